// K5: bandwidth-bound dequant-GEMV for decode-sized token counts (M <= 16):
//   Y = X W~^T + gamma (X A^T) B^T
// ("QLoRA, explained": serving the adapter unmerged on the 4-bit base).  The
// packed weight is streamed from HBM exactly once.
//
// One persistent CTA per SM: a producer warp and 16 consumer warps.
//   producer   pulls work units (16 rows of W x one contraction slice) from an
//              atomic counter and streams each unit as tiles of 16 rows x 32
//              NF4 blocks (16 rows x 1024 contiguous bytes) with one 3-D TMA
//              box per tile into a 4-stage ring (128-byte swizzle).  Its other
//              lanes read the tile's FP8 scale codes and fp32 meta scales and
//              publish c~ = e4m3(code) * c2 for every (row, block) of the
//              tile next to it, so consumers do no global loads at all.
//   consumers  each take 2 of the tile's 32 blocks for all 16 rows: swap-AB
//              mma.sync m16n8k16 with W rows on the MMA's M side and tokens on
//              its N side (one n8 tile for M <= 8, two for M <= 16).  A lane
//              turns each packed byte into the bf16 pair (q[lo], q[hi]) with
//              one byte permute and one shared-memory load from a
//              byte->bf16x2 table replicated per lane: table rows are 256
//              bytes apart from a 64 KiB-aligned base, so the permute drops the
//              byte straight into bits 8..15 of the lane's address.  Inside a
//              block the contraction order is permuted identically on both
//              operands (lane c of a row group covers k = 16c .. 16c+15), the
//              block's MMAs accumulate into fresh registers, and the block
//              partial is scaled by its c~ once.  At the end of a unit the 16
//              warps' partials are summed through shared memory.
// Each slice's first CTA also computes that slice's part of T = X A^T.  Slices
// write fp32 partials; the finalize kernel sums them, adds gamma T B^T and
// rounds Y to bf16.
//
// Deviation from the dequantise kernel, stated: the table holds bf16(q[i])
// rather than bf16(q[i] * c~), so each weight enters as bf16(q) * c~ in fp32;
// the difference from bf16_rne(q * c~) is below one bf16 ulp per weight, far
// inside the layer tolerance.
//
// Every mbarrier wait is bounded (common.cuh); a timeout sets the workspace
// error word and the kernel winds down.
#include <algorithm>

#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kConsumerWarps = 16;
constexpr int kThreads = (kConsumerWarps + 1) * 32;   // + producer warp
constexpr int kLutBytes = 256 * 256;                  // 256 rows of 256 bytes
constexpr int kSmemBytes = 227 * 1024;
constexpr int kStages = 4;
constexpr int kTileRows = 16;
constexpr int kTileBlocks = 32;                       // NF4 blocks per tile and row
constexpr int kTileBytes = kTileRows * kTileBlocks * 32;      // 16 KiB
constexpr int kScaleBytes = kTileRows * kTileBlocks * 4;      // 2 KiB of c~ per tile

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// bf16 pair of byte k of w: lane_reg = table base + 4*lane, bits 8..15 clear.
template <int k>
__device__ __forceinline__ uint32_t lut_pair(uint32_t w, uint32_t lane_reg) {
    return lds32(prmt(w, lane_reg, 0x7604u | (k << 4)));
}

__device__ __forceinline__ void tma_load_3d(uint32_t smem_dst, const CUtensorMap* map, int32_t c0,
                                            int32_t c1, int32_t c2, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// Shared-memory plan: the table sits at the first 64 KiB boundary; everything
// else is placed first-fit in the space before it, then after it.
struct SmemPlan {
    uint32_t lut, ring, scales, units, red, x, bars;
    bool ok;
};

__device__ __forceinline__ SmemPlan plan_smem(uint32_t start, uint32_t x_bytes, uint32_t red_bytes) {
    SmemPlan p;
    p.lut = (start + 0xFFFFu) & ~0xFFFFu;
    uint32_t lo = start;
    const uint32_t lo_end = p.lut;                             // region before the table
    uint32_t hi = p.lut + kLutBytes;
    const uint32_t hi_end = start + kSmemBytes;
    p.ok = true;
    auto take = [&](uint32_t bytes, uint32_t align) -> uint32_t {
        uint32_t at = (lo + align - 1) & ~(align - 1);
        if (at + bytes <= lo_end) {
            lo = at + bytes;
            return at;
        }
        at = (hi + align - 1) & ~(align - 1);
        if (at + bytes <= hi_end) {
            hi = at + bytes;
            return at;
        }
        p.ok = false;
        return start;
    };
    p.ring = take(kStages * kTileBytes, 1024);
    p.scales = take(kStages * kScaleBytes, 16);
    p.red = take(red_bytes, 16);
    p.x = take(x_bytes, 16);
    p.units = take(kStages * 8, 8);
    p.bars = take((2 * kStages + 4) * 8 + 8, 8);   // full, empty, rdone[2], rfree[2], flag
    return p;
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
gemv_kernel(const __grid_constant__ CUtensorMap tm_packed, GemvArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t start = smem_u32(smem);
    const int slice = blockIdx.y;
    const int64_t k_beg = int64_t(slice) * a.k_per_split;
    const int64_t k_end = min(a.K, k_beg + a.k_per_split);
    const int kslab = static_cast<int>(k_end - k_beg);
    const int nblk = kslab / QLORA_BLOCK;
    const int tiles_per_unit = (nblk + kTileBlocks - 1) / kTileBlocks;
    const uint32_t x_pitch = static_cast<uint32_t>(kslab * 2 + 8);
    const int xrows = static_cast<int>(a.M);
    constexpr int kTok = 8 * NT;
    constexpr uint32_t kRedHalf = kConsumerWarps * kTileRows * kTok * 4u;
    const SmemPlan sp = plan_smem(start, xrows * x_pitch, 2u * kRedHalf);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (sp.bars - start));
    uint64_t* empty = full + kStages;
    uint64_t* rdone = empty + kStages;          // [2] per reduction buffer: partials written
    uint64_t* rfree = rdone + 2;                // [2]: partials summed
    volatile int* abort_flag = reinterpret_cast<volatile int*>(rfree + 2);
    volatile int* uslot = reinterpret_cast<volatile int*>(smem + (sp.units - start));

    if (tid == 0) {
        *abort_flag = sp.ok ? 0 : 1;
        if (!sp.ok) atomicOr(a.err, 2);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        for (int p = 0; p < 2; ++p) {
            mbar_init(&rdone[p], kConsumerWarps);
            mbar_init(&rfree[p], 1);
        }
        fence_barrier_init();
        prefetch_tensormap(&tm_packed);
    }
    // lookup table: byte -> (bf16 q[lo nibble], bf16 q[hi nibble]), per lane
    for (int e = tid; e < 256 * 32; e += kThreads) {
        const int b = e >> 5, l = e & 31;
        const uint32_t v = pack_bf16x2(a.tab.code[b & 15], a.tab.code[b >> 4]);
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(sp.lut + b * 256 + l * 4), "r"(v) : "memory");
    }
    // activation slice, M rows (8-byte stores: the pitch is 8 mod 16 so that
    // fragment loads spread over all banks)
    const int vec_per_row = kslab / 8;
    for (int q = tid; q < xrows * vec_per_row; q += kThreads) {
        const int m = q / vec_per_row, v = q % vec_per_row;
        const uint4 val = *reinterpret_cast<const uint4*>(a.X + m * a.K + k_beg + v * 8);
        const uint32_t dst = sp.x + m * x_pitch + v * 16;
        asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(dst), "r"(val.x), "r"(val.y) : "memory");
        asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(dst + 8), "r"(val.z), "r"(val.w)
                     : "memory");
    }
    __syncthreads();
    if (*abort_flag) return;

    const int64_t nkb = a.K / QLORA_BLOCK;
    const int kb_beg = static_cast<int>(k_beg / QLORA_BLOCK);
    const int64_t nunits = (a.N + kTileRows - 1) / kTileRows;
    const int g = lane >> 2, c = lane & 3;

    if (warp == kConsumerWarps) {
        // -------------------------------------------------------- producer
        // Work items are (unit, tile) in order; the scale codes and meta
        // scales of the next two items are in flight while one is published,
        // and the unit after the current one is already claimed.
        const int row = lane >> 1;                  // this lane's (row, 16 blocks) of a tile
        const int bt0 = (lane & 1) * 16;
        const bool vec_codes = (nkb % 16) == 0 && (kb_beg % 16) == 0 &&
                               (reinterpret_cast<uintptr_t>(a.scale_codes) & 15u) == 0;
        struct Pref {
            uint4 codes;
            float m_first, m_last;
            int64_t ci0;
        };
        auto claim = [&]() -> int {
            int u = 0;
            if (lane == 0) u = atomicAdd(a.counters + slice, 1);
            return __shfl_sync(0xffffffffu, u, 0);
        };
        auto fetch = [&](int unit, int tile) -> Pref {
            Pref p;
            p.codes = make_uint4(0, 0, 0, 0);
            p.m_first = p.m_last = 0.f;
            const int64_t n = int64_t(unit) * kTileRows + row;
            const int bs0 = tile * kTileBlocks + bt0;
            p.ci0 = n * nkb + kb_beg + bs0;
            if (unit >= nunits || n >= a.N || bs0 >= nblk) return p;
            const int cnt = min(16, nblk - bs0);
            if (vec_codes && cnt == 16) {
                p.codes = __ldg(reinterpret_cast<const uint4*>(a.scale_codes + p.ci0));
            } else {
                uint32_t w[4] = {0, 0, 0, 0};
                for (int i = 0; i < cnt; ++i) w[i >> 2] |= uint32_t(__ldg(a.scale_codes + p.ci0 + i)) << (8 * (i & 3));
                p.codes = make_uint4(w[0], w[1], w[2], w[3]);
            }
            p.m_first = __ldg(a.meta + (p.ci0 >> 8));
            p.m_last = __ldg(a.meta + ((p.ci0 + cnt - 1) >> 8));
            return p;
        };
        uint32_t it = 0;
        int armed[kStages];
        for (int s = 0; s < kStages; ++s) armed[s] = -1;
        bool ok = true;
        int cur_u = claim(), next_u = claim(), cur_t = 0;
        // the item after (u, t): (u, t+1) or (next unit, 0)
        int nx_u = tiles_per_unit > 1 ? cur_u : next_u, nx_t = tiles_per_unit > 1 ? 1 : 0;
        Pref p0 = fetch(cur_u, cur_t);
        Pref p1 = fetch(nx_u, nx_t);
        for (;; ++it) {
            const int s = it % kStages;
            const uint32_t ph = (it / kStages) & 1;
            const bool done = cur_u >= nunits;
            if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, a.err)) {
                ok = false;
                break;
            }
            if (!done) {
                const uint32_t cw[4] = {p0.codes.x, p0.codes.y, p0.codes.z, p0.codes.w};
                float ct[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float mt = (((p0.ci0 + i) >> 8) == (p0.ci0 >> 8)) ? p0.m_first : p0.m_last;
                    ct[i] = __fmul_rn(e4m3_to_float(uint8_t(cw[i >> 2] >> (8 * (i & 3)))), mt);
                }
                // scales are stored [block][row] so that the consumers' reads
                // (8 rows of one block per warp) hit 8 consecutive words
                const uint32_t sdst = sp.scales + s * kScaleBytes + (bt0 * kTileRows + row) * 4;
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(sdst + i * kTileRows * 4), "f"(ct[i])
                                 : "memory");
            }
            if (lane == 0) {
                uslot[2 * s] = done ? -1 : cur_u;
                uslot[2 * s + 1] = cur_t;
            }
            __syncwarp();
            if (lane == 0) {
                if (done) {
                    mbar_arrive(&full[s]);
                } else {
                    mbar_arrive_expect_tx(&full[s], kTileBytes);
                    tma_load_3d(sp.ring + s * kTileBytes, &tm_packed, 0, cur_u * kTileRows,
                                static_cast<int>(k_beg / 256) + cur_t * (kTileBlocks / 4), &full[s]);
                    armed[s] = static_cast<int>(ph);
                }
            }
            if (done) break;
            // advance: the next item becomes current, fetch the one after it
            cur_u = nx_u;
            cur_t = nx_t;
            p0 = p1;
            if (cur_t == 0 && cur_u == next_u) next_u = claim();   // entered a new unit
            if (cur_t + 1 < tiles_per_unit) {
                nx_u = cur_u;
                nx_t = cur_t + 1;
            } else {
                nx_u = next_u;
                nx_t = 0;
            }
            p1 = fetch(nx_u, nx_t);
        }
        if (!ok && lane == 0) {
            for (int s = 0; s < kStages; ++s)
                if (armed[s] >= 0) mbar_drain(&full[s], armed[s], a.err);
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    if (blockIdx.x == 0) {
        // this slice's part of T = X A^T, k-steps split over the 16 warps;
        // reduced in the first reduction buffer, then published
        constexpr int kMaxJT = QLORA_MAX_RANK / 8;
        float tacc[kMaxJT][4];
#pragma unroll
        for (int j = 0; j < kMaxJT; ++j) tacc[j][0] = tacc[j][1] = tacc[j][2] = tacc[j][3] = 0.f;
        const int ksteps = kslab / 16;
        const int per = (ksteps + kConsumerWarps - 1) / kConsumerWarps;
        const int s0 = warp * per, s1 = min(ksteps, s0 + per);
        for (int st = s0; st < s1; ++st) {
            const int kk = st * 16 + 2 * c;
            const uint32_t a0 = g < xrows ? lds32(sp.x + g * x_pitch + kk * 2) : 0u;
            const uint32_t a2 = g < xrows ? lds32(sp.x + g * x_pitch + (kk + 8) * 2) : 0u;
            const uint32_t a1 = g + 8 < xrows ? lds32(sp.x + (g + 8) * x_pitch + kk * 2) : 0u;
            const uint32_t a3 = g + 8 < xrows ? lds32(sp.x + (g + 8) * x_pitch + (kk + 8) * 2) : 0u;
#pragma unroll
            for (int jt = 0; jt < kMaxJT; ++jt) {
                if (jt * 8 < a.r) {
                    const uint16_t* ap = a.A + int64_t(jt * 8 + g) * a.K + k_beg + kk;
                    const uint32_t b0 = __ldg(reinterpret_cast<const uint32_t*>(ap));
                    const uint32_t b1 = __ldg(reinterpret_cast<const uint32_t*>(ap + 8));
                    mma16816(tacc[jt], a0, a1, a2, a3, b0, b1);
                }
            }
        }
        // 16 rows x 128 columns of fp32 = 8 KiB, inside reduction buffer 0
        const uint32_t tred = sp.red;
        for (int e = lane; e < 16 * QLORA_MAX_RANK / kConsumerWarps; e += 32)
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(tred + (warp * 128 + e) * 4), "r"(0u)
                         : "memory");
        asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
#pragma unroll
        for (int jt = 0; jt < kMaxJT; ++jt) {
            if (jt * 8 < a.r) {
                const int j = jt * 8 + 2 * c;
                const uint32_t r0 = tred + (g * QLORA_MAX_RANK + j) * 4;
                const uint32_t r1 = tred + ((g + 8) * QLORA_MAX_RANK + j) * 4;
                asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(r0), "f"(tacc[jt][0]) : "memory");
                asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(r0 + 4), "f"(tacc[jt][1]) : "memory");
                asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(r1), "f"(tacc[jt][2]) : "memory");
                asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(r1 + 4), "f"(tacc[jt][3]) : "memory");
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
        for (int e = warp * 32 + lane; e < a.M * a.r; e += kConsumerWarps * 32) {
            const int m = e / a.r, j = e % a.r;
            a.Tpart[(int64_t(slice) * a.M + m) * a.r + j] =
                __uint_as_float(lds32(tred + (m * QLORA_MAX_RANK + j) * 4));
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
    }

    // main loop: 2 blocks of every tile, all 16 rows
    float acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
    const uint32_t lane_reg = sp.lut + lane * 4;
    float* part = a.part + int64_t(slice) * a.M * a.N;
    uint32_t it = 0, units_done = 0;
    for (;;) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!mbar_wait(&full[s], ph, abort_flag, a.err)) break;
        const int unit = uslot[2 * s];
        const int tile = uslot[2 * s + 1];
        if (unit < 0) break;                                  // no more work
        const uint32_t ring = sp.ring + s * kTileBytes;
        const uint32_t scl = sp.scales + s * kScaleBytes;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int bt = 2 * warp + j;                      // block within the tile
            const int bs = tile * kTileBlocks + bt;           // block within the slice
            if (bs >= nblk) break;
            // tile layout [chunk of 4 blocks][row][128 bytes], 16-byte units
            // swizzled by (row & 7); lane (g, c) reads 8 bytes of rows g, g+8
            const int within = (bt & 3) * 32 + c * 8;
            const uint32_t unit16 = static_cast<uint32_t>(within >> 4);
            const uint32_t chunk = ring + (bt >> 2) * (kTileRows * 128) + (within & 15);
            uint32_t wa0, wa1, wb0, wb1;
            asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];"
                         : "=r"(wa0), "=r"(wa1)
                         : "r"(chunk + g * 128 + ((unit16 ^ (g & 7)) << 4)));
            asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];"
                         : "=r"(wb0), "=r"(wb1)
                         : "r"(chunk + (g + 8) * 128 + ((unit16 ^ (g & 7)) << 4)));
            const float cta = __uint_as_float(lds32(scl + (bt * kTileRows + g) * 4));
            const float ctb = __uint_as_float(lds32(scl + (bt * kTileRows + g + 8) * 4));
            float blk[NT][4];
#pragma unroll
            for (int t = 0; t < NT; ++t) blk[t][0] = blk[t][1] = blk[t][2] = blk[t][3] = 0.f;
            const uint32_t xk = sp.x + static_cast<uint32_t>((bs * 64 + c * 16) * 2);
#pragma unroll
            for (int st = 0; st < 4; ++st) {
                const uint32_t wa = st < 2 ? wa0 : wa1;
                const uint32_t wb = st < 2 ? wb0 : wb1;
                uint32_t a0, a1, a2, a3;
                if (st & 1) {
                    a0 = lut_pair<2>(wa, lane_reg);
                    a2 = lut_pair<3>(wa, lane_reg);
                    a1 = lut_pair<2>(wb, lane_reg);
                    a3 = lut_pair<3>(wb, lane_reg);
                } else {
                    a0 = lut_pair<0>(wa, lane_reg);
                    a2 = lut_pair<1>(wa, lane_reg);
                    a1 = lut_pair<0>(wb, lane_reg);
                    a3 = lut_pair<1>(wb, lane_reg);
                }
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const int tok = g + 8 * t;
                    uint32_t b0 = 0, b1 = 0;
                    if (tok < xrows)
                        asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];"
                                     : "=r"(b0), "=r"(b1)
                                     : "r"(xk + tok * x_pitch + st * 8));
                    mma16816(blk[t], a0, a1, a2, a3, b0, b1);
                }
            }
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                acc[t][0] = fmaf(cta, blk[t][0], acc[t][0]);
                acc[t][1] = fmaf(cta, blk[t][1], acc[t][1]);
                acc[t][2] = fmaf(ctb, blk[t][2], acc[t][2]);
                acc[t][3] = fmaf(ctb, blk[t][3], acc[t][3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        ++it;
        if (tile == tiles_per_unit - 1) {
            // the unit is complete: sum the 16 warps' partials.  Buffer p is
            // reused every second unit; rfree[p] says its last sum was read.
            const int p = units_done & 1;
            const uint32_t use = units_done >> 1;
            const uint32_t red = sp.red + p * kRedHalf;
            bool ok = true;
            if (use > 0) ok = mbar_wait(&rfree[p], (use - 1) & 1, abort_flag, a.err);
            if (!ok) break;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int tok = 8 * t + 2 * c;
                const uint32_t base = red + (warp * kTileRows) * kTok * 4;
                asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(base + (g * kTok + tok) * 4),
                             "f"(acc[t][0]), "f"(acc[t][1]) : "memory");
                asm volatile("st.shared.v2.f32 [%0], {%1, %2};"
                             ::"r"(base + ((g + 8) * kTok + tok) * 4), "f"(acc[t][2]), "f"(acc[t][3])
                             : "memory");
                acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&rdone[p]);
            if (warp == unit % kConsumerWarps) {
                if (!mbar_wait(&rdone[p], use & 1, abort_flag, a.err)) break;
                for (int e = lane; e < kTileRows * kTok; e += 32) {
                    const int row = e / kTok, tok = e % kTok;
                    float sum = 0.f;
#pragma unroll 4
                    for (int w = 0; w < kConsumerWarps; ++w)
                        sum += __uint_as_float(lds32(red + ((w * kTileRows + row) * kTok + tok) * 4));
                    const int64_t n = int64_t(unit) * kTileRows + row;
                    if (tok < a.M && n < a.N) part[int64_t(tok) * a.N + n] = sum;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&rfree[p]);
            }
            ++units_done;
        }
    }
}

// One thread per output column n: T = sum of the slices' parts (staged in
// shared memory), Y[m][n] = bf16( sum_s part[s][m][n] + gamma * T[m] . B[n] ).
__global__ void __launch_bounds__(256)
gemv_finalize_kernel(GemvFinalizeArgs a) {
    __shared__ float st[16 * QLORA_MAX_RANK];
    for (int e = threadIdx.x; e < a.M * a.r; e += blockDim.x) {
        float t = 0.f;
        for (int s = 0; s < a.splits; ++s) t += a.Tpart[int64_t(s) * a.M * a.r + e];
        st[e] = t;
        if (blockIdx.x == 0 && a.T_save) a.T_save[e] = t;
    }
    __syncthreads();
    const int64_t n = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    if (n >= a.N) return;
    float acc[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) acc[m] = 0.f;
    for (int j0 = 0; j0 < a.r; j0 += 8) {
        const uint4 bv = *reinterpret_cast<const uint4*>(a.B + n * a.r + j0);
        float b[8];
        const uint32_t w[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            b[2 * q] = __uint_as_float(w[q] << 16);
            b[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
        }
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            if (m < a.M) {
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[m] = fmaf(st[m * a.r + j0 + q], b[q], acc[m]);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        if (m < a.M) {
            float s = a.gamma * acc[m];
            for (int k = 0; k < a.splits; ++k) s += a.part[(int64_t(k) * a.M + m) * a.N + n];
            __nv_bfloat16 y = __float2bfloat16_rn(s);
            a.Y[m * a.N + n] = *reinterpret_cast<uint16_t*>(&y);
        }
    }
}

}  // namespace

int gemv_max_activation_bytes() {
    // The table's 64 KiB alignment leaves the rest of shared memory in two
    // pieces whose sizes depend on where dynamic shared memory starts; 32 KiB
    // of activations fit next to the ring, scales and reduction buffers in
    // every split (the kernel re-checks its plan and reports a misfit).
    return 32 * 1024;
}

cudaError_t launch_gemv(const CUtensorMap& tm_packed, const GemvArgs& a, int num_sms,
                        cudaStream_t stream) {
    const unsigned per_slice = static_cast<unsigned>(std::max(1, num_sms / std::max(1, a.splits)));
    dim3 grid(per_slice, static_cast<unsigned>(a.splits));
    cudaError_t e;
    if (a.M > 8) {
        e = cudaFuncSetAttribute(gemv_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        gemv_kernel<2><<<grid, kThreads, kSmemBytes, stream>>>(tm_packed, a);
    } else {
        e = cudaFuncSetAttribute(gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        gemv_kernel<1><<<grid, kThreads, kSmemBytes, stream>>>(tm_packed, a);
    }
    return cudaGetLastError();
}

cudaError_t launch_gemv_finalize(const GemvFinalizeArgs& a, cudaStream_t stream) {
    if (a.M <= 0 || a.N <= 0) return cudaSuccess;
    const unsigned grid = static_cast<unsigned>((a.N + 255) / 256);
    gemv_finalize_kernel<<<grid, 256, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace qnf4
