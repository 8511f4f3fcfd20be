// K5: bandwidth-bound dequant-GEMV for decode-sized token counts (M <= 16):
//   Y = X W~^T + gamma (X A^T) B^T
// ("QLoRA, explained": serving the adapter unmerged on the 4-bit base).  The
// packed weight is streamed from HBM exactly once, and every weight enters
// the product as the W~ the page's dDQ defines, bf16_rne(fp32(q[idx] * c~)),
// the same value the dequantise kernel writes and the GEMM multiplies.
//
// One persistent CTA per SM: a producer warp and 16 consumer warps.
//   producer   pulls work units (R rows of W x one contraction slice) from an
//              atomic counter and streams each unit as tiles of R rows x D
//              256-wide chunks (R D = 256, 32 KiB of packed indices) with one
//              3-D TMA box per tile into a ring of stages (128-byte swizzle);
//              its lanes copy the tile's FP8 scale codes and each row's meta
//              scales next to it (cp.async), so consumers do no global loads.
//   consumers  warp w takes the tile's 16-row group w / D of chunk w % D: a
//              swap-AB mma.sync m16n8k16 with W rows on the MMA's M side and
//              tokens on its N side (one n8 tile for M <= 8, two for M <= 16).
//              The contraction order inside the chunk is permuted identically
//              on both operands so that lane (g, c) of the warp holds, over
//              the chunk's 16 MMAs, all 64 weights of NF4 block c of rows g
//              and g + 8 (MMA j feeds the block's positions 4j .. 4j + 3).
//              Each packed byte addresses a per-lane table of fp32 code pairs
//              (q[lo], q[hi]) in shared memory (one permute drops the byte
//              into the lane's address; one 8-byte load); the pair is
//              multiplied by the block's c~ in fp32 and rounded to a bf16 pair
//              (RNE): exactly bf16_rne(fp32(q * c~)), the A operand of the
//              MMA.  The activations sit in shared memory with 8-byte units
//              XOR-swizzled by block and token, so that a warp's 8-byte
//              fragment loads are free of bank conflicts.
//              At the end of a unit the D warps of each row group sum their
//              partials through shared memory.
// The first few CTAs of each slice also compute a share of T = X A^T.  Slices
// and T shares write fp32 partials; the finalize kernel sums them, adds
// gamma T B^T and rounds Y to bf16.
//
// Per two weights the expansion costs one permute, one 8-byte shared load
// (two wavefronts per warp), one paired fp32 multiply and one paired rounding.
// Measured alternatives that built each block's 16-entry bf16 table in
// registers and expanded nibbles with byte permutes (about 2.5 integer-pipe
// instructions per weight, entirely or for part of the rows) were slower: the
// integer pipe runs 64 such instructions per clock per SM on this GPU.
//
// Every mbarrier wait is bounded (common.cuh); a timeout sets the workspace
// error word and the kernel winds down.
#include <algorithm>

#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kConsumerWarps = 16;
constexpr int kThreads = (kConsumerWarps + 1) * 32;   // + producer warp
constexpr int kSmemBytes = 227 * 1024;
constexpr int kMaxStages = 6;
// A weight tile is 32 KiB: R rows x D chunks of 256 contraction positions
// (128 packed bytes), R D = 256, D in {1, 2, 4, 8} chosen per launch so that
// a contraction slice is a whole number of tiles; the 16 consumer warps take
// its 16 (16-row group, chunk) pieces.  A work unit is R rows x the whole
// slice.
constexpr int kTileBytes = 32768;
// Raw scale data of a tile, copied next to it by the producer: the FP8 codes
// [R rows][4 D + 4 bytes], then the meta scales [R rows][2] fp32 of each row's
// first and last block (a row's blocks in a tile span at most two groups of
// 256 scales).  1024 + 12 R <= 4096 bytes.
constexpr int kScaleBytes = 4096;
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0)
                 : "memory");
}
// Arrive on `bar` once this thread's earlier cp.async copies have landed (the
// arrival counts against the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

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

// The main loop's shared-memory loads and MMAs are plain (not volatile) asm so
// that the compiler may interleave them freely.  They are kept after the
// stage's full-barrier wait by taking their addresses from opaque_zero(),
// issued after the wait, and before the stage's release by feeding their
// results to keep_before() ahead of the arrive.
__device__ __forceinline__ uint32_t opaque_zero() {
    uint32_t z;
    asm volatile("mov.u32 %0, 0;" : "=r"(z)::"memory");
    return z;
}

__device__ __forceinline__ void keep_before(float v) { asm volatile("" ::"f"(v)); }


__device__ __forceinline__ uint32_t lds16_nv(uint32_t addr) {
    uint16_t v;
    asm("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ float2 lds64f_nv(uint32_t addr) {
    float2 v;
    asm("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint64_t lds64_nv(uint32_t addr) {
    uint64_t v;
    asm("ld.shared.b64 %0, [%1];" : "=l"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint64_t splat_f32x2(float x) {
    uint64_t v;
    asm("mov.b64 %0, {%1, %1};" : "=l"(v) : "f"(x));
    return v;
}

// Both fp32 lanes of q times those of c (each rounded to nearest, as two
// __fmul_rn), then rounded to one bf16 pair (RNE), low lane in the low half.
__device__ __forceinline__ uint32_t mul_f32x2_to_bf16x2(uint64_t q, uint64_t c) {
    uint32_t out;
    asm("{\n\t.reg .b64 p;\n\t.reg .f32 lo, hi;\n\t"
        "mul.rn.f32x2 p, %1, %2;\n\t"
        "mov.b64 {lo, hi}, p;\n\t"
        "cvt.rn.bf16x2.f32 %0, hi, lo;\n\t}"
        : "=r"(out)
        : "l"(q), "l"(c));
    return out;
}

// Two FP8 E4M3 codes (low byte first) to their exact fp32 values: E4M3 is a
// subset of f16, and f16 widens exactly to fp32.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t codes16) {
    uint32_t h2;
    asm("{ .reg .b16 c; cvt.u16.u32 c, %1; cvt.rn.f16x2.e4m3x2 %0, c; }" : "=r"(h2) : "r"(codes16));
    float2 v;
    asm("{ .reg .b16 lo, hi; mov.b32 {lo, hi}, %2; cvt.f32.f16 %0, lo; cvt.f32.f16 %1, hi; }"
        : "=f"(v.x), "=f"(v.y)
        : "r"(h2));
    return v;
}

__device__ __forceinline__ void mma16816_nv(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                            uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void tma_load_3d(uint32_t smem_dst, const CUtensorMap* map, int32_t c0,
                                            int32_t c1, int32_t c2, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// Shared-memory plan.  The code-pair table sits at the first 64 KiB boundary
// (its addresses are formed by dropping a byte into bits 8-15 of the lane's
// base, so bits 8-15 of the base must be clear); everything else is placed
// first-fit in the space before it, then after it.  The host evaluates the
// same plan to pick the stage count; the kernel re-checks it against its real
// shared-memory base and reports a misfit.
constexpr int kLutBytes = 256 * 256;      // 256 byte values x 32 lanes x 8 bytes

struct SmemPlan {
    uint32_t lut, ring, scales, units, red, x, zero, bars;
    bool ok;
};

__host__ __device__ inline SmemPlan plan_smem(uint32_t start, int stages, uint32_t x_bytes,
                                              uint32_t red_bytes) {
    SmemPlan p;
    p.lut = (start + 0xFFFFu) & ~0xFFFFu;
    uint32_t lo = start;
    const uint32_t lo_end = p.lut;                             // region before the table
    uint32_t hi = p.lut + kLutBytes;
    const uint32_t hi_end = start + kSmemBytes;
    p.ok = hi <= hi_end;
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
    p.ring = take(stages * kTileBytes, 1024);
    p.scales = take(stages * kScaleBytes, 16);
    p.red = take(red_bytes, 16);
    p.x = take(x_bytes, 128);
    p.zero = take(128, 128);                       // zero activations for absent tokens
    p.units = take(stages * 8, 8);
    p.bars = take((2 * stages + 4) * 8 + 8, 8);   // full, empty, rdone[2], rfree[2], flag
    return p;
}

// Activation slab bytes (M rows of kslab bf16, a row a whole number of 128-byte
// lines) and reduction-buffer bytes (two [warp][16 rows][M] fp32 buffers,
// which also hold the [M][r] reduction of T) for M tokens over a kslab-wide
// slice.
__host__ __device__ inline uint32_t gemv_x_bytes(int64_t M, int64_t kslab) {
    return static_cast<uint32_t>(M * kslab * 2);
}
__host__ __device__ inline uint32_t gemv_red_bytes(int64_t M) {
    return static_cast<uint32_t>(2 * kConsumerWarps * 16 * M * 4);
}

// Byte offset of activation (token m, slice position k) in the slab, k a
// multiple of 2: rows of kslab bf16; within each 64-position block the
// 8-byte units (4 positions) are permuted by u -> u ^ (4 (block mod 4) +
// (m mod 4)), so that the 16 lanes of a half-warp, which read unit j of
// blocks 0-3 for tokens 0-3 (or 4-7), hit 16 different bank pairs.
__device__ __forceinline__ uint32_t x_off(int m, int k, uint32_t x_pitch) {
    const int blk = k >> 6;
    const int u = ((k & 63) >> 2) ^ (((blk & 3) << 2) | (m & 3));
    return static_cast<uint32_t>(m) * x_pitch + static_cast<uint32_t>(blk * 128 + u * 8 + (k & 3) * 2);
}

template <int NT, int kStages, int D>
__global__ void __launch_bounds__(kThreads, 1)
gemv_kernel(const __grid_constant__ CUtensorMap tm_packed, GemvArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t start = smem_u32(smem);
    const int slice = blockIdx.y;
    launch_dependents();                         // the finalize waits for this grid
    const int64_t k_beg = int64_t(slice) * a.k_per_split;
    const int64_t k_end = min(a.K, k_beg + a.k_per_split);
    const int kslab = static_cast<int>(k_end - k_beg);
    const int nblk = kslab / QLORA_BLOCK;
    // D: 256-wide chunks per tile (= a.tile_chunks)
    constexpr int R = 256 / D;                   // rows per tile and unit
    constexpr int bpr = 4 * D;                   // blocks per tile row
    constexpr int code_pitch = bpr + 4;
    constexpr int meta_off = R * code_pitch;     // a multiple of 16
    const int tiles_per_unit = (nblk + bpr - 1) / bpr;
    const uint32_t x_pitch = static_cast<uint32_t>(kslab * 2);        // as gemv_x_bytes
    const int xrows = static_cast<int>(a.M);
    const uint32_t red_half = gemv_red_bytes(a.M) / 2;
    const SmemPlan sp = plan_smem(start, kStages, gemv_x_bytes(a.M, kslab), 2u * red_half);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (sp.bars - start));
    uint64_t* empty = full + kStages;
    uint64_t* rdone = empty + kStages;          // [2] per reduction buffer: partials written
    uint64_t* rfree = rdone + 2;                // [2]: partials summed
    volatile int* abort_flag = reinterpret_cast<volatile int*>(rfree + 2);
    volatile int* uslot = reinterpret_cast<volatile int*>(smem + (sp.units - start));

    if (tid == 0) {
        *abort_flag = sp.ok ? 0 : 1;
        if (!sp.ok) atomicOr(a.err, kErrSmemPlan);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1 + 32);           // producer lane 0 + the lanes' scale copies
            mbar_init(&empty[s], kConsumerWarps);
        }
        for (int p = 0; p < 2; ++p) {
            mbar_init(&rdone[p], kConsumerWarps);
            mbar_init(&rfree[p], min(kConsumerWarps, xrows));
        }
        fence_barrier_init();
        prefetch_tensormap(&tm_packed);
    }
    __syncthreads();                             // barriers initialised, plan checked
    if (*abort_flag) return;

    const int64_t nkb = a.K / QLORA_BLOCK;
    const int kb_beg = static_cast<int>(k_beg / QLORA_BLOCK);
    const int64_t nunits = (a.N + R - 1) / R;
    const int g = lane >> 2, c = lane & 3;

    if (warp == kConsumerWarps) {
        // -------------------------------------------------------- producer
        // Per work item (unit, tile), once its stage is free: lane 0 starts
        // the tile's TMA load; the lanes copy the tile's FP8 scale codes (8
        // 4-byte groups each, cp.async, zeros past the slice or the matrix)
        // and each row's two meta scales into the stage's scale area, and
        // arrive on the stage's full barrier when their copies land.  Units
        // are claimed one ahead.
        const int chunk0 = static_cast<int>(k_beg / 256);
        // Claims run one unit ahead: lane 0 holds the result of an atomic
        // issued a unit earlier, so no claim waits for its round trip.  Claims
        // increase, so once the work passes the last unit the claim still
        // outstanding lies past it too and no unit is left unprocessed.
        int pend = 0;
        if (lane == 0) pend = atomicAdd(a.counters + slice, 1);
        auto claim = [&]() -> int {
            const int u = __shfl_sync(0xffffffffu, pend, 0);
            if (lane == 0) pend = atomicAdd(a.counters + slice, 1);
            return u;
        };
        int u = claim(), t = 0;
        bool ok = true;
        int armed[kStages];
        for (int s = 0; s < kStages; ++s) armed[s] = -1;
        for (uint32_t it = 0;; ++it) {
            const int s = static_cast<int>(it % kStages);
            const uint32_t ph = (it / kStages) & 1;
            const bool done = u >= nunits;
            if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, a.err)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                uslot[2 * s] = done ? -1 : u;
                uslot[2 * s + 1] = t;
                if (done) {
                    mbar_arrive(&full[s]);
                } else {
                    mbar_arrive_expect_tx(&full[s], kTileBytes);
                    tma_load_3d(sp.ring + s * kTileBytes, &tm_packed, 0, u * R, chunk0 + t * D, &full[s]);
                    armed[s] = static_cast<int>(ph);
                }
            }
            if (!done) {
                // K is a multiple of 256, so a group of 4 blocks is all inside
                // or all outside the slice
                const uint32_t area = sp.scales + s * kScaleBytes;
                const int bs_row = t * bpr;                    // each row's first block
                const int cnt_full = max(0, min(bpr, nblk - bs_row));
#pragma unroll
                for (int q8 = 0; q8 < 8; ++q8) {
                    const int gi = lane + 32 * q8;             // 256 groups: R rows x D
                    const int row = gi / D, grp = gi % D;
                    const int64_t n = int64_t(u) * R + row;
                    const bool live = n < a.N && 4 * grp < cnt_full;
                    cp_async4(area + row * code_pitch + 4 * grp,
                              a.scale_codes + (live ? n * nkb + kb_beg + bs_row + 4 * grp : 0), live);
                }
                for (int mi = lane; mi < 2 * R; mi += 32) {
                    const int row = mi >> 1, last = mi & 1;
                    const int64_t n = int64_t(u) * R + row;
                    const bool live = n < a.N && cnt_full > 0;
                    const int64_t ci = n * nkb + kb_beg + bs_row + (last ? cnt_full - 1 : 0);
                    cp_async4(area + meta_off + mi * 4, a.meta + (live ? (ci >> 8) : 0), live);
                }
            }
            cp_async_arrive(&full[s]);
            if (done) break;
            if (++t == tiles_per_unit) {
                t = 0;
                u = claim();
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (!ok && lane == 0) {
            for (int s = 0; s < kStages; ++s)
                if (armed[s] >= 0) mbar_drain(&full[s], armed[s], a.err);
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    // While the producer's first tiles stream in, the consumer warps fill the
    // code-pair table and the activation slab, then meet on a named barrier.
    // Code-pair table: entry e (a packed byte) of lane l at lut + 256 e + 8 l
    // holds the fp32 codes (q[e & 15], q[e >> 4]); each thread writes two
    // lanes' copies of an entry at a time.
    for (int i = tid; i < 256 * 16; i += kConsumerWarps * 32) {
        const int e = i >> 4, l2 = (i & 15) * 2;
        const float q0 = a.tab.code[e & 15], q1 = a.tab.code[e >> 4];
        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %1, %2};" ::"r"(sp.lut + e * 256 + l2 * 8),
                     "f"(q0), "f"(q1)
                     : "memory");
    }
    // Activation slice, M rows of 8-byte units, swizzled (x_off); a zero line
    // stands in for tokens past M and blocks past the slice.
    if (tid < 32) asm volatile("st.shared.b32 [%0], %1;" ::"r"(sp.zero + tid * 4), "r"(0u) : "memory");
    {
        const int units_per_row = kslab / 4;
        for (int q = tid; q < xrows * units_per_row; q += kConsumerWarps * 32) {
            const int m = q / units_per_row, u = q % units_per_row;
            const uint2 val = *reinterpret_cast<const uint2*>(a.X + m * a.K + k_beg + u * 4);
            asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(sp.x + x_off(m, u * 4, x_pitch)),
                         "r"(val.x), "r"(val.y)
                         : "memory");
        }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
    if (blockIdx.x < a.t_ctas) {
        // a share of this slice's T = X A^T: CTA x of the first t_ctas takes
        // an equal run of the slice's 16-wide k-steps, spread over its warps.
        // Per round of 32 columns of T, each warp with k-steps stores its
        // [M][32] partial in its own slot of the reduction buffers (16 M 32
        // floats fill them exactly); the slots are then added in warp order
        // and written as this CTA's partial, so T is the same on every run.
        const int ksteps = kslab / 16;
        const int x = blockIdx.x;
        const int s0 = static_cast<int>(int64_t(ksteps) * x / a.t_ctas);
        const int s1 = static_cast<int>(int64_t(ksteps) * (x + 1) / a.t_ctas);
        const int nw = min(kConsumerWarps, s1 - s0);           // warps holding partials
        float* tp = a.Tpart + (int64_t(slice) * a.t_ctas + x) * a.M * a.r;
        const uint32_t slot = sp.red + static_cast<uint32_t>(warp * xrows * 32) * 4;
        // four 8-column tiles of T at a time keep the accumulators small
        for (int jg = 0; jg * 8 < a.r; jg += 4) {
            float tacc[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) tacc[j][0] = tacc[j][1] = tacc[j][2] = tacc[j][3] = 0.f;
            for (int st = s0 + warp; st < s1; st += kConsumerWarps) {
                const int kk = st * 16 + 2 * c;
                const uint32_t a0 = g < xrows ? lds32(sp.x + x_off(g, kk, x_pitch)) : 0u;
                const uint32_t a2 = g < xrows ? lds32(sp.x + x_off(g, kk + 8, x_pitch)) : 0u;
                const uint32_t a1 = g + 8 < xrows ? lds32(sp.x + x_off(g + 8, kk, x_pitch)) : 0u;
                const uint32_t a3 = g + 8 < xrows ? lds32(sp.x + x_off(g + 8, kk + 8, x_pitch)) : 0u;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if ((jg + j) * 8 < a.r) {
                        const uint16_t* ap = a.A + int64_t((jg + j) * 8 + g) * a.K + k_beg + kk;
                        const uint32_t b0 = __ldg(reinterpret_cast<const uint32_t*>(ap));
                        const uint32_t b1 = __ldg(reinterpret_cast<const uint32_t*>(ap + 8));
                        mma16816(tacc[j], a0, a1, a2, a3, b0, b1);
                    }
                }
            }
            if (warp < nw) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int col = j * 8 + 2 * c;                  // within the round
                    if (g < xrows) {
                        const uint32_t r0 = slot + (g * 32 + col) * 4;
                        asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(r0), "f"(tacc[j][0]),
                                     "f"(tacc[j][1]) : "memory");
                    }
                    if (g + 8 < xrows) {
                        const uint32_t r1 = slot + ((g + 8) * 32 + col) * 4;
                        asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(r1), "f"(tacc[j][2]),
                                     "f"(tacc[j][3]) : "memory");
                    }
                }
            }
            asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
            const int cols = min(32, a.r - jg * 8);
            for (int e = tid; e < xrows * 32; e += kConsumerWarps * 32) {
                const int m = e >> 5, col = e & 31;
                if (col < cols) {
                    float t = 0.f;
                    for (int w = 0; w < nw; ++w)
                        t += __uint_as_float(lds32(sp.red + static_cast<uint32_t>((w * xrows + m) * 32 + col) * 4));
                    tp[m * a.r + jg * 8 + col] = t;
                }
            }
            asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
        }
    }

    // Main loop.  Warp w takes row group rq = w / D (tile rows 16 rq + g and
    // 16 rq + g + 8 for MMA rows g, g + 8) of chunk cw = w % D; lane (g, c)
    // owns NF4 block bt = 4 cw + c of its two rows.  MMA j multiplies block
    // positions 4j .. 4j + 3: A fragment a0 / a2 = row g's positions
    // 4j, 4j+1 / 4j+2, 4j+3 (a1 / a3 the same of row g + 8), B fragment
    // b0, b1 = token g's activations at the same four positions.
    const int rq = warp / D, cw = warp % D;
    const int ra = rq * 16 + g, rb = ra + 8;
    const int bt = cw * 4 + c;
    const uint32_t lane_lut = sp.lut + lane * 8;       // bits 8-15 clear
    float acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
    float* part = a.part + int64_t(slice) * a.M * a.N;
    uint32_t it = 0, units_done = 0;
    for (;;) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!mbar_wait(&full[s], ph, abort_flag, a.err)) break;
        int unit, tile;
        asm volatile("ld.shared.v2.s32 {%0, %1}, [%2];" : "=r"(unit), "=r"(tile) : "r"(sp.units + s * 8) : "memory");
        if (unit < 0) break;                                  // no more work
        const uint32_t z = opaque_zero();
        const uint32_t ring = sp.ring + s * kTileBytes + z;
        const uint32_t scl = sp.scales + s * kScaleBytes + z;
        const int bs = tile * bpr + bt;                       // block within the slice
        // Blocks past the slice (only in a zero-filled last tile) take
        // c~ = 0 and zero activations, so they add nothing.
        const bool valid = bs < nblk;
        // c~ = fp32(e4m3 code * meta scale), one rounding; a row's blocks
        // before `split` belong to its first block's group of 256 scales
        // (the low 8 bits of the row's first scale index; 32-bit wrap-around
        // keeps them exact)
        const uint32_t ci_lo = static_cast<uint32_t>(unit) * static_cast<uint32_t>(R) * static_cast<uint32_t>(nkb) +
                               static_cast<uint32_t>(kb_beg + tile * bpr);
        const int split_a = 256 - static_cast<int>((ci_lo + ra * static_cast<uint32_t>(nkb)) & 255u);
        const int split_b = 256 - static_cast<int>((ci_lo + rb * static_cast<uint32_t>(nkb)) & 255u);
        const float2 mra = lds64f_nv(scl + meta_off + ra * 8);
        const float2 mrb = lds64f_nv(scl + meta_off + rb * 8);
        const uint32_t cab = lds16_nv(scl + ra * code_pitch + (bt & ~1)) >> (8 * (bt & 1));
        const uint32_t cbb = lds16_nv(scl + rb * code_pitch + (bt & ~1)) >> (8 * (bt & 1));
        const float2 va = e4m3x2_to_float2(cab & 0xffu), vb = e4m3x2_to_float2(cbb & 0xffu);
        const float cta = valid ? __fmul_rn(va.x, bt < split_a ? mra.x : mra.y) : 0.f;
        const float ctb = valid ? __fmul_rn(vb.x, bt < split_b ? mrb.x : mrb.y) : 0.f;
        const uint64_t cta2 = splat_f32x2(cta), ctb2 = splat_f32x2(ctb);
        // this lane's 32 packed bytes of each row: tile layout [chunk][R
        // rows][128 bytes], 16-byte units swizzled by (row & 7); block c is
        // units 2c, 2c + 1
        const uint32_t chunk = ring + cw * (R * 128);
        uint32_t wa[8], wb[8];
        {
            const uint32_t ua = chunk + ra * 128, ub = chunk + rb * 128;
            const uint32_t u0 = static_cast<uint32_t>((2 * c) ^ (ra & 7)) << 4;
            const uint32_t u1 = static_cast<uint32_t>((2 * c + 1) ^ (ra & 7)) << 4;
            asm("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(wa[0]), "=r"(wa[1]), "=r"(wa[2]), "=r"(wa[3]) : "r"(ua + u0));
            asm("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(wa[4]), "=r"(wa[5]), "=r"(wa[6]), "=r"(wa[7]) : "r"(ua + u1));
            asm("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(wb[0]), "=r"(wb[1]), "=r"(wb[2]), "=r"(wb[3]) : "r"(ub + u0));
            asm("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(wb[4]), "=r"(wb[5]), "=r"(wb[6]), "=r"(wb[7]) : "r"(ub + u1));
        }
        // activations of this lane's token(s) for block bs: the block's
        // 128-byte line of the slab (or the zero line past the slice or the
        // batch); unit j of it sits at line ^ ((j ^ key) << 3) (x_off)
        uint32_t xk[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const int tok = g + 8 * t;
            const uint32_t line = valid && tok < xrows ? sp.x + tok * x_pitch + bs * 128 : sp.zero;
            xk[t] = (line + z) | static_cast<uint32_t>((((bs & 3) << 2) | (tok & 3)) << 3);
        }
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            // each packed byte -> its two fp32 codes from the lane's pair
            // table -> fp32 products with c~ (one paired multiply) -> one
            // bf16 pair (RNE): exactly bf16_rne(fp32(q * c~)) for both
            uint32_t oa[4], ob[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                oa[k] = mul_f32x2_to_bf16x2(lds64_nv(prmt(wa[w], lane_lut, 0x7604u | (k << 4))), cta2);
                ob[k] = mul_f32x2_to_bf16x2(lds64_nv(prmt(wb[w], lane_lut, 0x7604u | (k << 4))), ctb2);
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = 2 * w + h;                          // MMA: positions 4j .. 4j + 3
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    uint32_t b0, b1;
                    asm("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(b0), "=r"(b1) : "r"(xk[t] ^ (j << 3)));
                    mma16816_nv(acc[t], oa[2 * h], ob[2 * h], oa[2 * h + 1], ob[2 * h + 1], b0, b1);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            keep_before(acc[t][0]);
            keep_before(acc[t][1]);
            keep_before(acc[t][2]);
            keep_before(acc[t][3]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        ++it;
        if (tile == tiles_per_unit - 1) {
            // The unit is complete.  Each warp writes its 16 rows x M
            // partials; then min(M, 16) warps, a different run of warps for
            // each unit, share the R M additions (each output adds the
            // partials of the D warps of its row group, in warp order).
            // Buffer p is reused every second unit; rfree[p] says the summing
            // warps have read its last contents.
            const int p = units_done & 1;
            const uint32_t use = units_done >> 1;
            const uint32_t red = sp.red + p * red_half;
            if (use > 0 && !mbar_wait(&rfree[p], (use - 1) & 1, abort_flag, a.err)) break;
            // buffer layout [warp][16 rows][M]; only existing tokens are kept
            const uint32_t base = red + static_cast<uint32_t>(warp * 16 * xrows) * 4;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int tok = 8 * t + 2 * c;
                const uint32_t r0 = base + (g * xrows + tok) * 4;
                const uint32_t r1 = base + ((g + 8) * xrows + tok) * 4;
                if (tok < xrows) {
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(r0), "f"(acc[t][0]) : "memory");
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(r1), "f"(acc[t][2]) : "memory");
                }
                if (tok + 1 < xrows) {
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(r0 + 4), "f"(acc[t][1]) : "memory");
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(r1 + 4), "f"(acc[t][3]) : "memory");
                }
                acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&rdone[p]);
            const int nsum = min(kConsumerWarps, xrows);
            const int idx = (warp - unit * nsum) & (kConsumerWarps - 1);
            if (idx < nsum) {
                if (!mbar_wait(&rdone[p], use & 1, abort_flag, a.err)) break;
                for (int e = idx * 32 + lane; e < R * xrows; e += nsum * 32) {
                    const int row = e / xrows, tok = e % xrows;
                    const int w0 = (row >> 4) * D, r16 = row & 15;
                    float sum = 0.f;
                    for (int w = w0; w < w0 + D; ++w)
                        sum += __uint_as_float(lds32(red + ((w * 16 + r16) * xrows + tok) * 4));
                    const int64_t n = int64_t(unit) * R + row;
                    if (n < a.N) part[int64_t(tok) * a.N + n] = sum;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&rfree[p]);
            }
            ++units_done;
        }
    }
}

// One thread per output column n: T = sum of the T partials (staged in
// shared memory), Y[m][n] = bf16( sum_s part[s][m][n] + gamma * T[m] . B[n] ).
__global__ void __launch_bounds__(256)
gemv_finalize_kernel(GemvFinalizeArgs a) {
    __shared__ float st[16 * QLORA_MAX_RANK];
    __shared__ float tsum[256];
    // launched as the GEMV's programmatic dependent: all inputs come from it
    grid_dependency_wait();
    // T: with E = M r <= 256 values, the 256 threads form 256 / E groups that
    // sum interleaved subsets of the partials, then the groups' sums are added
    // in group order; with more values each thread sums whole columns.  The
    // order is fixed either way.
    const int E = static_cast<int>(a.M) * a.r;
    if (E <= 256) {
        const int groups = 256 / E;
        const int e = threadIdx.x % E, gi = threadIdx.x / E;
        if (gi < groups) {
            float t = 0.f;
            for (int s = gi; s < a.t_parts; s += groups) t += a.Tpart[int64_t(s) * E + e];
            tsum[threadIdx.x] = t;
        }
        __syncthreads();
        if (threadIdx.x < E) {
            float t = 0.f;
            for (int g2 = 0; g2 < groups; ++g2) t += tsum[g2 * E + threadIdx.x];
            st[threadIdx.x] = t;
            if (blockIdx.x == 0 && a.T_save) a.T_save[threadIdx.x] = t;
        }
    } else {
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            float t = 0.f;
            for (int s = 0; s < a.t_parts; ++s) t += a.Tpart[int64_t(s) * E + e];
            st[e] = t;
            if (blockIdx.x == 0 && a.T_save) a.T_save[e] = t;
        }
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

int gemv_stages(int64_t M, int64_t kslab) {
    // dynamic shared memory starts after the 1 KiB the driver reserves; the
    // plan must also hold for a base 1 KiB either side of that.  Two stages
    // (64 KiB in flight per SM) still outrun what the consumers take; the
    // slice choice uses them to fit wider activation slabs.
    for (int st = kMaxStages; st >= 2; --st) {
        bool ok = true;
        for (uint32_t start : {0u, 1024u, 2048u})
            ok = ok && plan_smem(start, st, gemv_x_bytes(M, kslab), gemv_red_bytes(M)).ok;
        if (ok) return st;
    }
    return 0;
}

template <int NT, int ST, int D>
static cudaError_t launch_one(dim3 grid, const CUtensorMap& tm, const GemvArgs& a, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<NT, ST, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    gemv_kernel<NT, ST, D><<<grid, kThreads, kSmemBytes, stream>>>(tm, a);
    return cudaGetLastError();
}

template <int NT, int ST>
static cudaError_t launch_depth(dim3 grid, const CUtensorMap& tm, const GemvArgs& a, cudaStream_t stream) {
    switch (a.tile_chunks) {
        case 1: return launch_one<NT, ST, 1>(grid, tm, a, stream);
        case 2: return launch_one<NT, ST, 2>(grid, tm, a, stream);
        case 4: return launch_one<NT, ST, 4>(grid, tm, a, stream);
        case 8: return launch_one<NT, ST, 8>(grid, tm, a, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gemv(const CUtensorMap& tm_packed, const GemvArgs& a, int num_sms,
                        cudaStream_t stream) {
    const unsigned per_slice = static_cast<unsigned>(std::max(1, num_sms / std::max(1, a.splits)));
    dim3 grid(per_slice, static_cast<unsigned>(a.splits));
    const int st = gemv_stages(a.M, std::min<int64_t>(a.K, a.k_per_split));
    if (st == 0) return cudaErrorInvalidConfiguration;
    if (a.M > 8) {
        switch (st) {
            case 6: return launch_depth<2, 6>(grid, tm_packed, a, stream);
            case 5: return launch_depth<2, 5>(grid, tm_packed, a, stream);
            case 4: return launch_depth<2, 4>(grid, tm_packed, a, stream);
            case 3: return launch_depth<2, 3>(grid, tm_packed, a, stream);
            default: return launch_depth<2, 2>(grid, tm_packed, a, stream);
        }
    }
    switch (st) {
        case 6: return launch_depth<1, 6>(grid, tm_packed, a, stream);
        case 5: return launch_depth<1, 5>(grid, tm_packed, a, stream);
        case 4: return launch_depth<1, 4>(grid, tm_packed, a, stream);
        case 3: return launch_depth<1, 3>(grid, tm_packed, a, stream);
        default: return launch_depth<1, 2>(grid, tm_packed, a, stream);
    }
}

cudaError_t launch_gemv_finalize(const GemvFinalizeArgs& a, cudaStream_t stream) {
    if (a.M <= 0 || a.N <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((a.N + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_finalize_kernel, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace qnf4
