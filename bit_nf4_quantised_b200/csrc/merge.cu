// K7: merge for export, W_m = bf16_rne( W~ + gamma * B A ).
//
// "QLoRA, explained", "The forward pass and gradients": the model that was
// fine-tuned is W~ + gamma B A (the quantised base plus the adapter), not
// W0 + gamma B A.  The same page's "Failure modes", "Quality loss at merge
// time", gives dequantising W~ to bf16 and adding the adapter as the merge
// that keeps that model; "QLoRA" (finetunellm.com), "What it costs you", adds
// that a 4-bit deployment re-quantises the merged bf16 weight (qlora_quantize_bf16).
// W~ is rebuilt exactly as K6 does (c~ = fp32(e4m3 * c2), w~ = bf16_rne(fp32(q *
// c~))); the sum is formed in fp32 and rounded to bf16 once.
//
// HBM-bound: 0.516 B read and 2 B written per weight; A [r x K] and B [N x r]
// stay in L2.  The rank-r product B A is a contraction of depth r <= 128, done
// on the warp-level tensor cores (mma.sync m16n8k16, bf16 in, fp32
// accumulate): at r = 16 that is 16 MMAs per 1024 weights, a few per cent of
// the issue slots; the per-weight decode, the fused multiply-add and the two
// roundings make up most of the instruction stream.
//
// Work unit: one CTA tile of 16 rows x 512 columns, each of the 8 warps
// owning one 64-column strip (one NF4 block per row).  Units are ordered by
// column block (all row tiles of columns [c0, c0+512) before the next block)
// and cut into equal contiguous runs, one per CTA of a grid sized to the SMs'
// resident capacity.  Each warp keeps its strip's slice of A in its own
// shared-memory slab, reloaded only when its CTA's run enters the next column
// block, so no CTA-wide barrier is needed.  The 8 warps of a CTA read the same
// 16 rows of B and the same scale-code sectors at about the same time, so
// those reads are served by L1 once per CTA rather than once per warp.  The
// next unit's packed words, scale codes and group scales are loaded before
// the current unit is computed.
//
// Column ownership.  The MMA's output fragment gives lane (g, t) two adjacent
// columns of each 8-wide n-tile.  The 8 n-tiles are mapped to the strip's
// columns so that lane t of a quad owns columns 32i + 8t + (0..7) for i = 0, 1:
// each quad then writes 64 contiguous bytes per store (full 32-byte sectors)
// and needs one 32-bit word of packed indices per row and i (loaded by the
// quad as one 32-byte sector and exchanged by shuffles).  Logical
// column n (0..7) of n-tile nt is physical column
//     32 (nt / 4) + 8 (n / 2) + 2 (nt % 4) + (n % 2),
// and the slab stores A's columns in that logical order so that ldmatrix.trans
// yields the B-operand fragments directly.
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kStrip = 64;                 // columns per warp (one NF4 block per row)
constexpr int kTileRows = 16;              // rows per unit (the MMA's M)
constexpr int kSlabPitch = kStrip + 8;     // bf16 per slab row: 144 B, conflict-free ldmatrix

__host__ __device__ constexpr int slab_bytes(int rp) { return rp * kSlabPitch * 2; }

// Shared memory: the 16 codes; the pair table; the warps' slabs.  The pair
// table holds, for every byte value e of the packed indices, the codes of its
// two nibbles (q[e & 15], q[e >> 4]) as a float pair, one copy per lane:
// entry e of lane l at e * 256 + l * 8, so a warp's lookups never share a
// bank beyond the two wavefronts an 8-byte load takes, and one byte permute
// (the byte into bits 8-15) plus the lane's base address forms the address.
constexpr int kCodesOff = 0;
constexpr int kPairOff = 256;
constexpr int kPairBytes = 256 * 32 * 8;                         // 64 KiB
constexpr int kSlabOff = kPairOff + kPairBytes;

// One lane's weight inputs for a unit: the packed words of its columns in
// rows g and g+8, their blocks' FP8 scale codes and group scales.
struct WeightRegs {
    uint32_t w[2][2];
    uint32_t sc[2];
    float mt[2];
};

// The weights of one launch: their units in sequence (first[j] = the index of
// job j's first unit, first[n] = the total), the slabs sized for the largest
// rank among them.
struct MergeBatch {
    MergeArgs job[kMaxMergeJobs];
    int64_t first[kMaxMergeJobs + 1];
    int n;
    int rp_max;
};

// kMulti: the batch may hold several weights.  A one-weight launch indexes
// job 0 at compile time, so its arguments stay constant-bank operands; a
// batch copies the current job's arguments into registers once per unit.
template <bool kMulti>
__global__ void __launch_bounds__(kThreads)
merge_kernel(const __grid_constant__ MergeBatch bt, Nf4Table tab) {
    extern __shared__ __align__(16) uint8_t smem[];
    float* scode = reinterpret_cast<float*>(smem + kCodesOff);            // 16 codes
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint16_t* slab = reinterpret_cast<uint16_t*>(smem + kSlabOff + warp * slab_bytes(bt.rp_max));
    if (threadIdx.x == 0) {            // constant indices: no local copy of the table
#pragma unroll
        for (int q = 0; q < 16; ++q) scode[q] = tab.code[q];
    }
    __syncthreads();
    // Pair table: thread t writes 16-byte chunks t, t + 256, ...; chunk c holds
    // entry c / 16 for lanes 2 (c % 16) and 2 (c % 16) + 1 (consecutive
    // threads write consecutive chunks: no bank conflicts).
    for (int c = threadIdx.x; c < kPairBytes / 16; c += kThreads) {
        const int e = c >> 4;
        const float lo = scode[e & 15], hi = scode[e >> 4];
        *reinterpret_cast<float4*>(smem + kPairOff + c * 16) = make_float4(lo, hi, lo, hi);
    }
    __syncthreads();
    const uint8_t* pair_lane = smem + kPairOff + lane * 8;

    const int g = lane >> 2, tq = lane & 3;
    // N and K are below 2^31 (checked on the host); products of a row and K
    // are formed in 64 bits.
    const int64_t total = bt.first[bt.n];
    const int64_t u_begin = total * blockIdx.x / gridDim.x;
    const int64_t u_end = total * (blockIdx.x + 1) / gridDim.x;
    auto job = [&](int j) -> MergeArgs { return bt.job[kMulti ? j : 0]; };
    auto rows_of = [&](int j) { return (static_cast<int>(job(j).N) + kTileRows - 1) / kTileRows; };
    auto cblocks_of = [&](int j) { return (static_cast<int>(job(j).K) / kStrip + kWarps - 1) / kWarps; };

    // The slab position lane l fills: A's physical columns 2l, 2l+1 are
    // logical columns p0, p0 + 1 of the strip (see the column map above).
    const int pc = 2 * lane;
    const int p0 = 8 * (4 * (pc >> 5) + ((pc & 7) >> 1)) + 2 * ((pc & 31) >> 3);

    // ldmatrix.x4.trans addressing: matrix m = lane / 8 covers slab rows
    // (m & 1) * 8 + (lane & 7) of the k-step, n-tile (m >> 1) of the pair.
    const int lm_row = ((lane >> 3) & 1) * 8 + (lane & 7);
    const int lm_col = (lane >> 4) * 8;
    const uint32_t slab_s = smem_u32(slab);

    // Packed words: the quad loads its row's 32 bytes as four 8-byte pieces
    // (one sector, one request); lane t then needs words t and t + 4, held by
    // lanes t/2 and 2 + t/2 of its quad.
    const int qbase = lane & ~3;
    const int src_a = qbase + (tq >> 1), src_b = qbase + 2 + (tq >> 1);

    // Unit (job j, column block cb, row tile rt); units advance row tile
    // first, then column block, then job.
    auto load_unit = [&](int j, int cb, int rt, WeightRegs& wr) {
        const MergeArgs a = job(j);
        const int N = static_cast<int>(a.N), K = static_cast<int>(a.K);
        const int kblocks = K / kStrip;
        const int strip = cb * kWarps + warp;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            const int R = rt * kTileRows + g + 8 * s;
            uint2 v = make_uint2(0u, 0u);
            wr.sc[s] = 0u;
            wr.mt[s] = 0.f;
            if (R < N && strip < kblocks) {
                const uint64_t e0 = uint64_t(R) * uint64_t(K) + uint64_t(strip) * kStrip;
                v = __ldcs(reinterpret_cast<const uint2*>(a.packed + (e0 >> 3)) + tq);
                const uint64_t b = e0 >> 6;                     // flat block index
                wr.sc[s] = a.scale_codes[b];
                wr.mt[s] = a.meta[b >> 8];
            }
            wr.w[s][0] = v.x;       // exchanged below, after the loads have been issued
            wr.w[s][1] = v.y;
        }
    };
    auto exchange = [&](WeightRegs& wr) {
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            const uint32_t ax = __shfl_sync(0xffffffffu, wr.w[s][0], src_a);
            const uint32_t ay = __shfl_sync(0xffffffffu, wr.w[s][1], src_a);
            const uint32_t bx = __shfl_sync(0xffffffffu, wr.w[s][0], src_b);
            const uint32_t by = __shfl_sync(0xffffffffu, wr.w[s][1], src_b);
            wr.w[s][0] = (tq & 1) ? ay : ax;
            wr.w[s][1] = (tq & 1) ? by : bx;
        }
    };

    int j = 0;
    if (kMulti)
        while (j + 1 < bt.n && bt.first[j + 1] <= u_begin) ++j;
    int cb, rt;
    {
        const int64_t local = u_begin - bt.first[j];
        const int rtj = rows_of(j);
        cb = static_cast<int>(local / rtj);
        rt = static_cast<int>(local - int64_t(cb) * rtj);
    }
    // the unit after (j, cb, rt)
    auto advance = [&](int& jj, int& cc, int& rr) {
        if (++rr == rows_of(jj)) {
            rr = 0;
            if (++cc == cblocks_of(jj)) {
                cc = 0;
                ++jj;
            }
        }
    };
    int nj = j, ncb = cb, nrt = rt;
    advance(nj, ncb, nrt);
    WeightRegs cur, nxt;
    if (u_begin < u_end) load_unit(j, cb, rt, cur);
    int cur_j = -1, cur_cb = -1;
    for (int64_t u = u_begin; u < u_end; ++u) {
        if (u + 1 < u_end) load_unit(nj, ncb, nrt, nxt);
        exchange(cur);
        const MergeArgs a = job(j);
        const int N = static_cast<int>(a.N), K = static_cast<int>(a.K);
        const int kblocks = K / kStrip;
        const int strip = cb * kWarps + warp;
        if (strip < kblocks) {
            const int c0 = strip * kStrip;
            if (cb != cur_cb || j != cur_j) {
                __syncwarp();
                for (int k = 0; k < a.rp; ++k) {
                    uint32_t v = 0u;
                    if (k < a.r) v = *reinterpret_cast<const uint32_t*>(a.A + int64_t(k) * K + c0 + pc);
                    *reinterpret_cast<uint32_t*>(slab + k * kSlabPitch + p0) = v;
                }
                __syncwarp();
                cur_cb = cb;
                cur_j = j;
            }
            const int n0 = rt * kTileRows;

            // acc[nt][.] = (B A)[rows g, g+8][logical columns 2t, 2t+1 of n-tile nt]
            float acc[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;

            const int R0 = n0 + g, R1 = n0 + g + 8;
            for (int k0 = 0; k0 < a.rp; k0 += 16) {
                uint32_t af[4];
                const int ka = k0 + 2 * tq, kb = k0 + 8 + 2 * tq;
                const uint16_t* b0p = a.B + int64_t(R0) * a.r;
                const uint16_t* b1p = a.B + int64_t(R1) * a.r;
                af[0] = (R0 < N && ka < a.r) ? *reinterpret_cast<const uint32_t*>(b0p + ka) : 0u;
                af[1] = (R1 < N && ka < a.r) ? *reinterpret_cast<const uint32_t*>(b1p + ka) : 0u;
                af[2] = (R0 < N && kb < a.r) ? *reinterpret_cast<const uint32_t*>(b0p + kb) : 0u;
                af[3] = (R1 < N && kb < a.r) ? *reinterpret_cast<const uint32_t*>(b1p + kb) : 0u;
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(slab_s + 2u * uint32_t((k0 + lm_row) * kSlabPitch + np * 16 + lm_col),
                              b0, b1, b2, b3);
                    mma_bf16_16816(acc[2 * np], af[0], af[1], af[2], af[3], b0, b1);
                    mma_bf16_16816(acc[2 * np + 1], af[0], af[1], af[2], af[3], b2, b3);
                }
            }

            // Epilogue: W~ from the packed word, plus gamma * (B A), rounded once.
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const int R = n0 + g + 8 * s;
                uint16_t* orow = a.out + int64_t(R) * K + c0 + 8 * tq;
                const float ct = __fmul_rn(e4m3_to_float(static_cast<uint8_t>(cur.sc[s])), cur.mt[s]);
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const uint32_t v = cur.w[s][i];
                    uint32_t o[4];
#pragma unroll
                    for (int jp = 0; jp < 4; ++jp) {
                        // physical columns 32i + 8t + 2jp, +1 <- n-tile 4i + jp, logical 2t, 2t+1
                        const float2 qp = *reinterpret_cast<const float2*>(
                            pair_lane + prmt(v, 0u, 0x4404u | (uint32_t(jp) << 4)));
                        const uint32_t wb = pack_bf16x2(__fmul_rn(qp.x, ct), __fmul_rn(qp.y, ct));
                        const float wlo = __uint_as_float(wb << 16);
                        const float whi = __uint_as_float(wb & 0xffff0000u);
                        o[jp] = pack_bf16x2(__fmaf_rn(a.gamma, acc[4 * i + jp][2 * s], wlo),
                                            __fmaf_rn(a.gamma, acc[4 * i + jp][2 * s + 1], whi));
                    }
                    if (R < N)
                        __stcs(reinterpret_cast<uint4*>(orow + 32 * i), make_uint4(o[0], o[1], o[2], o[3]));
                }
            }
        }
        cur = nxt;
        j = nj;
        cb = ncb;
        rt = nrt;
        if (u + 1 < u_end) advance(nj, ncb, nrt);
    }
}

}  // namespace

int merge_smem_bytes(int r) {
    const int rp = (r + 15) / 16 * 16;
    return kSlabOff + kWarps * slab_bytes(rp);
}

cudaError_t launch_merge(const MergeArgs* jobs, int n, const Nf4Table& tab, int num_sms,
                         cudaStream_t stream) {
    if (n < 1 || n > kMaxMergeJobs) return cudaErrorInvalidValue;
    MergeBatch bt{};
    bt.n = 0;
    bt.rp_max = 16;
    int64_t total = 0;
    for (int i = 0; i < n; ++i) {
        MergeArgs a = jobs[i];
        a.rp = (a.r + 15) / 16 * 16;
        const int64_t col_blocks = (a.K / kStrip + kWarps - 1) / kWarps;
        a.tiles = col_blocks * ((a.N + kTileRows - 1) / kTileRows);   // CTA units
        if (a.tiles == 0) continue;
        bt.job[bt.n] = a;
        bt.first[bt.n] = total;
        total += a.tiles;
        if (a.rp > bt.rp_max) bt.rp_max = a.rp;
        ++bt.n;
    }
    bt.first[bt.n] = total;
    if (total == 0) return cudaSuccess;
    const int smem = merge_smem_bytes(bt.rp_max);
    const auto kernel = bt.n > 1 ? merge_kernel<true> : merge_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    int64_t grid = int64_t(num_sms) * per_sm;
    if (grid > total) grid = total;                               // at least one unit per CTA
    kernel<<<dim3(static_cast<unsigned>(grid)), kThreads, smem, stream>>>(bt, tab);
    return cudaGetLastError();
}

}  // namespace qnf4
