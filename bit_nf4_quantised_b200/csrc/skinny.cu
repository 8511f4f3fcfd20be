// K4: the rank-r LoRA side products of the adapted layer
// ("QLoRA, explained", "The forward pass and gradients"):
//   T = X A^T,  U = dY B,  dB = gamma dY^T T,  dA^T = X^T (gamma U).
// All are one long contraction (over K, N or the M tokens) with one short
// output side (r <= 128): HBM-bound streams over X or dY.  One kernel covers
// the four operand layouts.  A CTA of 4 warps owns 64 rows of the long output
// side and all r columns of one contraction slice, streams the slice through
// a deep cp.async ring (8 stages of 64 contraction positions for r <= 64: a
// CTA keeps 7 chunks in flight; one barrier per stage) and feeds mma.sync
// m16n8k16 (bf16 in, fp32 accumulate) through ldmatrix (.trans where the
// stored layout is the transpose).  The slices of a row block form one thread-block cluster (up to
// 8 CTAs): each parks its fp32 partial in shared memory, then every CTA sums
// one slice of the rows over all partials through distributed shared memory
// and writes the finished result -- scaled fp32 (optionally transposed or
// accumulated) and/or the zero-padded bf16 copy the tensor-core kernels
// consume.  No partial buffer in HBM, no separate reduction launch, and a
// fixed summation order.
#include <cooperative_groups.h>

#include "kernels.cuh"

namespace cg = cooperative_groups;

namespace qnf4 {

namespace {

constexpr int kThreads = 128;
constexpr int TI = 64;           // output rows per CTA
constexpr int TC = 64;           // contraction per stage
constexpr int kPitchK = TC * 2 + 16;   // bytes per 64-wide row (+16 against bank conflicts)

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <bool PK, bool QK, int JT16>
struct SkinnyTile {
    static constexpr int JP = JT16 * 16;
    static constexpr int kPBytes = TI * kPitchK;                        // 9216
    static constexpr int kQPitch = QK ? kPitchK : (JP * 2 + 16);
    static constexpr int kQBytes = QK ? JP * kPitchK : TC * kQPitch;
    static constexpr int kStage = kPBytes + kQBytes;
    // ring depth: 8 stages (7 chunks in flight per CTA), fewer where a stage
    // is large (r > 64) so that the ring stays within 200 KiB
    static constexpr int kStages = (200 * 1024 / kStage) < 8 ? (200 * 1024 / kStage) : 8;
    static constexpr int kRedBytes = TI * JP * 4;                       // fp32 partial tile
    static constexpr int kSmem = (kStages * kStage > kRedBytes) ? kStages * kStage : kRedBytes;
    static_assert(kStages >= 3, "skinny ring depth");
};

template <bool PK, bool QK, int JT16>
__global__ void __launch_bounds__(kThreads)
skinny_kernel(SkinnyArgs a) {
    using Tl = SkinnyTile<PK, QK, JT16>;
    extern __shared__ __align__(16) uint8_t smem[];
    // a dependent tensor-core GEMM may start streaming its weight tiles now;
    // it waits for this grid only before it reads this kernel's output
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the call's error word is cleared before a dependent may start
    if (a.err_zero != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) *a.err_zero = 0;
    if (a.trigger_dependents) launch_dependents();
    cg::cluster_group cluster = cg::this_cluster();
    const int64_t i0 = int64_t(blockIdx.x) * TI;
    const int split = blockIdx.y;
    const int64_t c_beg = int64_t(split) * a.c_per_split;
    const int64_t c_end = min(a.C, c_beg + a.c_per_split);
    const int nchunks = c_end > c_beg ? static_cast<int>((c_end - c_beg + TC - 1) / TC) : 0;
    const uint32_t sbase = smem_u32(smem);

    auto load_stage = [&](int chunk, int st) {
        const int64_t c0 = c_beg + int64_t(chunk) * TC;
        const uint32_t sp = sbase + st * Tl::kStage;
        const uint32_t sq = sp + Tl::kPBytes;
#pragma unroll
        for (int q = tid; q < TI * 8; q += kThreads) {          // P tile: 64 x 64
            const int row = q >> 3, ch = q & 7;
            const uint16_t* src;
            bool ok;
            if (PK) {
                ok = (i0 + row < a.I) && (c0 + ch * 8 < c_end);
                src = a.P + (i0 + row) * a.ldp + c0 + ch * 8;
            } else {
                ok = (c0 + row < c_end) && (i0 + ch * 8 < a.I);
                src = a.P + (c0 + row) * a.ldp + i0 + ch * 8;
            }
            cp_async16(sp + row * kPitchK + ch * 16, ok ? src : a.P, ok);
        }
        if (QK) {
            for (int q = tid; q < Tl::JP * 8; q += kThreads) {
                const int row = q >> 3, ch = q & 7;
                const bool ok = (row < a.J) && (c0 + ch * 8 < c_end);
                const uint16_t* src = a.Q + int64_t(row) * a.ldq + c0 + ch * 8;
                cp_async16(sq + row * Tl::kQPitch + ch * 16, ok ? src : a.Q, ok);
            }
        } else {
            constexpr int cpr = Tl::JP / 8;                        // chunks per row
            for (int q = tid; q < TC * cpr; q += kThreads) {
                const int row = q / cpr, ch = q % cpr;
                const bool ok = (c0 + row < c_end) && (ch * 8 < a.J);
                const uint16_t* src = a.Q + (c0 + row) * a.ldq + ch * 8;
                cp_async16(sq + row * Tl::kQPitch + ch * 16, ok ? src : a.Q, ok);
            }
        }
    };

    float acc[JT16][2][4];
#pragma unroll
    for (int j = 0; j < JT16; ++j)
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][t][e] = 0.f;

    constexpr int kStages = Tl::kStages;
#pragma unroll
    for (int st = 0; st < kStages - 1; ++st) {
        if (st < nchunks) load_stage(st, st);
        cp_async_commit();
    }
    for (int chunk = 0; chunk < nchunks; ++chunk) {
        const int st = chunk % kStages;
        // this chunk's copies have landed (the kStages - 2 later ones may
        // still fly); after the barrier every warp is also done with the
        // previous chunk's stage, which the next prefetch overwrites, so one
        // barrier per chunk suffices
        cp_async_wait<kStages - 2>();
        __syncthreads();
        if (chunk + kStages - 1 < nchunks) load_stage(chunk + kStages - 1, (chunk + kStages - 1) % kStages);
        cp_async_commit();
        const uint32_t sp = sbase + st * Tl::kStage;
        const uint32_t sq = sp + Tl::kPBytes;
        const int mi = lane >> 3, r8 = lane & 7;
#pragma unroll
        for (int kk = 0; kk < TC / 16; ++kk) {
            uint32_t a0, a1, a2, a3;
            if (PK) {
                const int row = warp * 16 + r8 + (mi & 1) * 8;
                const int col = kk * 16 + (mi >> 1) * 8;
                ldsm_x4(sp + row * kPitchK + col * 2, a0, a1, a2, a3);
            } else {
                const int row = kk * 16 + r8 + (mi >> 1) * 8;
                const int col = warp * 16 + (mi & 1) * 8;
                ldsm_x4_t(sp + row * kPitchK + col * 2, a0, a1, a2, a3);
            }
#pragma unroll
            for (int jt = 0; jt < JT16; ++jt) {
                uint32_t b0, b1, b2, b3;
                if (QK) {
                    const int row = jt * 16 + r8 + (mi >> 1) * 8;
                    const int col = kk * 16 + (mi & 1) * 8;
                    ldsm_x4(sq + row * Tl::kQPitch + col * 2, b0, b1, b2, b3);
                } else {
                    const int row = kk * 16 + r8 + (mi & 1) * 8;
                    const int col = jt * 16 + (mi >> 1) * 8;
                    ldsm_x4_t(sq + row * Tl::kQPitch + col * 2, b0, b1, b2, b3);
                }
                mma_bf16_16816(acc[jt][0], a0, a1, a2, a3, b0, b1);
                mma_bf16_16816(acc[jt][1], a0, a1, a2, a3, b2, b3);
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // park the partial tile [64][JP] in shared memory
    float* red = reinterpret_cast<float*>(smem);
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int jt = 0; jt < JT16; ++jt)
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = warp * 16 + g + h * 8;
                const int col = jt * 16 + t * 8 + 2 * c;
                *reinterpret_cast<float2*>(red + row * Tl::JP + col) =
                    make_float2(acc[jt][t][2 * h], acc[jt][t][2 * h + 1]);
            }
    cluster.sync();

    // Every CTA of the cluster finalises its own slice of the 64 rows, summing
    // the partials of all slices (float4 loads, issued before any use).
    const int nsplit = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int rows_per = (TI + nsplit - 1) / nsplit;
    const int r0 = rank * rows_per, r1 = min(TI, r0 + rows_per);
    constexpr int kC4 = Tl::JP / 4;
    const float4* parts[kMaxSkinnySplits];
#pragma unroll
    for (int q = 0; q < kMaxSkinnySplits; ++q)
        parts[q] = reinterpret_cast<const float4*>(cluster.map_shared_rank(red, q < nsplit ? q : 0));
    for (int g4 = tid; g4 < (r1 - r0) * kC4; g4 += kThreads) {
        const int li = r0 + g4 / kC4, c4 = g4 % kC4;
        const int64_t i = i0 + li;
        float4 v[kMaxSkinnySplits];
#pragma unroll
        for (int q = 0; q < kMaxSkinnySplits; ++q)
            if (q < nsplit) v[q] = parts[q][li * kC4 + c4];
        float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int q = 0; q < kMaxSkinnySplits; ++q)
            if (q < nsplit) {
                sum[0] += v[q].x;
                sum[1] += v[q].y;
                sum[2] += v[q].z;
                sum[3] += v[q].w;
            }
        if (i >= a.I) continue;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int j = c4 * 4 + e;
            const float val = sum[e] * a.alpha;
            if (j < a.J && a.out) {
                float* o = a.transpose ? (a.out + int64_t(j) * a.I + i) : (a.out + i * a.J + j);
                *o = a.accumulate ? (*o + val) : val;
            }
            if (a.out_bf16 && j < a.ldb) {
                __nv_bfloat16 bv = __float2bfloat16_rn(j < a.J ? val * a.beta : 0.f);
                a.out_bf16[i * a.ldb + j] = *reinterpret_cast<uint16_t*>(&bv);
            }
        }
    }
    if (a.out_bf16 && a.ldb > Tl::JP) {          // zero padding beyond the tile width
        const int padw = static_cast<int>(a.ldb) - Tl::JP;
        for (int e = tid; e < (r1 - r0) * padw; e += kThreads) {
            const int64_t i = i0 + r0 + e / padw;
            if (i < a.I) a.out_bf16[i * a.ldb + Tl::JP + e % padw] = 0;
        }
    }
    // side job: bf16 copy of a fp32 [I x J] source for the same rows
    if (a.cvt_src != nullptr) {
        const int c4w = static_cast<int>(a.ldb) / 4;
        for (int e = tid; e < (r1 - r0) * c4w; e += kThreads) {
            const int64_t i = i0 + r0 + e / c4w;
            const int j = (e % c4w) * 4;
            if (i >= a.I) continue;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j < a.J) v = *reinterpret_cast<const float4*>(a.cvt_src + i * a.J + j);
            const uint32_t lo = pack_bf16x2(v.x * a.cvt_scale, v.y * a.cvt_scale);
            const uint32_t hi = pack_bf16x2(v.z * a.cvt_scale, v.w * a.cvt_scale);
            *reinterpret_cast<uint2*>(a.cvt_dst + i * a.ldb + j) = make_uint2(lo, hi);
        }
    }
    cluster.sync();            // keep every partial alive until the sum is done
}

template <bool PK, bool QK, int JT16>
cudaError_t run_skinny(const SkinnyArgs& a, cudaStream_t stream) {
    using Tl = SkinnyTile<PK, QK, JT16>;
    cudaError_t e = cudaFuncSetAttribute(skinny_kernel<PK, QK, JT16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Tl::kSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((a.I + TI - 1) / TI), static_cast<unsigned>(a.splits));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = Tl::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = static_cast<unsigned>(a.splits);
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.programmatic ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, skinny_kernel<PK, QK, JT16>, a);
}

template <bool PK, bool QK>
cudaError_t dispatch_j(const SkinnyArgs& a, cudaStream_t stream) {
    switch ((a.J + 15) / 16) {
        case 1: return run_skinny<PK, QK, 1>(a, stream);
        case 2: return run_skinny<PK, QK, 2>(a, stream);
        case 3: return run_skinny<PK, QK, 3>(a, stream);
        case 4: return run_skinny<PK, QK, 4>(a, stream);
        case 5: return run_skinny<PK, QK, 5>(a, stream);
        case 6: return run_skinny<PK, QK, 6>(a, stream);
        case 7: return run_skinny<PK, QK, 7>(a, stream);
        case 8: return run_skinny<PK, QK, 8>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_skinny(bool p_kmajor, bool q_kmajor, const SkinnyArgs& a, cudaStream_t stream) {
    if (a.I <= 0 || a.J <= 0 || a.splits < 1 || a.splits > kMaxSkinnySplits)
        return a.I <= 0 ? cudaSuccess : cudaErrorInvalidValue;
    if (p_kmajor && q_kmajor) return dispatch_j<true, true>(a, stream);
    if (p_kmajor && !q_kmajor) return dispatch_j<true, false>(a, stream);
    if (!p_kmajor && !q_kmajor) return dispatch_j<false, false>(a, stream);
    return dispatch_j<false, true>(a, stream);
}

}  // namespace qnf4
