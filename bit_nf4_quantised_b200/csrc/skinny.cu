// K4: the rank-r LoRA side products of the adapted layer
// ("QLoRA, explained", "The forward pass and gradients"):
//   T = X A^T,  U = dY B,  dB = gamma dY^T T,  dA^T = X^T (gamma U).
// All are one long contraction (over K, N or the M tokens) with one short
// output side (r <= 128), so they are HBM-bound streams over X or dY.  One
// kernel covers the four operand layouts: a CTA of 4 warps owns 64 rows of
// the long output side and all r columns, streams its contraction slice
// through a 2-stage cp.async ring, and feeds mma.sync m16n8k16 (bf16 in, fp32
// accumulate) through ldmatrix (.trans where the stored layout is the
// transpose).  Slices write fp32 partials; a finalize pass sums them, applies
// gamma, and emits the fp32 result and/or the bf16 copy the tcgen05 kernels
// consume.
#include "kernels.cuh"

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

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <bool PK, bool QK, int JT16>
struct SkinnyTile {
    static constexpr int JP = JT16 * 16;
    static constexpr int kPBytes = TI * kPitchK;                        // 9216
    static constexpr int kQPitch = QK ? kPitchK : (JP * 2 + 16);
    static constexpr int kQBytes = QK ? JP * kPitchK : TC * kQPitch;
    static constexpr int kStage = kPBytes + kQBytes;
    static constexpr int kSmem = 2 * kStage;
};

template <bool PK, bool QK, int JT16>
__global__ void __launch_bounds__(kThreads)
skinny_kernel(SkinnyArgs a) {
    using Tl = SkinnyTile<PK, QK, JT16>;
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t i0 = int64_t(blockIdx.x) * TI;
    const int64_t c_beg = int64_t(blockIdx.y) * a.c_per_split;
    const int64_t c_end = min(a.C, c_beg + a.c_per_split);
    const int nchunks = static_cast<int>((c_end - c_beg + TC - 1) / TC);
    const uint32_t sbase = smem_u32(smem);

    auto load_stage = [&](int chunk, int st) {
        const int64_t c0 = c_beg + int64_t(chunk) * TC;
        const uint32_t sp = sbase + st * Tl::kStage;
        const uint32_t sq = sp + Tl::kPBytes;
        // P tile: 64 x 64 elements = 512 chunks of 16 B
#pragma unroll
        for (int q = tid; q < TI * 8; q += kThreads) {
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
            constexpr int cpr = Tl::JP / 8;            // chunks per row
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

    if (nchunks > 0) load_stage(0, 0);
    cp_async_commit();
    for (int chunk = 0; chunk < nchunks; ++chunk) {
        const int st = chunk & 1;
        if (chunk + 1 < nchunks) load_stage(chunk + 1, st ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
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
        __syncthreads();
    }

    // write the partial tile
    float* part = a.part + int64_t(blockIdx.y) * a.I * a.J;
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int jt = 0; jt < JT16; ++jt)
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int64_t j = jt * 16 + t * 8 + 2 * c;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t i = i0 + warp * 16 + g + h * 8;
                if (i < a.I && j < a.J)
                    *reinterpret_cast<float2*>(part + i * a.J + j) =
                        make_float2(acc[jt][t][2 * h], acc[jt][t][2 * h + 1]);
            }
        }
}

template <bool PK, bool QK, int JT16>
cudaError_t run_skinny(const SkinnyArgs& a, cudaStream_t stream) {
    using Tl = SkinnyTile<PK, QK, JT16>;
    cudaError_t e = cudaFuncSetAttribute(skinny_kernel<PK, QK, JT16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Tl::kSmem);
    if (e != cudaSuccess) return e;
    dim3 grid(static_cast<unsigned>((a.I + TI - 1) / TI), static_cast<unsigned>(a.splits));
    skinny_kernel<PK, QK, JT16><<<grid, kThreads, Tl::kSmem, stream>>>(a);
    return cudaGetLastError();
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

__global__ void finalize_kernel(FinalizeArgs a) {
    const int64_t total = a.I * (a.out_bf16 ? a.ldb : a.J);
    const int64_t width = a.out_bf16 ? a.ldb : a.J;
    for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total;
         idx += int64_t(gridDim.x) * blockDim.x) {
        const int64_t i = idx / width, j = idx % width;
        if (j >= a.J) {                              // zero padding of the bf16 copy
            a.out_bf16[i * a.ldb + j] = 0;
            continue;
        }
        float s = 0.f;
        for (int k = 0; k < a.splits; ++k) s += a.part[(int64_t(k) * a.I + i) * a.J + j];
        s *= a.alpha;
        if (a.out) {
            float* o = a.transpose ? (a.out + j * a.I + i) : (a.out + i * a.J + j);
            *o = a.accumulate ? (*o + s) : s;
        }
        if (a.out_bf16) {
            __nv_bfloat16 b = __float2bfloat16_rn(s * a.beta);
            a.out_bf16[i * a.ldb + j] = *reinterpret_cast<uint16_t*>(&b);
        }
    }
}

__global__ void pad_copy_kernel(const uint16_t* src, int64_t R1, int64_t C1, uint16_t* dst,
                                int64_t R2, int64_t C2) {
    const int64_t total = R2 * C2;
    for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total;
         idx += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = idx / C2, c = idx % C2;
        dst[idx] = (r < R1 && c < C1) ? src[r * C1 + c] : uint16_t(0);
    }
}

unsigned grid_for(int64_t n, int threads) {
    int64_t g = (n + threads - 1) / threads;
    if (g > 4096) g = 4096;
    if (g < 1) g = 1;
    return static_cast<unsigned>(g);
}

}  // namespace

cudaError_t launch_skinny(bool p_kmajor, bool q_kmajor, const SkinnyArgs& a, cudaStream_t stream) {
    if (a.I <= 0 || a.J <= 0) return cudaSuccess;
    if (p_kmajor && q_kmajor) return dispatch_j<true, true>(a, stream);
    if (p_kmajor && !q_kmajor) return dispatch_j<true, false>(a, stream);
    if (!p_kmajor && !q_kmajor) return dispatch_j<false, false>(a, stream);
    return dispatch_j<false, true>(a, stream);
}

cudaError_t launch_finalize(const FinalizeArgs& a, cudaStream_t stream) {
    const int64_t total = a.I * (a.out_bf16 ? a.ldb : a.J);
    if (total <= 0) return cudaSuccess;
    finalize_kernel<<<grid_for(total, 256), 256, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_pad_copy(const uint16_t* src, int64_t R1, int64_t C1, uint16_t* dst, int64_t R2,
                            int64_t C2, cudaStream_t stream) {
    if (R2 * C2 <= 0) return cudaSuccess;
    pad_copy_kernel<<<grid_for(R2 * C2, 256), 256, 0, stream>>>(src, R1, C1, dst, R2, C2);
    return cudaGetLastError();
}

}  // namespace qnf4
