// K5: bandwidth-bound dequant-GEMV for decode-sized token counts (M <= 16):
//   Y = X W~^T + (gamma T) B^T
// ("QLoRA, explained": serving the adapter unmerged on the 4-bit base, "Failure
// modes ..." / "When to use QLoRA").  The packed weight is streamed once from
// HBM; nothing about it is staged in shared memory.
//
// Swap-AB on mma.sync m16n8k16: rows of W are the MMA's M side, tokens its N
// side (one n8 tile for M <= 8, two for M <= 16).  A lane owns 8 contiguous
// bytes (16 nibbles) of rows g and g+8 of a 16-row tile per 64-wide block and
// turns each byte into the bf16 pair (q[lo], q[hi]) with one shared-memory
// lookup in a byte->bf16x2 table replicated per lane (256 entries x 32 lanes,
// so every lane always hits its own bank).  The contraction order inside a
// block is permuted (lane c of a row group covers k = 16c .. 16c+15, four
// k-values per MMA step) and the activation fragment is gathered with the
// same permutation, so each MMA step is still an exact dot product over its
// 16 k-values.  A block's MMAs accumulate into fresh fp32 registers that are
// then scaled by the block's c~ = e4m3(code) * c2: the per-block scale is
// applied once per 64 weights instead of once per weight.
//
// Deviation from the forward GEMM, stated: the table holds bf16(q[i]) rather
// than bf16(q[i] * c~), so each weight enters as bf16(q) * c~ in fp32; the
// difference from bf16_rne(q * c~) is below one bf16 ulp per weight, far
// inside the layer tolerance, and the bit-exact W~ contract is carried by the
// dequantise and GEMM kernels.
//
// A CTA owns 256 rows x one contraction slice; slices write fp32 partials
// that the finalize kernel sums together with the LoRA term.
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kThreads = 256;
constexpr int kRows = 256;                 // rows of W per CTA (16 row tiles)
constexpr int kLutBytes = 256 * 32 * 4;    // 32 KiB

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lut(uint32_t lut_base, uint32_t byte) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(lut_base + (byte << 7)));
    return v;
}

template <bool kTwoTiles>
__global__ void __launch_bounds__(kThreads)
gemv_kernel(GemvArgs a, int x_pitch_bytes) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t lut_base = smem_u32(smem) + lane * 4;
    uint8_t* sx = smem + kLutBytes;

    // byte -> (bf16 q[lo nibble], bf16 q[hi nibble])
    for (int e = tid; e < 256 * 32; e += kThreads) {
        const int b = e >> 5;
        reinterpret_cast<uint32_t*>(smem)[e] = pack_bf16x2(a.tab.code[b & 15], a.tab.code[b >> 4]);
    }
    // activation slice [16 tokens][kslab] bf16, zero beyond M and K
    const int64_t k_beg = int64_t(blockIdx.y) * a.k_per_split;
    const int64_t k_end = min(a.K, k_beg + a.k_per_split);
    const int kslab = static_cast<int>(k_end - k_beg);
    const int vec_per_row = kslab / 8;
    for (int q = tid; q < 16 * vec_per_row; q += kThreads) {
        const int m = q / vec_per_row, v = q % vec_per_row;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (m < a.M) val = *reinterpret_cast<const uint4*>(a.X + m * a.K + k_beg + v * 8);
        // rows are 8-byte aligned only (pitch = 8 mod 16): two 8-byte stores
        uint2* dst = reinterpret_cast<uint2*>(sx + m * x_pitch_bytes + v * 16);
        dst[0] = make_uint2(val.x, val.y);
        dst[1] = make_uint2(val.z, val.w);
    }
    __syncthreads();

    const int g = lane >> 2, c = lane & 3;
    const int64_t nkb = a.K / QLORA_BLOCK;
    const int kb_beg = static_cast<int>(k_beg / QLORA_BLOCK);
    const int nblk = kslab / QLORA_BLOCK;
    const uint32_t sx_base = smem_u32(sx);
    float* part = a.part + int64_t(blockIdx.y) * a.M * a.N;

#pragma unroll 1
    for (int rt = warp; rt < kRows / 16; rt += kThreads / 32) {
        const int64_t na = int64_t(blockIdx.x) * kRows + rt * 16 + g;
        const int64_t nb = na + 8;
        const bool va = na < a.N, vb = nb < a.N;
        const uint8_t* pa = a.packed + na * (a.K / 2) + c * 8;
        const uint8_t* pb = a.packed + nb * (a.K / 2) + c * 8;
        float acc0[4] = {0.f, 0.f, 0.f, 0.f};
        float acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int bi = 0; bi < nblk; ++bi) {
            const int64_t kb = kb_beg + bi;
            uint2 wa = make_uint2(0, 0), wb = make_uint2(0, 0);
            float cta = 0.f, ctb = 0.f;
            if (va) {
                wa = __ldcs(reinterpret_cast<const uint2*>(pa + kb * 32));
                const int64_t ci = na * nkb + kb;
                cta = __fmul_rn(e4m3_to_float(__ldg(a.scale_codes + ci)), __ldg(a.meta + (ci >> 8)));
            }
            if (vb) {
                wb = __ldcs(reinterpret_cast<const uint2*>(pb + kb * 32));
                const int64_t ci = nb * nkb + kb;
                ctb = __fmul_rn(e4m3_to_float(__ldg(a.scale_codes + ci)), __ldg(a.meta + (ci >> 8)));
            }
            float blk0[4] = {0.f, 0.f, 0.f, 0.f};
            float blk1[4] = {0.f, 0.f, 0.f, 0.f};
            const uint32_t xk = sx_base + static_cast<uint32_t>((bi * 64 + c * 16) * 2);
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint32_t wa_s = s < 2 ? wa.x : wa.y;
                const uint32_t wb_s = s < 2 ? wb.x : wb.y;
                const int sh = (s & 1) * 16;
                const uint32_t a0 = lut(lut_base, (wa_s >> sh) & 0xFFu);
                const uint32_t a2 = lut(lut_base, (wa_s >> (sh + 8)) & 0xFFu);
                const uint32_t a1 = lut(lut_base, (wb_s >> sh) & 0xFFu);
                const uint32_t a3 = lut(lut_base, (wb_s >> (sh + 8)) & 0xFFu);
                uint32_t b0, b1;
                asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];"
                             : "=r"(b0), "=r"(b1)
                             : "r"(xk + g * x_pitch_bytes + s * 8));
                mma16816(blk0, a0, a1, a2, a3, b0, b1);
                if (kTwoTiles) {
                    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];"
                                 : "=r"(b0), "=r"(b1)
                                 : "r"(xk + (g + 8) * x_pitch_bytes + s * 8));
                    mma16816(blk1, a0, a1, a2, a3, b0, b1);
                }
            }
            acc0[0] = fmaf(cta, blk0[0], acc0[0]);
            acc0[1] = fmaf(cta, blk0[1], acc0[1]);
            acc0[2] = fmaf(ctb, blk0[2], acc0[2]);
            acc0[3] = fmaf(ctb, blk0[3], acc0[3]);
            if (kTwoTiles) {
                acc1[0] = fmaf(cta, blk1[0], acc1[0]);
                acc1[1] = fmaf(cta, blk1[1], acc1[1]);
                acc1[2] = fmaf(ctb, blk1[2], acc1[2]);
                acc1[3] = fmaf(ctb, blk1[3], acc1[3]);
            }
        }
        // C fragment: (row g, tokens 2c, 2c+1) and (row g+8, same tokens)
        const int m0 = 2 * c;
        auto put = [&](int m, int64_t n, float v) {
            if (m < a.M && n < a.N) part[int64_t(m) * a.N + n] = v;
        };
        put(m0, na, acc0[0]);
        put(m0 + 1, na, acc0[1]);
        put(m0, nb, acc0[2]);
        put(m0 + 1, nb, acc0[3]);
        if (kTwoTiles) {
            put(m0 + 8, na, acc1[0]);
            put(m0 + 9, na, acc1[1]);
            put(m0 + 8, nb, acc1[2]);
            put(m0 + 9, nb, acc1[3]);
        }
    }
}

// One thread per output column n: sums the slice partials of all M tokens and
// adds the LoRA term sum_j G[m][j] B[n][j] (G = gamma*T in bf16, staged in
// shared memory).
__global__ void __launch_bounds__(256)
gemv_finalize_kernel(GemvFinalizeArgs a) {
    __shared__ float sg[16 * QLORA_MAX_RANK];
    for (int e = threadIdx.x; e < a.M * a.r; e += blockDim.x) {
        const int m = e / a.r, j = e % a.r;
        sg[e] = __uint_as_float(static_cast<uint32_t>(a.G[m * a.ldg + j]) << 16);
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
                for (int q = 0; q < 8; ++q) acc[m] = fmaf(sg[m * a.r + j0 + q], b[q], acc[m]);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        if (m < a.M) {
            float s = acc[m];
            for (int k = 0; k < a.splits; ++k) s += a.part[(int64_t(k) * a.M + m) * a.N + n];
            __nv_bfloat16 y = __float2bfloat16_rn(s);
            a.Y[m * a.N + n] = *reinterpret_cast<uint16_t*>(&y);
        }
    }
}

}  // namespace

int gemv_rows_per_cta() { return kRows; }

cudaError_t launch_gemv(const GemvArgs& a, int* smem_bytes_out, cudaStream_t stream) {
    const int x_pitch = static_cast<int>(a.k_per_split * 2 + 8);
    const int smem = kLutBytes + 16 * x_pitch;
    if (smem_bytes_out) *smem_bytes_out = smem;
    dim3 grid(static_cast<unsigned>((a.N + kRows - 1) / kRows), static_cast<unsigned>(a.splits));
    cudaError_t e;
    if (a.M > 8) {
        e = cudaFuncSetAttribute(gemv_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        gemv_kernel<true><<<grid, kThreads, smem, stream>>>(a, x_pitch);
    } else {
        e = cudaFuncSetAttribute(gemv_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        gemv_kernel<false><<<grid, kThreads, smem, stream>>>(a, x_pitch);
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
