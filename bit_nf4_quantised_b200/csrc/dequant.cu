// K6: dDQ of a whole stored tensor to bf16.
//
// "QLoRA, explained", "The forward pass and gradients": first the FP8 block
// scales are dequantised with their fp32 group constants, c~ = fp32(e4m3(code)
// * c2); then every index with its block's scale, w~ = bf16_rne(fp32(q[idx] *
// c~)).  This order of reconstruction is the bit-exact contract every fused
// kernel of the library also keeps.
//
// HBM-bound (0.516 B read, 2 B written per weight).  Each thread expands one
// 32-bit word of packed nibbles (8 weights) into one 16-byte store; the 16
// codes sit in shared memory (16 words on 16 banks: conflict-free).
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
dequantize_kernel(const uint32_t* __restrict__ packed, const uint8_t* __restrict__ scale_codes,
                  const float* __restrict__ meta, int64_t numel, uint16_t* __restrict__ out,
                  Nf4Table tab) {
    __shared__ float scode[16];
    if (threadIdx.x < 16) scode[threadIdx.x] = tab.code[threadIdx.x];
    __syncthreads();
    const int64_t nwords = (numel + 7) / 8;
    for (int64_t u = blockIdx.x * int64_t(kThreads) + threadIdx.x; u < nwords;
         u += int64_t(gridDim.x) * kThreads) {
        const uint32_t v = __ldcs(packed + u);
        const int64_t b = u >> 3;                       // 8 words per block of 64
        const float ct = __fmul_rn(e4m3_to_float(scale_codes[b]), meta[b >> 8]);
        uint32_t r[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float lo = __fmul_rn(scode[(v >> (8 * j)) & 15u], ct);
            const float hi = __fmul_rn(scode[(v >> (8 * j + 4)) & 15u], ct);
            r[j] = pack_bf16x2(lo, hi);
        }
        const int64_t e = u * 8;
        if (e + 8 <= numel) {
            __stcs(reinterpret_cast<uint4*>(out + e), make_uint4(r[0], r[1], r[2], r[3]));
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (e + j < numel) out[e + j] = static_cast<uint16_t>(r[j >> 1] >> (16 * (j & 1)));
        }
    }
}

}  // namespace

cudaError_t launch_dequantize(const uint8_t* packed, const uint8_t* scale_codes, const float* meta,
                              int64_t numel, uint16_t* out, const Nf4Table& tab, int num_sms,
                              cudaStream_t stream) {
    const int64_t nwords = (numel + 7) / 8;
    int64_t grid = (nwords + kThreads - 1) / kThreads;
    const int64_t cap = int64_t(num_sms) * 8;              // 8 resident CTAs per SM
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    dequantize_kernel<<<dim3(static_cast<unsigned>(grid)), kThreads, 0, stream>>>(
        reinterpret_cast<const uint32_t*>(packed), scale_codes, meta, numel, out, tab);
    return cudaGetLastError();
}

}  // namespace qnf4
