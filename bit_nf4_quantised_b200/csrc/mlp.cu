// Layer chaining with gradient checkpointing: the SwiGLU MLP of adapted NF4
// linears, y = down(silu(gate(x)) * up(x)).
//
// "QLoRA, explained", "The algorithm, step by step" runs the training step
// with gradient checkpointing enabled, and "Compute and memory cost" notes
// that checkpointing is effectively mandatory and that the recomputed forward
// dequantises every block a third time per step.  The pages print no block
// structure; the reading is the MLP of the Llama-shaped workloads, every
// linear an adapted NF4 layer (gate and up F x D, down D x F).  With
// checkpointing the forward keeps only x; the backward recomputes gate(x),
// up(x) and h = silu(gate(x)) * up(x) through the forward kernels, then runs
// the three linear backwards with the SwiGLU backward between them:
//   dH = dY W~_down^T ...            (down's backward, dA_down, dB_down)
//   dG = dH * u * silu'(g),  dU = dH * silu(g)
//   dX = dG W~_gate + dU W~_up + the adapters' terms, dA, dB of gate and up.
//
// The elementwise kernels here are HBM-bound (8 bf16 per thread, 16-byte
// loads and stores); silu'(g) = s (1 + g (1 - s)) with s the logistic
// sigmoid, evaluated in fp32 from the bf16 inputs.
#include <cmath>

#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ float sigmoid(float z) { return 1.0f / (1.0f + expf(-z)); }

// H = bf16(silu(G) * U), n elements (n % 8 == 0)
__global__ void __launch_bounds__(kThreads)
swiglu_forward_kernel(const uint16_t* __restrict__ G, const uint16_t* __restrict__ U,
                      uint16_t* __restrict__ H, int64_t n8) {
    for (int64_t i = blockIdx.x * int64_t(kThreads) + threadIdx.x; i < n8;
         i += int64_t(gridDim.x) * kThreads) {
        const uint4 g = __ldcs(reinterpret_cast<const uint4*>(G) + i);
        const uint4 u = __ldcs(reinterpret_cast<const uint4*>(U) + i);
        const uint32_t gw[4] = {g.x, g.y, g.z, g.w}, uw[4] = {u.x, u.y, u.z, u.w};
        uint32_t h[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float g0 = bf16_lo(gw[k]), g1 = bf16_hi(gw[k]);
            h[k] = pack_bf16x2(g0 * sigmoid(g0) * bf16_lo(uw[k]), g1 * sigmoid(g1) * bf16_hi(uw[k]));
        }
        __stcs(reinterpret_cast<uint4*>(H) + i, make_uint4(h[0], h[1], h[2], h[3]));
    }
}

// dG = bf16(dH * U * silu'(G)), dU = bf16(dH * silu(G)), written over G and U
__global__ void __launch_bounds__(kThreads)
swiglu_backward_kernel(uint16_t* __restrict__ G, uint16_t* __restrict__ U,
                       const uint16_t* __restrict__ dH, int64_t n8) {
    for (int64_t i = blockIdx.x * int64_t(kThreads) + threadIdx.x; i < n8;
         i += int64_t(gridDim.x) * kThreads) {
        const uint4 g = __ldcs(reinterpret_cast<const uint4*>(G) + i);
        const uint4 u = __ldcs(reinterpret_cast<const uint4*>(U) + i);
        const uint4 d = __ldcs(reinterpret_cast<const uint4*>(dH) + i);
        const uint32_t gw[4] = {g.x, g.y, g.z, g.w}, uw[4] = {u.x, u.y, u.z, u.w};
        const uint32_t dw[4] = {d.x, d.y, d.z, d.w};
        uint32_t dg[4], du[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float gg[2] = {bf16_lo(gw[k]), bf16_hi(gw[k])};
            float uu[2] = {bf16_lo(uw[k]), bf16_hi(uw[k])};
            float dd[2] = {bf16_lo(dw[k]), bf16_hi(dw[k])};
            float og[2], ou[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float s = sigmoid(gg[e]);
                const float silu = gg[e] * s;
                const float dsilu = s * (1.0f + gg[e] * (1.0f - s));
                og[e] = dd[e] * uu[e] * dsilu;
                ou[e] = dd[e] * silu;
            }
            dg[k] = pack_bf16x2(og[0], og[1]);
            du[k] = pack_bf16x2(ou[0], ou[1]);
        }
        __stcs(reinterpret_cast<uint4*>(G) + i, make_uint4(dg[0], dg[1], dg[2], dg[3]));
        __stcs(reinterpret_cast<uint4*>(U) + i, make_uint4(du[0], du[1], du[2], du[3]));
    }
}

// C = bf16(A + B) (fp32 sum of the two bf16 values), in place over C == A allowed
__global__ void __launch_bounds__(kThreads)
add_bf16_kernel(const uint16_t* A, const uint16_t* __restrict__ B, uint16_t* C, int64_t n8) {
    for (int64_t i = blockIdx.x * int64_t(kThreads) + threadIdx.x; i < n8;
         i += int64_t(gridDim.x) * kThreads) {
        const uint4 a = reinterpret_cast<const uint4*>(A)[i];
        const uint4 b = __ldcs(reinterpret_cast<const uint4*>(B) + i);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
        uint32_t c[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            c[k] = pack_bf16x2(bf16_lo(aw[k]) + bf16_lo(bw[k]), bf16_hi(aw[k]) + bf16_hi(bw[k]));
        reinterpret_cast<uint4*>(C)[i] = make_uint4(c[0], c[1], c[2], c[3]);
    }
}

// error word of the MLP call = OR of its linear calls' error words
__global__ void or_words_kernel(int* dst, const int* a, const int* b, const int* c, int accumulate) {
    if (threadIdx.x == 0) *dst = (accumulate ? *dst : 0) | *a | *b | *c;
}

unsigned grid_for(int64_t n8, int num_sms) {
    int64_t g = (n8 + kThreads - 1) / kThreads;
    const int64_t cap = int64_t(num_sms) * 8;
    if (g > cap) g = cap;
    return static_cast<unsigned>(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_swiglu_forward(const uint16_t* G, const uint16_t* U, uint16_t* H, int64_t n,
                                  int num_sms, cudaStream_t s) {
    swiglu_forward_kernel<<<grid_for(n / 8, num_sms), kThreads, 0, s>>>(G, U, H, n / 8);
    return cudaGetLastError();
}

cudaError_t launch_swiglu_backward(uint16_t* G, uint16_t* U, const uint16_t* dH, int64_t n,
                                   int num_sms, cudaStream_t s) {
    swiglu_backward_kernel<<<grid_for(n / 8, num_sms), kThreads, 0, s>>>(G, U, dH, n / 8);
    return cudaGetLastError();
}

cudaError_t launch_add_bf16(const uint16_t* A, const uint16_t* B, uint16_t* C, int64_t n,
                            int num_sms, cudaStream_t s) {
    add_bf16_kernel<<<grid_for(n / 8, num_sms), kThreads, 0, s>>>(A, B, C, n / 8);
    return cudaGetLastError();
}

cudaError_t launch_or_words(int* dst, const int* a, const int* b, const int* c, bool accumulate,
                            cudaStream_t s) {
    or_words_kernel<<<1, 32, 0, s>>>(dst, a, b, c, accumulate ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace qnf4
