// AdamW step over an adapter matrix with 8-bit blockwise optimiser state.
//
// "QLoRA, explained", "The algorithm, step by step" (AdamW over A and B only,
// 32-bit or 8-bit state) and "Hyperparameters that matter" (the 8-bit
// variant quantises Adam's moments blockwise).  The pages give no 8-bit
// format; the reading reuses the blockwise absmax scheme: blocks of 64 state
// entries with an fp32 absmax each, the first moment as the symmetric linear
// code rint(fp32(m / c) * 127), the second through its square root,
// rint(fp32(sqrt(v) / c) * 255) (the quotient rounded to fp32 first, then the
// product; a linear code of v flushes small v to zero while m is not, and the
// step then diverges).  Decoding is q * fp32(c / 127) (or / 255, squared).
//
// The update is AdamW in fp32 in a fixed operation order, every product,
// quotient and sum rounded on its own (no contraction into fused
// multiply-adds): p *= 1 - lr wd; m = b1 m + (1 - b1) g; v = b2 v + ((1 - b2)
// g) g; p -= (lr (m / (1 - b1^t))) / (sqrt(v / (1 - b2^t)) + eps).
//
// Elementwise work: per entry 4 B of p and 4 B of g read, 4 B of p written,
// 1 + 1 B of codes read and written (+ the bf16 copy of p if asked).  The
// five correctly rounded divisions and two square roots per entry cost more
// issue slots than the memory traffic needs time.  A half-warp covers one
// block of 64 (four entries per lane, 16-byte loads), reducing each block's
// new absmax values with four shuffles.
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kThreads = 256;
constexpr int kBlock = 64;

__device__ __forceinline__ float half_max(float a) {
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    return a;
}

__global__ void __launch_bounds__(kThreads)
adamw8_kernel(Adam8Args a) {
    const int lane = threadIdx.x & 31;
    const int sub = lane & 15;
    const int64_t nblocks = (a.n + kBlock - 1) / kBlock;
    const int64_t half_warps = int64_t(gridDim.x) * (kThreads / 16);
    const int64_t hw0 = (int64_t(blockIdx.x) * kThreads + threadIdx.x) / 16;
    // every lane of a warp runs the same number of iterations (shuffles)
    const int64_t iters = (nblocks + half_warps - 1) / half_warps;
    for (int64_t it = 0; it < iters; ++it) {
        const int64_t b = hw0 + it * half_warps;
        const bool blk_ok = b < nblocks;
        const int64_t e0 = b * kBlock + sub * 4;
        float p[4] = {0.f, 0.f, 0.f, 0.f}, g[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t mq = 0u, vq = 0u;
        float mc = 0.f, vc = 0.f;
        bool ok[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) ok[j] = blk_ok && e0 + j < a.n;
        if (blk_ok) {
            mc = a.m_absmax[b];
            vc = a.v_absmax[b];
            if (ok[3]) {
                const float4 pv = *reinterpret_cast<const float4*>(a.p + e0);
                const float4 gv = *reinterpret_cast<const float4*>(a.g + e0);
                p[0] = pv.x; p[1] = pv.y; p[2] = pv.z; p[3] = pv.w;
                g[0] = gv.x; g[1] = gv.y; g[2] = gv.z; g[3] = gv.w;
                mq = *reinterpret_cast<const uint32_t*>(a.m_codes + e0);
                vq = *reinterpret_cast<const uint32_t*>(a.v_codes + e0);
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (ok[j]) {
                        p[j] = a.p[e0 + j];
                        g[j] = a.g[e0 + j];
                        mq |= uint32_t(static_cast<uint8_t>(a.m_codes[e0 + j])) << (8 * j);
                        vq |= uint32_t(a.v_codes[e0 + j]) << (8 * j);
                    }
                }
            }
        }
        const float mstep = __fdiv_rn(mc, 127.0f), vstep = __fdiv_rn(vc, 255.0f);
        float m[4], u[4];
        float mmax = 0.f, umax = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float qm = static_cast<float>(static_cast<int8_t>((mq >> (8 * j)) & 0xffu));
            const float qv = static_cast<float>((vq >> (8 * j)) & 0xffu);
            float mj = __fmul_rn(qm, mstep);
            const float uj = __fmul_rn(qv, vstep);
            float vj = __fmul_rn(uj, uj);
            float pj = __fmul_rn(p[j], a.decay);                          // p (1 - lr wd)
            mj = __fadd_rn(__fmul_rn(a.beta1, mj), __fmul_rn(a.one_m_beta1, g[j]));
            vj = __fadd_rn(__fmul_rn(a.beta2, vj), __fmul_rn(__fmul_rn(a.one_m_beta2, g[j]), g[j]));
            const float mhat = __fdiv_rn(mj, a.bc1);
            const float vhat = __fdiv_rn(vj, a.bc2);
            pj = __fsub_rn(pj, __fdiv_rn(__fmul_rn(a.lr, mhat), __fadd_rn(__fsqrt_rn(vhat), a.eps)));
            p[j] = pj;
            m[j] = mj;
            u[j] = __fsqrt_rn(vj);
            if (ok[j]) {
                mmax = fmaxf(mmax, fabsf(mj));
                umax = fmaxf(umax, u[j]);
            }
        }
        mmax = half_max(mmax);
        umax = half_max(umax);
        if (!blk_ok) continue;
        uint32_t mo = 0u, vo = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int qm = 0, qv = 0;
            if (mmax > 0.f) qm = static_cast<int>(rintf(__fmul_rn(__fdiv_rn(m[j], mmax), 127.0f)));
            if (umax > 0.f) qv = static_cast<int>(rintf(__fmul_rn(__fdiv_rn(u[j], umax), 255.0f)));
            mo |= uint32_t(static_cast<uint8_t>(static_cast<int8_t>(qm))) << (8 * j);
            vo |= uint32_t(qv & 0xff) << (8 * j);
        }
        if (ok[3]) {
            *reinterpret_cast<float4*>(a.p + e0) = make_float4(p[0], p[1], p[2], p[3]);
            *reinterpret_cast<uint32_t*>(a.m_codes + e0) = mo;
            *reinterpret_cast<uint32_t*>(a.v_codes + e0) = vo;
            if (a.p_bf16)
                *reinterpret_cast<uint2*>(a.p_bf16 + e0) =
                    make_uint2(pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]));
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (ok[j]) {
                    a.p[e0 + j] = p[j];
                    a.m_codes[e0 + j] = static_cast<int8_t>((mo >> (8 * j)) & 0xffu);
                    a.v_codes[e0 + j] = static_cast<uint8_t>((vo >> (8 * j)) & 0xffu);
                    if (a.p_bf16)
                        a.p_bf16[e0 + j] = static_cast<uint16_t>(pack_bf16x2(p[j], 0.f) & 0xffffu);
                }
            }
        }
        if (sub == 0) {
            a.m_absmax[b] = mmax;
            a.v_absmax[b] = umax;
        }
    }
}

}  // namespace

cudaError_t launch_adamw8(const Adam8Args& a, int num_sms, cudaStream_t stream) {
    const int64_t nblocks = (a.n + kBlock - 1) / kBlock;
    int64_t grid = (nblocks + (kThreads / 16) - 1) / (kThreads / 16);
    const int64_t cap = int64_t(num_sms) * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    adamw8_kernel<<<dim3(static_cast<unsigned>(grid)), kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace qnf4
