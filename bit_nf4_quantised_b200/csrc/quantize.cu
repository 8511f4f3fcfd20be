// K1: blockwise absmax NF4 quantisation with double quantisation of the
// scales, one pass over the fp32 weight.
//
// "QLoRA, explained", "The algorithm, step by step": split the weight into
// blocks of 64 and take each block's absmax c1; store the index of the nearest
// NF4 code of w / c1; quantise c1 to FP8 in blocks of 256 with fp32 constants
// c2 ("Double quantisation").  Reading of the FP8 step: E4M3 (e4m3fn), c2 =
// max(c1 over the group) / 448, code = E4M3 round-to-nearest-even of c1 / c2,
// saturated to 448; an all-zero group stores c2 = 0 and codes 0.
//
// One CTA of 256 threads owns one group of 256 blocks (16384 weights, 64 KiB of
// fp32).  Each warp streams two blocks per step with fully coalesced 16-byte
// loads (lanes 0-15 on one block, 16-31 on the next), reduces the absmax with
// four shuffles, divides with a correctly rounded fp32 division (__fdiv_rn, as
// the method's normalisation is an fp32 quotient), finds the code by binary
// search over the midpoints in shared memory, and writes its four nibbles as
// one 16-bit store, so a warp writes 64 contiguous bytes.  The block scales
// stay in shared memory for the group-level FP8 pass at the end.
//
// The same kernel also takes a bf16 weight (a merged export being
// re-quantised): each lane then loads 8 bytes, widened exactly to fp32.
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kThreads = 256;
constexpr int kGroupElems = QLORA_BLOCK * QLORA_GROUP;   // 16384

__device__ __forceinline__ uint32_t nearest_code(float x, const float* smid) {
    // number of midpoints strictly below x (ties to the lower code)
    uint32_t i = 0;
    i += (x > smid[i + 7]) ? 8u : 0u;
    i += (x > smid[i + 3]) ? 4u : 0u;
    i += (x > smid[i + 1]) ? 2u : 0u;
    i += (x > smid[i + 0]) ? 1u : 0u;
    return i;
}

// Four consecutive weights as fp32: fp32 input directly, bf16 input widened
// exactly (a bf16 value is the top half of its fp32).
__device__ __forceinline__ float4 load4(const float* W, int64_t e0) {
    return __ldcs(reinterpret_cast<const float4*>(W + e0));
}
__device__ __forceinline__ float4 load4(const uint16_t* W, int64_t e0) {
    const uint2 u = __ldcs(reinterpret_cast<const uint2*>(W + e0));
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}
__device__ __forceinline__ float load1(const float* W, int64_t e) { return W[e]; }
__device__ __forceinline__ float load1(const uint16_t* W, int64_t e) {
    return __uint_as_float(uint32_t(W[e]) << 16);
}

template <bool kFull, typename Tin>
__global__ void __launch_bounds__(kThreads)
quantize_kernel(const Tin* __restrict__ W, int64_t numel, int64_t nblocks,
                uint8_t* __restrict__ packed, uint8_t* __restrict__ scale_codes,
                float* __restrict__ meta, int* __restrict__ nonfinite_flag, Nf4Table tab) {
    __shared__ float smid[16];
    __shared__ float sabs[QLORA_GROUP];
    __shared__ float sred[kThreads / 32];

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    if (tid < 15) smid[tid] = tab.mid[tid];
    __syncthreads();

    const int64_t group = blockIdx.x;
    const int64_t gbase = group * kGroupElems;
    const int half = lane >> 4, sub = lane & 15;
    bool bad = false;

    // 32 blocks per warp, two per step.
#pragma unroll 4
    for (int step = 0; step < 16; ++step) {
        const int blk = warp * 32 + step * 2 + half;          // block within group
        const int64_t e0 = gbase + int64_t(blk) * QLORA_BLOCK + sub * 4;
        float4 v;
        if (kFull) {
            v = load4(W, e0);
        } else {
            v.x = (e0 + 0 < numel) ? load1(W, e0 + 0) : 0.f;
            v.y = (e0 + 1 < numel) ? load1(W, e0 + 1) : 0.f;
            v.z = (e0 + 2 < numel) ? load1(W, e0 + 2) : 0.f;
            v.w = (e0 + 3 < numel) ? load1(W, e0 + 3) : 0.f;
        }
        bad |= !(isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w));
        float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        // a = c_b for this half-warp's block
        uint32_t q0 = 7, q1 = 7, q2 = 7, q3 = 7;               // zero block -> code 0
        if (a > 0.f) {
            q0 = nearest_code(__fdiv_rn(v.x, a), smid);
            q1 = nearest_code(__fdiv_rn(v.y, a), smid);
            q2 = nearest_code(__fdiv_rn(v.z, a), smid);
            q3 = nearest_code(__fdiv_rn(v.w, a), smid);
        }
        const int64_t gblk = group * QLORA_GROUP + blk;
        if (kFull || gblk < nblocks) {
            const uint16_t nib = static_cast<uint16_t>(q0 | (q1 << 4) | (q2 << 8) | (q3 << 12));
            reinterpret_cast<uint16_t*>(packed + gblk * (QLORA_BLOCK / 2))[sub] = nib;
        }
        if (sub == 0) sabs[blk] = a;
    }
    if (bad && nonfinite_flag != nullptr) atomicOr(nonfinite_flag, 1);
    __syncthreads();

    // Double quantisation of this group's 256 scales.
    const float c = sabs[tid];
    float m = c;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) sred[warp] = m;
    __syncthreads();
    float gmax = sred[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) gmax = fmaxf(gmax, sred[w]);
    const float c2 = __fdiv_rn(gmax, 448.0f);
    uint8_t code = 0;
    if (c2 > 0.f) {
        code = static_cast<uint8_t>(
            __nv_cvt_float_to_fp8(__fdiv_rn(c, c2), __NV_SATFINITE, __NV_E4M3));
    }
    const int64_t gblk = group * QLORA_GROUP + tid;
    if (kFull || gblk < nblocks) scale_codes[gblk] = code;
    if (tid == 0) meta[group] = c2;
}

template <typename Tin>
cudaError_t quantize_any(const Tin* W, int64_t numel, uint8_t* packed, uint8_t* scale_codes,
                         float* meta, int* nonfinite_flag, const Nf4Table& tab,
                         cudaStream_t stream) {
    const int64_t nblocks = (numel + QLORA_BLOCK - 1) / QLORA_BLOCK;
    const int64_t ngroups = (nblocks + QLORA_GROUP - 1) / QLORA_GROUP;
    const int64_t full = numel / kGroupElems;                  // groups with no tail
    if (full > 0) {
        quantize_kernel<true, Tin><<<dim3(static_cast<unsigned>(full)), kThreads, 0, stream>>>(
            W, numel, nblocks, packed, scale_codes, meta, nonfinite_flag, tab);
    }
    if (ngroups > full) {
        // the single trailing group, offset so blockIdx.x is its group index
        const int64_t off = full * kGroupElems;
        quantize_kernel<false, Tin><<<1, kThreads, 0, stream>>>(
            W + off, numel - off, nblocks - full * QLORA_GROUP, packed + full * (kGroupElems / 2),
            scale_codes + full * QLORA_GROUP, meta + full, nonfinite_flag, tab);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const float* W, int64_t numel, uint8_t* packed, uint8_t* scale_codes,
                            float* meta, int* nonfinite_flag, const Nf4Table& tab,
                            cudaStream_t stream) {
    return quantize_any(W, numel, packed, scale_codes, meta, nonfinite_flag, tab, stream);
}

cudaError_t launch_quantize_bf16(const uint16_t* W, int64_t numel, uint8_t* packed,
                                 uint8_t* scale_codes, float* meta, int* nonfinite_flag,
                                 const Nf4Table& tab, cudaStream_t stream) {
    return quantize_any(W, numel, packed, scale_codes, meta, nonfinite_flag, tab, stream);
}

}  // namespace qnf4
