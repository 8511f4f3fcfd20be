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
// One CTA of 512 threads owns one group of 256 blocks (16384 weights, 64 KiB
// of fp32); eight lanes cover a block, each lane the block's 32 consecutive
// bytes 32 s .. 32 s + 31 (s = lane mod 8), so a warp takes four blocks per
// step and a thread issues its four steps' loads (eight 16-byte loads) before
// using any: the whole group is in flight at once, and at 64 registers two
// CTAs (32 warps) share an SM.  (Layouts with four lanes per block, and
// persistent CTAs streaming groups through shared memory by bulk copies, were
// measured slower.)  Per block:
//   - absmax by three shuffles of NaN-propagating maxima (one test of the
//     result catches NaN and infinities);
//   - x = fp32(w / c) without a division per element: with r = RN(1/c)
//     computed once, q = RN(w r) is within one unit in the last place of
//     w / c, the fused multiply-add w - q c is then exact, and
//     RN(q + (w - q c) r) is the correctly rounded quotient (Markstein's
//     theorem); blocks whose absmax lies outside [2^-90, 2^90], where the
//     theorem's range conditions could fail, take the correctly rounded
//     division instead (clamped to [-1, 1], which also sends the NaN of an
//     infinite weight into range);
//   - the nearest code, the number of midpoints strictly below x (a value on
//     a midpoint takes the lower code): y = x + 3 lies in [2, 4], and the top
//     five mantissa bits of y cut [-1, 1] into buckets 1/16 wide, narrower
//     than the closest two midpoints (0.08 apart), so no bucket holds two.
//     A bucket's entry gives base = the number of midpoints below it (taken
//     2^-22 below, past the rounding of x + 3) and thr = midpoint number
//     base; every x of the bucket has base or base + 1 midpoints below it,
//     and idx = base + (x > thr) picks the right one.  The table (64 entries,
//     the top ones unused) is replicated per lane in shared memory, so the
//     lookups are free of bank conflicts;
//   - the lane's eight indices packed into one 32-bit store (a warp writes
//     128 contiguous bytes).
// The block scales stay in shared memory for the group-level FP8 pass.
//
// The same kernel also takes a bf16 weight (a merged export being
// re-quantised): each lane then loads its 8 weights as 16 bytes, widened
// exactly.
#include <cfloat>

#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kThreads = 512;
constexpr int kLanesPerBlock = 8;
constexpr int kPerLane = QLORA_BLOCK / kLanesPerBlock;                             // 8
constexpr int kBlocksPerWarpStep = 32 / kLanesPerBlock;                            // 4
constexpr int kSteps = QLORA_GROUP / (kThreads / 32 * kBlocksPerWarpStep);         // 4
constexpr int kGroupElems = QLORA_BLOCK * QLORA_GROUP;                             // 16384
constexpr int kLutBytes = kNf4LutEntries * 32 * 8;                                  // 16 KiB
// index 7 (the exact zero among the NF4 codes) in all eight nibbles: a zero block's word
constexpr uint32_t kNf4ZeroWord = 0x77777777u;

// eight consecutive weights of one lane
struct W8 {
    float v[kPerLane];
};
__device__ __forceinline__ W8 load8(const float* W, int64_t e0) {
    const float4 a = __ldcs(reinterpret_cast<const float4*>(W + e0));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(W + e0 + 4));
    return W8{{a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w}};
}
__device__ __forceinline__ W8 load8(const uint16_t* W, int64_t e0) {
    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(W + e0));   // bf16 = top half of fp32
    return W8{{__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
               __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u),
               __uint_as_float(u.z << 16), __uint_as_float(u.z & 0xffff0000u),
               __uint_as_float(u.w << 16), __uint_as_float(u.w & 0xffff0000u)}};
}
__device__ __forceinline__ float load1(const float* W, int64_t e) { return W[e]; }
__device__ __forceinline__ float load1(const uint16_t* W, int64_t e) {
    return __uint_as_float(uint32_t(W[e]) << 16);
}
template <typename Tin>
__device__ __forceinline__ W8 load8_tail(const Tin* W, int64_t e0, int64_t numel) {
    W8 r;
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) r.v[j] = e0 + j < numel ? load1(W, e0 + j) : 0.f;
    return r;
}

// max that returns NaN when either operand is NaN
__device__ __forceinline__ float max_nan(float a, float b) {
    float d;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}

// fp32(w / c), correctly rounded, from r = RN(1/c) (c in [2^-90, 2^90], |w| <= c)
__device__ __forceinline__ float quotient(float w, float c, float r) {
    const float q = __fmul_rn(w, r);
    const float rem = __fmaf_rn(-q, c, w);
    return __fmaf_rn(rem, r, q);
}

// Number of midpoints strictly below x in [-1, 1], from the bucket table.
// lane_lut is this lane's column of the table, minus the offset of key
// 0x1000 (the bucket of y = 2).
__device__ __forceinline__ uint32_t code_index(float x, uint32_t lane_lut) {
    const uint32_t key = __float_as_uint(__fadd_rn(x, 3.0f)) >> 18;   // 0x1000 + bucket
    uint32_t thr, base;
    asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(thr), "=r"(base) : "r"(lane_lut + (key << 8)));
    return base + (x > __uint_as_float(thr) ? 1u : 0u);
}

// One group of 256 blocks by one CTA (the body of both kernels below).
template <bool kFull, typename Tin>
__device__ __forceinline__ void quantize_group(const Tin* __restrict__ W, int64_t numel, int64_t nblocks,
                                               uint8_t* __restrict__ packed, void* __restrict__ scales,
                                               float* __restrict__ meta, int* __restrict__ nonfinite_flag,
                                               const Nf4IndexLut& lut, uint32_t zero_word, int scale_fmt,
                                               int64_t group) {
    extern __shared__ __align__(16) uint8_t smem[];                // the per-lane table
    __shared__ float sabs[QLORA_GROUP];
    __shared__ float sred[QLORA_GROUP / 32];

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int sub = lane & (kLanesPerBlock - 1), bq = lane / kLanesPerBlock;
    const int64_t gbase = group * kGroupElems;

    // every load of the group first
    W8 v[kSteps];
#pragma unroll
    for (int step = 0; step < kSteps; ++step) {
        const int blk = (step * (kThreads / 32) + warp) * kBlocksPerWarpStep + bq;
        const int64_t e0 = gbase + int64_t(blk) * QLORA_BLOCK + sub * kPerLane;
        v[step] = kFull ? load8(W, e0) : load8_tail(W, e0, numel);
    }
    // table entry e for lane l at byte 256 e + 8 l, written as 16-byte
    // chunks c = 16 e + l / 2 (two lanes each) by thread c mod 512: a warp's
    // stores cover 512 contiguous bytes, free of bank conflicts
    static_assert(kLutBytes / 16 == 2 * kThreads, "two chunks per thread");
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int c = tid + k * kThreads, e = c >> 4;
        const uint32_t t = lut.thr[e], b = lut.base[e];
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %1, %2};" ::"r"(smem_u32(smem) + c * 16), "r"(t), "r"(b)
                     : "memory");
    }
    __syncthreads();
    const uint32_t lane_lut = smem_u32(smem) + lane * 8 - (0x1000u << 8);
    uint32_t* packed_w = reinterpret_cast<uint32_t*>(packed + group * (kGroupElems / 2));

    bool bad = false;
#pragma unroll
    for (int step = 0; step < kSteps; ++step) {
        const int blk = (step * (kThreads / 32) + warp) * kBlocksPerWarpStep + bq;
        const float* f = v[step].v;
        float a = max_nan(max_nan(max_nan(fabsf(f[0]), fabsf(f[1])), max_nan(fabsf(f[2]), fabsf(f[3]))),
                          max_nan(max_nan(fabsf(f[4]), fabsf(f[5])), max_nan(fabsf(f[6]), fabsf(f[7]))));
#pragma unroll
        for (int o = 4; o >= 1; o >>= 1) a = max_nan(a, __shfl_xor_sync(0xffffffffu, a, o));
        bad |= !(a <= FLT_MAX);                                // NaN or infinity in the block
        // a = c_b for this block
        uint32_t word = zero_word;                              // zero block -> the code of 0
        if (a > 0.f) {
            word = 0;
            if (a >= 0x1p-90f && a <= 0x1p90f) {
                const float r = __frcp_rn(a);
#pragma unroll
                for (int j = 0; j < kPerLane; ++j) word += code_index(quotient(f[j], a, r), lane_lut) << (4 * j);
            } else {
#pragma unroll
                for (int j = 0; j < kPerLane; ++j)
                    word += code_index(fminf(fmaxf(__fdiv_rn(f[j], a), -1.0f), 1.0f), lane_lut) << (4 * j);
            }
        }
        if (kFull || group * QLORA_GROUP + blk < nblocks) packed_w[blk * (QLORA_BLOCK / 8) + sub] = word;
        if (sub == 0) sabs[blk] = a;
    }
    if (bad && sub == 0 && nonfinite_flag != nullptr) atomicOr(nonfinite_flag, 1);
    __syncthreads();

    // Double quantisation of this group's 256 scales (the first 8 warps), or
    // the fp32 scales themselves.
    if (tid < QLORA_GROUP) {
        const float c = sabs[tid];
        const int64_t gblk = group * QLORA_GROUP + tid;
        if (scale_fmt == QLORA_SCALES_FP32) {
            if (kFull || gblk < nblocks) reinterpret_cast<float*>(scales)[gblk] = c;
            return;
        }
        float m = c;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) sred[warp] = m;
        asm volatile("bar.sync 1, %0;" ::"n"(QLORA_GROUP) : "memory");
        float gmax = sred[0];
#pragma unroll
        for (int w = 1; w < QLORA_GROUP / 32; ++w) gmax = fmaxf(gmax, sred[w]);
        const float c2 = __fdiv_rn(gmax, scale8_top(scale_fmt));
        const uint8_t code = c2 > 0.f ? scale8_encode(__fdiv_rn(c, c2), scale_fmt) : uint8_t(0);
        if (kFull || gblk < nblocks) reinterpret_cast<uint8_t*>(scales)[gblk] = code;
        if (tid == 0) meta[group] = c2;
    }
}

template <bool kFull, typename Tin>
__global__ void __launch_bounds__(kThreads, 2)
quantize_kernel(const Tin* __restrict__ W, int64_t numel, int64_t nblocks,
                uint8_t* __restrict__ packed, void* __restrict__ scales,
                float* __restrict__ meta, int* __restrict__ nonfinite_flag, Nf4IndexLut lut,
                uint32_t zero_word, int scale_fmt) {
    quantize_group<kFull, Tin>(W, numel, nblocks, packed, scales, meta, nonfinite_flag, lut, zero_word,
                               scale_fmt, blockIdx.x);
}

// Several weights' whole groups in one launch: CTA x takes group
// x - first[j] of job j, first[j] <= x < first[j + 1].
struct QuantBatch {
    QuantizeJob job[kMaxQuantizeJobs];
    int64_t first[kMaxQuantizeJobs + 1];
    int n;
};

template <typename Tin>
__global__ void __launch_bounds__(kThreads, 2)
quantize_many_kernel(const __grid_constant__ QuantBatch bt, int* __restrict__ nonfinite_flag,
                     Nf4IndexLut lut) {
    // this CTA's job: the last whose first group is at or below blockIdx.x
    // (first[] rises strictly: jobs without whole groups are left out), one
    // lane per job, counted by a ballot
    const int lane = threadIdx.x & 31;
    const bool le = lane < bt.n && bt.first[lane] <= int64_t(blockIdx.x);
    const int j = __popc(__ballot_sync(0xffffffffu, le)) - 1;
    const QuantizeJob& q = bt.job[j];
    const int64_t nblocks = (q.numel + QLORA_BLOCK - 1) / QLORA_BLOCK;
    quantize_group<true, Tin>(static_cast<const Tin*>(q.W), q.numel, nblocks, q.packed, q.scale_codes,
                              q.meta, nonfinite_flag, lut, kNf4ZeroWord, QLORA_SCALES_E4M3,
                              int64_t(blockIdx.x) - bt.first[j]);
}

template <bool kFull, typename Tin>
cudaError_t launch_one(unsigned grid, const Tin* W, int64_t numel, int64_t nblocks, uint8_t* packed,
                       void* scales, float* meta, int* nonfinite_flag, const Nf4IndexLut& lut,
                       uint32_t zero_word, int scale_fmt, cudaStream_t stream) {
    quantize_kernel<kFull, Tin><<<grid, kThreads, kLutBytes, stream>>>(
        W, numel, nblocks, packed, scales, meta, nonfinite_flag, lut, zero_word, scale_fmt);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t quantize_any(const Tin* W, int64_t numel, uint8_t* packed, void* scales, float* meta,
                         int* nonfinite_flag, const Nf4IndexLut& lut, uint32_t zero_word,
                         int scale_fmt, cudaStream_t stream) {
    const int64_t nblocks = (numel + QLORA_BLOCK - 1) / QLORA_BLOCK;
    const int64_t ngroups = (nblocks + QLORA_GROUP - 1) / QLORA_GROUP;
    const int64_t full = numel / kGroupElems;                  // groups with no tail
    if (full > 0) {
        const cudaError_t e = launch_one<true>(static_cast<unsigned>(full), W, numel, nblocks, packed,
                                               scales, meta, nonfinite_flag, lut, zero_word,
                                               scale_fmt, stream);
        if (e != cudaSuccess) return e;
    }
    if (ngroups > full) {
        // the single trailing group, offset so blockIdx.x is its group index
        const int64_t off = full * kGroupElems;
        const int64_t blk_off = full * QLORA_GROUP;
        void* sc = scale_fmt == QLORA_SCALES_FP32
                       ? static_cast<void*>(static_cast<float*>(scales) + blk_off)
                       : static_cast<void*>(static_cast<uint8_t*>(scales) + blk_off);
        return launch_one<false>(1u, W + off, numel - off, nblocks - blk_off,
                                 packed + full * (kGroupElems / 2), sc,
                                 meta == nullptr ? nullptr : meta + full, nonfinite_flag, lut,
                                 zero_word, scale_fmt, stream);
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_quantize(const float* W, int64_t numel, uint8_t* packed, uint8_t* scale_codes,
                            float* meta, int* nonfinite_flag, const Nf4IndexLut& lut,
                            cudaStream_t stream) {
    return quantize_any(W, numel, packed, scale_codes, meta, nonfinite_flag, lut, kNf4ZeroWord,
                        QLORA_SCALES_E4M3, stream);
}

cudaError_t launch_quantize_b64(const float* W, int64_t numel, uint8_t* packed, void* scales,
                                float* meta, int* nonfinite_flag, const Nf4IndexLut& lut,
                                uint32_t zero_index, int scale_fmt, cudaStream_t stream) {
    return quantize_any(W, numel, packed, scales, meta, nonfinite_flag, lut, zero_index * 0x11111111u,
                        scale_fmt, stream);
}

template <typename Tin>
cudaError_t quantize_many_any(const QuantizeJob* jobs, int n, int* nonfinite_flag,
                              const Nf4IndexLut& lut, cudaStream_t stream) {
    for (int i0 = 0; i0 < n; i0 += kMaxQuantizeJobs) {
        QuantBatch bt{};
        int64_t total = 0;
        for (int i = i0; i < n && i < i0 + kMaxQuantizeJobs; ++i) {
            const int64_t full = jobs[i].numel / kGroupElems;
            if (full == 0) continue;
            bt.job[bt.n] = jobs[i];
            bt.first[bt.n] = total;
            total += full;
            ++bt.n;
        }
        bt.first[bt.n] = total;
        if (total > 0) {
            if (total > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
            quantize_many_kernel<Tin><<<static_cast<unsigned>(total), kThreads, kLutBytes, stream>>>(
                bt, nonfinite_flag, lut);
            const cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        // each weight's trailing partial group, if it has one
        for (int i = i0; i < n && i < i0 + kMaxQuantizeJobs; ++i) {
            const QuantizeJob& q = jobs[i];
            const int64_t full = q.numel / kGroupElems;
            const int64_t nblocks = (q.numel + QLORA_BLOCK - 1) / QLORA_BLOCK;
            if ((nblocks + QLORA_GROUP - 1) / QLORA_GROUP == full) continue;
            const int64_t off = full * kGroupElems;
            const cudaError_t e = launch_one<false>(
                1u, static_cast<const Tin*>(q.W) + off, q.numel - off, nblocks - full * QLORA_GROUP,
                q.packed + full * (kGroupElems / 2), q.scale_codes + full * QLORA_GROUP, q.meta + full,
                nonfinite_flag, lut, kNf4ZeroWord, QLORA_SCALES_E4M3, stream);
            if (e != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

cudaError_t launch_quantize_many(const QuantizeJob* jobs, int n, bool bf16, int* nonfinite_flag,
                                 const Nf4IndexLut& lut, cudaStream_t stream) {
    return bf16 ? quantize_many_any<uint16_t>(jobs, n, nonfinite_flag, lut, stream)
                : quantize_many_any<float>(jobs, n, nonfinite_flag, lut, stream);
}

cudaError_t launch_quantize_bf16(const uint16_t* W, int64_t numel, uint8_t* packed,
                                 uint8_t* scale_codes, float* meta, int* nonfinite_flag,
                                 const Nf4IndexLut& lut, cudaStream_t stream) {
    return quantize_any(W, numel, packed, scale_codes, meta, nonfinite_flag, lut, kNf4ZeroWord,
                        QLORA_SCALES_E4M3, stream);
}

}  // namespace qnf4
