// K1 / K6 format variants: blockwise absmax quantisation with any codebook of
// up to 16 codes, blocksizes 16 to 4096, and the block scales kept as fp32 or
// double-quantised to an 8-bit code (FP8 E4M3 or E5M2, or a linear code)
// with one fp32 constant per 256 blocks.
//
// "QLoRA, explained", "A toy run: how much does NF4 lose ...": the same scheme
// with the E2M1 FP4 and symmetric INT4 codebooks and blocksizes 16 and 4096
// next to NF4 at 64; "Double quantisation" is the optional second level.
// The steps are those of K1/K6: c_b = max |w| over the block, the index of
// the nearest code of fp32(w / c_b) as the number of midpoints strictly below
// it (a zero block and the padding of a final partial block take the index
// nearest to 0), two indices per byte with the even element in the low
// nibble; w~ = bf16_rne(fp32(q[idx] * c~_b)) with c~_b the fp32 absmax or
// fp32(decode(code) * c2).
//
// Quantise: one CTA per group of 256 blocks.  A block is covered by
// min(32, B/4) lanes that each load 16-byte pieces; the lanes reduce the
// absmax with shuffles and then re-read their pieces (from L1/L2) to write the
// indices, four per 16-bit store.  As in K1, x = fp32(w / c_b) comes from one
// correctly rounded reciprocal per block and two fused multiply-adds (exact,
// with a guarded fallback), and when the codebook's midpoints lie more than
// 1/16 apart (NF4, FP4, INT4) the index comes from K1's bucket table, one
// conflict-free shared-memory load per weight; other codebooks take a 4-step
// search over the midpoints.  The group's scales stay in shared memory for
// the FP8 pass, as in K1.  Dequantise: as K6, one packed word (8 weights)
// per thread and one 16-byte store; the block index is a shift.
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kThreads = 256;

// The correctly rounded a / b, given r = RN(1 / b): q = RN(a r) is within an
// ulp of a / b, the fused a - q b is then exact, and RN(q + (a - q b) r) is
// the correctly rounded quotient (Markstein's theorem), as long as no step
// overflows or underflows: a, b and q in [2^-100, 2^100] in magnitude.
// Elsewhere (zeros with their signs, NaN, infinities, extreme ranges) the
// plain correctly rounded division.  Both give the same bits.
__device__ __forceinline__ float div_rn_by(float a, float b, float r) {
    const float q = __fmul_rn(a, r);
    const float aa = fabsf(a), ab = fabsf(b), aq = fabsf(q);
    if (aa >= 0x1p-100f && aa <= 0x1p100f && ab >= 0x1p-100f && ab <= 0x1p100f && aq >= 0x1p-100f &&
        aq <= 0x1p100f)
        return __fmaf_rn(__fmaf_rn(-q, b, a), r, q);
    return __fdiv_rn(a, b);
}

// Number of midpoints strictly below x in [-1, 1], from K1's bucket table:
// bucket key = the top bits of x + 3; lane_lut is this lane's column of the
// table minus the offset of key 0x1000 (the bucket of x + 3 = 2).
__device__ __forceinline__ uint32_t bucket_code(float x, uint32_t lane_lut) {
    const uint32_t key = __float_as_uint(__fadd_rn(x, 3.0f)) >> 18;
    uint32_t thr, base;
    asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(thr), "=r"(base) : "r"(lane_lut + (key << 8)));
    return base + (x > __uint_as_float(thr) ? 1u : 0u);
}

__device__ __forceinline__ uint32_t nearest_code(float x, const float* smid) {
    // number of midpoints strictly below x; unused midpoints are +inf
    uint32_t i = 0;
    i += (x > smid[i + 7]) ? 8u : 0u;
    i += (x > smid[i + 3]) ? 4u : 0u;
    i += (x > smid[i + 1]) ? 2u : 0u;
    i += (x > smid[i + 0]) ? 1u : 0u;
    return i;
}

// kLP > 0 (full groups of blocks of 4 kLP <= 32 weights): kLP lanes cover a
// block, one 16-byte piece each, and a lane issues the loads of all its
// pieces of the group (4 kLP floats) before using any, keeping them in
// registers for the index pass; otherwise pieces are loaded block by block
// and re-read for the index pass.
template <bool kFull, int kLP>
__global__ void __launch_bounds__(kThreads)
quantize_fmt_kernel(const float* __restrict__ W, int64_t numel, int64_t nblocks, FmtArgs f,
                    uint8_t* __restrict__ packed, void* __restrict__ scales,
                    float* __restrict__ meta, int* __restrict__ nonfinite_flag, FmtTable tab) {
    __shared__ float smid[16];
    __shared__ float sabs[QLORA_GROUP];
    __shared__ float sred[kThreads / 32];
    __shared__ __align__(16) uint2 slut[kNf4LutEntries * 32];   // entry b of lane l at 256 b + 8 l

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {                    // constant indices: no local copy of the table
#pragma unroll
        for (int q = 0; q < 15; ++q) smid[q] = tab.mid[q];
        smid[15] = __int_as_float(0x7f800000);
    }
    if (tab.use_lut) {
        for (int i = tid; i < kNf4LutEntries * 32; i += kThreads)
            slut[i] = make_uint2(tab.lut.thr[i >> 5], tab.lut.base[i >> 5]);
    }
    __syncthreads();
    const uint32_t lane_lut = smem_u32(slut) + lane * 8 - (0x1000u << 8);

    const int64_t group = blockIdx.x;
    bool bad = false;
    if constexpr (kLP > 0) {
        constexpr int kBpw = 32 / kLP;                            // blocks per warp step
        constexpr int kIt = QLORA_GROUP / ((kThreads / 32) * kBpw);   // = kLP
        const int sub = lane % kLP;
        float4 v[kIt];
#pragma unroll
        for (int it = 0; it < kIt; ++it) {
            const int blk = warp * kBpw + lane / kLP + it * (kThreads / 32) * kBpw;
            const int64_t e0 = (group * QLORA_GROUP + blk) * (4 * kLP) + sub * 4;
            v[it] = __ldcs(reinterpret_cast<const float4*>(W + e0));
        }
#pragma unroll
        for (int it = 0; it < kIt; ++it) {
            const int blk = warp * kBpw + lane / kLP + it * (kThreads / 32) * kBpw;
            const int64_t e0 = (group * QLORA_GROUP + blk) * (4 * kLP) + sub * 4;
            const float4 w = v[it];
            bad |= !(isfinite(w.x) && isfinite(w.y) && isfinite(w.z) && isfinite(w.w));
            float a = fmaxf(fmaxf(fabsf(w.x), fabsf(w.y)), fmaxf(fabsf(w.z), fabsf(w.w)));
#pragma unroll
            for (int o = kLP / 2; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
            const float r = __frcp_rn(a);
            uint32_t q0 = tab.zero_index, q1 = tab.zero_index, q2 = tab.zero_index,
                     q3 = tab.zero_index;
            if (a > 0.f) {
                const float x0 = fminf(fmaxf(div_rn_by(w.x, a, r), -1.0f), 1.0f);
                const float x1 = fminf(fmaxf(div_rn_by(w.y, a, r), -1.0f), 1.0f);
                const float x2 = fminf(fmaxf(div_rn_by(w.z, a, r), -1.0f), 1.0f);
                const float x3 = fminf(fmaxf(div_rn_by(w.w, a, r), -1.0f), 1.0f);
                if (tab.use_lut) {
                    q0 = bucket_code(x0, lane_lut);
                    q1 = bucket_code(x1, lane_lut);
                    q2 = bucket_code(x2, lane_lut);
                    q3 = bucket_code(x3, lane_lut);
                } else {
                    q0 = nearest_code(x0, smid);
                    q1 = nearest_code(x1, smid);
                    q2 = nearest_code(x2, smid);
                    q3 = nearest_code(x3, smid);
                }
            }
            *reinterpret_cast<uint16_t*>(packed + e0 / 2) =
                static_cast<uint16_t>(q0 | (q1 << 4) | (q2 << 8) | (q3 << 12));
            if (sub == 0) sabs[blk] = a;
        }
    } else {
        const int lp = f.block >= 128 ? 32 : f.block / 4;        // lanes per block
        const int bpw = 32 / lp;                                  // blocks per warp step
        const int cpl = f.block / (4 * lp);                       // 16-byte pieces per lane
        const int sub = lane % lp;

        for (int blk = warp * bpw + lane / lp; blk < QLORA_GROUP; blk += (kThreads / 32) * bpw) {
            const int64_t gblk = group * QLORA_GROUP + blk;
            const int64_t ebase = gblk * f.block;
            float a = 0.f;
            for (int j = 0; j < cpl; ++j) {
                const int64_t e0 = ebase + int64_t(j * lp + sub) * 4;
                float4 v;
                if (kFull) {
                    v = *reinterpret_cast<const float4*>(W + e0);
                } else {
                    v.x = (e0 + 0 < numel) ? W[e0 + 0] : 0.f;
                    v.y = (e0 + 1 < numel) ? W[e0 + 1] : 0.f;
                    v.z = (e0 + 2 < numel) ? W[e0 + 2] : 0.f;
                    v.w = (e0 + 3 < numel) ? W[e0 + 3] : 0.f;
                }
                bad |= !(isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w));
                a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
            }
            for (int o = lp / 2; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
            const float r = __frcp_rn(a);
            const bool live = kFull || gblk < nblocks;
            for (int j = 0; j < cpl; ++j) {
                const int64_t e0 = ebase + int64_t(j * lp + sub) * 4;
                float4 v;
                if (kFull) {
                    v = *reinterpret_cast<const float4*>(W + e0);
                } else {
                    v.x = (e0 + 0 < numel) ? W[e0 + 0] : 0.f;
                    v.y = (e0 + 1 < numel) ? W[e0 + 1] : 0.f;
                    v.z = (e0 + 2 < numel) ? W[e0 + 2] : 0.f;
                    v.w = (e0 + 3 < numel) ? W[e0 + 3] : 0.f;
                }
                uint32_t q0 = tab.zero_index, q1 = tab.zero_index, q2 = tab.zero_index,
                         q3 = tab.zero_index;
                if (a > 0.f) {
                    // |w| <= c_b, so x lies in [-1, 1]; the clamp only sends the NaN
                    // of a non-finite weight (flagged above) into the table's range
                    const float x0 = fminf(fmaxf(div_rn_by(v.x, a, r), -1.0f), 1.0f);
                    const float x1 = fminf(fmaxf(div_rn_by(v.y, a, r), -1.0f), 1.0f);
                    const float x2 = fminf(fmaxf(div_rn_by(v.z, a, r), -1.0f), 1.0f);
                    const float x3 = fminf(fmaxf(div_rn_by(v.w, a, r), -1.0f), 1.0f);
                    if (tab.use_lut) {
                        q0 = bucket_code(x0, lane_lut);
                        q1 = bucket_code(x1, lane_lut);
                        q2 = bucket_code(x2, lane_lut);
                        q3 = bucket_code(x3, lane_lut);
                    } else {
                        q0 = nearest_code(x0, smid);
                        q1 = nearest_code(x1, smid);
                        q2 = nearest_code(x2, smid);
                        q3 = nearest_code(x3, smid);
                    }
                }
                if (live)
                    *reinterpret_cast<uint16_t*>(packed + e0 / 2) =
                        static_cast<uint16_t>(q0 | (q1 << 4) | (q2 << 8) | (q3 << 12));
            }
            if (sub == 0) sabs[blk] = a;
        }
    }
    if (bad && nonfinite_flag != nullptr) atomicOr(nonfinite_flag, 1);
    __syncthreads();

    const int64_t gblk = group * QLORA_GROUP + tid;
    const bool live = kFull || gblk < nblocks;
    const float c = sabs[tid];
    if (f.scale_fmt == QLORA_SCALES_FP32) {
        if (live) reinterpret_cast<float*>(scales)[gblk] = c;
        return;
    }
    float m = c;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) sred[warp] = m;
    __syncthreads();
    float gmax = sred[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) gmax = fmaxf(gmax, sred[w]);
    const float c2 = __fdiv_rn(gmax, scale8_top(f.scale_fmt));
    const uint8_t code = c2 > 0.f ? scale8_encode(__fdiv_rn(c, c2), f.scale_fmt) : uint8_t(0);
    if (live) reinterpret_cast<uint8_t*>(scales)[gblk] = code;
    if (tid == 0) meta[group] = c2;
}

__global__ void __launch_bounds__(kThreads)
dequantize_fmt_kernel(const uint32_t* __restrict__ packed, const void* __restrict__ scales,
                      const float* __restrict__ meta, int64_t numel, FmtArgs f,
                      uint16_t* __restrict__ out, FmtTable tab) {
    __shared__ float scode[16];
    if (threadIdx.x == 0) {
#pragma unroll
        for (int q = 0; q < 16; ++q) scode[q] = tab.code[q];
    }
    __syncthreads();
    const int64_t nwords = (numel + 7) / 8;
    for (int64_t u = blockIdx.x * int64_t(kThreads) + threadIdx.x; u < nwords;
         u += int64_t(gridDim.x) * kThreads) {
        const uint32_t v = packed[u];
        const int64_t b = (u * 8) >> f.log2_block;
        float ct;
        if (f.scale_fmt == QLORA_SCALES_FP32) {
            ct = reinterpret_cast<const float*>(scales)[b];
        } else {
            const uint8_t code = reinterpret_cast<const uint8_t*>(scales)[b];
            const float d = f.scale_fmt == QLORA_SCALES_E4M3 ? e4m3_to_float(code)
                          : f.scale_fmt == QLORA_SCALES_E5M2 ? e5m2_to_float(code)
                                                            : static_cast<float>(code);
            ct = __fmul_rn(d, meta[b >> 8]);
        }
        uint32_t r[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            r[j] = pack_bf16x2(__fmul_rn(scode[(v >> (8 * j)) & 15u], ct),
                               __fmul_rn(scode[(v >> (8 * j + 4)) & 15u], ct));
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

cudaError_t launch_quantize_fmt(const float* W, int64_t numel, const FmtArgs& f, uint8_t* packed,
                                void* scales, float* meta, int* nonfinite_flag,
                                const FmtTable& tab, cudaStream_t stream) {
    const int64_t nblocks = (numel + f.block - 1) / f.block;
    const int64_t ngroups = (nblocks + QLORA_GROUP - 1) / QLORA_GROUP;
    const int64_t group_elems = int64_t(QLORA_GROUP) * f.block;
    const int64_t full = numel / group_elems;                // groups with no tail
    if (f.block == 64 && tab.use_lut)      // K1's kernel, with this codebook and scale format
        return launch_quantize_b64(W, numel, packed, scales, meta, nonfinite_flag, tab.lut,
                                   tab.zero_index, f.scale_fmt, stream);
    if (full > 0) {
        const dim3 grid(static_cast<unsigned>(full));
        if (f.block == 16)
            quantize_fmt_kernel<true, 4><<<grid, kThreads, 0, stream>>>(W, numel, nblocks, f, packed, scales,
                                                                       meta, nonfinite_flag, tab);
        else if (f.block == 32)
            quantize_fmt_kernel<true, 8><<<grid, kThreads, 0, stream>>>(W, numel, nblocks, f, packed, scales,
                                                                       meta, nonfinite_flag, tab);
        else  // at B = 64 a lane would hold 64 floats; block by block measured faster there
            quantize_fmt_kernel<true, 0><<<grid, kThreads, 0, stream>>>(W, numel, nblocks, f, packed, scales,
                                                                       meta, nonfinite_flag, tab);
    }
    if (ngroups > full) {
        // the single trailing group, offset so blockIdx.x is its group index
        const int64_t off = full * group_elems;
        const int64_t blk_off = full * QLORA_GROUP;
        void* sc = f.scale_fmt == QLORA_SCALES_FP32
                       ? static_cast<void*>(static_cast<float*>(scales) + blk_off)
                       : static_cast<void*>(static_cast<uint8_t*>(scales) + blk_off);
        quantize_fmt_kernel<false, 0><<<1, kThreads, 0, stream>>>(
            W + off, numel - off, nblocks - blk_off, f, packed + off / 2, sc,
            meta == nullptr ? nullptr : meta + full, nonfinite_flag, tab);
    }
    return cudaGetLastError();
}

cudaError_t launch_dequantize_fmt(const uint8_t* packed, const void* scales, const float* meta,
                                  int64_t numel, const FmtArgs& f, uint16_t* out,
                                  const FmtTable& tab, int num_sms, cudaStream_t stream) {
    const int64_t nwords = (numel + 7) / 8;
    int64_t grid = (nwords + kThreads - 1) / kThreads;
    const int64_t cap = int64_t(num_sms) * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    dequantize_fmt_kernel<<<dim3(static_cast<unsigned>(grid)), kThreads, 0, stream>>>(
        reinterpret_cast<const uint32_t*>(packed), scales, meta, numel, f, out, tab);
    return cudaGetLastError();
}

}  // namespace qnf4
