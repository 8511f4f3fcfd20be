// K5: bandwidth-bound dequant-GEMV for decode-sized token counts (M <= 16):
//   Y = X W~^T + gamma (X A^T) B^T
// ("QLoRA, explained": serving the adapter unmerged on the 4-bit base, "Failure
// modes and how to detect them").  The packed weight is streamed from HBM once.
//
// Swap-AB on mma.sync m16n8k16: rows of W are the MMA's M side, tokens its N
// side (one n8 tile for M <= 8, two for M <= 16).  A lane owns 8 contiguous
// bytes (16 nibbles) of rows g and g+8 of a 16-row tile per 64-wide block and
// turns each byte into the bf16 pair (q[lo], q[hi]) with one shared-memory
// load from a byte->bf16x2 table replicated per lane (so every lane always
// hits its own bank).  The table rows are 256 bytes apart and start at a
// 64 KiB-aligned shared address, so a single byte permute writes the byte
// into bits 8..15 of the lane's base address: one permute and one load per
// two weights.  The contraction order inside a block is permuted (lane c of a
// row group covers k = 16c .. 16c+15, four k-values per MMA step) and the
// activation fragment is gathered with the same permutation, so each MMA step
// is still an exact dot product over its 16 k-values.  A block's MMAs
// accumulate into fresh fp32 registers that are then scaled by the block's
// c~ = e4m3(code) * c2 (per-block scaling of fp32 partial sums).
//
// Deviation from the dequantise kernel, stated: the table holds bf16(q[i])
// rather than bf16(q[i] * c~), so each weight enters as bf16(q) * c~ in fp32;
// the difference from bf16_rne(q * c~) is below one bf16 ulp per weight, far
// inside the layer tolerance.
//
// Work split: one persistent 512-thread CTA per SM.  The contraction is cut
// into S slices (the activation slice lives in shared memory); each slice's
// CTAs pull 16-row tiles of W from an atomic counter, so the load balances
// itself whatever N is.  Packed bytes, scale codes and meta scales of the next
// four blocks are loaded while the current four are processed.  Each slice's
// first CTA also computes that slice's part of T = X A^T.  Slices write fp32
// partials; the finalize kernel sums them, adds gamma T B^T and rounds Y.
#include <algorithm>

#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kLutBytes = 256 * 256;       // 256 entries x 256-byte rows (32 lanes x 4 used)
constexpr int kSmemBytes = 227 * 1024;     // all of it: room for the 64 KiB-aligned table
constexpr int kUnroll = 4;                 // blocks per prefetch group

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16 pair of the byte `k` of w: lane_reg = table base + 4*lane with bits
// 8..15 clear; the permute drops byte k of w into bits 8..15.
template <int k>
__device__ __forceinline__ uint32_t lut_pair(uint32_t w, uint32_t lane_reg) {
    const uint32_t addr = prmt(w, lane_reg, 0x7604u | (k << 4));
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

struct Group {                      // one prefetch group: kUnroll blocks of two rows
    uint2 wa[kUnroll], wb[kUnroll];
    uint32_t ca, cb;                // scale codes of the kUnroll blocks (byte i = block i)
    float ma, mb;                   // meta scales
};

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
gemv_kernel(GemvArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t start = smem_u32(smem);
    const uint32_t lut = (start + 0xFFFFu) & ~0xFFFFu;          // 64 KiB aligned
    constexpr int XR = 8 * NT;                                  // activation rows held
    const int slice = blockIdx.y;
    const int64_t k_beg = int64_t(slice) * a.k_per_split;
    const int64_t k_end = min(a.K, k_beg + a.k_per_split);
    const int kslab = static_cast<int>(k_end - k_beg);
    const uint32_t x_pitch = static_cast<uint32_t>(kslab * 2 + 8);
    const uint32_t x_bytes = XR * x_pitch;
    const uint32_t xs = (lut - start >= x_bytes) ? start : lut + kLutBytes;

    // byte -> (bf16 q[lo nibble], bf16 q[hi nibble]), one copy per lane
    for (int e = tid; e < 256 * 32; e += kThreads) {
        const int b = e >> 5, l = e & 31;
        const uint32_t v = pack_bf16x2(a.tab.code[b & 15], a.tab.code[b >> 4]);
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(lut + b * 256 + l * 4), "r"(v) : "memory");
    }
    // activation slice [XR rows][kslab] bf16, zero beyond M (8-byte stores: the
    // row pitch is 8 mod 16 so that fragment loads spread over all banks)
    const int vec_per_row = kslab / 8;
    for (int q = tid; q < XR * vec_per_row; q += kThreads) {
        const int m = q / vec_per_row, v = q % vec_per_row;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (m < a.M) val = *reinterpret_cast<const uint4*>(a.X + m * a.K + k_beg + v * 8);
        const uint32_t dst = xs + m * x_pitch + v * 16;
        asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(dst), "r"(val.x), "r"(val.y) : "memory");
        asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(dst + 8), "r"(val.z), "r"(val.w)
                     : "memory");
    }
    __syncthreads();

    const int g = lane >> 2, c = lane & 3;

    // this slice's part of T = X A^T: the slice's first CTA, all warps, each a
    // 16-aligned range of k; fragments are gathered with 4-byte loads
    if (blockIdx.x == 0) {
        constexpr int kMaxJT = QLORA_MAX_RANK / 8;
        float tacc[kMaxJT][4];
#pragma unroll
        for (int j = 0; j < kMaxJT; ++j) tacc[j][0] = tacc[j][1] = tacc[j][2] = tacc[j][3] = 0.f;
        const int ksteps = kslab / 16;
        const int per = (ksteps + kWarps - 1) / kWarps;
        const int s0 = warp * per, s1 = min(ksteps, s0 + per);
        for (int s = s0; s < s1; ++s) {
            const int kk = s * 16 + 2 * c;
            const uint32_t a0 = lds32(xs + g * x_pitch + kk * 2);
            const uint32_t a2 = lds32(xs + g * x_pitch + (kk + 8) * 2);
            const uint32_t a1 = NT == 2 ? lds32(xs + (g + 8) * x_pitch + kk * 2) : 0u;
            const uint32_t a3 = NT == 2 ? lds32(xs + (g + 8) * x_pitch + (kk + 8) * 2) : 0u;
#pragma unroll
            for (int jt = 0; jt < kMaxJT; ++jt) {
                if (jt * 8 < a.r) {
                    const uint16_t* ap = a.A + int64_t(jt * 8 + g) * a.K + k_beg + kk;
                    const uint32_t b0 = __ldg(reinterpret_cast<const uint32_t*>(ap));
                    const uint32_t b1 = __ldg(reinterpret_cast<const uint32_t*>(ap + 8));
                    mma16816(tacc[jt], a0, a1, a2, a3, b0, b1);
                }
            }
        }
        // reduce the warps' tiles in the unused upper half (bytes 128..255) of
        // the table rows: element e lives at row e / 32, word e % 32
        __syncthreads();
        auto red_addr = [&](int e) { return lut + (e >> 5) * 256 + 128 + (e & 31) * 4; };
        for (int e = tid; e < 16 * QLORA_MAX_RANK; e += kThreads)
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(red_addr(e)), "r"(0u) : "memory");
        __syncthreads();
#pragma unroll
        for (int jt = 0; jt < kMaxJT; ++jt) {
            if (jt * 8 < a.r) {
                const int j = jt * 8 + 2 * c;
                asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(red_addr(g * QLORA_MAX_RANK + j)),
                             "f"(tacc[jt][0]) : "memory");
                asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(red_addr(g * QLORA_MAX_RANK + j + 1)),
                             "f"(tacc[jt][1]) : "memory");
                asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(red_addr((g + 8) * QLORA_MAX_RANK + j)),
                             "f"(tacc[jt][2]) : "memory");
                asm volatile("red.shared.add.f32 [%0], %1;"
                             ::"r"(red_addr((g + 8) * QLORA_MAX_RANK + j + 1)), "f"(tacc[jt][3])
                             : "memory");
            }
        }
        __syncthreads();
        for (int e = tid; e < a.M * a.r; e += kThreads) {
            const int m = e / a.r, j = e % a.r;
            a.Tpart[(int64_t(slice) * a.M + m) * a.r + j] =
                __uint_as_float(lds32(red_addr(m * QLORA_MAX_RANK + j)));
        }
        __syncthreads();       // the table's spare halves are not touched again
    }

    const int64_t nkb = a.K / QLORA_BLOCK;
    const int kb_beg = static_cast<int>(k_beg / QLORA_BLOCK);
    const int nblk = kslab / QLORA_BLOCK;
    const int ngroups = (nblk + kUnroll - 1) / kUnroll;
    const bool vec_codes = (nkb % kUnroll) == 0 &&
                           (reinterpret_cast<uintptr_t>(a.scale_codes) & 3u) == 0;
    const uint32_t lane_reg = lut + lane * 4;
    float* part = a.part + int64_t(slice) * a.M * a.N;
    const int64_t ntiles = (a.N + 15) / 16;

    for (;;) {
        int64_t rt = 0;
        if (lane == 0) rt = atomicAdd(a.counters + slice, 1);
        rt = __shfl_sync(0xffffffffu, rt, 0);
        if (rt >= ntiles) break;
        const int64_t na = rt * 16 + g, nb = na + 8;
        const bool va = na < a.N, vb = nb < a.N;
        const uint8_t* pa = a.packed + na * (a.K / 2) + int64_t(kb_beg) * 32 + c * 8;
        const uint8_t* pb = a.packed + nb * (a.K / 2) + int64_t(kb_beg) * 32 + c * 8;
        const int64_t cia = na * nkb + kb_beg, cib = nb * nkb + kb_beg;

        auto fetch = [&](int grp, Group& G) {
#pragma unroll
            for (int i = 0; i < kUnroll; ++i) {
                const int bi = grp * kUnroll + i;
                const bool in = bi < nblk;
                G.wa[i] = (va && in) ? __ldcs(reinterpret_cast<const uint2*>(pa + bi * 32)) : make_uint2(0, 0);
                G.wb[i] = (vb && in) ? __ldcs(reinterpret_cast<const uint2*>(pb + bi * 32)) : make_uint2(0, 0);
            }
            const int b0 = grp * kUnroll;
            if (vec_codes && b0 + kUnroll <= nblk) {
                G.ca = va ? __ldg(reinterpret_cast<const uint32_t*>(a.scale_codes + cia + b0)) : 0u;
                G.cb = vb ? __ldg(reinterpret_cast<const uint32_t*>(a.scale_codes + cib + b0)) : 0u;
            } else {
                G.ca = G.cb = 0u;
#pragma unroll
                for (int i = 0; i < kUnroll; ++i) {
                    if (b0 + i < nblk) {
                        if (va) G.ca |= uint32_t(__ldg(a.scale_codes + cia + b0 + i)) << (8 * i);
                        if (vb) G.cb |= uint32_t(__ldg(a.scale_codes + cib + b0 + i)) << (8 * i);
                    }
                }
            }
            // a group of kUnroll aligned blocks never straddles a meta group
            // when codes are vector-loaded; otherwise each block's meta is read
            G.ma = va ? __ldg(a.meta + ((cia + b0) >> 8)) : 0.f;
            G.mb = vb ? __ldg(a.meta + ((cib + b0) >> 8)) : 0.f;
        };

        float acc[NT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
        Group cur, nxt;
        fetch(0, cur);
        for (int grp = 0; grp < ngroups; ++grp) {
            if (grp + 1 < ngroups) fetch(grp + 1, nxt);
#pragma unroll
            for (int i = 0; i < kUnroll; ++i) {
                const int bi = grp * kUnroll + i;
                if (bi >= nblk) break;
                float ma = cur.ma, mb = cur.mb;
                if (!vec_codes) {               // blocks may cross a meta group
                    ma = va ? __ldg(a.meta + ((cia + bi) >> 8)) : 0.f;
                    mb = vb ? __ldg(a.meta + ((cib + bi) >> 8)) : 0.f;
                }
                const float cta = __fmul_rn(e4m3_to_float(uint8_t(cur.ca >> (8 * i))), ma);
                const float ctb = __fmul_rn(e4m3_to_float(uint8_t(cur.cb >> (8 * i))), mb);
                float blk[NT][4];
#pragma unroll
                for (int t = 0; t < NT; ++t) blk[t][0] = blk[t][1] = blk[t][2] = blk[t][3] = 0.f;
                const uint32_t xk = xs + static_cast<uint32_t>((bi * 64 + c * 16) * 2);
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const uint32_t wa_s = s < 2 ? cur.wa[i].x : cur.wa[i].y;
                    const uint32_t wb_s = s < 2 ? cur.wb[i].x : cur.wb[i].y;
                    uint32_t a0, a1, a2, a3;
                    if (s & 1) {
                        a0 = lut_pair<2>(wa_s, lane_reg);
                        a2 = lut_pair<3>(wa_s, lane_reg);
                        a1 = lut_pair<2>(wb_s, lane_reg);
                        a3 = lut_pair<3>(wb_s, lane_reg);
                    } else {
                        a0 = lut_pair<0>(wa_s, lane_reg);
                        a2 = lut_pair<1>(wa_s, lane_reg);
                        a1 = lut_pair<0>(wb_s, lane_reg);
                        a3 = lut_pair<1>(wb_s, lane_reg);
                    }
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        uint32_t b0, b1;
                        asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];"
                                     : "=r"(b0), "=r"(b1)
                                     : "r"(xk + (g + 8 * t) * x_pitch + s * 8));
                        mma16816(blk[t], a0, a1, a2, a3, b0, b1);
                    }
                }
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    acc[t][0] = fmaf(cta, blk[t][0], acc[t][0]);
                    acc[t][1] = fmaf(cta, blk[t][1], acc[t][1]);
                    acc[t][2] = fmaf(ctb, blk[t][2], acc[t][2]);
                    acc[t][3] = fmaf(ctb, blk[t][3], acc[t][3]);
                }
            }
            cur = nxt;
        }
        // C fragment of tile t: (row g, tokens 8t+2c, 8t+2c+1) and (row g+8, same)
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const int m0 = 8 * t + 2 * c;
            if (va && m0 < a.M) part[int64_t(m0) * a.N + na] = acc[t][0];
            if (va && m0 + 1 < a.M) part[int64_t(m0 + 1) * a.N + na] = acc[t][1];
            if (vb && m0 < a.M) part[int64_t(m0) * a.N + nb] = acc[t][2];
            if (vb && m0 + 1 < a.M) part[int64_t(m0 + 1) * a.N + nb] = acc[t][3];
        }
    }
}

// One thread per output column n: T = sum of the slices' parts (staged in
// shared memory), Y[m][n] = bf16( sum_s part[s][m][n] + gamma * T[m] . B[n] ).
__global__ void __launch_bounds__(256)
gemv_finalize_kernel(GemvFinalizeArgs a) {
    __shared__ float st[16 * QLORA_MAX_RANK];
    for (int e = threadIdx.x; e < a.M * a.r; e += blockDim.x) {
        float t = 0.f;
        for (int s = 0; s < a.splits; ++s) t += a.Tpart[int64_t(s) * a.M * a.r + e];
        st[e] = t;
        if (blockIdx.x == 0 && a.T_save) a.T_save[e] = t;
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
                for (int q = 0; q < 8; ++q) acc[m] = fmaf(st[m * a.r + j0 + q], b[q], acc[m]);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        if (m < a.M) {
            float s = a.gamma * acc[m];
            for (int k = 0; k < a.splits; ++k) s += a.part[(int64_t(k) * a.M + m) * a.N + n];
            __nv_bfloat16 y = __float2bfloat16_rn(s);
            a.Y[m * a.N + n] = *reinterpret_cast<uint16_t*>(&y);
        }
    }
}

}  // namespace

int gemv_max_activation_bytes() { return kSmemBytes - 2 * kLutBytes; }

cudaError_t launch_gemv(const GemvArgs& a, int num_sms, cudaStream_t stream) {
    const unsigned per_slice = static_cast<unsigned>(std::max(1, num_sms / std::max(1, a.splits)));
    dim3 grid(per_slice, static_cast<unsigned>(a.splits));
    cudaError_t e;
    if (a.M > 8) {
        e = cudaFuncSetAttribute(gemv_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        gemv_kernel<2><<<grid, kThreads, kSmemBytes, stream>>>(a);
    } else {
        e = cudaFuncSetAttribute(gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        gemv_kernel<1><<<grid, kThreads, kSmemBytes, stream>>>(a);
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
