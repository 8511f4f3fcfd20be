// K2/K3: fused NF4 dequant-GEMM on the 5th-generation tensor cores (tcgen05,
// accumulators in TMEM), with the LoRA term folded into the same accumulator.
//
//   forward (kTrans = false):  Y  = X  W~^T + (gamma T) B^T        D = [M x N]
//   input grad (kTrans = true): dX = dY W~  + (gamma U) A          D = [M x K]
//
// "QLoRA, explained", "The forward pass and gradients": W~ is produced block by
// block from the stored NF4 indices and double-quantised scales, exists only
// transiently, and is produced a second time for the input gradient.
//
// Design (one CTA per 128 x 256 output tile, 320 threads, warp-specialised):
//   warp 0      TMA producer: the activation tile (X or dY, 128 x 64 bf16,
//               128-byte swizzle) and the packed-nibble tile of W for each
//               64-wide contraction step, into a 3-stage shared-memory ring.
//   warps 2..9  dequantisers: one thread per 64-element NF4 block per step.
//               A thread builds its block's 16-entry table of
//               bf16_rne(fp32(q[i] * c~)) once, then maps each nibble to its
//               bf16 with byte permutes (no per-element multiply or memory
//               lookup), and stores the row straight into the swizzled
//               operand layout tcgen05 reads: K-major rows of W~ for the
//               forward, MN-major rows (W~ untransposed) for dX, so the
//               "transposed dequant" is only a different descriptor.
//   warp 1      MMA issuer: 4 x tcgen05.mma (128 x 256 x 16) per step into a
//               128 x 256 fp32 TMEM accumulator; tcgen05.commit frees the
//               stage.  After the K loop, ceil(r/64) extra steps feed
//               (gamma T | gamma U) and (B | A) by TMA into the same ring and
//               accumulator: the LoRA term costs no separate pass over Y.
//   warps 2..9  then drain TMEM (tcgen05.ld), round to bf16 and store.
// Every mbarrier wait is bounded (see common.cuh); on a timeout the kernel
// records an error word, lets in-flight copies and MMAs land, frees TMEM and
// returns.
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int BM = 128;            // tokens per tile (MMA M)
constexpr int BN = 256;            // output columns per tile (MMA N)
constexpr int BK = 64;             // contraction per pipeline step (one NF4 block)
constexpr int kStages = 3;
constexpr int kThreads = 320;
constexpr int kDeqThreads = 256;
constexpr int kSA = BM * BK * 2;   // 16 KiB activation tile
constexpr int kSB = BN * BK * 2;   // 32 KiB W~ (or LoRA) tile
constexpr int kSP = BN * BK / 2;   //  8 KiB packed nibbles
constexpr int kStageBytes = kSA + kSB + kSP;
constexpr int kTmemCols = 256;
static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");

struct __align__(8) Barriers {
    uint64_t full_tma[kStages];
    uint64_t full_deq[kStages];
    uint64_t empty[kStages];
    uint64_t acc_full;
    uint64_t drain;
    uint32_t tmem_slot;
    int abort_flag;
};

constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align slack*/ + 256 /*barriers*/;
static_assert(sizeof(Barriers) <= 256, "barrier block");

// 64 nibbles (8 words) of one NF4 block -> 64 bf16, stored as 8 16-byte chunks
// of a 128-byte swizzled row.  Table entries are bf16_rne(fp32(q[i] * ct)).
__device__ __forceinline__ void dequant_block_to_smem(const uint32_t (&w)[8], float ct,
                                                      const Nf4Table& tab, uint32_t row_addr,
                                                      uint32_t swz) {
    uint32_t t2[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        t2[j] = pack_bf16x2(__fmul_rn(tab.code[2 * j], ct), __fmul_rn(tab.code[2 * j + 1], ct));
    uint32_t lo_plane[4], hi_plane[4];         // low / high bytes of entries 4p..4p+3
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        lo_plane[p] = prmt(t2[2 * p], t2[2 * p + 1], 0x6420u);
        hi_plane[p] = prmt(t2[2 * p], t2[2 * p + 1], 0x7531u);
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint32_t v = w[c];
        const uint32_t s7 = v & 0x77777777u;                            // entry within half
        const uint32_t s8 = ((v >> 1) & 0x44444444u) | 0x32103210u;      // which half
        uint32_t o[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t sa = h ? (s7 >> 16) : s7;
            const uint32_t sb = h ? (s8 >> 16) : s8;
            const uint32_t la = prmt(lo_plane[0], lo_plane[1], sa);
            const uint32_t lb = prmt(lo_plane[2], lo_plane[3], sa);
            const uint32_t ha = prmt(hi_plane[0], hi_plane[1], sa);
            const uint32_t hb = prmt(hi_plane[2], hi_plane[3], sa);
            const uint32_t lo = prmt(la, lb, sb);
            const uint32_t hi = prmt(ha, hb, sb);
            o[2 * h] = prmt(lo, hi, 0x5140u);
            o[2 * h + 1] = prmt(lo, hi, 0x7362u);
        }
        const uint32_t dst = row_addr + ((static_cast<uint32_t>(c) ^ swz) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(o[0]), "r"(o[1]),
                     "r"(o[2]), "r"(o[3])
                     : "memory");
    }
}

template <bool kTrans>
__global__ void __launch_bounds__(kThreads, 1)
qlora_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,    // X or dY   [M x Kc] bf16
                  const __grid_constant__ CUtensorMap tm_packed, // packed W  [N x K/2] u8
                  const __grid_constant__ CUtensorMap tm_lora_a, // gamma T|U [M x rp] bf16
                  const __grid_constant__ CUtensorMap tm_lora_b, // B [N x rp] | A [rp x K]
                  GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Barriers* bars = reinterpret_cast<Barriers*>(smem + kStages * kStageBytes);
    volatile int* abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m_tile = blockIdx.x % a.m_tiles;
    const int n_tile = blockIdx.x / a.m_tiles;
    const int m0 = m_tile * BM;
    const int n0 = n_tile * BN;          // first output column of this tile
    const int total_steps = a.main_steps + a.tail_steps;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->full_tma[s], 1);
            mbar_init(&bars->full_deq[s], kDeqThreads / 32);
            mbar_init(&bars->empty[s], 1);
        }
        mbar_init(&bars->acc_full, 1);
        mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm_act);
        prefetch_tensormap(&tm_packed);
        prefetch_tensormap(&tm_lora_a);
        prefetch_tensormap(&tm_lora_b);
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_slot, kTmemCols);
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = bars->tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            int armed[kStages];
            for (int s = 0; s < kStages; ++s) armed[s] = -1;
            for (int step = 0; step < total_steps; ++step) {
                const int s = step % kStages;
                const uint32_t ph = (step / kStages) & 1;
                if (!mbar_wait(&bars->empty[s], ph ^ 1, abort_flag, a.err)) break;
                uint8_t* sA = smem + s * kStageBytes;
                uint8_t* sB = sA + kSA;
                uint8_t* sP = sB + kSB;
                if (step < a.main_steps) {
                    mbar_arrive_expect_tx(&bars->full_tma[s], kSA + kSP);
                    tma_load_2d(sA, &tm_act, step * BK, m0, &bars->full_tma[s]);
                    if (!kTrans)
                        tma_load_2d(sP, &tm_packed, step * (BK / 2), n0, &bars->full_tma[s]);
                    else
                        tma_load_2d(sP, &tm_packed, n0 / 2, step * BK, &bars->full_tma[s]);
                } else {
                    const int j = step - a.main_steps;
                    mbar_arrive_expect_tx(&bars->full_tma[s], kSA + kSB);
                    tma_load_2d(sA, &tm_lora_a, j * BK, m0, &bars->full_tma[s]);
                    if (!kTrans) {
                        tma_load_2d(sB, &tm_lora_b, j * BK, n0, &bars->full_tma[s]);
                    } else {
#pragma unroll
                        for (int c = 0; c < BN / 64; ++c)
                            tma_load_2d(sB + c * (64 * 128), &tm_lora_b, n0 + 64 * c, j * BK,
                                        &bars->full_tma[s]);
                    }
                }
                armed[s] = static_cast<int>(ph);
            }
            if (*abort_flag) {
                for (int s = 0; s < kStages; ++s)
                    if (armed[s] >= 0) mbar_drain(&bars->full_tma[s], armed[s], a.err);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, false, kTrans);
            bool ok = true;
            for (int step = 0; step < total_steps && ok; ++step) {
                const int s = step % kStages;
                const uint32_t ph = (step / kStages) & 1;
                const bool main = step < a.main_steps;
                ok = mbar_wait(&bars->full_tma[s], ph, abort_flag, a.err);
                if (ok && main) ok = mbar_wait(&bars->full_deq[s], ph, abort_flag, a.err);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a_base = smem_u32(smem + s * kStageBytes);
                const uint32_t b_base = a_base + kSA;
                int nk = BK / 16;
                if (!main) {
                    const int rem = a.r - (step - a.main_steps) * BK;
                    nk = min(BK / 16, (rem + 15) / 16);
                }
                for (int kk = 0; kk < nk; ++kk) {
                    const uint64_t adesc = smem_desc_sw128(a_base + kk * 32, 16, 1024);
                    const uint64_t bdesc =
                        kTrans ? smem_desc_sw128(b_base + kk * 2048, 64 * 128, 1024)
                               : smem_desc_sw128(b_base + kk * 32, 16, 1024);
                    tc_mma_bf16(tmem_d, adesc, bdesc, idesc, (step | kk) != 0 ? 1u : 0u);
                }
                tc_commit(&bars->empty[s]);
            }
            if (ok) {
                tc_commit(&bars->acc_full);
            } else {
                tc_commit(&bars->drain);           // let issued MMAs finish before exit
                mbar_drain(&bars->drain, 0, a.err);
            }
        }
    } else {
        // ------------------------------------------------- dequantisers
        const int t = threadIdx.x - 64;            // 0..255
        const uint32_t swz = static_cast<uint32_t>(t & 7);
        // fwd: row n0+t of W, block = step.   dX: row step*64+(t&63), block k0/64+(t>>6).
        const int64_t nkb = a.nkb;
        const int kb_fixed = (n0 >> 6) + (t >> 6);
        auto code_index = [&](int step, int64_t& ci) -> bool {
            if (!kTrans) {
                const int64_t n = int64_t(n0) + t;
                ci = n * nkb + step;
                return n < a.Nw;
            } else {
                const int64_t n = int64_t(step) * BK + (t & 63);
                ci = n * nkb + kb_fixed;
                return n < a.Nw && kb_fixed < nkb;
            }
        };
        auto load_scale = [&](int step, uint32_t& code, float& meta) {
            int64_t ci;
            code = 0;
            meta = 0.f;
            if (step < a.main_steps && code_index(step, ci)) {
                code = __ldg(a.scale_codes + ci);
                meta = __ldg(a.meta + (ci >> 8));
            }
        };
        uint32_t code_cur, code_next;
        float meta_cur, meta_next;
        load_scale(0, code_cur, meta_cur);
        load_scale(1, code_next, meta_next);
        const uint32_t prow_off = kTrans ? static_cast<uint32_t>((t & 63) * 128 + (t >> 6) * 32)
                                         : static_cast<uint32_t>(t * 32);
        const uint32_t brow_off =
            kTrans ? static_cast<uint32_t>((t >> 6) * (64 * 128) + (t & 63) * 128)
                   : static_cast<uint32_t>(t * 128);
        for (int step = 0; step < a.main_steps; ++step) {
            const int s = step % kStages;
            const uint32_t ph = (step / kStages) & 1;
            if (!mbar_wait(&bars->full_tma[s], ph, abort_flag, a.err)) break;
            const uint32_t sbase = smem_u32(smem + s * kStageBytes);
            const uint32_t prow = sbase + kSA + kSB + prow_off;
            uint32_t w[8];
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                         : "r"(prow));
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                         : "r"(prow + 16));
            const float ct = __fmul_rn(e4m3_to_float(static_cast<uint8_t>(code_cur)), meta_cur);
            dequant_block_to_smem(w, ct, a.tab, sbase + kSA + brow_off, swz);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->full_deq[s]);
            code_cur = code_next;
            meta_cur = meta_next;
            load_scale(step + 2, code_next, meta_next);
        }

        // -------------------------------------------------- epilogue
        if (mbar_wait(&bars->acc_full, 0, abort_flag, a.err)) {
            tc_fence_after();
            const int q = warp & 3;                 // TMEM lane quarter of this warp
            const int half = (warp - 2) >> 2;       // which 128 columns
            const int64_t m = int64_t(m0) + q * 32 + lane;
            uint16_t* drow = a.D + m * a.d_cols;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                const int col = half * 128 + c * 32;
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_d + (static_cast<uint32_t>(q * 32) << 16) + col, r);
                tc_wait_ld();
                uint32_t p[16];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    p[j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
                if (m < a.M) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int64_t gc = int64_t(n0) + col + g * 8;
                        if (gc < a.d_cols)
                            *reinterpret_cast<uint4*>(drow + gc) =
                                make_uint4(p[4 * g], p[4 * g + 1], p[4 * g + 2], p[4 * g + 3]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_d, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_gemm(bool trans, const CUtensorMap& act, const CUtensorMap& packed,
                        const CUtensorMap& lora_a, const CUtensorMap& lora_b, const GemmArgs& args,
                        cudaStream_t stream) {
    const int64_t d_tiles = (args.d_cols + BN - 1) / BN;
    const int64_t grid = int64_t(args.m_tiles) * d_tiles;
    if (grid <= 0) return cudaSuccess;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (!trans) {
        cudaError_t e = cudaFuncSetAttribute(qlora_gemm_kernel<false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        qlora_gemm_kernel<false><<<dim3(static_cast<unsigned>(grid)), kThreads, kSmemBytes, stream>>>(
            act, packed, lora_a, lora_b, args);
    } else {
        cudaError_t e = cudaFuncSetAttribute(qlora_gemm_kernel<true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        qlora_gemm_kernel<true><<<dim3(static_cast<unsigned>(grid)), kThreads, kSmemBytes, stream>>>(
            act, packed, lora_a, lora_b, args);
    }
    return cudaGetLastError();
}

int gemm_tile_m() { return BM; }
int gemm_tile_n() { return BN; }

}  // namespace qnf4
