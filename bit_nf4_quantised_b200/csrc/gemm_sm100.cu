// K2/K3: fused NF4 dequant-GEMM on the 5th-generation tensor cores (tcgen05,
// accumulators in TMEM), with the LoRA term folded into the same accumulators.
//
//   forward (kTrans = false):  Y  = X  W~^T + (gamma T) B^T        D = [M x N]
//   input grad (kTrans = true): dX = dY W~  + (gamma U) A          D = [M x K]
//
// "QLoRA, explained", "The forward pass and gradients": W~ is produced block by
// block from the stored NF4 indices and double-quantised scales, exists only
// transiently, and is produced a second time for the input gradient.
//
// Design: a cluster of two CTAs on two SMs computes a 512 x 256 output tile
// with the pair MMA (tcgen05.mma.cta_group::2, 256 x 256 x 16): each CTA holds
// 128 of every 256 tokens (A operand) and 128 of the 256 output columns
// (B operand, its half of the W~ tile), and two accumulators of 128 lanes x
// 256 fp32 columns fill its 512-column TMEM.  One dequantised W~ element thus
// feeds 512 tokens, and each SM expands only half of the tile: this is what
// keeps the dequantisation (integer/permute work on the CUDA cores) below the
// tensor-core rate.
//   warp 0      TMA producer: two 128 x 64 activation tiles (X or dY, 128-byte
//               swizzle) per 64-wide contraction step, counted on the even
//               CTA's barrier, and this CTA's packed-nibble tile (32- or
//               64-byte swizzle, so the dequantisers read it conflict-free),
//               counted locally; 4-stage ring.
//   warps 2..9  dequantisers in two groups of four that take alternate steps:
//               one thread per 64-element NF4 block of this CTA's B half.  A
//               thread builds its block's 16-entry table of
//               bf16_rne(fp32(q[i] * c~)) once, maps each nibble to its bf16
//               with byte permutes, and stores the row straight into the
//               swizzled operand layout tcgen05 reads: K-major rows of W~ for
//               the forward, MN-major rows (W~ untransposed) for dX, so the
//               "transposed dequant" is only a different descriptor.  Each
//               warp then signals the even CTA's barrier.
//   warp 1      TMEM allocation (both CTAs); on the even CTA the MMA issuer:
//               8 pair MMAs per step, tcgen05.commit multicast to both CTAs
//               frees the stage.  After the K loop ceil(r/64) extra steps feed
//               (gamma T | gamma U) and (B | A) by TMA into the same ring and
//               accumulators: the LoRA term costs no separate pass over Y.
//   warps 2..9  then drain TMEM (tcgen05.ld), round to bf16 and store.
// Every mbarrier wait is bounded (common.cuh); on a timeout the kernel records
// an error word, lets in-flight copies and MMAs land, frees TMEM and returns.
#include "kernels.cuh"

namespace qnf4 {

namespace {

constexpr int kTileM = 512;        // tokens per pair tile (2 accumulators x 256)
constexpr int kTileN = 256;        // output columns per pair tile (MMA N)
constexpr int kHalfN = kTileN / 2; // B rows held by each CTA
constexpr int BK = 64;             // contraction per pipeline step (one NF4 block)
constexpr int kStages = 4;
constexpr int kGroups = 4;          // dequantiser groups, taking steps in turn
constexpr int kGroupThreads = 128;  // dequantisers per group: one per B row
constexpr int kThreads = 64 + kGroups * kGroupThreads;
constexpr int kSA1 = 128 * BK * 2; // 16 KiB: one 128-row activation tile
constexpr int kSA = 2 * kSA1;      // both accumulators' activation tiles
constexpr int kSB = kHalfN * BK * 2;   // 16 KiB: this CTA's half of W~ (or LoRA)
constexpr int kSP = kHalfN * BK / 2;   //  4 KiB: packed nibbles of that half
constexpr int kStageBytes = kSA + kSB + kSP;
constexpr int kTmemCols = 512;
static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");

struct __align__(8) Barriers {
    uint64_t a_full[kStages];      // even CTA: both CTAs' TMA bytes of a stage
    uint64_t pk_full[kStages];     // local: this CTA's packed tile
    uint64_t deq_full[kStages];    // even CTA: 8 dequant warps of the pair
    uint64_t empty[kStages];       // local: MMAs of the stage done
    uint64_t acc_full;             // local: all MMAs of a tile done
    uint64_t acc_empty;            // even CTA: 16 epilogue warps of the pair drained TMEM
    uint64_t drain;
    uint32_t tmem_slot;
    int abort_flag;
};

// Epilogue: the last two dequantiser groups (8 warps) drain the
// accumulators; each stages its output in two alternating 1 KiB buffers of
// 32 rows x 16 bf16 columns written out by TMA tensor stores.
constexpr int kEpiWarps = 8;
constexpr int kStageOut = 2048;
constexpr int kOutBytes = kEpiWarps * kStageOut;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align slack*/ + 1024 /*barriers*/ + kOutBytes;
static_assert(sizeof(Barriers) <= 1024, "barrier block");
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

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
    // chunk c lands at (c ^ swz) * 16 = row_addr ^ (c << 4) with swz folded in
    const uint32_t base = row_addr | (swz << 4);
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
        const uint32_t dst = base ^ (static_cast<uint32_t>(c) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(o[0]), "r"(o[1]),
                     "r"(o[2]), "r"(o[3])
                     : "memory");
    }
}

// The tiles of one CTA pair: its run [pair * col_budget, + col_budget) of the
// output taken as m_tiles x cols_lin in row-major order, cut at 512-token row
// boundaries and every 256 columns.
struct TileIter {
    int64_t pos, end, cols;
    __device__ TileIter(const GemmArgs& a, int pair)
        : pos(int64_t(pair) * a.col_budget),
          end(min(int64_t(pair + 1) * a.col_budget, int64_t(a.m_tiles) * a.cols_lin)),
          cols(a.cols_lin) {}
    // Widths are multiples of the host's granule (32, or 128 for dX so that
    // each CTA's half is whole NF4 blocks and its TMA x coordinates stay
    // 16-byte aligned); a schedule that breaks this ends the walk with an
    // error instead of issuing a misaligned copy.
    __device__ bool next(int& m0, int& n0, int& w, bool trans, int* err) {
        if (pos >= end) return false;
        const int64_t c = pos % cols;
        w = static_cast<int>(min(int64_t(kTileN), min(cols - c, end - pos)));
        if ((w & (trans ? 127 : 31)) != 0 || (c & (trans ? 127 : 31)) != 0) {
            atomicOr(err, kErrBadSchedule);
            pos = end;
            return false;
        }
        m0 = static_cast<int>(pos / cols) * kTileM;
        n0 = static_cast<int>(c);
        pos += w;
        return true;
    }
};

template <bool kTrans>
__global__ void __launch_bounds__(kThreads, 1)
qlora_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,    // X or dY   [M x Kc] bf16
                  const __grid_constant__ CUtensorMap tm_packed, // packed W  [N x K/2] u8
                  const __grid_constant__ CUtensorMap tm_lora_a, // gamma T|U [M x rp] bf16
                  const __grid_constant__ CUtensorMap tm_lora_b, // B [N x rp] | A [rp x K]
                  const __grid_constant__ CUtensorMap tm_out,    // D [M x d_cols] bf16, box {16, 32}
                  GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Barriers* bars = reinterpret_cast<Barriers*>(smem + kStages * kStageBytes);
    volatile int* abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();          // 0 = even CTA (issues the MMAs)
    const int pair = blockIdx.x >> 1;
    const int total_steps = a.main_steps + a.tail_steps;
    // The whole grid is resident at once (one wave, or persistent pairs), so
    // kernels launched as its programmatic dependents (the backward's LoRA
    // products, which do not read this kernel's output) may start now and
    // fill the SMs it leaves idle.
    launch_dependents();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->a_full[s], 1);
            mbar_init(&bars->pk_full[s], 1);
            mbar_init(&bars->deq_full[s], 2 * kGroupThreads / 32);
            mbar_init(&bars->empty[s], 1);
        }
        mbar_init(&bars->acc_full, 1);
        mbar_init(&bars->acc_empty, 2 * kEpiWarps);
        mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm_act);
        prefetch_tensormap(&tm_packed);
        prefetch_tensormap(&tm_lora_a);
        prefetch_tensormap(&tm_lora_b);
        prefetch_tensormap(&tm_out);
    }
    if (warp == 1) {
        tmem_alloc_pair(&bars->tmem_slot, kTmemCols);
        tc_fence_before();
    }
    cluster_sync();                                   // barrier inits visible pair-wide
    tc_fence_after();
    const uint32_t tmem_d = bars->tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            int armed[kStages];
            for (int s = 0; s < kStages; ++s) armed[s] = -1;
            TileIter tiles(a, pair);
            int m0, n0, w;
            uint32_t gstep = 0;                       // steps over all of this pair's tiles
            bool ok = true;
            while (ok && tiles.next(m0, n0, w, kTrans, a.err)) {
                const int nh0 = n0 + static_cast<int>(rank) * (w / 2);   // this CTA's B half
                const int arow = m0 + static_cast<int>(rank) * 128;
                for (int step = 0; step < total_steps; ++step, ++gstep) {
                    const int s = gstep % kStages;
                    const uint32_t ph = (gstep / kStages) & 1;
                    if (!mbar_wait(&bars->empty[s], ph ^ 1, abort_flag, a.err, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sA = smem + s * kStageBytes;
                    uint8_t* sB = sA + kSA;
                    uint8_t* sP = sB + kSB;
                    const uint32_t a_full0 = mapa_shared(smem_u32(&bars->a_full[s]), 0);
                    if (step < a.main_steps) {
                        if (rank == 0) mbar_arrive_expect_tx(&bars->a_full[s], 2 * kSA);
                        tma_load_2d_pair(sA, &tm_act, step * BK, arow, a_full0);
                        tma_load_2d_pair(sA + kSA1, &tm_act, step * BK, arow + 256, a_full0);
                        mbar_arrive_expect_tx(&bars->pk_full[s], kSP);
                        if (!kTrans)
                            tma_load_2d(sP, &tm_packed, step * (BK / 2), nh0, &bars->pk_full[s]);
                        else
                            tma_load_2d(sP, &tm_packed, nh0 / 2, step * BK, &bars->pk_full[s]);
                        armed[s] = static_cast<int>(ph);
                    } else {
                        const int j = step - a.main_steps;
                        // nothing to expand: the stage's packed-tile barrier
                        // still takes one phase per step, so that every
                        // stage's barriers stay in step over the tiles
                        mbar_arrive(&bars->pk_full[s]);
                        armed[s] = static_cast<int>(ph);
                        // (gamma T | gamma U) comes from the preceding kernel:
                        // with a programmatic launch, wait for it here, not
                        // before the main loop
                        if (j == 0) grid_dependency_wait();
                        if (rank == 0) mbar_arrive_expect_tx(&bars->a_full[s], 2 * (kSA + kSB));
                        tma_load_2d_pair(sA, &tm_lora_a, j * BK, arow, a_full0);
                        tma_load_2d_pair(sA + kSA1, &tm_lora_a, j * BK, arow + 256, a_full0);
                        if (!kTrans) {
                            tma_load_2d_pair(sB, &tm_lora_b, j * BK, nh0, a_full0);
                        } else {
                            tma_load_2d_pair(sB, &tm_lora_b, nh0, j * BK, a_full0);
                            tma_load_2d_pair(sB + 64 * 128, &tm_lora_b, nh0 + 64, j * BK, a_full0);
                        }
                    }
                }
            }
            if (*abort_flag) {
                for (int s = 0; s < kStages; ++s)
                    if (armed[s] >= 0) mbar_drain(&bars->pk_full[s], armed[s], a.err);
                // copies counted on the even CTA's barrier cannot be awaited
                // here: give them time to land before the CTA exits
                const unsigned long long t0 = globaltimer_ns();
                while (globaltimer_ns() - t0 < 50000ull) {
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (rank == 0 && lane == 0) {
            TileIter tiles(a, pair);
            int m0, n0, w;
            uint32_t gstep = 0;
            int tile = 0;
            bool ok = true;
            while (ok && tiles.next(m0, n0, w, kTrans, a.err)) {
                // the accumulators are free once both CTAs' epilogues of the
                // previous tile have read them
                if (tile > 0) {
                    ok = mbar_wait_cluster(&bars->acc_empty, (tile - 1) & 1, abort_flag, a.err, a.wait_ns);
                    if (!ok) break;
                    tc_fence_after();
                }
                const uint32_t idesc = idesc_bf16_f32(256, w, false, kTrans);
                for (int step = 0; step < total_steps; ++step, ++gstep) {
                    const int s = gstep % kStages;
                    const uint32_t ph = (gstep / kStages) & 1;
                    const bool main = step < a.main_steps;
                    ok = mbar_wait_cluster(&bars->a_full[s], ph, abort_flag, a.err, a.wait_ns);
                    // (deq_full takes a phase on LoRA steps too, with no expansion)
                    if (ok) ok = mbar_wait_cluster(&bars->deq_full[s], ph, abort_flag, a.err, a.wait_ns);
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
                        const uint64_t bdesc =
                            kTrans ? smem_desc_sw128(b_base + kk * 2048, 64 * 128, 1024)
                                   : smem_desc_sw128(b_base + kk * 32, 16, 1024);
#pragma unroll
                        for (int acc = 0; acc < 2; ++acc) {
                            const uint64_t adesc =
                                smem_desc_sw128(a_base + acc * kSA1 + kk * 32, 16, 1024);
                            tc_mma_bf16_pair(tmem_d + acc * kTileN, adesc, bdesc, idesc,
                                             (step | kk) != 0 ? 1u : 0u);
                        }
                    }
                    tc_commit_pair(&bars->empty[s], 0x3);
                }
                if (!ok) break;
                tc_commit_pair(&bars->acc_full, 0x3);
                ++tile;
            }
            if (ok) {
                if (tile > 0) mbar_drain(&bars->acc_full, (tile - 1) & 1, a.err);   // MMAs done before teardown
            } else {
                tc_commit_pair(&bars->drain, 0x1);
                mbar_drain(&bars->drain, 0, a.err);
            }
        }
    } else {
        // ------------------------------------------------- dequantisers
        const int group = (warp - 2) >> 2;                      // takes steps group, group+kGroups, ...
        const int t = ((warp - 2) & 3) * 32 + lane;             // 0..127
        const int64_t nkb = a.nkb;
        // forward: row nh0+t of W, block = step.
        // dX: row step*64 + (t & 63) of W, block nh0/64 + (t >> 6).
        // Threads past a narrower tile's half expand rows the MMA ignores.
        const int nr = t & 63, kbl = t >> 6;
        uint32_t p_off0, p_off1, b_off, swz;
        if (!kTrans) {
            const uint32_t x = static_cast<uint32_t>((t >> 2) & 1);       // 32-byte swizzle
            p_off0 = t * 32 + ((0u ^ x) << 4);
            p_off1 = t * 32 + ((1u ^ x) << 4);
            b_off = t * 128;
            swz = t & 7;
        } else {
            const uint32_t x = static_cast<uint32_t>((nr >> 1) & 3);      // 64-byte swizzle
            p_off0 = nr * 64 + (((2u * kbl) ^ x) << 4);
            p_off1 = nr * 64 + (((2u * kbl + 1u) ^ x) << 4);
            b_off = kbl * (64 * 128) + nr * 128;
            swz = nr & 7;
        }
        const int q = warp & 3;                     // TMEM lane quarter of this warp
        // groups kGroups-2 and kGroups-1 drain accumulators 0 and 1; the first
        // groups go straight on to the next tile's first steps
        const bool epi = group >= kGroups - 2;
        const int acc = group - (kGroups - 2);
        const uint32_t out_stage = smem_u32(smem + kStages * kStageBytes + 1024) +
                                   static_cast<uint32_t>((epi ? warp - 2 - 4 * (kGroups - 2) : 0) * kStageOut);
        uint32_t nbox = 0;                          // boxes this warp has staged (buffer = nbox & 1)
        TileIter tiles(a, pair);
        int m0, n0, w;
        uint32_t gbase = 0;                         // pair-wide index of the tile's first step
        int tile = 0;
        bool ok = true;
        while (ok && tiles.next(m0, n0, w, kTrans, a.err)) {
            const int nh0 = n0 + static_cast<int>(rank) * (w / 2);
            const int64_t kb_fixed = (nh0 >> 6) + kbl;
            auto scale_of = [&](int step, uint32_t& code, float& meta) {
                code = 0;
                meta = 0.f;
                if (step >= a.main_steps) return;
                int64_t n, ci;
                if (!kTrans) {
                    n = int64_t(nh0) + t;
                    ci = n * nkb + step;
                    if (n >= a.Nw) return;
                } else {
                    n = int64_t(step) * BK + nr;
                    ci = n * nkb + kb_fixed;
                    if (n >= a.Nw || kb_fixed >= nkb) return;
                }
                code = __ldg(a.scale_codes + ci);
                meta = __ldg(a.meta + (ci >> 8));
            };
            uint32_t code_cur, code_next;
            float meta_cur, meta_next;
            scale_of(group, code_cur, meta_cur);
            scale_of(group + kGroups, code_next, meta_next);
            // main steps are expanded; on the LoRA steps the group only passes
            // the stage's barriers on, keeping their phases in step
            for (int step = group; step < total_steps; step += kGroups) {
                const uint32_t gs = gbase + static_cast<uint32_t>(step);
                const int s = gs % kStages;
                const uint32_t ph = (gs / kStages) & 1;
                if (!mbar_wait(&bars->pk_full[s], ph, abort_flag, a.err, a.wait_ns)) {
                    ok = false;
                    break;
                }
                if (step >= a.main_steps) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&bars->deq_full[s]), 0));
                    continue;
                }
                const uint32_t sbase = smem_u32(smem + s * kStageBytes);
                const uint32_t pbase = sbase + kSA + kSB;
                uint32_t wv[8];
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(wv[0]), "=r"(wv[1]), "=r"(wv[2]), "=r"(wv[3])
                             : "r"(pbase + p_off0));
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(wv[4]), "=r"(wv[5]), "=r"(wv[6]), "=r"(wv[7])
                             : "r"(pbase + p_off1));
                const float ct = __fmul_rn(e4m3_to_float(static_cast<uint8_t>(code_cur)), meta_cur);
                dequant_block_to_smem(wv, ct, a.tab, sbase + kSA + b_off, swz);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&bars->deq_full[s]), 0));
                code_cur = code_next;
                meta_cur = meta_next;
                scale_of(step + 2 * kGroups, code_next, meta_next);
            }
            if (!ok) break;

            // Every group waits for the tile's MMAs to finish: then every phase
            // of every stage barrier of this tile is complete.  A stage's
            // owning group changes at a tile boundary (a tile's step count
            // need not be a multiple of kGroups), and a parity wait is only
            // sound when the waiter is at most one phase ahead of the last
            // completed phase, so no group may start the next tile earlier.
            if (!mbar_wait(&bars->acc_full, tile & 1, abort_flag, a.err, a.wait_ns)) break;

            // ---------------------------------------------- epilogue
            if (epi) {
                tc_fence_after();
                // Each 32-column TMEM chunk leaves as two 32-row x 16-column
                // bf16 boxes, staged alternately in this warp's two buffers
                // and written by TMA tensor stores (full 32-byte sectors; rows
                // past M, columns past d_cols are not written), so that one
                // box's copy-out overlaps the next box's staging.
                const int row0 = m0 + acc * 256 + static_cast<int>(rank) * 128 + q * 32;
#pragma unroll 1
                for (int c = 0; c < w / 32; ++c) {
                    const int col = c * 32;
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem_d + (static_cast<uint32_t>(q * 32) << 16) + acc * kTileN + col, r);
                    tc_wait_ld();
#pragma unroll
                    for (int h = 0; h < 2; ++h, ++nbox) {
                        const uint32_t buf = out_stage + (nbox & 1) * 1024;
                        uint32_t p[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            p[j] = pack_bf16x2(__uint_as_float(r[16 * h + 2 * j]),
                                               __uint_as_float(r[16 * h + 2 * j + 1]));
                        if (lane == 0) bulk_wait_read_all_but_one();   // this buffer's last box has left
                        __syncwarp();
                        const uint32_t dst = buf + lane * 32;
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(p[0]),
                                     "r"(p[1]), "r"(p[2]), "r"(p[3])
                                     : "memory");
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 16), "r"(p[4]),
                                     "r"(p[5]), "r"(p[6]), "r"(p[7])
                                     : "memory");
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tm_out, n0 + col + 16 * h, row0, buf);
                            bulk_commit();
                        }
                    }
                }
                // this warp's reads of the accumulator are done: the next
                // tile's MMAs may overwrite it
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&bars->acc_empty), 0));
            }
            gbase += static_cast<uint32_t>(total_steps);
            ++tile;
        }
        if (lane == 0) bulk_wait_all();             // this warp's output stores have landed
    }

    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_d, kTmemCols);
    }
}

template <bool kTrans>
cudaError_t launch_one(const CUtensorMap& act, const CUtensorMap& packed, const CUtensorMap& la,
                       const CUtensorMap& lb, const CUtensorMap& out, const GemmArgs& args,
                       unsigned pairs, bool after_lora, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(qlora_gemm_kernel<kTrans>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_lora ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, qlora_gemm_kernel<kTrans>, act, packed, la, lb, out, args);
}

}  // namespace

cudaError_t launch_gemm(bool trans, const CUtensorMap& act, const CUtensorMap& packed,
                        const CUtensorMap& lora_a, const CUtensorMap& lora_b, const CUtensorMap& out,
                        const GemmArgs& args, bool after_lora, cudaStream_t stream) {
    const int64_t total = int64_t(args.m_tiles) * args.cols_lin;
    if (total <= 0 || args.col_budget <= 0) return cudaSuccess;
    const int64_t pairs = (total + args.col_budget - 1) / args.col_budget;
    if (2 * pairs > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const cudaError_t e =
        trans ? launch_one<true>(act, packed, lora_a, lora_b, out, args, unsigned(pairs), after_lora, stream)
              : launch_one<false>(act, packed, lora_a, lora_b, out, args, unsigned(pairs), after_lora, stream);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

int gemm_tile_m() { return kTileM; }
int gemm_tile_n() { return kTileN; }
// TMA boxes the host must encode for the packed-weight map of this kernel:
// forward {32 bytes, 128 rows} with 32-byte swizzle; dX {64 bytes, 64 rows}
// with 64-byte swizzle.  The LoRA B-operand box is 128 rows (forward) or
// 64 x 64 (dX); activation boxes are {64, 128} with 128-byte swizzle.
int gemm_half_n() { return kHalfN; }
int gemm_col_granule(bool trans) { return trans ? 128 : 32; }

}  // namespace qnf4
