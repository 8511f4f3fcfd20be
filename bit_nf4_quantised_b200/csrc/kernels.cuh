// Internal launch interface between the host layer (qlora_api.cu) and the
// kernels.  Not part of the public C ABI.
#pragma once

#include "common.cuh"

namespace qnf4 {

// ---------------------------------------------------------------- K1 / K6
// Nearest-code table of the quantiser.  A normalised value x in [-1, 1] is
// bucketed by y = max(x + 3, 2) in [2, 4]: bucket b = (bits of y >> 18) -
// 0x1000 (the top five mantissa bits; b = 32 only at x = 1, entries past it
// are padding).  Each bucket is 1/16 wide in x, narrower than the closest two
// NF4 midpoints, so it holds at most one: base[b] = the number of midpoints
// below the bucket (counted 2^-22 below its lower edge, past the rounding of
// x + 3) and thr[b] = the bits of midpoint number base[b] (+inf when base is
// 15).  The code index of any x in bucket b is base[b] + (x > thr[b]).
constexpr int kNf4LutEntries = 64;
struct Nf4IndexLut {
    uint32_t thr[kNf4LutEntries];
    uint32_t base[kNf4LutEntries];
};

cudaError_t launch_quantize(const float* W, int64_t numel, uint8_t* packed, uint8_t* scale_codes,
                            float* meta, int* nonfinite_flag, const Nf4IndexLut& lut,
                            cudaStream_t stream);

cudaError_t launch_dequantize(const uint8_t* packed, const uint8_t* scale_codes, const float* meta,
                              int64_t numel, uint16_t* out, const Nf4Table& tab, int num_sms,
                              cudaStream_t stream);

// K1 with another codebook of the same blocksize (64): its bucket table, the
// index of a zero block, and the scales as fp32 (QLORA_SCALES_FP32: c_b per
// block, meta unused) or an 8-bit code with one fp32 constant per 256 blocks.
cudaError_t launch_quantize_b64(const float* W, int64_t numel, uint8_t* packed, void* scales,
                                float* meta, int* nonfinite_flag, const Nf4IndexLut& lut,
                                uint32_t zero_index, int scale_fmt, cudaStream_t stream);

// K1 over several weights (fp32, or bf16 when bf16 is set): up to
// kMaxQuantizeJobs weights' whole groups per launch, each partial trailing
// group by its own one-CTA launch.
constexpr int kMaxQuantizeJobs = 16;
struct QuantizeJob {
    const void* W;
    int64_t numel;
    uint8_t* packed;
    uint8_t* scale_codes;
    float* meta;
};
cudaError_t launch_quantize_many(const QuantizeJob* jobs, int n, bool bf16, int* nonfinite_flag,
                                 const Nf4IndexLut& lut, cudaStream_t stream);

// K1 on a bf16 weight (the re-quantisation of a merged export).
cudaError_t launch_quantize_bf16(const uint16_t* W, int64_t numel, uint8_t* packed,
                                 uint8_t* scale_codes, float* meta, int* nonfinite_flag,
                                 const Nf4IndexLut& lut, cudaStream_t stream);

// ------------------------------------------------- K1 / K6 format variants
struct FmtTable {
    float code[16];            // codebook (unused entries 0)
    float mid[15];             // fp32 midpoints; +inf past the last code
    uint32_t zero_index;       // index of the code nearest 0 (zero blocks, padding)
    uint32_t use_lut;          // the finite midpoints are more than 1/16 apart: the
    Nf4IndexLut lut;           // bucket table gives the code index (else a search)
};
struct FmtArgs {
    int block;                 // power of two, 16..4096
    int log2_block;
    int scale_fmt;             // a qlora_scale_format: fp32 absmax per block, or an 8-bit
                               // code (E4M3, E5M2, linear) + an fp32 constant per 256 blocks
};
cudaError_t launch_quantize_fmt(const float* W, int64_t numel, const FmtArgs& f, uint8_t* packed,
                                void* scales, float* meta, int* nonfinite_flag,
                                const FmtTable& tab, cudaStream_t stream);
cudaError_t launch_dequantize_fmt(const uint8_t* packed, const void* scales, const float* meta,
                                  int64_t numel, const FmtArgs& f, uint16_t* out,
                                  const FmtTable& tab, int num_sms, cudaStream_t stream);

// -------------------------------------------- 8-bit optimiser state (AdamW)
struct Adam8Args {
    float* p;                  // fp32 parameters, updated in place
    const float* g;            // fp32 gradients
    int8_t* m_codes;           // first moment, linear code of m
    float* m_absmax;
    uint8_t* v_codes;          // second moment, linear code of sqrt(v)
    float* v_absmax;
    uint16_t* p_bf16;          // optional bf16 copy of the updated p
    int64_t n;
    float lr, beta1, beta2, eps;
    float decay;               // fp32(1 - lr wd)
    float one_m_beta1, one_m_beta2;
    float bc1, bc2;            // fp32(1 - beta^t)
};
cudaError_t launch_adamw8(const Adam8Args& a, int num_sms, cudaStream_t stream);

// ---------------------------------------------------------------- K7 merge
struct MergeArgs {
    const uint32_t* packed;      // N*K/8 words of packed indices
    const uint8_t* scale_codes;
    const float* meta;
    const uint16_t* A;           // bf16 [r, K]
    const uint16_t* B;           // bf16 [N, r]
    uint16_t* out;               // bf16 [N, K]
    int64_t N, K;                // K % 64 == 0
    int r;                       // 8 <= r <= 128, r % 8 == 0
    int rp;                      // r rounded up to 16 (set by launch_merge)
    float gamma;
    int64_t tiles;               // CTA units of 16 rows x 512 columns (set by launch_merge)
};
int merge_smem_bytes(int r);
// Up to kMaxMergeJobs weights merged by one launch: their CTA units form one
// sequence (job 0's first), dealt to the CTAs in equal runs.
constexpr int kMaxMergeJobs = 16;
cudaError_t launch_merge(const MergeArgs* jobs, int n, const Nf4Table& tab, int num_sms,
                         cudaStream_t stream);

// ---------------------------------------------------------------- K2 / K3
struct GemmArgs {
    const uint8_t* scale_codes;
    const float* meta;
    uint16_t* D;          // output, row-major [M x d_cols]
    int64_t M;            // tokens
    int64_t Nw;           // rows of W (out features)
    int64_t d_cols;       // Nw (forward) or Kw (input gradient)
    int64_t nkb;          // NF4 blocks per row of W = Kw / 64
    int main_steps;       // 64-wide contraction steps over W
    int tail_steps;       // ceil(r / 64) LoRA steps
    int r;
    int m_tiles;
    // Tile schedule: the output, taken as m_tiles rows of cols_lin columns
    // (d_cols rounded up) in one linear order, is dealt to the CTA pairs in
    // runs of col_budget columns; a pair walks its run as tiles at most 256
    // columns wide, each ending at a 512-token row boundary or its run's end.
    int64_t cols_lin;
    int64_t col_budget;
    int* err;             // device error word
    unsigned long long wait_ns;   // bound of every operational mbarrier wait (teardown
                                  // drains keep kWaitLimitNs)
    Nf4Table tab;
};

// after_lora: the kernel directly before it in `stream` is the LoRA kernel
// that writes (gamma T | gamma U); the GEMM is then launched as its
// programmatic dependent and waits for it only before the LoRA steps.
// out: 2-D map of D [M x d_cols] bf16, box {16 columns, 32 rows}, no swizzle.
cudaError_t launch_gemm(bool trans, const CUtensorMap& act, const CUtensorMap& packed,
                        const CUtensorMap& lora_a, const CUtensorMap& lora_b, const CUtensorMap& out,
                        const GemmArgs& args, bool after_lora, cudaStream_t stream);
int gemm_tile_m();   // tokens per output tile (a CTA pair)
int gemm_tile_n();   // largest output tile width
int gemm_half_n();   // W~ rows each CTA of the pair expands for the widest tile
// Output-tile width granularity: a multiple of 32 columns for the forward
// (one TMEM load), of 128 for dX (each CTA's half holds whole NF4 blocks).
int gemm_col_granule(bool trans);

// -------------------------------------------------------------- K4 (LoRA)
// out = alpha * sum_c P(i,c) * Q(c,j) over i < I, j < J (J <= 128, J % 8 == 0),
// the contraction split over `splits` CTAs of one cluster (<= 8) and reduced
// in distributed shared memory by the first CTA, which also writes:
//   out       fp32 [I x J] (or [J x I] if transpose), += when accumulate;
//   out_bf16  bf16 of (alpha*sum*beta), [I x ldb], columns J..ldb-1 zero;
//   cvt_dst   bf16 of cvt_src*cvt_scale for the same rows ([I x J] fp32 in,
//             [I x ldb] out, zero padded) -- an optional side copy.
//   p_kmajor: P stored [I][C] (ld = ldp) else [C][I].
//   q_kmajor: Q stored [J][C] (ld = ldq) else [C][J].
//   err_zero: if set, one thread stores 0 there (clears the call's error word).
constexpr int kMaxSkinnySplits = 8;
struct SkinnyArgs {
    const uint16_t* P;
    const uint16_t* Q;
    int64_t I, J, C;
    int64_t ldp, ldq;
    int splits;
    int64_t c_per_split;  // multiple of 64
    float alpha;
    float* out;
    int transpose;
    int accumulate;
    uint16_t* out_bf16;
    int64_t ldb;
    float beta;
    const float* cvt_src;
    uint16_t* cvt_dst;
    float cvt_scale;
    int* err_zero;
    int trigger_dependents;   // let the next kernel (a programmatic dependent) start at once
    int programmatic;         // launch as the previous kernel's programmatic dependent; the
                              // kernel never waits for that grid, so its inputs must come
                              // from earlier work
};
cudaError_t launch_skinny(bool p_kmajor, bool q_kmajor, const SkinnyArgs& a, cudaStream_t stream);

// --------------------------------------------------------------------- K5
struct GemvArgs {
    const uint8_t* packed;
    const uint8_t* scale_codes;
    const float* meta;
    const uint16_t* X;    // [M x K] bf16, M <= 16
    const uint16_t* A;    // [r x K] bf16 (LoRA down-projection)
    int r;
    float* part;          // [splits][M][N] fp32 partial products
    float* Tpart;         // [splits][t_ctas][M][r] fp32 partial T = X A^T
    int* counters;        // [splits] work-unit counters, zero on entry
    int* err;             // device error word
    int64_t M, N, K;
    int splits;
    int64_t k_per_split;  // multiple of 256 (or K)
    int tile_chunks;      // D: 256-wide chunks per weight tile (1, 2, 4, 8); tiles are 256 / D rows
    int t_ctas;           // CTAs of each slice that compute a share of T
    Nf4Table tab;
};
// Pipeline stages the GEMV kernel runs with for M tokens over a kslab-wide
// contraction slice (0: its activations do not fit in shared memory).
int gemv_stages(int64_t M, int64_t kslab);
// tm_packed: 3-D view of the packed weight {128 bytes, N rows, K/256 chunks},
// strides {K/2, 128} bytes, box {128, 256 / D rows, D chunks}, 128-byte
// swizzle, D = a.tile_chunks.
cudaError_t launch_gemv(const CUtensorMap& tm_packed, const GemvArgs& a, int num_sms,
                        cudaStream_t stream);

// T = sum of the t_parts partials (also to T_save);
// Y = bf16(sum_s part[s] + gamma T B^T)
struct GemvFinalizeArgs {
    const float* part;
    const float* Tpart;
    int splits;           // partial outputs
    int t_parts;          // partial T
    const uint16_t* B;    // [N x r]
    int r;
    float gamma;
    float* T_save;        // nullable
    uint16_t* Y;
    int64_t M, N;
};
cudaError_t launch_gemv_finalize(const GemvFinalizeArgs& a, cudaStream_t stream);

// ----------------------------------------------- chained SwiGLU MLP (f3)
// n = elements, a multiple of 8; H = bf16(silu(G) U); (G, U) <- (dG, dU);
// C = bf16(A + B); dst = (accumulate ? dst : 0) | *a | *b | *c.
cudaError_t launch_swiglu_forward(const uint16_t* G, const uint16_t* U, uint16_t* H, int64_t n,
                                  int num_sms, cudaStream_t s);
cudaError_t launch_swiglu_backward(uint16_t* G, uint16_t* U, const uint16_t* dH, int64_t n,
                                   int num_sms, cudaStream_t s);
cudaError_t launch_add_bf16(const uint16_t* A, const uint16_t* B, uint16_t* C, int64_t n,
                            int num_sms, cudaStream_t s);
cudaError_t launch_or_words(int* dst, const int* a, const int* b, const int* c, bool accumulate,
                            cudaStream_t s);

}  // namespace qnf4
