/*
 * qlora_nf4.h -- C ABI of libqlora_nf4.so: the frozen-NF4 linear layer with a
 * bf16 LoRA adapter on one NVIDIA B200 (sm_100a).
 *
 * Method: "QLoRA, explained" (pofe.ai).  Storage follows its section "The
 * math: what is stored and what is computed" (sub-sections "Blockwise absmax
 * quantisation", "NormalFloat 4 (NF4)", "Double quantisation"); compute
 * follows "The forward pass and gradients" and "The algorithm, step by step".
 *
 * Conventions for every entry point
 *   - Every pointer argument named d_* or documented as "device" is device
 *     memory owned by the caller; the library never allocates, frees or keeps
 *     a pointer after the call returns.  Scratch space for the linear layer
 *     is a caller-provided workspace whose size
 *     qlora_linear_workspace_size() reports.
 *   - bf16 tensors are passed as uint16_t* holding IEEE bfloat16 bit patterns
 *     (the layout of __nv_bfloat16 and torch.bfloat16).
 *   - All matrices are row-major and densely packed (row stride = columns).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All device
 *     work is enqueued asynchronously on it; a call returns once its kernels
 *     are launched.  Outputs are valid after the stream reaches that point.
 *   - The return value is a qlora_status.  Argument errors are detected on
 *     the host before anything is launched and leave every output untouched.
 *     QLORA_ERR_CUDA reports a failed launch (cudaGetLastError()).
 *   - The only global state is the scratch array of
 *     qlora_linear_forward_noalloc and the wait limit that
 *     qlora_set_gemm_wait_limit_us sets.  Calls on different streams with
 *     disjoint outputs and workspaces may run concurrently.
 *   - Within a call, some kernels are launched as programmatic dependents of
 *     the kernel before them (they may start before it finishes and wait for
 *     it, if at all, only where they read its output).  The call's first
 *     kernel is an ordinary launch, so everything earlier on `stream` is
 *     complete before any of the call's kernels starts.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

struct CUstream_st;                       /* == cudaStream_t's pointee */
typedef struct CUstream_st* qlora_stream_t;

typedef enum {
    QLORA_OK = 0,
    QLORA_ERR_NULL = 1,         /* a required pointer is NULL               */
    QLORA_ERR_SHAPE = 2,        /* a size is negative or inconsistent       */
    QLORA_ERR_ALIGN = 3,        /* a pointer is not 16-byte aligned         */
    QLORA_ERR_UNSUPPORTED = 4,  /* a size outside what the kernels handle   */
    QLORA_ERR_NONFINITE = 5,    /* non-finite weight seen by qlora_quantize */
    QLORA_ERR_CUDA = 6,         /* a CUDA runtime call or launch failed     */
    QLORA_ERR_WORKSPACE = 7     /* workspace pointer NULL or too small      */
} qlora_status;

/* Fixed format parameters ("Blockwise absmax quantisation": blocks of 64;
 * "Double quantisation": one fp32 constant per 256 block scales). */
#define QLORA_BLOCK 64
#define QLORA_GROUP 256
/* Largest LoRA rank the linear layer accepts; the rank must be a multiple of 8. */
#define QLORA_MAX_RANK 128
/* Token counts up to this (with K % 256 == 0) go to the dequant-GEMV kernel. */
#define QLORA_GEMV_MAX_TOKENS 16

/*
 * A stored NF4 tensor: a non-owning view of three device buffers.
 *
 * The logical tensor is W[rows][cols] (fp32 before quantisation), flattened
 * in row-major order and cut into blocks of 64 consecutive elements
 * (nblocks = ceil(rows*cols / 64)); blocks are grouped 256 at a time
 * (ngroups = ceil(nblocks / 256)).
 *   packed      : nblocks*32 bytes.  Byte j holds element 2j in its low
 *                 nibble and element 2j+1 in its high nibble; each nibble is
 *                 the index (0..15) of the element's nearest NF4 code.  The
 *                 padding of a final partial block holds index 7, the code 0.
 *   scale_codes : nblocks bytes.  The FP8 E4M3 (e4m3fn) code of block b's
 *                 absmax c_b divided by its group's meta scale.
 *   meta_scale  : ngroups fp32.  The group's largest c_b divided by 448.
 * The dequantised weight is  w~ = bf16_rne( fp32( q[idx] * c~_b ) )  with
 * c~_b = fp32( e4m3(scale_code_b) * meta_scale_g ).
 */
typedef struct {
    uint8_t* packed;
    uint8_t* scale_codes;
    float* meta_scale;
    int64_t rows;   /* N: output features of the linear layer */
    int64_t cols;   /* K: input features                        */
} qlora_nf4_tensor;

/* Human-readable name of a qlora_status value (static string). */
QLORA_API const char* qlora_status_string(int status);

/*
 * nf4_build_codebook -- the 16 NF4 codes and the 15 decision midpoints.
 * "QLoRA, explained", "NormalFloat 4 (NF4)": codes at averages of adjacent
 * standard-normal quantiles, halves of 8 and 9 levels sharing an exact zero,
 * renormalised to [-1, 1].  Host only, deterministic, no CUDA call.
 *   codes     (host, 16 floats, written): ascending; codes[0] = -1,
 *             codes[7] = 0, codes[15] = 1.
 *   midpoints (host, 15 floats, written): midpoints[i] is the exact average
 *             of codes[i] and codes[i+1] rounded to nearest fp32.  An element
 *             x maps to the number of midpoints strictly below it (a value
 *             equal to a midpoint takes the lower code).
 * Errors: QLORA_ERR_NULL if either pointer is NULL.
 */
QLORA_API int nf4_build_codebook(float codes[16], float midpoints[15]);

/*
 * qlora_quantized_sizes -- byte sizes of the three buffers of a stored
 * rows x cols tensor (layout above).  Host only.
 * Errors: QLORA_ERR_NULL (an output pointer NULL), QLORA_ERR_SHAPE (a
 * negative size or rows*cols overflowing int64).
 */
QLORA_API int qlora_quantized_sizes(int64_t rows, int64_t cols, size_t* packed_bytes,
                          size_t* codes_bytes, size_t* meta_bytes);

/*
 * qlora_quantize -- blockwise absmax NF4 quantisation plus double
 * quantisation of the scales ("The algorithm, step by step": split into
 * blocks of 64, absmax, nearest NF4 code of w / c_b, FP8 scales in groups of
 * 256 with fp32 constants).
 *   W     (device, fp32, rows*cols, read): the weight, row-major.
 *   out   (host struct, read): rows, cols and the three device buffers to
 *         write, sized by qlora_quantized_sizes.  All of them are written.
 *   d_nonfinite_flag (device int, nullable): the caller's request for the
 *         non-finite check (a NaN or infinity leaves its block's absmax scale
 *         meaningless; "Failure modes", "Loss spikes and NaNs", asks for NaNs
 *         to be detected).  If given, the call zeroes it, enqueues
 *         the kernels (which set it when any element of W is NaN or +-Inf),
 *         then synchronises `stream` and returns QLORA_ERR_NONFINITE if it
 *         was set; the outputs are then unspecified.  If NULL, nothing is
 *         checked and the call returns as soon as the kernels are enqueued.
 *         rows * cols = 0 launches nothing and leaves the flag untouched.
 * Errors: QLORA_ERR_NULL, QLORA_ERR_SHAPE, QLORA_ERR_ALIGN (W, packed not
 * 16-byte aligned; scale_codes, meta_scale not 4-byte aligned),
 * QLORA_ERR_NONFINITE (only when d_nonfinite_flag is given), QLORA_ERR_CUDA.
 */
QLORA_API int qlora_quantize(const float* W, const qlora_nf4_tensor* out,
                   int* d_nonfinite_flag, qlora_stream_t stream);

/*
 * qlora_dequantize -- dDQ of a whole stored tensor to bf16 ("The forward
 * pass and gradients": dequantise the FP8 scales with the fp32 constants,
 * then the NF4 indices with those scales, producing bf16 W~).
 *   w     (host struct, read): the stored tensor.
 *   W_out (device, bf16 bits, rows*cols, written): W~ row-major; bit-exact
 *         to bf16_rne(fp32(q[idx] * c~_b)).
 * Errors: QLORA_ERR_NULL, QLORA_ERR_SHAPE, QLORA_ERR_ALIGN (W_out and packed
 * 16-byte aligned; scale_codes, meta_scale 4-byte aligned), QLORA_ERR_CUDA.
 */
QLORA_API int qlora_dequantize(const qlora_nf4_tensor* w, uint16_t* W_out,
                     qlora_stream_t stream);

/*
 * Format variants ("QLoRA, explained", "A toy run: how much does NF4 lose
 * ..."): the same blockwise absmax quantisation with another codebook (the
 * page compares E2M1 FP4 and a symmetric 15-level INT4 grid with NF4) and
 * blocksize (16 and 4096 next to 64), with the block scales either kept as
 * fp32 or double-quantised as in "Double quantisation" ("8-bit floats", no
 * format named: E4M3, E5M2, or a linear 8-bit code).
 * The stored layout generalises the NF4 one: nblocks = ceil(numel / block);
 *   packed : nblocks * block / 2 bytes, two indices per byte, the even
 *            element in the low nibble; a final partial block is padded with
 *            the index of the code nearest 0.
 *   scales : QLORA_SCALES_FP32 -- nblocks fp32, the block absmax c_b;
 *            otherwise nblocks bytes of 8-bit codes of c_b / c2, with meta =
 *            ceil(nblocks / 256) fp32 constants c2 = fp32(max c_b / TOP):
 *            QLORA_SCALES_E4M3 -- FP8 E4M3 (as NF4), TOP = 448;
 *            QLORA_SCALES_E5M2 -- FP8 E5M2, TOP = 57344;
 *            QLORA_SCALES_U8   -- linear, code = rint(fp32(c_b / c2)) (ties to
 *                                 even), TOP = 255.
 *            The FP8 codes round to nearest even and saturate at TOP.
 * Index of a weight: the number of midpoints strictly below fp32(w / c_b),
 * midpoint i being the exact average of codes i and i+1 rounded to fp32; a
 * zero block takes the index of the code nearest 0.  Dequantisation:
 * w~ = bf16_rne(fp32(codes[idx] * c~_b)), c~_b = c_b or fp32(decode(code) * c2).
 * With the NF4 codebook, block 64 and E4M3 scales the layout and every byte
 * equal those of qlora_quantize.
 */
typedef enum {
    QLORA_SCALES_FP32 = 0,
    QLORA_SCALES_E4M3 = 1,
    QLORA_SCALES_E5M2 = 2,
    QLORA_SCALES_U8 = 3
} qlora_scale_format;

typedef struct {
    int32_t block;       /* elements per block: a power of two, 16 ... 4096   */
    int32_t ncodes;      /* 2 ... 16                                          */
    float codes[16];     /* strictly ascending, finite; entries past ncodes   */
                         /* are ignored                                       */
    int32_t scales;      /* a qlora_scale_format                              */
} qlora_format;

/*
 * qlora_format_sizes -- byte sizes of the packed, scale and meta buffers of
 * numel weights in format f (meta is 0 bytes for fp32 scales).  Host only.
 * Errors: QLORA_ERR_NULL, QLORA_ERR_SHAPE (numel < 0), QLORA_ERR_UNSUPPORTED
 * (a format field out of range, codes not strictly ascending or not finite).
 */
QLORA_API int qlora_format_sizes(int64_t numel, const qlora_format* f, size_t* packed_bytes,
                                 size_t* scale_bytes, size_t* meta_bytes);

/*
 * qlora_quantize_fmt -- quantise numel fp32 weights (device, read) in format
 * f (host struct, read) into packed, scales and meta (device, written, sized
 * by qlora_format_sizes; meta may be NULL for fp32 scales).
 * d_nonfinite_flag as in qlora_quantize (given: the call synchronises the
 * stream and reports QLORA_ERR_NONFINITE).  numel = 0 launches nothing.
 * Errors: QLORA_ERR_NULL, QLORA_ERR_SHAPE, QLORA_ERR_UNSUPPORTED,
 * QLORA_ERR_ALIGN (W and packed 16-byte aligned; scales and meta 4-byte),
 * QLORA_ERR_NONFINITE, QLORA_ERR_CUDA.
 */
QLORA_API int qlora_quantize_fmt(const float* W, int64_t numel, const qlora_format* f,
                                 uint8_t* packed, void* scales, float* meta,
                                 int* d_nonfinite_flag, qlora_stream_t stream);

/*
 * qlora_dequantize_fmt -- w~ of numel weights stored in format f, written as
 * bf16 bits to out (device, numel, 16-byte aligned).  Other buffers as
 * qlora_quantize_fmt (read).  numel = 0 launches nothing.
 * Errors as qlora_quantize_fmt.
 */
QLORA_API int qlora_dequantize_fmt(const uint8_t* packed, const void* scales, const float* meta,
                                   int64_t numel, const qlora_format* f, uint16_t* out,
                                   qlora_stream_t stream);

/*
 * AdamW over an adapter matrix with 8-bit blockwise state ("QLoRA,
 * explained", "The algorithm, step by step": AdamW over A and B only, 32- or
 * 8-bit state; "Hyperparameters that matter": the 8-bit variant quantises
 * Adam's moments blockwise).  The state of n parameters: blocks of 64, an
 * fp32 absmax per block for each moment; m as int8 codes
 * rint(fp32(m / c) * 127), v through its square root as uint8 codes
 * rint(fp32(sqrt(v) / c) * 255) (quotient rounded to fp32, then the product
 * rounded to the nearest integer, ties to even).  Zero codes and absmax are
 * the initial (zero) state.
 */
typedef struct {
    float lr;
    float beta1;          /* 0 <= beta1 < 1 */
    float beta2;          /* 0 <= beta2 < 1 */
    float eps;
    float weight_decay;   /* decoupled: p *= 1 - lr weight_decay */
    int64_t step;         /* t >= 1, for the bias corrections 1 - beta^t */
} qlora_adamw_config;

/* Byte sizes of one moment's codes (n) and absmax array (4 ceil(n/64)). */
QLORA_API int qlora_adamw8_state_sizes(int64_t n, size_t* code_bytes, size_t* absmax_bytes);

/*
 * qlora_adamw8_step -- one AdamW step: decode the state, update in fp32
 * (p *= fp32(1 - lr wd); m = b1 m + fp32(1 - b1) g; v = b2 v + (fp32(1 - b2) g) g;
 * p -= (lr (m / fp32(1 - b1^t))) / (sqrt(v / fp32(1 - b2^t)) + eps), each
 * operation rounded on its own), re-encode the state.
 *   p (device, fp32, n, read and written); g (device, fp32, n, read);
 *   m_codes, m_absmax, v_codes, v_absmax (device, read and written);
 *   cfg (host, read); p_bf16 (device, bf16 bits, n, nullable, written): the
 *   updated p rounded to bf16, for the layer's A or B.
 * n = 0 launches nothing.
 * Non-finite values are not detected: a NaN or infinite gradient leaves p and
 * the state of its block unspecified (the block maximum that sets the new
 * absmax skips NaN).  Check gradients before the step if they may overflow.
 * Errors: QLORA_ERR_NULL, QLORA_ERR_SHAPE, QLORA_ERR_UNSUPPORTED (a
 * hyperparameter out of range: beta1 or beta2 outside [0, 1), step < 1,
 * eps <= 0, lr < 0, weight_decay < 0, lr * weight_decay >= 1, or any of them
 * not finite), QLORA_ERR_ALIGN (p, g 16-byte aligned; codes and absmax 4-byte;
 * p_bf16 8-byte), QLORA_ERR_CUDA.
 */
QLORA_API int qlora_adamw8_step(float* p, const float* g, int64_t n, int8_t* m_codes,
                                float* m_absmax, uint8_t* v_codes, float* v_absmax,
                                const qlora_adamw_config* cfg, uint16_t* p_bf16,
                                qlora_stream_t stream);

/*
 * qlora_merge -- the fine-tuned weight for bf16 export,
 *     W_out = bf16_rne( W~ + scale * B A ).
 * "QLoRA, explained", "The forward pass and gradients": the model that was
 * trained is W~ + gamma B A, the quantised base plus the adapter; the same
 * page's "Failure modes" ("Quality loss at merge time") gives dequantising W~
 * to bf16 and adding the adapter as the merge that keeps it.  W~ is rebuilt
 * bit for bit as qlora_dequantize does; the sum is formed in fp32 (B A
 * accumulated in fp32 from the exact bf16 products, then one fused
 * multiply-add with W~) and rounded to bf16 once.
 *   w     (host struct, read): the stored weight, rows = N, cols = K
 *   A     (device, bf16, r x K, read): LoRA down-projection
 *   B     (device, bf16, N x r, read): LoRA up-projection
 *   r     LoRA rank: 8 <= r <= 128, r % 8 == 0
 *   scale gamma = alpha / r
 *   W_out (device, bf16 bits, N x K, written, row-major); must not overlap
 *         the inputs.  Each element is within one bf16 rounding of the exact
 *         value, plus fp32 accumulation error (at most (2r+4) 2^-24 of
 *         |w~| + |gamma| sum_j |B_nj A_jk|).
 * N = 0 or K = 0 launches nothing; every buffer (the stored tensor's, A, B,
 * W_out) may then be NULL.
 * Shape rules: K % 64 == 0 (every NF4 block lies inside one row); N and K
 * below 2^31.
 * Errors: QLORA_ERR_NULL, QLORA_ERR_SHAPE, QLORA_ERR_UNSUPPORTED (K or r),
 * QLORA_ERR_ALIGN (A, B, W_out and packed 16-byte aligned; scale_codes,
 * meta_scale 4-byte), QLORA_ERR_CUDA.
 */
QLORA_API int qlora_merge(const qlora_nf4_tensor* w, const uint16_t* A, const uint16_t* B,
                          int r, float scale, uint16_t* W_out, qlora_stream_t stream);

/*
 * qlora_merge_many -- qlora_merge of several weights, e.g. every adapted
 * linear of a model at export, with up to 16 of them per kernel launch: a
 * launch deals the weights' units of work to the GPU as one sequence, so
 * small weights do not each pay a launch's ramp and tail.  Each job's result
 * is bit for bit what qlora_merge gives for it.
 *   jobs  (host array of n qlora_merge_job, read): one merge each, with the
 *         arguments and rules of qlora_merge; the jobs' W_out must not
 *         overlap one another or any job's inputs.  Ranks may differ.
 *   n     >= 0 (0 launches nothing).
 * Every job is checked before anything is launched; the first failing job's
 * status is returned and nothing runs.
 * Errors: those of qlora_merge; QLORA_ERR_NULL (jobs NULL with n > 0),
 * QLORA_ERR_SHAPE (n < 0).
 */
typedef struct {
    const qlora_nf4_tensor* w;   /* host struct, read */
    const uint16_t* A;           /* device, bf16, r x K */
    const uint16_t* B;           /* device, bf16, N x r */
    int r;
    float scale;
    uint16_t* W_out;             /* device, bf16, N x K */
} qlora_merge_job;

QLORA_API int qlora_merge_many(const qlora_merge_job* jobs, int n, qlora_stream_t stream);

/*
 * qlora_quantize_many -- qlora_quantize (or, with input_bf16, qlora_quantize_bf16)
 * of several weights, e.g. every linear of a model at load time or every
 * merged weight at export: the whole 256-block groups of up to 16 weights
 * share one kernel launch, so small weights do not each pay a launch's ramp
 * and tail; a weight's partial last group (numel % 16384 != 0) takes one more
 * small launch.  Each job's stored bytes are bit for bit what qlora_quantize
 * gives for it.
 *   jobs  (host array of n qlora_quantize_job, read): W (device, fp32 or bf16
 *         bits, rows*cols, read, 16-byte aligned) and out (host struct whose
 *         buffers are written); the outputs must not overlap one another or
 *         any input.  Empty weights (rows or cols 0) are skipped: their W
 *         and out's buffers may be NULL.
 *   n     >= 0 (0 launches nothing).
 *   input_bf16  0: every W is fp32; otherwise every W is bf16.
 *   d_nonfinite_flag (device int, nullable): as qlora_quantize, for all jobs
 *         together: cleared first, and with a flag the call synchronises the
 *         stream and returns QLORA_ERR_NONFINITE if any job held a NaN or an
 *         infinity.
 * Every job is checked before anything is launched; the first failing job's
 * status is returned and nothing runs.
 * Errors: QLORA_ERR_NULL, QLORA_ERR_SHAPE (n < 0, or a job's shape),
 * QLORA_ERR_ALIGN, QLORA_ERR_NONFINITE, QLORA_ERR_CUDA.
 */
typedef struct {
    const void* W;                 /* device, fp32 or bf16 (see input_bf16) */
    const qlora_nf4_tensor* out;   /* host struct, its buffers written */
} qlora_quantize_job;

QLORA_API int qlora_quantize_many(const qlora_quantize_job* jobs, int n, int input_bf16,
                                  int* d_nonfinite_flag, qlora_stream_t stream);

/*
 * qlora_quantize_bf16 -- qlora_quantize of a bf16 weight (each value widened
 * exactly to fp32 first), the re-quantisation of a merged weight for a 4-bit
 * deployment ("QLoRA" (finetunellm.com), "What it costs you": merging into
 * 4-bit weights means merging in bf16 and quantising again, a second
 * rounding).  Same result as qlora_quantize given the fp32 values of W.
 *   W (device, bf16 bits, rows*cols, read); other arguments as qlora_quantize,
 *   d_nonfinite_flag included (given: synchronise and report).
 * Errors: as qlora_quantize (W 16-byte aligned).
 */
QLORA_API int qlora_quantize_bf16(const uint16_t* W, const qlora_nf4_tensor* out,
                                  int* d_nonfinite_flag, qlora_stream_t stream);

/*
 * qlora_linear_workspace_size -- bytes of device workspace that
 * qlora_linear_forward and qlora_linear_backward need for these sizes.
 * M tokens, N = w.rows, K = w.cols, r the LoRA rank.  Host only.
 * Errors: QLORA_ERR_NULL, QLORA_ERR_SHAPE, QLORA_ERR_UNSUPPORTED (see the
 * shape rules of qlora_linear_forward).
 */
QLORA_API int qlora_linear_workspace_size(int64_t M, int64_t N, int64_t K, int r,
                                size_t* bytes);

/*
 * qlora_linear_forward -- Y = X W~^T + scale * (X A^T) B^T
 * ("The forward pass and gradients"; "The algorithm, step by step", forward).
 * W~ exists only tile by tile inside the kernels; it is never written out.
 *   X      (device, bf16, M x K, read)
 *   M      tokens, >= 0 (M = 0 launches nothing; X and Y may then be NULL)
 *   w      (host struct, read): the stored weight, rows = N, cols = K
 *   A      (device, bf16, r x K, read): LoRA down-projection
 *   B      (device, bf16, N x r, read): LoRA up-projection
 *   r      LoRA rank: 8 <= r <= 128, r % 8 == 0
 *   scale  gamma = alpha / r
 *   Y      (device, bf16, M x N, written)
 *   T_save (device, fp32, M x r, nullable, written): X A^T, for the backward
 *   ws, ws_bytes (device workspace, >= qlora_linear_workspace_size bytes,
 *          256-byte aligned); contents on entry are ignored.  After the
 *          call its first 4 bytes hold the kernels' error word (0 = none;
 *          bit 0 = a bounded wait inside a kernel expired; bit 1 = the
 *          GEMV's shared-memory plan did not fit; bit 2 = a GEMM tile
 *          schedule broke its width rules; with any bit set the outputs
 *          are unspecified).
 *   M <= 16 with K % 256 == 0 runs the bandwidth-bound dequant-GEMV kernel,
 *   every other shape the tensor-core dequant-GEMM; both multiply the same
 *   W~ (each weight bf16_rne(fp32(q[idx] * c~_b)), as qlora_dequantize
 *   writes it) in fp32 accumulation, so they differ only in the order of
 *   their fp32 additions.
 * Shape rules: K % 64 == 0, N % 8 == 0, K >= 64, N >= 8.
 * Errors: QLORA_ERR_NULL, QLORA_ERR_SHAPE, QLORA_ERR_ALIGN (every tensor
 * 16-byte aligned, except scale_codes and meta_scale: 4-byte),
 * QLORA_ERR_UNSUPPORTED, QLORA_ERR_WORKSPACE, QLORA_ERR_CUDA.
 */
QLORA_API int qlora_linear_forward(const uint16_t* X, int64_t M, const qlora_nf4_tensor* w,
                         const uint16_t* A, const uint16_t* B, int r, float scale,
                         uint16_t* Y, float* T_save, void* ws, size_t ws_bytes,
                         qlora_stream_t stream);

/*
 * qlora_linear_backward -- gradients of the adapted layer with W~ frozen
 * ("The forward pass and gradients": the input gradient dequantises the block
 * a second time; the adapter gradients are LoRA's with W~ in place of W0; no
 * gradient is formed for the stored NF4 weight).
 *   dX = dY W~ + scale * (dY B) A          (bf16, M x K)
 *   dA = scale * (dY B)^T X                (fp32, r x K)
 *   dB = scale * dY^T (X A^T)              (fp32, N x r)
 *   dY      (device, bf16, M x N, read)
 *   X       (device, bf16, M x K, read)
 *   T_saved (device, fp32, M x r, nullable): X A^T from the forward; NULL
 *           recomputes it
 *   dX      (device, bf16, M x K, nullable = not computed, written)
 *   dA, dB  (device, fp32, written; accumulate != 0 adds to their contents)
 *   M = 0 writes zero gradients (or leaves them unchanged when accumulating);
 *   dY and X may then be NULL.
 *   other arguments as in qlora_linear_forward.
 * The adapter-gradient kernels (dA, dB) are launched as programmatic
 * dependents of the dX GEMM and run beside it on the SMs it leaves idle;
 * they read only dY, X and the first kernel's output.
 * Errors as qlora_linear_forward.
 */
QLORA_API int qlora_linear_backward(const uint16_t* dY, const uint16_t* X, int64_t M,
                          const qlora_nf4_tensor* w, const uint16_t* A,
                          const uint16_t* B, int r, float scale,
                          const float* T_saved, uint16_t* dX, float* dA,
                          float* dB, int accumulate, void* ws, size_t ws_bytes,
                          qlora_stream_t stream);

/*
 * Layer chaining with gradient checkpointing: the SwiGLU MLP of adapted NF4
 * linears, y = down(silu(gate(x)) * up(x)) ("QLoRA, explained", "The
 * algorithm, step by step": the training step runs with gradient
 * checkpointing enabled; "Compute and memory cost": checkpointing is
 * effectively mandatory, and the recomputed forward dequantises every block
 * a third time per step).  The pages print no block structure; this is the
 * MLP of the Llama-shaped models.  gate and up are F x D stored weights, down
 * is D x F, each with its own LoRA adapter of rank r, all with the same
 * scale gamma.  silu(z) = z / (1 + exp(-z)).
 */
typedef struct {
    qlora_nf4_tensor gate, up, down;   /* F x D, F x D, D x F               */
    const uint16_t* A_gate;            /* bf16 r x D (device, read)         */
    const uint16_t* B_gate;            /* bf16 F x r                        */
    const uint16_t* A_up;              /* bf16 r x D                        */
    const uint16_t* B_up;              /* bf16 F x r                        */
    const uint16_t* A_down;            /* bf16 r x F                        */
    const uint16_t* B_down;            /* bf16 D x r                        */
    int r;                             /* 8 <= r <= 128, r % 8 == 0         */
} qlora_mlp;

/* Adapter gradients of the MLP (device fp32, written or accumulated):
 * dA_* r x (input features), dB_* (output features) x r. */
typedef struct {
    float* dA_gate;
    float* dB_gate;
    float* dA_up;
    float* dB_up;
    float* dA_down;
    float* dB_down;
} qlora_mlp_grads;

/*
 * qlora_mlp_workspace_size -- bytes of device workspace qlora_mlp_forward and
 * qlora_mlp_backward need for M tokens (the intermediate activations gate(x),
 * up(x), h and dh in bf16, M x F each, plus each linear call's own
 * workspace).  Host only.
 * Errors: QLORA_ERR_NULL, QLORA_ERR_SHAPE (negative M, or the three weights'
 * shapes not F x D, F x D, D x F), QLORA_ERR_ALIGN, QLORA_ERR_UNSUPPORTED (a
 * linear's shape rules, D and F both taking the roles of N and K).
 */
QLORA_API int qlora_mlp_workspace_size(int64_t M, const qlora_mlp* mlp, size_t* bytes);

/*
 * qlora_mlp_forward -- Y = down(silu(gate(X)) * up(X)), every linear the
 * adapted layer of qlora_linear_forward; gate(x) and up(x) are rounded to
 * bf16, h = bf16(silu(g) * u) in fp32 from them.
 *   X (device, bf16, M x D, read); Y (device, bf16, M x D, written); nothing
 *   else is kept for the backward (checkpointing: it recomputes from X).
 *   ws: >= qlora_mlp_workspace_size bytes, 256-byte aligned; its first 4
 *   bytes then hold the OR of the linear calls' error words (as
 *   qlora_linear_forward documents).
 * M = 0 launches nothing.
 * Errors: those of qlora_mlp_workspace_size and qlora_linear_forward.
 */
QLORA_API int qlora_mlp_forward(const uint16_t* X, int64_t M, const qlora_mlp* mlp, float scale,
                                uint16_t* Y, void* ws, size_t ws_bytes, qlora_stream_t stream);

/*
 * qlora_mlp_backward -- gradients of the MLP with the stored weights frozen,
 * recomputing the forward (the third dequantisation of gate and up):
 *   g = gate(X), u = up(X) (with their X A^T), h = silu(g) * u;
 *   dh, dA_down, dB_down from the down layer's backward at input h;
 *   dg = dh * u * silu'(g), du = dh * silu(g)  (silu' = s (1 + z (1 - s)),
 *   s the logistic sigmoid), rounded to bf16;
 *   dX = (dg's backward through gate) + (du's through up), each bf16, summed
 *   in fp32 and rounded; dA, dB of gate and up.
 *   dY (device, bf16, M x D, read); X (device, bf16, M x D, read);
 *   dX (device, bf16, M x D, written); grads (host struct of device
 *   pointers); accumulate != 0 adds to the adapter gradients.
 *   ws as qlora_mlp_forward (error word: OR over every linear call).
 * M = 0 writes zero adapter gradients (or leaves them when accumulating).
 * Errors: those of qlora_mlp_forward and qlora_linear_backward.
 */
QLORA_API int qlora_mlp_backward(const uint16_t* dY, const uint16_t* X, int64_t M,
                                 const qlora_mlp* mlp, float scale, uint16_t* dX,
                                 const qlora_mlp_grads* grads, int accumulate, void* ws,
                                 size_t ws_bytes, qlora_stream_t stream);

/*
 * qlora_set_gemm_wait_limit_us -- the bound, in microseconds, of every wait of
 * the tensor-core dequant-GEMM (the forward and dX kernel of
 * qlora_linear_forward / _backward) on its pipeline barriers, for GEMMs
 * launched after the call; 0 restores the default of 2 seconds.  A wait that
 * runs out sets bit 0 of the call's error word, and the kernel lets its
 * in-flight copies and MMAs land (those waits keep the default bound),
 * frees its tensor memory and returns; the call's outputs are then
 * unspecified and later calls are unaffected.  Under a limit below the
 * default the waits poll the barriers without blocking and count SM clock
 * cycles (1000 per microsecond of the limit: at most the stated time at
 * clocks of 1 GHz and above), so that even a microsecond is honoured.  This is a failure-detection control: a
 * healthy wait lasts microseconds, and a limit at or below that makes waits
 * run out on purpose.  Process-wide; host only.
 * Errors: QLORA_ERR_UNSUPPORTED (us < 0 or above 10 seconds).
 */
QLORA_API int qlora_set_gemm_wait_limit_us(int64_t us);

/*
 * Profiling variants.  Identical to qlora_linear_forward / _backward, plus
 * optional CUDA events (cudaEvent_t handles created by the caller, either may
 * be NULL) that are recorded on `stream` immediately before and after the
 * launch of the layer's main weight kernel (an event between two kernels
 * makes the second an ordinary launch, so with events the kernels no longer
 * overlap): the tensor-core dequant-GEMM
 * (forward Y, or dX in the backward), or the dequant-GEMV when M <= 16.  They
 * let a caller time that kernel inside a running workload without a profiler.
 * ev itself may be NULL.
 */
typedef struct {
    void* gemm_begin;
    void* gemm_end;
} qlora_events;

QLORA_API int qlora_linear_forward_ex(const uint16_t* X, int64_t M, const qlora_nf4_tensor* w,
                                      const uint16_t* A, const uint16_t* B, int r, float scale,
                                      uint16_t* Y, float* T_save, void* ws, size_t ws_bytes,
                                      qlora_stream_t stream, const qlora_events* ev);

QLORA_API int qlora_linear_backward_ex(const uint16_t* dY, const uint16_t* X, int64_t M,
                                       const qlora_nf4_tensor* w, const uint16_t* A,
                                       const uint16_t* B, int r, float scale,
                                       const float* T_saved, uint16_t* dX, float* dA, float* dB,
                                       int accumulate, void* ws, size_t ws_bytes,
                                       qlora_stream_t stream, const qlora_events* ev);

/*
 * qlora_linear_forward_noalloc -- qlora_linear_forward for callers that cannot
 * allocate device memory.  The paper has no counterpart to this entry point;
 * it exists for callers such as plug-ins inside a host framework that owns
 * every device allocation and exposes no allocator, or deployments that ban
 * device allocation after start-up, which therefore cannot hand over the
 * workspace qlora_linear_forward needs.
 *   Same arguments and result as qlora_linear_forward, without ws/ws_bytes:
 *   the scratch is a fixed 16 MiB device array inside this library, present
 *   on every GPU that loads it until the process exits.  No cudaMalloc,
 *   cudaFree or other allocating routine is called.
 *   The first call on a device looks up that array's device address with
 *   cudaGetSymbolAddress (the device must be current); make that first call
 *   before any stream capture.  Every call on a device shares the one array:
 *   calls that may overlap on the GPU (unordered streams) race on it.
 * Errors: as qlora_linear_forward; QLORA_ERR_WORKSPACE when these sizes need
 * more than the 16 MiB array (qlora_linear_workspace_size reports the need);
 * QLORA_ERR_CUDA if the address lookup fails.
 */
QLORA_API int qlora_linear_forward_noalloc(const uint16_t* X, int64_t M,
                                           const qlora_nf4_tensor* w, const uint16_t* A,
                                           const uint16_t* B, int r, float scale, uint16_t* Y,
                                           float* T_save, qlora_stream_t stream);

/*
 * qlora_linear_forward_noalloc_error_word -- the kernels' error word of the
 * last qlora_linear_forward_noalloc call on the current device (the word
 * qlora_linear_forward leaves in the first 4 bytes of a caller's workspace:
 * 0 = none, bits as documented there).  That word lives in the library's
 * scratch array, which callers cannot address, so this call enqueues a copy
 * of it on `stream` into *h_word (host memory; pinned memory keeps the copy
 * asynchronous).  The value is valid once `stream` has reached the copy;
 * order the copy after the forward call whose word it should report.  Like
 * the forward it allocates nothing; its first call on a device performs the
 * same address look-up.  The paper has no counterpart to this call.
 * Errors: QLORA_ERR_NULL (h_word NULL), QLORA_ERR_CUDA.
 */
QLORA_API int qlora_linear_forward_noalloc_error_word(int* h_word, qlora_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_NF4_H */
