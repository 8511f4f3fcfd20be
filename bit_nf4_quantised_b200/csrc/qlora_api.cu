// Host layer of libqlora_nf4.so: the exported C ABI (include/qlora_nf4.h).
// Argument validation, the workspace plan, TMA descriptors, the NF4 codebook
// construction, and the launch sequence of each entry point.  No device
// memory is allocated here; every buffer is the caller's.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <limits>
#include <atomic>
#include <mutex>
#include <vector>

#include "kernels.cuh"

using namespace qnf4;

namespace {

// ------------------------------------------------------------- codebook
// Standard-normal CDF and its inverse by safeguarded Newton iteration on
// erfc, in double precision.
double norm_cdf(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }

double norm_quantile(double p) {
    double lo = -40.0, hi = 40.0, x = 0.0;
    const double inv_sqrt_2pi = 0.3989422804014327;
    for (int it = 0; it < 200; ++it) {
        const double f = norm_cdf(x) - p;
        if (f < 0) lo = x; else hi = x;
        const double dens = inv_sqrt_2pi * std::exp(-0.5 * x * x);
        double xn = x - f / dens;
        if (!(xn > lo && xn < hi)) xn = 0.5 * (lo + hi);
        if (xn == x) break;
        x = xn;
    }
    return x;
}

// "QLoRA, explained", "NormalFloat 4 (NF4)": averages of adjacent quantiles,
// a 9-level positive half and an 8-level negative half sharing zero (the
// offset delta averages the two halves' outermost probabilities), scaled to
// [-1, 1].
void build_table(float codes[16], float mids[15]) {
    const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
    double v[16];
    int n = 0;
    for (int j = 6; j >= 0; --j) v[n++] = -norm_quantile(delta - j * (delta - 0.5) / 7.0);
    v[n++] = 0.0;
    for (int i = 7; i >= 0; --i) v[n++] = norm_quantile(delta - i * (delta - 0.5) / 8.0);
    std::sort(v, v + 16);
    const double top = norm_quantile(delta);
    for (int i = 0; i < 16; ++i) codes[i] = static_cast<float>(v[i] / top);
    codes[0] = -1.0f;      // exact by construction; pinned against rounding of v/top
    codes[7] = 0.0f;
    codes[15] = 1.0f;
    for (int i = 0; i < 15; ++i)
        mids[i] = static_cast<float>((static_cast<double>(codes[i]) + codes[i + 1]) / 2.0);
}

const Nf4Table& table() {
    static Nf4Table t;
    static std::once_flag once;
    std::call_once(once, [] { build_table(t.code, t.mid); });
    return t;
}

// The quantiser's bucket table (kernels.cuh): bucket b covers x + 3 in
// [2 + b/16, 2 + (b+1)/16); base = the number of midpoints below
// 2 + b/16 - 3 - 2^-22, thr = midpoint number base (+inf past the last).
// Returns false unless every bucket spans at most one midpoint (true for the
// NF4 codes, whose midpoints lie at least 0.08 apart).
bool build_index_lut(const float mids[15], Nf4IndexLut* lut) {
    // consecutive finite midpoints (a codebook of fewer than 16 codes pads
    // its midpoints with +inf) must be more than a bucket apart
    for (int i = 0; i + 1 < 15 && std::isfinite(mids[i + 1]); ++i)
        if (!(double(mids[i + 1]) - double(mids[i]) > 1.0 / 16.0 + std::ldexp(1.0, -20))) return false;
    for (int b = 0; b < kNf4LutEntries; ++b) {
        const double lo = 2.0 + b / 16.0 - 3.0 - std::ldexp(1.0, -22);
        uint32_t base = 0;
        for (int i = 0; i < 15; ++i) base += double(mids[i]) < lo ? 1u : 0u;
        const float thr = base < 15 ? mids[base] : std::numeric_limits<float>::infinity();
        std::memcpy(&lut->thr[b], &thr, 4);
        lut->base[b] = base;
    }
    return true;
}

// nullptr if the table could not be built
const Nf4IndexLut* index_lut() {
    static Nf4IndexLut lut;
    static bool ok = false;
    static std::once_flag once;
    std::call_once(once, [] { ok = build_index_lut(table().mid, &lut); });
    return ok ? &lut : nullptr;
}

// ---------------------------------------------------------------- TMA
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed weight seen as {128 bytes, N rows, K/256 chunks of 128 bytes}; box
// {128, 256 / chunks, chunks} = a 32 KiB tile, 128-byte swizzle.
bool make_map_3d_packed(CUtensorMap* map, const void* packed, int64_t N, int64_t K, int chunks) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(K / 256)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K / 2), 128};
    const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(256 / chunks), static_cast<cuuint32_t>(chunks)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(packed), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------- validation
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_tensor(const qlora_nf4_tensor* w) {
    if (!w || !w->packed || !w->scale_codes || !w->meta_scale) return QLORA_ERR_NULL;
    if (w->rows < 0 || w->cols < 0) return QLORA_ERR_SHAPE;
    if (w->cols > 0 && w->rows > INT64_MAX / w->cols) return QLORA_ERR_SHAPE;
    if (!aligned(w->packed, 16) || !aligned(w->scale_codes, 4) || !aligned(w->meta_scale, 4))
        return QLORA_ERR_ALIGN;
    return QLORA_OK;
}

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// ------------------------------------------------------- workspace plan
constexpr int64_t kAlign = 256;
constexpr int64_t kControlBytes = 1024;     // error word + GEMV tile counters
constexpr int64_t kMaxGemvSlices = 200;

int64_t up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct Split {
    int splits;
    int64_t per;     // contraction slice width (the last slice may be shorter)
    int chunks;      // weight tile depth D in 256-wide chunks
};

// contraction slices of a LoRA side product: one cluster of up to 8 CTAs
// Contraction slices of a skinny product with `rows` output rows (64 per
// CTA): enough slices for about 128 CTAs, at most 8 (one cluster) and at most
// one per 64-wide chunk.  With the deep ring, fewer and longer slices keep
// more bytes in flight per CTA; measured on the 4096-token layer, 2 slices
// (128 CTAs) beat 4 and 8, and leave SMs free for the GEMM that follows.
constexpr int64_t kSkinnyTargetCtas = 128;
Split skinny_split(int64_t C, int64_t rows) {
    const int64_t chunks = std::max<int64_t>(1, cdiv(C, 64));
    const int64_t row_tiles = std::max<int64_t>(1, cdiv(rows, 64));
    const int64_t want = std::max<int64_t>(1, cdiv(kSkinnyTargetCtas, row_tiles));
    const int64_t s = std::min<int64_t>({int64_t(kMaxSkinnySplits), chunks, want});
    const int64_t per = cdiv(chunks, s) * 64;
    return {static_cast<int>(cdiv(std::max<int64_t>(C, 1), per)), per, 0};
}

// Contraction slices for the GEMV.  Each slice's activations must fit in
// shared memory (cap); among the slice widths that do, the one with the
// shortest estimated makespan is taken, in weight-tile times per CTA: the
// slice's units (R = 256 / D rows x the slice) are dealt to its CTAs in
// waves, so a CTA streams waves x ceil(chunks / D) tiles, and every slice
// adds M x N fp32 partials that are written and read again (counted as
// 32 KiB tiles spread over all CTAs).  D, the chunks per tile, is the
// largest power of two up to 8 that divides the slice's 256-wide chunks
// (8 for a single slice, whose last tile past K is zero-filled).
Split gemv_split(int64_t M, int64_t N, int64_t K) {
    int64_t cap = 256;
    for (int64_t c = std::min<int64_t>(K, 32768) / 256 * 256; c >= 256; c -= 256)
        if (gemv_stages(M, c) > 0) {
            cap = c;
            break;
        }
    const int64_t sms = std::max(1, num_sms());
    Split best{0, 0, 0};
    double best_cost = 0.0;
    const int64_t s_max = std::min<int64_t>(kMaxGemvSlices, std::max<int64_t>(1, K / 256));
    for (int64_t s = std::max<int64_t>(1, cdiv(K, cap)); s <= s_max; ++s) {
        for (int64_t q : {256, 512, 1024, 2048}) {
            const int64_t per = up(cdiv(K, s), q);
            if (per > cap || cdiv(K, per) != s) continue;
            const int64_t chunks = per / 256;
            int d = 1;
            if (s == 1 && chunks >= 8) {
                d = 8;
            } else {
                while (d < 8 && chunks % (2 * d) == 0) d *= 2;
            }
            const int64_t units = cdiv(N, 256 / d);
            const int64_t ctas = std::max<int64_t>(1, sms / s);
            const double cost = double(cdiv(units, ctas) * cdiv(chunks, d)) +
                                double(s * M * N * 8) / 32768.0 / double(ctas * s);
            if (best.splits == 0 || cost < best_cost - 1e-9) {
                best = {static_cast<int>(s), s == 1 ? K : per, d};
                best_cost = cost;
            }
        }
    }
    if (best.splits == 0) best = {static_cast<int>(cdiv(K, 256)), 256, 1};   // one chunk per slice
    return best;
}

// M <= 16 with K % 256 == 0 runs the bandwidth-bound GEMV (its 3-D weight view
// takes 256-wide chunks); every other shape runs the tensor-core GEMM.
bool use_gemv(int64_t M, int64_t K) { return M <= QLORA_GEMV_MAX_TOKENS && K % 256 == 0; }

// T = X A^T is spread thinly over the CTAs of each slice, so that each share
// is a k-step or two that overlaps the first weight tile's latency; every CTA
// of the share writes one fp32 partial, which the finalize sums.  The shares
// stop growing once the finalize would read more than kGemvTReadCap partial
// values per CTA, and never exceed kGemvTParts partials in all.
constexpr int kGemvTParts = 256;
constexpr int64_t kGemvTReadCap = 8192;
int gemv_t_ctas(int splits, int sms, int64_t M, int r) {
    const int sp = std::max(1, splits);
    const int per_slice = std::max(1, sms / sp);
    const int64_t by_read = kGemvTReadCap / std::max<int64_t>(1, M * r * sp);
    const int64_t by_total = kGemvTParts / sp;
    return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>({per_slice, by_read, by_total})));
}

struct Plan {
    int64_t rp;          // rank padded to 64
    int64_t off_err, off_part, off_tpart, off_gt, off_gu, total;
};

Plan make_plan(int64_t M, int64_t N, int64_t K, int r) {
    Plan p;
    p.rp = up(r, 64);
    int64_t part = 0, tpart = 0;
    if (use_gemv(M, K)) {
        const Split sp = gemv_split(M, N, K);
        part = int64_t(sp.splits) * M * N;
        tpart = int64_t(std::max(sp.splits, kGemvTParts)) * M * r;
    }
    int64_t o = 0;
    p.off_err = o;  o += kControlBytes;
    p.off_part = o; o += up(part * 4, kAlign);
    p.off_tpart = o; o += up(tpart * 4, kAlign);
    p.off_gt = o;   o += up(M * p.rp * 2, kAlign);
    p.off_gu = o;   o += up(M * p.rp * 2, kAlign);
    p.total = o;
    return p;
}

int check_linear_shapes(int64_t M, int64_t N, int64_t K, int r) {
    if (M < 0 || N < 0 || K < 0) return QLORA_ERR_SHAPE;
    if (K < 64 || N < 8 || K % 64 != 0 || N % 8 != 0) return QLORA_ERR_UNSUPPORTED;
    if (r < 8 || r > QLORA_MAX_RANK || r % 8 != 0) return QLORA_ERR_UNSUPPORTED;
    if (M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1 || K > (int64_t(1) << 31) - 1)
        return QLORA_ERR_UNSUPPORTED;
    return QLORA_OK;
}

// Tile schedule of the dequant-GEMM.  With one wave of 512 x 256 tiles, one
// tile per CTA pair.  With more, the pairs are persistent and take equal runs
// of whole 256-wide tiles (the same makespan as waves, and each pair's TMA
// loads of its next tile overlap the epilogue of its current one).  Narrower
// tiles are not used: they were measured slower per column than full ones
// (each step's dequantisation does not shrink with the tile width).
void gemm_schedule(GemmArgs& g, bool trans) {
    (void)trans;
    const int64_t tn = gemm_tile_n();
    const int64_t pairs = std::max(1, num_sms() / 2);
    const int64_t n_tiles = cdiv(g.d_cols, tn);
    const int64_t tiles = int64_t(g.m_tiles) * n_tiles;
    g.cols_lin = n_tiles * tn;
    g.col_budget = tn;
    if (tiles > pairs) g.col_budget = cdiv(tiles, pairs) * tn;
}

// Format variants: validate a qlora_format and build the kernels' table.
int check_format(const qlora_format* f, FmtTable* t, FmtArgs* a) {
    if (!f) return QLORA_ERR_NULL;
    const int b = f->block;
    if (b < 16 || b > 4096 || (b & (b - 1)) != 0) return QLORA_ERR_UNSUPPORTED;
    if (f->ncodes < 2 || f->ncodes > 16) return QLORA_ERR_UNSUPPORTED;
    if (f->scales != QLORA_SCALES_FP32 && f->scales != QLORA_SCALES_E4M3 &&
        f->scales != QLORA_SCALES_E5M2 && f->scales != QLORA_SCALES_U8)
        return QLORA_ERR_UNSUPPORTED;
    for (int i = 0; i < f->ncodes; ++i) {
        if (!std::isfinite(f->codes[i])) return QLORA_ERR_UNSUPPORTED;
        if (i > 0 && !(f->codes[i] > f->codes[i - 1])) return QLORA_ERR_UNSUPPORTED;
    }
    if (t) {
        std::memset(t, 0, sizeof(*t));
        for (int i = 0; i < f->ncodes; ++i) t->code[i] = f->codes[i];
        uint32_t z = 0;
        for (int i = 0; i < 15; ++i) {
            if (i < f->ncodes - 1) {
                // exact average of two fp32 values (exact in double), rounded to fp32
                t->mid[i] = static_cast<float>((double(f->codes[i]) + double(f->codes[i + 1])) / 2.0);
                if (0.0f > t->mid[i]) ++z;
            } else {
                t->mid[i] = std::numeric_limits<float>::infinity();
            }
        }
        t->zero_index = z;
        t->use_lut = build_index_lut(t->mid, &t->lut) ? 1u : 0u;
    }
    if (a) {
        a->block = b;
        a->log2_block = 0;
        while ((1 << a->log2_block) < b) ++a->log2_block;
        a->scale_fmt = f->scales;
    }
    return QLORA_OK;
}

// Bound of the tensor-core GEMM's operational waits (qlora_set_gemm_wait_limit_us).
std::atomic<unsigned long long> g_gemm_wait_ns{kWaitLimitNs};

cudaError_t record(const qlora_events* ev, bool begin, cudaStream_t s) {
    if (!ev) return cudaSuccess;
    void* e = begin ? ev->gemm_begin : ev->gemm_end;
    return e ? cudaEventRecord(reinterpret_cast<cudaEvent_t>(e), s) : cudaSuccess;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

// The quantisers' optional non-finite check.  When the caller passes a flag,
// the call clears it ahead of its kernels, and afterwards waits for the
// stream and returns QLORA_ERR_NONFINITE if a kernel raised it.
int begin_checked(int* d_flag, cudaStream_t s) {
    if (!d_flag) return QLORA_OK;
    return cuda_status(cudaMemsetAsync(d_flag, 0, sizeof(int), s));
}

int end_checked(int status, int* d_flag, cudaStream_t s) {
    if (status != QLORA_OK || !d_flag) return status;
    int h = 0;
    if (cudaMemcpyAsync(&h, d_flag, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return QLORA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return QLORA_ERR_CUDA;
    return h != 0 ? QLORA_ERR_NONFINITE : QLORA_OK;
}

#define QTRY(expr)                                   \
    do {                                             \
        cudaError_t _e = (expr);                     \
        if (_e != cudaSuccess) return QLORA_ERR_CUDA; \
    } while (0)

template <class T>
T* at(void* ws, int64_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

SkinnyArgs skinny_args(const uint16_t* P, const uint16_t* Q, int64_t I, int64_t J, int64_t C,
                       int64_t ldp, int64_t ldq) {
    SkinnyArgs a{};
    a.P = P;
    a.Q = Q;
    a.I = I;
    a.J = J;
    a.C = C;
    a.ldp = ldp;
    a.ldq = ldq;
    const Split sp = skinny_split(C, I);
    a.splits = sp.splits;
    a.c_per_split = sp.per;
    a.alpha = 1.0f;
    a.beta = 1.0f;
    a.cvt_scale = 1.0f;
    return a;
}

// T = X A^T -> optional fp32 T_save and bf16 gamma*T padded to rp columns.
// trigger: a GEMM launched next as its programmatic dependent may start at once.
cudaError_t run_T(const uint16_t* X, const uint16_t* A, int64_t M, int64_t K, int r, float gamma,
                  float* T_save, uint16_t* Gt, int64_t rp, int* err_zero, bool trigger,
                  cudaStream_t s) {
    SkinnyArgs a = skinny_args(X, A, M, r, K, K, K);
    a.out = T_save;
    a.out_bf16 = Gt;
    a.ldb = rp;
    a.beta = gamma;
    a.err_zero = err_zero;
    a.trigger_dependents = trigger ? 1 : 0;
    return launch_skinny(true, true, a, s);
}

}  // namespace

// ===================================================================== ABI
extern "C" {

const char* qlora_status_string(int status) {
    switch (status) {
        case QLORA_OK: return "ok";
        case QLORA_ERR_NULL: return "null pointer";
        case QLORA_ERR_SHAPE: return "bad shape";
        case QLORA_ERR_ALIGN: return "misaligned pointer";
        case QLORA_ERR_UNSUPPORTED: return "unsupported size";
        case QLORA_ERR_NONFINITE: return "non-finite weight";
        case QLORA_ERR_CUDA: return "CUDA error";
        case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

int qlora_set_gemm_wait_limit_us(int64_t us) {
    if (us < 0 || us > 10000000) return QLORA_ERR_UNSUPPORTED;
    g_gemm_wait_ns.store(us == 0 ? kWaitLimitNs : static_cast<unsigned long long>(us) * 1000ull,
                         std::memory_order_relaxed);
    return QLORA_OK;
}

int nf4_build_codebook(float codes[16], float midpoints[15]) {
    if (!codes || !midpoints) return QLORA_ERR_NULL;
    const Nf4Table& t = table();
    std::memcpy(codes, t.code, sizeof(t.code));
    std::memcpy(midpoints, t.mid, sizeof(t.mid));
    return QLORA_OK;
}

int qlora_quantized_sizes(int64_t rows, int64_t cols, size_t* packed_bytes, size_t* codes_bytes,
                          size_t* meta_bytes) {
    if (!packed_bytes || !codes_bytes || !meta_bytes) return QLORA_ERR_NULL;
    if (rows < 0 || cols < 0) return QLORA_ERR_SHAPE;
    if (cols > 0 && rows > INT64_MAX / cols) return QLORA_ERR_SHAPE;
    const int64_t numel = rows * cols;
    const int64_t nblocks = cdiv(numel, QLORA_BLOCK);
    const int64_t ngroups = cdiv(nblocks, QLORA_GROUP);
    *packed_bytes = static_cast<size_t>(nblocks) * (QLORA_BLOCK / 2);
    *codes_bytes = static_cast<size_t>(nblocks);
    *meta_bytes = static_cast<size_t>(ngroups) * 4;
    return QLORA_OK;
}

int qlora_quantize(const float* W, const qlora_nf4_tensor* out, int* d_nonfinite_flag,
                   qlora_stream_t stream) {
    if (!W) return QLORA_ERR_NULL;
    int st = check_tensor(out);
    if (st != QLORA_OK) return st;
    if (!aligned(W, 16)) return QLORA_ERR_ALIGN;
    const int64_t numel = out->rows * out->cols;
    if (numel == 0) return QLORA_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    st = begin_checked(d_nonfinite_flag, s);
    if (st != QLORA_OK) return st;
    const Nf4IndexLut* lut = index_lut();
    if (!lut) return QLORA_ERR_UNSUPPORTED;
    st = cuda_status(launch_quantize(W, numel, out->packed, out->scale_codes, out->meta_scale,
                                     d_nonfinite_flag, *lut, s));
    return end_checked(st, d_nonfinite_flag, s);
}

int qlora_dequantize(const qlora_nf4_tensor* w, uint16_t* W_out, qlora_stream_t stream) {
    if (!W_out) return QLORA_ERR_NULL;
    int st = check_tensor(w);
    if (st != QLORA_OK) return st;
    if (!aligned(W_out, 16)) return QLORA_ERR_ALIGN;
    const int64_t numel = w->rows * w->cols;
    if (numel == 0) return QLORA_OK;
    return cuda_status(launch_dequantize(w->packed, w->scale_codes, w->meta_scale, numel, W_out,
                                         table(), num_sms(),
                                         reinterpret_cast<cudaStream_t>(stream)));
}

int qlora_quantize_bf16(const uint16_t* W, const qlora_nf4_tensor* out, int* d_nonfinite_flag,
                        qlora_stream_t stream) {
    if (!W) return QLORA_ERR_NULL;
    int st = check_tensor(out);
    if (st != QLORA_OK) return st;
    if (!aligned(W, 16)) return QLORA_ERR_ALIGN;
    const int64_t numel = out->rows * out->cols;
    if (numel == 0) return QLORA_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    st = begin_checked(d_nonfinite_flag, s);
    if (st != QLORA_OK) return st;
    const Nf4IndexLut* lut = index_lut();
    if (!lut) return QLORA_ERR_UNSUPPORTED;
    st = cuda_status(launch_quantize_bf16(W, numel, out->packed, out->scale_codes,
                                          out->meta_scale, d_nonfinite_flag, *lut, s));
    return end_checked(st, d_nonfinite_flag, s);
}

int qlora_quantize_many(const qlora_quantize_job* jobs, int n, int input_bf16,
                        int* d_nonfinite_flag, qlora_stream_t stream) {
    if (n < 0) return QLORA_ERR_SHAPE;
    if (n > 0 && !jobs) return QLORA_ERR_NULL;
    // every job is checked before anything is launched
    std::vector<QuantizeJob> q;
    q.reserve(static_cast<size_t>(n));
    for (int i = 0; i < n; ++i) {
        const qlora_nf4_tensor* o = jobs[i].out;
        if (!o) return QLORA_ERR_NULL;
        if (o->rows < 0 || o->cols < 0) return QLORA_ERR_SHAPE;
        if (o->rows == 0 || o->cols == 0) continue;   // empty: W and buffers may be NULL
        const int st = check_tensor(o);
        if (st != QLORA_OK) return st;
        const int64_t numel = o->rows * o->cols;
        if (!jobs[i].W) return QLORA_ERR_NULL;
        if (!aligned(jobs[i].W, 16)) return QLORA_ERR_ALIGN;
        q.push_back({jobs[i].W, numel, jobs[i].out->packed, jobs[i].out->scale_codes,
                     jobs[i].out->meta_scale});
    }
    if (q.empty()) return QLORA_OK;
    const Nf4IndexLut* lut = index_lut();
    if (!lut) return QLORA_ERR_UNSUPPORTED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int st = begin_checked(d_nonfinite_flag, s);
    if (st != QLORA_OK) return st;
    st = cuda_status(launch_quantize_many(q.data(), static_cast<int>(q.size()), input_bf16 != 0,
                                          d_nonfinite_flag, *lut, s));
    return end_checked(st, d_nonfinite_flag, s);
}

int qlora_format_sizes(int64_t numel, const qlora_format* f, size_t* packed_bytes,
                       size_t* scale_bytes, size_t* meta_bytes) {
    if (!packed_bytes || !scale_bytes || !meta_bytes) return QLORA_ERR_NULL;
    int st = check_format(f, nullptr, nullptr);
    if (st != QLORA_OK) return st;
    if (numel < 0) return QLORA_ERR_SHAPE;
    const int64_t nblocks = cdiv(numel, f->block);
    *packed_bytes = static_cast<size_t>(nblocks) * (f->block / 2);
    if (f->scales == QLORA_SCALES_FP32) {
        *scale_bytes = static_cast<size_t>(nblocks) * 4;
        *meta_bytes = 0;
    } else {
        *scale_bytes = static_cast<size_t>(nblocks);
        *meta_bytes = static_cast<size_t>(cdiv(nblocks, QLORA_GROUP)) * 4;
    }
    return QLORA_OK;
}

int qlora_quantize_fmt(const float* W, int64_t numel, const qlora_format* f, uint8_t* packed,
                       void* scales, float* meta, int* d_nonfinite_flag, qlora_stream_t stream) {
    FmtTable t;
    FmtArgs a;
    int st = check_format(f, &t, &a);
    if (st != QLORA_OK) return st;
    if (numel < 0) return QLORA_ERR_SHAPE;
    if (numel == 0) return QLORA_OK;
    if (!W || !packed || !scales || (a.scale_fmt != QLORA_SCALES_FP32 && !meta)) return QLORA_ERR_NULL;
    if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(scales, 4) || (meta && !aligned(meta, 4)))
        return QLORA_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    st = begin_checked(d_nonfinite_flag, s);
    if (st != QLORA_OK) return st;
    st = cuda_status(launch_quantize_fmt(W, numel, a, packed, scales, meta, d_nonfinite_flag, t, s));
    return end_checked(st, d_nonfinite_flag, s);
}

int qlora_dequantize_fmt(const uint8_t* packed, const void* scales, const float* meta,
                         int64_t numel, const qlora_format* f, uint16_t* out,
                         qlora_stream_t stream) {
    FmtTable t;
    FmtArgs a;
    int st = check_format(f, &t, &a);
    if (st != QLORA_OK) return st;
    if (numel < 0) return QLORA_ERR_SHAPE;
    if (numel == 0) return QLORA_OK;
    if (!packed || !scales || !out || (a.scale_fmt != QLORA_SCALES_FP32 && !meta)) return QLORA_ERR_NULL;
    if (!aligned(packed, 16) || !aligned(out, 16) || !aligned(scales, 4) || (meta && !aligned(meta, 4)))
        return QLORA_ERR_ALIGN;
    return cuda_status(launch_dequantize_fmt(packed, scales, meta, numel, a, out, t, num_sms(),
                                             reinterpret_cast<cudaStream_t>(stream)));
}

int qlora_adamw8_state_sizes(int64_t n, size_t* code_bytes, size_t* absmax_bytes) {
    if (!code_bytes || !absmax_bytes) return QLORA_ERR_NULL;
    if (n < 0) return QLORA_ERR_SHAPE;
    *code_bytes = static_cast<size_t>(n);
    *absmax_bytes = static_cast<size_t>(cdiv(n, QLORA_BLOCK)) * 4;
    return QLORA_OK;
}

int qlora_adamw8_step(float* p, const float* g, int64_t n, int8_t* m_codes, float* m_absmax,
                      uint8_t* v_codes, float* v_absmax, const qlora_adamw_config* cfg,
                      uint16_t* p_bf16, qlora_stream_t stream) {
    if (!cfg) return QLORA_ERR_NULL;
    if (n < 0) return QLORA_ERR_SHAPE;
    // eps > 0 keeps every division finite (a block whose gradient and moments
    // are all zero divides 0 by eps); lr >= 0, wd >= 0 and lr wd < 1 keep the
    // decoupled decay factor 1 - lr wd in (0, 1]
    if (cfg->step < 1 || !(cfg->beta1 >= 0.f && cfg->beta1 < 1.f) ||
        !(cfg->beta2 >= 0.f && cfg->beta2 < 1.f) || !std::isfinite(cfg->lr) ||
        !std::isfinite(cfg->eps) || !std::isfinite(cfg->weight_decay) || !(cfg->eps > 0.f) ||
        !(cfg->lr >= 0.f) || !(cfg->weight_decay >= 0.f) ||
        !(double(cfg->lr) * double(cfg->weight_decay) < 1.0))
        return QLORA_ERR_UNSUPPORTED;
    if (n == 0) return QLORA_OK;
    if (!p || !g || !m_codes || !m_absmax || !v_codes || !v_absmax) return QLORA_ERR_NULL;
    if (!aligned(p, 16) || !aligned(g, 16) || !aligned(m_codes, 4) || !aligned(v_codes, 4) ||
        !aligned(m_absmax, 4) || !aligned(v_absmax, 4) || (p_bf16 && !aligned(p_bf16, 8)))
        return QLORA_ERR_ALIGN;
    Adam8Args a{};
    a.p = p;
    a.g = g;
    a.m_codes = m_codes;
    a.m_absmax = m_absmax;
    a.v_codes = v_codes;
    a.v_absmax = v_absmax;
    a.p_bf16 = p_bf16;
    a.n = n;
    // constants formed in double from the fp32 arguments, rounded once
    const double lr = cfg->lr, b1 = cfg->beta1, b2 = cfg->beta2, wd = cfg->weight_decay;
    const double t = static_cast<double>(cfg->step);
    a.lr = cfg->lr;
    a.beta1 = cfg->beta1;
    a.beta2 = cfg->beta2;
    a.eps = cfg->eps;
    a.decay = static_cast<float>(1.0 - lr * wd);
    a.one_m_beta1 = static_cast<float>(1.0 - b1);
    a.one_m_beta2 = static_cast<float>(1.0 - b2);
    a.bc1 = static_cast<float>(1.0 - std::pow(b1, t));
    a.bc2 = static_cast<float>(1.0 - std::pow(b2, t));
    return cuda_status(launch_adamw8(a, num_sms(), reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// Checks one merge and fills its kernel arguments; *skip = true when the
// weight is empty (nothing read or written).
int merge_job_args(const qlora_nf4_tensor* w, const uint16_t* A, const uint16_t* B, int r,
                   float scale, uint16_t* W_out, MergeArgs* a, bool* skip) {
    *skip = false;
    if (!w) return QLORA_ERR_NULL;
    const int64_t N = w->rows, K = w->cols;
    if (N < 0 || K < 0 || (K > 0 && N > INT64_MAX / K)) return QLORA_ERR_SHAPE;
    if (K % QLORA_BLOCK != 0) return QLORA_ERR_UNSUPPORTED;
    if (r < 8 || r > QLORA_MAX_RANK || r % 8 != 0) return QLORA_ERR_UNSUPPORTED;
    if (N > (int64_t(1) << 31) - 1 || K > (int64_t(1) << 31) - 1) return QLORA_ERR_UNSUPPORTED;
    if (N == 0 || K == 0) {
        *skip = true;
        return QLORA_OK;
    }
    int st = check_tensor(w);
    if (st != QLORA_OK) return st;
    if (!A || !B || !W_out) return QLORA_ERR_NULL;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(W_out, 16)) return QLORA_ERR_ALIGN;
    *a = MergeArgs{};
    a->packed = reinterpret_cast<const uint32_t*>(w->packed);
    a->scale_codes = w->scale_codes;
    a->meta = w->meta_scale;
    a->A = A;
    a->B = B;
    a->out = W_out;
    a->N = N;
    a->K = K;
    a->r = r;
    a->gamma = scale;
    return QLORA_OK;
}

}  // namespace

extern "C" {

int qlora_merge(const qlora_nf4_tensor* w, const uint16_t* A, const uint16_t* B, int r,
                float scale, uint16_t* W_out, qlora_stream_t stream) {
    MergeArgs a;
    bool skip = false;
    const int st = merge_job_args(w, A, B, r, scale, W_out, &a, &skip);
    if (st != QLORA_OK || skip) return st;
    return cuda_status(launch_merge(&a, 1, table(), num_sms(), reinterpret_cast<cudaStream_t>(stream)));
}

int qlora_merge_many(const qlora_merge_job* jobs, int n, qlora_stream_t stream) {
    if (n < 0) return QLORA_ERR_SHAPE;
    if (n > 0 && !jobs) return QLORA_ERR_NULL;
    // every job is checked before anything is launched
    for (int i = 0; i < n; ++i) {
        MergeArgs a;
        bool skip = false;
        const int st = merge_job_args(jobs[i].w, jobs[i].A, jobs[i].B, jobs[i].r, jobs[i].scale,
                                      jobs[i].W_out, &a, &skip);
        if (st != QLORA_OK) return st;
    }
    MergeArgs batch[kMaxMergeJobs];
    int k = 0;
    for (int i = 0; i < n; ++i) {
        bool skip = false;
        merge_job_args(jobs[i].w, jobs[i].A, jobs[i].B, jobs[i].r, jobs[i].scale, jobs[i].W_out,
                       &batch[k], &skip);
        if (skip) continue;
        if (++k == kMaxMergeJobs) {
            QTRY(launch_merge(batch, k, table(), num_sms(), reinterpret_cast<cudaStream_t>(stream)));
            k = 0;
        }
    }
    if (k > 0) QTRY(launch_merge(batch, k, table(), num_sms(), reinterpret_cast<cudaStream_t>(stream)));
    return QLORA_OK;
}

int qlora_linear_workspace_size(int64_t M, int64_t N, int64_t K, int r, size_t* bytes) {
    if (!bytes) return QLORA_ERR_NULL;
    int st = check_linear_shapes(M, N, K, r);
    if (st != QLORA_OK) return st;
    *bytes = static_cast<size_t>(make_plan(M, N, K, r).total);
    return QLORA_OK;
}

int qlora_linear_forward_ex(const uint16_t* X, int64_t M, const qlora_nf4_tensor* w,
                            const uint16_t* A, const uint16_t* B, int r, float scale, uint16_t* Y,
                            float* T_save, void* ws, size_t ws_bytes, qlora_stream_t stream,
                            const qlora_events* ev) {
    // an empty batch may come with NULL activation pointers
    if (!A || !B || (M != 0 && (!X || !Y))) return QLORA_ERR_NULL;
    int st = check_tensor(w);
    if (st != QLORA_OK) return st;
    const int64_t N = w->rows, K = w->cols;
    st = check_linear_shapes(M, N, K, r);
    if (st != QLORA_OK) return st;
    if (!aligned(X, 16) || !aligned(A, 16) || !aligned(B, 16) || !aligned(Y, 16) ||
        (T_save && !aligned(T_save, 16)))
        return QLORA_ERR_ALIGN;
    const Plan p = make_plan(M, N, K, r);
    if (!ws || ws_bytes < static_cast<size_t>(p.total)) return QLORA_ERR_WORKSPACE;
    if (!aligned(ws, kAlign)) return QLORA_ERR_ALIGN;
    if (M == 0) return QLORA_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int* err = at<int>(ws, p.off_err);
    float* part = at<float>(ws, p.off_part);
    uint16_t* Gt = at<uint16_t>(ws, p.off_gt);
    if (use_gemv(M, K)) {
        // decode path: T is computed inside the GEMV kernel; the control
        // words (error word, work-unit counters) start at zero
        const Split sp = gemv_split(M, N, K);
        if (sp.splits > kMaxGemvSlices) return QLORA_ERR_UNSUPPORTED;
        float* tpart = at<float>(ws, p.off_tpart);
        int* counters = err + 4;
        QTRY(cudaMemsetAsync(err, 0, size_t(4 + sp.splits) * sizeof(int), s));
        GemvArgs g{};
        g.packed = w->packed;
        g.scale_codes = w->scale_codes;
        g.meta = w->meta_scale;
        g.X = X;
        g.A = A;
        g.r = r;
        g.part = part;
        g.Tpart = tpart;
        g.counters = counters;
        g.M = M;
        g.N = N;
        g.K = K;
        g.splits = sp.splits;
        g.k_per_split = sp.per;
        g.tile_chunks = sp.chunks;
        g.t_ctas = gemv_t_ctas(sp.splits, num_sms(), M, r);
        g.err = err;
        g.tab = table();
        CUtensorMap m_w;
        if (!make_map_3d_packed(&m_w, w->packed, N, K, sp.chunks)) return QLORA_ERR_CUDA;
        QTRY(record(ev, true, s));
        QTRY(launch_gemv(m_w, g, num_sms(), s));
        QTRY(record(ev, false, s));
        GemvFinalizeArgs f{part, tpart, sp.splits, sp.splits * g.t_ctas, B, r, scale, T_save, Y, M, N};
        QTRY(launch_gemv_finalize(f, s));
        return QLORA_OK;
    }
    QTRY(run_T(X, A, M, K, r, scale, T_save, Gt, p.rp, err, true, s));

    // B [N x r] is read in place: the 64-wide TMA box zero-fills columns >= r
    CUtensorMap m_act, m_packed, m_la, m_lb, m_out;
    bool ok = make_map_2d(&m_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, N * 2, 16, 32,
                          CU_TENSOR_MAP_SWIZZLE_NONE) &&
              make_map_2d(&m_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, K * 2, 64, 128,
                          CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map_2d(&m_packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->packed, K / 2, N, K / 2, 32,
                          gemm_half_n(), CU_TENSOR_MAP_SWIZZLE_32B) &&
              make_map_2d(&m_la, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Gt, p.rp, M, p.rp * 2, 64, 128,
                          CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map_2d(&m_lb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, r, N, int64_t(r) * 2, 64,
                          gemm_half_n(), CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return QLORA_ERR_CUDA;
    GemmArgs g{};
    g.scale_codes = w->scale_codes;
    g.meta = w->meta_scale;
    g.D = Y;
    g.M = M;
    g.Nw = N;
    g.d_cols = N;
    g.nkb = K / 64;
    g.main_steps = static_cast<int>(K / 64);
    g.tail_steps = static_cast<int>(cdiv(r, 64));
    g.r = r;
    g.m_tiles = static_cast<int>(cdiv(M, gemm_tile_m()));
    gemm_schedule(g, false);
    g.err = err;
    g.wait_ns = g_gemm_wait_ns.load(std::memory_order_relaxed);
    g.tab = table();
    // an event record between the two kernels would serialise them fully
    QTRY(record(ev, true, s));
    QTRY(launch_gemm(false, m_act, m_packed, m_la, m_lb, m_out, g, ev == nullptr, s));
    QTRY(record(ev, false, s));
    return QLORA_OK;
}

int qlora_linear_forward(const uint16_t* X, int64_t M, const qlora_nf4_tensor* w,
                         const uint16_t* A, const uint16_t* B, int r, float scale, uint16_t* Y,
                         float* T_save, void* ws, size_t ws_bytes, qlora_stream_t stream) {
    return qlora_linear_forward_ex(X, M, w, A, B, r, scale, Y, T_save, ws, ws_bytes, stream,
                                   nullptr);
}

int qlora_linear_backward_ex(const uint16_t* dY, const uint16_t* X, int64_t M,
                             const qlora_nf4_tensor* w, const uint16_t* A, const uint16_t* B,
                             int r, float scale, const float* T_saved, uint16_t* dX, float* dA,
                             float* dB, int accumulate, void* ws, size_t ws_bytes,
                             qlora_stream_t stream, const qlora_events* ev) {
    if (!A || !B || !dA || !dB || (M != 0 && (!dY || !X))) return QLORA_ERR_NULL;
    int st = check_tensor(w);
    if (st != QLORA_OK) return st;
    const int64_t N = w->rows, K = w->cols;
    st = check_linear_shapes(M, N, K, r);
    if (st != QLORA_OK) return st;
    if (!aligned(dY, 16) || !aligned(X, 16) || !aligned(A, 16) || !aligned(B, 16) ||
        !aligned(dA, 16) || !aligned(dB, 16) || (dX && !aligned(dX, 16)) ||
        (T_saved && !aligned(T_saved, 16)))
        return QLORA_ERR_ALIGN;
    const Plan p = make_plan(M, N, K, r);
    if (!ws || ws_bytes < static_cast<size_t>(p.total)) return QLORA_ERR_WORKSPACE;
    if (!aligned(ws, kAlign)) return QLORA_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (M == 0) {
        // empty batch: gradients are zero (or unchanged when accumulating)
        if (!accumulate) {
            QTRY(cudaMemsetAsync(dA, 0, size_t(r) * K * 4, s));
            QTRY(cudaMemsetAsync(dB, 0, size_t(N) * r * 4, s));
        }
        return QLORA_OK;
    }
    int* err = at<int>(ws, p.off_err);
    uint16_t* Gt = at<uint16_t>(ws, p.off_gt);
    uint16_t* Gu = at<uint16_t>(ws, p.off_gu);
    int* err_first = err;                 // cleared by the first kernel of the call

    if (!T_saved) {                       // recompute gamma * T in bf16
        QTRY(run_T(X, A, M, K, r, scale, nullptr, Gt, p.rp, err_first, false, s));
        err_first = nullptr;
    }
    // U = dY B -> gamma * U in bf16; converts a saved T to gamma * T on the side
    {
        SkinnyArgs a = skinny_args(dY, B, M, r, N, N, r);
        a.out_bf16 = Gu;
        a.ldb = p.rp;
        a.beta = scale;
        if (T_saved) {
            a.cvt_src = T_saved;
            a.cvt_dst = Gt;
            a.cvt_scale = scale;
        }
        a.err_zero = err_first;
        QTRY(launch_skinny(true, false, a, s));
    }
    // dX = dY W~ + (gamma U) A, launched as U's programmatic dependent (U does
    // not signal early, so the GEMM starts as U completes; it waits for U
    // again only before its LoRA steps).  dB = dY^T (gamma T) and
    // dA^T = X^T (gamma U) follow as the GEMM's programmatic dependents: the
    // GEMM signals on entry and they never wait for it (they read only U's
    // outputs, dY and X), so they run beside it on the SMs it leaves idle.
    // Profiling events between the kernels make the launches ordinary.
    if (dX) {
        // A [r x K] is read in place: the 64-row TMA box zero-fills rows >= r
        CUtensorMap m_act, m_packed, m_la, m_lb, m_out;
        bool ok = make_map_2d(&m_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dX, K, M, K * 2, 16, 32,
                              CU_TENSOR_MAP_SWIZZLE_NONE) &&
                  make_map_2d(&m_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, N, M, N * 2, 64, 128,
                              CU_TENSOR_MAP_SWIZZLE_128B) &&
                  make_map_2d(&m_packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->packed, K / 2, N, K / 2,
                              gemm_half_n() / 2, 64, CU_TENSOR_MAP_SWIZZLE_64B) &&
                  make_map_2d(&m_la, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Gu, p.rp, M, p.rp * 2, 64,
                              128, CU_TENSOR_MAP_SWIZZLE_128B) &&
                  make_map_2d(&m_lb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, K, r, K * 2, 64, 64,
                              CU_TENSOR_MAP_SWIZZLE_128B);
        if (!ok) return QLORA_ERR_CUDA;
        GemmArgs g{};
        g.scale_codes = w->scale_codes;
        g.meta = w->meta_scale;
        g.D = dX;
        g.M = M;
        g.Nw = N;
        g.d_cols = K;
        g.nkb = K / 64;
        g.main_steps = static_cast<int>(cdiv(N, 64));
        g.tail_steps = static_cast<int>(cdiv(r, 64));
        g.r = r;
        g.m_tiles = static_cast<int>(cdiv(M, gemm_tile_m()));
        gemm_schedule(g, true);
        g.err = err;
        g.wait_ns = g_gemm_wait_ns.load(std::memory_order_relaxed);
        g.tab = table();
        QTRY(record(ev, true, s));
        QTRY(launch_gemm(true, m_act, m_packed, m_la, m_lb, m_out, g, ev == nullptr, s));
        QTRY(record(ev, false, s));
    }
    {
        SkinnyArgs a = skinny_args(dY, Gt, N, r, M, N, p.rp);
        a.out = dB;
        a.accumulate = accumulate;
        a.programmatic = 1;
        a.trigger_dependents = 1;      // dA need not wait for dB either
        QTRY(launch_skinny(false, false, a, s));
    }
    {
        SkinnyArgs a = skinny_args(X, Gu, K, r, M, K, p.rp);
        a.out = dA;
        a.transpose = 1;
        a.accumulate = accumulate;
        a.programmatic = 1;
        QTRY(launch_skinny(false, false, a, s));
    }
    return QLORA_OK;
}

int qlora_linear_backward(const uint16_t* dY, const uint16_t* X, int64_t M,
                          const qlora_nf4_tensor* w, const uint16_t* A, const uint16_t* B, int r,
                          float scale, const float* T_saved, uint16_t* dX, float* dA, float* dB,
                          int accumulate, void* ws, size_t ws_bytes, qlora_stream_t stream) {
    return qlora_linear_backward_ex(dY, X, M, w, A, B, r, scale, T_saved, dX, dA, dB, accumulate,
                                    ws, ws_bytes, stream, nullptr);
}

// ------------------------------------------------ chained SwiGLU MLP (f3)
}  // extern "C"

namespace {

struct MlpPlan {
    int64_t D, F;
    size_t lin;                          // one linear call's workspace
    // linear calls' workspaces, each keeping its own error word: [0] gate
    // and [1] up forward (or recompute), [2] down, [3] gate and [4] up backward
    int64_t off_lin[5], off_g, off_u, off_h, off_dh, off_dxg, off_tg, off_tu, total;
};

int mlp_plan(int64_t M, const qlora_mlp* m, MlpPlan* p) {
    if (!m) return QLORA_ERR_NULL;
    int st = check_tensor(&m->gate);
    if (st == QLORA_OK) st = check_tensor(&m->up);
    if (st == QLORA_OK) st = check_tensor(&m->down);
    if (st != QLORA_OK) return st;
    const int64_t F = m->gate.rows, D = m->gate.cols;
    if (m->up.rows != F || m->up.cols != D || m->down.rows != D || m->down.cols != F)
        return QLORA_ERR_SHAPE;
    if (M < 0) return QLORA_ERR_SHAPE;
    st = check_linear_shapes(M, F, D, m->r);
    if (st == QLORA_OK) st = check_linear_shapes(M, D, F, m->r);
    if (st != QLORA_OK) return st;
    p->D = D;
    p->F = F;
    p->lin = static_cast<size_t>(std::max(make_plan(M, F, D, m->r).total, make_plan(M, D, F, m->r).total));
    int64_t o = kAlign;                                   // header: the call's error word
    for (int i = 0; i < 5; ++i) {
        p->off_lin[i] = o;
        o += up(static_cast<int64_t>(p->lin), kAlign);
    }
    const int64_t mf = up(M * F * 2, kAlign);
    p->off_g = o;   o += mf;
    p->off_u = o;   o += mf;
    p->off_h = o;   o += mf;
    p->off_dh = o;  o += mf;
    p->off_dxg = o; o += up(M * D * 2, kAlign);
    p->off_tg = o;  o += up(M * m->r * 4, kAlign);
    p->off_tu = o;  o += up(M * m->r * 4, kAlign);
    p->total = o;
    return QLORA_OK;
}

int check_mlp_adapters(const qlora_mlp* m) {
    if (!m->A_gate || !m->B_gate || !m->A_up || !m->B_up || !m->A_down || !m->B_down)
        return QLORA_ERR_NULL;
    return QLORA_OK;
}

}  // namespace

extern "C" {

int qlora_mlp_workspace_size(int64_t M, const qlora_mlp* mlp, size_t* bytes) {
    if (!bytes) return QLORA_ERR_NULL;
    MlpPlan p;
    const int st = mlp_plan(M, mlp, &p);
    if (st != QLORA_OK) return st;
    *bytes = static_cast<size_t>(p.total);
    return QLORA_OK;
}

int qlora_mlp_forward(const uint16_t* X, int64_t M, const qlora_mlp* mlp, float scale, uint16_t* Y,
                      void* ws, size_t ws_bytes, qlora_stream_t stream) {
    MlpPlan p;
    int st = mlp_plan(M, mlp, &p);
    if (st != QLORA_OK) return st;
    st = check_mlp_adapters(mlp);
    if (st != QLORA_OK) return st;
    if (M != 0 && (!X || !Y)) return QLORA_ERR_NULL;
    if (!aligned(X, 16) || !aligned(Y, 16)) return QLORA_ERR_ALIGN;
    if (!ws || ws_bytes < static_cast<size_t>(p.total)) return QLORA_ERR_WORKSPACE;
    if (!aligned(ws, kAlign)) return QLORA_ERR_ALIGN;
    if (M == 0) return QLORA_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint16_t* G = at<uint16_t>(ws, p.off_g);
    uint16_t* U = at<uint16_t>(ws, p.off_u);
    uint16_t* H = at<uint16_t>(ws, p.off_h);
    const int r = mlp->r;
    void* w0 = at<void>(ws, p.off_lin[0]);
    void* w1 = at<void>(ws, p.off_lin[1]);
    void* w2 = at<void>(ws, p.off_lin[2]);
    st = qlora_linear_forward(X, M, &mlp->gate, mlp->A_gate, mlp->B_gate, r, scale, G, nullptr, w0,
                              p.lin, stream);
    if (st == QLORA_OK)
        st = qlora_linear_forward(X, M, &mlp->up, mlp->A_up, mlp->B_up, r, scale, U, nullptr, w1,
                                  p.lin, stream);
    if (st != QLORA_OK) return st;
    QTRY(launch_swiglu_forward(G, U, H, M * p.F, num_sms(), s));
    st = qlora_linear_forward(H, M, &mlp->down, mlp->A_down, mlp->B_down, r, scale, Y, nullptr, w2,
                              p.lin, stream);
    if (st != QLORA_OK) return st;
    QTRY(launch_or_words(at<int>(ws, 0), at<int>(ws, p.off_lin[0]), at<int>(ws, p.off_lin[1]),
                         at<int>(ws, p.off_lin[2]), false, s));
    return QLORA_OK;
}

int qlora_mlp_backward(const uint16_t* dY, const uint16_t* X, int64_t M, const qlora_mlp* mlp,
                       float scale, uint16_t* dX, const qlora_mlp_grads* g, int accumulate,
                       void* ws, size_t ws_bytes, qlora_stream_t stream) {
    MlpPlan p;
    int st = mlp_plan(M, mlp, &p);
    if (st != QLORA_OK) return st;
    st = check_mlp_adapters(mlp);
    if (st != QLORA_OK) return st;
    if (!g || !g->dA_gate || !g->dB_gate || !g->dA_up || !g->dB_up || !g->dA_down || !g->dB_down)
        return QLORA_ERR_NULL;
    if (M != 0 && (!dY || !X || !dX)) return QLORA_ERR_NULL;
    if (!aligned(dY, 16) || !aligned(X, 16) || !aligned(dX, 16)) return QLORA_ERR_ALIGN;
    if (!ws || ws_bytes < static_cast<size_t>(p.total)) return QLORA_ERR_WORKSPACE;
    if (!aligned(ws, kAlign)) return QLORA_ERR_ALIGN;
    const int r = mlp->r;
    void* w0 = at<void>(ws, p.off_lin[0]);
    void* w1 = at<void>(ws, p.off_lin[1]);
    void* w2 = at<void>(ws, p.off_lin[2]);
    void* w3 = at<void>(ws, p.off_lin[3]);
    void* w4 = at<void>(ws, p.off_lin[4]);
    if (M == 0) {
        // empty batch: the linear backwards write zero gradients (or leave
        // them when accumulating)
        st = qlora_linear_backward(nullptr, nullptr, 0, &mlp->down, mlp->A_down, mlp->B_down, r,
                                   scale, nullptr, nullptr, g->dA_down, g->dB_down, accumulate, w2,
                                   p.lin, stream);
        if (st == QLORA_OK)
            st = qlora_linear_backward(nullptr, nullptr, 0, &mlp->gate, mlp->A_gate, mlp->B_gate, r,
                                       scale, nullptr, nullptr, g->dA_gate, g->dB_gate, accumulate,
                                       w0, p.lin, stream);
        if (st == QLORA_OK)
            st = qlora_linear_backward(nullptr, nullptr, 0, &mlp->up, mlp->A_up, mlp->B_up, r, scale,
                                       nullptr, nullptr, g->dA_up, g->dB_up, accumulate, w1, p.lin,
                                       stream);
        return st;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint16_t* G = at<uint16_t>(ws, p.off_g);
    uint16_t* U = at<uint16_t>(ws, p.off_u);
    uint16_t* H = at<uint16_t>(ws, p.off_h);
    uint16_t* dH = at<uint16_t>(ws, p.off_dh);
    uint16_t* dXg = at<uint16_t>(ws, p.off_dxg);
    float* Tg = at<float>(ws, p.off_tg);
    float* Tu = at<float>(ws, p.off_tu);
    // recompute (checkpointing): gate(x), up(x) with their T = X A^T, h
    st = qlora_linear_forward(X, M, &mlp->gate, mlp->A_gate, mlp->B_gate, r, scale, G, Tg, w0, p.lin,
                              stream);
    if (st == QLORA_OK)
        st = qlora_linear_forward(X, M, &mlp->up, mlp->A_up, mlp->B_up, r, scale, U, Tu, w1, p.lin,
                                  stream);
    if (st != QLORA_OK) return st;
    QTRY(launch_swiglu_forward(G, U, H, M * p.F, num_sms(), s));
    // down: dH, dA_down, dB_down (its T recomputed from h)
    st = qlora_linear_backward(dY, H, M, &mlp->down, mlp->A_down, mlp->B_down, r, scale, nullptr, dH,
                               g->dA_down, g->dB_down, accumulate, w2, p.lin, stream);
    if (st != QLORA_OK) return st;
    // SwiGLU backward: (G, U) <- (dG, dU)
    QTRY(launch_swiglu_backward(G, U, dH, M * p.F, num_sms(), s));
    st = qlora_linear_backward(G, X, M, &mlp->gate, mlp->A_gate, mlp->B_gate, r, scale, Tg, dXg,
                               g->dA_gate, g->dB_gate, accumulate, w3, p.lin, stream);
    if (st == QLORA_OK)
        st = qlora_linear_backward(U, X, M, &mlp->up, mlp->A_up, mlp->B_up, r, scale, Tu, dX,
                                   g->dA_up, g->dB_up, accumulate, w4, p.lin, stream);
    if (st != QLORA_OK) return st;
    QTRY(launch_add_bf16(dX, dXg, dX, M * p.D, num_sms(), s));
    QTRY(launch_or_words(at<int>(ws, 0), at<int>(ws, p.off_lin[0]), at<int>(ws, p.off_lin[1]),
                         at<int>(ws, p.off_lin[2]), false, s));
    QTRY(launch_or_words(at<int>(ws, 0), at<int>(ws, p.off_lin[3]), at<int>(ws, p.off_lin[4]),
                         at<int>(ws, p.off_lin[4]), true, s));
    return QLORA_OK;
}

}  // extern "C"
