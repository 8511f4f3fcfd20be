// qlora_linear_forward_noalloc: the forward of the adapted layer for callers
// that cannot allocate device memory at all.
//
// Who needs it: code that runs inside a host framework which owns every
// device allocation and offers no allocator handle to plug-ins, and
// deployments that forbid any device allocation after start-up (fixed memory
// budgets, certified or real-time runtimes).  Such callers cannot provide the
// workspace that qlora_linear_forward asks for, because providing it means
// allocating it.
//
// How: the scratch lives in one file-scope device array of this library,
// kNoAllocScratchBytes (16 MiB) on every GPU that loads the library, held
// until the process exits.  Host code cannot use the array's name as a
// device address (on the host it is only a stand-in symbol), so the first
// call on each device looks the address up with cudaGetSymbolAddress while
// that device is current, checks the result and caches it; later calls on
// that device reuse it.  The call then runs the ordinary forward with that
// array as its workspace.  The forward path zeroes the only part of the
// workspace that must start at zero (its error word) and overwrites the
// rest, so the contents left by the previous call do no harm.  All calls on
// a device share the one array: calls that can overlap on the GPU (different
// streams with no ordering between them) race on it and must not be issued.
//
// The ordinary forward reports kernel-side failures (a bounded wait that
// expired, a shared-memory plan or tile schedule that did not fit) in the
// first 4 bytes of the caller's workspace.  Here that word lives in the
// library's array, which the caller cannot address, so
// qlora_linear_forward_noalloc_error_word copies it out.
#include <mutex>

#include "kernels.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB per device

__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];
cudaError_t g_scratch_status[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];

// Device address of g_noalloc_scratch on the current device (set-up on the
// first call per device, with that device current).
int scratch_on_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return QLORA_ERR_UNSUPPORTED;
    std::call_once(g_scratch_once[dev], [dev] {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        g_scratch_status[dev] = e;
        g_scratch_addr[dev] = (e == cudaSuccess) ? p : nullptr;
    });
    if (g_scratch_status[dev] != cudaSuccess || g_scratch_addr[dev] == nullptr)
        return QLORA_ERR_CUDA;
    *out = g_scratch_addr[dev];
    return QLORA_OK;
}

}  // namespace

extern "C" QLORA_API int qlora_linear_forward_noalloc(const uint16_t* X, int64_t M,
                                                      const qlora_nf4_tensor* w,
                                                      const uint16_t* A, const uint16_t* B, int r,
                                                      float scale, uint16_t* Y, float* T_save,
                                                      qlora_stream_t stream) {
    if (!w) return QLORA_ERR_NULL;
    size_t need = 0;
    int st = qlora_linear_workspace_size(M, w->rows, w->cols, r, &need);
    if (st != QLORA_OK) return st;
    if (need > kNoAllocScratchBytes) return QLORA_ERR_WORKSPACE;   // beyond the fixed array
    void* ws = nullptr;
    st = scratch_on_current_device(&ws);
    if (st != QLORA_OK) return st;
    return qlora_linear_forward(X, M, w, A, B, r, scale, Y, T_save, ws, kNoAllocScratchBytes,
                                stream);
}

extern "C" QLORA_API int qlora_linear_forward_noalloc_error_word(int* h_word,
                                                                qlora_stream_t stream) {
    if (!h_word) return QLORA_ERR_NULL;
    void* ws = nullptr;
    const int st = scratch_on_current_device(&ws);
    if (st != QLORA_OK) return st;
    return cudaMemcpyAsync(h_word, ws, sizeof(int), cudaMemcpyDeviceToHost,
                           reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? QLORA_OK
               : QLORA_ERR_CUDA;
}
