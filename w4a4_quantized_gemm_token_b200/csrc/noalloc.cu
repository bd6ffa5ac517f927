// w4a4_linear_noalloc: the fused linear layer with its scratch in a
// file-scope device array of this library instead of a caller workspace.
//
// Who needs it: a caller that holds no device allocator of its own (a plain
// C host program that drives one layer, a runtime whose device memory plan
// is fixed before the layer is chosen) and so cannot provide the workspace
// w4a4_linear asks for.  The scratch is this library's static device memory:
// W4A4_NOALLOC_SCRATCH_BYTES per device, reserved when the library's module
// is loaded on that device.  Nothing here calls cudaMalloc, cudaFree or any
// allocating library routine.
//
// Set-up: the first call in a CUDA context (with its device current) looks up
// the array's device address there (cudaGetSymbolAddress) and caches it for
// that context; make that first call before any stream capture.  The array is
// per module and context, so a caller that drives its own driver-API context
// or re-creates the primary context (cudaDeviceReset) gets the address of the
// copy in the context that is current at the call.
//
// Zero state: no byte of the scratch has to start at zero.  Every byte a
// call reads is written earlier in the same call (quantized activation codes
// and scales, the FP32 second-level scales, the split-K partial sums), and
// the TENSOR-mode amax slot is cleared by the call itself.
//
// Races: one scratch per device, shared by every call on that device.  Two
// calls whose kernels can run at the same time (different streams without an
// ordering between them, or several host threads) overwrite each other's
// scratch; such calls must be ordered (one stream, or events).
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/w4a4.h"

namespace {

static __device__ __align__(256) unsigned char g_linear_scratch[W4A4_NOALLOC_SCRATCH_BYTES];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// A few cached (context, address) pairs; a context not among them is looked up
// (and replaces the oldest entry).
constexpr int kSlots = 64;
struct Slot {
    CUcontext ctx;
    void* ptr;
};
std::mutex g_scratch_mutex;
Slot g_slots[kSlots] = {};
int g_next_slot = 0;
CtxGetCurrentFn g_ctx_get_current = nullptr;

// Device address of g_linear_scratch in the current context.
int scratch_for_current_context(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return W4A4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_ctx_get_current) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return W4A4_ERR_CUDA;
        g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    }
    CUcontext ctx = nullptr;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return W4A4_ERR_CUDA;
    if (ctx)
        for (int i = 0; i < kSlots; ++i)
            if (g_slots[i].ctx == ctx) {
                *out = g_slots[i].ptr;
                return W4A4_OK;
            }
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return W4A4_ERR_CUDA;
    if (major != 10) return W4A4_ERR_ARCH;
    // (with no context current yet, this runtime call makes the device's
    // primary context current)
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_linear_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return W4A4_ERR_CUDA;
    }
    if (!ctx && (g_ctx_get_current(&ctx) != CUDA_SUCCESS || !ctx)) return W4A4_ERR_CUDA;
    g_slots[g_next_slot] = Slot{ctx, p};
    g_next_slot = (g_next_slot + 1) % kSlots;
    *out = p;
    return W4A4_OK;
}

}  // namespace

extern "C" int w4a4_linear_noalloc(const uint16_t* X, int M, int K, int ldx, const w4a4_qtensor* Wq, int scale_mode,
                                   const int32_t* S, int nS, uint16_t* Y, int ldy, void* stream) {
    if (!Wq) return W4A4_ERR_INVALID_ARG;
    // bad arguments give 0 here and are reported by w4a4_linear below
    const size_t need = w4a4_linear_workspace(M, Wq->rows, K, Wq->format, nS);
    if (need > (size_t)W4A4_NOALLOC_SCRATCH_BYTES) return W4A4_ERR_WORKSPACE;
    void* scratch = nullptr;
    const int rc = scratch_for_current_context(&scratch);
    if (rc != W4A4_OK) return rc;
    return w4a4_linear(X, M, K, ldx, Wq, scale_mode, S, nS, Y, ldy, scratch, (size_t)W4A4_NOALLOC_SCRATCH_BYTES,
                       stream);
}
