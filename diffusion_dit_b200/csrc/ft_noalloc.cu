// fourtune_quantize_block16_noalloc: the block quantizer (with its optional fused
// down-projection) for callers that must not allocate device memory.
//
// Some hosts cannot call cudaMalloc: a plugin interface that hands the library only
// its input and output buffers, or a process whose device memory is budgeted and
// owned by another runtime from start-up on.  This entry point takes the scratch the
// quantizer needs (status word, tensor max, padded down factor, per-slice partial sums)
// from a fixed array in the library's own device memory instead of a caller workspace.
#include <cudaTypedefs.h>

#include <mutex>

#include "fourtune.h"
#include "ft_internal.h"

namespace {

// Every GPU that loads the library holds this array until the process exits.  Device
// memory is zero at module load, so the status word (its first bytes) starts at FT_OK.
constexpr size_t kScratchBytes = FT_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the array, looked up once per device and CUDA context: the symbol
// is only a host-side stand-in, and a new context (after cudaDeviceReset, say) loads
// the module again at another address, so the cache is keyed on the context's
// process-unique id.
struct ScratchAddr {
    unsigned long long ctx_id = 0;
    void* ptr = nullptr;
};
std::mutex g_mu;
ScratchAddr g_addr[64];

struct CtxFns {
    PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    PFN_cuCtxGetId_v12000 get_id = nullptr;
};

const CtxFns& ctx_fns() {
    static CtxFns f;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            f.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            f.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    return f;
}

// Id of the context current on this thread, 0 if none is current or it cannot be read.
unsigned long long current_ctx_id() {
    const CtxFns& f = ctx_fns();
    if (!f.get_current || !f.get_id) return 0;
    CUcontext ctx = nullptr;
    if (f.get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

}  // namespace

namespace ft {

ft_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FT_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    ScratchAddr& a = g_addr[dev];
    const unsigned long long id = current_ctx_id();
    if (!a.ptr || id == 0 || id != a.ctx_id) {
        // Set-up (the device is current): host code needs the array's device address.
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FT_ERR_CUDA;
        a.ptr = p;
        a.ctx_id = current_ctx_id();  // the lookup has made the runtime's context current
    }
    *out = a.ptr;
    return FT_OK;
}

}  // namespace ft

extern "C" ft_status fourtune_quantize_block16_noalloc(const void* x_dev, int32_t x_dtype, int64_t rows,
                                                       int64_t cols, int64_t ld, const float* amax_or_null,
                                                       const void* down_dev, int32_t r_down, float* down_out_dev,
                                                       const ft_fp4* out, const ft_fp4* out_t, void* stream) {
    if (rows < 0 || cols < 0 || r_down < 0) return FT_ERR_INVALID_ARG;
    const size_t need = fourtune_quantize_workspace_bytes(rows, cols, r_down);
    if (need > kScratchBytes) return FT_ERR_WORKSPACE;  // beyond the fixed scratch array
    void* scratch = nullptr;
    const ft_status s = ft::noalloc_scratch(&scratch);
    if (s != FT_OK) return s;
    // The status word at the start of the array is sticky, as in a caller workspace: the
    // kernels only ever set it, and fourtune_device_status(NULL, ...) reads and clears it.
    // The tensor-max slot is cleared by the call's own kernels, and the other regions are
    // fully written before they are read, so nothing left by an earlier call leaks in.
    return fourtune_quantize_block16(x_dev, x_dtype, rows, cols, ld, amax_or_null, down_dev, r_down,
                                     down_out_dev, out, out_t, scratch, kScratchBytes, stream);
}
