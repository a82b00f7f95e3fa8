// fourtune_quantize_block16_noalloc: the block quantizer (with its optional fused
// down-projection) for callers that must not allocate device memory.
//
// Some hosts cannot call cudaMalloc: a plugin interface that hands the library only
// its input and output buffers, or a process whose device memory is budgeted and
// owned by another runtime from start-up on.  This entry point takes the scratch the
// quantizer needs (status word, tensor max, padded down factor, per-slice partial sums)
// from a fixed array in the library's own device memory instead of a caller workspace.
#include <mutex>

#include "fourtune.h"

namespace {

// Every GPU that loads the library holds this array until the process exits.
constexpr size_t kScratchBytes = FT_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[64] = {};  // device address of the array, per device (set up once)

}  // namespace

extern "C" ft_status fourtune_quantize_block16_noalloc(const void* x_dev, int32_t x_dtype, int64_t rows,
                                                       int64_t cols, int64_t ld, const float* amax_or_null,
                                                       const void* down_dev, int32_t r_down, float* down_out_dev,
                                                       const ft_fp4* out, const ft_fp4* out_t, void* stream) {
    if (rows < 0 || cols < 0 || r_down < 0) return FT_ERR_INVALID_ARG;
    const size_t need = fourtune_quantize_workspace_bytes(rows, cols, r_down);
    if (need > kScratchBytes) return FT_ERR_WORKSPACE;  // beyond the fixed scratch array
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FT_ERR_CUDA;
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_scratch_ptr[dev]) {
            // First call on this device (the device is current): host code needs the
            // array's device address; the symbol itself is only a host-side stand-in.
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FT_ERR_CUDA;
            g_scratch_ptr[dev] = p;
        }
        scratch = g_scratch_ptr[dev];
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents: clear the status word the kernels
    // report through (the other regions are fully written before they are read).
    if (cudaMemsetAsync(scratch, 0, 256, st) != cudaSuccess) return FT_ERR_CUDA;
    return fourtune_quantize_block16(x_dev, x_dtype, rows, cols, ld, amax_or_null, down_dev, r_down,
                                     down_out_dev, out, out_t, scratch, kScratchBytes, stream);
}
