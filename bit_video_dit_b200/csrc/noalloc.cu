// noalloc.cu -- nvfp4_quantize_noalloc: nvfp4_quantize for callers that may
// not allocate device memory (no workspace argument).
//
// The fused quantize kernel needs a little device scratch besides its inputs
// and outputs: its error record and grid-barrier words (a 256-byte block).
// Here that scratch is one file-scope __device__ array instead of a caller
// workspace.  Every GPU that loads the library holds the array until the
// process exits.
#include <mutex>

#include "common.cuh"

namespace {

// Largest scratch the no-allocation quantize can use (the fused kernel's
// control block).  Problems whose workspace would be larger are rejected.
constexpr size_t kNoAllocScratchBytes = NVFP4_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name only stands in for it: it is not a device pointer, and a
// kernel given it would fault (or, where the GPU can reach host memory, use
// the wrong memory).  The address is looked up once per device, with that
// device current.
nvfp4_status scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return NVFP4_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                               void* codes, void* scales, float* global_scale, unsigned flags,
                                               nvfp4_stream_t stream) {
    // every argument check first: a rejected call puts nothing on the stream
    // and leaves the shared array alone (another stream may be using it)
    const nvfp4_status chk = nvfp4::quantize_check_args(x_bf16, rows, cols, ld, codes, scales, global_scale, flags);
    if (chk != NVFP4_OK) return chk;
    if (rows == 0) return NVFP4_OK;
    if (nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, rows, 0, cols) > kNoAllocScratchBytes) return NVFP4_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    const nvfp4_status st = scratch_for_current_device(&scratch);
    if (st != NVFP4_OK) return st;
    // the array keeps whatever the previous call left: start from zero
    if (cudaMemsetAsync(scratch, 0, kNoAllocScratchBytes, (cudaStream_t)stream) != cudaSuccess) return NVFP4_ERR_CUDA;
    return nvfp4_quantize(x_bf16, rows, cols, ld, codes, scales, global_scale, flags, scratch, kNoAllocScratchBytes,
                          stream);
}
