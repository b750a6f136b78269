// api.cu -- size queries, status strings and the device error read-back of
// libnvfp4 (host code only).
#include "common.cuh"

namespace {
// Every call's workspace starts with a 256-byte control block: the device
// error record (bytes 0..15) and, for quantize / KV append, the fused
// kernel's grid-barrier words (the launch epoch at word 8, the two arrival
// counters at words 16..17, the per-parity tensor maxima at words 20..23).
// Nothing follows the block for those calls: their whole workspace is 256
// bytes, which is also what the no-allocation quantize keeps in its static
// array.  The LayerNorm quantize keeps its row statistics after the block.
constexpr size_t kWsControl = 256;
constexpr size_t kWsQuantize = kWsControl;
}

extern "C" const char* nvfp4_status_string(nvfp4_status s) {
    switch (s) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_INVALID_ARG: return "invalid argument";
        case NVFP4_ERR_UNSUPPORTED: return "unsupported shape or device";
        case NVFP4_ERR_MISALIGNED: return "pointer or leading dimension not 16-byte aligned";
        case NVFP4_ERR_CUDA: return "CUDA runtime or driver error";
        case NVFP4_ERR_TIMEOUT: return "bounded device-side wait ran out";
        case NVFP4_ERR_DEVICE: return "device-detected error";
    }
    return "unknown status";
}

extern "C" int nvfp4_version(void) { return (1 << 16) | 0; }

extern "C" size_t nvfp4_codes_bytes(int64_t rows, int64_t cols) {
    if (rows < 0 || cols < 0 || (cols & 1)) return 0;
    return (size_t)(rows * (cols / 2));
}

extern "C" size_t nvfp4_scales_bytes(int64_t rows, int64_t cols, int swizzled) {
    if (rows < 0 || cols < 0 || cols % 16 != 0) return 0;
    if (!swizzled) return (size_t)(rows * (cols / 16));
    const int64_t rp = (rows + 127) / 128 * 128;
    const int64_t cp = (cols + 63) / 64 * 4;
    return (size_t)(rp * cp);
}

extern "C" size_t nvfp4_workspace_bytes(int op, int64_t m, int64_t n, int64_t k) {
    (void)n;
    (void)k;
    switch (op) {
        case NVFP4_OP_QUANTIZE:
        case NVFP4_OP_KV_APPEND: return kWsQuantize;
        case NVFP4_OP_GEMM:
        case NVFP4_OP_KV_DEQUANT:
        case NVFP4_OP_QUANTIZE_2D:  // error record, then the amax word at byte 128
        case NVFP4_OP_QUANTIZE_T:
        case NVFP4_OP_KV_ATTENTION: return kWsControl;
        case NVFP4_OP_LN_QUANTIZE:  // control block, then (mean, rstd) per row
            return kWsControl + (size_t)(m > 0 ? m : 0) * 8;
    }
    return kWsQuantize;
}

extern "C" nvfp4_status nvfp4_read_device_error(void* workspace, nvfp4_stream_t stream, int* code, uint32_t* info) {
    if (!workspace || !code) return NVFP4_ERR_INVALID_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return NVFP4_ERR_CUDA;
    nvfp4::DevError e;
    if (cudaMemcpy(&e, workspace, sizeof e, cudaMemcpyDeviceToHost) != cudaSuccess) return NVFP4_ERR_CUDA;
    // after an error the whole control block is reset (a wait that ran out
    // may have left the grid-barrier words of the fused quantize mid-way)
    const size_t n = e.code ? kWsControl : sizeof e;
    if (cudaMemset(workspace, 0, n) != cudaSuccess) return NVFP4_ERR_CUDA;
    *code = (int)e.code;
    if (info) *info = e.info;
    return NVFP4_OK;
}
