// quantize.cu -- NVFP4 quantize (bf16 -> E2M1 codes + E4M3 block scales +
// FP32 tensor scale) and the NVFP4 KV-cache append / dequant-gather.
//
// Format: "LongLive-2.0：用 NVFP4 并行底座做长视频生成" (yingwang.github.io
// reading note), section 二 方法 / "NVFP4 量化格式" (three-level scaling and
// the Dequant equation); KV store: same note, "推理底座" (per-frame-chunk K/V
// quantization, 9/8 * T_c * H * d bytes, dequant in a CUDA kernel) and the
// anzhuoshouzhuan.com article's in-place quantized KV-cache update.
//
// All kernels here are HBM-bandwidth bound.  Layout of the work:
//  * amax pass: 16-byte streaming loads, |x| max on the bf16 bit patterns
//    (two 16-bit lanes per 32-bit SIMD max), one partial per CTA -- no atomics
//    and no memset launch.
//  * encode pass: a warp owns a 512-element run of one row; lane i loads the
//    16-byte chunks i and i+32 (each warp-wide load is 512 contiguous bytes),
//    a block of 16 elements is a lane pair (one shuffle for the block amax),
//    and the 4-byte code stores of a warp are 128 contiguous bytes.
//  * dequant-gather: a warp owns 256 elements of a slot: 4-byte code loads,
//    16-byte bf16 stores (512 contiguous bytes per warp store).
#include "common.cuh"

namespace nvfp4 {

constexpr int kThreads = 256;
constexpr int kMaxPartials = 1024;  // amax partials per tensor (one per CTA)

// Workspace layout shared by quantize and kv_append:
//   [0, 16)        DevError
//   [256, 256+4K)  amax partials of tensor 0
//   [256+4K, ..)   amax partials of tensor 1
constexpr size_t kWsPartials = 256;
constexpr size_t kWsQuantize = kWsPartials + 2 * kMaxPartials * sizeof(float);

struct AmaxArgs {
    const uint8_t* x[2];
    int64_t rows, cols, ld;  // elements
    float* partials;         // [2][kMaxPartials]
};

// max of |bf16| over 8 values, on the bit patterns (exact for finite values)
__device__ __forceinline__ uint32_t absmax_bits8(const uint4& v) {
    const uint32_t m = 0x7FFF7FFFu;
    uint32_t a = __vmaxu2(v.x & m, v.y & m);
    uint32_t b = __vmaxu2(v.z & m, v.w & m);
    return __vmaxu2(a, b);
}

__global__ void __launch_bounds__(kThreads) amax_kernel(AmaxArgs a) {
    const uint8_t* base = a.x[blockIdx.y];
    const int64_t cpr = a.cols / 8;  // 16-byte chunks per row
    const int64_t total = a.rows * cpr;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    uint32_t m2 = 0;
    if (a.ld == a.cols) {
        for (; i + 3 * stride < total; i += 4 * stride) {
            uint4 v0 = ld_stream16(base + i * 16);
            uint4 v1 = ld_stream16(base + (i + stride) * 16);
            uint4 v2 = ld_stream16(base + (i + 2 * stride) * 16);
            uint4 v3 = ld_stream16(base + (i + 3 * stride) * 16);
            m2 = __vmaxu2(m2, __vmaxu2(__vmaxu2(absmax_bits8(v0), absmax_bits8(v1)),
                                       __vmaxu2(absmax_bits8(v2), absmax_bits8(v3))));
        }
        for (; i < total; i += stride) m2 = __vmaxu2(m2, absmax_bits8(ld_stream16(base + i * 16)));
    } else {
        for (; i < total; i += stride) {
            const int64_t r = i / cpr, c = i - r * cpr;
            m2 = __vmaxu2(m2, absmax_bits8(ld_stream16(base + (r * a.ld + c * 8) * 2)));
        }
    }
    uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ uint32_t red[kThreads / 32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t r = 0;
        for (int w = 0; w < kThreads / 32; w++) r = max(r, red[w]);
        a.partials[blockIdx.y * kMaxPartials + blockIdx.x] = __uint_as_float(r << 16);
    }
}

struct EncodeArgs {
    const uint8_t* x[2];
    uint8_t* codes[2];
    uint8_t* scales[2];
    float* gscale[2];        // a32: written (computed) or read (given)
    int64_t rows, cols, ld;  // elements
    const float* partials;   // [2][kMaxPartials] when computed
    int nparts;
    int given;
    int swizzled;
    int64_t tiles_c;         // ceil(cols / 64)
};

__global__ void __launch_bounds__(kThreads) encode_kernel(EncodeArgs a) {
    const int t = blockIdx.y;
    __shared__ float s_a32;
    if (threadIdx.x < 32) {
        float a32;
        if (a.given) {
            a32 = *a.gscale[t];
        } else {
            float m = 0.0f;
            for (int i = threadIdx.x; i < a.nparts; i += 32) m = fmaxf(m, a.partials[t * kMaxPartials + i]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
            a32 = __fdiv_rn(m, 2688.0f);  // a32 = amax / (6 * 448)
            if (blockIdx.x == 0 && threadIdx.x == 0) *a.gscale[t] = a32;
        }
        if (threadIdx.x == 0) s_a32 = a32;
    }
    __syncthreads();
    const float a32 = s_a32;

    const int lane = threadIdx.x & 31;
    const int64_t upr = (a.cols + 511) / 512;  // 512-element runs per row
    const int64_t units = a.rows * upr;
    const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
    const uint8_t* xb = a.x[t];
    uint8_t* cb = a.codes[t];
    uint8_t* sb = a.scales[t];
    const int64_t sc_row = a.cols / 16;

    for (int64_t unit = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); unit < units;
         unit += nwarps) {
        const int64_t r = unit / upr;
        const int64_t c0 = (unit - r * upr) * 512;
        const int64_t L = min((int64_t)512, a.cols - c0);
        const int nchunks = (int)(L / 8);
        const bool v0 = lane < nchunks, v1 = lane + 32 < nchunks;
        const uint8_t* row = xb + (r * a.ld + c0) * 2;
        uint4 q0 = make_uint4(0, 0, 0, 0), q1 = make_uint4(0, 0, 0, 0);
        if (v0) q0 = ld_stream16(row + lane * 16);
        if (v1) q1 = ld_stream16(row + (lane + 32) * 16);
        float f0[8], f1[8];
        bf16x8_to_f32(q0, f0);
        bf16x8_to_f32(q1, f1);
        float am0 = absmax8(f0), am1 = absmax8(f1);
        am0 = fmaxf(am0, __shfl_xor_sync(0xFFFFFFFFu, am0, 1));
        am1 = fmaxf(am1, __shfl_xor_sync(0xFFFFFFFFu, am1, 1));
        const BlockScale b0 = block_scale(am0, a32);
        const BlockScale b1 = block_scale(am1, a32);
        const uint32_t w0 = encode8(f0, b0.inv);
        const uint32_t w1 = encode8(f1, b1.inv);
        uint8_t* crow = cb + r * (a.cols / 2) + c0 / 2;
        if (v0) *reinterpret_cast<uint32_t*>(crow + 4 * lane) = w0;
        if (v1) *reinterpret_cast<uint32_t*>(crow + 128 + 4 * lane) = w1;
        // even lanes store the scale of their first-half block, odd lanes the
        // scale of their second-half block
        const bool odd = lane & 1;
        const bool vs = odd ? v1 : v0;
        if (vs) {
            const int64_t bj = c0 / 16 + (odd ? 16 : 0) + (lane >> 1);
            const uint8_t code = (uint8_t)(odd ? b1.code : b0.code);
            if (a.swizzled)
                sb[swz_offset(r, bj, a.tiles_c)] = code;
            else
                sb[r * sc_row + bj] = code;
        }
    }

    // zero the padding rows of the swizzled scale tiles (cols % 64 == 0, so
    // only rows past `rows` up to the next multiple of 128 are padding)
    if (a.swizzled) {
        const int64_t rows_pad = (a.rows + 127) / 128 * 128;
        const int64_t sc_pad = a.tiles_c * 4;
        const int64_t npad = (rows_pad - a.rows) * sc_pad;
        for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < npad; i += (int64_t)gridDim.x * kThreads) {
            const int64_t r = a.rows + i / sc_pad, c = i % sc_pad;
            sb[swz_offset(r, c, a.tiles_c)] = 0;
        }
    }
}

struct DequantArgs {
    const uint8_t* codes[2];
    const uint8_t* scales[2];
    const float* gscale[2];  // [n_slots]
    uint8_t* out[2];         // bf16
    const int32_t* slots;
    int32_t n;
    int32_t n_slots;
    int64_t slot_elems;      // T * H * d
    DevError* err;
};

__global__ void __launch_bounds__(kThreads) kv_dequant_kernel(DequantArgs a) {
    const int t = blockIdx.y;
    const int lane = threadIdx.x & 31;
    const int64_t ups = (a.slot_elems + 255) / 256;  // 256-element runs per slot
    const int64_t units = (int64_t)a.n * ups;
    const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
    const uint8_t* cb = a.codes[t];
    const uint8_t* sb = a.scales[t];
    uint8_t* ob = a.out[t];
    for (int64_t unit = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); unit < units;
         unit += nwarps) {
        const int64_t i = unit / ups;
        const int64_t u = unit - i * ups;
        const int32_t s = __ldg(a.slots + i);
        if (s < 0 || s >= a.n_slots) {
            if (lane == 0 && u == 0 && t == 0) record_error(a.err, NVFP4_ERR_DEVICE, (uint32_t)i);
            continue;
        }
        const int64_t e0 = u * 256 + 8 * lane;
        if (e0 >= a.slot_elems) continue;
        const int64_t sbase = (int64_t)s * a.slot_elems;
        const uint32_t q = __ldg(reinterpret_cast<const uint32_t*>(cb + (sbase + e0) / 2));
        const uint8_t sc = __ldg(sb + (sbase + e0) / 16);
        const float a32 = __ldg(a.gscale[t] + s);
        const __half2 s2 = e4m3x2_to_half2((uint16_t)(sc | (sc << 8)));
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const __half2 v = __hmul2(e2m1x2_to_half2((q >> (8 * j)) & 0xFFu), s2);  // exact
            const float2 f = __half22float2(v);
            const __nv_bfloat162 b = __floats2bfloat162_rn(__fmul_rn(f.x, a32), __fmul_rn(f.y, a32));
            o[j] = *reinterpret_cast<const uint32_t*>(&b);
        }
        *reinterpret_cast<uint4*>(ob + ((int64_t)i * a.slot_elems + e0) * 2) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// Test support: run the device encoders on arbitrary binary32 inputs.
__global__ void encoder_probe_kernel(const float* x, int64_t n, uint8_t* e2m1, uint8_t* e4m3) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float v = x[i];
        if (e2m1) {
            float y[8] = {v, 0, 0, 0, 0, 0, 0, 0};
            e2m1[i] = (uint8_t)(e2m1x8(y) & 0xFu);
        }
        if (e4m3) e4m3[i] = (uint8_t)e4m3_code(v);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static int g_sms = 0;

static int num_sms() {
    if (g_sms == 0) {
        int dev = 0, n = 0;
        if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
            g_sms = n;
        else
            return 148;
    }
    return g_sms;
}

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int grid_for(int64_t work_items, int per_cta, int cap) {
    int64_t g = (work_items + per_cta - 1) / per_cta;
    if (g < 1) g = 1;
    if (g > cap) g = cap;
    return (int)g;
}

static nvfp4_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// amax + encode over one or two tensors of the same shape
static nvfp4_status quantize_impl(int ntensors, const void* const* x, int64_t rows, int64_t cols, int64_t ld,
                                  void* const* codes, void* const* scales, float* const* gscale, bool given,
                                  bool swizzled, void* workspace, cudaStream_t stream) {
    const int sms = num_sms();
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* partials = reinterpret_cast<float*>(ws + kWsPartials);
    int nparts = 0;
    const int64_t chunks = rows * (cols / 8);
    if (!given) {
        AmaxArgs aa{};
        for (int t = 0; t < ntensors; t++) aa.x[t] = static_cast<const uint8_t*>(x[t]);
        aa.rows = rows;
        aa.cols = cols;
        aa.ld = ld;
        aa.partials = partials;
        nparts = grid_for(chunks, kThreads * 8, std::min(kMaxPartials, sms * 4));
        amax_kernel<<<dim3(nparts, ntensors), kThreads, 0, stream>>>(aa);
        if (launch_status() != NVFP4_OK) return NVFP4_ERR_CUDA;
    }
    EncodeArgs ea{};
    for (int t = 0; t < ntensors; t++) {
        ea.x[t] = static_cast<const uint8_t*>(x[t]);
        ea.codes[t] = static_cast<uint8_t*>(codes[t]);
        ea.scales[t] = static_cast<uint8_t*>(scales[t]);
        ea.gscale[t] = gscale[t];
    }
    ea.rows = rows;
    ea.cols = cols;
    ea.ld = ld;
    ea.partials = partials;
    ea.nparts = nparts;
    ea.given = given ? 1 : 0;
    ea.swizzled = swizzled ? 1 : 0;
    ea.tiles_c = (cols + 63) / 64;
    const int64_t units = rows * ((cols + 511) / 512);
    const int g = grid_for(units, kThreads / 32, sms * 8);
    encode_kernel<<<dim3(g, ntensors), kThreads, 0, stream>>>(ea);
    return launch_status();
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status nvfp4_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld, void* codes,
                                       void* scales, float* global_scale, unsigned flags, void* workspace,
                                       size_t ws_bytes, nvfp4_stream_t stream) {
    if (flags & ~(NVFP4_Q_GIVEN_GLOBAL | NVFP4_Q_ROWMAJOR_SCALES)) return NVFP4_ERR_INVALID_ARG;
    if (rows < 0 || cols <= 0 || ld < cols) return NVFP4_ERR_INVALID_ARG;
    if (cols % 64 != 0) return NVFP4_ERR_UNSUPPORTED;
    if (rows > ((int64_t)1 << 31) || cols > ((int64_t)1 << 31)) return NVFP4_ERR_UNSUPPORTED;
    if (!global_scale || !workspace) return NVFP4_ERR_INVALID_ARG;
    if (ws_bytes < nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, rows, 0, cols)) return NVFP4_ERR_INVALID_ARG;
    if (rows == 0) return NVFP4_OK;
    if (!x_bf16 || !codes || !scales) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scales) || (ld % 8) != 0 ||
        (reinterpret_cast<uintptr_t>(global_scale) & 3u) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return NVFP4_ERR_MISALIGNED;
    const void* xs[1] = {x_bf16};
    void* cs[1] = {codes};
    void* ss[1] = {scales};
    float* gs[1] = {global_scale};
    return quantize_impl(1, xs, rows, cols, ld, cs, ss, gs, (flags & NVFP4_Q_GIVEN_GLOBAL) != 0,
                         (flags & NVFP4_Q_ROWMAJOR_SCALES) == 0, workspace, (cudaStream_t)stream);
}

static nvfp4_status check_cache(const nvfp4_kv_cache* c) {
    if (!c) return NVFP4_ERR_INVALID_ARG;
    if (!c->k_codes || !c->k_scales || !c->v_codes || !c->v_scales || !c->k_global || !c->v_global)
        return NVFP4_ERR_INVALID_ARG;
    if (c->n_slots <= 0 || c->tokens_per_slot <= 0 || c->heads <= 0 || c->head_dim <= 0) return NVFP4_ERR_INVALID_ARG;
    if (c->head_dim % 16 != 0) return NVFP4_ERR_UNSUPPORTED;
    const int64_t e = (int64_t)c->tokens_per_slot * c->heads * c->head_dim;
    if (e % 64 != 0 || e > ((int64_t)1 << 40)) return NVFP4_ERR_UNSUPPORTED;
    if (!aligned16(c->k_codes) || !aligned16(c->k_scales) || !aligned16(c->v_codes) || !aligned16(c->v_scales) ||
        (reinterpret_cast<uintptr_t>(c->k_global) & 3u) || (reinterpret_cast<uintptr_t>(c->v_global) & 3u))
        return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

extern "C" nvfp4_status nvfp4_kv_append(const nvfp4_kv_cache* cache, int32_t slot, const void* k_bf16,
                                        const void* v_bf16, void* workspace, size_t ws_bytes, nvfp4_stream_t stream) {
    nvfp4_status st = check_cache(cache);
    if (st != NVFP4_OK) return st;
    if (slot < 0 || slot >= cache->n_slots) return NVFP4_ERR_INVALID_ARG;
    if (!k_bf16 || !v_bf16 || !workspace) return NVFP4_ERR_INVALID_ARG;
    const int64_t rows = (int64_t)cache->tokens_per_slot * cache->heads;
    const int64_t e = rows * cache->head_dim;
    if (ws_bytes < nvfp4_workspace_bytes(NVFP4_OP_KV_APPEND, rows, 0, cache->head_dim)) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(k_bf16) || !aligned16(v_bf16) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return NVFP4_ERR_MISALIGNED;
    // The chunk is quantized as one flat row of T*H*d elements: with
    // row-major scales over rows of head_dim this is the same byte layout.
    const void* xs[2] = {k_bf16, v_bf16};
    void* cs[2] = {static_cast<uint8_t*>(cache->k_codes) + (int64_t)slot * (e / 2),
                   static_cast<uint8_t*>(cache->v_codes) + (int64_t)slot * (e / 2)};
    void* ss[2] = {static_cast<uint8_t*>(cache->k_scales) + (int64_t)slot * (e / 16),
                   static_cast<uint8_t*>(cache->v_scales) + (int64_t)slot * (e / 16)};
    float* gs[2] = {cache->k_global + slot, cache->v_global + slot};
    return quantize_impl(2, xs, 1, e, e, cs, ss, gs, false, false, workspace, (cudaStream_t)stream);
}

extern "C" nvfp4_status nvfp4_kv_dequant(const nvfp4_kv_cache* cache, const int32_t* slots_dev, int32_t n,
                                         void* k_out_bf16, void* v_out_bf16, void* workspace, size_t ws_bytes,
                                         nvfp4_stream_t stream) {
    nvfp4_status st = check_cache(cache);
    if (st != NVFP4_OK) return st;
    if (n < 0 || !workspace) return NVFP4_ERR_INVALID_ARG;
    if (ws_bytes < nvfp4_workspace_bytes(NVFP4_OP_KV_DEQUANT, 0, 0, 0)) return NVFP4_ERR_INVALID_ARG;
    if (n == 0) return NVFP4_OK;
    if (!slots_dev || !k_out_bf16 || !v_out_bf16) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(k_out_bf16) || !aligned16(v_out_bf16) || (reinterpret_cast<uintptr_t>(slots_dev) & 3u) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return NVFP4_ERR_MISALIGNED;
    DequantArgs a{};
    a.codes[0] = static_cast<const uint8_t*>(cache->k_codes);
    a.codes[1] = static_cast<const uint8_t*>(cache->v_codes);
    a.scales[0] = static_cast<const uint8_t*>(cache->k_scales);
    a.scales[1] = static_cast<const uint8_t*>(cache->v_scales);
    a.gscale[0] = cache->k_global;
    a.gscale[1] = cache->v_global;
    a.out[0] = static_cast<uint8_t*>(k_out_bf16);
    a.out[1] = static_cast<uint8_t*>(v_out_bf16);
    a.slots = slots_dev;
    a.n = n;
    a.n_slots = cache->n_slots;
    a.slot_elems = (int64_t)cache->tokens_per_slot * cache->heads * cache->head_dim;
    a.err = static_cast<DevError*>(workspace);
    const int64_t units = (int64_t)n * ((a.slot_elems + 255) / 256);
    const int g = grid_for(units, kThreads / 32, num_sms() * 8);
    kv_dequant_kernel<<<dim3(g, 2), kThreads, 0, (cudaStream_t)stream>>>(a);
    return launch_status();
}

extern "C" nvfp4_status nvfp4_test_encode(const float* x, int64_t n, uint8_t* e2m1_out, uint8_t* e4m3_out,
                                          nvfp4_stream_t stream) {
    if (n < 0 || (n > 0 && !x) || (!e2m1_out && !e4m3_out)) return NVFP4_ERR_INVALID_ARG;
    if (n == 0) return NVFP4_OK;
    const int g = grid_for(n, 256, num_sms() * 16);
    encoder_probe_kernel<<<g, 256, 0, (cudaStream_t)stream>>>(x, n, e2m1_out, e4m3_out);
    return launch_status();
}
