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
//  * quantize / KV append: one cooperative launch (see quantize_fused_kernel):
//    bulk copies into shared memory, |x| max on the bf16 bit patterns (two
//    16-bit lanes per 32-bit SIMD max), a bounded grid barrier for the tensor
//    scale, then the encode from shared memory.  In the encode a warp owns a
//    512-element run of one row; lane i holds the 16-byte chunks i and i+32,
//    a block of 16 elements is a lane pair (one shuffle for the block amax),
//    and a warp's 4-byte code stores are 128 contiguous bytes.
//  * dequant-gather: a warp owns 512-element runs of a slot; lane i decodes
//    elements 8i..8i+7 and 256+8i..256+8i+7 (4-byte code loads, 16-byte bf16
//    stores, each warp-wide access contiguous), two runs in flight per lane.
#include <algorithm>

#include "common.cuh"

namespace nvfp4 {

constexpr int kThreads = 256;  // dequant / probe kernels

// ---------------------------------------------------------------------------
// Fused quantize: one cooperative launch, one CTA per SM.
//   phase 1  every CTA bulk-copies (cp.async.bulk, no registers involved) its
//            contiguous share of 512-element row runs into shared memory and
//            takes the |x| max of it;
//   barrier  the CTA maxima meet in one atomicMax word per tensor; the last
//            CTA to arrive turns it into a32 = amax / 2688 and releases the
//            grid (bounded wait everywhere else);
//   phase 2  every CTA encodes its runs straight from shared memory.
// HBM is read once and written once.  Runs that do not fit in shared memory
// (tensors larger than ~#SMs x 200 KB) are read from global memory in both
// phases instead.
// ---------------------------------------------------------------------------
constexpr int kQThreads = 512;
constexpr int kQWarps = kQThreads / 32;
constexpr int kRunBytes = 1024;  // one 512-element bf16 run

// Control block in the first 256 bytes of the workspace (zero before first use).
constexpr int kCtlCount = 8;   // uint32 index: CTAs arrived at the grid barrier
constexpr int kCtlGen = 9;     // barrier generation
constexpr int kCtlAmax = 10;   // [2] bf16 magnitude bit patterns, reset by the releasing CTA
constexpr int kCtlAlpha = 12;  // [2] a32 bits

struct QuantArgs {
    const uint8_t* x[2];
    uint8_t* codes[2];
    uint8_t* scales[2];
    float* gscale[2];
    int64_t rows, cols, ld;   // per tensor, elements
    int64_t upr;              // 512-element runs per row
    int64_t runs_per_tensor;
    int64_t total_runs;       // ntensors * runs_per_tensor
    int given;
    int swizzled;
    int64_t tiles_c;          // ceil(cols / 64)
    int cap;                  // runs cached in shared memory per CTA
    uint32_t* ctl;
    DevError* err;
    uint64_t limit_ns;
};

// max of |bf16| over 8 values, on the bit patterns (two 16-bit lanes per
// 32-bit SIMD max; exact for finite values)
__device__ __forceinline__ uint32_t absmax_bits8(const uint4& v) {
    const uint32_t m = 0x7FFF7FFFu;
    const uint32_t a = __vmaxu2(v.x & m, v.y & m);
    const uint32_t b = __vmaxu2(v.z & m, v.w & m);
    return __vmaxu2(a, b);
}

struct Run {
    int t;            // tensor
    int64_t r, c0;    // row, first column
    int nchunks;      // valid 16-byte chunks (L / 8)
};

__device__ __forceinline__ Run run_of(const QuantArgs& a, int64_t g) {
    Run u;
    u.t = g >= a.runs_per_tensor ? 1 : 0;
    const int64_t gl = g - (u.t ? a.runs_per_tensor : 0);
    u.r = gl / a.upr;
    u.c0 = (gl - u.r * a.upr) * 512;
    u.nchunks = (int)(min((int64_t)512, a.cols - u.c0) / 8);
    return u;
}

__device__ __forceinline__ const uint8_t* run_src(const QuantArgs& a, const Run& u) {
    return (u.t ? a.x[1] : a.x[0]) + (u.r * a.ld + u.c0) * 2;
}

__global__ void __launch_bounds__(kQThreads, 1) quantize_fused_kernel(const __grid_constant__ QuantArgs a) {
    extern __shared__ __align__(128) uint8_t qsmem[];
    uint4* cache = reinterpret_cast<uint4*>(qsmem);  // [cap][64]
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ uint32_t s_red[2][kQWarps];
    __shared__ float s_alpha[2];
    __shared__ int s_ok;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t G = gridDim.x;
    const int64_t begin = a.total_runs * (int64_t)blockIdx.x / G;
    const int64_t end = a.total_runs * ((int64_t)blockIdx.x + 1) / G;
    const int64_t ncached = min(end - begin, (int64_t)a.cap);

    // ---- phase 1: bulk-copy this CTA's runs into shared memory
    if (threadIdx.x == 0) {
        mbar_init(&s_bar, 1);
        fence_barrier_init();
        fence_proxy_async_smem();
        s_ok = 1;
    }
    __syncthreads();
    {
        // every thread announces its own bytes, then issues its copies; the
        // single arrival comes after all announcements (the __syncthreads)
        uint32_t mine = 0;
        for (int64_t l = threadIdx.x; l < ncached; l += kQThreads) mine += (uint32_t)run_of(a, begin + l).nchunks * 16u;
        if (mine) mbar_expect_tx_only(&s_bar, mine);
        for (int64_t l = threadIdx.x; l < ncached; l += kQThreads) {
            const Run u = run_of(a, begin + l);
            bulk_load(cache + l * 64, run_src(a, u), (uint32_t)u.nchunks * 16u, &s_bar);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_arrive(&s_bar);
    if (ncached > 0) {
        volatile int never = 0;
        if (!mbar_wait_bounded(&s_bar, 0, &never, a.limit_ns)) {
            record_error(a.err, NVFP4_ERR_TIMEOUT, 1);
            s_ok = 0;  // the copies may still land: wait for them once more below
        }
    }
    __syncthreads();
    if (!s_ok) {
        if (threadIdx.x == 0) {
            volatile int never = 0;
            mbar_wait_bounded(&s_bar, 0, &never, a.limit_ns);
        }
        return;
    }

    if (!a.given) {
        uint32_t m0 = 0, m1 = 0;
        for (int64_t g = begin + warp; g < end; g += kQWarps) {
            const Run u = run_of(a, g);
            const int64_t l = g - begin;
            const bool v0 = lane < u.nchunks, v1 = lane + 32 < u.nchunks;
            uint4 q0 = make_uint4(0, 0, 0, 0), q1 = make_uint4(0, 0, 0, 0);
            if (l < ncached) {
                if (v0) q0 = cache[l * 64 + lane];
                if (v1) q1 = cache[l * 64 + 32 + lane];
            } else {
                const uint8_t* src = run_src(a, u);
                if (v0) q0 = ld_stream16(src + lane * 16);
                if (v1) q1 = ld_stream16(src + (lane + 32) * 16);
            }
            const uint32_t mm = __vmaxu2(absmax_bits8(q0), absmax_bits8(q1));
            if (u.t) m1 = __vmaxu2(m1, mm);
            else m0 = __vmaxu2(m0, mm);
        }
        m0 = max(m0 & 0xFFFFu, m0 >> 16);
        m1 = max(m1 & 0xFFFFu, m1 >> 16);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            m0 = max(m0, __shfl_xor_sync(0xFFFFFFFFu, m0, o));
            m1 = max(m1, __shfl_xor_sync(0xFFFFFFFFu, m1, o));
        }
        if (lane == 0) {
            s_red[0][warp] = m0;
            s_red[1][warp] = m1;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t c0 = 0, c1 = 0;
            for (int w = 0; w < kQWarps; w++) {
                c0 = max(c0, s_red[0][w]);
                c1 = max(c1, s_red[1][w]);
            }
            volatile uint32_t* vctl = a.ctl;
            const uint32_t gen = vctl[kCtlGen];
            atomicMax(&a.ctl[kCtlAmax + 0], c0);
            atomicMax(&a.ctl[kCtlAmax + 1], c1);
            __threadfence();
            const uint32_t arrived = atomicAdd(&a.ctl[kCtlCount], 1u);
            if (arrived == (uint32_t)G - 1) {
                // last CTA: finish the tensor maxima and release the grid
                __threadfence();
                for (int t = 0; t < 2; t++) {
                    const uint32_t bits = atomicExch(&a.ctl[kCtlAmax + t], 0u);
                    const float a32 = __fdiv_rn(__uint_as_float(bits << 16), 2688.0f);  // amax / (6 * 448)
                    vctl[kCtlAlpha + t] = __float_as_uint(a32);
                    if (t < (a.total_runs > a.runs_per_tensor ? 2 : 1)) *(t ? a.gscale[1] : a.gscale[0]) = a32;
                }
                vctl[kCtlCount] = 0;
                __threadfence();
                atomicAdd(&a.ctl[kCtlGen], 1u);
            } else {
                const uint64_t t0 = global_ns();
                uint32_t it = 0;
                while (vctl[kCtlGen] == gen) {
                    if ((++it & 255u) == 0 && global_ns() - t0 > a.limit_ns) {
                        record_error(a.err, NVFP4_ERR_TIMEOUT, 2);
                        s_ok = 0;
                        break;
                    }
                }
                __threadfence();
            }
            s_alpha[0] = __uint_as_float(vctl[kCtlAlpha + 0]);
            s_alpha[1] = __uint_as_float(vctl[kCtlAlpha + 1]);
        }
        __syncthreads();
        if (!s_ok) return;
    } else {
        const int nt = a.total_runs > a.runs_per_tensor ? 2 : 1;  // gscale[1] is NULL for one tensor
        if (threadIdx.x < nt) s_alpha[threadIdx.x] = *(threadIdx.x ? a.gscale[1] : a.gscale[0]);
        __syncthreads();
    }

    // ---- phase 2: encode
    const int64_t sc_row = a.cols / 16;
    for (int64_t g = begin + warp; g < end; g += kQWarps) {
        const Run u = run_of(a, g);
        const int64_t l = g - begin;
        const bool v0 = lane < u.nchunks, v1 = lane + 32 < u.nchunks;
        uint4 q0 = make_uint4(0, 0, 0, 0), q1 = make_uint4(0, 0, 0, 0);
        if (l < ncached) {
            if (v0) q0 = cache[l * 64 + lane];
            if (v1) q1 = cache[l * 64 + 32 + lane];
        } else {
            const uint8_t* src = run_src(a, u);
            if (v0) q0 = ld_stream16(src + lane * 16);
            if (v1) q1 = ld_stream16(src + (lane + 32) * 16);
        }
        const float a32 = s_alpha[u.t];
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
        uint8_t* crow = (u.t ? a.codes[1] : a.codes[0]) + u.r * (a.cols / 2) + u.c0 / 2;
        if (v0) *reinterpret_cast<uint32_t*>(crow + 4 * lane) = w0;
        if (v1) *reinterpret_cast<uint32_t*>(crow + 128 + 4 * lane) = w1;
        // even lanes store the scale of their first-half block, odd lanes
        // the scale of their second-half block
        const bool odd = lane & 1;
        if (odd ? v1 : v0) {
            const int64_t bj = u.c0 / 16 + (odd ? 16 : 0) + (lane >> 1);
            const uint8_t code = (uint8_t)(odd ? b1.code : b0.code);
            uint8_t* sb = u.t ? a.scales[1] : a.scales[0];
            if (a.swizzled)
                sb[swz_offset(u.r, bj, a.tiles_c)] = code;
            else
                sb[u.r * sc_row + bj] = code;
        }
    }

    // zero the padding rows of the swizzled scale tiles (cols % 64 == 0, so
    // only the rows past `rows` up to the next multiple of 128 are padding)
    if (a.swizzled) {
        const int64_t rows_pad = (a.rows + 127) / 128 * 128;
        const int64_t sc_pad = a.tiles_c * 4;
        const int64_t npad = (rows_pad - a.rows) * sc_pad;
        const int nt = a.total_runs > a.runs_per_tensor ? 2 : 1;
        for (int t = 0; t < nt; t++) {
            uint8_t* sb = t ? a.scales[1] : a.scales[0];
            for (int64_t i = (int64_t)blockIdx.x * kQThreads + threadIdx.x; i < npad; i += G * kQThreads) {
                const int64_t r = a.rows + i / sc_pad, c = i % sc_pad;
                sb[swz_offset(r, c, a.tiles_c)] = 0;
            }
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

// 8 E2M1 codes (32 bits) with one block scale and the slot's a32 -> 8 bf16
// (16 bytes): bf16_rne(fl32(fl32(e2m1 * s) * a32)); e2m1 * s is exact in
// binary16, so the only roundings are the two the definition has.
__device__ __forceinline__ uint4 dequant8(uint32_t q, uint8_t sc, float a32) {
    const __half2 s2 = e4m3x2_to_half2((uint16_t)(sc | (sc << 8)));
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const __half2 v = __hmul2(e2m1x2_to_half2((q >> (8 * j)) & 0xFFu), s2);  // exact
        const float2 f = __half22float2(v);
        const __nv_bfloat162 b = __floats2bfloat162_rn(__fmul_rn(f.x, a32), __fmul_rn(f.y, a32));
        o[j] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__global__ void __launch_bounds__(kThreads) kv_dequant_kernel(DequantArgs a) {
    const int t = blockIdx.y;
    const int lane = threadIdx.x & 31;
    const int64_t ups = (a.slot_elems + 511) / 512;  // 512-element runs per slot
    const int64_t units = (int64_t)a.n * ups;
    const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
    const uint8_t* cb = t ? a.codes[1] : a.codes[0];
    const uint8_t* sb = t ? a.scales[1] : a.scales[0];
    const float* gb = t ? a.gscale[1] : a.gscale[0];
    uint8_t* ob = t ? a.out[1] : a.out[0];
    const int64_t w0 = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    for (int64_t base = w0; base < units; base += 2 * nwarps) {
        // two runs per iteration: all loads first, then decode and store
        uint32_t q[2][2];
        uint8_t sc[2][2];
        float a32[2];
        bool ok[2][2];
        int64_t obase[2], e0[2];
#pragma unroll
        for (int k = 0; k < 2; k++) {
            const int64_t unit = base + k * nwarps;
            ok[k][0] = ok[k][1] = false;
            a32[k] = 0.0f;
            obase[k] = e0[k] = 0;
            q[k][0] = q[k][1] = 0;
            sc[k][0] = sc[k][1] = 0;
            if (unit >= units) continue;
            const int64_t i = unit / ups;
            const int64_t u = unit - i * ups;
            const int32_t s = __ldg(a.slots + i);
            if (s < 0 || s >= a.n_slots) {
                if (lane == 0 && u == 0 && t == 0) record_error(a.err, NVFP4_ERR_DEVICE, (uint32_t)i);
                continue;
            }
            const int64_t sbase = (int64_t)s * a.slot_elems;
            e0[k] = u * 512 + 8 * lane;
            obase[k] = (int64_t)i * a.slot_elems;
            a32[k] = __ldg(gb + s);
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const int64_t e = e0[k] + 256 * h;
                ok[k][h] = e < a.slot_elems;
                if (ok[k][h]) {
                    q[k][h] = __ldg(reinterpret_cast<const uint32_t*>(cb + (sbase + e) / 2));
                    sc[k][h] = __ldg(sb + (sbase + e) / 16);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < 2; k++)
#pragma unroll
            for (int h = 0; h < 2; h++)
                if (ok[k][h])
                    *reinterpret_cast<uint4*>(ob + (obase[k] + e0[k] + 256 * h) * 2) = dequant8(q[k][h], sc[k][h], a32[k]);
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

static int g_q_dev = -1;
static int g_q_smem = 0;

// one fused, cooperative launch over one or two tensors of the same shape
static nvfp4_status quantize_impl(int ntensors, const void* const* x, int64_t rows, int64_t cols, int64_t ld,
                                  void* const* codes, void* const* scales, float* const* gscale, bool given,
                                  bool swizzled, void* workspace, cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (g_q_dev != dev) {
        int optin = 0;
        if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        // leave room for the kernel's static shared memory
        const int smem = (optin - 2048) / kRunBytes * kRunBytes;
        if (cudaFuncSetAttribute(quantize_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
            return NVFP4_ERR_CUDA;
        g_q_smem = smem;
        g_q_dev = dev;
    }
    QuantArgs a{};
    for (int t = 0; t < ntensors; t++) {
        a.x[t] = static_cast<const uint8_t*>(x[t]);
        a.codes[t] = static_cast<uint8_t*>(codes[t]);
        a.scales[t] = static_cast<uint8_t*>(scales[t]);
        a.gscale[t] = gscale[t];
    }
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.upr = (cols + 511) / 512;
    a.runs_per_tensor = rows * a.upr;
    a.total_runs = a.runs_per_tensor * ntensors;
    a.given = given ? 1 : 0;
    a.swizzled = swizzled ? 1 : 0;
    a.tiles_c = (cols + 63) / 64;
    a.ctl = static_cast<uint32_t*>(workspace);
    a.err = static_cast<DevError*>(workspace);
    a.limit_ns = 2000000000ull;
    const int G = (int)std::min<int64_t>(num_sms(), a.total_runs);
    const int64_t per_cta = (a.total_runs + G - 1) / G;
    a.cap = (int)std::min<int64_t>(per_cta, g_q_smem / kRunBytes);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kQThreads);
    cfg.dynamicSmemBytes = (size_t)a.cap * kRunBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, quantize_fused_kernel, a) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
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
    const int64_t units = (int64_t)n * ((a.slot_elems + 511) / 512);
    const int g = grid_for(units, 2 * (kThreads / 32), num_sms() * 8);
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
