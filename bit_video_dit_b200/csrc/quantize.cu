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
//    the input held in registers across a bounded grid barrier, |x| max on
//    the bf16 bit patterns (two 16-bit lanes per 32-bit SIMD max), then the
//    encode: a warp per 512-element run, a lane per 16-element block.
//  * dequant-gather: a warp owns 512-element runs of a slot; lane i decodes
//    elements 8i..8i+7 and 256+8i..256+8i+7 (4-byte code loads, 16-byte bf16
//    stores, each warp-wide access contiguous), two runs in flight per lane.
//  * value transforms ahead of the encode (template variants of the fused
//    kernel): LayerNorm + adaLN modulate of activation rows; for a KV chunk the
//    keys' rotary embedding (the article's fused RoPE; interleaved pairs turned
//    by a per-token cos / sin table) and the K-smoothing mean subtraction, whose
//    channel means come from a separate fixed-order kernel (of the turned keys
//    when both apply).
//  * LayerNorm + modulate + quantize in one cooperative launch when each CTA's
//    rows fit in shared memory (ln_quantize_smem_kernel: the rows copied in
//    once, statistics, tensor maximum and encode all read them there); larger
//    inputs take the statistics kernel and the fused kernel's LN variant.
#include <algorithm>

#include "common.cuh"

namespace nvfp4 {

constexpr int kThreads = 256;  // dequant / probe kernels

// ---------------------------------------------------------------------------
// Fused quantize: one cooperative launch, one CTA of 512 threads per SM.
//   phase 1  every warp takes a contiguous share of one tensor's 512-element
//            runs (the tensor's elements in row order, 32 blocks of 16 a run)
//            and loads up to kMaxRuns of them straight into registers -- a
//            lane holds one 16-element block per run, all loads in flight at
//            once -- and takes their |x| max (on the bf16 bit patterns);
//   barrier  each CTA folds its maxima into two global maxima (fire-and-
//            forget reductions) and counts itself in with an acquire-release
//            add; every CTA polls the count (bounded wait), then reads the
//            maxima: a32 = amax / 2688;
//   phase 2  every warp encodes the blocks it holds: one block scale per
//            lane (the reciprocal 1 / (s * a32) from a 256-entry table per
//            tensor, built once per CTA), 8-byte code stores (256 contiguous
//            bytes per warp).
// A block's row comes from its index by a multiply-high with a per-shape
// magic number (no division, no state carried from run to run), so the runs
// a lane holds are independent and their encodes interleave; the scale
// layout is a template parameter.  HBM is read once and written once; runs
// beyond kMaxRuns per warp (tensors larger than ~#SMs x 176 KB) are read
// again in phase 2, several at a time (from L2 when the tensor fits there).
// ---------------------------------------------------------------------------
constexpr int kQThreads = 512;
constexpr int kQWarps = kQThreads / 32;
constexpr int kMaxRuns = 11;   // runs held in registers per warp (11 x 32 B per lane)
constexpr int kBatch = 2;      // runs past the held ones, loaded together (phase 1)
constexpr int kBatch2 = 6;     // the same in phase 2, once the held runs are encoded
constexpr int kMaxGrid = 1024;

// Control block (uint32 words of the workspace's first 256 bytes, zero before
// first use; words 0..3 are the error record):
constexpr int kCtlEpoch = 8;   // epoch of the last completed launch
constexpr int kCtlCount = 16;  // [2] arrivals of the launch with epoch parity p
constexpr int kCtlMax = 20;    // [2][2] magnitude maxima per parity, per tensor

struct QuantArgs {
    const uint8_t* x[2];
    uint8_t* codes[2];
    uint8_t* scales[2];
    float* gscale[2];
    int64_t ld_bytes;      // row stride of x in bytes
    int64_t tiles_c;       // swizzled scales: 4-column tiles per row block (cols / 64)
    uint32_t nblk;         // 16-element blocks per tensor (rows * cols / 16 < 2^31)
    uint32_t nb;           // blocks per row (cols / 16)
    uint32_t nb_magic;     // block b's row = umulhi(b, nb_magic) >> nb_shift
    int nb_shift;
    int runs_per_tensor;   // ceil(nblk / 32)
    int ntensors;
    int given;
    // LayerNorm + modulate ahead of the quantize (LN kernels only): per-row
    // (mean, rstd) and the bf16 [cols] modulation vectors (NULL: 0)
    const float2* ln_stats;
    const __nv_bfloat16* mod_scale;
    const __nv_bfloat16* mod_shift;
    // K-smoothing ahead of the quantize (smoothing kernels only, one row per
    // tensor): binary32 channel means [smooth_hd] per tensor (NULL: none);
    // the element at flat index i belongs to channel i mod smooth_hd
    const float* smooth_mean[2];
    int smooth_hd;
    // rotary position embedding of tensor 0 (the keys) ahead of the quantize
    // (smoothing kernels only, one row per tensor): binary32 cos / sin
    // [tokens][rope_d / 2]; the element at flat index i is channel i mod rope_d
    // of a head of token i / rope_hd (NULL: none)
    const float* rope_cos;
    const float* rope_sin;
    int rope_d;
    int rope_hd;
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

// 16-byte streaming load, or zeros when `pred` is false (no branch)
__device__ __forceinline__ uint4 ld_stream16_if(const void* p, bool pred) {
    uint4 v;
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %5, 0;\n\t"
        "mov.b32 %0, 0;\n\tmov.b32 %1, 0;\n\tmov.b32 %2, 0;\n\tmov.b32 %3, 0;\n\t"
        "@q ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];\n\t}"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p), "r"((int)pred));
    return v;
}

// Where the lane's block of run `run` (tensor t) lives: block index b in the
// tensor, its row r and block column cb; valid when b is inside the tensor.
struct Blk {
    uint32_t b, r, cb;
    bool valid;
    __device__ __forceinline__ Blk(const QuantArgs& a, int run, int lane) {
        b = (uint32_t)run * 32u + (uint32_t)lane;
        valid = b < a.nblk;
        r = __umulhi(b, a.nb_magic) >> a.nb_shift;
        cb = b - r * a.nb;
    }
    __device__ __forceinline__ const uint8_t* src(const QuantArgs& a, int t) const {
        return (t ? a.x[1] : a.x[0]) + (int64_t)r * a.ld_bytes + (int64_t)cb * 32;
    }
};

// Per-tensor constants of the encode: a32, 6 a32, 4 a32 (targets of the
// block max) and the reciprocal 1 / (s * a32) of every E4M3 code s.
struct EncodeConsts {
    float a32, d6, d4;
    const float* inv_tab;
};

// E2M1 codes of 16 binary32 ratios x * inv (two 32-bit words, element 2i in
// the low nibble); a flushed block (inv == 0) is +0 codes.
__device__ __forceinline__ uint2 encode16(const float* f, float inv) {
    float y[16];
    const float2 iv = make_float2(inv, inv);
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const float2 t = mul2(make_float2(f[2 * i], f[2 * i + 1]), iv);
        y[2 * i] = t.x;
        y[2 * i + 1] = t.y;
    }
    return make_uint2(inv == 0.0f ? 0u : e2m1x8(y), inv == 0.0f ? 0u : e2m1x8(y + 8));
}

// Squared error of an encoding of the block, binary32, in element order:
// sum += (x - fl32(fl32(e2m1 * s) * a32))^2 (the dequant product, exact up to
// the last multiply).  e2m1 * s is exact in binary16 (at most 6 significant
// bits, between 2^-10 and 2688), so it is formed there, two at a time; the
// multiply by a32, the difference and the square run on binary32 pairs (each
// lane rounded alone); only the sum is taken one element at a time.
__device__ __forceinline__ float block_sq_error(const float* f, uint2 c, uint32_t code, float a32) {
    float sum = 0.0f;
    const __half2 s2 = e4m3x2_to_half2((uint16_t)(code | (code << 8)));
    const float2 aa = make_float2(a32, a32), m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int w = 0; w < 2; w++) {
        const uint32_t word = w ? c.y : c.x;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const float2 v = __half22float2(__hmul2(e2m1x2_to_half2((word >> (8 * j)) & 0xFFu), s2));
            const float2 d = mul2(v, aa);
            const float2 e = fma2(d, m1, make_float2(f[8 * w + 2 * j], f[8 * w + 2 * j + 1]));
            const float2 e2 = mul2(e, e);
            sum = __fadd_rn(sum, e2.x);
            sum = __fadd_rn(sum, e2.y);
        }
    }
    return sum;
}

// encode the lane's 16-element block and store its codes + scale.  SEARCH:
// also encode with the block max aimed at 4 instead of 6 and keep that
// encoding when its squared error is smaller.
template <bool SWZ, bool SEARCH>
__device__ __forceinline__ void encode_block(const QuantArgs& a, int t, const Blk& k, const float* f, float amax_b,
                                             const EncodeConsts& kc) {
    // s = E4M3(amax_b / (6 a32)); a zero tensor scale flushes every block
    uint32_t code = kc.d6 == 0.0f ? 0u : e4m3_code(__fdiv_rn(amax_b, kc.d6));
    uint2 c = encode16(f, kc.inv_tab[code]);
    if (SEARCH) {
        const uint32_t code4 = kc.d4 == 0.0f ? 0u : e4m3_code(__fdiv_rn(amax_b, kc.d4));
        const uint2 c4 = encode16(f, kc.inv_tab[code4]);
        if (block_sq_error(f, c4, code4, kc.a32) < block_sq_error(f, c, code, kc.a32)) {
            code = code4;
            c = c4;
        }
    }
    if (k.valid) {
        *reinterpret_cast<uint2*>((t ? a.codes[1] : a.codes[0]) + (int64_t)k.b * 8) = c;
        uint8_t* sc = t ? a.scales[1] : a.scales[0];
        if (SWZ)
            sc[swz_offset(k.r, k.cb, a.tiles_c)] = (uint8_t)code;
        else
            sc[k.b] = (uint8_t)code;
    }
}

// Value transforms ahead of the encode (a template parameter of the kernel).
constexpr int kXfNone = 0;    // the bf16 input as is
constexpr int kXfLn = 1;      // LayerNorm + adaLN modulate of each row
constexpr int kXfSmooth = 2;  // RoPE of the keys, then minus the channel mean (KV chunk)

// The 16 binary32 values of the lane's block k (tensor t): the bf16 input;
// with LN its LayerNorm + modulate, in this order and rounding:
// m = fl32(fl32(fl32(fl32(x - mean) * rstd) * fl32(1 + scale)) + shift);
// for a KV chunk, the keys' rotary embedding where a table is given (pair
// (x0, x1) -> (fl32(fl32(x0 c) - fl32(x1 s)), fl32(fl32(x0 s) + fl32(x1 c))),
// c and s of the element's token and pair), then fl32(y - mean[channel]) where
// means are given.
template <int XF>
__device__ __forceinline__ void block_values(const QuantArgs& a, const Blk& k, int t, const uint4& q0, const uint4& q1,
                                             float* f) {
    bf16x8_to_f32(q0, f);
    bf16x8_to_f32(q1, f + 8);
    if (XF == kXfSmooth && t == 0 && a.rope_cos && k.valid) {
        // one row per tensor, fewer than 2^31 elements: the block's 16
        // elements are 8 whole pairs of one head of one token (rope_d % 16 == 0)
        const uint32_t i0 = k.cb * 16u;
        const uint32_t tok = i0 / (uint32_t)a.rope_hd;
        const uint32_t p0 = (i0 % (uint32_t)a.rope_d) >> 1;
        const size_t off = (size_t)tok * (uint32_t)(a.rope_d >> 1) + p0;  // a multiple of 8 floats
        const float4* pc = reinterpret_cast<const float4*>(a.rope_cos + off);
        const float4* ps = reinterpret_cast<const float4*>(a.rope_sin + off);
        const float4 c0 = __ldg(pc), c1 = __ldg(pc + 1), s0 = __ldg(ps), s1 = __ldg(ps + 1);
        const float c[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const float sn[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const float x0 = f[2 * j], x1 = f[2 * j + 1];
            f[2 * j] = __fsub_rn(__fmul_rn(x0, c[j]), __fmul_rn(x1, sn[j]));
            f[2 * j + 1] = __fadd_rn(__fmul_rn(x0, sn[j]), __fmul_rn(x1, c[j]));
        }
    }
    if (XF == kXfSmooth) {
        const float* mean = t ? a.smooth_mean[1] : a.smooth_mean[0];
        if (k.valid && mean) {
            // one row per tensor: the block's 16 channels are consecutive
            // (smooth_hd is a multiple of 16)
            const uint32_t c0 = (k.cb * 16u) % (uint32_t)a.smooth_hd;
            const float4* p = reinterpret_cast<const float4*>(mean + c0);
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const float4 v = __ldg(p + j);
                f[4 * j] = __fsub_rn(f[4 * j], v.x);
                f[4 * j + 1] = __fsub_rn(f[4 * j + 1], v.y);
                f[4 * j + 2] = __fsub_rn(f[4 * j + 2], v.z);
                f[4 * j + 3] = __fsub_rn(f[4 * j + 3], v.w);
            }
        }
    }
    if (XF == kXfLn) {
        const float2 st = k.valid ? __ldg(a.ln_stats + k.r) : make_float2(0.0f, 0.0f);
        const uint32_t c0 = k.cb * 16u;
        float sc[16], sh[16];
#pragma unroll
        for (int i = 0; i < 16; i++) sc[i] = sh[i] = 0.0f;
        if (k.valid && a.mod_scale) {
            const uint4* p = reinterpret_cast<const uint4*>(a.mod_scale + c0);
            bf16x8_to_f32(__ldg(p), sc);
            bf16x8_to_f32(__ldg(p + 1), sc + 8);
        }
        if (k.valid && a.mod_shift) {
            const uint4* p = reinterpret_cast<const uint4*>(a.mod_shift + c0);
            bf16x8_to_f32(__ldg(p), sh);
            bf16x8_to_f32(__ldg(p + 1), sh + 8);
        }
#pragma unroll
        for (int i = 0; i < 16; i++) {
            const float h = __fmul_rn(__fsub_rn(f[i], st.x), st.y);
            f[i] = __fadd_rn(__fmul_rn(h, __fadd_rn(1.0f, sc[i])), sh[i]);
        }
    }
}

// a block's |x| max as an order-preserving 32-bit key: the bf16 magnitude
// bits (F32, after a transform: the binary32 magnitude bits of the values)
template <bool F32>
__device__ __forceinline__ uint32_t block_max_key(const uint4& q0, const uint4& q1, const float* f) {
    if (F32) {
        float mx = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; i++) mx = fmaxf(mx, fabsf(f[i]));
        return __float_as_uint(mx);
    }
    const uint32_t mm = __vmaxu2(absmax_bits8(q0), absmax_bits8(q1));
    return max(mm & 0xFFFFu, mm >> 16);
}

template <bool F32>
__device__ __forceinline__ float key_value(uint32_t key) { return __uint_as_float(F32 ? key : key << 16); }

// ---------------------------------------------------------------------------
// Grid-wide maximum of the cooperative quantize kernels (thread 0 of each
// CTA): fold the CTA's per-tensor maxima into the launch's global maxima and
// count the CTA in (acquire-release), wait until every CTA of the launch has
// (bounded), then read the maxima into total[2].  False when the wait ran out
// (error recorded).
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool grid_max_exchange(uint32_t* ctl, DevError* err, uint64_t limit_ns, int par, int G,
                                                  uint32_t c0, uint32_t c1, uint32_t* total) {
    uint32_t* cnt = ctl + kCtlCount + par;
    uint32_t* mx = ctl + kCtlMax + 2 * par;
    asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(mx), "r"(c0) : "memory");
    asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(mx + 1), "r"(c1) : "memory");
    uint32_t old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(old) : "l"(cnt) : "memory");
    const uint64_t t_start = global_ns();
    uint32_t n = old + 1u;
    bool ok = true;
    while (n < (uint32_t)G) {
        __nanosleep(20);
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(n) : "l"(cnt) : "memory");
        if (n < (uint32_t)G && global_ns() - t_start > limit_ns) {
            record_error(err, NVFP4_ERR_TIMEOUT, 2);
            ok = false;
            break;
        }
    }
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(total[0]) : "l"(mx) : "memory");
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(total[1]) : "l"(mx + 1) : "memory");
    return ok;
}

// After every CTA has counted itself in (so has read the epoch and is done
// with the other parity's words): reset those for the next launch, then
// publish this launch's epoch.  One thread of one CTA.
__device__ __forceinline__ void grid_barrier_retire(uint32_t* ctl, int par, uint32_t epoch) {
    ctl[kCtlCount + (par ^ 1)] = 0u;
    ctl[kCtlMax + 2 * (par ^ 1)] = 0u;
    ctl[kCtlMax + 2 * (par ^ 1) + 1] = 0u;
    __threadfence();
    *(volatile uint32_t*)&ctl[kCtlEpoch] = epoch;
}

template <bool SWZ, bool SEARCH, int XF>
__global__ void __launch_bounds__(kQThreads, 1) quantize_fused_kernel(const __grid_constant__ QuantArgs a) {
    constexpr bool F32 = XF != kXfNone;       // 32-bit keys of transformed values
    constexpr int kRuns = F32 ? 4 : kMaxRuns;  // a transform needs registers
    __shared__ uint32_t s_red[kQWarps];
    __shared__ float s_d6[2], s_d4[2], s_a32[2];
    __shared__ float s_inv[2][256];
    __shared__ uint32_t s_total[2];
    __shared__ int s_ok;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x;
    // warps [0, nw / ntensors) take tensor 0, the rest tensor 1
    const int nw = G * kQWarps, nwt = nw / a.ntensors;
    const int wg = blockIdx.x * kQWarps + warp;
    const int t = wg / nwt;
    const int wl = wg - t * nwt;
    const int wb = (int)((int64_t)a.runs_per_tensor * wl / nwt);
    const int we = (int)((int64_t)a.runs_per_tensor * (wl + 1) / nwt);
    const uint32_t epoch = *(volatile uint32_t*)&a.ctl[kCtlEpoch] + 1u;  // same for every CTA of this launch
    const int par = (int)(epoch & 1u);

    // ---- phase 1: this warp's runs wb .. we-1 of tensor t, one block per lane
    uint4 q[kRuns][2];
#pragma unroll
    for (int k = 0; k < kRuns; k++) {
        const Blk kb(a, wb + k, lane);
        const bool ld = wb + k < we && kb.valid;
        const uint8_t* src = kb.src(a, t);
        q[k][0] = ld_stream16_if(src, ld);
        q[k][1] = ld_stream16_if(src + 16, ld);
    }
    uint32_t m = 0;  // the lane's max key over its runs (each block's max is taken again in phase 2)
#pragma unroll
    for (int k = 0; k < kRuns; k++) {
        if constexpr (!F32) {
            // blocks past the data were loaded as zeros: key 0
            const uint32_t mm = __vmaxu2(absmax_bits8(q[k][0]), absmax_bits8(q[k][1]));
            m = max(m, max(mm & 0xFFFFu, mm >> 16));
        } else {
            const Blk kb(a, wb + k, lane);
            float f[16];
            block_values<XF>(a, kb, t, q[k][0], q[k][1], f);
            if (wb + k < we && kb.valid) m = max(m, block_max_key<F32>(q[k][0], q[k][1], f));
        }
    }
    if (threadIdx.x == 0) s_ok = 1;
    if (!a.given) {
        // the runs past the held ones, kBatch loads in flight per lane
        for (int g = wb + kRuns; g < we; g += kBatch) {
            uint4 v[kBatch][2];
#pragma unroll
            for (int u = 0; u < kBatch; u++) {
                const Blk kb(a, g + u, lane);
                const bool ld = g + u < we && kb.valid;
                const uint8_t* src = kb.src(a, t);
                v[u][0] = ld_stream16_if(src, ld);
                v[u][1] = ld_stream16_if(src + 16, ld);
            }
#pragma unroll
            for (int u = 0; u < kBatch; u++) {
                const Blk kb(a, g + u, lane);
                float f[16];
                block_values<XF>(a, kb, t, v[u][0], v[u][1], f);
                if (g + u < we && kb.valid) m = max(m, block_max_key<F32>(v[u][0], v[u][1], f));
            }
        }
        // 16-bit keys: one word per lane, tensor-1 max in the high half and
        // tensor-0 in the low, reduced as pairs; 32-bit keys (after a
        // transform): a warp covers one tensor, so its max, then per tensor
        // over the CTA's warps
        if (!F32) m = t ? (m << 16) : m;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, m, o);
            m = F32 ? max(m, other) : __vmaxu2(m, other);
        }
        if (lane == 0) s_red[warp] = m;
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t c0 = 0u, c1 = 0u;
            if (F32) {
#pragma unroll
                for (int i = 0; i < kQWarps; i++) {
                    if ((blockIdx.x * kQWarps + i) / nwt)
                        c1 = max(c1, s_red[i]);
                    else
                        c0 = max(c0, s_red[i]);
                }
            } else {
                uint32_t c = 0u;
#pragma unroll
                for (int i = 0; i < kQWarps; i++) c = __vmaxu2(c, s_red[i]);
                c0 = c & 0xFFFFu;
                c1 = c >> 16;
            }
            uint32_t tot[2];
            if (!grid_max_exchange(a.ctl, a.err, a.limit_ns, par, G, c0, c1, tot)) s_ok = 0;
            s_total[0] = tot[0];
            s_total[1] = tot[1];
        }
        __syncthreads();
        if (!s_ok) return;
        if (threadIdx.x < a.ntensors) {
            const float a32 = __fdiv_rn(key_value<F32>(s_total[threadIdx.x]), 2688.0f);  // amax / (6 * 448)
            s_d6[threadIdx.x] = a32;  // a32 for now; the table below needs it
            if (blockIdx.x == 0) *(threadIdx.x ? a.gscale[1] : a.gscale[0]) = a32;
        }
        if (blockIdx.x == 0 && threadIdx.x == 32) grid_barrier_retire(a.ctl, par, epoch);
    } else {
        if (threadIdx.x < a.ntensors) s_d6[threadIdx.x] = *(threadIdx.x ? a.gscale[1] : a.gscale[0]);
    }
    __syncthreads();
    // per tensor: inv[code] = 1 / (s * a32) for every E4M3 code (0 when s = 0
    // or a32 = 0), then 6 a32 and 4 a32
    {
        const int tt = threadIdx.x >> 8, c = threadIdx.x & 255;
        if (tt < a.ntensors) {
            const float a32 = s_d6[tt];
            const float sv = e4m3_value((uint32_t)c);
            s_inv[tt][c] = (a32 == 0.0f || sv == 0.0f) ? 0.0f : __frcp_rn(__fmul_rn(sv, a32));
        }
        __syncthreads();
        if (threadIdx.x < a.ntensors) {
            const float a32 = s_d6[threadIdx.x];
            s_a32[threadIdx.x] = a32;
            s_d6[threadIdx.x] = __fmul_rn(6.0f, a32);
            s_d4[threadIdx.x] = __fmul_rn(4.0f, a32);
        }
        __syncthreads();
    }

    // ---- phase 2: encode
    {
        const EncodeConsts kc{s_a32[t], s_d6[t], s_d4[t], s_inv[t]};
#pragma unroll
        for (int k = 0; k < kRuns; k++) {
            if (wb + k < we) {
                const Blk kb(a, wb + k, lane);
                float f[16];
                block_values<XF>(a, kb, t, q[k][0], q[k][1], f);
                encode_block<SWZ, SEARCH>(a, t, kb, f, key_value<F32>(block_max_key<F32>(q[k][0], q[k][1], f)), kc);
            }
        }
        for (int g = wb + kRuns; g < we; g += kBatch2) {
            uint4 v[kBatch2][2];
#pragma unroll
            for (int u = 0; u < kBatch2; u++) {
                const Blk kb(a, g + u, lane);
                const bool ld = g + u < we && kb.valid;
                const uint8_t* src = kb.src(a, t);
                v[u][0] = ld_stream16_if(src, ld);
                v[u][1] = ld_stream16_if(src + 16, ld);
            }
#pragma unroll
            for (int u = 0; u < kBatch2; u++) {
                if (g + u < we) {
                    const Blk kb(a, g + u, lane);
                    float f[16];
                    block_values<XF>(a, kb, t, v[u][0], v[u][1], f);
                    encode_block<SWZ, SEARCH>(a, t, kb, f, key_value<F32>(block_max_key<F32>(v[u][0], v[u][1], f)), kc);
                }
            }
        }
    }

    // zero the padding rows of the swizzled scale tiles (cols % 64 == 0, so
    // only the rows past `rows` up to the next multiple of 128 are padding)
    if (SWZ) {
        const int64_t rows = a.nblk / a.nb;
        const int64_t rows_pad = (rows + 127) / 128 * 128;
        const int64_t sc_pad = a.tiles_c * 4;
        const int64_t npad = (rows_pad - rows) * sc_pad;
        for (int tt = 0; tt < a.ntensors; tt++) {
            uint8_t* sb = a.scales[tt];
            for (int64_t i = (int64_t)blockIdx.x * kQThreads + threadIdx.x; i < npad; i += (int64_t)G * kQThreads) {
                const int64_t r = rows + i / sc_pad, c = i % sc_pad;
                sb[swz_offset(r, c, a.tiles_c)] = 0;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// LayerNorm + adaLN modulate + quantize in one cooperative launch, for inputs
// whose rows fit in shared memory (one CTA of 512 threads per SM holds
// ceil(rows / #SMs) rows):
//   load     thread 0 bulk-copies the CTA's rows into shared memory, one copy
//            per row, kLnGroups groups of rows each on its own mbarrier;
//   stats    a warp per row, as its group lands: S1 = sum of x, lane j
//            adding elements 256c + 8j .. 256c + 8j + 7 of c = 0, 1, ... in
//            order (16 contiguous bytes a lane: conflict-free), the 32 partials
//            met in an xor butterfly (16, 8, 4, 2, 1); mean = fl32(S1 / cols);
//            S2 the same over fl32(x - mean)^2; rstd = 1 / sqrt(S2 / cols +
//            eps) -- the order of the two-launch path's statistics kernel, so
//            both paths give the same bits;
//   max      the (512-column chunk, row) tasks in chunk-major order, split
//            evenly over the warps, lane i holding block i of the chunk (its
//            modulation columns stay in registers while the warp's chunk
//            stays the same):
//            m = fl32(fl32(fl32(fl32(x - mean) * rstd) * fl32(1 + scale)) + shift)
//            (binary32 pairs) and the CTA's max |m|;
//   barrier  the bounded grid barrier: a32 = max |m| / 2688;
//   encode   the same tasks: m and its block max again, one scale and 8
//            bytes of codes a lane.
// A lane reads its 32-byte block as two 16-byte halves, lanes 4..7 of every
// eight taking the second half first, so each warp-wide read covers all 32
// banks four times (no conflicts).  HBM: the input is read once and the codes
// and scales written once.
// ---------------------------------------------------------------------------
constexpr int kLnGroups = 8;  // groups of rows, each copied in on its own mbarrier

struct LnArgs {
    const uint8_t* x;
    int64_t ld_bytes;
    int rows, cols;
    float eps;
    const __nv_bfloat16* mod_scale;  // NULL: 0
    const __nv_bfloat16* mod_shift;  // NULL: 0
    uint8_t* codes;
    uint8_t* scales;
    float* gscale;
    int given;
    int swizzled;
    int64_t tile_row;  // swizzled scales: bytes per 128-row block (cols / 64 * 512)
    float2* stats;     // (mean, rstd) per row, written for the caller
    uint32_t* ctl;
    DevError* err;
    uint64_t limit_ns;
};

__device__ __forceinline__ float ln_butterfly(float s) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s = __fadd_rn(s, __shfl_xor_sync(0xFFFFFFFFu, s, o));
    return s;
}

// The lane's 16 modulation columns c0 .. c0+15: fl32(1 + scale) and shift
// (1 and 0 where the vector is absent or the block is past the row).
__device__ __forceinline__ void ln_columns(const LnArgs& a, int c0, bool valid, float* sc1, float* sh) {
#pragma unroll
    for (int i = 0; i < 16; i++) {
        sc1[i] = 1.0f;
        sh[i] = 0.0f;
    }
    if (valid && a.mod_scale) {
        const uint4* p = reinterpret_cast<const uint4*>(a.mod_scale + c0);
        float v[16];
        bf16x8_to_f32(__ldg(p), v);
        bf16x8_to_f32(__ldg(p + 1), v + 8);
#pragma unroll
        for (int i = 0; i < 16; i++) sc1[i] = __fadd_rn(1.0f, v[i]);
    }
    if (valid && a.mod_shift) {
        const uint4* p = reinterpret_cast<const uint4*>(a.mod_shift + c0);
        bf16x8_to_f32(__ldg(p), sh);
        bf16x8_to_f32(__ldg(p + 1), sh + 8);
    }
}

// The lane's 16 bf16 of a row staged in shared memory (32 bytes at `p`) as
// binary32, the halves read in the order that spreads a warp over all banks.
__device__ __forceinline__ void ln_load16(const uint8_t* p, int lane, float* f) {
    const int h = (lane >> 2) & 1;
    const uint4 first = *reinterpret_cast<const uint4*>(p + 16 * h);
    const uint4 second = *reinterpret_cast<const uint4*>(p + 16 * (h ^ 1));
    bf16x8_to_f32(h ? second : first, f);
    bf16x8_to_f32(h ? first : second, f + 8);
}

// m of 16 elements (in place over x) and their |m| max, binary32 pairs:
// fl32(fl32(fl32(fl32(x - mean) * rstd) * sc1) + sh)
__device__ __forceinline__ float ln_modulate16(float* f, float mean, float rstd, const float* sc1, const float* sh) {
    const float2 nm = make_float2(-mean, -mean), rs = make_float2(rstd, rstd);
    float mx = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const float2 h = mul2(add2(make_float2(f[2 * i], f[2 * i + 1]), nm), rs);
        const float2 m = add2(mul2(h, make_float2(sc1[2 * i], sc1[2 * i + 1])), make_float2(sh[2 * i], sh[2 * i + 1]));
        f[2 * i] = m.x;
        f[2 * i + 1] = m.y;
        mx = fmaxf(mx, fmaxf(fabsf(m.x), fabsf(m.y)));
    }
    return mx;
}

template <bool SEARCH>
__global__ void __launch_bounds__(kQThreads, 1) ln_quantize_smem_kernel(const __grid_constant__ LnArgs a) {
    extern __shared__ __align__(128) uint8_t ln_smem[];
    __shared__ uint64_t bars[kLnGroups];
    __shared__ uint32_t s_red[kQWarps];
    __shared__ float s_inv[256];
    __shared__ float s_a32, s_d6, s_d4;
    __shared__ uint32_t s_total;
    __shared__ int s_ok;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x;
    const int r0 = (int)((int64_t)a.rows * blockIdx.x / G), r1 = (int)((int64_t)a.rows * (blockIdx.x + 1) / G);
    const int nr = r1 - r0, cols = a.cols;
    const int nch = (cols + 255) / 256;   // 256-element chunks per row (statistics)
    const int nrun = (cols + 511) / 512;  // 512-element chunks per row (a block per lane)
    const int64_t row_bytes = (int64_t)cols * 2;
    uint8_t* xs = ln_smem;                                                      // [nr][cols] bf16
    float2* st = reinterpret_cast<float2*>(ln_smem + (int64_t)nr * row_bytes);  // [nr] (mean, rstd)
    const uint32_t epoch = *(volatile uint32_t*)&a.ctl[kCtlEpoch] + 1u;  // same for every CTA of this launch
    const int par = (int)(epoch & 1u);
    if (threadIdx.x == 0) {
        s_ok = 1;
        for (int g = 0; g < kLnGroups; g++) mbar_init(&bars[g], 1);
        fence_barrier_init();
        int r = 0;
        for (int g = 0; g < kLnGroups; g++) {
            const int re = (int)((int64_t)nr * (g + 1) / kLnGroups);
            for (; r < re; r++) {
                mbar_expect_tx_only(&bars[g], (uint32_t)row_bytes);
                bulk_load(xs + r * row_bytes, a.x + (int64_t)(r0 + r) * a.ld_bytes, (uint32_t)row_bytes, &bars[g]);
            }
            mbar_arrive(&bars[g]);
        }
    }
    __syncthreads();
    // ---- statistics, a warp per row (as its group lands)
    const float n = (float)cols;
    bool landed = true;
    {
        volatile int never = 0;
        int g = 0;
        for (int r = warp; r < nr && landed; r += kQWarps) {
            while ((int64_t)(g + 1) * nr / kLnGroups <= r) g++;  // the group holding row r
            landed = mbar_wait_bounded(&bars[g], 0, &never, a.limit_ns);
            if (!landed) break;
            const uint8_t* row = xs + r * row_bytes;
            float s1 = 0.0f;
            for (int c = 0; c < nch; c++) {
                const int e0 = 256 * c + 8 * lane;
                if (e0 < cols) {
                    float f[8];
                    bf16x8_to_f32(*reinterpret_cast<const uint4*>(row + 2 * e0), f);
#pragma unroll
                    for (int i = 0; i < 8; i++) s1 = __fadd_rn(s1, f[i]);
                }
            }
            const float mean = __fdiv_rn(ln_butterfly(s1), n);
            float s2 = 0.0f;
            for (int c = 0; c < nch; c++) {
                const int e0 = 256 * c + 8 * lane;
                if (e0 < cols) {
                    float f[8];
                    bf16x8_to_f32(*reinterpret_cast<const uint4*>(row + 2 * e0), f);
#pragma unroll
                    for (int i = 0; i < 8; i++) {
                        const float d = __fsub_rn(f[i], mean);
                        s2 = __fadd_rn(s2, __fmul_rn(d, d));
                    }
                }
            }
            const float var = __fdiv_rn(ln_butterfly(s2), n);
            const float rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, a.eps)));
            if (lane == 0) {
                st[r] = make_float2(mean, rstd);
                a.stats[r0 + r] = make_float2(mean, rstd);
            }
        }
    }
    // every row's group has been waited on by the warp that took the row
    if (!__syncthreads_and(landed)) {
        if (threadIdx.x == 0) record_error(a.err, NVFP4_ERR_TIMEOUT, 6);
        return;
    }
    // the warp's tasks: [tb, te) of the (512-column chunk, row) tasks in chunk-major order
    const int ntask = nrun * nr;
    const int tb = (int)((int64_t)ntask * warp / kQWarps), te = (int)((int64_t)ntask * (warp + 1) / kQWarps);
    if (!a.given) {
        // ---- max |m| over the CTA's rows
        float lmax = 0.0f;
        int c = tb / max(nr, 1), r = tb - c * nr;  // task tb's chunk and row
        float sc1[16], sh[16];
        ln_columns(a, 512 * c + 16 * lane, 512 * c + 16 * lane < cols, sc1, sh);
        for (int k = 0; tb + k < te; k++) {
            const int e0 = 512 * c + 16 * lane;
            float mx = 0.0f;
            if (e0 < cols) {
                float f[16];
                ln_load16(xs + r * row_bytes + 2 * e0, lane, f);
                const float2 rs = st[r];
                mx = ln_modulate16(f, rs.x, rs.y, sc1, sh);
            }
            lmax = fmaxf(lmax, mx);
            if (++r == nr && tb + k + 1 < te) {
                r = 0;
                ++c;
                ln_columns(a, 512 * c + 16 * lane, 512 * c + 16 * lane < cols, sc1, sh);
            }
        }
        uint32_t m = __float_as_uint(lmax);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0) s_red[warp] = m;
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t c0 = 0u;
#pragma unroll
            for (int i = 0; i < kQWarps; i++) c0 = max(c0, s_red[i]);
            uint32_t tot[2];
            if (!grid_max_exchange(a.ctl, a.err, a.limit_ns, par, G, c0, 0u, tot)) s_ok = 0;
            s_total = tot[0];
        }
        __syncthreads();
        if (!s_ok) return;
        if (threadIdx.x == 0) {
            const float a32 = __fdiv_rn(__uint_as_float(s_total), 2688.0f);  // amax / (6 * 448)
            s_a32 = a32;
            if (blockIdx.x == 0) *a.gscale = a32;
        }
        if (blockIdx.x == 0 && threadIdx.x == 32) grid_barrier_retire(a.ctl, par, epoch);
    } else if (threadIdx.x == 0) {
        s_a32 = *a.gscale;
    }
    __syncthreads();
    {
        const int c = threadIdx.x;
        if (c < 256) {
            const float sv = e4m3_value((uint32_t)c);
            s_inv[c] = (s_a32 == 0.0f || sv == 0.0f) ? 0.0f : __frcp_rn(__fmul_rn(sv, s_a32));
        }
        if (threadIdx.x == 0) {
            s_d6 = __fmul_rn(6.0f, s_a32);
            s_d4 = __fmul_rn(4.0f, s_a32);
        }
        __syncthreads();
    }
    // ---- encode every block of m, the same tasks
    const EncodeConsts kc{s_a32, s_d6, s_d4, s_inv};
    const int64_t tiles_c = cols / 64;
    {
        int c = tb / max(nr, 1), r = tb - c * nr;
        float sc1[16], sh[16];
        ln_columns(a, 512 * c + 16 * lane, 512 * c + 16 * lane < cols, sc1, sh);
        for (int k = 0; tb + k < te; k++) {
            const int e0 = 512 * c + 16 * lane;
            if (e0 < cols) {
                float f[16];
                ln_load16(xs + r * row_bytes + 2 * e0, lane, f);
                const float2 rs = st[r];
                const float mx = ln_modulate16(f, rs.x, rs.y, sc1, sh);
                uint32_t code = kc.d6 == 0.0f ? 0u : e4m3_code(__fdiv_rn(mx, kc.d6));
                uint2 cw = encode16(f, kc.inv_tab[code]);
                if (SEARCH) {
                    const uint32_t code4 = kc.d4 == 0.0f ? 0u : e4m3_code(__fdiv_rn(mx, kc.d4));
                    const uint2 c4 = encode16(f, kc.inv_tab[code4]);
                    if (block_sq_error(f, c4, code4, kc.a32) < block_sq_error(f, cw, code, kc.a32)) {
                        code = code4;
                        cw = c4;
                    }
                }
                const int64_t gr = r0 + r;
                const int b = e0 >> 4;
                *reinterpret_cast<uint2*>(a.codes + gr * (cols / 2) + (e0 >> 1)) = cw;
                if (a.swizzled)
                    a.scales[swz_offset(gr, b, tiles_c)] = (uint8_t)code;
                else
                    a.scales[gr * (cols / 16) + b] = (uint8_t)code;
            }
            if (++r == nr && tb + k + 1 < te) {
                r = 0;
                ++c;
                ln_columns(a, 512 * c + 16 * lane, 512 * c + 16 * lane < cols, sc1, sh);
            }
        }
    }
    // zero the padding rows of the swizzled scale tiles (rows past `rows` up to the next multiple of 128)
    if (a.swizzled) {
        const int64_t rows_pad = ((int64_t)a.rows + 127) / 128 * 128;
        const int64_t sc_pad = tiles_c * 4;
        const int64_t npad = (rows_pad - a.rows) * sc_pad;
        for (int64_t i = (int64_t)blockIdx.x * kQThreads + threadIdx.x; i < npad; i += (int64_t)G * kQThreads) {
            const int64_t r = a.rows + i / sc_pad, c = i % sc_pad;
            a.scales[swz_offset(r, c, tiles_c)] = 0;
        }
    }
}

// LayerNorm statistics of each row (one warp per row), in the fixed order of
// the one-launch LayerNorm + modulate + quantize: lane j adds elements
// 256c + 8j .. 256c + 8j + 7 of chunks c = 0, 1, ... in order, the 32 partial
// sums meet in an xor butterfly (16, 8, 4, 2, 1); mean = S1 / cols,
// var = S2 / cols with S2 over fl32(x - mean)^2, rstd = 1 / sqrt(var + eps),
// every step correctly rounded binary32.
__device__ __forceinline__ float warp_butterfly_sum(float s) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s = __fadd_rn(s, __shfl_xor_sync(0xFFFFFFFFu, s, o));
    return s;
}

constexpr int kStatRegChunks = 16;  // 256-element chunks a warp holds in registers (rows up to 4096 columns)

__device__ __forceinline__ float stat_sum(const uint4& v, float s) {
    float f[8];
    bf16x8_to_f32(v, f);
#pragma unroll
    for (int i = 0; i < 8; i++) s = __fadd_rn(s, f[i]);
    return s;
}

__device__ __forceinline__ float stat_sq_sum(const uint4& v, float mean, float s2) {
    float f[8];
    bf16x8_to_f32(v, f);
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const float d = __fsub_rn(f[i], mean);
        s2 = __fadd_rn(s2, __fmul_rn(d, d));
    }
    return s2;
}

__global__ void __launch_bounds__(256) ln_stats_kernel(const uint8_t* x, int64_t ld_bytes, int rows, int cols,
                                                       float eps, float2* out) {
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const uint8_t* xr = x + (int64_t)row * ld_bytes;
    const int nch = (cols + 255) / 256;
    const float n = (float)cols;
    float s = 0.0f, s2 = 0.0f, mean;
    if (nch <= kStatRegChunks) {
        // the lane's 16 bytes of every chunk loaded at once and kept for both sums
        uint4 v[kStatRegChunks];
#pragma unroll
        for (int c = 0; c < kStatRegChunks; c++) {
            const int e0 = 256 * c + 8 * lane;
            v[c] = (c < nch && e0 < cols) ? __ldg(reinterpret_cast<const uint4*>(xr + 2 * e0)) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int c = 0; c < kStatRegChunks; c++)
            if (c < nch && 256 * c + 8 * lane < cols) s = stat_sum(v[c], s);
        mean = __fdiv_rn(warp_butterfly_sum(s), n);
#pragma unroll
        for (int c = 0; c < kStatRegChunks; c++)
            if (c < nch && 256 * c + 8 * lane < cols) s2 = stat_sq_sum(v[c], mean, s2);
    } else {
        for (int c = 0; c < nch; c++) {
            const int e0 = 256 * c + 8 * lane;
            if (e0 < cols) s = stat_sum(__ldg(reinterpret_cast<const uint4*>(xr + 2 * e0)), s);
        }
        mean = __fdiv_rn(warp_butterfly_sum(s), n);
        for (int c = 0; c < nch; c++) {
            const int e0 = 256 * c + 8 * lane;
            if (e0 < cols) s2 = stat_sq_sum(__ldg(reinterpret_cast<const uint4*>(xr + 2 * e0)), mean, s2);
        }
    }
    const float var = __fdiv_rn(warp_butterfly_sum(s2), n);
    if (lane == 0) out[row] = make_float2(mean, __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, eps))));
}

// Channel means of a KV chunk for K-smoothing, in a fixed binary32 order:
// channel c = h * d + j of the chunk [T][H*d]; partial p (p = 0..31) sums
// tokens p, p+32, p+64, ... in increasing order from +0, the 32 partials meet
// in an xor butterfly (16, 8, 4, 2, 1), and mean = S / T, each step one
// correctly rounded binary32 operation.  A block of 1024 threads covers 32
// channels of one tensor: warp p computes partial p of one channel per lane
// (a 2-byte load a token, 64 contiguous bytes a warp), the partials meet in
// shared memory, and warp w finishes channel w.
struct MeanArgs {
    const uint8_t* x[2];  // bf16 [T][hd]
    float* mean[2];       // [hd], NULL: tensor not smoothed
    int T;
    int hd;               // H * d, a multiple of 16
    // ROPE kernels: the keys (tensor 0) are turned first, as the quantize does
    const float* rope_cos;  // [T][d / 2]
    const float* rope_sin;
    int d;
};

// the bf16 value at p as binary32
__device__ __forceinline__ float ldg_bf16(const uint8_t* p) {
    return __uint_as_float((uint32_t)__ldg(reinterpret_cast<const uint16_t*>(p)) << 16);
}

template <bool ROPE>
__global__ void __launch_bounds__(1024) kv_channel_mean_kernel(MeanArgs a) {
    __shared__ float part[32][33];
    const int t = blockIdx.y;
    const uint8_t* x = t ? a.x[1] : a.x[0];
    float* out = t ? a.mean[1] : a.mean[0];
    if (out == nullptr) return;  // the whole block
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x * 32 + lane;
    float s0 = 0.0f;
    if (ROPE && t == 0) {
        // each key is turned with its pair partner, the neighbouring lane's
        // channel (channels 2p, 2p + 1 sit in lanes 2i, 2i + 1; hd is even, so
        // both are in range or neither), by its token's angle.  Every lane
        // loads (lanes past hd read channel 0 and their sums are dropped), so
        // the exchanges are warp-wide; token loops are uniform per warp.
        const int cc = c < a.hd ? c : 0;
        const int hp = a.d >> 1;
        const int pr = (cc % a.d) >> 1;
        const bool odd = (lane & 1) != 0;
        const int64_t stride = (int64_t)32 * a.hd * 2;
        const uint8_t* p = x + ((int64_t)warp * a.hd + cc) * 2;
        const float* pc = a.rope_cos + (int64_t)warp * hp + pr;
        const float* ps = a.rope_sin + (int64_t)warp * hp + pr;
        const int64_t tstride = (int64_t)32 * hp;
        auto turn = [&](float xv, float cs, float sn) {
            const float xp = __shfl_xor_sync(0xFFFFFFFFu, xv, 1);
            return odd ? __fadd_rn(__fmul_rn(xp, sn), __fmul_rn(xv, cs))
                       : __fsub_rn(__fmul_rn(xv, cs), __fmul_rn(xp, sn));
        };
        int tok = warp;
        for (; tok + 7 * 32 < a.T; tok += 8 * 32, p += 8 * stride, pc += 8 * tstride, ps += 8 * tstride) {
            float xv[8], cs[8], sn[8];
#pragma unroll
            for (int k = 0; k < 8; k++) {
                xv[k] = ldg_bf16(p + k * stride);
                cs[k] = __ldg(pc + k * tstride);
                sn[k] = __ldg(ps + k * tstride);
            }
#pragma unroll
            for (int k = 0; k < 8; k++) s0 = __fadd_rn(s0, turn(xv[k], cs[k], sn[k]));
        }
        for (; tok < a.T; tok += 32, p += stride, pc += tstride, ps += tstride)
            s0 = __fadd_rn(s0, turn(ldg_bf16(p), __ldg(pc), __ldg(ps)));
    } else if (c < a.hd) {
        const uint8_t* p = x + ((int64_t)warp * a.hd + c) * 2;
        const int64_t stride = (int64_t)32 * a.hd * 2;
        // up to 24 tokens' loads in flight before their (in-order) adds
        int tok = warp;
        for (; tok + 23 * 32 < a.T; tok += 24 * 32, p += 24 * stride) {
            uint32_t v[24];
#pragma unroll
            for (int k = 0; k < 24; k++) v[k] = __ldg(reinterpret_cast<const uint16_t*>(p + k * stride));
#pragma unroll
            for (int k = 0; k < 24; k++) s0 = __fadd_rn(s0, __uint_as_float(v[k] << 16));
        }
        for (; tok < a.T; tok += 32, p += stride)
            s0 = __fadd_rn(s0, __uint_as_float((uint32_t)__ldg(reinterpret_cast<const uint16_t*>(p)) << 16));
    }
    part[warp][lane] = s0;
    __syncthreads();
    float sum = part[lane][warp];  // lane p holds partial p of channel `warp`
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xFFFFFFFFu, sum, o));
    const int cc = blockIdx.x * 32 + warp;
    if (lane == 0 && cc < a.hd) out[cc] = __fdiv_rn(sum, (float)a.T);
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
    const float* mean[2];    // K-smoothing channel means [n_slots][hd] (NULL: none)
    int hd;                  // H * d
};

// 8 E2M1 codes (32 bits) with one block scale and the slot's a32 -> 8 bf16
// (16 bytes): bf16_rne(fl32(fl32(e2m1 * s) * a32)); e2m1 * s is exact in
// binary16, so the only roundings are the two the definition has.  The
// binary32 products go two at a time (mul.rn.f32x2, each lane rounded as a
// binary32 multiply).  ADD (K-smoothing): the 8 channel means m are added to
// the products first, bf16_rne(fl32(fl32(fl32(e2m1 * s) * a32) + m)).
template <bool ADD>
__device__ __forceinline__ uint4 dequant8(uint32_t q, uint8_t sc, unsigned long long a2, const float4* m) {
    const __half2 s2 = e4m3x2_to_half2((uint16_t)(sc | (sc << 8)));
    float mv[8];
    if (ADD) {
        const float4 m0 = __ldg(m), m1 = __ldg(m + 1);
        mv[0] = m0.x; mv[1] = m0.y; mv[2] = m0.z; mv[3] = m0.w;
        mv[4] = m1.x; mv[5] = m1.y; mv[6] = m1.z; mv[7] = m1.w;
    }
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const __half2 v = __hmul2(e2m1x2_to_half2((q >> (8 * j)) & 0xFFu), s2);  // exact
        const float2 f = __half22float2(v);
        unsigned long long p;
        asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(p) : "l"(*reinterpret_cast<const unsigned long long*>(&f)), "l"(a2));
        float2 y = *reinterpret_cast<const float2*>(&p);
        if (ADD) {
            // scalar adds: the compiler may contract a packed multiply and a
            // packed add into one fused multiply-add, which would skip the
            // product's own rounding; __fadd_rn is never contracted
            y.x = __fadd_rn(y.x, mv[2 * j]);
            y.y = __fadd_rn(y.y, mv[2 * j + 1]);
        }
        const __nv_bfloat162 b = __floats2bfloat162_rn(y.x, y.y);
        o[j] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// 16 bytes to global memory with the streaming hint: the dequantized output
// is written once and not read back by this kernel, so it should not push the
// codes out of L2.
__device__ __forceinline__ void st_stream16(void* p, const uint4& v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// One resident wave of warps (at most 32 registers a thread, so 8 blocks of
// 256 fit an SM); each warp walks units (512-element runs of the listed
// slots) two at a time with a stride of twice the warp count.  A lane loads
// 4 code bytes and a scale byte per half unit and stores 16 bytes, so every
// warp store covers 512 contiguous bytes.  Positions are 32-bit: the list
// index is below 2^31 and the run index below slot_elems / 512 <= 2^31.
// SMOOTH: the tensor's channel means (when it has them) are added back.
template <bool SMOOTH>
__global__ void __launch_bounds__(kThreads, SMOOTH ? 6 : 8) kv_dequant_kernel(DequantArgs a) {
    const int t = blockIdx.y;
    const int lane = threadIdx.x & 31;
    const int64_t ups = (a.slot_elems + 511) / 512;  // 512-element runs per slot
    const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
    const uint8_t* cb = t ? a.codes[1] : a.codes[0];
    const uint8_t* sb = t ? a.scales[1] : a.scales[0];
    const float* gb = t ? a.gscale[1] : a.gscale[0];
    uint8_t* ob = t ? a.out[1] : a.out[0];
    const float* mb = SMOOTH ? (t ? a.mean[1] : a.mean[0]) : nullptr;
    const int64_t w0 = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    const uint32_t ups32 = (uint32_t)ups;
    const uint32_t qs = (uint32_t)(2 * nwarps / ups), rs = (uint32_t)(2 * nwarps - (int64_t)qs * ups);
    const uint32_t n = (uint32_t)a.n;
    uint32_t pi[2], pu[2];
#pragma unroll
    for (int k = 0; k < 2; k++) {
        const int64_t unit = w0 + k * nwarps;
        pi[k] = (uint32_t)(unit / ups);
        pu[k] = (uint32_t)(unit - (int64_t)pi[k] * ups);
    }
    while (pi[0] < n) {
        // both units' loads first, then decode and store
        uint32_t q[2][2], sc[2];
        float a32[2];
        int64_t o0[2];
        const float* mk[2];  // SMOOTH: the slot's channel means
        int halves[2];
#pragma unroll
        for (int k = 0; k < 2; k++) {
            q[k][0] = q[k][1] = 0;
            sc[k] = 0;
            a32[k] = 0.0f;
            o0[k] = 0;
            halves[k] = 0;
            mk[k] = nullptr;
            if (pi[k] >= n) continue;
            const int32_t s = __ldg(a.slots + pi[k]);
            if (s < 0 || s >= a.n_slots) {
                if (lane == 0 && pu[k] == 0 && t == 0) record_error(a.err, NVFP4_ERR_DEVICE, pi[k]);
                continue;
            }
            const int64_t e0 = (int64_t)pu[k] * 512 + 8 * lane;
            const int64_t src = (int64_t)s * a.slot_elems + e0;
            o0[k] = (int64_t)pi[k] * a.slot_elems + e0;
            a32[k] = __ldg(gb + s);
            if (SMOOTH && mb) mk[k] = mb + (int64_t)s * a.hd;
            // slot_elems is a multiple of 64 and e0 of 8: a word that starts
            // inside the slot ends inside it
            if (e0 < a.slot_elems) {
                q[k][0] = __ldg(reinterpret_cast<const uint32_t*>(cb + src / 2));
                sc[k] = __ldg(sb + src / 16);
                halves[k] = 1;
            }
            if (e0 + 256 < a.slot_elems) {
                q[k][1] = __ldg(reinterpret_cast<const uint32_t*>(cb + (src + 256) / 2));
                sc[k] |= (uint32_t)__ldg(sb + (src + 256) / 16) << 8;
                halves[k] = 2;
            }
        }
#pragma unroll
        for (int k = 0; k < 2; k++) {
            const float2 aa = make_float2(a32[k], a32[k]);
            const unsigned long long a2 = *reinterpret_cast<const unsigned long long*>(&aa);
#pragma unroll
            for (int h = 0; h < 2; h++) {
                if (h >= halves[k]) continue;
                uint4 v;
                if (SMOOTH && mk[k]) {
                    // fewer than 2^31 elements a slot (checked on the host): the
                    // lane's 8 channels are consecutive (hd is a multiple of 16)
                    const uint32_t e = (uint32_t)(pu[k] * 512 + 8 * lane + 256 * h);
                    const float4* m = reinterpret_cast<const float4*>(mk[k] + e % (uint32_t)a.hd);
                    v = dequant8<true>(q[k][h], (uint8_t)(sc[k] >> (8 * h)), a2, m);
                } else {
                    v = dequant8<false>(q[k][h], (uint8_t)(sc[k] >> (8 * h)), a2, nullptr);
                }
                st_stream16(ob + (o0[k] + 256 * h) * 2, v);
            }
        }
#pragma unroll
        for (int k = 0; k < 2; k++) {
            pi[k] += qs;
            pu[k] += rs;
            if (pu[k] >= ups32) {
                pu[k] -= ups32;
                pi[k] += 1;
            }
        }
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
static PerDevice<int> g_sms;

// SMs of the current device (148 on B200 if the query fails)
static int num_sms() {
    int n = 0;
    const nvfp4_status st = g_sms.get(&n, [](int dev, int& v) {
        return cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? NVFP4_OK
                                                                                               : NVFP4_ERR_CUDA;
    });
    return st == NVFP4_OK && n > 0 ? n : 148;
}

// resident 256-thread blocks per SM of the two dequant kernels on the current device
struct DequantResidency {
    int blocks[2];
};
static PerDevice<DequantResidency> g_dequant_resident;

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// dynamic shared memory of the one-launch LayerNorm quantize (rows and their
// statistics); larger inputs take the two-launch path
constexpr int64_t kLnSmemMax = 224 * 1024;
static PerDevice<bool> g_ln_attr;

static int grid_for(int64_t work_items, int per_cta, int cap) {
    int64_t g = (work_items + per_cta - 1) / per_cta;
    if (g < 1) g = 1;
    if (g > cap) g = cap;
    return (int)g;
}

static nvfp4_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// Magic number for b / d with b < 2^31 (division by an invariant integer,
// Granlund and Montgomery): l = ceil(log2 d), m = floor(2^(31 + l) / d) + 1
// (fits in 32 bits), b / d = umulhi(b, m) >> (l - 1).  d >= 2.
static void div_magic(uint32_t d, uint32_t* m, int* shift) {
    int l = 0;
    while ((1ull << l) < d) l++;
    *m = (uint32_t)(((uint64_t)1 << (31 + l)) / d + 1);
    *shift = l - 1;
}

// one fused, cooperative launch over one or two tensors of the same shape
static nvfp4_status quantize_impl(int ntensors, const void* const* x, int64_t rows, int64_t cols, int64_t ld,
                                  void* const* codes, void* const* scales, float* const* gscale, bool given,
                                  bool swizzled, bool search, void* workspace, cudaStream_t stream,
                                  const float2* ln_stats = nullptr, const void* mod_scale = nullptr,
                                  const void* mod_shift = nullptr, const float* const* smooth_mean = nullptr,
                                  int smooth_hd = 0, const float* rope_cos = nullptr, const float* rope_sin = nullptr,
                                  int rope_d = 0) {
    QuantArgs a{};
    for (int t = 0; t < ntensors; t++) {
        a.x[t] = static_cast<const uint8_t*>(x[t]);
        a.codes[t] = static_cast<uint8_t*>(codes[t]);
        a.scales[t] = static_cast<uint8_t*>(scales[t]);
        a.gscale[t] = gscale[t];
    }
    // the kernel indexes a tensor's 16-element blocks in 32 bits
    if (cols > ((int64_t)1 << 30) || rows * (cols / 16) >= ((int64_t)1 << 31)) return NVFP4_ERR_UNSUPPORTED;
    a.ld_bytes = ld * 2;
    a.tiles_c = cols / 64;
    a.nblk = (uint32_t)(rows * (cols / 16));
    a.nb = (uint32_t)(cols / 16);
    div_magic(a.nb, &a.nb_magic, &a.nb_shift);
    a.runs_per_tensor = (int)((a.nblk + 31u) / 32u);
    a.ntensors = ntensors;
    a.given = given ? 1 : 0;
    a.ctl = static_cast<uint32_t*>(workspace);
    a.err = static_cast<DevError*>(workspace);
    a.limit_ns = 2000000000ull;
    a.ln_stats = ln_stats;
    a.mod_scale = static_cast<const __nv_bfloat16*>(mod_scale);
    a.mod_shift = static_cast<const __nv_bfloat16*>(mod_shift);
    if (smooth_mean) {
        a.smooth_mean[0] = smooth_mean[0];
        a.smooth_mean[1] = ntensors > 1 ? smooth_mean[1] : nullptr;
        a.smooth_hd = smooth_hd;
    }
    if (rope_cos) {
        a.rope_cos = rope_cos;
        a.rope_sin = rope_sin;
        a.rope_d = rope_d;
        a.rope_hd = smooth_hd;
    }
    const int64_t total_runs = (int64_t)a.runs_per_tensor * ntensors;
    const int G = (int)std::min<int64_t>(std::min(num_sms(), kMaxGrid), (total_runs + kQWarps - 1) / kQWarps);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kQThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void (*kern)(QuantArgs);
    if (ln_stats)
        kern = swizzled ? (search ? quantize_fused_kernel<true, true, kXfLn> : quantize_fused_kernel<true, false, kXfLn>)
                        : (search ? quantize_fused_kernel<false, true, kXfLn> : quantize_fused_kernel<false, false, kXfLn>);
    else if (smooth_mean || rope_cos)  // KV chunks only: row-major scales
        kern = search ? quantize_fused_kernel<false, true, kXfSmooth> : quantize_fused_kernel<false, false, kXfSmooth>;
    else
        kern = swizzled ? (search ? quantize_fused_kernel<true, true, kXfNone> : quantize_fused_kernel<true, false, kXfNone>)
                        : (search ? quantize_fused_kernel<false, true, kXfNone> : quantize_fused_kernel<false, false, kXfNone>);
    if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

}  // namespace nvfp4

using namespace nvfp4;

namespace nvfp4 {
// nvfp4_quantize's argument checks apart from the workspace (shared with the
// no-allocation entry point, which must run them before touching its scratch).
nvfp4_status quantize_check_args(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld, const void* codes,
                                 const void* scales, const float* global_scale, unsigned flags) {
    if (flags & ~(NVFP4_Q_GIVEN_GLOBAL | NVFP4_Q_ROWMAJOR_SCALES | NVFP4_Q_SCALE_SEARCH)) return NVFP4_ERR_INVALID_ARG;
    if (rows < 0 || cols <= 0 || ld < cols) return NVFP4_ERR_INVALID_ARG;
    if (cols % 64 != 0) return NVFP4_ERR_UNSUPPORTED;
    // the kernel indexes a tensor's 16-element blocks in 32 bits
    if (cols > ((int64_t)1 << 30) || rows >= ((int64_t)1 << 31) || rows * (cols / 16) >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED;
    if (!global_scale) return NVFP4_ERR_INVALID_ARG;
    if (rows == 0) return NVFP4_OK;
    if (!x_bf16 || !codes || !scales) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scales) || (ld % 8) != 0 ||
        (reinterpret_cast<uintptr_t>(global_scale) & 3u))
        return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}
}  // namespace nvfp4

extern "C" nvfp4_status nvfp4_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld, void* codes,
                                       void* scales, float* global_scale, unsigned flags, void* workspace,
                                       size_t ws_bytes, nvfp4_stream_t stream) {
    const nvfp4_status chk = quantize_check_args(x_bf16, rows, cols, ld, codes, scales, global_scale, flags);
    if (chk != NVFP4_OK) return chk;
    if (!workspace) return NVFP4_ERR_INVALID_ARG;
    if (ws_bytes < nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, rows, 0, cols)) return NVFP4_ERR_INVALID_ARG;
    if (rows == 0) return NVFP4_OK;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return NVFP4_ERR_MISALIGNED;
    const void* xs[1] = {x_bf16};
    void* cs[1] = {codes};
    void* ss[1] = {scales};
    float* gs[1] = {global_scale};
    return quantize_impl(1, xs, rows, cols, ld, cs, ss, gs, (flags & NVFP4_Q_GIVEN_GLOBAL) != 0,
                         (flags & NVFP4_Q_ROWMAJOR_SCALES) == 0, (flags & NVFP4_Q_SCALE_SEARCH) != 0, workspace,
                         (cudaStream_t)stream);
}

extern "C" nvfp4_status nvfp4_ln_modulate_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                                   const void* mod_scale, const void* mod_shift, float eps,
                                                   void* codes, void* scales, float* global_scale, unsigned flags,
                                                   void* workspace, size_t ws_bytes, nvfp4_stream_t stream) {
    if (flags & ~(NVFP4_Q_GIVEN_GLOBAL | NVFP4_Q_ROWMAJOR_SCALES | NVFP4_Q_SCALE_SEARCH)) return NVFP4_ERR_INVALID_ARG;
    if (rows < 0 || cols <= 0 || ld < cols || !(eps >= 0.0f)) return NVFP4_ERR_INVALID_ARG;
    if (cols % 64 != 0) return NVFP4_ERR_UNSUPPORTED;
    if (rows > ((int64_t)1 << 30) || cols > ((int64_t)1 << 24) || rows * (cols / 16) >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED;
    if (!global_scale || !workspace) return NVFP4_ERR_INVALID_ARG;
    if (ws_bytes < nvfp4_workspace_bytes(NVFP4_OP_LN_QUANTIZE, rows, 0, cols)) return NVFP4_ERR_INVALID_ARG;
    if (rows == 0) return NVFP4_OK;
    if (!x_bf16 || !codes || !scales) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scales) || (ld % 8) != 0 ||
        (mod_scale && !aligned16(mod_scale)) || (mod_shift && !aligned16(mod_shift)) ||
        (reinterpret_cast<uintptr_t>(global_scale) & 3u) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return NVFP4_ERR_MISALIGNED;
    // the row statistics follow the 256-byte control block
    float2* stats = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) + 256);
    // one launch when each CTA's rows fit in shared memory with the staged vectors
    const int G = (int)std::min<int64_t>(std::min(num_sms(), kMaxGrid), rows);
    const int64_t rows_per_cta = (rows + G - 1) / G;
    const int64_t smem = rows_per_cta * cols * 2 + rows_per_cta * 8;
    if (smem <= kLnSmemMax) {
        LnArgs la{};
        la.x = static_cast<const uint8_t*>(x_bf16);
        la.ld_bytes = ld * 2;
        la.rows = (int)rows;
        la.cols = (int)cols;
        la.eps = eps;
        la.mod_scale = static_cast<const __nv_bfloat16*>(mod_scale);
        la.mod_shift = static_cast<const __nv_bfloat16*>(mod_shift);
        la.codes = static_cast<uint8_t*>(codes);
        la.scales = static_cast<uint8_t*>(scales);
        la.gscale = global_scale;
        la.given = (flags & NVFP4_Q_GIVEN_GLOBAL) != 0;
        la.swizzled = (flags & NVFP4_Q_ROWMAJOR_SCALES) == 0;
        la.tile_row = cols / 64 * 512;
        la.stats = stats;
        la.ctl = static_cast<uint32_t*>(workspace);
        la.err = static_cast<DevError*>(workspace);
        la.limit_ns = 2000000000ull;
        const bool search = (flags & NVFP4_Q_SCALE_SEARCH) != 0;
        void (*kern)(LnArgs) = search ? ln_quantize_smem_kernel<true> : ln_quantize_smem_kernel<false>;
        bool attr_ok = false;
        const nvfp4_status ast = g_ln_attr.get(&attr_ok, [](int, bool& v) {
            if (cudaFuncSetAttribute(ln_quantize_smem_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kLnSmemMax) != cudaSuccess ||
                cudaFuncSetAttribute(ln_quantize_smem_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kLnSmemMax) != cudaSuccess)
                return NVFP4_ERR_CUDA;
            v = true;
            return NVFP4_OK;
        });
        if (ast != NVFP4_OK) return ast;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(G);
        cfg.blockDim = dim3(kQThreads);
        cfg.dynamicSmemBytes = (size_t)smem;
        cfg.stream = (cudaStream_t)stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kern, la) != cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_CUDA;
        }
        return NVFP4_OK;
    }
    ln_stats_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, (cudaStream_t)stream>>>(
        static_cast<const uint8_t*>(x_bf16), ld * 2, (int)rows, (int)cols, eps, stats);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
    const void* xs[1] = {x_bf16};
    void* cs[1] = {codes};
    void* ss[1] = {scales};
    float* gs[1] = {global_scale};
    return quantize_impl(1, xs, rows, cols, ld, cs, ss, gs, (flags & NVFP4_Q_GIVEN_GLOBAL) != 0,
                         (flags & NVFP4_Q_ROWMAJOR_SCALES) == 0, (flags & NVFP4_Q_SCALE_SEARCH) != 0, workspace,
                         (cudaStream_t)stream, stats, mod_scale, mod_shift);
}

static nvfp4_status check_cache(const nvfp4_kv_cache* c) {
    if (!c) return NVFP4_ERR_INVALID_ARG;
    if (!c->k_codes || !c->k_scales || !c->v_codes || !c->v_scales || !c->k_global || !c->v_global)
        return NVFP4_ERR_INVALID_ARG;
    if (c->n_slots <= 0 || c->tokens_per_slot <= 0 || c->heads <= 0 || c->head_dim <= 0) return NVFP4_ERR_INVALID_ARG;
    if (c->head_dim % 16 != 0) return NVFP4_ERR_UNSUPPORTED;
    if (c->flags & ~(NVFP4_KV_SCALE_SEARCH | NVFP4_KV_SMOOTH_K | NVFP4_KV_SMOOTH_V)) return NVFP4_ERR_INVALID_ARG;
    const int64_t e = (int64_t)c->tokens_per_slot * c->heads * c->head_dim;
    if (e % 64 != 0 || e > ((int64_t)1 << 40)) return NVFP4_ERR_UNSUPPORTED;
    if (c->flags & (NVFP4_KV_SMOOTH_K | NVFP4_KV_SMOOTH_V)) {
        // smoothing indexes channels with 32-bit arithmetic
        // and divides by the token count in binary32 (exact below 2^24)
        if (e >= ((int64_t)1 << 31) || (int64_t)c->heads * c->head_dim >= ((int64_t)1 << 24) ||
            c->tokens_per_slot >= (1 << 24))
            return NVFP4_ERR_UNSUPPORTED;
        if (((c->flags & NVFP4_KV_SMOOTH_K) && !c->k_mean) || ((c->flags & NVFP4_KV_SMOOTH_V) && !c->v_mean))
            return NVFP4_ERR_INVALID_ARG;
        if (((c->flags & NVFP4_KV_SMOOTH_K) && !aligned16(c->k_mean)) ||
            ((c->flags & NVFP4_KV_SMOOTH_V) && !aligned16(c->v_mean)))
            return NVFP4_ERR_MISALIGNED;
    }
    if (!aligned16(c->k_codes) || !aligned16(c->k_scales) || !aligned16(c->v_codes) || !aligned16(c->v_scales) ||
        (reinterpret_cast<uintptr_t>(c->k_global) & 3u) || (reinterpret_cast<uintptr_t>(c->v_global) & 3u))
        return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

// The chunk's append: channel means first where a tensor is smoothed (of
// the turned keys where a RoPE table is given), then the fused quantize.
static nvfp4_status kv_append_impl(const nvfp4_kv_cache* cache, int32_t slot, const void* k_bf16,
                                   const void* v_bf16, const float* rope_cos, const float* rope_sin,
                                   void* workspace, size_t ws_bytes, cudaStream_t stream) {
    nvfp4_status st = check_cache(cache);
    if (st != NVFP4_OK) return st;
    if (slot < 0 || slot >= cache->n_slots) return NVFP4_ERR_INVALID_ARG;
    if (!k_bf16 || !v_bf16 || !workspace) return NVFP4_ERR_INVALID_ARG;
    const int64_t rows = (int64_t)cache->tokens_per_slot * cache->heads;
    const int64_t e = rows * cache->head_dim;
    if (ws_bytes < nvfp4_workspace_bytes(NVFP4_OP_KV_APPEND, rows, 0, cache->head_dim)) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(k_bf16) || !aligned16(v_bf16) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return NVFP4_ERR_MISALIGNED;
    const bool rope = rope_cos != nullptr;
    if (rope) {
        // flat element and channel indexes are 32-bit in the kernels
        if (e >= ((int64_t)1 << 31) || (int64_t)cache->heads * cache->head_dim >= ((int64_t)1 << 24))
            return NVFP4_ERR_UNSUPPORTED;
        if (!aligned16(rope_cos) || !aligned16(rope_sin)) return NVFP4_ERR_MISALIGNED;
    }
    // The chunk is quantized as one flat row of T*H*d elements: with
    // row-major scales over rows of head_dim this is the same byte layout.
    const void* xs[2] = {k_bf16, v_bf16};
    void* cs[2] = {static_cast<uint8_t*>(cache->k_codes) + (int64_t)slot * (e / 2),
                   static_cast<uint8_t*>(cache->v_codes) + (int64_t)slot * (e / 2)};
    void* ss[2] = {static_cast<uint8_t*>(cache->k_scales) + (int64_t)slot * (e / 16),
                   static_cast<uint8_t*>(cache->v_scales) + (int64_t)slot * (e / 16)};
    float* gs[2] = {cache->k_global + slot, cache->v_global + slot};
    const bool search = (cache->flags & NVFP4_KV_SCALE_SEARCH) != 0;
    const bool sk = (cache->flags & NVFP4_KV_SMOOTH_K) != 0, sv = (cache->flags & NVFP4_KV_SMOOTH_V) != 0;
    const int hd = cache->heads * cache->head_dim;
    if (!sk && !sv)
        return quantize_impl(2, xs, 1, e, e, cs, ss, gs, false, false, search, workspace, stream, nullptr, nullptr,
                             nullptr, nullptr, hd, rope_cos, rope_sin, cache->head_dim);
    // K-smoothing: the slot's channel means first, then the quantize of x - mean
    MeanArgs m{};
    m.x[0] = static_cast<const uint8_t*>(k_bf16);
    m.x[1] = static_cast<const uint8_t*>(v_bf16);
    m.mean[0] = sk ? cache->k_mean + (int64_t)slot * hd : nullptr;
    m.mean[1] = sv ? cache->v_mean + (int64_t)slot * hd : nullptr;
    m.T = cache->tokens_per_slot;
    m.hd = hd;
    m.rope_cos = rope_cos;
    m.rope_sin = rope_sin;
    m.d = cache->head_dim;
    const dim3 grid((unsigned)((hd + 31) / 32), 2);
    if (rope && sk)
        kv_channel_mean_kernel<true><<<grid, 1024, 0, stream>>>(m);
    else
        kv_channel_mean_kernel<false><<<grid, 1024, 0, stream>>>(m);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
    const float* means[2] = {m.mean[0], m.mean[1]};
    return quantize_impl(2, xs, 1, e, e, cs, ss, gs, false, false, search, workspace, stream, nullptr, nullptr,
                         nullptr, means, hd, rope_cos, rope_sin, cache->head_dim);
}

extern "C" nvfp4_status nvfp4_kv_append(const nvfp4_kv_cache* cache, int32_t slot, const void* k_bf16,
                                        const void* v_bf16, void* workspace, size_t ws_bytes, nvfp4_stream_t stream) {
    return kv_append_impl(cache, slot, k_bf16, v_bf16, nullptr, nullptr, workspace, ws_bytes, (cudaStream_t)stream);
}

extern "C" nvfp4_status nvfp4_kv_append_rope(const nvfp4_kv_cache* cache, int32_t slot, const void* k_bf16,
                                             const void* v_bf16, const float* rope_cos, const float* rope_sin,
                                             void* workspace, size_t ws_bytes, nvfp4_stream_t stream) {
    if (!rope_cos || !rope_sin) return NVFP4_ERR_INVALID_ARG;
    return kv_append_impl(cache, slot, k_bf16, v_bf16, rope_cos, rope_sin, workspace, ws_bytes,
                          (cudaStream_t)stream);
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
    const bool smooth = (cache->flags & (NVFP4_KV_SMOOTH_K | NVFP4_KV_SMOOTH_V)) != 0;
    if (smooth) {
        a.mean[0] = (cache->flags & NVFP4_KV_SMOOTH_K) ? cache->k_mean : nullptr;
        a.mean[1] = (cache->flags & NVFP4_KV_SMOOTH_V) ? cache->v_mean : nullptr;
        a.hd = cache->heads * cache->head_dim;
    }
    // one resident wave over K and V together (blockIdx.y picks the tensor)
    void (*kern)(DequantArgs) = smooth ? kv_dequant_kernel<true> : kv_dequant_kernel<false>;
    DequantResidency res{};
    st = g_dequant_resident.get(&res, [](int, DequantResidency& v) {
        for (int sm = 0; sm < 2; sm++) {
            int b = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, sm ? kv_dequant_kernel<true> : kv_dequant_kernel<false>,
                                                              kThreads, 0) != cudaSuccess || b < 2) {
                cudaGetLastError();
                b = 2;
            }
            v.blocks[sm] = b;
        }
        return NVFP4_OK;
    });
    if (st != NVFP4_OK) return st;
    const int64_t units = (int64_t)n * ((a.slot_elems + 511) / 512);
    const int g = grid_for(units, 2 * (kThreads / 32), num_sms() * res.blocks[smooth] / 2);
    kern<<<dim3(g, 2), kThreads, 0, (cudaStream_t)stream>>>(a);
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

