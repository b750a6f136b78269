// Attention of bf16 queries over NVFP4 KV-cache slots, reading the cache
// directly (the reading note's KV store, section 二 推理底座, and its attention
// anchors: the caller lists the slots of A_g | A_s | KV[t - W, t)).
//
// One CTA per (128-query tile, head), 128 threads: thread i owns query row i
// and TMEM lane i.  K and V tiles of 128 tokens are dequantized from the slot
// (E2M1 codes, E4M3 block scales, the slot's a32, the K-smoothing mean when
// the cache has one) straight into shared memory in the layouts the tensor
// cores read, with each thread writing its token's row as 16-byte chunks:
//   Q, K, P: K-major, no swizzle (P is written over K, which the Q K^T
//            product has finished with): element (row r, column c) at
//            (c / 8) * 2048 + r * 16 + (c % 8) * 2 (8-row core matrices 128
//            bytes apart, 8-column chunks 2048 bytes apart);
//   V:       MN-major (the d columns are the MMA's N): element (token t, dim j)
//            at (j / 8) * 2048 + t * 16 + (j % 8) * 2.
// S = Q K^T and O += P V run as tcgen05.mma kind::f16 (bf16 operands, binary32
// accumulators in TMEM: S in columns [0, 128), O in [128, 256)), issued by
// thread 0 and waited on through an mbarrier.  The softmax is one pass with a
// lazy row maximum: P = exp(scale * (s - m)) in bf16 against a reference max m
// that moves only when a tile exceeds it by more than 2^8 (then the row of O
// in TMEM and the running sum are rescaled by the thread that owns the row),
// and O / sum is stored as bf16.  Every wait is
// bounded; a timeout records NVFP4_ERR_TIMEOUT and the CTA stops.
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "common.cuh"

namespace nvfp4 {
namespace attn {

constexpr int kD = 128;       // head_dim (the tile's K for Q K^T, N for P V)
constexpr int kTile = 128;    // queries per CTA, keys per KV tile
constexpr int kThreads = 128;
constexpr int kOperandBytes = kTile * kD * 2;  // 32 KB per bf16 128 x 128 operand
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kSCol = 0, kOCol = 128;
constexpr float kLazyLog2 = 8.0f;  // a row's reference max moves when exceeded by more than 2^8

struct AttnArgs {
    const uint8_t* q;            // bf16 [Tq][H][d]
    uint8_t* o;                  // bf16 [Tq][H][d]
    const uint8_t* codes[2];     // K, V codes of slot 0 (slot s at + s * slot_elems / 2)
    const uint8_t* scales[2];    // K, V row-major scales
    const float* gscale[2];      // [n_slots]
    const float* mean[2];        // K-smoothing means [n_slots][H * d] or NULL
    const int32_t* slots;
    int n, n_slots, tq, tokens, heads;
    int64_t slot_elems;
    float scale_log2;            // softmax scale * log2(e)
    DevError* err;
    uint32_t* rescales;          // count of warp-level rescales of O (diagnostic)
    uint64_t limit_ns;
};

// instruction descriptor of kind::f16: binary32 accumulator, A and B both
// binary16 (bf = 0) or both bf16 (bf = 1), A K-major, B K-major (b_mn = 0) or
// MN-major (1), M = N = 128
__host__ __device__ constexpr uint32_t idesc_f16(int b_mn, int bf) {
    return (1u << 4) | ((uint32_t)bf << 7) | ((uint32_t)bf << 10) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(kTile >> 3) << 17) | ((uint32_t)(kTile >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        "}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void st_shared16(uint32_t addr, const uint4& v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// 8 E2M1 codes with their block scale and the slot's a32 -> 8 bf16, as the
// cache's dequant: bf16_rne(fl32(fl32(e2m1 * s) * a32) [+ mean]).
__device__ __forceinline__ uint4 dq8(uint32_t q, uint32_t sc, float a32, const float* m) {
    const __half2 s2 = e4m3x2_to_half2((uint16_t)(sc | (sc << 8)));
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const float2 f = __half22float2(__hmul2(e2m1x2_to_half2((q >> (8 * j)) & 0xFFu), s2));
        float y0 = __fmul_rn(f.x, a32), y1 = __fmul_rn(f.y, a32);
        if (m) {
            y0 = __fadd_rn(y0, __ldg(m + 2 * j));
            y1 = __fadd_rn(y1, __ldg(m + 2 * j + 1));
        }
        const __nv_bfloat162 b = __floats2bfloat162_rn(y0, y1);
        o[j] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// 8 E2M1 codes times their block scale, exactly, as binary16 (every product
// e2m1 * s of an E2M1 value and an E4M3 scale is exact in binary16): the
// operand values of the binary16 path, whose tensor scale a32 is applied to
// the products instead.
__device__ __forceinline__ uint4 raw8(uint32_t q, uint32_t sc) {
    const __half2 s2 = e4m3x2_to_half2((uint16_t)(sc | (sc << 8)));
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const __half2 v = __hmul2(e2m1x2_to_half2((q >> (8 * j)) & 0xFFu), s2);
        o[j] = *reinterpret_cast<const uint32_t*>(&v);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// One token row (token `tok` of slot s, head h) of K or V as stored: 64 code
// bytes, 8 scale bytes and the slot's a32; zeros when the token is past the
// slot's end.  Fetched a tile ahead so the loads overlap the tile in flight.
struct RowRaw {
    uint4 c[4];
    uint2 sc;
    float a32;
    bool valid;
};

__device__ __forceinline__ RowRaw fetch_row(const AttnArgs& a, int t, int s, int tok, int h) {
    RowRaw r;
    r.valid = tok < a.tokens;
    if (r.valid) {
        const int64_t e = (int64_t)s * a.slot_elems + ((int64_t)tok * a.heads + h) * kD;
        const uint4* cp = reinterpret_cast<const uint4*>(a.codes[t] + e / 2);
#pragma unroll
        for (int k = 0; k < 4; k++) r.c[k] = __ldg(cp + k);
        r.sc = __ldg(reinterpret_cast<const uint2*>(a.scales[t] + e / 16));
        r.a32 = __ldg(a.gscale[t] + s);
    } else {
#pragma unroll
        for (int k = 0; k < 4; k++) r.c[k] = make_uint4(0u, 0u, 0u, 0u);
        r.sc = make_uint2(0u, 0u);
        r.a32 = 0.0f;
    }
    return r;
}

// The row's 128 dequantized bf16 values into the operand at `base` (K-major
// and MN-major layouts put a row at the same places); a row past the slot's
// end (codes 0, a32 0, no mean) decodes to zeros.
template <bool RAW>
__device__ __forceinline__ void store_row(const AttnArgs& a, int t, int s, int h, const RowRaw& r, uint32_t base,
                                         int row) {
    const float* m = (a.mean[t] && r.valid) ? a.mean[t] + ((int64_t)s * a.heads + h) * kD : nullptr;
    const uint32_t sw[2] = {r.sc.x, r.sc.y};
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const uint32_t cw[4] = {r.c[k].x, r.c[k].y, r.c[k].z, r.c[k].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int chunk = 4 * k + j;  // elements 8 * chunk .. + 7; block chunk / 2
            const uint32_t sc = (sw[chunk / 8] >> (8 * ((chunk / 2) % 4))) & 0xFFu;
            st_shared16(base + chunk * 2048 + row * 16,
                        RAW ? raw8(cw[j], sc) : dq8(cw[j], sc, r.a32, m ? m + 8 * chunk : nullptr));
        }
    }
}

// RAW (no smoothing mean on either tensor): binary16 operands.  Each Q row is
// scaled by a power of two 2^k (exact) so that its largest magnitude lies in
// [2^14, 2^15), then rounded to binary16; K and V tiles hold e2m1 * s exactly;
// the row's 2^-k and the slot's K scale a32_K multiply the products inside the
// exponent, and P carries a32_V / a32_ref (a32_ref: the largest V scale of the
// listed slots), O being multiplied by a32_ref at the end.  Otherwise: bf16
// operands holding the cache's bf16 dequant (with the smoothing means).
template <bool RAW>
__global__ void __launch_bounds__(kThreads, 2) kv_attention_kernel(const __grid_constant__ AttnArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ uint64_t bar_s, bar_o;
    __shared__ uint32_t tmem_base;
    __shared__ int s_abort;
    const int i = threadIdx.x;  // query row, TMEM lane
    const int warp = i >> 5;
    const int qt = blockIdx.x, h = blockIdx.y;
    // P is written over K: the Q K^T product is done with K before P is formed
    const uint32_t q_s = smem_u32(smem), k_s = q_s + kOperandBytes, v_s = k_s + kOperandBytes, p_s = k_s;
    if (i == 0) {
        mbar_init(&bar_s, 1);
        mbar_init(&bar_o, 1);
        s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, kTmemCols);
        tmem_relinquish();
    }
    // Q row i (zeros past the last query); RAW: times 2^k into binary16
    float q_inv = 1.0f;  // RAW: 2^-k
    {
        const int qrow = qt * kTile + i;
        uint4 v[16];
        if (qrow < a.tq) {
            const uint4* src = reinterpret_cast<const uint4*>(a.q + ((int64_t)qrow * a.heads + h) * kD * 2);
#pragma unroll
            for (int c = 0; c < 16; c++) v[c] = __ldg(src + c);
        } else {
#pragma unroll
            for (int c = 0; c < 16; c++) v[c] = make_uint4(0u, 0u, 0u, 0u);
        }
        if (RAW) {
            uint32_t mx = 0u;  // largest bf16 magnitude bits of the row
#pragma unroll
            for (int c = 0; c < 16; c++)
                mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(v[c].x & 0x7FFF7FFFu, v[c].y & 0x7FFF7FFFu),
                                           __vmaxu2(v[c].z & 0x7FFF7FFFu, v[c].w & 0x7FFF7FFFu)));
            mx = max(mx & 0xFFFFu, mx >> 16);
            // 2^k brings the largest magnitude into [2^14, 2^15): k = 141 - its biased exponent
            const int k = mx == 0u ? 0 : min(100, max(-100, 141 - (int)(mx >> 7)));
            const float pk = __uint_as_float((uint32_t)(127 + k) << 23);
            q_inv = __uint_as_float((uint32_t)(127 - k) << 23);
#pragma unroll
            for (int c = 0; c < 16; c++) {
                uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const __half2 hv = __floats2half2_rn(__uint_as_float(w[e] << 16) * pk,
                                                         __uint_as_float(w[e] & 0xFFFF0000u) * pk);
                    w[e] = *reinterpret_cast<const uint32_t*>(&hv);
                }
                v[c] = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
#pragma unroll
        for (int c = 0; c < 16; c++) st_shared16(q_s + c * 2048 + i * 16, v[c]);
    }
    // RAW: the largest V tensor scale of the listed slots (the same in every thread)
    float a_ref = 1.0f;
    if (RAW) {
        a_ref = 0.0f;
        for (int si = 0; si < a.n; si++) {
            const int s = __ldg(a.slots + si);
            if (s >= 0 && s < a.n_slots) a_ref = fmaxf(a_ref, __ldg(a.gscale[1] + s));
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    const uint32_t t_s = tmem + kSCol, t_o = tmem + kOCol;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    constexpr uint32_t ID_QK = idesc_f16(0, RAW ? 0 : 1), ID_PV = idesc_f16(1, RAW ? 0 : 1);
    const int tiles_per_slot = (a.tokens + kTile - 1) / kTile;
    uint32_t ph_s = 0, ph_o = 0;
    bool ok = true;
    float m_run = -INFINITY, l_run = 0.0f;
    bool first_pv = true;

    if (i == 0 && qt == 0 && h == 0)
        for (int si = 0; si < a.n; si++) {
            const int s = __ldg(a.slots + si);
            if (s < 0 || s >= a.n_slots) record_error(a.err, NVFP4_ERR_DEVICE, (uint32_t)si);
        }
    // the key tiles: tile g is tile g % tiles_per_slot of list entry g / tiles_per_slot;
    // entries with an out-of-range slot are skipped (uniform over the CTA)
    const int G = a.n * tiles_per_slot;
    auto slot_of = [&](int g) { return __ldg(a.slots + g / tiles_per_slot); };
    auto next_tile = [&](int g) {
        while (g < G) {
            const int s = slot_of(g);
            if (s >= 0 && s < a.n_slots) break;
            g += tiles_per_slot - g % tiles_per_slot;
        }
        return g;
    };
    int g = next_tile(0);
    RowRaw kr, vr;
    if (g < G) {
        kr = fetch_row(a, 0, slot_of(g), (g % tiles_per_slot) * kTile + i, h);
        vr = fetch_row(a, 1, slot_of(g), (g % tiles_per_slot) * kTile + i, h);
    }
    while (g < G && ok) {
        const int s = slot_of(g), kt = g % tiles_per_slot;
        const int valid = min(kTile, a.tokens - kt * kTile);
        const int gn = next_tile(g + 1);
        // the previous P V product must be done with K, V and P and with O
        // (every wait's outcome is made uniform over the CTA before anyone
        // acts on it, so all threads take the same barriers)
        if (!first_pv) {
            const bool got = mbar_wait_bounded(&bar_o, ph_o, &s_abort, a.limit_ns);
            ph_o ^= 1u;
            if (!__syncthreads_and(got)) {
                ok = false;
                break;
            }
            tc_fence_after();
        }
        store_row<RAW>(a, 0, s, h, kr, k_s, i);
        store_row<RAW>(a, 1, s, h, vr, v_s, i);
        fence_proxy_async_smem();
        __syncthreads();
        if (i == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < kD / 16; k++)
                mma_f16(t_s, smem_desc(q_s + k * 4096, 2048, 128, kLayoutNone),
                        smem_desc(k_s + k * 4096, 2048, 128, kLayoutNone), ID_QK, k > 0);
            tc_commit(&bar_s);
        }
        // the next tile's rows load while the product and the softmax run
        if (gn < G) {
            kr = fetch_row(a, 0, slot_of(gn), (gn % tiles_per_slot) * kTile + i, h);
            vr = fetch_row(a, 1, slot_of(gn), (gn % tiles_per_slot) * kTile + i, h);
        }
        {
            const bool got = mbar_wait_bounded(&bar_s, ph_s, &s_abort, a.limit_ns);
            ph_s ^= 1u;
            if (!__syncthreads_and(got)) {
                ok = false;
                break;
            }
        }
        tc_fence_after();
        uint32_t r[4][32];
#pragma unroll
        for (int c = 0; c < 4; c++) tmem_ld_32cols(t_s + lane_off + 32 * c, r[c]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 4; c++) tmem_regs_ready(r[c]);
        // online softmax with a lazy maximum, in exponent units t = c_s * S
        // (exp(scale * q.k) = 2^t; RAW: c_s also carries the row's 2^-k and the
        // slot's a32_K): the row's reference max moves only when this tile
        // exceeds it by more than 8, and then O (in TMEM) and the running sum
        // are rescaled; otherwise P stays below 2^8
        const float c_s = RAW ? q_inv * __ldg(a.gscale[0] + s) * a.scale_log2 : a.scale_log2;
        const float w_s = RAW ? (a_ref > 0.0f ? __fdiv_rn(__ldg(a.gscale[1] + s), a_ref) : 0.0f) : 1.0f;
        float smax = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; c++)
#pragma unroll
            for (int j = 0; j < 32; j++)
                if (32 * c + j < valid) smax = fmaxf(smax, __uint_as_float(r[c][j]));
        const float mt = smax * c_s;  // c_s >= 0
        float factor = 1.0f;  // O's rescale, applied after P is formed (S's registers are free then)
        if (mt - m_run > kLazyLog2) {
            factor = ex2(m_run - mt);  // 0 on the first tile (m_run = -inf)
            l_run *= factor;
            m_run = mt;
        }
        // P row i: 2^(t - m_run) times w_s (RAW: a32_V / a32_ref) in binary16
        // (RAW) or bf16, zero for keys past the slot's end
#pragma unroll
        for (int c = 0; c < 4; c++)
#pragma unroll
            for (int q4 = 0; q4 < 4; q4++) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int j0 = 32 * c + 8 * q4 + 2 * e;
                    const float p0 = j0 < valid ? ex2(fmaf(__uint_as_float(r[c][8 * q4 + 2 * e]), c_s, -m_run)) : 0.0f;
                    const float p1 =
                        j0 + 1 < valid ? ex2(fmaf(__uint_as_float(r[c][8 * q4 + 2 * e + 1]), c_s, -m_run)) : 0.0f;
                    l_run += p0 + p1;
                    if (RAW) {
                        const __half2 hv = __floats2half2_rn(p0 * w_s, p1 * w_s);
                        w[e] = *reinterpret_cast<const uint32_t*>(&hv);
                    } else {
                        const __nv_bfloat162 b = __floats2bfloat162_rn(p0, p1);
                        w[e] = *reinterpret_cast<const uint32_t*>(&b);
                    }
                }
                st_shared16(p_s + (4 * c + q4) * 2048 + i * 16, make_uint4(w[0], w[1], w[2], w[3]));
            }
        // tcgen05.ld / st are warp-collective: the warp rescales together when any
        // of its rows needs it (the others multiply by exactly 1)
        if (__any_sync(0xFFFFFFFFu, factor != 1.0f) && !first_pv) {
            if ((i & 31) == 0) atomicAdd(a.rescales, 1u);
            uint32_t o[32];
#pragma unroll 1
            for (int c = 0; c < 4; c++) {
                tmem_ld_32cols(t_o + lane_off + 32 * c, o);
                tmem_ld_wait();
                tmem_regs_ready(o);
#pragma unroll
                for (int j = 0; j < 32; j++) o[j] = __float_as_uint(__uint_as_float(o[j]) * factor);
                tmem_st_32cols(t_o + lane_off + 32 * c, o);
            }
            tmem_st_wait();
        }
        // every row's S is read (and O rescaled) before the next MMAs
        tc_fence_before();
        fence_proxy_async_smem();
        __syncthreads();
        if (i == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < kTile / 16; k++)
                mma_f16(t_o, smem_desc(p_s + k * 4096, 2048, 128, kLayoutNone),
                        smem_desc(v_s + k * 256, 128, 2048, kLayoutNone), ID_PV, (!first_pv || k > 0) ? 1u : 0u);
            tc_commit(&bar_o);
        }
        first_pv = false;
        g = gn;
    }
    // O row i / l -> bf16
    if (ok && !first_pv) {
        const bool got = mbar_wait_bounded(&bar_o, ph_o, &s_abort, a.limit_ns);
        ok = __syncthreads_and(got) != 0;
        tc_fence_after();
    }
    if (!ok) {
        if (i == 0) record_error(a.err, NVFP4_ERR_TIMEOUT, 3);
    } else {
        const int qrow = qt * kTile + i;
        const float inv_l = l_run > 0.0f ? __fdiv_rn(a_ref, l_run) : 0.0f;  // a_ref = 1 unless RAW
        uint32_t r[4][32];
        if (!first_pv) {
#pragma unroll
            for (int c = 0; c < 4; c++) tmem_ld_32cols(t_o + lane_off + 32 * c, r[c]);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 4; c++) tmem_regs_ready(r[c]);
        } else {
#pragma unroll
            for (int c = 0; c < 4; c++)
#pragma unroll
                for (int j = 0; j < 32; j++) r[c][j] = 0u;
        }
        if (qrow < a.tq) {
            uint4* dst = reinterpret_cast<uint4*>(a.o + ((int64_t)qrow * a.heads + h) * kD * 2);
#pragma unroll
            for (int c = 0; c < 4; c++)
#pragma unroll
                for (int g = 0; g < 4; g++) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const __nv_bfloat162 b =
                            __floats2bfloat162_rn(__uint_as_float(r[c][8 * g + 2 * e]) * inv_l,
                                                  __uint_as_float(r[c][8 * g + 2 * e + 1]) * inv_l);
                        w[e] = *reinterpret_cast<const uint32_t*>(&b);
                    }
                    dst[4 * c + g] = make_uint4(w[0], w[1], w[2], w[3]);
                }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace attn
}  // namespace nvfp4

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
using namespace nvfp4;
using namespace nvfp4::attn;

extern "C" int32_t nvfp4_attention_chunks(int32_t t, int32_t sink_global, int32_t shot_start, int32_t sink_shot,
                                          int32_t window, int32_t* out, int32_t max_out) {
    if (t < 0 || sink_global < 0 || sink_shot < 0 || window < 0 || shot_start < 0 || max_out < 0 ||
        (max_out > 0 && !out))
        return -1;
    // ascending walk over [0, t): a chunk is in the set when it lies in any of
    // the three ranges (so each appears once)
    int32_t n = 0;
    const int64_t w0 = (int64_t)t - window;
    for (int64_t c = 0; c < t; c++) {
        const bool in = c < sink_global || (c >= shot_start && c < (int64_t)shot_start + sink_shot) || c >= w0;
        if (!in) {
            // skip the gap up to the next range start in one step
            int64_t next = t;
            if (c < shot_start) next = std::min<int64_t>(next, shot_start);
            if (c < w0) next = std::min<int64_t>(next, w0);
            c = next - 1;
            continue;
        }
        if (n >= max_out) return -1;
        out[n++] = (int32_t)c;
    }
    return n;
}

extern "C" nvfp4_status nvfp4_kv_attention(const nvfp4_kv_cache* cache, const int32_t* slots_dev, int32_t n,
                                           const void* q_bf16, int32_t tq, float scale, void* o_bf16, void* workspace,
                                           size_t ws_bytes, nvfp4_stream_t stream) {
    if (!cache || n < 0 || tq < 0 || !workspace || !(scale >= 0.0f)) return NVFP4_ERR_INVALID_ARG;
    if (ws_bytes < nvfp4_workspace_bytes(NVFP4_OP_KV_ATTENTION, 0, 0, 0)) return NVFP4_ERR_INVALID_ARG;
    if (!cache->k_codes || !cache->k_scales || !cache->v_codes || !cache->v_scales || !cache->k_global ||
        !cache->v_global || cache->n_slots <= 0 || cache->tokens_per_slot <= 0 || cache->heads <= 0)
        return NVFP4_ERR_INVALID_ARG;
    if (cache->head_dim != kD) return NVFP4_ERR_UNSUPPORTED;
    if (cache->flags & ~(NVFP4_KV_SCALE_SEARCH | NVFP4_KV_SMOOTH_K | NVFP4_KV_SMOOTH_V)) return NVFP4_ERR_INVALID_ARG;
    const bool sk = (cache->flags & NVFP4_KV_SMOOTH_K) != 0, sv = (cache->flags & NVFP4_KV_SMOOTH_V) != 0;
    if ((sk && !cache->k_mean) || (sv && !cache->v_mean)) return NVFP4_ERR_INVALID_ARG;
    // the kernel counts key tiles over the whole list in 32 bits
    if ((int64_t)n * ((cache->tokens_per_slot + kTile - 1) / kTile) >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED;
    if (tq == 0) return NVFP4_OK;
    if (!q_bf16 || !o_bf16 || (n > 0 && !slots_dev)) return NVFP4_ERR_INVALID_ARG;
    auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!a16(q_bf16) || !a16(o_bf16) || !a16(cache->k_codes) || !a16(cache->v_codes) || !a16(cache->k_scales) ||
        !a16(cache->v_scales) || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        (reinterpret_cast<uintptr_t>(slots_dev) & 3u))
        return NVFP4_ERR_MISALIGNED;
    AttnArgs a{};
    a.q = static_cast<const uint8_t*>(q_bf16);
    a.o = static_cast<uint8_t*>(o_bf16);
    a.codes[0] = static_cast<const uint8_t*>(cache->k_codes);
    a.codes[1] = static_cast<const uint8_t*>(cache->v_codes);
    a.scales[0] = static_cast<const uint8_t*>(cache->k_scales);
    a.scales[1] = static_cast<const uint8_t*>(cache->v_scales);
    a.gscale[0] = cache->k_global;
    a.gscale[1] = cache->v_global;
    a.mean[0] = sk ? cache->k_mean : nullptr;
    a.mean[1] = sv ? cache->v_mean : nullptr;
    a.slots = slots_dev;
    a.n = n;
    a.n_slots = cache->n_slots;
    a.tq = tq;
    a.tokens = cache->tokens_per_slot;
    a.heads = cache->heads;
    a.slot_elems = (int64_t)cache->tokens_per_slot * cache->heads * cache->head_dim;
    const float sc = scale > 0.0f ? scale : 1.0f / sqrtf((float)kD);
    a.scale_log2 = sc * 1.4426950408889634f;  // log2(e)
    a.err = static_cast<DevError*>(workspace);
    a.rescales = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + 16);
    a.limit_ns = 2000000000ull;
    const int smem = 3 * kOperandBytes;
    // caches without smoothing means take the binary16 path
    const bool raw = !sk && !sv;
    void (*kern)(AttnArgs) = raw ? kv_attention_kernel<true> : kv_attention_kernel<false>;
    // the shared-memory attribute of both variants, set once per device
    static PerDevice<bool> attr_set;
    bool done = false;
    const nvfp4_status ast = attr_set.get(&done, [smem](int, bool& v) {
        if (cudaFuncSetAttribute(kv_attention_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess ||
            cudaFuncSetAttribute(kv_attention_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess)
            return NVFP4_ERR_CUDA;
        v = true;
        return NVFP4_OK;
    });
    if (ast != NVFP4_OK) return ast;
    const dim3 grid((unsigned)((tq + kTile - 1) / kTile), (unsigned)cache->heads);
    kern<<<grid, kThreads, smem, (cudaStream_t)stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
