// Attention of bf16 queries over NVFP4 KV-cache slots, reading the cache
// directly (the reading note's KV store, section 二 推理底座, and its attention
// anchors: the caller lists the slots of A_g | A_s | KV[t - W, t)).
//
// Work unit: one head and two 128-query tiles of it (A and B), which share
// every dequantized K and V tile.  Persistent CTAs, one per SM, walk the units;
// inside a CTA the warps split the work:
//   warps 0-3   softmax of tile A (thread = query row = TMEM lane),
//   warps 4-7   softmax of tile B,
//   warps 8-11  K / V producers: each thread dequantizes one key row of the
//               128-key tile (E2M1 codes, E4M3 block scales, the slot's a32,
//               the K-smoothing mean when the cache has one) straight into
//               shared memory in the layout the tensor cores read,
//   warp 12     one thread issuing the tcgen05 products and their commits.
// Shared memory (224 KB): Q_A, Q_B, K, V[2], P_A, P_B, each a 128 x 128
// 16-bit operand of 8 x 8 core matrices without swizzle, element (row r,
// column c) at (c / 8) * 2048 + r * 16 + (c % 8) * 2 (8-row core matrices 128
// bytes apart, 8-column chunks 2048 bytes apart): Q, K and P K-major; V
// MN-major (rows = keys, columns = the d outputs).  TMEM (512 columns): S_A,
// S_B (binary32 scores) and O_A, O_B (binary32 outputs), 128 columns each.
// S = Q K^T and O += P V run as tcgen05.mma kind::f16 (binary32 accumulation)
// in the order PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1) per key tile j, so
// while one query tile's softmax runs the tensor cores work on the other
// tile's products.  The softmax forms P = exp(scale * (s - m)) in one pass
// against a reference row maximum m; only a row whose weights in the tile sum
// above 2^15 (always the first tile) reads the tile's maximum, moves m to it
// when it exceeds m by more than 2^8 (then the row of O in TMEM and the
// running sum are rescaled by the thread that owns the row) and forms P
// again.  O / sum is stored as bf16.  Every wait is bounded; a timeout
// records NVFP4_ERR_TIMEOUT and every role stops.
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "common.cuh"

namespace nvfp4 {
namespace attn {

constexpr int kD = 128;                         // head_dim (the K of Q K^T, the N of P V)
constexpr int kTile = 128;                      // queries per query tile, keys per key tile
constexpr int kProducerWarp0 = 8;               // warps 0-7 softmax, 8-11 producers
constexpr int kMmaWarp = 12;
constexpr int kThreads = (kMmaWarp + 1) * 32;   // 416
constexpr int kGroup = 128;                     // threads of one softmax group, of the producers
constexpr int kOperandBytes = kTile * kD * 2;   // 32 KB per 16-bit 128 x 128 operand
constexpr uint32_t kSmemQ = 0, kSmemK = 2 * kOperandBytes, kSmemV = 3 * kOperandBytes, kSmemP = 5 * kOperandBytes;
constexpr int kSmemBytes = 7 * kOperandBytes;   // Q_A Q_B K V0 V1 P_A P_B
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 0, kOCol = 256;      // S_X at 128 X, O_X at 256 + 128 X
constexpr float kLazyLog2 = 8.0f;  // a row's reference max moves when exceeded by more than 2^8
constexpr float kPMax = 32768.0f;  // a tile's weights summing above 2^15 make the row check its max

struct AttnArgs {
    const uint8_t* q;            // bf16 [Tq][H][d]
    uint8_t* o;                  // bf16 [Tq][H][d]
    const uint8_t* codes[2];     // K, V codes of slot 0 (slot s at + s * slot_elems / 2)
    const uint8_t* scales[2];    // K, V row-major scales
    const float* gscale[2];      // [n_slots]
    const float* mean[2];        // K-smoothing means [n_slots][H * d] or NULL
    const int32_t* slots;
    int n, n_slots, tq, tokens, heads;
    int n_qt, n_qp, n_units;     // query tiles, pairs of them, units (pairs x heads)
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
    // the row's eight block scales, two per conversion
    __half2 sp[4];
#pragma unroll
    for (int b2 = 0; b2 < 4; b2++)
        sp[b2] = e4m3x2_to_half2((uint16_t)(((b2 < 2 ? r.sc.x : r.sc.y) >> (16 * (b2 & 1))) & 0xFFFFu));
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const uint32_t cw[4] = {r.c[k].x, r.c[k].y, r.c[k].z, r.c[k].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int chunk = 4 * k + j;  // elements 8 * chunk .. + 7; block chunk / 2
            const int blk = chunk / 2;
            const __half2 s2 = (blk & 1) ? __high2half2(sp[blk / 2]) : __low2half2(sp[blk / 2]);
            if (RAW) {
                // e2m1 * s exactly as binary16 (every product of an E2M1 value and an
                // E4M3 scale is exact there); a32 is applied to the products instead
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const __half2 v = __hmul2(e2m1x2_to_half2((cw[j] >> (8 * e)) & 0xFFu), s2);
                    o[e] = *reinterpret_cast<const uint32_t*>(&v);
                }
                st_shared16(base + chunk * 2048 + row * 16, make_uint4(o[0], o[1], o[2], o[3]));
            } else {
                const uint32_t sc = (((blk < 4 ? r.sc.x : r.sc.y) >> (8 * (blk % 4))) & 0xFFu);
                st_shared16(base + chunk * 2048 + row * 16, dq8(cw[j], sc, r.a32, m ? m + 8 * chunk : nullptr));
            }
        }
    }
}

// Barriers and flags of one CTA (static shared memory).
struct AttnShared {
    uint64_t q_full[2];  // softmax X -> MMA: Q_X of the unit written (128 arrivals)
    uint64_t s_full[2];  // MMA -> softmax X: S_X = Q_X K^T done (commit), so is every earlier product
    uint64_t p_full[2];  // softmax X -> MMA: P_X written, S_X read, O_X rescaled (128 arrivals)
    uint64_t o_full[2];  // MMA -> softmax X: the unit's last P V product into O_X done (commit)
    uint64_t k_full;     // producers -> MMA: K tile written (128 arrivals)
    uint64_t k_empty;    // MMA -> producers: both Q K^T products of the K tile done (commit)
    uint64_t v_full[2];  // producers -> MMA: V buffer b written (128 arrivals)
    uint64_t v_empty[2]; // MMA -> producers: both P V products of V buffer b done (commit)
    uint64_t done;       // MMA thread: every product it issued is done (before TMEM is freed)
    uint32_t tmem_base;
    int abort;           // set by the first role whose wait gives up; the others stop at their next wait
};

// The key tiles of the listed slots: tile g is tile g % tps of list entry
// g / tps; entries with an out-of-range slot are skipped.
struct KeyTiles {
    const int32_t* slots;
    int n_slots, tps, G;
    __device__ __forceinline__ int slot(int g) const { return __ldg(slots + g / tps); }
    __device__ __forceinline__ int next(int g) const {
        while (g < G) {
            const int s = slot(g);
            if (s >= 0 && s < n_slots) break;
            g += tps - g % tps;
        }
        return g;
    }
};

// Bounded wait; on giving up it records the timeout (the first error wins) and
// raises the CTA's abort flag.
__device__ __forceinline__ bool wait_or_stop(uint64_t* bar, uint32_t parity, AttnShared& sh, const AttnArgs& a,
                                             uint32_t where) {
    volatile int* abort = &sh.abort;
    if (mbar_wait_bounded(bar, parity, abort, a.limit_ns)) return true;
    record_error(a.err, NVFP4_ERR_TIMEOUT, where);
    *abort = 1;
    return false;
}

// Query row `qrow` of head h into Q at row `row` (zeros past the last query).
// RAW: the row is scaled by a power of two 2^k (exact) so that its largest
// magnitude lies in [2^14, 2^15), then rounded to binary16; returns 2^-k.
template <bool RAW>
__device__ __forceinline__ float load_q_row(const AttnArgs& a, uint32_t q_s, int qrow, int h, int row) {
    uint4 v[16];
    if (qrow < a.tq) {
        const uint4* src = reinterpret_cast<const uint4*>(a.q + ((int64_t)qrow * a.heads + h) * kD * 2);
#pragma unroll
        for (int c = 0; c < 16; c++) v[c] = __ldg(src + c);
    } else {
#pragma unroll
        for (int c = 0; c < 16; c++) v[c] = make_uint4(0u, 0u, 0u, 0u);
    }
    float q_inv = 1.0f;
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
    for (int c = 0; c < 16; c++) st_shared16(q_s + c * 2048 + row * 16, v[c]);
    return q_inv;
}

// The largest score of the thread's S row over the tile's first `valid` keys
// (four independent chains).
__device__ __forceinline__ float tile_max(uint32_t t_s, int valid) {
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int c2 = 0; c2 < 2; c2++) {
        uint32_t r[2][32];
        tmem_ld_32cols(t_s + 64 * c2, r[0]);
        tmem_ld_32cols(t_s + 64 * c2 + 32, r[1]);
        tmem_ld_wait();
        tmem_regs_ready(r[0]);
        tmem_regs_ready(r[1]);
#pragma unroll
        for (int c = 0; c < 2; c++)
#pragma unroll
            for (int j = 0; j < 32; j++)
                if (valid == kTile || 64 * c2 + 32 * c + j < valid) mx[j & 3] = fmaxf(mx[j & 3], __uint_as_float(r[c][j]));
    }
    return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
}

// P row: 2^(c_s * s - m) for the tile's first `valid` keys (zero past them),
// times w_s (RAW: a32_V / a32_ref) rounded to binary16, else bf16, written to
// P at row `row`; returns the row's sum of the unrounded, unweighted values.
// 32 columns a TMEM load (the chunk loop is kept rolled: fewer live registers).
template <bool RAW>
__device__ __forceinline__ float write_p(uint32_t t_s, uint32_t p_s, int row, int valid, float c_s, float m,
                                         float w_s) {
    float2 sum[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
    const float2 cc = make_float2(c_s, c_s), mm = make_float2(-m, -m), ww = make_float2(w_s, w_s);
#pragma unroll 1
    for (int c = 0; c < 4; c++) {
        uint32_t rc[32];
        tmem_ld_32cols(t_s + 32 * c, rc);
        tmem_ld_wait();
        tmem_regs_ready(rc);
#pragma unroll
        for (int q4 = 0; q4 < 4; q4++) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int j = 8 * q4 + 2 * e;
                const float2 t = fma2(make_float2(__uint_as_float(rc[j]), __uint_as_float(rc[j + 1])), cc, mm);
                float2 p = make_float2(ex2(t.x), ex2(t.y));
                if (valid < kTile) {
                    if (32 * c + j >= valid) p.x = 0.0f;
                    if (32 * c + j + 1 >= valid) p.y = 0.0f;
                }
                sum[e & 1] = add2(sum[e & 1], p);
                if (RAW) {
                    const float2 pw = mul2(p, ww);
                    const __half2 hv = __floats2half2_rn(pw.x, pw.y);
                    w[e] = *reinterpret_cast<const uint32_t*>(&hv);
                } else {
                    const __nv_bfloat162 b = __floats2bfloat162_rn(p.x, p.y);
                    w[e] = *reinterpret_cast<const uint32_t*>(&b);
                }
            }
            st_shared16(p_s + (4 * c + q4) * 2048 + row * 16, make_uint4(w[0], w[1], w[2], w[3]));
        }
    }
    return (sum[0].x + sum[1].x) + (sum[0].y + sum[1].y);
}

// Softmax group X (warps 4X .. 4X + 3; `row` = query row in the tile = TMEM lane).
// RAW: binary16 operands; the row's 2^-k and the slot's a32_K multiply the
// scores inside the exponent, P carries a32_V / a32_ref (a32_ref: the largest
// V scale of the listed slots) and O is multiplied by a32_ref at the end.
template <bool RAW>
__device__ __forceinline__ void softmax_role(const AttnArgs& a, AttnShared& sh, const KeyTiles& kt, uint32_t smem0,
                                             uint32_t tmem, int X, int row) {
    const uint32_t lane_off = (uint32_t)(row & ~31) << 16;
    const uint32_t t_s = tmem + kSCol + 128 * X + lane_off, t_o = tmem + kOCol + 128 * X + lane_off;
    const uint32_t q_s = smem0 + kSmemQ + X * kOperandBytes, p_s = smem0 + kSmemP + X * kOperandBytes;
    float a_ref = 1.0f;
    if (RAW) {
        a_ref = 0.0f;
        for (int si = 0; si < a.n; si++) {
            const int s = __ldg(kt.slots + si);
            if (s >= 0 && s < kt.n_slots) a_ref = fmaxf(a_ref, __ldg(a.gscale[1] + s));
        }
    }
    uint32_t ph_s = 0u, ph_o = 0u;
    for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
        const int h = u / a.n_qp, qt = 2 * (u % a.n_qp) + X;
        if (qt >= a.n_qt) continue;  // tile B of the last pair may be empty
        const int qrow = qt * kTile + row;
        const float q_inv = load_q_row<RAW>(a, q_s, qrow, h, row);
        fence_proxy_async_smem();
        mbar_arrive(&sh.q_full[X]);
        float m_run = -INFINITY, l_run = 0.0f;
        bool first = true;
        int cur_s = -1;
        float c_s = 0.0f, w_s = 0.0f;
        for (int g = kt.next(0); g < kt.G; g = kt.next(g + 1)) {
            // the tile's scalars load before the wait: exponent units t = c_s * S
            // (exp(scale * q.k) = 2^t; RAW: c_s also carries the row's 2^-k and the
            // slot's a32_K), w_s = a32_V / a32_ref (RAW)
            const int s = kt.slot(g);
            const int valid = min(kTile, a.tokens - (g % kt.tps) * kTile);
            if (s != cur_s) {
                cur_s = s;
                c_s = RAW ? q_inv * __ldg(a.gscale[0] + s) * a.scale_log2 : a.scale_log2;
                w_s = RAW ? (a_ref > 0.0f ? __fdiv_rn(__ldg(a.gscale[1] + s), a_ref) : 0.0f) : 1.0f;
            }
            // (a wait's outcome is made uniform over the warp: the TMEM loads are warp-collective)
            const bool got = __all_sync(0xFFFFFFFFu, wait_or_stop(&sh.s_full[X], ph_s, sh, a, 1));
            ph_s ^= 1u;
            if (!got) return;
            tc_fence_after();
            // P against the current reference max m; every weight is at most 2^15
            // (binary16 holds it) when their sum is.  A row whose sum is larger, or not
            // finite (the first tile: m = -inf), takes the tile's largest score: the
            // reference moves to it when it exceeds m by more than 8 (2^8 in the
            // weights), O (in TMEM; its last product is done, s_full says so) and the
            // running sum are rescaled, and P is formed again.
            float tsum = write_p<RAW>(t_s, p_s, row, valid, c_s, m_run, w_s);
            const bool redo = !(tsum <= kPMax);
            if (__any_sync(0xFFFFFFFFu, redo)) {
                // tcgen05.ld / st are warp-collective: the whole warp takes part
                const float mt = tile_max(t_s, valid) * c_s;  // c_s >= 0
                float factor = 1.0f;
                if (redo && mt - m_run > kLazyLog2) {
                    factor = ex2(m_run - mt);  // 0 on the first tile (m_run = -inf)
                    l_run *= factor;
                    m_run = mt;
                }
                // rows that keep their reference multiply by exactly 1
                if (!first && __any_sync(0xFFFFFFFFu, factor != 1.0f)) {
                    if ((row & 31) == 0) atomicAdd(a.rescales, 1u);
                    uint32_t o[32];
#pragma unroll 1
                    for (int c = 0; c < 4; c++) {
                        tmem_ld_32cols(t_o + 32 * c, o);
                        tmem_ld_wait();
                        tmem_regs_ready(o);
#pragma unroll
                        for (int j = 0; j < 32; j++) o[j] = __float_as_uint(__uint_as_float(o[j]) * factor);
                        tmem_st_32cols(t_o + 32 * c, o);
                    }
                    tmem_st_wait();
                }
                tsum = write_p<RAW>(t_s, p_s, row, valid, c_s, m_run, w_s);
            }
            l_run += tsum;
            // S read, O rescaled and P written before the MMA thread goes on
            tc_fence_before();
            fence_proxy_async_smem();
            mbar_arrive(&sh.p_full[X]);
            first = false;
        }
        // O row / l -> bf16
        if (!first) {
            const bool got = __all_sync(0xFFFFFFFFu, wait_or_stop(&sh.o_full[X], ph_o, sh, a, 2));
            ph_o ^= 1u;
            if (!got) return;
            tc_fence_after();
        }
        const float inv_l = l_run > 0.0f ? __fdiv_rn(a_ref, l_run) : 0.0f;  // a_ref = 1 unless RAW
        uint4* dst = reinterpret_cast<uint4*>(a.o + ((int64_t)qrow * a.heads + h) * kD * 2);
#pragma unroll
        for (int c = 0; c < 4; c++) {
            uint32_t r[32];
            if (!first) {
                tmem_ld_32cols(t_o + 32 * c, r);
                tmem_ld_wait();
                tmem_regs_ready(r);
            } else {
#pragma unroll
                for (int j = 0; j < 32; j++) r[j] = 0u;
            }
            if (qrow < a.tq) {
#pragma unroll
                for (int g4 = 0; g4 < 4; g4++) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(r[8 * g4 + 2 * e]) * inv_l,
                                                                       __uint_as_float(r[8 * g4 + 2 * e + 1]) * inv_l);
                        w[e] = *reinterpret_cast<const uint32_t*>(&b);
                    }
                    dst[4 * c + g4] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
        // O read before the next unit's first P V product overwrites it
        tc_fence_before();
    }
}

// Producers (warps 8-11; `row` = key row of the tile): K into its one buffer,
// V into two alternating buffers; the next tile's rows load while the current
// ones wait for their buffers.
template <bool RAW>
__device__ __forceinline__ void producer_role(const AttnArgs& a, AttnShared& sh, const KeyTiles& kt, uint32_t smem0,
                                              int row) {
    uint32_t ph_k = 0u, nv = 0u;
    for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
        const int h = u / a.n_qp;
        int g = kt.next(0);
        RowRaw kr, vr;
        if (g < kt.G) {
            const int s = kt.slot(g), tok = (g % kt.tps) * kTile + row;
            kr = fetch_row(a, 0, s, tok, h);
            vr = fetch_row(a, 1, s, tok, h);
        }
        while (g < kt.G) {
            const int s = kt.slot(g);
            const int gn = kt.next(g + 1);
            // a buffer's first fill passes at once (parity 1 of a fresh barrier)
            if (!wait_or_stop(&sh.k_empty, ph_k ^ 1u, sh, a, 4)) return;
            ph_k ^= 1u;
            store_row<RAW>(a, 0, s, h, kr, smem0 + kSmemK, row);
            fence_proxy_async_smem();
            mbar_arrive(&sh.k_full);
            const uint32_t vb = nv & 1u;
            if (!wait_or_stop(&sh.v_empty[vb], ((nv >> 1) & 1u) ^ 1u, sh, a, 5)) return;
            store_row<RAW>(a, 1, s, h, vr, smem0 + kSmemV + vb * kOperandBytes, row);
            fence_proxy_async_smem();
            mbar_arrive(&sh.v_full[vb]);
            nv++;
            if (gn < kt.G) {
                const int sn = kt.slot(gn), tok = (gn % kt.tps) * kTile + row;
                kr = fetch_row(a, 0, sn, tok, h);
                vr = fetch_row(a, 1, sn, tok, h);
            }
            g = gn;
        }
    }
}

// The MMA thread (lane 0 of warp 12).  Per unit: QK_A(0), QK_B(0), then per
// key tile j: PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1).  The hazards:
//  - QK_X(j+1) overwrites S_X: issued only after p_full[X] of tile j (its
//    softmax has read S_X);
//  - K is single-buffered: k_empty is committed after the tile's last Q K^T;
//  - softmax X(j) writes P_X and may rescale O_X once s_full[X](j) has fired,
//    which covers PV_X(j-1) (a commit tracks every earlier product of this
//    thread, and PV_X(j-1) is issued before QK_X(j));
//  - V buffer b is released (v_empty) after the tile's last P V product.
template <bool RAW>
__device__ __forceinline__ void mma_role(const AttnArgs& a, AttnShared& sh, const KeyTiles& kt, uint32_t smem0,
                                         uint32_t tmem) {
    constexpr uint32_t ID_QK = idesc_f16(0, RAW ? 0 : 1), ID_PV = idesc_f16(1, RAW ? 0 : 1);
    auto qk = [&](int X) {
        const uint32_t q_s = smem0 + kSmemQ + X * kOperandBytes, k_s = smem0 + kSmemK;
#pragma unroll
        for (int k = 0; k < kD / 16; k++)
            mma_f16(tmem + kSCol + 128 * X, smem_desc(q_s + k * 4096, 2048, 128, kLayoutNone),
                    smem_desc(k_s + k * 4096, 2048, 128, kLayoutNone), ID_QK, k > 0);
        tc_commit(&sh.s_full[X]);
    };
    auto pv = [&](int X, uint32_t vb, bool acc) {
        const uint32_t p_s = smem0 + kSmemP + X * kOperandBytes, v_s = smem0 + kSmemV + vb * kOperandBytes;
#pragma unroll
        for (int k = 0; k < kTile / 16; k++)
            mma_f16(tmem + kOCol + 128 * X, smem_desc(p_s + k * 4096, 2048, 128, kLayoutNone),
                    smem_desc(v_s + k * 256, 128, 2048, kLayoutNone), ID_PV, (acc || k > 0) ? 1u : 0u);
    };
    uint32_t ph_q[2] = {0u, 0u}, ph_p[2] = {0u, 0u}, ph_k = 0u, nv = 0u;
    bool ok = true;
    for (int u = blockIdx.x; u < a.n_units && ok; u += gridDim.x) {
        const bool hasB = 2 * (u % a.n_qp) + 1 < a.n_qt;
        if (!wait_or_stop(&sh.q_full[0], ph_q[0], sh, a, 6)) break;
        ph_q[0] ^= 1u;
        if (hasB) {
            if (!wait_or_stop(&sh.q_full[1], ph_q[1], sh, a, 6)) break;
            ph_q[1] ^= 1u;
        }
        int g = kt.next(0);
        if (g >= kt.G) continue;
        if (!wait_or_stop(&sh.k_full, ph_k, sh, a, 7)) break;
        ph_k ^= 1u;
        tc_fence_after();
        qk(0);
        if (hasB) qk(1);
        tc_commit(&sh.k_empty);
        bool first = true;
        while (g < kt.G) {
            const int gn = kt.next(g + 1);
            const uint32_t vb = nv & 1u;
            if (!wait_or_stop(&sh.v_full[vb], (nv >> 1) & 1u, sh, a, 8) ||
                !wait_or_stop(&sh.p_full[0], ph_p[0], sh, a, 9)) {
                ok = false;
                break;
            }
            ph_p[0] ^= 1u;
            tc_fence_after();
            pv(0, vb, !first);
            if (gn < kt.G) {
                if (!wait_or_stop(&sh.k_full, ph_k, sh, a, 7)) {
                    ok = false;
                    break;
                }
                ph_k ^= 1u;
                tc_fence_after();
                qk(0);
            } else {
                tc_commit(&sh.o_full[0]);
            }
            if (hasB) {
                if (!wait_or_stop(&sh.p_full[1], ph_p[1], sh, a, 9)) {
                    ok = false;
                    break;
                }
                ph_p[1] ^= 1u;
                tc_fence_after();
                pv(1, vb, !first);
            }
            tc_commit(&sh.v_empty[vb]);
            nv++;
            if (gn < kt.G) {
                if (hasB) qk(1);
                tc_commit(&sh.k_empty);
            } else if (hasB) {
                tc_commit(&sh.o_full[1]);
            }
            first = false;
            g = gn;
        }
    }
    // every product issued is done before the TMEM is released (also after a stop)
    tc_commit(&sh.done);
    volatile int never = 0;
    if (!mbar_wait_bounded(&sh.done, 0, &never, a.limit_ns)) record_error(a.err, NVFP4_ERR_TIMEOUT, 10);
}

template <bool RAW>
__global__ void __launch_bounds__(kThreads, 1) kv_attention_kernel(const __grid_constant__ AttnArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ AttnShared sh;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        for (int X = 0; X < 2; X++) {
            mbar_init(&sh.q_full[X], kGroup);
            mbar_init(&sh.s_full[X], 1);
            mbar_init(&sh.p_full[X], kGroup);
            mbar_init(&sh.o_full[X], 1);
            mbar_init(&sh.v_full[X], kGroup);
            mbar_init(&sh.v_empty[X], 1);
        }
        mbar_init(&sh.k_full, kGroup);
        mbar_init(&sh.k_empty, 1);
        mbar_init(&sh.done, 1);
        sh.abort = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&sh.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base, smem0 = smem_u32(smem);
    KeyTiles kt;
    kt.slots = a.slots;
    kt.n_slots = a.n_slots;
    kt.tps = (a.tokens + kTile - 1) / kTile;
    kt.G = a.n * kt.tps;
    if (blockIdx.x == 0 && threadIdx.x == 0)
        for (int si = 0; si < a.n; si++) {
            const int s = __ldg(a.slots + si);
            if (s < 0 || s >= a.n_slots) record_error(a.err, NVFP4_ERR_DEVICE, (uint32_t)si);
        }
    if (warp < kProducerWarp0)
        softmax_role<RAW>(a, sh, kt, smem0, tmem, warp >> 2, threadIdx.x & (kGroup - 1));
    else if (warp < kMmaWarp)
        producer_role<RAW>(a, sh, kt, smem0, threadIdx.x - kProducerWarp0 * 32);
    else if ((threadIdx.x & 31) == 0)
        mma_role<RAW>(a, sh, kt, smem0, tmem);
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
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
    // and its work units (pairs of 128-query tiles x heads) in 32 bits
    if (((int64_t)tq + 2 * kTile - 1) / (2 * kTile) * cache->heads >= ((int64_t)1 << 31)) return NVFP4_ERR_UNSUPPORTED;
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
    a.n_qt = (int)((tq + kTile - 1) / kTile);
    a.n_qp = (a.n_qt + 1) / 2;
    a.n_units = a.n_qp * cache->heads;
    const int smem = kSmemBytes;
    // caches without smoothing means take the binary16 path
    const bool raw = !sk && !sv;
    void (*kern)(AttnArgs) = raw ? kv_attention_kernel<true> : kv_attention_kernel<false>;
    // the SM count and the shared-memory attribute of both variants, once per device
    static PerDevice<int> dev_sms;
    int sms = 0;
    const nvfp4_status ast = dev_sms.get(&sms, [smem](int dev, int& v) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v < 1 ||
            cudaFuncSetAttribute(kv_attention_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess ||
            cudaFuncSetAttribute(kv_attention_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess)
            return NVFP4_ERR_CUDA;
        return NVFP4_OK;
    });
    if (ast != NVFP4_OK) return ast;
    // persistent: one CTA per SM at most, each walking units blockIdx.x, + gridDim.x, ...
    const int grid = std::min(a.n_units, sms);
    kern<<<grid, kThreads, smem, (cudaStream_t)stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
