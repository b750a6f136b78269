// gemm.cu -- W4A4 NVFP4 GEMM for sm_100a with a fused epilogue.
//
//   C[M x N] = a32_A * a32_B * (A_q . S_A)(B_q . S_B)^T  -> epilogue -> bf16
//              and/or NVFP4 re-quantization for the next layer.
//
// Method: the W4A4 linear layers of "LongLive-2.0：用 NVFP4 并行底座做长视频生成"
// (yingwang.github.io reading note), sections "NVFP4 训练的工程细节" (weights and
// activations in NVFP4, 1D block scaling along K, self-written CUDA kernels)
// and "推理底座" (4-bit weights and activations at inference); the Dequant
// equation of section "NVFP4 量化格式" is what the block-scaled MMA applies
// per 16-element block.  The adaLN modulate/gate epilogue stands in for the
// fused adaLN kernels of the anzhuoshouzhuan.com article ("NVFP4 量化").
//
// Kernel design (B200):
//  * persistent grid, one CTA per SM, static tile schedule with the N blocks
//    of an M block consecutive.  Two variants of one template: a CTA pair
//    (cluster of 2, tcgen05 cta_group::2) computing 256 x 256 tiles -- each
//    CTA loads its 128 rows of A, its 128 rows of B and all 256 rows of B's
//    scales, the leader CTA issues the MMAs for both -- and a single-CTA
//    128 x 256 variant used when M <= 128;
//  * warp 0: TMA producer (A/B code tiles with 128B swizzle, the 512-byte
//    scale-factor tiles as 3-D boxes whose K tail the TMA zero-fills); a ring
//    of K-slices of 256 elements (5 x 38 KB per CTA for the pair, 3 x 54 KB
//    for one CTA);
//  * warp 1: owns TMEM (512 columns: two overlapping 256-column accumulators
//    and two or three 48-column scale buffers) and issues, from one thread,
//    tcgen05.mma.kind::mxf4nvf4.block_scale (M=128 or 256 for the pair,
//    N=256, K=64), releasing each stage with tcgen05.commit;
//  * warps 10..: tcgen05.cp of the stage's scale tiles into a free TMEM scale
//    buffer, a stage ahead of the MMAs;
//  * warps 2..9: epilogue, two warps per TMEM lane quarter, each taking every
//    other 32-column chunk: tcgen05.ld, binary32 math, bf16 through TMA stores
//    and/or the NVFP4 requant with the same encoder as the quantize kernel;
//    the columns both accumulators share are drained first, so the next
//    tile's MMAs run while the rest of the epilogue proceeds;
//  * every mbarrier wait is bounded (globaltimer); on expiry the kernel
//    records NVFP4_ERR_TIMEOUT in the workspace, raises a CTA-wide abort flag,
//    drains what it issued and frees TMEM before returning.
#include <algorithm>
#include <cstring>

#include "common.cuh"

namespace nvfp4 {
namespace gemm {

constexpr int BM = 128;  // rows of A per CTA
constexpr int BN = 256;  // output columns per tile
constexpr int BK = 256;  // K elements per stage
constexpr int BKB = BK / 2;  // bytes per row per stage (128: one swizzle atom row)
constexpr int KB_PER_STAGE = BK / 64;
// Block: producer, MMA, 8 epilogue warps (two per TMEM lane quarter, each
// taking every other 32-column chunk, so every scheduler has two epilogue
// warps to switch between) and NC scale-copy warps.  Two variants: NC = 3
// (416 threads, at most 152 registers a thread) for long K, where the
// mainloop dominates, and NC = 2 (384 threads, 168 registers) for short K,
// where the epilogue takes its shared accumulator columns into registers at
// once so the next tile starts sooner.
constexpr int EPI_WARPS = 8;
constexpr int EPI_THREADS = EPI_WARPS * 32;
constexpr int FIRST_COPY_WARP = 2 + EPI_WARPS;
constexpr int threads_for(int nc) { return (FIRST_COPY_WARP + nc) * 32; }
constexpr uint32_t TMEM_COLS = 512;
constexpr int A_BYTES = BM * BKB;                  // 16 KB
constexpr int SFA_BYTES = KB_PER_STAGE * 512;      // 2 KB
constexpr int SFB_BYTES = 2 * KB_PER_STAGE * 512;  // 4 KB (two 128-row halves of the tile's N)

// Per-tile shared memory of the epilogue: the tile's per-column vectors
// (bias, modulate scale, modulate shift, gate; bf16 pairs, two buffers by
// tile parity) and each warp's 32 x 32 bf16 staging buffer for the TMA store
// of C (64-byte rows, 64B swizzle: 16-byte unit u of row r at
// (u ^ (r / 2 % 4)) * 16).
constexpr int EPI_BUF_BYTES = 32 * 64;
constexpr int EPI_STAGE_BYTES = EPI_WARPS * EPI_BUF_BYTES;  // 16 KB
constexpr int VEC_BYTES = 2 * 4 * BN * 4;  // two tile parities x 4 binary32 vectors x BN: 8 KB
constexpr int INV_TAB_BYTES = 256 * 4;    // requant reciprocal per E4M3 code

// Two accumulators of BN columns share TMEM with NSF 48-column scale buffers
// that the stages take in turn (the copy warps fill one while the MMAs read
// another).  The accumulators overlap; the epilogue drains the shared columns
// first and then lets the next tile's MMAs start, so the rest of the
// epilogue overlaps the next mainloop.  Short K (NC = 2): two scale buffers,
// acc0 = [0, 256), acc1 = [160, 416), scales = [416, 512), 3 shared chunks
// (acc0: its chunks 5..7, acc1: 0..2).  Long K (NC = 3): three scale buffers,
// so the copy warps can run two stages ahead of the MMAs and the tensor pipe
// never waits for a copy to be seen; acc1 = [96, 352), scales = [352, 496),
// 5 shared chunks -- a longer hand-over between tiles, which long K
// amortises.
constexpr uint32_t SF_COLS = 4 * KB_PER_STAGE + 8 * KB_PER_STAGE;  // 48 per buffer
constexpr int MAX_NSF = 3;
template <int NC>
struct Tm {
    static constexpr int NSF = NC == 3 ? 3 : 2;
    static constexpr uint32_t ACC1_COL = NC == 3 ? 96 : 160;
    static constexpr uint32_t SFA_COL = ACC1_COL + BN;               // scale buffer 0
    static constexpr uint32_t SFB_COL = SFA_COL + 4 * KB_PER_STAGE;
    static constexpr int OVERLAP_CHUNKS = (BN - (int)ACC1_COL) / 32;
    static_assert(SFA_COL + NSF * SF_COLS <= TMEM_COLS, "TMEM budget");
    static_assert(NSF <= MAX_NSF, "scale-buffer barriers");
    static_assert(ACC1_COL % 32 == 0 && (BN - (int)ACC1_COL) % 32 == 0, "overlap must be whole 32-column chunks");
};

// instruction descriptor: E2M1 x E2M1, UE4M3 scales, f32 accumulate, K-major
// A and B, M x N, K = 64 (dense).
constexpr uint32_t make_idesc(int m, int n) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

template <bool PAIR>
struct Cfg {
    static constexpr int CTAS = PAIR ? 2 : 1;
    static constexpr int TILE_M = BM * CTAS;        // 256 or 128
    static constexpr int B_ROWS = PAIR ? 128 : 256;  // rows of B each CTA loads
    static constexpr int STAGES = PAIR ? 5 : 3;
    static constexpr int B_BYTES = B_ROWS * BKB;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_STAGE_BYTES + VEC_BYTES + INV_TAB_BYTES + 1024 + 256;
    static constexpr uint32_t TX_BYTES = (uint32_t)(CTAS * STAGE_BYTES);  // per stage, both CTAs
    static constexpr uint32_t IDESC = make_idesc(TILE_M, BN);
    static_assert(STAGE_BYTES % 1024 == 0, "stage must keep 1024-byte alignment for 128B swizzle");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

struct Params {
    int M, N, K;
    int tiles_m, tiles_n, num_tiles;  // tiles_m counts TILE_M-row blocks
    int kt_count;                     // ceil(K / BK)
    int kb_total;                     // K / 64
    const float* ga;
    const float* gb;
    __nv_bfloat16* c;
    int64_t ldc;
    const __nv_bfloat16* bias;
    const __nv_bfloat16* mod_scale;
    const __nv_bfloat16* mod_shift;
    const __nv_bfloat16* gate;
    const __nv_bfloat16* residual;
    int64_t ld_res;
    int act;
    uint8_t* out_codes;
    uint8_t* out_scales;
    const float* out_gscale;
    int q_col0, q_col1;  // requant / out_amax window [q_col0, q_col1): multiples of 64 (requant)
    float* out_amax;
    float* debug_y;
    DevError* err;
    uint64_t limit_ns;
    uint32_t dbg;
};

template <int STAGES>
struct Smem {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tmem_full;
    uint64_t tmem_empty;
    uint64_t drain;
    uint64_t sf_full[MAX_NSF];   // scale buffer filled (one commit per copy warp)
    uint64_t sf_empty[MAX_NSF];  // scale buffer no longer read by the MMAs
    uint32_t tmem_base;
    int abort_flag;
};

// Tile order: the N blocks of one M block are consecutive, so the tiles
// running at once share a few A row blocks (each fetched from HBM once and
// then read from L2 by every N block) while the whole weight B stays in L2
// across waves when it fits (a DiT linear's weight is at most ~25 MB).
__device__ __forceinline__ void tile_coords(const Params& p, int tile, int& mb, int& nb) {
    nb = tile % p.tiles_n;
    mb = tile / p.tiles_n;
}

template <class S>
__device__ __forceinline__ void raise_abort(S* s, const Params& p, uint32_t where) {
    record_error(p.err, NVFP4_ERR_TIMEOUT, where);
    *(volatile int*)&s->abort_flag = 1;
}

// work unit of this CTA (pair: one per cluster) and the stride between them
template <bool PAIR>
__device__ __forceinline__ void tile_range(int& first, int& step) {
    if (PAIR) {
        first = blockIdx.x >> 1;
        step = gridDim.x >> 1;
    } else {
        first = blockIdx.x;
        step = gridDim.x;
    }
}

// ---------------------------------------------------------------- producer --
template <bool PAIR>
__device__ void producer(const Params& p, Smem<Cfg<PAIR>::STAGES>* s, uint8_t* ring, const CUtensorMap* tma_a,
                         const CUtensorMap* tma_b, const CUtensorMap* tma_sfa, const CUtensorMap* tma_sfb,
                         uint32_t rank) {
    using C = Cfg<PAIR>;
    prefetch_tmap(tma_a);
    prefetch_tmap(tma_b);
    prefetch_tmap(tma_sfa);
    prefetch_tmap(tma_sfb);
    volatile int* abort = &s->abort_flag;
    uint32_t issued_mask = 0, parity_mask = 0;  // per stage: a load was issued / its phase parity
    if (p.dbg & NVFP4_DBG_SKIP_LOADS) return;
    int first, step;
    tile_range<PAIR>(first, step);
    uint32_t it = 0;
    for (int tile = first; tile < p.num_tiles; tile += step) {
        int mb, nb;
        tile_coords(p, tile, mb, nb);
        const int a_row = mb * C::TILE_M + (int)rank * BM;
        const int b_row = nb * BN + (int)rank * C::B_ROWS;
        const int sfa_blk = mb * C::CTAS + (int)rank;
        for (int kt = 0; kt < p.kt_count; kt++, it++) {
            const int st = it % C::STAGES;
            const uint32_t round = it / C::STAGES;
            if (!mbar_wait_bounded(&s->empty[st], (round & 1) ^ 1, abort, p.limit_ns)) {
                if (!*abort) raise_abort(s, p, 1);
                goto drain;
            }
            {
                uint8_t* a_s = ring + st * C::STAGE_BYTES;
                uint8_t* b_s = a_s + A_BYTES;
                uint8_t* sfa_s = b_s + C::B_BYTES;
                uint8_t* sfb_s = sfa_s + SFA_BYTES;
                const int kx = kt * BKB, ks = kt * KB_PER_STAGE;
                if (PAIR) {
                    // all transaction bytes of the pair are counted on the leader's barrier
                    const uint32_t bar = mapa_shared(smem_u32(&s->full[st]), 0);
                    if (rank == 0) mbar_expect_tx(&s->full[st], C::TX_BYTES);
                    tma_load_2d_pair(a_s, tma_a, bar, kx, a_row);
                    tma_load_2d_pair(b_s, tma_b, bar, kx, b_row);
                    tma_load_3d_pair(sfa_s, tma_sfa, bar, 0, ks, sfa_blk);
                    tma_load_3d_pair(sfb_s, tma_sfb, bar, 0, ks, nb * 2);
                    tma_load_3d_pair(sfb_s + SFA_BYTES, tma_sfb, bar, 0, ks, nb * 2 + 1);
                } else {
                    mbar_expect_tx(&s->full[st], C::TX_BYTES);
                    tma_load_2d(a_s, tma_a, &s->full[st], kx, a_row);
                    tma_load_2d(b_s, tma_b, &s->full[st], kx, b_row);
                    tma_load_3d(sfa_s, tma_sfa, &s->full[st], 0, ks, sfa_blk);
                    tma_load_3d(sfb_s, tma_sfb, &s->full[st], 0, ks, nb * 2);
                    tma_load_3d(sfb_s + SFA_BYTES, tma_sfb, &s->full[st], 0, ks, nb * 2 + 1);
                }
                issued_mask |= 1u << st;
                parity_mask = (parity_mask & ~(1u << st)) | ((round & 1u) << st);
            }
        }
    }
    return;
drain:
    // the only loads that can still be in flight are the last one per stage
    // (for the pair they are all counted on the leader's barriers)
    if (!PAIR || rank == 0) {
        for (int i = 0; i < C::STAGES; i++)
            if (issued_mask & (1u << i)) {
                volatile int never = 0;
                mbar_wait_bounded(&s->full[i], (parity_mask >> i) & 1u, &never, p.limit_ns);
            }
    }
}

// ---------------------------------------------------------------- MMA -------
// One thread (of the leader CTA for the pair) issues the MMAs; the scale-factor
// copies into TMEM are issued by the copy warps below.  tcgen05.cp costs about
// 50 cycles per instruction and a stage needs 12 of them against 512 cycles of
// MMA work, so they run on other threads, a stage ahead, into the other scale
// buffer.  Descriptors are built once; a stage / k-block step only adds to the
// 14-bit start-address field (shared memory addresses are < 2^18, so the field
// never carries).
template <bool PAIR, int NC>
__device__ void mma_issuer(const Params& p, Smem<Cfg<PAIR>::STAGES>* s, uint8_t* ring, uint32_t tmem) {
    using C = Cfg<PAIR>;
    using T = Tm<NC>;
    volatile int* abort = &s->abort_flag;
    const uint32_t ring_s = smem_u32(ring);
    const uint64_t a_desc0 = smem_desc(ring_s, 16, 1024, kLayoutSw128);
    const uint64_t b_desc0 = smem_desc(ring_s + A_BYTES, 16, 1024, kLayoutSw128);
    const uint32_t sfa_t = tmem + T::SFA_COL, sfb_t = tmem + T::SFB_COL;
    int first, step;
    tile_range<PAIR>(first, step);
    uint32_t it = 0;
    uint32_t tcount = 0;
    bool issued = false;
    for (int tile = first; tile < p.num_tiles; tile += step, tcount++) {
        if (!mbar_wait_bounded(&s->tmem_empty, (tcount & 1) ^ 1, abort, p.limit_ns)) {
            if (!*abort) raise_abort(s, p, 2);
            goto drain;
        }
        tc_fence_after();
        const uint32_t acc = tmem + ((tcount & 1) ? T::ACC1_COL : 0u);
        for (int kt = 0; kt < p.kt_count; kt++, it++) {
            const int st = it % C::STAGES;
            const uint32_t sb = it % T::NSF;
            // the stage's scales are in TMEM (the copy warps saw its data arrive)
            if (!mbar_wait_bounded(&s->sf_full[sb], (it / T::NSF) & 1, abort, p.limit_ns)) {
                if (!*abort) raise_abort(s, p, 3);
                goto drain;
            }
            tc_fence_after();
            const uint64_t off = (uint64_t)((st * C::STAGE_BYTES) >> 4);
            const int nkb = min(KB_PER_STAGE, p.kb_total - kt * KB_PER_STAGE);
            const uint32_t sfo = sb * SF_COLS;
#pragma unroll
            for (int kb = 0; kb < KB_PER_STAGE; kb++) {
                if (kb < nkb) {
                    const uint64_t ad = a_desc0 + off + kb * (32 >> 4);
                    const uint64_t bd = b_desc0 + off + kb * (32 >> 4);
                    const uint32_t acc_flag = (kt > 0 || kb > 0) ? 1u : 0u;
                    if (PAIR)
                        tc_mma_nvf4_pair(acc, ad, bd, C::IDESC, sfa_t + sfo + 4 * kb, sfb_t + sfo + 8 * kb, acc_flag);
                    else
                        tc_mma_nvf4(acc, ad, bd, C::IDESC, sfa_t + sfo + 4 * kb, sfb_t + sfo + 8 * kb, acc_flag);
                }
            }
            issued = true;
            if (PAIR) {
                tc_commit_pair(&s->empty[st], 0x3);
                tc_commit_pair(&s->sf_empty[sb], 0x1);
            } else {
                tc_commit(&s->empty[st]);
                tc_commit(&s->sf_empty[sb]);
            }
        }
        if (PAIR)
            tc_commit_pair(&s->tmem_full, 0x3);
        else
            tc_commit(&s->tmem_full);
    }
    return;
drain:
    if (issued) {
        // wait until every tcgen05 op issued so far has finished
        if (PAIR)
            tc_commit_pair(&s->drain, 0x1);
        else
            tc_commit(&s->drain);
        volatile int never = 0;
        mbar_wait_bounded(&s->drain, 0, &never, p.limit_ns);
    }
}

// ---------------------------------------------------------------- copies ----
// Copy warp `part` moves its share of the stage's twelve 512-byte scale tiles
// (4 SFA, 4 SFB rows 0..127, 4 SFB rows 128..255; NC = 3: four each, NC = 2:
// six each) from shared memory into the stage's TMEM scale buffer
// (tcgen05.cp 32x128b.warpx4: one tile into lanes 0..31, copied to all four
// lane quarters), then commits to sf_full.
template <bool PAIR, int NC>
__device__ void scale_copier(const Params& p, Smem<Cfg<PAIR>::STAGES>* s, uint8_t* ring, uint32_t tmem, int part) {
    using C = Cfg<PAIR>;
    using T = Tm<NC>;
    constexpr int PER = 3 * KB_PER_STAGE / NC;  // tiles per copy warp and stage: 6 (NC = 2) or 4 (NC = 3)
    volatile int* abort = &s->abort_flag;
    const uint32_t sf_s = smem_u32(ring) + A_BYTES + C::B_BYTES;  // SFA, then SFB rows 0..127, then 128..255
    const uint64_t desc0 = smem_desc(sf_s, 0, 128, kLayoutNone);
    int first, step;
    tile_range<PAIR>(first, step);
    uint32_t it = 0;
    for (int tile = first; tile < p.num_tiles; tile += step) {
        for (int kt = 0; kt < p.kt_count; kt++, it++) {
            const int st = it % C::STAGES;
            const uint32_t sb = it % T::NSF;
            if (!mbar_wait_bounded(&s->full[st], (it / C::STAGES) & 1, abort, p.limit_ns) ||
                !mbar_wait_bounded(&s->sf_empty[sb], ((it / T::NSF) & 1) ^ 1, abort, p.limit_ns)) {
                if (!*abort) raise_abort(s, p, 5);
                return;
            }
            tc_fence_after();
            const uint64_t d = desc0 + (uint64_t)((st * C::STAGE_BYTES) >> 4);
            const uint32_t t = tmem + sb * SF_COLS;
#pragma unroll
            for (int c = 0; c < PER; c++) {
                // tile g of the stage: which = g / 4 (SFA, SFB rows 0..127, SFB rows
                // 128..255: 2 KB apart in shared memory), k-block g % 4
                const int g = part * PER + c;
                const int which = g / KB_PER_STAGE, kb = g % KB_PER_STAGE;
                const uint32_t dst =
                    t + (which == 0 ? T::SFA_COL + 4u * kb : T::SFB_COL + 8u * kb + 4u * (uint32_t)(which - 1));
                const uint64_t src = d + (uint64_t)((which * SFA_BYTES + kb * 512) >> 4);
                if (PAIR)
                    tc_cp_32x128b_x4_pair(dst, src);
                else
                    tc_cp_32x128b_x4(dst, src);
            }
            if (PAIR)
                tc_commit_pair(&s->sf_full[sb], 0x1);
            else
                tc_commit(&s->sf_full[sb]);
        }
    }
}

// ---------------------------------------------------------------- epilogue --
// GELU, tanh form, on a pair: (y / 2) (1 + tanh(u)) with u = sqrt(2/pi) (y +
// 0.044715 y^3) = y * (sqrt(2/pi) + sqrt(2/pi) 0.044715 y^2) and the hardware
// tanh (tanh.approx.f32): the value moves by at most ~3e-4 |y| from the exact
// tanh form.  The product form keeps the sign of a negative y whose tanh
// rounds to -1 (a -0 result, as the exact value's tiny negative), which a
// fused h + h tanh(u) would turn into +0.
__device__ __forceinline__ float2 gelu2(float2 y) {
    const float2 k = make_float2(0.7978845608028654f, 0.7978845608028654f);       // sqrt(2 / pi)
    const float2 kc = make_float2(0.0356774081363001f, 0.0356774081363001f);      // sqrt(2 / pi) * 0.044715
    const float2 half = make_float2(0.5f, 0.5f);
    const float2 one = make_float2(1.0f, 1.0f);
    const float2 u = mul2(y, fma2(kc, mul2(y, y), k));
    float2 th;
    asm("tanh.approx.f32 %0, %1;" : "=f"(th.x) : "f"(u.x));
    asm("tanh.approx.f32 %0, %1;" : "=f"(th.y) : "f"(u.y));
    return mul2(mul2(half, y), add2(one, th));
}

// 32 consecutive bf16 (as binary32), columns n0.. with `valid` of them in
// range (fully unrolled: the values stay in registers)
__device__ __forceinline__ void load_row32(const __nv_bfloat16* p, int valid, float* out) {
    if (valid >= 32) {
        const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
        for (int i = 0; i < 4; i++) bf16x8_to_f32(__ldg(q + i), out + 8 * i);
    } else {
#pragma unroll
        for (int i = 0; i < 32; i++) out[i] = (i < valid) ? __bfloat162float(p[i]) : 0.0f;
    }
}

// Per-tile staged column vectors in shared memory, binary32 [VEC_N][BN]:
// bias, 1 + modulate scale (fl32 of the sum), modulate shift, gate.
constexpr int VEC_BIAS = 0, VEC_SCALE1 = 1, VEC_SHIFT = 2, VEC_GATE = 3, VEC_N = 4;

// 32 binary32 of a staged vector (the same for every lane: broadcast loads)
__device__ __forceinline__ void smem_vec32(const float* v, float2* out) {
    const float4* q = reinterpret_cast<const float4*>(v);
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const float4 f = q[i];
        out[2 * i] = make_float2(f.x, f.y);
        out[2 * i + 1] = make_float2(f.z, f.w);
    }
}

// Requant constants of one launch: the output tensor scale a32, 6 a32, and
// the reciprocal 1 / (s * a32) of every E4M3 code s (0 for s == 0 or
// a32 == 0), a table each CTA fills once.
struct RequantConsts {
    float a32, d6;
    const float* inv_tab;
};

// E4M3 code of the block max and the block's reciprocal scale: the quantize
// rule s = E4M3_rne_satfinite(amax / (6 a32)), 1 / (s a32) from the table.
__device__ __forceinline__ uint32_t requant_scale(float amax_b, const RequantConsts& k, float& inv) {
    const uint32_t code = k.d6 == 0.0f ? 0u : e4m3_code(__fdiv_rn(amax_b, k.d6));
    inv = k.inv_tab[code];
    return code;
}

// Eight pairs (16 elements of one block) times inv -> 64 bits of E2M1 codes.
__device__ __forceinline__ uint2 encode16x2(const float2* y, float inv) {
    const float2 iv = make_float2(inv, inv);
    float q[16];
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const float2 t = mul2(y[i], iv);
        q[2 * i] = t.x;
        q[2 * i + 1] = t.y;
    }
    // a flushed block (s == 0 or a32 == 0: inv == 0) is +0 codes (not the -0
    // that negative values times 0 would give)
    return inv == 0.0f ? make_uint2(0u, 0u) : make_uint2(e2m1x8(q), e2m1x8(q + 8));
}

// One 32-column chunk of one output row: epilogue math and outputs.  `r`
// holds the accumulator (binary32 bits), `tv` the tile's staged vectors,
// `stage` this warp's staging buffer.  The arithmetic is binary32 on pairs:
// y = fma(acc, a32_A a32_B, bias) (one rounding), then GELU, y (1 + scale),
// + shift, gate * y, residual + y as the header states.  The NVFP4 requant and
// out_amax cover the column window [q_col0, q_col1) only (its ends are
// multiples of 64 when requantizing, so a chunk is inside or outside it as a
// whole); requant column n lands at n - q_col0 of an [M x (q_col1 - q_col0)]
// operand with tiles_on scale tiles along its row.
__device__ __forceinline__ void epilogue_chunk(const Params& p, const uint32_t* r, float alpha, int64_t m, bool row_ok,
                                               int64_t n0, int j, int valid, const RequantConsts& rq,
                                               int64_t tiles_on, float& amax_run, const float* tv, uint8_t* stage,
                                               int lane) {
    float2 y[16];
    float2 v[16];
    const float2 al = make_float2(alpha, alpha);
    if (p.bias) {
        smem_vec32(tv + VEC_BIAS * BN + j * 32, v);
#pragma unroll
        for (int i = 0; i < 16; i++) y[i] = fma2(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), al, v[i]);
    } else {
#pragma unroll
        for (int i = 0; i < 16; i++) y[i] = mul2(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), al);
    }
    if (p.act == NVFP4_ACT_GELU_TANH) {
#pragma unroll
        for (int i = 0; i < 16; i++) y[i] = gelu2(y[i]);
    }
    if (p.mod_scale) {
        smem_vec32(tv + VEC_SCALE1 * BN + j * 32, v);
#pragma unroll
        for (int i = 0; i < 16; i++) y[i] = mul2(y[i], v[i]);
    }
    if (p.mod_shift) {
        smem_vec32(tv + VEC_SHIFT * BN + j * 32, v);
#pragma unroll
        for (int i = 0; i < 16; i++) y[i] = add2(y[i], v[i]);
    }
    if (p.gate) {
        smem_vec32(tv + VEC_GATE * BN + j * 32, v);
#pragma unroll
        for (int i = 0; i < 16; i++) y[i] = mul2(v[i], y[i]);
    }
    if (p.residual && row_ok) {
        float rv[32];
        load_row32(p.residual + m * p.ld_res + n0, valid, rv);
#pragma unroll
        for (int i = 0; i < 16; i++) y[i] = add2(make_float2(rv[2 * i], rv[2 * i + 1]), y[i]);
    }
    const bool in_win = n0 >= p.q_col0 && n0 < p.q_col1;
    if (p.out_amax && row_ok && in_win) {
        const int wv = (int)min((int64_t)valid, (int64_t)p.q_col1 - n0);
#pragma unroll
        for (int i = 0; i < 16; i++) {
            if (2 * i < wv) amax_run = fmaxf(amax_run, fabsf(y[i].x));
            if (2 * i + 1 < wv) amax_run = fmaxf(amax_run, fabsf(y[i].y));
        }
    }
    if (p.debug_y && row_ok) {
        float* d = p.debug_y + m * p.N + n0;
#pragma unroll
        for (int i = 0; i < 16; i++) {
            if (2 * i < valid) d[2 * i] = y[i].x;
            if (2 * i + 1 < valid) d[2 * i + 1] = y[i].y;
        }
    }
    if (p.c) {
        // row `lane` of the staging buffer; the TMA store drops rows >= M and columns >= N
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; i++) {
            __nv_bfloat162 bb = __floats2bfloat162_rn(y[i].x, y[i].y);
            w[i] = *reinterpret_cast<uint32_t*>(&bb);
        }
        uint8_t* row = stage + lane * 64;
        const int sw = (lane >> 1) & 3;
#pragma unroll
        for (int u = 0; u < 4; u++)
            *reinterpret_cast<uint4*>(row + ((u ^ sw) << 4)) = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
    }
    if (p.out_codes && in_win) {
        // the window's ends are multiples of 64, so a 32-column chunk inside it is whole
        const int64_t nq = n0 - p.q_col0;
        const int64_t bj = nq / 16;
        uint16_t sc2 = 0;
        if (row_ok) {
            float am0 = 0.0f, am1 = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                am0 = fmaxf(am0, fmaxf(fabsf(y[i].x), fabsf(y[i].y)));
                am1 = fmaxf(am1, fmaxf(fabsf(y[8 + i].x), fabsf(y[8 + i].y)));
            }
            float inv0, inv1;
            const uint32_t c0 = requant_scale(am0, rq, inv0);
            const uint32_t c1 = requant_scale(am1, rq, inv1);
            const uint2 w0 = encode16x2(y, inv0);
            const uint2 w1 = encode16x2(y + 8, inv1);
            *reinterpret_cast<uint4*>(p.out_codes + m * ((p.q_col1 - p.q_col0) / 2) + nq / 2) =
                make_uint4(w0.x, w0.y, w1.x, w1.y);
            sc2 = (uint16_t)(c0 | (c1 << 8));
        }
        // rows past M up to the next multiple of 128 are scale padding: zero
        // (a 256-row pair tile can reach past that; those rows have no scales)
        if (m < ((int64_t)p.M + 127) / 128 * 128)
            *reinterpret_cast<uint16_t*>(p.out_scales + swz_offset(m, bj, tiles_on)) = sc2;
    }
}

// Epilogue warp w (2..9) reads TMEM lane quarter w % 4 (rows 32 (w % 4) ..
// of the CTA's 128) and the 32-column chunks j = h, h + 2, h + 4, h + 6 of
// the tile (h = (w - 2) / 4).  The chunks this accumulator shares with the
// other one (Tm::OVERLAP_CHUNKS at the high end of buffer 0, at the low end
// of buffer 1) come first; once they are in registers the warp arrives on
// tmem_empty (8 warps per CTA), so the next tile's MMAs can start.
template <bool PAIR, int NC, bool EARLY>
__device__ void epilogue(const Params& p, Smem<Cfg<PAIR>::STAGES>* s, uint32_t tmem, int warp, int lane, uint32_t rank,
                         const CUtensorMap* tma_c, uint8_t* epi_stage, float* vecs, float* inv_tab) {
    using C = Cfg<PAIR>;
    constexpr int OV = Tm<NC>::OVERLAP_CHUNKS;
    static_assert(!EARLY || OV <= 4, "an early warp holds at most two shared chunks");
    volatile int* abort = &s->abort_flag;
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int h = (warp - 2) >> 2;          // column chunks h, h + 2, h + 4, h + 6
    const int et = (warp - 2) * 32 + lane;  // 0..255 over the epilogue warps
    const float alpha = __fmul_rn(__ldg(p.ga), __ldg(p.gb));
    const float oa32 = p.out_codes ? __ldg(p.out_gscale) : 0.0f;
    // the requant's reciprocal table: one entry per epilogue thread (256 codes)
    if (p.out_codes) {
        const float sv = e4m3_value((uint32_t)et);
        inv_tab[et] = (oa32 == 0.0f || sv == 0.0f) ? 0.0f : __frcp_rn(__fmul_rn(sv, oa32));
    }
    const RequantConsts rq{oa32, __fmul_rn(6.0f, oa32), inv_tab};
    const int64_t tiles_on = ((int64_t)(p.q_col1 - p.q_col0) + 63) / 64;  // scale tiles along the requant window
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    // the leader's MMA waits for the epilogue warps of both CTAs
    const uint32_t empty_bar = PAIR ? mapa_shared(smem_u32(&s->tmem_empty), 0) : smem_u32(&s->tmem_empty);
    const __nv_bfloat16* vsrc[4] = {p.bias, p.mod_scale, p.mod_shift, p.gate};
    uint8_t* stage = epi_stage + (warp - 2) * EPI_BUF_BYTES;
    if (p.c && lane == 0) prefetch_tmap(tma_c);
    int first, step;
    tile_range<PAIR>(first, step);
    float amax_run = 0.0f;
    uint32_t tcount = 0;
    for (int tile = first; tile < p.num_tiles; tile += step, tcount++) {
        int mb, nb;
        tile_coords(p, tile, mb, nb);
        // stage this tile's per-column vectors as binary32 (one column per
        // epilogue thread; past N: 0, and 1 + scale = 1)
        float* tv = vecs + (tcount & 1) * VEC_N * BN;
        {
            const int64_t n = (int64_t)nb * BN + et;
#pragma unroll
            for (int v = 0; v < VEC_N; v++) {
                if (vsrc[v]) {
                    const float x = n < p.N ? __bfloat162float(vsrc[v][n]) : 0.0f;
                    tv[v * BN + et] = v == VEC_SCALE1 ? __fadd_rn(1.0f, x) : x;
                }
            }
        }
        const bool ok = mbar_wait_bounded(&s->tmem_full, tcount & 1, abort, p.limit_ns);
        if (!ok && !*abort) raise_abort(s, p, 4);
        // the staged vectors are visible, and all epilogue warps take the same exit
        if (named_barrier_or(1, EPI_THREADS, !ok)) break;
        tc_fence_after();
        const int64_t m0 = (int64_t)mb * C::TILE_M + (int64_t)rank * BM + q * 32;  // the warp's first row
        const int64_t m = m0 + lane;
        const bool row_ok = m < p.M;
        const int ncols = min(BN, p.N - nb * BN);
        const int nchunks = (ncols + 31) / 32;
        const int nmy = (nchunks - h + 1) >> 1;  // this warp's chunks: i = 0 .. nmy - 1, j = h + 2 i
        const bool buf1 = tcount & 1;
        const uint32_t acc = lane_base + (buf1 ? Tm<NC>::ACC1_COL : 0u);
        // shared chunks: buffer 1's first OV, buffer 0's last OV; as indices i of this warp's
        // chunks they are a prefix (buffer 1) or a suffix starting at s0 (buffer 0)
        const int s0 = (BN / 32 - OV - h + 1) >> 1;
        const int n_ov = buf1 ? min(nmy, (OV - h + 1) >> 1) : max(0, nmy - s0);
        // processing order t = 0 .. nmy - 1: shared chunks first
        auto chunk_of = [&](int t) { return h + 2 * (buf1 ? t : (t < n_ov ? s0 + t : t - n_ov)); };
        auto out_chunk = [&](const uint32_t* r, int j) {
            const int64_t n0 = (int64_t)nb * BN + j * 32;
            const int valid = (int)min((int64_t)32, p.N - n0);
            if (p.c) {
                // the previous store has finished reading the staging buffer
                if (lane == 0) bulk_wait_group_read<0>();
                __syncwarp();
            }
            epilogue_chunk(p, r, alpha, m, row_ok, n0, j, valid, rq, tiles_on, amax_run, tv, stage, lane);
            if (p.c) {
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(tma_c, stage, (int32_t)n0, (int32_t)m0);
                    bulk_commit_group();
                }
            }
        };
        if (EARLY) {
            // the shared chunks (at most two) go to registers first; then the next tile may start
            uint32_t ov0[32], ov1[32];
            if (n_ov > 0) tmem_ld_32cols(acc + chunk_of(0) * 32, ov0);
            if (n_ov > 1) tmem_ld_32cols(acc + chunk_of(1) * 32, ov1);
            tmem_ld_wait();
            tmem_regs_ready(ov0);
            tmem_regs_ready(ov1);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(empty_bar);
            for (int t = 0; t < nmy; t++) {
                const int j = chunk_of(t);
                uint32_t r[32];
                if (t < n_ov) {
#pragma unroll
                    for (int e = 0; e < 32; e++) r[e] = t == 0 ? ov0[e] : ov1[e];
                } else {
                    tmem_ld_32cols(acc + j * 32, r);
                    tmem_ld_wait();
                    tmem_regs_ready(r);
                }
                out_chunk(r, j);
            }
        } else {
            if (n_ov == 0) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(empty_bar);
            }
            for (int t = 0; t < nmy; t++) {
                const int j = chunk_of(t);
                uint32_t r[32];
                tmem_ld_32cols(acc + j * 32, r);
                tmem_ld_wait();
                tmem_regs_ready(r);
                if (t == n_ov - 1) {
                    // this warp's shared columns are in registers: the next tile may start
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(empty_bar);
                }
                out_chunk(r, j);
            }
        }
    }
    if (p.c && lane == 0) bulk_wait_group_all();
    if (p.out_amax) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax_run = fmaxf(amax_run, __shfl_xor_sync(0xFFFFFFFFu, amax_run, o));
        if (lane == 0) atomicMax(reinterpret_cast<unsigned int*>(p.out_amax), __float_as_uint(amax_run));
    }
}

template <bool PAIR, int NC>
__global__ void __launch_bounds__(threads_for(NC), 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                const __grid_constant__ CUtensorMap tma_sfa, const __grid_constant__ CUtensorMap tma_sfb,
                const __grid_constant__ CUtensorMap tma_c, const __grid_constant__ Params p) {
    using C = Cfg<PAIR>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // the next kernel on the stream (if launched with programmatic stream
    // serialization) may be scheduled now; it waits for this grid to complete
    // before it touches global memory
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* epi_stage = ring + C::STAGES * C::STAGE_BYTES;  // 1024-aligned (STAGE_BYTES % 1024 == 0)
    float* vecs = reinterpret_cast<float*>(epi_stage + EPI_STAGE_BYTES);
    float* inv_tab = reinterpret_cast<float*>(epi_stage + EPI_STAGE_BYTES + VEC_BYTES);
    Smem<C::STAGES>* s = reinterpret_cast<Smem<C::STAGES>*>(epi_stage + EPI_STAGE_BYTES + VEC_BYTES + INV_TAB_BYTES);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::STAGES; i++) {
            mbar_init(&s->full[i], 1);
            mbar_init(&s->empty[i], 1);
        }
        mbar_init(&s->tmem_full, 1);
        mbar_init(&s->tmem_empty, EPI_WARPS * C::CTAS);
        mbar_init(&s->drain, 1);
        for (int i = 0; i < Tm<NC>::NSF; i++) {
            mbar_init(&s->sf_full[i], NC);
            mbar_init(&s->sf_empty[i], 1);
        }
        s->abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        if (PAIR) {
            tmem_alloc_pair(&s->tmem_base, TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(&s->tmem_base, TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    if (PAIR)
        cluster_sync_all();  // peer barriers initialized before any remote arrive / multicast
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s->tmem_base;
    // Launched with programmatic stream serialization, this grid may start
    // while the previous kernel on the stream is still finishing (its CTAs
    // free SMs one by one): everything above touches only this CTA's shared
    // memory and TMEM; wait for that kernel to complete, with its memory
    // visible, before any global access (its outputs are read here, and it may
    // still read what this kernel writes).
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        if (lane == 0) producer<PAIR>(p, s, ring, &tma_a, &tma_b, &tma_sfa, &tma_sfb, rank);
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) mma_issuer<PAIR, NC>(p, s, ring, tmem);
        __syncwarp();
    } else if (warp >= FIRST_COPY_WARP) {
        if (lane == 0 && rank == 0) scale_copier<PAIR, NC>(p, s, ring, tmem, warp - FIRST_COPY_WARP);
        __syncwarp();
    } else {
        epilogue<PAIR, NC, NC == 2>(p, s, tmem, warp, lane, rank, &tma_c, epi_stage, vecs, inv_tab);
    }
    tc_fence_before();
    if (PAIR)
        cluster_sync_all();  // neither CTA leaves while the pair's MMAs may touch it
    else
        __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        if (PAIR)
            tmem_dealloc_pair(tmem, TMEM_COLS);
        else
            tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace gemm

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn g_encode_tiled = nullptr;  // driver entry point, looked up once per process
static std::once_flag g_encode_once;

struct GemmDevice {
    int sms;
    int pair_clusters;
};
static PerDevice<GemmDevice> g_gemm_dev;

static nvfp4_status gemm_setup(int& sms, int& pair_clusters) {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess && fn != nullptr)
            g_encode_tiled = reinterpret_cast<EncodeTiledFn>(fn);
        else
            cudaGetLastError();
    });
    if (g_encode_tiled == nullptr) return NVFP4_ERR_CUDA;
    GemmDevice gd{};
    const nvfp4_status st = g_gemm_dev.get(&gd, [](int dev, GemmDevice& v) {
        int major = 0, minor = 0, n = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (major != 10 || minor != 0) return NVFP4_ERR_UNSUPPORTED;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return NVFP4_ERR_CUDA;
        if (cudaFuncSetAttribute(gemm::gemm_kernel<false, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 gemm::Cfg<false>::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(gemm::gemm_kernel<false, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 gemm::Cfg<false>::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(gemm::gemm_kernel<true, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 gemm::Cfg<true>::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(gemm::gemm_kernel<true, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 gemm::Cfg<true>::SMEM_BYTES) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        // how many CTA pairs can be resident at once (bounds the persistent grid)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (n / 2));
        cfg.blockDim = dim3(gemm::threads_for(3));
        cfg.dynamicSmemBytes = gemm::Cfg<true>::SMEM_BYTES;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;  // shared memory bounds both variants alike: one CTA per SM
        if (cudaOccupancyMaxActiveClusters(&clusters, gemm::gemm_kernel<true, 3>, &cfg) != cudaSuccess || clusters < 1) {
            cudaGetLastError();
            clusters = 0;  // pair variant unavailable: single-CTA tiles only
        }
        v.sms = n;
        v.pair_clusters = clusters;
        return NVFP4_OK;
    });
    if (st != NVFP4_OK) return st;
    sms = gd.sms;
    pair_clusters = gd.pair_clusters;
    return NVFP4_OK;
}

// packed E2M1 codes [rows x K/2] bytes, 128-byte (256-element) boxes of box_rows rows
static bool make_code_map(CUtensorMap* map, const void* codes, int64_t rows, int64_t K, int box_rows) {
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {(cuuint32_t)gemm::BKB, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// bf16 C [M x N], row stride ldc elements; a box is one epilogue warp's 32 rows
// x 32 columns (64-byte rows, 64B swizzle)
static bool make_c_map(CUtensorMap* map, void* c, int64_t M, int64_t N, int64_t ldc) {
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)(ldc * 2)};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, c, dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// swizzled scales viewed as [row blocks][K/64 tiles][128 x u32]; a box is the
// 4 tiles (2 KB) of one stage of one 128-row block.  Tiles past K/64 read as 0.
static bool make_scale_map(CUtensorMap* map, const void* scales, int64_t rows, int64_t K) {
    const int64_t tiles_k = K / 64, blocks = (rows + 127) / 128;
    cuuint64_t dims[3] = {128, (cuuint64_t)tiles_k, (cuuint64_t)blocks};
    cuuint64_t strides[2] = {512, (cuuint64_t)(tiles_k * 512)};
    cuuint32_t box[3] = {128, (cuuint32_t)gemm::KB_PER_STAGE, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(scales), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

static inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status nvfp4_gemm(const nvfp4_tensor* A, const nvfp4_tensor* B, void* c_bf16, int64_t ldc,
                                   const nvfp4_epilogue* ep, void* workspace, size_t ws_bytes,
                                   nvfp4_stream_t stream) {
    if (!A || !B || !workspace) return NVFP4_ERR_INVALID_ARG;
    if (!A->codes || !A->scales || !A->global_scale || !B->codes || !B->scales || !B->global_scale)
        return NVFP4_ERR_INVALID_ARG;
    const int64_t M = A->rows, N = B->rows, K = A->cols;
    if (M <= 0 || N <= 0 || K <= 0 || B->cols != K) return NVFP4_ERR_INVALID_ARG;
    if (K % 64 != 0) return NVFP4_ERR_UNSUPPORTED;
    if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return NVFP4_ERR_UNSUPPORTED;
    if (ws_bytes < nvfp4_workspace_bytes(NVFP4_OP_GEMM, M, N, K)) return NVFP4_ERR_INVALID_ARG;
    const bool requant = ep && ep->out_codes;
    if (!c_bf16 && !requant) return NVFP4_ERR_INVALID_ARG;
    if (requant && (!ep->out_scales || !ep->out_global_scale)) return NVFP4_ERR_INVALID_ARG;
    // the requant / out_amax column window (out_cols == 0: all N columns)
    const int64_t win0 = ep ? ep->out_col0 : 0;
    const int64_t wcols = (ep && ep->out_cols) ? ep->out_cols : N - win0;
    if (win0 < 0 || wcols <= 0 || win0 + wcols > N) return NVFP4_ERR_INVALID_ARG;
    if (requant && (win0 % 64 != 0 || wcols % 64 != 0)) return NVFP4_ERR_UNSUPPORTED;
    if (ep && ep->act != NVFP4_ACT_NONE && ep->act != NVFP4_ACT_GELU_TANH) return NVFP4_ERR_INVALID_ARG;
    if (ep && (ep->debug_flags & ~NVFP4_DBG_SKIP_LOADS)) return NVFP4_ERR_INVALID_ARG;
    if (ep && ep->residual && ep->ld_residual < N) return NVFP4_ERR_INVALID_ARG;
    if (c_bf16 && ldc < N) return NVFP4_ERR_INVALID_ARG;
    if (!al16(A->codes) || !al16(A->scales) || !al16(B->codes) || !al16(B->scales) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return NVFP4_ERR_MISALIGNED;
    if (c_bf16 && (!al16(c_bf16) || ldc % 8 != 0)) return NVFP4_ERR_MISALIGNED;
    if (ep) {
        const void* vecs[4] = {ep->bias, ep->mod_scale, ep->mod_shift, ep->gate};
        for (const void* v : vecs)
            if (v && !al16(v)) return NVFP4_ERR_MISALIGNED;
        if (ep->residual && (!al16(ep->residual) || ep->ld_residual % 8 != 0)) return NVFP4_ERR_MISALIGNED;
        if (requant && (!al16(ep->out_codes) || !al16(ep->out_scales))) return NVFP4_ERR_MISALIGNED;
        if (ep->out_amax && (reinterpret_cast<uintptr_t>(ep->out_amax) & 3u)) return NVFP4_ERR_MISALIGNED;
        if (ep->debug_y && (reinterpret_cast<uintptr_t>(ep->debug_y) & 3u)) return NVFP4_ERR_MISALIGNED;
    }
    int sms = 0, pair_clusters = 0;
    nvfp4_status st = gemm_setup(sms, pair_clusters);
    if (st != NVFP4_OK) return st;
    // CTA pairs (256-row tiles) whenever there is more than one 128-row block
    const bool pair = M > gemm::BM && pair_clusters > 0;

    CUtensorMap ma, mb, msa, msb, mc;
    memset(&mc, 0, sizeof(mc));
    if (c_bf16 && !make_c_map(&mc, c_bf16, M, N, ldc)) return NVFP4_ERR_CUDA;
    if (!make_code_map(&ma, A->codes, M, K, gemm::BM) ||
        !make_code_map(&mb, B->codes, N, K, pair ? gemm::Cfg<true>::B_ROWS : gemm::Cfg<false>::B_ROWS) ||
        !make_scale_map(&msa, A->scales, M, K) || !make_scale_map(&msb, B->scales, N, K))
        return NVFP4_ERR_CUDA;

    gemm::Params p{};
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    const int tile_m = pair ? gemm::Cfg<true>::TILE_M : gemm::Cfg<false>::TILE_M;
    p.tiles_m = (int)((M + tile_m - 1) / tile_m);
    p.tiles_n = (int)((N + gemm::BN - 1) / gemm::BN);
    p.num_tiles = p.tiles_m * p.tiles_n;
    p.kt_count = (int)((K + gemm::BK - 1) / gemm::BK);
    p.kb_total = (int)(K / 64);
    p.ga = A->global_scale;
    p.gb = B->global_scale;
    p.c = static_cast<__nv_bfloat16*>(c_bf16);
    p.ldc = ldc;
    if (ep) {
        p.bias = static_cast<const __nv_bfloat16*>(ep->bias);
        p.mod_scale = static_cast<const __nv_bfloat16*>(ep->mod_scale);
        p.mod_shift = static_cast<const __nv_bfloat16*>(ep->mod_shift);
        p.gate = static_cast<const __nv_bfloat16*>(ep->gate);
        p.residual = static_cast<const __nv_bfloat16*>(ep->residual);
        p.ld_res = ep->ld_residual;
        p.act = ep->act;
        p.out_codes = static_cast<uint8_t*>(ep->out_codes);
        p.out_scales = static_cast<uint8_t*>(ep->out_scales);
        p.out_gscale = ep->out_global_scale;
        p.out_amax = ep->out_amax;
        p.q_col0 = (int)win0;
        p.q_col1 = (int)(win0 + wcols);
        p.debug_y = ep->debug_y;
        p.dbg = ep->debug_flags;
        p.limit_ns = (uint64_t)(ep->wait_limit_us ? ep->wait_limit_us : 2000000u) * 1000ull;
    } else {
        p.limit_ns = 2000000000ull;
        p.q_col0 = 0;
        p.q_col1 = (int)N;
    }
    p.err = static_cast<DevError*>(workspace);
    // short K (at most 16 stages per tile): the epilogue bounds the tile rate,
    // so take the variant whose epilogue frees the accumulator soonest
    const int nc = p.kt_count <= 16 ? 2 : 3;
    if (pair) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * std::min(p.num_tiles, pair_clusters));
        cfg.blockDim = dim3(gemm::threads_for(nc));
        cfg.dynamicSmemBytes = gemm::Cfg<true>::SMEM_BYTES;
        cfg.stream = (cudaStream_t)stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        // programmatic dependent launch: the grid's prologue (barriers, TMEM,
        // cluster sync) overlaps the previous kernel's last tiles
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        if (cudaLaunchKernelEx(&cfg, nc == 2 ? gemm::gemm_kernel<true, 2> : gemm::gemm_kernel<true, 3>, ma, mb, msa, msb,
                               mc, p) != cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_CUDA;
        }
        return NVFP4_OK;
    }
    const int grid = std::min(p.num_tiles, sms);
    if (nc == 2)
        gemm::gemm_kernel<false, 2><<<grid, gemm::threads_for(2), gemm::Cfg<false>::SMEM_BYTES, (cudaStream_t)stream>>>(
            ma, mb, msa, msb, mc, p);
    else
        gemm::gemm_kernel<false, 3><<<grid, gemm::threads_for(3), gemm::Cfg<false>::SMEM_BYTES, (cudaStream_t)stream>>>(
            ma, mb, msa, msb, mc, p);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
