/*
 * nvfp4.h -- C ABI of libnvfp4.so: the NVFP4 W4A4 linear layer and the NVFP4
 * KV-cache store, hand-written for NVIDIA B200 (sm_100a).
 *
 * Sources (page title + section):
 *  [RN]   "LongLive-2.0：用 NVFP4 并行底座做长视频生成" (yingwang.github.io
 *         reading note), section 二 方法 / "NVFP4 量化格式": E2M1 element codes,
 *         three-level scaling (FP32 tensor factor, FP8 E4M3 factor per
 *         16-element block, FP4 element) and the Dequant equation
 *         Dequant(X) = X^FP4 * a^FP8 * a^FP32.
 *  [RN-T] same note, "NVFP4 训练的工程细节": weights and activations both 4-bit
 *         (W4A4) through self-written CUDA kernels; 1D block scaling along K.
 *  [RN-I] same note, "推理底座": 4-bit weights and activations at inference;
 *         per-frame-chunk KV quantization, K and V separately, storage
 *         9/8 * T_c * H * d bytes, dequant in a self-written CUDA kernel.
 *  [NEWS] anzhuoshouzhuan.com LongLive 2.0 article, "NVFP4 量化" section:
 *         fused RoPE/adaLN kernels and an in-place quantized KV-cache update.
 *
 * Data formats (all buffers are device memory owned by the caller):
 *  - codes: packed E2M1, two per byte, element 2i in bits 3:0 and element
 *    2i+1 in bits 7:4; a [rows x cols] tensor takes rows*cols/2 bytes,
 *    row-major with rows of cols/2 bytes.
 *  - block scales: one E4M3 byte per 16 consecutive elements of a row.
 *    GEMM operands use the tensor-core scale-factor tile layout ("swizzled"):
 *    rows padded to a multiple of 128 and scale columns to a multiple of 4;
 *    tile (i, j) (rows 128i.., scale columns 4j..) is 512 contiguous bytes at
 *    (i * ceil(cols/64) + j) * 512; inside it element (r, c) is at byte
 *    (r % 32) * 16 + (r / 32) * 4 + c.  Padding bytes are zero.  KV slots use
 *    plain row-major scales [rows x cols/16].
 *  - tensor scale a32: one binary32 in device memory.
 *  Quantization of x with tensor scale a32 (readings of [RN]; the pages give
 *  no rounding rule):  a32 = amax|x| / 2688 (2688 = 6 * 448) when computed;
 *  per block  s = E4M3_rne_satfinite(amax_b / (6 * a32));  if s == 0 the
 *  block's codes are +0, else  code = E2M1_rne_satfinite(x * (1 / (s * a32)))
 *  with the sign of the product kept (negative values that round to zero give
 *  code 0x8).  Every step is one binary32 operation rounded to nearest-even.
 *
 * Conventions:
 *  - The library never allocates, frees or synchronizes (except
 *    nvfp4_read_device_error).  All work is enqueued on `stream`.
 *  - Host-side argument checks run before any launch and return a status;
 *    nothing is launched when a check fails.  Launch failures return
 *    NVFP4_ERR_CUDA.  Errors found on the device (a bounded wait that ran out,
 *    a page-table entry out of range) are recorded in the first 16 bytes of
 *    the workspace and read back with nvfp4_read_device_error.
 *  - Device pointers must be 16-byte aligned.  Inputs must be finite.
 *  - Thread safety: calls may be issued from several host threads on
 *    different streams as long as each call has its own workspace.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream (NULL = the legacy default stream). */
typedef struct CUstream_st* nvfp4_stream_t;

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad flag */
    NVFP4_ERR_UNSUPPORTED = 2, /* shape the kernels do not handle, or no sm_100 device */
    NVFP4_ERR_MISALIGNED = 3,  /* pointer or leading dimension not 16-byte aligned */
    NVFP4_ERR_CUDA = 4,        /* a CUDA runtime / driver call failed */
    NVFP4_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out (device error) */
    NVFP4_ERR_DEVICE = 6       /* other device-detected error, e.g. slot out of range */
} nvfp4_status;

/* Static text for a status; never NULL. */
const char* nvfp4_status_string(nvfp4_status s);

/* Library version, (major << 16) | minor. */
int nvfp4_version(void);

/* Bytes of packed E2M1 codes for a [rows x cols] tensor: rows * cols / 2.
 * Returns 0 for negative sizes or odd cols. */
size_t nvfp4_codes_bytes(int64_t rows, int64_t cols);

/* Bytes of block scales for a [rows x cols] tensor (cols % 16 == 0):
 * swizzled != 0 -> ceil(rows/128)*128 * ceil(cols/64)*4 (GEMM operand layout);
 * swizzled == 0 -> rows * cols / 16 (row-major, KV slots).  0 on bad sizes. */
size_t nvfp4_scales_bytes(int64_t rows, int64_t cols, int swizzled);

enum {
    NVFP4_OP_QUANTIZE = 0,  /* nvfp4_quantize: m = rows, k = cols, n unused */
    NVFP4_OP_GEMM = 1,      /* nvfp4_gemm */
    NVFP4_OP_KV_APPEND = 2, /* nvfp4_kv_append */
    NVFP4_OP_KV_DEQUANT = 3, /* nvfp4_kv_dequant */
    NVFP4_OP_LN_QUANTIZE = 4, /* nvfp4_ln_modulate_quantize (m = rows) */
    NVFP4_OP_QUANTIZE_2D = 5, /* nvfp4_quantize_2d */
    NVFP4_OP_QUANTIZE_T = 6,  /* nvfp4_quantize_t */
    NVFP4_OP_KV_ATTENTION = 7 /* nvfp4_kv_attention */
};

/* Workspace bytes the caller must pass to the call `op` (device memory,
 * 256-byte aligned).  Never 0.  Its first 256 bytes are a control block (the
 * device error record in bytes 0..15; for quantize and KV append also the
 * grid-barrier words of the fused kernel): they must be zero before a
 * workspace is first used, and the calls leave them ready for the next call.
 * A workspace may be reused by calls that are ordered on one stream; calls
 * that can run concurrently need their own workspaces. */
size_t nvfp4_workspace_bytes(int op, int64_t m, int64_t n, int64_t k);

/* Synchronizes `stream`, then reads and clears the device error record of
 * `workspace` (written by the calls that used it); after an error the whole
 * 256-byte control block is reset.  *code receives
 * NVFP4_OK, NVFP4_ERR_TIMEOUT or NVFP4_ERR_DEVICE; *info (may be NULL) a
 * call-specific detail (which wait ran out, the offending page-table index).
 * Returns NVFP4_ERR_CUDA if the synchronization or the copy fails. */
nvfp4_status nvfp4_read_device_error(void* workspace, nvfp4_stream_t stream, int* code, uint32_t* info);

/* ------------------------------------------------------------------------ */
/* Quantize  [RN] three-level scaling, [RN-T] 1D blocks of 16 along a row     */
/* ------------------------------------------------------------------------ */
#define NVFP4_Q_COMPUTE_GLOBAL 0u /* compute a32 = amax / 2688 and write *global_scale */
#define NVFP4_Q_GIVEN_GLOBAL 1u   /* read a32 from *global_scale (delayed scaling) */
#define NVFP4_Q_ROWMAJOR_SCALES 2u /* write row-major scales instead of the swizzled tiles */
/* Adaptive scale search over the block-max targets {4, 6} ([RN] "NVFP4 训练的
 *工程细节" and "推理底座": "adaptive scale search" / "adaptive scale 选择"):
 * per 16-element block, also encode with the block max aimed at 4, i.e.
 * s4 = E4M3(amax_b / fl32(4 * a32)), and keep that encoding when its squared
 * error is smaller.  The error is binary32, summed over the block's elements
 * in order: sum += (x - fl32(fl32(e2m1 * s) * a32))^2; a tie keeps the
 * standard encoding.  The tensor scale a32 is unchanged. */
#define NVFP4_Q_SCALE_SEARCH 4u

/* x_bf16: bf16 [rows x cols], row stride ld elements (ld >= cols, ld % 8 == 0).
 * cols % 64 == 0, rows >= 0; cols <= 2^30 and rows * cols / 16 < 2^31 (the
 * tensor's 16-element blocks), else NVFP4_ERR_UNSUPPORTED.
 * codes: nvfp4_codes_bytes(rows, cols) bytes, rows of cols/2 bytes.
 * scales: nvfp4_scales_bytes(rows, cols, swizzled) bytes (padding zeroed).
 * global_scale: device binary32, written (COMPUTE) or read (GIVEN).
 * workspace: nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, rows, 0, cols) bytes.
 * One cooperative launch (one CTA per SM): the input is read from HBM once
 * (held in registers across a bounded grid barrier that turns the CTAs'
 * maxima into a32) unless it exceeds ~#SMs x 176 KB, in which case the
 * excess is read twice. */
nvfp4_status nvfp4_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld, void* codes,
                            void* scales, float* global_scale, unsigned flags, void* workspace,
                            size_t ws_bytes, nvfp4_stream_t stream);

/* LayerNorm + adaLN modulate + quantize, the step before a DiT linear layer
 * (the pages' fused adaLN kernels, [NEWS] "NVFP4 量化"; here fused with the
 * NVFP4 quantize so the modulated activation never goes to memory in bf16).
 * Per row of x (bf16 [rows x cols], row stride ld): LayerNorm without affine
 * parameters (population variance, eps inside the square root), then
 * m = h * (1 + mod_scale[c]) + mod_shift[c] (bf16 [cols] each, or NULL for
 * 0), all in binary32:
 *   mean = S1 / cols, var = S2 / cols, rstd = 1 / sqrt(var + eps),
 *   m = fl32(fl32(fl32(fl32(x - mean) * rstd) * fl32(1 + scale)) + shift),
 * where S1 = sum x and S2 = sum fl32(x - mean)^2 are summed as 32 partial
 * sums (partial j over elements 256c + 8j .. 256c + 8j + 7 of c = 0, 1, ...
 * in order) combined by an xor butterfly over 16, 8, 4, 2, 1.  m is then quantized exactly as
 * nvfp4_quantize quantizes a tensor (flags as there), a32 from max |m|.
 * cols % 64 == 0, cols <= 2^24, rows <= 2^30, rows * cols / 16 < 2^31;
 * pointers 16-byte aligned.
 * workspace: nvfp4_workspace_bytes(NVFP4_OP_LN_QUANTIZE, rows, 0, cols)
 * bytes (the control block, then the binary32 (mean, rstd) of every row,
 * which the call leaves there).  One cooperative launch when ceil(rows /
 * #SMs) rows fit in a CTA's shared memory (224 KB: 4096 x 3072 does,
 * 8192 x 3072 does not): the rows are bulk-copied in once, the statistics,
 * the tensor maximum and the encode all read them there.  Otherwise two
 * launches: the row statistics, then the fused quantize.  Both give the same
 * bits. */
nvfp4_status nvfp4_ln_modulate_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                        const void* mod_scale, const void* mod_shift, float eps, void* codes,
                                        void* scales, float* global_scale, unsigned flags, void* workspace,
                                        size_t ws_bytes, nvfp4_stream_t stream);

/* nvfp4_quantize without a workspace, for callers that cannot allocate
 * device memory: code hosted inside a framework that owns every device
 * allocation (an engine or server plugin handed only its input and output
 * buffers), or a loop that must not call cudaMalloc because it would
 * synchronize the device or break a fixed memory budget.  The pages have no
 * counterpart of this call; it is a convenience of this library.
 * Same arguments, rules and results as nvfp4_quantize, minus the workspace:
 * the scratch it needs (the 256-byte control block of the grid barrier)
 * lives in one static device array of the library
 * (NVFP4_NOALLOC_SCRATCH_BYTES; a problem that would need more is rejected
 * with NVFP4_ERR_UNSUPPORTED), which every GPU that loads the
 * library holds until the process exits.  The first call on a device looks
 * up the array's device address (cudaGetSymbolAddress), so make that first
 * call before any stream capture.  Each call clears the array (one
 * cudaMemsetAsync on `stream`) and then launches the quantize kernel; it
 * allocates nothing.  Every argument check runs before the clear, so a
 * rejected call enqueues nothing and leaves the array alone.  All calls share
 * the array, so calls that can overlap on the GPU (different streams,
 * different host threads) race: order them on one stream.  Errors found on
 * the device are not reported by this call: if the kernel's bounded
 * grid-barrier wait ever ran out, it would return without writing the codes,
 * scales or tensor scale, leaving those outputs as they were, and the next
 * call's clear erases the record. */
#define NVFP4_NOALLOC_SCRATCH_BYTES 256
nvfp4_status nvfp4_quantize_noalloc(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld, void* codes,
                                    void* scales, float* global_scale, unsigned flags, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* W4A4 GEMM  [RN-T] / [RN-I] W4A4 linears; [NEWS] fused adaLN epilogue        */
/* ------------------------------------------------------------------------ */
/* One NVFP4 operand: codes [rows x cols/2], swizzled scales, device a32. */
typedef struct {
    const void* codes;
    const void* scales;
    const float* global_scale;
    int64_t rows, cols;
} nvfp4_tensor;

#define NVFP4_ACT_NONE 0
#define NVFP4_ACT_GELU_TANH 1 /* 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))) */

/* Debug / test flags of nvfp4_epilogue.debug_flags (0 in production). */
#define NVFP4_DBG_SKIP_LOADS 1u /* producer issues no loads: the consumer's bounded wait
                                   must run out and record NVFP4_ERR_TIMEOUT (tests only) */

/* Epilogue, in binary32, in this order:
 *   y = a32_A * a32_B * acc + bias[n]  (one fused multiply-add; y = a32_A *
 *   a32_B * acc without a bias);  y = act(y);  y = y * (1 + mod_scale[n]);
 *   y = y + mod_shift[n];  y = gate[n] * y;  y = residual[m, n] + y
 * (each step skipped when its pointer is NULL / act is NONE; a32_A * a32_B
 * and 1 + mod_scale[n] rounded to binary32 first).  Then y is
 * stored as bf16 to c (if non-NULL; every column) and/or re-quantized to
 * NVFP4 with the given output tensor scale (if out_codes is non-NULL):
 * blocks of 16 along N, exactly the quantize rule above, over the column
 * window [out_col0, out_col0 + out_cols) (out_cols == 0: every column from
 * out_col0 on; both multiples of 64 for a requant), written as an
 * [M x out_cols] operand: codes [M x out_cols/2], swizzled scales.  A DiT
 * QKV projection can so hand its V third straight to the next GEMM.
 * out_amax (optional) receives atomically max(|y|) over the same window, for
 * calibrating out_global_scale; the caller initializes it.
 * debug_y (optional, tests) receives y as binary32 [M x N] before the store. */
typedef struct {
    const void* bias;      /* bf16 [N] or NULL */
    const void* mod_scale; /* bf16 [N] or NULL (adaLN scale) */
    const void* mod_shift; /* bf16 [N] or NULL (adaLN shift) */
    const void* gate;      /* bf16 [N] or NULL (adaLN gate) */
    const void* residual;  /* bf16 [M x N], row stride ld_residual, or NULL */
    int64_t ld_residual;
    int act;               /* NVFP4_ACT_* */
    void* out_codes;       /* NVFP4 requant: codes [M x out_cols/2] or NULL */
    void* out_scales;      /* swizzled scales for [M x out_cols] */
    const float* out_global_scale; /* device binary32 a32 of the output */
    float* out_amax;       /* device binary32 or NULL */
    float* debug_y;        /* device binary32 [M x N] or NULL */
    unsigned debug_flags;  /* NVFP4_DBG_*, 0 in production */
    uint32_t wait_limit_us; /* bound of every device-side wait; 0 = default (2 s) */
    int64_t out_col0;      /* first column of the requant / out_amax window (0: from column 0) */
    int64_t out_cols;      /* columns in the window (0: through column N - 1) */
} nvfp4_epilogue;

/* C[M x N] = a32_A * a32_B * (A_q . S_A)(B_q . S_B)^T, then the epilogue.
 * A: [M x K] activations, B: [N x K] weights (both K-major, K = A->cols =
 * B->cols, K % 64 == 0).  M, N >= 1, arbitrary (tails handled); M, N, K
 * <= 2^30 (else NVFP4_ERR_UNSUPPORTED).
 * c_bf16: [M x N] with row stride ldc (ldc >= N, ldc % 8 == 0) or NULL when
 * ep->out_codes is set.  ep may be NULL (plain bf16 output).
 * A requant window that is not a multiple of 64 at both ends returns
 * NVFP4_ERR_UNSUPPORTED; one outside [0, N), NVFP4_ERR_INVALID_ARG.
 * workspace: nvfp4_workspace_bytes(NVFP4_OP_GEMM, M, N, K) bytes.
 * One persistent launch (tcgen05 block-scaled MMA, TMEM accumulators, TMA). */
nvfp4_status nvfp4_gemm(const nvfp4_tensor* A, const nvfp4_tensor* B, void* c_bf16, int64_t ldc,
                        const nvfp4_epilogue* ep, void* workspace, size_t ws_bytes, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* NVFP4 KV cache  [RN-I] per-chunk K/V quantization; [NEWS] in-place update  */
/* ------------------------------------------------------------------------ */
/* n_slots slots (frame-chunks), each tokens_per_slot x heads x head_dim.
 * Slot s of K: k_codes + s * T*H*d/2 (T*H*d/2 bytes), k_scales + s * T*H*d/16
 * (row-major scales over rows of head_dim), k_global[s]; same for V.
 * head_dim % 16 == 0; T*H*d % 64 == 0. */
typedef struct {
    void* k_codes;
    void* k_scales;
    void* v_codes;
    void* v_scales;
    float* k_global; /* [n_slots] device binary32 */
    float* v_global; /* [n_slots] device binary32 */
    int32_t n_slots, tokens_per_slot, heads, head_dim;
    uint32_t flags; /* NVFP4_KV_* (0: the standard encoding) */
    float* k_mean;  /* [n_slots][H*d] device binary32, with NVFP4_KV_SMOOTH_K (else unused, may be NULL) */
    float* v_mean;  /* [n_slots][H*d] device binary32, with NVFP4_KV_SMOOTH_V (else unused, may be NULL) */
} nvfp4_kv_cache;

#define NVFP4_KV_SCALE_SEARCH 1u /* appends use the scale search of NVFP4_Q_SCALE_SEARCH */
/* K-smoothing [RN-I] (K and V each, independently): the append takes each
 * channel's mean over the chunk's tokens (channel c = h*d + j; binary32:
 * partial p sums tokens p, p+32, ... in order, the 32 partials meet in an xor
 * butterfly 16, 8, 4, 2, 1, mean = S / T), stores it at *_mean[slot][c] and
 * quantizes fl32(x - mean[c]) (tensor scale from max |x - mean|); the dequant
 * returns bf16_rne(fl32(fl32(fl32(e2m1 * s) * a32) + mean[c])).  Needs
 * T*H*d < 2^31 (the append, as any append, T*H*d <= 2^30), T < 2^24 and the
 * mean array 16-byte aligned; the append is then two launches (the means, then
 * the quantize). */
#define NVFP4_KV_SMOOTH_K 2u
#define NVFP4_KV_SMOOTH_V 4u

/* Quantizes one chunk's K and V (bf16, token-major [T][H][d], contiguous)
 * in place into slot `slot`: one tensor scale per (slot, K|V) = amax / 2688
 * over the whole chunk, then the quantize rule above with row-major scales
 * (with the scale search when cache->flags has NVFP4_KV_SCALE_SEARCH).
 * workspace: nvfp4_workspace_bytes(NVFP4_OP_KV_APPEND, T*H, 0, d) bytes.
 * One cooperative launch covering K and V (as nvfp4_quantize), which takes
 * the chunk as one row of T*H*d elements: T*H*d <= 2^30, else
 * NVFP4_ERR_UNSUPPORTED (the dequant takes slots of up to 2^40 elements). */
nvfp4_status nvfp4_kv_append(const nvfp4_kv_cache* cache, int32_t slot, const void* k_bf16,
                             const void* v_bf16, void* workspace, size_t ws_bytes, nvfp4_stream_t stream);

/* nvfp4_kv_append with the keys' rotary position embedding fused ahead of
 * their quantize ([NEWS]: fused RoPE and the in-place KV update).  rope_cos,
 * rope_sin: device binary32 [T][d/2], row t the token's cos / sin per pair,
 * 16-byte aligned, read only.  In every head of token t, pair p (channels 2p
 * and 2p+1, interleaved) becomes, with c = rope_cos[t][p], s = rope_sin[t][p]:
 *   y[2p]   = fl32(fl32(x[2p] * c) - fl32(x[2p+1] * s))
 *   y[2p+1] = fl32(fl32(x[2p] * s) + fl32(x[2p+1] * c))
 * and the slot holds the quantize of y (binary32, never rounded to bf16):
 * tensor scale from max |y|, and with NVFP4_KV_SMOOTH_K the channel means of y
 * (the cache's dequant then returns the turned keys).  V is stored as by
 * nvfp4_kv_append.  Angles (positions, 1D or 3D frequency bands) are the
 * caller's.  T*H*d <= 2^30 as for nvfp4_kv_append; NULL tables:
 * NVFP4_ERR_INVALID_ARG.
 * Same workspace and launches as nvfp4_kv_append. */
nvfp4_status nvfp4_kv_append_rope(const nvfp4_kv_cache* cache, int32_t slot, const void* k_bf16,
                                  const void* v_bf16, const float* rope_cos, const float* rope_sin,
                                  void* workspace, size_t ws_bytes, nvfp4_stream_t stream);

/* Gathers the n slots listed in slots_dev (device int32 [n], values in
 * [0, n_slots)) back to bf16: output i covers rows i*T*H .. of k_out / v_out
 * (bf16 [n][T][H][d]).  Each value is bf16_rne(fl32(fl32(e2m1 * s) * a32))
 * (plus the channel mean before the bf16 rounding for a smoothed tensor).
 * An out-of-range slot index records NVFP4_ERR_DEVICE (info = list position)
 * in the workspace and leaves that output chunk unwritten.
 * workspace: nvfp4_workspace_bytes(NVFP4_OP_KV_DEQUANT, 0, 0, 0) bytes. */
nvfp4_status nvfp4_kv_dequant(const nvfp4_kv_cache* cache, const int32_t* slots_dev, int32_t n, void* k_out_bf16,
                              void* v_out_bf16, void* workspace, size_t ws_bytes, nvfp4_stream_t stream);


/* Attention over the cache [RN-I, RN multi-shot anchors].  The chunk set of
 * step t: A_g (the first sink_global chunks) | A_s (the current shot's first
 * sink_shot chunks; the shot starts at chunk shot_start) | KV[t - window, t),
 * without repeats, only chunks < t, ascending, written to the host array out
 * (at most max_out).  Returns the count, or -1 on a negative argument or a
 * full array.  Host only; mapping chunks to slots is the caller's page table. */
int32_t nvfp4_attention_chunks(int32_t t, int32_t sink_global, int32_t shot_start, int32_t sink_shot,
                               int32_t window, int32_t* out, int32_t max_out);

/* O = softmax(scale * Q K^T) V over every key of the n slots listed in
 * slots_dev (device int32, values in [0, n_slots)), reading K and V from the
 * cache directly, no mask inside the set.  For a cache without smoothing the
 * keys and values are the exact e2m1 * s * a32 (tiles of e2m1 * s in binary16,
 * the slot's a32 applied to the products); with K- or V-smoothing they are the
 * cache's bf16 dequant with the means added (bf16 tiles).  q_bf16 and o_bf16
 * are bf16 [tq][heads][head_dim] (token-major like the cache's chunks); scale
 * = 0 means 1 / sqrt(head_dim).  head_dim must be 128, n * ceil(T / 128) < 2^31
 * and ceil(tq / 256) * heads < 2^31 (else NVFP4_ERR_UNSUPPORTED).  Products on the tensor cores with
 * binary32 accumulation, a one-pass softmax in binary32 against a reference
 * maximum per query row: a row whose weights in a 128-key tile would sum
 * above 2^15 (always the first tile) takes the tile's largest score, and the
 * reference moves to it when it exceeds the reference by more than 2^8 (O
 * rescaled in TMEM then); P rounded to the tiles' 16-bit type.  One launch of
 * min(ceil(tq / 256) x heads, SMs) persistent CTAs, each taking one head and
 * two 128-query tiles at a time.  An out-of-range slot records NVFP4_ERR_DEVICE
 * (info = list position) and is skipped; a wait that runs out records
 * NVFP4_ERR_TIMEOUT (info = which wait) and leaves O incomplete.  workspace:
 * nvfp4_workspace_bytes(NVFP4_OP_KV_ATTENTION, 0, 0, 0) bytes; its bytes
 * 16..19 (a uint32 after the error record) count the rescales of O, one per
 * warp and key tile in which a row's reference maximum moved after the first
 * tile (a diagnostic: each call adds to it, the caller clears it). */
nvfp4_status nvfp4_kv_attention(const nvfp4_kv_cache* cache, const int32_t* slots_dev, int32_t n, const void* q_bf16,
                                int32_t tq, float scale, void* o_bf16, void* workspace, size_t ws_bytes,
                                nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Training-side operands  [RN-T] "NVFP4 训练的工程细节"                        */
/* ------------------------------------------------------------------------ */
/* 2D block scaling of a weight x (bf16 [rows x cols], row stride ld elements;
 * rows % 64 == 0, cols % 64 == 0, both <= 2^30): one E4M3 scale per 16 x 16 block,
 * s = E4M3_rne_sat(amax_block / (6 * a32)), every element encoded with it as
 * in nvfp4_quantize (a32 = amax / 2688 over the tensor, or given with
 * NVFP4_Q_GIVEN_GLOBAL).  Writes the GEMM operand of x (codes [rows x cols/2],
 * swizzled scales of [rows x cols/16], each row holding its block's scale)
 * and/or the operand of x^T (codes_t [cols x rows/2], swizzled scales_t of
 * [cols x rows/16]): the same codes and scales, transposed (pass NULL for a
 * pair not wanted, not both).  Two launches (amax, encode); workspace:
 * nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE_2D, rows, 0, cols) bytes. */
nvfp4_status nvfp4_quantize_2d(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld, void* codes,
                               void* scales, void* codes_t, void* scales_t, float* global_scale, unsigned flags,
                               void* workspace, size_t ws_bytes, nvfp4_stream_t stream);

/* The operand of a GEMM that contracts over x's rows (the weight gradient
 * dW = dY^T X contracts over tokens): x^T [cols x rows] quantized with 1D
 * blocks of 16 along the rows of x (codes_t [cols x rows/2], swizzled
 * scales_t of [cols x rows/16]).  With rht_sign (host array of 16 int8 values,
 * each +1 or -1; NULL: no transform), each 16-element block along the rows
 * first goes through the Random Hadamard Transform y = (1/4) H_16 diag(sign) v
 * in binary32 (signs, then butterflies h = 1, 2, 4, 8 with (a + b, a - b),
 * then * 0.25), and a32 comes from max |y|.  Use the same signs for both
 * operands of the product so the transform cancels.  rows % 64 == 0,
 * cols % 16 == 0, both <= 2^30.  Two launches; workspace:
 * nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE_T, rows, 0, cols) bytes. */
nvfp4_status nvfp4_quantize_t(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld, void* codes_t,
                              void* scales_t, float* global_scale, const int8_t* rht_sign, unsigned flags,
                              void* workspace, size_t ws_bytes, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Test support                                                              */
/* ------------------------------------------------------------------------ */
/* Runs the device encoders used by every kernel above on n arbitrary
 * binary32 inputs: e2m1_out[i] = E2M1 code of x[i] (nearest-even, saturating
 * at 6, sign kept), e4m3_out[i] = E4M3 code of x[i] (nearest-even, saturating
 * at 448; meant for x >= 0).  Either output may be NULL.  Lets a test sweep
 * all 2^32 inputs against the CPU definition.  One launch. */
nvfp4_status nvfp4_test_encode(const float* x, int64_t n, uint8_t* e2m1_out, uint8_t* e4m3_out,
                               nvfp4_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
