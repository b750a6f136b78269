// Training-side NVFP4 operands ("NVFP4 训练的工程细节" in the LongLive-2.0
// reading note): weights with 2D block scaling (one E4M3 scale per 16 x 16
// block, so W and W^T share codes and scales), and the operands of the
// weight-gradient GEMM, which contracts over tokens: x^T quantized with 1D
// blocks along the tokens, after a 16-point Random Hadamard Transform.
//
// Both run as two launches on the caller's stream: an amax pass (the tensor
// scale a32 = amax / 2688 needs the whole tensor) and an encode pass.  A warp
// owns a 32-row x 64-column tile of x (rows % 64 == 0): lane l holds columns
// 2l and 2l + 1 of the tile for all 32 rows (32 four-byte loads, each warp
// load 128 contiguous bytes), so a 16-element block along the rows is one
// lane's register column and a 16 x 16 block is eight lanes.  Per column the
// lane writes the transposed operand's 16 code bytes (one 16-byte store) and
// its 2 scale bytes (one 2-byte store into the swizzled tile); the 2D mode
// also writes the row-wise operand (a byte per row and lane, 32 contiguous
// bytes per warp store) and its scales.  The grid is one resident wave.
#include <algorithm>
#include <cstdint>

#include "common.cuh"

namespace nvfp4 {
namespace train {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTileRows = 32;

struct TrainArgs {
    const uint8_t* x;      // bf16 [rows][ld]
    int64_t ld;            // elements
    int rows, cols;
    uint8_t* codes;        // 2D: row-wise operand [rows][cols/2] (NULL: not written)
    uint8_t* scales;       //     swizzled [rows x cols/16]
    uint8_t* codes_t;      // transposed operand [cols][rows/2] (NULL: not written)
    uint8_t* scales_t;     //     swizzled [cols x rows/16]
    float* gscale;         // a32 out (COMPUTE) or in (GIVEN)
    int given;
    uint32_t* amax_word;   // workspace word: max |value| as binary32 bits
    uint32_t sign_mask;    // RHT: bit i set -> sign_i = -1
    int tiles_c, ntiles;
    DevError* err;
};

// Two binary32 -> two E2M1 codes in the low byte: lo -> bits 3:0, hi -> 7:4.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
    uint16_t out;
    asm("{\n\t.reg .b8 b;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b, %2, %1;\n\t"
        "cvt.u16.u8 %0, b;\n\t}"
        : "=h"(out)
        : "f"(lo), "f"(hi));
    return out;
}

// The 16-point Random Hadamard Transform of a block, binary32: the signs
// (exact), butterflies h = 1, 2, 4, 8 with (a + b, a - b), then * 0.25 (the
// 1 / sqrt(16) normalisation): y = (1/4) H_16 diag(sign) v, H_16 the
// Sylvester Hadamard matrix.
// The same transform on two blocks at once (columns c and c + 1 of a lane):
// element i of both blocks in one 64-bit pair, the packed binary32 add, sub
// and multiply rounding each lane as the scalar operation does.  The signs
// are applied by the caller (on the packed bf16 words, exact), and SCALE =
// false leaves out the final * 0.25, which the amax pass applies to its
// maximum instead (exact: rounding is monotone, so it commutes with max).
__device__ __forceinline__ uint64_t pk(float lo, float hi) {
    return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
template <bool SCALE>
__device__ __forceinline__ void rht16x2(float* f0, float* f1) {
    uint64_t v[16];
#pragma unroll
    for (int i = 0; i < 16; i++) v[i] = pk(f0[i], f1[i]);
#pragma unroll
    for (int h = 1; h < 16; h <<= 1)
#pragma unroll
        for (int i = 0; i < 16; i++)
            if ((i & h) == 0) {
                const uint64_t a = v[i], b = v[i + h];
                asm("add.rn.f32x2 %0, %1, %2;" : "=l"(v[i]) : "l"(a), "l"(b));
                asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(v[i + h]) : "l"(a), "l"(b));
            }
    const uint64_t q = pk(0.25f, 0.25f);
#pragma unroll
    for (int i = 0; i < 16; i++) {
        uint64_t r = v[i];
        if (SCALE) asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(v[i]), "l"(q));
        f0[i] = __uint_as_float((uint32_t)r);
        f1[i] = __uint_as_float((uint32_t)(r >> 32));
    }
}

__device__ __forceinline__ float absmax16(const float* f) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; i++) m = fmaxf(m, fabsf(f[i]));
    return m;
}

// E4M3 scale code of a block (R3) and its reciprocal 1 / (s * a32) (R5; 0
// when the block is flushed or a32 == 0).
__device__ __forceinline__ uint32_t block_code(float amax_b, float d6) {
    return d6 == 0.0f ? 0u : e4m3_code(__fdiv_rn(amax_b, d6));
}
__device__ __forceinline__ float block_inv(uint32_t code, float a32) {
    const float s = e4m3_value(code);
    return (s == 0.0f || a32 == 0.0f) ? 0.0f : __frcp_rn(__fmul_rn(s, a32));
}

// TWO_D: 16 x 16 blocks, both operands.  Otherwise the transposed operand
// with 1D blocks along the rows (RHT: after the transform).  ENCODE = false
// is the amax pass.
template <bool TWO_D, bool RHT, bool ENCODE>
__global__ void __launch_bounds__(kThreads, (RHT && ENCODE) ? 2 : 3) train_quant_kernel(const __grid_constant__ TrainArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;
    float a32 = 0.0f, d6 = 0.0f;
    if (ENCODE) {
        a32 = a.given ? *a.gscale : __fdiv_rn(__uint_as_float(*(volatile uint32_t*)a.amax_word), 2688.0f);
        d6 = __fmul_rn(6.0f, a32);
        if (!a.given && blockIdx.x == 0 && threadIdx.x == 0) *a.gscale = a32;
    }
    float lane_max = 0.0f;
    const int64_t code_ld_t = a.rows / 2;           // bytes per row of x^T's codes
    const int64_t tiles_c_t = a.rows / 64;          // 128 x 4 scale tiles per 128 rows of x^T
    const int64_t tiles_c_r = a.cols / 64;          // row-wise operand (2D)
    for (int64_t t = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); t < a.ntiles; t += nwarps) {
        const int tr = (int)(t / a.tiles_c), tc = (int)(t - (int64_t)tr * a.tiles_c);
        const int r0 = tr * kTileRows, c = tc * 64 + 2 * lane;
        const bool active = c < a.cols;  // cols % 16 == 0: whole 8-lane groups
        uint32_t v[kTileRows];
        const uint8_t* src = a.x + ((int64_t)r0 * a.ld + c) * 2;
#pragma unroll
        for (int i = 0; i < kTileRows; i++)
            v[i] = active ? __ldg(reinterpret_cast<const uint32_t*>(src + (int64_t)i * a.ld * 2)) : 0u;
        uint32_t ct[2][4];  // transposed codes of the two columns: 32 rows -> 4 words each
        uint32_t st[2] = {0u, 0u};
#pragma unroll
        for (int b = 0; b < kTileRows / 16; b++) {
            float f0[16], f1[16];
#pragma unroll
            for (int i = 0; i < 16; i++) {
                // RHT signs on the packed bf16 pair (both columns share row i's sign)
                const uint32_t w = RHT ? v[16 * b + i] ^ (((a.sign_mask >> i) & 1u) * 0x80008000u) : v[16 * b + i];
                f0[i] = __uint_as_float(w << 16);
                f1[i] = __uint_as_float(w & 0xFFFF0000u);
            }
            if (RHT) rht16x2<ENCODE>(f0, f1);
            const float m0 = absmax16(f0), m1 = absmax16(f1);
            if (!ENCODE) {
                lane_max = fmaxf(lane_max, fmaxf(m0, m1));
                continue;
            }
            uint32_t code0, code1;
            if (TWO_D) {
                // the 16 x 16 block is 8 lanes x 2 columns x these 16 rows
                float m = fmaxf(m0, m1);
#pragma unroll
                for (int o = 1; o < 8; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
                code0 = code1 = block_code(m, d6);
            } else {
                code0 = block_code(m0, d6);
                code1 = block_code(m1, d6);
            }
            const float inv0 = block_inv(code0, a32), inv1 = block_inv(code1, a32);
            float y0[16], y1[16];
            const uint64_t inv2 = pk(inv0, inv1);
#pragma unroll
            for (int i = 0; i < 16; i++) {
                uint64_t r;
                asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk(f0[i], f1[i])), "l"(inv2));
                y0[i] = __uint_as_float((uint32_t)r);
                y1[i] = __uint_as_float((uint32_t)(r >> 32));
            }
            ct[0][2 * b] = inv0 == 0.0f ? 0u : e2m1x8(y0);
            ct[0][2 * b + 1] = inv0 == 0.0f ? 0u : e2m1x8(y0 + 8);
            ct[1][2 * b] = inv1 == 0.0f ? 0u : e2m1x8(y1);
            ct[1][2 * b + 1] = inv1 == 0.0f ? 0u : e2m1x8(y1 + 8);
            st[0] |= code0 << (8 * b);
            st[1] |= code1 << (8 * b);
            if (TWO_D && a.codes && active) {
                // row-wise operand: one byte per row (columns c, c + 1), and
                // the block's scale on each of its 16 rows
                uint8_t* crow = a.codes + (int64_t)(r0 + 16 * b) * (a.cols / 2) + c / 2;
#pragma unroll
                for (int i = 0; i < 16; i++)
                    crow[(int64_t)i * (a.cols / 2)] = (uint8_t)(inv0 == 0.0f ? 0u : e2m1x2(y0[i], y1[i]));
                const int k = lane & 7;
#pragma unroll
                for (int j = 0; j < 2; j++) {
                    const int64_t r = r0 + 16 * b + 2 * k + j;
                    a.scales[swz_offset(r, c / 16, tiles_c_r)] = (uint8_t)code0;
                }
            }
        }
        if (ENCODE && a.codes_t && active) {
#pragma unroll
            for (int j = 0; j < 2; j++) {
                uint8_t* dst = a.codes_t + (int64_t)(c + j) * code_ld_t + r0 / 2;
                *reinterpret_cast<uint4*>(dst) = make_uint4(ct[j][0], ct[j][1], ct[j][2], ct[j][3]);
                // scale columns r0/16 and r0/16 + 1 of row c + j: 2 contiguous
                // bytes (r0/16 is even, so they share a 4-byte group)
                *reinterpret_cast<uint16_t*>(a.scales_t + swz_offset(c + j, r0 / 16, tiles_c_t)) = (uint16_t)st[j];
            }
        }
    }
    if (!ENCODE) {
        if (RHT) lane_max = __fmul_rn(lane_max, 0.25f);  // the transform's normalisation, left out above
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lane_max = fmaxf(lane_max, __shfl_xor_sync(0xFFFFFFFFu, lane_max, o));
        if (lane == 0 && lane_max > 0.0f) atomicMax(a.amax_word, __float_as_uint(lane_max));
    }
}

}  // namespace train
}  // namespace nvfp4

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

using namespace nvfp4;
using namespace nvfp4::train;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PerDevice<int> g_train_sms;

// SMs of the current device (148 on B200 if the query fails)
int sm_count() {
    int n = 0;
    const nvfp4_status st = g_train_sms.get(&n, [](int dev, int& v) {
        return cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? NVFP4_OK
                                                                                               : NVFP4_ERR_CUDA;
    });
    return st == NVFP4_OK && n > 0 ? n : 148;
}

struct TrainResidency {
    int blocks[2];  // resident blocks per SM of the amax pass and of the encode pass
};

// Zero a swizzled scale buffer when its layout has padding rows (rows not a
// multiple of 128): the kernels write only real rows.
nvfp4_status zero_padding(uint8_t* scales, int64_t rows, int64_t sc, cudaStream_t s) {
    if (rows % 128 == 0) return NVFP4_OK;
    const size_t bytes = (size_t)((rows + 127) / 128 * 128) * (size_t)((sc + 3) / 4 * 4);
    return cudaMemsetAsync(scales, 0, bytes, s) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

template <bool TWO_D, bool RHT>
nvfp4_status run(TrainArgs& a, cudaStream_t s) {
    a.tiles_c = (a.cols + 63) / 64;
    a.ntiles = (a.rows / kTileRows) * a.tiles_c;
    const int64_t want = ((int64_t)a.ntiles + kWarps - 1) / kWarps;
    // one resident wave of each pass (blocks per SM from the occupancy query, per device)
    static PerDevice<TrainResidency> g_resident;
    TrainResidency res{};
    const nvfp4_status rst = g_resident.get(&res, [](int, TrainResidency& v) {
        for (int e = 0; e < 2; e++) {
            int b = 0;
            auto k = e ? train_quant_kernel<TWO_D, RHT, true> : train_quant_kernel<TWO_D, RHT, false>;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, k, kThreads, 0) != cudaSuccess || b < 1) {
                cudaGetLastError();
                b = 1;
            }
            v.blocks[e] = b;
        }
        return NVFP4_OK;
    });
    if (rst != NVFP4_OK) return rst;
    const int* resident = res.blocks;
    if (!a.given) {
        if (cudaMemsetAsync(a.amax_word, 0, 4, s) != cudaSuccess) return NVFP4_ERR_CUDA;
        const int g = (int)std::min<int64_t>(want, (int64_t)sm_count() * resident[0]);
        train_quant_kernel<TWO_D, RHT, false><<<g, kThreads, 0, s>>>(a);
        if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
    }
    const int g = (int)std::min<int64_t>(want, (int64_t)sm_count() * resident[1]);
    train_quant_kernel<TWO_D, RHT, true><<<g, kThreads, 0, s>>>(a);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

nvfp4_status common_checks(const void* x, int64_t rows, int64_t cols, int64_t ld, const float* gscale, unsigned flags,
                           const void* ws, size_t ws_bytes, int op) {
    if (flags & ~NVFP4_Q_GIVEN_GLOBAL) return NVFP4_ERR_INVALID_ARG;
    if (rows < 0 || cols <= 0 || ld < cols || !gscale || !ws) return NVFP4_ERR_INVALID_ARG;
    if (ws_bytes < nvfp4_workspace_bytes(op, rows, 0, cols)) return NVFP4_ERR_INVALID_ARG;
    if (rows % 64 != 0 || cols % 16 != 0 || rows > ((int64_t)1 << 30) || cols > ((int64_t)1 << 30))
        return NVFP4_ERR_UNSUPPORTED;
    if (rows > 0 && !x) return NVFP4_ERR_INVALID_ARG;
    if ((x && !aligned16(x)) || ld % 8 != 0 || (reinterpret_cast<uintptr_t>(gscale) & 3u) ||
        (reinterpret_cast<uintptr_t>(ws) & 255u))
        return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status nvfp4_quantize_2d(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld, void* codes,
                                          void* scales, void* codes_t, void* scales_t, float* global_scale,
                                          unsigned flags, void* workspace, size_t ws_bytes, nvfp4_stream_t stream) {
    nvfp4_status st = common_checks(x_bf16, rows, cols, ld, global_scale, flags, workspace, ws_bytes,
                                    NVFP4_OP_QUANTIZE_2D);
    if (st != NVFP4_OK) return st;
    if (cols % 64 != 0) return NVFP4_ERR_UNSUPPORTED;
    if ((codes == nullptr) != (scales == nullptr) || (codes_t == nullptr) != (scales_t == nullptr) ||
        (!codes && !codes_t))
        return NVFP4_ERR_INVALID_ARG;
    if ((codes && (!aligned16(codes) || !aligned16(scales))) || (codes_t && (!aligned16(codes_t) || !aligned16(scales_t))))
        return NVFP4_ERR_MISALIGNED;
    if (rows == 0) return NVFP4_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (codes && (st = zero_padding(static_cast<uint8_t*>(scales), rows, cols / 16, s)) != NVFP4_OK) return st;
    if (codes_t && (st = zero_padding(static_cast<uint8_t*>(scales_t), cols, rows / 16, s)) != NVFP4_OK) return st;
    TrainArgs a{};
    a.x = static_cast<const uint8_t*>(x_bf16);
    a.ld = ld;
    a.rows = (int)rows;
    a.cols = (int)cols;
    a.codes = static_cast<uint8_t*>(codes);
    a.scales = static_cast<uint8_t*>(scales);
    a.codes_t = static_cast<uint8_t*>(codes_t);
    a.scales_t = static_cast<uint8_t*>(scales_t);
    a.gscale = global_scale;
    a.given = (flags & NVFP4_Q_GIVEN_GLOBAL) ? 1 : 0;
    a.amax_word = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + 128);
    a.err = static_cast<DevError*>(workspace);
    return run<true, false>(a, s);
}

extern "C" nvfp4_status nvfp4_quantize_t(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld, void* codes_t,
                                         void* scales_t, float* global_scale, const int8_t* rht_sign, unsigned flags,
                                         void* workspace, size_t ws_bytes, nvfp4_stream_t stream) {
    nvfp4_status st = common_checks(x_bf16, rows, cols, ld, global_scale, flags, workspace, ws_bytes,
                                    NVFP4_OP_QUANTIZE_T);
    if (st != NVFP4_OK) return st;
    if (!codes_t || !scales_t) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(codes_t) || !aligned16(scales_t)) return NVFP4_ERR_MISALIGNED;
    uint32_t mask = 0;
    if (rht_sign)
        for (int i = 0; i < 16; i++) {
            if (rht_sign[i] != 1 && rht_sign[i] != -1) return NVFP4_ERR_INVALID_ARG;
            mask |= (rht_sign[i] < 0 ? 1u : 0u) << i;
        }
    if (rows == 0) return NVFP4_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if ((st = zero_padding(static_cast<uint8_t*>(scales_t), cols, rows / 16, s)) != NVFP4_OK) return st;
    TrainArgs a{};
    a.x = static_cast<const uint8_t*>(x_bf16);
    a.ld = ld;
    a.rows = (int)rows;
    a.cols = (int)cols;
    a.codes_t = static_cast<uint8_t*>(codes_t);
    a.scales_t = static_cast<uint8_t*>(scales_t);
    a.gscale = global_scale;
    a.given = (flags & NVFP4_Q_GIVEN_GLOBAL) ? 1 : 0;
    a.amax_word = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + 128);
    a.sign_mask = mask;
    a.err = static_cast<DevError*>(workspace);
    return rht_sign ? run<false, true>(a, s) : run<false, false>(a, s);
}
