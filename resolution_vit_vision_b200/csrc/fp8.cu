// fp8.cu -- E4M3 quantisation for the fp8 tower ("Qwen2-VL-2B-Instruct -- LiteRT-LM", file table:
// the vision tower ships with 8-bit weights; the pages fix no scheme):
//   * quantize_rows_kernel: bf16 rows -> E4M3 codes and one power-of-two scale per row (weights
//     once per output channel; at run time the inputs of the out-proj and fc2 products)
//   * layernorm_fp8_kernel: the LayerNorm of the tower, its output row quantised the same way
//     (the inputs of the QKV and fc1 products)
// A row with max |x| = a > 0 gets the scale 2^e, e the smallest integer with a <= 448 * 2^e (448:
// the largest finite E4M3 value), found from the bits of a: a = M 2^E, M in [1, 2), 448 =
// 1.75 * 2^8, so e = E - 8, plus one when M > 1.75; e is kept >= -126 so that 2^e and 2^-e are
// normal floats (a row whose max is below 448 * 2^-126, an all-zero row included, gets 2^-126).
// Codes are x * 2^-e, an exact product, rounded to the nearest E4M3 value (ties to even) by
// cvt.rn.satfinite.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace vitk {

__device__ __forceinline__ int fp8_scale_exp(float amax) {
    const uint32_t b = __float_as_uint(amax);
    const int field = static_cast<int>((b >> 23) & 0xFF);
    if (field == 0) return -126;                            // zero or below 2^-126
    const int e = field - 127 - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    return max(e, -126);
}
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float(static_cast<uint32_t>(e + 127) << 23); }

// two floats -> two E4M3 codes (lo in the low byte)
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
    return e4m3x2(a, b) | (e4m3x2(c, d) << 16);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_add(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

constexpr int kQWarps = 8;

// One warp per row of `cols` bf16 values (cols a multiple of 8), eight values per lane per step.
// CH > 0: the row is CH * 256 values wide and stays in registers between the max and the codes
// (one read of the row); CH == 0: any width, the row is read twice (the second time mostly from
// L1 or L2).
template <int CH>
__global__ void __launch_bounds__(kQWarps * 32)
    quantize_rows_kernel(const __nv_bfloat16 *__restrict__ x, int64_t rows, int cols, uint8_t *__restrict__ codes,
                         float *__restrict__ scales) {
    pdl_wait();                                   // the rows are the previous kernel's output
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kQWarps + warp;
    if (row >= rows) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + row * cols);
    uint2 *dst = reinterpret_cast<uint2 *>(codes + row * cols);
    float amax = 0.f;
    if (CH > 0) {
        uint4 u[CH > 0 ? CH : 1];
#pragma unroll
        for (int i = 0; i < CH; ++i) u[i] = __ldcs(src + lane + 32 * i);
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
        }
        const int e = fp8_scale_exp(warp_max(amax));
        const float inv = exp2i(-e);
#pragma unroll
        for (int i = 0; i < CH; ++i)
            dst[lane + 32 * i] =
                make_uint2(e4m3x4(bf16_lo(u[i].x) * inv, bf16_hi(u[i].x) * inv, bf16_lo(u[i].y) * inv, bf16_hi(u[i].y) * inv),
                           e4m3x4(bf16_lo(u[i].z) * inv, bf16_hi(u[i].z) * inv, bf16_lo(u[i].w) * inv, bf16_hi(u[i].w) * inv));
        if (lane == 0) scales[row] = exp2i(e);
        return;
    }
    const int n8 = cols >> 3;
    for (int c = lane; c < n8; c += 32) {
        const uint4 u = src[c];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
    }
    const int e = fp8_scale_exp(warp_max(amax));
    const float inv = exp2i(-e);
    for (int c = lane; c < n8; c += 32) {
        const uint4 u = src[c];
        dst[c] = make_uint2(e4m3x4(bf16_lo(u.x) * inv, bf16_hi(u.x) * inv, bf16_lo(u.y) * inv, bf16_hi(u.y) * inv),
                            e4m3x4(bf16_lo(u.z) * inv, bf16_hi(u.z) * inv, bf16_lo(u.w) * inv, bf16_hi(u.w) * inv));
    }
    if (lane == 0) scales[row] = exp2i(e);
}

// LayerNorm of a 1280-wide fp32 row (as layernorm_kernel: two-pass mean / variance, the row in
// registers), then the normalised row quantised: codes [rows, 1280], scales [rows].
constexpr int kLnWarps8 = 8;
__global__ void __launch_bounds__(kLnWarps8 * 32)
    layernorm_fp8_kernel(const float *__restrict__ X, const __nv_bfloat16 *__restrict__ gamma,
                         const __nv_bfloat16 *__restrict__ beta, uint8_t *__restrict__ codes,
                         float *__restrict__ scales, int64_t rows, float eps) {
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kLnWarps8 + warp;
    if (row >= rows) return;
    const float4 *x4 = reinterpret_cast<const float4 *>(X + row * VIT_WIDTH);
    float4 v[10];
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 10; ++i) {
        v[i] = __ldcs(x4 + lane + 32 * i);
        s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
    }
    const float mean = warp_add(s) * (1.0f / VIT_WIDTH);
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < 10; ++i) {
        const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
        q += (a * a + b * b) + (c * c + d * d);
    }
    const float rstd = rsqrtf(warp_add(q) * (1.0f / VIT_WIDTH) + eps);
    const uint2 *g2 = reinterpret_cast<const uint2 *>(gamma);
    const uint2 *b2 = reinterpret_cast<const uint2 *>(beta);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 10; ++i) {
        const int c4 = lane + 32 * i;
        const uint2 g = __ldg(g2 + c4);
        v[i].x = (v[i].x - mean) * rstd * bf16_lo(g.x);
        v[i].y = (v[i].y - mean) * rstd * bf16_hi(g.x);
        v[i].z = (v[i].z - mean) * rstd * bf16_lo(g.y);
        v[i].w = (v[i].w - mean) * rstd * bf16_hi(g.y);
        if (beta) {
            const uint2 b = __ldg(b2 + c4);
            v[i].x += bf16_lo(b.x); v[i].y += bf16_hi(b.x); v[i].z += bf16_lo(b.y); v[i].w += bf16_hi(b.y);
        }
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
    }
    const int e = fp8_scale_exp(warp_max(amax));
    const float inv = exp2i(-e);
    uint32_t *dst = reinterpret_cast<uint32_t *>(codes + row * VIT_WIDTH);
#pragma unroll
    for (int i = 0; i < 10; ++i)
        dst[lane + 32 * i] = e4m3x4(v[i].x * inv, v[i].y * inv, v[i].z * inv, v[i].w * inv);
    if (lane == 0) scales[row] = exp2i(e);
}

}  // namespace vitk

namespace vith {

int quantize_rows_launch(const void *x, int64_t rows, int cols, void *codes, float *scales, cudaStream_t s) {
    if (rows <= 0) return VIT_OK;
    const int64_t blocks = (rows + vitk::kQWarps - 1) / vitk::kQWarps;
    const auto *xb = static_cast<const __nv_bfloat16 *>(x);
    auto *cb = static_cast<uint8_t *>(codes);
    const dim3 grid(static_cast<unsigned>(blocks)), block(vitk::kQWarps * 32);
    // the widths of the tower's product inputs keep their rows in registers (one read)
    auto *k = cols == VIT_MLP     ? vitk::quantize_rows_kernel<VIT_MLP / 256>
              : cols == VIT_WIDTH ? vitk::quantize_rows_kernel<VIT_WIDTH / 256>
                                  : vitk::quantize_rows_kernel<0>;
    if (launch_pdl(k, grid, block, 0, s, 1, xb, rows, cols, cb, scales) != cudaSuccess) return VIT_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}

int layernorm_fp8_launch(const float *X, const void *gamma, const void *beta, void *codes, float *scales,
                         int64_t rows, float eps, cudaStream_t s) {
    if (rows <= 0) return VIT_OK;
    const int64_t blocks = (rows + vitk::kLnWarps8 - 1) / vitk::kLnWarps8;
    if (launch_pdl(vitk::layernorm_fp8_kernel, dim3(static_cast<unsigned>(blocks)), dim3(vitk::kLnWarps8 * 32), 0, s,
                   1, X, static_cast<const __nv_bfloat16 *>(gamma), static_cast<const __nv_bfloat16 *>(beta),
                   static_cast<uint8_t *>(codes), scales, rows, eps) != cudaSuccess)
        return VIT_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}

}  // namespace vith
