// misc.cu -- the HBM-bound and integer kernels of the path:
//   * LayerNorm rows of 1280 (fp32 residual in, bf16 out, optional row scatter for the merger)
//   * the 2-D rope cos/sin table and the per-patch (row, column) positions
//   * the decoder's 3-D M-RoPE position ids
#include <cuda_bf16.h>

#include <cmath>
#include <memory>

#include "internal.h"
#include "ptx.cuh"

namespace vitk {

// ------------------------------------------------------------------------------ LayerNorm
// "Qwen2-VL (Native-Resolution VLM)", Structure table (pre-norm ViT blocks) and the exported
// PatchMerger's nn.LayerNorm: y = (x - mean) / sqrt(var + eps) * gamma + beta over 1280
// features, biased variance. One warp per row, the row held in registers (two passes).
constexpr int kLnWarps = 8;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void __launch_bounds__(kLnWarps * 32)
    layernorm_kernel(const float *__restrict__ X, const __nv_bfloat16 *__restrict__ gamma,
                     const __nv_bfloat16 *__restrict__ beta, __nv_bfloat16 *__restrict__ Y, int64_t rows, float eps,
                     const int32_t *__restrict__ out_row) {
    pdl_wait();                                   // the rows are the previous kernel's output
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kLnWarps + warp;
    if (row >= rows) return;
    const float4 *x4 = reinterpret_cast<const float4 *>(X + row * VIT_WIDTH);
    float4 v[10];
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 10; ++i) {
        v[i] = __ldcs(x4 + lane + 32 * i);
        s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
    }
    const float mean = warp_sum(s) * (1.0f / VIT_WIDTH);
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < 10; ++i) {
        const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
        q += (a * a + b * b) + (c * c + d * d);
    }
    const float rstd = rsqrtf(warp_sum(q) * (1.0f / VIT_WIDTH) + eps);
    const int64_t orow = out_row ? static_cast<int64_t>(out_row[row]) : row;
    uint2 *y2 = reinterpret_cast<uint2 *>(Y + orow * VIT_WIDTH);
    const uint2 *g2 = reinterpret_cast<const uint2 *>(gamma);
    const uint2 *b2 = reinterpret_cast<const uint2 *>(beta);
#pragma unroll
    for (int i = 0; i < 10; ++i) {
        const int c4 = lane + 32 * i;
        const uint2 g = __ldg(g2 + c4);
        float o0 = (v[i].x - mean) * rstd * bf16_lo(g.x);
        float o1 = (v[i].y - mean) * rstd * bf16_hi(g.x);
        float o2 = (v[i].z - mean) * rstd * bf16_lo(g.y);
        float o3 = (v[i].w - mean) * rstd * bf16_hi(g.y);
        if (beta) {
            const uint2 b = __ldg(b2 + c4);
            o0 += bf16_lo(b.x); o1 += bf16_hi(b.x); o2 += bf16_lo(b.y); o3 += bf16_hi(b.y);
        }
        y2[c4] = make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
    }
}

// ------------------------------------------------------------------------------ 2-D rope
// cs[p][k] = (cos(p f_k), sin(p f_k)), f_k = 10000^(-2k/40), k < 20: the 20 frequencies of each
// 40-dim half (row half, column half) of the 80-wide head. Computed in double, stored fp32.
__global__ void rope_table_kernel(float2 *cs, int n_pos) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_pos * 20) return;
    const int p = i / 20, k = i % 20;
    const double f = pow(10000.0, -2.0 * k / 40.0);
    double s, c;
    sincos(static_cast<double>(p) * f, &s, &c);
    cs[i] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

// Packed-image table for the positions kernel (kernel parameter).
struct ImageTable {
    int n;
    int row_start[VIT_MAX_IMAGES];
    int t[VIT_MAX_IMAGES], h[VIT_MAX_IMAGES], w[VIT_MAX_IMAGES];
};

// pos[r] = (h << 16) | w of patch r inside its frame. patch_order 0: per frame the patches run
// (bh, bw, dh, dw), dw fastest, so four consecutive rows are one 2x2 merge group; 1: raster.
// merge_row[r]: the row patch r takes in block order (the merger reads four consecutive rows).
__global__ void positions_kernel(const __grid_constant__ ImageTable tab, int64_t P, int patch_order,
                                 int32_t *__restrict__ pos, int32_t *__restrict__ merge_row) {
    pdl_wait();                                   // the previous encode may still read pos / merge_row
    pdl_trigger();
    const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (r >= P) return;
    int lo = 0, hi = tab.n - 1;   // last image with row_start <= r
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tab.row_start[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int h = tab.h[lo], w = tab.w[lo];
    const int64_t j = r - tab.row_start[lo];
    const int64_t frame_start = tab.row_start[lo] + (j / (h * w)) * (h * w);
    const int jj = static_cast<int>(j % (h * w));
    int hp, wp;
    if (patch_order == 0) {
        const int g = jj >> 2;
        hp = 2 * (g / (w >> 1)) + ((jj >> 1) & 1);
        wp = 2 * (g % (w >> 1)) + (jj & 1);
        if (merge_row) merge_row[r] = static_cast<int32_t>(r);
    } else {
        hp = jj / w;
        wp = jj % w;
        if (merge_row)
            merge_row[r] = static_cast<int32_t>(frame_start + (((hp >> 1) * (w >> 1) + (wp >> 1)) << 2) +
                                                ((hp & 1) << 1) + (wp & 1));
    }
    pos[r] = (hp << 16) | wp;
}

// ------------------------------------------------------------------------------ M-RoPE ids
// "Qwen2-VL": the decoder's rotary positions split across time / height / width
// (mrope_section (16, 24, 24) splits the frequencies, the ids are what this builds);
// "Qwen2-VL-2B-Instruct -- LiteRT-LM", M-RoPE note: text tokens keep 1-D positions.
// Closed form of the cursor rule: with vision runs k = 0.. (start s_k, length n_k, advance
// a_k = max(t, h', w')), a token i outside every run gets i - sum over runs ending at or before
// i of (n_k - a_k); the j-th token of run k gets base_k + (j / h'w', (j / w') % h', j % w') with
// base_k = s_k - sum_{k' < k} (n_k' - a_k'). One CTA: ballot-compacts the runs, prefix-sums the
// shifts, validates every run, then writes every token in parallel.
constexpr int kMropeThreads = 1024;

struct MropeGrids {
    int n;
    int t[VIT_MAX_MROPE_GRIDS], h[VIT_MAX_MROPE_GRIDS], w[VIT_MAX_MROPE_GRIDS];
};

__global__ void __launch_bounds__(kMropeThreads)
    mrope_kernel(const int32_t *__restrict__ ids, int64_t L, const __grid_constant__ MropeGrids g,
                 int32_t *__restrict__ out, int32_t *__restrict__ delta, int32_t *__restrict__ status) {
    __shared__ int s_start[VIT_MAX_MROPE_GRIDS + 1];
    __shared__ int s_len[VIT_MAX_MROPE_GRIDS];
    __shared__ int s_base[VIT_MAX_MROPE_GRIDS];
    __shared__ int s_shift[VIT_MAX_MROPE_GRIDS];   // sum of (n - a) over runs 0..k
    __shared__ int s_hw[VIT_MAX_MROPE_GRIDS];      // (h' << 16) | w'
    __shared__ int s_tok[VIT_MAX_MROPE_GRIDS];
    __shared__ int s_warp[kMropeThreads / 32];
    __shared__ int s_count, s_err;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cap = g.n + 1;   // one more than the grids, to notice a run without a grid
    if (tid == 0) { s_count = 0; s_err = 0; }
    __syncthreads();

    // 1. vision runs, in token order: i + 1 where ids[i] is vision_start and ids[i+1] a placeholder
    for (int64_t base = 0; base < L; base += kMropeThreads) {
        const int64_t i = base + tid;
        bool f = false;
        if (i + 1 < L && ids[i] == VIT_VISION_START_TOKEN_ID) {
            const int nx = ids[i + 1];
            f = (nx == VIT_IMAGE_TOKEN_ID || nx == VIT_VIDEO_TOKEN_ID);
        }
        const unsigned bal = __ballot_sync(0xffffffffu, f);
        if (lane == 0) s_warp[warp] = __popc(bal);
        __syncthreads();
        if (warp == 0) {   // exclusive scan of the 32 warp counts
            int v = s_warp[lane], x = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            s_warp[lane] = x - v;
        }
        __syncthreads();
        const int idx = s_count + s_warp[warp] + __popc(bal & ((1u << lane) - 1u));
        if (f && idx < cap) s_start[idx] = static_cast<int>(i + 1);
        __syncthreads();
        if (tid == kMropeThreads - 1) s_count = idx + (f ? 1 : 0);
        __syncthreads();
    }
    const int n_runs = s_count;

    // 2. per-run sizes and prefix sums (sequential: at most 1024 runs)
    if (tid == 0) {
        if (n_runs > g.n) s_err = 1;
        int shift = 0, prev_end = 0;
        for (int k = 0; k < n_runs && !s_err; ++k) {
            // a grid is checked only when a run consumes it (unused trailing grids are ignored);
            // every factor of a run's length is at most the prompt length, so each is bounded by
            // L before the product is formed
            const int64_t gt = g.t[k], gh = g.h[k], gw = g.w[k];
            if (gt < 1 || gh < 2 || gw < 2 || (gh & 1) || (gw & 1) || gt > L || gh / 2 > L || gw / 2 > L ||
                gt * (gh / 2) > L || gt * (gh / 2) * (gw / 2) > L) {
                s_err = 1;
                break;
            }
            const int hh = static_cast<int>(gh >> 1), ww = static_cast<int>(gw >> 1);
            const int n = static_cast<int>(gt) * hh * ww;
            const int a = max(g.t[k], max(hh, ww));
            const int s = s_start[k];
            if (s < prev_end || static_cast<int64_t>(s) + n > L) { s_err = 1; break; }
            s_len[k] = n;
            s_base[k] = s - shift;
            shift += n - a;
            s_shift[k] = shift;
            s_hw[k] = (hh << 16) | ww;
            s_tok[k] = ids[s];
            prev_end = s + n;
        }
    }
    __syncthreads();

    // 3. every run is exactly n tokens of its placeholder id
    if (!s_err) {
        for (int k = 0; k < n_runs; ++k) {
            const int s = s_start[k], n = s_len[k], tok = s_tok[k];
            for (int j = tid; j <= n; j += kMropeThreads) {
                const int64_t i = static_cast<int64_t>(s) + j;
                if (j < n) {
                    if (ids[i] != tok) s_err = 1;
                } else if (i < L && ids[i] == tok) {
                    s_err = 1;   // run longer than its grid
                }
            }
        }
    }
    __syncthreads();
    if (s_err) {
        if (tid == 0 && status) *status = VIT_ERR_TOKENS;
        return;
    }

    // 4. ids
    for (int64_t i = tid; i < L; i += kMropeThreads) {
        int lo = -1, hi = n_runs - 1;   // last run with start <= i
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_start[mid] <= i) lo = mid; else hi = mid - 1;
        }
        int a0, a1, a2;
        if (lo >= 0 && i < static_cast<int64_t>(s_start[lo]) + s_len[lo]) {
            const int j = static_cast<int>(i - s_start[lo]);
            const int hh = s_hw[lo] >> 16, ww = s_hw[lo] & 0xFFFF;
            const int b = s_base[lo];
            a0 = b + j / (hh * ww);
            a1 = b + (j / ww) % hh;
            a2 = b + j % ww;
        } else {
            a0 = a1 = a2 = static_cast<int>(i) - (lo >= 0 ? s_shift[lo] : 0);
        }
        out[i] = a0;
        out[L + i] = a1;
        out[2 * L + i] = a2;
    }
    if (tid == 0 && delta) *delta = n_runs > 0 ? -s_shift[n_runs - 1] : 0;
}

// ------------------------------------------------------------------------------ wait self-test
// Exercises the bounded-wait path on the GPU without any fault: every thread waits on an
// mbarrier that nothing arrives on. Each wait must give up after `limit` cycles (or as soon as
// another thread has raised the abort flag), write VIT_ERR_TIMEOUT to *status and return, so the
// kernel ends normally and the context stays usable.
__global__ void wait_selftest_kernel(int32_t *status, long long limit) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    WaitCtx wc{&abort_flag, status};
    wc.limit = limit;
    if (mbar_wait(&bar, 0, wc) && status) atomicExch(status, -1);   // a wait with no arrival succeeded
}

}  // namespace vitk

namespace vith {

int wait_selftest_launch(int32_t *status, long long limit, cudaStream_t s) {
    vitk::wait_selftest_kernel<<<1, 64, 0, s>>>(status, limit);
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}


int layernorm_launch(const float *X, const void *gamma, const void *beta, void *Y, int64_t rows, float eps,
                     const int32_t *out_row, cudaStream_t s) {
    if (rows <= 0) return VIT_OK;
    const int64_t blocks = (rows + vitk::kLnWarps - 1) / vitk::kLnWarps;
    if (launch_pdl(vitk::layernorm_kernel, dim3(static_cast<unsigned>(blocks)), dim3(vitk::kLnWarps * 32), 0, s, 1, X,
                   static_cast<const __nv_bfloat16 *>(gamma), static_cast<const __nv_bfloat16 *>(beta),
                   static_cast<__nv_bfloat16 *>(Y), rows, eps, out_row) != cudaSuccess)
        return VIT_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}

int rope_table_launch(float *cs, int n_pos, cudaStream_t s) {
    const int n = n_pos * 20;
    vitk::rope_table_kernel<<<(n + 255) / 256, 256, 0, s>>>(reinterpret_cast<float2 *>(cs), n_pos);
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}

int positions_launch(const int32_t *grid_thw, int n_images, int64_t P, int patch_order, int32_t *pos,
                           int32_t *merge_row, cudaStream_t s) {
    auto tab = std::make_unique<vitk::ImageTable>();
    tab->n = n_images;
    int64_t row = 0;
    for (int i = 0; i < n_images; ++i) {
        tab->row_start[i] = static_cast<int>(row);
        tab->t[i] = grid_thw[3 * i];
        tab->h[i] = grid_thw[3 * i + 1];
        tab->w[i] = grid_thw[3 * i + 2];
        row += static_cast<int64_t>(tab->t[i]) * tab->h[i] * tab->w[i];
    }
    if (P <= 0) return VIT_OK;
    if (launch_pdl(vitk::positions_kernel, dim3(static_cast<unsigned>((P + 255) / 256)), dim3(256), 0, s, 1, *tab, P,
                   patch_order, pos, merge_row) != cudaSuccess)
        return VIT_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}

// positions_launch with the image table on the host stack, for callers that must not allocate.
int positions_launch_stack(const int32_t *grid_thw, int n_images, int64_t P, int patch_order, int32_t *pos,
                           int32_t *merge_row, cudaStream_t s) {
    if (n_images < 0 || n_images > VIT_MAX_IMAGES) return VIT_ERR_LIMIT;
    vitk::ImageTable tab;
    tab.n = n_images;
    int64_t row = 0;
    for (int i = 0; i < n_images; ++i) {
        tab.row_start[i] = static_cast<int>(row);
        tab.t[i] = grid_thw[3 * i];
        tab.h[i] = grid_thw[3 * i + 1];
        tab.w[i] = grid_thw[3 * i + 2];
        row += static_cast<int64_t>(tab.t[i]) * tab.h[i] * tab.w[i];
    }
    if (P <= 0) return VIT_OK;
    if (launch_pdl(vitk::positions_kernel, dim3(static_cast<unsigned>((P + 255) / 256)), dim3(256), 0, s, 1, tab, P,
                   patch_order, pos, merge_row) != cudaSuccess)
        return VIT_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}

int mrope_launch(const int32_t *ids, int64_t L, const int32_t *grid_thw, int n_grids, int32_t *out, int32_t *delta,
                 int32_t *status, cudaStream_t s) {
    auto g = std::make_unique<vitk::MropeGrids>();
    g->n = n_grids;
    for (int i = 0; i < n_grids; ++i) {
        g->t[i] = grid_thw[3 * i];
        g->h[i] = grid_thw[3 * i + 1];
        g->w[i] = grid_thw[3 * i + 2];
    }
    vitk::mrope_kernel<<<1, vitk::kMropeThreads, 0, s>>>(ids, L, *g, out, delta, status);
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}

}  // namespace vith
