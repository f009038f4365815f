// decoder.cu -- the two decoder-side steps that consume the vision encoder's output.
//
// mrope_apply_kernel  3-D M-RoPE rotation of q and k in place ("Qwen2-VL", intro and Qwen2VLModel
//                     table: rope_theta 1e6, mrope_section (16, 24, 24) across time / height /
//                     width; "Qwen2.5-VL-7B-Instruct" record: head_dim 128, 28 / 4 heads). One CTA
//                     per token: its q / k vectors are loaded first, then its D/2 angles
//                     pos[axis(j)] * theta^(-2j/D) are formed and reduced modulo 2 pi in double
//                     precision (positions reach 10^5 and an fp32 angle would be off by ~10^-2
//                     rad), cos / sin of the reduced angle in fp32 into shared memory, and every
//                     head's pairs (j, j + D/2) are turned in fp32 with 16-byte loads and stores.
//                     HBM-bound.
// scatter_kernel      the decoder's input sequence ("Qwen2-VL (Native-Resolution VLM)", Structure
//                     rows 6-10; "Qwen2-VL", several images: each marker expands to its image's
//                     tokens): the k-th image / video placeholder takes merged vision token k, every
//                     other token its embedding row. One CTA per chunk of tokens (8, or more for
//                     long prompts so that at most ~1200 CTAs recount the ids): placeholders before
//                     the chunk counted straight from the ids (no scratch, no inter-CTA waits),
//                     ranks inside the chunk from warp ballots, then the CTA copies the chunk's
//                     rows with 16-byte accesses. HBM-bound.
#include <cuda_bf16.h>

#include <cmath>

#include "internal.h"

namespace vitk {

constexpr int kMaxRopeFreq = 128;   // head_dim <= 256

struct MropeParams {
    int n_freq;                       // head_dim / 2
    int axis_end0, axis_end1;         // frequencies [0, e0) follow t, [e0, e1) h, [e1, n_freq) w
    double inv_freq[kMaxRopeFreq];
};

// Thread t of a token handles 8 consecutive frequencies j0 = 8 (t % (D/16)) of head t / (D/16):
// dims j0..j0+7 and j0+D/2..j0+D/2+7 of that head (two 16-byte vectors).
__device__ __forceinline__ void rotate_pair(uint4 &lo, uint4 &hi, const float *cs, int j0) {
    __nv_bfloat162 *l2 = reinterpret_cast<__nv_bfloat162 *>(&lo);
    __nv_bfloat162 *h2 = reinterpret_cast<__nv_bfloat162 *>(&hi);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 a = __bfloat1622float2(l2[e]), b = __bfloat1622float2(h2[e]);
        const float c0 = cs[2 * (j0 + 2 * e)], s0 = cs[2 * (j0 + 2 * e) + 1];
        const float c1 = cs[2 * (j0 + 2 * e + 1)], s1 = cs[2 * (j0 + 2 * e + 1) + 1];
        l2[e] = __floats2bfloat162_rn(a.x * c0 - b.x * s0, a.y * c1 - b.y * s1);
        h2[e] = __floats2bfloat162_rn(b.x * c0 + a.x * s0, b.y * c1 + a.y * s1);
    }
}

// 128 threads holding two items each: 16 CTAs (4 KB of loads each) in flight per SM
constexpr int kRopeThreads = 128, kRopeHeld = 2;

__global__ void __launch_bounds__(kRopeThreads) mrope_apply_kernel(__nv_bfloat16 *__restrict__ q, int Hq,
                                                                   __nv_bfloat16 *__restrict__ k, int Hk, int D,
                                                                   const int32_t *__restrict__ pos, int64_t L,
                                                                   const __grid_constant__ MropeParams prm) {
    __shared__ float cs[2 * kMaxRopeFreq];
    const int64_t l = blockIdx.x;
    const int per_head = D / 16;
    const int nq = Hq * per_head, n = nq + Hk * per_head;   // work items of this token
    auto addr = [&](int t, bool upper) -> uint4 * {
        const bool is_q = t < nq;
        const int tt = is_q ? t : t - nq;
        __nv_bfloat16 *row = is_q ? q + l * Hq * D : k + l * Hk * D;
        return reinterpret_cast<uint4 *>(row + (tt / per_head) * D + (tt % per_head) * 8 + (upper ? D / 2 : 0));
    };
    // the first items' vectors are in flight while the angles are formed
    uint4 lo[kRopeHeld], hi[kRopeHeld];
#pragma unroll
    for (int i = 0; i < kRopeHeld; ++i) {
        const int t = threadIdx.x + i * kRopeThreads;
        if (t < n) {
            lo[i] = *addr(t, false);
            hi[i] = *addr(t, true);
        }
    }
    for (int j = threadIdx.x; j < prm.n_freq; j += kRopeThreads) {
        const int axis = j < prm.axis_end0 ? 0 : (j < prm.axis_end1 ? 1 : 2);
        const double a = static_cast<double>(pos[axis * L + l]) * prm.inv_freq[j];
        const double r = a - 6.283185307179586476925 * rint(a * 0.159154943091895335768883763);   // |r| <= pi
        float sv, cv;
        sincosf(static_cast<float>(r), &sv, &cv);
        cs[2 * j] = cv;
        cs[2 * j + 1] = sv;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kRopeHeld; ++i) {
        const int t = threadIdx.x + i * kRopeThreads;
        if (t < n) {
            rotate_pair(lo[i], hi[i], cs, (t < nq ? t : t - nq) % per_head * 8);
            *addr(t, false) = lo[i];
            *addr(t, true) = hi[i];
        }
    }
    for (int t = threadIdx.x + kRopeHeld * kRopeThreads; t < n; t += kRopeThreads) {   // very wide rows
        uint4 a = *addr(t, false), b = *addr(t, true);
        rotate_pair(a, b, cs, (t < nq ? t : t - nq) % per_head * 8);
        *addr(t, false) = a;
        *addr(t, true) = b;
    }
}

// ---------------------------------------------------------------- token scatter
constexpr int kScatterMaxChunk = 512, kScatterThreads = 256, kScatterCtas = 1184, kScatterUnroll = 8;

__device__ __forceinline__ int is_vision(int id) {
    return (id == VIT_IMAGE_TOKEN_ID || id == VIT_VIDEO_TOKEN_ID) ? 1 : 0;
}

__global__ void __launch_bounds__(kScatterThreads) scatter_kernel(const int32_t *__restrict__ ids, int64_t L,
                                                                  const uint4 *__restrict__ table, int64_t vocab,
                                                                  const uint4 *__restrict__ vision, int64_t n_vision,
                                                                  int row_vecs, uint4 *__restrict__ out,
                                                                  int chunk, int32_t *status) {
    __shared__ int s_warp[kScatterThreads / 32];
    __shared__ int s_rank[kScatterMaxChunk];
    __shared__ int s_total;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * chunk;
    const int64_t c1 = c0 + chunk < L ? c0 + chunk : L;
    // placeholders before this chunk
    int cnt = 0;
    for (int64_t i = tid; i < c0; i += kScatterThreads) cnt += is_vision(__ldg(ids + i));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) s_warp[warp] = cnt;
    __syncthreads();
    if (warp == 0) {   // ranks inside the chunk, 32 tokens per ballot
        int base = 0;
        for (int w = 0; w < kScatterThreads / 32; ++w) base += s_warp[w];
        for (int b = 0; b < chunk; b += 32) {
            const int64_t i = c0 + b + lane;
            const int f = i < c1 ? is_vision(__ldg(ids + i)) : 0;
            const unsigned m = __ballot_sync(0xffffffffu, f);
            s_rank[b + lane] = f ? base + __popc(m & ((1u << lane) - 1u)) : -1;
            base += __popc(m);
        }
        if (lane == 0) s_total = base;
    }
    __syncthreads();
    if (tid == 0 && c1 == L && s_total != n_vision && status) atomicExch(status, VIT_ERR_TOKENS);
    // rows: each warp copies rows of the chunk
    for (int64_t i = c0 + warp; i < c1; i += kScatterThreads / 32) {
        const int rank = s_rank[i - c0];
        const uint4 *src;
        if (rank >= 0) {
            if (rank >= n_vision) {   // more placeholders than vision tokens: leave the row, flag it
                if (lane == 0 && status) atomicExch(status, VIT_ERR_TOKENS);
                continue;
            }
            src = vision + static_cast<int64_t>(rank) * row_vecs;
        } else {
            const int id = __ldg(ids + i);
            if (id < 0 || id >= vocab) {
                if (lane == 0 && status) atomicExch(status, VIT_ERR_TOKENS);
                continue;
            }
            src = table + static_cast<int64_t>(id) * row_vecs;
        }
        uint4 *dst = out + i * row_vecs;
        for (int c = lane; c < row_vecs; c += 32 * kScatterUnroll) {   // 8 loads in flight per lane
            uint4 v[kScatterUnroll];
#pragma unroll
            for (int e = 0; e < kScatterUnroll; ++e)
                if (c + 32 * e < row_vecs) v[e] = __ldg(src + c + 32 * e);
#pragma unroll
            for (int e = 0; e < kScatterUnroll; ++e)
                if (c + 32 * e < row_vecs) dst[c + 32 * e] = v[e];
        }
    }
}

}  // namespace vitk

namespace vith {

int mrope_apply_launch(void *q, int Hq, void *k, int Hk, int D, const int32_t *pos, int64_t L, double theta,
                       const int32_t *sections, cudaStream_t s) {
    vitk::MropeParams prm;
    prm.n_freq = D / 2;
    prm.axis_end0 = sections[0];
    prm.axis_end1 = sections[0] + sections[1];
    for (int j = 0; j < prm.n_freq; ++j) prm.inv_freq[j] = std::pow(theta, -2.0 * j / D);
    if (L <= 0) return VIT_OK;
    vitk::mrope_apply_kernel<<<static_cast<unsigned>(L), vitk::kRopeThreads, 0, s>>>(
        static_cast<__nv_bfloat16 *>(q), Hq, static_cast<__nv_bfloat16 *>(k), Hk, D, pos, L, prm);
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}

int scatter_launch(const int32_t *ids, int64_t L, const void *table, int64_t vocab, int dim, const void *vision,
                   int64_t n_vision, void *out, int32_t *status, cudaStream_t s) {
    if (L <= 0) return VIT_OK;
    // about 8 CTAs per SM: chunks of 8 tokens or more (a multiple of 8), so that at most ~1200
    // CTAs recount the prefix of the ids
    int64_t chunk = (L + vitk::kScatterCtas - 1) / vitk::kScatterCtas;
    chunk = chunk < 8 ? 8 : (chunk + 7) / 8 * 8;
    if (chunk > vitk::kScatterMaxChunk) return VIT_ERR_LIMIT;
    const int64_t chunks = (L + chunk - 1) / chunk;
    vitk::scatter_kernel<<<static_cast<unsigned>(chunks), vitk::kScatterThreads, 0, s>>>(
        ids, L, static_cast<const uint4 *>(table), vocab, static_cast<const uint4 *>(vision), n_vision, dim / 8,
        static_cast<uint4 *>(out), static_cast<int>(chunk), status);
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}

}  // namespace vith
