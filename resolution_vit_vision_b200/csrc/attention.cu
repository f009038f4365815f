// attention.cu -- varlen, block-diagonal attention on the tcgen05 tensor cores.
//
// "Qwen2-VL-2B-Instruct -- LiteRT-LM": the tower uses full attention, one image is one
// sequence, and the dynamic tower packs all images with cu_seqlens. Here a segment is one
// (image, frame); every query attends to every key of its own segment and to nothing else:
// out = softmax(q k^T / sqrt(80)) v per segment and head (16 heads x 80).
//
// One CTA = two 128-query tiles (A and B) of one (segment, head); keys stream through in tiles
// of 112 that both query tiles share:
//   warp 0      TMA producer: Q of both tiles once, K_j and V_j into a 4-deep ring (32-byte
//               swizzle, the 80-wide head read as five 16-column boxes straight from the [P, 3840]
//               QKV buffer)
//   warps 1, 2  one MMA-issuing thread per query tile: S_x(j) = Q_x K_j^T into the tile's TMEM
//               score buffer (M=128, N=112, K=5x16), then O_x += P_x(j) V_j (M=128, N=80,
//               K=7x16) with P_x read from TMEM
//   warps 3..6  softmax of tile A, 7..10 of tile B, one query row per thread: scores from TMEM,
//               online max / sum in fp32 with a lazy rescale (the exponent offset moves only when
//               the running max, in log2 units, grows by more than 8), P in bf16 back to TMEM, O
//               rescaled after the exponentials; the two warpgroups take turns at the
//               exponentials (named barriers) so one group's loads and stores overlap the
//               other's MUFU work; final O / l written as bf16.
// Work items are (segment, pair of query tiles), longest segments first; the work list travels
// as a kernel parameter.
#include <cuda_bf16.h>

#include <algorithm>
#include <memory>
#include <vector>

#include "internal.h"
#include "ptx.cuh"

namespace vitk {

constexpr int kAttnThreads = 352;                 // 11 warps
constexpr int kBQ = 128, kBKV = 112, kD = 80;     // query tile, key tile, head dim
constexpr int kQTilesPerCta = 2;                  // query tiles A and B share every K/V tile
constexpr int kKVStages = 4;
constexpr int kQBytes = kBQ * kD * 2;             // 20480: 5 boxes of 128 rows x 32 bytes
constexpr int kQBox = kBQ * 32;
constexpr int kKVBytes = kBKV * kD * 2;           // 17920: 5 boxes of 112 rows x 32 bytes
constexpr int kKVBox = kBKV * 32;
constexpr int kAttnSmem = 1024 + kQBytes * kQTilesPerCta + kKVBytes * 2 * kKVStages + 256;
constexpr int kMaxSegPerLaunch = 512;
constexpr int kMaxWorkPerLaunch = 4096;
// Lazy rescaling: a row's exponent offset only moves when its running max grows by more than
// this (log2 units), so P stays below 2^8 and O is rarely rescaled.
constexpr float kRescaleThreshold = 8.0f;

// TMEM columns of query tile x: scores S_x (112), P_x (bf16 pairs, 56 used of 64), O_x (80).
__host__ __device__ constexpr uint32_t col_s(int x) { return x * 112; }
__host__ __device__ constexpr uint32_t col_p(int x) { return 224 + x * 64; }
__host__ __device__ constexpr uint32_t col_o(int x) { return 352 + x * 80; }
static_assert(col_o(1) + 80 <= 512, "TMEM budget");

// Work list and segment starts travel as a kernel parameter (no device-side plan buffer).
struct AttnPlan {
    int n_work;
    int n_seg;
    int start[kMaxSegPerLaunch];      // absolute first row of each segment of this launch
    int len[kMaxSegPerLaunch];        // its number of rows
    int work[kMaxWorkPerLaunch];      // (local segment << 16) | pair of query tiles
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Warp roles: 0 TMA producer; 1 and 2 issue the tensor-core products of query tile A and B
// (one thread each, so neither tile's products wait behind the other's events); 3..6 softmax of
// tile A, 7..10 of tile B (one query row per thread). Each tile has its own score and P buffers,
// so S_x(j+1) = Q_x K_(j+1)^T runs while the softmax warpgroup still turns S_x(j) into P_x(j).
// 11 warps put 3 warps on three of the SM's four sub-partitions (16K registers each), which caps
// a thread at 168 registers.
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm, const __grid_constant__ CUtensorMap tkv,
                   const __grid_constant__ AttnPlan plan,
                   __nv_bfloat16 *__restrict__ out, int32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;                                   // [2][5 boxes]
    uint8_t *sK = sQ + kQTilesPerCta * kQBytes;
    uint8_t *sV = sK + kKVStages * kKVBytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sV + kKVStages * kKVBytes);
    uint64_t *q_full = bars;
    uint64_t *k_full = bars + 1;
    uint64_t *v_full = k_full + kKVStages;
    uint64_t *kv_empty = v_full + kKVStages;
    uint64_t *s_full = kv_empty + kKVStages;     // [2] per query tile
    uint64_t *s_free = s_full + 2;               // [2]
    uint64_t *p_full = s_free + 2;               // [2]
    uint64_t *o_done = p_full + 2;               // [2]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(o_done + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int item = blockIdx.x / VIT_HEADS, head = blockIdx.x % VIT_HEADS;
    const int wk = plan.work[item];
    const int seg = wk >> 16, pair = wk & 0xFFFF;
    const int seg_start = plan.start[seg], seg_len = plan.len[seg];
    const int q0 = seg_start + pair * kQTilesPerCta * kBQ;
    const int n_kv = (seg_len + kBKV - 1) / kBKV;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < kKVStages; ++s) {
            mbar_init(k_full + s, 1);
            mbar_init(v_full + s, 1);
            mbar_init(kv_empty + s, 2);              // released by both tiles' issuers
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(s_full + x, 1);
            mbar_init(s_free + x, 128);
            mbar_init(p_full + x, 128);
            mbar_init(o_done + x, 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    // the previous kernel of the stream (the QKV product) has completed from here on; tensor
    // memory is taken only after it
    pdl_wait();
    pdl_trigger();
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx wc{abort_flag, status};

    if (warp == 0) {
        if (lane == 0 && seg_len > 0) {
            tma_prefetch(&tm);
            tma_prefetch(&tkv);
            mbar_expect_tx(q_full, kQTilesPerCta * kQBytes);
            for (int x = 0; x < kQTilesPerCta; ++x)
                for (int c = 0; c < 5; ++c)
                    tma_load_2d(sQ + x * kQBytes + c * kQBox, &tm, q_full, head * kD + c * 16, q0 + x * kBQ);
            for (int j = 0; j < n_kv; ++j) {
                const int st = j % kKVStages;
                const uint32_t ph = (j / kKVStages) & 1;
                if (!mbar_wait(kv_empty + st, ph ^ 1u, wc)) break;
                const int r0 = seg_start + j * kBKV;
                mbar_expect_tx(k_full + st, kKVBytes);
                for (int c = 0; c < 5; ++c)
                    tma_load_2d(sK + st * kKVBytes + c * kKVBox, &tkv, k_full + st, VIT_WIDTH + head * kD + c * 16, r0);
                mbar_expect_tx(v_full + st, kKVBytes);
                for (int c = 0; c < 5; ++c)
                    tma_load_2d(sV + st * kKVBytes + c * kKVBox, &tkv, v_full + st,
                                2 * VIT_WIDTH + head * kD + c * 16, r0);
            }
        }
    } else if (warp == 1 || warp == 2) {
        if (lane == 0 && seg_len > 0) {
            const int x = warp - 1;                                // query tile of this issuer
            constexpr uint32_t idS = idesc_bf16(kBQ, kBKV, false, false);
            constexpr uint32_t idO = idesc_bf16(kBQ, kD, false, true);   // V is N(=head dim)-major
            const uint32_t qa = smem_u32(sQ) + x * kQBytes, ka = smem_u32(sK), va = smem_u32(sV);
            auto issue_s = [&](int j) {          // S_x = Q_x K_j^T
                const int st = j % kKVStages;
#pragma unroll
                for (int c = 0; c < 5; ++c) {
                    const uint64_t da = smem_desc(qa + c * kQBox, 16, 256, kSwizzle32B);
                    const uint64_t db = smem_desc(ka + st * kKVBytes + c * kKVBox, 16, 256, kSwizzle32B);
                    mma_bf16_ss(tmem + col_s(x), da, db, idS, c > 0 ? 1u : 0u);
                }
                mma_commit(s_full + x);
            };
            auto issue_pv = [&](int j) {         // O_x += P_x V_j, P_x read from TMEM (8 columns per 16 keys)
                const int st = j % kKVStages;
#pragma unroll
                for (int kk = 0; kk < kBKV / 16; ++kk) {
                    const uint64_t db = smem_desc(va + st * kKVBytes + kk * 512, kKVBox, 256, kSwizzle32B);
                    mma_bf16_ts(tmem + col_o(x), tmem + col_p(x) + kk * 8, db, idO, (j > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(o_done + x);
                mma_commit(kv_empty + st);
            };
            auto wait_k = [&](int j) { return mbar_wait(k_full + j % kKVStages, (j / kKVStages) & 1, wc); };
            bool ok = mbar_wait(q_full, 0, wc) && wait_k(0);
            if (ok) {
                tc_fence_after();
                issue_s(0);
            }
            for (int j = 0; ok && j < n_kv; ++j) {
                if (j + 1 < n_kv) {   // next scores once this tile's softmax has read S_x(j)
                    if (!mbar_wait(s_free + x, j & 1, wc) || !wait_k(j + 1)) break;
                    tc_fence_after();
                    issue_s(j + 1);
                }
                if (!mbar_wait(p_full + x, j & 1, wc) ||
                    !mbar_wait(v_full + j % kKVStages, (j / kKVStages) & 1, wc))
                    break;
                tc_fence_after();
                issue_pv(j);
            }
        }
    } else if (seg_len > 0) {
        const int x = (warp - 3) >> 2;                             // query tile of this warpgroup
        const int quarter = warp & 3;                              // TMEM lanes 32*quarter ..
        const int r = quarter * 32 + lane;                         // query row inside the tile
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tS = tmem + col_s(x) + lane_off;
        const uint32_t tP = tmem + col_p(x) + lane_off;
        const uint32_t tO = tmem + col_o(x) + lane_off;
        const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(kD));
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        // Ping-pong: the two warpgroups take turns for the exponentials (named barriers 2 and 3),
        // so one group's loads, max and stores run while the other keeps the MUFU busy.
        // Group A goes first; B's initial arrive on barrier 2 opens A's first turn.
        const int my_turn = 2 + x, their_turn = 3 - x;
        if (x == 1) named_bar_arrive(2, 256);
        for (int j = 0; j < n_kv; ++j) {
            // a failed (timed-out) wait does not leave the loop: both groups must keep taking
            // their turns on the named barriers; the results are then discarded
            if (!mbar_wait(s_full + x, j & 1, wc)) ok = false;
            tc_fence_after();
            uint32_t sr[112];
            tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(sr));
            tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
            tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(sr + 64));
            tmem_ld16(tS + 96, sr + 96);
            tmem_wait_ld();
            reg_fence32(sr);
            reg_fence32(sr + 32);
            reg_fence32(sr + 64);
            reg_fence16(sr + 96);
            tc_fence_before();
            mbar_arrive(s_free + x);                               // S_x may be overwritten now
            const int kv_valid = min(kBKV, seg_len - j * kBKV);
            if (kv_valid < kBKV) {   // last key tile of the segment
#pragma unroll
                for (int k = 0; k < kBKV; ++k)
                    if (k >= kv_valid) sr[k] = __float_as_uint(-INFINITY);
            }
            // row max: eight independent chains of three-input maxima (max.f32 with three sources)
            float m8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) m8[i] = __uint_as_float(sr[i]);
#pragma unroll
            for (int k = 8; k + 16 <= kBKV; k += 16)
#pragma unroll
                for (int i = 0; i < 8; ++i) m8[i] = fmax3(m8[i], __uint_as_float(sr[k + i]), __uint_as_float(sr[k + 8 + i]));
#pragma unroll
            for (int i = 0; i < 8; ++i) m8[i] = fmaxf(m8[i], __uint_as_float(sr[kBKV - 8 + i]));
            const float mx =
                fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) *
                scale_log2;
            // the rescale decision needs no tensor memory; O itself is scaled after the
            // exponentials, once P_x(j-1) V_(j-1) has completed
            const bool need = mx > m_used + kRescaleThreshold;
            const float alpha = (j > 0 && need) ? ex2(m_used - mx) : 1.0f;
            l *= alpha;
            if (need) m_used = mx;
            const float neg_m = -m_used;
            float r8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            uint32_t pk[56];
            named_bar_sync(my_turn, 256);                           // this group's turn
            // groups of four pairs: eight independent exponentials in flight before their results
            // are summed and packed, so the MUFU latency overlaps within one thread
#pragma unroll
            for (int k = 0; k < kBKV; k += 8) {
                float p[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) p[e] = fmaf(__uint_as_float(sr[k + e]), scale_log2, neg_m);
#pragma unroll
                for (int e = 0; e < 8; ++e) p[e] = ex2(p[e]);
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    r8[(e >> 1) + 4 * ((k >> 3) & 1)] += p[e] + p[e + 1];
                    pk[(k + e) >> 1] = pack_bf16x2(p[e], p[e + 1]);
                }
            }
            // hand the MUFU to the other group (B's arrive after its last turn has no partner)
            if (x == 0 || j + 1 < n_kv) named_bar_arrive(their_turn, 256);
            l += ((r8[0] + r8[1]) + (r8[2] + r8[3])) + ((r8[4] + r8[5]) + (r8[6] + r8[7]));
            // P_x(j-1) V_(j-1) must be complete before O_x is rescaled or P_x is overwritten
            if (j > 0) {
                if (!mbar_wait(o_done + x, (j - 1) & 1, wc)) ok = false;
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
                    for (int c = 0; c < 5; ++c) {
                        uint32_t o[16];
                        tmem_ld16(tO + c * 16, o);
                        tmem_wait_ld();
                        reg_fence16(o);
#pragma unroll
                        for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st16(tO + c * 16, o);
                    }
                }
            }
            tmem_st32(tP, pk);
            tmem_st16(tP + 32, pk + 32);
            {
                uint32_t pad[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) pad[e] = pk[48 + e];
                tmem_st8(tP + 48, pad);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_full + x);
        }
        if (ok && mbar_wait(o_done + x, (n_kv - 1) & 1, wc)) {
            tc_fence_after();
            uint32_t o[80];
#pragma unroll
            for (int c = 0; c < 5; ++c) tmem_ld16(tO + c * 16, o + c * 16);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 5; ++c) reg_fence16(o + c * 16);
            const int row = pair * kQTilesPerCta * kBQ + x * kBQ + r;   // row inside the segment
            if (row < seg_len) {
                const float inv = 1.0f / l;
                uint4 *dst = reinterpret_cast<uint4 *>(out + static_cast<int64_t>(seg_start + row) * VIT_WIDTH + head * kD);
#pragma unroll
                for (int q = 0; q < 10; ++q)
                    dst[q] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * q]) * inv, __uint_as_float(o[8 * q + 1]) * inv),
                                        pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv),
                                        pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv),
                                        pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) __nanosleep(200000);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// y[i] = exp2_fma2(x[i]): the FMA-pipe exponential of the softmax, elementwise, so that its error
// can be checked on a dense sweep against the exact 2^x.
__global__ void exp2_fma_kernel(const float *__restrict__ x, float *__restrict__ y, int64_t n) {
    for (int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x); i < n;
         i += 2 * static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float a = x[i], b = i + 1 < n ? x[i + 1] : 0.0f;
        exp2_fma2(a, b);
        y[i] = a;
        if (i + 1 < n) y[i + 1] = b;
    }
}

}  // namespace vitk

namespace vith {

int exp2_fma_launch(const float *x, float *y, int64_t n, cudaStream_t s) {
    if (n <= 0) return VIT_OK;
    const int64_t pairs = (n + 1) / 2;
    const int blocks = static_cast<int>(std::min<int64_t>((pairs + 255) / 256, 148 * 16));
    vitk::exp2_fma_kernel<<<blocks, 256, 0, s>>>(x, y, n);
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}


// Two views of the [P, 3840] QKV buffer, 16-column boxes with 32-byte swizzle: query tiles of
// 128 rows and key / value tiles of kBKV rows.
int attn_make_maps(AttnMaps *m, const void *qkv, int64_t P) {
    int rc = tmap_2d(&m->q, qkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 3 * VIT_WIDTH, static_cast<uint64_t>(P),
                     3 * VIT_WIDTH * 2, 16, vitk::kBQ, CU_TENSOR_MAP_SWIZZLE_32B);
    if (rc == VIT_OK)
        rc = tmap_2d(&m->kv, qkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 3 * VIT_WIDTH, static_cast<uint64_t>(P),
                     3 * VIT_WIDTH * 2, 16, vitk::kBKV, CU_TENSOR_MAP_SWIZZLE_32B);
    return rc;
}

namespace {

bool configure_attention() {
    static bool configured[64] = {};   // the attribute is set once per device
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && configured[dev]) return true;
    if (cudaFuncSetAttribute(vitk::attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, vitk::kAttnSmem) !=
        cudaSuccess)
        return false;
    if (dev < 64) configured[dev] = true;
    return true;
}

// Packs the (segment, pair of query tiles) work of the segments in `order` into as many launches
// as the per-launch tables need. A segment whose tiles do not all fit into the current launch
// continues in the next one (its start and length are repeated there), so one segment of any
// length up to VIT_MAX_PATCHES runs.
int launch_plans(vitk::AttnPlan &plan, const int *order, int n_seg,
                 const int32_t *cu_seqlens, const AttnMaps &tqkv, void *out, int32_t *status, cudaStream_t s) {
    constexpr int kRowsPerItem = vitk::kBQ * vitk::kQTilesPerCta;
    plan.n_seg = 0;
    plan.n_work = 0;
    auto flush = [&]() {
        if (plan.n_work > 0) {
            if (launch_pdl(vitk::attn_tc_kernel, dim3(plan.n_work * VIT_HEADS), dim3(vitk::kAttnThreads),
                           vitk::kAttnSmem, s, 1, tqkv.q, tqkv.kv, plan, static_cast<__nv_bfloat16 *>(out),
                           status) != cudaSuccess ||
                cudaGetLastError() != cudaSuccess)
                return false;
        }
        plan.n_seg = 0;
        plan.n_work = 0;
        return true;
    };
    for (int i = 0; i < n_seg; ++i) {
        const int sg = order[i];
        const int len = cu_seqlens[sg + 1] - cu_seqlens[sg];
        const int tiles = (len + kRowsPerItem - 1) / kRowsPerItem;
        for (int t = 0; t < tiles;) {
            if (plan.n_seg == vitk::kMaxSegPerLaunch || plan.n_work == vitk::kMaxWorkPerLaunch)
                if (!flush()) return VIT_ERR_CUDA;
            const int ls = plan.n_seg++;
            plan.start[ls] = cu_seqlens[sg];
            plan.len[ls] = len;
            for (; t < tiles && plan.n_work < vitk::kMaxWorkPerLaunch; ++t) plan.work[plan.n_work++] = (ls << 16) | t;
        }
    }
    return flush() ? VIT_OK : VIT_ERR_CUDA;
}

}  // namespace

// cu_seqlens: HOST [n_seg + 1]. Builds the (segment, q-tile) list, longest segments first
// (longest-processing-time-first over the CTA waves), and launches as many kernels as the
// per-launch limits need.
int attn_launch(const AttnMaps &tqkv, const int32_t *cu_seqlens, int n_seg, void *out, int32_t *status,
                cudaStream_t s) {
    if (n_seg < 0 || n_seg > VIT_MAX_SEGMENTS) return VIT_ERR_LIMIT;
    if (!configure_attention()) return VIT_ERR_CUDA;
    std::vector<int> order(n_seg);
    for (int i = 0; i < n_seg; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
        return (cu_seqlens[a + 1] - cu_seqlens[a]) > (cu_seqlens[b + 1] - cu_seqlens[b]);
    });
    auto plan = std::make_unique<vitk::AttnPlan>();
    return launch_plans(*plan, order.data(), n_seg, cu_seqlens, tqkv, out, status, s);
}

// attn_launch with the schedule kept on the host stack and an in-place sort (ties broken by
// segment index, the order attn_launch's stable sort gives), for callers that must not allocate.
int attn_launch_stack(const AttnMaps &tqkv, const int32_t *cu_seqlens, int n_seg, void *out, int32_t *status,
                      cudaStream_t s) {
    if (n_seg < 0 || n_seg > VIT_MAX_SEGMENTS) return VIT_ERR_LIMIT;
    if (!configure_attention()) return VIT_ERR_CUDA;
    int order[VIT_MAX_SEGMENTS];
    for (int i = 0; i < n_seg; ++i) order[i] = i;
    std::sort(order, order + n_seg, [&](int a, int b) {
        const int la = cu_seqlens[a + 1] - cu_seqlens[a], lb = cu_seqlens[b + 1] - cu_seqlens[b];
        return la != lb ? la > lb : a < b;
    });
    vitk::AttnPlan plan;
    return launch_plans(plan, order, n_seg, cu_seqlens, tqkv, out, status, s);
}

}  // namespace vith
