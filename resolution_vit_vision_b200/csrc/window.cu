// window.cu -- windowed attention of the Qwen2.5-VL tower.
//
// "Qwen2.5-VL-7B-Instruct" (inference-research model record), architecture note: the tower is
// Qwen2-VL's, but its blocks attend inside windows of 112 px (8 x 8 patches), except a few
// full-attention blocks (depths 7, 15, 23, 31). A patch belongs to window (h / 8, w / 8) of its
// frame; border windows are cut short.
//
// Layout. The encoder keeps its activations in WINDOW ORDER when windows are on: per image, per
// frame, the windows in raster order, inside a window its 2x2 merge groups in raster order, inside
// a group the patches (dh, dw). Every window is then a contiguous run of rows (a window side is
// even, so it holds whole merge groups), and so is every frame, so the full-attention blocks see
// the same per-frame segments as before. Everything else in a block works row by row, and each
// row keeps its own (h, w) for the rope, so only attention sees the order. The patches are
// gathered into this order once, before the patch embed; the merger's LayerNorm scatters the rows
// back to 2x2-block order, so the merged tokens come out in the usual order.
//
// Kernels:
//   window_positions_kernel  per window-order row: (h, w), the input row it comes from, and the
//                            2x2-block-order row the merger reads it from; the first row of each
//                            window also writes that window's (first row, rows) to a table
//   gather_rows_kernel       patches into window order (16-byte copies, HBM-bound)
//   win_attn_kernel          attention inside windows of at most 64 patches: two windows share
//                            one 128-row tile (one per 64-row half, loaded by TMA straight from
//                            the [P, 3840] QKV buffer: columns 0..63 of a head as 128-byte
//                            swizzled rows, 64..79 as 32-byte rows), S = Q K^T and O = P V on the
//                            tensor cores with the two off-diagonal 64 x 64 blocks of P set to
//                            zero; each window fits in one tile, so the softmax is exact in one
//                            pass. Persistent: one CTA per SM walks (window pair, head) items;
//                            Q and K come through a 3-stage TMA ring freed as soon as S is
//                            computed, V through a 5-stage ring freed after P V, so more of the
//                            item loads are in flight; two softmax warpgroups take alternate
//                            items, each with its own MMA-issuing thread, and a group stores
//                            item k's output while P V of item k + 2 runs. The kernel is bound
//                            by HBM (q, k, v read once, the output written once).
#include <cuda_bf16.h>

#include <algorithm>
#include <memory>
#include <vector>

#include "internal.h"
#include "ptx.cuh"

namespace vitk {

// ---------------------------------------------------------------- window geometry
// Closed forms over the merged grid (H2 x W2 merge groups per frame, windows of wm x wm groups):
// window row a holds ha = min(wm, H2 - a wm) group rows and every group column, so the groups
// before window (a, b) number a wm W2 + ha b wm; inside a window the groups run in raster order
// with width wb = min(wm, W2 - b wm).
struct WinGeom {
    int H2, W2, wm, nwh, nww;
    __host__ __device__ WinGeom(int h, int w, int wm_) : H2(h >> 1), W2(w >> 1), wm(wm_) {
        nwh = (H2 + wm - 1) / wm;
        nww = (W2 + wm - 1) / wm;
    }
    __host__ __device__ int per_frame() const { return nwh * nww; }
    // first row (inside the frame) and number of rows of window widx of a frame
    __host__ __device__ void window(int widx, int &first, int &rows) const {
        const int a = widx / nww, b = widx % nww;
        const int ha = min(wm, H2 - a * wm), wb = min(wm, W2 - b * wm);
        first = 4 * (a * wm * W2 + ha * b * wm);
        rows = 4 * ha * wb;
    }
    // merge group (mh, mw) of group index u inside the frame, in window order; widx = its window
    // (a nww + b), in_win = its index inside the window, rows = the window's number of rows
    __host__ __device__ void group(int u, int &mh, int &mw, int &widx, int &in_win, int &rows) const {
        const int a = u / (wm * W2);
        const int ha = min(wm, H2 - a * wm);
        const int rem = u - a * wm * W2;
        const int b = rem / (ha * wm);
        const int wb = min(wm, W2 - b * wm);
        in_win = rem - b * ha * wm;
        mh = a * wm + in_win / wb;
        mw = b * wm + in_win % wb;
        widx = a * nww + b;
        rows = 4 * ha * wb;
    }
};

// Grid table (kernel parameter): per image its first row, (h, w), and its first window index.
struct WinTable {
    int n_images, wm, n_windows;
    int row_start[VIT_MAX_IMAGES];
    int win_start[VIT_MAX_IMAGES + 1];
    int h[VIT_MAX_IMAGES], w[VIT_MAX_IMAGES];
};

__device__ __forceinline__ int last_le(const int *a, int n, int v) {   // last i < n with a[i] <= v
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a[mid] <= v) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// pos[r] = (h << 16) | w of window-order row r; src_row[r] = its row in the caller's packed order
// (patch_order 0: 2x2-block, 1: raster); merge_row[r] = its row in 2x2-block order. The first row
// of window wi writes win_tab[wi] = (that row, the window's rows).
__global__ void window_positions_kernel(const __grid_constant__ WinTable T, int64_t P, int patch_order,
                                        int32_t *__restrict__ pos, int32_t *__restrict__ merge_row,
                                        int32_t *__restrict__ src_row, int2 *__restrict__ win_tab) {
    pdl_wait();                                   // the previous encode may still read these tables
    pdl_trigger();
    const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (r >= P) return;
    const int i = last_le(T.row_start, T.n_images, static_cast<int>(r));
    const int h = T.h[i], w = T.w[i];
    const WinGeom g(h, w, T.wm);
    const int j = static_cast<int>(r - T.row_start[i]);
    const int f = j / (h * w);
    const int frame_start = T.row_start[i] + f * (h * w);
    const int q = j % (h * w);
    int mh, mw, widx, in_win, rows;
    g.group(q >> 2, mh, mw, widx, in_win, rows);
    if (in_win == 0 && (q & 3) == 0)
        win_tab[T.win_start[i] + f * g.per_frame() + widx] = make_int2(static_cast<int>(r), rows);
    const int hp = 2 * mh + ((q >> 1) & 1), wp = 2 * mw + (q & 1);
    const int block_row = frame_start + 4 * (mh * g.W2 + mw) + (q & 3);
    pos[r] = (hp << 16) | wp;
    merge_row[r] = block_row;
    src_row[r] = patch_order == 0 ? block_row : frame_start + hp * w + wp;
}

// dst[r, :] = src[src_row[r], :] for rows of `row_bytes` (a multiple of 16); one warp per row.
__global__ void gather_rows_kernel(const uint4 *__restrict__ src, const int32_t *__restrict__ src_row,
                                   uint4 *__restrict__ dst, int64_t rows, int row_vecs) {
    pdl_wait();                                   // src is the previous kernel's output
    pdl_trigger();
    const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const uint4 *s = src + static_cast<int64_t>(src_row[r]) * row_vecs;
    uint4 *d = dst + r * row_vecs;
    for (int c = lane; c < row_vecs; c += 32) d[c] = s[c];
}

// ---------------------------------------------------------------- attention inside windows
constexpr int kWThreads = 352;                      // 11 warps
constexpr int kWQKStages = 3, kWVStages = 5;        // Q+K ring (freed after S), V ring (after P V)
constexpr int kWRows = 128, kWHalf = 64, kWD = 80;  // tile rows, rows per window slot, head dim
constexpr int kWChunk = kWRows * 32;                // one 16-column box column of the tile: 4096 B
constexpr int kWTensor = 5 * kWChunk;               // Q, K or V of one tile: 20480 B
constexpr int kW128 = kWRows * 128;                 // its columns 0..63 (128-byte rows): 16384 B
constexpr int kWQK = 2 * kWTensor;                  // 40960 B
constexpr int kWSmem = 1024 + kWQKStages * kWQK + kWVStages * kWTensor + 256;
// TMEM columns: scores of group g at 128 g (P, bf16 pairs, written over their first 64 columns),
// the output of group g at 256 + 80 g.
__host__ __device__ constexpr uint32_t wcol_s(int g) { return 128 * g; }
__host__ __device__ constexpr uint32_t wcol_o(int g) { return 256 + 80 * g; }
static_assert(wcol_o(1) + kWD <= 512, "TMEM budget");

__device__ __forceinline__ float wex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// (first row, rows) of window wi; an absent second window of the last pair reads as empty
__device__ __forceinline__ int2 window_entry(const int2 *tab, int n_windows, int wi) {
    return wi < n_windows ? __ldg(tab + wi) : make_int2(0, 0);
}

// Warp roles: 0 TMA producer; 1 and 2 issue the products of the even and of the odd items (one
// thread each); 3..6 softmax + output of the even items, 7..10 of the odd items (one tile row
// per thread; warp w reads TMEM lanes 32 (w % 4) ..). Rows 0..63 of a tile are window 2p, rows
// 64..127 window 2p + 1. The window table is trusted for its rows (each within [0, P), at most 64
// long); stores stay below P. 11 warps put three on three of the four sub-partitions, which caps a
// thread at 168 registers.
__global__ void __launch_bounds__(kWThreads, 1)
    win_attn_kernel(const __grid_constant__ CUtensorMap tm32, const __grid_constant__ CUtensorMap tm128,
                    const int2 *__restrict__ win_tab, int n_windows, int n_items, int P,
                    __nv_bfloat16 *__restrict__ out, int32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sV = smem + kWQKStages * kWQK;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sV + kWVStages * kWTensor);
    uint64_t *qk_full = bars;                   // [QK stages] Q, K of an item landed
    uint64_t *qk_empty = qk_full + kWQKStages;  // [QK stages] S is done with them
    uint64_t *v_full = qk_empty + kWQKStages;   // [V stages]
    uint64_t *v_empty = v_full + kWVStages;     // [V stages] P V is done with it
    uint64_t *s_full = v_empty + kWVStages;     // [2] scores of group g ready
    uint64_t *p_full = s_full + 2;              // [2] P of group g written
    uint64_t *o_full = p_full + 2;              // [2] O of group g ready (P consumed)
    uint64_t *o_free = o_full + 2;              // [2] O of group g read out
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(o_free + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_mine = n_items > static_cast<int>(blockIdx.x)
                           ? (n_items - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                           : 0;
    auto item_of = [&](int k) { return static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kWQKStages; ++s) {
            mbar_init(qk_full + s, 1);
            mbar_init(qk_empty + s, 1);
        }
        for (int s = 0; s < kWVStages; ++s) {
            mbar_init(v_full + s, 1);
            mbar_init(v_empty + s, 1);
        }
        for (int g = 0; g < 2; ++g) {
            mbar_init(s_full + g, 1);
            mbar_init(p_full + g, 128);
            mbar_init(o_full + g, 1);
            mbar_init(o_free + g, 128);
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
        if (lane == 0 && n_mine > 0) {
            tma_prefetch(&tm32);
            tma_prefetch(&tm128);
            // window entries are read one item ahead, so their latency hides behind the ring wait
            int pair = item_of(0) / VIT_HEADS;
            int2 w0 = window_entry(win_tab, n_windows, 2 * pair), w1 = window_entry(win_tab, n_windows, 2 * pair + 1);
            for (int k = 0; k < n_mine; ++k) {
                const int sq = k % kWQKStages, sv = k % kWVStages;
                const int head = item_of(k) % VIT_HEADS;
                const int s0 = w0.x, s1 = w1.y > 0 ? w1.x : w0.x;   // no second window: load the first
                if (k + 1 < n_mine) {                                 // again, so every row is finite
                    pair = item_of(k + 1) / VIT_HEADS;
                    w0 = window_entry(win_tab, n_windows, 2 * pair);
                    w1 = window_entry(win_tab, n_windows, 2 * pair + 1);
                }
                // per tensor: columns 0..63 of the head, then 64..79, for both windows
                auto load_tensor = [&](uint8_t *dst, int t, uint64_t *bar) {
                    const int col = t * VIT_WIDTH + head * kWD;
                    tma_load_2d(dst, &tm128, bar, col, s0);
                    tma_load_2d(dst + kWHalf * 128, &tm128, bar, col, s1);
                    tma_load_2d(dst + kW128, &tm32, bar, col + 64, s0);
                    tma_load_2d(dst + kW128 + kWHalf * 32, &tm32, bar, col + 64, s1);
                };
                if (!mbar_wait(qk_empty + sq, ((k / kWQKStages) & 1) ^ 1u, wc)) break;
                mbar_expect_tx(qk_full + sq, kWQK);
                load_tensor(smem + sq * kWQK, 0, qk_full + sq);
                load_tensor(smem + sq * kWQK + kWTensor, 1, qk_full + sq);
                if (!mbar_wait(v_empty + sv, ((k / kWVStages) & 1) ^ 1u, wc)) break;
                mbar_expect_tx(v_full + sv, kWTensor);
                load_tensor(sV + sv * kWTensor, 2, v_full + sv);
            }
        }
    } else if (warp == 1 || warp == 2) {
        if (lane == 0 && n_mine > warp - 1) {
            constexpr uint32_t idS = idesc_bf16(kWRows, kWRows, false, false);
            constexpr uint32_t idO64 = idesc_bf16(kWRows, 64, false, true);   // V is N(=head dim)-major
            constexpr uint32_t idO16 = idesc_bf16(kWRows, 16, false, true);
            const uint32_t base = smem_u32(smem);
            auto issue_s = [&](int k) {   // S_g = Q K^T over both windows of the tile
                const int st = k % kWQKStages, g = k & 1;
                if (!mbar_wait(qk_full + st, (k / kWQKStages) & 1, wc)) return false;
                // P_g of item k - 2 (written over S_g) must have been consumed
                if (k >= 2 && !mbar_wait(o_full + g, ((k >> 1) - 1) & 1, wc)) return false;
                tc_fence_after();
                const uint32_t qa = base + st * kWQK, ka = qa + kWTensor;
#pragma unroll
                for (int c = 0; c < 4; ++c)   // head dims 0..63: K-major, 128-byte swizzle, +32 B per 16
                    mma_bf16_ss(tmem + wcol_s(g), smem_desc(qa + c * 32, 16, 1024, kSwizzle128B),
                                smem_desc(ka + c * 32, 16, 1024, kSwizzle128B), idS, c > 0 ? 1u : 0u);
                mma_bf16_ss(tmem + wcol_s(g), smem_desc(qa + kW128, 16, 256, kSwizzle32B),
                            smem_desc(ka + kW128, 16, 256, kSwizzle32B), idS, 1u);   // dims 64..79
                mma_commit(s_full + g);
                mma_commit(qk_empty + st);
                return true;
            };
            auto issue_pv = [&](int k) {   // O_g = P_g V, P_g read from TMEM (8 columns per 16 keys)
                const int st = k % kWVStages, g = k & 1, u = k >> 1;
                if (!mbar_wait(p_full + g, u & 1, wc)) return false;
                if (u > 0 && !mbar_wait(o_free + g, (u - 1) & 1, wc)) return false;
                if (!mbar_wait(v_full + st, (k / kWVStages) & 1, wc)) return false;
                tc_fence_after();
                const uint32_t va = base + kWQKStages * kWQK + st * kWTensor;
#pragma unroll
                for (int kk = 0; kk < kWRows / 16; ++kk) {   // O[:, 0:64] and O[:, 64:80], 16 keys a step
                    mma_bf16_ts(tmem + wcol_o(g), tmem + wcol_s(g) + kk * 8,
                                smem_desc(va + kk * 2048, kW128, 1024, kSwizzle128B), idO64, kk > 0 ? 1u : 0u);
                    mma_bf16_ts(tmem + wcol_o(g) + 64, tmem + wcol_s(g) + kk * 8,
                                smem_desc(va + kW128 + kk * 512, kWChunk, 256, kSwizzle32B), idO16, kk > 0 ? 1u : 0u);
                }
                mma_commit(o_full + g);
                mma_commit(v_empty + st);
                return true;
            };
            // the items of one softmax group, in order: S(k) needs its data and P V of item k - 2
            // (whose P lies where S(k) goes); P V(k) needs P(k) and O of item k - 2 read out
            const int g = warp - 1;
            for (int k = g; k < n_mine; k += 2)
                if (!issue_s(k) || !issue_pv(k)) break;
        }
    } else {
        const int g = (warp - 3) >> 2;                       // items k with k % 2 == g
        const int quarter = warp & 3;                        // TMEM lanes 32 * quarter ..
        const int r = quarter * 32 + lane;                   // tile row
        const int half = r >> 6;                             // window slot of this row
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tS = tmem + wcol_s(g) + lane_off;
        const uint32_t tO = tmem + wcol_o(g) + lane_off;
        const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(kWD));
        int2 wnext = g < n_mine ? window_entry(win_tab, n_windows, 2 * (item_of(g) / VIT_HEADS) + half)
                                : make_int2(0, 0);
        // the output of item k - 2 is held packed in registers and stored while P V of item k runs
        uint4 ob[10];
        uint4 *ob_dst = nullptr;
        auto flush_out = [&]() {
            if (ob_dst) {
#pragma unroll
                for (int q = 0; q < 10; ++q) ob_dst[q] = ob[q];
            }
            ob_dst = nullptr;
        };
        for (int u = 0;; ++u) {
            const int k = 2 * u + g;
            if (k >= n_mine) break;
            const int head = item_of(k) % VIT_HEADS;
            const int start = wnext.x, len = min(wnext.y, kWHalf);
            if (k + 2 < n_mine) wnext = window_entry(win_tab, n_windows, 2 * (item_of(k + 2) / VIT_HEADS) + half);
            if (!mbar_wait(s_full + g, u & 1, wc)) break;
            tc_fence_after();
            uint32_t sr[64];
            tmem_ld32(tS + kWHalf * half, *reinterpret_cast<uint32_t(*)[32]>(sr));
            tmem_ld32(tS + kWHalf * half + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
            tmem_wait_ld();
            reg_fence32(sr);
            reg_fence32(sr + 32);
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < kWHalf; ++c) {
                if (c >= len) sr[c] = __float_as_uint(-INFINITY);
                mx = fmaxf(mx, __uint_as_float(sr[c]));
            }
            const float neg_m = len > 0 ? -mx * scale_log2 : 0.f;
            float l0 = 0.f, l1 = 0.f;
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < kWHalf; c += 2) {
                const float p0 = wex2(fmaf(__uint_as_float(sr[c]), scale_log2, neg_m));
                const float p1 = wex2(fmaf(__uint_as_float(sr[c + 1]), scale_log2, neg_m));
                l0 += p0;
                l1 += p1;
                pk[c >> 1] = pack_bf16x2(p0, p1);
            }
            uint32_t zero[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) zero[c] = 0u;
            // P row: this window's 64 keys, zeros on the other window's
            tmem_st32(tS + 32 * half, pk);
            tmem_st32(tS + 32 * (1 - half), zero);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_full + g);
            flush_out();
            if (!mbar_wait(o_full + g, u & 1, wc)) break;
            tc_fence_after();
            uint32_t o[80];
#pragma unroll
            for (int c = 0; c < 5; ++c) tmem_ld16(tO + c * 16, o + c * 16);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 5; ++c) reg_fence16(o + c * 16);
            tc_fence_before();
            mbar_arrive(o_free + g);
            const int row = r & (kWHalf - 1);
            if (row < len && start + row < P) {
                const float inv = 1.0f / (l0 + l1);
                ob_dst = reinterpret_cast<uint4 *>(out + static_cast<int64_t>(start + row) * VIT_WIDTH + head * kWD);
#pragma unroll
                for (int q = 0; q < 10; ++q)
                    ob[q] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * q]) * inv, __uint_as_float(o[8 * q + 1]) * inv),
                                       pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv),
                                       pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv),
                                       pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv));
            }
        }
        flush_out();
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) __nanosleep(200000);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace vitk

namespace vith {

namespace {
// Fills the grid table (grids validated by the caller); returns the number of windows.
int fill_table(vitk::WinTable &T, const int32_t *grid_thw, int n_images, int window) {
    T.n_images = n_images;
    T.wm = window / 2;
    int row = 0, win = 0;
    for (int i = 0; i < n_images; ++i) {
        const int t = grid_thw[3 * i], h = grid_thw[3 * i + 1], w = grid_thw[3 * i + 2];
        T.row_start[i] = row;
        T.win_start[i] = win;
        T.h[i] = h;
        T.w[i] = w;
        row += t * h * w;
        win += t * vitk::WinGeom(h, w, T.wm).per_frame();
    }
    T.win_start[n_images] = win;
    T.n_windows = win;
    return win;
}
}  // namespace

int window_cu_seqlens(const int32_t *grid_thw, int n_images, int window, std::vector<int32_t> &cu) {
    if (window < 2 || window % 2) return VIT_ERR_ARG;
    cu.assign(1, 0);
    for (int i = 0; i < n_images; ++i) {
        const int t = grid_thw[3 * i], h = grid_thw[3 * i + 1], w = grid_thw[3 * i + 2];
        const vitk::WinGeom g(h, w, window / 2);
        for (int f = 0; f < t; ++f)
            for (int x = 0; x < g.per_frame(); ++x) {
                int first, rows;
                g.window(x, first, rows);
                cu.push_back(cu.back() + rows);
            }
    }
    return VIT_OK;
}

int window_count(const int32_t *grid_thw, int n_images, int window) {
    int win = 0;
    for (int i = 0; i < n_images; ++i)
        win += grid_thw[3 * i] * vitk::WinGeom(grid_thw[3 * i + 1], grid_thw[3 * i + 2], window / 2).per_frame();
    return win;
}

int window_positions_launch(const int32_t *grid_thw, int n_images, int64_t P, int patch_order, int window,
                            int32_t *pos, int32_t *merge_row, int32_t *src_row, int32_t *win_tab, cudaStream_t s) {
    if (window < 2 || window % 2) return VIT_ERR_ARG;
    auto T = std::make_unique<vitk::WinTable>();
    fill_table(*T, grid_thw, n_images, window);
    if (P <= 0) return VIT_OK;
    if (launch_pdl(vitk::window_positions_kernel, dim3(static_cast<unsigned>((P + 255) / 256)), dim3(256), 0, s, 1,
                   *T, P, patch_order, pos, merge_row, src_row, reinterpret_cast<int2 *>(win_tab)) != cudaSuccess)
        return VIT_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}

int gather_rows_launch(const void *src, const int32_t *src_row, void *dst, int64_t rows, int row_bytes,
                       cudaStream_t s) {
    if (row_bytes % 16 || (reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) % 16)
        return VIT_ERR_ALIGN;
    if (rows <= 0) return VIT_OK;
    const int64_t threads = rows * 32;
    if (launch_pdl(vitk::gather_rows_kernel, dim3(static_cast<unsigned>((threads + 255) / 256)), dim3(256), 0, s, 1,
                   static_cast<const uint4 *>(src), src_row, static_cast<uint4 *>(dst), rows, row_bytes / 16) !=
        cudaSuccess)
        return VIT_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}

// The [P, 3840] QKV buffer as 64-row boxes: 16 columns with 32-byte swizzle, 64 with 128-byte.
int win_make_maps(WinMaps *m, const void *qkv, int64_t P) {
    int rc = tmap_2d(&m->m32, qkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 3 * VIT_WIDTH, static_cast<uint64_t>(P),
                     3 * VIT_WIDTH * 2, 16, vitk::kWHalf, CU_TENSOR_MAP_SWIZZLE_32B);
    if (rc == VIT_OK)
        rc = tmap_2d(&m->m128, qkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 3 * VIT_WIDTH, static_cast<uint64_t>(P),
                     3 * VIT_WIDTH * 2, 64, vitk::kWHalf, CU_TENSOR_MAP_SWIZZLE_128B);
    return rc;
}

int win_attn_launch(const WinMaps &m, const int32_t *win_tab, int n_windows, int64_t P, void *out, int32_t *status,
                    cudaStream_t s) {
    if (n_windows < 0 || !win_tab) return VIT_ERR_ARG;
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !configured[dev]) {
        if (cudaFuncSetAttribute(vitk::win_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, vitk::kWSmem) !=
            cudaSuccess)
            return VIT_ERR_CUDA;
        configured[dev] = true;
    }
    const int n_items = ((n_windows + 1) / 2) * VIT_HEADS;
    if (n_items == 0) return VIT_OK;
    const int grid = std::min(n_items, device_sm_count());
    if (launch_pdl(vitk::win_attn_kernel, dim3(grid), dim3(vitk::kWThreads), vitk::kWSmem, s, 1, m.m32, m.m128,
                   reinterpret_cast<const int2 *>(win_tab), n_windows, n_items, static_cast<int>(P),
                   static_cast<__nv_bfloat16 *>(out), status) != cudaSuccess)
        return VIT_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}

}  // namespace vith
