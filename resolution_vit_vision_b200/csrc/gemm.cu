// gemm.cu -- persistent, warp-specialised tcgen05 GEMM C = A B^T with fused epilogues.
//
// Used for every dense contraction of the tower ("Qwen2-VL (Native-Resolution VLM)", Structure
// table: Patchify 14x14 as a [P,1176]x[1176,1280] product, the ViT blocks' QKV / out-proj /
// MLP linears, and the Patch Merger's two linears).
//
// Two SMs share each output tile of 256 x BN (a cluster of two CTAs, tcgen05 cta_group::2): each
// CTA holds its 128 rows of A and half of the tile's BN rows of B in its own shared memory, so
// every SM streams 64 bytes of operands per 128 x BN x 16 product share instead of 96 -- the
// operand feed from L2, not the tensor pipe, had bounded the one-SM tiles. The even CTA issues
// the M = 256 products; each CTA receives its 128 rows of the accumulator in its own TMEM.
// Per CTA (persistent, the pair walks the 256 x BN tiles together):
//   warp 0      TMA producer: its A rows and its half of B (128B-swizzled, K-major) into a
//               STAGES-deep ring; both CTAs' loads complete on the even CTA's barrier
//   warp 1      (even CTA, one thread) MMA issuer: tcgen05.mma 256xBNx16 into the pair's TMEM
//               accumulators, commits multicast to both CTAs; two accumulators so the epilogue of
//               tile i overlaps the mainloop of tile i+1
//   warps 2..5  epilogue (and 6..9: a second warpgroup for the products whose epilogue would
//               otherwise hold the mainloop back -- E4M3, rope, small-batch tiles -- each group
//               taking every other column chunk or head of a tile): tcgen05.ld of the
//               accumulator rows (one row per thread), bias, GELU / 2-D rope, then the chunk
//               leaves through a swizzled shared staging buffer and a TMA store -- or a TMA
//               reduce-add into the fp32 residual stream, so the residual update never reads the
//               residual into the SM.
// The same kernel runs the fp8 tower's products (F8 = true): A and B are E4M3 codes with a
// power-of-two scale per row of A and per row of B ("Qwen2-VL-2B-Instruct -- LiteRT-LM", file
// table: an 8-bit vision tower); a 128-byte k-block then holds 128 elements instead of 64, the
// tensor core runs kind::f8f6f4 (K = 32 per instruction) at twice the bf16 rate, and the epilogue
// multiplies every accumulator by its row's and column's scales before the bias.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace vitk {

constexpr int kBM = 128;
constexpr int kBK = 64;           // 64 bf16 = 128 bytes: one 128B swizzle atom per row
constexpr int kEpiBarrier = 1;    // named barriers kEpiBarrier + g of the 128 threads of group g

// Epilogue warpgroups of a product: two, each taking every other column chunk (or head) of a tile,
// where the epilogue would otherwise hold the mainloop back -- the E4M3 products (twice the
// product rate), the rope epilogue, the 256 x 128 tiles of small batches -- else one. The two
// staging buffers are double-buffered by one group or split between two.
template <int BN, int EPI, bool F8>
struct GemmCfg {
    static constexpr int GROUPS = (F8 || EPI == VIT_EPI_QKV_ROPE || BN == 128) ? 2 : 1;
    static constexpr int THREADS = 64 + 128 * GROUPS;
    static constexpr int NBUF = 2 / GROUPS;   // staging buffers per group
};

template <int BN>
struct GemmShape {
    static constexpr int STAGES = BN == 240 ? 5 : (BN == 128 ? 8 : 6);
    static constexpr int A_BYTES = kBM * kBK * 2;
    static constexpr int B_BYTES = (BN / 2) * kBK * 2;   // this CTA's half of the B tile
    static constexpr int ACC_STRIDE = 256;    // TMEM columns between the two accumulators
    static constexpr int TMEM_COLS = 512;
    // output staging chunk: 128 rows x 128 bytes (32 fp32 or 64 bf16 columns), or for QKV one
    // 80-wide head as five 128 x 32-byte boxes
    static constexpr int STG_BYTES = BN == 240 ? 5 * 4096 : 16384;
    static constexpr int SMEM = 1024 + STAGES * (A_BYTES + B_BYTES) + 2 * STG_BYTES + 256;
    static_assert(B_BYTES % 1024 == 0, "B stage must keep 1024-byte alignment");
    static_assert(SMEM <= 232448, "shared memory per block");
};

struct GemmParams {
    const __nv_bfloat16 *bias;
    const float *a_scale;             // F8 only: [M] power-of-two scale of each row of A
    const float *b_scale;             // F8 only: [N] scale of each row of B (output column)
    const int32_t *pos;
    const float2 *rope_cs;
    int32_t *status;
    int M, N, K;
    int m_tiles, n_tiles, k_blocks;   // m_tiles: 256-row tiles of the CTA pair
};

// GELU(x) = x Phi(x) = 0.5 x (1 + erf(x / sqrt 2)), with erf from Abramowitz & Stegun,
// Handbook of Mathematical Functions, eq. 7.1.26 (Hastings' approximation): for z >= 0,
// erfc(z) = t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-z^2) + e(z), t = 1 / (1 + p z),
// |e(z)| <= 1.5e-7. For x < 0, 1 + erf(x / sqrt 2) = erfc(|x| / sqrt 2) is taken directly from
// that product, so large negative x keep their relative accuracy. Two MUFU operations (rcp, ex2)
// per element. Evaluated on two values at once: the FMA-pipe work as packed fp32x2 instructions
// (half the instruction count), the reciprocals and exponentials on the MUFU. The epilogue warps
// share the SM sub-partitions with the TMA and MMA warps, and their instruction volume had been
// slowing the mainloop of the next tile (fc1 188 -> 171 us per launch).
__device__ __forceinline__ void gelu_erf2(float &x0, float &x1) {
    float z0, z1, q0, q1, t0, t1, p0, p1, w0, w1, e0, e1;
    fmul2(z0, z1, fabsf(x0), fabsf(x1), 0.70710678118654752f, 0.70710678118654752f);
    ffma2(q0, q1, 0.3275911f, 0.3275911f, z0, z1, 1.0f, 1.0f);
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t0) : "f"(q0));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t1) : "f"(q1));
    ffma2(p0, p1, t0, t1, 1.061405429f, 1.061405429f, -1.453152027f, -1.453152027f);
    ffma2(p0, p1, t0, t1, p0, p1, 1.421413741f, 1.421413741f);
    ffma2(p0, p1, t0, t1, p0, p1, -0.284496736f, -0.284496736f);
    ffma2(p0, p1, t0, t1, p0, p1, 0.254829592f, 0.254829592f);
    fmul2(p0, p1, p0, p1, t0, t1);
    fmul2(w0, w1, z0, z1, z0, z1);                                        // z^2
    fmul2(w0, w1, w0, w1, -1.4426950408889634f, -1.4426950408889634f);    // -z^2 log2 e
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e0) : "f"(w0));
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(w1));
    fmul2(e0, e1, p0, p1, e0, e1);   // erfc(|x| / sqrt 2)
    const float s0 = x0 >= 0.f ? 2.0f - e0 : e0, s1 = x1 >= 0.f ? 2.0f - e1 : e1;
    fmul2(w0, w1, x0, x1, 0.5f, 0.5f);
    fmul2(x0, x1, w0, w1, s0, s1);
}

// v[0..NV) += bias[col0 ..] (bias 16-byte aligned, col0 a multiple of 8), columns >= N skipped
template <int NV>
__device__ __forceinline__ void add_bias(float *v, const __nv_bfloat16 *bias, int col0, int N) {
    if (bias == nullptr) return;
#pragma unroll
    for (int q = 0; q < NV / 8; ++q) {
        if (col0 + 8 * q < N) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(bias + col0) + q);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) fadd2(v[q * 8 + 2 * j], v[q * 8 + 2 * j + 1], bf16_lo(w[j]), bf16_hi(w[j]));
        }
    }
}

// v[j] *= sa * b_scale[col0 + j] (the fp8 products' dequantisation; b_scale 16-byte aligned,
// col0 a multiple of 4), columns >= N skipped
template <int NV>
__device__ __forceinline__ void scale_cols(float *v, float sa, const float *b_scale, int col0, int N) {
#pragma unroll
    for (int q = 0; q < NV / 4; ++q) {
        if (col0 + 4 * q < N) {
            const float4 b = __ldg(reinterpret_cast<const float4 *>(b_scale + col0) + q);
            float s0, s1, s2, s3;
            fmul2(s0, s1, sa, sa, b.x, b.y);
            fmul2(s2, s3, sa, sa, b.z, b.w);
            fmul2(v[4 * q], v[4 * q + 1], v[4 * q], v[4 * q + 1], s0, s1);
            fmul2(v[4 * q + 2], v[4 * q + 3], v[4 * q + 2], v[4 * q + 3], s2, s3);
        }
    }
}

// Writes one thread's row r of 128 bytes (eight 16-byte pieces) into a 128B-swizzled staging
// chunk: piece q lands at piece q ^ (r % 8), the layout a SWIZZLE_128B TMA box expects.
__device__ __forceinline__ void stage_row128(uint8_t *stg, int r, const uint32_t *w) {
    uint8_t *row = stg + r * 128;
#pragma unroll
    for (int q = 0; q < 8; ++q)
        *reinterpret_cast<uint4 *>(row + ((q ^ (r & 7)) << 4)) = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
}

// The 2-D rope on one 80-wide q or k head held in registers: pair (d, d+40) turns by the angle
// of dim d, row position h for d < 20, column w for d >= 20. Two dims at a time (d and d + 1 lie on
// the same side of 20) in packed fp32x2, like the GELU above.
__device__ __forceinline__ void rope_head(float *v, int hw, const float2 *cs) {
    const float2 *ch = cs + (hw >> 16) * 20;
    const float2 *cw = cs + (hw & 0xFFFF) * 20;
#pragma unroll
    for (int d = 0; d < 40; d += 2) {
        const float2 a = __ldg(d < 20 ? ch + d : cw + (d - 20));       // (cos, sin) of dim d
        const float2 b = __ldg(d < 20 ? ch + d + 1 : cw + (d - 19));   // and of dim d + 1
        float t0, t1, u0, u1;
        fmul2(t0, t1, v[d], v[d + 1], a.x, b.x);              // x0 cos
        fmul2(u0, u1, v[d + 40], v[d + 41], a.x, b.x);        // x1 cos
        ffma2(u0, u1, v[d], v[d + 1], a.y, b.y, u0, u1);      // x1 cos + x0 sin
        ffma2(t0, t1, v[d + 40], v[d + 41], -a.y, -b.y, t0, t1);   // x0 cos - x1 sin
        v[d] = t0;
        v[d + 1] = t1;
        v[d + 40] = u0;
        v[d + 41] = u1;
    }
}

// instruction descriptor of kind::f8f6f4 with E4M3 A and B (format code 0), fp32 D
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
    return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

template <int BN, int EPI, bool F8>
__global__ void __launch_bounds__(GemmCfg<BN, EPI, F8>::THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb,
                   const __grid_constant__ CUtensorMap tmc, GemmParams p) {
    using S = GemmShape<BN>;
    using C = GemmCfg<BN, EPI, F8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + S::STAGES * S::A_BYTES;
    uint8_t *sStg = sB + S::STAGES * S::B_BYTES;            // [2][STG_BYTES], 1024-aligned
    uint64_t *full = reinterpret_cast<uint64_t *>(sStg + 2 * S::STG_BYTES);
    uint64_t *empty = full + S::STAGES;
    uint64_t *tfull = empty + S::STAGES;
    uint64_t *tempty = tfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();                 // 0: issues the pair's products
    const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S::STAGES; ++s) {
            mbar_init(full + s, 1);                       // (used in CTA 0: both CTAs' loads land on it)
            mbar_init(empty + s, 1);                      // the pair's products are done with stage s
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, 8 * C::GROUPS);         // (CTA 0) every epilogue warp of the pair
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    // The previous kernel of the stream has completed from here on (the operands are its output);
    // tensor memory is taken only after it, so no CTA holds any while it waits.
    pdl_wait();
    pdl_trigger();
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, S::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                                       // both CTAs' barriers exist before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const WaitCtx wc{abort_flag, p.status};
    const int total = p.m_tiles * p.n_tiles;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch(&tma);
            tma_prefetch(&tmb);
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = cluster; tile < total; tile += n_clusters) {
                // this CTA's 128 rows of the pair's 256, and its half of the BN rows of B
                const int m0 = (tile / p.n_tiles) * 2 * kBM + static_cast<int>(rank) * kBM;
                const int n0 = (tile % p.n_tiles) * BN + static_cast<int>(rank) * (BN / 2);
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(empty + stage, phase ^ 1u, wc)) goto producer_done;
                    const uint32_t bar0 = cluster_addr(full + stage, 0);
                    if (rank == 0) mbar_expect_tx(full + stage, 2 * (S::A_BYTES + S::B_BYTES));
                    // a k-block is 128 bytes of each row: 64 bf16 or 128 E4M3 elements
                    const int kx = kb * (F8 ? 2 * kBK : kBK);
                    tma_load_2d_pair(sA + stage * S::A_BYTES, &tma, bar0, kx, m0);
                    tma_load_2d_pair(sB + stage * S::B_BYTES, &tmb, bar0, kx, n0);
                    if (++stage == S::STAGES) { stage = 0; phase ^= 1u; }
                }
            }
        producer_done:;
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = F8 ? idesc_e4m3(2 * kBM, BN) : idesc_bf16(2 * kBM, BN, false, false);
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            for (int tile = cluster; tile < total; tile += n_clusters, ++local) {
                const int acc = local & 1;
                const uint32_t acc_phase = (local >> 1) & 1;
                if (!mbar_wait(tempty + acc, acc_phase ^ 1u, wc)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * S::ACC_STRIDE;
                bool ok = true;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(full + stage, phase, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sA + stage * S::A_BYTES);
                    const uint32_t b_addr = smem_u32(sB + stage * S::B_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        // +32 bytes per K step (16 bf16 or 32 E4M3) inside the 128-byte swizzle atom
                        const uint64_t da = smem_desc(a_addr + k * 32, 16, 1024, kSwizzle128B);
                        const uint64_t db = smem_desc(b_addr + k * 32, 16, 1024, kSwizzle128B);
                        if (F8) mma_e4m3_ss_pair(d_tmem, da, db, idesc, (kb | k) != 0 ? 1u : 0u);
                        else mma_bf16_ss_pair(d_tmem, da, db, idesc, (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair(empty + stage, 0x3);
                    if (++stage == S::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit_pair(tfull + acc, 0x3);
            }
        }
    } else {
        const int grp = (warp - 2) >> 2;                        // epilogue group
        const int quarter = warp & 3;   // TMEM lanes [32*quarter, 32*quarter+32) belong to this warp
        const int r = quarter * 32 + lane;                      // row inside the tile
        const bool leader = threadIdx.x == 64 + 128 * grp;      // issues the group's TMA stores
        int sc = 0;                                             // staging chunks used so far
        // Before refilling one of the group's staging buffers, the store that last read it must be
        // done.
        auto stage_acquire = [&]() {
            if (leader && sc >= C::NBUF) bulk_wait_read<C::NBUF - 1>();
            named_bar_sync(kEpiBarrier + grp, 128);
            return sStg + (grp * C::NBUF + sc % C::NBUF) * S::STG_BYTES;
        };
        auto stage_publish = [&]() {
            fence_proxy_async_smem();
            named_bar_sync(kEpiBarrier + grp, 128);
        };
        const uint32_t tempty0 = cluster_addr(tempty, 0);   // CTA 0's accumulator-free barriers
        // this warp's share of the accumulator is read: one arrival per warp on CTA 0's barrier
        auto release_acc = [&](int acc) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty0 + acc * 8);
        };
        int local = 0;
        for (int tile = cluster; tile < total; tile += n_clusters, ++local) {
            const int acc = local & 1;
            const uint32_t acc_phase = (local >> 1) & 1;
            if (!mbar_wait(tfull + acc, acc_phase, wc)) break;
            tc_fence_after();
            const int m0 = (tile / p.n_tiles) * 2 * kBM + static_cast<int>(rank) * kBM, n0 = (tile % p.n_tiles) * BN;
            const uint32_t t0 = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * S::ACC_STRIDE;
            if (EPI == VIT_EPI_QKV_ROPE) {
#pragma unroll 1
                for (int hh = grp; hh < BN / 80; hh += C::GROUPS) {
                    uint32_t u[80];
#pragma unroll
                    for (int c = 0; c < 5; ++c) tmem_ld16(t0 + hh * 80 + c * 16, u + c * 16);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 5; ++c) reg_fence16(u + c * 16);
                    if (hh + C::GROUPS >= BN / 80) release_acc(acc);   // this warp's reads are done
                    float v[80];
#pragma unroll
                    for (int j = 0; j < 80; ++j) v[j] = __uint_as_float(u[j]);
                    const int col0 = n0 + hh * 80;
                    const int row = m0 + r;
                    if (F8) scale_cols<80>(v, row < p.M ? __ldg(p.a_scale + row) : 0.0f, p.b_scale, col0, p.N);
                    add_bias<80>(v, p.bias, col0, p.N);
                    if (col0 < 2 * VIT_WIDTH) rope_head(v, row < p.M ? p.pos[row] : 0, p.rope_cs);
                    uint8_t *stg = stage_acquire();
                    // five 32-byte-swizzled boxes of 16 columns: the 16-byte half h of row r goes
                    // to half h ^ ((r >> 2) & 1)
#pragma unroll
                    for (int c = 0; c < 5; ++c) {
                        uint8_t *rowp = stg + c * 4096 + r * 32;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const float *x = v + 16 * c + 8 * h;
                            *reinterpret_cast<uint4 *>(rowp + ((h ^ ((r >> 2) & 1)) << 4)) =
                                make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                                           pack_bf16x2(x[6], x[7]));
                        }
                    }
                    stage_publish();
                    if (leader) {
#pragma unroll
                        for (int c = 0; c < 5; ++c) tma_store_2d(&tmc, stg + c * 4096, col0 + 16 * c, m0);
                        bulk_commit();
                    }
                    ++sc;
                }
            } else if (EPI == VIT_EPI_STORE_F32 || EPI == VIT_EPI_ADD_F32) {
#pragma unroll 1
                for (int c = grp; c < BN / 32; c += C::GROUPS) {   // 32 fp32 columns = a 128-byte row
                    uint32_t u[32];
                    tmem_ld32(t0 + c * 32, u);
                    tmem_wait_ld();
                    reg_fence32(u);
                    if (c + C::GROUPS >= BN / 32) release_acc(acc);
                    const int col0 = n0 + c * 32;
                    if (col0 < p.N) {                   // uniform across the CTA
                        float v[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(u[j]);
                        if (F8) scale_cols<32>(v, m0 + r < p.M ? __ldg(p.a_scale + m0 + r) : 0.0f, p.b_scale, col0, p.N);
                        add_bias<32>(v, p.bias, col0, p.N);
#pragma unroll
                        for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(v[j]);
                        uint8_t *stg = stage_acquire();
                        stage_row128(stg, r, u);
                        stage_publish();
                        if (leader) {
                            if (EPI == VIT_EPI_ADD_F32) tma_reduce_add_2d(&tmc, stg, col0, m0);
                            else tma_store_2d(&tmc, stg, col0, m0);
                            bulk_commit();
                        }
                        ++sc;
                    }
                }
            } else {
#pragma unroll 1
                for (int c = grp; c < BN / 64; c += C::GROUPS) {   // 64 bf16 columns = a 128-byte row
                    uint32_t u[64];
                    tmem_ld32(t0 + c * 64, *reinterpret_cast<uint32_t(*)[32]>(u));
                    tmem_ld32(t0 + c * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(u + 32));
                    tmem_wait_ld();
                    reg_fence32(u);
                    reg_fence32(u + 32);
                    if (c + C::GROUPS >= BN / 64) release_acc(acc);
                    const int col0 = n0 + c * 64;
                    if (col0 < p.N) {
                        float v[64];
#pragma unroll
                        for (int j = 0; j < 64; ++j) v[j] = __uint_as_float(u[j]);
                        if (F8) scale_cols<64>(v, m0 + r < p.M ? __ldg(p.a_scale + m0 + r) : 0.0f, p.b_scale, col0, p.N);
                        add_bias<64>(v, p.bias, col0, p.N);
                        uint32_t w[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            float a = v[2 * j], b = v[2 * j + 1];
                            if (EPI == VIT_EPI_GELU_BF16) gelu_erf2(a, b);
                            w[j] = pack_bf16x2(a, b);
                        }
                        uint8_t *stg = stage_acquire();
                        stage_row128(stg, r, w);
                        stage_publish();
                        if (leader) {
                            tma_store_2d(&tmc, stg, col0, m0);
                            bulk_commit();
                        }
                        ++sc;
                    }
                }
            }
        }
        if (leader) bulk_wait<0>();             // every store has landed before the CTA exits
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) __nanosleep(200000);   // let copies already in flight land before exit
    cluster_sync();                          // no remote arrival or product still targets either CTA
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
    }
}

}  // namespace vitk

namespace vith {

int gemm_make_a_map(CUtensorMap *map, const void *A, int64_t M, int K, bool f8) {
    // 128-byte boxes along K: 64 bf16 or 128 E4M3 codes
    if (f8)
        return tmap_2d(map, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, static_cast<uint64_t>(K), 2 * vitk::kBK,
                       vitk::kBM, CU_TENSOR_MAP_SWIZZLE_128B);
    return tmap_2d(map, A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, M, static_cast<uint64_t>(K) * 2, vitk::kBK,
                   vitk::kBM, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Narrow tiles (256 x 128) when the 256 x 256 tiles of a product would not fill the device's SM
// pairs once (a single small image: M = 1024 gives 20 tiles of N = 1280 for 74 pairs).
bool gemm_use_narrow(int64_t M, int N, int epilogue) {
    if (epilogue == VIT_EPI_QKV_ROPE) return false;   // the rope epilogue needs whole 80-wide heads
    const int64_t tiles = ((M + 2 * vitk::kBM - 1) / (2 * vitk::kBM)) * ((N + 255) / 256);
    return tiles < device_sm_count() / 2;
}

int gemm_make_b_map(CUtensorMap *map, const void *B, int N, int K, int epilogue, bool f8, bool narrow) {
    const uint32_t bn = (epilogue == VIT_EPI_QKV_ROPE) ? 240 : (narrow ? 128 : 256);   // each CTA of a pair loads half
    if (f8)
        return tmap_2d(map, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N, static_cast<uint64_t>(K), 2 * vitk::kBK,
                       bn / 2, CU_TENSOR_MAP_SWIZZLE_128B);
    return tmap_2d(map, B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, N, static_cast<uint64_t>(K) * 2, vitk::kBK, bn / 2,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

int gemm_make_c_map(CUtensorMap *map, void *C, int64_t M, int N, int epilogue) {
    switch (epilogue) {
        case VIT_EPI_STORE_F32:
        case VIT_EPI_ADD_F32:
            return tmap_2d(map, C, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, N, M, static_cast<uint64_t>(N) * 4, 32,
                           vitk::kBM, CU_TENSOR_MAP_SWIZZLE_128B);
        case VIT_EPI_QKV_ROPE:
            return tmap_2d(map, C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M, static_cast<uint64_t>(N) * 2, 16,
                           vitk::kBM, CU_TENSOR_MAP_SWIZZLE_32B);
        default:
            return tmap_2d(map, C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M, static_cast<uint64_t>(N) * 2, 64,
                           vitk::kBM, CU_TENSOR_MAP_SWIZZLE_128B);
    }
}

template <int BN, int EPI, bool F8>
static int launch_one(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tc, const vitk::GemmParams &p,
                      cudaStream_t s) {
    using S = vitk::GemmShape<BN>;
    using C = vitk::GemmCfg<BN, EPI, F8>;
    static bool configured[64] = {};   // the attribute is set once per device
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !configured[dev]) {
        if (cudaFuncSetAttribute(vitk::gemm_tc_kernel<BN, EPI, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM) !=
            cudaSuccess)
            return VIT_ERR_CUDA;
        if (dev < 64) configured[dev] = true;
    }
    static int max_clusters[64] = {};   // pairs that fit on the device at once (set with the attribute)
    if (dev < 64 && max_clusters[dev] == 0) {
        cudaLaunchConfig_t cfg{};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.blockDim = dim3(C::THREADS);
        cfg.dynamicSmemBytes = S::SMEM;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cfg.gridDim = dim3(2 * 74);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, vitk::gemm_tc_kernel<BN, EPI, F8>, &cfg) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = device_sm_count() / 2;
        }
        max_clusters[dev] = n;
    }
    const int total = p.m_tiles * p.n_tiles;
    const int pairs = dev < 64 ? max_clusters[dev] : device_sm_count() / 2;
    const dim3 grid(2 * (total < pairs ? total : pairs));
    if (launch_pdl(vitk::gemm_tc_kernel<BN, EPI, F8>, grid, dim3(C::THREADS), S::SMEM, s, 2, ta, tb, tc, p) !=
        cudaSuccess)
        return VIT_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? VIT_OK : VIT_ERR_CUDA;
}

int gemm_launch(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tc, const void *bias, int64_t M,
                int N, int K, int epilogue, const int32_t *pos, const float *rope_cs, int32_t *status,
                cudaStream_t s, const float *a_scale, const float *b_scale) {
    if (M <= 0) return VIT_OK;
    const bool f8 = a_scale != nullptr;
    if (f8 && (!b_scale || K % 16)) return VIT_ERR_ARG;
    vitk::GemmParams p{};
    p.bias = static_cast<const __nv_bfloat16 *>(bias);
    p.a_scale = a_scale;
    p.b_scale = b_scale;
    p.pos = pos;
    p.rope_cs = reinterpret_cast<const float2 *>(rope_cs);
    p.status = status;
    p.M = static_cast<int>(M);
    p.N = N;
    p.K = K;
    p.m_tiles = static_cast<int>((M + 2 * vitk::kBM - 1) / (2 * vitk::kBM));
    const int kblk = f8 ? 2 * vitk::kBK : vitk::kBK;   // elements per 128-byte k-block
    p.k_blocks = (K + kblk - 1) / kblk;
    if (gemm_use_narrow(M, N, epilogue)) {   // the B map was made with narrow = true
        p.n_tiles = (N + 127) / 128;
        switch (epilogue) {
            case VIT_EPI_STORE_F32:
                return f8 ? launch_one<128, VIT_EPI_STORE_F32, true>(ta, tb, tc, p, s)
                          : launch_one<128, VIT_EPI_STORE_F32, false>(ta, tb, tc, p, s);
            case VIT_EPI_ADD_F32:
                return f8 ? launch_one<128, VIT_EPI_ADD_F32, true>(ta, tb, tc, p, s)
                          : launch_one<128, VIT_EPI_ADD_F32, false>(ta, tb, tc, p, s);
            case VIT_EPI_STORE_BF16:
                return f8 ? launch_one<128, VIT_EPI_STORE_BF16, true>(ta, tb, tc, p, s)
                          : launch_one<128, VIT_EPI_STORE_BF16, false>(ta, tb, tc, p, s);
            case VIT_EPI_GELU_BF16:
                return f8 ? launch_one<128, VIT_EPI_GELU_BF16, true>(ta, tb, tc, p, s)
                          : launch_one<128, VIT_EPI_GELU_BF16, false>(ta, tb, tc, p, s);
            default:
                return VIT_ERR_ARG;
        }
    }
    switch (epilogue) {
        case VIT_EPI_QKV_ROPE:
            p.n_tiles = N / 240;
            return f8 ? launch_one<240, VIT_EPI_QKV_ROPE, true>(ta, tb, tc, p, s)
                      : launch_one<240, VIT_EPI_QKV_ROPE, false>(ta, tb, tc, p, s);
        case VIT_EPI_STORE_F32:
            p.n_tiles = (N + 255) / 256;
            return f8 ? launch_one<256, VIT_EPI_STORE_F32, true>(ta, tb, tc, p, s)
                      : launch_one<256, VIT_EPI_STORE_F32, false>(ta, tb, tc, p, s);
        case VIT_EPI_ADD_F32:
            p.n_tiles = (N + 255) / 256;
            return f8 ? launch_one<256, VIT_EPI_ADD_F32, true>(ta, tb, tc, p, s)
                      : launch_one<256, VIT_EPI_ADD_F32, false>(ta, tb, tc, p, s);
        case VIT_EPI_STORE_BF16:
            p.n_tiles = (N + 255) / 256;
            return f8 ? launch_one<256, VIT_EPI_STORE_BF16, true>(ta, tb, tc, p, s)
                      : launch_one<256, VIT_EPI_STORE_BF16, false>(ta, tb, tc, p, s);
        case VIT_EPI_GELU_BF16:
            p.n_tiles = (N + 255) / 256;
            return f8 ? launch_one<256, VIT_EPI_GELU_BF16, true>(ta, tb, tc, p, s)
                      : launch_one<256, VIT_EPI_GELU_BF16, false>(ta, tb, tc, p, s);
        default:
            return VIT_ERR_ARG;
    }
}

}  // namespace vith
