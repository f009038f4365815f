// internal.h -- host-side declarations shared by the C ABI (api.cpp) and the kernel files.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include <utility>
#include <vector>

#include "../../include/vit.h"
#include "../../include/vit_decoder.h"
#include "../../include/vit_ops.h"

namespace vith {

// Launches kernel k with programmatic stream serialisation: k may start while the previous kernel
// of stream s finishes, so every such kernel calls pdl_wait() (ptx.cuh) before it touches global
// memory. cluster_x > 1 also launches it in clusters of that many CTAs.
template <typename... P, typename... A>
inline cudaError_t launch_pdl(void (*k)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster_x,
                              A &&...args) {
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(cluster_x);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = cluster_x > 1 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, k, std::forward<A>(args)...);
}

// ---- tensor maps (driver entry point fetched through the runtime, no -lcuda needed)
int tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes, uint64_t inner,
            uint64_t outer, uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_outer,
            CUtensorMapSwizzle swizzle);

int device_sm_count();
int check_device();   // VIT_OK when the current device is sm_100

// ---- GEMM (gemm.cu). A bf16 [M, K], B bf16 [N, K]. The B map may be prebuilt (weights).
// f8: E4M3 codes (one byte per element) instead of bf16
int gemm_make_a_map(CUtensorMap *map, const void *A, int64_t M, int K, bool f8 = false);
// narrow: the map of 256 x 128 tiles, which gemm_launch uses when gemm_use_narrow(M, N, epilogue)
int gemm_make_b_map(CUtensorMap *map, const void *B, int N, int K, int epilogue, bool f8 = false,
                    bool narrow = false);
bool gemm_use_narrow(int64_t M, int N, int epilogue);
// C [M, N]: fp32 for STORE_F32 / ADD_F32 (the output is written, or added, by TMA), else bf16
int gemm_make_c_map(CUtensorMap *map, void *C, int64_t M, int N, int epilogue);
// The B map must be made with narrow = gemm_use_narrow(M, N, epilogue).
// a_scale != NULL selects the E4M3 product: A and B are codes (maps made with f8), a_scale [M] and
// b_scale [N] their per-row power-of-two scales, applied to the accumulator before the bias
int gemm_launch(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tc, const void *bias, int64_t M,
                int N, int K, int epilogue, const int32_t *pos, const float *rope_cs, int32_t *status,
                cudaStream_t s, const float *a_scale = nullptr, const float *b_scale = nullptr);

// ---- attention (attention.cu). qkv bf16 [P, 3840].
struct AttnMaps {
    CUtensorMap q, kv;
};
int attn_make_maps(AttnMaps *m, const void *qkv, int64_t P);
// cu_seqlens: HOST [n_seg + 1]; the (segment, q-tile) work list is built here, longest first
int attn_launch(const AttnMaps &tqkv, const int32_t *cu_seqlens, int n_seg, void *out, int32_t *status,
                cudaStream_t s);

// the FMA-pipe exponential of the attention softmax, elementwise (parity checks)
int exp2_fma_launch(const float *x, float *y, int64_t n, cudaStream_t s);

// ---- E4M3 quantisation (fp8.cu): per-row power-of-two scales, codes rounded to nearest even
int quantize_rows_launch(const void *x, int64_t rows, int cols, void *codes, float *scales, cudaStream_t s);
int layernorm_fp8_launch(const float *X, const void *gamma, const void *beta, void *codes, float *scales,
                         int64_t rows, float eps, cudaStream_t s);

// ---- small kernels (misc.cu)
int layernorm_launch(const float *X, const void *gamma, const void *beta, void *Y, int64_t rows, float eps,
                     const int32_t *out_row, cudaStream_t s);
int rope_table_launch(float *cs, int n_pos, cudaStream_t s);
// grid_thw: HOST [n_images, 3] (validated); the table travels as a kernel parameter
int positions_launch(const int32_t *grid_thw, int n_images, int64_t P, int patch_order, int32_t *pos,
                     int32_t *merge_row, cudaStream_t s);
// the same launches with their host-side tables on the stack (no heap use)
int attn_launch_stack(const AttnMaps &tqkv, const int32_t *cu_seqlens, int n_seg, void *out, int32_t *status,
                      cudaStream_t s);
int positions_launch_stack(const int32_t *grid_thw, int n_images, int64_t P, int patch_order, int32_t *pos,
                           int32_t *merge_row, cudaStream_t s);
// ---- windowed attention (window.cu); window = side in patches (even)
int window_cu_seqlens(const int32_t *grid_thw, int n_images, int window, std::vector<int32_t> &cu);
int window_count(const int32_t *grid_thw, int n_images, int window);
// win_tab: int32 [2 * window_count] device, receives (first row, rows) per window
int window_positions_launch(const int32_t *grid_thw, int n_images, int64_t P, int patch_order, int window,
                            int32_t *pos, int32_t *merge_row, int32_t *src_row, int32_t *win_tab, cudaStream_t s);
int gather_rows_launch(const void *src, const int32_t *src_row, void *dst, int64_t rows, int row_bytes,
                       cudaStream_t s);
struct WinMaps {
    CUtensorMap m32, m128;
};
int win_make_maps(WinMaps *m, const void *qkv, int64_t P);
// windows of at most 64 rows, from the table window_positions_launch wrote
int win_attn_launch(const WinMaps &m, const int32_t *win_tab, int n_windows, int64_t P, void *out, int32_t *status,
                    cudaStream_t s);
// ---- decoder-side steps (decoder.cu)
int mrope_apply_launch(void *q, int Hq, void *k, int Hk, int D, const int32_t *pos, int64_t L, double theta,
                       const int32_t *sections, cudaStream_t s);
int scatter_launch(const int32_t *ids, int64_t L, const void *table, int64_t vocab, int dim, const void *vision,
                   int64_t n_vision, void *out, int32_t *status, cudaStream_t s);
int wait_selftest_launch(int32_t *status, long long limit, cudaStream_t s);
int mrope_launch(const int32_t *ids, int64_t L, const int32_t *grid_thw, int n_grids, int32_t *out, int32_t *delta,
                 int32_t *status, cudaStream_t s);

}  // namespace vith
