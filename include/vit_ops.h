/*
 * vit_ops.h -- kernel-level entry points of the B200 vision encoder.
 *
 * Each function launches ONE of the kernels vit_encode chains together, on caller-owned device
 * buffers, asynchronously on `stream`. They exist so that every step of the encoder can be
 * checked and timed on its own; vit_encode does not go through them. Same conventions as
 * vit.h: device pointers, 16-byte alignment for every matrix, bf16 row-major, host-side
 * argument errors returned before launch, device-side errors (VIT_ERR_TIMEOUT) written to
 * *dev_status when it is not NULL.
 */
#ifndef RESOLUTION_VIT_VISION_B200_VIT_OPS_H
#define RESOLUTION_VIT_VISION_B200_VIT_OPS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Epilogues of the tensor-core GEMM C = A B^T (+ bias): A bf16 [M, K], B bf16 [N, K]
 * (nn.Linear weight), fp32 accumulation in tensor memory. */
#define VIT_EPI_STORE_F32   0  /* C fp32 [M, N]  = acc + bias       (patch embed -> residual)  */
#define VIT_EPI_ADD_F32     1  /* C fp32 [M, N] += acc + bias       (out-proj, fc2 residual)   */
#define VIT_EPI_STORE_BF16  2  /* C bf16 [M, N]  = acc + bias       (merger output)            */
#define VIT_EPI_GELU_BF16   3  /* C bf16 [M, N]  = GELU_erf(acc + bias)   (fc1, merger fc 1)   */
#define VIT_EPI_QKV_ROPE    4  /* C bf16 [M, 3840] = acc + bias, then the 2-D rope on the q and
                                  k columns (< 2560) of every 80-wide head; needs pos, rope_cs */

/* GEMM: the patch-embed, QKV, out-proj, fc1, fc2 and merger products ("Qwen2-VL (Native-
 * Resolution VLM)", Structure table rows 2, 4-6; "Qwen2-VL" Qwen2VLModel table widths).
 * Requirements: M >= 1, 16 <= N, N % 16 == 0, K >= 8, K % 8 == 0 (row pitch a multiple of 16
 * bytes); QKV_ROPE needs N == 3840. bias: bf16 [N] or NULL. pos: int32 [M], (h << 16) | w of
 * each row (QKV_ROPE only). rope_cs: fp32 [n_pos][20][2] (cos, sin) from vit_op_rope_table,
 * n_pos > max(h, w). */
int vit_op_gemm(const void *A, const void *B, const void *bias, void *C, int64_t M, int N, int K,
                int epilogue, const int32_t *pos, const float *rope_cs, int32_t *dev_status,
                void *stream);

/* The fp8 tower's product (vit.h, vit_layer_fp8): C = (a_scale[m] * b_scale[n]) * (A B^T)[m, n]
 * (+ bias) with A E4M3 codes [M, K], B E4M3 codes [N, K] (one byte each), a_scale fp32 [M],
 * b_scale fp32 [N] (16-byte aligned), the same epilogues as vit_op_gemm (the scales are applied
 * to the fp32 accumulator first). Requirements as vit_op_gemm, and K % 16 == 0. */
int vit_op_gemm_fp8(const void *A, const float *a_scale, const void *B, const float *b_scale, const void *bias,
                    void *C, int64_t M, int N, int K, int epilogue, const int32_t *pos, const float *rope_cs,
                    int32_t *dev_status, void *stream);

/* LayerNorm of fp32 rows of 1280 (as vit_op_layernorm), the output row quantised as by
 * vit_quantize_fp8: codes [rows, 1280] bytes, scales fp32 [rows] (one power of two per row). */
int vit_op_layernorm_fp8(const float *X, const void *gamma, const void *beta, void *codes, float *scales,
                         int64_t rows, float eps, void *stream);

/* Rope table ("Qwen2-VL (Native-Resolution VLM)", Structure row 3, 2D RoPE; LiteRT-LM card,
 * Conversion notes: precomputed 2-D rope): cs[p][k] = (cos(p f_k), sin(p f_k)), f_k =
 * 10000^(-2k/40), k < 20, p < n_pos. cs: fp32 [n_pos * 40]. */
int vit_op_rope_table(float *cs, int n_pos, void *stream);

/* Positions of the packed patches: pos[r] = (h << 16) | w of row r inside its frame, for the
 * images of grid_thw (HOST [n_images, 3]) packed in patch_order (0 block, 1 raster). For
 * patch_order 1, merge_row[r] (int32 [P], or NULL) receives the row that patch r takes in the
 * 2x2-block order used by the merger; for patch_order 0 it is r. */
int vit_op_positions(const int32_t *grid_thw, int n_images, int patch_order, int32_t *pos,
                     int32_t *merge_row, void *stream);

/* LayerNorm over rows of 1280 ("Qwen2-VL (Native-Resolution VLM)", ViT Block rows; exported
 * PatchMerger's LayerNorm): Y[out_row[r]] = (X[r] - mean) / sqrt(var + eps) * gamma + beta,
 * X fp32 [rows, 1280], Y bf16 [rows, 1280], gamma bf16 [1280], beta bf16 [1280] or NULL,
 * out_row int32 [rows] or NULL (identity). */
int vit_op_layernorm(const float *X, const void *gamma, const void *beta, void *Y, int64_t rows,
                     float eps, const int32_t *out_row, void *stream);

/* Varlen block-diagonal attention ("Qwen2-VL-2B-Instruct -- LiteRT-LM", Vision row: full
 * attention; Conversion notes: packed patches with cu_seqlens, one image = one sequence).
 * qkv: bf16 [P, 3840] = q | k | v, each [16 heads][80] (rope already applied to q and k).
 * cu_seqlens: HOST int32 [n_seg + 1], cu_seqlens[0] = 0, cu_seqlens[n_seg] = P, non-decreasing;
 * empty segments are allowed. out: bf16 [P, 1280], out = softmax(q k^T / sqrt(80)) v per
 * segment and head. The (segment, 128-query tile) list is scheduled longest segment first. */
int vit_op_attention(const void *qkv, int64_t P, const int32_t *cu_seqlens, int n_seg, void *out,
                     int32_t *dev_status, void *stream);

/* The exponential that the attention softmax computes on the FMA pipe for a share of its scores
 * (no counterpart on the pages, which fix only softmax itself: "Qwen2-VL-2B-Instruct --
 * LiteRT-LM", Vision row, full attention). y[i] = 2^x[i] for x, y fp32 [n] device, n >= 0: range
 * reduction x = j + f (j = rint x, |f| <= 1/2), 2^f by a degree-3 minimax polynomial, j added to
 * the exponent; relative error <= 7.5e-5 for x in [-125, 127); 0 for x <= -127.5 (and -inf);
 * between those, 0 or a value of at most 2^-124 (2^f's exponent field may underflow there). |x| must stay below 2^22 (inputs beyond are not
 * rejected and give meaningless results). */
int vit_op_exp2_fma(const float *x, float *y, int64_t n, void *stream);

/* Window order of the windowed (Qwen2.5-VL) tower ("Qwen2.5-VL-7B-Instruct", inference-research
 * model record, architecture note: 112-px windows). Rows in window order run, per image and frame,
 * over the windows of window x window patches (window even, >= 2) in raster order, inside a window
 * over its 2x2 merge groups in raster order, inside a group (dh, dw). For each window-order row r:
 * pos[r] = (h << 16) | w inside its frame, src_row[r] = the row holding that patch when the images
 * are packed in patch_order (0 block, 1 raster), merge_row[r] = its row in 2x2-block order (int32
 * [P] device buffers each). win_table: int32 [2 * n_windows] device (n_windows <= P / 4), receives
 * (first row, number of rows) of every window in window order; *n_windows (HOST int) receives the
 * number of windows. All outputs required. grid_thw: HOST [n_images, 3]. */
int vit_op_window_positions(const int32_t *grid_thw, int n_images, int patch_order, int window, int32_t *pos,
                            int32_t *merge_row, int32_t *src_row, int32_t *win_table, int *n_windows,
                            void *stream);

/* dst[r, :] = src[src_row[r], :] for rows of row_bytes bytes (a multiple of 16; src, dst
 * 16-byte aligned). src_row: int32 [rows] device, each in range of src (not checked). */
int vit_op_gather_rows(const void *src, const int32_t *src_row, void *dst, int64_t rows, int row_bytes,
                       void *stream);

/* Attention inside windows (same architecture note): qkv bf16 [P, 3840]; win_table: int32
 * [2 * n_windows] device, (first row, rows) of each window as vit_op_window_positions writes it
 * (windows of at most 8 x 8 patches: rows <= 64; the table is trusted, the kernel only keeps its
 * stores below row P). Every window is one segment, attended exactly as by vit_op_attention.
 * out: bf16 [P, 1280], same row order. dev_status as for vit_op_attention. */
int vit_op_window_attention(const void *qkv, int64_t P, const int32_t *win_table, int n_windows, void *out,
                            int32_t *dev_status, void *stream);

/* Bounded-wait self-test (the failure path of every tensor-core kernel's mbarrier waits, run on
 * purpose and without any fault): one CTA waits on a barrier nothing arrives on; each wait gives
 * up after limit_cycles SM cycles (1000 .. 4e9), the kernel writes VIT_ERR_TIMEOUT to *dev_status
 * (device int32, required) and ends normally, leaving the context usable. */
int vit_op_wait_selftest(int32_t *dev_status, int64_t limit_cycles, void *stream);

#ifdef __cplusplus
}
#endif
#endif
