/*
 * vit_decoder.h -- C ABI of the two decoder-side steps that consume the vision encoder's output.
 *
 * What they compute (the passages that define them):
 *   - mrope_apply: "Qwen2-VL" (ZeroModels Keras docs), intro (the decoder's rotary embedding is split
 *     across time / height / width) and Qwen2VLModel table (rope_theta 1e6, mrope_section
 *     (16, 24, 24)); "Qwen2.5-VL-7B-Instruct" (inference-research model record): 28 query / 4
 *     key-value heads of head_dim 128, the t and h indices share the head-dim halves with w;
 *     "Qwen2-VL-2B-Instruct -- LiteRT-LM" card, M-RoPE note: text tokens reduce to 1-D positions.
 *   - scatter_vision_tokens: "Qwen2-VL (Native-Resolution VLM)", Structure table rows 6-10 (merged
 *     image tokens and embedded text tokens form one sequence of the decoder's width); "Qwen2-VL",
 *     several images in one conversation (each marker expands to its image's own token count).
 *
 * Conventions as in vit.h: device pointers unless marked HOST, bf16 row-major, asynchronous on
 * `stream`, argument errors returned before any launch, data errors written to dev_status.
 */
#ifndef RESOLUTION_VIT_VISION_B200_VIT_DECODER_H
#define RESOLUTION_VIT_VISION_B200_VIT_DECODER_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* 3-D M-RoPE, in place. q: bf16 [L, n_heads, head_dim], k: bf16 [L, n_kv_heads, head_dim] (either
 * may be NULL with its head count 0); pos: int32 [3, L], the (t, h, w) ids mrope_index writes.
 * head_dim even, 16..256, a multiple of 16; sections: HOST int32 [3] with sum = head_dim / 2 (16,
 * 24, 24 for head_dim 128). Frequency j < head_dim / 2 is theta^(-2j / head_dim); it is driven by
 * pos[t] for the first sections[0] frequencies, pos[h] for the next sections[1], pos[w] for the
 * rest, and turns dims (j, j + head_dim/2) of every head: x_j' = x_j cos - x_(j+D/2) sin,
 * x_(j+D/2)' = x_(j+D/2) cos + x_j sin. Angles in double precision, the turn in fp32, rounded to
 * bf16. Pointers 16-byte aligned (VIT_ERR_ALIGN). VIT_ERR_ARG on bad sizes or sections. */
int mrope_apply(void *q, int n_heads, void *k, int n_kv_heads, int head_dim, const int32_t *pos, int64_t L,
                double theta, const int32_t *sections, void *stream);

/* The decoder's input sequence: out[i] = vision[k] when input_ids[i] is the k-th image or video
 * placeholder (VIT_IMAGE_TOKEN_ID / VIT_VIDEO_TOKEN_ID, counted in order), else
 * embed_table[input_ids[i]]. input_ids: int32 [L]; embed_table: bf16 [vocab, dim]; vision: bf16
 * [n_vision, dim] (vit_encode's output, the images in prompt order); out: bf16 [L, dim]. dim a
 * multiple of 8; pointers 16-byte aligned. Data errors (placeholder count != n_vision, a text id
 * outside [0, vocab)) write VIT_ERR_TOKENS to dev_status (int32 [1] device, or NULL) and leave
 * the offending rows unwritten; every other row is written. L <= 2^18; L = 0 with n_vision = 0 is a
 * no-op that reads no pointer. */
int scatter_vision_tokens(const int32_t *input_ids, int64_t L, const void *embed_table, int64_t vocab, int dim,
                          const void *vision, int64_t n_vision, void *out, int32_t *dev_status, void *stream);

#ifdef __cplusplus
}
#endif
#endif
