/*
 * vit.h -- C ABI of the B200 (sm_100a) Qwen2-VL native-resolution vision encoder and the
 * decoder's 3-D M-RoPE position-id builder.
 *
 * What the library computes (the passages that define it):
 *   - "Qwen2-VL" (ZeroModels Keras docs), API, Qwen2VLVisionModel: patch-embed -> rotary blocks
 *     -> 2x2 merger; Qwen2VLModel table: vision depth 32, width 1280, 16 heads, mlp ratio 4,
 *     patch 14, spatial merge 2, temporal patch 2, 3 channels, the special token ids and
 *     mrope_section (16, 24, 24).
 *   - "Qwen2-VL (Native-Resolution VLM)", Structure table (Patchify 14x14 -> 2D RoPE -> ViT
 *     blocks -> Patch Merger 2x2) and its exported PatchMerger (LayerNorm, 2x2 group, Linear,
 *     GELU, Linear).
 *   - "Qwen2-VL-2B-Instruct -- LiteRT-LM", Conversion notes: packed patches with cu_seqlens,
 *     per-image full attention, 2-D rope per patch, Conv3d patch embed over 2 frames, the 2x2
 *     merge of raster patches by strided slices; M-RoPE note (text tokens get 1-D positions).
 *
 * Conventions
 *   - Every tensor argument is caller-owned DEVICE memory unless the comment says "host".
 *     The library never frees caller memory. bf16 = IEEE bfloat16, row-major, nn.Linear
 *     weights are [out_features, in_features].
 *   - Device pointers given to vit_encode / vit_weights_create must be 16-byte aligned
 *     (the kernels read them with TMA); misaligned pointers return VIT_ERR_ALIGN.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *     default stream) except vit_device_status, which synchronises that stream.
 *   - The encoder's kernels are launched with programmatic stream serialisation: each may start
 *     while the stream's previous kernel drains, and waits for that kernel to complete before it
 *     reads or writes any memory, so stream order holds for every caller. A kernel of the caller
 *     launched next on the stream with the same attribute may likewise start early: it must wait
 *     (griddepcontrol.wait / cudaGridDependencySynchronize) before reading the library's output.
 *   - Argument errors are returned synchronously, before anything is launched. Errors that
 *     depend on device data (a malformed M-RoPE prompt, a kernel wait that timed out) are
 *     written to a device status word and never trap.
 *   - One handle is used by one stream at a time (its workspace is shared by its calls).
 */
#ifndef RESOLUTION_VIT_VISION_B200_VIT_H
#define RESOLUTION_VIT_VISION_B200_VIT_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------------------------- */
#define VIT_OK               0
#define VIT_ERR_ARG          1   /* null pointer, bad size, bad enum value                      */
#define VIT_ERR_GRID         2   /* grid_thw row with t < 1, or h / w odd or < 2                 */
#define VIT_ERR_ALIGN        3   /* a device pointer is not 16-byte aligned                      */
#define VIT_ERR_NOMEM        4   /* workspace allocation failed                                 */
#define VIT_ERR_CUDA         5   /* a CUDA runtime / driver call failed                         */
#define VIT_ERR_TOKENS       6   /* (device) M-RoPE prompt malformed: run length != t*h*w/4,
                                    or a vision run with no grid left                           */
#define VIT_ERR_TIMEOUT      7   /* (device) a kernel's bounded wait expired; outputs invalid   */
#define VIT_ERR_UNSUPPORTED  8   /* the current device is not sm_100 (B200 class)               */
#define VIT_ERR_LIMIT        9   /* a size beyond the library's documented limits               */

/* ---- model constants ("Qwen2-VL", Qwen2VLModel table) -------------------------------------- */
#define VIT_WIDTH            1280
#define VIT_HEADS            16
#define VIT_HEAD_DIM         80
#define VIT_MLP              5120
#define VIT_PATCH_DIM        1176   /* 3 channels x 2 frames x 14 x 14, flattened (c, t, ph, pw) */
#define VIT_MERGE_DIM        5120   /* 2 x 2 x 1280                                               */
#define VIT_IMAGE_TOKEN_ID        151655
#define VIT_VIDEO_TOKEN_ID        151656
#define VIT_VISION_START_TOKEN_ID 151652
#define VIT_VISION_END_TOKEN_ID   151653

/* ---- limits -------------------------------------------------------------------------------- */
#define VIT_MAX_IMAGES       512       /* grid_thw rows per vit_encode call                     */
#define VIT_MAX_SEGMENTS     4096      /* attention segments = sum of t over the images         */
#define VIT_MAX_PATCHES      (1 << 21) /* patches per vit_encode call                           */
#define VIT_MAX_SIDE         4096      /* h and w, in patches                                   */
#define VIT_MAX_MROPE_GRIDS  1024      /* grid_thw rows per mrope_index call                    */

/* ---- weights ------------------------------------------------------------------------------- */
/* One pre-norm ViT block ("Qwen2-VL (Native-Resolution VLM)", Structure table, ViT Block rows):
 * all bf16 device pointers. Biases may be NULL (treated as zero); LayerNorm gamma must be given,
 * beta may be NULL. qkv_w is [3*1280, 1280] with q, k, v stacked in that order, head-major
 * (head h owns rows h*80 .. h*80+79 of each). */
typedef struct {
    const void *ln1_w, *ln1_b;     /* [1280]                 */
    const void *qkv_w, *qkv_b;     /* [3840, 1280], [3840]   */
    const void *proj_w, *proj_b;   /* [1280, 1280], [1280]   */
    const void *ln2_w, *ln2_b;     /* [1280]                 */
    const void *fc1_w, *fc1_b;     /* [5120, 1280], [5120]   */
    const void *fc2_w, *fc2_b;     /* [1280, 5120], [1280]   */
} vit_layer_w;

/* The fp8 variant of one block's four linears ("Qwen2-VL-2B-Instruct -- LiteRT-LM", file table:
 * the vision tower ships with 8-bit weights; correlation note: 0.90 with them). Codes: FP8 E4M3
 * (OCP "e4m3fn": bias 7, max 448, no infinities), [out, in] row-major, one byte each; scales:
 * fp32 [out], one power of two per output channel, weight = scale * code. vit_quantize_fp8 makes
 * both from bf16 weights. All device pointers, 16-byte aligned. */
typedef struct {
    const void *qkv_q;  const float *qkv_s;    /* [3840, 1280], [3840] */
    const void *proj_q; const float *proj_s;   /* [1280, 1280], [1280] */
    const void *fc1_q;  const float *fc1_s;    /* [5120, 1280], [5120] */
    const void *fc2_q;  const float *fc2_s;    /* [1280, 5120], [1280] */
} vit_layer_fp8;

typedef struct {
    int depth;                 /* number of ViT blocks, 1..64 (32 for Qwen2-VL)                  */
    int out_dim;               /* merger output width: a multiple of 16, 16..16384 (1536, 3584)  */
    float ln_eps;              /* LayerNorm epsilon (1e-6), used by every LayerNorm incl. ln_q   */
    int patch_order;           /* 0: patches of each frame in 2x2-block order (bh, bw, dh, dw);
                                  1: raster order (h, w) -- the merge then gathers 2x2 groups    */
    const void *pe_w;          /* [1280, 1176] patch-embed (Conv3d kernel flattened c,t,ph,pw)   */
    const void *pe_b;          /* [1280] or NULL                                                */
    const vit_layer_w *layers; /* HOST array [depth]; copied by vit_weights_create              */
    const void *lnq_w, *lnq_b; /* merger LayerNorm [1280]                                       */
    const void *m0_w, *m0_b;   /* merger Linear 1 [5120, 5120], [5120]                          */
    const void *m2_w, *m2_b;   /* merger Linear 2 [out_dim, 5120], [out_dim]                    */
    /* Windowed attention, the Qwen2.5-VL tower ("Qwen2.5-VL-7B-Instruct", inference-research
     * model record, architecture note: 112-px windows, full attention only at depths 7, 15, 23,
     * 31). 0 (or zero-initialised): every block attends over its whole (image, frame) segment, the
     * Qwen2-VL tower. window > 0: the side of a window in patches, even, 2..VIT_MAX_SIDE (8 =
     * 112 px); windows tile each frame from its top-left corner, border windows are cut short,
     * and a patch at (h, w) attends only to the patches of its window (h / window, w / window).
     * Windows of up to 8 x 8 patches run on a dedicated kernel; larger ones on the segment kernel. */
    int window;
    const uint8_t *full_attention; /* HOST [depth] or NULL; copied by vit_weights_create. With
                                      window > 0, block l attends over the whole frame where
                                      full_attention[l] != 0 (Qwen2.5-VL: l = 7, 15, 23, 31) */
    /* HOST array [depth] or NULL (zero-initialised: the bf16 tower). Given, every block's four
     * linears run as E4M3 products on the tensor cores: the input rows of each product are
     * quantised at run time (E4M3 codes, one power-of-two scale per row, taken from the row's max
     * |x|: the LayerNorm kernels emit them for QKV and fc1, a quantisation pass for out-proj and
     * fc2), the accumulator is multiplied by the row's and the channel's scales, then the bias
     * is added in fp32. The layers' qkv_w, proj_w, fc1_w and fc2_w may then be NULL. Everything
     * else (LayerNorms, rope, attention, GELU, the fp32 residual stream, the patch embed and the
     * merger) is as in the bf16 tower. Copied by vit_weights_create. */
    const vit_layer_fp8 *fp8_layers;
} vit_weights_desc;

typedef struct vit_handle vit_handle;  /* validated weight view + workspace + device status word */

/* Validates the descriptor (pointers non-NULL where required, 16-byte aligned, sizes in range),
 * copies it (not the weight data: the caller keeps the weights alive and unchanged until
 * vit_weights_destroy) and prepares the tensor maps of the weights on the current device.
 * Returns VIT_ERR_ARG / VIT_ERR_ALIGN on a bad descriptor (*out untouched), VIT_ERR_CUDA or
 * VIT_ERR_UNSUPPORTED when no sm_100 device is current. */
int vit_weights_create(const vit_weights_desc *desc, vit_handle **out);

/* Frees the handle and its workspace. Synchronises the device first. NULL is a no-op. */
void vit_weights_destroy(vit_handle *h);

/* Host-only: number of patches P = sum t*h*w and merged tokens P/4 for a host grid_thw [n,3].
 * Validates the grids exactly as vit_encode does. */
int vit_encode_sizes(const int32_t *grid_thw, int n_images, int64_t *n_patches, int64_t *n_merged);

/* Pre-sizes the handle's workspace for up to max_patches patches (a synchronous allocation).
 * vit_encode grows the workspace on demand otherwise; call this before capturing vit_encode
 * into a CUDA graph so that no allocation happens inside the capture. */
int vit_reserve(vit_handle *h, int64_t max_patches);

/* The encoder forward ("Qwen2-VL", Qwen2VLVisionModel: patch-embed -> rotary blocks -> 2x2
 * merger). patches: bf16 [P, 1176], the images of grid_thw one after another, each image's
 * frames in temporal order, each frame's patches in desc.patch_order. grid_thw: HOST int32
 * [n_images, 3] = (t, h, w) in patch units (h, w even). out: bf16 [P/4, out_dim]; row order =
 * images in grid_thw order, then t, then the merged (h/2, w/2) grid in raster order.
 * Attention is full within each (image, frame) segment and never crosses segments (inside
 * windows for the windowed blocks of a handle made with desc.window > 0; the output order is the
 * same). May allocate (synchronously) if the workspace is too small, see vit_reserve. */
int vit_encode(const void *patches, const int32_t *grid_thw, int n_images, vit_handle *h,
               void *out, void *stream);

/* CUDA-graph replay for repeated encodes (off by default). When enabled, the first vit_encode
 * with a given (grid_thw values, patches pointer, out pointer) records its whole launch sequence
 * into a CUDA graph on a private stream (nothing runs during the recording) and launches that
 * graph on `stream`; later calls with the same signature replay it as one launch. Up to 4
 * signatures are kept (least recently used evicted); growing the workspace or disabling drops
 * them. The inputs are read when the graph runs, so new data in the same buffers is encoded.
 * Profiling (vit_profile_enable) bypasses the graphs. */
int vit_graph_enable(vit_handle *h, int enable);

/* vit_encode with HOST patches and HOST out (pinned memory gives asynchronous copies): copies
 * the patches into the handle's workspace, encodes, copies the tokens back, all on `stream`.
 * The host buffers must stay valid until the stream reaches that point. With vit_graph_enable on,
 * the encode between the two copies is replayed from a recorded graph as in vit_encode. To overlap
 * one batch's copies with another's kernels, use one handle per stream (handles share weights). */
int vit_encode_host(const void *host_patches, const int32_t *grid_thw, int n_images,
                    vit_handle *h, void *host_out, void *stream);

/* 3-D M-RoPE position ids for the decoder ("Qwen2-VL" intro and Qwen2VLModel table, mrope;
 * LiteRT-LM card, M-RoPE note). input_ids: int32 [L]. grid_thw: HOST int32 [n_grids, 3], the
 * grids of the prompt's images and videos in order of appearance (n_grids may be 0; unused
 * trailing grids are ignored, their values are not even checked). out: int32 [3, L] (t, h, w
 * axes). delta: int32 [1] or NULL, receives (largest id + 1) - L. dev_status: int32 [1] or NULL;
 * on a malformed prompt the kernel writes VIT_ERR_TOKENS there and leaves out/delta untouched
 * (with NULL the error is silent). Malformed means: a vision run whose length is not the
 * t*(h/2)*(w/2) of the grid it consumes, a vision run with no grid left, or a consumed grid with
 * t < 1, h or w odd or < 2, or a run length above L.
 * The rule: text tokens (incl. vision_start/end) take (c, c, c) from a cursor c that counts up;
 * a vision run follows a vision_start, is t*(h/2)*(w/2) image or video tokens, its j-th token
 * takes c + (j / (h'w'), (j / w') % h', j % w'), then c += max(t, h', w').
 * Host-side returns: VIT_ERR_ARG (NULL pointers, L < 0, n_grids out of range), VIT_ERR_LIMIT
 * (L > 2^30). */
int mrope_index(const int32_t *input_ids, int64_t L, const int32_t *grid_thw, int n_grids,
                int32_t *out, int32_t *delta, int32_t *dev_status, void *stream);

/* E4M3 codes of bf16 rows with one power-of-two scale per row (the fp8 tower's weights: one row =
 * one output channel). x: bf16 [rows, cols]; codes: [rows, cols] bytes; scales: fp32 [rows]. Row r
 * with a = max |x[r]| gets scale 2^e, e the smallest integer with a <= 448 * 2^e but at least
 * -126; codes[r][c] = x[r][c] / 2^e (exact) rounded to the nearest E4M3 value, ties to even.
 * cols: a multiple of 8, 8..65536; rows >= 0; x and codes 16-byte aligned. Async on stream. */
int vit_quantize_fp8(const void *x, int64_t rows, int cols, void *codes, float *scales, void *stream);

/* ---- for callers that cannot allocate device memory ----------------------------------------
 * No counterpart on the pages: this is a deployment variant of vit_encode, not part of the method.
 * vit_encode keeps its activations in a workspace the handle grows with cudaMalloc. Callers whose
 * device memory is owned by another allocator, or that forbid device allocation after start-up
 * (cudaMalloc can synchronise the whole device and can fail at run time), use this instead: it
 * computes exactly what vit_encode computes, with the activations in a fixed file-scope device
 * array inside the library, and it calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Limit: at most VIT_NOALLOC_MAX_PATCHES patches per call (the sum of t*h*w), so the array
 *     is about 26.3 MB (activations of 1024 patches + the rope table). Every GPU on which the
 *     array has been set up holds it until process exit. Larger batches return VIT_ERR_LIMIT and
 *     launch nothing.
 *   - The first call on a device sets the array up on that device: it looks up the array's
 *     device address and fills its rope table with one kernel on `stream`, then waits for that
 *     kernel (a synchronize of `stream`), so later calls on any stream find the table ready.
 *     Under CUDA's default lazy module loading, that first call is also when the library's
 *     module holding the array is loaded on the device, i.e. when the array's 26.3 MB are
 *     allocated. Make the first call on each device at start-up, before another allocator
 *     takes the device's memory and before any stream capture (or run with
 *     CUDA_MODULE_LOADING=EAGER, which allocates the array when the CUDA context is created).
 *     Every later call allocates nothing and does not synchronise.
 *   - Every call, on every stream, shares the one array and leaves the last call's activations in
 *     it. Calls whose work overlaps on the GPU race with each other: issue them on one stream or
 *     order them. Nothing in the array needs clearing between calls: each buffer is fully
 *     written before it is read.
 *   - Arguments as for vit_encode; weights from vit_weights_create on the current device, made
 *     without windows and without fp8 layers (desc.window == 0, desc.fp8_layers == NULL; other
 *     handles return VIT_ERR_ARG). A grid row with
 *     h or w above VIT_NOALLOC_MAX_PATCHES / 2, or t above VIT_NOALLOC_MAX_PATCHES / 4, returns
 *     VIT_ERR_LIMIT before any product of its values is formed.
 *     dev_status: int32 [1] device or NULL; a kernel wait that timed out writes VIT_ERR_TIMEOUT
 *     there (it is not cleared by the call). */
#define VIT_NOALLOC_MAX_PATCHES 1024
int vit_encode_noalloc(const void *patches, const int32_t *grid_thw, int n_images, vit_handle *weights,
                       void *out, int32_t *dev_status, void *stream);

/* Synchronises `stream`, reads the handle's device status word into *host_status (VIT_OK or
 * VIT_ERR_TIMEOUT from a kernel) and clears it. */
int vit_device_status(vit_handle *h, void *stream, int32_t *host_status);

/* Number of kernels this handle has launched so far (for launch accounting). */
int64_t vit_launch_count(const vit_handle *h);

/* Per-kernel-class timing with CUDA events recorded on the launch stream around each kernel of
 * vit_encode. enable != 0 starts recording (clearing earlier totals). vit_profile_read fills
 * up to n entries of ms_total[] / launches[] in the order of vit_profile_name(i) and returns
 * the number of classes; it synchronises the stream of the last encode. */
int vit_profile_enable(vit_handle *h, int enable);
int vit_profile_read(vit_handle *h, double *ms_total, int64_t *launches, int n);
const char *vit_profile_name(int i);

const char *vit_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif
