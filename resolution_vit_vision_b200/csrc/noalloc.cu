// noalloc.cu -- vit_encode_noalloc: the encoder forward for callers that cannot allocate device
// memory.
//
// vit_encode keeps its activations in a workspace that the handle grows with cudaMalloc. Some
// callers cannot allow that: a process whose device memory is owned entirely by another
// allocator (a framework that reserved the GPU up front), or a real-time / certified deployment
// that forbids device allocation after start-up, because cudaMalloc can synchronise the whole
// device and can fail at run time. For them this file holds the activations of one encode in a
// fixed, file-scope device array instead, sized for at most VIT_NOALLOC_MAX_PATCHES patches.
// The array exists on every GPU where the module holding it is loaded: from the first call on
// that device (CUDA's default lazy module loading) or from context creation (eager loading),
// until process exit.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "handle.h"
#include "internal.h"

namespace {

constexpr int64_t kMaxP = VIT_NOALLOC_MAX_PATCHES;
constexpr int kMaxSide = static_cast<int>(kMaxP / 2);   // h * w <= kMaxP with h, w >= 2
constexpr size_t al(size_t x) { return (x + 255) / 256 * 256; }

// scratch layout (byte offsets, each 256-aligned)
constexpr size_t kOffX = 0;                                                   // fp32 [P, 1280]
constexpr size_t kOffH = kOffX + al(kMaxP * VIT_WIDTH * 4);                   // bf16 [P, 1280]
constexpr size_t kOffQKV = kOffH + al(kMaxP * VIT_WIDTH * 2);                 // bf16 [P, 3840]
constexpr size_t kOffF = kOffQKV + al(kMaxP * 3 * VIT_WIDTH * 2);             // bf16 [P, 5120]
constexpr size_t kOffPos = kOffF + al(kMaxP * VIT_MLP * 2);                   // int32 [P]
constexpr size_t kOffMr = kOffPos + al(kMaxP * 4);                            // int32 [P]
constexpr size_t kOffCs = kOffMr + al(kMaxP * 4);                             // fp32 [kMaxSide+1][20][2]
constexpr size_t kScratchBytes = kOffCs + al(static_cast<size_t>(kMaxSide + 1) * 40 * 4);

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_setup_mu;
unsigned char *g_scratch_dev[64] = {};   // device address of g_scratch, per device

// Once per device, with that device current: look up the array's device address (host code may
// not use the symbol itself as an address) and fill the rope cos/sin table it holds. Under CUDA's
// lazy module loading (the default) the address lookup is what loads this file's module on the
// device, and with it allocates the array. The set-up waits for the table fill, so a later call on
// any other stream finds the table complete.
int setup_device(int dev, cudaStream_t s) {
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (g_scratch_dev[dev]) return VIT_OK;
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return VIT_ERR_CUDA;
    }
    unsigned char *base = static_cast<unsigned char *>(p);
    const int rc = vith::rope_table_launch(reinterpret_cast<float *>(base + kOffCs), kMaxSide + 1, s);
    if (rc != VIT_OK) return rc;
    if (cudaStreamSynchronize(s) != cudaSuccess) return VIT_ERR_CUDA;
    g_scratch_dev[dev] = base;
    return VIT_OK;
}

#define NA_TRY(expr)                   \
    do {                               \
        const int _rc = (expr);        \
        if (_rc != VIT_OK) return _rc; \
    } while (0)

}  // namespace

extern "C" int vit_encode_noalloc(const void *patches, const int32_t *grid_thw, int n_images, vit_handle *h,
                                  void *out, int32_t *dev_status, void *stream) {
    if (!patches || !h || !out || !grid_thw || n_images < 1 || n_images > VIT_MAX_IMAGES) return VIT_ERR_ARG;
    if (h->desc.window != 0 || !h->fp8.empty()) return VIT_ERR_ARG;   // windowed / fp8 towers: vit_encode only
    int64_t P = 0;
    for (int i = 0; i < n_images; ++i) {
        const int t = grid_thw[3 * i], hh = grid_thw[3 * i + 1], ww = grid_thw[3 * i + 2];
        if (t < 1 || hh < 2 || ww < 2 || (hh & 1) || (ww & 1)) return VIT_ERR_GRID;
        // each factor is bounded before the product is formed: t * hh * ww <= kMaxP follows
        if (hh > kMaxSide || ww > kMaxSide || t > kMaxP / 4) return VIT_ERR_LIMIT;
        if (static_cast<int64_t>(hh) * ww > kMaxP) return VIT_ERR_LIMIT;
        P += static_cast<int64_t>(t) * hh * ww;
        if (P > kMaxP) return VIT_ERR_LIMIT;   // more patches than the fixed scratch holds
    }
    if ((reinterpret_cast<uintptr_t>(patches) & 15u) || (reinterpret_cast<uintptr_t>(out) & 15u))
        return VIT_ERR_ALIGN;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return VIT_ERR_CUDA;
    if (dev >= 64 || dev != h->device) return VIT_ERR_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    NA_TRY(setup_device(dev, s));
    unsigned char *base = g_scratch_dev[dev];
    float *X = reinterpret_cast<float *>(base + kOffX);
    void *H = base + kOffH, *QKV = base + kOffQKV, *F = base + kOffF;
    int32_t *pos = reinterpret_cast<int32_t *>(base + kOffPos);
    int32_t *merge_row = reinterpret_cast<int32_t *>(base + kOffMr);
    const float *rope_cs = reinterpret_cast<const float *>(base + kOffCs);

    // one attention segment per (image, frame); at most kMaxP / 4 of them
    int32_t cu[kMaxP / 4 + 1];
    int n_seg = 0;
    cu[0] = 0;
    for (int i = 0; i < n_images; ++i)
        for (int t = 0; t < grid_thw[3 * i]; ++t, ++n_seg) cu[n_seg + 1] = cu[n_seg] + grid_thw[3 * i + 1] * grid_thw[3 * i + 2];
    const int64_t M4 = P / 4;
    const vit_weights_desc &d = h->desc;
    auto nw = vith::gemm_use_narrow;   // the weight map matching the tile width gemm_launch picks

    NA_TRY(vith::positions_launch_stack(grid_thw, n_images, P, d.patch_order, pos, merge_row, s));
    CUtensorMap mPatch, mH, mF, mH4, mF4;
    vith::AttnMaps mQKV;
    NA_TRY(vith::gemm_make_a_map(&mPatch, patches, P, VIT_PATCH_DIM));
    NA_TRY(vith::gemm_make_a_map(&mH, H, P, VIT_WIDTH));
    NA_TRY(vith::gemm_make_a_map(&mF, F, P, VIT_MLP));
    NA_TRY(vith::gemm_make_a_map(&mH4, H, M4, VIT_MERGE_DIM));
    NA_TRY(vith::gemm_make_a_map(&mF4, F, M4, VIT_MERGE_DIM));
    NA_TRY(vith::attn_make_maps(&mQKV, QKV, P));
    CUtensorMap cX, cQKV, cF, cF4, cOut;
    NA_TRY(vith::gemm_make_c_map(&cX, X, P, VIT_WIDTH, VIT_EPI_ADD_F32));
    NA_TRY(vith::gemm_make_c_map(&cQKV, QKV, P, 3 * VIT_WIDTH, VIT_EPI_QKV_ROPE));
    NA_TRY(vith::gemm_make_c_map(&cF, F, P, VIT_MLP, VIT_EPI_GELU_BF16));
    NA_TRY(vith::gemm_make_c_map(&cF4, F, M4, VIT_MERGE_DIM, VIT_EPI_GELU_BF16));
    NA_TRY(vith::gemm_make_c_map(&cOut, out, M4, d.out_dim, VIT_EPI_STORE_BF16));
    NA_TRY(vith::gemm_launch(mPatch, nw(P, VIT_WIDTH, VIT_EPI_STORE_F32) ? h->pe_map_n : h->pe_map, cX, d.pe_b, P, VIT_WIDTH, VIT_PATCH_DIM, VIT_EPI_STORE_F32, nullptr,
                             nullptr, dev_status, s));
    for (int l = 0; l < d.depth; ++l) {
        const vit_layer_w &L = h->layers[l];
        const vith::LayerMaps &lm = h->maps[l];
        NA_TRY(vith::layernorm_launch(X, L.ln1_w, L.ln1_b, H, P, d.ln_eps, nullptr, s));
        NA_TRY(vith::gemm_launch(mH, lm.qkv, cQKV, L.qkv_b, P, 3 * VIT_WIDTH, VIT_WIDTH, VIT_EPI_QKV_ROPE, pos,
                                 rope_cs, dev_status, s));
        NA_TRY(vith::attn_launch_stack(mQKV, cu, n_seg, H, dev_status, s));
        NA_TRY(vith::gemm_launch(mH, nw(P, VIT_WIDTH, VIT_EPI_ADD_F32) ? lm.proj_n : lm.proj, cX, L.proj_b, P, VIT_WIDTH, VIT_WIDTH, VIT_EPI_ADD_F32, nullptr, nullptr,
                                 dev_status, s));
        NA_TRY(vith::layernorm_launch(X, L.ln2_w, L.ln2_b, H, P, d.ln_eps, nullptr, s));
        NA_TRY(vith::gemm_launch(mH, nw(P, VIT_MLP, VIT_EPI_GELU_BF16) ? lm.fc1_n : lm.fc1, cF, L.fc1_b, P, VIT_MLP, VIT_WIDTH, VIT_EPI_GELU_BF16, nullptr, nullptr,
                                 dev_status, s));
        NA_TRY(vith::gemm_launch(mF, nw(P, VIT_WIDTH, VIT_EPI_ADD_F32) ? lm.fc2_n : lm.fc2, cX, L.fc2_b, P, VIT_WIDTH, VIT_MLP, VIT_EPI_ADD_F32, nullptr, nullptr,
                                 dev_status, s));
        h->launches += 7;
    }
    NA_TRY(vith::layernorm_launch(X, d.lnq_w, d.lnq_b, H, P, d.ln_eps, d.patch_order == 1 ? merge_row : nullptr, s));
    NA_TRY(vith::gemm_launch(mH4, nw(M4, VIT_MERGE_DIM, VIT_EPI_GELU_BF16) ? h->m0_map_n : h->m0_map, cF4, d.m0_b, M4, VIT_MERGE_DIM, VIT_MERGE_DIM, VIT_EPI_GELU_BF16, nullptr,
                             nullptr, dev_status, s));
    NA_TRY(vith::gemm_launch(mF4, nw(M4, d.out_dim, VIT_EPI_STORE_BF16) ? h->m2_map_n : h->m2_map, cOut, d.m2_b, M4, d.out_dim, VIT_MERGE_DIM, VIT_EPI_STORE_BF16, nullptr,
                             nullptr, dev_status, s));
    h->launches += 5;
    return VIT_OK;
}
