// api.cpp -- the C ABI: argument validation, the host-side plan of a packed batch (segments,
// positions, work lists), the handle's workspace and the launch sequence of vit_encode.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <memory>
#include <mutex>
#include <new>
#include <vector>

#include "handle.h"
#include "internal.h"

// ============================================================================ device helpers
namespace vith {

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;
int g_sms[64] = {};
}  // namespace

int tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes, uint64_t inner,
            uint64_t outer, uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_outer,
            CUtensorMapSwizzle swizzle) {
    (void)elem_bytes;
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    if (!g_encode) return VIT_ERR_CUDA;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_pitch_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? VIT_OK : VIT_ERR_CUDA;
}

int device_sm_count() {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && g_sms[dev]) return g_sms[dev];
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    if (dev < 64) g_sms[dev] = n;
    return n;
}

int check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return VIT_ERR_CUDA;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return VIT_ERR_CUDA;
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    return (major == 10 && minor == 0) ? VIT_OK : VIT_ERR_UNSUPPORTED;
}

}  // namespace vith

// ============================================================================ handle
namespace {

const char *kProfNames[vith::kProfClasses] = {"patch_embed", "layernorm",  "qkv_rope",   "attention",
                                              "out_proj",    "fc1_gelu",   "fc2",        "merger_fc1",
                                              "merger_fc2",  "positions",  "attention_window", "quantize_fp8"};
enum ProfClass { P_PE, P_LN, P_QKV, P_ATT, P_PROJ, P_FC1, P_FC2, P_M0, P_M2, P_POS, P_WATT, P_Q8 };

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace


namespace {

int validate_grids(const int32_t *g, int n, int max_n, int64_t *P_out) {
    if (!g || n < 1 || n > max_n) return VIT_ERR_ARG;
    int64_t P = 0;
    for (int i = 0; i < n; ++i) {
        const int t = g[3 * i], h = g[3 * i + 1], w = g[3 * i + 2];
        if (t < 1 || h < 2 || w < 2 || (h & 1) || (w & 1)) return VIT_ERR_GRID;
        if (h > VIT_MAX_SIDE || w > VIT_MAX_SIDE) return VIT_ERR_LIMIT;
        P += static_cast<int64_t>(t) * h * w;
        if (P > VIT_MAX_PATCHES) return VIT_ERR_LIMIT;
    }
    *P_out = P;
    return VIT_OK;
}

// Profiling: an event pair around one launch.
struct ProfScope {
    vit_handle *h;
    cudaStream_t s;
    int cls;
    size_t idx = 0;
    bool on;
    ProfScope(vit_handle *h_, cudaStream_t s_, int cls_) : h(h_), s(s_), cls(cls_), on(h_ && h_->prof) {
        if (!on) return;
        idx = h->ev_used++;
        while (h->ev_pool.size() < 2 * h->ev_used) {
            cudaEvent_t e;
            cudaEventCreate(&e);
            h->ev_pool.push_back(e);
        }
        if (h->ev_class.size() < h->ev_used) h->ev_class.resize(h->ev_used);
        h->ev_class[idx] = cls;
        cudaEventRecord(h->ev_pool[2 * idx], s);
    }
    ~ProfScope() {
        if (on) cudaEventRecord(h->ev_pool[2 * idx + 1], s);
    }
};

// Fold the recorded event pairs into the per-class totals (synchronises on the last event).
void prof_collect(vit_handle *h) {
    if (h->ev_used == 0) return;
    cudaEventSynchronize(h->ev_pool[2 * (h->ev_used - 1) + 1]);
    for (size_t i = 0; i < h->ev_used; ++i) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, h->ev_pool[2 * i], h->ev_pool[2 * i + 1]) == cudaSuccess) {
            h->prof_ms[h->ev_class[i]] += ms;
            h->prof_n[h->ev_class[i]] += 1;
        }
    }
    h->ev_used = 0;
}

void graph_clear(vit_handle *h);

int ensure_workspace(vit_handle *h, int64_t P) {
    if (P <= h->ws_patches && h->ws) return VIT_OK;
    const int64_t Pn = P > 0 ? P : 1;
    const int out_dim = h->desc.out_dim;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = round_up(off + bytes, 256);
        return o;
    };
    const size_t oX = take(static_cast<size_t>(Pn) * VIT_WIDTH * 4);
    const size_t oH = take(static_cast<size_t>(Pn) * VIT_WIDTH * 2);
    const size_t oQKV = take(static_cast<size_t>(Pn) * 3 * VIT_WIDTH * 2);
    const size_t oF = take(static_cast<size_t>(Pn) * VIT_MLP * 2);
    const size_t oPos = take(static_cast<size_t>(Pn) * 4);
    const size_t oMr = take(static_cast<size_t>(Pn) * 4);
    const size_t oWt = take(static_cast<size_t>(Pn / 4 + 1) * 8);
    const size_t oPs = take(static_cast<size_t>(Pn) * VIT_PATCH_DIM * 2);
    const size_t oOs = take(static_cast<size_t>(Pn / 4 + 1) * out_dim * 2);
    const size_t oCs = take(static_cast<size_t>(VIT_MAX_SIDE) * 40 * 4);
    const size_t oSt = take(256);
    const bool f8 = !h->fp8.empty();
    const size_t oQ8 = f8 ? take(static_cast<size_t>(Pn) * VIT_MLP) : 0;
    const size_t oS8 = f8 ? take(static_cast<size_t>(Pn) * 4) : 0;
    if (h->ws) {
        cudaDeviceSynchronize();
        graph_clear(h);           // recorded graphs point into the old workspace
        cudaFree(h->ws);
        h->ws = nullptr;
    }
    void *p = nullptr;
    if (cudaMalloc(&p, off) != cudaSuccess) {
        cudaGetLastError();
        h->ws_patches = 0;
        return VIT_ERR_NOMEM;
    }
    uint8_t *b = static_cast<uint8_t *>(p);
    h->ws = p;
    h->ws_bytes = off;
    h->ws_patches = Pn;
    h->X = reinterpret_cast<float *>(b + oX);
    h->H = b + oH;
    h->QKV = b + oQKV;
    h->F = b + oF;
    h->pos = reinterpret_cast<int32_t *>(b + oPos);
    h->merge_row = reinterpret_cast<int32_t *>(b + oMr);
    h->win_tab = reinterpret_cast<int32_t *>(b + oWt);
    h->patch_stage = b + oPs;
    h->out_stage = b + oOs;
    h->rope_cs = reinterpret_cast<float *>(b + oCs);
    h->status = reinterpret_cast<int32_t *>(b + oSt);
    h->Q8 = f8 ? b + oQ8 : nullptr;
    h->S8 = f8 ? reinterpret_cast<float *>(b + oS8) : nullptr;
    h->rope_ready = false;
    if (cudaMemset(h->status, 0, 4) != cudaSuccess) return VIT_ERR_CUDA;
    return VIT_OK;
}

#define VIT_TRY(expr)                \
    do {                             \
        int _rc = (expr);            \
        if (_rc != VIT_OK) return _rc; \
    } while (0)

int encode_device(vit_handle *h, const void *patches, const int32_t *grid, int n_images, int64_t P, void *out,
                  cudaStream_t s) {
    const vit_weights_desc &d = h->desc;
    auto nw = vith::gemm_use_narrow;   // which prebuilt weight map (256 x 256 or 256 x 128 tiles) a product takes
    if (h->prof && h->ev_used) prof_collect(h);
    h->last_stream = s;
    int64_t &nl = h->launches;

    // host plan: one attention segment per (image, frame)
    std::vector<int32_t> cu;
    cu.push_back(0);
    for (int i = 0; i < n_images; ++i)
        for (int t = 0; t < grid[3 * i]; ++t) cu.push_back(cu.back() + grid[3 * i + 1] * grid[3 * i + 2]);
    const int n_seg = static_cast<int>(cu.size()) - 1;
    if (n_seg > VIT_MAX_SEGMENTS) return VIT_ERR_LIMIT;
    const int64_t M4 = P / 4;
    // windowed blocks: rows live in window order (window.cu); windows of up to 8 x 8 patches go to
    // the packed window kernel, larger ones to the segment kernel with one segment per window
    const int window = d.window;
    std::vector<int32_t> cu_win;
    if (window > 8) VIT_TRY(vith::window_cu_seqlens(grid, n_images, window, cu_win));

    if (!h->rope_ready) {
        ProfScope ps(h, s, P_POS);
        VIT_TRY(vith::rope_table_launch(h->rope_cs, VIT_MAX_SIDE, s));
        ++nl;
        h->rope_ready = true;
    }
    if (window == 0) {
        ProfScope ps(h, s, P_POS);
        VIT_TRY(vith::positions_launch(grid, n_images, P, d.patch_order, h->pos, h->merge_row, s));
        ++nl;
    } else {
        // the gather's source rows sit in the QKV buffer and the gathered patches in F, both free
        // until the first block
        int32_t *src_row = static_cast<int32_t *>(h->QKV);
        ProfScope ps(h, s, P_POS);
        VIT_TRY(vith::window_positions_launch(grid, n_images, P, d.patch_order, window, h->pos, h->merge_row,
                                              src_row, h->win_tab, s));
        ++nl;
        VIT_TRY(vith::gather_rows_launch(patches, src_row, h->F, P, VIT_PATCH_DIM * 2, s));
        ++nl;
        patches = h->F;
    }

    const bool f8 = !h->fp8.empty();
    CUtensorMap mPatch, mH, mF, mH4, mF4, mQ8w, mQ8m;   // mQ8w / mQ8m: E4M3 rows of 1280 / 5120
    vith::WinMaps mWin;
    const int n_windows = window > 0 ? vith::window_count(grid, n_images, window) : 0;
    vith::AttnMaps mQKV;
    VIT_TRY(vith::gemm_make_a_map(&mPatch, patches, P, VIT_PATCH_DIM));
    if (window > 0 && window <= 8) VIT_TRY(vith::win_make_maps(&mWin, h->QKV, P));
    VIT_TRY(vith::gemm_make_a_map(&mH, h->H, P, VIT_WIDTH));
    VIT_TRY(vith::gemm_make_a_map(&mF, h->F, P, VIT_MLP));
    VIT_TRY(vith::gemm_make_a_map(&mH4, h->H, M4, VIT_MERGE_DIM));
    VIT_TRY(vith::gemm_make_a_map(&mF4, h->F, M4, VIT_MERGE_DIM));
    VIT_TRY(vith::attn_make_maps(&mQKV, h->QKV, P));
    if (f8) {
        VIT_TRY(vith::gemm_make_a_map(&mQ8w, h->Q8, P, VIT_WIDTH, true));
        VIT_TRY(vith::gemm_make_a_map(&mQ8m, h->Q8, P, VIT_MLP, true));
    }
    CUtensorMap cX, cQKV, cF, cF4, cOut;
    VIT_TRY(vith::gemm_make_c_map(&cX, h->X, P, VIT_WIDTH, VIT_EPI_ADD_F32));
    VIT_TRY(vith::gemm_make_c_map(&cQKV, h->QKV, P, 3 * VIT_WIDTH, VIT_EPI_QKV_ROPE));
    VIT_TRY(vith::gemm_make_c_map(&cF, h->F, P, VIT_MLP, VIT_EPI_GELU_BF16));
    VIT_TRY(vith::gemm_make_c_map(&cF4, h->F, M4, VIT_MERGE_DIM, VIT_EPI_GELU_BF16));
    VIT_TRY(vith::gemm_make_c_map(&cOut, out, M4, d.out_dim, VIT_EPI_STORE_BF16));

    {
        ProfScope ps(h, s, P_PE);
        VIT_TRY(vith::gemm_launch(mPatch, nw(P, VIT_WIDTH, VIT_EPI_STORE_F32) ? h->pe_map_n : h->pe_map, cX, d.pe_b, P,
                                  VIT_WIDTH, VIT_PATCH_DIM, VIT_EPI_STORE_F32,
                                  nullptr, nullptr, h->status, s));
        ++nl;
    }
    for (int l = 0; l < d.depth; ++l) {
        const vit_layer_w &L = h->layers[l];
        const vith::LayerMaps &lm = h->maps[l];
        const vit_layer_fp8 *L8 = f8 ? &h->fp8[l] : nullptr;
        {
            ProfScope ps(h, s, P_LN);
            if (f8) VIT_TRY(vith::layernorm_fp8_launch(h->X, L.ln1_w, L.ln1_b, h->Q8, h->S8, P, d.ln_eps, s));
            else VIT_TRY(vith::layernorm_launch(h->X, L.ln1_w, L.ln1_b, h->H, P, d.ln_eps, nullptr, s));
            ++nl;
        }
        {
            ProfScope ps(h, s, P_QKV);
            VIT_TRY(vith::gemm_launch(f8 ? mQ8w : mH, lm.qkv, cQKV, L.qkv_b, P, 3 * VIT_WIDTH, VIT_WIDTH,
                                      VIT_EPI_QKV_ROPE, h->pos, h->rope_cs, h->status, s, f8 ? h->S8 : nullptr,
                                      f8 ? L8->qkv_s : nullptr));
            ++nl;
        }
        if (window == 0 || h->full_attention[l]) {
            ProfScope ps(h, s, P_ATT);
            VIT_TRY(vith::attn_launch(mQKV, cu.data(), n_seg, h->H, h->status, s));
            ++nl;
        } else if (window <= 8) {
            ProfScope ps(h, s, P_WATT);
            VIT_TRY(vith::win_attn_launch(mWin, h->win_tab, n_windows, P, h->H, h->status, s));
            ++nl;
        } else {
            ProfScope ps(h, s, P_WATT);
            VIT_TRY(vith::attn_launch(mQKV, cu_win.data(), static_cast<int>(cu_win.size()) - 1, h->H, h->status, s));
            ++nl;
        }
        if (f8) {
            ProfScope ps(h, s, P_Q8);
            VIT_TRY(vith::quantize_rows_launch(h->H, P, VIT_WIDTH, h->Q8, h->S8, s));
            ++nl;
        }
        {
            ProfScope ps(h, s, P_PROJ);
            VIT_TRY(vith::gemm_launch(f8 ? mQ8w : mH, nw(P, VIT_WIDTH, VIT_EPI_ADD_F32) ? lm.proj_n : lm.proj, cX,
                                      L.proj_b, P, VIT_WIDTH, VIT_WIDTH, VIT_EPI_ADD_F32,
                                      nullptr, nullptr, h->status, s, f8 ? h->S8 : nullptr,
                                      f8 ? L8->proj_s : nullptr));
            ++nl;
        }
        {
            ProfScope ps(h, s, P_LN);
            if (f8) VIT_TRY(vith::layernorm_fp8_launch(h->X, L.ln2_w, L.ln2_b, h->Q8, h->S8, P, d.ln_eps, s));
            else VIT_TRY(vith::layernorm_launch(h->X, L.ln2_w, L.ln2_b, h->H, P, d.ln_eps, nullptr, s));
            ++nl;
        }
        {
            ProfScope ps(h, s, P_FC1);
            VIT_TRY(vith::gemm_launch(f8 ? mQ8w : mH, nw(P, VIT_MLP, VIT_EPI_GELU_BF16) ? lm.fc1_n : lm.fc1, cF,
                                      L.fc1_b, P, VIT_MLP, VIT_WIDTH, VIT_EPI_GELU_BF16,
                                      nullptr, nullptr, h->status, s, f8 ? h->S8 : nullptr,
                                      f8 ? L8->fc1_s : nullptr));
            ++nl;
        }
        if (f8) {
            ProfScope ps(h, s, P_Q8);
            VIT_TRY(vith::quantize_rows_launch(h->F, P, VIT_MLP, h->Q8, h->S8, s));
            ++nl;
        }
        {
            ProfScope ps(h, s, P_FC2);
            VIT_TRY(vith::gemm_launch(f8 ? mQ8m : mF, nw(P, VIT_WIDTH, VIT_EPI_ADD_F32) ? lm.fc2_n : lm.fc2, cX,
                                      L.fc2_b, P, VIT_WIDTH, VIT_MLP, VIT_EPI_ADD_F32,
                                      nullptr, nullptr, h->status, s, f8 ? h->S8 : nullptr,
                                      f8 ? L8->fc2_s : nullptr));
            ++nl;
        }
    }
    {
        ProfScope ps(h, s, P_LN);
        VIT_TRY(vith::layernorm_launch(h->X, d.lnq_w, d.lnq_b, h->H, P, d.ln_eps,
                                       (d.patch_order == 1 || window > 0) ? h->merge_row : nullptr, s));
        ++nl;
    }
    {
        ProfScope ps(h, s, P_M0);
        VIT_TRY(vith::gemm_launch(mH4, nw(M4, VIT_MERGE_DIM, VIT_EPI_GELU_BF16) ? h->m0_map_n : h->m0_map, cF4, d.m0_b,
                                  M4, VIT_MERGE_DIM, VIT_MERGE_DIM, VIT_EPI_GELU_BF16,
                                  nullptr, nullptr, h->status, s));
        ++nl;
    }
    {
        ProfScope ps(h, s, P_M2);
        VIT_TRY(vith::gemm_launch(mF4, nw(M4, d.out_dim, VIT_EPI_STORE_BF16) ? h->m2_map_n : h->m2_map, cOut, d.m2_b,
                                  M4, d.out_dim, VIT_MERGE_DIM, VIT_EPI_STORE_BF16,
                                  nullptr, nullptr, h->status, s));
        ++nl;
    }
    return VIT_OK;
}

void graph_clear(vit_handle *h) {
    for (auto &g : h->graphs)
        if (g.exec) cudaGraphExecDestroy(g.exec);
    h->graphs.clear();
}

// vit_encode through a CUDA graph: the first call with a given (grid, patches, out) records the
// whole launch sequence on a private stream and instantiates it; later calls replay it on the
// caller's stream (one launch instead of ~229). At most kGraphCache signatures are kept.
constexpr size_t kGraphCache = 4;

int encode_graph(vit_handle *h, const void *patches, const int32_t *grid, int n_images, int64_t P, void *out,
                 cudaStream_t s) {
    std::vector<int32_t> key(grid, grid + 3 * n_images);
    for (auto &g : h->graphs) {
        if (g.patches == patches && g.out == out && g.grid == key) {
            if (cudaGraphLaunch(g.exec, s) != cudaSuccess) return VIT_ERR_CUDA;
            g.last_use = ++h->graph_clock;
            h->launches += g.launches;
            h->last_stream = s;
            return VIT_OK;
        }
    }
    if (!h->capture_stream &&
        cudaStreamCreateWithFlags(&h->capture_stream, cudaStreamNonBlocking) != cudaSuccess)
        return VIT_ERR_CUDA;
    if (!h->rope_ready) {   // the once-per-workspace table is not part of the replayed graph
        int rc = vith::rope_table_launch(h->rope_cs, VIT_MAX_SIDE, s);
        if (rc != VIT_OK) return rc;
        ++h->launches;
        h->rope_ready = true;
    }
    // the caller's earlier work on `s` must precede the replay, which runs on `s` itself; the
    // capture only records, so nothing else orders it
    if (cudaStreamBeginCapture(h->capture_stream, cudaStreamCaptureModeThreadLocal) != cudaSuccess)
        return VIT_ERR_CUDA;
    const int64_t n0 = h->launches;
    int rc = encode_device(h, patches, grid, n_images, P, out, h->capture_stream);
    cudaGraph_t graph = nullptr;
    const cudaError_t e = cudaStreamEndCapture(h->capture_stream, &graph);
    const int64_t recorded = h->launches - n0;
    h->launches = n0;
    if (rc != VIT_OK || e != cudaSuccess || !graph) {
        if (graph) cudaGraphDestroy(graph);
        cudaGetLastError();
        return rc != VIT_OK ? rc : VIT_ERR_CUDA;
    }
    cudaGraphExec_t exec = nullptr;
    const cudaError_t ie = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (ie != cudaSuccess) return VIT_ERR_CUDA;
    if (h->graphs.size() == kGraphCache) {   // evict the least recently used signature
        size_t lru = 0;
        for (size_t i = 1; i < h->graphs.size(); ++i)
            if (h->graphs[i].last_use < h->graphs[lru].last_use) lru = i;
        cudaGraphExecDestroy(h->graphs[lru].exec);
        h->graphs.erase(h->graphs.begin() + lru);
    }
    vit_handle::GraphEntry g;
    g.grid = std::move(key);
    g.patches = patches;
    g.out = out;
    g.exec = exec;
    g.launches = recorded;
    g.last_use = ++h->graph_clock;
    h->graphs.push_back(std::move(g));
    if (cudaGraphLaunch(exec, s) != cudaSuccess) return VIT_ERR_CUDA;
    h->launches += recorded;
    h->last_stream = s;
    return VIT_OK;
}

}  // namespace

// ============================================================================ C ABI
extern "C" {

const char *vit_status_string(int st) {
    switch (st) {
        case VIT_OK: return "ok";
        case VIT_ERR_ARG: return "invalid argument";
        case VIT_ERR_GRID: return "invalid grid_thw (need t >= 1 and even h, w >= 2)";
        case VIT_ERR_ALIGN: return "device pointer not 16-byte aligned";
        case VIT_ERR_NOMEM: return "device allocation failed";
        case VIT_ERR_CUDA: return "CUDA error";
        case VIT_ERR_TOKENS: return "malformed M-RoPE prompt (vision run length or grid count)";
        case VIT_ERR_TIMEOUT: return "a kernel wait timed out";
        case VIT_ERR_UNSUPPORTED: return "device is not sm_100 (B200 class)";
        case VIT_ERR_LIMIT: return "size beyond the library limits";
        default: return "unknown status";
    }
}

int vit_encode_sizes(const int32_t *grid_thw, int n_images, int64_t *n_patches, int64_t *n_merged) {
    if (!n_patches || !n_merged) return VIT_ERR_ARG;
    int64_t P = 0;
    const int rc = validate_grids(grid_thw, n_images, VIT_MAX_IMAGES, &P);
    if (rc != VIT_OK) return rc;
    *n_patches = P;
    *n_merged = P / 4;
    return VIT_OK;
}

int vit_weights_create(const vit_weights_desc *d, vit_handle **out) {
    if (!d || !out) return VIT_ERR_ARG;
    if (d->depth < 1 || d->depth > 64 || d->out_dim < 16 || d->out_dim > 16384 || (d->out_dim % 16) != 0 ||
        !(d->ln_eps > 0.0f) || (d->patch_order != 0 && d->patch_order != 1) || !d->layers)
        return VIT_ERR_ARG;
    if (d->window < 0 || d->window > VIT_MAX_SIDE || (d->window % 2) != 0) return VIT_ERR_ARG;
    const void *req[] = {d->pe_w, d->lnq_w, d->m0_w, d->m2_w};
    for (const void *p : req)
        if (!p) return VIT_ERR_ARG;
    const void *opt[] = {d->pe_w, d->pe_b, d->lnq_w, d->lnq_b, d->m0_w, d->m0_b, d->m2_w, d->m2_b};
    for (const void *p : opt)
        if (p && !aligned16(p)) return VIT_ERR_ALIGN;
    for (int l = 0; l < d->depth; ++l) {
        const vit_layer_w &L = d->layers[l];
        const void *lr[] = {L.ln1_w, L.ln2_w};
        for (const void *p : lr)
            if (!p) return VIT_ERR_ARG;
        if (d->fp8_layers) {   // the E4M3 codes and scales replace the four bf16 block linears
            const vit_layer_fp8 &Q = d->fp8_layers[l];
            const void *q[] = {Q.qkv_q, Q.qkv_s, Q.proj_q, Q.proj_s, Q.fc1_q, Q.fc1_s, Q.fc2_q, Q.fc2_s};
            for (const void *p : q) {
                if (!p) return VIT_ERR_ARG;
                if (!aligned16(p)) return VIT_ERR_ALIGN;
            }
        } else {
            const void *w[] = {L.qkv_w, L.proj_w, L.fc1_w, L.fc2_w};
            for (const void *p : w)
                if (!p) return VIT_ERR_ARG;
        }
        const void *la[] = {L.ln1_w, L.ln1_b, L.qkv_w, L.qkv_b, L.proj_w, L.proj_b,
                            L.ln2_w, L.ln2_b, L.fc1_w, L.fc1_b, L.fc2_w, L.fc2_b};
        for (const void *p : la)
            if (p && !aligned16(p)) return VIT_ERR_ALIGN;
    }
    int rc = vith::check_device();
    if (rc != VIT_OK) return rc;
    std::unique_ptr<vit_handle> h(new (std::nothrow) vit_handle());
    if (!h) return VIT_ERR_NOMEM;
    h->desc = *d;
    h->layers.assign(d->layers, d->layers + d->depth);
    h->desc.layers = nullptr;
    h->full_attention.assign(d->depth, 0);
    if (d->window > 0 && d->full_attention)
        for (int l = 0; l < d->depth; ++l) h->full_attention[l] = d->full_attention[l] ? 1 : 0;
    h->desc.full_attention = nullptr;
    if (d->fp8_layers) h->fp8.assign(d->fp8_layers, d->fp8_layers + d->depth);
    h->desc.fp8_layers = nullptr;
    cudaGetDevice(&h->device);
    h->maps.resize(d->depth);
    rc = vith::gemm_make_b_map(&h->pe_map, d->pe_w, VIT_WIDTH, VIT_PATCH_DIM, VIT_EPI_STORE_F32);
    if (rc == VIT_OK) rc = vith::gemm_make_b_map(&h->m0_map, d->m0_w, VIT_MERGE_DIM, VIT_MERGE_DIM, VIT_EPI_GELU_BF16);
    if (rc == VIT_OK) rc = vith::gemm_make_b_map(&h->m2_map, d->m2_w, d->out_dim, VIT_MERGE_DIM, VIT_EPI_STORE_BF16);
    if (rc == VIT_OK)
        rc = vith::gemm_make_b_map(&h->pe_map_n, d->pe_w, VIT_WIDTH, VIT_PATCH_DIM, VIT_EPI_STORE_F32, false, true);
    if (rc == VIT_OK)
        rc = vith::gemm_make_b_map(&h->m0_map_n, d->m0_w, VIT_MERGE_DIM, VIT_MERGE_DIM, VIT_EPI_GELU_BF16, false, true);
    if (rc == VIT_OK)
        rc = vith::gemm_make_b_map(&h->m2_map_n, d->m2_w, d->out_dim, VIT_MERGE_DIM, VIT_EPI_STORE_BF16, false, true);
    for (int l = 0; l < d->depth && rc == VIT_OK; ++l) {
        const vit_layer_w &L = h->layers[l];
        vith::LayerMaps &m = h->maps[l];
        const bool f8 = !h->fp8.empty();
        const vit_layer_fp8 *Q = f8 ? &h->fp8[l] : nullptr;
        rc = vith::gemm_make_b_map(&m.qkv, f8 ? Q->qkv_q : L.qkv_w, 3 * VIT_WIDTH, VIT_WIDTH, VIT_EPI_QKV_ROPE, f8);
        if (rc == VIT_OK)
            rc = vith::gemm_make_b_map(&m.proj, f8 ? Q->proj_q : L.proj_w, VIT_WIDTH, VIT_WIDTH, VIT_EPI_ADD_F32, f8);
        if (rc == VIT_OK)
            rc = vith::gemm_make_b_map(&m.fc1, f8 ? Q->fc1_q : L.fc1_w, VIT_MLP, VIT_WIDTH, VIT_EPI_GELU_BF16, f8);
        if (rc == VIT_OK)
            rc = vith::gemm_make_b_map(&m.fc2, f8 ? Q->fc2_q : L.fc2_w, VIT_WIDTH, VIT_MLP, VIT_EPI_ADD_F32, f8);
        if (rc == VIT_OK)
            rc = vith::gemm_make_b_map(&m.proj_n, f8 ? Q->proj_q : L.proj_w, VIT_WIDTH, VIT_WIDTH, VIT_EPI_ADD_F32, f8,
                                       true);
        if (rc == VIT_OK)
            rc = vith::gemm_make_b_map(&m.fc1_n, f8 ? Q->fc1_q : L.fc1_w, VIT_MLP, VIT_WIDTH, VIT_EPI_GELU_BF16, f8,
                                       true);
        if (rc == VIT_OK)
            rc = vith::gemm_make_b_map(&m.fc2_n, f8 ? Q->fc2_q : L.fc2_w, VIT_WIDTH, VIT_MLP, VIT_EPI_ADD_F32, f8,
                                       true);
    }
    if (rc != VIT_OK) return rc;
    *out = h.release();
    return VIT_OK;
}

void vit_weights_destroy(vit_handle *h) {
    if (!h) return;
    cudaDeviceSynchronize();
    graph_clear(h);
    if (h->capture_stream) cudaStreamDestroy(h->capture_stream);
    for (cudaEvent_t e : h->ev_pool) cudaEventDestroy(e);
    if (h->ws) cudaFree(h->ws);
    delete h;
}

int vit_reserve(vit_handle *h, int64_t max_patches) {
    if (!h || max_patches < 0) return VIT_ERR_ARG;
    if (max_patches > VIT_MAX_PATCHES) return VIT_ERR_LIMIT;
    return ensure_workspace(h, max_patches);
}

int vit_encode(const void *patches, const int32_t *grid_thw, int n_images, vit_handle *h, void *out, void *stream) {
    if (!patches || !h || !out) return VIT_ERR_ARG;
    int64_t P = 0;
    int rc = validate_grids(grid_thw, n_images, VIT_MAX_IMAGES, &P);
    if (rc != VIT_OK) return rc;
    if (!aligned16(patches) || !aligned16(out)) return VIT_ERR_ALIGN;
    rc = ensure_workspace(h, P);
    if (rc != VIT_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!h->graph_on || h->prof) return encode_device(h, patches, grid_thw, n_images, P, out, s);
    return encode_graph(h, patches, grid_thw, n_images, P, out, s);
}

int vit_graph_enable(vit_handle *h, int enable) {
    if (!h) return VIT_ERR_ARG;
    h->graph_on = enable != 0;
    if (!h->graph_on) graph_clear(h);
    return VIT_OK;
}

int vit_encode_host(const void *host_patches, const int32_t *grid_thw, int n_images, vit_handle *h, void *host_out,
                    void *stream) {
    if (!host_patches || !h || !host_out) return VIT_ERR_ARG;
    int64_t P = 0;
    int rc = validate_grids(grid_thw, n_images, VIT_MAX_IMAGES, &P);
    if (rc != VIT_OK) return rc;
    rc = ensure_workspace(h, P);
    if (rc != VIT_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t in_bytes = static_cast<size_t>(P) * VIT_PATCH_DIM * 2;
    const size_t out_bytes = static_cast<size_t>(P / 4) * h->desc.out_dim * 2;
    if (cudaMemcpyAsync(h->patch_stage, host_patches, in_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return VIT_ERR_CUDA;
    rc = (h->graph_on && !h->prof) ? encode_graph(h, h->patch_stage, grid_thw, n_images, P, h->out_stage, s)
                                   : encode_device(h, h->patch_stage, grid_thw, n_images, P, h->out_stage, s);
    if (rc != VIT_OK) return rc;
    if (cudaMemcpyAsync(host_out, h->out_stage, out_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return VIT_ERR_CUDA;
    return VIT_OK;
}

int mrope_index(const int32_t *input_ids, int64_t L, const int32_t *grid_thw, int n_grids, int32_t *out,
                int32_t *delta, int32_t *dev_status, void *stream) {
    if (L < 0 || n_grids < 0 || n_grids > VIT_MAX_MROPE_GRIDS) return VIT_ERR_ARG;
    if (L > 0 && (!input_ids || !out)) return VIT_ERR_ARG;
    if (n_grids > 0 && !grid_thw) return VIT_ERR_ARG;
    if (L > (int64_t(1) << 30)) return VIT_ERR_LIMIT;
    // grid values are checked on the device, only for the grids the prompt's vision runs consume
    return vith::mrope_launch(input_ids, L, grid_thw, n_grids, out, delta, dev_status,
                              static_cast<cudaStream_t>(stream));
}

int vit_device_status(vit_handle *h, void *stream, int32_t *host_status) {
    if (!h || !host_status) return VIT_ERR_ARG;
    if (!h->status) {
        *host_status = VIT_OK;
        return VIT_OK;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return VIT_ERR_CUDA;
    int32_t v = 0;
    if (cudaMemcpy(&v, h->status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return VIT_ERR_CUDA;
    if (cudaMemset(h->status, 0, 4) != cudaSuccess) return VIT_ERR_CUDA;
    *host_status = v;
    return VIT_OK;
}

int64_t vit_launch_count(const vit_handle *h) { return h ? h->launches : -1; }

int vit_profile_enable(vit_handle *h, int enable) {
    if (!h) return VIT_ERR_ARG;
    if (h->ev_used) prof_collect(h);
    h->prof = enable != 0;
    for (int i = 0; i < vith::kProfClasses; ++i) {
        h->prof_ms[i] = 0;
        h->prof_n[i] = 0;
    }
    return VIT_OK;
}

int vit_profile_read(vit_handle *h, double *ms_total, int64_t *launches, int n) {
    if (!h) return VIT_ERR_ARG;
    prof_collect(h);
    for (int i = 0; i < n && i < vith::kProfClasses; ++i) {
        if (ms_total) ms_total[i] = h->prof_ms[i];
        if (launches) launches[i] = h->prof_n[i];
    }
    return vith::kProfClasses;
}

const char *vit_profile_name(int i) { return (i >= 0 && i < vith::kProfClasses) ? kProfNames[i] : nullptr; }

// ---------------------------------------------------------------------------- kernel-level ops
int vit_op_gemm(const void *A, const void *B, const void *bias, void *C, int64_t M, int N, int K, int epilogue,
                const int32_t *pos, const float *rope_cs, int32_t *dev_status, void *stream) {
    if (!A || !B || !C || M < 1 || N < 16 || (N % 16) != 0 || K < 8 || (K % 8) != 0) return VIT_ERR_ARG;
    if (epilogue < VIT_EPI_STORE_F32 || epilogue > VIT_EPI_QKV_ROPE) return VIT_ERR_ARG;
    if (epilogue == VIT_EPI_QKV_ROPE && (N != 3 * VIT_WIDTH || !pos || !rope_cs)) return VIT_ERR_ARG;
    if (M > (int64_t(1) << 30)) return VIT_ERR_LIMIT;
    if (!aligned16(A) || !aligned16(B) || !aligned16(C) || (bias && !aligned16(bias))) return VIT_ERR_ALIGN;
    CUtensorMap ta, tb, tc;
    int rc = vith::gemm_make_a_map(&ta, A, M, K);
    if (rc == VIT_OK) rc = vith::gemm_make_b_map(&tb, B, N, K, epilogue, false, vith::gemm_use_narrow(M, N, epilogue));
    if (rc == VIT_OK) rc = vith::gemm_make_c_map(&tc, C, M, N, epilogue);
    if (rc != VIT_OK) return rc;
    return vith::gemm_launch(ta, tb, tc, bias, M, N, K, epilogue, pos, rope_cs, dev_status,
                             static_cast<cudaStream_t>(stream));
}

int vit_op_gemm_fp8(const void *A, const float *a_scale, const void *B, const float *b_scale, const void *bias,
                    void *C, int64_t M, int N, int K, int epilogue, const int32_t *pos, const float *rope_cs,
                    int32_t *dev_status, void *stream) {
    if (!A || !B || !C || !a_scale || !b_scale || M < 1 || N < 16 || (N % 16) != 0 || K < 16 || (K % 16) != 0)
        return VIT_ERR_ARG;
    if (epilogue < VIT_EPI_STORE_F32 || epilogue > VIT_EPI_QKV_ROPE) return VIT_ERR_ARG;
    if (epilogue == VIT_EPI_QKV_ROPE && (N != 3 * VIT_WIDTH || !pos || !rope_cs)) return VIT_ERR_ARG;
    if (M > (int64_t(1) << 30)) return VIT_ERR_LIMIT;
    if (!aligned16(A) || !aligned16(B) || !aligned16(C) || !aligned16(b_scale) || (bias && !aligned16(bias)))
        return VIT_ERR_ALIGN;
    CUtensorMap ta, tb, tc;
    int rc = vith::gemm_make_a_map(&ta, A, M, K, true);
    if (rc == VIT_OK) rc = vith::gemm_make_b_map(&tb, B, N, K, epilogue, true, vith::gemm_use_narrow(M, N, epilogue));
    if (rc == VIT_OK) rc = vith::gemm_make_c_map(&tc, C, M, N, epilogue);
    if (rc != VIT_OK) return rc;
    return vith::gemm_launch(ta, tb, tc, bias, M, N, K, epilogue, pos, rope_cs, dev_status,
                             static_cast<cudaStream_t>(stream), a_scale, b_scale);
}

int vit_op_layernorm_fp8(const float *X, const void *gamma, const void *beta, void *codes, float *scales,
                         int64_t rows, float eps, void *stream) {
    if (!X || !gamma || !codes || !scales || rows < 0 || !(eps > 0.0f)) return VIT_ERR_ARG;
    if (!aligned16(X) || !aligned16(codes) || !aligned16(gamma) || (beta && !aligned16(beta))) return VIT_ERR_ALIGN;
    return vith::layernorm_fp8_launch(X, gamma, beta, codes, scales, rows, eps, static_cast<cudaStream_t>(stream));
}

int vit_quantize_fp8(const void *x, int64_t rows, int cols, void *codes, float *scales, void *stream) {
    if (rows < 0 || cols < 8 || cols > 65536 || (cols % 8) != 0) return VIT_ERR_ARG;
    if (rows > 0 && (!x || !codes || !scales)) return VIT_ERR_ARG;
    if (rows > (int64_t(1) << 31)) return VIT_ERR_LIMIT;
    if (rows > 0 && (!aligned16(x) || !aligned16(codes))) return VIT_ERR_ALIGN;
    return vith::quantize_rows_launch(x, rows, cols, codes, scales, static_cast<cudaStream_t>(stream));
}

int vit_op_rope_table(float *cs, int n_pos, void *stream) {
    if (!cs || n_pos < 1 || n_pos > VIT_MAX_SIDE) return VIT_ERR_ARG;
    return vith::rope_table_launch(cs, n_pos, static_cast<cudaStream_t>(stream));
}

int vit_op_positions(const int32_t *grid_thw, int n_images, int patch_order, int32_t *pos, int32_t *merge_row,
                     void *stream) {
    if (!pos || (patch_order != 0 && patch_order != 1)) return VIT_ERR_ARG;
    int64_t P = 0;
    const int rc = validate_grids(grid_thw, n_images, VIT_MAX_IMAGES, &P);
    if (rc != VIT_OK) return rc;
    return vith::positions_launch(grid_thw, n_images, P, patch_order, pos, merge_row,
                                  static_cast<cudaStream_t>(stream));
}

int vit_op_layernorm(const float *X, const void *gamma, const void *beta, void *Y, int64_t rows, float eps,
                     const int32_t *out_row, void *stream) {
    if (!X || !gamma || !Y || rows < 0 || !(eps > 0.0f)) return VIT_ERR_ARG;
    if (!aligned16(X) || !aligned16(Y) || !aligned16(gamma) || (beta && !aligned16(beta))) return VIT_ERR_ALIGN;
    return vith::layernorm_launch(X, gamma, beta, Y, rows, eps, out_row, static_cast<cudaStream_t>(stream));
}

int vit_op_attention(const void *qkv, int64_t P, const int32_t *cu_seqlens, int n_seg, void *out,
                     int32_t *dev_status, void *stream) {
    if (!qkv || !out || !cu_seqlens || n_seg < 1 || n_seg > VIT_MAX_SEGMENTS || P < 1) return VIT_ERR_ARG;
    if (cu_seqlens[0] != 0 || cu_seqlens[n_seg] != P) return VIT_ERR_ARG;
    for (int i = 0; i < n_seg; ++i)
        if (cu_seqlens[i + 1] < cu_seqlens[i]) return VIT_ERR_ARG;
    if (P > VIT_MAX_PATCHES) return VIT_ERR_LIMIT;
    if (!aligned16(qkv) || !aligned16(out)) return VIT_ERR_ALIGN;
    vith::AttnMaps t;
    const int rc = vith::attn_make_maps(&t, qkv, P);
    if (rc != VIT_OK) return rc;
    return vith::attn_launch(t, cu_seqlens, n_seg, out, dev_status, static_cast<cudaStream_t>(stream));
}

int vit_op_exp2_fma(const float *x, float *y, int64_t n, void *stream) {
    if (n < 0 || (n > 0 && (!x || !y))) return VIT_ERR_ARG;
    return vith::exp2_fma_launch(x, y, n, static_cast<cudaStream_t>(stream));
}

int vit_op_window_positions(const int32_t *grid_thw, int n_images, int patch_order, int window, int32_t *pos,
                            int32_t *merge_row, int32_t *src_row, int32_t *win_table, int *n_windows,
                            void *stream) {
    if (!pos || !merge_row || !src_row || !win_table || !n_windows || (patch_order != 0 && patch_order != 1))
        return VIT_ERR_ARG;
    if (window < 2 || window > VIT_MAX_SIDE || window % 2) return VIT_ERR_ARG;
    int64_t P = 0;
    const int rc = validate_grids(grid_thw, n_images, VIT_MAX_IMAGES, &P);
    if (rc != VIT_OK) return rc;
    *n_windows = vith::window_count(grid_thw, n_images, window);
    return vith::window_positions_launch(grid_thw, n_images, P, patch_order, window, pos, merge_row, src_row,
                                         win_table, static_cast<cudaStream_t>(stream));
}

int vit_op_gather_rows(const void *src, const int32_t *src_row, void *dst, int64_t rows, int row_bytes,
                       void *stream) {
    if (!src || !src_row || !dst || rows < 0 || row_bytes <= 0) return VIT_ERR_ARG;
    return vith::gather_rows_launch(src, src_row, dst, rows, row_bytes, static_cast<cudaStream_t>(stream));
}

int vit_op_window_attention(const void *qkv, int64_t P, const int32_t *win_table, int n_windows, void *out,
                            int32_t *dev_status, void *stream) {
    if (!qkv || !out || !win_table || P < 1 || n_windows < 1 || n_windows > P / 4) return VIT_ERR_ARG;
    if (P > VIT_MAX_PATCHES) return VIT_ERR_LIMIT;
    if (!aligned16(qkv) || !aligned16(out)) return VIT_ERR_ALIGN;
    vith::WinMaps m;
    const int rc = vith::win_make_maps(&m, qkv, P);
    if (rc != VIT_OK) return rc;
    return vith::win_attn_launch(m, win_table, n_windows, P, out, dev_status, static_cast<cudaStream_t>(stream));
}

int mrope_apply(void *q, int n_heads, void *k, int n_kv_heads, int head_dim, const int32_t *pos, int64_t L,
                double theta, const int32_t *sections, void *stream) {
    if (!pos || !sections || L < 0 || L > (int64_t(1) << 31) - 1 || !(theta > 1.0)) return VIT_ERR_ARG;
    if (head_dim < 16 || head_dim > 256 || head_dim % 16) return VIT_ERR_ARG;
    if (n_heads < 0 || n_kv_heads < 0 || (n_heads > 0 && !q) || (n_kv_heads > 0 && !k)) return VIT_ERR_ARG;
    if (n_heads * head_dim > 65536 || n_kv_heads * head_dim > 65536) return VIT_ERR_ARG;
    if (sections[0] < 0 || sections[1] < 0 || sections[2] < 0 || sections[0] + sections[1] + sections[2] != head_dim / 2)
        return VIT_ERR_ARG;
    if ((q && !aligned16(q)) || (k && !aligned16(k))) return VIT_ERR_ALIGN;
    return vith::mrope_apply_launch(n_heads > 0 ? q : nullptr, n_heads, n_kv_heads > 0 ? k : nullptr, n_kv_heads,
                                    head_dim, pos, L, theta, sections, static_cast<cudaStream_t>(stream));
}

int scatter_vision_tokens(const int32_t *input_ids, int64_t L, const void *embed_table, int64_t vocab, int dim,
                          const void *vision, int64_t n_vision, void *out, int32_t *dev_status, void *stream) {
    if (L == 0 && n_vision == 0) return VIT_OK;   // an empty prompt: nothing to read or write
    if (!input_ids || !embed_table || !out || L < 0 || L > (int64_t(1) << 18) || vocab < 1 || dim < 8 ||
        dim % 8 || n_vision < 0 || (n_vision > 0 && !vision))
        return VIT_ERR_ARG;
    if (!aligned16(embed_table) || !aligned16(out) || (vision && !aligned16(vision))) return VIT_ERR_ALIGN;
    return vith::scatter_launch(input_ids, L, embed_table, vocab, dim, vision, n_vision, out, dev_status,
                                static_cast<cudaStream_t>(stream));
}

int vit_op_wait_selftest(int32_t *dev_status, int64_t limit_cycles, void *stream) {
    if (!dev_status || limit_cycles < 1000 || limit_cycles > 4000000000LL) return VIT_ERR_ARG;
    return vith::wait_selftest_launch(dev_status, limit_cycles, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
