// handle.h -- the vit_handle behind the C ABI: the validated weight view (descriptor copy and
// the weights' TMA descriptors), the lazily grown workspace and the profiling state.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "../../include/vit.h"

namespace vith {
struct LayerMaps {
    CUtensorMap qkv, proj, fc1, fc2;
    CUtensorMap proj_n, fc1_n, fc2_n;   // the same weights for 256 x 128 tiles (small batches)
};
constexpr int kProfClasses = 12;
}  // namespace vith

struct vit_handle {
    vit_weights_desc desc{};
    std::vector<vit_layer_w> layers;
    std::vector<uint8_t> full_attention;   // [depth], windowed handles only
    std::vector<vit_layer_fp8> fp8;        // [depth] when the block linears run in E4M3, else empty
    std::vector<vith::LayerMaps> maps;     // of the bf16 weights, or of the E4M3 codes
    CUtensorMap pe_map{}, m0_map{}, m2_map{};
    CUtensorMap pe_map_n{}, m0_map_n{}, m2_map_n{};   // for 256 x 128 tiles
    int device = 0;

    // workspace
    void *ws = nullptr;
    size_t ws_bytes = 0;
    int64_t ws_patches = 0;
    float *X = nullptr;            // fp32 [P, 1280] residual stream
    void *H = nullptr;             // bf16 [P, 1280] LayerNorm output / attention output / merger input
    void *QKV = nullptr;           // bf16 [P, 3840]; with windows, first the gather's source rows
    void *F = nullptr;             // bf16 [P, 5120] fc1 output / merger hidden; with windows, first
                                   // the patches gathered into window order (bf16 [P, 1176])
    int32_t *pos = nullptr;        // [P]
    int32_t *merge_row = nullptr;  // [P]
    int32_t *win_tab = nullptr;    // [2 * (P/4 + 1)] (first row, rows) per attention window
    void *Q8 = nullptr;            // fp8 handles: E4M3 codes of a product's input rows [P, <= 5120]
    float *S8 = nullptr;           // fp8 handles: their per-row scales [P]
    void *patch_stage = nullptr;   // bf16 [P, 1176] (vit_encode_host)
    void *out_stage = nullptr;     // bf16 [P/4, out_dim] (vit_encode_host)
    float *rope_cs = nullptr;      // [VIT_MAX_SIDE][20][2]
    int32_t *status = nullptr;     // device status word
    bool rope_ready = false;

    // accounting / profiling
    int64_t launches = 0;
    bool prof = false;
    std::vector<cudaEvent_t> ev_pool;
    std::vector<int> ev_class;     // class of event pair i (events 2i, 2i+1)
    size_t ev_used = 0;
    double prof_ms[vith::kProfClasses] = {};
    int64_t prof_n[vith::kProfClasses] = {};
    cudaStream_t last_stream = nullptr;

    // CUDA-graph replay of vit_encode (opt-in): the last few (grid, patches, out) signatures
    struct GraphEntry {
        std::vector<int32_t> grid;
        const void *patches = nullptr;
        void *out = nullptr;
        cudaGraphExec_t exec = nullptr;
        int64_t launches = 0;
        uint64_t last_use = 0;
    };
    bool graph_on = false;
    std::vector<GraphEntry> graphs;
    uint64_t graph_clock = 0;
    cudaStream_t capture_stream = nullptr;
};
