// Internal launcher interface between the step orchestrator (focus_api.cu) and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace focus {

// Every kernel of the step asks for the largest shared-memory carveout, so consecutive kernels never
// need the SMs to drain and reconfigure the L1 / shared split between them.  The configure_* functions
// set it (for the current device) at init and return false if an attribute could not be set.
inline bool max_shared_carveout(const void* fn) {
    return cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                (int)cudaSharedmemCarveoutMaxShared) == cudaSuccess;
}
bool configure_rows_kernels();
bool configure_attention_kernels();
bool configure_attention_tc_kernels();
bool configure_select_decode_kernels();
bool configure_select_kernel();
bool configure_simt_gemm_kernels();

// Launch with programmatic stream serialisation (the kernel starts with pdl_entry()); cluster_x > 0
// launches clusters of cluster_x CTAs along x.
template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              unsigned cluster_x, Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_x > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}
inline int launched(cudaError_t e) { return e == cudaSuccess ? 1 : -1; }

struct Dims {
    int L, D, Hq, Hkv, d, F, V, qkv;  // qkv = (Hq + 2 Hkv) d
    float eps;
};

// ---- row-wise kernels (rows.cu) ---------------------------------------------
template <typename T>
int launch_embed_norm(const int32_t* tokens, int rows, int V, const T* embed, const T* gamma, float eps, int D,
                       float* x, T* h, int* err, cudaStream_t s);

// x_out[r] = x_in[src] + sum_s part[s][src]  (src = src_map ? src_map[r] : r), then h_out[r] = RMSNorm(x_out[r]) * gamma.
// Rows r < (n_rows_dev ? *n_rows_dev : rows_bound).  h_out may be null (residual only).
template <typename T>
int launch_residual_norm(const float* x_in, const int32_t* src_map, const int32_t* n_rows_dev, int rows_bound,
                          const float* part, int n_splits, size_t part_stride, float* x_out, const T* gamma,
                          float eps, int D, T* h_out, cudaStream_t s);

// Sum the QKV GEMM partials, rotate q and k (rotate-half RoPE at P_b + j), write q rows and the
// row's K/V into the intra-block cache at (b, layer, :, :, j).
template <typename T>
int launch_qkv_finalize(const float* part, int n_splits, size_t part_stride, RowMap rm, const int32_t* prefix_len,
                         int max_prefix, const double* inv_freq, Dims dm, int layer, T* q_out, T* ibc, int* err,
                         cudaStream_t s);

// ---- attention (attention.cu) ------------------------------------------------
struct AttnArgs {
    const void* q;              // [rows, Hq d]
    void* o;                    // [rows, Hq d]
    const void* kv_pool;        // [n_pages, L, 2, Hkv, S, d]
    const void* ibc;            // [N, L, 2, Hkv, B, d]
    const int32_t* prefix_len;  // [N]
    const int32_t* page_table;  // [N, max_pages]
    const int32_t* row_offsets; // compacted phase: request b's rows are [row_offsets[b], row_offsets[b+1]); null = full phase
    float* imp_part;            // full phase: [N, Hkv, B] block-column sums of this layer (null = not wanted)
    int N, B, layer, L, Hq, Hkv, d;
    int max_pages, page_size, n_pages;
    int* err;
    // split-KV (tensor-core kernel): each (request, KV head, query tile) unit is walked by `pieces` CTAs;
    // pieces > 1 needs the scratch below for units * pieces <= split_cap (and units <= split_cap)
    int pieces;
    float* part_o;              // [unit * pieces + piece][64][128] unnormalised partial outputs
    float* part_ml;             // [unit * pieces + piece][64][2] partial row max / denominator (log2 domain)
    float* sb_buf;              // [unit][64][64] raw block-key scores (layers 0-1)
    int* counters;              // [unit] arrival counters, zero between launches
    int q_rows;                 // bound on query rows per request in this launch (B, or the kept-row cap)
    int q_rows_cap;             // rows the query buffer holds
    const int32_t* order;       // tcgen05 kernel: [N] request of each grid slot (null: slot b is request b)
};

constexpr int kAttnSplitCap = 1280;  // unit-pieces the split-KV scratch holds
// pieces for a launch of `units` work units whose longest key walk is `max_chunks` 64-key chunks
int attention_pieces(int units, int max_chunks);
template <typename T> int launch_attention(const AttnArgs& a, cudaStream_t s);
// bf16, head_dim 128: tensor-core kernel (attention_tc.cu); the full phase writes its importance column
// sums per (KV head, 64-vector query tile): imp_part [N, Hkv, q_tiles, B]
// Returns the number of launches, or -1 if a tensor map could not be built.
int launch_attention_tc(const AttnArgs& a, int q_tiles, cudaStream_t s);
int attention_q_tiles(int B, int G);
// tcgen05 kernel (attention_t5.cu) for units of more than 32 query vectors: 128-vector query tiles
bool attention_t5_used(int q_rows, int G);
int attention_t5_q_tiles(int q_rows, int G);
int launch_attention_t5(const AttnArgs& a, int q_tiles, cudaStream_t s);
bool configure_attention_t5_kernels();
bool attention_tc_page_size_ok(int page_size);  // KV page sizes the TMA page loader handles: 16, 32, 64

// ---- selection + compaction metadata (select.cu) ------------------------------
struct SelectArgs {
    const float* imp_part;      // [2, N, groups, B]: per-group importance partials, summed in group order
    const uint8_t* mask;        // [N, B]
    int N, B, groups, max_keep;
    float tau, alpha, forced_frac;
    int k_min, k_max;
    const int32_t* forced_idx;  // optional [N, max_keep]
    const int32_t* forced_cnt;  // optional [N]
    int32_t* keep_count;        // [N]
    int32_t* retained_idx;      // [N, max_keep]
    int32_t* row_offsets;       // [N + 1]
    float* importance_out;      // optional [2, N, B]
    int32_t* row_req;           // [R_max]
    int32_t* row_pos;           // [R_max]
    int32_t* row_src;           // [R_max] = b * B + j
    int32_t* n_rows;            // [1] = R
    int* err;
    const int32_t* prefix_len;  // [N] (clamped to [0, max_prefix] for the order)
    int max_prefix;
    int32_t* order;             // [N] requests by descending prefix length, ties by index (null: not wanted)
};
int launch_select(const SelectArgs& a, cudaStream_t s);

// ---- GEMM C = A B^T with fused epilogues (gemm_simt.cu, gemm_tc.cu) -------------
enum Epi { EPI_PARTIAL = 0, EPI_SWIGLU = 1, EPI_LMHEAD = 2, EPI_RESID = 3, EPI_QKV = 4 };

struct GemmArgs {
    const void* A;              // [M, K] row-major
    const void* B;              // [N, K] row-major (gate rows for SWIGLU)
    const void* B2;             // SWIGLU: up rows [N, K]
    int M_bound;                // rows bound (grid is sized for it)
    const int32_t* M_dev;       // live row count on the device (null = M_bound)
    int N, K;
    int splits;                 // split-K count (EPI_PARTIAL only)
    float* part;                // EPI_PARTIAL: [splits][M_bound][N] float32
    size_t split_stride;        //   elements between splits
    void* act;                  // EPI_SWIGLU: [M_bound, N] T = silu(A Bg^T) * (A Bu^T)
    float* lm_max;              // EPI_LMHEAD: [M_bound, n_tiles] tile max, sum exp(z - max), first argmax
    float* lm_sum;
    int32_t* lm_arg;
    int n_tiles;
    int tile_n;                 // EPI_LMHEAD: columns per stats tile
    // tcgen05 fused epilogues
    float* resid;               // EPI_RESID: [rows, N] float32 residual stream, resid += A B^T
    void* q_out;                // EPI_QKV: [rows, Hq d] rotated queries (bf16)
    void* ibc;                  // EPI_QKV: intra-block KV cache [N, L, 2, Hkv, B, d]: rotated K and V at (b, j)
    const int32_t* row_req;     // EPI_QKV: compacted rows -> request / block position (null: row = b * B + j)
    const int32_t* row_pos;
    const int32_t* prefix_len;
    const double* inv_freq;     // [d / 2] RoPE frequencies
    const float2* rope_tab;     // tensor-core epilogues: [positions][d / 2] (cos, sin) of pos * inv_freq
    int max_prefix, block, n_layers, layer, Hq, Hkv;
    int* err;
    // Row bounds above 256 with a live count known only on the device: the few-row and the many-row kernel
    // are both launched, and each works only if the live count is in its range (else it exits after its
    // programmatic-launch wait).  0: no gate, 1: live <= 256 only (few-row kernel), 2: live > 256 only.
    int live_gate;
};
constexpr int kGateFewRows = 1, kGateManyRows = 2;
template <typename T> int launch_gemm_simt(Epi epi, const GemmArgs& g, cudaStream_t s);
constexpr int kSimtTileN = 64;

// ---- LM-head combine + threshold decode (decode.cu) ------------------------------
struct DecodeArgs {
    const float* lm_max;
    const float* lm_sum;
    const int32_t* lm_arg;
    int n_tiles;
    const int32_t* row_offsets;
    const int32_t* keep_count;
    const int32_t* retained_idx;
    int max_keep;
    int32_t* tokens;
    uint8_t* mask;
    int N, B;
    float threshold;
    int32_t* decoded_ids;
    float* conf_out;
    int32_t* top_out;
    float* row_conf;            // [R_max] per kept row: confidence (written by the combine kernel)
    int32_t* row_top;           // [R_max] per kept row: top id
};
int launch_lm_combine(const DecodeArgs& a, int rows_bound, const int32_t* n_rows, cudaStream_t s);
int launch_decode(const DecodeArgs& a, cudaStream_t s);

}  // namespace focus
