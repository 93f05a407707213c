// Internal launcher interface between the step orchestrator (focus_api.cu) and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace focus {

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
};
template <typename T> int launch_attention(const AttnArgs& a, cudaStream_t s);
// bf16, head_dim 128: tensor-core kernel (attention_tc.cu); the full phase writes its importance column
// sums per (KV head, 64-vector query tile): imp_part [N, Hkv, q_tiles, B]
int launch_attention_tc(const AttnArgs& a, int q_tiles, cudaStream_t s);
int attention_q_tiles(int B, int G);

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
};
int launch_select(const SelectArgs& a, cudaStream_t s);

// ---- GEMM C = A B^T with fused epilogues (gemm_simt.cu, gemm_tc.cu) -------------
enum Epi { EPI_PARTIAL = 0, EPI_SWIGLU = 1, EPI_LMHEAD = 2 };

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
};
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
};
int launch_decode(const DecodeArgs& a, cudaStream_t s);

}  // namespace focus
