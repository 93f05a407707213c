// C ABI of one FOCUS focused denoising step: validation, workspace, and the launch sequence.
//
// Step order ("FOCUS: DLLMs Know How to Tame Their Compute Bound", project page, Overview):
//   embed + RMSNorm -> layers 0, 1 on all N*B rows (attention with fused importance column sums)
//   -> delta / budget / top-k / row map -> gather of the kept rows -> layers 2..L-1 on the kept rows
//   (intra-block KV-cache write, ragged paged attention) -> LM head with fused max / sum-exp / argmax
//   -> confidence-threshold decode.
// Every launch is sized from host-visible values (N, B, limits); the data-dependent kept-row count
// R lives in device memory and the compacted-phase kernels read it, so the step never syncs.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <new>
#include <vector>

#include <nvtx3/nvToolsExt.h>  // header-only; ranges are no-ops unless a profiler is attached

#include "launch.h"
#include "tc_gemm.h"
#include "block.h"

using namespace focus;

struct focus_ctx {
    focus_model_cfg cfg;
    focus_limits lim;
    int device;
    int sms;                // streaming multiprocessors of the device
    Dims dm;
    size_t elt;  // bytes per T
    // borrowed weights
    const void *embed, *final_norm, *lm_head;
    std::vector<const void*> wqkv, wo, wgate, wup, wdown, attn_norm, mlp_norm;
    // workspace (one allocation)
    void* ws;
    size_t ws_bytes;
    float *x_full, *x_c, *part, *imp_part, *lm_max, *lm_sum;
    void *h, *q, *o, *act;
    int32_t *row_req, *row_pos, *row_src, *n_rows, *lm_arg;
    double* inv_freq;
    float2* rope_tab;     // bf16 path: [rope_positions][head_dim / 2] (cos, sin)
    int32_t* masked_count;  // block loop: masked positions left after a step
    int32_t* req_order;     // [max_requests] requests by descending prefix length (kept-row attention order)
    int* err;
    float *att_part_o, *att_part_ml, *att_sb;
    int* att_counters;
    float* row_conf;
    int32_t* row_top;
    size_t part_rows;     // rows of the partial-sum buffer
    size_t split_stride;  // elements between split-K slices
    int lm_tiles_cap;
    TcPlan* tc;        // tcgen05 GEMM plan (bf16), null for float32
    int last_launches = -1;
    // per-class event timing (focus_profile_begin / _end)
    bool prof_active = false;
    int prof_class = -1, prof_cap = 0, prof_n = 0;
    std::vector<cudaEvent_t> prof_ev;
};

namespace {

constexpr int kMaxSplits = 8;

// NVTX range names, one per focus_kernel_class (profilers group the step's launches by these)
const char* const kClassNames[] = {"embed_norm", "qkv_finalize", "attn_score", "attn_ragged", "row_norm",
                                   "select", "decode", "gemm_full_qkv", "gemm_full_o", "gemm_full_gateup",
                                   "gemm_full_down", "gemm_qkv", "gemm_o", "gemm_gateup", "gemm_down",
                                   "gemm_lmhead"};
static_assert(sizeof(kClassNames) / sizeof(kClassNames[0]) == FOCUS_K_COUNT, "one name per kernel class");

struct Layout {
    size_t off[32];
    size_t total;
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool cfg_ok(const focus_model_cfg* c) {
    if (!c) return false;
    if (c->n_layers < 2 || c->hidden <= 0 || c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->ffn <= 0 || c->vocab <= 1)
        return false;
    if (c->n_q_heads % c->n_kv_heads) return false;
    if (c->dtype != FOCUS_DTYPE_F32 && c->dtype != FOCUS_DTYPE_BF16) return false;
    if (!(c->rms_eps >= 0.f) || !(c->rope_theta > 0.f)) return false;
    return true;
}

int shape_supported(const focus_model_cfg* c) {
    if (c->head_dim != 64 && c->head_dim != 128) return FOCUS_ERR_UNSUPPORTED;
    if (c->dtype == FOCUS_DTYPE_BF16 && c->head_dim != 128) return FOCUS_ERR_UNSUPPORTED;
    if (c->hidden % 128 || c->hidden > 4096 || c->ffn % 64) return FOCUS_ERR_UNSUPPORTED;
    return FOCUS_OK;
}

bool lim_ok(const focus_limits* l) {
    return l && l->max_requests > 0 && l->max_block > 0 && l->max_block <= 64 && l->max_keep > 0 &&
           l->max_keep <= l->max_block && l->max_pages_per_req > 0;
}

int lm_tiles(const focus_model_cfg* c) { return (c->vocab + kSimtTileN - 1) / kSimtTileN; }

// query tiles per (request, KV head) of the full-block attention (bf16 tensor-core kernel), 1 otherwise
int imp_tiles(const focus_model_cfg* c, const focus_limits* l) {
    return c->dtype == FOCUS_DTYPE_BF16 ? attention_q_tiles(l->max_block, c->n_q_heads / c->n_kv_heads) : 1;
}

// rotary positions a step can reach: the longest prefix (largest page size) plus the block
size_t rope_positions(const focus_limits* l) { return (size_t)l->max_pages_per_req * 64 + l->max_block; }

Layout plan(const focus_model_cfg* c, const focus_limits* l) {
    const size_t elt = c->dtype == FOCUS_DTYPE_BF16 ? 2 : 4;
    const size_t rows_full = (size_t)l->max_requests * l->max_block;
    const size_t rows_c = (size_t)l->max_requests * l->max_keep;
    const size_t D = c->hidden, HD = (size_t)c->n_q_heads * c->head_dim, F = c->ffn;
    const size_t qkv = (size_t)(c->n_q_heads + 2 * c->n_kv_heads) * c->head_dim;
    const size_t part_rows = rows_full > kMaxSplits * rows_c ? rows_full : kMaxSplits * rows_c;
    const size_t widest = qkv > D ? qkv : D;
    const size_t split = c->dtype == FOCUS_DTYPE_BF16 ? 1 : 0;
    const size_t sizes[] = {
        rows_full * D * 4,                                  // 0 x_full
        rows_c * D * 4,                                     // 1 x_c
        rows_full * D * elt,                                // 2 h
        rows_full * HD * elt,                               // 3 q
        rows_full * HD * elt,                               // 4 o
        rows_full * F * elt,                                // 5 act
        part_rows * widest * 4,                             // 6 part
        2 * (size_t)l->max_requests * c->n_kv_heads * imp_tiles(c, l) * l->max_block * 4,  // 7 imp_part
        rows_c * 4, rows_c * 4, rows_c * 4,                 // 8-10 row_req, row_pos, row_src
        64,                                                 // 11 n_rows
        rows_c * lm_tiles(c) * 4,                           // 12 lm_max
        rows_c * lm_tiles(c) * 4,                           // 13 lm_sum
        rows_c * lm_tiles(c) * 4,                           // 14 lm_arg
        (size_t)c->head_dim / 2 * 8,                        // 15 inv_freq
        64,                                                 // 16 err
        split * (size_t)kAttnSplitCap * 64 * 128 * 4,       // 17 attention split partial outputs
        split * (size_t)kAttnSplitCap * 64 * 2 * 4,         // 18 partial row max / denominator
        split * (size_t)kAttnSplitCap * 64 * 64 * 4,        // 19 raw block scores
        split * (size_t)kAttnSplitCap * 4,                  // 20 arrival counters
        rows_c * 4, rows_c * 4,                             // 21-22 per-row confidence / top id
        split * rope_positions(l) * (size_t)c->head_dim / 2 * 8,  // 23 RoPE (cos, sin) table
        64,                                                 // 24 block loop: masked-position count
        (size_t)l->max_requests * 4,                        // 25 request order
    };
    Layout lay{};
    size_t at = 0;
    for (int i = 0; i < 26; ++i) {
        lay.off[i] = at;
        at = align_up(at + sizes[i], 1024);
    }
    lay.total = at;
    return lay;
}

bool all_nonnull(const void* const* arr, int n) {
    if (!arr) return false;
    for (int i = 0; i < n; ++i)
        if (!arr[i]) return false;
    return true;
}

#define FOCUS_CUDA_TRY(x)                              \
    do {                                               \
        cudaError_t e_ = (x);                          \
        if (e_ != cudaSuccess) return FOCUS_ERR_CUDA;  \
    } while (0)

template <typename T>
int run_step(focus_ctx* c, const focus_batch* in, const focus_params* p, focus_step_out* out, cudaStream_t s,
             int k_cap) {
    const Dims& dm = c->dm;
    const int N = in->n_requests, B = in->block_size;
    const int rows_full = N * B;
    const int R_bound = N * k_cap;
    const int max_prefix = c->lim.max_pages_per_req * in->page_size;
    // split z of a GEMM's partial sums starts at z * stride; only compacted-row GEMMs split K, and
    // kMaxSplits slices of (max kept rows x widest output) fit in the buffer
    const size_t stride = c->split_stride;
    T* h = reinterpret_cast<T*>(c->h);
    T* q = reinterpret_cast<T*>(c->q);
    T* ibc = reinterpret_cast<T*>(in->ibc);
    auto W = [](const void* ptr) { return reinterpret_cast<const T*>(ptr); };
    const bool tc = c->cfg.dtype == FOCUS_DTYPE_BF16 && c->tc != nullptr;
    const bool bf = c->cfg.dtype == FOCUS_DTYPE_BF16;
    const int G = dm.Hq / dm.Hkv;
    const int qt_full = bf ? attention_q_tiles(B, G) : 1;         // importance partial groups per KV head
    const int qt_kept = bf ? attention_q_tiles(k_cap, G) : 1;
    auto attention = [&](const AttnArgs& args, int q_tiles) {
        return bf ? launch_attention_tc(args, q_tiles, s) : launch_attention<T>(args, s);
    };

    // every launch goes through here: launch accounting and optional per-class event timing
    int launches = 0;
    bool launch_failed = false;
    // inside a stream capture the profiling pairs are recorded as external event nodes of the graph,
    // so they time every replay; outside a capture they are plain records
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (c->prof_active) FOCUS_CUDA_TRY(cudaStreamIsCapturing(s, &cap));
    const unsigned rec_flags = cap == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
    auto run = [&](int kclass, auto&& launch) {
        nvtxRangePushA(kClassNames[kclass]);
        const bool timed = c->prof_active && c->prof_class == kclass && c->prof_n < c->prof_cap;
        if (timed && cudaEventRecordWithFlags(c->prof_ev[2 * c->prof_n], s, rec_flags) != cudaSuccess)
            launch_failed = true;
        const int n = launch();
        if (n < 0) launch_failed = true;
        else launches += n;
        if (timed) {
            if (cudaEventRecordWithFlags(c->prof_ev[2 * c->prof_n + 1], s, rec_flags) != cudaSuccess)
                launch_failed = true;
            ++c->prof_n;
        }
        nvtxRangePop();
    };
    auto gemm = [&](int kclass, Epi epi, const void* A, const void* Bw, const void* B2, int Mb, const int32_t* Md,
                    int Nn, int K, int splits, void* act_out, float* resid = nullptr, int layer = 0,
                    bool compact = false) {
        GemmArgs g{};
        g.A = A; g.B = Bw; g.B2 = B2; g.M_bound = Mb; g.M_dev = Md; g.N = Nn; g.K = K; g.splits = splits;
        g.part = c->part; g.split_stride = stride; g.act = act_out;
        g.lm_max = c->lm_max; g.lm_sum = c->lm_sum; g.lm_arg = c->lm_arg;
        g.resid = resid; g.q_out = c->q; g.ibc = in->ibc;
        g.row_req = compact ? c->row_req : nullptr; g.row_pos = compact ? c->row_pos : nullptr;
        g.prefix_len = in->prefix_len; g.inv_freq = c->inv_freq; g.rope_tab = c->rope_tab; g.max_prefix = max_prefix;
        g.block = B;
        g.n_layers = dm.L; g.layer = layer; g.Hq = dm.Hq; g.Hkv = dm.Hkv; g.err = c->err;
        run(kclass, [&] {
            if (tc) return tc_gemm(c->tc, epi, g, s);
            g.n_tiles = (Nn + kSimtTileN - 1) / kSimtTileN;
            g.tile_n = kSimtTileN;
            return launch_gemm_simt<T>(epi, g, s);
        });
    };

    AttnArgs at{};
    at.q = c->q; at.o = c->o; at.kv_pool = in->kv_pool; at.ibc = in->ibc; at.prefix_len = in->prefix_len;
    at.page_table = in->page_table; at.N = N; at.B = B; at.L = dm.L; at.Hq = dm.Hq; at.Hkv = dm.Hkv; at.d = dm.d;
    at.max_pages = c->lim.max_pages_per_req; at.page_size = in->page_size; at.n_pages = in->n_pages; at.err = c->err;
    at.part_o = c->att_part_o; at.part_ml = c->att_part_ml; at.sb_buf = c->att_sb; at.counters = c->att_counters;
    at.q_rows_cap = c->lim.max_requests * c->lim.max_block;
    const int max_chunks = (c->lim.max_pages_per_req * in->page_size + 63) / 64 + 1;
    const int pieces_full = bf ? attention_pieces(N * dm.Hkv * qt_full, max_chunks) : 1;
    const int pieces_kept = bf ? attention_pieces(N * dm.Hkv * qt_kept, max_chunks) : 1;
    if (bf) FOCUS_CUDA_TRY(cudaMemsetAsync(c->att_counters, 0, (size_t)kAttnSplitCap * 4, s));

    const RowMap full{nullptr, nullptr, nullptr, rows_full, B};
    const RowMap comp{c->row_req, c->row_pos, c->n_rows, R_bound, B};

    run(FOCUS_K_EMBED_NORM, [&] {
        return launch_embed_norm<T>(in->block_tokens, rows_full, dm.V, W(c->embed), W(c->attn_norm[0]), dm.eps, dm.D,
                                    c->x_full, h, c->err, s);
    });
    // tensor-core path: the GEMM epilogues apply RoPE + the cache write (QKV) and the residual adds
    // (O, down) themselves, reducing any split-K slices inside the GEMM; the row kernels only normalise
    // ---- layers 0 and 1: full block, importance at both
    for (int l = 0; l < 2; ++l) {
        if (tc) {
            gemm(FOCUS_K_GEMM_FULL_QKV, EPI_QKV, c->h, c->wqkv[l], nullptr, rows_full, nullptr, dm.qkv, dm.D, 1, nullptr, nullptr, l, false);
        } else {
            gemm(FOCUS_K_GEMM_FULL_QKV, EPI_PARTIAL, c->h, c->wqkv[l], nullptr, rows_full, nullptr, dm.qkv, dm.D, 1, nullptr);
            run(FOCUS_K_QKV_FINALIZE, [&] {
                return launch_qkv_finalize<T>(c->part, 1, stride, full, in->prefix_len, max_prefix, c->inv_freq, dm,
                                              l, q, ibc, c->err, s);
            });
        }
        at.layer = l;
        at.q_rows = B;
        at.row_offsets = nullptr;
        at.imp_part = c->imp_part + (size_t)l * N * dm.Hkv * qt_full * B;
        at.pieces = pieces_full;
        run(FOCUS_K_ATTN_SCORE, [&] { return attention(at, qt_full); });
        const int nsp_full = tc ? 0 : 1;  // partial slices the norm kernels still add (CUDA-core path)
        gemm(FOCUS_K_GEMM_FULL_O, tc ? EPI_RESID : EPI_PARTIAL, c->o, c->wo[l], nullptr, rows_full, nullptr, dm.D,
             dm.Hq * dm.d, 1, nullptr, c->x_full, l, false);
        run(FOCUS_K_ROW_NORM, [&] {
            return launch_residual_norm<T>(c->x_full, nullptr, nullptr, rows_full, c->part, nsp_full, stride, c->x_full,
                                           W(c->mlp_norm[l]), dm.eps, dm.D, h, s);
        });
        gemm(FOCUS_K_GEMM_FULL_GATEUP, EPI_SWIGLU, c->h, c->wgate[l], c->wup[l], rows_full, nullptr, dm.F, dm.D, 1, c->act);
        gemm(FOCUS_K_GEMM_FULL_DOWN, tc ? EPI_RESID : EPI_PARTIAL, c->act, c->wdown[l], nullptr, rows_full, nullptr,
             dm.D, dm.F, 1, nullptr, c->x_full, l, false);
        if (l == 0)
            run(FOCUS_K_ROW_NORM, [&] {
                return launch_residual_norm<T>(c->x_full, nullptr, nullptr, rows_full, c->part, nsp_full, stride,
                                               c->x_full, W(c->attn_norm[1]), dm.eps, dm.D, h, s);
            });
    }
    // ---- delta, budget, top-k, row map
    SelectArgs sa{};
    sa.imp_part = c->imp_part; sa.mask = in->mask; sa.N = N; sa.B = B; sa.groups = dm.Hkv * qt_full;
    sa.max_keep = c->lim.max_keep;
    sa.tau = p->tau; sa.alpha = p->alpha; sa.forced_frac = p->forced_keep_frac; sa.k_min = p->k_min; sa.k_max = p->k_max;
    sa.forced_idx = p->forced_keep_idx; sa.forced_cnt = p->forced_keep_count;
    sa.keep_count = out->keep_count; sa.retained_idx = out->retained_idx; sa.row_offsets = out->row_offsets;
    sa.importance_out = out->importance; sa.row_req = c->row_req; sa.row_pos = c->row_pos; sa.row_src = c->row_src;
    sa.n_rows = c->n_rows; sa.err = c->err;
    sa.prefix_len = in->prefix_len; sa.max_prefix = max_prefix; sa.order = bf ? c->req_order : nullptr;
    run(FOCUS_K_SELECT, [&] { return launch_select(sa, s); });
    // ---- gather the kept rows (folding in layer 1's MLP partial sums) and normalise for layer 2
    const void* g_next = dm.L > 2 ? c->attn_norm[2] : c->final_norm;
    run(FOCUS_K_ROW_NORM, [&] {
        return launch_residual_norm<T>(c->x_full, c->row_src, c->n_rows, R_bound, c->part, tc ? 0 : 1, stride, c->x_c,
                                       W(g_next), dm.eps, dm.D, h, s);
    });
    // ---- layers 2..L-1 on the kept rows
    // the tensor-core GEMMs pick their own split-K for the kept rows and reduce it in the epilogue
    const int sp_qkv = 1, sp_o = 1, sp_dn = 1;
    for (int l = 2; l < dm.L; ++l) {
        if (tc) {
            gemm(FOCUS_K_GEMM_QKV, EPI_QKV, c->h, c->wqkv[l], nullptr, R_bound, c->n_rows, dm.qkv, dm.D, sp_qkv,
                 nullptr, nullptr, l, true);
        } else {
            gemm(FOCUS_K_GEMM_QKV, EPI_PARTIAL, c->h, c->wqkv[l], nullptr, R_bound, c->n_rows, dm.qkv, dm.D, sp_qkv, nullptr);
            run(FOCUS_K_QKV_FINALIZE, [&] {
                return launch_qkv_finalize<T>(c->part, sp_qkv, stride, comp, in->prefix_len, max_prefix, c->inv_freq,
                                              dm, l, q, ibc, c->err, s);
            });
        }
        at.layer = l;
        at.q_rows = k_cap;
        at.row_offsets = out->row_offsets;
        at.imp_part = nullptr;
        // longest prefix first (written by the row-map kernel) when the units outnumber the CTAs resident at
        // once (two per SM); a single wave gains nothing and keeps the mma.sync kernel's early chunk copies
        at.order = bf && (attention_t5_used(k_cap, dm.Hq / dm.Hkv) || N * dm.Hkv * qt_kept > 2 * c->sms)
                       ? c->req_order
                       : nullptr;
        at.pieces = pieces_kept;
        run(FOCUS_K_ATTN_RAGGED, [&] { return attention(at, qt_kept); });
        gemm(FOCUS_K_GEMM_O, tc ? EPI_RESID : EPI_PARTIAL, c->o, c->wo[l], nullptr, R_bound, c->n_rows, dm.D,
             dm.Hq * dm.d, sp_o, nullptr, c->x_c, l, true);
        run(FOCUS_K_ROW_NORM, [&] {
            return launch_residual_norm<T>(c->x_c, nullptr, c->n_rows, R_bound, c->part, tc ? 0 : sp_o, stride, c->x_c,
                                           W(c->mlp_norm[l]), dm.eps, dm.D, h, s);
        });
        gemm(FOCUS_K_GEMM_GATEUP, EPI_SWIGLU, c->h, c->wgate[l], c->wup[l], R_bound, c->n_rows, dm.F, dm.D, 1, c->act);
        gemm(FOCUS_K_GEMM_DOWN, tc ? EPI_RESID : EPI_PARTIAL, c->act, c->wdown[l], nullptr, R_bound, c->n_rows, dm.D,
             dm.F, sp_dn, nullptr, c->x_c, l, true);
        const void* gn = l + 1 < dm.L ? c->attn_norm[l + 1] : c->final_norm;
        run(FOCUS_K_ROW_NORM, [&] {
            return launch_residual_norm<T>(c->x_c, nullptr, c->n_rows, R_bound, c->part, tc ? 0 : sp_dn, stride, c->x_c,
                                           W(gn), dm.eps, dm.D, h, s);
        });
    }
    // ---- LM head (fused max / sum-exp / argmax per vocabulary tile), combine, decode
    gemm(FOCUS_K_GEMM_LMHEAD, EPI_LMHEAD, c->h, c->lm_head, nullptr, R_bound, c->n_rows, dm.V, dm.D, 1, nullptr);
    DecodeArgs da{};
    da.lm_max = c->lm_max; da.lm_sum = c->lm_sum; da.lm_arg = c->lm_arg;
    da.n_tiles = tc ? tc_lm_tiles(c->tc) : (dm.V + kSimtTileN - 1) / kSimtTileN;
    da.row_offsets = out->row_offsets; da.keep_count = out->keep_count; da.retained_idx = out->retained_idx;
    da.max_keep = c->lim.max_keep; da.tokens = in->block_tokens; da.mask = in->mask; da.N = N; da.B = B;
    da.threshold = p->conf_threshold; da.decoded_ids = out->decoded_ids; da.conf_out = out->conf;
    da.top_out = out->top_id;
    da.row_conf = c->row_conf; da.row_top = c->row_top;
    run(FOCUS_K_DECODE, [&] { return launch_lm_combine(da, R_bound, c->n_rows, s); });
    run(FOCUS_K_DECODE, [&] { return launch_decode(da, s); });
    c->last_launches = launches;
    if (launch_failed) return FOCUS_ERR_CUDA;
    if (out->hidden && R_bound > 0)
        FOCUS_CUDA_TRY(cudaMemcpyAsync(out->hidden, c->x_c, (size_t)R_bound * dm.D * sizeof(float),
                                       cudaMemcpyDeviceToDevice, s));
    FOCUS_CUDA_TRY(cudaGetLastError());
    return FOCUS_OK;
}

void prof_release(focus_ctx* c) {
    for (cudaEvent_t e : c->prof_ev) cudaEventDestroy(e);
    c->prof_ev.clear();
    c->prof_active = false;
    c->prof_cap = c->prof_n = 0;
}

}  // namespace

extern "C" {

const char* focus_status_string(int status) {
    switch (status) {
        case FOCUS_OK: return "ok";
        case FOCUS_ERR_INVALID_ARG: return "invalid argument";
        case FOCUS_ERR_LIMITS: return "request exceeds the context's limits";
        case FOCUS_ERR_CUDA: return "CUDA runtime error";
        case FOCUS_ERR_TIMEOUT: return "device-side bounded wait expired";
        case FOCUS_ERR_DEVICE_BOUNDS: return "device-side index check failed";
        case FOCUS_ERR_UNSUPPORTED: return "unsupported model shape";
        case FOCUS_ERR_NO_MEMORY: return "workspace allocation failed";
        default: return "unknown status";
    }
}

size_t focus_workspace_bytes(const focus_model_cfg* cfg, const focus_limits* lim) {
    if (!cfg_ok(cfg) || !lim_ok(lim)) return 0;
    return plan(cfg, lim).total;
}

int focus_init(const focus_model_cfg* cfg, const focus_weights* w, const focus_limits* lim, focus_ctx** out) {
    if (!out) return FOCUS_ERR_INVALID_ARG;
    *out = nullptr;
    if (!cfg_ok(cfg) || !w || !lim_ok(lim)) return FOCUS_ERR_INVALID_ARG;
    const int sup = shape_supported(cfg);
    if (sup != FOCUS_OK) return sup;
    const int L = cfg->n_layers;
    if (!w->embed || !w->final_norm || !w->lm_head || !all_nonnull(w->wqkv, L) || !all_nonnull(w->wo, L) ||
        !all_nonnull(w->wgate, L) || !all_nonnull(w->wup, L) || !all_nonnull(w->wdown, L) ||
        !all_nonnull(w->attn_norm, L) || !all_nonnull(w->mlp_norm, L))
        return FOCUS_ERR_INVALID_ARG;
    focus_ctx* c = new (std::nothrow) focus_ctx();
    if (!c) return FOCUS_ERR_NO_MEMORY;
    c->cfg = *cfg;
    c->lim = *lim;
    if (cudaGetDevice(&c->device) != cudaSuccess) {
        delete c;
        return FOCUS_ERR_CUDA;
    }
    if (cudaDeviceGetAttribute(&c->sms, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess) {
        delete c;
        return FOCUS_ERR_CUDA;
    }
    c->dm = Dims{L, cfg->hidden, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim, cfg->ffn, cfg->vocab,
                 (cfg->n_q_heads + 2 * cfg->n_kv_heads) * cfg->head_dim, cfg->rms_eps};
    c->elt = cfg->dtype == FOCUS_DTYPE_BF16 ? 2 : 4;
    c->embed = w->embed;
    c->final_norm = w->final_norm;
    c->lm_head = w->lm_head;
    c->wqkv.assign(w->wqkv, w->wqkv + L);
    c->wo.assign(w->wo, w->wo + L);
    c->wgate.assign(w->wgate, w->wgate + L);
    c->wup.assign(w->wup, w->wup + L);
    c->wdown.assign(w->wdown, w->wdown + L);
    c->attn_norm.assign(w->attn_norm, w->attn_norm + L);
    c->mlp_norm.assign(w->mlp_norm, w->mlp_norm + L);

    const Layout lay = plan(cfg, lim);
    if (cudaMalloc(&c->ws, lay.total) != cudaSuccess) {
        cudaGetLastError();
        delete c;
        return FOCUS_ERR_NO_MEMORY;
    }
    c->ws_bytes = lay.total;
    char* base = static_cast<char*>(c->ws);
    c->x_full = reinterpret_cast<float*>(base + lay.off[0]);
    c->x_c = reinterpret_cast<float*>(base + lay.off[1]);
    c->h = base + lay.off[2];
    c->q = base + lay.off[3];
    c->o = base + lay.off[4];
    c->act = base + lay.off[5];
    c->part = reinterpret_cast<float*>(base + lay.off[6]);
    c->imp_part = reinterpret_cast<float*>(base + lay.off[7]);
    c->row_req = reinterpret_cast<int32_t*>(base + lay.off[8]);
    c->row_pos = reinterpret_cast<int32_t*>(base + lay.off[9]);
    c->row_src = reinterpret_cast<int32_t*>(base + lay.off[10]);
    c->n_rows = reinterpret_cast<int32_t*>(base + lay.off[11]);
    c->lm_max = reinterpret_cast<float*>(base + lay.off[12]);
    c->lm_sum = reinterpret_cast<float*>(base + lay.off[13]);
    c->lm_arg = reinterpret_cast<int32_t*>(base + lay.off[14]);
    c->inv_freq = reinterpret_cast<double*>(base + lay.off[15]);
    c->rope_tab = reinterpret_cast<float2*>(base + lay.off[23]);
    c->masked_count = reinterpret_cast<int32_t*>(base + lay.off[24]);
    c->req_order = reinterpret_cast<int32_t*>(base + lay.off[25]);
    c->err = reinterpret_cast<int*>(base + lay.off[16]);
    c->att_part_o = reinterpret_cast<float*>(base + lay.off[17]);
    c->att_part_ml = reinterpret_cast<float*>(base + lay.off[18]);
    c->att_sb = reinterpret_cast<float*>(base + lay.off[19]);
    c->att_counters = reinterpret_cast<int*>(base + lay.off[20]);
    c->row_conf = reinterpret_cast<float*>(base + lay.off[21]);
    c->row_top = reinterpret_cast<int32_t*>(base + lay.off[22]);
    const size_t rows_full = (size_t)lim->max_requests * lim->max_block;
    const size_t rows_c = (size_t)lim->max_requests * lim->max_keep;
    c->part_rows = rows_full > kMaxSplits * rows_c ? rows_full : kMaxSplits * rows_c;
    c->split_stride = rows_c * (size_t)(c->dm.qkv > c->dm.D ? c->dm.qkv : c->dm.D);
    c->lm_tiles_cap = lm_tiles(cfg);

    std::vector<double> inv(cfg->head_dim / 2);
    for (int i = 0; i < cfg->head_dim / 2; ++i)
        inv[i] = pow((double)cfg->rope_theta, -2.0 * i / (double)cfg->head_dim);
    int rc = FOCUS_OK;
    if (cfg->dtype == FOCUS_DTYPE_BF16) {
        const size_t npos = rope_positions(lim), half = (size_t)cfg->head_dim / 2;
        std::vector<float2> tab(npos * half);
        for (size_t pos = 0; pos < npos; ++pos)
            for (size_t i = 0; i < half; ++i) {
                const double ang = (double)pos * inv[i];
                tab[pos * half + i] = make_float2((float)cos(ang), (float)sin(ang));
            }
        if (cudaMemcpy(c->rope_tab, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess)
            rc = FOCUS_ERR_CUDA;
    }
    if (cudaMemcpy(c->inv_freq, inv.data(), inv.size() * sizeof(double), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemset(c->err, 0, sizeof(int)) != cudaSuccess || cudaMemset(c->n_rows, 0, sizeof(int)) != cudaSuccess ||
        (cfg->dtype == FOCUS_DTYPE_BF16 &&
         cudaMemset(c->att_counters, 0, (size_t)kAttnSplitCap * 4) != cudaSuccess))
        rc = FOCUS_ERR_CUDA;
    if (rc == FOCUS_OK && !(configure_rows_kernels() && configure_attention_kernels() &&
                            configure_select_decode_kernels() && configure_simt_gemm_kernels()))
        rc = FOCUS_ERR_CUDA;
    c->tc = nullptr;
    if (rc == FOCUS_OK && cfg->dtype == FOCUS_DTYPE_BF16) {
        TcWeights tw{};
        tw.L = L;
        tw.wqkv = c->wqkv.data(); tw.wo = c->wo.data(); tw.wgate = c->wgate.data(); tw.wup = c->wup.data();
        tw.wdown = c->wdown.data(); tw.lm_head = c->lm_head;
        rc = tc_plan_create(&c->tc, c->dm, tw, c->h, c->o, c->act, (int)rows_full, (int)rows_c, c->lm_tiles_cap,
                            c->err);
    }
    if (rc != FOCUS_OK) {
        cudaFree(c->ws);
        delete c;
        return rc;
    }
    *out = c;
    return FOCUS_OK;
}

int focus_step(focus_ctx* c, const focus_batch* in, const focus_params* p, focus_step_out* out, void* stream) {
    if (!c || !in || !p || !out) return FOCUS_ERR_INVALID_ARG;
    const int N = in->n_requests, B = in->block_size;
    if (N < 0 || B <= 0 || in->page_size <= 0 || in->n_pages < 0) return FOCUS_ERR_INVALID_ARG;
    if (N > c->lim.max_requests || B > c->lim.max_block) return FOCUS_ERR_LIMITS;
    if (!in->block_tokens || !in->mask || !in->prefix_len || !in->page_table || !in->ibc ||
        (in->n_pages > 0 && !in->kv_pool))
        return FOCUS_ERR_INVALID_ARG;
    if (!out->keep_count || !out->retained_idx || !out->row_offsets || !out->decoded_ids || !out->conf ||
        !out->top_id)
        return FOCUS_ERR_INVALID_ARG;
    if (!(p->alpha >= 0.f) || p->k_min < 0 || p->k_max < 0 || p->tau != p->tau || p->conf_threshold != p->conf_threshold)
        return FOCUS_ERR_INVALID_ARG;
    if ((p->forced_keep_idx == nullptr) != (p->forced_keep_count == nullptr)) return FOCUS_ERR_INVALID_ARG;
    int k_cap;
    if (p->forced_keep_idx) {
        k_cap = c->lim.max_keep < B ? c->lim.max_keep : B;
    } else if (p->forced_keep_frac >= 0.f) {
        if (p->forced_keep_frac > 1.f) return FOCUS_ERR_INVALID_ARG;
        k_cap = (int)ceilf(p->forced_keep_frac * (float)B);
        if (k_cap > B) k_cap = B;
        if (k_cap > c->lim.max_keep) return FOCUS_ERR_LIMITS;
    } else {
        if (p->k_max > B || p->k_min > p->k_max) return FOCUS_ERR_INVALID_ARG;
        if (p->k_max > c->lim.max_keep) return FOCUS_ERR_LIMITS;
        k_cap = p->k_max;
    }
    if (c->cfg.dtype == FOCUS_DTYPE_BF16 && !attention_tc_page_size_ok(in->page_size)) return FOCUS_ERR_UNSUPPORTED;
    if (N == 0) return FOCUS_OK;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != c->device) return FOCUS_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    nvtxRangePushA("focus_step");
    const int rc = c->cfg.dtype == FOCUS_DTYPE_BF16 ? run_step<bf16>(c, in, p, out, s, k_cap)
                                                    : run_step<float>(c, in, p, out, s, k_cap);
    nvtxRangePop();
    return rc;
}

int focus_commit_block(focus_ctx* c, const focus_batch* in, void* stream) {
    if (!c || !in) return FOCUS_ERR_INVALID_ARG;
    const int N = in->n_requests, B = in->block_size;
    if (N < 0 || B <= 0 || in->page_size <= 0 || in->n_pages <= 0) return FOCUS_ERR_INVALID_ARG;
    if (N > c->lim.max_requests || B > c->lim.max_block) return FOCUS_ERR_LIMITS;
    if (!in->prefix_len || !in->page_table || !in->ibc || !in->kv_pool) return FOCUS_ERR_INVALID_ARG;
    if (N == 0) return FOCUS_OK;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != c->device) return FOCUS_ERR_INVALID_ARG;
    CommitArgs a{};
    a.ibc = in->ibc;
    // the step only reads the pages and prefix lengths; the commit is the one call that writes them
    a.kv_pool = const_cast<void*>(in->kv_pool);
    a.prefix_len = const_cast<int32_t*>(in->prefix_len);
    a.page_table = in->page_table;
    a.N = N;
    a.L = c->dm.L;
    a.Hkv = c->dm.Hkv;
    a.B = B;
    a.d = c->dm.d;
    a.S = in->page_size;
    a.max_pages = c->lim.max_pages_per_req;
    a.n_pages = in->n_pages;
    a.elt = (int)c->elt;
    a.err = c->err;
    return launch_commit_block(a, static_cast<cudaStream_t>(stream)) < 0 ? FOCUS_ERR_CUDA : FOCUS_OK;
}

int focus_decode_block(focus_ctx* c, const focus_batch* in, const focus_params* p, int32_t max_steps,
                       focus_step_out* out, int32_t* steps_taken, void* stream) {
    if (!c || !in || !p || !out || max_steps < 1) return FOCUS_ERR_INVALID_ARG;
    if (steps_taken) *steps_taken = 0;
    const int N = in->n_requests, B = in->block_size;
    if (B > c->lim.max_keep) return FOCUS_ERR_LIMITS;  // the dense steps keep every position
    if (p->forced_keep_idx) return FOCUS_ERR_INVALID_ARG;
    if (N <= 0) return N == 0 ? FOCUS_OK : FOCUS_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    focus_params dense = *p, focused = *p;
    dense.forced_keep_frac = 1.f;
    focused.forced_keep_frac = -1.f;
    auto masked_left = [&](int32_t* left) {
        if (launch_count_masked(in->mask, N * B, c->masked_count, s) < 0 ||
            cudaMemcpyAsync(left, c->masked_count, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return FOCUS_ERR_CUDA;
        return FOCUS_OK;
    };
    // the block's first step is dense; then focused steps until nothing is masked
    int rc = focus_step(c, in, &dense, out, stream);
    int steps = 1;
    int32_t left = 0;
    if (rc == FOCUS_OK) rc = masked_left(&left);
    while (rc == FOCUS_OK && left > 0 && steps < max_steps) {
        rc = focus_step(c, in, &focused, out, stream);
        ++steps;
        if (rc == FOCUS_OK) rc = masked_left(&left);
    }
    if (steps_taken) *steps_taken = steps;
    if (rc != FOCUS_OK) return rc;
    if (left > 0) return FOCUS_ERR_LIMITS;  // not decoded within max_steps: nothing is committed
    // one dense refresh of the decoded block (its cache then holds the final tokens' K/V), then commit
    rc = focus_step(c, in, &dense, out, stream);
    if (rc != FOCUS_OK) return rc;
    return focus_commit_block(c, in, stream);
}

int focus_destroy(focus_ctx* c) {
    if (!c) return FOCUS_OK;
    int prev = -1;
    cudaGetDevice(&prev);
    cudaSetDevice(c->device);
    int rc = cudaDeviceSynchronize() == cudaSuccess ? FOCUS_OK : FOCUS_ERR_CUDA;
    prof_release(c);
    if (c->tc) tc_plan_destroy(c->tc);
    if (cudaFree(c->ws) != cudaSuccess) rc = FOCUS_ERR_CUDA;
    if (prev >= 0) cudaSetDevice(prev);
    delete c;
    return rc;
}

int focus_get_device_error(focus_ctx* c, int32_t* bits) {
    if (!c) return FOCUS_ERR_INVALID_ARG;
    int prev = -1;
    cudaGetDevice(&prev);
    if (cudaSetDevice(c->device) != cudaSuccess) return FOCUS_ERR_CUDA;
    int v = 0;
    int rc = FOCUS_OK;
    if (cudaDeviceSynchronize() != cudaSuccess || cudaMemcpy(&v, c->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(c->err, 0, sizeof(int)) != cudaSuccess)
        rc = FOCUS_ERR_CUDA;
    if (prev >= 0) cudaSetDevice(prev);
    if (bits) *bits = v;
    if (rc != FOCUS_OK) return rc;
    if (v & FOCUS_DEVERR_TIMEOUT) return FOCUS_ERR_TIMEOUT;
    return v ? FOCUS_ERR_DEVICE_BOUNDS : FOCUS_OK;
}

int focus_probe_wait_timeout(focus_ctx* c, void* stream) {
    if (!c) return FOCUS_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != c->device) return FOCUS_ERR_INVALID_ARG;
    return launch_wait_timeout_probe(c->err, static_cast<cudaStream_t>(stream)) == 1 ? FOCUS_OK : FOCUS_ERR_CUDA;
}

int focus_last_step_launches(const focus_ctx* c) { return c ? c->last_launches : -1; }

int focus_profile_begin(focus_ctx* c, int kernel_class, int max_launches) {
    if (!c || kernel_class < 0 || kernel_class >= FOCUS_K_COUNT || max_launches <= 0) return FOCUS_ERR_INVALID_ARG;
    int prev = -1;
    cudaGetDevice(&prev);
    cudaSetDevice(c->device);
    prof_release(c);
    int rc = FOCUS_OK;
    c->prof_ev.resize(2 * (size_t)max_launches);
    for (auto& e : c->prof_ev)
        if (cudaEventCreate(&e) != cudaSuccess) rc = FOCUS_ERR_CUDA;
    if (rc == FOCUS_OK) {
        c->prof_class = kernel_class;
        c->prof_cap = max_launches;
        c->prof_n = 0;
        c->prof_active = true;
    } else {
        c->prof_ev.clear();
    }
    if (prev >= 0) cudaSetDevice(prev);
    return rc;
}

int focus_profile_end(focus_ctx* c, float* total_ms, int32_t* launches) {
    if (!c) return FOCUS_ERR_INVALID_ARG;
    c->prof_active = false;
    int prev = -1;
    cudaGetDevice(&prev);
    cudaSetDevice(c->device);
    int rc = cudaDeviceSynchronize() == cudaSuccess ? FOCUS_OK : FOCUS_ERR_CUDA;
    float tot = 0.f;
    for (int i = 0; rc == FOCUS_OK && i < c->prof_n; ++i) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, c->prof_ev[2 * i], c->prof_ev[2 * i + 1]) != cudaSuccess) rc = FOCUS_ERR_CUDA;
        tot += ms;
    }
    if (total_ms) *total_ms = tot;
    if (launches) *launches = c->prof_n;
    prof_release(c);
    if (prev >= 0) cudaSetDevice(prev);
    return rc;
}

}  // extern "C"
