// bf16 GEMM C = A B^T on the 5th-generation tensor cores (tcgen05.mma, accumulators in TMEM,
// operands staged by TMA), with the step's fused epilogues:
//   EPI_SWIGLU:  the B tile is BN/2 gate rows followed by BN/2 up rows; writes silu(g) * u (bf16)
//   EPI_LMHEAD:  per row and vocabulary tile: max logit, sum exp(z - max), first argmax (no logits in HBM)
//   EPI_RESID:   resid += A B^T (float32 residual stream)
//   EPI_QKV:     rotary embedding of the query / key heads, queries to q, keys and values to the cache
//
// GEMMs of at most 256 rows (the kept rows and the LM head) run on the swapped kernel (features on the
// MMA's M side, tokens on N, split K over a thread-block cluster).  GEMMs with more rows (the full-block
// GEMMs of layers 0-1, the kept rows of large batches) run on the persistent kernel (tc_gemm_persist.cuh:
// one CTA per SM, 128 x 256 or 128 x 128 tiles, two TMEM accumulators so that epilogues overlap the next
// tile's MMAs) when they have enough tiles to fill the SMs, else on the one-tile-per-CTA row-major kernel.
//
// One CTA computes a (128 * MSUB) x BN tile (MSUB accumulators of 128 x BN fp32 in TMEM) over a range of
// 64-wide K blocks.  Warp roles: warp 0 lane 0 issues TMA loads into a STAGES-deep shared-memory ring,
// warp 1 owns the TMEM allocation and its lane 0 issues tcgen05.mma (one elected thread), warps 2..5
// read the accumulators back with tcgen05.ld (each warp reads its own 32-lane quarter) and run the
// epilogue.  Operand tiles are K-major with the 128-byte swizzle that TMA writes; no cluster multicast.
// The weights are written by no kernel of the step, so the producer issues the weight tiles of the first
// ring stages before the programmatic-launch wait; the activation / token tiles are issued after it.
// Every mbarrier wait is bounded: on expiry the kernel flags FOCUS_DEVERR_TIMEOUT, still waits (bounded)
// for its own in-flight copies, frees its TMEM and returns.
#include <unordered_map>

#include "tc_gemm.h"
#include "tc_gemm_kernel.cuh"
#include "tc_gemm_persist.cuh"

namespace focus {

namespace {

using namespace tc;

// ------------------------------------------------------------------ host side
// Many rows (layers 0-1: N*B rows): 256 x 128 tiles, two 128-row TMEM accumulators sharing each weight
// tile, or 128 x 128 tiles for the residual and QKV GEMMs when 256-row tiles would leave SMs idle.  At
// most 256 rows (layers 2..L-1 and the LM head: at most N*k_max kept rows, typically a few dozen): the
// swapped kernel.  More kept rows than that (large batches) take the row-major kernel, whose CTAs with
// all rows beyond the live row count exit after the wait.
constexpr int kBN = 128, kStages = 4;
constexpr int kSmallRows = kTcFewRows;  // GEMMs with at most this many rows run on the swapped kernel
constexpr bool kUsePairs = true;   // many-row GEMMs on CTA pairs (tc_gemmp2_kernel) where they fill the GPU
using Big = TcShape<kBN, 2, kStages>;
using Small = TcShape<kBN, 1, kStages>;

}  // namespace

struct TcPlan {
    Dims dm;
    int rows_full, rows_c;
    const void *h, *o, *act;
    CUtensorMap map_h, map_o, map_act;        // 256-row boxes
    CUtensorMap map_h1, map_o1, map_act1;     // 128-row boxes
    CUtensorMap map_h32, map_o32, map_act32;  // 32-row boxes: token operand of the swapped kernel
    std::unordered_map<const void*, CUtensorMap> wmap;   // weight pointer -> map (box rows = tile N or N/2)
    std::unordered_map<const void*, CUtensorMap> wmap2;  // the same with 256-row boxes (128 for gate / up)
    std::unordered_map<const void*, CUtensorMap> wmap32; // O and down weights in 32-row boxes (column slabs)
    int* err;
    int sms;
    int max_clusters[kTMaxSplits + 1];  // co-resident clusters of the swapped kernel with s CTAs (0: not launchable)
    int max_pairs;                      // co-resident CTA pairs of the paired persistent kernel (0: not used)
    // fp32 maps of the residual streams and the split-tile partial buffer (pointer -> rows, map), built on
    // first use: the residual epilogue adds and stores through them
    std::unordered_map<const void*, std::pair<uint64_t, CUtensorMap>> fmap;
};



int tc_plan_create(TcPlan** out, const Dims& dm, const TcWeights& w, void* h, void* o, void* act, int rows_full,
                   int rows_c, int lm_tiles_cap, int* err) {
    *out = nullptr;
    if (dm.D % BK || dm.F % BK || (dm.Hq * dm.d) % BK || dm.qkv % kBN || dm.D % kBN || dm.F % (kBN / 2))
        return FOCUS_OK;  // shapes outside the tiling run on the CUDA-core GEMM
    if ((dm.V + kBN - 1) / kBN > lm_tiles_cap) return FOCUS_ERR_INVALID_ARG;
    if (!encode_fn()) return FOCUS_ERR_CUDA;
    TcPlan* p = new TcPlan();
    p->dm = dm;
    p->rows_full = rows_full;
    p->rows_c = rows_c;
    p->h = h;
    p->o = o;
    p->act = act;
    p->err = err;
    const uint64_t HD = (uint64_t)dm.Hq * dm.d;
    bool ok = make_map(&p->map_h, h, rows_full, dm.D, Big::BM) && make_map(&p->map_o, o, rows_full, HD, Big::BM) &&
              make_map(&p->map_act, act, rows_full, dm.F, Big::BM) &&
              make_map(&p->map_h1, h, rows_full, dm.D, Small::BM) && make_map(&p->map_o1, o, rows_full, HD, Small::BM) &&
              make_map(&p->map_act1, act, rows_full, dm.F, Small::BM) && make_map(&p->map_h32, h, rows_full, dm.D, 32) &&
              make_map(&p->map_o32, o, rows_full, HD, 32) && make_map(&p->map_act32, act, rows_full, dm.F, 32);
    for (int l = 0; ok && l < w.L; ++l) {
        CUtensorMap m;
        ok = ok && make_map(&m, w.wqkv[l], dm.qkv, dm.D, kBN);
        p->wmap[w.wqkv[l]] = m;
        ok = ok && make_map(&m, w.wo[l], dm.D, HD, kBN);
        p->wmap[w.wo[l]] = m;
        ok = ok && make_map(&m, w.wgate[l], dm.F, dm.D, kBN / 2);
        p->wmap[w.wgate[l]] = m;
        ok = ok && make_map(&m, w.wup[l], dm.F, dm.D, kBN / 2);
        p->wmap[w.wup[l]] = m;
        ok = ok && make_map(&m, w.wdown[l], dm.D, dm.F, kBN);
        p->wmap[w.wdown[l]] = m;
        ok = ok && make_map(&m, w.wqkv[l], dm.qkv, dm.D, 2 * kBN);
        p->wmap2[w.wqkv[l]] = m;
        ok = ok && make_map(&m, w.wo[l], dm.D, HD, 2 * kBN);
        p->wmap2[w.wo[l]] = m;
        ok = ok && make_map(&m, w.wgate[l], dm.F, dm.D, kBN);
        p->wmap2[w.wgate[l]] = m;
        ok = ok && make_map(&m, w.wup[l], dm.F, dm.D, kBN);
        p->wmap2[w.wup[l]] = m;
        ok = ok && make_map(&m, w.wdown[l], dm.D, dm.F, 2 * kBN);
        p->wmap2[w.wdown[l]] = m;
        ok = ok && make_map(&m, w.wo[l], dm.D, HD, 32);
        p->wmap32[w.wo[l]] = m;
        ok = ok && make_map(&m, w.wdown[l], dm.D, dm.F, 32);
        p->wmap32[w.wdown[l]] = m;
    }
    CUtensorMap m;
    ok = ok && make_map(&m, w.lm_head, dm.V, dm.D, kBN);
    p->wmap[w.lm_head] = m;
    ok = ok && make_map(&m, w.lm_head, dm.V, dm.D, 2 * kBN);
    p->wmap2[w.lm_head] = m;
    if (!ok) {
        delete p;
        return FOCUS_ERR_CUDA;
    }
    auto set_smem = [](const void* fn, int bytes) {
        return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess &&
               max_shared_carveout(fn);
    };
    ok = set_smem((const void*)tc_gemm_kernel<kBN, 2, kStages, EPI_SWIGLU>, Big::SMEM) &&
         set_smem((const void*)tc_gemm_kernel<kBN, 2, kStages, EPI_LMHEAD>, Big::SMEM) &&
         set_smem((const void*)tc_gemm_kernel<kBN, 2, kStages, EPI_RESID>, Big::SMEM) &&
         set_smem((const void*)tc_gemm_kernel<kBN, 2, kStages, EPI_QKV>, Big::SMEM) &&
         set_smem((const void*)tc_gemm_kernel<kBN, 1, kStages, EPI_RESID>, Small::SMEM) &&
         set_smem((const void*)tc_gemm_kernel<kBN, 1, kStages, EPI_QKV>, Small::SMEM) &&
         set_smem((const void*)tc_gemmt_kernel<EPI_RESID>, kTSmem) &&
         set_smem((const void*)tc_gemmt_kernel<EPI_QKV>, kTSmem) &&
         set_smem((const void*)tc_gemmt_kernel<EPI_SWIGLU>, kTSmem) &&
         set_smem((const void*)tc_gemmt_kernel<EPI_LMHEAD>, kTSmem) &&
         set_smem((const void*)tc_gemmp_kernel<256, EPI_SWIGLU>, PShape<256>::SMEM) &&
         set_smem((const void*)tc_gemmp_kernel<256, EPI_LMHEAD>, PShape<256>::SMEM) &&
         set_smem((const void*)tc_gemmp_kernel<256, EPI_RESID>, PShape<256>::SMEM_RESID) &&
         set_smem((const void*)tc_gemmp_kernel<256, EPI_QKV>, PShape<256>::SMEM) &&
         set_smem((const void*)tc_gemmp_kernel<128, EPI_SWIGLU>, PShape<128>::SMEM) &&
         set_smem((const void*)tc_gemmp_kernel<128, EPI_LMHEAD>, PShape<128>::SMEM) &&
         set_smem((const void*)tc_gemmp_kernel<128, EPI_RESID>, PShape<128>::SMEM_RESID) &&
         set_smem((const void*)tc_gemmp_kernel<128, EPI_QKV>, PShape<128>::SMEM) &&
         set_smem((const void*)tc_gemmp2_kernel<EPI_SWIGLU>, kP2Smem) &&
         set_smem((const void*)tc_gemmp2_kernel<EPI_LMHEAD>, kP2Smem) &&
         set_smem((const void*)tc_gemmp2_kernel<EPI_RESID>, kP2Smem) &&
         set_smem((const void*)tc_gemmp2_kernel<EPI_QKV>, kP2Smem);
    int dev = 0;
    p->sms = 0;
    ok = ok && cudaGetDevice(&dev) == cudaSuccess &&
         cudaDeviceGetAttribute(&p->sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && p->sms > 0;
    // how many clusters of each size fit at once (a cluster's CTAs share one GPC, so this is not
    // simply SMs / size)
    p->max_clusters[0] = 0;
    for (int cs = 1; ok && cs <= kTMaxSplits; ++cs) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(cs, 1, 1);
        cfg.blockDim = dim3(192, 1, 1);
        cfg.dynamicSmemBytes = kTSmem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cs;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, tc_gemmt_kernel<EPI_RESID>, &cfg) != cudaSuccess) {
            (void)cudaGetLastError();  // a cluster shape the device does not take is simply not used
            n = 0;
        }
        p->max_clusters[cs] = n;
    }
    ok = ok && p->max_clusters[1] > 0;
    p->max_pairs = 0;
    if (ok && kUsePairs) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(2, 1, 1);
        cfg.blockDim = dim3(192, 1, 1);
        cfg.dynamicSmemBytes = kP2Smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, tc_gemmp2_kernel<EPI_RESID>, &cfg) != cudaSuccess) {
            (void)cudaGetLastError();
            n = 0;
        }
        p->max_pairs = n;
    }
    if (!ok) {
        delete p;
        return FOCUS_ERR_CUDA;
    }
    *out = p;
    return FOCUS_OK;
}

void tc_plan_destroy(TcPlan* p) { delete p; }

int tc_lm_tiles(const TcPlan* p) { return p ? (p->dm.V + kBN - 1) / kBN : 0; }

namespace {

// fp32 [rows, cols] map of `base` (cached per pointer; rebuilt when the row count changes); null on failure
const CUtensorMap* f32_map(TcPlan* p, const void* base, uint64_t rows, uint64_t cols) {
    auto it = p->fmap.find(base);
    if (it != p->fmap.end() && it->second.first == rows) return &it->second.second;
    CUtensorMap m;
    if (!make_map_f32(&m, base, rows, cols)) return nullptr;
    auto& slot = p->fmap[base];
    slot = {rows, m};
    return &slot.second;
}

// Slabs per tile when a residual GEMM has fewer pair tiles than co-resident pairs (then all its tiles form
// one partial round): 4 or 2 if that many slabs of every tile still fit on the pairs.
int launch_slabs(Epi epi, long long tiles, int max_pairs) {
    if (epi != EPI_RESID || tiles >= max_pairs) return 1;
    return tiles * 4 <= max_pairs ? 4 : tiles * 2 <= max_pairs ? 2 : 1;
}

// Swapped GEMM: 128-feature tiles x all live tokens, split K over a cluster of 1..8 CTAs (each slice keeps
// at least one K block).  The LM head (many feature tiles) does not split.
int tc_gemm_swapped(TcPlan* p, Epi epi, GemmArgs g, cudaStream_t s) {
    const CUtensorMap* x = g.A == p->h ? &p->map_h32 : g.A == p->o ? &p->map_o32 : &p->map_act32;
    const CUtensorMap* w = &p->wmap.find(g.B)->second;  // 128-row boxes; 64-row boxes for gate / up
    const CUtensorMap* w2 = epi == EPI_SWIGLU ? &p->wmap.find(g.B2)->second : w;
    const int n_tiles = epi == EPI_SWIGLU ? g.N / 64 : (g.N + 127) / 128;
    // split K into the largest power of two of slices (at most 8, each with at least one K block) that
    // keeps the grid within the two CTAs per SM that the shared-memory ring allows (measured on the
    // 1.7B shapes: O, down and QKV best at 8 slices, gate/up at 2; three-CTA clusters place poorly)
    int splits = 1;
    if (epi != EPI_LMHEAD)
        while (splits * 2 <= kTMaxSplits && splits * 2 <= g.K / BK && n_tiles * splits * 2 <= 2 * p->sms &&
               p->max_clusters[splits * 2] > 0)
            splits *= 2;
    if (epi == EPI_LMHEAD) {
        g.n_tiles = n_tiles;
        g.tile_n = 128;
    }
    const dim3 grid(splits, n_tiles, 1), blk(192);
    const unsigned cx = (unsigned)splits;
    cudaError_t e;
    switch (epi) {
        case EPI_RESID: e = launch_pdl(tc_gemmt_kernel<EPI_RESID>, grid, blk, kTSmem, s, cx, *w, *w2, *x, g, p->err); break;
        case EPI_QKV: e = launch_pdl(tc_gemmt_kernel<EPI_QKV>, grid, blk, kTSmem, s, cx, *w, *w2, *x, g, p->err); break;
        case EPI_LMHEAD:
            e = launch_pdl(tc_gemmt_kernel<EPI_LMHEAD>, grid, blk, kTSmem, s, cx, *w, *w2, *x, g, p->err);
            break;
        default: e = launch_pdl(tc_gemmt_kernel<EPI_SWIGLU>, grid, blk, kTSmem, s, cx, *w, *w2, *x, g, p->err); break;
    }
    return e == cudaSuccess ? 1 : -1;
}

// Persistent kernel for many rows: 128 x bn tiles over min(SMs, tiles) CTAs.
template <int BN>
int tc_gemm_persistent(TcPlan* p, Epi epi, GemmArgs g, int tiles, cudaStream_t s) {
    const CUtensorMap* a = g.A == p->h ? &p->map_h1 : g.A == p->o ? &p->map_o1 : &p->map_act1;
    auto& wm = BN == 256 ? p->wmap2 : p->wmap;
    const CUtensorMap* b = &wm.find(g.B)->second;
    const CUtensorMap* b2 = epi == EPI_SWIGLU ? &wm.find(g.B2)->second : b;
    if (epi == EPI_LMHEAD) {
        g.n_tiles = (g.N + kBN - 1) / kBN;  // statistics per 128 vocabulary columns, as the combine reads them
        g.tile_n = kBN;
    }
    const CUtensorMap* c = a;  // the residual stream (EPI_RESID), unused otherwise
    if (epi == EPI_RESID && !(c = f32_map(p, g.resid, (uint64_t)g.M_bound, (uint64_t)g.N))) return -1;
    const dim3 grid(tiles < p->sms ? tiles : p->sms, 1, 1), blk(192);
    const int smem = PShape<BN>::SMEM;
    switch (epi) {
        case EPI_SWIGLU: return launched(launch_pdl(tc_gemmp_kernel<BN, EPI_SWIGLU>, grid, blk, smem, s, 0, *a, *b, *b2, *c, g, p->err));
        case EPI_LMHEAD: return launched(launch_pdl(tc_gemmp_kernel<BN, EPI_LMHEAD>, grid, blk, smem, s, 0, *a, *b, *b2, *c, g, p->err));
        case EPI_RESID:
            return launched(launch_pdl(tc_gemmp_kernel<BN, EPI_RESID>, grid, blk, PShape<BN>::SMEM_RESID, s, 0, *a, *b, *b2,
                                       *c, g, p->err));
        case EPI_QKV: return launched(launch_pdl(tc_gemmp_kernel<BN, EPI_QKV>, grid, blk, smem, s, 0, *a, *b, *b2, *c, g, p->err));
        default: return -1;
    }
}

// Paired persistent kernel: 256 x 256 tiles over min(co-resident pairs, tiles) clusters of 2 CTAs.
int tc_gemm_pairs(TcPlan* p, Epi epi, GemmArgs g, int tiles, cudaStream_t s) {
    const CUtensorMap* a = g.A == p->h ? &p->map_h1 : g.A == p->o ? &p->map_o1 : &p->map_act1;
    // 128-row weight boxes: each rank loads half of the tile's 256 weight rows (gate or up for SwiGLU)
    const CUtensorMap* b = &p->wmap2.find(g.B)->second;
    const CUtensorMap* b2 = b;
    if (epi == EPI_SWIGLU) {
        b = &p->wmap2.find(g.B)->second;
        b2 = &p->wmap2.find(g.B2)->second;
    } else {
        b = &p->wmap.find(g.B)->second;
        b2 = b;
    }
    if (epi == EPI_LMHEAD) {
        g.n_tiles = (g.N + kBN - 1) / kBN;
        g.tile_n = kBN;
    }
    // EPI_RESID: the residual stream, and the weights in 32-row boxes for the column slabs of a last round
    const CUtensorMap *c = a, *bt = a;
    if (epi == EPI_RESID) {
        if (!(c = f32_map(p, g.resid, (uint64_t)g.M_bound, (uint64_t)g.N))) return -1;
        auto it = p->wmap32.find(g.B);
        if (it == p->wmap32.end()) return -1;
        bt = &it->second;
    }
    // fewer tiles than pairs: enough pairs for the column slabs of every tile
    const int pairs = tiles < p->max_pairs ? tiles * launch_slabs(epi, tiles, p->max_pairs) : p->max_pairs;
    const dim3 grid(2 * pairs, 1, 1), blk(192);
    switch (epi) {
        case EPI_SWIGLU: return launched(launch_pdl(tc_gemmp2_kernel<EPI_SWIGLU>, grid, blk, kP2Smem, s, 2, *a, *b, *b2, *c, *bt, g, p->err));
        case EPI_LMHEAD: return launched(launch_pdl(tc_gemmp2_kernel<EPI_LMHEAD>, grid, blk, kP2Smem, s, 2, *a, *b, *b2, *c, *bt, g, p->err));
        case EPI_RESID: return launched(launch_pdl(tc_gemmp2_kernel<EPI_RESID>, grid, blk, kP2Smem, s, 2, *a, *b, *b2, *c, *bt, g, p->err));
        case EPI_QKV: return launched(launch_pdl(tc_gemmp2_kernel<EPI_QKV>, grid, blk, kP2Smem, s, 2, *a, *b, *b2, *c, *bt, g, p->err));
        default: return -1;
    }
}

// Column slabs per tile of a last partial round of `tiles` pair tiles over `pairs` pairs (residual GEMMs:
// the most of 4 or 2 that keeps that round within the pairs; the kernel applies the same rule).
int slabs(Epi epi, long long tiles, int pairs) {
    const long long rem = tiles % pairs;
    if (epi != EPI_RESID || rem == 0) return 1;
    return rem * 4 <= pairs ? 4 : rem * 2 <= pairs ? 2 : 1;
}

// Rounds of tile-MMA time a pair launch takes: the full rounds, plus a slab's share of a round for the last.
double pair_rounds(Epi epi, long long tiles, int max_pairs) {
    const int pairs = (int)(tiles < max_pairs ? tiles * launch_slabs(epi, tiles, max_pairs) : max_pairs);
    const long long full = tiles / pairs, rem = tiles % pairs;
    return (double)full + (rem ? 1.0 / slabs(epi, tiles, pairs) : 0.0);
}

// Column tiles of width bn (0 if the epilogue needs whole tiles and N does not divide).
int persist_col_tiles(Epi epi, int N, int bn) {
    if (epi == EPI_SWIGLU) return N % (bn / 2) ? 0 : N / (bn / 2);
    if (epi == EPI_LMHEAD) return (N + bn - 1) / bn;  // a partial last tile is masked column by column
    return N % bn ? 0 : N / bn;
}

}  // namespace

namespace {

// GEMMs of more than kSmallRows rows (at the row bound)
int tc_gemm_many(TcPlan* p, Epi epi, GemmArgs g, cudaStream_t s) {
    {
        // Persistent kernel when there are enough tiles to fill the SMs.  Of 256- and 128-wide tiles take the
        // one with the shorter expected time: full waves of tiles (at the row bound) x tile width, a 128-wide
        // tile costing 15 % more per column (half-width MMAs, twice the A traffic per flop).
        const int mt = (g.M_bound + 127) / 128;
        const int n256 = persist_col_tiles(epi, g.N, 256), n128 = persist_col_tiles(epi, g.N, 128);
        const long long t256 = (long long)mt * n256, t128 = (long long)mt * n128;
        const double c256 = n256 ? (double)((t256 + p->sms - 1) / p->sms) * 256.0 : 1e30;
        const double c128 = n128 ? (double)((t128 + p->sms - 1) / p->sms) * 128.0 * 1.15 : 1e30;
        if (p->max_pairs > 0 && n256) {
            // pairs: 256 x 256 tiles, one round = max_pairs tiles; a round takes about as long as a round of
            // 128 x 256 tiles on single CTAs, at two thirds of their operand bytes per flop.  Residual GEMMs cut
            // the tiles of a last partial round into 64- or 128-column slabs (pair_rounds).
            const long long tp = (long long)((g.M_bound + 255) / 256) * n256;
            const double cp = pair_rounds(epi, tp, p->max_pairs) * 256.0 * (2.0 * p->max_pairs / p->sms);
            if ((tp >= p->max_pairs || epi == EPI_RESID) && cp <= c256 && cp <= c128)
                return tc_gemm_pairs(p, epi, g, (int)tp, s);
        }
        if (n256 && t256 >= p->sms && c256 <= c128) return tc_gemm_persistent<256>(p, epi, g, (int)t256, s);
        if (n128 && t128 >= p->sms) return tc_gemm_persistent<128>(p, epi, g, (int)t128, s);
    }
    // residual and QKV GEMMs whose 256-row tiles would leave SMs idle take 128-row tiles
    const int n_tiles_big = (g.N + kBN - 1) / kBN;
    const bool rows128 = (epi == EPI_RESID || epi == EPI_QKV) &&
                         n_tiles_big * ((g.M_bound + Big::BM - 1) / Big::BM) < p->sms;
    const CUtensorMap* a = g.A == p->h ? (rows128 ? &p->map_h1 : &p->map_h)
                         : g.A == p->o ? (rows128 ? &p->map_o1 : &p->map_o)
                                       : (rows128 ? &p->map_act1 : &p->map_act);
    const CUtensorMap* b = &p->wmap.find(g.B)->second;
    const CUtensorMap* b2 = epi == EPI_SWIGLU ? &p->wmap.find(g.B2)->second : b;
    const int n_tiles = epi == EPI_SWIGLU ? g.N / (kBN / 2) : (g.N + kBN - 1) / kBN;
    if (epi == EPI_LMHEAD) {
        g.n_tiles = n_tiles;
        g.tile_n = kBN;
    }
    const int bm = rows128 ? Small::BM : Big::BM;
    const dim3 grid(n_tiles, (g.M_bound + bm - 1) / bm, 1), blk(192);
    if (rows128 && epi == EPI_RESID)
        return launched(launch_pdl(tc_gemm_kernel<kBN, 1, kStages, EPI_RESID>, grid, blk, Small::SMEM, s, 0, *a, *b, *b2,
                                   g, p->err));
    if (rows128 && epi == EPI_QKV)
        return launched(launch_pdl(tc_gemm_kernel<kBN, 1, kStages, EPI_QKV>, grid, blk, Small::SMEM, s, 0, *a, *b, *b2, g,
                                   p->err));
    switch (epi) {
        case EPI_SWIGLU:
            return launched(launch_pdl(tc_gemm_kernel<kBN, 2, kStages, EPI_SWIGLU>, grid, blk, Big::SMEM, s, 0, *a, *b,
                                       *b2, g, p->err));
        case EPI_LMHEAD:
            return launched(launch_pdl(tc_gemm_kernel<kBN, 2, kStages, EPI_LMHEAD>, grid, blk, Big::SMEM, s, 0, *a, *b,
                                       *b2, g, p->err));
        case EPI_RESID:
            return launched(launch_pdl(tc_gemm_kernel<kBN, 2, kStages, EPI_RESID>, grid, blk, Big::SMEM, s, 0, *a, *b,
                                       *b2, g, p->err));
        case EPI_QKV:
            return launched(launch_pdl(tc_gemm_kernel<kBN, 2, kStages, EPI_QKV>, grid, blk, Big::SMEM, s, 0, *a, *b, *b2,
                                       g, p->err));
        default:
            return -1;
    }
}

}  // namespace

int tc_gemm(TcPlan* p, Epi epi, const GemmArgs& g0, cudaStream_t s) {
    if (g0.M_bound <= 0) return 0;
    if (epi == EPI_PARTIAL) return -1;  // partial sums are the CUDA-core path's; these kernels fuse their epilogues
    GemmArgs g = g0;
    if (g.M_bound <= kSmallRows) return tc_gemm_swapped(p, epi, g, s);
    if (g.M_dev == nullptr) return tc_gemm_many(p, epi, g, s);
    // kept rows whose bound exceeds the few-row kernel but whose live count may not: launch both kernels;
    // each reads the live count after its programmatic wait and only one of them works
    GemmArgs gf = g;
    gf.live_gate = kGateFewRows;
    const int n_few = tc_gemm_swapped(p, epi, gf, s);
    if (n_few < 0) return -1;
    g.live_gate = kGateManyRows;
    const int n_many = tc_gemm_many(p, epi, g, s);
    return n_many < 0 ? -1 : n_few + n_many;
}

}  // namespace focus
