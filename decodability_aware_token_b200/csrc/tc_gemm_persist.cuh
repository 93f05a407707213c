// Persistent row-major tcgen05 GEMM for GEMMs with many rows: the full-block GEMMs of layers 0-1 (N*B rows)
// and the kept-row GEMMs once more than 256 rows are kept.  C = A B^T, A [M, K] activations, B [N, K]
// weights, bf16 operands, fp32 accumulation in TMEM, the step's fused epilogues.
//
// One CTA per SM walks output tiles of 128 rows x BN columns (BN = 256: one M = 128, N = 256 MMA per
// 16-wide K slice; BN = 128 where 256-wide tiles would leave a poorly filled last wave).  Warp roles:
// warp 0 lane 0 streams A and B tiles by TMA into a ring of STAGES stages that runs on across tile
// boundaries; warp 1 owns TMEM and its lane 0 issues the MMAs; warps 2..5 drain accumulators through
// tcgen05.ld and run the epilogue.  TMEM holds two accumulators, so the epilogue of one tile runs while
// the MMAs of the next fill the other: the tensor pipe does not wait for epilogues, and a CTA pays its
// set-up (barriers, TMEM allocation, tensor-map prefetch) once rather than once per tile.
//
// Tile order: bands of consecutive 128-row tiles (about 32 MB of A each), and within a band all column
// tiles, row tile fastest.  The CTAs in flight at any moment then share a band of A and a few weight
// slices, both L2-resident, so A comes from DRAM once per launch and the weights once per band.
//
// Every mbarrier wait is bounded: on expiry the waiting role flags FOCUS_DEVERR_TIMEOUT and stops; the
// producer still waits (bounded) for its own copies in flight, the MMA thread waits (bounded) for all MMAs
// it issued to complete, and TMEM is released only after both.  No cluster multicast.
#pragma once
#include "tc_gemm_kernel.cuh"

namespace focus {
namespace tc {
namespace {

template <int BN>
struct PShape {
    static constexpr int A_BYTES = 128 * BK * 2;                // 16 KB
    static constexpr int B_BYTES = BN * BK * 2;                 // 32 KB at BN = 256
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES = (192 * 1024) / STAGE;         // 4 stages at BN = 256, 6 at BN = 128
    static constexpr int SMEM = STAGES * STAGE + 1024;          // + alignment slack
    static constexpr int SMEM_RESID = SMEM + 32 * 1024;         // + the residual epilogue's staging boxes
    static constexpr uint32_t TMEM_COLS = 2 * BN;               // two accumulators
    static_assert(BN == 128 || BN == 256, "MMA N");
    static_assert(STAGES >= 2 && STAGES <= 8, "ring depth");
};

constexpr size_t kBandBytes = 32u << 20;  // A bytes per band of row tiles

// Output tile `t` of the launch -> (row tile, column tile).
__device__ __forceinline__ void persist_tile(int t, int Mt, int Nt, int Bm, int& m, int& n) {
    const int band_tiles = Bm * Nt;
    const int band = t / band_tiles;
    const int r = t - band * band_tiles;
    const int bw = min(Bm, Mt - band * Bm);   // only the last band may be narrower
    n = r / bw;
    m = band * Bm + (r - n * bw);
}

// ---- residual epilogue through TMA reductions
// Each epilogue warp moves 32 rows x 32 columns of the accumulator at a time into a 4 KB staging box in
// shared memory (fp32 rows of 128 bytes with the 128-byte swizzle the tensor map names: 16-byte piece q of
// row r sits at piece q ^ (r % 8)), and one lane adds the box into the residual stream with a TMA reduction
// (cp.reduce.async.bulk.tensor, .add on f32).  The residual never enters the SM, every global access is a
// whole 128-byte line, and each element receives exactly one addition (x + acc, rounded once, as a plain
// read-modify-write would give).  Rows at or past the live row count add +0; boxes wholly past it are not
// sent.  Two boxes per warp alternate; a box is rewritten only after the reduction issued from it two boxes
// earlier has finished reading it.
constexpr int kResidBox = 32 * 32 * 4;            // one staging box: 4 KB
constexpr int kResidStage = 4 * 2 * kResidBox;    // four epilogue warps x two boxes: 32 KB
static_assert(PShape<256>::SMEM_RESID - PShape<256>::SMEM == kResidStage &&
                  PShape<128>::SMEM_RESID - PShape<128>::SMEM == kResidStage,
              "staging boxes after the ring");
static_assert(PShape<256>::SMEM_RESID <= 227 * 1024 && PShape<128>::SMEM_RESID <= 227 * 1024, "one CTA per SM");

__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int x, int y) {
    asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];"
                 ::"l"(map), "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// at most one bulk group of this thread still reading shared memory
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// every bulk group of this thread complete (its global writes performed)
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// `cols` (a multiple of 32) accumulator columns of this warp's 32 TMEM lanes through the staging boxes, added
// into rows row0 .. row0 + 31, columns col0 .. of the residual stream.  Rows at or past `row_end` add +0 and
// boxes wholly past it are skipped.  `boxes` = this warp's two staging boxes, `nbox` = boxes this warp has
// sent so far.
__device__ __forceinline__ void resid_add_tma(const CUtensorMap* map, uint8_t* boxes, uint32_t tacc, int cols, int row0,
                                              int col0, int row_end, uint32_t& nbox) {
    const int lane = threadIdx.x & 31;
    const bool live = row0 + lane < row_end;
    const bool any = row0 < row_end;  // warp-uniform
#pragma unroll 1
    for (int c0 = 0; c0 < cols; c0 += 32) {
        float v[32];
        tmem_ld32(tacc + c0, v);  // warp-collective: every lane
        if (!any) continue;
        uint8_t* box = boxes + (nbox & 1u) * kResidBox;
        if (lane == 0 && nbox >= 2) bulk_wait_read_1();
        __syncwarp();
        uint8_t* rowp = box + lane * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(rowp + ((q ^ (lane & 7)) << 4)) =
                live ? make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]) : make_float4(0.f, 0.f, 0.f, 0.f);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the box is visible to the TMA unit
        __syncwarp();
        if (lane == 0) tma_reduce_add_2d(map, box, col0 + c0, row0);
        ++nbox;
    }
}

// Epilogue of one accumulator (128 rows x BN columns) for this thread's row; `tacc` is the TMEM address
// of the warp's lane quarter at column 0 of the accumulator.  Every lane executes every tcgen05.ld;
// `live` only guards the stores.
template <int BN, int EPI>
__device__ __forceinline__ void persist_epilogue(const GemmArgs& g, uint32_t tacc, int row, bool live, int n_tile) {
    if constexpr (EPI == EPI_RESID) {
        float* xr = g.resid + (size_t)row * g.N + (size_t)n_tile * BN;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
            float v[32];
            tmem_ld32(tacc + c0, v);
            if (live) {
                float4* x4 = reinterpret_cast<float4*>(xr + c0);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float4 x = x4[q];
                    x.x += v[4 * q];
                    x.y += v[4 * q + 1];
                    x.z += v[4 * q + 2];
                    x.w += v[4 * q + 3];
                    x4[q] = x;
                }
            }
        }
    } else if constexpr (EPI == EPI_QKV) {
        // 128-column heads; rotate pairs (i, i + 64) of query and key heads, then q rows or the cache
        int b = 0, j = 0, pos = 0;
        if (live) qkv_row(g, row, b, j, pos);
#pragma unroll 1
        for (int hs = 0; hs < BN / 128; ++hs) {
            const int head = n_tile * (BN / 128) + hs;
            const bool rotate = head < g.Hq + g.Hkv;
            bf16* dst = live ? qkv_dst(g, row, head, b, j) : nullptr;
#pragma unroll 1
            for (int c0 = 0; c0 < 64; c0 += 32) {
                float lo[32], hi[32];
                tmem_ld32(tacc + hs * 128 + c0, lo);
                tmem_ld32(tacc + hs * 128 + 64 + c0, hi);
                if (live) {
#pragma unroll
                    for (int t = 0; t < 32; t += 8) {
                        float a[8], bb[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            a[e] = lo[t + e];
                            bb[e] = hi[t + e];
                            if (rotate) {
                                float cn, sn;
                                rope_cs(g, pos, c0 + t + e, cn, sn);
                                a[e] = lo[t + e] * cn - hi[t + e] * sn;
                                bb[e] = hi[t + e] * cn + lo[t + e] * sn;
                            }
                        }
                        uint32_t wa[4], wb[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            __nv_bfloat162 pa = __floats2bfloat162_rn(a[2 * e], a[2 * e + 1]);
                            __nv_bfloat162 pb = __floats2bfloat162_rn(bb[2 * e], bb[2 * e + 1]);
                            wa[e] = *reinterpret_cast<uint32_t*>(&pa);
                            wb[e] = *reinterpret_cast<uint32_t*>(&pb);
                        }
                        *reinterpret_cast<uint4*>(dst + c0 + t) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
                        *reinterpret_cast<uint4*>(dst + 64 + c0 + t) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
                    }
                }
            }
        }
    } else if constexpr (EPI == EPI_SWIGLU) {
        // columns [0, BN/2) of the accumulator are gate rows, [BN/2, BN) the matching up rows
        constexpr int H = BN / 2;
        bf16* out = reinterpret_cast<bf16*>(g.act) + (size_t)row * g.N + (size_t)n_tile * H;
#pragma unroll 1
        for (int c0 = 0; c0 < H; c0 += 32) {
            float gt[32], up[32];
            tmem_ld32(tacc + c0, gt);
            tmem_ld32(tacc + H + c0, up);
            if (live) {
                uint4* o4 = reinterpret_cast<uint4*>(out + c0);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i0 = 8 * q + 2 * e;
                        const float a0 = gt[i0] / (1.f + expf(-gt[i0])) * up[i0];
                        const float a1 = gt[i0 + 1] / (1.f + expf(-gt[i0 + 1])) * up[i0 + 1];
                        __nv_bfloat162 p2 = __floats2bfloat162_rn(a0, a1);
                        w[e] = *reinterpret_cast<uint32_t*>(&p2);
                    }
                    o4[q] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
    } else {
        // LM head: per row and 128-column vocabulary tile, the max logit, sum exp(z - max) and first argmax
#pragma unroll 1
        for (int hs = 0; hs < BN / 128; ++hs) {
            const int st = n_tile * (BN / 128) + hs;
            const int col0 = st * 128;
            float mx = -CUDART_INF_F, se = 0.f;
            int arg = 0x7fffffff;
#pragma unroll 1
            for (int c0 = 0; c0 < 128; c0 += 32) {
                float v[32];
                tmem_ld32(tacc + hs * 128 + c0, v);
                float cm = -CUDART_INF_F;
                int ca = 0x7fffffff;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (col0 + c0 + i < g.N && v[i] > cm) {
                        cm = v[i];
                        ca = col0 + c0 + i;
                    }
                if (cm > mx) {
                    se = (mx == -CUDART_INF_F) ? 0.f : se * expf(mx - cm);
                    mx = cm;
                    arg = ca;
                }
                if (cm != -CUDART_INF_F) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (col0 + c0 + i < g.N) se += expf(v[i] - mx);
                }
            }
            if (live && st < g.n_tiles) {
                const size_t idx = (size_t)row * g.n_tiles + st;
                g.lm_max[idx] = mx;
                g.lm_sum[idx] = se;
                g.lm_arg[idx] = arg;
            }
        }
    }
}

// tmC: the fp32 residual stream (box 32 columns x 32 rows, 128-byte swizzle), read by EPI_RESID only.
template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1) tc_gemmp_kernel(const __grid_constant__ CUtensorMap tmA,
                                                          const __grid_constant__ CUtensorMap tmB,
                                                          const __grid_constant__ CUtensorMap tmB2,
                                                          const __grid_constant__ CUtensorMap tmC, GemmArgs g,
                                                          int* err) {
    pdl_trigger();
    using S = PShape<BN>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[S::STAGES];
    __shared__ __align__(8) uint64_t empty_bar[S::STAGES];
    __shared__ __align__(8) uint64_t acc_full[2];
    __shared__ __align__(8) uint64_t acc_empty[2];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint32_t tmem_slot;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    if (threadIdx.x == 0) {
        for (int s = 0; s < S::STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);  // one arrival per epilogue warp
        }
        mbar_init(&done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                     "r"(S::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB) : "memory");
        if (EPI == EPI_SWIGLU) asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB2) : "memory");
    }
    pdl_wait();

    const int live = min(g.M_dev ? *g.M_dev : g.M_bound, g.M_bound);
    const int M = g.live_gate == kGateManyRows && live <= 256 ? 0 : live;  // 0: the few-row kernel's launch
    const int Mt = (M + 127) / 128;
    const int Nt = EPI == EPI_SWIGLU ? g.N / (BN / 2) : (g.N + BN - 1) / BN;
    const int T = Mt * Nt;
    const int nk = g.K / BK;
    const int Bm = max(1, min(Mt, (int)(kBandBytes / ((size_t)128 * g.K * 2))));

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer: one ring across all of this CTA's tiles
            uint32_t q = 0;  // stages issued
            bool ok = true;
            for (int t = blockIdx.x; ok && t < T; t += gridDim.x) {
                int m, n;
                persist_tile(t, Mt, Nt, Bm, m, n);
                for (int kb = 0; kb < nk; ++kb) {
                    const int s = (int)(q % S::STAGES);
                    const uint32_t ph = (q / S::STAGES) & 1u;
                    if (!mbar_wait(&empty_bar[s], ph ^ 1u, err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + s * S::STAGE;
                    mbar_expect_tx(&full_bar[s], (uint32_t)S::STAGE);
                    tma_load_2d(&tmA, &full_bar[s], st, kb * BK, m * 128);
                    if (EPI == EPI_SWIGLU) {
                        tma_load_2d(&tmB, &full_bar[s], st + S::A_BYTES, kb * BK, n * (BN / 2));
                        tma_load_2d(&tmB2, &full_bar[s], st + S::A_BYTES + (BN / 2) * BK * 2, kb * BK, n * (BN / 2));
                    } else {
                        tma_load_2d(&tmB, &full_bar[s], st + S::A_BYTES, kb * BK, n * BN);
                    }
                    ++q;
                }
            }
            // never leave with copies in flight: wait (bounded) for the last stages issued
            for (uint32_t i = q > (uint32_t)S::STAGES ? q - S::STAGES : 0; i < q; ++i)
                mbar_wait(&full_bar[i % S::STAGES], (i / S::STAGES) & 1u, err);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer (one thread)
            constexpr uint32_t idesc = idesc_bf16(128, BN);
            uint32_t q = 0;
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < T; t += gridDim.x, ++it) {
                const int b = it & 1;
                const uint32_t u = (uint32_t)(it >> 1) & 1u;
                if (!mbar_wait(&acc_empty[b], u ^ 1u, err)) {  // the epilogue has drained accumulator b
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(b * BN);
                for (int kb = 0; kb < nk; ++kb) {
                    const int s = (int)(q % S::STAGES);
                    const uint32_t ph = (q / S::STAGES) & 1u;
                    if (!mbar_wait(&full_bar[s], ph, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * S::STAGE);
                    const uint32_t b_addr = a_addr + S::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_bf16(d, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32), idesc,
                                 (kb > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&empty_bar[s]);  // the stage is free once these MMAs have read it
                    ++q;
                }
                if (ok) mma_commit(&acc_full[b]);  // accumulator b complete
            }
            // TMEM is released only after every MMA issued here has completed
            mma_commit(&done_bar);
            mbar_wait(&done_bar, 0u, err);
        }
        __syncwarp();
    } else {
        // ---- epilogue: warps 2..5, TMEM lane quarter = warp % 4, one output row per thread
        const int quarter = warp & 3;
        uint8_t* boxes = smem + S::STAGES * S::STAGE + quarter * 2 * kResidBox;  // EPI_RESID staging
        uint32_t nbox = 0;
        int it = 0;
        if (EPI == EPI_RESID && lane == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(&tmC) : "memory");
        for (int t = blockIdx.x; t < T; t += gridDim.x, ++it) {
            const int b = it & 1;
            const uint32_t u = (uint32_t)(it >> 1) & 1u;
            int m, n;
            persist_tile(t, Mt, Nt, Bm, m, n);
            const int row = m * 128 + quarter * 32 + lane;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[b], u, err));
            if (!ok) break;  // warp-uniform: no tcgen05.ld of an accumulator that is not complete
            tc_fence_after();
            const uint32_t tacc = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * BN);
            if constexpr (EPI == EPI_RESID)
                resid_add_tma(&tmC, boxes, tacc, BN, m * 128 + quarter * 32, n * BN, M, nbox);
            else
                persist_epilogue<BN, EPI>(g, tacc, row, row < M, n);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
        }
        if (EPI == EPI_RESID && lane == 0) bulk_wait_all();  // reductions done before the CTA's memory goes
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(S::TMEM_COLS) : "memory");
}


// ------------------------------------------------------------------ CTA pairs (cta_group::2)
// The same persistent GEMM on pairs of CTAs (a cluster of 2) that compute 256 x 256 output tiles together:
// rank r of the pair loads rows [128 r, 128 r + 128) of the tile's A rows and rows [128 r, 128 r + 128) of
// its 256 weight rows (for SwiGLU: rank 0 the 128 gate rows, rank 1 the matching up rows), each into its
// own shared memory, without multicast.  The leader (rank 0) issues M = 256, N = 256 MMAs that read A and
// B from both CTAs; each CTA's TMEM holds its 128 rows of the tile for all 256 columns.  Per SM this halves
// the weight bytes per flop against a 128 x 256 tile of one CTA.
//
// Synchronisation: both ranks' TMA copies count their bytes on the leader's full barrier (the leader arrives
// with the pair's byte total); the leader's commits arrive on both ranks' empty / accumulator-full / done
// barriers (multicast commit); both ranks' epilogue warps arrive on the leader's accumulator-empty barrier.
// Cluster barriers after set-up (barriers initialised before any copy may signal them) and before TMEM is
// released (no rank leaves while its shared memory or TMEM is still read), both reached only after bounded
// waits.
constexpr int kP2Stage = 2 * 128 * BK * 2;        // A 16 KB + B 16 KB per CTA
constexpr int kP2Stages = 6;
constexpr int kP2Smem = kP2Stages * kP2Stage + kResidStage + 1024;  // ring, residual staging, alignment slack
constexpr uint32_t kP2TmemCols = 512;             // two 256-column accumulators

__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap* map, uint32_t bar_cluster, void* dst, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(bar_cluster), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

// Arrive (once) on the barrier at this offset in both CTAs of the pair when the leader's MMAs so far complete.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
        ::"r"(smem_u32(bar)), "h"((uint16_t)3)
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

// tmC: the fp32 residual stream (box 32 columns x 32 rows, 128-byte swizzle), tmBt: the weights in 32-row
// boxes, for the column slabs of a last partial round (both EPI_RESID only).
template <int EPI>
__global__ void __launch_bounds__(192, 1) tc_gemmp2_kernel(const __grid_constant__ CUtensorMap tmA,
                                                           const __grid_constant__ CUtensorMap tmB,
                                                           const __grid_constant__ CUtensorMap tmB2,
                                                           const __grid_constant__ CUtensorMap tmC,
                                                           const __grid_constant__ CUtensorMap tmBt, GemmArgs g,
                                                           int* err) {
    pdl_trigger();
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kP2Stages];
    __shared__ __align__(8) uint64_t empty_bar[kP2Stages];
    __shared__ __align__(8) uint64_t acc_full[2];
    __shared__ __align__(8) uint64_t acc_empty[2];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint32_t tmem_slot;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    if (threadIdx.x == 0) {
        for (int s = 0; s < kP2Stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);  // four epilogue warps in each CTA of the pair
        }
        mbar_init(&done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                     "r"(kP2TmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();  // both ranks' barriers are initialised and TMEM is allocated
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB) : "memory");
        if (EPI == EPI_SWIGLU) asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB2) : "memory");
    }
    pdl_wait();

    const int live = min(g.M_dev ? *g.M_dev : g.M_bound, g.M_bound);
    const int M = g.live_gate == kGateManyRows && live <= 256 ? 0 : live;  // 0: the few-row kernel's launch
    const int Mt = (M + 255) / 256;
    const int Nt = EPI == EPI_SWIGLU ? g.N / 128 : (g.N + 255) / 256;
    const int T = Mt * Nt;
    const int nk = g.K / BK;
    const int Bm = max(1, min(Mt, (int)(kBandBytes / ((size_t)256 * g.K * 2))));
    const int pair = blockIdx.x >> 1, pairs = gridDim.x >> 1;
    // Work items: the full rounds' tiles, then the tiles of a last, partial round (all tiles, when there are
    // fewer than pairs) cut into S column slabs of 256 / S columns (S = 4 or 2, the most that keeps one
    // round; residual GEMMs only), so that the last round keeps more pairs busy.  A slab is computed whole
    // (full K) by one pair: no partial sums.  Item w >= T_full is slab (w - T_full) % S of tile
    // T_full + (w - T_full) / S.
    int T_full = T, S = 1;
    if (EPI == EPI_RESID) {
        const int rem = T % pairs;
        if (rem > 0) {
            S = rem * 4 <= pairs ? 4 : rem * 2 <= pairs ? 2 : 1;
            if (S > 1) T_full = T - rem;
        }
    }
    const int W = T_full + (T - T_full) * S;
    // tile, first column of the item within the tile, columns of the item
    auto item = [&](int w, int& tile, int& c0, int& cw) {
        if (w < T_full) {
            tile = w;
            c0 = 0;
            cw = 256;
        } else {
            tile = T_full + (w - T_full) / S;
            cw = 256 / S;
            c0 = ((w - T_full) % S) * cw;
        }
    };
    const uint32_t full0 = cluster_map(smem_u32(&full_bar[0]), 0);      // the leader's full barriers
    const uint32_t empty0 = cluster_map(smem_u32(&acc_empty[0]), 0);    // the leader's accumulator-empty

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer of this rank's halves
            uint32_t q = 0;
            bool ok = true;
            for (int w = pair; ok && w < W; w += pairs) {
                int t, c0, cw, m, n;
                item(w, t, c0, cw);
                persist_tile(t, Mt, Nt, Bm, m, n);
                // a slab: each rank brings cw / 2 weight rows, in 32-row boxes
                const uint32_t pair_bytes = cw == 256 ? 2u * kP2Stage : 2u * (kP2Stage / 2 + (uint32_t)cw / 2 * 128u);
                for (int kb = 0; kb < nk; ++kb) {
                    const int s = (int)(q % kP2Stages);
                    const uint32_t ph = (q / kP2Stages) & 1u;
                    if (!mbar_wait(&empty_bar[s], ph ^ 1u, err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + s * kP2Stage;
                    const uint32_t fb = full0 + (uint32_t)(s * sizeof(uint64_t));
                    if (leader) mbar_expect_tx(&full_bar[s], pair_bytes);  // the pair's bytes
                    tma_load_2d_pair(&tmA, fb, st, kb * BK, m * 256 + (int)rank * 128);
                    if (EPI == EPI_SWIGLU)
                        tma_load_2d_pair(rank == 0 ? &tmB : &tmB2, fb, st + kP2Stage / 2, kb * BK, n * 128);
                    else if (cw == 256)
                        tma_load_2d_pair(&tmB, fb, st + kP2Stage / 2, kb * BK, n * 256 + (int)rank * 128);
                    else
                        for (int j = 0; j < cw / 64; ++j)
                            tma_load_2d_pair(&tmBt, fb, st + kP2Stage / 2 + j * 32 * 128, kb * BK,
                                             n * 256 + c0 + (int)rank * (cw / 2) + j * 32);
                    ++q;
                }
            }
            // the stages issued last are free again once the MMAs consumed them: then no copy is in flight
            for (uint32_t i = q > (uint32_t)kP2Stages ? q - kP2Stages : 0; i < q; ++i)
                mbar_wait(&empty_bar[i % kP2Stages], (i / kP2Stages) & 1u, err);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            if (leader) {
                // ---- MMA issuer for the pair (one thread of the leader)
                uint32_t q = 0;
                int it = 0;
                bool ok = true;
                for (int w = pair; ok && w < W; w += pairs, ++it) {
                    int t, c0, cw;
                    item(w, t, c0, cw);
                    const uint32_t idesc = cw == 256 ? idesc_bf16(256, 256) : cw == 128 ? idesc_bf16(256, 128)
                                                                                        : idesc_bf16(256, 64);
                    const int b = it & 1;
                    const uint32_t u = (uint32_t)(it >> 1) & 1u;
                    if (!mbar_wait(&acc_empty[b], u ^ 1u, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d = tmem + (uint32_t)(b * 256);
                    for (int kb = 0; kb < nk; ++kb) {
                        const int s = (int)(q % kP2Stages);
                        const uint32_t ph = (q / kP2Stages) & 1u;
                        if (!mbar_wait(&full_bar[s], ph, err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a_addr = smem_u32(smem + s * kP2Stage);
                        const uint32_t b_addr = a_addr + kP2Stage / 2;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            mma_bf16_pair(d, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32), idesc,
                                          (kb > 0 || kk > 0) ? 1u : 0u);
                        mma_commit_pair(&empty_bar[s]);
                        ++q;
                    }
                    if (ok) mma_commit_pair(&acc_full[b]);
                }
                mma_commit_pair(&done_bar);
            }
            // both ranks: every MMA the leader issued has completed before TMEM or shared memory is released
            mbar_wait(&done_bar, 0u, err);
        }
        __syncwarp();
    } else {
        // ---- epilogue: this rank's 128 rows of the pair tile, one row per thread
        const int quarter = warp & 3;
        const int r128 = quarter * 32 + lane;  // row within this rank's half of the tile
        uint8_t* boxes = smem + kP2Stages * kP2Stage + quarter * 2 * kResidBox;  // EPI_RESID staging
        uint32_t nbox = 0;
        int it = 0;
        if (EPI == EPI_RESID && lane == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(&tmC) : "memory");
        for (int w = pair; w < W; w += pairs, ++it) {
            int t, c0, cw, m, n;
            item(w, t, c0, cw);
            const int b = it & 1;
            const uint32_t u = (uint32_t)(it >> 1) & 1u;
            persist_tile(t, Mt, Nt, Bm, m, n);
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[b], u, err));
            if (!ok) break;  // warp-uniform: no tcgen05.ld of an accumulator that is not complete
            tc_fence_after();
            const uint32_t tacc = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * 256);
            if constexpr (EPI == EPI_RESID)
                resid_add_tma(&tmC, boxes, tacc, cw, m * 256 + (int)rank * 128 + quarter * 32, n * 256 + c0, M,
                                    nbox);
            else
                persist_epilogue<256, EPI>(g, tacc, m * 256 + (int)rank * 128 + r128, m * 256 + (int)rank * 128 + r128 < M,
                                           n);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(empty0 + (uint32_t)(b * sizeof(uint64_t)));
        }
        if (EPI == EPI_RESID && lane == 0) bulk_wait_all();  // reductions done before the CTA's memory goes
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // neither rank releases TMEM or leaves while the pair still works on it
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kP2TmemCols) : "memory");
}

}  // namespace
}  // namespace tc
}  // namespace focus
