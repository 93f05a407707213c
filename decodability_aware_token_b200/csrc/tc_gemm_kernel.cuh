// Device side of the tcgen05 / TMEM / TMA bf16 GEMM (see tc_gemm.cu for the description), plus the
// host helper that builds its 2-D tensor maps.  Included by the translation units that launch it.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include <math_constants.h>

#include "launch.h"

namespace focus {
namespace tc {
namespace {  // each including translation unit gets its own kernel instances

constexpr int BK = 64;                     // K elements per stage (128 bytes of bf16: one swizzle row)
constexpr long long kWaitCycles = 2000000000LL;  // ~1 s at 2 GHz

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// Raise the bytes the current phase waits for without arriving (the arrival comes later).
__device__ __forceinline__ void mbar_add_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(addr), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with `parity` to complete; false (and the timeout bit) if it does not in ~1 s.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try(a, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try(a, parity)) {
        if (clock64() - t0 > kWaitCycles) {
            raise_err(err, FOCUS_DEVERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint64_t* bar, void* dst, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major tile written by TMA with the 128-byte swizzle;
// 8-row core groups 1024 bytes apart (stride byte offset), leading byte offset unused for this layout.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);        // start address
    d |= (uint64_t)1 << 16;                       // leading byte offset (16 B, unused)
    d |= (uint64_t)(1024 >> 4) << 32;             // stride byte offset
    d |= (uint64_t)1 << 46;                       // descriptor version for tcgen05
    d |= (uint64_t)2 << 61;                       // 128-byte swizzle
    return d;
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator, both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4)                    // D format: f32
           | (1u << 7)                  // A format: bf16
           | (1u << 10)                 // B format: bf16
           | ((uint32_t)(N >> 3) << 17) // N / 8
           | ((uint32_t)(M >> 4) << 24);// M / 16
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes (one row per thread).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// RoPE (cos, sin) of rotary position pos for pair i (head dim 128): a table the context fills once in
// double precision, rounded to float (positions up to the longest prefix plus the block).
__device__ __forceinline__ void rope_cs(const GemmArgs& g, int pos, int i, float& cn, float& sn) {
    const float2 cs = __ldg(g.rope_tab + (size_t)pos * 64 + i);
    cn = cs.x;
    sn = cs.y;
}

// (request, block position, rotary position) of a GEMM row in the QKV epilogue
__device__ __forceinline__ void qkv_row(const GemmArgs& g, int row, int& b, int& j, int& pos) {
    if (g.row_req) {
        b = g.row_req[row];
        j = g.row_pos[row];
    } else {
        b = row / g.block;
        j = row - b * g.block;
    }
    pos = checked_prefix(g.prefix_len, b, g.max_prefix, g.err) + j;
}

// destination of 128-wide head tile `head` of a QKV row: query rows, or K / V of the intra-block cache
__device__ __forceinline__ bf16* qkv_dst(const GemmArgs& g, int row, int head, int b, int j) {
    if (head < g.Hq) return reinterpret_cast<bf16*>(g.q_out) + ((size_t)row * g.Hq + head) * 128;
    const int kv = head < g.Hq + g.Hkv ? 0 : 1;
    const int gh = head - g.Hq - kv * g.Hkv;
    return reinterpret_cast<bf16*>(g.ibc) +
           ((((size_t)b * g.n_layers + g.layer) * 2 + kv) * g.Hkv + gh) * (size_t)g.block * 128 + (size_t)j * 128;
}

__device__ __forceinline__ void named_sync_epilogue() { asm volatile("bar.sync 1, 128;" ::: "memory"); }


template <int BN, int MSUB, int STAGES>
struct TcShape {
    static constexpr int BM = 128 * MSUB;
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int SMEM = STAGES * STAGE_BYTES + 1024;  // + alignment slack
    static constexpr int TMEM_COLS = (MSUB * BN <= 32) ? 32 : (MSUB * BN <= 64) ? 64 : (MSUB * BN <= 128) ? 128
                                     : (MSUB * BN <= 256) ? 256 : 512;
    static_assert(MSUB * BN <= 512, "accumulators exceed TMEM");
    static_assert(BN % 16 == 0 && BN >= 32 && BN <= 256, "tcgen05 N for M = 128");
};

template <int BN, int MSUB, int STAGES, int EPI>
__global__ void __launch_bounds__(192, 1) tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                                                         const __grid_constant__ CUtensorMap tmB,
                                                         const __grid_constant__ CUtensorMap tmB2, GemmArgs g,
                                                         int* err) {
    pdl_trigger();
    using S = TcShape<BN, MSUB, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[STAGES];
    __shared__ __align__(8) uint64_t empty_bar[STAGES];
    __shared__ __align__(8) uint64_t accum_bar;
    __shared__ uint32_t tmem_slot;

    const int m0 = blockIdx.y * S::BM;
    if (m0 >= g.M_bound) return;  // whole CTA, before any barrier, copy or TMEM use
    const int n_tile = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    // K blocks of this split
    const int nk_all = g.K / BK;
    const int split = blockIdx.z, splits = gridDim.z;
    const int kb0 = (int)((long long)nk_all * split / splits);
    const int kb1 = (int)((long long)nk_all * (split + 1) / splits);
    const int nk = kb1 - kb0;
    // stages whose weight tiles go out before the programmatic wait (none when the few-row kernel may take
    // this launch: the copies would be wasted there)
    const int n_pre = g.live_gate == kGateManyRows ? 0 : min(nk, STAGES);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&accum_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                     "r"((uint32_t)S::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    // the weight (B) tiles of the first stages depend on nothing an earlier kernel writes
    auto load_b = [&](int s, int kx) {
        uint8_t* b_dst = smem + s * S::STAGE_BYTES + S::A_BYTES;
        if (EPI == EPI_SWIGLU) {
            tma_load_2d(&tmB, &full_bar[s], b_dst, kx, n_tile * (BN / 2));
            tma_load_2d(&tmB2, &full_bar[s], b_dst + (BN / 2) * BK * 2, kx, n_tile * (BN / 2));
        } else {
            tma_load_2d(&tmB, &full_bar[s], b_dst, kx, n_tile * BN);
        }
    };
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB) : "memory");
        if (EPI == EPI_SWIGLU) asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB2) : "memory");
        for (int s = 0; s < n_pre; ++s) {  // fresh stages: nothing to wait for
            mbar_add_tx(&full_bar[s], (uint32_t)S::B_BYTES);
            load_b(s, (kb0 + s) * BK);
        }
    }
    pdl_wait();

    const int M = g.live_gate == kGateManyRows && (g.M_dev ? *g.M_dev : g.M_bound) <= 256
                      ? 0  // the few-row kernel's launch
                      : (g.M_dev ? *g.M_dev : g.M_bound);
    if (m0 >= M) {  // whole CTA: let the early weight copies land, release TMEM, leave
        if (warp == 0 && lane == 0)
            for (int s = 0; s < n_pre; ++s) {
                mbar_arrive(&full_bar[s]);
                mbar_wait(&full_bar[s], 0u, err);
            }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 1)
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)S::TMEM_COLS)
                         : "memory");
        return;
    }

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer
            int issued = 0;
            for (int i = 0; i < nk; ++i) {
                const int s = i % STAGES;
                const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
                const int kx = (kb0 + i) * BK;
                if (i < n_pre) {  // weight tile already on its way: arrive with the activation bytes
                    mbar_expect_tx(&full_bar[s], S::A_BYTES);
                } else {
                    if (!mbar_wait(&empty_bar[s], ph ^ 1u, err)) break;
                    mbar_expect_tx(&full_bar[s], S::STAGE_BYTES);
                    load_b(s, kx);
                }
                tma_load_2d(&tmA, &full_bar[s], smem + s * S::STAGE_BYTES, kx, m0);
                ++issued;
            }
            // never leave with copies in flight: wait (bounded) for the last stages issued
            for (int i = issued - 1; i >= 0 && i >= issued - STAGES; --i)
                mbar_wait(&full_bar[i % STAGES], (uint32_t)(i / STAGES) & 1u, err);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer (one thread)
            constexpr uint32_t idesc = idesc_bf16(128, BN);
            for (int i = 0; i < nk; ++i) {
                const int s = i % STAGES;
                const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
                if (!mbar_wait(&full_bar[s], ph, err)) break;
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + s * S::STAGE_BYTES);
                const uint32_t b_addr = a_addr + S::A_BYTES;
#pragma unroll
                for (int ms = 0; ms < MSUB; ++ms) {
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t ad = smem_desc_sw128(a_addr + ms * 128 * 128 + kk * 32);
                        const uint64_t bd = smem_desc_sw128(b_addr + kk * 32);
                        mma_bf16(tmem + ms * BN, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                mma_commit(&empty_bar[s]);  // slot free once these MMAs have read it
            }
            mma_commit(&accum_bar);         // accumulators complete
        }
        __syncwarp();
    } else {
        // ---- epilogue: warps 2..5, TMEM lane quarter = warp % 4
        const int quarter = warp & 3;
        const bool ok = mbar_wait(&accum_bar, 0, err);
        tc_fence_after();
#pragma unroll 1
        for (int ms = 0; ms < MSUB; ++ms) {
            const int row = m0 + ms * 128 + quarter * 32 + lane;
            const bool live = ok && row < M && nk > 0;
            const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + ms * BN;
            if (EPI == EPI_RESID || EPI == EPI_QKV) {
                if (EPI == EPI_RESID) {
                    float* xr = g.resid + (size_t)row * g.N + (size_t)n_tile * BN;
#pragma unroll 1
                    for (int c0 = 0; c0 < BN; c0 += 32) {
                        float v[32];
                        tmem_ld32(tbase + c0, v);
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
                } else {
                    // one head per 128-column tile: rotate pairs (i, i + 64), then q rows or the cache
                    const int head = n_tile;
                    const bool rotate = head < g.Hq + g.Hkv;
                    int b = 0, j = 0, pos = 0;
                    if (live) qkv_row(g, row, b, j, pos);
#pragma unroll 1
                    for (int c0 = 0; c0 < 64; c0 += 32) {
                        float lo[32], hi[32];
                        tmem_ld32(tbase + c0, lo);
                        tmem_ld32(tbase + 64 + c0, hi);
                        if (live) {
                            bf16* dst = qkv_dst(g, row, head, b, j);
#pragma unroll
                            for (int t = 0; t < 32; t += 2) {
                                float a0 = lo[t], a1 = lo[t + 1], b0 = hi[t], b1 = hi[t + 1];
                                if (rotate) {
                                    float c_0, s_0, c_1, s_1;
                                    rope_cs(g, pos, c0 + t, c_0, s_0);
                                    rope_cs(g, pos, c0 + t + 1, c_1, s_1);
                                    a0 = lo[t] * c_0 - hi[t] * s_0;
                                    b0 = hi[t] * c_0 + lo[t] * s_0;
                                    a1 = lo[t + 1] * c_1 - hi[t + 1] * s_1;
                                    b1 = hi[t + 1] * c_1 + lo[t + 1] * s_1;
                                }
                                *reinterpret_cast<__nv_bfloat162*>(dst + c0 + t) = __floats2bfloat162_rn(a0, a1);
                                *reinterpret_cast<__nv_bfloat162*>(dst + 64 + c0 + t) = __floats2bfloat162_rn(b0, b1);
                            }
                        }
                    }
                }
            } else if (EPI == EPI_SWIGLU) {
                bf16* out = reinterpret_cast<bf16*>(g.act) + (size_t)row * g.N + (size_t)n_tile * (BN / 2);
#pragma unroll 1
                for (int c0 = 0; c0 < BN / 2; c0 += 32) {
                    float gt[32], up[32];
                    tmem_ld32(tbase + c0, gt);
                    tmem_ld32(tbase + BN / 2 + c0, up);
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
                // vocabulary tile statistics of this row, online over 32-column chunks
                float mx = -CUDART_INF_F, se = 0.f;
                int arg = 0x7fffffff;
                const int col0 = n_tile * BN;
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    float v[32];
                    tmem_ld32(tbase + c0, v);
                    float cm = -CUDART_INF_F;
                    int ca = 0x7fffffff;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const bool in = col0 + c0 + i < g.N;
                        if (in && v[i] > cm) {
                            cm = v[i];
                            ca = col0 + c0 + i;
                        }
                    }
                    // (no early exit: every lane must reach the next tcgen05.ld)
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
                if (live) {
                    const size_t idx = (size_t)row * g.n_tiles + n_tile;
                    g.lm_max[idx] = mx;
                    g.lm_sum[idx] = se;
                    g.lm_arg[idx] = arg;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)S::TMEM_COLS)
                     : "memory");
    }
}

// ------------------------------------------------------------------ swapped GEMM for few rows
// For the kept rows (at most 256 tokens, typically a few dozen) the GEMMs stream weights.  The product is
// computed transposed, D^T = W X^T: the 128 output features of a tile sit on the MMA's M side and every
// live token on its N side (N = the live count rounded up to 32, at most 256), so one CTA covers all
// tokens of its feature tile, no CTA is spent on absent rows and no tensor work or operand bytes go to
// them.  A stage holds the 16 KB weight tile and one 4 KB box per live 32-token group; the 100 KB
// operand ring (two CTAs per SM) holds 5 stages for up to 32 tokens.
//
// Split K runs inside a thread-block cluster: the `splits` CTAs of one output tile are the cluster's
// ranks, each accumulates its K slice in TMEM and parks it (128 tokens at a time) in its own shared memory
// as [token][feature] fp32; after a cluster barrier rank r sums the slices of its share of the tokens in rank order through
// distributed shared memory and applies the epilogue to them.  No partial sums go through global memory
// and no CTA waits on an arrival counter.  Epilogue threads own one output feature each, so for every
// token a warp touches 32 consecutive features.  Pairs of features f and f + 64 (the RoPE halves of a
// head; gate and up of SwiGLU, loaded as two 64-row weight boxes) are both in the parked tile.  The
// LM-head epilogue (no split) reduces each token's 128 vocabulary features of the tile to the max
// logit, sum exp(z - max) and first argmax, so no logits reach global memory.
//
// Grid: (splits, feature tiles), cluster (splits, 1, 1).
constexpr int kTMaxTok = 256;                    // tokens per CTA (MMA N <= 256)
constexpr int kTW = 128 * BK * 2;                // weight tile bytes (16 KB)
constexpr int kTXBox = 32 * BK * 2;              // one 32-token box of the token tile (4 KB)
constexpr int kTRing = 100 * 1024;               // operand ring bytes (two CTAs per SM)
constexpr int kTMaxStages = kTRing / (kTW + kTXBox);
constexpr int kTSmem = kTRing + 1024;            // + alignment slack
constexpr int kTMaxSplits = 8;                   // portable cluster size
constexpr int kTChunk = 128;                     // tokens parked at a time
constexpr int kTPark = 129;                      // parked tile row stride (odd: token-major scans are conflict free)
static_assert(kTChunk * kTPark * 4 <= kTRing, "parked tile reuses the operand ring");

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_map(uint32_t local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

template <int EPI>
__global__ void __launch_bounds__(192, 2) tc_gemmt_kernel(const __grid_constant__ CUtensorMap tmW,
                                                          const __grid_constant__ CUtensorMap tmW2,
                                                          const __grid_constant__ CUtensorMap tmX, GemmArgs g,
                                                          int* err) {
    pdl_trigger();
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kTMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kTMaxStages];
    __shared__ __align__(8) uint64_t accum_bar;
    __shared__ uint32_t tmem_slot;

    // Before the programmatic-launch wait only what the launch fixes is known: the token bound, the K
    // slice and the weights.  The ring keeps its weight tiles apart from its token tiles (weights of
    // stage s at s x 16 KB, token tiles after the last weight stage), so the first stages' weight tiles
    // can be fetched while the predecessor drains; the live token count, read after the wait, only
    // sets where the token tiles go and how many stages the ring holds.
    const int Mb = min(g.M_bound, kTMaxTok);  // the launcher keeps M_bound in [1, 256]
    const int xb_bound = (Mb + 31) / 32;
    const uint32_t tmem_cols = xb_bound <= 1 ? 32u : xb_bound <= 2 ? 64u : xb_bound <= 4 ? 128u : 256u;
    const int n_tile = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int splits = gridDim.x;
    const int split = (int)cluster_rank();
    const int nk_all = g.K / BK;
    const int kb0 = (int)((long long)nk_all * split / splits);
    const int nk = (int)((long long)nk_all * (split + 1) / splits) - kb0;
    // output features of the tile: 128 (QKV: one head; residual GEMMs; LM head), or 64 gate + 64 up (SwiGLU)
    const int fbase = EPI == EPI_SWIGLU ? n_tile * 64 : n_tile * 128;
    // stages whose weight tiles go out before the wait: as many as the ring holds at the token bound
    // (none when the many-row kernel may take this launch: the copies would be wasted there)
    const int n_pre = g.live_gate == kGateFewRows ? 0 : min(nk, min(kTMaxStages, kTRing / (kTW + xb_bound * kTXBox)));

    if (threadIdx.x == 0) {
        for (int st = 0; st < kTMaxStages; ++st) {
            mbar_init(&full_bar[st], 1);
            mbar_init(&empty_bar[st], 1);
        }
        mbar_init(&accum_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                     "r"(tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmW) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmX) : "memory");
        if (EPI == EPI_SWIGLU) asm volatile("prefetch.tensormap [%0];" ::"l"(&tmW2) : "memory");
        for (int st = 0; st < n_pre; ++st) {  // fresh stages: nothing to wait for
            mbar_add_tx(&full_bar[st], (uint32_t)kTW);
            uint8_t* w_dst = smem + st * kTW;
            tma_load_2d(&tmW, &full_bar[st], w_dst, (kb0 + st) * BK, fbase);
            if (EPI == EPI_SWIGLU) tma_load_2d(&tmW2, &full_bar[st], w_dst + kTW / 2, (kb0 + st) * BK, fbase);
        }
    }
    pdl_wait();

    const int live_rows = g.M_dev ? *g.M_dev : g.M_bound;
    const int M = g.live_gate == kGateFewRows && live_rows > kTMaxTok ? 0 : min(live_rows, Mb);  // 0: the many-row kernel's
    if (M <= 0) {  // the whole grid: let the early weight copies land, release TMEM, leave
        if (warp == 0 && lane == 0)
            for (int st = 0; st < n_pre; ++st) {
                mbar_arrive(&full_bar[st]);
                mbar_wait(&full_bar[st], 0u, err);
            }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 1)
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tmem_cols) : "memory");
        return;
    }
    const int x_boxes = (M + 31) / 32;
    const int n_cols = x_boxes * 32;               // MMA N and TMEM columns read back (<= tmem_cols)
    const int x_stage = x_boxes * kTXBox;          // token-tile bytes of a stage (a multiple of 1024)
    const int nst = min(kTMaxStages, kTRing / (kTW + x_stage));  // >= n_pre, since M <= Mb
    uint8_t* xring = smem + nst * kTW;             // 1024-aligned (swizzle atom)
    float* park = reinterpret_cast<float*>(smem);  // [token][kTPark] features, once the ring is idle

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer
            int issued = 0;
            for (int i = 0; i < nk; ++i) {
                const int st = i % nst;
                const uint32_t ph = (uint32_t)(i / nst) & 1u;
                uint8_t* w_dst = smem + st * kTW;
                uint8_t* x_dst = xring + st * x_stage;
                const int kx = (kb0 + i) * BK;
                if (i < n_pre) {  // weight tile already on its way: arrive with the token bytes
                    mbar_expect_tx(&full_bar[st], (uint32_t)x_stage);
                } else {
                    if (!mbar_wait(&empty_bar[st], ph ^ 1u, err)) break;
                    mbar_expect_tx(&full_bar[st], (uint32_t)(kTW + x_stage));
                    tma_load_2d(&tmW, &full_bar[st], w_dst, kx, fbase);
                    if (EPI == EPI_SWIGLU) tma_load_2d(&tmW2, &full_bar[st], w_dst + kTW / 2, kx, fbase);
                }
                for (int bx = 0; bx < x_boxes; ++bx)
                    tma_load_2d(&tmX, &full_bar[st], x_dst + bx * kTXBox, kx, bx * 32);
                ++issued;
            }
            // never leave with copies in flight: wait (bounded) for the last stages issued
            for (int i = issued - 1; i >= 0 && i >= issued - nst; --i)
                mbar_wait(&full_bar[i % nst], (uint32_t)(i / nst) & 1u, err);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer (one thread): 128 features x n_cols tokens per instruction
            const uint32_t idesc = idesc_bf16(128, n_cols);
            for (int i = 0; i < nk; ++i) {
                const int st = i % nst;
                const uint32_t ph = (uint32_t)(i / nst) & 1u;
                if (!mbar_wait(&full_bar[st], ph, err)) break;
                tc_fence_after();
                const uint32_t w_addr = smem_u32(smem + st * kTW);
                const uint32_t x_addr = smem_u32(xring + st * x_stage);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    mma_bf16(tmem, smem_desc_sw128(w_addr + kk * 32), smem_desc_sw128(x_addr + kk * 32), idesc,
                             (i > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&empty_bar[st]);
            }
            mma_commit(&accum_bar);
        }
        __syncwarp();
    }
    // ---- epilogue warps: accumulators ready?
    const int f_own = (warp & 3) * 32 + lane;  // warp w holds TMEM lanes 32 (w % 4) .. +31, i.e. features f
    const uint32_t tbase = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    bool live = false;  // otherwise this slice contributes zeros (a timeout is flagged)
    if (warp >= 2) {
        live = mbar_wait(&accum_bar, 0, err) && nk > 0;
        tc_fence_after();
    }
    // tokens in chunks of kTChunk, each parked, reduced across the cluster and finished
#pragma unroll 1
    for (int c = 0; c < M; c += kTChunk) {
        const int cm = min(kTChunk, M - c);
        if (c > 0) cluster_sync_all();  // the previous chunk's parked tiles are no longer read
        if (warp >= 2) {
#pragma unroll 1
            for (int c0 = 0; c0 < cm; c0 += 32) {  // CTA-uniform: all lanes of the warp execute the load
                float v[32];
                tmem_ld32(tbase + c + c0, v);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (c0 + i < cm) park[(c0 + i) * kTPark + f_own] = live ? v[i] : 0.f;
            }
        }
        cluster_sync_all();  // every slice of the chunk is parked
        if (warp < 2) continue;
        const int e = threadIdx.x - 64;
        if (EPI == EPI_LMHEAD) {
            // ---- per token: the tile's max logit, first argmax and sum exp(z - max) (no split)
            const int n_valid = min(128, g.N - fbase);
            for (int t = e; t < cm; t += 128) {
                const float* z = park + t * kTPark;
                float mx = -CUDART_INF_F;
                int arg = 0x7fffffff;
                for (int q = 0; q < n_valid; ++q)
                    if (z[q] > mx) {
                        mx = z[q];
                        arg = fbase + q;
                    }
                float se = 0.f;
                for (int q = 0; q < n_valid; ++q) se += expf(z[q] - mx);
                const size_t idx = (size_t)(c + t) * g.n_tiles + n_tile;
                g.lm_max[idx] = mx;
                g.lm_sum[idx] = se;
                g.lm_arg[idx] = arg;
            }
            continue;
        }
        // ---- this rank's tokens [t0, t1) of the chunk: sum the slices in rank order, then the epilogue
        const int t0 = cm * split / splits, t1 = cm * (split + 1) / splits;
        const uint32_t park_local = smem_u32(park);
        uint32_t peer[kTMaxSplits];
#pragma unroll
        for (int sp = 0; sp < kTMaxSplits; ++sp) peer[sp] = sp < splits ? cluster_map(park_local, sp) : 0u;
        if (EPI == EPI_RESID) {
            const int f = e;
            float* xc = g.resid + (size_t)c * g.N + fbase + f;
            for (int t = t0; t < t1; t += 4) {
                float pv[4][kTMaxSplits], xv[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    xv[q] = t + q < t1 ? xc[(size_t)(t + q) * g.N] : 0.f;
#pragma unroll
                    for (int sp = 0; sp < kTMaxSplits; ++sp)
                        pv[q][sp] = (sp < splits && t + q < t1) ? ld_cluster_f32(peer[sp] + ((t + q) * kTPark + f) * 4)
                                                                 : 0.f;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float acc = 0.f;
#pragma unroll
                    for (int sp = 0; sp < kTMaxSplits; ++sp) acc += pv[q][sp];
                    if (t + q < t1) xc[(size_t)(t + q) * g.N] = xv[q] + acc;
                }
            }
        } else {
            // thread e finishes feature pair (fp, fp + 64) for the tokens of parity e / 64
            const int fp = e & 63;
            for (int t = t0 + (e >> 6); t < t1; t += 4) {
                float lo_p[2][kTMaxSplits], hi_p[2][kTMaxSplits];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int tt = t + 2 * q;
#pragma unroll
                    for (int sp = 0; sp < kTMaxSplits; ++sp) {
                        const bool in = sp < splits && tt < t1;
                        lo_p[q][sp] = in ? ld_cluster_f32(peer[sp] + (tt * kTPark + fp) * 4) : 0.f;
                        hi_p[q][sp] = in ? ld_cluster_f32(peer[sp] + (tt * kTPark + fp + 64) * 4) : 0.f;
                    }
                }
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int tt = t + 2 * q;
                    if (tt >= t1) continue;
                    float a = 0.f, bb = 0.f;
#pragma unroll
                    for (int sp = 0; sp < kTMaxSplits; ++sp) {
                        a += lo_p[q][sp];
                        bb += hi_p[q][sp];
                    }
                    const int row = c + tt;
                    if (EPI == EPI_SWIGLU) {
                        bf16* out = reinterpret_cast<bf16*>(g.act) + (size_t)row * g.N + fbase + fp;
                        *out = __float2bfloat16_rn(a / (1.f + expf(-a)) * bb);
                    } else {  // EPI_QKV: one head per tile; queries and keys rotate (fp, fp + 64)
                        const int head = n_tile;
                        int b, j, pos;
                        qkv_row(g, row, b, j, pos);
                        float lo = a, hi = bb;
                        if (head < g.Hq + g.Hkv) {
                            float cn, sn;
                            rope_cs(g, pos, fp, cn, sn);
                            lo = a * cn - bb * sn;
                            hi = bb * cn + a * sn;
                        }
                        bf16* dst = qkv_dst(g, row, head, b, j);
                        dst[fp] = __float2bfloat16_rn(lo);
                        dst[fp + 64] = __float2bfloat16_rn(hi);
                    }
                }
            }
        }
    }
    tc_fence_before();
    cluster_sync_all();  // no rank leaves (or reuses its shared memory) while others still read it
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tmem_cols) : "memory");
    }
}

// ------------------------------------------------------------------ tensor maps
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D bf16 row-major [rows, cols] tensor, box = [box_rows, 64 cols], 128-byte swizzle.  L2 promotion of
// each 128-byte box row to 256 bytes suits operands walked along K (the promoted half is the next K
// block); tiles whose two column halves are copied together take promote_256 = false.
inline bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                     bool promote_256 = true) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              promote_256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 row-major [rows, cols] array, box = [32 rows, 32 cols] (128-byte rows), 128-byte swizzle: the
// staging boxes of the persistent GEMMs' residual epilogue (TMA reductions into the residual stream, TMA
// stores of split-tile partial sums).
inline bool make_map_f32(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 4};
    const cuuint32_t box[2] = {32u, 32u};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace tc
}  // namespace focus
