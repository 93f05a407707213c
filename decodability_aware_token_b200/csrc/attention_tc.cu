// bf16 attention of block queries over paged prefix KV plus the intra-block KV cache, on tensor cores
// (mma.sync m16n8k16, fp32 accumulate), with the importance column sums fused in for layers 0 and 1.
//
// "FOCUS: DLLMs Know How to Tame Their Compute Bound", project page, Overview -- Design / Decodability
// Signal (importance from the early layers' Q/K attention) and Runtime Action (ragged execution and the
// intra-block KV cache); news article on the same paper, "Arquitetura do FOCUS" (ragged paged attention).
//
// Work unit (one CTA): request b, KV head g, and a tile of up to 64 query vectors of that group
// (query vector qi = row * G + head-in-group).  Keys are walked in 64-key chunks: the prefix in page
// order (each page's K and V rows copied by TMA with the 128-byte swizzle; pages of 16, 32 or 64
// tokens), then the block's B keys from the intra-block cache as the last chunk.  A ring of three chunk
// stages keeps two chunks in flight while one is consumed; the first prefix chunks are requested before
// the programmatic-launch wait.  The 4 warps split the work as RT row tiles x KS key slices (RT * KS = 4): 64 query
// vectors -> 4 x 1, 32 -> 2 x 2, <= 16 (the usual ragged case) -> 1 x 4.  Each warp keeps an online
// softmax (base 2) over its key slice; slices are merged through shared memory at the end.
//
// Importance: the block chunk's raw scores stay in registers until the final row max M and denominator
// L are known; then p = 2^(s - M) / L is summed over the tile's query vectors per block key and written
// to imp_part[b][g][tile][j] (fixed order, no atomics); the selection kernel adds those in order.
//
// The kernel is HBM-bound at these shapes (about 2 x rows flops per byte of K/V), so the legacy mma.sync
// path -- whose 16-row tile granularity fits ragged query counts of 2..16 -- keeps the tensor work far
// below the time to stream the keys.
#include <math_constants.h>

#include "launch.h"
#include "attention_pages.cuh"

namespace focus {

namespace {

using tc::mbar_expect_tx;
using tc::mbar_init;
using tc::mbar_wait;
using tc::tma_load_2d;

constexpr int kQTile = 64;      // query vectors per CTA
constexpr int kStages = 3;      // chunks in the ring (2 in flight while one is consumed)
constexpr int kAttnSmem = kStages * kStageBytes + 1024;  // dynamic shared memory: 97 KB, two CTAs per SM

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Byte offset of 16-byte column chunk c (0..15) of key row r in a K or V tile held as two [64][64]
// bf16 halves written by TMA with the 128-byte swizzle (chunk c & 7 of row r sits at (c & 7) ^ (r & 7)).
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return (uint32_t)((c >> 3) * kHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

template <bool FULL>
__global__ void __launch_bounds__(128, 2) attention_tc_kernel(const __grid_constant__ CUtensorMap pool_map,
                                                              const __grid_constant__ CUtensorMap ibc_map, AttnArgs a,
                                                              int q_tiles) {
    pdl_trigger();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* kv = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full_bar[kStages];
    __shared__ uint64_t valid_s[kStages];
    __shared__ float ml_s[4][16][2];      // per warp: row max / denominator (log2 domain)
    __shared__ float col_s[4][kChunk];    // per row tile: block-key column sums
    __shared__ int32_t pt_s[kPtCache];     // this request's page-table row
    __shared__ float fin_s[kQTile][2];     // split merge: final row max / denominator
    __shared__ int last_s;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.Hq / a.Hkv;
    Unit u{};
    // grid (KV heads x pieces, query tiles, request slots): a request's CTAs are adjacent.  With a request
    // order (kept-row launches with more units than resident CTAs: longest prefix first, written by the
    // row-map kernel earlier in the step), slot z walks request order[z], read after the wait; the early
    // chunk copies below then also come after it.
    if (a.order) pdl_wait();
    u.b = a.order ? a.order[blockIdx.z] : (int)blockIdx.z;
    u.g = blockIdx.x % a.Hkv;
    u.qt = blockIdx.y;
    // Before the programmatic-launch wait this kernel reads only what no kernel of the step writes: the
    // prefix lengths, the page table and the prefix pages of the KV pool (the step's first kernel lets
    // its successors start only after everything queued before the step has completed).  The block's
    // cache rows, the queries and the kept-row offsets are written earlier in the step and wait.
    u.P = checked_prefix(a.prefix_len, u.b, a.max_pages * a.page_size, a.err);
    u.q0 = u.qt * kQTile;
    const int n_prefix_chunks = (u.P + kChunk - 1) / kChunk;
    const int n_chunks = n_prefix_chunks + 1;
    // split-KV: this CTA walks chunks [c_begin, c_end) of the unit's n_chunks
    const int pieces = a.pieces;  // grid.y = Hkv * pieces
    const int cpp = (n_chunks + pieces - 1) / pieces;  // chunks per piece
    const int piece = blockIdx.x / a.Hkv;
    const int c_begin = piece * cpp, c_end = min(n_chunks, c_begin + cpp);
    if (c_begin >= c_end) return;
    const int n_active = (n_chunks + cpp - 1) / cpp;
    const int unit = (u.b * a.Hkv + u.g) * q_tiles + u.qt;

    // page-table row -> shared (one latency for the whole CTA instead of one per issued chunk)
    const bool pt_cached = a.max_pages <= kPtCache;
    for (int i = threadIdx.x; pt_cached && i < a.max_pages; i += 128)
        pt_s[i] = a.page_table[(size_t)u.b * a.max_pages + i];
    const int32_t* pt = pt_cached ? pt_s : a.page_table + (size_t)u.b * a.max_pages;

    if (threadIdx.x == 0) {
        for (int s2 = 0; s2 < kStages; ++s2) mbar_init(&full_bar[s2], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    int issued = 0;  // chunks whose copies thread 0 has issued
    // the first query tile of every unit (the only one in the ragged layers' usual case) starts its
    // leading prefix chunks now
    if (threadIdx.x == 0 && u.qt == 0)
        for (; issued < kStages - 1 && c_begin + issued < c_end && c_begin + issued < n_prefix_chunks; ++issued)
            valid_s[issued] = issue_chunk(a, u, &pool_map, &ibc_map, kv + issued * kStageBytes, &full_bar[issued],
                                          c_begin + issued, n_prefix_chunks, pt);
    pdl_wait();

    if (FULL) {
        u.row_base = u.b * a.B;
        u.n_rows = a.B;
    } else {
        u.row_base = a.row_offsets[u.b];
        u.n_rows = a.row_offsets[u.b + 1] - u.row_base;
    }
    u.nq = min(kQTile, u.n_rows * G - u.q0);
    if (u.nq <= 0) {  // CTA-uniform: let the early copies land, then leave
        if (threadIdx.x == 0)
            for (int i = 0; i < issued; ++i) mbar_wait(&full_bar[i], 0u, a.err);
        return;
    }
    const int RT = u.nq <= 16 ? 1 : (u.nq <= 32 ? 2 : 4);
    const int KS = 4 / RT;
    const int rt = warp % RT, ks = warp / RT;
    const int keys_per_warp = kChunk / KS;  // 64, 32 or 16
    const int key0 = ks * keys_per_warp;
    if (threadIdx.x == 0)
        for (; issued < kStages - 1 && c_begin + issued < c_end; ++issued)
            valid_s[issued] = issue_chunk(a, u, &pool_map, &ibc_map, kv + issued * kStageBytes, &full_bar[issued],
                                          c_begin + issued, n_prefix_chunks, pt);

    // ---- Q fragments (A operand) of this warp's 16 query vectors, straight from global memory
    const int gq = lane >> 2, tq = lane & 3;
    uint32_t qf[8][4];
    {
        const bf16* qg = reinterpret_cast<const bf16*>(a.q);
        const uint32_t* rowp[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int v = rt * 16 + gq + 8 * h;
            const int qi = u.q0 + (v < u.nq ? v : 0);
            const int row = qi / G, hh = u.g * G + (qi - row * G);
            rowp[h] = v < u.nq ? reinterpret_cast<const uint32_t*>(qg + ((size_t)(u.row_base + row) * a.Hq + hh) * kD)
                               : nullptr;
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int c = kk * 8 + tq;  // 32-bit word: columns 16 kk + 2 tq, +1
            qf[kk][0] = rowp[0] ? rowp[0][c] : 0u;
            qf[kk][1] = rowp[1] ? rowp[1][c] : 0u;
            qf[kk][2] = rowp[0] ? rowp[0][c + 4] : 0u;
            qf[kk][3] = rowp[1] ? rowp[1][c + 4] : 0u;
        }
    }
    __syncthreads();  // valid_s of the first chunks
    const float sl2 = rsqrtf((float)kD) * 1.4426950408889634f;  // 1/sqrt(d) * log2(e)
    float m_r[2] = {-CUDART_INF_F, -CUDART_INF_F}, l_r[2] = {0.f, 0.f};
    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float sb[8][4];  // raw (scaled) scores of the block chunk, kept for the importance
#pragma unroll
    for (int n = 0; n < 8; ++n) sb[n][0] = sb[n][1] = sb[n][2] = sb[n][3] = -CUDART_INF_F;

    bool alive = true;
    for (int ci = c_begin; ci < c_end; ++ci) {
        const int i = ci - c_begin;       // position in this CTA's ring
        const int st = i % kStages;
        if (threadIdx.x == 0 && ci + kStages - 1 < c_end) {
            const int sn = (i + kStages - 1) % kStages;  // stage of chunk ci - 1: free since the last sync
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // V rows zeroed below, before TMA
            valid_s[sn] = issue_chunk(a, u, &pool_map, &ibc_map, kv + sn * kStageBytes, &full_bar[sn],
                                      ci + kStages - 1, n_prefix_chunks, pt);
            ++issued;
        }
        const bool landed = mbar_wait(&full_bar[st], (uint32_t)(i / kStages) & 1u, a.err);
        if (__syncthreads_or(!landed)) {  // block-uniform: nobody is left waiting at a barrier
            alive = false;
            break;
        }
        const uint64_t vmask = valid_s[st];
        const uint32_t kbase = smem_u32(kv + st * kStageBytes);
        const uint32_t vbase = kbase + 2 * kHalf;
        if (vmask != ~0ull) {  // block-uniform: V rows of keys the copies left unfilled (skipped pages,
                               // a short block) may hold stale bits; P is 0 there, so make V 0 too
            uint8_t* vb = kv + st * kStageBytes + 2 * kHalf;
            for (int t = threadIdx.x; t < kChunk * 16; t += 128) {
                const int r = t >> 4, c = t & 15;
                if (!((vmask >> r) & 1ull)) *reinterpret_cast<uint4*>(vb + swz(r, c)) = make_uint4(0, 0, 0, 0);
            }
            __syncthreads();
        }
        // S = Q K^T over this warp's key slice: keys_per_warp / 8 n-tiles (up to 8)
        float s[8][4];
        const int n_nt = keys_per_warp / 8;
#pragma unroll
        for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
        for (int np = 0; np < 4; ++np) {  // pairs of n-tiles (16 keys)
            if (2 * np >= n_nt) break;
            const int kr = key0 + np * 16 + (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int c = kk * 2 + ((lane >> 3) & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kbase + swz(kr, c), b0, b1, b2, b3);
                mma16816(s[2 * np], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
                mma16816(s[2 * np + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
            }
        }
        // mask, scale, online softmax (rows gq and gq + 8 of this warp's tile)
        float mx[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            if (n >= n_nt) break;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = key0 + n * 8 + 2 * tq + (e & 1);
                const float v = ((vmask >> key) & 1ull) ? s[n][e] * sl2 : -CUDART_INF_F;
                s[n][e] = v;
                mx[e >> 1] = fmaxf(mx[e >> 1], v);
            }
        }
        if (FULL && ci == n_chunks - 1) {
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) sb[n][e] = s[n][e];
        }
        float scale[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
            const float m_new = fmaxf(m_r[h], mx[h]);
            const float m_use = m_new == -CUDART_INF_F ? 0.f : m_new;
            scale[h] = exp2f(m_r[h] - m_use);   // 0 when m_r is -inf
            m_r[h] = m_new;
            mx[h] = m_use;
        }
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            if (n >= n_nt) break;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float p = exp2f(s[n][e] - mx[e >> 1]);  // 0 for masked keys
                s[n][e] = p;
                rs[e >> 1] += p;
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 1);
            rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 2);
            l_r[h] = l_r[h] * scale[h] + rs[h];
        }
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            o[n][0] *= scale[0];
            o[n][1] *= scale[0];
            o[n][2] *= scale[1];
            o[n][3] *= scale[1];
        }
        // O += P V over this warp's key slice: keys_per_warp / 16 k-steps
#pragma unroll
        for (int ksp = 0; ksp < 4; ++ksp) {
            if (2 * ksp >= n_nt) break;
            const uint32_t pa0 = pack_bf16(s[2 * ksp][0], s[2 * ksp][1]);
            const uint32_t pa1 = pack_bf16(s[2 * ksp][2], s[2 * ksp][3]);
            const uint32_t pa2 = pack_bf16(s[2 * ksp + 1][0], s[2 * ksp + 1][1]);
            const uint32_t pa3 = pack_bf16(s[2 * ksp + 1][2], s[2 * ksp + 1][3]);
            const int vr = key0 + ksp * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
            for (int dp = 0; dp < 8; ++dp) {  // pairs of 8-wide d tiles
                const int c = dp * 2 + (lane >> 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vbase + swz(vr, c), b0, b1, b2, b3);
                mma16816(o[2 * dp], pa0, pa1, pa2, pa3, b0, b1);
                mma16816(o[2 * dp + 1], pa0, pa1, pa2, pa3, b2, b3);
            }
        }
        __syncthreads();  // stage st is refilled two iterations later
    }
    if (!alive) {
        // a copy never landed: wait (bounded) for the chunks still in the ring so that no TMA write
        // lands in a CTA that has exited; the outputs of this unit stay unwritten (error flagged)
        if (threadIdx.x == 0)
            for (int c = issued - kStages < 0 ? 0 : issued - kStages; c < issued; ++c)
                mbar_wait(&full_bar[c % kStages], (uint32_t)(c / kStages) & 1u, a.err);
        return;
    }

    // ---- merge the key slices: final M, L per row of each row tile
    if (tq == 0) {
        ml_s[warp][gq][0] = m_r[0];
        ml_s[warp][gq][1] = l_r[0];
        ml_s[warp][gq + 8][0] = m_r[1];
        ml_s[warp][gq + 8][1] = l_r[1];
    }
    __syncthreads();
    float M[2], L[2], f[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int r = gq + 8 * h;
        float mm = -CUDART_INF_F;
        for (int k2 = 0; k2 < KS; ++k2) mm = fmaxf(mm, ml_s[k2 * RT + rt][r][0]);
        const float mu = mm == -CUDART_INF_F ? 0.f : mm;
        float ll = 0.f;
        for (int k2 = 0; k2 < KS; ++k2) ll += ml_s[k2 * RT + rt][r][1] * exp2f(ml_s[k2 * RT + rt][r][0] - mu);
        M[h] = mu;
        L[h] = ll;
        f[h] = exp2f(m_r[h] - mu);  // this slice's weight
    }
    // o slices -> shared (fp32), summed over the key slices by the ks == 0 warp of each row tile
    float* osum = reinterpret_cast<float*>(kv);  // reuses the ring: [warps][16][128]
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        const int d0 = n * 8 + 2 * tq;
        float* r0 = osum + ((size_t)warp * 16 + gq) * kD + d0;
        float* r1 = osum + ((size_t)warp * 16 + gq + 8) * kD + d0;
        r0[0] = o[n][0] * f[0];
        r0[1] = o[n][1] * f[0];
        r1[0] = o[n][2] * f[1];
        r1[1] = o[n][3] * f[1];
    }
    __syncthreads();
    const bool split = n_active > 1;
    if (ks == 0) {
        bf16* og = reinterpret_cast<bf16*>(a.o);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = gq + 8 * h;
            const int v = rt * 16 + r;  // query vector within the tile
            if (v >= u.nq) continue;
            const int qi = u.q0 + v;
            const int row = qi / G, hh = u.g * G + (qi - row * G);
            bf16* dst = og + ((size_t)(u.row_base + row) * a.Hq + hh) * kD;
            const float inv = L[h] > 0.f ? 1.f / L[h] : 0.f;
            const size_t pofs = ((size_t)unit * a.pieces + piece) * kQTile + v;
            if (split && tq == 0) {
                a.part_ml[2 * pofs] = M[h];
                a.part_ml[2 * pofs + 1] = L[h];
            }
            for (int n = 0; n < 16; ++n) {
                const int d0 = n * 8 + 2 * tq;
                float v0 = 0.f, v1 = 0.f;
                for (int k2 = 0; k2 < KS; ++k2) {
                    const float* src = osum + ((size_t)(k2 * RT + rt) * 16 + r) * kD + d0;
                    v0 += src[0];
                    v1 += src[1];
                }
                if (split) {
                    *reinterpret_cast<float2*>(a.part_o + pofs * kD + d0) = make_float2(v0, v1);
                } else {
                    *reinterpret_cast<__nv_bfloat162*>(dst + d0) = __floats2bfloat162_rn(v0 * inv, v1 * inv);
                }
            }
        }
    }
    if (split) {
        // the piece holding the block chunk leaves its raw block scores for the importance
        if (FULL && a.imp_part != nullptr && c_end == n_chunks) {
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                if (n >= keys_per_warp / 8) continue;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int v = rt * 16 + gq + 8 * (e >> 1);
                    const int key = key0 + n * 8 + 2 * tq + (e & 1);
                    if (v < u.nq) a.sb_buf[((size_t)unit * kQTile + v) * kChunk + key] = sb[n][e];
                }
            }
        }
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) last_s = atomicAdd(&a.counters[unit], 1) == n_active - 1;
        __syncthreads();
        if (!last_s) return;
        __threadfence();
        // last piece of the unit: merge the pieces in piece order (deterministic)
        bf16* og = reinterpret_cast<bf16*>(a.o);
        for (int v = warp; v < u.nq; v += 4) {
            float mm = -CUDART_INF_F;
            for (int p2 = 0; p2 < n_active; ++p2)
                mm = fmaxf(mm, __ldcg(a.part_ml + 2 * (((size_t)unit * a.pieces + p2) * kQTile + v)));
            const float mu = mm == -CUDART_INF_F ? 0.f : mm;
            float ll = 0.f;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int p2 = 0; p2 < n_active; ++p2) {
                const size_t pofs = ((size_t)unit * a.pieces + p2) * kQTile + v;
                const float w = exp2f(__ldcg(a.part_ml + 2 * pofs) - mu);
                ll += __ldcg(a.part_ml + 2 * pofs + 1) * w;
                const float4 x = __ldcg(reinterpret_cast<const float4*>(a.part_o + pofs * kD) + lane);
                acc[0] += x.x * w;
                acc[1] += x.y * w;
                acc[2] += x.z * w;
                acc[3] += x.w * w;
            }
            if (lane == 0) {
                fin_s[v][0] = mu;
                fin_s[v][1] = ll;
            }
            const float inv = ll > 0.f ? 1.f / ll : 0.f;
            const int qi = u.q0 + v;
            const int row = qi / G, hh = u.g * G + (qi - row * G);
            bf16* dst = og + ((size_t)(u.row_base + row) * a.Hq + hh) * kD + lane * 4;
            *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
            *reinterpret_cast<__nv_bfloat162*>(dst + 2) = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
        }
        __syncthreads();
        if (threadIdx.x == 0) a.counters[unit] = 0;  // ready for the next launch
        if constexpr (FULL) {
            if (a.imp_part == nullptr) return;
            for (int j = threadIdx.x; j < a.B; j += 128) {
                float col = 0.f;
                for (int v = 0; v < u.nq; ++v) {
                    const float sv = __ldcg(a.sb_buf + ((size_t)unit * kQTile + v) * kChunk + j);
                    if (sv != -CUDART_INF_F && fin_s[v][1] > 0.f) col += exp2f(sv - fin_s[v][0]) / fin_s[v][1];
                }
                a.imp_part[(size_t)unit * a.B + j] = col;
            }
        }
        return;
    }
    if constexpr (FULL) {
    if (a.imp_part == nullptr) return;
    // ---- importance: column sums of the final probabilities of the block keys over this tile's vectors
    float cs[8][2];
#pragma unroll
    for (int n = 0; n < 8; ++n) {
        cs[n][0] = cs[n][1] = 0.f;
        if (n >= keys_per_warp / 8) continue;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int h = e >> 1;
            const bool row_ok = rt * 16 + gq + 8 * h < u.nq;
            const float p = (row_ok && sb[n][e] != -CUDART_INF_F && L[h] > 0.f) ? exp2f(sb[n][e] - M[h]) / L[h] : 0.f;
            cs[n][e & 1] += p;
        }
    }
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float v = cs[n][e];
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            cs[n][e] = v;
        }
    if (gq == 0) {
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            if (n >= keys_per_warp / 8) continue;
            col_s[rt][key0 + n * 8 + 2 * tq] = cs[n][0];
            col_s[rt][key0 + n * 8 + 2 * tq + 1] = cs[n][1];
        }
    }
    __syncthreads();
    for (int j = threadIdx.x; j < a.B; j += 128) {
        float v = 0.f;
        for (int t = 0; t < RT; ++t) v += col_s[t][j];
        a.imp_part[(size_t)unit * a.B + j] = v;
    }
    }  // FULL
}

}  // namespace

bool configure_attention_tc_kernels() {
    // once per context (device current): the shared-memory opt-in is not a stream operation, so it is
    // never made at launch time, where it would break stream capture
    return configure_attention_t5_kernels() && cudaFuncSetAttribute(attention_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem) ==
               cudaSuccess &&
           cudaFuncSetAttribute(attention_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem) ==
               cudaSuccess &&
           max_shared_carveout((const void*)attention_tc_kernel<true>) &&
           max_shared_carveout((const void*)attention_tc_kernel<false>);
}

int attention_q_tiles(int B, int G) {
    return attention_t5_used(B, G) ? attention_t5_q_tiles(B, G) : (B * G + kQTile - 1) / kQTile;
}

bool attention_tc_page_size_ok(int S) { return S == 16 || S == 32 || S == 64; }

int attention_pieces(int units, int max_chunks) {
    // aim at about four resident CTAs per SM-slot pair (148 SMs x 2 CTAs x 2) so that no single long
    // request walk sets the kernel's duration; capped by the split scratch
    constexpr int kTargetCtas = 4 * 148;
    // with at least one unit per SM the walks are long-lived streams already: splitting them only adds
    // start-up and merge cost per piece (measured, also with length-aware pieces), so only few-unit
    // launches are split
    if (units <= 0 || units >= 148 || units > kAttnSplitCap) return 1;
    int p = (kTargetCtas + units - 1) / units;
    if (p > max_chunks) p = max_chunks;
    if (p > kAttnSplitCap / units) p = kAttnSplitCap / units;
    return p < 1 ? 1 : p;
}

int launch_attention_tc(const AttnArgs& a, int q_tiles, cudaStream_t s) {
    if (a.N <= 0 || q_tiles <= 0) return 0;
    if (attention_t5_used(a.q_rows, a.Hq / a.Hkv)) return launch_attention_t5(a, q_tiles, s);
    // 2-D views for TMA: every (page, layer, K|V, head) block of S rows and every (request, layer,
    // K|V, head) cache block of B rows is a run of consecutive 256-byte rows
    CUtensorMap pool_map, ibc_map;
    const uint64_t ibc_rows = (uint64_t)a.N * a.L * 2 * a.Hkv * a.B;
    if (!tc::make_map(&ibc_map, a.ibc, ibc_rows, kD, (uint32_t)a.B, false)) return -1;
    if (a.n_pages > 0) {
        const uint64_t pool_rows = (uint64_t)a.n_pages * a.L * 2 * a.Hkv * a.page_size;
        if (!tc::make_map(&pool_map, a.kv_pool, pool_rows, kD, (uint32_t)a.page_size, false)) return -1;
    } else {
        pool_map = ibc_map;  // never used: with no pages every prefix key is invalid
    }
    const int smem = kAttnSmem;  // opted in by configure_attention_tc_kernels (at focus_init, per device)
    dim3 grid(a.Hkv * a.pieces, q_tiles, a.N);
    if (a.row_offsets == nullptr)
        return launched(launch_pdl(attention_tc_kernel<true>, grid, dim3(128), smem, s, 0, pool_map, ibc_map, a, q_tiles));
    return launched(launch_pdl(attention_tc_kernel<false>, grid, dim3(128), smem, s, 0, pool_map, ibc_map, a, q_tiles));
}

}  // namespace focus
