// bf16 attention of block queries over paged prefix KV plus the intra-block KV cache, on tensor cores
// (mma.sync m16n8k16, fp32 accumulate), with the importance column sums fused in for layers 0 and 1.
//
// "FOCUS: DLLMs Know How to Tame Their Compute Bound", project page, Overview -- Design / Decodability
// Signal (importance from the early layers' Q/K attention) and Runtime Action (ragged execution and the
// intra-block KV cache); news article on the same paper, "Arquitetura do FOCUS" (ragged paged attention).
//
// Work unit (one CTA): request b, KV head g, and a tile of up to 64 query vectors of that group
// (query vector qi = row * G + head-in-group).  Keys are walked in 64-key chunks: the prefix in page
// order (page-table lookups per 16-byte copy, so any page size works), then the block's B keys from the
// intra-block cache as the last chunk.  Chunks are double-buffered through XOR-swizzled shared memory
// with cp.async.  The 4 warps split the work as RT row tiles x KS key slices (RT * KS = 4): 64 query
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

namespace focus {

namespace {

constexpr int kChunk = 64;      // keys per chunk
constexpr int kD = 128;         // head dim (bf16 path)
constexpr int kQTile = 64;      // query vectors per CTA
constexpr int kRowBytes = kD * 2;
constexpr int kTileBytes = kChunk * kRowBytes;  // 16 KB

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// byte offset of 16-byte column chunk c of row r in a swizzled [rows][128] bf16 tile
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * kRowBytes + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    const int n = valid ? 16 : 0;  // 0 source bytes: zero-fill
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

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

struct Unit {
    int b, g, qt, P, row_base, n_rows, nq, q0;
};

template <bool FULL>
__global__ void __launch_bounds__(128, 2) attention_tc_kernel(AttnArgs a, int q_tiles) {
    extern __shared__ __align__(128) uint8_t smem[];
    // [0, 64K): K/V double buffer (stage s: K at 2s*16K, V at (2s+1)*16K); [64K, 80K): Q tile
    uint8_t* kv = smem;
    uint8_t* qs = smem + 4 * kTileBytes;
    __shared__ float ml_s[4][16][2];      // per warp: row max / denominator (log2 domain)
    __shared__ float col_s[4][kChunk];    // per row tile: block-key column sums

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.Hq / a.Hkv;
    Unit u;
    u.b = blockIdx.x;
    u.g = blockIdx.y;
    u.qt = blockIdx.z;
    u.P = checked_prefix(a.prefix_len, u.b, a.max_pages * a.page_size, a.err);
    if (FULL) {
        u.row_base = u.b * a.B;
        u.n_rows = a.B;
    } else {
        u.row_base = a.row_offsets[u.b];
        u.n_rows = a.row_offsets[u.b + 1] - u.row_base;
    }
    u.q0 = u.qt * kQTile;
    u.nq = min(kQTile, u.n_rows * G - u.q0);
    if (u.nq <= 0) return;
    const int RT = u.nq <= 16 ? 1 : (u.nq <= 32 ? 2 : 4);
    const int KS = 4 / RT;
    const int rt = warp % RT, ks = warp / RT;
    const int keys_per_warp = kChunk / KS;  // 64, 32 or 16
    const int key0 = ks * keys_per_warp;

    const bf16* qg = reinterpret_cast<const bf16*>(a.q);
    const bf16* pool = reinterpret_cast<const bf16*>(a.kv_pool);
    const bf16* ibc = reinterpret_cast<const bf16*>(a.ibc);
    const size_t ibc_k = ((((size_t)u.b * a.L + a.layer) * 2 + 0) * a.Hkv + u.g) * (size_t)a.B * kD;
    const size_t ibc_v = ((((size_t)u.b * a.L + a.layer) * 2 + 1) * a.Hkv + u.g) * (size_t)a.B * kD;
    const int n_prefix_chunks = (u.P + kChunk - 1) / kChunk;
    const int n_chunks = n_prefix_chunks + 1;

    // ---- Q tile -> shared (rows beyond nq zero-filled)
    for (int i = threadIdx.x; i < kQTile * 16; i += 128) {
        const int r = i >> 4, c = i & 15;
        const int qi = u.q0 + r;
        const bool ok = r < u.nq;
        const int row = qi / G, hh = u.g * G + (qi - (qi / G) * G);
        const bf16* src = qg + ((size_t)(u.row_base + (ok ? row : 0)) * a.Hq + (ok ? hh : 0)) * kD + c * 8;
        cp_async16(smem_u32(qs) + swz(r, c), src, ok);
    }
    // ---- chunk loader: K and V rows of chunk `ci` into stage `st`
    auto load_chunk = [&](int ci, int st) {
        const uint32_t kdst = smem_u32(kv) + (2 * st) * kTileBytes;
        const uint32_t vdst = kdst + kTileBytes;
        for (int i = threadIdx.x; i < kChunk * 16; i += 128) {
            const int r = i >> 4, c = i & 15;
            const bf16* ks_src = pool;
            const bf16* vs_src = pool;
            bool ok;
            if (ci < n_prefix_chunks) {
                const int t = ci * kChunk + r;
                ok = t < u.P;
                if (ok) {
                    const int page = a.page_table[(size_t)u.b * a.max_pages + t / a.page_size];
                    if (page < 0 || page >= a.n_pages) {
                        raise_err(a.err, FOCUS_DEVERR_PAGE_ID);
                        ok = false;
                    } else {
                        const size_t base = ((((size_t)page * a.L + a.layer) * 2) * a.Hkv + u.g) * (size_t)a.page_size * kD +
                                            (size_t)(t % a.page_size) * kD + c * 8;
                        ks_src = pool + base;
                        vs_src = pool + base + (size_t)a.Hkv * a.page_size * kD;
                    }
                }
            } else {
                ok = r < a.B;
                if (ok) {
                    ks_src = ibc + ibc_k + (size_t)r * kD + c * 8;
                    vs_src = ibc + ibc_v + (size_t)r * kD + c * 8;
                }
            }
            cp_async16(kdst + swz(r, c), ks_src, ok);
            cp_async16(vdst + swz(r, c), vs_src, ok);
        }
    };
    auto key_valid = [&](int ci, int key) -> bool {
        if (ci < n_prefix_chunks) {
            const int t = ci * kChunk + key;
            if (t >= u.P) return false;
            const int page = a.page_table[(size_t)u.b * a.max_pages + t / a.page_size];
            return page >= 0 && page < a.n_pages;
        }
        return key < a.B;
    };

    load_chunk(0, 0);
    cp_commit();

    // ---- Q fragments (A operand) for this warp's 16 rows, all 8 k-steps of d
    cp_wait<0>();
    __syncthreads();
    uint32_t qf[8][4];
    {
        const int r = rt * 16 + (lane & 15);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int c = kk * 2 + (lane >> 4);
            ldsm_x4(smem_u32(qs) + swz(r, c), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
        }
    }
    const float sl2 = rsqrtf((float)kD) * 1.4426950408889634f;  // 1/sqrt(d) * log2(e)
    float m_r[2] = {-CUDART_INF_F, -CUDART_INF_F}, l_r[2] = {0.f, 0.f};
    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float sb[8][4];  // raw (scaled) scores of the block chunk, kept for the importance
#pragma unroll
    for (int n = 0; n < 8; ++n) sb[n][0] = sb[n][1] = sb[n][2] = sb[n][3] = -CUDART_INF_F;

    const int gq = lane >> 2, tq = lane & 3;
    for (int ci = 0; ci < n_chunks; ++ci) {
        const int st = ci & 1;
        if (ci + 1 < n_chunks) load_chunk(ci + 1, st ^ 1);
        cp_commit();
        cp_wait<1>();
        __syncthreads();
        const uint32_t kbase = smem_u32(kv) + (2 * st) * kTileBytes;
        const uint32_t vbase = kbase + kTileBytes;
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
                const float v = key_valid(ci, key) ? s[n][e] * sl2 : -CUDART_INF_F;
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
        __syncthreads();  // stage st is refilled by the next iteration's prefetch
    }
    cp_wait<0>();

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
    // o slices -> shared (fp32), summed by the ks == 0 warp of each row tile
    float* osum = reinterpret_cast<float*>(smem);  // reuses the K/V buffers: [warps][16][128]
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
    if (ks == 0) {
        bf16* og = reinterpret_cast<bf16*>(a.o);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = gq + 8 * h;
            const int qi = u.q0 + rt * 16 + r;
            if (rt * 16 + r >= u.nq) continue;
            const int row = qi / G, hh = u.g * G + (qi - (qi / G) * G);
            bf16* dst = og + ((size_t)(u.row_base + row) * a.Hq + hh) * kD;
            const float inv = L[h] > 0.f ? 1.f / L[h] : 0.f;
            for (int n = 0; n < 16; ++n) {
                const int d0 = n * 8 + 2 * tq;
                float v0 = 0.f, v1 = 0.f;
                for (int k2 = 0; k2 < KS; ++k2) {
                    const float* src = osum + ((size_t)(k2 * RT + rt) * 16 + r) * kD + d0;
                    v0 += src[0];
                    v1 += src[1];
                }
                *reinterpret_cast<__nv_bfloat162*>(dst + d0) = __floats2bfloat162_rn(v0 * inv, v1 * inv);
            }
        }
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
        a.imp_part[(((size_t)u.b * a.Hkv + u.g) * q_tiles + u.qt) * a.B + j] = v;
    }
    }  // FULL
}

}  // namespace

int attention_q_tiles(int B, int G) { return (B * G + kQTile - 1) / kQTile; }

int launch_attention_tc(const AttnArgs& a, int q_tiles, cudaStream_t s) {
    if (a.N <= 0 || q_tiles <= 0) return 0;
    const int smem = 4 * kTileBytes + kQTile * kRowBytes;  // 80 KB
    dim3 grid(a.N, a.Hkv, q_tiles);
    if (a.row_offsets == nullptr) {
        cudaFuncSetAttribute(attention_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        attention_tc_kernel<true><<<grid, 128, smem, s>>>(a, q_tiles);
    } else {
        cudaFuncSetAttribute(attention_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        attention_tc_kernel<false><<<grid, 128, smem, s>>>(a, q_tiles);
    }
    return 1;
}

}  // namespace focus
