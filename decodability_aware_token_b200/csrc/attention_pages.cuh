// Paged K/V chunks for the attention kernels: one TMA-fed 64-key chunk of a request's keys is either
// 64 / S prefix pages (each page's K and V rows of one layer and KV head) or the request's B block keys
// from the intra-block KV cache.  A chunk lands in shared memory as four [64 keys][64 d] bf16 half-tiles
// with the 128-byte swizzle: K of dims 0-63, K of dims 64-127, V of dims 0-63, V of dims 64-127.
#pragma once
#include "launch.h"
#include "tc_gemm_kernel.cuh"

namespace focus {
namespace {

using tc::mbar_expect_tx;
using tc::mbar_init;
using tc::mbar_wait;
using tc::tma_load_2d;

constexpr int kChunk = 64;                  // keys per chunk
constexpr int kD = 128;                     // head dim (bf16 path)
constexpr int kHalf = kChunk * 128;         // one [64 keys][64 d] bf16 half-tile: 8 KB
constexpr int kStageBytes = 4 * kHalf;      // K lo, K hi, V lo, V hi: 32 KB
constexpr int kPtCache = 512;               // page-table entries cached in shared memory

struct Unit {
    int b, g, qt, P, row_base, n_rows, nq, q0;
};

// Issue the TMA copies of chunk `ci` into stage `st` (one thread).  Prefix chunks copy whole pages
// (64 / S pages, each as K and V halves); the last chunk copies the block's B cache rows.  Pages past
// the prefix or with an out-of-range id are skipped (their keys stay masked).  Returns the valid-key
// mask of the chunk.
__device__ __forceinline__ uint64_t issue_chunk(const AttnArgs& a, const Unit& u, const CUtensorMap* pool_map,
                                                const CUtensorMap* ibc_map, uint8_t* stage, uint64_t* bar, int ci,
                                                int n_prefix_chunks, const int32_t* pt) {
    const int S = a.page_size;
    uint64_t mask = 0;
    if (ci < n_prefix_chunks) {
        uint32_t bytes = 0;
        for (int p = 0; p < kChunk / S; ++p) {
            const int t0 = ci * kChunk + p * S;
            if (t0 >= u.P) break;
            const int page = pt[t0 / S];
            if (page < 0 || page >= a.n_pages) {
                raise_err(a.err, FOCUS_DEVERR_PAGE_ID);
                continue;
            }
            bytes += 4u * S * 128u;
            const int n = min(S, u.P - t0);
            mask |= (n == 64 ? ~0ull : ((1ull << n) - 1ull)) << (p * S);
        }
        mbar_expect_tx(bar, bytes);
        for (int p = 0; p < kChunk / S; ++p) {
            const int t0 = ci * kChunk + p * S;
            if (t0 >= u.P) break;
            const int page = pt[t0 / S];
            if (page < 0 || page >= a.n_pages) continue;
            const int krow = (int)(((((size_t)page * a.L + a.layer) * 2 + 0) * a.Hkv + u.g) * S);
            const int vrow = krow + a.Hkv * S;
            uint8_t* dst = stage + p * S * 128;
            tma_load_2d(pool_map, bar, dst, 0, krow);
            tma_load_2d(pool_map, bar, dst + kHalf, 64, krow);
            tma_load_2d(pool_map, bar, dst + 2 * kHalf, 0, vrow);
            tma_load_2d(pool_map, bar, dst + 3 * kHalf, 64, vrow);
        }
    } else {
        const int krow = (int)(((((size_t)u.b * a.L + a.layer) * 2 + 0) * a.Hkv + u.g) * a.B);
        const int vrow = krow + a.Hkv * a.B;
        mbar_expect_tx(bar, 4u * a.B * 128u);
        tma_load_2d(ibc_map, bar, stage, 0, krow);
        tma_load_2d(ibc_map, bar, stage + kHalf, 64, krow);
        tma_load_2d(ibc_map, bar, stage + 2 * kHalf, 0, vrow);
        tma_load_2d(ibc_map, bar, stage + 3 * kHalf, 64, vrow);
        mask = a.B == 64 ? ~0ull : ((1ull << a.B) - 1ull);
    }
    return mask;
}

// Ask L2 for the K and V rows of prefix chunk `ci` (one bulk prefetch per page and K / V; no shared memory,
// no barrier), issued one chunk ahead of the ring's copies: one more chunk of DRAM requests in flight per CTA
// than the shared-memory ring holds, with an L2 footprint (one chunk per CTA, ~10 MB) far below its capacity.
// (Four chunks ahead raised DRAM reads by a fifth: the lines were evicted before their copies came.)
// Pages past the prefix or with an out-of-range id are skipped; the block chunk is not prefetched.
__device__ __forceinline__ void prefetch_chunk_l2(const AttnArgs& a, const Unit& u, int ci, int n_prefix_chunks,
                                                  const int32_t* pt) {
    if (ci >= n_prefix_chunks) return;
    const int S = a.page_size;
    const uint32_t bytes = (uint32_t)S * kD * 2;  // S rows of 256 bytes: a multiple of 16
    for (int p = 0; p < kChunk / S; ++p) {
        const int t0 = ci * kChunk + p * S;
        if (t0 >= u.P) break;
        const int page = pt[t0 / S];
        if (page < 0 || page >= a.n_pages) continue;
        const size_t krow = ((((size_t)page * a.L + a.layer) * 2 + 0) * a.Hkv + u.g) * (size_t)S;
        const uint8_t* kp = reinterpret_cast<const uint8_t*>(a.kv_pool) + krow * kD * 2;
        const uint8_t* vp = kp + (size_t)a.Hkv * S * kD * 2;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(kp), "r"(bytes) : "memory");
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(vp), "r"(bytes) : "memory");
    }
}

}  // namespace
}  // namespace focus
