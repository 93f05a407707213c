// Importance delta -> adaptive budget -> top-k with index tie-break -> ragged row map.
//
// "FOCUS: DLLMs Know How to Tame Their Compute Bound", project page, Overview -- Decodability Signal
// (layer-0-to-1 importance delta), Design (keep likely-decodable candidates under an adaptive budget)
// and Runtime Action (dynamic budgeting, token eviction, ragged execution); news article on the same
// paper, "Arquitetura do FOCUS" (target token selection, state compaction).
//
// Rules: c = #{masked j : delta_j > tau};  k = min(clamp(ceil(alpha c), k_min, k_max), #masked)
// (product and ceil in float32); kept = the k best masked positions under (delta desc, j asc),
// written ascending.  Forced fraction f >= 0: k = min(B, ceil(f B)) over all positions under
// (masked first, delta desc, j asc).
//
// Two kernels.  select_kernel: a warp per request, eight requests per CTA (B <= 64: each lane owns positions
// lane and lane + 32): the request's importance partials summed in group order, ballots for the counts, an
// O(B) rank per position (B^2 <= 4096 compares per request), the kept positions written ascending.
// rowmap_kernel: one CTA scans the kept counts (block-wide, in order of requests) into the row offsets and
// writes the ragged row map.  Both are latency-bound; spreading the requests over CTAs keeps the read of
// the importance partials (4 MB at 256 requests of block 64 with 32 groups) parallel.
#include "launch.h"

namespace focus {

namespace {

__device__ __forceinline__ bool key_less(bool forced, bool ma, float da, int ja, bool mb, float db, int jb) {
    if (forced && ma != mb) return ma;  // masked positions first
    if (da != db) return da > db;       // larger delta first
    return ja < jb;                     // lower position first
}

constexpr int kSelWarps = 8;  // requests per select CTA

__global__ void __launch_bounds__(32 * kSelWarps) select_kernel(SelectArgs a) {
    pdl_entry();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = a.B;
    const bool forced = a.forced_frac >= 0.f;
    const size_t layer_stride = (size_t)a.N * a.groups * B;

    const int b = blockIdx.x * kSelWarps + warp;
    if (b < a.N) {
        float dl[2];
        bool valid[2], msk[2], keep[2];
        for (int h = 0; h < 2; ++h) {
            const int j = lane + 32 * h;
            valid[h] = j < B;
            dl[h] = 0.f;
            msk[h] = false;
            if (valid[h]) {
                float i0 = 0.f, i1 = 0.f;
#pragma unroll 8
                for (int g = 0; g < a.groups; ++g) {  // partial groups in order: deterministic
                    i0 += a.imp_part[((size_t)b * a.groups + g) * B + j];
                    i1 += a.imp_part[layer_stride + ((size_t)b * a.groups + g) * B + j];
                }
                dl[h] = i1 - i0;
                msk[h] = a.mask[(size_t)b * B + j] != 0;
                if (a.importance_out) {
                    a.importance_out[(size_t)b * B + j] = i0;
                    a.importance_out[(size_t)a.N * B + (size_t)b * B + j] = i1;
                }
            }
        }
        if (a.forced_idx) {
            // caller-chosen set: ascending positions in [0, B), count <= max_keep
            const int cnt = a.forced_cnt[b];
            bool bad = cnt < 0 || cnt > a.max_keep || cnt > B;
            unsigned long long bits = 0ull;
            if (!bad) {
                for (int t = lane; t < cnt; t += 32) {
                    const int j = a.forced_idx[(size_t)b * a.max_keep + t];
                    const int prev = t > 0 ? a.forced_idx[(size_t)b * a.max_keep + t - 1] : -1;
                    if (j < 0 || j >= B || j <= prev) bad = true;
                    else bits |= 1ull << j;
                }
            }
            for (int o = 16; o > 0; o >>= 1) bits |= __shfl_xor_sync(0xffffffffu, bits, o);
            bad = __any_sync(0xffffffffu, bad);
            if (bad) {
                if (lane == 0) raise_err(a.err, FOCUS_DEVERR_FORCED_SET);
                bits = 0ull;
            }
            for (int h = 0; h < 2; ++h) keep[h] = valid[h] && ((bits >> (lane + 32 * h)) & 1ull);
        } else {
            bool elig[2];
            for (int h = 0; h < 2; ++h) elig[h] = valid[h] && (forced || msk[h]);
            int k;
            if (forced) {
                k = min(B, (int)ceilf(a.forced_frac * (float)B));
            } else {
                const int c = __popc(__ballot_sync(0xffffffffu, elig[0] && dl[0] > a.tau)) +
                              __popc(__ballot_sync(0xffffffffu, elig[1] && dl[1] > a.tau));
                const int n_el = __popc(__ballot_sync(0xffffffffu, elig[0])) + __popc(__ballot_sync(0xffffffffu, elig[1]));
                k = (int)ceilf(a.alpha * (float)c);
                k = max(k, a.k_min);
                k = min(k, a.k_max);
                k = min(k, n_el);
            }
            int rank[2] = {0, 0};
            for (int jj = 0; jj < B; ++jj) {
                const int src = jj & 31, hh = jj >> 5;
                const float d2 = __shfl_sync(0xffffffffu, hh ? dl[1] : dl[0], src);
                const bool m2 = __shfl_sync(0xffffffffu, (int)(hh ? msk[1] : msk[0]), src) != 0;
                const bool e2 = __shfl_sync(0xffffffffu, (int)(hh ? elig[1] : elig[0]), src) != 0;
                for (int h = 0; h < 2; ++h)
                    if (e2 && key_less(forced, m2, d2, jj, msk[h], dl[h], lane + 32 * h)) ++rank[h];
            }
            for (int h = 0; h < 2; ++h) keep[h] = elig[h] && rank[h] < k;
        }
        const unsigned lo = __ballot_sync(0xffffffffu, keep[0]);
        const unsigned hi = __ballot_sync(0xffffffffu, keep[1]);
        const int kept = __popc(lo) + __popc(hi);
        const unsigned lt = (1u << lane) - 1u;
        int32_t* ret = a.retained_idx + (size_t)b * a.max_keep;
        if (keep[0]) ret[__popc(lo & lt)] = lane;
        if (keep[1]) ret[__popc(lo) + __popc(hi & lt)] = lane + 32;
        for (int t = kept + lane; t < a.max_keep; t += 32) ret[t] = -1;
        if (lane == 0) a.keep_count[b] = kept;
    }
}

// Exclusive scan of the kept counts (requests in order) into row_offsets and the live row count, then the
// row map: compacted row row_offsets[b] + t is position retained_idx[b][t] of request b.
__global__ void __launch_bounds__(1024) rowmap_kernel(SelectArgs a) {
    pdl_entry();
    __shared__ int32_t warp_sum[32];
    __shared__ int32_t carry_s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) carry_s = 0;
    __syncthreads();
    for (int base = 0; base < a.N; base += 1024) {
        const int b = base + tid;
        const int v = b < a.N ? a.keep_count[b] : 0;
        int inc = v;  // inclusive scan within the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        if (lane == 31) warp_sum[warp] = inc;
        __syncthreads();
        if (warp == 0) {
            int w = warp_sum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            warp_sum[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        const int carry = carry_s;
        if (b < a.N) a.row_offsets[b] = carry + (warp > 0 ? warp_sum[warp - 1] : 0) + inc - v;
        __syncthreads();
        if (tid == 0) carry_s = carry + warp_sum[31];
        __syncthreads();
    }
    if (tid == 0) {
        a.row_offsets[a.N] = carry_s;
        *a.n_rows = carry_s;
    }
    __syncthreads();  // the offsets this CTA wrote are visible to all of its threads
    for (int b = warp; b < a.N; b += 32) {
        const int off = a.row_offsets[b], k = a.keep_count[b];
        for (int t = lane; t < k; t += 32) {
            const int j = a.retained_idx[(size_t)b * a.max_keep + t];
            a.row_req[off + t] = b;
            a.row_pos[off + t] = j;
            a.row_src[off + t] = b * a.B + j;
        }
    }
    if (a.order) {
        // requests by descending prefix length (ties by index): request b goes to the slot of its rank
        auto len = [&](int b) { return min(max(a.prefix_len[b], 0), a.max_prefix); };
        for (int b = tid; b < a.N; b += 1024) {
            const int pb = len(b);
            int rank = 0;
            for (int c = 0; c < a.N; ++c) {
                const int pc = len(c);
                rank += (pc > pb || (pc == pb && c < b)) ? 1 : 0;
            }
            a.order[rank] = b;
        }
    }
}

}  // namespace

bool configure_select_kernel() {
    return max_shared_carveout((const void*)select_kernel) && max_shared_carveout((const void*)rowmap_kernel);
}

int launch_select(const SelectArgs& a, cudaStream_t s) {
    if (a.N <= 0) return 0;
    const dim3 grid((a.N + kSelWarps - 1) / kSelWarps);
    if (launch_pdl(select_kernel, grid, dim3(32 * kSelWarps), 0, s, 0, a) != cudaSuccess) return -1;
    return launch_pdl(rowmap_kernel, dim3(1), dim3(1024), 0, s, 0, a) == cudaSuccess ? 2 : -1;
}

}  // namespace focus
