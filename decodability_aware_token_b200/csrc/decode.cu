// LM-head combine (one CTA per kept row) + confidence-threshold decode (one CTA per request).
//
// The LM-head GEMM leaves, per kept row and vocabulary tile, the tile's max logit, the sum of
// exp(z - tile max) and the first (lowest-id) argmax, so logits never reach HBM.  Merging the tiles
// gives conf = max softmax = 1 / sum_v exp(z_v - z_max) and the top id (lowest id among equal maxima).
//
// Decode ("FOCUS: DLLMs Know How to Tame Their Compute Bound", project page, Quality table: the
// "Conf." threshold): a kept masked position decodes when conf > threshold; if none does and the
// request kept a masked position, the kept masked position with the highest conf decodes (lowest
// position on ties) so that each step makes progress.
#include <math_constants.h>

#include "launch.h"

namespace focus {

namespace {

constexpr int kDecodeWarps = 8;

__device__ __forceinline__ void merge_stats(float& m, float& s, int& a, float m2, float s2, int a2) {
    if (m2 > m) {
        s = (m == -CUDART_INF_F ? 0.f : s * expf(m - m2)) + s2;
        m = m2;
        a = a2;
    } else if (m2 == m) {
        s += s2;
        a = min(a, a2);
    } else if (m2 != -CUDART_INF_F) {
        s += s2 * expf(m2 - m);
    }
}

// One CTA per kept row: merge the row's vocabulary-tile statistics into its confidence and top id.
// Each thread loads its tiles (8 at a time, all in flight) before merging them; threads, then warps,
// are merged in a fixed order.
constexpr int kCombineThreads = 256;
constexpr int kCombineBatch = 8;
__global__ void __launch_bounds__(kCombineThreads) lm_combine_kernel(const float* __restrict__ lm_max,
                                                                     const float* __restrict__ lm_sum,
                                                                     const int32_t* __restrict__ lm_arg, int n_tiles,
                                                                     const int32_t* __restrict__ n_rows,
                                                                     float* __restrict__ row_conf,
                                                                     int32_t* __restrict__ row_top) {
    pdl_entry();
    __shared__ float wm[kCombineThreads / 32], ws[kCombineThreads / 32];
    __shared__ int wa[kCombineThreads / 32];
    const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (r >= *n_rows) return;
    const size_t base = (size_t)r * n_tiles;
    float m = -CUDART_INF_F, s = 0.f;
    int arg = 0x7fffffff;
    for (int t0 = 0; t0 < n_tiles; t0 += kCombineThreads * kCombineBatch) {
        float bm[kCombineBatch], bs[kCombineBatch];
        int ba[kCombineBatch];
#pragma unroll
        for (int i = 0; i < kCombineBatch; ++i) {
            const int t = t0 + i * kCombineThreads + tid;
            const bool ok = t < n_tiles;
            bm[i] = ok ? lm_max[base + t] : -CUDART_INF_F;
            bs[i] = ok ? lm_sum[base + t] : 0.f;
            ba[i] = ok ? lm_arg[base + t] : 0x7fffffff;
        }
#pragma unroll
        for (int i = 0; i < kCombineBatch; ++i) merge_stats(m, s, arg, bm[i], bs[i], ba[i]);
    }
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
        const int a2 = __shfl_xor_sync(0xffffffffu, arg, o);
        merge_stats(m, s, arg, m2, s2, a2);
    }
    if (lane == 0) {
        wm[warp] = m;
        ws[warp] = s;
        wa[warp] = arg;
    }
    __syncthreads();
    if (tid == 0) {
        for (int w = 1; w < kCombineThreads / 32; ++w) merge_stats(m, s, arg, wm[w], ws[w], wa[w]);
        row_conf[r] = 1.f / s;
        row_top[r] = arg;
    }
}

__global__ void __launch_bounds__(kDecodeWarps * 32) decode_kernel(DecodeArgs a) {
    pdl_entry();
    __shared__ float conf_s[64];
    __shared__ int top_s[64];
    const int b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k = a.keep_count[b], off = a.row_offsets[b], B = a.B;
    for (int j = threadIdx.x; j < B; j += blockDim.x) a.decoded_ids[(size_t)b * B + j] = -1;
    for (int t = threadIdx.x; t < k; t += blockDim.x) {
        conf_s[t] = a.row_conf[off + t];
        top_s[t] = a.row_top[off + t];
    }
    __syncthreads();
    for (int t = threadIdx.x; t < a.max_keep; t += blockDim.x) {
        a.conf_out[(size_t)b * a.max_keep + t] = t < k ? conf_s[t] : 0.f;
        a.top_out[(size_t)b * a.max_keep + t] = t < k ? top_s[t] : -1;
    }
    if (warp != 0) return;
    bool cand[2], dec[2];
    int pos[2];
    float cf[2];
    for (int h = 0; h < 2; ++h) {
        const int t = lane + 32 * h;
        pos[h] = t < k ? a.retained_idx[(size_t)b * a.max_keep + t] : -1;
        cand[h] = pos[h] >= 0 && a.mask[(size_t)b * B + pos[h]] != 0;
        cf[h] = cand[h] ? conf_s[t] : -1.f;
        dec[h] = cand[h] && cf[h] > a.threshold;
    }
    const bool any_dec = __any_sync(0xffffffffu, dec[0] || dec[1]);
    const bool any_cand = __any_sync(0xffffffffu, cand[0] || cand[1]);
    if (!any_dec && any_cand) {
        // highest confidence; ties -> lowest slot, i.e. lowest position (slots are ascending)
        float best = -1.f;
        int slot = 1 << 30;
        for (int h = 0; h < 2; ++h)
            if (cand[h] && (cf[h] > best || (cf[h] == best && lane + 32 * h < slot))) {
                best = cf[h];
                slot = lane + 32 * h;
            }
        for (int o = 16; o > 0; o >>= 1) {
            const float b2 = __shfl_xor_sync(0xffffffffu, best, o);
            const int s2 = __shfl_xor_sync(0xffffffffu, slot, o);
            if (b2 > best || (b2 == best && s2 < slot)) {
                best = b2;
                slot = s2;
            }
        }
        for (int h = 0; h < 2; ++h) dec[h] = (lane + 32 * h) == slot;
    }
    for (int h = 0; h < 2; ++h) {
        if (!dec[h]) continue;
        const int t = lane + 32 * h, j = pos[h];
        const int id = top_s[t];
        a.decoded_ids[(size_t)b * B + j] = id;
        a.tokens[(size_t)b * B + j] = id;
        a.mask[(size_t)b * B + j] = 0;
    }
}

}  // namespace

bool configure_select_decode_kernels() {
    return configure_select_kernel() && max_shared_carveout((const void*)decode_kernel) &&
           max_shared_carveout((const void*)lm_combine_kernel);
}

int launch_lm_combine(const DecodeArgs& a, int rows_bound, const int32_t* n_rows, cudaStream_t s) {
    if (rows_bound <= 0) return 0;
    return launched(launch_pdl(lm_combine_kernel, dim3(rows_bound), dim3(kCombineThreads), 0, s, 0, a.lm_max, a.lm_sum,
                               a.lm_arg, a.n_tiles, n_rows, a.row_conf, a.row_top));
}

int launch_decode(const DecodeArgs& a, cudaStream_t s) {
    if (a.N <= 0) return 0;
    return launched(launch_pdl(decode_kernel, dim3(a.N), dim3(kDecodeWarps * 32), 0, s, 0, a));
}

}  // namespace focus
