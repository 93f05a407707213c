// LM-head combine + confidence-threshold decode.
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

__global__ void __launch_bounds__(kDecodeWarps * 32) decode_kernel(DecodeArgs a) {
    __shared__ float conf_s[64];
    __shared__ int top_s[64];
    const int b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k = a.keep_count[b], off = a.row_offsets[b], B = a.B;
    for (int j = threadIdx.x; j < B; j += blockDim.x) a.decoded_ids[(size_t)b * B + j] = -1;
    for (int t = warp; t < k; t += kDecodeWarps) {
        const size_t r = (size_t)(off + t);
        float m = -CUDART_INF_F, s = 0.f;
        int arg = 0x7fffffff;
        for (int tile = lane; tile < a.n_tiles; tile += 32)
            merge_stats(m, s, arg, a.lm_max[r * a.n_tiles + tile], a.lm_sum[r * a.n_tiles + tile],
                        a.lm_arg[r * a.n_tiles + tile]);
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
            const int a2 = __shfl_xor_sync(0xffffffffu, arg, o);
            merge_stats(m, s, arg, m2, s2, a2);
        }
        if (lane == 0) {
            conf_s[t] = 1.f / s;
            top_s[t] = arg;
        }
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

int launch_decode(const DecodeArgs& a, cudaStream_t s) {
    if (a.N <= 0) return 0;
    decode_kernel<<<a.N, kDecodeWarps * 32, 0, s>>>(a);
    return 1;
}

}  // namespace focus
