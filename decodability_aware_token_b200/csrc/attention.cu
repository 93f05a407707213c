// Attention of the block queries over paged prefix KV plus the intra-block KV cache, with the
// importance column sums fused in (layers 0 and 1).  SIMT version: one CTA per (request, KV head),
// one warp per query vector, online softmax over 32-key chunks.
//
// Importance ("FOCUS: DLLMs Know How to Tame Their Compute Bound", project page, Overview -- Design
// and Decodability Signal): for block key column j, sum over the group's query heads and all block
// query rows of the FINAL softmax probability.  Online softmax only knows the final row max m and
// denominator l at the end, so the raw block-column scores are kept in shared memory and turned into
// probabilities exp(s - m) / l once the row is done; each CTA writes the column sums of its KV group
// (fixed summation order, no float atomics) and the selection kernel adds the groups in order.
#include <math_constants.h>

#include "launch.h"

namespace focus {

namespace {

constexpr int kAttnWarps = 4;

template <typename T>
__device__ __forceinline__ const T* key_row(const AttnArgs& a, int b, int g, int t, int P, int kv, bool& ok) {
    const int d = a.d;
    if (t < P) {
        const int page = a.page_table[(size_t)b * a.max_pages + t / a.page_size];
        if (page < 0 || page >= a.n_pages) {
            ok = false;
            return nullptr;
        }
        const int slot = t % a.page_size;
        return reinterpret_cast<const T*>(a.kv_pool) +
               ((((size_t)page * a.L + a.layer) * 2 + kv) * a.Hkv + g) * (size_t)a.page_size * d + (size_t)slot * d;
    }
    const int j = t - P;
    return reinterpret_cast<const T*>(a.ibc) + ((((size_t)b * a.L + a.layer) * 2 + kv) * a.Hkv + g) * (size_t)a.B * d +
           (size_t)j * d;
}

template <typename T>
__global__ void __launch_bounds__(kAttnWarps * 32) attention_simt_kernel(AttnArgs a) {
    pdl_entry();
    extern __shared__ float smem[];
    const int b = blockIdx.x, g = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int d = a.d, G = a.Hq / a.Hkv;
    const int P = checked_prefix(a.prefix_len, b, a.max_pages * a.page_size, a.err);
    int row_base, n_rows;
    if (a.row_offsets) {
        row_base = a.row_offsets[b];
        n_rows = a.row_offsets[b + 1] - row_base;
    } else {
        row_base = b * a.B;
        n_rows = a.B;
    }
    const int nq = n_rows * G;
    const bool want_imp = a.imp_part != nullptr && a.row_offsets == nullptr;
    float* q_s = smem;                          // [warps][d]
    float* ml_s = q_s + kAttnWarps * d;         // [nq][2]
    float* sblk = ml_s + 2 * nq;                // [nq][B] raw block-column scores
    const int T_keys = P + a.B;
    const float scale = rsqrtf((float)d);
    const int per_lane = d / 32;
    const T* qsrc = reinterpret_cast<const T*>(a.q);
    T* odst = reinterpret_cast<T*>(a.o);

    for (int qi = warp; qi < nq; qi += kAttnWarps) {
        const int rr = qi / G, hh = g * G + (qi - rr * G);
        const size_t qoff = (size_t)(row_base + rr) * a.Hq * d + (size_t)hh * d;
        for (int u = 0; u < per_lane; ++u) q_s[warp * d + lane + 32 * u] = to_f(qsrc[qoff + lane + 32 * u]);
        __syncwarp();
        float m = -CUDART_INF_F, l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int kb = 0; kb < T_keys; kb += 32) {
            const int t = kb + lane;
            float s = -CUDART_INF_F;
            bool ok = t < T_keys;
            if (ok) {
                const T* kr = key_row<T>(a, b, g, t, P, 0, ok);
                if (ok) {
                    float dot = 0.f;
                    for (int i = 0; i < d; ++i) dot += q_s[warp * d + i] * to_f(kr[i]);
                    s = dot * scale;
                } else {
                    raise_err(a.err, FOCUS_DEVERR_PAGE_ID);
                }
            }
            if (want_imp && t >= P && t < T_keys) sblk[(size_t)qi * a.B + (t - P)] = s;
            const float m_new = fmaxf(m, warp_max(s));
            if (m_new == -CUDART_INF_F) continue;  // nothing valid yet
            const float p = ok ? expf(s - m_new) : 0.f;
            const float corr = expf(m - m_new);
            l = l * corr + warp_sum(p);
            for (int u = 0; u < per_lane; ++u) acc[u] *= corr;
            const int n_here = min(32, T_keys - kb);
            for (int k2 = 0; k2 < n_here; ++k2) {
                const float pk = __shfl_sync(0xffffffffu, p, k2);
                if (pk == 0.f) continue;
                bool vok = true;
                const T* vr = key_row<T>(a, b, g, kb + k2, P, 1, vok);
                if (!vok) continue;
                for (int u = 0; u < per_lane; ++u) acc[u] += pk * to_f(vr[lane + 32 * u]);
            }
            m = m_new;
        }
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        const size_t ooff = (size_t)(row_base + rr) * a.Hq * d + (size_t)hh * d;
        for (int u = 0; u < per_lane; ++u) odst[ooff + lane + 32 * u] = from_f<T>(acc[u] * inv_l);
        if (lane == 0) {
            ml_s[2 * qi] = m;
            ml_s[2 * qi + 1] = inv_l;
        }
        __syncwarp();
    }
    if (!want_imp) return;
    __syncthreads();
    for (int j = threadIdx.x; j < a.B; j += blockDim.x) {
        float col = 0.f;
        for (int qi = 0; qi < nq; ++qi) {
            const float s = sblk[(size_t)qi * a.B + j];
            if (s != -CUDART_INF_F) col += expf(s - ml_s[2 * qi]) * ml_s[2 * qi + 1];
        }
        a.imp_part[((size_t)b * a.Hkv + g) * a.B + j] = col;
    }
}

}  // namespace

bool configure_attention_kernels() {
    return max_shared_carveout((const void*)attention_simt_kernel<float>) &&
           max_shared_carveout((const void*)attention_simt_kernel<bf16>) && configure_attention_tc_kernels();
}

template <typename T>
int launch_attention(const AttnArgs& a, cudaStream_t s) {
    if (a.N <= 0) return 0;
    const int G = a.Hq / a.Hkv;
    const int nq_max = a.B * G;
    const bool imp = a.imp_part != nullptr && a.row_offsets == nullptr;
    size_t smem = sizeof(float) * ((size_t)kAttnWarps * a.d + 2 * (size_t)nq_max + (imp ? (size_t)nq_max * a.B : 0));
    if (smem > 48 * 1024)
        cudaFuncSetAttribute(attention_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 grid(a.N, a.Hkv);
    return launched(launch_pdl(attention_simt_kernel<T>, grid, dim3(kAttnWarps * 32), smem, s, 0, a));
}

template int launch_attention<float>(const AttnArgs&, cudaStream_t);
template int launch_attention<bf16>(const AttnArgs&, cudaStream_t);

}  // namespace focus
