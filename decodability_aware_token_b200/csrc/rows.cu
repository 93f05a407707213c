// Row-wise kernels of the step: embedding + RMSNorm, residual reduction + RMSNorm (optionally
// gathering the kept rows), and the QKV finalisation (RoPE + intra-block KV-cache write).
// With a few dozen kept rows these kernels are latency-bound, so each CTA takes one row and issues
// every load of the row (float4, all in flight together) before using any; reductions run in a fixed
// order.
#include "launch.h"

namespace focus {

namespace {

constexpr int kRowThreads = 256;
constexpr int kMaxNormSplits = 8;  // split-K partial slices a norm kernel adds (CUDA-core path: at most 1)

// One CTA per row: x = E[token], h = RMSNorm(x) * gamma.
template <typename T>
__global__ void __launch_bounds__(kNormThreads) embed_norm_kernel(const int32_t* __restrict__ tokens, int V,
                                                                  const T* __restrict__ embed,
                                                                  const T* __restrict__ gamma, float eps, int D,
                                                                  float* __restrict__ x, T* __restrict__ h, int* err) {
    // the step's first kernel: its successors may start only once everything queued before the step
    // (a block commit writing the KV pool and prefix lengths, the caller's copies) has completed, so the
    // step's kernels can read such inputs before their own programmatic-launch wait
    pdl_wait();
    pdl_trigger();
    __shared__ float red[32];
    const int r = blockIdx.x, tid = threadIdx.x;
    int tok = tokens[r];
    if (tok < 0 || tok >= V) {
        if (tid == 0) raise_err(err, FOCUS_DEVERR_TOKEN_ID);
        tok = 0;
    }
    const T* e = embed + (size_t)tok * D;
    float* xr = x + (size_t)r * D;
    float4 v[kNormVec];
#pragma unroll
    for (int i = 0; i < kNormVec; ++i) {
        const int c = (i * kNormThreads + tid) * 4;
        v[i] = c < D ? load4<T>(e + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < kNormVec; ++i) {
        const int c = (i * kNormThreads + tid) * 4;
        if (c < D) *reinterpret_cast<float4*>(xr + c) = v[i];
    }
    rmsnorm_finish_cta<T>(v, D, gamma, eps, h + (size_t)r * D, red);
}

// One CTA per row: x_out[r] = x_in[src] + the split partials (src = src_map ? src_map[r] : r), then
// h_out[r] = RMSNorm(x_out[r]) * gamma.  Every load of the row is issued before any is used.
template <typename T>
__global__ void __launch_bounds__(kNormThreads) residual_norm_kernel(
    const float* __restrict__ x_in, const int32_t* __restrict__ src_map, const int32_t* __restrict__ n_rows_dev,
    const float* __restrict__ part, int n_splits, size_t part_stride, float* x_out, const T* __restrict__ gamma,
    float eps, int D, T* __restrict__ h_out) {
    pdl_entry();
    __shared__ float red[32];
    const int r = blockIdx.x, tid = threadIdx.x;
    if (n_rows_dev && r >= *n_rows_dev) return;
    const int src = src_map ? src_map[r] : r;
    const float* xi = x_in + (size_t)src * D;
    float* xo = x_out + (size_t)r * D;
    float4 v[kNormVec];
#pragma unroll
    for (int i = 0; i < kNormVec; ++i) {
        const int c = (i * kNormThreads + tid) * 4;
        v[i] = c < D ? *reinterpret_cast<const float4*>(xi + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (n_splits > 0) {
        float4 p[kNormVec][kMaxNormSplits];
#pragma unroll
        for (int i = 0; i < kNormVec; ++i)
#pragma unroll
            for (int sp = 0; sp < kMaxNormSplits; ++sp) {
                const int c = (i * kNormThreads + tid) * 4;
                p[i][sp] = (c < D && sp < n_splits)
                               ? *reinterpret_cast<const float4*>(part + (size_t)sp * part_stride + (size_t)src * D + c)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
        for (int i = 0; i < kNormVec; ++i)
#pragma unroll
            for (int sp = 0; sp < kMaxNormSplits; ++sp) {
                v[i].x += p[i][sp].x;
                v[i].y += p[i][sp].y;
                v[i].z += p[i][sp].z;
                v[i].w += p[i][sp].w;
            }
    }
    if (n_splits > 0 || xo != xi) {  // in-place normalisation alone leaves x untouched
#pragma unroll
        for (int i = 0; i < kNormVec; ++i) {
            const int c = (i * kNormThreads + tid) * 4;
            if (c < D) *reinterpret_cast<float4*>(xo + c) = v[i];
        }
    }
    if (h_out) rmsnorm_finish_cta<T>(v, D, gamma, eps, h_out + (size_t)r * D, red);
}

template <typename T>
__global__ void __launch_bounds__(kRowThreads) qkv_finalize_kernel(const float* __restrict__ part, int n_splits,
                                                                   size_t part_stride, RowMap rm,
                                                                   const int32_t* __restrict__ prefix_len,
                                                                   int max_prefix, const double* __restrict__ inv_freq,
                                                                   Dims dm, int layer, T* __restrict__ q_out,
                                                                   T* __restrict__ ibc, int* err) {
    pdl_entry();
    extern __shared__ float cs[];  // [d/2] cos, [d/2] sin
    const int r = blockIdx.x;
    if (r >= rm.rows()) return;
    int b, j;
    rm.coords(r, b, j);
    const int d = dm.d, half = d / 2;
    const int P = checked_prefix(prefix_len, b, max_prefix, err);
    const double pos = (double)(P + j);
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
        // angle reduced to [-pi, pi] in double (two-term 2*pi, Cody-Waite), then a float sincos
        const double ang = pos * inv_freq[i];
        const double k = rint(ang * 0.15915494309189535);
        const double red = (ang - k * 6.283185307179586) - k * 2.4492935982947064e-16;
        float sn, cn;
        sincosf((float)red, &sn, &cn);
        cs[i] = cn;
        cs[half + i] = sn;
    }
    __syncthreads();
    const int B = rm.block;
    const float* pr = part + (size_t)r * dm.qkv;
    auto col = [&](int c) {
        float v = pr[c];
        for (int s = 1; s < n_splits; ++s) v += pr[(size_t)s * part_stride + c];
        return v;
    };
    // rotated heads: Hq query heads then Hkv key heads, one (i, i + d/2) pair per item
    const int n_rot = (dm.Hq + dm.Hkv) * half;
    for (int it = threadIdx.x; it < n_rot; it += blockDim.x) {
        const int head = it / half, i = it - head * half;
        const int c0 = head * d + i;
        const float a = col(c0), bb = col(c0 + half);
        const float cn = cs[i], sn = cs[half + i];
        const float lo = a * cn - bb * sn, hi = bb * cn + a * sn;
        if (head < dm.Hq) {
            T* qr = q_out + (size_t)r * dm.Hq * d + head * d;
            qr[i] = from_f<T>(lo);
            qr[i + half] = from_f<T>(hi);
        } else {
            const int g = head - dm.Hq;
            T* kr = ibc + ((((size_t)b * dm.L + layer) * 2 + 0) * dm.Hkv + g) * B * d + (size_t)j * d;
            kr[i] = from_f<T>(lo);
            kr[i + half] = from_f<T>(hi);
        }
    }
    const int n_v = dm.Hkv * d;
    for (int it = threadIdx.x; it < n_v; it += blockDim.x) {
        const int g = it / d, i = it - g * d;
        T* vr = ibc + ((((size_t)b * dm.L + layer) * 2 + 1) * dm.Hkv + g) * B * d + (size_t)j * d;
        vr[i] = from_f<T>(col((dm.Hq + dm.Hkv) * d + it));
    }
}

}  // namespace

template <typename T>
int launch_embed_norm(const int32_t* tokens, int rows, int V, const T* embed, const T* gamma, float eps, int D,
                       float* x, T* h, int* err, cudaStream_t s) {
    if (rows <= 0) return 0;
    return launched(launch_pdl(embed_norm_kernel<T>, dim3(rows), dim3(kNormThreads), 0, s, 0, tokens, V, embed, gamma,
                               eps, D, x, h, err));
}

template <typename T>
int launch_residual_norm(const float* x_in, const int32_t* src_map, const int32_t* n_rows_dev, int rows_bound,
                          const float* part, int n_splits, size_t part_stride, float* x_out, const T* gamma,
                          float eps, int D, T* h_out, cudaStream_t s) {
    if (rows_bound <= 0) return 0;
    return launched(launch_pdl(residual_norm_kernel<T>, dim3(rows_bound), dim3(kNormThreads), 0, s, 0, x_in, src_map,
                               n_rows_dev, part, n_splits, part_stride, x_out, gamma, eps, D, h_out));
}

template <typename T>
int launch_qkv_finalize(const float* part, int n_splits, size_t part_stride, RowMap rm, const int32_t* prefix_len,
                         int max_prefix, const double* inv_freq, Dims dm, int layer, T* q_out, T* ibc, int* err,
                         cudaStream_t s) {
    if (rm.rows_static <= 0) return 0;
    return launched(launch_pdl(qkv_finalize_kernel<T>, dim3(rm.rows_static), dim3(kRowThreads), dm.d * sizeof(float), s,
                               0, part, n_splits, part_stride, rm, prefix_len, max_prefix, inv_freq, dm, layer, q_out,
                               ibc, err));
}

bool configure_rows_kernels() {
    return max_shared_carveout((const void*)embed_norm_kernel<float>) &&
           max_shared_carveout((const void*)embed_norm_kernel<bf16>) &&
           max_shared_carveout((const void*)residual_norm_kernel<float>) &&
           max_shared_carveout((const void*)residual_norm_kernel<bf16>) &&
           max_shared_carveout((const void*)qkv_finalize_kernel<float>) &&
           max_shared_carveout((const void*)qkv_finalize_kernel<bf16>);
}

#define FOCUS_INST_ROWS(T)                                                                                         \
    template int launch_embed_norm<T>(const int32_t*, int, int, const T*, const T*, float, int, float*, T*, int*, \
                                       cudaStream_t);                                                              \
    template int launch_residual_norm<T>(const float*, const int32_t*, const int32_t*, int, const float*, int,    \
                                          size_t, float*, const T*, float, int, T*, cudaStream_t);                 \
    template int launch_qkv_finalize<T>(const float*, int, size_t, RowMap, const int32_t*, int, const double*,    \
                                         Dims, int, T*, T*, int*, cudaStream_t);
FOCUS_INST_ROWS(float)
FOCUS_INST_ROWS(bf16)

}  // namespace focus
