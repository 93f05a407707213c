// CUDA-core GEMM C = A B^T (A [M, K], B [N, K], both row-major) with the step's fused epilogues.
// This is the float32 path (the tiny fp32 model); bf16 GEMMs run on the tcgen05 kernel.
//   EPI_PARTIAL: split-K slice z writes its float32 partial sums to part[z][m][n];
//   EPI_SWIGLU:  computes A Bg^T and A Bu^T together and writes silu(g) * u;
//   EPI_LMHEAD:  per row and 64-column vocabulary tile: max logit, sum exp(z - max), first argmax.
// 64x64 tiles, 256 threads, 4x4 outputs per thread, K staged 16 at a time through shared memory.
#include <math_constants.h>

#include "launch.h"

namespace focus {

namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <typename T, int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs g) {
    pdl_entry();
    __shared__ float As[TK][TM + 4];
    __shared__ float Bs[TK][TN + 4];
    __shared__ float Bs2[EPI == EPI_SWIGLU ? TK : 1][TN + 4];
    const int M = g.M_dev ? *g.M_dev : g.M_bound;
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
    if (m0 >= M) return;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int K = g.K, N = g.N;
    int kchunk = (K + g.splits - 1) / g.splits;
    kchunk = (kchunk + TK - 1) / TK * TK;
    const int k0 = blockIdx.z * kchunk, k1 = min(K, k0 + kchunk);
    const T* A = reinterpret_cast<const T*>(g.A);
    const T* Bm = reinterpret_cast<const T*>(g.B);
    const T* Bu = reinterpret_cast<const T*>(g.B2);
    float acc[4][4] = {}, acc2[4][4] = {};
    const int lr = tid >> 2, lk = (tid & 3) * 4;
    for (int kk = k0; kk < k1; kk += TK) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int k = kk + lk + u;
            const int am = m0 + lr, bn = n0 + lr;
            As[lk + u][lr] = (am < M && k < k1) ? to_f(A[(size_t)am * K + k]) : 0.f;
            Bs[lk + u][lr] = (bn < N && k < k1) ? to_f(Bm[(size_t)bn * K + k]) : 0.f;
            if (EPI == EPI_SWIGLU) Bs2[lk + u][lr] = (bn < N && k < k1) ? to_f(Bu[(size_t)bn * K + k]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < TK; ++k) {
            float av[4], bv[4], bv2[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) av[i] = As[k][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                bv[j] = Bs[k][tx * 4 + j];
                if (EPI == EPI_SWIGLU) bv2[j] = Bs2[k][tx * 4 + j];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[i][j] += av[i] * bv[j];
                    if (EPI == EPI_SWIGLU) acc2[i][j] += av[i] * bv2[j];
                }
        }
        __syncthreads();
    }
    if (EPI == EPI_PARTIAL) {
        float* out = g.part + (size_t)blockIdx.z * g.split_stride;
        for (int i = 0; i < 4; ++i) {
            const int m = m0 + ty * 4 + i;
            if (m >= M) continue;
            for (int j = 0; j < 4; ++j) {
                const int n = n0 + tx * 4 + j;
                if (n < N) out[(size_t)m * N + n] = acc[i][j];
            }
        }
    } else if (EPI == EPI_SWIGLU) {
        T* out = reinterpret_cast<T*>(g.act);
        for (int i = 0; i < 4; ++i) {
            const int m = m0 + ty * 4 + i;
            if (m >= M) continue;
            for (int j = 0; j < 4; ++j) {
                const int n = n0 + tx * 4 + j;
                const float x = acc[i][j];
                if (n < N) out[(size_t)m * N + n] = from_f<T>(x / (1.f + expf(-x)) * acc2[i][j]);
            }
        }
    } else {
        // 16 threads (tx) share a row: half a warp, reduce with xor shuffles of width 16
        for (int i = 0; i < 4; ++i) {
            const int m = m0 + ty * 4 + i;
            float mx = -CUDART_INF_F;
            int arg = 0x7fffffff;
            for (int j = 0; j < 4; ++j) {
                const int n = n0 + tx * 4 + j;
                if (n < N && acc[i][j] > mx) {
                    mx = acc[i][j];
                    arg = n;
                }
            }
            for (int o = 8; o > 0; o >>= 1) {
                const float m2 = __shfl_xor_sync(0xffffffffu, mx, o, 16);
                const int a2 = __shfl_xor_sync(0xffffffffu, arg, o, 16);
                if (m2 > mx || (m2 == mx && a2 < arg)) {
                    mx = m2;
                    arg = a2;
                }
            }
            float se = 0.f;
            for (int j = 0; j < 4; ++j) {
                const int n = n0 + tx * 4 + j;
                if (n < N) se += expf(acc[i][j] - mx);
            }
            for (int o = 8; o > 0; o >>= 1) se += __shfl_xor_sync(0xffffffffu, se, o, 16);
            if (tx == 0 && m < M) {
                const size_t idx = (size_t)m * g.n_tiles + blockIdx.x;
                g.lm_max[idx] = mx;
                g.lm_sum[idx] = se;
                g.lm_arg[idx] = arg;
            }
        }
    }
}

}  // namespace

bool configure_simt_gemm_kernels() {
    return max_shared_carveout((const void*)gemm_simt_kernel<float, EPI_PARTIAL>) &&
           max_shared_carveout((const void*)gemm_simt_kernel<float, EPI_SWIGLU>) &&
           max_shared_carveout((const void*)gemm_simt_kernel<float, EPI_LMHEAD>) &&
           max_shared_carveout((const void*)gemm_simt_kernel<bf16, EPI_PARTIAL>) &&
           max_shared_carveout((const void*)gemm_simt_kernel<bf16, EPI_SWIGLU>) &&
           max_shared_carveout((const void*)gemm_simt_kernel<bf16, EPI_LMHEAD>);
}

template <typename T>
int launch_gemm_simt(Epi epi, const GemmArgs& g, cudaStream_t s) {
    if (g.M_bound <= 0) return 0;
    dim3 grid((g.N + TN - 1) / TN, (g.M_bound + TM - 1) / TM, epi == EPI_PARTIAL ? g.splits : 1);
    GemmArgs a = g;
    if (epi != EPI_PARTIAL) a.splits = 1;
    switch (epi) {
        case EPI_PARTIAL: return launched(launch_pdl(gemm_simt_kernel<T, EPI_PARTIAL>, grid, dim3(256), 0, s, 0, a));
        case EPI_SWIGLU: return launched(launch_pdl(gemm_simt_kernel<T, EPI_SWIGLU>, grid, dim3(256), 0, s, 0, a));
        case EPI_LMHEAD: return launched(launch_pdl(gemm_simt_kernel<T, EPI_LMHEAD>, grid, dim3(256), 0, s, 0, a));
        default: return -1;
    }
}

template int launch_gemm_simt<float>(Epi, const GemmArgs&, cudaStream_t);
template int launch_gemm_simt<bf16>(Epi, const GemmArgs&, cudaStream_t);

}  // namespace focus
