// LM-head confidence of caller-supplied hidden rows, with no memory allocation at all.
//
// Who needs this: code that is not allowed to call the CUDA allocator -- for example a host thread that
// is recording a CUDA graph (cudaMalloc is not a stream operation and cannot be captured), a real-time
// serving loop with a fixed memory budget that must never block on or fail in the allocator, or a
// plug-in running inside another framework whose caching allocator owns all device memory.  Such
// callers can still run the final stage of the step (final RMSNorm, LM head, max-softmax confidence
// and top id) on hidden rows they hold, passing only their own input and output buffers.
//
// The intermediate data (normalised bf16 rows and per-vocabulary-tile statistics) lives in one
// file-scope __device__ array of fixed size, so every GPU that loads this library holds it from load
// until process exit.  All calls on a device share that array: calls that may overlap on the GPU (on
// different streams, or from different threads without ordering) race on it and must be serialised by
// the caller.  Nothing in the array needs to survive from one call to the next; the one word that must
// start at zero (the bounded-wait flag) is cleared at the start of every call.
#include <mutex>

#include "tc_gemm_kernel.cuh"

namespace focus {

namespace {

using namespace tc;

// maximum sizes served by the fixed scratch array
constexpr int kNaRows = 256;                    // hidden rows per call
constexpr int kNaDim = 4096;                    // hidden size (a multiple of 128)
constexpr int kNaVocab = 163840;                // vocabulary size
constexpr int kNaBN = 128;                      // vocabulary columns per statistics tile
constexpr int kNaTiles = kNaVocab / kNaBN;      // 1280 tiles
constexpr size_t kNaNormBytes = (size_t)kNaRows * kNaDim * 2;   // normalised bf16 rows: 2 MiB
constexpr size_t kNaStatBytes = (size_t)kNaRows * kNaTiles * 4; // one statistic per row and tile: 1.25 MiB
constexpr size_t kNaBytes = kNaNormBytes + 3 * kNaStatBytes + 256;  // + the bounded-wait flag: ~5.75 MiB

static __device__ __align__(256) unsigned char g_lm_conf_scratch[kNaBytes];

using NaShape = TcShape<kNaBN, 2, 4>;

// RMSNorm of float32 rows into bf16, one CTA per row, with the very routine the step's own norm
// kernels use, so both paths produce bit-identical normalised rows.
__global__ void __launch_bounds__(kNormThreads) na_norm_kernel(const float* __restrict__ x, int D,
                                                               const bf16* __restrict__ gamma, float eps,
                                                               bf16* __restrict__ h) {
    __shared__ float red[32];
    const int r = blockIdx.x, tid = threadIdx.x;
    float4 v[kNormVec];
#pragma unroll
    for (int i = 0; i < kNormVec; ++i) {
        const int c = (i * kNormThreads + tid) * 4;
        v[i] = c < D ? *reinterpret_cast<const float4*>(x + (size_t)r * D + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    rmsnorm_finish_cta<bf16>(v, D, gamma, eps, h + (size_t)r * D, red);
}

__device__ __forceinline__ void na_merge(float& m, float& s, int& a, float m2, float s2, int a2) {
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

// One warp per row: merge the vocabulary tiles into conf = 1 / sum exp(z - max) and the top id.
__global__ void __launch_bounds__(256) na_combine_kernel(const float* __restrict__ mx, const float* __restrict__ se,
                                                         const int* __restrict__ arg, int n_tiles, int rows,
                                                         const int* flag, float* conf, int32_t* top) {
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (r >= rows) return;
    float m = -CUDART_INF_F, s = 0.f;
    int a = 0x7fffffff;
    for (int t = lane; t < n_tiles; t += 32)
        na_merge(m, s, a, mx[(size_t)r * n_tiles + t], se[(size_t)r * n_tiles + t], arg[(size_t)r * n_tiles + t]);
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
        const int a2 = __shfl_xor_sync(0xffffffffu, a, o);
        na_merge(m, s, a, m2, s2, a2);
    }
    if (lane == 0) {
        const bool bad = *flag != 0;  // a bounded wait in the GEMM expired: the statistics are not valid
        conf[r] = bad ? CUDART_NAN_F : 1.f / s;
        top[r] = bad ? -1 : a;
    }
}

// Device address of the scratch array, looked up once per device (with that device current).
std::mutex g_na_mu;
constexpr int kNaMaxDevices = 64;
void* g_na_base[kNaMaxDevices] = {};

int na_setup(int dev, void** base) {
    if (dev < 0 || dev >= kNaMaxDevices) return FOCUS_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_na_mu);
    if (!g_na_base[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_lm_conf_scratch) != cudaSuccess || !p) return FOCUS_ERR_CUDA;
        if (cudaFuncSetAttribute(tc_gemm_kernel<kNaBN, 2, 4, EPI_LMHEAD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 NaShape::SMEM) != cudaSuccess ||
            !max_shared_carveout((const void*)tc_gemm_kernel<kNaBN, 2, 4, EPI_LMHEAD>) ||
            !max_shared_carveout((const void*)na_norm_kernel) || !max_shared_carveout((const void*)na_combine_kernel))
            return FOCUS_ERR_CUDA;
        g_na_base[dev] = p;
    }
    *base = g_na_base[dev];
    return FOCUS_OK;
}

}  // namespace

}  // namespace focus

using namespace focus;

extern "C" int focus_lm_head_conf_noalloc(const float* hidden, int32_t rows, int32_t hidden_dim,
                                          const void* final_norm, const void* lm_head, int32_t vocab, float rms_eps,
                                          float* conf, int32_t* top_id, void* stream) {
    if (!hidden || !final_norm || !lm_head || !conf || !top_id || rows < 0 || hidden_dim <= 0 || vocab <= 0 ||
        !(rms_eps >= 0.f))
        return FOCUS_ERR_INVALID_ARG;
    // the kernels read hidden rows as float4, final_norm four bf16 at a time, and lm_head through a TMA tensor
    // map (16-byte base); outputs are written per element
    if (reinterpret_cast<uintptr_t>(hidden) % 16 || reinterpret_cast<uintptr_t>(final_norm) % 8 ||
        reinterpret_cast<uintptr_t>(lm_head) % 16 || reinterpret_cast<uintptr_t>(conf) % 4 ||
        reinterpret_cast<uintptr_t>(top_id) % 4)
        return FOCUS_ERR_INVALID_ARG;
    if (rows > kNaRows || hidden_dim > kNaDim || vocab > kNaVocab) return FOCUS_ERR_LIMITS;
    if (hidden_dim % 128) return FOCUS_ERR_UNSUPPORTED;
    if (rows == 0) return FOCUS_OK;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return FOCUS_ERR_CUDA;
    void* base = nullptr;
    const int rc = na_setup(dev, &base);
    if (rc != FOCUS_OK) return rc;
    unsigned char* b = static_cast<unsigned char*>(base);
    bf16* h = reinterpret_cast<bf16*>(b);
    float* mx = reinterpret_cast<float*>(b + kNaNormBytes);
    float* se = reinterpret_cast<float*>(b + kNaNormBytes + kNaStatBytes);
    int* arg = reinterpret_cast<int*>(b + kNaNormBytes + 2 * kNaStatBytes);
    int* flag = reinterpret_cast<int*>(b + kNaNormBytes + 3 * kNaStatBytes);
    // tensor maps are host-side descriptors: building them allocates nothing on the device
    CUtensorMap map_a, map_b;
    if (!make_map(&map_a, h, kNaRows, (uint64_t)hidden_dim, NaShape::BM) ||
        !make_map(&map_b, lm_head, (uint64_t)vocab, (uint64_t)hidden_dim, kNaBN))
        return FOCUS_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(flag, 0, sizeof(int), s) != cudaSuccess) return FOCUS_ERR_CUDA;
    na_norm_kernel<<<rows, kNormThreads, 0, s>>>(hidden, hidden_dim, static_cast<const bf16*>(final_norm), rms_eps, h);
    GemmArgs g{};
    g.A = h;
    g.B = lm_head;
    g.M_bound = rows;
    g.M_dev = nullptr;
    g.N = vocab;
    g.K = hidden_dim;
    g.splits = 1;
    g.lm_max = mx;
    g.lm_sum = se;
    g.lm_arg = arg;
    g.n_tiles = (vocab + kNaBN - 1) / kNaBN;
    g.tile_n = kNaBN;
    tc_gemm_kernel<kNaBN, 2, 4, EPI_LMHEAD><<<dim3(g.n_tiles, 1, 1), 192, NaShape::SMEM, s>>>(map_a, map_b, map_b, g,
                                                                                          flag);
    na_combine_kernel<<<(rows + 7) / 8, 256, 0, s>>>(mx, se, arg, g.n_tiles, rows, flag, conf, top_id);
    return cudaGetLastError() == cudaSuccess ? FOCUS_OK : FOCUS_ERR_CUDA;
}
