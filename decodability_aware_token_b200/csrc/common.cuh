// Shared device helpers of the FOCUS step kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/focus.h"

namespace focus {

using bf16 = __nv_bfloat16;

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ void raise_err(int* err, int bit) { atomicOr(err, bit); }

// Programmatic dependent launch: every kernel of the step is launched so that it may start while its
// predecessor drains.  On entry it lets its own successor launch (pdl_trigger), then waits until the
// predecessor has completed and its memory is visible (pdl_wait).  Before that wait a kernel touches
// nothing that an earlier kernel of the step writes: only inputs that no kernel of the step writes (the
// model weights; the prefix lengths, page table and prefix pages of the KV pool) may be read there.  The
// step's first kernel triggers only after its own wait, so nothing queued before the step is still
// running when any later kernel of the step starts.  (Without a programmatic launch both are no-ops.)
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_entry() {
    pdl_trigger();
    pdl_wait();
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Block-wide sum for blockDim.x a multiple of 32 (<= 1024); `red` holds >= 32 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = 0.f;
    for (int i = 0; i < nw; ++i) t += red[i];  // fixed order: deterministic
    return t;
}

template <typename T> __device__ __forceinline__ void store4(T* p, float a, float b, float c, float d);
template <> __device__ __forceinline__ void store4<float>(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
template <> __device__ __forceinline__ void store4<bf16>(bf16* p, float a, float b, float c, float d) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&lo);
    u.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p) = u;
}
template <typename T> __device__ __forceinline__ float4 load4(const T* p);
template <> __device__ __forceinline__ float4 load4<float>(const float* p) { return *reinterpret_cast<const float4*>(p); }
template <> __device__ __forceinline__ float4 load4<bf16>(const bf16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// RMSNorm of one float32 row by one CTA of kNormThreads threads.  Thread t holds the row's float4
// number i * kNormThreads + t in v[i] (i < kNormVec, D % 4 == 0, D <= 4 * kNormThreads * kNormVec);
// the gamma loads are issued before the reduction so that the row costs two memory round trips.
// h = x / sqrt(mean(x^2) + eps) * gamma.  Every kernel that normalises a residual row goes through
// this routine, so all of them produce bit-identical results.  Contains __syncthreads().
constexpr int kNormThreads = 256;
constexpr int kNormVec = 4;  // D <= 4096
template <typename T>
__device__ __forceinline__ void rmsnorm_finish_cta(const float4 (&v)[kNormVec], int D, const T* gamma, float eps,
                                                   T* hr, float* red) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float4 g[kNormVec];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kNormVec; ++i) {
        const int c = (i * kNormThreads + tid) * 4;
        g[i] = c < D ? load4<T>(gamma + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < kNormVec; ++i) {
        const int c = (i * kNormThreads + tid) * 4;
        if (c < D) {
            ss = fmaf(v[i].x, v[i].x, ss);
            ss = fmaf(v[i].y, v[i].y, ss);
            ss = fmaf(v[i].z, v[i].z, ss);
            ss = fmaf(v[i].w, v[i].w, ss);
        }
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kNormThreads / 32; ++w) tot += red[w];  // fixed order: deterministic
    const float inv = rsqrtf(tot / D + eps);
#pragma unroll
    for (int i = 0; i < kNormVec; ++i) {
        const int c = (i * kNormThreads + tid) * 4;
        if (c < D)
            store4<T>(hr + c, __fmul_rn(__fmul_rn(v[i].x, inv), g[i].x), __fmul_rn(__fmul_rn(v[i].y, inv), g[i].y),
                      __fmul_rn(__fmul_rn(v[i].z, inv), g[i].z), __fmul_rn(__fmul_rn(v[i].w, inv), g[i].w));
    }
}

// Where the rows of the current phase come from.
//  full phase:      row r is block position (r / B, r % B)
//  compacted phase: row r is (row_req[r], row_pos[r]); the live row count is *n_rows
struct RowMap {
    const int32_t* row_req;  // nullptr in the full phase
    const int32_t* row_pos;
    const int32_t* n_rows;   // device count (compacted phase) or nullptr
    int32_t rows_static;     // row count of the full phase / upper bound of the compacted phase
    int32_t block;           // B
    __device__ __forceinline__ int rows() const { return n_rows ? *n_rows : rows_static; }
    __device__ __forceinline__ void coords(int r, int& b, int& j) const {
        if (row_req) { b = row_req[r]; j = row_pos[r]; }
        else { b = r / block; j = r - (r / block) * block; }
    }
};

// Clamp a request's prefix length to what its page-table row can address.
__device__ __forceinline__ int checked_prefix(const int32_t* prefix_len, int b, int max_prefix, int* err) {
    int p = prefix_len[b];
    if (p < 0 || p > max_prefix) {
        raise_err(err, FOCUS_DEVERR_PREFIX);
        p = p < 0 ? 0 : max_prefix;
    }
    return p;
}

}  // namespace focus
