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
