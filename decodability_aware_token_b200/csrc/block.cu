// Around the focused step: a block that has been decoded becomes part of the exactly cached prefix
// ("FOCUS: DLLMs Know How to Tame Their Compute Bound", project page, Overview -- Motivation: each
// denoising step runs the block on top of an exactly cached prefix).  The commit copies the block's
// K/V -- the intra-block cache after the block's final dense refresh -- into the request's pages at
// positions P_b .. P_b + B - 1, then grows P_b by B.  Pure data movement: 16-byte vector copies, one CTA
// per (request, layer, K|V, KV head) so that both sides are read and written in contiguous 256-byte
// (bf16, d = 128) rows.
#include "block.h"

#include "common.cuh"

namespace focus {

namespace {

__global__ void __launch_bounds__(256) commit_block_kernel(CommitArgs a) {
    const int b = blockIdx.x;
    const int layer_kv_head = blockIdx.y;  // (l * 2 + kv) * Hkv + h
    int P = a.prefix_len[b];
    if (P < 0 || P > a.max_pages * a.S) {  // the step would have clamped it: nothing sensible to commit
        if (threadIdx.x == 0) raise_err(a.err, FOCUS_DEVERR_PREFIX);
        return;
    }
    const int row_bytes = a.d * a.elt;  // 128 .. 512, a multiple of 16
    const int vec = row_bytes / 16;
    const size_t src_base = (((size_t)b * a.L * 2 * a.Hkv) + layer_kv_head) * a.B;  // rows of the cache
    for (int t = threadIdx.x; t < a.B * vec; t += blockDim.x) {
        const int j = t / vec, c = t - j * vec;
        const int pos = P + j;
        const int slot = pos / a.S;
        const int page = slot < a.max_pages ? a.page_table[(size_t)b * a.max_pages + slot] : -1;
        if (page < 0 || page >= a.n_pages) {
            if (c == 0) raise_err(a.err, FOCUS_DEVERR_PAGE_ID);  // no page for this block position
            continue;
        }
        const size_t dst_row = ((size_t)page * a.L * 2 * a.Hkv + layer_kv_head) * a.S + (pos - slot * a.S);
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const char*>(a.ibc) + (src_base + j) * row_bytes);
        uint4* dst = reinterpret_cast<uint4*>(static_cast<char*>(a.kv_pool) + dst_row * row_bytes);
        dst[c] = src[c];
    }
}

// After every copy of the launch above has read the old prefix length.
__global__ void advance_prefix_kernel(int32_t* prefix_len, int N, int B, int limit) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < N) {
        const int P = prefix_len[b];
        if (P >= 0 && P <= limit) prefix_len[b] = P + B;
    }
}

__global__ void __launch_bounds__(256) count_masked_kernel(const uint8_t* mask, int n, int32_t* out) {
    __shared__ float red[32];
    float c = 0.f;  // exact: counts stay far below 2^24
    for (int i = threadIdx.x; i < n; i += blockDim.x) c += mask[i] != 0 ? 1.f : 0.f;
    const float tot = block_sum(c, red);
    if (threadIdx.x == 0) *out = (int32_t)tot;
}

}  // namespace

int launch_commit_block(const CommitArgs& a, cudaStream_t s) {
    if (a.N <= 0 || a.B <= 0) return 0;
    commit_block_kernel<<<dim3(a.N, a.L * 2 * a.Hkv), 256, 0, s>>>(a);
    advance_prefix_kernel<<<(a.N + 255) / 256, 256, 0, s>>>(a.prefix_len, a.N, a.B, a.max_pages * a.S);
    return cudaGetLastError() == cudaSuccess ? 2 : -1;
}

int launch_count_masked(const uint8_t* mask, int n, int32_t* out, cudaStream_t s) {
    count_masked_kernel<<<1, 256, 0, s>>>(mask, n, out);
    return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace focus
