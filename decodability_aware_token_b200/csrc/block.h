// Kernels around the focused step: committing a decoded block's K/V into the prefix pages, and the
// masked-position count the block loop polls.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace focus {

struct CommitArgs {
    const void* ibc;            // [N, L, 2, Hkv, B, d] T
    void* kv_pool;              // [n_pages, L, 2, Hkv, S, d] T
    int32_t* prefix_len;        // [N], grown by B
    const int32_t* page_table;  // [N, max_pages]
    int N, L, Hkv, B, d, S, max_pages, n_pages, elt;
    int* err;
};
// Enqueue the copy and the prefix update (two launches); returns the launch count or -1.
int launch_commit_block(const CommitArgs& a, cudaStream_t s);
// Number of nonzero bytes in mask[0 .. n) into *out (one launch).
int launch_count_masked(const uint8_t* mask, int n, int32_t* out, cudaStream_t s);
// One CTA whose bounded pipeline wait is never satisfied: sets FOCUS_DEVERR_TIMEOUT in *err after about a
// second and returns (probe.cu); returns the launch count or -1.
int launch_wait_timeout_probe(int* err, cudaStream_t s);

}  // namespace focus
