// bf16 attention of block queries over paged prefix KV plus the intra-block KV cache on the 5th-generation
// tensor cores (tcgen05.mma with S and O accumulators in TMEM), with the importance column sums fused in
// for layers 0 and 1.  Used for launches whose (request, KV head) units hold more than 32 query vectors --
// many kept rows, or four query heads per KV head -- where the legacy mma.sync kernel (attention_tc.cu)
// runs out of tensor throughput before it runs out of memory bandwidth.
//
// "FOCUS: DLLMs Know How to Tame Their Compute Bound", project page, Overview -- Design / Decodability
// Signal (importance from the early layers' Q/K attention) and Runtime Action (ragged execution and the
// intra-block KV cache); news article on the same paper, "Arquitetura do FOCUS" (ragged paged attention).
//
// Work unit (one CTA): request b, KV head g and a tile of up to QT = 128 (or 64) query vectors of that group
// (query vector qi = row * G + head-in-group; the MMAs have M = 128).  Keys are walked in 64-key chunks:
// the prefix pages in order, then the B block keys from the intra-block cache as the last chunk (the same
// TMA chunk loads as the mma.sync kernel).  Per chunk i:
//   S_i = Q K_i^T         tcgen05.mma M = 128, N = 64, K = 128 (both operands K-major), into one of two
//                         64-column TMEM buffers, issued before the softmax of chunk i - 1 has finished;
//   softmax (8 warps, two threads per query vector): S_i from TMEM, masked and scaled to base 2, online
//                         max / denominator; P_i = 2^(s - m) rounded to bf16 into shared memory (two
//                         buffers: chunk i's P waits only for P_{i-2} V_{i-2}, so the softmax of one chunk
//                         overlaps the P V of the one before; only a raise of the running max waits for
//                         P_{i-1} V_{i-1}, which O must have absorbed before it is rescaled);
//   O += P_i V_i          tcgen05.mma M = 128, N = 128, K = 64, V taken MN-major straight from the page
//                         tile, into a 128-column TMEM accumulator.
// The running max m is raised only when a chunk exceeds it by more than 8 (a factor of 256 in the
// weights); O and the denominator are then rescaled in TMEM.  Between raises, weights up to 2^8 are
// summed exactly as the plain online softmax would sum them after its rescale, so the result is the same
// softmax.  Warp roles: one lane issues the TMA copies, the MMA warp owns TMEM and one of its lanes issues
// the MMAs, the softmax warps run the softmax and the output, two threads per query vector (one per half of
// the keys of a chunk and of the output columns).
//
// Importance: the block chunk's scaled scores stay in registers until the final m and denominator are
// known; the probabilities of the block keys are then summed over the tile's query vectors per key in
// fixed order (through shared memory) into imp_part[b][g][tile][j]; the selection kernel adds those in order.
//
// Every mbarrier wait is bounded; on expiry the role flags FOCUS_DEVERR_TIMEOUT and stops, the producer
// waits (bounded) for its own copies, the MMA thread for its own MMAs, and TMEM is released after both.
#include <math_constants.h>

#include "attention_pages.cuh"

namespace focus {

namespace {

using tc::idesc_bf16;
using tc::mbar_arrive;
using tc::mma_bf16;
using tc::mma_commit;
using tc::smem_desc_sw128;
using tc::smem_u32;
using tc::tc_fence_after;
using tc::tc_fence_before;
using tc::tmem_ld32;

// Two shapes of the kernel, by query tile height QT:
//   QT = 128: one CTA per SM (193 KB of shared memory), four K/V stages, eight softmax warps (two threads per
//             query vector); warp 0 issues the copies, warp 1 the MMAs.
//   QT = 64:  units of at most 64 query vectors (a few kept rows per request), two CTAs per SM (97 KB each),
//             two K/V stages each, four softmax warps; warp 2 issues the copies, warp 3 the MMAs, so that the
//             softmax warps 0, 1, 4, 5 sit on TMEM lane quarters 0 and 1, where the tile's rows are.  Each SM
//             then runs two independent chunk chains (S, softmax, P V), which hides the latency of one chain.
//             The MMAs keep M = 128: rows 64..127 of the A operands read the next 8 KB of shared memory (the
//             other Q half, the next P buffer, the first stage), land in TMEM lanes 64..127 and are never read.
template <int QT> struct T5;
template <> struct T5<128> {
    static constexpr int kStages = 4, kSoftWarps = 8, kTmaWarp = 0, kMmaWarp = 1, kMinBlocks = 1;
};
template <> struct T5<64> {
    static constexpr int kStages = 2, kSoftWarps = 4, kTmaWarp = 2, kMmaWarp = 3, kMinBlocks = 2;
};
template <int QT> constexpr int t5_threads() { return 64 + 32 * T5<QT>::kSoftWarps; }
template <int QT> constexpr int t5_qhalf() { return QT * 128; }  // [QT q][64 d] bf16
template <int QT> constexpr int t5_pbytes() { return QT * 128; }  // [QT q][64 keys] bf16
// Q halves, P, then the K/V ring (all 1024-byte aligned); the M = 128 operand reads of the QT = 64 shape stay
// inside this allocation
template <int QT> constexpr int t5_smem() {
    return 2 * t5_qhalf<QT>() + 2 * t5_pbytes<QT>() + T5<QT>::kStages * kStageBytes + 1024;
}
static_assert(t5_smem<128>() == 193 * 1024 && t5_smem<64>() == 97 * 1024, "shared memory per CTA");
constexpr uint32_t kT5TmemCols = 256;             // S (two 64-column buffers) + O (128 columns)
constexpr uint32_t kT5OCol = 128;                 // first TMEM column of O
constexpr float kT5Raise = 8.f;                   // base-2 headroom before the running max is raised

// The softmax warps' own barrier (named barrier 1, all of their threads).
template <int N> __device__ __forceinline__ void named_sync_softmax() { asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory"); }

// 3-D TMA load (q rows: d, head, row).
__device__ __forceinline__ void tma_load_3d(const CUtensorMap* map, uint64_t* bar, void* dst, int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes, written back.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    uint32_t r[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i]);
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory descriptor of an MN-major operand written by TMA with the 128-byte swizzle: 64 elements of
// the MN dimension per 128-byte row, consecutive K indices on consecutive rows; the next 64 MN elements
// `lbo` bytes on, the next 8 K rows 1024 bytes on.
__device__ __forceinline__ uint64_t smem_desc_sw128_mn(uint32_t addr, uint32_t lbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);        // start address
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;   // leading byte offset: next 64 MN elements
    d |= (uint64_t)(1024 >> 4) << 32;             // stride byte offset: next 8 K rows
    d |= (uint64_t)1 << 46;                       // descriptor version for tcgen05
    d |= (uint64_t)2 << 61;                       // 128-byte swizzle
    return d;
}

template <bool FULL, int QT>
__global__ void __launch_bounds__(t5_threads<QT>(), T5<QT>::kMinBlocks) attention_t5_kernel(const __grid_constant__ CUtensorMap pool_map,
                                                              const __grid_constant__ CUtensorMap ibc_map,
                                                              const __grid_constant__ CUtensorMap q_map, AttnArgs a,
                                                              int q_tiles) {
    constexpr int kStages = T5<QT>::kStages, kSoftWarps = T5<QT>::kSoftWarps, kQHalf = t5_qhalf<QT>();
    pdl_trigger();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* q_s = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* p_s = q_s + 2 * kQHalf;
    uint8_t* kv_s = p_s + 2 * t5_pbytes<QT>();  // P buffers 0 and 1, then the K/V ring
    __shared__ __align__(8) uint64_t q_full;
    __shared__ __align__(8) uint64_t kv_full[kStages];
    __shared__ __align__(8) uint64_t kv_empty[kStages];
    __shared__ __align__(8) uint64_t s_full[2];
    __shared__ __align__(8) uint64_t s_free[2];
    __shared__ __align__(8) uint64_t p_full[2];
    __shared__ __align__(8) uint64_t pv_bar[2];  // P_j V_j complete, j even / odd
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint64_t valid_s[kStages];
    __shared__ int32_t pt_s[kPtCache];
    __shared__ float xm_s[2][2][QT];   // per chunk parity and column half: the half-row maxima
    __shared__ float lx_s[2][QT];      // per column half: the row's partial denominators
    __shared__ uint32_t tmem_slot;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.Hq / a.Hkv;
    Unit u{};
    // grid (query tiles, KV heads, request slots): the query tiles of one unit run side by side (the walks
    // after the first find the unit's pages in L2), and the CTAs of one request are adjacent.  With a
    // request order (kept-row launches: longest prefix first, written by the row-map kernel earlier in
    // the step) slot z walks request order[z], so the longest walks start first and the launch's tail is
    // made of the shortest ones; the order is read after the programmatic-launch wait.
    u.qt = blockIdx.x;
    u.g = blockIdx.y;

    if (threadIdx.x == 0) {
        mbar_init(&q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], kSoftWarps);  // one arrival per softmax warp
            mbar_init(&p_full[b], kSoftWarps);
        }
        mbar_init(&pv_bar[0], 1);
        mbar_init(&pv_bar[1], 1);
        mbar_init(&done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == T5<QT>::kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                     "r"(kT5TmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    pdl_wait();

    u.b = a.order ? a.order[blockIdx.z] : (int)blockIdx.z;
    u.P = checked_prefix(a.prefix_len, u.b, a.max_pages * a.page_size, a.err);
    u.q0 = u.qt * QT;
    const int n_prefix_chunks = (u.P + kChunk - 1) / kChunk;
    const int n_chunks = n_prefix_chunks + 1;
    const int unit = (u.b * a.Hkv + u.g) * q_tiles + u.qt;
    const bool pt_cached = a.max_pages <= kPtCache;
    for (int i = threadIdx.x; pt_cached && i < a.max_pages; i += blockDim.x)
        pt_s[i] = a.page_table[(size_t)u.b * a.max_pages + i];
    const int32_t* pt = pt_cached ? pt_s : a.page_table + (size_t)u.b * a.max_pages;
    __syncthreads();  // the cached page-table row

    if (FULL) {
        u.row_base = u.b * a.B;
        u.n_rows = a.B;
    } else {
        u.row_base = a.row_offsets[u.b];
        u.n_rows = a.row_offsets[u.b + 1] - u.row_base;
    }
    u.nq = min(QT, u.n_rows * G - u.q0);
    if (u.nq > 0) {
        if (warp == T5<QT>::kTmaWarp) {
            if (lane == 0) {
                // ---- TMA producer: the query tile once, then the key / value chunks through the ring
                asm volatile("prefetch.tensormap [%0];" ::"l"(&q_map) : "memory");
                mbar_expect_tx(&q_full, 2u * kQHalf);
                const int row0 = u.row_base + u.q0 / G;
                tma_load_3d(&q_map, &q_full, q_s, 0, u.g * G, row0);
                tma_load_3d(&q_map, &q_full, q_s + kQHalf, 64, u.g * G, row0);
                int issued = 0;
                for (int i = 0; i < n_chunks; ++i) {
                    const int st = i % kStages;
                    if (!mbar_wait(&kv_empty[st], ((uint32_t)(i / kStages) & 1u) ^ 1u, a.err)) break;
                    valid_s[st] = issue_chunk(a, u, &pool_map, &ibc_map, kv_s + st * kStageBytes, &kv_full[st], i,
                                              n_prefix_chunks, pt);
                    // kept-row units of the two-CTAs-per-SM shape: ask L2 for the next chunk while it waits for
                    // a stage (measured: the full-block units' query tiles walk the same pages side by side,
                    // and the four-stage shape has its chunks in flight already; both lost time to it)
                    if (!FULL && QT == 64) prefetch_chunk_l2(a, u, i + 3, n_prefix_chunks, pt);  // three ahead
                    ++issued;
                }
                // never leave with copies in flight
                mbar_wait(&q_full, 0u, a.err);
                for (int i = issued > kStages ? issued - kStages : 0; i < issued; ++i)
                    mbar_wait(&kv_full[i % kStages], (uint32_t)(i / kStages) & 1u, a.err);
            }
            __syncwarp();
        } else if (warp == T5<QT>::kMmaWarp) {
            if (lane == 0) {
                // ---- MMA issuer: S_i, then P_{i-1} V_{i-1}, so the S of the next chunk overlaps the softmax
                constexpr uint32_t idesc_s = idesc_bf16(128, 64);
                constexpr uint32_t idesc_o = idesc_bf16(128, 128) | (1u << 16);  // B (V) MN-major
                const uint32_t q_addr = smem_u32(q_s);
                bool ok = mbar_wait(&q_full, 0u, a.err);
                auto pv = [&](int j) {
                    const int pb = j & 1, st = j % kStages;
                    if (!mbar_wait(&p_full[pb], (uint32_t)(j >> 1) & 1u, a.err)) return false;
                    tc_fence_after();
                    const uint32_t p_addr = smem_u32(p_s + (j & 1) * t5_pbytes<QT>());
                    const uint32_t v_addr = smem_u32(kv_s + st * kStageBytes + 2 * kHalf);
#pragma unroll
                    for (int kk = 0; kk < kChunk / 16; ++kk)
                        mma_bf16(tmem + kT5OCol, smem_desc_sw128(p_addr + kk * 32),
                                 smem_desc_sw128_mn(v_addr + kk * 2048, kHalf), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&pv_bar[j & 1]);
                    mma_commit(&kv_empty[st]);  // K and V of chunk j have been read
                    return true;
                };
                int i = 0;
                for (; ok && i < n_chunks; ++i) {
                    const int st = i % kStages, sb = i & 1;
                    if (!mbar_wait(&kv_full[st], (uint32_t)(i / kStages) & 1u, a.err) ||
                        !mbar_wait(&s_free[sb], ((uint32_t)(i >> 1) & 1u) ^ 1u, a.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t k_addr = smem_u32(kv_s + st * kStageBytes);
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        const uint32_t off = (uint32_t)((kk >> 2) * kHalf + (kk & 3) * 32);
                        mma_bf16(tmem + (uint32_t)(sb * 64), smem_desc_sw128(q_addr + (uint32_t)((kk >> 2) * kQHalf) +
                                                                             (uint32_t)((kk & 3) * 32)),
                                 smem_desc_sw128(k_addr + off), idesc_s, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&s_full[sb]);
                    if (i >= 1 && !pv(i - 1)) {
                        ok = false;
                        break;
                    }
                }
                if (ok) pv(n_chunks - 1);
                mma_commit(&done_bar);
                mbar_wait(&done_bar, 0u, a.err);
            }
            __syncwarp();
        } else {
            // ---- softmax and output: two threads per query vector (each thread owns one half of the 64 keys
            // of a chunk and one half of the 128 output columns).  A softmax warp reads TMEM lane quarter
            // warp % 4 (the query vectors 32 (warp % 4) .. + 31); its column half is (warp - 2) / 4 for QT = 128
            // (warps 2..9) and warp / 4 for QT = 64 (warps 0, 1, 4, 5).  The two halves of a row exchange their
            // chunk maxima through shared memory behind a named barrier; every softmax warp passes that
            // barrier once per chunk even after one of its waits gave up (it then only skips its
            // tensor-memory work), so no warp is left waiting there.
            const int quarter = warp & 3, half = QT == 128 ? (warp - 2) >> 2 : warp >> 2;
            const int t = quarter * 32 + lane;                   // query vector within the tile
            const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
            const float sl2 = rsqrtf((float)kD) * 1.4426950408889634f;  // 1/sqrt(d) * log2(e)
            float m_used = -CUDART_INF_F, l = 0.f;
            float sb[32];                                        // block chunk: this half's scaled scores
            bool alive = true;
            for (int i = 0; i < n_chunks; ++i) {
                const int st = i % kStages, sbuf = i & 1;
                bool ok = alive && mbar_wait(&s_full[sbuf], (uint32_t)(i >> 1) & 1u, a.err) &&
                          mbar_wait(&kv_full[st], (uint32_t)(i / kStages) & 1u, a.err);  // valid_s is written
                alive = __all_sync(0xffffffffu, ok);
                float s[32];
                float cm = -CUDART_INF_F;
                const uint32_t vm = (uint32_t)(valid_s[st] >> (32 * half));
                if (alive) {
                    tc_fence_after();
                    tmem_ld32(trow + (uint32_t)(sbuf * 64 + half * 32), s);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s_free[sbuf]);
                    if (vm != 0xffffffffu) {
#pragma unroll
                        for (int c = 0; c < 32; ++c) s[c] = ((vm >> c) & 1u) ? s[c] : -CUDART_INF_F;
                    }
#pragma unroll
                    for (int c = 0; c < 32; ++c) cm = fmaxf(cm, s[c]);
                }
                xm_s[sbuf][half][t] = cm == -CUDART_INF_F ? cm : cm * sl2;
                named_sync_softmax<32 * kSoftWarps>();
                const float cmax = fmaxf(xm_s[sbuf][0][t], xm_s[sbuf][1][t]);  // the same value in both halves
                // P buffer i % 2 is free once P_{i-2} V_{i-2} has completed (phase (i - 2) / 2 of its barrier;
                // every earlier phase was waited for, and P_i V_i needs this chunk's P: the barrier is at most
                // one phase past the one asked for, so the parity is unambiguous)
                if (alive && i >= 2)
                    alive = __all_sync(0xffffffffu, mbar_wait(&pv_bar[i & 1], (uint32_t)((i - 2) >> 1) & 1u, a.err));
                if (!alive) continue;
                tc_fence_after();
                // raise the running max only by more than kT5Raise; O and the denominator follow it
                float f = 1.f;
                if (m_used == -CUDART_INF_F) {
                    m_used = cmax;  // no weight has been summed yet: O and l are zero
                } else if (cmax > m_used + kT5Raise) {
                    f = exp2f(m_used - cmax);
                    l *= f;
                    m_used = cmax;
                }
                if (__any_sync(0xffffffffu, f != 1.f)) {  // TMEM access is warp-collective: factor 1 elsewhere
                    // O must hold P_{i-1} V_{i-1} before it is scaled (a raise needs an earlier summed chunk)
                    if (i >= 1 && !__all_sync(0xffffffffu, mbar_wait(&pv_bar[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u,
                                                                     a.err))) {
                        alive = false;
                        continue;
                    }
                    tc_fence_after();
#pragma unroll 1
                    for (int c0 = 0; c0 < kD / 2; c0 += 32) {
                        float v[32];
                        tmem_ld32(trow + kT5OCol + (uint32_t)(half * 64 + c0), v);
#pragma unroll
                        for (int c = 0; c < 32; ++c) v[c] *= f;
                        tmem_st32(trow + kT5OCol + (uint32_t)(half * 64 + c0), v);
                    }
                }
                const float mu = m_used == -CUDART_INF_F ? 0.f : m_used;
                float rs = 0.f;
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float p0 = exp2f(fmaf(s[c], sl2, -mu)), p1 = exp2f(fmaf(s[c + 1], sl2, -mu));
                    rs += p0 + p1;
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                    pk[c / 2] = *reinterpret_cast<uint32_t*>(&b2);
                }
                l += rs;
                if (FULL && i == n_chunks - 1) {
#pragma unroll
                    for (int c = 0; c < 32; ++c) sb[c] = s[c] == -CUDART_INF_F ? s[c] : s[c] * sl2;
                }
                // P row t: 128 bytes, 16-byte chunk cc at (cc ^ (t & 7)) (the 128-byte swizzle); this half writes
                // chunks 4 half .. 4 half + 3
                uint8_t* prow = p_s + (i & 1) * t5_pbytes<QT>() + (t >> 3) * 1024 + (t & 7) * 128;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    *reinterpret_cast<uint4*>(prow + (((4 * half + c) ^ (t & 7)) << 4)) =
                        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                // V rows of keys the copies left unfilled may hold stale bits: P is 0 there, so make V 0 too
                // (QT = 128: the half-0 threads, key t % 64 of V half t / 64; QT = 64: key t of V half `half`)
                if ((QT == 64 || half == 0) && valid_s[st] != ~0ull) {
                    const int r = QT == 128 ? (t & 63) : t, h = QT == 128 ? (t >> 6) : half;
                    if (!((valid_s[st] >> r) & 1ull)) {
                        uint4* vr = reinterpret_cast<uint4*>(kv_s + st * kStageBytes + 2 * kHalf + h * kHalf + r * 128);
#pragma unroll
                        for (int c = 0; c < 8; ++c) vr[c] = make_uint4(0, 0, 0, 0);
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor core
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[sbuf]);
            }
            // the last P V has completed: normalise and write this thread's half of the query vector
            if (alive)
                alive = __all_sync(0xffffffffu, mbar_wait(&pv_bar[(n_chunks - 1) & 1], (uint32_t)((n_chunks - 1) >> 1) & 1u,
                                                          a.err));
            lx_s[half][t] = l;
            named_sync_softmax<32 * kSoftWarps>();
            const float lt = lx_s[0][t] + lx_s[1][t];            // fixed order: the same in both halves
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
            const bool live = t < u.nq;
            if (alive) {
                tc_fence_after();
                const int qi = u.q0 + t;
                const int row = qi / G, hh = u.g * G + (qi - row * G);
                bf16* dst = reinterpret_cast<bf16*>(a.o) + ((size_t)(u.row_base + row) * a.Hq + hh) * kD + half * 64;
#pragma unroll 1
                for (int c0 = 0; c0 < kD / 2; c0 += 32) {
                    float v[32];
                    tmem_ld32(trow + kT5OCol + (uint32_t)(half * 64 + c0), v);
                    if (live) {
#pragma unroll
                        for (int c = 0; c < 32; c += 8) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                __nv_bfloat162 b2 = __floats2bfloat162_rn(v[c + 2 * e] * inv, v[c + 2 * e + 1] * inv);
                                w[e] = *reinterpret_cast<uint32_t*>(&b2);
                            }
                            *reinterpret_cast<uint4*>(dst + c0 + c) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
            }
            if constexpr (FULL) {
                if (a.imp_part != nullptr) {
                    // column sums of the block keys' final probabilities over the tile's query vectors, in fixed
                    // order through shared memory (the K / V ring is idle once the last P V completed).  Every
                    // softmax warp reaches the named barrier, whether or not its waits succeeded; a timeout
                    // contributes zeros (and the error word says the outputs are not valid).
                    float* colbuf = reinterpret_cast<float*>(kv_s);  // [QT query vectors][65]
                    const float mu = m_used == -CUDART_INF_F ? 0.f : m_used;
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        colbuf[t * 65 + half * 32 + c] =
                            (alive && live && sb[c] != -CUDART_INF_F && lt > 0.f) ? exp2f(sb[c] - mu) * inv : 0.f;
                    named_sync_softmax<32 * kSoftWarps>();
                    const int j = half * QT + t;
                    if (j < a.B) {
                        float col = 0.f;
                        for (int r = 0; r < QT; ++r) col += colbuf[r * 65 + j];
                        a.imp_part[(size_t)unit * a.B + j] = col;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == T5<QT>::kMmaWarp)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kT5TmemCols) : "memory");
}

}  // namespace

}  // namespace focus

namespace focus {

namespace {

// 3-D view of the query rows for TMA: (d, query head, row), box (64, G, QT / G): one box is the d half of a
// QT-vector query tile of one KV group, laid out as QT rows of 128 bytes with the 128-byte swizzle.
bool make_q_map(CUtensorMap* m, const void* q, int rows_cap, int Hq, int G, int QT) {
    auto fn = tc::encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)Hq, (cuuint64_t)rows_cap};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)Hq * kD * 2};
    const cuuint32_t box[3] = {64u, (cuuint32_t)G, (cuuint32_t)(QT / G)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// query tile height: 64 when every unit fits one 64-vector tile (two CTAs per SM), else 128
int t5_tile(int q_rows, int G) { return q_rows * G <= 64 ? 64 : 128; }

template <bool FULL, int QT> bool configure_t5() {
    return cudaFuncSetAttribute(attention_t5_kernel<FULL, QT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                t5_smem<QT>()) == cudaSuccess &&
           max_shared_carveout((const void*)attention_t5_kernel<FULL, QT>);
}

template <int QT>
int launch_t5(const AttnArgs& a, int q_tiles, const CUtensorMap& pool_map, const CUtensorMap& ibc_map, cudaStream_t s) {
    CUtensorMap q_map;
    if (!make_q_map(&q_map, a.q, a.q_rows_cap, a.Hq, a.Hq / a.Hkv, QT)) return -1;
    const dim3 grid(q_tiles, a.Hkv, a.N), block(t5_threads<QT>());
    if (a.row_offsets == nullptr)
        return launched(launch_pdl(attention_t5_kernel<true, QT>, grid, block, t5_smem<QT>(), s, 0, pool_map, ibc_map,
                                   q_map, a, q_tiles));
    return launched(launch_pdl(attention_t5_kernel<false, QT>, grid, block, t5_smem<QT>(), s, 0, pool_map, ibc_map, q_map,
                               a, q_tiles));
}

}  // namespace

bool attention_t5_used(int q_rows, int G) { return q_rows * G > 32 && G >= 1 && G <= 16 && (G & (G - 1)) == 0; }

int attention_t5_q_tiles(int q_rows, int G) {
    const int qt = t5_tile(q_rows, G);
    return (q_rows * G + qt - 1) / qt;
}

bool configure_attention_t5_kernels() {
    return configure_t5<true, 128>() && configure_t5<false, 128>() && configure_t5<true, 64>() &&
           configure_t5<false, 64>();
}

int launch_attention_t5(const AttnArgs& a, int q_tiles, cudaStream_t s) {
    if (a.N <= 0 || q_tiles <= 0) return 0;
    CUtensorMap pool_map, ibc_map;
    const uint64_t ibc_rows = (uint64_t)a.N * a.L * 2 * a.Hkv * a.B;
    if (!tc::make_map(&ibc_map, a.ibc, ibc_rows, kD, (uint32_t)a.B, false)) return -1;
    if (a.n_pages > 0) {
        const uint64_t pool_rows = (uint64_t)a.n_pages * a.L * 2 * a.Hkv * a.page_size;
        if (!tc::make_map(&pool_map, a.kv_pool, pool_rows, kD, (uint32_t)a.page_size, false)) return -1;
    } else {
        pool_map = ibc_map;  // never used: with no pages every prefix key is invalid
    }
    if (t5_tile(a.q_rows, a.Hq / a.Hkv) == 64) return launch_t5<64>(a, q_tiles, pool_map, ibc_map, s);
    return launch_t5<128>(a, q_tiles, pool_map, ibc_map, s);
}

}  // namespace focus
