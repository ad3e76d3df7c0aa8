// permute.cuh -- token reordering by expert.
//
// The "token reordering" step of "Qwen3MoeSparseMoeBlock performance
// optimisation in practice" (section 2.2: sort_tokens_by_expert, then gather
// the hidden states and routing weights in that order), done as a stable
// counting sort over the T*k flat assignments a = t*k + j, in 64-token chunks:
//   hist       : each chunk's assignment count per expert, stored expert-major
//                counts[e][chunk] (the router's softmax kernel can produce
//                the same table as a by-product)
//   chunk_scan : one block per expert turns its row of chunk counts into
//                exclusive chunk bases inside the expert's group and writes
//                the expert's total
//   rank       : one block per chunk recomputes the group offsets (an
//                exclusive scan of the totals), then eight warps walk their
//                slices of the chunk in order; __match_any_sync ranks each
//                lane among same-expert lanes, so every group lists its
//                assignments in ascending a -- deterministic, no global
//                atomics.
//   gather     : x_perm[inv[t*k + j]] = x[t]: one warp per token reads the
//                row once and writes its k copies (16-byte vectors).
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace moe {
namespace permute {

constexpr int kTokensPerChunk = 64;
constexpr int kThreads = 256;       // 8 warps
constexpr int kWarps = kThreads / 32;
constexpr int kMaxE = 512;

// Chunk histogram for callers that bring their own expert ids.
__global__ void __launch_bounds__(kThreads) hist_kernel(const int32_t* __restrict__ ids, int64_t T, int k, int E,
                                                        int32_t* __restrict__ counts_em, int n_tchunks)
{
    __shared__ int s_hist[kMaxE];
    pdl_trigger();
    pdl_wait();
    for (int e = threadIdx.x; e < E; e += kThreads) s_hist[e] = 0;
    __syncthreads();
    const int64_t a0 = (int64_t)blockIdx.x * kTokensPerChunk * k;
    const int64_t a1 = min(T * k, a0 + (int64_t)kTokensPerChunk * k);
    bool bad = false;
    for (int64_t a = a0 + threadIdx.x; a < a1; a += kThreads) {
        const int e = __ldg(ids + a);
        if ((unsigned)e < (unsigned)E)
            atomicAdd(&s_hist[e], 1);
        else
            bad = true;
    }
    if (bad) record_status(kStatusDeviceBounds);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kThreads) counts_em[(int64_t)e * n_tchunks + blockIdx.x] = s_hist[e];
}

// Block e: exclusive scan of counts_em[e][0..n_tchunks) in place; totals[e].
__global__ void __launch_bounds__(kThreads) chunk_scan_kernel(int32_t* __restrict__ counts_em, int n_tchunks,
                                                              int32_t* __restrict__ totals)
{
    __shared__ int s_warp[32];
    pdl_trigger();
    pdl_wait();
    int32_t* row = counts_em + (int64_t)blockIdx.x * n_tchunks;
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    int carry = 0;
    for (int base = 0; base < n_tchunks; base += 4 * kThreads) {
        const int n = min(4 * kThreads, n_tchunks - base);
        int v[4], local = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int idx = tid * 4 + i;
            v[i] = idx < n ? row[base + idx] : 0;
            local += v[i];
        }
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int nb = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += nb;
        }
        if (lane == 31) s_warp[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int w = lane < kWarps ? s_warp[lane] : 0;
            int wi = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int nb = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += nb;
            }
            s_warp[lane] = wi;  // inclusive over warps
        }
        __syncthreads();
        int run = carry + (warp > 0 ? s_warp[warp - 1] : 0) + incl - local;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int idx = tid * 4 + i;
            if (idx < n) row[base + idx] = run;
            run += v[i];
        }
        carry += s_warp[kWarps - 1];
        __syncthreads();
    }
    if (tid == 0) totals[blockIdx.x] = carry;
}

// Rows a group occupies: its size, or (PAD64) its size rounded up to a
// multiple of 64, so that every group starts on a 64-row boundary.
template <bool PAD64>
__device__ __forceinline__ int group_span(int n)
{
    return PAD64 ? (n + 63) & ~63 : n;
}

// One block per 64-token chunk.  chunk_base_em[e][c] holds the chunk's first
// position inside group e (relative to the group start); totals[e] the group
// sizes.  Block 0 also writes offsets[0..E] (the group starts; with PAD64
// each group's rows are followed by padding up to the next multiple of 64,
// which this kernel leaves unwritten).
template <bool PAD64>
__global__ void __launch_bounds__(kThreads) rank_kernel(const int32_t* __restrict__ ids,
                                                        const float* __restrict__ wts, int64_t T, int k, int E,
                                                        const int32_t* __restrict__ chunk_base_em, int n_tchunks,
                                                        const int32_t* __restrict__ totals,
                                                        int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
                                                        int32_t* __restrict__ inv, float* __restrict__ w_perm)
{
    __shared__ int s_off[kMaxE + 1];
    __shared__ int s_next[kWarps * kMaxE];   // next free position per warp and expert
    __shared__ int s_warp[32];
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int chunk = blockIdx.x;
    pdl_trigger();
    pdl_wait();

    // group offsets = exclusive scan of the totals (E <= 512 <= 4 * 256)
    for (int e = tid; e < E; e += kThreads) s_off[e] = totals[e];
    __syncthreads();
    {
        int v[4], local = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int idx = tid * 4 + i;
            v[i] = idx < E ? group_span<PAD64>(s_off[idx]) : 0;
            local += v[i];
        }
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int nb = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += nb;
        }
        if (lane == 31) s_warp[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int w = lane < kWarps ? s_warp[lane] : 0;
            int wi = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int nb = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += nb;
            }
            s_warp[lane] = wi;
        }
        __syncthreads();
        int run = (warp > 0 ? s_warp[warp - 1] : 0) + incl - local;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int idx = tid * 4 + i;
            if (idx < E) s_off[idx] = run;
            run += v[i];
        }
        if (tid == 0) s_off[E] = s_warp[kWarps - 1];
        __syncthreads();
    }
    if (chunk == 0)
        for (int e = tid; e <= E; e += kThreads) offsets[e] = s_off[e];

    // per-warp slices of this chunk's assignments
    const int64_t a_begin = (int64_t)chunk * kTokensPerChunk * k;
    const int64_t a_end = min(T * k, a_begin + (int64_t)kTokensPerChunk * k);
    const int per_warp = (kTokensPerChunk * k + kWarps - 1) / kWarps;
    const int64_t w0 = min(a_end, a_begin + (int64_t)warp * per_warp);
    const int64_t w1 = min(a_end, w0 + per_warp);
    int* mine = s_next + warp * E;
    for (int i = tid; i < kWarps * E; i += kThreads) s_next[i] = 0;
    __syncthreads();
    for (int64_t a = w0 + lane; a < w1; a += 32) {
        const int e = __ldg(ids + a);
        if ((unsigned)e < (unsigned)E) atomicAdd(&mine[e], 1);
    }
    __syncthreads();
    for (int e = tid; e < E; e += kThreads) {
        int run = s_off[e] + chunk_base_em[(int64_t)e * n_tchunks + chunk];
        for (int w = 0; w < kWarps; ++w) {
            const int c = s_next[w * E + e];
            s_next[w * E + e] = run;
            run += c;
        }
    }
    __syncthreads();
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int64_t b = w0; b < w1; b += 32) {
        const int64_t a = b + lane;
        int e = a < w1 ? __ldg(ids + a) : -1;
        const bool valid = (unsigned)e < (unsigned)E;
        if (!valid) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & lt_mask);
        const int base = valid ? mine[e] : 0;
        __syncwarp();
        if (valid && rank == 0) mine[e] = base + __popc(peers);
        __syncwarp();
        if (valid) {
            const int pos = base + rank;
            perm[pos] = (int32_t)a;
            inv[a] = pos;
            w_perm[pos] = __ldg(wts + a);
        }
    }
}

// x_perm[inv[t*k + j]] = x[t] for every slot j: one warp per token reads the
// token's row once (16-byte vectors, eight in flight per lane) and writes it
// to its k grouped positions, so x is read from HBM once and every write is
// a whole contiguous row.  rows: the rows x_perm holds (T*k, or more when
// the groups are padded); a position outside is reported and skipped.
__global__ void __launch_bounds__(kThreads) gather_kernel(const uint4* __restrict__ x,
                                                          const int32_t* __restrict__ inv, int64_t T, int k,
                                                          int nvec, int64_t rows, uint4* __restrict__ x_perm)
{
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t t = (int64_t)blockIdx.x * kWarps + warp;
    pdl_trigger();
    pdl_wait();
    if (t >= T) return;
    const int64_t n = rows;
    int pos = -1;
    if (lane < k) {
        pos = __ldg(inv + t * k + lane);
        if ((unsigned long long)(unsigned)pos >= (unsigned long long)n) {
            record_status(kStatusDeviceBounds);
            pos = -1;
        }
    }
    const uint4* src = x + t * nvec;
    constexpr int kUnroll = 8;
    for (int v0 = 0; v0 < nvec; v0 += 32 * kUnroll) {
        uint4 buf[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int v = v0 + u * 32 + lane;
            if (v < nvec) buf[u] = __ldg(src + v);
        }
        for (int j = 0; j < k; ++j) {
            const int pj = __shfl_sync(0xffffffffu, pos, j);  // warp-uniform
            if (pj < 0) continue;
            uint4* dst = x_perm + (int64_t)pj * nvec;
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < nvec) dst[v] = buf[u];
            }
        }
    }
}

// dst[i] = src[idx[i]] for whole rows of nvec 16-byte vectors: one warp per
// row.  An index outside [0, n_src) is reported and its row is zero-filled.
__global__ void __launch_bounds__(kThreads) gather_rows_idx_kernel(const uint4* __restrict__ src,
                                                                   const int32_t* __restrict__ idx, int64_t n,
                                                                   int64_t n_src, int nvec, uint4* __restrict__ dst)
{
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t i = (int64_t)blockIdx.x * kWarps + warp;
    pdl_trigger();
    pdl_wait();
    if (i >= n) return;
    const int r = __ldg(idx + i);
    const bool ok = r >= 0 && (int64_t)r < n_src;
    if (!ok && lane == 0) record_status(kStatusDeviceBounds);
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int v = lane; v < nvec; v += 32) dst[i * nvec + v] = ok ? __ldg(src + (int64_t)r * nvec + v) : z;
}

// The same for rows of nword 4-byte words (rows that are not a multiple of
// 16 bytes, such as one routing weight per row).
__global__ void __launch_bounds__(kThreads) gather_words_idx_kernel(const uint32_t* __restrict__ src,
                                                                    const int32_t* __restrict__ idx, int64_t n,
                                                                    int64_t n_src, int nword, uint32_t* __restrict__ dst)
{
    const int64_t i0 = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    pdl_trigger();
    pdl_wait();
    const int64_t total = n * nword;
    if (i0 >= total) return;
    const int64_t i = i0 / nword;
    const int wd = (int)(i0 - i * nword);
    const int r = __ldg(idx + i);
    const bool ok = r >= 0 && (int64_t)r < n_src;
    if (!ok && wd == 0) record_status(kStatusDeviceBounds);
    dst[i0] = ok ? __ldg(src + (int64_t)r * nword + wd) : 0u;
}

}  // namespace permute
}  // namespace moe
