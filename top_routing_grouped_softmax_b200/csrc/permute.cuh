// permute.cuh -- token reordering by expert.
//
// The "token reordering" step of "Qwen3MoeSparseMoeBlock performance
// optimisation in practice" (section 2.2: sort_tokens_by_expert, then gather
// the hidden states and routing weights in that order), done as a stable
// counting sort over the T*k flat assignments a = t*k + j:
//   hist  : per-chunk expert histograms (chunk = 4096 assignments)
//   scan  : per-expert totals, exclusive offsets, and each chunk's starting
//           position inside every expert group
//   rank  : inside a chunk, eight warps walk their 512 assignments in order;
//           __match_any_sync gives each lane its rank among same-expert lanes
//           so group order is ascending a -- deterministic, no global atomics
//   gather: one warp per grouped row copies x[t] with 16-byte vectors
#pragma once

#include <cuda_bf16.h>

#include "status.cuh"

namespace moe {
namespace permute {

constexpr int kChunk = 4096;        // assignments per chunk
constexpr int kThreads = 256;       // 8 warps
constexpr int kWarps = kThreads / 32;
constexpr int kPerWarp = kChunk / kWarps;
constexpr int kScanThreads = 512;   // >= max E

__global__ void __launch_bounds__(kThreads) hist_kernel(const int32_t* __restrict__ ids, int64_t n, int E,
                                                        int32_t* __restrict__ chunk_counts)
{
    extern __shared__ int s_hist[];
    for (int e = threadIdx.x; e < E; e += kThreads) s_hist[e] = 0;
    __syncthreads();
    const int64_t a0 = (int64_t)blockIdx.x * kChunk;
    const int64_t a1 = min(n, a0 + kChunk);
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
    for (int e = threadIdx.x; e < E; e += kThreads) chunk_counts[(int64_t)blockIdx.x * E + e] = s_hist[e];
}

// One block.  Thread e walks the chunks of expert e (running sum), then a
// block-wide exclusive scan over experts gives the group offsets.
// chunk_counts is rewritten in place into absolute chunk starting positions.
__global__ void __launch_bounds__(kScanThreads) scan_kernel(int32_t* __restrict__ chunk_counts, int nchunks, int E,
                                                            int32_t* __restrict__ counts,
                                                            int32_t* __restrict__ offsets)
{
    __shared__ int s_warp[kScanThreads / 32];
    const int e = threadIdx.x;
    const int lane = e % 32, warp = e / 32;
    int total = 0;
    if (e < E) {
#pragma unroll 8
        for (int c = 0; c < nchunks; ++c) {
            const int v = chunk_counts[(int64_t)c * E + e];
            chunk_counts[(int64_t)c * E + e] = total;
            total += v;
        }
        counts[e] = total;
    }
    int incl = total;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int nb = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += nb;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kScanThreads / 32 ? s_warp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int nb = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += nb;
        }
        if (lane < kScanThreads / 32) s_warp[lane] = wi - w;  // exclusive warp prefix
    }
    __syncthreads();
    const int excl = s_warp[warp] + incl - total;
    if (e < E) {
        offsets[e] = excl;
        if (e == E - 1) offsets[E] = excl + total;
#pragma unroll 8
        for (int c = 0; c < nchunks; ++c) chunk_counts[(int64_t)c * E + e] += excl;
    }
}

__global__ void __launch_bounds__(kThreads) rank_kernel(const int32_t* __restrict__ ids,
                                                        const float* __restrict__ wts, int64_t n, int E,
                                                        const int32_t* __restrict__ chunk_base,
                                                        int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                        float* __restrict__ w_perm)
{
    extern __shared__ int s_next[];  // [kWarps][E]: next free position per warp and expert
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int i = threadIdx.x; i < kWarps * E; i += kThreads) s_next[i] = 0;
    __syncthreads();
    const int64_t w0 = (int64_t)blockIdx.x * kChunk + (int64_t)warp * kPerWarp;
    const int64_t w1 = min(n, w0 + kPerWarp);
    int* mine = s_next + warp * E;
    for (int64_t a = w0 + lane; a < w1; a += 32) {
        const int e = __ldg(ids + a);
        if ((unsigned)e < (unsigned)E) atomicAdd(&mine[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kThreads) {
        int run = chunk_base[(int64_t)blockIdx.x * E + e];
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

// x_perm[pos] = x[perm[pos] / k]; one warp per row, 16-byte vectors.
__global__ void __launch_bounds__(kThreads) gather_kernel(const uint4* __restrict__ x,
                                                          const int32_t* __restrict__ perm, int64_t n, int nvec,
                                                          int k, uint4* __restrict__ x_perm)
{
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t row = (int64_t)blockIdx.x * kWarps + warp;
    if (row >= n) return;
    const int a = __ldg(perm + row);
    if ((unsigned)a >= (unsigned long long)n) {
        record_status(kStatusDeviceBounds);
        return;
    }
    const uint4* src = x + (int64_t)(a / k) * nvec;
    uint4* dst = x_perm + row * nvec;
#pragma unroll 4
    for (int v = lane; v < nvec; v += 32) dst[v] = __ldg(src + v);
}

}  // namespace permute
}  // namespace moe
