// rounding.cuh -- token rounding: every expert's token count rounded to a
// multiple of the GEMM tile, so the grouped GEMMs compute no padding rows.
//
// The "token rounding" scheduling of "SonicMoE vs conventional MoE: how
// token rounding lifts training efficiency" (core difference 3).  The page's
// pseudocode is garbled; the rule implemented, per expert e and independently
// of the other experts, starting from the top-k routing:
//   c = tokens routed to e, r = c mod R;
//   r == 0      : unchanged;
//   2 r <= R    : drop the r routed tokens with the smallest p[t][e] (equal p:
//                 the larger token index first);
//   2 r >  R    : add the R - r unrouted tokens with the largest p[t][e]
//                 (equal p: the smaller token index first), if there are that
//                 many; otherwise drop r as above.
// A token's weight for an expert it keeps or gains is p[t][e], the softmax
// probability the router computed (the top-k weights are those same values).
//
// Kernels:
//   round_kernel  one CTA per expert: a T-bit membership bitmap in shared
//                 memory; the r-th smallest (or a-th largest) key is found by
//                 an 8-pass radix select over distinct 64-bit keys
//                 (p's bits << 32 | ~t); the bitmap is updated and written out
//                 with the new count.
//   scan_kernel   exclusive scan of the new counts -> group offsets.
//   place_kernel  one CTA per expert: walks its bitmap in token order and
//                 writes the grouped rows' weights and posmap[t][e]
//                 (the row of (t, e); -1, set by a memset, elsewhere).
//   gather_rows   x_perm[posmap[t][e]] = x[t]: a warp per token reads its row
//                 once and writes it to each of the token's rows.
//   combine_kernel_masked: out[t] = sum over e ascending with posmap[t][e] >= 0
//                 of y[posmap[t][e]] (fp16 rows widened, fp32 sum).
#pragma once

#include <cuda_fp16.h>

#include "ptx.cuh"

namespace moe {
namespace rounding {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxTokens = 1 << 20;   // bitmap of one expert: 128 KB of shared memory

__host__ __device__ inline int bitmap_words(int T) { return (T + 31) / 32; }

// Shared memory of round_kernel: 64 B of scratch, 256 histogram bins, bitmap
// words and, when T <= kCachedTokens, the expert's probability row (read by
// all eight radix passes).
constexpr int kCachedTokens = 40960;
__host__ __device__ inline bool round_caches_row(int T) { return T <= kCachedTokens; }
__host__ inline size_t round_smem_bytes(int T)
{
    return 64 + 256 * 4 + (size_t)bitmap_words(T) * 4 + (round_caches_row(T) ? (size_t)T * 4 : 0);
}

__device__ __forceinline__ uint64_t round_key(float p, int t)
{
    return ((uint64_t)__float_as_uint(p) << 32) | (uint64_t)(~(uint32_t)t);
}

// Block-wide: the m-th smallest key (1-based) among the candidates `cand(i)`
// for i in [0, n).  Keys are distinct.  Every thread returns the same value.
// hist: 256 ints of shared memory; sh: 4 words of shared memory.
template <typename Cand>
__device__ uint64_t select_kth(int n, int m, Cand cand, int* hist, unsigned long long* sh)
{
    uint64_t prefix = 0;
    int rem = m;
    for (int shift = 56; shift >= 0; shift -= 8) {
        const uint64_t hi_mask = shift == 56 ? 0ull : (~0ull << (shift + 8));
        for (int i = threadIdx.x; i < 256; i += kThreads) hist[i] = 0;
        __syncthreads();
        // warp-aggregated: the lanes with the same digit add once (most keys
        // share their top bytes, so per-lane atomics would serialise)
        const int lane = threadIdx.x & 31;
        for (int i0 = threadIdx.x - lane; i0 < n; i0 += kThreads) {
            const int i = i0 + lane;
            uint64_t key = 0;
            const bool live = i < n && cand(i, key) && (key & hi_mask) == (prefix & hi_mask);
            const int digit = live ? (int)((key >> shift) & 255u) : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, digit);
            if (live && (__ffs(peers) - 1) == lane) atomicAdd(&hist[digit], __popc(peers));
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // warp 0: find the digit whose bucket holds the rem-th key
            const int lane = threadIdx.x;
            int cnt[8], local = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                cnt[j] = hist[lane * 8 + j];
                local += cnt[j];
            }
            int incl = local;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int nb = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += nb;
            }
            const int before = incl - local;
            if (before < rem && rem <= incl) {
                int run = before;
                for (int j = 0; j < 8; ++j) {
                    if (rem <= run + cnt[j]) {
                        sh[0] = (unsigned long long)(lane * 8 + j);
                        sh[1] = (unsigned long long)(rem - run);
                        break;
                    }
                    run += cnt[j];
                }
            }
        }
        __syncthreads();
        prefix |= (uint64_t)sh[0] << shift;
        rem = (int)sh[1];
        __syncthreads();
    }
    return prefix;
}

// One CTA per expert.  counts/offsets/perm: the top-k grouping (group e =
// rows offsets[e]..offsets[e+1], perm[row] = t*k + j).  probs_t [E][T].
__global__ void __launch_bounds__(kThreads, 1)
    round_kernel(const int32_t* __restrict__ offsets, const int32_t* __restrict__ perm, int k,
                 const float* __restrict__ probs_t, int T, int E, int R, uint32_t* __restrict__ bitmaps,
                 int32_t* __restrict__ new_counts)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int nw = bitmap_words(T);
    unsigned long long* sh = reinterpret_cast<unsigned long long*>(smem_raw);  // 8 words (64 B), 8-byte aligned
    int* hist = reinterpret_cast<int*>(smem_raw + 64);                        // 256 bins
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem_raw + 64 + 256 * 4);    // nw words
    float* s_p = reinterpret_cast<float*>(bits + nw);                          // T floats when cached
    const bool cached = round_caches_row(T);
    const int e = blockIdx.x;
    pdl_trigger();
    pdl_wait();
    for (int i = threadIdx.x; i < nw; i += kThreads) bits[i] = 0u;
    if (cached)
        for (int t = threadIdx.x; t < T; t += kThreads) s_p[t] = __ldg(probs_t + (int64_t)e * T + t);
    __syncthreads();
    const int g0 = __ldg(offsets + e), g1 = __ldg(offsets + e + 1);
    const int c = g1 - g0;
    bool bad = false;
    for (int i = g0 + threadIdx.x; i < g1; i += kThreads) {
        const int t = __ldg(perm + i) / k;
        if ((unsigned)t < (unsigned)T)
            atomicOr(&bits[t >> 5], 1u << (t & 31));
        else
            bad = true;
    }
    bad = __syncthreads_or(bad) != 0;
    if (bad) {
        // corrupt grouping: report it and leave the expert empty, so the
        // later kernels still see a consistent (if wrong) routing
        if (threadIdx.x == 0) record_status(kStatusDeviceBounds);
        for (int i = threadIdx.x; i < nw; i += kThreads) bits[i] = 0u;
        __syncthreads();
    }
    const float* pe = cached ? s_p : probs_t + (int64_t)e * T;
    const int r = bad ? 0 : c % R;
    const int add = R - r;
    if (r != 0) {
        if (2 * r > R && T - c >= add) {
            // the add-th largest unrouted key = the (n - add + 1)-th smallest
            const int n = T - c;
            const uint64_t kth = select_kth(T, n - add + 1, [&](int t, uint64_t& key) {
                if ((bits[t >> 5] >> (t & 31)) & 1u) return false;
                key = round_key(pe[t], t);
                return true;
            }, hist, sh);
            __syncthreads();
            for (int t = threadIdx.x; t < T; t += kThreads)
                if (!((bits[t >> 5] >> (t & 31)) & 1u) && round_key(pe[t], t) >= kth)
                    atomicOr(&bits[t >> 5], 1u << (t & 31));
        } else {
            const uint64_t kth = select_kth(c, r, [&](int i, uint64_t& key) {
                const int t = __ldg(perm + g0 + i) / k;
                key = round_key(pe[t], t);
                return true;
            }, hist, sh);
            __syncthreads();
            for (int i = threadIdx.x; i < c; i += kThreads) {
                const int t = __ldg(perm + g0 + i) / k;
                if (round_key(pe[t], t) <= kth) atomicAnd(&bits[t >> 5], ~(1u << (t & 31)));
            }
        }
    }
    __syncthreads();
    int cnt = 0;
    uint32_t* out = bitmaps + (int64_t)e * nw;
    for (int i = threadIdx.x; i < nw; i += kThreads) {
        out[i] = bits[i];
        cnt += __popc(bits[i]);
    }
    // block sum of cnt (hist is free again: the selects are done)
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if ((threadIdx.x & 31) == 0) hist[threadIdx.x >> 5] = cnt;
    __syncthreads();
    if (threadIdx.x == 0) {
        int s = 0;
        for (int w = 0; w < kWarps; ++w) s += hist[w];
        new_counts[e] = s;
    }
}

// Exclusive scan of counts[0..E) into offsets[0..E] (one block, E <= 512).
__global__ void __launch_bounds__(kThreads) scan_kernel(const int32_t* __restrict__ counts, int E,
                                                         int32_t* __restrict__ offsets)
{
    __shared__ int s_warp[kWarps];
    pdl_trigger();
    pdl_wait();
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    const int v = tid < E ? counts[tid] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int nb = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += nb;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int nb = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += nb;
        }
        s_warp[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int excl = (warp > 0 ? s_warp[warp - 1] : 0) + incl - v;
    if (tid < E) offsets[tid] = excl;
    if (tid == 0) offsets[E] = s_warp[kWarps - 1];
}

// One CTA per expert: group e's rows, in token order: w[pos] = p[t][e] and
// posmap[t * E + e] = pos (the caller fills posmap with -1 first).
__global__ void __launch_bounds__(kThreads) place_kernel(const uint32_t* __restrict__ bitmaps,
                                                          const int32_t* __restrict__ offsets,
                                                          const float* __restrict__ probs_t, int T, int E,
                                                          int64_t capacity, float* __restrict__ w,
                                                          int32_t* __restrict__ posmap)
{
    __shared__ int s_warp[kWarps];
    __shared__ int s_carry;
    pdl_trigger();
    pdl_wait();
    const int e = blockIdx.x;
    const int nw = bitmap_words(T);
    const uint32_t* bits = bitmaps + (int64_t)e * nw;
    const float* pe = probs_t + (int64_t)e * T;
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    if (tid == 0) s_carry = 0;
    __syncthreads();
    const int base = __ldg(offsets + e);
    for (int w0 = 0; w0 < nw; w0 += kThreads) {
        const int wi = w0 + tid;
        const uint32_t word = wi < nw ? __ldg(bits + wi) : 0u;
        const int v = __popc(word);
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int nb = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += nb;
        }
        if (lane == 31) s_warp[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int x = s_warp[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int nb = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += nb;
            }
            s_warp[lane] = x;
        }
        __syncthreads();
        int pos = base + s_carry + (warp > 0 ? s_warp[warp - 1] : 0) + incl - v;
        if (wi < nw) {
            for (int b = 0; b < 32; ++b) {
                const int t = wi * 32 + b;
                if (t >= T) break;
                if (!((word >> b) & 1u)) continue;  // posmap was filled with -1 beforehand
                if ((unsigned long long)(unsigned)pos < (unsigned long long)capacity) {
                    w[pos] = pe[t];
                    posmap[(int64_t)t * E + e] = pos;
                    ++pos;
                } else {
                    record_status(kStatusDeviceBounds);
                }
            }
        }
        __syncthreads();
        if (tid == 0) s_carry += s_warp[kWarps - 1];
        __syncthreads();
    }
}

// x_perm[posmap[t][e]] = x[t] for every row of token t: one warp per token
// reads the row once (16-byte vectors, eight in flight per lane) and writes
// it to each of the token's rows, found 32 experts at a time with a ballot.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x,
                                                           const int32_t* __restrict__ posmap, int E, int64_t T,
                                                           int64_t capacity, int nvec, uint4* __restrict__ x_perm)
{
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t t = (int64_t)blockIdx.x * 8 + warp;
    pdl_trigger();
    pdl_wait();
    if (t >= T) return;
    const uint4* src = x + t * nvec;
    constexpr int kUnroll = 8;
    for (int v0 = 0; v0 < nvec; v0 += 32 * kUnroll) {
        uint4 buf[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int v = v0 + u * 32 + lane;
            if (v < nvec) buf[u] = __ldg(src + v);
        }
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            int pos = e < E ? __ldg(posmap + t * E + e) : -1;
            if (pos >= 0 && (unsigned long long)pos >= (unsigned long long)capacity) {
                record_status(kStatusDeviceBounds);
                pos = -1;
            }
            unsigned m = __ballot_sync(0xffffffffu, pos >= 0);
            while (m) {  // warp-uniform
                const int src_lane = __ffs(m) - 1;
                m &= m - 1;
                const int pj = __shfl_sync(0xffffffffu, pos, src_lane);
                uint4* dst = x_perm + (int64_t)pj * nvec;
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec) dst[v] = buf[u];
                }
            }
        }
    }
}

// out[t] = sum over experts e ascending with posmap[t][e] >= 0 of y[row]
// (fp16 widened, fp32 sum).  One block per token; warp 0 compacts the token's
// rows into shared memory in expert order first.
__global__ void __launch_bounds__(256) combine_masked_kernel(const uint4* __restrict__ y,
                                                              const int32_t* __restrict__ posmap, int E,
                                                              int64_t rows, int nvec, float4* __restrict__ out)
{
    __shared__ int s_pos[512];
    __shared__ int s_chunk[17];  // per 32-expert chunk: its row count, then the exclusive prefix; [16]: total
    const int64_t t = blockIdx.x;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nwarps = blockDim.x / 32;
    const int nchunks = (E + 31) / 32;
    pdl_trigger();
    pdl_wait();
    auto row_of = [&](int e) {
        int p = e < E ? __ldg(posmap + t * E + e) : -1;
        if (p >= 0 && (unsigned long long)p >= (unsigned long long)rows) {
            record_status(kStatusDeviceBounds);
            p = -1;
        }
        return p;
    };
    // the token's rows, compacted in ascending expert order by all warps:
    // chunk counts, their prefix, then each chunk writes at its offset
    for (int ch = warp; ch < nchunks; ch += nwarps) {
        const unsigned m = __ballot_sync(0xffffffffu, row_of(ch * 32 + lane) >= 0);
        if (lane == 0) s_chunk[ch] = __popc(m);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int ch = 0; ch < nchunks; ++ch) {
            const int c = s_chunk[ch];
            s_chunk[ch] = run;
            run += c;
        }
        s_chunk[16] = run;
    }
    __syncthreads();
    for (int ch = warp; ch < nchunks; ch += nwarps) {
        const int p = row_of(ch * 32 + lane);
        const unsigned m = __ballot_sync(0xffffffffu, p >= 0);
        if (p >= 0) s_pos[s_chunk[ch] + __popc(m & ((1u << lane) - 1u))] = p;
    }
    __syncthreads();
    const int n = s_chunk[16];
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int j = 0; j < n; ++j) {
            const uint4 q = __ldg(y + (int64_t)s_pos[j] * nvec + v);
            const __half2* h = reinterpret_cast<const __half2*>(&q);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __half22float2(h[i]);
                acc[2 * i] += f.x;
                acc[2 * i + 1] += f.y;
            }
        }
        float4* o = out + (t * nvec + v) * 2;
        o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

}  // namespace rounding
}  // namespace moe
