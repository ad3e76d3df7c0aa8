// route.cuh -- router GEMM, fp32 softmax and top-k.
//
// Stages 1 and 2 of the MoE block ("Qwen3MoeSparseMoeBlock performance
// optimisation in practice", section 1: router linear, softmax over the
// experts, topk; the routing weights are the top-k probabilities, not
// renormalised).
//
// Two kernels:
//   logits_kernel   tcgen05 GEMM.  A CTA owns 128 tokens and one slice of
//                   the hidden dimension (split-K, so that even a short batch
//                   spreads the x read over all SMs).  TMA streams x
//                   [128 tokens, 64 k] (K-major) and W_router [64 k, E]
//                   (E contiguous, MN-major) into a shared-memory ring; one
//                   thread issues tcgen05.mma into a 128 x E fp32 TMEM
//                   accumulator; the epilogue writes the slice's partial
//                   logits (fp32, never rounded) to part[slice][t][e].
//   softmax_topk_kernel
//                   one warp per token: logit = sum of the slices in slice
//                   order + bias; max and sum of exp(l - max) by warp
//                   reductions in a fixed order; then k rounds of a warp
//                   arg-max that prefers the lower expert index on equal
//                   logits.  Selection compares fp32 logits (softmax is
//                   monotone).  Optionally counts each 64-token chunk's
//                   assignments per expert for the permutation.
// Work shape: router_slices() on the host picks the split of the hidden
// dimension (at most kMaxSlices).
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace moe {
namespace route {

constexpr int kBM = 128;                    // tokens per CTA = TMEM lanes
constexpr int kBK = 64;                     // K per pipeline stage (128 B of bf16)
constexpr int kThreads = 128;
constexpr int kABytes = kBM * kBK * 2;      // 16 KB token tile
constexpr int kChunkBytes = 64 * kBK * 2;   // 8 KB: 64 experts x 64 k
constexpr int kTokensPerChunk = 64;         // permutation chunk (tokens)
constexpr int kSoftmaxWarps = 8;            // tokens per softmax block
constexpr int kMaxSlices = 16;

struct Params {
    float* part;         // [slices][T][E] partial logits
    int32_t* zero;       // optional table the softmax kernel accumulates into (zeroed here)
    int64_t zero_count;  // its length in int32
    int T, d, E;
    int n_chunks;        // ceil(E / 64): 64-expert column chunks of W_router
    int stages;          // pipeline depth
    int slices;          // split of the hidden dimension
    uint32_t tmem_cols;  // power of two >= 64 * n_chunks
};

__host__ __device__ inline int stage_bytes(int n_chunks) { return kABytes + n_chunks * kChunkBytes; }

// Dynamic shared memory: 1 KB alignment slack, the stage ring, barriers,
// TMEM slot + abort flag.
__host__ inline size_t smem_bytes(int n_chunks, int stages)
{
    return 1024 + (size_t)stages * stage_bytes(n_chunks) + (size_t)(2 * stages + 1) * 8 + 16;
}

// k-block range [kb0, kb1) of slice s when num_kb blocks are split S ways.
__host__ __device__ inline void slice_range(int num_kb, int S, int s, int& kb0, int& kb1)
{
    kb0 = (int)((int64_t)num_kb * s / S);
    kb1 = (int)((int64_t)num_kb * (s + 1) / S);
}

__global__ void __launch_bounds__(kThreads, 1)
    logits_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int sbytes = stage_bytes(p.n_chunks);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)p.stages * sbytes);
    uint64_t* empty = full + p.stages;
    uint64_t* done = empty + p.stages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint64_t limit = g_wait_limit_ns;
    const int tile0 = (blockIdx.x / p.slices) * kBM;
    const int slice = blockIdx.x % p.slices;
    int kb0, kb1;
    slice_range(p.d / kBK, p.slices, slice, kb0, kb1);
    const int num_kb = kb1 - kb0;

    if (p.zero)
        for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < p.zero_count; i += (int64_t)gridDim.x * kThreads)
            p.zero[i] = 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_map(&tm_x);
        tma_prefetch_map(&tm_w);
    }
    if (warp == 1) {
        __syncwarp();
        tmem_alloc(tmem_slot, p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // TMA producer
            int issued = 0;
            for (int i = 0; i < num_kb; ++i) {
                const int s = i % p.stages;
                const uint32_t ph = (uint32_t)(i / p.stages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, limit)) {
                    *abort_flag = 1;
                    break;
                }
                const int kb = kb0 + i;
                uint8_t* sa = smem + (size_t)s * sbytes;
                mbar_arrive_expect_tx(&full[s], (uint32_t)sbytes);
                tma_load_2d(sa, &tm_x, &full[s], kb * kBK, tile0);
                for (int c = 0; c < p.n_chunks; ++c)
                    tma_load_2d(sa + kABytes + c * kChunkBytes, &tm_w, &full[s], c * 64, kb * kBK);
                ++issued;
            }
            // Never leave the CTA with a copy still landing in its shared memory.
            for (int s = 0; s < p.stages; ++s) {
                const int cnt = issued / p.stages + (s < issued % p.stages ? 1 : 0);
                if (cnt > 0) mbar_wait(&full[s], (uint32_t)(cnt - 1) & 1u, limit);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // MMA issuer: up to two N <= 256 MMAs per k-step cover all experts.
            for (int i = 0; i < num_kb; ++i) {
                const int s = i % p.stages;
                const uint32_t ph = (uint32_t)(i / p.stages) & 1u;
                if (!mbar_wait(&full[s], ph, limit)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t a_base = smem_u32(smem + (size_t)s * sbytes);
                const uint32_t b_base = a_base + kABytes;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    const uint64_t adesc = smem_desc_sw128(a_base + kk * 32, 16, 1024);
                    for (int m = 0; m * 4 < p.n_chunks; ++m) {
                        const int chunks = min(4, p.n_chunks - 4 * m);
                        const uint64_t bdesc =
                            smem_desc_sw128(b_base + m * 4 * kChunkBytes + kk * 2048, kChunkBytes, 1024);
                        mma_bf16_ss(tmem + m * 256, adesc, bdesc, idesc_bf16_f32(128, 64 * chunks, false, true),
                                    (i | kk) != 0);
                    }
                }
                mma_commit(&empty[s]);
            }
            mma_commit(done);  // arrives once every MMA issued above has completed
        }
        __syncwarp();
    }
    __syncthreads();

    // Epilogue: thread r owns token tile0 + r (TMEM lane r) and writes its
    // row of partial logits.
    const bool have = __all_sync(0xffffffffu, mbar_wait(done, 0, limit));
    tc_fence_after_sync();
    if (have && *abort_flag == 0) {
        const int64_t t = (int64_t)tile0 + warp * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        float* dst = p.part + ((int64_t)slice * p.T + t) * p.E;
        for (int c0 = 0; c0 < p.E; c0 += 16) {
            uint32_t acc[16];
            tmem_ld16(trow + c0, acc);
            tmem_ld_wait();
            if (t < p.T) {
                if (c0 + 16 <= p.E) {
                    float4* d4 = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        d4[v] = make_float4(__uint_as_float(acc[4 * v]), __uint_as_float(acc[4 * v + 1]),
                                            __uint_as_float(acc[4 * v + 2]), __uint_as_float(acc[4 * v + 3]));
                } else {
                    // E % 8 == 0: the last 8 columns
                    float4* d4 = reinterpret_cast<float4*>(dst + c0);
                    d4[0] = make_float4(__uint_as_float(acc[0]), __uint_as_float(acc[1]), __uint_as_float(acc[2]),
                                        __uint_as_float(acc[3]));
                    d4[1] = make_float4(__uint_as_float(acc[4]), __uint_as_float(acc[5]), __uint_as_float(acc[6]),
                                        __uint_as_float(acc[7]));
                }
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, p.tmem_cols);
    }
}

// (value, index) order for the top-k: larger logit first, then lower index.
__device__ __forceinline__ bool ranks_before(float v, int i, float w, int j) { return v > w || (v == w && i < j); }

// One warp per token; lane l holds experts e = l + 32 j, j < VPL.  With
// chunk_counts set, every block (8 tokens, all inside one 64-token chunk)
// adds its tokens' selections to chunk_counts[e][chunk] (zeroed by the
// logits kernel); integer atomics, so the totals do not depend on order.
template <int VPL>
__global__ void __launch_bounds__(kSoftmaxWarps * 32)
    softmax_topk_kernel(const float* __restrict__ part, const float* __restrict__ bias, int T, int E, int k,
                        int slices, int32_t* __restrict__ ids, float* __restrict__ wts,
                        int32_t* __restrict__ chunk_counts, int n_tchunks)
{
    __shared__ int s_sel[kSoftmaxWarps * 32];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t t = (int64_t)blockIdx.x * kSoftmaxWarps + warp;
    const bool active = t < T;  // warp-uniform
    if (active) {
        float v[VPL];
        bool taken[VPL];
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int e = lane + 32 * j;
            taken[j] = e >= E;
            float parts[kMaxSlices];
#pragma unroll
            for (int sl = 0; sl < kMaxSlices; ++sl)
                parts[sl] = (e < E && sl < slices) ? __ldg(part + ((int64_t)sl * T + t) * E + e) : 0.0f;
            float l = -INFINITY;
            if (e < E) {
                l = parts[0];
#pragma unroll
                for (int sl = 1; sl < kMaxSlices; ++sl)
                    if (sl < slices) l += parts[sl];
                if (bias) l += __ldg(bias + e);
            }
            v[j] = l;
        }
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < VPL; ++j) mx = fmaxf(mx, v[j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.0f;
#pragma unroll
        for (int j = 0; j < VPL; ++j)
            if (!taken[j]) sum += expf(v[j] - mx);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        int my_id = 0;
        float my_w = 0.0f;
        for (int slot = 0; slot < k; ++slot) {
            // this lane's best remaining (value, index)
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < VPL; ++j) {
                const int e = lane + 32 * j;
                if (!taken[j] && ranks_before(v[j], e, bv, bi)) {
                    bv = v[j];
                    bi = e;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (ranks_before(ov, oi, bv, bi)) {
                    bv = ov;
                    bi = oi;
                }
            }
            // every lane now holds the winner; its owner retires it
            if ((bi & 31) == lane) {
#pragma unroll
                for (int j = 0; j < VPL; ++j)
                    if (lane + 32 * j == bi) taken[j] = true;
            }
            if (lane == slot) {
                my_id = bi;
                my_w = expf(bv - mx) / sum;
            }
        }
        // lane j < k writes slot j (coalesced)
        if (lane < k) {
            ids[t * k + lane] = my_id;
            wts[t * k + lane] = my_w;
        }
        if (chunk_counts) s_sel[warp * 32 + lane] = lane < k ? my_id : -1;
    } else if (chunk_counts) {
        s_sel[warp * 32 + lane] = -1;
    }
    if (chunk_counts) {
        __syncthreads();
        const int chunk = (int)(((int64_t)blockIdx.x * kSoftmaxWarps) / kTokensPerChunk);
        const int e = s_sel[threadIdx.x];
        if (e >= 0) atomicAdd(&chunk_counts[(int64_t)e * n_tchunks + chunk], 1);
    }
}

}  // namespace route
}  // namespace moe
