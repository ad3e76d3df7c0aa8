// route.cuh -- router GEMM + fp32 softmax + top-k in one kernel.
//
// Stages 1 and 2 of the MoE block ("Qwen3MoeSparseMoeBlock performance
// optimisation in practice", section 1: router linear, softmax over the
// experts, topk; the routing weights are the top-k probabilities, not
// renormalised).
//
// One CTA owns 128 tokens.  TMA streams x[128 tokens, 64 k] (K-major) and
// W_router[64 k, E] (E contiguous, i.e. MN-major) into a shared-memory ring;
// one thread issues tcgen05.mma into a 128 x E fp32 accumulator in TMEM
// (token m -> TMEM lane m, expert e -> column e).  After the K loop each of
// the 128 threads owns one token's whole logit row: it adds the bias, keeps
// a sorted top-KMAX list in registers while tracking the maximum, then sums
// exp(l - max) in a second pass and writes the k ids and probabilities.
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

struct Params {
    const float* bias;   // [E] or nullptr
    int32_t* ids;        // [T, k]
    float* wts;          // [T, k]
    int T, d, E, k;
    int n_chunks;        // ceil(E / 64): 64-expert column chunks of W_router
    int stages;          // pipeline depth
    uint32_t tmem_cols;  // power of two >= 64 * n_chunks
};

__host__ __device__ inline int stage_bytes(int n_chunks) { return kABytes + n_chunks * kChunkBytes; }

// Dynamic shared memory: 1 KB alignment slack, the stage ring, barriers,
// TMEM slot + abort flag, bias copy.
__host__ inline size_t smem_bytes(int n_chunks, int stages, int E)
{
    return 1024 + (size_t)stages * stage_bytes(n_chunks) + (size_t)(2 * stages + 1) * 8 + 16 + (size_t)E * 4;
}

// Insert (x, col) into a list sorted by descending value.  Columns arrive in
// ascending order, so an equal value stays behind the earlier (lower) index.
template <int KMAX>
__device__ __forceinline__ void topk_insert(float (&v)[KMAX], int (&ix)[KMAX], float x, int col)
{
    if (!(x > v[KMAX - 1])) return;
    // Walk from the tail: slot j takes the old v[j-1] when x belongs in front
    // of it, or x itself when x lands exactly at j.
#pragma unroll
    for (int j = KMAX - 1; j > 0; --j) {
        if (x > v[j - 1]) {
            v[j] = v[j - 1];
            ix[j] = ix[j - 1];
        } else if (x > v[j]) {
            v[j] = x;
            ix[j] = col;
        }
    }
    if (x > v[0]) {
        v[0] = x;
        ix[0] = col;
    }
}

template <int KMAX>
__global__ void __launch_bounds__(kThreads, 1)
    route_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int sbytes = stage_bytes(p.n_chunks);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)p.stages * sbytes);
    uint64_t* empty = full + p.stages;
    uint64_t* done = empty + p.stages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* s_bias = reinterpret_cast<float*>(tmem_slot + 4);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint64_t limit = g_wait_limit_ns;
    const int tile0 = blockIdx.x * kBM;
    const int num_kb = p.d / kBK;

    for (int e = threadIdx.x; e < p.E; e += kThreads) s_bias[e] = p.bias ? p.bias[e] : 0.0f;
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
            for (int kb = 0; kb < num_kb; ++kb) {
                const int s = kb % p.stages;
                const uint32_t ph = (uint32_t)(kb / p.stages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, limit)) {
                    *abort_flag = 1;
                    break;
                }
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
            for (int kb = 0; kb < num_kb; ++kb) {
                const int s = kb % p.stages;
                const uint32_t ph = (uint32_t)(kb / p.stages) & 1u;
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
                                    (kb | kk) != 0);
                    }
                }
                mma_commit(&empty[s]);
            }
            mma_commit(done);  // arrives once every MMA issued above has completed
        }
        __syncwarp();
    }
    __syncthreads();

    // Epilogue: every thread owns one token (TMEM lane = warp*32 + lane).
    const bool have = __all_sync(0xffffffffu, mbar_wait(done, 0, limit));
    tc_fence_after_sync();
    if (have && *abort_flag == 0) {
        const int r = warp * 32 + lane;
        const int64_t t = (int64_t)tile0 + r;
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        float v[KMAX];
        int ix[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            v[j] = -INFINITY;
            ix[j] = 0x7fffffff;
        }
        float mx = -INFINITY;
        for (int c0 = 0; c0 < p.E; c0 += 16) {
            uint32_t acc[16];
            tmem_ld16(trow + c0, acc);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int col = c0 + i;
                if (col < p.E) {
                    const float l = __uint_as_float(acc[i]) + s_bias[col];
                    mx = fmaxf(mx, l);
                    topk_insert<KMAX>(v, ix, l, col);
                }
            }
        }
        float sum = 0.0f;
        for (int c0 = 0; c0 < p.E; c0 += 16) {
            uint32_t acc[16];
            tmem_ld16(trow + c0, acc);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int col = c0 + i;
                if (col < p.E) sum += expf(__uint_as_float(acc[i]) + s_bias[col] - mx);
            }
        }
        if (t < p.T) {
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j < p.k) {
                    p.ids[t * p.k + j] = ix[j];
                    p.wts[t * p.k + j] = expf(v[j] - mx) / sum;
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

}  // namespace route
}  // namespace moe
