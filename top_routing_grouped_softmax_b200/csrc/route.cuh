// route.cuh -- router GEMM, fp32 softmax and top-k in one kernel.
//
// Stages 1 and 2 of the MoE block ("Qwen3MoeSparseMoeBlock performance
// optimisation in practice", section 1: router linear, softmax over the
// experts, topk; the routing weights are the top-k probabilities, not
// renormalised).
//
// One CTA owns 128 tokens and the whole hidden dimension.  TMA streams
// x[128 tokens, 64 k] (K-major) and W_router[64 k, E] (E contiguous,
// MN-major) through a shared-memory ring; one thread issues tcgen05.mma into
// a 128 x E fp32 accumulator in TMEM (token m -> TMEM lane m, expert e ->
// column e).  The logits never leave the SM and are never rounded below fp32.
//
// Epilogue, 4 * NG warps.  Warp w may only read TMEM lane quarter w % 4 (32
// tokens), so it takes column group w / 4: NG threads share each token, one
// NG-th of the experts each.  Each thread adds the bias, keeps its maximum
// and a sorted top-KMAX list of (logit, expert) in registers (ranking
// compares fp32 logits -- softmax is monotone -- and equal logits rank the
// lower expert index first), then sums exp(l - max) over its columns.  The
// NG partial results meet in shared memory; one thread per token combines
// them: overall maximum, the partial sums rescaled by exp(m_g - max) in group
// order, and an NG-way merge of the sorted lists for the k winners.  The
// winners' probabilities exp(l - max) / sum are the routing weights.  The same thread counts its winners into the CTA's two
// 64-token chunk histograms, which the permutation needs and which the CTA
// writes out whole (expert-major table, no global atomics, no zeroing).
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace moe {
namespace route {

constexpr int kBM = 128;                    // tokens per CTA = TMEM lanes
constexpr int kBK = 64;                     // K per pipeline stage (128 B of bf16)
constexpr int kABytes = kBM * kBK * 2;      // 16 KB token tile
constexpr int kChunkBytes = 64 * kBK * 2;   // 8 KB: 64 experts x 64 k
constexpr int kTokensPerChunk = 64;         // permutation chunk (tokens)
constexpr int kChunksPerTile = kBM / kTokensPerChunk;
constexpr int kMaxStages = 8;

struct Params {
    const float* bias;       // [E] or nullptr
    int32_t* ids;            // [T, k]
    float* wts;              // [T, k]
    int32_t* chunk_counts;   // [E][n_tchunks] or nullptr
    int n_tchunks;
    int T, d, E, k;
    int n_chunks;            // ceil(E / 64): 64-expert column chunks of W_router
    int stages;              // pipeline depth
    uint32_t tmem_cols;      // power of two >= 64 * n_chunks
};

__host__ __device__ inline int stage_bytes(int n_chunks) { return kABytes + n_chunks * kChunkBytes; }

// Column groups (threads per token) for a top-KMAX list: eight keep 32
// warps busy while the short lists fit 64 registers; longer lists need the
// registers of a 16-warp CTA.
template <int KMAX>
struct Shape {
    static constexpr int groups = KMAX <= 8 ? 8 : 4;
    static constexpr int threads = 128 * groups;
};

// Columns per group: a multiple of 16 (the TMEM load width) such that the
// groups cover all E columns.  Groups past E are empty; a 16-column load
// that starts below E (a multiple of 8) ends at or below 64 * n_chunks.
__host__ __device__ inline int group_cols(int E, int groups)
{
    return ((E + groups * 16 - 1) / (groups * 16)) * 16;
}

// Epilogue scratch (reuses the stage ring once every MMA has completed):
// the groups' lists [group][j][token] (values, then indices), their maxima
// and sums [group][token], and the winners [token][j] (ids, then weights).
__host__ __device__ inline size_t epi_bytes(int kmax, int groups)
{
    return (size_t)4 * kBM * (2 * groups * kmax + 2 * groups + 2 * kmax);
}

__host__ __device__ inline size_t region_bytes(int n_chunks, int stages, int kmax, int groups)
{
    const size_t ring = (size_t)stages * stage_bytes(n_chunks);
    const size_t epi = epi_bytes(kmax, groups);
    return ring > epi ? ring : epi;
}

// Dynamic shared memory: 1 KB alignment slack, ring/scratch region,
// barriers, TMEM slot, abort flag, bias [E], chunk histograms [2][E].
template <int KMAX>
__host__ inline size_t smem_bytes(int n_chunks, int stages, int E)
{
    return 1024 + region_bytes(n_chunks, stages, KMAX, Shape<KMAX>::groups) + (size_t)(2 * stages + 1) * 8 + 16 +
           (size_t)3 * E * 4;
}

// (value, index) order of the top-k: larger logit first; equal logits rank
// the lower expert index first.
__device__ __forceinline__ bool ranks_before(float v, int i, float w, int j) { return v > w || (v == w && i < j); }

// Insert (x, col) into a list sorted by ranks_before, dropping its last
// entry.  The caller visits its columns in ascending index order, so every
// entry already in the list has a lower index than col and x ranks before
// entry j exactly when x > v[j].  All KMAX comparisons are independent and
// every slot takes its new value by selection (no branches, no dependent
// chain): slot j keeps its entry, takes x, or takes the old entry j-1.
template <int KMAX>
__device__ __forceinline__ void topk_insert_ascending(float (&v)[KMAX], int (&ix)[KMAX], float x, int col)
{
    bool gt[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) gt[j] = x > v[j];
#pragma unroll
    for (int j = KMAX - 1; j > 0; --j) {
        v[j] = gt[j - 1] ? v[j - 1] : (gt[j] ? x : v[j]);
        ix[j] = gt[j - 1] ? ix[j - 1] : (gt[j] ? col : ix[j]);
    }
    v[0] = gt[0] ? x : v[0];
    ix[0] = gt[0] ? col : ix[0];
}

template <int KMAX>
__global__ void __launch_bounds__(Shape<KMAX>::threads, 1)
    route_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, Params p)
{
    constexpr int kGroups = Shape<KMAX>::groups;
    constexpr int kThreads = Shape<KMAX>::threads;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int sbytes = stage_bytes(p.n_chunks);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + region_bytes(p.n_chunks, p.stages, KMAX, kGroups));
    uint64_t* empty = full + p.stages;
    uint64_t* done = empty + p.stages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* s_bias = reinterpret_cast<float*>(tmem_slot + 4);
    int* s_hist = reinterpret_cast<int*>(s_bias + p.E);  // [2][E]
    // epilogue scratch, valid once every MMA has completed
    float* s_lval = reinterpret_cast<float*>(smem);                       // [groups][KMAX][128]
    int* s_lidx = reinterpret_cast<int*>(s_lval + kGroups * KMAX * kBM);  // [groups][KMAX][128]
    float* s_gmax = reinterpret_cast<float*>(s_lidx + kGroups * KMAX * kBM);  // [groups][128]
    float* s_gsum = s_gmax + kGroups * kBM;                                   // [groups][128]
    int* s_oid = reinterpret_cast<int*>(s_gsum + kGroups * kBM);              // [128][KMAX]
    float* s_ow = reinterpret_cast<float*>(s_oid + kBM * KMAX);               // [128][KMAX]

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint64_t limit = g_wait_limit_ns;
    const int tile0 = blockIdx.x * kBM;
    const int num_kb = p.d / kBK;

    for (int e = threadIdx.x; e < p.E; e += kThreads) s_bias[e] = p.bias ? p.bias[e] : 0.0f;
    for (int e = threadIdx.x; e < kChunksPerTile * p.E; e += kThreads) s_hist[e] = 0;
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

    // ------------------------------------------------------------ epilogue
    bool have = true;
    if (lane == 0) have = mbar_wait(done, 0, limit);
    have = __shfl_sync(0xffffffffu, have ? 1 : 0, 0) != 0;
    tc_fence_after_sync();
    // a timed-out wait already recorded the device status; every thread of
    // the CTA reaches the same decision from the flag and its warp's wait
    const bool ok = __syncthreads_and(have && *abort_flag == 0) != 0;
    const int q = warp & 3;          // TMEM lane quarter
    const int g = warp >> 2;         // column group
    const int row = q * 32 + lane;   // token within the tile
    if (ok) {
        const int cg = group_cols(p.E, kGroups);
        const int c_begin = g * cg;
        const int c_end = min(p.E, c_begin + cg);
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
        float v[KMAX];
        int ix[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            v[j] = -INFINITY;
            ix[j] = 0x7fffffff;
        }
        float mx = -INFINITY;
        for (int c0 = c_begin; c0 < c_end; c0 += 16) {  // warp-uniform bounds
            uint32_t acc[16];
            tmem_ld16(trow + c0, acc);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int col = c0 + i;
                if (col < c_end) {
                    const float l = __uint_as_float(acc[i]) + s_bias[col];
                    mx = fmaxf(mx, l);
                    topk_insert_ascending<KMAX>(v, ix, l, col);
                }
            }
        }
        float sum = 0.0f;
        for (int c0 = c_begin; c0 < c_end; c0 += 16) {
            uint32_t acc[16];
            tmem_ld16(trow + c0, acc);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int col = c0 + i;
                if (col < c_end) sum += expf(__uint_as_float(acc[i]) + s_bias[col] - mx);
            }
        }
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            s_lval[(g * KMAX + j) * kBM + row] = v[j];
            s_lidx[(g * KMAX + j) * kBM + row] = ix[j];
        }
        s_gmax[g * kBM + row] = mx;
        s_gsum[g * kBM + row] = sum;
    }
    __syncthreads();
    const int64_t t = (int64_t)tile0 + row;
    if (ok && g == 0 && t < p.T) {
        float mx = s_gmax[row];
        for (int h = 1; h < kGroups; ++h) mx = fmaxf(mx, s_gmax[h * kBM + row]);
        float sum = 0.0f;
        for (int h = 0; h < kGroups; ++h) {
            const float mh = s_gmax[h * kBM + row];
            if (mh != -INFINITY) sum += s_gsum[h * kBM + row] * expf(mh - mx);
        }
        // kGroups-way merge: each list is sorted and holds its group's
        // KMAX >= k best, so the k best overall are among the heads
        int head[kGroups];
#pragma unroll
        for (int h = 0; h < kGroups; ++h) head[h] = 0;
        const int hc = row / kTokensPerChunk;
        for (int j = 0; j < p.k; ++j) {
            int bg = -1;
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int h = 0; h < kGroups; ++h) {
                if (head[h] < KMAX) {
                    const float hv = s_lval[(h * KMAX + head[h]) * kBM + row];
                    const int hi = s_lidx[(h * KMAX + head[h]) * kBM + row];
                    if (hi < p.E && (bg < 0 || ranks_before(hv, hi, bv, bi))) {
                        bg = h;
                        bv = hv;
                        bi = hi;
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < kGroups; ++h)
                if (h == bg) ++head[h];
            s_oid[row * KMAX + j] = bi;
            s_ow[row * KMAX + j] = expf(bv - mx) / sum;
            if (p.chunk_counts && bg >= 0) atomicAdd(&s_hist[hc * p.E + bi], 1);
        }
    }
    __syncthreads();
    if (ok) {
        // the tile's ids and weights are contiguous in [T, k]: coalesced copy
        const int n_tok = min(kBM, p.T - tile0);
        for (int i = threadIdx.x; i < n_tok * p.k; i += kThreads) {
            const int r = i / p.k, j = i % p.k;
            p.ids[(int64_t)tile0 * p.k + i] = s_oid[r * KMAX + j];
            p.wts[(int64_t)tile0 * p.k + i] = s_ow[r * KMAX + j];
        }
        if (p.chunk_counts) {
            const int chunk0 = tile0 / kTokensPerChunk;
            for (int i = threadIdx.x; i < kChunksPerTile * p.E; i += kThreads) {
                const int hc = i / p.E, e = i % p.E;
                if (chunk0 + hc < p.n_tchunks)
                    p.chunk_counts[(int64_t)e * p.n_tchunks + chunk0 + hc] = s_hist[i];
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
