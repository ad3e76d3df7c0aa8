// route.cuh -- router GEMM, fp32 softmax and top-k in one kernel.
//
// Stages 1 and 2 of the MoE block ("Qwen3MoeSparseMoeBlock performance
// optimisation in practice", section 1: router linear, softmax over the
// experts, topk; the routing weights are the top-k probabilities, not
// renormalised).
//
// A tile is 128 tokens.  TMA streams x[128 tokens, 64 k] (K-major) and
// W_router[64 k, E] (E contiguous, MN-major) through a shared-memory ring;
// one thread issues tcgen05.mma into a 128 x E fp32 accumulator in TMEM
// (token m -> TMEM lane m, expert e -> column e).  The logits are never
// rounded below fp32.
//
// Split K over a CTA pair.  When the batch has few tiles (fewer than half the
// SMs), a cluster of two CTAs shares a tile: CTA r accumulates k-blocks
// [r*nkb/2, (r+1)*nkb/2), and CTA r owns token rows [64r, 64r+64) of the
// tile.  After both mainloops, each CTA copies its partial logits from TMEM
// into the owner's shared memory (distributed shared memory stores), one
// buffer slot per sender; the owner adds the slots in rank order, so the
// result does not depend on timing.  With one CTA per tile the same code
// runs with a single slot (and, for E > 256, in two passes of 64 rows so
// the buffer fits).
//
// Softmax and top-k.  For k <= 8, a group of L lanes of one warp takes a
// token (L = 8 when a CTA owns 128 rows, 16 when it owns 64, so all 32 warps
// are busy).  Lane j of the group visits experts j, j + L, j + 2L, ... in
// ascending order: it adds the split-K partials and the bias once, writes
// the logit back to shared memory, and keeps its maximum and its best
// (logit, expert); the group's maximum and the sum of exp(l - max) are
// butterfly reductions in a fixed order.  k rounds of a butterfly arg-max
// over the lanes' best candidates then pick the winners in order; the lane
// that owned a winner marks it taken and rescans its experts (from a
// register copy when a lane has at most 16).  For k > 8, a whole warp takes a
// token and picks the winners in k rounds of a butterfly arg-max.  Both
// rank by the (value, index) order -- larger logit first, equal logits rank
// the lower expert index first -- on fp32 logits (softmax is monotone).
// Lane j < k of the token's group writes slot j: the expert and its
// probability exp(l - max) / sum -- or, with renorm, exp(l - max) divided by
// the sum over the k selected experts only (weights summing to one).  The same lanes count their experts into
// the tile's 64-token chunk histograms, which the permutation needs and
// which the CTA writes out whole (expert-major table, no global atomics, no
// zeroing).
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace moe {
namespace route {

constexpr int kBM = 128;                    // tokens per tile = TMEM lanes
constexpr int kBK = 64;                     // K per pipeline stage (128 B of bf16)
constexpr int kThreads = 1024;              // 32 warps
constexpr int kWarps = kThreads / 32;
constexpr int kABytes = kBM * kBK * 2;      // 16 KB token tile
constexpr int kChunkBytes = 64 * kBK * 2;   // 8 KB: 64 experts x 64 k
constexpr int kTokensPerChunk = 64;         // permutation chunk (tokens)
constexpr int kColGroups = kWarps / 4;      // warps sharing a TMEM lane quarter
constexpr int kMaxStages = 8;

struct Params {
    const float* bias;       // [E] or nullptr
    int32_t* ids;            // [T, k]
    float* wts;              // [T, k]
    int32_t* chunk_counts;   // [E][n_tchunks] or nullptr
    int n_tchunks;
    int T, d, E, k;
    int n_chunks;            // ceil(E / 64): 64-expert column chunks of W_router
    int w_one_copy;          // 1: all chunks of a k-block come in one 3-D copy (E % 64 == 0)
    int stages;              // pipeline depth
    uint32_t tmem_cols;      // power of two >= 64 * n_chunks
    int split;               // CTAs per tile: 1, or 2 (cluster of two, split K)
    int passes;              // row passes of the exchange buffer (1, or 2 when split == 1 and E > 256)
    int renorm;              // 1: divide each token's k weights by their sum
    float* probs;            // every expert's probability, or nullptr: p[t][e] at t * probs_tstride + e * probs_estride
    int64_t probs_tstride;   // [E][T] for token rounding (1, T); [T][E] for the backward (E, 1)
    int64_t probs_estride;
};

__host__ __device__ inline int stage_bytes(int n_chunks) { return kABytes + n_chunks * kChunkBytes; }

// Token rows one CTA owns in one pass, and the exchange buffer
// [split slots][E][pitch] fp32 with pitch = own + 32 / L (own is a multiple
// of 32, so pitch = 32 / L mod 32 banks).  A warp writing 32 rows of one
// column hits 32 consecutive words; a warp reading, for 32 / L tokens, the
// columns j + L m of its L lanes hits bank (32 / L) * j + token: distinct.
__host__ __device__ inline int own_rows(int split, int passes) { return kBM / (split * passes); }
__host__ __device__ inline int group_lanes(int own) { return kThreads / own; }  // 8 or 16
__host__ __device__ inline int buffer_pitch(int own) { return own + 32 / group_lanes(own); }
__host__ __device__ inline size_t buffer_bytes(int E, int split, int passes)
{
    return (size_t)split * E * buffer_pitch(own_rows(split, passes)) * 4;
}

__host__ __device__ inline size_t region_bytes(int n_chunks, int stages, int E, int split, int passes)
{
    const size_t ring = (size_t)stages * stage_bytes(n_chunks);
    const size_t buf = buffer_bytes(E, split, passes);
    return ring > buf ? ring : buf;
}

// Dynamic shared memory: 1 KB alignment slack, ring / exchange region,
// barriers, TMEM slot, abort flag, bias [E], chunk histograms [2][E].
__host__ inline size_t smem_bytes(int n_chunks, int stages, int E, int split, int passes)
{
    return 1024 + region_bytes(n_chunks, stages, E, split, passes) + (size_t)(2 * stages + 1) * 8 + 16 +
           (size_t)3 * E * 4;
}

// Columns per warp column group: a multiple of 16 (the TMEM load width) such
// that the groups cover all E columns.  Groups past E are empty; a 16-column
// load that starts below E (a multiple of 8) ends at or below 64 * n_chunks.
__host__ __device__ inline int group_cols(int E) { return ((E + kColGroups * 16 - 1) / (kColGroups * 16)) * 16; }

// (value, index) order of the top-k: larger logit first; equal logits rank
// the lower expert index first.
__device__ __forceinline__ bool ranks_before(float v, int i, float w, int j) { return v > w || (v == w && i < j); }

// Softmax and top-k of one token by a whole warp (k > 8).  `col(j)` is the
// logit of expert lane + 32 j (called only for lane + 32 j < E).  Lane
// j < k receives slot j.
template <int VPL, typename Logit>
__device__ __forceinline__ void warp_topk(int E, int k, bool renorm, int lane, Logit col, int& my_id, float& my_w,
                                          float* pcol, int64_t pstride)
{
    float v[VPL];
    unsigned taken = 0;  // bit j: value j is not a candidate
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        const int c = lane + 32 * j;
        if (c < E) {
            v[j] = col(j);
        } else {
            v[j] = -INFINITY;
            taken |= 1u << j;
        }
    }
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < VPL; ++j) mx = fmaxf(mx, v[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.0f;
#pragma unroll
    for (int j = 0; j < VPL; ++j)
        if (!((taken >> j) & 1u)) sum += expf(v[j] - mx);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (pcol) {  // every expert's probability, by the same formula as the weights below
#pragma unroll
        for (int j = 0; j < VPL; ++j)
            if (!((taken >> j) & 1u)) pcol[(int64_t)(lane + 32 * j) * pstride] = expf(v[j] - mx) / sum;
    }
    my_id = 0;
    my_w = 0.0f;
    for (int slot = 0; slot < k; ++slot) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int c = lane + 32 * j;
            if (!((taken >> j) & 1u) && ranks_before(v[j], c, bv, bi)) {
                bv = v[j];
                bi = c;
            }
        }
        // a strict total order: both partners of every exchange keep the
        // same winner, so all lanes end with the token's best
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ranks_before(ov, oi, bv, bi)) {
                bv = ov;
                bi = oi;
            }
        }
        if ((bi & 31) == lane) taken |= 1u << ((bi >> 5) & 31);
        if (lane == slot) {
            my_id = bi;
            my_w = expf(bv - mx);
        }
    }
    if (renorm) {
        // the selected terms only (lanes >= k hold 0), in a fixed order
        sum = my_w;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    }
    my_w /= sum;
}

// Softmax and top-k of one token by a group of L lanes (lane j of the group
// = lane % L).  Lane j owns experts j, j + L, j + 2L, ...  `combine(c)` returns
// expert c's logit (the sum of the split-K partials plus the bias) and
// `cell(c)` is a shared-memory slot for it: the first pass writes the
// combined logits there, tracks the lane's maximum and its best (value,
// index), and the group's maximum and sum follow by butterfly reductions in
// a fixed order.  Then k rounds of a butterfly arg-max over the lanes' best
// candidates pick the winners in (value, index) order; the lane that owned
// a winner marks it taken (-inf in its slot) and rescans its experts for its
// next best.  Lane j < k receives slot j.  With VPL > 0 (E <= L * VPL) the
// rescans run over a register copy of the lane's logits, unrolled, instead
// of the shared-memory cells; the passes before stay rolled loops, because
// the epilogue runs once per CTA and unrolled code there is fetched cold.
template <int L, int VPL, typename Combine, typename Cell>
__device__ __forceinline__ void group_topk(int E, int k, bool renorm, int j, Combine combine, Cell cell, int& my_id,
                                           float& my_w, float* pcol, int64_t pstride)
{
    float mx = -INFINITY, bv = -INFINITY;
    int bc = 0x7fffffff;
    for (int c = j; c < E; c += L) {
        const float l = combine(c);
        cell(c) = l;
        mx = fmaxf(mx, l);
        if (l > bv) {  // ascending c: among equal values the lower index stays
            bv = l;
            bc = c;
        }
    }
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.0f;
    for (int c = j; c < E; c += L) sum += __expf(cell(c) - mx);
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (pcol)  // every expert's probability, by the same formula as the weights below
        for (int c = j; c < E; c += L) pcol[c * pstride] = __expf(cell(c) - mx) / sum;
    // VPL > 0: a register copy of the lane's logits (slots at or past E hold
    // -inf, never a candidate) serves the rescans below
    float v[VPL > 0 ? VPL : 1];
    if constexpr (VPL > 0) {
#pragma unroll
        for (int m = 0; m < VPL; ++m) v[m] = j + L * m < E ? cell(j + L * m) : -INFINITY;
    }
    float my_v = -INFINITY;
    my_id = 0;
    for (int slot = 0; slot < k; ++slot) {
        float wv = bv;
        int wc = bc;
#pragma unroll
        for (int o = L / 2; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
            const int oc = __shfl_xor_sync(0xffffffffu, wc, o);
            if (ranks_before(ov, oc, wv, wc)) {
                wv = ov;
                wc = oc;
            }
        }
        if (j == slot) {
            my_id = wc;
            my_v = wv;
        }
        // this lane owned the winner: take it, find the next best (a lane with
        // no candidate left -- NaN logits -- holds the sentinel, never an index)
        if (wc == bc && wc < E) {
            bv = -INFINITY;
            bc = 0x7fffffff;
            if constexpr (VPL > 0) {
#pragma unroll
                for (int m = 0; m < VPL; ++m) {
                    const int c = j + L * m;
                    if (c == wc) v[m] = -INFINITY;
                    if (v[m] > bv) {
                        bv = v[m];
                        bc = c;
                    }
                }
            } else {
                cell(wc) = -INFINITY;
                for (int c = j; c < E; c += L) {
                    const float l = cell(c);
                    if (l > bv) {
                        bv = l;
                        bc = c;
                    }
                }
            }
        }
    }
    if (renorm) {
        // the selected terms only (lanes >= k hold 0), in a fixed order
        float s = j < k ? __expf(my_v - mx) : 0.0f;
#pragma unroll
        for (int o = L / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        sum = s;
    }
    my_w = __expf(my_v - mx) / sum;
}

// One pass of softmax + top-k over the `own` buffered rows, L lanes per
// token (32 / L tokens per warp).  VPL > 0: the rescans of the top-k rounds
// over VPL registers per lane (E <= L * VPL); VPL == 0: over the
// shared-memory buffer cells (any E).
template <int L, int KMAX, int VPL>
__device__ __forceinline__ void topk_rows(const Params& p, float* buf, const float* s_bias, int* s_hist,
                                          int S, int own, int pitch, int tile0, int row0, bool ok, int warp,
                                          int lane)
{
    static_assert(L >= KMAX, "lane j of a group writes slot j: a group needs at least k lanes");
    const int E = p.E;
    const int j = lane % L;
    for (int i = warp * (32 / L) + lane / L; i - lane / L < own; i += kWarps * (32 / L)) {
        // i < own for every group of the warp: own is a multiple of 32 / L
        const int64_t t = (int64_t)tile0 + row0 + i;
        int my_id;
        float my_w;
        const auto combine = [&](int c) {
            const float* col = buf + (size_t)c * pitch + i;
            float l = col[0];
            for (int s = 1; s < S; ++s) l += col[(size_t)s * E * pitch];
            return l + s_bias[c];
        };
        float* const pcol = (p.probs && ok && t < p.T) ? p.probs + t * p.probs_tstride : nullptr;
        group_topk<L, VPL>(
            E, p.k, p.renorm != 0, j, combine, [&](int c) -> float& { return buf[(size_t)c * pitch + i]; }, my_id,
            my_w, pcol, p.probs_estride);
        if (ok && t < p.T && j < p.k) {
            p.ids[t * p.k + j] = my_id;
            p.wts[t * p.k + j] = my_w;
            if (p.chunk_counts && (unsigned)my_id < (unsigned)E)
                atomicAdd(&s_hist[((row0 + i) / kTokensPerChunk) * E + my_id], 1);
        }
    }
}

// topk_rows with the smallest register count per lane that holds the
// lane's ceil(E / L) experts (up to 16), else the shared-memory version.
template <int L, int KMAX>
__device__ __forceinline__ void topk_rows_any(const Params& p, float* buf, const float* s_bias, int* s_hist,
                                              int S, int own, int pitch, int tile0, int row0, bool ok, int warp,
                                              int lane)
{
    const int vpl = (p.E + L - 1) / L;
    if (vpl <= 1)
        topk_rows<L, KMAX, 1>(p, buf, s_bias, s_hist, S, own, pitch, tile0, row0, ok, warp, lane);
    else if (vpl <= 2)
        topk_rows<L, KMAX, 2>(p, buf, s_bias, s_hist, S, own, pitch, tile0, row0, ok, warp, lane);
    else if (vpl <= 4)
        topk_rows<L, KMAX, 4>(p, buf, s_bias, s_hist, S, own, pitch, tile0, row0, ok, warp, lane);
    else if (vpl <= 8)
        topk_rows<L, KMAX, 8>(p, buf, s_bias, s_hist, S, own, pitch, tile0, row0, ok, warp, lane);
    else if (vpl <= 16)
        topk_rows<L, KMAX, 16>(p, buf, s_bias, s_hist, S, own, pitch, tile0, row0, ok, warp, lane);
    else
        topk_rows<L, KMAX, 0>(p, buf, s_bias, s_hist, S, own, pitch, tile0, row0, ok, warp, lane);
}

template <int KMAX>
__global__ void __launch_bounds__(kThreads, 1)
    route_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                 const __grid_constant__ CUtensorMap tm_w3, Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = p.split;
    const int sbytes = stage_bytes(p.n_chunks);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + region_bytes(p.n_chunks, p.stages, p.E, S, p.passes));
    uint64_t* empty = full + p.stages;
    uint64_t* done = empty + p.stages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* s_bias = reinterpret_cast<float*>(tmem_slot + 4);
    int* s_hist = reinterpret_cast<int*>(s_bias + p.E);  // [2][E]
    float* buf = reinterpret_cast<float*>(smem);         // exchange buffer, once the ring is idle

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint64_t limit = g_wait_limit_ns;
    const uint32_t r = S > 1 ? cluster_ctarank() : 0u;
    const int tile0 = (int)(blockIdx.x / S) * kBM;
    const int nkb = p.d / kBK;
    const int kb0 = (int)((int64_t)nkb * r / S);
    const int kb1 = (int)((int64_t)nkb * (r + 1) / S);
    const int E = p.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_map(&tm_x);
        tma_prefetch_map(p.w_one_copy ? &tm_w3 : &tm_w);
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
    // x may come from an earlier kernel on the stream, and earlier kernels
    // may still read the ids, weights and histograms this launch writes
    pdl_trigger();
    pdl_wait();
    for (int e = threadIdx.x; e < E; e += kThreads) s_bias[e] = p.bias ? p.bias[e] : 0.0f;
    for (int e = threadIdx.x; e < 2 * E; e += kThreads) s_hist[e] = 0;
    __syncthreads();

    if (warp == 0) {
        if (lane == 0) {
            // TMA producer over this CTA's k-blocks
            int issued = 0;
            for (int kb = kb0; kb < kb1; ++kb) {
                const int i = kb - kb0;
                const int s = i % p.stages;
                const uint32_t ph = (uint32_t)(i / p.stages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, limit)) {
                    *abort_flag = 1;
                    break;
                }
                uint8_t* sa = smem + (size_t)s * sbytes;
                mbar_arrive_expect_tx(&full[s], (uint32_t)sbytes);
                tma_load_2d(sa, &tm_x, &full[s], kb * kBK, tile0);
                if (p.w_one_copy) {
                    // W_router viewed as [E/64][d][64]: every 64-expert chunk of the k-block
                    tma_load_3d(sa + kABytes, &tm_w3, &full[s], 0, kb * kBK, 0);
                } else {
                    for (int c = 0; c < p.n_chunks; ++c)
                        tma_load_2d(sa + kABytes + c * kChunkBytes, &tm_w, &full[s], c * 64, kb * kBK);
                }
                ++issued;
            }
            // Never leave the CTA with a copy still landing in its shared memory.
            for (int s = 0; s < p.stages; ++s) {
                const int cnt = issued / p.stages + (s < issued % p.stages ? 1 : 0);
                if (cnt > 0) mbar_wait(&full[s], (uint32_t)(cnt - 1) & 1u, drain_limit(limit));
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // MMA issuer: up to two N <= 256 MMAs per k-step cover all experts.
            for (int kb = kb0; kb < kb1; ++kb) {
                const int i = kb - kb0;
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

    // ---------------------------------------------------------- epilogue
    bool have = true;
    if (lane == 0) have = mbar_wait(done, 0, drain_limit(limit));
    have = __shfl_sync(0xffffffffu, have ? 1 : 0, 0) != 0;
    tc_fence_after_sync();
    // a timed-out wait already recorded the device status; every thread of
    // the CTA reaches the same decision, and every thread of both CTAs of a
    // pair still takes part in every cluster barrier below
    const bool ok = __syncthreads_and(have && *abort_flag == 0) != 0;
    const int q = warp & 3;          // TMEM lane quarter
    const int g = warp >> 2;         // column group
    const int cg = group_cols(E);
    const int c_begin = g * cg;
    const int c_end = min(E, c_begin + cg);
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    const int own = own_rows(S, p.passes);
    const int pitch = buffer_pitch(own);

    for (int pass = 0; pass < p.passes; ++pass) {
        // the ring (and the previous pass's buffer) is idle in every CTA of the tile
        if (S > 1)
            cluster_sync();
        else
            __syncthreads();
        // stage this CTA's partial logits for the rows of this pass into the
        // owner's buffer slot r: buf[r][col][row - owner's first row]
        const int qrow = q * 32;
        const int owner = S > 1 ? qrow / own : 0;
        const int first = S > 1 ? owner * own : pass * own;
        const bool stage = ok && qrow >= first && qrow < first + own;  // warp-uniform
        if (stage) {
            float* dst = buf + (size_t)r * E * pitch + (qrow + lane - first);
            for (int c0 = c_begin; c0 < c_end; c0 += 16) {  // warp-uniform bounds
                uint32_t acc[16];
                tmem_ld16(trow + c0, acc);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int col = c0 + i;
                    if (col < c_end) {
                        float* a = dst + (size_t)col * pitch;
                        if (S > 1)
                            st_cluster_f32(mapa_shared(a, (uint32_t)owner), __uint_as_float(acc[i]));
                        else
                            *a = __uint_as_float(acc[i]);
                    }
                }
            }
        }
        if (S > 1)
            cluster_sync();  // every slot of this CTA's buffer is written
        else
            __syncthreads();
        // softmax + top-k of the rows this CTA owns in this pass
        const int row0 = S > 1 ? (int)r * own : pass * own;
        if constexpr (KMAX <= 8) {
            if (own == 128)
                topk_rows_any<8, KMAX>(p, buf, s_bias, s_hist, S, own, pitch, tile0, row0, ok, warp, lane);
            else
                topk_rows_any<16, KMAX>(p, buf, s_bias, s_hist, S, own, pitch, tile0, row0, ok, warp, lane);
        } else {
            for (int i = warp; i < own; i += kWarps) {
                const int64_t t = (int64_t)tile0 + row0 + i;
                if (t >= p.T) break;  // warp-uniform; later rows are past the end too
                int my_id;
                float my_w;
                warp_topk<16>(E, p.k, p.renorm != 0, lane, [&](int jj) {
                    const int c = lane + 32 * jj;
                    const float* col = buf + (size_t)c * pitch + i;
                    float l = col[0];
                    for (int s = 1; s < S; ++s) l += col[(size_t)s * E * pitch];
                    return l + s_bias[c];
                }, my_id, my_w, (p.probs && ok) ? p.probs + t * p.probs_tstride : nullptr, p.probs_estride);
                if (ok && lane < p.k) {
                    p.ids[t * p.k + lane] = my_id;
                    p.wts[t * p.k + lane] = my_w;
                    if (p.chunk_counts && (unsigned)my_id < (unsigned)E)
                        atomicAdd(&s_hist[((row0 + i) / kTokensPerChunk) * E + my_id], 1);
                }
            }
        }
    }
    __syncthreads();
    if (ok && p.chunk_counts) {
        // chunks whose tokens this CTA ranked: both of the tile (one CTA), or
        // chunk r (pair)
        const int chunk0 = tile0 / kTokensPerChunk;
        for (int i = threadIdx.x; i < 2 * E; i += kThreads) {
            const int hc = i / E, e = i % E;
            if ((S == 1 || hc == (int)r) && chunk0 + hc < p.n_tchunks)
                p.chunk_counts[(int64_t)e * p.n_tchunks + chunk0 + hc] = s_hist[i];
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
