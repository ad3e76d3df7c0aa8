// backward.cuh -- the memory-bound kernels of the MoE block's backward.
//
// The gradient is that of L = sum_t dout[t] . out[t] (the block's forward as
// in "Qwen3MoeSparseMoeBlock performance optimisation in practice", section
// 1), computed the way the SonicMoE comparison page's memory rule asks ("core
// differences", item 1): nothing but the routing is kept from the forward;
// the permutation, x_perm and the expert activations are rebuilt.  The
// grouped GEMMs are in grouped_gemm_bwd.cuh; these kernels move rows and
// finish the router's part:
//
//   gather_dout   dout_perm[inv[t*k+j]] = bf16(dout[t])   (one warp per token)
//   zero_pad      zero the padding rows between a group's end and the next
//                 64-row boundary in x_perm and dout_perm, and their routing
//                 weights, so every row operand of the weight gradients is
//                 zero there
//   route_bwd     per token (one warp): dw_j = sum of the down GEMM's partial
//                 dot products of slot j; dp = dw at the selected experts
//                 (renormalised weights: (dw_j - sum_m w_m dw_m) / S);
//                 dlogit = p (dp - sum_e p_e dp_e) (the softmax Jacobian);
//                 stores dlogit in bf16 (the operand of the two router GEMMs)
//                 and the block's fp32 sums of dlogit for the bias gradient
//   colsum        dbias[e] = sum over blocks of those sums, in a fixed order
//   sum_partials  dW_router = the sum of its split-K partials, in a fixed order
//   combine_dx    dx[t] = dx_router[t] + sum_j dx_perm[inv[t*k+j]]  (fp32 sums of bf16 dx_perm rows)
#pragma once

#include <cuda_bf16.h>

#include "grouped_gemm_bwd.cuh"
#include "ptx.cuh"

namespace moe {
namespace bwd {

constexpr int kRowThreads = 256;  // 8 warps
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kMaxTopK = 32;
constexpr int kMaxExperts = 512;

// dout (fp32 [T][d]) -> dout_perm (bf16, grouped rows): one warp per token
// reads the row once (eight columns per lane per step) and writes its k
// copies.  nvec = d / 8.
__global__ void __launch_bounds__(kRowThreads) gather_dout_kernel(const float4* __restrict__ dout,
                                                                  const int32_t* __restrict__ inv, int64_t T, int k,
                                                                  int nvec, int64_t rows, uint4* __restrict__ dout_perm)
{
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t t = (int64_t)blockIdx.x * kRowWarps + warp;
    pdl_trigger();
    pdl_wait();
    if (t >= T) return;
    int pos = -1;
    if (lane < k) {
        pos = __ldg(inv + t * k + lane);
        if ((unsigned long long)(unsigned)pos >= (unsigned long long)rows) {
            record_status(kStatusDeviceBounds);
            pos = -1;
        }
    }
    for (int v = lane; v < nvec; v += 32) {
        const float4 a = __ldg(dout + (t * nvec + v) * 2);
        const float4 b = __ldg(dout + (t * nvec + v) * 2 + 1);
        __nv_bfloat162 q[4] = {__floats2bfloat162_rn(a.x, a.y), __floats2bfloat162_rn(a.z, a.w),
                               __floats2bfloat162_rn(b.x, b.y), __floats2bfloat162_rn(b.z, b.w)};
        const uint4 packed = *reinterpret_cast<const uint4*>(q);
        for (int j = 0; j < k; ++j) {
            const int pj = __shfl_sync(0xffffffffu, pos, j);
            if (pj >= 0) dout_perm[(int64_t)pj * nvec + v] = packed;
        }
    }
}

// One block per expert: rows [offsets[e] + counts[e], offsets[e+1]) of the
// two row operands (nvec 16-byte vectors per row) and their routing weights
// are set to zero.
__global__ void __launch_bounds__(kRowThreads) zero_pad_kernel(const int32_t* __restrict__ offsets,
                                                               const int32_t* __restrict__ counts, int nvec,
                                                               uint4* __restrict__ a, uint4* __restrict__ b,
                                                               float* __restrict__ w_perm)
{
    const int e = blockIdx.x;
    pdl_trigger();
    pdl_wait();
    const int64_t r0 = (int64_t)__ldg(offsets + e) + __ldg(counts + e);
    const int64_t r1 = __ldg(offsets + e + 1);
    const int64_t n = (r1 - r0) * nvec;
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int64_t i = threadIdx.x; i < n; i += kRowThreads) {
        a[r0 * nvec + i] = z;
        b[r0 * nvec + i] = z;
    }
    for (int64_t r = r0 + threadIdx.x; r < r1; r += kRowThreads) w_perm[r] = 0.0f;
}

// One warp per token, eight tokens per block.  probs [T][E] fp32 (the
// router's probabilities, recomputed), ids / wts [T][k], inv [T*k], dwp
// [rows][n_tiles] (the down GEMM's partial dot products; n_tiles counts
// them per row).  Writes dlogit
// [T][ld_dl] bf16 (columns past E zero) and, per block, the fp32 sum of its tokens' dlogit rows
// (db_part [gridDim.x][E], added in warp order).
__global__ void __launch_bounds__(kRowThreads) route_bwd_kernel(
    const float* __restrict__ probs, const int32_t* __restrict__ ids, const float* __restrict__ wts,
    const int32_t* __restrict__ inv, const float* __restrict__ dwp, int n_tiles, int64_t rows, int64_t T, int E,
    int k, int renorm, __nv_bfloat16* __restrict__ dlogit, float* __restrict__ db_part, int ld_dl)
{
    __shared__ float s_dp[kRowWarps][kMaxExperts];
    __shared__ float s_dl[kRowWarps][kMaxExperts];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t t = (int64_t)blockIdx.x * kRowWarps + warp;
    pdl_trigger();
    pdl_wait();
    const bool live = t < T;
    for (int e = lane; e < E; e += 32) {
        s_dp[warp][e] = 0.0f;
        s_dl[warp][e] = 0.0f;
    }
    __syncwarp();
    if (live) {
        // slot j on lane j: its expert, weight and weight gradient
        int id = -1;
        float wj = 0.0f, dwj = 0.0f, pj = 0.0f;
        if (lane < k) {
            id = __ldg(ids + t * k + lane);
            wj = __ldg(wts + t * k + lane);
            int pos = __ldg(inv + t * k + lane);
            if ((unsigned)id >= (unsigned)E || (unsigned long long)(unsigned)pos >= (unsigned long long)rows) {
                record_status(kStatusDeviceBounds);
                id = -1;
            } else {
                for (int n = 0; n < n_tiles; ++n) dwj += __ldg(dwp + (int64_t)pos * n_tiles + n);
                pj = __ldg(probs + t * E + id);
            }
        }
        // sums over the k slots in slot order (a fixed butterfly order)
        float dot = wj * dwj, ssum = pj;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            dot += __shfl_xor_sync(0xffffffffu, dot, o);
            ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
        }
        if (id >= 0) s_dp[warp][id] = renorm ? (dwj - dot) / ssum : dwj;
        __syncwarp();
        float pdp = 0.0f;
        for (int e = lane; e < E; e += 32) pdp += __ldg(probs + t * E + e) * s_dp[warp][e];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) pdp += __shfl_xor_sync(0xffffffffu, pdp, o);
        for (int e = lane; e < E; e += 32) {
            const float pe = __ldg(probs + t * E + e);
            const float dl = pe * (s_dp[warp][e] - pdp);
            s_dl[warp][e] = dl;
            dlogit[t * ld_dl + e] = __float2bfloat16_rn(dl);
        }
        // columns E .. ld_dl - 1 pad the row to a multiple of 64: zero
        for (int e = E + lane; e < ld_dl; e += 32) dlogit[t * ld_dl + e] = __float2bfloat16_rn(0.0f);
    }
    __syncthreads();
    if (db_part)
        for (int e = threadIdx.x; e < E; e += kRowThreads) {
            float acc = 0.0f;
            for (int w = 0; w < kRowWarps; ++w) acc += s_dl[w][e];
            db_part[(int64_t)blockIdx.x * E + e] = acc;
        }
}

// dbias[e] = sum over blocks b of db_part[b][e]: one block per expert;
// thread i sums blocks i, i + 256, ... in order, then a fixed tree adds the
// 256 partial sums (the same order on every run).
__global__ void __launch_bounds__(kRowThreads) colsum_kernel(const float* __restrict__ db_part, int nblk, int E,
                                                             float* __restrict__ dbias)
{
    __shared__ float s_part[kRowThreads];
    const int e = blockIdx.x;
    pdl_trigger();
    pdl_wait();
    float acc = 0.0f;
    for (int b = threadIdx.x; b < nblk; b += kRowThreads) acc += __ldg(db_part + (int64_t)b * E + e);
    s_part[threadIdx.x] = acc;
    __syncthreads();
    for (int w = kRowThreads / 2; w > 0; w >>= 1) {
        if (threadIdx.x < w) s_part[threadIdx.x] += s_part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) dbias[e] = s_part[0];
}

// out[i] = sum over s = 0..S-1 of part[s][i], in ascending s (fp32): the
// split-K partial products of the router's weight gradient.  n4 = elements / 4.
// BF16OUT: the fp32 sum rounded to bf16 once.
template <bool BF16OUT>
__global__ void __launch_bounds__(kRowThreads) sum_partials_kernel(const float4* __restrict__ part, int S,
                                                                   int64_t n4, void* __restrict__ out)
{
    pdl_trigger();
    pdl_wait();
    for (int64_t i = blockIdx.x * (int64_t)kRowThreads + threadIdx.x; i < n4; i += (int64_t)gridDim.x * kRowThreads) {
        float4 acc = __ldg(part + i);
        for (int s = 1; s < S; ++s) {
            const float4 a = __ldg(part + (int64_t)s * n4 + i);
            acc.x += a.x;
            acc.y += a.y;
            acc.z += a.z;
            acc.w += a.w;
        }
        if constexpr (BF16OUT)
            static_cast<uint2*>(out)[i] = make_uint2(gemm::pack_bf16x2(acc.x, acc.y), gemm::pack_bf16x2(acc.z, acc.w));
        else
            static_cast<float4*>(out)[i] = acc;
    }
}

// dx[t] = dx_router[t] + sum_j dx_perm[inv[t*k+j]] (fp32 sums, slots in
// order; dx_perm bf16, widened exactly): one block per token, eight columns
// per thread.  nvec = d / 8.
__global__ void __launch_bounds__(kRowThreads) combine_dx_kernel(const uint4* __restrict__ dx_perm,
                                                                 const float4* __restrict__ dx_router,
                                                                 const int32_t* __restrict__ inv, int64_t rows, int k,
                                                                 int nvec, float4* __restrict__ dx)
{
    __shared__ int s_pos[kMaxTopK];
    const int64_t t = blockIdx.x;
    pdl_trigger();
    pdl_wait();
    if (threadIdx.x < k) {
        int p = __ldg(inv + t * k + threadIdx.x);
        if ((unsigned long long)(unsigned)p >= (unsigned long long)rows) {
            record_status(kStatusDeviceBounds);
            p = -1;
        }
        s_pos[threadIdx.x] = p;
    }
    __syncthreads();
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        const float4 r0 = __ldg(dx_router + (t * nvec + v) * 2), r1 = __ldg(dx_router + (t * nvec + v) * 2 + 1);
        float acc[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
        for (int j = 0; j < k; ++j) {
            const int p = s_pos[j];
            if (p < 0) continue;
            float a[8];
            unpack_bf16x8(__ldg(dx_perm + (int64_t)p * nvec + v), a);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] += a[i];
        }
        dx[(t * nvec + v) * 2] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        dx[(t * nvec + v) * 2 + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

}  // namespace bwd
}  // namespace moe
