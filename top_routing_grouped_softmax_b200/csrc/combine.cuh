// combine.cuh -- routing-weighted aggregation back to token order.
//
// Stage 4 of "Qwen3MoeSparseMoeBlock performance optimisation in practice"
// (section 1: expert outputs summed per token, weighted by the routing
// weights; section 2.2 scatter_outputs).  The weight is already folded into
// y by the down-projection epilogue, so each token gathers its k grouped
// fp16 rows through inv, widens them to fp32 and sums them in fp32 in slot
// order -- a gather, not a scatter-add, so no atomics and a deterministic
// result.  The sum is fp32 and by default is stored as fp32; an output
// option rounds it to fp16 once, at the store.
#pragma once

#include <cuda_fp16.h>

#include "ptx.cuh"

namespace moe {
namespace combine {

constexpr int kMaxK = 32;

// Widen eight fp16 values and add them to acc.
__device__ __forceinline__ void add_f16x8(float (&acc)[8], const uint4& q)
{
    const __half2* h = reinterpret_cast<const __half2*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
    }
}

// One block per token; thread v handles 8 consecutive columns (16 bytes of
// y, 32 bytes of out), with all k <= 8 row loads in flight at once.  The
// kernel is launched after the down GEMM ends, not early beside its CTAs.
// With shared experts (n_s > 0), their rows y_s[s][t] (weight one, already
// applied) are added after the k routed slots, in ascending s.  F16OUT: the fp32 sum is rounded to fp16 once, at
// the store (16 bytes of out per thread); a value whose rounding leaves the
// fp16 range (|v| >= 65520, or NaN) is stored as such and reported as
// kStatusDeviceRange, as for y.
template <bool F16OUT>
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ y, const int32_t* __restrict__ inv,
                                                      int64_t n, int nvec, int k, const uint4* __restrict__ y_s,
                                                      int n_s, int64_t T, void* __restrict__ out_)
{
    __shared__ int s_pos[kMaxK];
    const int64_t t = blockIdx.x;
    pdl_trigger();
    pdl_wait();
    if (threadIdx.x < k) {
        int p = __ldg(inv + t * k + threadIdx.x);
        if ((unsigned)p >= (unsigned long long)n) {
            record_status(kStatusDeviceBounds);
            p = -1;
        }
        s_pos[threadIdx.x] = p;
    }
    __syncthreads();
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        if (k <= 8) {
            // every slot's load in flight before the sums (slot order kept)
            uint4 q[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int p = j < k ? s_pos[j] : -1;
                q[j] = p >= 0 ? __ldg(y + (int64_t)p * nvec + v) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j < k && s_pos[j] >= 0) add_f16x8(acc, q[j]);
        } else {
#pragma unroll 4
            for (int j = 0; j < k; ++j) {
                const int p = s_pos[j];
                if (p >= 0) add_f16x8(acc, __ldg(y + (int64_t)p * nvec + v));
            }
        }
        for (int sh = 0; sh < n_s; ++sh) add_f16x8(acc, __ldg(y_s + ((int64_t)sh * T + t) * nvec + v));
        if constexpr (F16OUT) {
            bool bad = false;
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                bad |= !(fabsf(acc[2 * i]) < 65520.0f) || !(fabsf(acc[2 * i + 1]) < 65520.0f);
                const __half2 h2 = __floats2half2_rn(acc[2 * i], acc[2 * i + 1]);
                pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            static_cast<uint4*>(out_)[t * nvec + v] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            if (bad) record_status(kStatusDeviceRange);
        } else {
            float4* o = static_cast<float4*>(out_) + (t * nvec + v) * 2;
            o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
    }
}

}  // namespace combine
}  // namespace moe
