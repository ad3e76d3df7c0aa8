// combine.cuh -- routing-weighted aggregation back to token order.
//
// Stage 4 of "Qwen3MoeSparseMoeBlock performance optimisation in practice"
// (section 1: expert outputs summed per token, weighted by the routing
// weights; section 2.2 scatter_outputs).  The weight is already folded into
// y by the down-projection epilogue, so each token gathers its k grouped
// fp32 rows through inv and sums them in fp32 in slot order -- a gather, not
// a scatter-add, so no atomics and a deterministic result.  The output stays
// fp32: the accumulation is never rounded to a narrower type.
#pragma once

#include "status.cuh"

namespace moe {
namespace combine {

constexpr int kMaxK = 32;

// One block per token; thread v handles 4 consecutive columns (16 bytes).
__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ y, const int32_t* __restrict__ inv,
                                                      int64_t n, int nvec, int k, float4* __restrict__ out)
{
    __shared__ int s_pos[kMaxK];
    const int64_t t = blockIdx.x;
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
        float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll 4
        for (int j = 0; j < k; ++j) {
            const int p = s_pos[j];
            if (p >= 0) {
                const float4 q = __ldg(y + (int64_t)p * nvec + v);
                acc.x += q.x;
                acc.y += q.y;
                acc.z += q.z;
                acc.w += q.w;
            }
        }
        out[t * nvec + v] = acc;
    }
}

}  // namespace combine
}  // namespace moe
