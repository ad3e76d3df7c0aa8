/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse Mixture-of-Experts block forward.
 *
 * The operation is the forward pass of a top-k routed MoE block as defined by
 * the article "Qwen3MoeSparseMoeBlock performance optimisation in practice"
 * (parallelising a sparse mixture-of-experts system), section 1: the forward()
 * code and the four-stage workflow above it (router linear + softmax,
 * top-k selection, per-expert computation, routing-weighted aggregation),
 * restaged in its section 2.2 as route -> sort tokens by expert -> batched
 * expert compute -> scatter back.  Notation: T tokens, d hidden size, E
 * experts, k experts per token, f expert intermediate size, M = T*k
 * token-expert assignments.
 *
 *   logits[t,e] = sum_i x[t,i] * W_router[i,e] + bias[e]     (fp32)
 *   p[t,:]      = softmax over e of logits[t,:]                (fp32)
 *   ids[t,:]    = the k experts with the largest p, in descending order;
 *                 equal values rank the lower expert index first
 *   w[t,j]      = p[t, ids[t,j]]                      (NOT renormalised)
 *   h           = silu(x[t] . W_gate[e]) * (x[t] . W_up[e]),  silu(z) = z/(1+e^-z)
 *   y[t,j]      = w[t,j] * (h . W_down[e]),  e = ids[t,j]      (fp32, stored fp16)
 *   out[t]      = sum_j y[t,j]                                  (fp32)
 * Precision: bf16 inputs, fp32 accumulation everywhere.  h is rounded to
 * bf16 once, because it is the operand of the second bf16 tensor-core GEMM.
 * Each slot's contribution y is computed in fp32 and stored once as IEEE
 * fp16 (11-bit significand, relative error <= 2^-11): it is the block's
 * largest intermediate, and fp16 keeps the output within its tolerance
 * where bf16 would not.  The k-way sum and out stay fp32.  A y outside the
 * fp16 range (|y| >= 65520) or NaN is stored as inf / NaN and reported as
 * MOE_ERR_DEVICE_RANGE.
 * Types at the boundary: out is fp32 and y fp16, where a bf16 interface
 * would round both to bf16.  Rounding out to bf16 alone puts the worst
 * element at about 0.024 x RMS from the exact fp64 result on the
 * Qwen3-shaped layer (a CPU emulation of the rounding points), above the
 * block's 0.02 x RMS tolerance; a bf16 y alone gives 0.022 x RMS; fp16 y
 * with fp32 out gives 0.012 x RMS.
 * The optional per-expert bias follows the gate G(x) = Softmax(W_g x + b_g)
 * of the Hunyuan-Large overview page, section 2.1.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named x, w_*, h, x_perm are DEVICE pointers to bf16 (IEEE
 *   bfloat16 bit patterns, type moe_bf16); y is a DEVICE pointer to IEEE
 *   fp16 bit patterns (type moe_f16); out is a DEVICE pointer to fp32.  All are row-major, contiguous and 16-byte aligned.  Other int32 /
 *   fp32 arrays are device pointers, 4-byte aligned.
 *   The caller owns every buffer; the library never allocates, frees or
 *   synchronises (except moe_get_status), in line with the article's
 *   "memory pre-allocation" point (section 2.1, point 3).
 * - Work is enqueued on `stream` and runs asynchronously; a return value of
 *   MOE_OK means the arguments were valid and every launch was accepted.
 * - Errors detected on the device (an expert id out of range, corrupt group
 *   offsets, a pipeline wait that ran past its time limit, a y value outside
 *   the fp16 range) are written to a
 *   per-device status word and reported by moe_get_status.  The kernel that
 *   detects one skips the offending access and finishes without faulting.
 * - Shapes (MOE_ERR_UNSUPPORTED_SHAPE otherwise):
 *     d % 64 == 0 and 64 <= d <= 32768;  f % 64 == 0 and 64 <= f <= 65536;
 *     E % 8 == 0 and 8 <= E <= 512;  1 <= k <= min(E, 32);
 *     0 <= T and T*k < 2^31.  T == 0 is a valid no-op.
 * - The device must be compute capability 10.0 (B200); the library carries
 *   sm_100a code only (MOE_ERR_UNSUPPORTED_DEVICE otherwise).
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* IEEE bfloat16 bit pattern. */
typedef uint16_t moe_bf16;
/* IEEE binary16 (fp16) bit pattern. */
typedef uint16_t moe_f16;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,         /* null / misaligned pointer, negative size */
    MOE_ERR_UNSUPPORTED_SHAPE = 2,   /* shape outside the limits listed above */
    MOE_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes below the *_workspace_size value */
    MOE_ERR_CUDA = 4,                /* a CUDA runtime call or a launch failed */
    MOE_ERR_DEVICE_TIMEOUT = 5,      /* device: a pipeline wait ran past its limit */
    MOE_ERR_DEVICE_BOUNDS = 6,       /* device: index data out of range (ids, offsets, inv) */
    MOE_ERR_UNSUPPORTED_DEVICE = 7,  /* not a compute-capability 10.0 GPU */
    MOE_ERR_STATIC_SCRATCH_TOO_SMALL = 8, /* moe_permute_static: E * ceil(T/64) > 262144 */
    MOE_ERR_DEVICE_RANGE = 9         /* device: a y value outside the fp16 range, or NaN */
} moe_status_t;

/* Human-readable name of a status code (static string, never NULL). */
const char* moe_strerror(int status);

/* ABI version of this header (major * 100 + minor). */
int moe_version(void);

/*
 * Bytes of scratch that moe_forward needs for these sizes (0 if the shape is
 * unsupported).  The pieces, each 256-byte aligned, are: topk ids and
 * weights [M], counts [E], offsets [E+1], per-chunk group bases, perm / inv /
 * w_perm [M], x_perm [M,d] bf16 (the rows of x in grouped order, which the
 * gate/up GEMM reads; moe_forward builds it), h [M,f] bf16 and y [M,d] fp16.
 * Only moe_forward_ex with MOE_FLAG_FUSED_GATHER leaves x_perm unwritten
 * (its gate/up GEMM gathers the rows of x through perm itself); the size
 * still includes it.
 */
size_t moe_workspace_size(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f);

/* Bytes of scratch that moe_route needs: 0 for every supported shape (the
 * logits stay on chip).  Kept so that callers size the argument the same
 * way for every entry point. */
size_t moe_route_workspace_size(int64_t T, int64_t d, int64_t E);

/* Bytes of scratch that moe_permute needs (per-chunk expert counts). */
size_t moe_permute_workspace_size(int64_t T, int64_t E, int64_t k);

/*
 * Stage 1-2: router GEMM, fp32 softmax over E, top-k (section 1: gate
 * linear, softmax over the experts, topk; no renormalisation follows).
 *   x        [T, d]    bf16
 *   w_router [d, E]    bf16
 *   bias     [E]       fp32, or NULL for no bias
 *   topk_ids [T, k]    int32 out, slot j = j-th largest probability
 *   topk_w   [T, k]    fp32  out, the softmax probability of that expert
 *   workspace          device scratch of moe_route_workspace_size bytes
 *                      (NULL when that is 0), 16-byte aligned
 * One kernel: logits are accumulated in fp32 on the tensor cores over the
 * whole hidden dimension, stay in tensor memory and are never rounded to
 * bf16; softmax and top-k run in the same kernel's epilogue.
 * Selection compares the fp32 logits (softmax is monotone); ties go to the
 * lower expert index.
 */
int moe_route(const moe_bf16* x, const moe_bf16* w_router, const float* bias,
              int64_t T, int64_t d, int64_t E, int64_t k,
              int32_t* topk_ids, float* topk_w,
              void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Flag of moe_route_ex and moe_forward_ex: renormalise the routing
 * weights, w[t,j] = p[t,ids[t,j]] / sum_m p[t,ids[t,m]] (each token's k
 * weights sum to one).  Not part of the article's listing, which keeps the
 * top-k probabilities as they are; the default (no flag) follows the
 * listing. */
#define MOE_FLAG_RENORMALIZE 2u

/*
 * moe_route with flags: 0 or MOE_FLAG_RENORMALIZE (other bits:
 * MOE_ERR_INVALID_ARG).  Same ids as moe_route; with the flag each weight
 * is exp(l - max) divided by the sum of exp(l_m - max) over the token's k
 * selected experts.
 */
int moe_route_ex(const moe_bf16* x, const moe_bf16* w_router, const float* bias,
                 int64_t T, int64_t d, int64_t E, int64_t k,
                 int32_t* topk_ids, float* topk_w,
                 void* workspace, size_t workspace_bytes, cudaStream_t stream, unsigned flags);

/*
 * Token reordering by expert (section 2.2: sort_tokens_by_expert, then
 * gather hidden states and routing weights in that order).
 *   topk_ids [T, k] int32 in (each in [0, E); otherwise MOE_ERR_DEVICE_BOUNDS
 *                   is reported and those assignments are skipped)
 *   topk_w   [T, k] fp32 in
 *   counts   [E]    int32 out: assignments per expert
 *   offsets  [E+1]  int32 out: exclusive prefix sum, offsets[E] = T*k
 *   perm     [T*k]  int32 out: perm[pos] = t*k + j (grouped row -> assignment)
 *   inv      [T*k]  int32 out: inv[t*k + j] = pos
 *   x_perm   [T*k, d] bf16 out: x_perm[pos] = x[perm[pos] / k]; may be NULL
 *                   to skip the row gather
 *   w_perm   [T*k]  fp32 out: w_perm[pos] = topk_w[perm[pos]]
 *   workspace       device scratch of moe_permute_workspace_size bytes
 * Inside one expert's group the assignments keep ascending t*k + j order,
 * so the result is deterministic and bit-reproducible.
 */
int moe_permute(const moe_bf16* x, const int32_t* topk_ids, const float* topk_w,
                int64_t T, int64_t d, int64_t E, int64_t k,
                int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                moe_bf16* x_perm, float* w_perm,
                void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * moe_permute for callers that cannot allocate device memory when they call
 * it -- for example a plugin inside an inference engine that plans all
 * device memory ahead of time and may not allocate while enqueueing work, or
 * a latency-critical loop that cannot afford cudaMalloc's implicit device
 * synchronisation.  (The pages have no counterpart: this is an interface
 * convenience, not part of the method.)  Same arguments, outputs and
 * results as moe_permute, without the workspace: the per-chunk expert counts
 * live in a fixed 1 MiB array inside the library, which every GPU that loads
 * the library keeps until the process exits.
 *   Limit: E * ceil(T / 64) <= 262144 (for E = 128: T <= 131072); larger
 *          sizes return MOE_ERR_STATIC_SCRATCH_TOO_SMALL.
 *   The call allocates nothing and calls no allocating routine.  The first
 *   call on each device looks up the array's device address (a one-time
 *   set-up for that device, repeated once in a new context if the caller
 *   destroyed the old one with cudaDeviceReset); make that first call before
 *   any stream capture.
 *   All calls share the one array and it keeps the last call's contents;
 *   each call writes every entry it later reads, so nothing needs clearing,
 *   but calls whose work overlaps on the GPU (for example on two streams)
 *   race on the array and must be serialised by the caller.
 */
int moe_permute_static(const moe_bf16* x, const int32_t* topk_ids, const float* topk_w,
                       int64_t T, int64_t d, int64_t E, int64_t k,
                       int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                       moe_bf16* x_perm, float* w_perm, cudaStream_t stream);

/*
 * Batched expert compute (section 2.1, point 1: the experts' weights stacked
 * into one buffer and evaluated together; section 2.2 parallel_expert_compute)
 * as two grouped GEMMs on the tcgen05 tensor cores:
 *   h[pos] = silu(x_perm[pos] . W_gate[e]) * (x_perm[pos] . W_up[e])
 *   y[pos] = w_perm[pos] * (h[pos] . W_down[e])
 * for offsets[e] <= pos < offsets[e+1].
 *   x_perm  [M, d] bf16,  w_perm [M] fp32,  offsets [E+1] int32 (device)
 *   w_gate, w_up [E, d, f] bf16;  w_down [E, f, d] bf16
 *   h [M, f] bf16 out (also the caller's scratch),  y [M, d] fp16 out
 * offsets must be non-decreasing with offsets[0] = 0 and offsets[E] = M;
 * otherwise MOE_ERR_DEVICE_BOUNDS is reported and nothing is written.
 */
int moe_expert_ffn(const moe_bf16* x_perm, const float* w_perm, const int32_t* offsets,
                   const moe_bf16* w_gate, const moe_bf16* w_up, const moe_bf16* w_down,
                   int64_t M, int64_t d, int64_t E, int64_t f,
                   moe_bf16* h, moe_f16* y, cudaStream_t stream);

/*
 * Weighted aggregation back to token order (section 1, stage 4; section 2.2
 * scatter_outputs), without atomics:
 *   out[t] = sum_{j = 0..k-1} y[inv[t*k + j]]   (fp32 sum in slot order)
 *   y [T*k, d] fp16 (already multiplied by the routing weight; widened to
 *   fp32 before the sum),
 *   inv [T*k] int32 (entries outside [0, T*k) are reported as
 *   MOE_ERR_DEVICE_BOUNDS and skipped), out [T, d] fp32.
 */
int moe_combine(const moe_f16* y, const int32_t* inv, int64_t T, int64_t d, int64_t k,
                float* out, cudaStream_t stream);

/*
 * The whole block: moe_route -> moe_permute -> moe_expert_ffn -> moe_combine
 * on one stream, with every intermediate in `workspace`
 * (moe_workspace_size bytes).  Gives bit-identical results to calling the
 * four stages one by one.
 *   out          [T, d] fp32 out
 *   topk_ids_out [T, k] int32 out, or NULL (kept in the workspace)
 *   topk_w_out   [T, k] fp32 out, or NULL
 */
int moe_forward(const moe_bf16* x, const moe_bf16* w_router, const float* bias,
                const moe_bf16* w_gate, const moe_bf16* w_up, const moe_bf16* w_down,
                int64_t T, int64_t d, int64_t E, int64_t k, int64_t f,
                float* out, int32_t* topk_ids_out, float* topk_w_out,
                void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* moe_forward_ex flag: the gate/up GEMM gathers its operand rows from x
 * through the permutation while it loads them, instead of reading a
 * materialised x_perm.  Same results bit for bit. */
#define MOE_FLAG_FUSED_GATHER 1u

/* moe_forward_ex flag: `out` is [T, d] fp16 instead of fp32.  The combine
 * sums in fp32 exactly as without the flag and rounds each sum to fp16
 * (round to nearest even) once, at the store, so the result equals the
 * fp32 output rounded to fp16 bit for bit; it halves the bytes written and
 * read back.  An output whose rounding leaves the fp16 range (|v| >= 65520)
 * or is NaN is stored as such and reported as MOE_ERR_DEVICE_RANGE.  The
 * article's block returns bf16 (section 1); fp16 keeps three more mantissa
 * bits.  Accepted by moe_forward_ex only. */
#define MOE_FLAG_OUT_F16 4u

/*
 * moe_forward with options.  events (may be NULL): n_events >= 6
 * caller-created CUDA events recorded on `stream` before routing, after
 * routing, after the permutation, after the gate/up GEMM, after the down
 * GEMM and after the combine, for timing stages; a NULL entry skips that
 * boundary.  A recorded event makes the next kernel wait for the previous
 * one to finish (it cannot begin its launch early), so record only the
 * boundaries you need.  flags: any of MOE_FLAG_FUSED_GATHER,
 * MOE_FLAG_RENORMALIZE and MOE_FLAG_OUT_F16 (other bits:
 * MOE_ERR_INVALID_ARG).  out: fp32 [T, d], or fp16 [T, d] with
 * MOE_FLAG_OUT_F16 (16-byte aligned either way).  Without
 * MOE_FLAG_RENORMALIZE and MOE_FLAG_OUT_F16 the arithmetic is identical to
 * moe_forward.
 *
 * Every kernel of the library but the combine is launched with
 * programmatic dependent launch: it may begin launching while the previous
 * kernel on the stream drains, and waits for that kernel's completion before
 * its first global memory access.  The combine starts after the down GEMM
 * ends (waiting beside the GEMM's CTAs measured slower).
 */
int moe_forward_ex(const moe_bf16* x, const moe_bf16* w_router, const float* bias,
                   const moe_bf16* w_gate, const moe_bf16* w_up, const moe_bf16* w_down,
                   int64_t T, int64_t d, int64_t E, int64_t k, int64_t f,
                   void* out, int32_t* topk_ids_out, float* topk_w_out,
                   void* workspace, size_t workspace_bytes, cudaStream_t stream,
                   cudaEvent_t* events, int n_events, unsigned flags);

/*
 * Shared experts (optional; not in the article's block).  n_shared SwiGLU
 * experts that every token passes through with weight one, on top of its k
 * routed experts -- the "shared expert" routing of the Hunyuan-Large
 * overview page, section 2.1:
 *   out[t] = sum_j y[t,j] + sum_{s = 0..n_shared-1} down_s(silu(gate_s x[t]) * up_s x[t])
 * with the shared sum added after the routed slots, in ascending s, in fp32.
 *   w_gate_s, w_up_s [n_shared, d, f_shared] bf16;  w_down_s [n_shared, f_shared, d] bf16
 *   1 <= n_shared <= 8; f_shared follows the rules for f.
 * Each shared expert runs through the same grouped GEMMs as one group of all
 * T rows of x (no permutation).
 */

/* Bytes of scratch for moe_forward_shared (0 if a shape is unsupported). */
size_t moe_workspace_size_shared(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f,
                                 int64_t n_shared, int64_t f_shared);

/* Stage: y_s[s][t] = down_s(silu(gate_s x[t]) * up_s x[t]) for every shared
 * expert s, stored fp16 (range errors as for y).  h_s [T, f_shared] bf16 is
 * the caller's scratch; y_s is [n_shared, T, d] fp16. */
int moe_shared_ffn(const moe_bf16* x, const moe_bf16* w_gate_s, const moe_bf16* w_up_s,
                   const moe_bf16* w_down_s, int64_t T, int64_t d, int64_t n_shared, int64_t f_shared,
                   moe_bf16* h_s, moe_f16* y_s, cudaStream_t stream);

/* Stage: moe_combine plus the shared rows: out[t] = sum_j y[inv[t*k+j]] +
 * sum_s y_s[s][t] (fp32, routed slots first, then ascending s).
 * n_shared = 0 is moe_combine (y_s may then be NULL). */
int moe_combine_shared(const moe_f16* y, const int32_t* inv, const moe_f16* y_s, int64_t n_shared,
                       int64_t T, int64_t d, int64_t k, float* out, cudaStream_t stream);

/* The whole block with shared experts: moe_forward_ex's stages, with the
 * shared GEMMs after the routed down GEMM (inside the "after down" event)
 * and moe_combine_shared; workspace of moe_workspace_size_shared bytes.
 * events and flags as for moe_forward_ex, except MOE_FLAG_OUT_F16 (out stays
 * fp32; the flag gives MOE_ERR_INVALID_ARG). */
int moe_forward_shared(const moe_bf16* x, const moe_bf16* w_router, const float* bias,
                       const moe_bf16* w_gate, const moe_bf16* w_up, const moe_bf16* w_down,
                       const moe_bf16* w_gate_s, const moe_bf16* w_up_s, const moe_bf16* w_down_s,
                       int64_t T, int64_t d, int64_t E, int64_t k, int64_t f,
                       int64_t n_shared, int64_t f_shared,
                       float* out, int32_t* topk_ids_out, float* topk_w_out,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream,
                       cudaEvent_t* events, int n_events, unsigned flags);

/*
 * Token rounding (optional; an approximation, not the article's block): the
 * "token rounding" scheduling of the SonicMoE comparison page (core
 * difference 3), which adjusts how many tokens each expert receives so the
 * grouped GEMMs need no tile padding.  The page's pseudocode is garbled; the
 * rule implemented, per expert e and independently of the other experts,
 * starting from the top-k routing (c tokens routed to e, r = c mod tile):
 *   r == 0         unchanged;
 *   2 r <= tile    drop the r routed tokens with the smallest p[t,e]
 *                  (equal p: the larger token index first);
 *   2 r >  tile    add the tile - r unrouted tokens with the largest p[t,e]
 *                  (equal p: the smaller token index first) when there are
 *                  that many, else drop r as above.
 * Every count becomes a multiple of `tile` (256 matches the CTA-pair GEMM
 * tile, leaving it no padding).  A token's weight for each expert it keeps or
 * gains is the softmax probability p[t,e]; a token can end with more or
 * fewer than k experts (or none):
 *   out[t] = sum over its experts e, ascending, of p[t,e] * expert_e(x[t]).
 * Limits: T <= 2^20, 1 <= tile <= 65536, T*k + E*(tile-1) < 2^31.
 */

/* Bytes of scratch for moe_forward_rounded (0 if a shape is unsupported). */
size_t moe_workspace_size_rounded(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, int64_t tile);

/*
 * The block with token rounding.  out [T, d] fp32.  counts_out [E] int32 (or
 * NULL): the rounded token count of every expert.  rows_out [T, E] int32 (or
 * NULL): the grouped row of (t, e), -1 where token t does not go to expert e
 * (so rows_out >= 0 is the rounded routing mask).  events as for
 * moe_forward_ex (the "after permute" event follows the rounding).
 */
int moe_forward_rounded(const moe_bf16* x, const moe_bf16* w_router, const float* bias,
                        const moe_bf16* w_gate, const moe_bf16* w_up, const moe_bf16* w_down,
                        int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, int64_t tile,
                        float* out, int32_t* counts_out, int32_t* rows_out,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream,
                        cudaEvent_t* events, int n_events);

/*
 * Backward of the block (optional; the article's block is forward only): the
 * gradient of L = sum_t dout[t] . out[t] with respect to x, W_router, the
 * bias and the three expert weight tensors, following the memory rule of
 * the SonicMoE comparison page ("SonicMoE vs conventional MoE", core
 * difference 1): nothing from the forward is kept beyond the inputs; the
 * routing, the permutation and the expert activations g, u and h are
 * recomputed.  With e = ids[t][j], w = w[t][j], s = 1/(1+e^-g):
 *   dh          = w * dout[t] . W_down[e]^T
 *   dg          = dh * u * s * (1 + g * (1 - s)),   du = dh * g * s
 *   dW_down[e] += (w h)^T dout[t],  dW_gate[e] += x[t]^T dg,  dW_up[e] += x[t]^T du
 *   dx[t]      += dg . W_gate[e]^T + du . W_up[e]^T
 *   dw_j        = dout[t] . (h . W_down[e])          (the routing weight's gradient)
 *   dp[e]       = dw_j at e = ids[t][j], else 0      (with MOE_FLAG_RENORMALIZE:
 *                 (dw_j - sum_m w_m dw_m) / S, S = sum of the k probabilities)
 *   dlogit      = p * (dp - sum_e p_e dp_e)
 *   dW_router  += x[t]^T dlogit,  dbias += dlogit,  dx[t] += dlogit . W_router^T
 * The top-k choice itself passes no gradient.
 *   dout [T, d] fp32 in; dx [T, d] fp32 out; dw_router [d, E], dbias [E]
 *   (NULL to skip), dw_gate / dw_up [E, d, f], dw_down [E, f, d]: fp32 out
 *   (with MOE_FLAG_GRAD_BF16: dw_router, dw_gate, dw_up and dw_down bf16,
 *   each the fp32 result rounded once; dx and dbias stay fp32), overwritten
 *   (experts no token selects get zeros).  All 16-byte aligned.
 * Precision: the GEMM operands are bf16 (x, the weights, dout, dg, du, w h
 * and dlogit rounded once each), every sum fp32; each slot's contribution
 * to dx (dg . W_gate^T + du . W_up^T) is rounded to bf16 once before the
 * fp32 sum over the token's k slots.  flags: any of MOE_FLAG_RENORMALIZE
 * (the routing the forward used) and MOE_FLAG_GRAD_BF16.  Workspace:
 * moe_backward_workspace_size bytes, 256-byte aligned; grouped rows are
 * padded so that each expert's group starts on a 64-row boundary.
 */
size_t moe_backward_workspace_size(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f);

/* moe_backward flag: the weight gradients are bf16 (the fp32 accumulators
 * rounded to nearest even once, at the store), half the bytes of the
 * weight-gradient GEMMs' outputs, which bound those GEMMs' time. */
#define MOE_FLAG_GRAD_BF16 8u

int moe_backward(const moe_bf16* x, const moe_bf16* w_router, const float* bias,
                 const moe_bf16* w_gate, const moe_bf16* w_up, const moe_bf16* w_down, const float* dout,
                 int64_t T, int64_t d, int64_t E, int64_t k, int64_t f,
                 float* dx, void* dw_router, float* dbias, void* dw_gate, void* dw_up, void* dw_down,
                 void* workspace, size_t workspace_bytes, cudaStream_t stream, unsigned flags);

/*
 * Row gather for moving grouped rows between layouts (the expert-parallel
 * dispatch regroups the rows it receives by local expert and returns them in
 * the order they came; the pages' hierarchical all-to-all of the
 * Hunyuan-Large overview, section 5.1, leaves the layout open):
 *   dst[i] = src[idx[i]] for i < n, whole rows of row_bytes bytes
 *   src [n_src rows], dst [n rows]: device; row_bytes % 4 == 0; 16-byte
 *   aligned when row_bytes % 16 == 0 (copied in 16-byte vectors), else 4-byte
 *   idx [n] int32 device; an index outside [0, n_src) is reported as
 *   MOE_ERR_DEVICE_BOUNDS and its row is zero-filled.
 */
int moe_gather_rows(const void* src, const int32_t* idx, int64_t n_src, int64_t n, int64_t row_bytes, void* dst,
                    cudaStream_t stream);

/*
 * Synchronises `stream`, then returns and clears the current device's status
 * word (MOE_OK if no device-side error was recorded since the last call).
 */
int moe_get_status(cudaStream_t stream);

/*
 * Upper bound, in nanoseconds, on any single pipeline wait inside the
 * library's kernels on the current device (default 1e9).  A wait that runs
 * past it records MOE_ERR_DEVICE_TIMEOUT and the kernel winds down
 * without faulting: before it frees its tensor memory or exits, each CTA
 * waits for its own copies and MMAs still in flight, for up to the larger of
 * this limit and one second.  Values <= 0 restore the default; values below
 * 1e6 (1 ms) are raised to 1e6.
 */
int moe_set_wait_limit_ns(int64_t limit_ns);

/*
 * Failure-path self test: launches one block whose bounded wait on a barrier
 * that nothing signals runs out after `limit_ns`; afterwards
 * moe_get_status reports MOE_ERR_DEVICE_TIMEOUT.  Needs no input data.
 */
int moe_selftest_wait_timeout(int64_t limit_ns, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
