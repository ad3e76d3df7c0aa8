// moe.cu -- the C ABI declared in include/moe.h: argument validation,
// workspace planning, TMA descriptor encoding and kernel launches.  All
// device code is included here so the library is one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "moe.h"

#include "status.cuh"
#include "ptx.cuh"
#include "route.cuh"
#include "rounding.cuh"
#include "permute.cuh"
#include "grouped_gemm.cuh"
#include "grouped_gemm_pair.cuh"
#include "combine.cuh"
#include "grouped_gemm_bwd.cuh"
#include "backward.cuh"

namespace {

// ------------------------------------------------------------ self test
__global__ void wait_timeout_kernel(unsigned long long limit_ns)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        moe::mbar_init(&bar, 1);
        moe::fence_mbar_init();
    }
    __syncthreads();
    // Nothing ever arrives on `bar`: the bounded wait must give up.
    if (threadIdx.x == 0) moe::mbar_wait(&bar, 0, limit_ns);
    __syncthreads();
}

// ------------------------------------------------------ per-device state
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int kMaxDevices = 64;

// Per-device state lives as long as the context it was set up in: kernel
// attributes and symbol addresses belong to a context, and a caller may
// destroy the device's primary context (cudaDeviceReset) and carry on in a
// new one.  Each entry records the unique id of its context and is set up
// again when the current context's id differs.
struct DeviceState {
    bool init = false;
    bool supported = false;
    int sm_count = 0;
    int max_pairs = 0;  // co-resident 2-CTA clusters of the pair GEMM
    unsigned long long ctx_id = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

// Process-unique id of the calling thread's current context on device `dev`
// (its primary context is made current first if the thread has none).
// Called with g_mu held.
int current_context_id(int dev, unsigned long long* id)
{
    cudaDriverEntryPointQueryResult q;
    if (!g_ctx_get_current) {
        void* fn = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 12000, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return MOE_ERR_CUDA;
        g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    }
    if (!g_ctx_get_id) {
        void* fn = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return MOE_ERR_CUDA;
        g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(fn);
    }
    CUcontext ctx = nullptr;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return MOE_ERR_CUDA;
    if (!ctx) {
        // no context current on this thread yet: cudaSetDevice initialises the
        // device's primary context and makes it current
        if (cudaSetDevice(dev) != cudaSuccess || g_ctx_get_current(&ctx) != CUDA_SUCCESS || !ctx)
            return MOE_ERR_CUDA;
    }
    return g_ctx_get_id(ctx, id) == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

constexpr int kMaxDynSmem = 227 * 1024;

// moe_forward's variant: the gate/up GEMM reads a materialised x_perm (the
// fused row gather measured slower on B200, see MOE_FLAG_FUSED_GATHER).
constexpr unsigned kDefaultForwardFlags = 0;

// Grouped GEMMs on CTA pairs (tcgen05 cta_group::2) instead of single CTAs.
#ifndef MOE_GEMM_PAIR
#define MOE_GEMM_PAIR 1
#endif

// Programmatic dependent launch for every kernel of the library: a launch
// may begin while the previous kernel on the stream drains; each kernel
// waits (griddepcontrol.wait) before its first global-memory access.
#ifndef MOE_PDL
#define MOE_PDL 1
#endif

// A launch without the PDL attribute: the kernel starts once its
// predecessor on the stream has finished, and its grid-dependency wait is a
// no-op.  For the combine: launched early it would wait in blocks resident
// beside the down GEMM's CTAs (it needs no shared memory), which measured
// 3-4 us slower per forward than waiting for the GEMM to end.
template <typename... KArgs, typename... Args>
int launch_after(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = nullptr;
    cfg.numAttrs = 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// cudaLaunchKernelEx with the PDL attribute and, for cluster > 1, a 1-D
// cluster of that many CTAs.
template <typename... KArgs, typename... Args>
int launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, unsigned cluster,
           Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    if (cluster > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    if (MOE_PDL) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

template <int EPI, int SC = moe::gemm::kSlabCols>
int launch_pair_gemm(const DeviceState& st, int64_t work, const CUtensorMap& ta, const CUtensorMap& tb0,
                     const CUtensorMap& tb1, const CUtensorMap& tout, const moe::gemm::Params& p, cudaStream_t s)
{
    int64_t pairs = st.max_pairs > 0 ? st.max_pairs : st.sm_count / 2;
    if (work < pairs) pairs = work;
    if (pairs < 1) pairs = 1;
    return launch(moe::gemm::grouped_gemm_pair_kernel<EPI, SC>, dim3((unsigned)(2 * pairs)),
                  dim3(moe::gemm::kThreads), moe::gemm::pair_smem_bytes<EPI, SC>(), s, 2u, ta, tb0, tb1, tout, p);
}

int setup_device(DeviceState** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& st = g_dev[dev];
    unsigned long long ctx_id = 0;
    if (current_context_id(dev, &ctx_id)) return MOE_ERR_CUDA;
    if (st.init && st.ctx_id != ctx_id) st = DeviceState{};  // a new context: set up again
    if (!st.init) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        st.supported = (major == 10 && minor == 0);
        st.sm_count = sms;
        if (st.supported) {
            if (!g_encode) {
                void* fn = nullptr;
                cudaDriverEntryPointQueryResult q;
                if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
                        cudaSuccess ||
                    q != cudaDriverEntryPointSuccess || !fn)
                    return MOE_ERR_CUDA;
                g_encode = reinterpret_cast<EncodeTiledFn>(fn);
            }
            cudaError_t e = cudaSuccess;
            e = e ? e : cudaFuncSetAttribute(moe::route::route_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::route::route_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::route::route_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::route::route_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::route::route_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::rounding::round_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::gemm::grouped_gemm_kernel<moe::gemm::kSwiGLU, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::gemm::grouped_gemm_kernel<moe::gemm::kSwiGLU, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::gemm::grouped_gemm_kernel<moe::gemm::kWeighted, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::gemm::grouped_gemm_pair_kernel<moe::gemm::kSwiGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::gemm::grouped_gemm_pair_kernel<moe::gemm::kWeighted>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::gemm::grouped_gemm_pair_kernel<moe::gemm::kWeighted, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::bwd::pair_bwd_kernel<moe::bwd::kGU>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::bwd::pair_bwd_kernel<moe::bwd::kDH>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::bwd::pair_bwd_kernel<moe::bwd::kDX>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            e = e ? e : cudaFuncSetAttribute(moe::bwd::pair_bwd_kernel<moe::bwd::kDW>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            if (e == cudaSuccess) {
                // CTA pairs that can be resident at once (clusters need two
                // SMs of one GPC, so this can be below sm_count / 2)
                cudaLaunchConfig_t cfg = {};
                cudaLaunchAttribute attr[1];
                attr[0].id = cudaLaunchAttributeClusterDimension;
                attr[0].val.clusterDim.x = 2;
                attr[0].val.clusterDim.y = 1;
                attr[0].val.clusterDim.z = 1;
                cfg.gridDim = dim3(2 * (sms / 2));
                cfg.blockDim = dim3(moe::gemm::kThreads);
                cfg.dynamicSmemBytes = moe::gemm::pair_smem_bytes<moe::gemm::kSwiGLU>();
                cfg.attrs = attr;
                cfg.numAttrs = 1;
                int n = 0;
                if (cudaOccupancyMaxActiveClusters(&n, moe::gemm::grouped_gemm_pair_kernel<moe::gemm::kSwiGLU>,
                                                   &cfg) != cudaSuccess) {
                    cudaGetLastError();  // not fatal: fall back to sm_count / 2 pairs
                    n = 0;
                }
                st.max_pairs = n;
            }
            if (e != cudaSuccess) return MOE_ERR_CUDA;
        }
        st.ctx_id = ctx_id;
        st.init = true;
    }
    if (!st.supported) return MOE_ERR_UNSUPPORTED_DEVICE;
    *out = &st;
    return MOE_OK;
}

// ------------------------------------------------------------ validation
inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_common(int64_t T, int64_t d, int64_t E, int64_t k)
{
    if (T < 0 || d <= 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (d % 64 != 0 || d > 32768) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (E % 8 != 0 || E < 8 || E > moe::gemm::kMaxE) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (k > E || k > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T * k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

int check_f(int64_t f)
{
    if (f <= 0) return MOE_ERR_INVALID_ARG;
    if (f % 64 != 0 || f > 65536) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

int launch_status()
{
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// 2-D row-major tensor map, zero fill outside the tensor.  Default: bf16
// with 128-byte swizzle (the layout the tcgen05 descriptors expect).
int make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
             uint32_t box_outer, CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
             uint32_t elem_bytes = 2, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B)
{
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * elem_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// A bf16 weight matrix [rows = k, cols] viewed as [cols/64][rows][64]
// (64-column chunks outermost), 128-byte swizzle, box of 64 rows x two
// chunks: one copy fetches 128 columns as the two 8 KB chunks an MN-major
// operand uses.  Chunks past the last column read zeros.
int make_weight_chunk_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows)
{
    cuuint64_t dims[3] = {64, rows, (cols + 63) / 64};
    cuuint64_t strides[2] = {cols * 2, 128};
    cuuint32_t box[3] = {64, 64, 2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// ---------------------------------------------------------- work shapes
inline int64_t token_chunks(int64_t T) { return (T + moe::permute::kTokensPerChunk - 1) / moe::permute::kTokensPerChunk; }

// The router keeps its logits on chip (a CTA pair that splits K exchanges
// its partial logits through distributed shared memory) and needs no
// scratch; moe_route keeps its workspace argument so that every stage entry
// point is sized the same way.
size_t route_ws_bytes(int64_t, int64_t, int64_t) { return 0; }

size_t permute_ws_bytes(int64_t T, int64_t E) { return align256((size_t)token_chunks(T) * (size_t)E * 4); }

// Workspace carve-up for moe_forward.
struct Layout {
    size_t ids, wts, counts, offsets, chunk, perm, inv, w_perm, x_perm, h, y, h_s, y_s, total;
};

// n_s shared experts of intermediate size f_s add h_s [T, f_s] bf16 (reused
// by every shared expert) and y_s [n_s, T, d] fp16.
Layout plan(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, int64_t n_s = 0, int64_t f_s = 0)
{
    const size_t M = (size_t)(T * k);
    Layout L{};
    size_t o = 0;
    L.ids = o;     o += align256(M * 4);
    L.wts = o;     o += align256(M * 4);
    L.counts = o;  o += align256((size_t)E * 4);
    L.offsets = o; o += align256((size_t)(E + 1) * 4);
    L.chunk = o;   o += permute_ws_bytes(T, E);
    L.perm = o;    o += align256(M * 4);
    L.inv = o;     o += align256(M * 4);
    L.w_perm = o;  o += align256(M * 4);
    L.x_perm = o;  o += align256(M * (size_t)d * 2);
    L.h = o;       o += align256(M * (size_t)f * 2);
    L.y = o;       o += align256(M * (size_t)d * 2);
    L.h_s = o;     o += n_s > 0 ? align256((size_t)T * (size_t)f_s * 2) : 0;
    L.y_s = o;     o += align256((size_t)n_s * (size_t)T * (size_t)d * 2);
    L.total = o;
    return L;
}

// ------------------------------------------------------------ launchers
// Router GEMM, softmax and top-k in one kernel.  With chunk_counts set, it
// also writes the per-chunk expert histogram the permutation needs.
template <int KMAX>
int launch_route(const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& tw3, moe::route::Params p,
                 unsigned tiles, cudaStream_t s)
{
    using moe::route::smem_bytes;
    // one CTA per SM: the deepest ring that fits (2 to 8 stages)
    p.stages = moe::route::kMaxStages;
    while (p.stages > 2 && smem_bytes(p.n_chunks, p.stages, p.E, p.split, p.passes) > (size_t)kMaxDynSmem)
        --p.stages;
    return launch(moe::route::route_kernel<KMAX>, dim3(tiles * (unsigned)p.split), dim3(moe::route::kThreads),
                  smem_bytes(p.n_chunks, p.stages, p.E, p.split, p.passes), s, (unsigned)p.split, tx, tw, tw3, p);
}

int run_route(const DeviceState& st, const moe_bf16* x, const moe_bf16* w_router, const float* bias, int64_t T,
              int64_t d, int64_t E, int64_t k, int32_t* ids, float* wts, int32_t* chunk_counts, bool renorm,
              cudaStream_t s, float* probs_t = nullptr, float* probs_tm = nullptr)
{
    if (T == 0) return MOE_OK;
    CUtensorMap tx, tw;
    int rc = make_map(&tx, x, (uint64_t)d, (uint64_t)T, 64, moe::route::kBM);
    if (rc) return rc;
    rc = make_map(&tw, w_router, (uint64_t)E, (uint64_t)d, 64, 64);
    if (rc) return rc;
    // E a multiple of 64: every expert chunk of a k-block in one 3-D copy
    // (W_router viewed as [E/64][d][64]); otherwise one copy per chunk, the
    // last one zero-filled past E
    CUtensorMap tw3 = tw;
    const bool w_one_copy = E % 64 == 0 && E / 64 <= 16;
    if (w_one_copy) {
        cuuint64_t dims[3] = {64, (cuuint64_t)d, (cuuint64_t)(E / 64)};
        cuuint64_t strides[2] = {(cuuint64_t)E * 2, 128};
        cuuint32_t box[3] = {64, 64, (cuuint32_t)(E / 64)};
        cuuint32_t estr[3] = {1, 1, 1};
        if (g_encode(&tw3, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<moe_bf16*>(w_router), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MOE_ERR_CUDA;
    }
    const int64_t tiles = (T + moe::route::kBM - 1) / moe::route::kBM;
    moe::route::Params p;
    p.bias = bias;
    p.ids = ids;
    p.wts = wts;
    p.chunk_counts = chunk_counts;
    p.n_tchunks = (int)token_chunks(T);
    p.T = (int)T;
    p.d = (int)d;
    p.E = (int)E;
    p.k = (int)k;
    p.n_chunks = (int)((E + 63) / 64);
    p.w_one_copy = w_one_copy ? 1 : 0;
    p.stages = 0;  // set by the launcher
    uint32_t cols = 64;
    while (cols < (uint32_t)(64 * p.n_chunks)) cols <<= 1;
    p.tmem_cols = cols;
    // Split K over a CTA pair while the pairs of all tiles can be resident
    // at once: more SMs stream x.  The exchange buffer of a pair holds
    // 128 x E fp32 partials, which fits the ring for E <= 256.
    const int64_t pairs = st.max_pairs > 0 ? st.max_pairs : st.sm_count / 2;
    p.split = (E <= 256 && d >= 2 * moe::route::kBK && tiles <= pairs) ? 2 : 1;
    p.passes = (p.split == 1 && E > 256) ? 2 : 1;
    p.renorm = renorm ? 1 : 0;
    // every expert's probability, [E][T] (token rounding) or [T][E] (backward)
    p.probs = probs_t ? probs_t : probs_tm;
    p.probs_tstride = probs_t ? 1 : E;
    p.probs_estride = probs_t ? T : 1;
    // top-k list length: the power of two >= k for lane groups (k <= 8), or
    // the whole-warp rounds (k > 8)
    const unsigned ut = (unsigned)tiles;
    if (k <= 1) return launch_route<1>(tx, tw, tw3, p, ut, s);
    if (k <= 2) return launch_route<2>(tx, tw, tw3, p, ut, s);
    if (k <= 4) return launch_route<4>(tx, tw, tw3, p, ut, s);
    if (k <= 8) return launch_route<8>(tx, tw, tw3, p, ut, s);
    return launch_route<32>(tx, tw, tw3, p, ut, s);
}

// Grouping by expert.  have_hist: chunk_em already holds the per-chunk
// histogram (from the router); otherwise it is computed here.
int run_permute(const moe_bf16* x, const int32_t* ids, const float* wts, int64_t T, int64_t d, int64_t E,
                int64_t k, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv, moe_bf16* x_perm,
                float* w_perm, int32_t* chunk_em, bool have_hist, cudaStream_t s)
{
    if (T == 0) {
        // Empty batch: every group is empty.
        if (cudaMemsetAsync(counts, 0, (size_t)E * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemsetAsync(offsets, 0, (size_t)(E + 1) * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    using namespace moe::permute;
    const int nch = (int)token_chunks(T);
    const int32_t* cids = ids;
    const float* cw = wts;
    const int ik = (int)k, iE = (int)E;
    if (!have_hist && launch(hist_kernel, dim3(nch), dim3(kThreads), 0, s, 1u, cids, T, ik, iE, chunk_em, nch))
        return MOE_ERR_CUDA;
    if (launch(chunk_scan_kernel, dim3((unsigned)E), dim3(kThreads), 0, s, 1u, chunk_em, nch, counts))
        return MOE_ERR_CUDA;
    if (launch(rank_kernel<false>, dim3(nch), dim3(kThreads), 0, s, 1u, cids, cw, T, ik, iE,
               static_cast<const int32_t*>(chunk_em), nch, static_cast<const int32_t*>(counts), offsets, perm, inv,
               w_perm))
        return MOE_ERR_CUDA;
    if (x_perm) {
        if (launch(gather_kernel, dim3((unsigned)((T + kWarps - 1) / kWarps)), dim3(kThreads), 0, s, 1u,
                   reinterpret_cast<const uint4*>(x), static_cast<const int32_t*>(inv), T, ik, (int)(d / 8), T * k,
                   reinterpret_cast<uint4*>(x_perm)))
            return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

// The two grouped GEMMs.  With x_gather/perm set, the gate/up GEMM reads its
// A rows straight from x through perm (row pos -> token perm[pos] / k) and
// x_perm is not used.
int run_ffn(const DeviceState& st, const moe_bf16* x_perm, const moe_bf16* x_gather, const int32_t* perm,
            int64_t T, int64_t k, const float* w_perm, const int32_t* offsets, const moe_bf16* w_gate,
            const moe_bf16* w_up, const moe_bf16* w_down, int64_t M, int64_t d, int64_t E, int64_t f, moe_bf16* h,
            moe_f16* y, cudaStream_t s, cudaEvent_t mid_event, bool m_capacity = false)
{
    if (M == 0) {
        if (mid_event && cudaEventRecord(mid_event, s) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    using namespace moe::gemm;
    const bool gather = x_gather != nullptr;
    CUtensorMap ta1, tg, tu, ta2, td, ty;
    // In gather mode the A rows are copied by the producer warp itself; the
    // A map is unused (the x_perm map is encoded over x only as a placeholder).
    int rc = gather ? make_map(&ta1, x_gather, (uint64_t)d, (uint64_t)T, 64, kBM)
                    : make_map(&ta1, x_perm, (uint64_t)d, (uint64_t)M, 64, kBM);
    rc = rc ? rc : make_map(&tg, w_gate, (uint64_t)f, (uint64_t)(E * d), 64, 64);
    rc = rc ? rc : make_map(&tu, w_up, (uint64_t)f, (uint64_t)(E * d), 64, 64);
    rc = rc ? rc : make_map(&ta2, h, (uint64_t)f, (uint64_t)M, 64, kBM);
    rc = rc ? rc : make_map(&td, w_down, (uint64_t)d, (uint64_t)(E * f), 64, 64);
    rc = rc ? rc : make_map(&ty, y, (uint64_t)d, (uint64_t)M, kSlabCols, 32, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                            CU_TENSOR_MAP_SWIZZLE_64B);
    // the CTA-pair kernels fetch weight columns in 128-column copies
    CUtensorMap tg3, tu3, td3;
    rc = rc ? rc : make_weight_chunk_map(&tg3, w_gate, (uint64_t)f, (uint64_t)(E * d));
    rc = rc ? rc : make_weight_chunk_map(&tu3, w_up, (uint64_t)f, (uint64_t)(E * d));
    rc = rc ? rc : make_weight_chunk_map(&td3, w_down, (uint64_t)d, (uint64_t)(E * f));
    if (rc) return rc;
    const size_t smem1 = smem_bytes<kSwiGLU>();
    const size_t smem2 = smem_bytes<kWeighted>();
    const int64_t max_mtiles = (M + kBM - 1) / kBM + E;

    Params p1;
    p1.offsets = offsets;
    p1.w_perm = nullptr;
    p1.perm = perm;
    p1.x = reinterpret_cast<const __nv_bfloat16*>(x_gather);
    p1.ldx = d;
    p1.out = h;
    p1.E = (int)E;
    p1.M = (int)M;
    p1.K = (int)d;
    p1.n_out = (int)f;
    p1.n_tiles = (int)((f + 127) / 128);
    p1.k_top = (int)k;
    p1.m_capacity = m_capacity ? 1 : 0;
    const int64_t work1 = max_mtiles * p1.n_tiles;
    const unsigned grid1 = (unsigned)(work1 < st.sm_count ? work1 : st.sm_count);
    const int64_t max_pair_tiles = (M + kPairRows - 1) / kPairRows + E;
    if (MOE_GEMM_PAIR && !gather) {
        if (launch_pair_gemm<kSwiGLU>(st, max_pair_tiles * p1.n_tiles, ta1, tg3, tu3, ty, p1, s)) return MOE_ERR_CUDA;
    } else if (gather) {
        if (launch(grouped_gemm_kernel<kSwiGLU, true>, dim3(grid1), dim3(kThreads), smem1, s, 1u, ta1, tg, tu, ty, p1))
            return MOE_ERR_CUDA;
    } else {
        if (launch(grouped_gemm_kernel<kSwiGLU, false>, dim3(grid1), dim3(kThreads), smem1, s, 1u, ta1, tg, tu, ty,
                   p1))
            return MOE_ERR_CUDA;
    }
    if (mid_event && cudaEventRecord(mid_event, s) != cudaSuccess) return MOE_ERR_CUDA;

    Params p2;
    p2.offsets = offsets;
    p2.w_perm = w_perm;
    p2.perm = nullptr;
    p2.x = nullptr;
    p2.ldx = 0;
    p2.out = y;
    p2.E = (int)E;
    p2.M = (int)M;
    p2.K = (int)f;
    p2.n_out = (int)d;
    p2.n_tiles = (int)((d + kBN - 1) / kBN);
    p2.k_top = 1;
    p2.m_capacity = m_capacity ? 1 : 0;
    const int64_t work2 = max_mtiles * p2.n_tiles;
    const unsigned grid2 = (unsigned)(work2 < st.sm_count ? work2 : st.sm_count);
    if (MOE_GEMM_PAIR) {
        if (f <= kDownShortK) {  // y through 32 x 64 slabs (128-byte rows)
            CUtensorMap ty64;
            if (make_map(&ty64, y, (uint64_t)d, (uint64_t)M, 64, 32, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                         CU_TENSOR_MAP_SWIZZLE_128B))
                return MOE_ERR_CUDA;
            return launch_pair_gemm<kWeighted, 64>(st, max_pair_tiles * p2.n_tiles, ta2, td3, td3, ty64, p2, s);
        }
        return launch_pair_gemm<kWeighted>(st, max_pair_tiles * p2.n_tiles, ta2, td3, td3, ty, p2, s);
    }
    return launch(grouped_gemm_kernel<kWeighted, false>, dim3(grid2), dim3(kThreads), smem2, s, 1u, ta2, td, td, ty,
                  p2);
}

// out: fp32 [T, d], or fp16 [T, d] with f16_out.
int run_combine(const moe_f16* y, const int32_t* inv, int64_t T, int64_t d, int64_t k, void* out, cudaStream_t s,
                const moe_f16* y_s = nullptr, int64_t n_s = 0, bool f16_out = false)
{
    if (T == 0) return MOE_OK;
    const int nvec = (int)(d / 8);
    const int threads = nvec < 256 ? ((nvec + 31) / 32) * 32 : 256;
    if (f16_out)
        return launch_after(moe::combine::combine_kernel<true>, dim3((unsigned)T), dim3(threads), 0, s,
                            reinterpret_cast<const uint4*>(y), inv, T * k, nvec, (int)k,
                            reinterpret_cast<const uint4*>(y_s), (int)n_s, T, out);
    return launch_after(moe::combine::combine_kernel<false>, dim3((unsigned)T), dim3(threads), 0, s,
                        reinterpret_cast<const uint4*>(y), inv, T * k, nvec, (int)k,
                        reinterpret_cast<const uint4*>(y_s), (int)n_s, T, out);
}

// Shared experts: each is one group of all T rows of x (no permutation, no
// gather, weight one) through the same grouped GEMMs: h_s = SwiGLU input
// projections of shared expert s, y_s[s] = h_s . W_down_s[s] in fp16.
int run_shared(const DeviceState& st, const moe_bf16* x, const moe_bf16* w_gate_s, const moe_bf16* w_up_s,
               const moe_bf16* w_down_s, int64_t T, int64_t d, int64_t n_s, int64_t f_s, moe_bf16* h_s, moe_f16* y_s,
               cudaStream_t s)
{
    for (int64_t i = 0; i < n_s; ++i) {
        const int rc = run_ffn(st, x, nullptr, nullptr, T, 1, nullptr, nullptr, w_gate_s + i * d * f_s,
                               w_up_s + i * d * f_s, w_down_s + i * f_s * d, T, d, 1, f_s, h_s, y_s + i * T * d, s,
                               nullptr);
        if (rc) return rc;
    }
    return MOE_OK;
}

constexpr int64_t kMaxShared = 8;

int check_shared(const moe_bf16* w_gate_s, const moe_bf16* w_up_s, const moe_bf16* w_down_s, int64_t T,
                 int64_t n_s, int64_t f_s)
{
    if (n_s < 0 || n_s > kMaxShared) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (n_s == 0) return MOE_OK;
    int rc = check_f(f_s);
    if (rc) return rc;
    if (T > 0 && (!w_gate_s || !w_up_s || !w_down_s)) return MOE_ERR_INVALID_ARG;
    if (!aligned(w_gate_s, 16) || !aligned(w_up_s, 16) || !aligned(w_down_s, 16)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

int forward_impl(const moe_bf16* x, const moe_bf16* w_router, const float* bias, const moe_bf16* w_gate,
                 const moe_bf16* w_up, const moe_bf16* w_down, int64_t T, int64_t d, int64_t E, int64_t k, int64_t f,
                 void* out, int32_t* ids_out, float* w_out, void* ws, size_t ws_bytes, cudaStream_t s,
                 cudaEvent_t* ev, int n_ev, unsigned flags, const moe_bf16* w_gate_s = nullptr,
                 const moe_bf16* w_up_s = nullptr, const moe_bf16* w_down_s = nullptr, int64_t n_s = 0,
                 int64_t f_s = 0)
{
    int rc = check_common(T, d, E, k);
    if (rc) return rc;
    if ((rc = check_f(f))) return rc;
    if ((rc = check_shared(w_gate_s, w_up_s, w_down_s, T, n_s, f_s))) return rc;
    if (flags & ~(unsigned)(MOE_FLAG_FUSED_GATHER | MOE_FLAG_RENORMALIZE | MOE_FLAG_OUT_F16))
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !w_router || !w_gate || !w_up || !w_down || !out)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(w_gate, 16) || !aligned(w_up, 16) ||
        !aligned(w_down, 16) || !aligned(out, 16) || !aligned(bias, 4) || !aligned(ids_out, 4) ||
        !aligned(w_out, 4))
        return MOE_ERR_INVALID_ARG;
    if (ev && n_ev < 6) return MOE_ERR_INVALID_ARG;
    const Layout L = plan(T, d, E, k, f, n_s, f_s);
    if (T > 0 && (!ws || !aligned(ws, 256))) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    DeviceState* st = nullptr;
    if ((rc = setup_device(&st))) return rc;
    auto rec = [&](int i) {
        return (ev && ev[i] && cudaEventRecord(ev[i], s) != cudaSuccess) ? MOE_ERR_CUDA : MOE_OK;
    };
    if ((rc = rec(0))) return rc;
    if (T == 0) {
        for (int i = 1; i < 6; ++i)
            if ((rc = rec(i))) return rc;
        return MOE_OK;
    }
    uint8_t* w = static_cast<uint8_t*>(ws);
    int32_t* ids = ids_out ? ids_out : reinterpret_cast<int32_t*>(w + L.ids);
    float* wts = w_out ? w_out : reinterpret_cast<float*>(w + L.wts);
    int32_t* counts = reinterpret_cast<int32_t*>(w + L.counts);
    int32_t* offsets = reinterpret_cast<int32_t*>(w + L.offsets);
    int32_t* chunk = reinterpret_cast<int32_t*>(w + L.chunk);
    int32_t* perm = reinterpret_cast<int32_t*>(w + L.perm);
    int32_t* inv = reinterpret_cast<int32_t*>(w + L.inv);
    float* w_perm = reinterpret_cast<float*>(w + L.w_perm);
    moe_bf16* x_perm = reinterpret_cast<moe_bf16*>(w + L.x_perm);
    moe_bf16* h = reinterpret_cast<moe_bf16*>(w + L.h);
    moe_f16* y = reinterpret_cast<moe_f16*>(w + L.y);
    const bool gather = (flags & MOE_FLAG_FUSED_GATHER) != 0;

    if ((rc = run_route(*st, x, w_router, bias, T, d, E, k, ids, wts, chunk, (flags & MOE_FLAG_RENORMALIZE) != 0,
                        s)))
        return rc;
    if ((rc = rec(1))) return rc;
    if ((rc = run_permute(x, ids, wts, T, d, E, k, counts, offsets, perm, inv, gather ? nullptr : x_perm, w_perm,
                          chunk, true, s)))
        return rc;
    if ((rc = rec(2))) return rc;
    if ((rc = run_ffn(*st, gather ? nullptr : x_perm, gather ? x : nullptr, perm, T, k, w_perm, offsets, w_gate,
                      w_up, w_down, T * k, d, E, f, h, y, s, ev ? ev[3] : nullptr)))
        return rc;
    moe_f16* y_s = reinterpret_cast<moe_f16*>(w + L.y_s);
    if (n_s > 0 && (rc = run_shared(*st, x, w_gate_s, w_up_s, w_down_s, T, d, n_s, f_s,
                                    reinterpret_cast<moe_bf16*>(w + L.h_s), y_s, s)))
        return rc;
    if ((rc = rec(4))) return rc;
    if ((rc = run_combine(y, inv, T, d, k, out, s, y_s, n_s, (flags & MOE_FLAG_OUT_F16) != 0))) return rc;
    return rec(5);
}

// ------------------------------------------------------------ token rounding
// Rows of the rounded grouping: every expert gains fewer than `tile` rows.
inline int64_t round_capacity(int64_t T, int64_t E, int64_t k, int64_t tile) { return T * k + E * (tile - 1); }

int check_rounding(int64_t T, int64_t E, int64_t k, int64_t tile)
{
    if (tile < 1) return MOE_ERR_INVALID_ARG;
    if (tile > 65536 || T > moe::rounding::kMaxTokens || round_capacity(T, E, k, tile) >= (int64_t(1) << 31))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

struct RLayout {
    size_t ids, wts, counts, offsets, chunk, perm, inv, w_perm, probs_t, bitmaps, new_counts, offsets2, w2,
        posmap, x_perm, h, y, total;
};

RLayout plan_rounded(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, int64_t tile)
{
    const size_t M = (size_t)(T * k);
    const size_t cap = (size_t)round_capacity(T, E, k, tile);
    RLayout L{};
    size_t o = 0;
    L.ids = o;        o += align256(M * 4);
    L.wts = o;        o += align256(M * 4);
    L.counts = o;     o += align256((size_t)E * 4);
    L.offsets = o;    o += align256((size_t)(E + 1) * 4);
    L.chunk = o;      o += permute_ws_bytes(T, E);
    L.perm = o;       o += align256(M * 4);
    L.inv = o;        o += align256(M * 4);
    L.w_perm = o;     o += align256(M * 4);
    L.probs_t = o;    o += align256((size_t)E * (size_t)T * 4);
    L.bitmaps = o;    o += align256((size_t)E * (size_t)moe::rounding::bitmap_words((int)T) * 4);
    L.new_counts = o; o += align256((size_t)E * 4);
    L.offsets2 = o;   o += align256((size_t)(E + 1) * 4);
    L.w2 = o;         o += align256(cap * 4);
    L.posmap = o;     o += align256((size_t)T * (size_t)E * 4);
    L.x_perm = o;     o += align256(cap * (size_t)d * 2);
    L.h = o;          o += align256(cap * (size_t)f * 2);
    L.y = o;          o += align256(cap * (size_t)d * 2);
    L.total = o;
    return L;
}

int forward_rounded_impl(const moe_bf16* x, const moe_bf16* w_router, const float* bias, const moe_bf16* w_gate,
                         const moe_bf16* w_up, const moe_bf16* w_down, int64_t T, int64_t d, int64_t E, int64_t k,
                         int64_t f, int64_t tile, float* out, int32_t* counts_out, int32_t* posmap_out, void* ws,
                         size_t ws_bytes, cudaStream_t s, cudaEvent_t* ev, int n_ev)
{
    int rc = check_common(T, d, E, k);
    if (rc) return rc;
    if ((rc = check_f(f))) return rc;
    if ((rc = check_rounding(T, E, k, tile))) return rc;
    if (T > 0 && (!x || !w_router || !w_gate || !w_up || !w_down || !out)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(w_gate, 16) || !aligned(w_up, 16) ||
        !aligned(w_down, 16) || !aligned(out, 16) || !aligned(bias, 4) || !aligned(counts_out, 4) ||
        !aligned(posmap_out, 4))
        return MOE_ERR_INVALID_ARG;
    if (ev && n_ev < 6) return MOE_ERR_INVALID_ARG;
    const RLayout L = plan_rounded(T, d, E, k, f, tile);
    if (T > 0 && (!ws || !aligned(ws, 256))) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    DeviceState* st = nullptr;
    if ((rc = setup_device(&st))) return rc;
    auto rec = [&](int i) {
        return (ev && ev[i] && cudaEventRecord(ev[i], s) != cudaSuccess) ? MOE_ERR_CUDA : MOE_OK;
    };
    if ((rc = rec(0))) return rc;
    if (T == 0) {
        if (counts_out && cudaMemsetAsync(counts_out, 0, (size_t)E * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
        for (int i = 1; i < 6; ++i)
            if ((rc = rec(i))) return rc;
        return MOE_OK;
    }
    uint8_t* w = static_cast<uint8_t*>(ws);
    auto at = [&](size_t off) { return static_cast<void*>(w + off); };
    int32_t* ids = static_cast<int32_t*>(at(L.ids));
    float* wts = static_cast<float*>(at(L.wts));
    int32_t* counts = static_cast<int32_t*>(at(L.counts));
    int32_t* offsets = static_cast<int32_t*>(at(L.offsets));
    int32_t* chunk = static_cast<int32_t*>(at(L.chunk));
    int32_t* perm = static_cast<int32_t*>(at(L.perm));
    int32_t* inv = static_cast<int32_t*>(at(L.inv));
    float* w_perm = static_cast<float*>(at(L.w_perm));
    float* probs_t = static_cast<float*>(at(L.probs_t));
    uint32_t* bitmaps = static_cast<uint32_t*>(at(L.bitmaps));
    int32_t* new_counts = counts_out ? counts_out : static_cast<int32_t*>(at(L.new_counts));
    int32_t* offsets2 = static_cast<int32_t*>(at(L.offsets2));
    float* w2 = static_cast<float*>(at(L.w2));
    int32_t* posmap = posmap_out ? posmap_out : static_cast<int32_t*>(at(L.posmap));
    moe_bf16* x_perm = static_cast<moe_bf16*>(at(L.x_perm));
    moe_bf16* h = static_cast<moe_bf16*>(at(L.h));
    moe_f16* y = static_cast<moe_f16*>(at(L.y));
    const int64_t cap = round_capacity(T, E, k, tile);
    using namespace moe::rounding;

    if ((rc = run_route(*st, x, w_router, bias, T, d, E, k, ids, wts, chunk, false, s, probs_t))) return rc;
    if ((rc = rec(1))) return rc;
    if ((rc = run_permute(x, ids, wts, T, d, E, k, counts, offsets, perm, inv, nullptr, w_perm, chunk, true, s)))
        return rc;
    const int iT = (int)T, iE = (int)E;
    if (launch(round_kernel, dim3((unsigned)E), dim3(kThreads), round_smem_bytes(iT), s, 1u,
               static_cast<const int32_t*>(offsets), static_cast<const int32_t*>(perm), (int)k,
               static_cast<const float*>(probs_t), iT, iE, (int)tile, bitmaps, new_counts))
        return MOE_ERR_CUDA;
    if (launch(scan_kernel, dim3(1), dim3(kThreads), 0, s, 1u, static_cast<const int32_t*>(new_counts), iE, offsets2))
        return MOE_ERR_CUDA;
    if (cudaMemsetAsync(posmap, 0xff, (size_t)T * (size_t)E * 4, s) != cudaSuccess) return MOE_ERR_CUDA;  // -1
    if (launch(place_kernel, dim3((unsigned)E), dim3(kThreads), 0, s, 1u, static_cast<const uint32_t*>(bitmaps),
               static_cast<const int32_t*>(offsets2), static_cast<const float*>(probs_t), iT, iE, cap, w2,
               posmap))
        return MOE_ERR_CUDA;
    if (launch(gather_rows_kernel, dim3((unsigned)((T + 7) / 8)), dim3(256), 0, s, 1u,
               reinterpret_cast<const uint4*>(x), static_cast<const int32_t*>(posmap), iE, T, cap, (int)(d / 8),
               reinterpret_cast<uint4*>(x_perm)))
        return MOE_ERR_CUDA;
    if ((rc = rec(2))) return rc;
    if ((rc = run_ffn(*st, x_perm, nullptr, nullptr, T, k, w2, offsets2, w_gate, w_up, w_down, cap, d, E, f, h, y, s,
                      ev ? ev[3] : nullptr, true)))
        return rc;
    if ((rc = rec(4))) return rc;
    const int nvec = (int)(d / 8);
    const int threads = nvec < 256 ? ((nvec + 31) / 32) * 32 : 256;
    if (launch(combine_masked_kernel, dim3((unsigned)T), dim3(threads), 0, s, 1u, reinterpret_cast<const uint4*>(y),
               static_cast<const int32_t*>(posmap), iE, cap, nvec, reinterpret_cast<float4*>(out)))
        return MOE_ERR_CUDA;
    return rec(5);
}

// ------------------------------------------------------------ backward
// Workspace of moe_backward.  Grouped rows are padded: every expert group
// starts on a 64-row boundary, so the grouped buffers hold up to
// T*k + 63*E rows.
// The router's weight gradient x^T . dlogit reduces over all T tokens into a
// small d x E matrix: (d / 256) x (E / 256) output tiles, too few to fill the
// GPU.  It is split over up to this many chunks of tokens, each writing a
// partial product, summed afterwards in a fixed order.
constexpr int64_t kRouterGradSplits = 16;

struct BLayout {
    size_t ids, wts, probs, counts, offsets, chunk, perm, inv, w_perm, x_perm, dout_perm, g, u, hw, dwp, dx_perm,
        dlogit, db_part, dx_router, dwr_part, total;
    int64_t rows;    // padded row capacity
    int64_t e_pad;   // E rounded up to 64 (row length of dlogit)
    int n_tiles_f;   // 256-column tiles over f (the down-projection gradient's partial dots)
};

BLayout plan_backward(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f)
{
    const size_t M = (size_t)(T * k);
    BLayout L{};
    L.rows = (int64_t)M + 63 * E;
    L.e_pad = (E + 63) / 64 * 64;
    L.n_tiles_f = (int)((f + moe::gemm::kBN - 1) / moe::gemm::kBN);
    const size_t R = (size_t)L.rows;
    size_t o = 0;
    L.ids = o;       o += align256(M * 4);
    L.wts = o;       o += align256(M * 4);
    L.probs = o;     o += align256((size_t)T * (size_t)E * 4);
    L.counts = o;    o += align256((size_t)E * 4);
    L.offsets = o;   o += align256((size_t)(E + 1) * 4);
    L.chunk = o;     o += permute_ws_bytes(T, E);
    L.perm = o;      o += align256(R * 4);
    L.inv = o;       o += align256(M * 4);
    L.w_perm = o;    o += align256(R * 4);
    L.x_perm = o;    o += align256(R * (size_t)d * 2);
    L.dout_perm = o; o += align256(R * (size_t)d * 2);
    L.g = o;         o += align256(R * (size_t)f * 2);   // g, then dg in place
    L.u = o;         o += align256(R * (size_t)f * 2);   // u, then du in place
    L.hw = o;        o += align256(R * (size_t)f * 2);
    L.dwp = o;       o += align256(R * (size_t)(2 * L.n_tiles_f) * 4);
    L.dx_perm = o;   o += align256(R * (size_t)d * 2);  // bf16
    L.dlogit = o;    o += align256((size_t)T * (size_t)L.e_pad * 2);
    L.db_part = o;   o += align256((size_t)((T + moe::bwd::kRowWarps - 1) / moe::bwd::kRowWarps) * (size_t)E * 4);
    L.dx_router = o; o += align256((size_t)T * (size_t)d * 4);
    L.dwr_part = o;  o += align256((size_t)kRouterGradSplits * (size_t)d * (size_t)E * 4);
    L.total = o;
    return L;
}

// to0 / to1: the output maps of the TMA-store epilogues: the two weight-gradient
// views of kDW (fp32 or bf16), the bf16 dx_perm rows of kDX (to0), the dg
// and du chunks of kDH (to0, to1); kGU ignores them.
template <int KIND>
int launch_pair_bwd(const DeviceState& st, int64_t work, const CUtensorMap& ta, const CUtensorMap& ta2,
                    const CUtensorMap& tb0, const CUtensorMap& tb1, const moe::bwd::Params& p, cudaStream_t s,
                    const CUtensorMap* to0 = nullptr, const CUtensorMap* to1 = nullptr)
{
    int64_t pairs = st.max_pairs > 0 ? st.max_pairs : st.sm_count / 2;
    if (work < pairs) pairs = work;
    if (pairs < 1) pairs = 1;
    return launch(moe::bwd::pair_bwd_kernel<KIND>, dim3((unsigned)(2 * pairs)), dim3(moe::bwd::kThreads),
                  moe::bwd::smem_bytes<KIND>(), s, 2u, ta, ta2, tb0, tb1, to0 ? *to0 : ta, to1 ? *to1 : ta, p);
}

// bf16 [groups][rows][cols] viewed for 32 x 32 TMA stores (2 KB slabs,
// 64-byte swizzle); elements outside the extents are clipped by the store.
int make_out3_map_bf16(CUtensorMap* m, void* base, uint64_t cols, uint64_t rows, uint64_t groups)
{
    cuuint64_t dims[3] = {cols, rows, groups};
    cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
    cuuint32_t box[3] = {32, 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// The same for fp32 (4 KB slabs, 128-byte swizzle).
int make_out3_map(CUtensorMap* m, float* base, uint64_t cols, uint64_t rows, uint64_t groups)
{
    cuuint64_t dims[3] = {cols, rows, groups};
    cuuint64_t strides[2] = {cols * 4, rows * cols * 4};
    cuuint32_t box[3] = {32, 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

moe::bwd::Params bwd_params()
{
    moe::bwd::Params p;
    std::memset(&p, 0, sizeof(p));
    return p;
}

int backward_impl(const moe_bf16* x, const moe_bf16* w_router, const float* bias, const moe_bf16* w_gate,
                  const moe_bf16* w_up, const moe_bf16* w_down, const float* dout, int64_t T, int64_t d, int64_t E,
                  int64_t k, int64_t f, float* dx, void* dw_router, float* dbias, void* dw_gate, void* dw_up,
                  void* dw_down, void* ws, size_t ws_bytes, cudaStream_t s, unsigned flags)
{
    int rc = check_common(T, d, E, k);
    if (rc) return rc;
    if ((rc = check_f(f))) return rc;
    if (flags & ~(unsigned)(MOE_FLAG_RENORMALIZE | MOE_FLAG_GRAD_BF16)) return MOE_ERR_INVALID_ARG;
    const bool grad_bf16 = (flags & MOE_FLAG_GRAD_BF16) != 0;
    const size_t gbytes = grad_bf16 ? 2 : 4;  // bytes per weight-gradient element
    if (!w_router || !w_gate || !w_up || !w_down || !dw_router || !dw_gate || !dw_up || !dw_down)
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !dout || !dx)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(w_gate, 16) || !aligned(w_up, 16) ||
        !aligned(w_down, 16) || !aligned(dout, 16) || !aligned(dx, 16) || !aligned(dw_router, 16) ||
        !aligned(dw_gate, 16) || !aligned(dw_up, 16) || !aligned(dw_down, 16) || !aligned(bias, 4) ||
        !aligned(dbias, 4))
        return MOE_ERR_INVALID_ARG;
    const BLayout L = plan_backward(T, d, E, k, f);
    if (L.rows >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T > 0 && (!ws || !aligned(ws, 256))) return MOE_ERR_INVALID_ARG;
    if (T > 0 && ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    DeviceState* st = nullptr;
    if ((rc = setup_device(&st))) return rc;
    if (T == 0) {
        // no tokens: every weight gradient is zero
        const size_t we = (size_t)E * (size_t)d * (size_t)f * gbytes;
        if (cudaMemsetAsync(dw_gate, 0, we, s) != cudaSuccess || cudaMemsetAsync(dw_up, 0, we, s) != cudaSuccess ||
            cudaMemsetAsync(dw_down, 0, we, s) != cudaSuccess ||
            cudaMemsetAsync(dw_router, 0, (size_t)d * (size_t)E * gbytes, s) != cudaSuccess ||
            (dbias && cudaMemsetAsync(dbias, 0, (size_t)E * 4, s) != cudaSuccess))
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    using namespace moe::bwd;
    uint8_t* w = static_cast<uint8_t*>(ws);
    auto at = [&](size_t off) { return static_cast<void*>(w + off); };
    int32_t* ids = static_cast<int32_t*>(at(L.ids));
    float* wts = static_cast<float*>(at(L.wts));
    float* probs = static_cast<float*>(at(L.probs));
    int32_t* counts = static_cast<int32_t*>(at(L.counts));
    int32_t* offsets = static_cast<int32_t*>(at(L.offsets));
    int32_t* chunk = static_cast<int32_t*>(at(L.chunk));
    int32_t* perm = static_cast<int32_t*>(at(L.perm));
    int32_t* inv = static_cast<int32_t*>(at(L.inv));
    float* w_perm = static_cast<float*>(at(L.w_perm));
    moe_bf16* x_perm = static_cast<moe_bf16*>(at(L.x_perm));
    moe_bf16* dout_perm = static_cast<moe_bf16*>(at(L.dout_perm));
    moe_bf16* g = static_cast<moe_bf16*>(at(L.g));
    moe_bf16* u = static_cast<moe_bf16*>(at(L.u));
    moe_bf16* hw = static_cast<moe_bf16*>(at(L.hw));
    float* dwp = static_cast<float*>(at(L.dwp));
    moe_bf16* dx_perm = static_cast<moe_bf16*>(at(L.dx_perm));
    moe_bf16* dlogit = static_cast<moe_bf16*>(at(L.dlogit));
    float* db_part = static_cast<float*>(at(L.db_part));
    float* dx_router = static_cast<float*>(at(L.dx_router));
    const int64_t R = L.rows;
    const int iE = (int)E, ik = (int)k;
    const bool renorm = (flags & MOE_FLAG_RENORMALIZE) != 0;

    // 1. routing again (ids, weights, every probability [T][E], chunk histograms)
    if ((rc = run_route(*st, x, w_router, bias, T, d, E, k, ids, wts, chunk, renorm, s, nullptr, probs))) return rc;
    // 2. grouping with 64-row aligned groups, x_perm, dout_perm, zero padding
    {
        using namespace moe::permute;
        const int nch = (int)token_chunks(T);
        if (launch(chunk_scan_kernel, dim3((unsigned)E), dim3(moe::permute::kThreads), 0, s, 1u, chunk, nch, counts))
            return MOE_ERR_CUDA;
        if (launch(rank_kernel<true>, dim3(nch), dim3(moe::permute::kThreads), 0, s, 1u,
                   static_cast<const int32_t*>(ids), static_cast<const float*>(wts), T, ik, iE,
                   static_cast<const int32_t*>(chunk), nch, static_cast<const int32_t*>(counts), offsets, perm, inv,
                   w_perm))
            return MOE_ERR_CUDA;
        if (launch(gather_kernel, dim3((unsigned)((T + moe::permute::kWarps - 1) / moe::permute::kWarps)),
                   dim3(moe::permute::kThreads), 0, s, 1u, reinterpret_cast<const uint4*>(x),
                   static_cast<const int32_t*>(inv), T, ik, (int)(d / 8), R, reinterpret_cast<uint4*>(x_perm)))
            return MOE_ERR_CUDA;
    }
    if (launch(gather_dout_kernel, dim3((unsigned)((T + kRowWarps - 1) / kRowWarps)), dim3(kRowThreads), 0, s, 1u,
               reinterpret_cast<const float4*>(dout), static_cast<const int32_t*>(inv), T, ik, (int)(d / 8), R,
               reinterpret_cast<uint4*>(dout_perm)))
        return MOE_ERR_CUDA;
    if (launch(zero_pad_kernel, dim3((unsigned)E), dim3(kRowThreads), 0, s, 1u, static_cast<const int32_t*>(offsets),
               static_cast<const int32_t*>(counts), (int)(d / 8), reinterpret_cast<uint4*>(x_perm),
               reinterpret_cast<uint4*>(dout_perm), w_perm))
        return MOE_ERR_CUDA;

    using moe::gemm::kBN;
    using moe::gemm::kBM;
    using moe::gemm::kPairRows;
    const int64_t max_mtiles = (R + kPairRows - 1) / kPairRows + E;
    // 3. recompute g, u = x_perm . [W_gate | W_up], and w h for the W_down gradient
    {
        CUtensorMap ta, tg3, tu3;
        rc = make_map(&ta, x_perm, (uint64_t)d, (uint64_t)R, 64, kBM);
        rc = rc ? rc : make_weight_chunk_map(&tg3, w_gate, (uint64_t)f, (uint64_t)(E * d));
        rc = rc ? rc : make_weight_chunk_map(&tu3, w_up, (uint64_t)f, (uint64_t)(E * d));
        if (rc) return rc;
        Params p = bwd_params();
        p.offsets = offsets;
        p.w_perm = w_perm;
        p.out_g = reinterpret_cast<__nv_bfloat16*>(g);
        p.out_u = reinterpret_cast<__nv_bfloat16*>(u);
        p.out_hw = reinterpret_cast<__nv_bfloat16*>(hw);
        p.ld_f = f;
        p.E = iE;
        p.M = (int)R;
        p.K = (int)d;
        p.n_out = (int)f;
        p.n_tiles = (int)((f + 127) / 128);
        p.b_rows = (int)d;
        if (launch_pair_bwd<kGU>(*st, max_mtiles * p.n_tiles, ta, ta, tg3, tu3, p, s)) return MOE_ERR_CUDA;
    }
    // 4. dh = w . dout_perm . W_down^T and the SwiGLU derivative: dg, du (in place of g, u), partial dots
    {
        CUtensorMap ta, tb, tog, tou;
        rc = make_map(&ta, dout_perm, (uint64_t)d, (uint64_t)R, 64, kBM);
        rc = rc ? rc : make_map(&tb, w_down, (uint64_t)d, (uint64_t)(E * f), 64, kBM);
        // dg and du (in place over g and u) for the epilogue's 32 x 16 TMA stores
        rc = rc ? rc : make_map(&tog, g, (uint64_t)f, (uint64_t)R, 16, 32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                                CU_TENSOR_MAP_SWIZZLE_NONE);
        rc = rc ? rc : make_map(&tou, u, (uint64_t)f, (uint64_t)R, 16, 32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                                CU_TENSOR_MAP_SWIZZLE_NONE);
        if (rc) return rc;
        Params p = bwd_params();
        p.offsets = offsets;
        p.w_perm = w_perm;
        p.g = reinterpret_cast<const __nv_bfloat16*>(g);
        p.u = reinterpret_cast<const __nv_bfloat16*>(u);
        p.out_g = reinterpret_cast<__nv_bfloat16*>(g);
        p.out_u = reinterpret_cast<__nv_bfloat16*>(u);
        p.dwp = dwp;
        p.ld_f = f;
        p.E = iE;
        p.M = (int)R;
        p.K = (int)d;
        p.n_out = (int)f;
        p.n_tiles = L.n_tiles_f;
        p.b_rows = (int)f;
        if (launch_pair_bwd<kDH>(*st, max_mtiles * p.n_tiles, ta, ta, tb, tb, p, s, &tog, &tou)) return MOE_ERR_CUDA;
    }
    // 5. dx_perm = dg . W_gate^T + du . W_up^T (fp32 accumulators, stored bf16)
    {
        CUtensorMap ta, ta2, tb0, tb1, to0;
        rc = make_map(&ta, g, (uint64_t)f, (uint64_t)R, 64, kBM);
        rc = rc ? rc : make_map(&ta2, u, (uint64_t)f, (uint64_t)R, 64, kBM);
        rc = rc ? rc : make_map(&tb0, w_gate, (uint64_t)f, (uint64_t)(E * d), 64, kBM);
        rc = rc ? rc : make_map(&tb1, w_up, (uint64_t)f, (uint64_t)(E * d), 64, kBM);
        rc = rc ? rc : make_map(&to0, dx_perm, (uint64_t)d, (uint64_t)R, 32, 32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                                CU_TENSOR_MAP_SWIZZLE_64B);
        if (rc) return rc;
        Params p = bwd_params();
        p.offsets = offsets;
        p.out0 = reinterpret_cast<float*>(dx_perm);
        p.out_bf16 = 1;
        p.ld_out = d;
        p.E = iE;
        p.M = (int)R;
        p.K = (int)(2 * f);
        p.k_split = (int)(f / 64);
        p.n_out = (int)d;
        p.n_tiles = (int)((d + kBN - 1) / kBN);
        p.b_rows = (int)d;
        if (launch_pair_bwd<kDX>(*st, max_mtiles * p.n_tiles, ta, ta2, tb0, tb1, p, s, &to0, &to0))
            return MOE_ERR_CUDA;
    }
    // 6. dW_gate[e], dW_up[e] = x_perm_e^T . dg_e, x_perm_e^T . du_e
    {
        CUtensorMap ta, tb0, tb1, to0, to1;
        rc = make_weight_chunk_map(&ta, x_perm, (uint64_t)d, (uint64_t)R);
        rc = rc ? rc : make_weight_chunk_map(&tb0, g, (uint64_t)f, (uint64_t)R);
        rc = rc ? rc : make_weight_chunk_map(&tb1, u, (uint64_t)f, (uint64_t)R);
        if (grad_bf16) {
            rc = rc ? rc : make_out3_map_bf16(&to0, dw_gate, (uint64_t)f, (uint64_t)d, (uint64_t)E);
            rc = rc ? rc : make_out3_map_bf16(&to1, dw_up, (uint64_t)f, (uint64_t)d, (uint64_t)E);
        } else {
            rc = rc ? rc : make_out3_map(&to0, static_cast<float*>(dw_gate), (uint64_t)f, (uint64_t)d, (uint64_t)E);
            rc = rc ? rc : make_out3_map(&to1, static_cast<float*>(dw_up), (uint64_t)f, (uint64_t)d, (uint64_t)E);
        }
        if (rc) return rc;
        Params p = bwd_params();
        p.offsets = offsets;
        p.out0 = static_cast<float*>(dw_gate);
        p.out1 = static_cast<float*>(dw_up);
        p.out_bf16 = grad_bf16 ? 1 : 0;
        p.ld_out = f;
        p.E = iE;
        p.M = (int)R;
        p.n_out = (int)f;
        p.n_tiles = (int)((f + 127) / 128);
        p.m_total = (int)d;
        p.m_tiles = (int)((d + kPairRows - 1) / kPairRows);
        p.split_b = 1;
        if (launch_pair_bwd<kDW>(*st, E * p.m_tiles * p.n_tiles, ta, ta, tb0, tb1, p, s, &to0, &to1))
            return MOE_ERR_CUDA;
    }
    // 7. dW_down[e] = (w h)_e^T . dout_perm_e
    {
        CUtensorMap ta, tb, to0;
        rc = make_weight_chunk_map(&ta, hw, (uint64_t)f, (uint64_t)R);
        rc = rc ? rc : make_weight_chunk_map(&tb, dout_perm, (uint64_t)d, (uint64_t)R);
        rc = rc ? rc
                : (grad_bf16 ? make_out3_map_bf16(&to0, dw_down, (uint64_t)d, (uint64_t)f, (uint64_t)E)
                             : make_out3_map(&to0, static_cast<float*>(dw_down), (uint64_t)d, (uint64_t)f,
                                             (uint64_t)E));
        if (rc) return rc;
        Params p = bwd_params();
        p.offsets = offsets;
        p.out0 = static_cast<float*>(dw_down);
        p.out_bf16 = grad_bf16 ? 1 : 0;
        p.ld_out = d;
        p.E = iE;
        p.M = (int)R;
        p.n_out = (int)d;
        p.n_tiles = (int)((d + kBN - 1) / kBN);
        p.m_total = (int)f;
        p.m_tiles = (int)((f + kPairRows - 1) / kPairRows);
        p.split_b = 0;
        if (launch_pair_bwd<kDW>(*st, E * p.m_tiles * p.n_tiles, ta, ta, tb, tb, p, s, &to0, &to0))
            return MOE_ERR_CUDA;
    }
    // 8. router: dlogit (bf16 [T][E_pad]) and the bias gradient
    const unsigned nblk = (unsigned)((T + kRowWarps - 1) / kRowWarps);
    if (launch(route_bwd_kernel, dim3(nblk), dim3(kRowThreads), 0, s, 1u, static_cast<const float*>(probs),
               static_cast<const int32_t*>(ids), static_cast<const float*>(wts), static_cast<const int32_t*>(inv),
               static_cast<const float*>(dwp), 2 * L.n_tiles_f, R, T, iE, ik, renorm ? 1 : 0,
               reinterpret_cast<__nv_bfloat16*>(dlogit), dbias ? db_part : nullptr, (int)L.e_pad))
        return MOE_ERR_CUDA;
    if (dbias && launch(colsum_kernel, dim3((unsigned)E), dim3(kRowThreads), 0, s, 1u,
                        static_cast<const float*>(db_part), (int)nblk, iE, dbias))
        return MOE_ERR_CUDA;
    // 9. dW_router = x^T . dlogit: the T rows in S chunks of a multiple of 64
    //    rows (as many as fill one wave of CTA pairs, at most
    //    kRouterGradSplits), one fp32 partial product per chunk, then their
    //    sum in chunk order
    {
        const int m_tiles = (int)((d + kPairRows - 1) / kPairRows);
        const int n_tiles = (int)((E + kBN - 1) / kBN);
        const int64_t pairs = st->max_pairs > 0 ? st->max_pairs : st->sm_count / 2;
        int64_t S = pairs / ((int64_t)m_tiles * n_tiles);
        S = S < 1 ? 1 : (S > kRouterGradSplits ? kRouterGradSplits : S);
        const int64_t chunk = ((T + S - 1) / S + 63) / 64 * 64;
        S = (T + chunk - 1) / chunk;
        float* part = static_cast<float*>(at(L.dwr_part));
        CUtensorMap ta, tb, to0;
        rc = make_weight_chunk_map(&ta, x, (uint64_t)d, (uint64_t)T);
        rc = rc ? rc : make_weight_chunk_map(&tb, dlogit, (uint64_t)L.e_pad, (uint64_t)T);
        rc = rc ? rc : make_out3_map(&to0, part, (uint64_t)E, (uint64_t)d, (uint64_t)S);
        if (rc) return rc;
        Params p = bwd_params();
        p.offsets = nullptr;
        p.out0 = part;
        p.ld_out = E;
        p.E = (int)S;
        p.M = (int)T;
        p.k_chunk = (int)chunk;
        p.n_out = iE;
        p.n_tiles = n_tiles;
        p.m_total = (int)d;
        p.m_tiles = m_tiles;
        p.split_b = 0;
        if (launch_pair_bwd<kDW>(*st, S * p.m_tiles * p.n_tiles, ta, ta, tb, tb, p, s, &to0, &to0))
            return MOE_ERR_CUDA;
        const int64_t n4 = d * E / 4;
        const unsigned blocks = (unsigned)((n4 + kRowThreads - 1) / kRowThreads);
        const dim3 grid(blocks < 1184u ? blocks : 1184u);
        if (grad_bf16 ? launch(sum_partials_kernel<true>, grid, dim3(kRowThreads), 0, s, 1u,
                               reinterpret_cast<const float4*>(part), (int)S, n4, dw_router)
                      : launch(sum_partials_kernel<false>, grid, dim3(kRowThreads), 0, s, 1u,
                               reinterpret_cast<const float4*>(part), (int)S, n4, dw_router))
            return MOE_ERR_CUDA;
    }
    // 10. dx_router = dlogit . W_router^T (fp32)
    {
        CUtensorMap ta, tb, to0;
        rc = make_map(&ta, dlogit, (uint64_t)L.e_pad, (uint64_t)T, 64, kBM);
        rc = rc ? rc : make_map(&tb, w_router, (uint64_t)E, (uint64_t)d, 64, kBM);
        rc = rc ? rc : make_out3_map(&to0, dx_router, (uint64_t)d, (uint64_t)T, 1);
        if (rc) return rc;
        Params p = bwd_params();
        p.offsets = nullptr;
        p.out0 = dx_router;
        p.ld_out = d;
        p.E = 1;
        p.M = (int)T;
        p.K = (int)L.e_pad;
        p.k_split = (int)(L.e_pad / 64);
        p.n_out = (int)d;
        p.n_tiles = (int)((d + kBN - 1) / kBN);
        p.b_rows = 0;
        if (launch_pair_bwd<kDX>(*st, ((T + kPairRows - 1) / kPairRows) * p.n_tiles, ta, ta, tb, tb, p, s, &to0,
                                 &to0))
            return MOE_ERR_CUDA;
    }
    // 11. dx = dx_router + sum over slots of dx_perm (fp32 sums)
    if (launch(combine_dx_kernel, dim3((unsigned)T), dim3(kRowThreads), 0, s, 1u,
               reinterpret_cast<const uint4*>(dx_perm), reinterpret_cast<const float4*>(dx_router),
               static_cast<const int32_t*>(inv), R, ik, (int)(d / 8), reinterpret_cast<float4*>(dx)))
        return MOE_ERR_CUDA;
    return MOE_OK;
}

// ------------------------------------------- fixed scratch for moe_permute_static
// Some callers cannot allocate device memory when they run the permutation:
// for example a plugin inside an inference engine that plans all device
// memory ahead of time and must not allocate while it enqueues work, or a
// latency-critical loop where cudaMalloc's implicit synchronisation is not
// acceptable.  moe_permute_static serves them from this array instead of a
// caller-provided workspace.  It holds the per-chunk expert counts, one
// int32 per (expert, 64-token chunk), so it caps E * ceil(T / 64).  Every
// GPU that loads the library keeps the array (1 MiB) until the process ends.
constexpr int64_t kStaticPermuteScratchInts = int64_t(1) << 18;
static __device__ __align__(256) int32_t g_static_permute_scratch[kStaticPermuteScratchInts];

int32_t* g_static_scratch_addr[kMaxDevices] = {};
unsigned long long g_static_scratch_ctx[kMaxDevices] = {};

// The array's device address for the current device.  In host code the
// symbol name is only a host-side stand-in, so the address is looked up once
// per device (and context) with that device current, checked, and cached;
// a new context on the device (after cudaDeviceReset) gets a new lookup.
int static_permute_scratch(int32_t** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    unsigned long long ctx_id = 0;
    if (current_context_id(dev, &ctx_id)) return MOE_ERR_CUDA;
    if (!g_static_scratch_addr[dev] || g_static_scratch_ctx[dev] != ctx_id) {
        void* addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_static_permute_scratch) != cudaSuccess || !addr) return MOE_ERR_CUDA;
        g_static_scratch_addr[dev] = static_cast<int32_t*>(addr);
        g_static_scratch_ctx[dev] = ctx_id;
    }
    *out = g_static_scratch_addr[dev];
    return MOE_OK;
}

}  // namespace

// ===================================================================== ABI
extern "C" {

const char* moe_strerror(int status)
{
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: null or misaligned pointer, or negative size";
        case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE: shape outside the supported limits";
        case MOE_ERR_WORKSPACE_TOO_SMALL: return "MOE_ERR_WORKSPACE_TOO_SMALL";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call or kernel launch failed";
        case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT: a device pipeline wait ran past its limit";
        case MOE_ERR_DEVICE_BOUNDS: return "MOE_ERR_DEVICE_BOUNDS: index data out of range on the device";
        case MOE_ERR_UNSUPPORTED_DEVICE: return "MOE_ERR_UNSUPPORTED_DEVICE: needs a compute capability 10.0 GPU";
        case MOE_ERR_STATIC_SCRATCH_TOO_SMALL:
            return "MOE_ERR_STATIC_SCRATCH_TOO_SMALL: moe_permute_static needs E * ceil(T / 64) <= 262144";
        case MOE_ERR_DEVICE_RANGE:
            return "MOE_ERR_DEVICE_RANGE: a y value outside the fp16 range (|y| >= 65520) or NaN on the device";
        default: return "unknown moe status";
    }
}

int moe_version(void) { return 203; }

size_t moe_workspace_size(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f)
{
    if (check_common(T, d, E, k) || check_f(f)) return 0;
    return plan(T, d, E, k, f).total;
}

size_t moe_workspace_size_shared(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, int64_t n_shared,
                                 int64_t f_shared)
{
    if (check_common(T, d, E, k) || check_f(f) || n_shared < 1 || n_shared > kMaxShared || check_f(f_shared))
        return 0;
    return plan(T, d, E, k, f, n_shared, f_shared).total;
}

size_t moe_route_workspace_size(int64_t T, int64_t d, int64_t E)
{
    if (check_common(T, d, E, 1)) return 0;
    return route_ws_bytes(T, d, E);
}

size_t moe_permute_workspace_size(int64_t T, int64_t E, int64_t k)
{
    if (T < 0 || E <= 0 || k <= 0 || E > moe::gemm::kMaxE || k > E) return 0;
    return permute_ws_bytes(T, E);
}

int moe_route(const moe_bf16* x, const moe_bf16* w_router, const float* bias, int64_t T, int64_t d, int64_t E,
              int64_t k, int32_t* topk_ids, float* topk_w, void* workspace, size_t workspace_bytes,
              cudaStream_t stream)
{
    return moe_route_ex(x, w_router, bias, T, d, E, k, topk_ids, topk_w, workspace, workspace_bytes, stream, 0u);
}

int moe_route_ex(const moe_bf16* x, const moe_bf16* w_router, const float* bias, int64_t T, int64_t d, int64_t E,
                 int64_t k, int32_t* topk_ids, float* topk_w, void* workspace, size_t workspace_bytes,
                 cudaStream_t stream, unsigned flags)
{
    if (flags & ~(unsigned)MOE_FLAG_RENORMALIZE) return MOE_ERR_INVALID_ARG;
    int rc = check_common(T, d, E, k);
    if (rc) return rc;
    if (T > 0 && (!x || !w_router || !topk_ids || !topk_w)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(bias, 4) || !aligned(topk_ids, 4) ||
        !aligned(topk_w, 4) || !aligned(workspace, 16))
        return MOE_ERR_INVALID_ARG;
    if (workspace_bytes < route_ws_bytes(T, d, E)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    DeviceState* st = nullptr;
    if ((rc = setup_device(&st))) return rc;
    return run_route(*st, x, w_router, bias, T, d, E, k, topk_ids, topk_w, nullptr,
                     (flags & MOE_FLAG_RENORMALIZE) != 0, stream);
}

int moe_permute(const moe_bf16* x, const int32_t* topk_ids, const float* topk_w, int64_t T, int64_t d, int64_t E,
                int64_t k, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv, moe_bf16* x_perm,
                float* w_perm, void* workspace, size_t workspace_bytes, cudaStream_t stream)
{
    int rc = check_common(T, d, E, k);
    if (rc) return rc;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!topk_ids || !topk_w || !perm || !inv || !w_perm)) return MOE_ERR_INVALID_ARG;
    if (x_perm && !x) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(x_perm, 16) || !aligned(topk_ids, 4) || !aligned(topk_w, 4) ||
        !aligned(counts, 4) || !aligned(offsets, 4) || !aligned(perm, 4) || !aligned(inv, 4) || !aligned(w_perm, 4))
        return MOE_ERR_INVALID_ARG;
    const size_t need = permute_ws_bytes(T, E);
    if (workspace_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (T > 0 && (!workspace || !aligned(workspace, 4))) return MOE_ERR_INVALID_ARG;
    DeviceState* st = nullptr;
    if ((rc = setup_device(&st))) return rc;
    return run_permute(x, topk_ids, topk_w, T, d, E, k, counts, offsets, perm, inv, x_perm, w_perm,
                       static_cast<int32_t*>(workspace), false, stream);
}

int moe_permute_static(const moe_bf16* x, const int32_t* topk_ids, const float* topk_w, int64_t T, int64_t d,
                       int64_t E, int64_t k, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                       moe_bf16* x_perm, float* w_perm, cudaStream_t stream)
{
    int rc = check_common(T, d, E, k);
    if (rc) return rc;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!topk_ids || !topk_w || !perm || !inv || !w_perm)) return MOE_ERR_INVALID_ARG;
    if (x_perm && !x) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(x_perm, 16) || !aligned(topk_ids, 4) || !aligned(topk_w, 4) ||
        !aligned(counts, 4) || !aligned(offsets, 4) || !aligned(perm, 4) || !aligned(inv, 4) || !aligned(w_perm, 4))
        return MOE_ERR_INVALID_ARG;
    if (E * token_chunks(T) > kStaticPermuteScratchInts) return MOE_ERR_STATIC_SCRATCH_TOO_SMALL;
    DeviceState* st = nullptr;
    if ((rc = setup_device(&st))) return rc;
    int32_t* scratch = nullptr;
    if ((rc = static_permute_scratch(&scratch))) return rc;
    // The histogram kernel writes every (expert, chunk) entry that the scan
    // and rank kernels later read, so nothing left by an earlier call needs
    // clearing first.
    return run_permute(x, topk_ids, topk_w, T, d, E, k, counts, offsets, perm, inv, x_perm, w_perm, scratch, false,
                       stream);
}

int moe_expert_ffn(const moe_bf16* x_perm, const float* w_perm, const int32_t* offsets, const moe_bf16* w_gate,
                   const moe_bf16* w_up, const moe_bf16* w_down, int64_t M, int64_t d, int64_t E, int64_t f,
                   moe_bf16* h, moe_f16* y, cudaStream_t stream)
{
    if (M < 0 || d <= 0 || E <= 0) return MOE_ERR_INVALID_ARG;
    int rc = check_common(M, d, E, 1);
    if (rc) return rc;
    if ((rc = check_f(f))) return rc;
    if (M > 0 && (!x_perm || !w_perm || !offsets || !w_gate || !w_up || !w_down || !h || !y))
        return MOE_ERR_INVALID_ARG;
    if (!aligned(x_perm, 16) || !aligned(w_gate, 16) || !aligned(w_up, 16) || !aligned(w_down, 16) ||
        !aligned(h, 16) || !aligned(y, 16) || !aligned(w_perm, 4) || !aligned(offsets, 4))
        return MOE_ERR_INVALID_ARG;
    DeviceState* st = nullptr;
    if ((rc = setup_device(&st))) return rc;
    return run_ffn(*st, x_perm, nullptr, nullptr, 0, 1, w_perm, offsets, w_gate, w_up, w_down, M, d, E, f, h, y,
                   stream, nullptr);
}

int moe_combine(const moe_f16* y, const int32_t* inv, int64_t T, int64_t d, int64_t k, float* out,
                cudaStream_t stream)
{
    if (T < 0 || d <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (d % 64 != 0 || d > 32768 || k > 32 || T * k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T > 0 && (!y || !inv || !out)) return MOE_ERR_INVALID_ARG;
    if (!aligned(y, 16) || !aligned(out, 16) || !aligned(inv, 4)) return MOE_ERR_INVALID_ARG;
    DeviceState* st = nullptr;
    int rc = setup_device(&st);
    if (rc) return rc;
    return run_combine(y, inv, T, d, k, out, stream);
}

int moe_shared_ffn(const moe_bf16* x, const moe_bf16* w_gate_s, const moe_bf16* w_up_s, const moe_bf16* w_down_s,
                   int64_t T, int64_t d, int64_t n_shared, int64_t f_shared, moe_bf16* h_s, moe_f16* y_s,
                   cudaStream_t stream)
{
    if (T < 0 || d <= 0 || n_shared < 1) return MOE_ERR_INVALID_ARG;
    if (d % 64 != 0 || d > 32768 || T >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
    int rc;
    if ((rc = check_shared(w_gate_s, w_up_s, w_down_s, T, n_shared, f_shared))) return rc;
    if (T > 0 && (!x || !h_s || !y_s)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(h_s, 16) || !aligned(y_s, 16)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    DeviceState* st = nullptr;
    if ((rc = setup_device(&st))) return rc;
    return run_shared(*st, x, w_gate_s, w_up_s, w_down_s, T, d, n_shared, f_shared, h_s, y_s, stream);
}

int moe_combine_shared(const moe_f16* y, const int32_t* inv, const moe_f16* y_s, int64_t n_shared, int64_t T,
                       int64_t d, int64_t k, float* out, cudaStream_t stream)
{
    if (T < 0 || d <= 0 || k <= 0 || n_shared < 0) return MOE_ERR_INVALID_ARG;
    if (d % 64 != 0 || d > 32768 || k > 32 || T * k >= (int64_t(1) << 31) || n_shared > kMaxShared)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T > 0 && (!y || !inv || !out || (n_shared > 0 && !y_s))) return MOE_ERR_INVALID_ARG;
    if (!aligned(y, 16) || !aligned(out, 16) || !aligned(inv, 4) || !aligned(y_s, 16)) return MOE_ERR_INVALID_ARG;
    DeviceState* st = nullptr;
    int rc = setup_device(&st);
    if (rc) return rc;
    return run_combine(y, inv, T, d, k, out, stream, y_s, n_shared);
}

int moe_forward_shared(const moe_bf16* x, const moe_bf16* w_router, const float* bias, const moe_bf16* w_gate,
                       const moe_bf16* w_up, const moe_bf16* w_down, const moe_bf16* w_gate_s,
                       const moe_bf16* w_up_s, const moe_bf16* w_down_s, int64_t T, int64_t d, int64_t E, int64_t k,
                       int64_t f, int64_t n_shared, int64_t f_shared, float* out, int32_t* topk_ids_out,
                       float* topk_w_out, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                       cudaEvent_t* events, int n_events, unsigned flags)
{
    if (n_shared < 1 || (flags & MOE_FLAG_OUT_F16)) return MOE_ERR_INVALID_ARG;
    return forward_impl(x, w_router, bias, w_gate, w_up, w_down, T, d, E, k, f, out, topk_ids_out, topk_w_out,
                        workspace, workspace_bytes, stream, events, n_events, flags, w_gate_s, w_up_s, w_down_s,
                        n_shared, f_shared);
}

size_t moe_workspace_size_rounded(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, int64_t tile)
{
    if (check_common(T, d, E, k) || check_f(f) || check_rounding(T, E, k, tile)) return 0;
    return plan_rounded(T, d, E, k, f, tile).total;
}

int moe_forward_rounded(const moe_bf16* x, const moe_bf16* w_router, const float* bias, const moe_bf16* w_gate,
                        const moe_bf16* w_up, const moe_bf16* w_down, int64_t T, int64_t d, int64_t E, int64_t k,
                        int64_t f, int64_t tile, float* out, int32_t* counts_out, int32_t* rows_out,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream, cudaEvent_t* events,
                        int n_events)
{
    return forward_rounded_impl(x, w_router, bias, w_gate, w_up, w_down, T, d, E, k, f, tile, out, counts_out,
                                rows_out, workspace, workspace_bytes, stream, events, n_events);
}

int moe_forward(const moe_bf16* x, const moe_bf16* w_router, const float* bias, const moe_bf16* w_gate,
                const moe_bf16* w_up, const moe_bf16* w_down, int64_t T, int64_t d, int64_t E, int64_t k, int64_t f,
                float* out, int32_t* topk_ids_out, float* topk_w_out, void* workspace, size_t workspace_bytes,
                cudaStream_t stream)
{
    return forward_impl(x, w_router, bias, w_gate, w_up, w_down, T, d, E, k, f, out, topk_ids_out, topk_w_out,
                        workspace, workspace_bytes, stream, nullptr, 0, kDefaultForwardFlags);
}

int moe_forward_ex(const moe_bf16* x, const moe_bf16* w_router, const float* bias, const moe_bf16* w_gate,
                   const moe_bf16* w_up, const moe_bf16* w_down, int64_t T, int64_t d, int64_t E, int64_t k,
                   int64_t f, void* out, int32_t* topk_ids_out, float* topk_w_out, void* workspace,
                   size_t workspace_bytes, cudaStream_t stream, cudaEvent_t* events, int n_events, unsigned flags)
{
    return forward_impl(x, w_router, bias, w_gate, w_up, w_down, T, d, E, k, f, out, topk_ids_out, topk_w_out,
                        workspace, workspace_bytes, stream, events, n_events, flags);
}

int moe_gather_rows(const void* src, const int32_t* idx, int64_t n_src, int64_t n, int64_t row_bytes, void* dst,
                    cudaStream_t stream)
{
    if (n_src < 0 || n < 0 || row_bytes <= 0) return MOE_ERR_INVALID_ARG;
    if (row_bytes % 4 != 0 || row_bytes / 4 > (int64_t(1) << 24) || n >= (int64_t(1) << 31) ||
        n * (row_bytes / 4) >= (int64_t(1) << 40))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (n > 0 && (!src || !idx || !dst)) return MOE_ERR_INVALID_ARG;
    const bool wide = row_bytes % 16 == 0;
    if (!aligned(src, wide ? 16 : 4) || !aligned(dst, wide ? 16 : 4) || !aligned(idx, 4)) return MOE_ERR_INVALID_ARG;
    if (n == 0) return MOE_OK;
    DeviceState* st = nullptr;
    int rc = setup_device(&st);
    if (rc) return rc;
    using namespace moe::permute;
    if (wide)
        return launch(gather_rows_idx_kernel, dim3((unsigned)((n + kWarps - 1) / kWarps)), dim3(kThreads), 0, stream,
                      1u, static_cast<const uint4*>(src), idx, n, n_src, (int)(row_bytes / 16),
                      static_cast<uint4*>(dst));
    const int64_t words = n * (row_bytes / 4);
    return launch(gather_words_idx_kernel, dim3((unsigned)((words + kThreads - 1) / kThreads)), dim3(kThreads), 0,
                  stream, 1u, static_cast<const uint32_t*>(src), idx, n, n_src, (int)(row_bytes / 4),
                  static_cast<uint32_t*>(dst));
}

size_t moe_backward_workspace_size(int64_t T, int64_t d, int64_t E, int64_t k, int64_t f)
{
    if (check_common(T, d, E, k) || check_f(f)) return 0;
    const BLayout L = plan_backward(T, d, E, k, f);
    if (L.rows >= (int64_t(1) << 31)) return 0;
    return L.total;
}

int moe_backward(const moe_bf16* x, const moe_bf16* w_router, const float* bias, const moe_bf16* w_gate,
                 const moe_bf16* w_up, const moe_bf16* w_down, const float* dout, int64_t T, int64_t d, int64_t E,
                 int64_t k, int64_t f, float* dx, void* dw_router, float* dbias, void* dw_gate, void* dw_up,
                 void* dw_down, void* workspace, size_t workspace_bytes, cudaStream_t stream, unsigned flags)
{
    return backward_impl(x, w_router, bias, w_gate, w_up, w_down, dout, T, d, E, k, f, dx, dw_router, dbias, dw_gate,
                         dw_up, dw_down, workspace, workspace_bytes, stream, flags);
}

int moe_get_status(cudaStream_t stream)
{
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
    int v = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&v, moe::g_status, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpyToSymbol(moe::g_status, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    return v;
}

int moe_set_wait_limit_ns(int64_t limit_ns)
{
    // <= 0: the default (1 s); otherwise at least 1 ms
    const unsigned long long v =
        limit_ns <= 0 ? 1000000000ull : (limit_ns < 1000000 ? 1000000ull : (unsigned long long)limit_ns);
    return cudaMemcpyToSymbol(moe::g_wait_limit_ns, &v, sizeof(v)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_selftest_wait_timeout(int64_t limit_ns, cudaStream_t stream)
{
    if (limit_ns <= 0 || limit_ns > 10000000000ll) return MOE_ERR_INVALID_ARG;
    DeviceState* st = nullptr;
    int rc = setup_device(&st);
    if (rc) return rc;
    wait_timeout_kernel<<<1, 32, 0, stream>>>((unsigned long long)limit_ns);
    return launch_status();
}

}  // extern "C"
