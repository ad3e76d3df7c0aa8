// grouped_gemm.cuh -- persistent grouped GEMM over variable-size expert
// groups on the tcgen05 tensor cores, with the two epilogues of the expert
// MLP fused in.
//
// This is the "batched expert compute" of "Qwen3MoeSparseMoeBlock
// performance optimisation in practice": the experts' weight matrices are
// stacked in one buffer and evaluated together (section 2.1, point 1), with
// work spread over the SMs dynamically (section 2.1, point 2) and operands
// staged in shared memory (section 2.2, point 3).  The compute/IO overlap
// through a producer-consumer queue that the SonicMoE comparison page
// describes for Hopper is realised here with Blackwell's own machinery.
//
// Rows of the A operand are grouped by expert: group e is rows
// [offsets[e], offsets[e+1]).  Each group is cut into 128-row M tiles (the
// last may be partial; its extra rows belong to the next group or are past
// the end, are computed, and are not stored).  A work item is one M tile x
// one N tile; persistent CTAs take items blockIdx.x, +gridDim.x, ...  Each
// CTA rebuilds the tile list from the device offsets itself, so nothing is
// read back to the host.
//
// Warp roles (192 threads):
//   warp 0       TMA producer: A [128 rows x 64 k] K-major, B 4 x [64 k x 64 n]
//                (weights are [K, N] with N contiguous: MN-major operand).
//                With GATHER, the A rows are fetched straight from the token
//                matrix x through the permutation (row pos -> token
//                perm[pos] / k): the 32 lanes issue 16-byte cp.async copies,
//                8 lanes per 128-byte row segment so each warp instruction
//                reads four whole segments, write them in the 128-byte
//                swizzled layout the MMA expects, and each lane's completion
//                is counted on the stage barrier.  The permuted copy of x is
//                never written.  (A tile::gather4 TMA per 4 rows was measured
//                3x slower here: too many small TMA requests per stage.)
//   warp 1       TMEM allocation + single-thread tcgen05.mma issuer,
//                M=128 N=256 K=16 per instruction, fp32 accumulators
//   warps 2..9   epilogue: tcgen05.ld of the 128 x 256 accumulator, one row
//                per thread, fused math, stores; the two warps of a TMEM lane
//                quarter split the columns.  (Eight warps against four: the
//                same time where the MMA bounds the tile, and 7 % off the
//                fine-grained layer, f = 256, whose short K leaves each tile's
//                epilogue longer than its MMAs.)
// Two accumulator buffers (2 x 256 TMEM columns) let the epilogue of one
// tile overlap the MMAs of the next.
//
// Epilogues:
//   kSwiGLU   : B columns 0..127 come from W_gate, 128..255 from W_up for the
//               same 128 output columns; h = silu(g) * u, silu(z) = z/(1+e^-z),
//               stored as bf16 (h is the next GEMM's bf16 operand)
//   kWeighted : y = w_perm[row] * acc, computed in fp32 and stored as IEEE
//               fp16 (the routing weight applied after the down projection).
//               One rounding to an 11-bit significand (relative error
//               <= 2^-11) keeps the combine's fp32 k-way sum well inside the
//               output tolerance, where bf16 (8 bits) would not, at half the
//               bytes of fp32 -- y is the largest stream of the block.  A value
//               that fp16 cannot hold (|y| >= 65520, or NaN) is stored as is
//               (inf / NaN) and reported as a range error.
//               Each warp stages 32 rows x 32 columns in shared memory and
//               writes them with one TMA store, so global writes are whole
//               64-byte row segments instead of per-thread scattered stores.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace moe {
namespace gemm {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kMaxStages = 4;
// Tuning constants (overridable at build time for measurements).  The CTA
// pair kernels (the default path) take 8 epilogue warps: even with 4 where
// the MMA bounds the tile, 7 % faster on the fine-grained layer.  For the
// single-CTA kernel, 4 down-GEMM stages beat 3 with more store staging.
#ifndef MOE_GEMM_EPI_WARPS
#define MOE_GEMM_EPI_WARPS 8
#endif
#ifndef MOE_GEMM_DOWN_STAGES
#define MOE_GEMM_DOWN_STAGES 4
#endif
constexpr int kEpiWarps = MOE_GEMM_EPI_WARPS;      // 4 or 8: 1 or 2 warps per TMEM lane quarter
constexpr int kColGroups = kEpiWarps / 4;          // warps sharing a lane quarter split the columns
constexpr int kThreads = 64 + kEpiWarps * 32;
static_assert(kEpiWarps == 4 || kEpiWarps == 8, "epilogue warps");
constexpr int kABytes = kBM * kBK * 2;      // 16 KB
constexpr int kChunkBytes = 64 * kBK * 2;   // 8 KB: 64 n x 64 k
constexpr int kBBytes = 4 * kChunkBytes;    // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr uint32_t kTmemCols = 512;         // 2 accumulators x 256 columns
constexpr int kMaxE = 512;
constexpr int kSlabCols = 32;               // fp16 columns per TMA-store slab (64 B rows)
constexpr int kSlabBytes = 32 * kSlabCols * 2;     // 32 rows x 32 fp16 = 2 KB
constexpr int kSlabBufs = kEpiWarps == 8 ? 1 : 2;  // y staging slabs per epilogue warp
constexpr int kStoreBytes = kEpiWarps * kSlabBufs * kSlabBytes;

// Ring depth and store staging per epilogue: the down GEMM gives up one
// stage to the staging buffers its TMA stores read from.
template <int EPI>
struct Stages {
    static constexpr int value = EPI == 0 ? 4 : MOE_GEMM_DOWN_STAGES;
    static constexpr int store_bytes = EPI == 0 ? 0 : kStoreBytes;
};

enum EpiKind { kSwiGLU = 0, kWeighted = 1 };

struct Params {
    const int32_t* offsets;  // [E+1] group boundaries (device), or nullptr: one group of M rows
    const float* w_perm;     // [M] routing weight per grouped row (kWeighted), or nullptr: weight one
    const int32_t* perm;     // [M] grouped row -> flat assignment t*k + j (GATHER)
    const __nv_bfloat16* x;  // [T, ldx] token matrix the A rows are gathered from (GATHER)
    int64_t ldx;             // row length of x in elements (= K for the gate/up GEMM)
    void* out;               // [M, n_out]: bf16 h (kSwiGLU) or fp16 y (kWeighted)
    int E;
    int M;        // grouped rows
    int K;        // reduction length (multiple of 64)
    int n_out;    // output columns (multiple of 64)
    int n_tiles;  // N tiles per M tile
    int k_top;    // experts per token (GATHER: token = perm[row] / k_top)
    int m_capacity;  // 0: offsets[E] must equal M; 1: M is a capacity, offsets[E] <= M
};

// Shared memory after the stage ring and the store staging buffers.
struct alignas(8) Ctrl {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t done;
    uint32_t tmem_slot;
    volatile int abort_flag;
    int bad;
    int total_mtiles;
    int off[kMaxE + 1];   // group offsets
    int tp[kMaxE + 1];    // exclusive prefix of M tiles per group
    int tok[kBM];         // GATHER: token row of x for each row of the current M tile
};

template <int EPI>
__host__ inline size_t smem_bytes()
{
    return 1024 + (size_t)Stages<EPI>::value * kStageBytes + Stages<EPI>::store_bytes + sizeof(Ctrl);
}
static_assert(1024 + (size_t)Stages<kSwiGLU>::value * kStageBytes + Stages<kSwiGLU>::store_bytes + sizeof(Ctrl) <=
                  227 * 1024,
              "gate/up ring, staging and control exceed 227 KB of shared memory");
static_assert(1024 + (size_t)Stages<kWeighted>::value * kStageBytes + Stages<kWeighted>::store_bytes + sizeof(Ctrl) <=
                  227 * 1024,
              "down ring, staging and control exceed 227 KB of shared memory");

// Work item -> (expert, first row, group end, N tile), for M tiles of
// TILE_ROWS rows: tp[e] is the exclusive prefix of M tiles per group.
template <int TILE_ROWS = kBM>
__device__ __forceinline__ void decode_tile(int64_t w, int n_tiles, const int* tp, const int* off, int E, int& e,
                                            int& row0, int& row_end, int& nt)
{
    const int mt = (int)(w / n_tiles);
    nt = (int)(w - (int64_t)mt * n_tiles);
    int lo = 0, hi = E;  // tp[lo] <= mt < tp[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tp[mid] <= mt)
            lo = mid;
        else
            hi = mid;
    }
    e = lo;
    row0 = off[e] + (mt - tp[e]) * TILE_ROWS;
    row_end = off[e + 1];
}

__device__ __forceinline__ void decode(int64_t w, int n_tiles, const Ctrl& c, int E, int& e, int& row0,
                                       int& row_end, int& nt)
{
    decode_tile<kBM>(w, n_tiles, c.tp, c.off, E, e, row0, row_end, nt);
}

// Reads the group offsets into off[0..E] and, with warp 0, builds tp (the
// exclusive prefix of ceil(count / TILE_ROWS) per group).  The offsets are
// validated: non-decreasing, off[0] = 0, off[E] = M; *bad is set otherwise.
// Contains __syncthreads: every thread of the block must call it.
template <int TILE_ROWS>
__device__ __forceinline__ void build_tile_list(const int32_t* offsets, int E, int M, int* off, int* tp,
                                                int* total, int* bad_out, bool capacity = false)
{
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // offsets == nullptr: a single group of all M rows (E == 1)
    for (int i = threadIdx.x; i <= E; i += blockDim.x) off[i] = offsets ? offsets[i] : (i == 0 ? 0 : M);
    __syncthreads();
    if (warp == 0) {
        int run = 0;
        bool bad = false;
        for (int base = 0; base < E; base += 32) {
            const int e = base + lane;
            int tiles = 0;
            if (e < E) {
                const int cnt = off[e + 1] - off[e];
                if (cnt < 0) bad = true;
                tiles = cnt > 0 ? (cnt + TILE_ROWS - 1) / TILE_ROWS : 0;
            }
            int incl = tiles;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int nb = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += nb;
            }
            if (e < E) tp[e] = run + incl - tiles;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        bad = __any_sync(0xffffffffu, bad);
        if (lane == 0) {
            tp[E] = run;
            *bad_out = (bad || off[0] != 0 || (capacity ? off[E] > M : off[E] != M)) ? 1 : 0;
            *total = run;
            if (*bad_out && blockIdx.x == 0) record_status(kStatusDeviceBounds);
        }
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + __expf(-z)); }

// fp16 pair of w * a, w * b (round to nearest even); `bad` is set when either
// product is outside the fp16 range (|v| >= 65520 rounds to inf) or NaN.
// The two products are one packed fp32 multiply (each rounded as a scalar
// multiply would be), which took 2 us off the down GEMM on the Qwen3-shaped
// and fine-grained layers.
__device__ __forceinline__ uint32_t scaled_f16x2(float w, uint32_t a, uint32_t b, bool& bad)
{
    const float2 v = __fmul2_rn(make_float2(__uint_as_float(a), __uint_as_float(b)), make_float2(w, w));
    bad |= !(fabsf(v.x) < 65520.0f) || !(fabsf(v.y) < 65520.0f);
    const __half2 h = __floats2half2_rn(v.x, v.y);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Token row of x for grouped row r (clamped into range; rows past the group
// end only feed accumulator rows that are never stored).
__device__ __forceinline__ int gather_token(const Params& p, int r)
{
    r = r < p.M ? r : p.M - 1;
    int a = __ldg(p.perm + r);
    if ((unsigned)a >= (unsigned)p.M) {
        record_status(kStatusDeviceBounds);
        a = 0;
    }
    return a / p.k_top;
}

// Drains one 128 x 256 fp32 accumulator tile from TMEM and stores it.  The
// calling warp reads TMEM lane quarter q (rows q*32 .. +31 of the tile, row
// row0 + r for thread r) and column group hf; rows at or past row_end are
// not stored.  tbase addresses the accumulator at this warp's lane quarter.
// kWeighted stages y through NBUF slab buffers of this warp (slab, in turn
// by slab_buf): a buffer is rewritten once the store that last read it is
// done, so up to NBUF stores per warp are in flight.  A slab is 32 rows x SC
// fp16 columns (SC = 32: 64-byte rows, 64-byte swizzle; SC = 64: 128-byte
// rows, 128-byte swizzle), the box of the caller's y map.
template <int EPI, int NBUF = 2, int SC = kSlabCols>
__device__ __forceinline__ void epilogue_tile(const Params& p, const CUtensorMap* tm_out, uint32_t tbase, int row0,
                                              int row_end, int nt, int q, int lane, int hf, float* slab,
                                              int& slab_buf)
{
    const int r = q * 32 + lane;        // tile row owned by this thread
    const int row = row0 + r;
    const bool valid = row < row_end;
    if (EPI == kSwiGLU) {
        // this warp: output columns [cbeg, cbeg + 128 / kColGroups) of the tile
        constexpr int kIters = 128 / kColGroups / 16;
        const int cbeg = hf * (128 / kColGroups);
        __nv_bfloat16* orow =
            static_cast<__nv_bfloat16*>(p.out) + (int64_t)row * p.n_out + nt * 128;
        const int ncols = min(128, p.n_out - nt * 128);
        uint32_t g[2][16], u[2][16];
        tmem_ld16(tbase + cbeg, g[0]);
        tmem_ld16(tbase + 128 + cbeg, u[0]);
        tmem_ld_wait();
#pragma unroll
        for (int it = 0; it < kIters; ++it) {
            const int c0 = cbeg + 16 * it;
            if (it + 1 < kIters) {  // next chunk in flight while this one is processed
                tmem_ld16(tbase + c0 + 16, g[(it + 1) & 1]);
                tmem_ld16(tbase + 128 + c0 + 16, u[(it + 1) & 1]);
            }
            if (valid && c0 < ncols) {
                const uint32_t* gg = g[it & 1];
                const uint32_t* uu = u[it & 1];
                uint32_t packed[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float h0 = silu(__uint_as_float(gg[2 * i])) * __uint_as_float(uu[2 * i]);
                    const float h1 = silu(__uint_as_float(gg[2 * i + 1])) * __uint_as_float(uu[2 * i + 1]);
                    packed[i] = pack_bf16x2(h0, h1);
                }
                uint4* dst = reinterpret_cast<uint4*>(orow + c0);
                dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            }
            tmem_ld_wait();
        }
    } else {
        // this warp: columns [cbeg, cbeg + 256 / kColGroups) of the tile, in
        // slabs of SC columns
        constexpr int kIters = kBN / kColGroups / SC;
        constexpr int kSlabB = 32 * SC * 2;
        const int cbeg = hf * (kBN / kColGroups);
        const float wgt = valid ? (p.w_perm ? __ldg(p.w_perm + row) : 1.0f) : 0.0f;  // no weights: one
        const int wrow0 = row0 + q * 32;                   // first row of this warp's slab
        const bool whole = wrow0 + 31 < row_end;           // all 32 rows belong to the group
        __half* orow = static_cast<__half*>(p.out) + (int64_t)row * p.n_out + nt * kBN;
        const int ncols = min(kBN, p.n_out - nt * kBN);
        bool bad = false;
        if constexpr (SC == 64) {
#pragma unroll 1
            for (int it = 0; it < kIters; ++it) {
                const int c0 = cbeg + SC * it;
                if (c0 < ncols) {  // warp-uniform (n_out % 64 == 0)
                    uint32_t pk[32];
#pragma unroll
                    for (int h4 = 0; h4 < 4; h4 += 2) {
                        uint32_t a0[16], a1[16];
                        tmem_ld16(tbase + c0 + 16 * h4, a0);
                        tmem_ld16(tbase + c0 + 16 * h4 + 16, a1);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            pk[8 * h4 + i] = scaled_f16x2(wgt, a0[2 * i], a0[2 * i + 1], bad);
                            pk[8 * h4 + 8 + i] = scaled_f16x2(wgt, a1[2 * i], a1[2 * i + 1], bad);
                        }
                    }
                    if (whole) {
                        uint32_t* buf = reinterpret_cast<uint32_t*>(slab) + slab_buf * (kSlabB / 4);
                        if (lane == 0) bulk_wait_group_read<NBUF - 1>();  // the store that last read `buf` is done
                        __syncwarp();
                        // row `lane` of the slab: 8 x 16 B chunks, 128-byte swizzle
                        uint4* rowp = reinterpret_cast<uint4*>(buf + lane * (SC / 2));
                        const int sw = lane & 7;
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            rowp[v ^ sw] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(tm_out, buf, nt * kBN + c0, wrow0);
                            bulk_commit_group();
                        }
                        slab_buf = slab_buf + 1 == NBUF ? 0 : slab_buf + 1;
                    } else if (valid) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
                        for (int v = 0; v < 8; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                    }
                }
            }
        } else {
            uint32_t lo[2][16], hi[2][16];  // columns 0..15 and 16..31 of a slab
            tmem_ld16(tbase + cbeg, lo[0]);
            tmem_ld16(tbase + cbeg + 16, hi[0]);
            tmem_ld_wait();
#pragma unroll
            for (int it = 0; it < kIters; ++it) {
                const int c0 = cbeg + SC * it;
                if (it + 1 < kIters) {
                    tmem_ld16(tbase + c0 + SC, lo[(it + 1) & 1]);
                    tmem_ld16(tbase + c0 + SC + 16, hi[(it + 1) & 1]);
                }
                const uint32_t* al = lo[it & 1];
                const uint32_t* ah = hi[it & 1];
                if (c0 < ncols) {  // warp-uniform (n_out % 64 == 0)
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        pk[i] = scaled_f16x2(wgt, al[2 * i], al[2 * i + 1], bad);
                        pk[8 + i] = scaled_f16x2(wgt, ah[2 * i], ah[2 * i + 1], bad);
                    }
                    if (whole) {
                        uint32_t* buf = reinterpret_cast<uint32_t*>(slab) + slab_buf * (kSlabB / 4);
                        if (lane == 0) bulk_wait_group_read<NBUF - 1>();  // the store that last read `buf` is done
                        __syncwarp();
                        // row `lane` of the slab: 4 x 16 B chunks, 64-byte swizzle
                        uint4* rowp = reinterpret_cast<uint4*>(buf + lane * (SC / 2));
                        const int sw = (lane >> 1) & 3;
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            rowp[v ^ sw] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(tm_out, buf, nt * kBN + c0, wrow0);
                            bulk_commit_group();
                        }
                        slab_buf = slab_buf + 1 == NBUF ? 0 : slab_buf + 1;
                    } else if (valid) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
                        for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                    }
                }
                tmem_ld_wait();
            }
        }
        if (__any_sync(0xffffffffu, bad && valid) && lane == 0) record_status(kStatusDeviceRange);
    }
}

template <int EPI, bool GATHER>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                        const __grid_constant__ CUtensorMap tm_b1, const __grid_constant__ CUtensorMap tm_out,
                        Params p)
{
    constexpr int kStages = Stages<EPI>::value;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stage_out = smem + (size_t)kStages * kStageBytes;
    Ctrl& c = *reinterpret_cast<Ctrl*>(stage_out + Stages<EPI>::store_bytes);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint64_t limit = g_wait_limit_ns;
    const int E = p.E;

    if (threadIdx.x == 32) {
        for (int s = 0; s < kStages; ++s) {
            // GATHER: the TMA arrival plus one cp.async completion per lane
            mbar_init(&c.full[s], GATHER ? 1 + 32 : 1);
            mbar_init(&c.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&c.acc_full[b], 1);
            mbar_init(&c.acc_empty[b], kEpiWarps * 32);
        }
        mbar_init(&c.done, 1);
        c.abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_map(&tm_a);
        tma_prefetch_map(&tm_b0);
        if (EPI == kSwiGLU) tma_prefetch_map(&tm_b1);
        if (EPI == kWeighted) tma_prefetch_map(&tm_out);
    }
    if (warp == 1) {
        __syncwarp();
        tmem_alloc(&c.tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = c.tmem_slot;
    // the offsets and A rows come from earlier kernels on the stream
    pdl_trigger();
    pdl_wait();
    // ---- tile list from the device offsets (validated) ----
    build_tile_list<kBM>(p.offsets, E, p.M, c.off, c.tp, &c.total_mtiles, &c.bad, p.m_capacity != 0);
    __syncthreads();
    const int64_t total_work = c.bad ? 0 : (int64_t)c.total_mtiles * p.n_tiles;
    const int num_kb = p.K / kBK;

    if (warp == 0 && (GATHER || lane == 0)) {
        // ---------------------------------------------------- TMA producer
        // GATHER: the whole warp (it copies the A rows); otherwise lane 0.
        constexpr unsigned pmask = GATHER ? 0xffffffffu : 1u;
        int s = 0;
        uint32_t ph = 0;
        int64_t issued = 0;
        for (int64_t w = blockIdx.x; w < total_work; w += gridDim.x) {
            if (__shfl_sync(pmask, c.abort_flag, 0)) break;  // uniform exit
            int e, row0, row_end, nt;
            decode(w, p.n_tiles, c, E, e, row0, row_end, nt);
            if (GATHER) {
                __syncwarp(pmask);  // every lane is done issuing copies that read c.tok
#pragma unroll
                for (int i = 0; i < kBM / 32; ++i) c.tok[lane + 32 * i] = gather_token(p, row0 + lane + 32 * i);
                __syncwarp(pmask);
            }
            const int krow0 = e * p.K;
            bool ok = true;
            for (int kb = 0; kb < num_kb; ++kb) {
                bool ready = true;
                if (lane == 0) ready = mbar_wait(&c.empty[s], ph ^ 1u, limit);
                if (!__shfl_sync(pmask, ready ? 1 : 0, 0)) {
                    ok = false;
                    break;
                }
                uint8_t* sa = smem + (size_t)s * kStageBytes;
                uint8_t* sb = sa + kABytes;
                if (lane == 0) mbar_arrive_expect_tx(&c.full[s], (uint32_t)(GATHER ? kBBytes : kStageBytes));
                if (GATHER) {
                    // lane = 8 * g + ch: 16-byte chunk ch of rows 4i + g, i = 0..31
                    const int g = lane >> 3, ch = lane & 7;
                    const __nv_bfloat16* xk = p.x + (size_t)kb * kBK + ch * 8;
#pragma unroll 8
                    for (int i = 0; i < kBM / 4; ++i) {
                        const int r = 4 * i + g;
                        cp_async_16(sa + r * 128 + ((ch ^ (r & 7)) << 4), xk + (size_t)c.tok[r] * p.ldx);
                    }
                    cp_async_arrive_noinc(&c.full[s]);
                }
                if (lane == 0) {
                    if (!GATHER) tma_load_2d(sa, &tm_a, &c.full[s], kb * kBK, row0);
                    const int kr = krow0 + kb * kBK;
                    if (EPI == kSwiGLU) {
                        const int n0 = nt * 128;
                        tma_load_2d(sb + 0 * kChunkBytes, &tm_b0, &c.full[s], n0, kr);
                        tma_load_2d(sb + 1 * kChunkBytes, &tm_b0, &c.full[s], n0 + 64, kr);
                        tma_load_2d(sb + 2 * kChunkBytes, &tm_b1, &c.full[s], n0, kr);
                        tma_load_2d(sb + 3 * kChunkBytes, &tm_b1, &c.full[s], n0 + 64, kr);
                    } else {
                        const int n0 = nt * kBN;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            tma_load_2d(sb + q * kChunkBytes, &tm_b0, &c.full[s], n0 + 64 * q, kr);
                    }
                }
                ++issued;
                if (++s == kStages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (!ok) {
                if (lane == 0) c.abort_flag = 1;
                break;
            }
        }
        // Never leave the CTA with a copy still landing in its shared memory.
        if (GATHER) cp_async_wait_all();
        if (lane == 0) {
            for (int q = 0; q < kStages; ++q) {
                const int64_t cnt = issued / kStages + (q < issued % kStages ? 1 : 0);
                if (cnt > 0) mbar_wait(&c.full[q], (uint32_t)(cnt - 1) & 1u, drain_limit(limit));
            }
        }
        __syncwarp(pmask);
    } else if (warp == 0) {
        // lanes 1..31 of the producer warp have nothing to do without GATHER
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, false, true);
            int s = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t acc_ph = 0;
            for (int64_t w = blockIdx.x; w < total_work && !c.abort_flag; w += gridDim.x) {
                if (!mbar_wait(&c.acc_empty[acc], acc_ph ^ 1u, limit)) {
                    c.abort_flag = 1;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * kBN);
                bool ok = true;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&c.full[s], ph, limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_base = smem_u32(smem + (size_t)s * kStageBytes);
                    const uint32_t b_base = a_base + kABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t adesc = smem_desc_sw128(a_base + kk * 32, 16, 1024);
                        const uint64_t bdesc = smem_desc_sw128(b_base + kk * 2048, kChunkBytes, 1024);
                        mma_bf16_ss(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit(&c.empty[s]);  // frees the stage once these MMAs are done
                    if (++s == kStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) {
                    c.abort_flag = 1;
                    break;
                }
                mma_commit(&c.acc_full[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_ph ^= 1u;
                }
            }
            mma_commit(&c.done);
            mbar_wait(&c.done, 0, drain_limit(limit));
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue
        // Warp w may only touch TMEM lanes 32*(w%4)..+31: warps 2..5 and 6..9
        // each cover the four lane quarters; the two groups split the columns.
        const int ew = warp - 2;            // 0..7
        const int q = warp & 3;             // TMEM lane quarter
        const int hf = ew >> 2;             // column group (0 when kColGroups == 1)
        float* slab = reinterpret_cast<float*>(stage_out + ew * kSlabBufs * kSlabBytes);
        int slab_buf = 0;
        int acc = 0;
        uint32_t acc_ph = 0;
        for (int64_t w = blockIdx.x; w < total_work; w += gridDim.x) {
            int e, row0, row_end, nt;
            decode(w, p.n_tiles, c, E, e, row0, row_end, nt);
            // Lane 0 polls (so idle epilogue warps do not steal issue slots
            // from the MMA thread); the warp continues together, since the
            // TMEM loads below are warp-collective.
            bool ready = true;
            if (lane == 0) ready = mbar_wait(&c.acc_full[acc], acc_ph, limit);
            ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
            if (!ready) {
                c.abort_flag = 1;
                break;
            }
            tc_fence_after_sync();
            const uint32_t tbase = tmem + (uint32_t)(acc * kBN) + ((uint32_t)(q * 32) << 16);
            epilogue_tile<EPI, kSlabBufs>(p, &tm_out, tbase, row0, row_end, nt, q, lane, hf, slab, slab_buf);
            tc_fence_before_sync();
            mbar_arrive(&c.acc_empty[acc]);
            if (++acc == 2) {
                acc = 0;
                acc_ph ^= 1u;
            }
        }
        if (EPI == kWeighted && lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace gemm
}  // namespace moe
