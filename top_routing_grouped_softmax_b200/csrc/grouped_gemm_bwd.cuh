// grouped_gemm_bwd.cuh -- the grouped GEMMs of the MoE block's backward on
// CTA pairs (tcgen05 cta_group::2), with their epilogues fused in.
//
// The backward follows the memory rule of the SonicMoE comparison page ("SonicMoE
// vs conventional MoE", core difference 1): only the routing is kept, and the
// expert activations g, u and h are recomputed from the grouped rows of x.
// Rows are grouped by expert with every group starting on a 64-row boundary
// (the rows between a group's end and the next boundary are zero in every
// row operand), so a group's rows can also serve as the reduction axis of
// the weight gradients in whole 64-row blocks.
//
// Four kinds share one pipeline (the CTA-pair ring of the forward's grouped
// GEMM: TMA producer, one MMA thread in the even CTA issuing M=256 N=256 K=16
// pair MMAs, eight epilogue warps per CTA over a double-buffered accumulator):
//
//   kGU  g, u = x_perm . W_gate[e], x_perm . W_up[e]      (recompute)
//        A = x_perm rows (K-major), B = weight columns (MN-major): the even
//        CTA loads W_gate's 128 columns, the odd CTA the matching W_up ones,
//        so accumulator columns 0..127 are g and 128..255 are u.  Stores g, u
//        and hw = w silu(g) u (the operand of the W_down gradient), bf16.
//   kDH  dh = w . (dout_perm . W_down[e]^T), then the SwiGLU derivative:
//          s = 1/(1+e^-g),  h = g s u,
//          dg = dh u s (1 + g (1 - s)),  du = dh g s,
//        and the routing-weight gradient's partial dot products
//          dwp[row][2 nt + half] = sum over that half of the tile's columns of (dh / w) h
//        (dh / w is the unweighted accumulator: dout . (h W_down) = (dout W_down^T) . h).
//        A = dout_perm rows (K-major), B = W_down[e] rows (K-major: W_down[e] is
//        [f][d], its rows are the output columns).  Stores dg and du as bf16
//        (in place of g and u).
//   kDX  out = A1 . B1^T + A2 . B2^T with K split in two halves (the first
//        k_split 64-blocks read A1/B1, the rest A2/B2):
//        dx_perm = dg . W_gate[e]^T + du . W_up[e]^T (out rounded to bf16), and
//        (one group, one half) the router's dx = dlogit . W_router^T (fp32 out).
//        Whole 32-row slabs go out by TMA store; a slab that crosses the
//        group's end is stored row by row.
//   kDW  out[e] = A_e^T . B_e, reduced over the rows of group e:
//        A = the group's rows read MN-major (x_perm or hw, or x), B likewise
//        (dg | du split over the pair, or dout_perm / dlogit).  One work item
//        is (expert, 256-row M tile, 256-column N tile); an empty group writes
//        zeros.  fp32 out (or, as an option, the fp32 result rounded to bf16)
//        by 3-D TMA store ([E][rows][cols] views clip the partial tiles).  With
//        k_chunk the "groups" are fixed chunks of one operand pair's rows, so a
//        long reduction (the router's weight gradient over all tokens) is split
//        over many CTA pairs and the partial results are summed afterwards.
//
// No TMA load uses multicast.  Every wait is bounded (see ptx.cuh).
#pragma once

#include "grouped_gemm_pair.cuh"

namespace moe {
namespace bwd {

using gemm::kABytes;
using gemm::kBK;
using gemm::kBM;
using gemm::kBN;
using gemm::kChunkBytes;
using gemm::kMaxE;
using gemm::kPairRows;
using gemm::kPairStageBytes;
using gemm::kPairStages;
using gemm::kTmemCols;

enum Kind { kGU = 0, kDH = 1, kDX = 2, kDW = 3 };

// Eight epilogue warps: two per TMEM lane quarter, each taking half of the
// tile's columns.  The backward's epilogues do more per element than the
// forward's (kDH reads g and u and writes three bf16 outputs; kDW and kDX
// write fp32), so they need the issue slots of eight warps to keep pace
// with the MMAs.
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + kEpiWarps * 32;

struct Params {
    const int32_t* offsets;  // [E+1] group starts; nullptr: one group of M rows
    const float* w_perm;     // kGU, kDH: routing weight of each grouped row
    const __nv_bfloat16* g;  // kDH: recomputed g, u [rows][ld_f]
    const __nv_bfloat16* u;
    __nv_bfloat16* out_g;    // kGU: g;  kDH: dg        [rows][ld_f]
    __nv_bfloat16* out_u;    // kGU: u;  kDH: du
    __nv_bfloat16* out_hw;   // kGU: w * h
    float* dwp;              // kDH: [rows][2 * n_tiles] partial dot products (two column halves per tile)
    float* out0;             // kDX: [rows][ld_out];  kDW: [E][m_total][ld_out] (gate part when split)
    float* out1;             // kDW split: the up part
    int64_t ld_f;            // row length of g, u, dg, du, hw
    int64_t ld_out;          // row length of out0 / out1
    int E;
    int M;                   // grouped rows (capacity: offsets[E] <= M)
    int K;                   // kGU, kDH, kDX: reduction length (kDX: both halves)
    int k_split;             // kDX: 64-blocks read from A1/B1 below this, A2/B2 from it on
    int n_out;               // output columns
    int n_tiles;             // N tiles per item (kGU: 128 output columns each, else 256)
    int b_rows;              // kGU: weight rows per expert (d); kDH, kDX: B rows per expert (f, d)
    int m_total;             // kDW: output rows per expert
    int m_tiles;             // kDW: 256-row M tiles per expert
    int split_b;             // kDW: 1 = B halves from two tensors (dg | du), two outputs
    int out_bf16;            // kDX: 1 = out0 holds bf16 values (rows of ld_out), stored through a 2-D map;
                             // kDW: 1 = out0 / out1 hold bf16 values (32 x 32 slabs of 2 KB, 64-byte swizzle)
    int k_chunk;             // kDW: > 0 = group e is rows [e k_chunk, min((e + 1) k_chunk, M)) of one
                             // M-row operand pair (split K; offsets unused), else the offsets' groups
};

struct alignas(8) Ctrl {
    uint64_t full[kPairStages];
    uint64_t empty[kPairStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t done;
    uint32_t tmem_slot;
    volatile int abort_flag;
    int bad;
    int total_mtiles;
    int off[kMaxE + 1];
    int tp[kMaxE + 1];
};

// Ring depth per kind: kDW and kDX give a stage to the staging slabs of
// their TMA-store epilogues (eight warps x 32 x 32 fp32 slabs).
// Tuning constants (overridable at build time for measurements): staging
// slabs per epilogue warp and the ring depth of the TMA-store kinds.  One
// slab per warp and five stages measured 4 % faster over the whole backward
// on the Qwen3-shaped layer than two slabs and four stages (2.25 against
// 2.35 ms): the deeper operand ring matters more than a second slab.
#ifndef MOE_BWD_SLAB_BUFS
#define MOE_BWD_SLAB_BUFS 1
#endif
#ifndef MOE_BWD_STORE_STAGES
#define MOE_BWD_STORE_STAGES 5
#endif
constexpr int kSlabBufs = MOE_BWD_SLAB_BUFS;
constexpr int kSlabBytes = 32 * 32 * 4;
constexpr int kStoreBytes = kEpiWarps * kSlabBufs * kSlabBytes;
static_assert(kSlabBufs == 1 || kSlabBufs == 2, "staging slabs per warp");
// kDH stages each warp's 32-row x 16-column dg and du chunk in one 2 KB
// slab (dg in the first KB, du in the second) for two 2-D TMA stores.
constexpr int kDhSlabBytes = 2048;
__host__ __device__ constexpr int slab_stride_for(int kind)
{
    return kind == kDH ? kDhSlabBytes : kSlabBufs * kSlabBytes;
}
__host__ __device__ constexpr int stages_for(int kind)
{
    return (kind == kDW || kind == kDX) ? MOE_BWD_STORE_STAGES : kPairStages;
}
__host__ __device__ constexpr int store_bytes_for(int kind)
{
    return (kind == kDW || kind == kDX) ? kStoreBytes : (kind == kDH ? kEpiWarps * kDhSlabBytes : 0);
}

template <int KIND>
__host__ inline size_t smem_bytes()
{
    return 1024 + (size_t)stages_for(KIND) * kPairStageBytes + store_bytes_for(KIND) + sizeof(Ctrl);
}
static_assert(1024 + (size_t)stages_for(kDH) * kPairStageBytes + store_bytes_for(kDH) + sizeof(Ctrl) <= 227 * 1024,
              "dh ring, staging and control exceed 227 KB of shared memory");
static_assert(1024 + (size_t)stages_for(kDW) * kPairStageBytes + store_bytes_for(kDW) + sizeof(Ctrl) <= 227 * 1024,
              "weight-gradient ring, staging and control exceed 227 KB of shared memory");

// One work item of kind KIND: the expert, the first grouped row (M-grouped
// kinds) or M tile (kDW), the group's row range, the N tile and the number
// of 64-row k-blocks.
struct Item {
    int e, row0, row_end, nt, mt, kstart, num_kb;
};

template <int KIND>
__device__ __forceinline__ Item decode_item(int64_t w, const Params& p, const Ctrl& c)
{
    Item it;
    if constexpr (KIND == kDW) {
        const int64_t per_e = (int64_t)p.m_tiles * p.n_tiles;
        it.e = (int)(w / per_e);
        const int rem = (int)(w - (int64_t)it.e * per_e);
        it.mt = rem / p.n_tiles;
        it.nt = rem - it.mt * p.n_tiles;
        if (p.k_chunk > 0) {
            it.kstart = it.e * p.k_chunk;
            it.row_end = min(it.kstart + p.k_chunk, p.M);
        } else {
            it.kstart = c.off[it.e];
            it.row_end = c.off[it.e + 1];
        }
        it.num_kb = (it.row_end - it.kstart + kBK - 1) / kBK;
        it.row0 = it.kstart;
    } else {
        gemm::decode_tile<kPairRows>(w, p.n_tiles, c.tp, c.off, p.E, it.e, it.row0, it.row_end, it.nt);
        it.mt = 0;
        it.kstart = 0;
        it.num_kb = p.K / kBK;
    }
    return it;
}

// 1 / (1 + e^-z) with the fast reciprocal division (about 2 ulp in fp32; the
// results are rounded to bf16).
__device__ __forceinline__ float sigmoid(float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); }

__device__ __forceinline__ void unpack_bf16x8(const uint4& q, float (&v)[8])
{
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

// Sixteen fp32 values to one row segment (four 16-byte stores).
__device__ __forceinline__ void store_f32x16(float* dst, const uint32_t (&r)[16])
{
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int v = 0; v < 4; ++v)
        d4[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]), __uint_as_float(r[4 * v + 2]),
                            __uint_as_float(r[4 * v + 3]));
}

__device__ __forceinline__ void store_zero_f32x16(float* dst)
{
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int v = 0; v < 4; ++v) d4[v] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// Drains one accumulator tile.  The calling warp reads TMEM lane quarter q:
// row q*32 + lane of this CTA's 128 rows.  tbase addresses the accumulator
// at this warp's lane quarter.
// `half` selects the columns this warp drains: half of the tile's output
// columns (kGU: 64 of 128; the others: 128 of 256).  kDW and kDX stage their
// output in `slab` (kSlabBufs 4 KB buffers of this warp, taken in turn)
// and store it with TMA: kDW through tm_o0 / tm_o1 ([E][m_total][n_out]
// fp32 views; rows past m_total and columns past n_out are not written),
// kDX through tm_o0 ([1][rows][n_out] fp32, or with p.out_bf16 a 2-D
// [rows][n_out] bf16 map whose 32 x 32 box is a 2 KB slab).
template <int KIND>
__device__ __forceinline__ void epilogue(const Params& p, const Item& it, uint32_t tbase, uint32_t rank, int q,
                                         int lane, int half, const CUtensorMap* tm_o0, const CUtensorMap* tm_o1,
                                         float* slab, int& slab_buf)
{
    const int r = (int)rank * kBM + q * 32 + lane;  // row of the 256-row pair tile
    if constexpr (KIND == kGU) {
        // g and u (bf16, for the dh epilogue) and w h = w silu(g) u (bf16,
        // the A operand of the W_down gradient) from the fp32 accumulators
        const int row = it.row0 + r;
        const bool valid = row < it.row_end;
        const int c_base = it.nt * 128;
        const int ncols = min(128, p.n_out - c_base);
        const float w = valid ? __ldg(p.w_perm + row) : 0.0f;
#pragma unroll 1
        for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 16) {
            uint32_t g[16], u[16];
            tmem_ld16(tbase + c0, g);
            tmem_ld16(tbase + 128 + c0, u);
            tmem_ld_wait();
            if (valid && c0 < ncols) {
                uint32_t pg[8], pu[8], ph[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
                    const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
                    pg[i] = gemm::pack_bf16x2(g0, g1);
                    pu[i] = gemm::pack_bf16x2(u0, u1);
                    ph[i] = gemm::pack_bf16x2(w * (g0 * sigmoid(g0) * u0), w * (g1 * sigmoid(g1) * u1));
                }
                const int64_t off = (int64_t)row * p.ld_f + c_base + c0;
                uint4* dg = reinterpret_cast<uint4*>(p.out_g + off);
                uint4* du = reinterpret_cast<uint4*>(p.out_u + off);
                uint4* dh = reinterpret_cast<uint4*>(p.out_hw + off);
                dg[0] = make_uint4(pg[0], pg[1], pg[2], pg[3]);
                dg[1] = make_uint4(pg[4], pg[5], pg[6], pg[7]);
                du[0] = make_uint4(pu[0], pu[1], pu[2], pu[3]);
                du[1] = make_uint4(pu[4], pu[5], pu[6], pu[7]);
                dh[0] = make_uint4(ph[0], ph[1], ph[2], ph[3]);
                dh[1] = make_uint4(ph[4], ph[5], ph[6], ph[7]);
            }
        }
    } else if constexpr (KIND == kDH) {
        const int row = it.row0 + r;
        const bool valid = row < it.row_end;
        const int c_base = it.nt * kBN;
        const int ncols = min(kBN, p.n_out - c_base);
        const float w = valid ? __ldg(p.w_perm + row) : 0.0f;
        const int64_t row_off = (int64_t)row * p.ld_f + c_base;
        const int wrow0 = it.row0 + (int)rank * kBM + q * 32;
        const bool whole = wrow0 + 31 < it.row_end;  // warp-uniform: all 32 rows belong to the group
        float dot = 0.0f;
        // g and u of the next two 16-column chunks are in flight while this
        // chunk is processed (the loads are row-strided across the warp and
        // would otherwise expose their latency once per chunk)
        uint4 gq[3][2], uq[3][2];
        auto fetch = [&](int c0, int b) {
            if (valid && c0 < ncols) {
                const uint4* gp = reinterpret_cast<const uint4*>(p.g + row_off + c0);
                const uint4* up = reinterpret_cast<const uint4*>(p.u + row_off + c0);
                gq[b][0] = __ldg(gp);
                gq[b][1] = __ldg(gp + 1);
                uq[b][0] = __ldg(up);
                uq[b][1] = __ldg(up + 1);
            }
        };
        fetch(half * 128, 0);
        fetch(half * 128 + 16, 1);
        // the accumulator of the next chunk is read from TMEM while this one
        // is processed (tcgen05.wait::ld waits for all of a thread's loads,
        // so the wait comes after the math)
        uint32_t accb[2][16];
        tmem_ld16(tbase + half * 128, accb[0]);
        tmem_ld_wait();
#pragma unroll
        for (int ci = 0; ci < 8; ++ci) {
            const int c0 = half * 128 + ci * 16;
            if (ci + 2 < 8) fetch(c0 + 32, (ci + 2) % 3);
            if (ci + 1 < 8) tmem_ld16(tbase + c0 + 16, accb[(ci + 1) & 1]);
            const uint32_t* acc = accb[ci & 1];
            if (valid && c0 < ncols) {
                float g[16], u[16];
                unpack_bf16x8(gq[ci % 3][0], *reinterpret_cast<float(*)[8]>(&g[0]));
                unpack_bf16x8(gq[ci % 3][1], *reinterpret_cast<float(*)[8]>(&g[8]));
                unpack_bf16x8(uq[ci % 3][0], *reinterpret_cast<float(*)[8]>(&u[0]));
                unpack_bf16x8(uq[ci % 3][1], *reinterpret_cast<float(*)[8]>(&u[8]));
                uint32_t pdg[8], pdu[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    // two columns at a time: packed fp32 multiplies and FMAs
                    // (each lane rounded as the scalar operation would be);
                    // dh = w dhu, where dhu = dout . W_down^T is the
                    // unweighted accumulator, and dot is a serial sum
                    const float2 dhu = make_float2(__uint_as_float(acc[2 * i]), __uint_as_float(acc[2 * i + 1]));
                    const float2 gg = make_float2(g[2 * i], g[2 * i + 1]);
                    const float2 uu = make_float2(u[2 * i], u[2 * i + 1]);
                    const float2 sg = make_float2(sigmoid(gg.x), sigmoid(gg.y));
                    const float2 gs = __fmul2_rn(gg, sg);
                    const float2 dh = __fmul2_rn(make_float2(w, w), dhu);
                    const float2 hu = __fmul2_rn(gs, uu);
                    dot = fmaf(dhu.x, hu.x, dot);
                    dot = fmaf(dhu.y, hu.y, dot);
                    const float2 om = __ffma2_rn(sg, make_float2(-1.0f, -1.0f), make_float2(1.0f, 1.0f));
                    const float2 t = __ffma2_rn(gg, om, make_float2(1.0f, 1.0f));
                    const float2 dg = __fmul2_rn(__fmul2_rn(__fmul2_rn(dh, uu), sg), t);
                    const float2 du = __fmul2_rn(dh, gs);
                    pdg[i] = gemm::pack_bf16x2(dg.x, dg.y);
                    pdu[i] = gemm::pack_bf16x2(du.x, du.y);
                }
                if (whole) {
                    // the warp's 32 x 16 chunk of dg and du through the slab:
                    // two 2-D TMA stores instead of 64 row-strided 32-byte ones
                    uint4* sg = reinterpret_cast<uint4*>(slab) + lane * 2;
                    uint4* su = reinterpret_cast<uint4*>(slab) + 64 + lane * 2;
                    if (lane == 0) bulk_wait_group_read<0>();  // the slab's last stores have read it
                    __syncwarp();
                    sg[0] = make_uint4(pdg[0], pdg[1], pdg[2], pdg[3]);
                    sg[1] = make_uint4(pdg[4], pdg[5], pdg[6], pdg[7]);
                    su[0] = make_uint4(pdu[0], pdu[1], pdu[2], pdu[3]);
                    su[1] = make_uint4(pdu[4], pdu[5], pdu[6], pdu[7]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(tm_o0, slab, c_base + c0, wrow0);
                        tma_store_2d(tm_o1, reinterpret_cast<uint8_t*>(slab) + 1024, c_base + c0, wrow0);
                        bulk_commit_group();
                    }
                } else {
                    uint4* dgp = reinterpret_cast<uint4*>(p.out_g + row_off + c0);
                    uint4* dup = reinterpret_cast<uint4*>(p.out_u + row_off + c0);
                    dgp[0] = make_uint4(pdg[0], pdg[1], pdg[2], pdg[3]);
                    dgp[1] = make_uint4(pdg[4], pdg[5], pdg[6], pdg[7]);
                    dup[0] = make_uint4(pdu[0], pdu[1], pdu[2], pdu[3]);
                    dup[1] = make_uint4(pdu[4], pdu[5], pdu[6], pdu[7]);
                }
            }
            tmem_ld_wait();
        }
        if (valid) p.dwp[(int64_t)row * (2 * p.n_tiles) + 2 * it.nt + half] = dot;
    } else if constexpr (KIND == kDX) {
        // 32 x 32 fp32 slabs written by TMA when all 32 rows of this warp
        // belong to the group (the rows past a group's end belong to the next
        // group and are left alone); a warp with a partial slab stores its
        // valid rows itself
        const int row = it.row0 + r;
        const bool valid = row < it.row_end;
        const int c_base = it.nt * kBN;
        const int ncols = min(kBN, p.n_out - c_base);
        const int wrow0 = it.row0 + (int)rank * kBM + q * 32;
        const bool whole = wrow0 + 31 < it.row_end;  // warp-uniform
        uint32_t lob[2][16], hib[2][16];  // this slab and the next one in flight
        tmem_ld16(tbase + half * 128, lob[0]);
        tmem_ld16(tbase + half * 128 + 16, hib[0]);
        tmem_ld_wait();
#pragma unroll
        for (int si = 0; si < 4; ++si) {
            const int c0 = half * 128 + si * 32;
            if (si + 1 < 4) {
                tmem_ld16(tbase + c0 + 32, lob[(si + 1) & 1]);
                tmem_ld16(tbase + c0 + 48, hib[(si + 1) & 1]);
            }
            const uint32_t(&lo)[16] = lob[si & 1];
            const uint32_t(&hi)[16] = hib[si & 1];
            if (p.out_bf16) {
                // bf16 rows: a 32 x 32 slab is 2 KB (64-byte rows, 64-byte swizzle)
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    pk[i] = gemm::pack_bf16x2(__uint_as_float(lo[2 * i]), __uint_as_float(lo[2 * i + 1]));
                    pk[8 + i] = gemm::pack_bf16x2(__uint_as_float(hi[2 * i]), __uint_as_float(hi[2 * i + 1]));
                }
                if (c0 < ncols && whole) {
                    uint32_t* buf = reinterpret_cast<uint32_t*>(slab) + slab_buf * (kSlabBytes / 4);
                    if (lane == 0) bulk_wait_group_read<kSlabBufs - 1>();
                    __syncwarp();
                    uint4* rowp = reinterpret_cast<uint4*>(buf + lane * 16);
                    const int sw = (lane >> 1) & 3;
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        rowp[v ^ sw] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(tm_o0, buf, c_base + c0, wrow0);
                        bulk_commit_group();
                    }
                    slab_buf = (slab_buf + 1) % kSlabBufs;
                } else if (c0 < ncols && valid) {
                    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out0) +
                                                          (int64_t)row * p.ld_out + c_base + c0);
#pragma unroll
                    for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                }
            } else if (c0 < ncols && whole) {  // c0 < ncols is warp-uniform (n_out % 64 == 0)
                uint32_t* buf = reinterpret_cast<uint32_t*>(slab) + slab_buf * (kSlabBytes / 4);
                if (lane == 0) bulk_wait_group_read<kSlabBufs - 1>();
                __syncwarp();
                uint4* rowp = reinterpret_cast<uint4*>(buf + lane * 32);
                const int sw = lane & 7;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    rowp[v ^ sw] = make_uint4(lo[4 * v], lo[4 * v + 1], lo[4 * v + 2], lo[4 * v + 3]);
                    rowp[(4 + v) ^ sw] = make_uint4(hi[4 * v], hi[4 * v + 1], hi[4 * v + 2], hi[4 * v + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(tm_o0, buf, c_base + c0, wrow0, 0);
                    bulk_commit_group();
                }
                slab_buf = (slab_buf + 1) % kSlabBufs;
            } else if (c0 < ncols && valid) {
                float* dst = p.out0 + (int64_t)row * p.ld_out + c_base + c0;
                store_f32x16(dst, lo);
                store_f32x16(dst + 16, hi);
            }
            tmem_ld_wait();
        }
    } else {  // kDW: 32 x 32 fp32 slabs staged in shared memory, written by TMA
        const bool empty = it.num_kb == 0;
        const int m0 = it.mt * kPairRows + (int)rank * kBM + q * 32;  // first row of this warp's slabs
        uint32_t lob[2][16], hib[2][16];  // this slab and the next one in flight
        tmem_ld16(tbase + half * 128, lob[0]);
        tmem_ld16(tbase + half * 128 + 16, hib[0]);
        tmem_ld_wait();
#pragma unroll
        for (int si = 0; si < 4; ++si) {
            const int c0 = half * 128 + si * 32;
            if (si + 1 < 4) {
                tmem_ld16(tbase + c0 + 32, lob[(si + 1) & 1]);
                tmem_ld16(tbase + c0 + 48, hib[(si + 1) & 1]);
            }
            const uint32_t(&lo)[16] = lob[si & 1];
            const uint32_t(&hi)[16] = hib[si & 1];
            uint32_t* buf = reinterpret_cast<uint32_t*>(slab) + slab_buf * (kSlabBytes / 4);
            if (lane == 0) bulk_wait_group_read<kSlabBufs - 1>();  // the store that last read `buf` is done
            __syncwarp();
            if (p.out_bf16) {
                // row `lane` of a 32 x 32 bf16 slab: 4 x 16 B chunks, 64-byte swizzle
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    pk[i] = empty ? 0u : gemm::pack_bf16x2(__uint_as_float(lo[2 * i]), __uint_as_float(lo[2 * i + 1]));
                    pk[8 + i] = empty ? 0u
                                      : gemm::pack_bf16x2(__uint_as_float(hi[2 * i]), __uint_as_float(hi[2 * i + 1]));
                }
                uint4* rowp = reinterpret_cast<uint4*>(buf + lane * 16);
                const int sw = (lane >> 1) & 3;
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    rowp[v ^ sw] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            } else {
                // row `lane` of the slab: 8 x 16 B chunks, 128-byte swizzle
                uint4* rowp = reinterpret_cast<uint4*>(buf + lane * 32);
                const int sw = lane & 7;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    rowp[v ^ sw] = empty ? make_uint4(0u, 0u, 0u, 0u)
                                         : make_uint4(lo[4 * v], lo[4 * v + 1], lo[4 * v + 2], lo[4 * v + 3]);
                    rowp[(4 + v) ^ sw] = empty ? make_uint4(0u, 0u, 0u, 0u)
                                               : make_uint4(hi[4 * v], hi[4 * v + 1], hi[4 * v + 2], hi[4 * v + 3]);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const bool second = p.split_b && c0 >= 128;
                const int col = p.split_b ? it.nt * 128 + (c0 & 127) : it.nt * kBN + c0;
                tma_store_3d(second ? tm_o1 : tm_o0, buf, col, m0, it.e);
                bulk_commit_group();
            }
            slab_buf = (slab_buf + 1) % kSlabBufs;
            tmem_ld_wait();
        }
    }
}

template <int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    pair_bwd_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a2,
                    const __grid_constant__ CUtensorMap tm_b0, const __grid_constant__ CUtensorMap tm_b1,
                    const __grid_constant__ CUtensorMap tm_o0, const __grid_constant__ CUtensorMap tm_o1, Params p)
{
    constexpr bool kAMN = KIND == kDW;                   // A read MN-major
    constexpr bool kBK_MAJOR = KIND == kDH || KIND == kDX;  // B read K-major
    constexpr int kStages = stages_for(KIND);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stage_out = smem + (size_t)kStages * kPairStageBytes;
    Ctrl& c = *reinterpret_cast<Ctrl*>(stage_out + store_bytes_for(KIND));

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint64_t limit = g_wait_limit_ns;
    const int E = p.E;
    const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs
    const bool leader = rank == 0;
    const int64_t pair = cluster_id_x();
    const int64_t npairs = num_clusters_x();

    if (threadIdx.x == 32) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&c.full[s], 1);
            mbar_init(&c.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&c.acc_full[b], 1);
            mbar_init(&c.acc_empty[b], 2 * kEpiWarps);
        }
        mbar_init(&c.done, 1);
        c.abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_map(&tm_a);
        tma_prefetch_map(&tm_b0);
        if (KIND == kDX) tma_prefetch_map(&tm_a2);
        if (KIND == kGU || KIND == kDX || KIND == kDW) tma_prefetch_map(&tm_b1);
        if (KIND == kDW || KIND == kDX || KIND == kDH) {
            tma_prefetch_map(&tm_o0);
            tma_prefetch_map(&tm_o1);
        }
    }
    if (warp == 1) {
        __syncwarp();
        tmem_alloc_pair(&c.tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    cluster_sync();
    tc_fence_after_sync();
    const uint32_t tmem = c.tmem_slot;
    pdl_trigger();
    pdl_wait();
    gemm::build_tile_list<kPairRows>(p.offsets, E, p.M, c.off, c.tp, &c.total_mtiles, &c.bad, true);
    __syncthreads();
    int64_t total_work = 0;
    if (!c.bad) total_work = KIND == kDW ? (int64_t)E * p.m_tiles * p.n_tiles : (int64_t)c.total_mtiles * p.n_tiles;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer (both CTAs)
            int s = 0;
            uint32_t ph = 0;
            int64_t issued = 0;
            for (int64_t w = pair; w < total_work && !c.abort_flag; w += npairs) {
                const Item it = decode_item<KIND>(w, p, c);
                // M-grouped kinds: on a tail tile whose odd half lies wholly past
                // the group's end (rows never stored), the odd CTA loads no A
                const bool odd_idle = KIND != kDW && it.row0 + kBM >= it.row_end;
                const uint32_t stage_tx = (uint32_t)(2 * kPairStageBytes - (odd_idle ? kABytes : 0));
                const bool load_a = leader || !odd_idle;
                bool ok = true;
                for (int kb = 0; kb < it.num_kb; ++kb) {
                    if (!mbar_wait(&c.empty[s], ph ^ 1u, limit)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + (size_t)s * kPairStageBytes;
                    uint8_t* sb = sa + kABytes;
                    if (leader) mbar_arrive_expect_tx(&c.full[s], stage_tx);
                    const uint32_t bar = mapa_shared(&c.full[s], 0);
                    if constexpr (KIND == kGU) {
                        if (load_a) tma_load_2d_pair(sa, &tm_a, bar, kb * kBK, it.row0 + (int)rank * kBM);
                        tma_load_3d_pair(sb, leader ? &tm_b0 : &tm_b1, bar, 0, it.e * p.b_rows + kb * kBK, it.nt * 2);
                    } else if constexpr (KIND == kDH) {
                        if (load_a) tma_load_2d_pair(sa, &tm_a, bar, kb * kBK, it.row0 + (int)rank * kBM);
                        tma_load_2d_pair(sb, &tm_b0, bar, kb * kBK, it.e * p.b_rows + it.nt * kBN + (int)rank * kBM);
                    } else if constexpr (KIND == kDX) {
                        const bool second = kb >= p.k_split;
                        const int kc = (second ? kb - p.k_split : kb) * kBK;
                        if (load_a) tma_load_2d_pair(sa, second ? &tm_a2 : &tm_a, bar, kc, it.row0 + (int)rank * kBM);
                        tma_load_2d_pair(sb, second ? &tm_b1 : &tm_b0, bar, kc,
                                         it.e * p.b_rows + it.nt * kBN + (int)rank * kBM);
                    } else {
                        const int kr = it.kstart + kb * kBK;
                        tma_load_3d_pair(sa, &tm_a, bar, 0, kr, (it.mt * kPairRows + (int)rank * kBM) / 64);
                        if (p.split_b)
                            tma_load_3d_pair(sb, leader ? &tm_b0 : &tm_b1, bar, 0, kr, it.nt * 2);
                        else
                            tma_load_3d_pair(sb, &tm_b0, bar, 0, kr, it.nt * (kBN / 64) + (int)rank * 2);
                    }
                    ++issued;
                    if (++s == kStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) {
                    c.abort_flag = 1;
                    break;
                }
            }
            for (int qq = 0; qq < kStages; ++qq) {
                const int64_t cnt = issued / kStages + (qq < issued % kStages ? 1 : 0);
                if (cnt > 0)
                    mbar_wait(leader ? &c.full[qq] : &c.empty[qq], (uint32_t)(cnt - 1) & 1u, drain_limit(limit));
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------ MMA issuer (even CTA)
            constexpr uint32_t idesc = idesc_bf16_f32(kPairRows, kBN, kAMN, !kBK_MAJOR);
            int s = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t acc_ph = 0;
            for (int64_t w = pair; w < total_work && !c.abort_flag; w += npairs) {
                const Item it = decode_item<KIND>(w, p, c);
                if (!mbar_wait(&c.acc_empty[acc], acc_ph ^ 1u, limit)) {
                    c.abort_flag = 1;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * kBN);
                bool ok = true;
                for (int kb = 0; kb < it.num_kb; ++kb) {
                    if (!mbar_wait(&c.full[s], ph, limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_base = smem_u32(smem + (size_t)s * kPairStageBytes);
                    const uint32_t b_base = a_base + kABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t adesc = kAMN ? smem_desc_sw128(a_base + kk * 2048, kChunkBytes, 1024)
                                                    : smem_desc_sw128(a_base + kk * 32, 16, 1024);
                        const uint64_t bdesc = kBK_MAJOR ? smem_desc_sw128(b_base + kk * 32, 16, 1024)
                                                         : smem_desc_sw128(b_base + kk * 2048, kChunkBytes, 1024);
                        mma_bf16_ss_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair_multicast(&c.empty[s], 0x3);
                    if (++s == kStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) {
                    c.abort_flag = 1;
                    break;
                }
                // an empty group issues no MMA: the commit still arrives (once
                // the earlier MMAs are done) and the epilogue writes zeros
                mma_commit_pair_multicast(&c.acc_full[acc], 0x3);
                if (++acc == 2) {
                    acc = 0;
                    acc_ph ^= 1u;
                }
            }
            mma_commit_pair(&c.done);
            mbar_wait(&c.done, 0, drain_limit(limit));
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;                 // TMEM lane quarter
        const int half = (warp - 2) >> 2;       // column half: warps 2-5 and 6-9
        float* slab = reinterpret_cast<float*>(stage_out + (warp - 2) * slab_stride_for(KIND));
        int slab_buf = 0;
        int acc = 0;
        uint32_t acc_ph = 0;
        for (int64_t w = pair; w < total_work; w += npairs) {
            const Item it = decode_item<KIND>(w, p, c);
            bool ready = true;
            if (lane == 0) ready = mbar_wait(&c.acc_full[acc], acc_ph, limit);
            ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
            if (!ready) {
                c.abort_flag = 1;
                break;
            }
            tc_fence_after_sync();
            const uint32_t tbase = tmem + (uint32_t)(acc * kBN) + ((uint32_t)(q * 32) << 16);
            epilogue<KIND>(p, it, tbase, rank, q, lane, half, &tm_o0, &tm_o1, slab, slab_buf);
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(&c.acc_empty[acc], 0));
            if (++acc == 2) {
                acc = 0;
                acc_ph ^= 1u;
            }
        }
        if ((KIND == kDW || KIND == kDX || KIND == kDH) && lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    tc_fence_before_sync();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace bwd
}  // namespace moe
