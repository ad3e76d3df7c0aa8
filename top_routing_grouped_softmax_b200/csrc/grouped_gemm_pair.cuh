// grouped_gemm_pair.cuh -- the grouped expert GEMM on CTA pairs
// (tcgen05 cta_group::2), for the same work and epilogues as
// grouped_gemm_kernel.
//
// A cluster of two CTAs on two SMs owns a 256-row M tile of one expert group
// and a 256-column N tile.  Each CTA loads its own 128 rows of A and its own
// half of the B tile (128 columns), so per SM a pipeline stage is 32 KB
// instead of 48 KB for the same tensor work: less shared-memory fill and
// L2->SM traffic per flop, and a deeper ring (6 stages).  The B half is
// fetched by one 3-D copy (two 64-column chunks), so a CTA issues two
// copies per stage.  The even CTA issues the pair MMAs (M=256, N=256,
// K=16); each CTA's TMEM receives its own 128 rows of the accumulator, so
// each CTA's epilogue drains its own rows exactly like the single-CTA
// kernel.
//
// Synchronisation across the pair:
//   full[s]      lives in the even CTA; both CTAs' TMA loads complete on it
//                (the even CTA's producer expects the bytes of both halves)
//   empty[s]     one per CTA; the MMA commit is multicast to both
//   acc_full[b]  one per CTA; multicast commit
//   acc_empty[b] lives in the even CTA; the epilogue warps of each CTA
//                arrive on it (remotely, for the odd CTA)
// The pair meets at a cluster barrier after set-up and before releasing TMEM.
// No TMA load uses multicast.
#pragma once

#include "grouped_gemm.cuh"

namespace moe {
namespace gemm {

constexpr int kPairRows = 256;                        // M rows per CTA pair
constexpr int kPairBHalfBytes = 2 * kChunkBytes;      // 128 columns x 64 k
constexpr int kPairStageBytes = kABytes + kPairBHalfBytes;  // 32 KB per CTA
constexpr int kPairStages = 6;
// Ring depth of the down-projection (kWeighted) kernel and y staging slabs
// per epilogue warp: build-time tuning constants (the ring and the slabs
// share the 227 KB of shared memory).  Six stages and one slab per warp for
// eight epilogue warps measured the same as five stages with two or three
// slabs on the fine-grained layer and 4 us faster on the Qwen3-shaped one.
#ifndef MOE_PAIR_DOWN_STAGES
#define MOE_PAIR_DOWN_STAGES 6
#endif
#ifndef MOE_PAIR_SLAB_BUFS
#define MOE_PAIR_SLAB_BUFS 1
#endif
constexpr int kPairSlabBufs = MOE_PAIR_SLAB_BUFS;
static_assert(MOE_PAIR_DOWN_STAGES >= 2 && MOE_PAIR_DOWN_STAGES <= kPairStages, "down ring depth");
static_assert(kPairSlabBufs >= 1 && kPairSlabBufs <= 8, "slab buffers per epilogue warp");

// The down kernel's y slabs are 32 x SC fp16: SC = 32 by default; SC = 64
// (128-byte rows, half as many fences and stores per tile, with a five-stage
// ring to make room) where the reduction is short (f <= kDownShortK), whose
// tiles are bound by their epilogue: 7 % off that layer's down GEMM, while
// a long K lost the ring stage (qwen's down GEMM 5 us slower).
constexpr int kDownShortK = 512;
constexpr int kDownShortKStages = 5;

template <int EPI, int SC = kSlabCols>
__host__ __device__ constexpr int pair_stages()
{
    return EPI == kWeighted ? (SC == 64 ? kDownShortKStages : MOE_PAIR_DOWN_STAGES) : kPairStages;
}

template <int EPI, int SC = kSlabCols>
__host__ __device__ constexpr int pair_store_bytes()
{
    return EPI == kWeighted ? kEpiWarps * kPairSlabBufs * (32 * SC * 2) : 0;
}

struct alignas(8) PairCtrl {
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

template <int EPI, int SC = kSlabCols>
__host__ inline size_t pair_smem_bytes()
{
    return 1024 + (size_t)pair_stages<EPI, SC>() * kPairStageBytes + pair_store_bytes<EPI, SC>() + sizeof(PairCtrl);
}
static_assert(1024 + (size_t)pair_stages<kSwiGLU>() * kPairStageBytes + sizeof(PairCtrl) <= 227 * 1024,
              "gate/up pair ring and control exceed 227 KB of shared memory");
static_assert(1024 + (size_t)pair_stages<kWeighted>() * kPairStageBytes + pair_store_bytes<kWeighted>() +
                      sizeof(PairCtrl) <= 227 * 1024,
              "down pair ring, staging and control exceed 227 KB of shared memory");
static_assert(1024 + (size_t)pair_stages<kWeighted, 64>() * kPairStageBytes + pair_store_bytes<kWeighted, 64>() +
                      sizeof(PairCtrl) <= 227 * 1024,
              "down pair ring, staging and control exceed 227 KB of shared memory (short-K form)");

template <int EPI, int SC = kSlabCols>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                             const __grid_constant__ CUtensorMap tm_b1, const __grid_constant__ CUtensorMap tm_out,
                             Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int NS = pair_stages<EPI, SC>();
    uint8_t* stage_out = smem + (size_t)NS * kPairStageBytes;
    PairCtrl& c = *reinterpret_cast<PairCtrl*>(stage_out + pair_store_bytes<EPI, SC>());

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint64_t limit = g_wait_limit_ns;
    const int E = p.E;
    const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs
    const bool leader = rank == 0;
    const int64_t pair = cluster_id_x();
    const int64_t npairs = num_clusters_x();

    if (threadIdx.x == 32) {
        for (int s = 0; s < NS; ++s) {
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
        if (EPI == kSwiGLU) tma_prefetch_map(&tm_b1);
        if (EPI == kWeighted) tma_prefetch_map(&tm_out);
    }
    if (warp == 1) {
        __syncwarp();
        tmem_alloc_pair(&c.tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
    tc_fence_after_sync();
    const uint32_t tmem = c.tmem_slot;
    // the offsets and operands come from earlier kernels on the stream
    pdl_trigger();
    pdl_wait();
    build_tile_list<kPairRows>(p.offsets, E, p.M, c.off, c.tp, &c.total_mtiles, &c.bad, p.m_capacity != 0);
    __syncthreads();
    const int64_t total_work = c.bad ? 0 : (int64_t)c.total_mtiles * p.n_tiles;
    const int num_kb = p.K / kBK;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer (both CTAs)
            int s = 0;
            uint32_t ph = 0;
            int64_t issued = 0;
            for (int64_t w = pair; w < total_work && !c.abort_flag; w += npairs) {
                int e, row0, row_end, nt;
                decode_tile<kPairRows>(w, p.n_tiles, c.tp, c.off, E, e, row0, row_end, nt);
                const int krow0 = e * p.K;
                const int arow = row0 + (int)rank * kBM;
                // A tail tile of at most 128 rows: the odd CTA's rows all lie past
                // the group's end (its accumulator rows are never stored), so it
                // loads no A and the stage expects 16 KB less.  Both CTAs decode
                // the same tile, so they agree on this.
                const bool odd_idle = row0 + kBM >= row_end;
                const uint32_t stage_tx = (uint32_t)(2 * kPairStageBytes - (odd_idle ? kABytes : 0));
                bool ok = true;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&c.empty[s], ph ^ 1u, limit)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + (size_t)s * kPairStageBytes;
                    uint8_t* sb = sa + kABytes;
                    if (leader) mbar_arrive_expect_tx(&c.full[s], stage_tx);
                    const uint32_t bar = mapa_shared(&c.full[s], 0);
                    const int kr = krow0 + kb * kBK;
                    if (leader || !odd_idle) tma_load_2d_pair(sa, &tm_a, bar, kb * kBK, arow);
                    // 128 weight columns as two 64-column chunks in one copy (the
                    // weight maps view [K, N] as [N/64][K][64])
                    if (EPI == kSwiGLU) {
                        // even CTA: the gate columns, odd CTA: the matching up columns
                        const CUtensorMap* tb = leader ? &tm_b0 : &tm_b1;
                        tma_load_3d_pair(sb, tb, bar, 0, kr, nt * 2);
                    } else {
                        tma_load_3d_pair(sb, &tm_b0, bar, 0, kr, nt * (kBN / 64) + (int)rank * 2);
                    }
                    ++issued;
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) {
                    c.abort_flag = 1;
                    break;
                }
            }
            // Never leave a copy landing in shared memory.  The even CTA's full
            // barriers count both CTAs' copies; the odd CTA instead waits until
            // the MMAs that read each of its stages released it (which they do
            // only after the stage's bytes arrived).
            for (int q = 0; q < NS; ++q) {
                const int64_t cnt = issued / NS + (q < issued % NS ? 1 : 0);
                if (cnt > 0)
                    mbar_wait(leader ? &c.full[q] : &c.empty[q], (uint32_t)(cnt - 1) & 1u, drain_limit(limit));
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------ MMA issuer (even CTA)
            constexpr uint32_t idesc = idesc_bf16_f32(kPairRows, kBN, false, true);
            int s = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t acc_ph = 0;
            for (int64_t w = pair; w < total_work && !c.abort_flag; w += npairs) {
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
                    const uint32_t a_base = smem_u32(smem + (size_t)s * kPairStageBytes);
                    const uint32_t b_base = a_base + kABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t adesc = smem_desc_sw128(a_base + kk * 32, 16, 1024);
                        const uint64_t bdesc = smem_desc_sw128(b_base + kk * 2048, kChunkBytes, 1024);
                        mma_bf16_ss_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair_multicast(&c.empty[s], 0x3);  // frees the stage in both CTAs
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) {
                    c.abort_flag = 1;
                    break;
                }
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
        const int ew = warp - 2;
        const int q = warp & 3;
        const int hf = ew >> 2;
        float* slab = reinterpret_cast<float*>(stage_out + ew * kPairSlabBufs * (32 * SC * 2));
        int slab_buf = 0;
        int acc = 0;
        uint32_t acc_ph = 0;
        for (int64_t w = pair; w < total_work; w += npairs) {
            int e, row0, row_end, nt;
            decode_tile<kPairRows>(w, p.n_tiles, c.tp, c.off, E, e, row0, row_end, nt);
            bool ready = true;
            if (lane == 0) ready = mbar_wait(&c.acc_full[acc], acc_ph, limit);
            ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
            if (!ready) {
                c.abort_flag = 1;
                break;
            }
            tc_fence_after_sync();
            const uint32_t tbase = tmem + (uint32_t)(acc * kBN) + ((uint32_t)(q * 32) << 16);
            epilogue_tile<EPI, kPairSlabBufs, SC>(p, &tm_out, tbase, row0 + (int)rank * kBM, row_end, nt, q, lane, hf,
                                                  slab, slab_buf);
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(&c.acc_empty[acc], 0));
            if (++acc == 2) {
                acc = 0;
                acc_ph ^= 1u;
            }
        }
        if (EPI == kWeighted && lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    tc_fence_before_sync();
    cluster_sync();  // both CTAs are done with TMEM and with each other's barriers
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace gemm
}  // namespace moe
