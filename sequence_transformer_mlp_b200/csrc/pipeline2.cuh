// pipeline2.cuh -- the tcgen05 pipeline on CTA pairs (cta_group::2).
//
// A cluster of two CTAs on two SMs computes one 256 x 256 tile with paired
// UMMAs (M = 256, N = 256, K = 16): CTA r of the pair stages rows
// [128 r, 128 r + 128) of A and columns [128 r, 128 r + 128) of B in its own
// shared memory, the leader (r = 0) issues every MMA, and each CTA's tensor
// memory receives its own 128 rows of the accumulator.  Per SM a stage is
// 32 KB for the same 128 x 256 x 64 of work that takes 48 KB on one CTA, so
// the operand traffic from L2 into each SM drops by a third.
//
// Synchronisation across the pair:
//   full[s]   leader only: the leader's producer expects the bytes of both
//             CTAs' loads; both CTAs' TMA loads complete on it.
//   empty[s]  both CTAs: the leader's commit arrives on both (multicast).
//   tfull[b]  both CTAs: the leader's commit arrives on both (multicast).
//   tempty[b] leader: the 4 epilogue warps of each CTA arrive (8 in all).
// Every wait is bounded as in pipeline.cuh; a CTA whose partner stops
// signalling times out on its own.  Both CTAs meet at a cluster barrier
// before freeing tensor memory and leaving, so no CTA leaves while the
// leader's MMAs may still read its shared memory.  No load uses cluster
// multicast; only the commit arrivals are multicast.
//
// A pair recipe R supplies, like a recipe of pipeline.cuh: Params, kStages,
// kStageBytes (per CTA), num_tiles, tile, num_kb, prefetch, and
//   void load(const Params&, const Tile&, int kb, uint32_t rank, uint32_t stage,
//             uint32_t leader_full_bar)               (1 thread in each CTA)
//   void mma(const Tile&, int kb, uint32_t stage, uint32_t acc)   (leader, 1 thread)
//   void epilogue(const Params&, const Tile&, uint32_t rank, uint32_t acc, int q, int lane,
//                 uint32_t stg)   (stg: the warp's 4 KB staging buffer for warp_store_*)
#pragma once

#include "pipeline.cuh"
#include "recipes.cuh"

namespace tspmlp {

template <class R>
constexpr int pair_smem_bytes() {
    return R::kStages * R::kStageBytes + 256 + kEpiStageBytes + 1024;
}

template <class R>
__global__ void __launch_bounds__(kPipelineThreads, 1)
    umma_pair_pipeline_kernel(const __grid_constant__ typename R::Params p) {
    constexpr int S = R::kStages;
    constexpr int NB = R::kAccBufs;
    constexpr uint32_t kAccCols = R::kAccCols;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t ring = (raw + 1023u) & ~1023u;
    uint8_t* ring_ptr = smem_raw + (ring - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(ring_ptr + S * R::kStageBytes);
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * S + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * S + NB + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * S + 2 * NB);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 2 * NB + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 8);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), 512);
        tmem_relinquish_pair();
    }
    if (warp == 0 && lane == 0) R::prefetch(p);
    tc_fence_before();
    cluster_sync_all();  // barrier inits and the allocation visible to both CTAs
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int num_tiles = R::num_tiles(p);
    const int pair = static_cast<int>(cluster_id_x());
    const int npairs = static_cast<int>(num_clusters_x());

    if (warp == 0) {
        // ------------------------------------------------------------ producers (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_par = 0;
            // the leader's full barriers in the cluster window, mapped once
            // (the barriers are contiguous; checked, else mapped per load)
            const uint32_t full0_leader = map_to_cta(full_bar(0), 0);
            const bool linear_map = map_to_cta(full_bar(S - 1), 0) == full0_leader + 8u * (S - 1);
            for (int t = pair; t < num_tiles && !*abort_flag; t += npairs) {
                const auto ti = R::tile(p, t);
                const int nkb = R::num_kb(p, ti);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) break;
                    if (leader) mbar_arrive_expect_tx(full_bar(stage), 2u * R::kStageBytes);
                    R::load(p, ti, kb, rank, ring + stage * R::kStageBytes,
                            linear_map ? full0_leader + 8u * stage : map_to_cta(full_bar(stage), 0));
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // the leader's full barriers count both CTAs' loads: waiting on them
            // lets every load of the pair land before shared memory goes away
            if (leader)
                for (int s = 0; s < S; ++s)
                    if (armed & (1u << s)) mbar_wait_drain(full_bar(s), (armed_par >> s) & 1u);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (lane == 0 && leader) {
            int stage = 0, local = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += npairs, ++local) {
                const auto ti = R::tile(p, t);
                const int nkb = R::num_kb(p, ti);
                const int buf = local % NB;
                const uint32_t use = static_cast<uint32_t>(local / NB);
                if (!mbar_wait(tempty_bar(buf), (use & 1u) ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t acc = tmem_base + static_cast<uint32_t>(buf) * kAccCols;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(full_bar(stage), phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    R::mma(ti, kb, ring + stage * R::kStageBytes, acc);
                    umma_commit_pair_mc(empty_bar(stage), 0x3);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit_pair_mc(tfull_bar(buf), 0x3);
            }
            umma_commit_pair_mc(drain_bar, 0x1);
            mbar_wait_drain(drain_bar, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        const uint32_t stg = ring + S * R::kStageBytes + 256 + q * kEpiStageBytesPerWarp;
        int local = 0;
        for (int t = pair; t < num_tiles; t += npairs, ++local) {
            const int buf = local % NB;
            const uint32_t use = static_cast<uint32_t>(local / NB);
            int ok = 0;
            if (lane == 0) ok = mbar_wait(tfull_bar(buf), use & 1u, abort_flag) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const auto ti = R::tile(p, t);
            R::epilogue(p, ti, rank, tmem_base + static_cast<uint32_t>(buf) * kAccCols, q, lane, stg);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader)
                    mbar_arrive(tempty_bar(buf));
                else
                    mbar_arrive_remote(map_to_cta(tempty_bar(buf), 0));
            }
        }
    }

    tc_fence_before();
    cluster_sync_all();  // no CTA leaves while the pair's MMAs may read its shared memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
}

// ============================================================================
// Paired gate/up projection with the fused activation (see FwdHidden).
// Tile = 256 token rows (128 per CTA).  SwiGLU: CTA 0 stages the gate columns,
// CTA 1 the up columns of the same 128 hidden units, so TMEM columns 0-127
// hold the gate and 128-255 the up pre-activations of each CTA's rows.
// GeLU: 256 hidden units a tile, 128 staged by each CTA.
template <int ACT>
struct FwdHiddenPair {
    using Params = typename FwdHidden<ACT>::Params;
    static constexpr const char* kName = ACT == 1 ? "fwd_hidden_swiglu" : "fwd_hidden_gelu";
    // 128-deep k-blocks: each operand is two 64-column TMA boxes (16 KB each
    // a CTA); half as many stages, barrier round trips and producer/MMA-issuer
    // iterations per FLOP as 64-deep blocks (measured 3-6% faster)
    static constexpr int kBK = 128;
    static constexpr int kOut = ACT == 1 ? 128 : 256;
    static constexpr int kABytes = 128 * kBK * 2;
    static constexpr int kStageBytes = kABytes + 128 * kBK * 2;
    static constexpr int kStages = 3;
    static constexpr int kAccCols = 256, kAccBufs = 2;
    static constexpr uint32_t kIdesc = make_idesc_bf16(256, 256, false, true);
    struct Tile {
        int s, mi, nj;
        int c;     // first weight column of the tile (shard base + nj kOut)
        int xrow;  // first X row of the pair's 256 rows
    };
    __host__ __device__ static int pair_mtiles(const SegGeom& g) { return (g.seg_rows + 255) >> 8; }
    __host__ __device__ static int ntiles_n(const Params& p) { return (p.width + kOut - 1) / kOut; }
    __host__ __device__ static int num_tiles(const Params& p) {
        return p.g.num_segs * pair_mtiles(p.g) * ntiles_n(p);
    }
    __device__ static Tile tile(const Params& p, int t) {
        const int mt = pair_mtiles(p.g), per_seg = mt * ntiles_n(p);
        const int s = t / per_seg, r = t - s * per_seg;
        const int nj = r / mt;
        const int mi = r - nj * mt;
        // everything the per-k-block loads need, computed once a tile
        return Tile{s, mi, nj, p.g.shard_col(s) + nj * kOut, (p.g.seg_begin + s) * p.g.seg_rows + mi * 256};
    }
    __device__ static int num_kb(const Params& p, const Tile&) { return (p.d + kBK - 1) / kBK; }
    __device__ static void prefetch(const Params& p) { FwdHidden<ACT>::prefetch(p); }
    __device__ static void load(const Params& p, const Tile& ti, int kb, uint32_t rank, uint32_t st,
                                uint32_t bar) {
        const int k0 = kb * kBK;
        const int xr = ti.xrow + static_cast<int>(rank) * 128;
        tma_load_2d_pair(st, &p.tmX, bar, k0, xr);  // X: two {64 k, 128 rows} boxes
        tma_load_2d_pair(st + 16384, &p.tmX, bar, k0 + 64, xr);
        const int c = ti.c;  // weights: two {64 cols, 128 k} boxes
        if (ACT == 1) {
            const CUtensorMap* w = rank == 0 ? &p.tmG : &p.tmU;
            tma_load_2d_pair(st + kABytes, w, bar, c, k0);
            tma_load_2d_pair(st + kABytes + 16384, w, bar, c + 64, k0);
        } else {
            const int cr = c + static_cast<int>(rank) * 128;
            tma_load_2d_pair(st + kABytes, &p.tmG, bar, cr, k0);
            tma_load_2d_pair(st + kABytes + 16384, &p.tmG, bar, cr + 64, k0);
        }
    }
    __device__ static void mma(const Tile&, int kb, uint32_t st, uint32_t acc) {
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
            // A: K-major, 32 B a K16 step inside a 64-k box, the next box 16 KB on
            // B: MN-major, 2 KB a K16 step; its second 64-column box 16 KB on
            const uint64_t a =
                make_smem_desc(st + (kk >> 2) * 16384 + 32 * (kk & 3), 16, 1024, kLayoutSW128);
            const uint64_t b = make_smem_desc(st + kABytes + 2048 * kk, 16384, 1024, kLayoutSW128);
            umma_bf16_pair(acc, a, b, kIdesc, (kb | kk) != 0 ? 1u : 0u);
        }
    }
    __device__ static void epilogue(const Params& p, const Tile& ti, uint32_t rank, uint32_t acc,
                                    int q, int lane, uint32_t stg) {
        // the same per-row work as the single-CTA tile, on this CTA's 128 rows
        typename FwdHidden<ACT>::Tile t1{ti.s, 2 * ti.mi + static_cast<int>(rank), ti.nj};
        FwdHidden<ACT>::epilogue(p, t1, acc, q, lane, stg);
    }
};

// ============================================================================
// Paired down projection / input gradient with in-place fp32 accumulation
// (see DownAccum).  Tile = 256 rows x BN output columns; CTA r stages output
// columns [r BN/2, (r+1) BN/2) of the B tile.  BN = 128 gives twice the tiles
// of BN = 256 for the same problem (fewer idle SMs in the last wave).
template <bool B_MN, int NSEG, int BN = 256>
struct DownAccumPair {
    using Base = DownAccum<B_MN, NSEG>;
    using Params = typename Base::Params;
    static constexpr const char* kName = Base::kName;
    // 128-deep k-blocks, each operand two 64-wide TMA boxes (see FwdHiddenPair)
    static constexpr int kBK = 128;
    static constexpr int kHalf = BN / 2;
    static_assert(kHalf == 128, "a CTA stages 128 output columns");
    static constexpr int kABytes = 128 * kBK * 2;
    static constexpr int kStageBytes = kABytes + kHalf * kBK * 2;
    static constexpr int kStages = 3;
    static constexpr int kAccCols = 256, kAccBufs = 2;
    static constexpr uint32_t kIdesc = make_idesc_bf16(256, BN, false, B_MN);
    struct Tile {
        int s, mi, nj;
        int kbase;  // hidden unit of the K loop's first column (shard base, or the
                    // ring start (seg_begin + s) fs with rot_P)
        int kwrap;  // rot_P fs: the K loop's hidden units wrap at this column
        int arow;   // first A row of the pair's 256 rows
        int half;   // -1 whole tile; 0 / 1: first / second half of a split tile's K loop
        int kb0;    // first k-block of this unit
        int nkb;    // k-blocks of this unit
        int slot;   // split tiles: index of the tile among them
    };
    __host__ __device__ static int pair_mtiles(const SegGeom& g) { return (g.seg_rows + 255) >> 8; }
    __host__ __device__ static int ntiles_n(const Params& p) { return (p.n_out + BN - 1) / BN; }
    __host__ __device__ static int whole_tiles(const Params& p) {
        return p.g.num_segs * pair_mtiles(p.g) * ntiles_n(p);
    }
    __host__ __device__ static int kblocks(const Params& p) { return NSEG * ((p.kdim + kBK - 1) / kBK); }
    // work units: the whole tiles before split_from, then two halves of each
    // later tile (units split_from + 2 j and + 2 j + 1)
    __host__ __device__ static int num_tiles(const Params& p) {
        const int w = whole_tiles(p);
        return p.split_from > 0 ? p.split_from + 2 * (w - p.split_from) : w;
    }
    __device__ static Tile tile(const Params& p, int u) {
        int t = u, half = -1;
        if (p.split_from > 0 && u >= p.split_from) {
            const int j = u - p.split_from;
            t = p.split_from + (j >> 1);
            half = j & 1;
        }
        const int mt = pair_mtiles(p.g), per_seg = mt * ntiles_n(p);
        const int s = t / per_seg, r = t - s * per_seg;
        const int nj = r / mt;
        const int mi = r - nj * mt;
        const int nkb = kblocks(p), h0 = nkb >> 1;
        // everything the per-k-block loads need, computed once a tile
        return Tile{s, mi, nj,
                    p.rot_P > 0 ? (p.g.seg_begin + s) * p.g.fs : p.g.shard_col(s),
                    p.rot_P * p.g.fs, s * p.g.seg_rows + mi * 256, half,
                    half == 1 ? h0 : 0, half < 0 ? nkb : (half == 0 ? h0 : nkb - h0),
                    t - p.split_from};
    }
    __device__ static int num_kb(const Params&, const Tile& ti) { return ti.nkb; }
    __device__ static void prefetch(const Params& p) { Base::prefetch(p); }
    __device__ static void load(const Params& p, const Tile& ti, int kb, uint32_t rank, uint32_t st,
                                uint32_t bar) {
        kb += ti.kb0;  // the unit's k-blocks within the tile's K loop
        // K segment of this k-block (NSEG <= 2), without a division: this runs
        // once per k-block in the producer thread
        static_assert(NSEG == 1 || NSEG == 2, "one or two K segments");
        const int nkb1 = (p.kdim + kBK - 1) / kBK;
        const int seg = (NSEG > 1 && kb >= nkb1) ? 1 : 0;
        const int k = (kb - seg * nkb1) * kBK;
        const CUtensorMap* ta = seg ? &p.tmA1 : &p.tmA0;
        const CUtensorMap* tb = seg ? &p.tmB1 : &p.tmB0;
        // hidden column of this k-block in H (ka) and in the weights (kw)
        // hidden column of each 64-wide half of this k-block, in H (ka) and in
        // the weights (kw)
        int ka[2], kw[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            ka[h] = k + 64 * h;
            kw[h] = ti.kbase + ka[h];
            if (p.rot_P > 0) {
                // H holds every hidden unit; segment s visits the shards in ring
                // order, starting at shard seg_begin + s (< P): column k of the
                // loop is hidden unit (k + (seg_begin + s) fs) mod (P fs).  The
                // planner takes this path only with fs % 128 == 0, so the wrap
                // falls on a k-block edge.  No division: this runs once per
                // k-block in the producer thread.
                ka[h] = kw[h] = kw[h] >= ti.kwrap ? kw[h] - ti.kwrap : kw[h];
            }
        }
        const int ar = ti.arow + static_cast<int>(rank) * 128;
        tma_load_2d_pair(st, ta, bar, ka[0], ar);  // A: two {64 k, 128 rows} boxes
        tma_load_2d_pair(st + 16384, ta, bar, ka[1], ar);
        const int n0 = ti.nj * BN + static_cast<int>(rank) * kHalf;
        if (B_MN) {  // two {64 cols, 128 k} boxes (K rows kw[0] .. kw[0] + 127)
            tma_load_2d_pair(st + kABytes, tb, bar, n0, kw[0]);
            tma_load_2d_pair(st + kABytes + 16384, tb, bar, n0 + 64, kw[0]);
        } else {  // K-major: two {64 k, 128 rows} boxes
            tma_load_2d_pair(st + kABytes, tb, bar, kw[0], n0);
            tma_load_2d_pair(st + kABytes + 16384, tb, bar, kw[1], n0);
        }
    }
    __device__ static void mma(const Tile&, int kb, uint32_t st, uint32_t acc) {
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t kmaj = (kk >> 2) * 16384 + 32 * (kk & 3);  // K-major K16 step
            const uint64_t a = make_smem_desc(st + kmaj, 16, 1024, kLayoutSW128);
            const uint64_t b = B_MN ? make_smem_desc(st + kABytes + 2048 * kk, 16384, 1024, kLayoutSW128)
                                    : make_smem_desc(st + kABytes + kmaj, 16, 1024, kLayoutSW128);
            umma_bf16_pair(acc, a, b, kIdesc, (kb | kk) != 0 ? 1u : 0u);
        }
    }
    __device__ static void epilogue(const Params& p, const Tile& ti, uint32_t rank, uint32_t acc,
                                    int q, int lane, uint32_t stg) {
        const int wr0 = ti.mi * 256 + static_cast<int>(rank) * 128 + q * 32;  // warp's first row
        const uint32_t t0 = acc + (static_cast<uint32_t>(q * 32) << 16);
        if (ti.half < 0) {
            Base::template store_rows<BN / 32>(p, ti.s, wr0, lane, ti.nj * BN, t0, stg);
            return;
        }
        // a split tile: this warp's 32 rows x 256 columns of the partial sum
        float* part = p.part + static_cast<long long>(ti.slot) * (256 * 256) +
                      (static_cast<int>(rank) * 128 + q * 32) * 256;
        int* flag = p.flags + ti.slot * 8 + static_cast<int>(rank) * 4 + q;
        if (ti.half == 0) {
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(t0 + 32 * cc, v);
                tmem_ld_wait();
                warp_store_f32x32(stg, part + 32 * cc, 256, 32, v, 32, lane);
            }
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release_gpu(flag, 1);
            return;
        }
        // second half: wait (bounded) for the first half's rows of this warp,
        // then round first-half + second-half sums to bf16
        if (lane == 0) wait_flag_gpu(flag);
        __syncwarp();
        const int nrows = min(32, p.g.seg_rows - wr0);
        const long long row0 = static_cast<long long>(p.g.seg_begin + ti.s) * p.g.seg_rows + wr0;
        const float* prow = part + lane * 256;
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
            uint32_t v[32], pk[16];
            tmem_ld_32x32b_x32(t0 + 32 * cc, v);
            tmem_ld_wait();
            const int c0 = ti.nj * BN + 32 * cc;
            const int valid = p.n_out - c0;
            if (valid <= 0) continue;
            const float4* a4 = reinterpret_cast<const float4*>(prow + 32 * cc);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 a = __ldcg(a4 + i);
                pk[2 * i] = pack_bf16x2(a.x + __uint_as_float(v[4 * i]), a.y + __uint_as_float(v[4 * i + 1]));
                pk[2 * i + 1] =
                    pack_bf16x2(a.z + __uint_as_float(v[4 * i + 2]), a.w + __uint_as_float(v[4 * i + 3]));
            }
            warp_store_16x32(stg, p.out + row0 * p.ldo + c0, p.ldo, nrows, pk, valid, lane);
        }
    }
};

}  // namespace tspmlp
