// pipeline.cuh -- the persistent, warp-specialised tcgen05 pipeline shared by
// every tensor-core kernel of the library.
//
// One CTA per SM (192 threads, 1 CTA/SM by shared-memory size):
//   warp 0      TMA producer: one elected thread fills a ring of shared-memory
//               stages (mbarrier "full"/"empty" pairs, transaction counts).
//   warp 1      MMA issuer: allocates tensor memory, one elected thread issues
//               tcgen05.mma for every stage and commits the stage back to the
//               producer; after a tile it commits the accumulator to the
//               epilogue.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4) .. +31, i.e. tile rows), fused elementwise
//               work, stores to global memory, then hand the accumulator
//               buffer back to the MMA warp.
// Tiles are visited persistently: CTA b takes tiles b, b + gridDim.x, ...
// With two accumulator buffers the epilogue of tile i overlaps the main loop
// of tile i+1.
//
// Every wait is bounded (ptx.cuh: mbar_wait).  When one runs out the kernel
// raises a shared abort flag, every role leaves its loop, the producer waits
// (bounded) for its loads in flight, the MMA thread waits (bounded) for its
// MMAs, tensor memory is freed and the kernel returns.
//
// A recipe R supplies the tile space, the per-stage loads, the MMAs of one
// stage and the epilogue:
//   R::Params, R::kStages, R::kStageBytes, R::kAccCols, R::kAccBufs, R::kTmemCols
//   int  R::num_tiles(const Params&)
//   Tile R::tile(const Params&, int t)
//   int  R::num_kb(const Params&, const Tile&)
//   void R::prefetch(const Params&)                                       (1 thread)
//   uint32_t R::load(const Params&, const Tile&, int kb, uint32_t stage, uint32_t bar)
//        issues the TMA loads of k-block kb and returns the bytes they move (1 thread)
//   void R::mma(const Tile&, int kb, uint32_t stage, uint32_t acc_tmem)   (1 thread)
//   void R::epilogue(const Params&, const Tile&, uint32_t acc_tmem, int q, int lane)
//        (128 threads; q = warp % 4 owns tile rows 32q .. 32q+31)
#pragma once

#include "ptx.cuh"

namespace tspmlp {

constexpr int kPipelineThreads = 192;

// Each epilogue warp stages its 32 x 32 blocks for coalesced stores in 4 KB
// of shared memory after the barriers (recipes.cuh: warp_store_*).
constexpr int kEpiStageBytesPerWarp = 4096;
constexpr int kEpiStageBytes = 4 * kEpiStageBytesPerWarp;

// Bytes of dynamic shared memory a recipe needs (stages + barriers + the
// epilogue staging buffers + slack for 1024-byte alignment of the stage ring).
template <class R>
constexpr int pipeline_smem_bytes() {
    return R::kStages * R::kStageBytes + 256 + kEpiStageBytes + 1024;
}

// Bounded wait that ignores the abort flag (used while draining).
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 31u) == 0u && global_timer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_device_error, kDevErrTimeout);
            return false;
        }
    }
}

// kDropFirstLoad (self-test only): the producer arms the first stage of
// CTA 0's first tile but issues none of its loads, so that stage never fills
// and every role must leave through the bounded-wait abort path.
template <class R, bool kDropFirstLoad = false>
__global__ void __launch_bounds__(kPipelineThreads, 1)
    umma_pipeline_kernel(const __grid_constant__ typename R::Params p) {
    constexpr int S = R::kStages;
    constexpr int NB = R::kAccBufs;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t ring = (raw + 1023u) & ~1023u;
    uint8_t* ring_ptr = smem_raw + (ring - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(ring_ptr + S * R::kStageBytes);
    // barrier map: full[S], empty[S], tfull[NB], tempty[NB], drain
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

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 4);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), R::kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) R::prefetch(p);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int num_tiles = R::num_tiles(p);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0;        // bit s: stage s has loads issued
            uint32_t armed_par = 0;    // bit s: parity of that stage's phase
            for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
                const auto ti = R::tile(p, t);
                const int nkb = R::num_kb(p, ti);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) break;
                    const uint32_t sbase = ring + stage * R::kStageBytes;
                    const uint32_t bytes = R::load_bytes(p, ti, kb);
                    mbar_arrive_expect_tx(full_bar(stage), bytes);
                    if (!(kDropFirstLoad && blockIdx.x == 0 && t == 0 && kb == 0))
                        R::load(p, ti, kb, sbase, full_bar(stage));
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // let every load in flight land before shared memory goes away
            // (returns at once in a normal run: each armed phase has landed
            // or lands within microseconds)
            for (int s = 0; s < S; ++s)
                if (armed & (1u << s)) mbar_wait_drain(full_bar(s), (armed_par >> s) & 1u);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++local) {
                const auto ti = R::tile(p, t);
                const int nkb = R::num_kb(p, ti);
                const int buf = local % NB;
                const uint32_t use = static_cast<uint32_t>(local / NB);
                if (!mbar_wait(tempty_bar(buf), (use & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem_base + static_cast<uint32_t>(buf * R::kAccCols);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(full_bar(stage), phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    R::mma(ti, kb, ring + stage * R::kStageBytes, acc);
                    umma_commit(empty_bar(stage));
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(tfull_bar(buf));
            }
            // every MMA issued must finish before tensor memory is released
            umma_commit(drain_bar);
            mbar_wait_drain(drain_bar, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const uint32_t stg = ring + S * R::kStageBytes + 256 + q * kEpiStageBytesPerWarp;
        int local = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++local) {
            const int buf = local % NB;
            const uint32_t use = static_cast<uint32_t>(local / NB);
            int ok = 0;
            if (lane == 0) ok = mbar_wait(tfull_bar(buf), use & 1u, abort_flag) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const auto ti = R::tile(p, t);
            R::epilogue(p, ti, tmem_base + static_cast<uint32_t>(buf * R::kAccCols), q, lane, stg);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar(buf));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, R::kTmemCols);
    }
}

}  // namespace tspmlp
