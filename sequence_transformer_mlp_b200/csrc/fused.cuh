// fused.cuh -- the whole forward pass in one persistent launch.
//
// Work is cut into row blocks of 128 tokens.  Each row block has
//   gate/up tiles  (nJ of them): H[rows, j*kOut ..] = act(X[rows] . W[:, j*kOut ..])
//   down tiles     (nC of them): Y[rows, c*256 ..] = H[rows, :] . W_down[:, c*256 ..]
// The down tile's K loop runs over all d_ff hidden units in shard order
// (shard 0, 1, ..., P-1; for the folded tensor-and-sequence ring, sequence
// shard s starts at weight shard s and wraps), so each shard's partial output
// is added into the fp32 tensor-memory accumulator in shard order and Y is
// written once ("Tensor Parallelism: Splitting the Math", steps 4-6; "Folding
// Tensor and Sequence Parallelism ...", Abstract).
//
// Tile list.  Row blocks form groups of GM.  Phase p holds the gate/up tiles
// of group p (weight-column slab outer, row block inner, so a slab is read
// from HBM once per group while the group's X rows stay in L2) merged with
// the down tiles of group p-1 (output slab outer, row block inner): first a
// head of up to one wave of gate/up tiles, then both lists interleaved in
// proportion to their lengths.  Tiles are handed out in list order through a
// global atomic counter (dynamic scheduling).
//
// Dependencies.  A down tile's producer waits until all gate/up tiles of its
// row block have stored their H.  H lives in a ring of R = 3*GM row-block
// slots (or one slot per row block), so a gate/up tile's producer waits until
// the down tiles of the row block R earlier -- two phases back -- are done.
// Every dependency points to an earlier tile of the list and tiles are taken
// in list order by running CTAs, so the waits always end; they are bounded
// anyway.  Ordering: the gate/up epilogue stores H with st.global, fences the
// async proxy and releases the row block's counter; the consumer acquires the
// counter and fences the async proxy before its TMA loads of H.
//
// Roles as in pipeline.cuh (warp 0 TMA producer, warp 1 MMA issuer, warps 2-5
// epilogue); the producer also takes the tiles and passes their indices to
// the other roles through a small shared-memory queue.
#pragma once

#include "recipes.cuh"

namespace tspmlp {

struct FusedFwdParams {
    CUtensorMap tmX;  // X [n][d], box {64, 128}
    CUtensorMap tmG;  // W_gate / A [d][f], box {64, 64}
    CUtensorMap tmU;  // W_up [d][f], box {64, 64} (SwiGLU)
    CUtensorMap tmH;  // H ring [R*128][f], box {64, 128}
    CUtensorMap tmD;  // W_down / B [f][d], box {64, 64}
    int n, d, f;
    int seg_rows;     // rows per sequence segment (n for the weight-shard schedule)
    int mts;          // row blocks per segment
    int ring;         // 1: segment s starts its K loop over hidden units at s*fs
    int fs;           // hidden units per weight shard
    int MB;           // row blocks in total
    int nJ, nC;       // gate/up and down tiles per row block
    int GM, G;        // row blocks per group, groups
    int head;         // gate/up tiles that open a phase before any down tile
    int R;            // H ring slots
    int total;        // tiles in the list
    __nv_bfloat16* H; // ring base, [R*128][f]
    __nv_bfloat16* Y; // [n][d]
    unsigned* sync;   // [0] next tile; [1+m] gate/up warps done; [1+MB+m] down warps done
};

enum : int { kFusedGateUp = 0, kFusedDown = 1 };

struct FusedTile {
    int type, mb, j;
};

__host__ __device__ inline int fused_group_rows(const FusedFwdParams& p, int g) {
    const int r = p.MB - g * p.GM;
    return r < p.GM ? r : p.GM;
}

// Tile t of the list (see the header comment).
__host__ __device__ inline FusedTile fused_tile(const FusedFwdParams& p, int t) {
    int start = 0;
    for (int ph = 0; ph <= p.G; ++ph) {
        const int ga = ph < p.G ? fused_group_rows(p, ph) : 0;      // gate/up rows
        const int gb = ph >= 1 ? fused_group_rows(p, ph - 1) : 0;   // down rows
        const int a = ga * p.nJ, b = gb * p.nC;
        if (t >= start + a + b) {
            start += a + b;
            continue;
        }
        const int u = t - start;
        int ia = -1, ib = -1;
        if (b == 0) {
            ia = u;
        } else if (a == 0) {
            ib = u;
        } else {
            const int h = a < p.head ? a : p.head;
            if (u < h) {
                ia = u;
            } else {
                const long long v = u - h, tot = static_cast<long long>(a - h) + b;
                const int nb0 = static_cast<int>(v * b / tot);
                const int nb1 = static_cast<int>((v + 1) * b / tot);
                if (nb1 > nb0)
                    ib = nb0;
                else
                    ia = h + static_cast<int>(v) - nb0;
            }
        }
        if (ia >= 0) return FusedTile{kFusedGateUp, ph * p.GM + ia % ga, ia / ga};
        return FusedTile{kFusedDown, (ph - 1) * p.GM + ib % gb, ib / gb};
    }
    return FusedTile{kFusedDown, 0, 0};  // not reached for t < total
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_gpu_add(unsigned* p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bounded wait for *p >= target (acquire).  False on timeout (recorded) or abort.
__device__ __forceinline__ bool wait_counter(const unsigned* p, unsigned target,
                                             volatile int* abort) {
    if (ld_acquire_gpu(p) >= target) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
        asm volatile("nanosleep.u32 %0;" ::"r"(128u));
        if (ld_acquire_gpu(p) >= target) return true;
        if ((i & 15u) == 0u) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                atomicOr(&g_device_error, kDevErrTimeout);
                *abort = 1;
                return false;
            }
        }
    }
}

template <int ACT>
struct FusedFwd {
    static constexpr const char* kName = ACT == 1 ? "fused_fwd_swiglu" : "fused_fwd_gelu";
    static constexpr int kBK = 64;
    static constexpr int kOut = ACT == 1 ? 128 : 256;  // hidden columns per gate/up tile
    static constexpr int kABytes = 128 * kBK * 2;
    static constexpr int kStageBytes = kABytes + 256 * kBK * 2;
    static constexpr int kStages = 4;
    static constexpr int kQueue = 8;
    static constexpr int kAccCols = 256;
    static constexpr uint32_t kIdesc = make_idesc_bf16(128, 256, false, true);
    static constexpr int kSmemBytes = kStages * kStageBytes + 512 + 1024;
};

template <int ACT>
__global__ void __launch_bounds__(kPipelineThreads, 1)
    fused_mlp_fwd_kernel(const __grid_constant__ FusedFwdParams p) {
    using C = FusedFwd<ACT>;
    constexpr int S = C::kStages, Q = C::kQueue;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t ring = (raw + 1023u) & ~1023u;
    uint8_t* ring_ptr = smem_raw + (ring - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(ring_ptr + S * C::kStageBytes);
    // barrier map: full[S], empty[S], tfull[2], tempty[2], qfull[Q], qempty[Q], drain
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * S + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * S + 2 + b); };
    auto qfull_bar = [&](int s) { return bar0 + 8u * (2 * S + 4 + s); };
    auto qempty_bar = [&](int s) { return bar0 + 8u * (2 * S + 4 + Q + s); };
    const uint32_t drain_bar = bar0 + 8u * (2 * S + 4 + 2 * Q);
    volatile int* tile_q = reinterpret_cast<volatile int*>(bars + 2 * S + 4 + 2 * Q + 1);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(tile_q) + Q);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nkb_up = (p.d + C::kBK - 1) / C::kBK;
    const int nkb_down = (p.f + C::kBK - 1) / C::kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 4);
        }
        for (int s = 0; s < Q; ++s) {
            mbar_init(qfull_bar(s), 1);
            mbar_init(qempty_bar(s), 5);  // MMA thread + one lane per epilogue warp
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.tmX);
        tma_prefetch_desc(&p.tmG);
        if (ACT == 1) tma_prefetch_desc(&p.tmU);
        tma_prefetch_desc(&p.tmH);
        tma_prefetch_desc(&p.tmD);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer + scheduler
        if (lane == 0) {
            int stage = 0, qs = 0;
            uint32_t phase = 0, qph = 0;
            uint32_t armed = 0, armed_par = 0;
            for (;;) {
                const int t = static_cast<int>(atomicAdd(p.sync, 1u));
                if (!mbar_wait(qempty_bar(qs), qph ^ 1u, abort_flag)) break;
                tile_q[qs] = t;
                mbar_arrive(qfull_bar(qs));
                if (++qs == Q) {
                    qs = 0;
                    qph ^= 1u;
                }
                if (t >= p.total) break;
                const FusedTile ti = fused_tile(p, t);
                const int slot = ti.mb % p.R;
                int nkb;
                if (ti.type == kFusedDown) {
                    if (!wait_counter(p.sync + 1 + ti.mb, 4u * p.nJ, abort_flag)) break;
                    fence_proxy_async_global();
                    nkb = nkb_down;
                } else {
                    if (ti.mb >= p.R &&
                        !wait_counter(p.sync + 1 + p.MB + (ti.mb - p.R), 4u * p.nC, abort_flag))
                        break;
                    nkb = nkb_up;
                }
                const int seg = ti.mb / p.mts, mi = ti.mb % p.mts;
                const int kstart = p.ring ? (seg * p.fs) / C::kBK : 0;
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = ring + stage * C::kStageBytes;
                    const uint32_t fb = full_bar(stage);
                    mbar_arrive_expect_tx(fb, C::kStageBytes);
                    const uint32_t b = st + C::kABytes;
                    if (ti.type == kFusedGateUp) {
                        const int k0 = kb * C::kBK;
                        tma_load_2d(st, &p.tmX, fb, k0, seg * p.seg_rows + mi * 128);
                        const int c = ti.j * C::kOut;
                        if (ACT == 1) {
                            tma_load_2d(b, &p.tmG, fb, c, k0);
                            tma_load_2d(b + 8192, &p.tmG, fb, c + 64, k0);
                            tma_load_2d(b + 16384, &p.tmU, fb, c, k0);
                            tma_load_2d(b + 24576, &p.tmU, fb, c + 64, k0);
                        } else {
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                tma_load_2d(b + 8192 * i, &p.tmG, fb, c + 64 * i, k0);
                        }
                    } else {
                        int kr = kb + kstart;
                        if (kr >= nkb) kr -= nkb;
                        const int k0 = kr * C::kBK;
                        tma_load_2d(st, &p.tmH, fb, k0, slot * 128);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            tma_load_2d(b + 8192 * i, &p.tmD, fb, ti.j * 256 + 64 * i, k0);
                    }
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
            }
            for (int s = 0; s < S; ++s)
                if (armed & (1u << s)) mbar_wait_drain(full_bar(s), (armed_par >> s) & 1u);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0, qs = 0, local = 0;
            uint32_t phase = 0, qph = 0;
            for (;;) {
                if (!mbar_wait(qfull_bar(qs), qph, abort_flag)) break;
                const int t = tile_q[qs];
                mbar_arrive(qempty_bar(qs));
                if (++qs == Q) {
                    qs = 0;
                    qph ^= 1u;
                }
                if (t >= p.total) break;
                const FusedTile ti = fused_tile(p, t);
                const int nkb = ti.type == kFusedDown ? nkb_down : nkb_up;
                const int buf = local & 1;
                const uint32_t use = static_cast<uint32_t>(local >> 1);
                if (!mbar_wait(tempty_bar(buf), (use & 1u) ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t acc = tmem_base + static_cast<uint32_t>(buf * C::kAccCols);
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(full_bar(stage), phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = ring + stage * C::kStageBytes;
#pragma unroll
                    for (int kk = 0; kk < C::kBK / 16; ++kk) {
                        const uint64_t a = make_smem_desc(st + 32 * kk, 16, 1024, kLayoutSW128);
                        const uint64_t b =
                            make_smem_desc(st + C::kABytes + 2048 * kk, 8192, 1024, kLayoutSW128);
                        umma_bf16(acc, a, b, C::kIdesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(empty_bar(stage));
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(tfull_bar(buf));
                ++local;
            }
            umma_commit(drain_bar);
            mbar_wait_drain(drain_bar, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        int qs = 0, local = 0;
        uint32_t qph = 0;
        for (;;) {
            int ok = 0, t = 0;
            if (lane == 0) {
                ok = mbar_wait(qfull_bar(qs), qph, abort_flag) ? 1 : 0;
                if (ok) t = tile_q[qs];
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            t = __shfl_sync(0xffffffffu, t, 0);
            if (!ok) break;
            if (lane == 0) mbar_arrive(qempty_bar(qs));
            if (++qs == Q) {
                qs = 0;
                qph ^= 1u;
            }
            if (t >= p.total) break;
            const FusedTile ti = fused_tile(p, t);
            const int buf = local & 1;
            const uint32_t use = static_cast<uint32_t>(local >> 1);
            if (lane == 0) ok = mbar_wait(tfull_bar(buf), use & 1u, abort_flag) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const uint32_t t0 = tmem_base + static_cast<uint32_t>(buf * C::kAccCols) +
                                (static_cast<uint32_t>(q * 32) << 16);
            const int seg = ti.mb / p.mts, mi = ti.mb % p.mts;
            const int rl = mi * 128 + q * 32 + lane;
            const bool row_ok = rl < p.seg_rows;
            if (ti.type == kFusedGateUp) {
                __nv_bfloat16* hrow = p.H + static_cast<long long>((ti.mb % p.R) * 128 + q * 32 + lane) * p.f;
                if (ACT == 1) {
#pragma unroll 1
                    for (int cc = 0; cc < 4; ++cc) {
                        uint32_t g[32], u[32], pk[16];
                        tmem_ld_32x32b_x32(t0 + 32 * cc, g);
                        tmem_ld_32x32b_x32(t0 + 128 + 32 * cc, u);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            pk[i] = pack_bf16x2(
                                silu_f(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]),
                                silu_f(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]));
                        const int c0 = ti.j * 128 + 32 * cc;
                        if (row_ok) store_bf16x32(hrow + c0, pk, p.f - c0);
                    }
                } else {
#pragma unroll 1
                    for (int cc = 0; cc < 8; ++cc) {
                        uint32_t z[32], pk[16];
                        tmem_ld_32x32b_x32(t0 + 32 * cc, z);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            pk[i] = pack_bf16x2(gelu_f(__uint_as_float(z[2 * i])),
                                                gelu_f(__uint_as_float(z[2 * i + 1])));
                        const int c0 = ti.j * 256 + 32 * cc;
                        if (row_ok) store_bf16x32(hrow + c0, pk, p.f - c0);
                    }
                }
            } else {
                const long long row = static_cast<long long>(seg) * p.seg_rows + rl;
#pragma unroll 1
                for (int cc = 0; cc < 8; ++cc) {
                    uint32_t v[32], pk[16];
                    tmem_ld_32x32b_x32(t0 + 32 * cc, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                    const int c0 = ti.j * 256 + 32 * cc;
                    if (row_ok && c0 < p.d) store_bf16x32(p.Y + row * p.d + c0, pk, p.d - c0);
                }
            }
            tc_fence_before();
            // this warp's stores, then the async-proxy fence, then one release
            // per warp on the row block's counter
            if (ti.type == kFusedGateUp) fence_proxy_async_global();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(tempty_bar(buf));
                red_release_gpu_add(p.sync + 1 + (ti.type == kFusedGateUp ? 0 : p.MB) + ti.mb, 1u);
            }
            ++local;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace tspmlp
