// fused2.cuh -- the chunked weight-shard forward in one persistent launch on
// CTA pairs.
//
// The hidden units are cut into chunks (runs of whole shards, in shard
// order).  Per chunk c and pair of 128-token row blocks (row pair) there are
//   gate/up tiles (nJ_c): H_c[rows, j*kOut ..] = act(X[rows] . W[:, cb_c + j*kOut ..])
//   down tiles    (nN):   acc[rows, n*256 ..] (+)= H_c[rows, :] . W_down[cb_c .., n*256 ..]
// with the down tiles adding chunk c's partial output into the fp32
// accumulator in place (store for the first chunk, add, and bf16(acc + tile)
// into Y for the last; a single chunk writes Y directly) -- the partial
// outputs of the shards summed in shard order ("Tensor Parallelism: Splitting
// the Math", steps 4-6).  The tiles are the 256 x 256 paired tiles of
// pipeline2.cuh; gate/up and down tiles share one stage geometry and one
// instruction descriptor, so the MMA issue is the same for both.
//
// Tile list.  Phase p holds the gate/up tiles of chunk p (weight slab outer,
// row pair inner) merged with the down tiles of chunk p-1 (output slab outer,
// row pair inner): one wave of gate/up tiles first, then both in proportion.
// The pair leader takes tile indices from a global atomic counter in list
// order and passes each to both CTAs through their shared-memory queues.
//
// Dependencies (per chunk and row pair, counted in epilogue warps: 4 per CTA,
// 8 per paired tile, each releasing its counter after its stores):
//   down(c, m)    waits for all gate/up(c, m) (its H) and, for c > 0, all
//                 down(c-1, m) (the accumulator rows it adds to);
//   gate/up(c, m) waits, for c > 1, for all down(c-2, m): H is double-
//                 buffered by chunk parity.
// Each points to an earlier tile of the list, so the waits end (and are
// bounded).  H is stored with st.global + an async-proxy fence before the
// release; consumers acquire and fence before their TMA loads.  The
// accumulator is read back by generic loads after a fresh acquire.
#pragma once

#include "fused.cuh"
#include "pipeline2.cuh"

namespace tspmlp {

constexpr int kFusedMaxChunks = 32;

struct FusedPassesParams {
    CUtensorMap tmX;   // X [n][d], box {64, 128}
    CUtensorMap tmG;   // W_gate / A [d][f], box {64, 64}
    CUtensorMap tmU;   // W_up [d][f], box {64, 64} (SwiGLU)
    CUtensorMap tmH0;  // H buffer 0 [n][wmax], box {64, 128}
    CUtensorMap tmH1;  // H buffer 1
    CUtensorMap tmD;   // W_down / B [f][d], box {64, 64}
    int n, d, f;
    int MP;            // row pairs
    int C;             // chunks
    int cb[kFusedMaxChunks];  // chunk column base
    int cw[kFusedMaxChunks];  // chunk width (multiple of 64)
    int nN;            // down tiles per row pair
    int wmax;          // H buffer row pitch
    int head;          // gate/up tiles that open a phase
    int total;
    __nv_bfloat16* H0;
    __nv_bfloat16* H1;
    float* acc;        // [n][d] fp32 (C > 1)
    __nv_bfloat16* Y;  // [n][d]
    unsigned* sync;    // [0] tile counter; [1 + c*MP + m] gate/up warps; [1 + (C+c)*MP + m] down warps
};

struct PassTile {
    int type, c, m, j;  // type 0 gate/up (j = hidden tile), 1 down (j = output tile)
};

template <int KOUT>
__host__ __device__ inline int pass_nj(const FusedPassesParams& p, int c) {
    return (p.cw[c] + KOUT - 1) / KOUT;
}

template <int KOUT>
__host__ __device__ inline PassTile pass_tile(const FusedPassesParams& p, int t) {
    int start = 0;
    for (int ph = 0; ph <= p.C; ++ph) {
        const int a = ph < p.C ? pass_nj<KOUT>(p, ph) * p.MP : 0;
        const int b = ph >= 1 ? p.nN * p.MP : 0;
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
        if (ia >= 0) return PassTile{0, ph, ia % p.MP, ia / p.MP};
        return PassTile{1, ph - 1, ib % p.MP, ib / p.MP};
    }
    return PassTile{1, 0, 0, 0};  // not reached for t < total
}

template <int ACT>
struct FusedPassesCfg {
    static constexpr const char* kName = ACT == 1 ? "fused_passes_swiglu" : "fused_passes_gelu";
    static constexpr int kBK = 64;
    static constexpr int kOut = ACT == 1 ? 128 : 256;
    static constexpr int kABytes = 128 * kBK * 2;
    static constexpr int kStageBytes = kABytes + 128 * kBK * 2;
    static constexpr int kStages = 6;
    static constexpr int kQueue = 8;
    static constexpr uint32_t kIdesc = make_idesc_bf16(256, 256, false, true);
    static constexpr int kSmemBytes = kStages * kStageBytes + 512 + 1024;
};

template <int ACT>
__global__ void __launch_bounds__(kPipelineThreads, 1)
    fused_passes_pair_kernel(const __grid_constant__ FusedPassesParams p) {
    using Cfg = FusedPassesCfg<ACT>;
    constexpr int S = Cfg::kStages, Q = Cfg::kQueue;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t ring = (raw + 1023u) & ~1023u;
    uint8_t* ring_ptr = smem_raw + (ring - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(ring_ptr + S * Cfg::kStageBytes);
    // full[S], empty[S], tfull[2], tempty[2], qfull[Q], qempty[Q], drain
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
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int nkb_up = (p.d + Cfg::kBK - 1) / Cfg::kBK;
    const unsigned target_down = 8u * static_cast<unsigned>(p.nN);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 8);
        }
        for (int s = 0; s < Q; ++s) {
            mbar_init(qfull_bar(s), 1);
            mbar_init(qempty_bar(s), 10);  // leader MMA + 4 leader + 5 partner consumers
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
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.tmX);
        tma_prefetch_desc(&p.tmG);
        if (ACT == 1) tma_prefetch_desc(&p.tmU);
        tma_prefetch_desc(&p.tmH0);
        tma_prefetch_desc(&p.tmH1);
        tma_prefetch_desc(&p.tmD);
    }
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // One queue entry: the leader producer takes a tile and writes it to both
    // CTAs' queues; consumers read their own queue and release the entry on
    // the leader's qempty barrier.
    auto consume_entry = [&](int qs, uint32_t qph, int* t_out) -> bool {
        const bool ok = leader ? mbar_wait(qfull_bar(qs), qph, abort_flag)
                               : mbar_wait_cluster(qfull_bar(qs), qph, abort_flag);
        if (!ok) return false;
        *t_out = tile_q[qs];
        if (leader)
            mbar_arrive(qempty_bar(qs));
        else
            mbar_arrive_remote(map_to_cta(qempty_bar(qs), 0));
        return true;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producers
        if (lane == 0) {
            int stage = 0, qs = 0;
            uint32_t phase = 0, qph = 0, armed = 0, armed_par = 0;
            for (;;) {
                int t;
                if (leader) {
                    t = static_cast<int>(atomicAdd(p.sync, 1u));
                    if (!mbar_wait(qempty_bar(qs), qph ^ 1u, abort_flag)) break;
                    tile_q[qs] = t;
                    st_cluster_u32(map_to_cta(smem_u32(const_cast<int*>(tile_q + qs)), 1),
                                   static_cast<uint32_t>(t));
                    mbar_arrive(qfull_bar(qs));
                    mbar_arrive_remote(map_to_cta(qfull_bar(qs), 1));
                } else {
                    if (!consume_entry(qs, qph, &t)) break;
                }
                if (++qs == Q) {
                    qs = 0;
                    qph ^= 1u;
                }
                if (t >= p.total) break;
                const PassTile ti = pass_tile<Cfg::kOut>(p, t);
                const unsigned* k1done = p.sync + 1 + ti.c * p.MP + ti.m;
                int nkb;
                if (ti.type == 1) {
                    const unsigned tgt = 8u * static_cast<unsigned>(pass_nj<Cfg::kOut>(p, ti.c));
                    if (!wait_counter(k1done, tgt, abort_flag)) break;
                    if (ti.c > 0 &&
                        !wait_counter(p.sync + 1 + (p.C + ti.c - 1) * p.MP + ti.m, target_down,
                                      abort_flag))
                        break;
                    fence_proxy_async_global();
                    nkb = p.cw[ti.c] / Cfg::kBK;
                } else {
                    if (ti.c > 1 &&
                        !wait_counter(p.sync + 1 + (p.C + ti.c - 2) * p.MP + ti.m, target_down,
                                      abort_flag))
                        break;
                    nkb = nkb_up;
                }
                const int row = ti.m * 256 + static_cast<int>(rank) * 128;
                const int cbase = p.cb[ti.c];  // read once a tile, not per k-block
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = ring + stage * Cfg::kStageBytes;
                    if (leader) mbar_arrive_expect_tx(full_bar(stage), 2u * Cfg::kStageBytes);
                    const uint32_t fb = map_to_cta(full_bar(stage), 0);
                    const int k0 = kb * Cfg::kBK;
                    if (ti.type == 0) {
                        tma_load_2d_pair(st, &p.tmX, fb, k0, row);
                        const int c = cbase + ti.j * Cfg::kOut;
                        if (ACT == 1) {
                            const CUtensorMap* w = leader ? &p.tmG : &p.tmU;
                            tma_load_2d_pair(st + Cfg::kABytes, w, fb, c, k0);
                            tma_load_2d_pair(st + Cfg::kABytes + 8192, w, fb, c + 64, k0);
                        } else {
                            const int cr = c + static_cast<int>(rank) * 128;
                            tma_load_2d_pair(st + Cfg::kABytes, &p.tmG, fb, cr, k0);
                            tma_load_2d_pair(st + Cfg::kABytes + 8192, &p.tmG, fb, cr + 64, k0);
                        }
                    } else {
                        tma_load_2d_pair(st, (ti.c & 1) ? &p.tmH1 : &p.tmH0, fb, k0, row);
                        const int n0 = ti.j * 256 + static_cast<int>(rank) * 128;
                        tma_load_2d_pair(st + Cfg::kABytes, &p.tmD, fb, n0, cbase + k0);
                        tma_load_2d_pair(st + Cfg::kABytes + 8192, &p.tmD, fb, n0 + 64, cbase + k0);
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
            if (leader)
                for (int s = 0; s < S; ++s)
                    if (armed & (1u << s)) mbar_wait_drain(full_bar(s), (armed_par >> s) & 1u);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (lane == 0 && leader) {
            int stage = 0, qs = 0, local = 0;
            uint32_t phase = 0, qph = 0;
            for (;;) {
                int t;
                if (!consume_entry(qs, qph, &t)) break;
                if (++qs == Q) {
                    qs = 0;
                    qph ^= 1u;
                }
                if (t >= p.total) break;
                const PassTile ti = pass_tile<Cfg::kOut>(p, t);
                const int nkb = ti.type == 1 ? p.cw[ti.c] / Cfg::kBK : nkb_up;
                const int buf = local & 1;
                const uint32_t use = static_cast<uint32_t>(local >> 1);
                if (!mbar_wait(tempty_bar(buf), (use & 1u) ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t acc = tmem_base + static_cast<uint32_t>(buf) * 256u;
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(full_bar(stage), phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = ring + stage * Cfg::kStageBytes;
#pragma unroll
                    for (int kk = 0; kk < Cfg::kBK / 16; ++kk) {
                        const uint64_t a = make_smem_desc(st + 32 * kk, 16, 1024, kLayoutSW128);
                        const uint64_t b =
                            make_smem_desc(st + Cfg::kABytes + 2048 * kk, 8192, 1024, kLayoutSW128);
                        umma_bf16_pair(acc, a, b, Cfg::kIdesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit_pair_mc(empty_bar(stage), 0x3);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit_pair_mc(tfull_bar(buf), 0x3);
                ++local;
            }
            umma_commit_pair_mc(drain_bar, 0x1);
            mbar_wait_drain(drain_bar, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        int qs = 0, local = 0;
        uint32_t qph = 0;
        for (;;) {
            int ok = 0, t = 0;
            if (lane == 0) ok = consume_entry(qs, qph, &t) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            t = __shfl_sync(0xffffffffu, t, 0);
            if (!ok) break;
            if (++qs == Q) {
                qs = 0;
                qph ^= 1u;
            }
            if (t >= p.total) break;
            const PassTile ti = pass_tile<Cfg::kOut>(p, t);
            const int buf = local & 1;
            const uint32_t use = static_cast<uint32_t>(local >> 1);
            if (lane == 0) ok = mbar_wait_cluster(tfull_bar(buf), use & 1u, abort_flag) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const uint32_t t0 =
                tmem_base + static_cast<uint32_t>(buf) * 256u + (static_cast<uint32_t>(q * 32) << 16);
            const int row = ti.m * 256 + static_cast<int>(rank) * 128 + q * 32 + lane;
            const bool row_ok = row < p.n;
            if (ti.type == 0) {
                __nv_bfloat16* hrow = ((ti.c & 1) ? p.H1 : p.H0) + static_cast<long long>(row) * p.wmax;
                const int width = p.cw[ti.c];
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
                        if (row_ok) store_bf16x32(hrow + c0, pk, width - c0);
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
                        if (row_ok) store_bf16x32(hrow + c0, pk, width - c0);
                    }
                }
                fence_proxy_async_global();
            } else {
                // mode: single chunk -> bf16(tile); first -> store fp32; last -> bf16(acc + tile)
                const int mode = p.C == 1 ? 3 : (ti.c == 0 ? 0 : (ti.c == p.C - 1 ? 2 : 1));
                if (mode == 1 || mode == 2)
                    (void)ld_acquire_gpu(p.sync + 1 + (p.C + ti.c - 1) * p.MP + ti.m);
                const long long roff = static_cast<long long>(row) * p.d;
#pragma unroll 1
                for (int cc = 0; cc < 8; ++cc) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(t0 + 32 * cc, v);
                    tmem_ld_wait();
                    const int c0 = ti.j * 256 + 32 * cc;
                    const int valid = p.d - c0;
                    if (!row_ok || valid <= 0) continue;
                    if (mode == 0) {
                        store_f32x32(p.acc + roff + c0, v, valid);
                    } else if (mode == 1) {
                        float* a = p.acc + roff + c0;
                        if (valid >= 32) {
                            float4* a4 = reinterpret_cast<float4*>(a);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                float4 o = a4[i];
                                o.x += __uint_as_float(v[4 * i]);
                                o.y += __uint_as_float(v[4 * i + 1]);
                                o.z += __uint_as_float(v[4 * i + 2]);
                                o.w += __uint_as_float(v[4 * i + 3]);
                                a4[i] = o;
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (i < valid) a[i] += __uint_as_float(v[i]);
                        }
                    } else {
                        uint32_t pk[16];
                        if (mode == 2) {
                            const float* a = p.acc + roff + c0;
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const float x0 = (2 * i < valid ? a[2 * i] : 0.f) + __uint_as_float(v[2 * i]);
                                const float x1 = (2 * i + 1 < valid ? a[2 * i + 1] : 0.f) +
                                                 __uint_as_float(v[2 * i + 1]);
                                pk[i] = pack_bf16x2(x0, x1);
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]),
                                                    __uint_as_float(v[2 * i + 1]));
                        }
                        store_bf16x32(p.Y + roff + c0, pk, valid);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader)
                    mbar_arrive(tempty_bar(buf));
                else
                    mbar_arrive_remote(map_to_cta(tempty_bar(buf), 0));
                red_release_gpu_add(p.sync + 1 + (ti.type == 0 ? ti.c : p.C + ti.c) * p.MP + ti.m, 1u);
            }
            ++local;
        }
    }

    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
}

}  // namespace tspmlp
