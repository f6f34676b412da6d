// attn.cuh -- the attention core of the TSP attention schedule on tcgen05.
//
// "Folding Tensor and Sequence Parallelism for Memory-Efficient Transformer
// Training & Inference", Abstract: for attention every rank owns a sequence
// shard of tokens, iterates over the broadcast parameter shards (groups of
// heads), and reconstructs the whole context through a sequence-wise
// key/value exchange.  On one GPU the P sequence shards are logical: the
// queries of sequence shard s visit the key/value shards in ring order
// s, s+1, ..., s-1 (mod P), 128 keys a block, and every block is merged into
// a running row maximum, row sum and weighted value sum (the exact softmax
// merge), so no shard ever needs the whole score row at once.  With the
// causal mask the shards after s hold only future keys and are skipped.
//
// One CTA per SM, persistent, 576 threads:
//   warp 0      TMA producer: per work item the two 128-row query tiles, then
//               the key and value blocks in the item's ring order (each key
//               block one block ahead of its value block) through a ring of
//               three 32 KB stages.
//   warp 1      MMA issuer: S_a = Q_a K^T into tensor memory and O_a += P_a V
//               (a = 0, 1).  A tile's next scores are issued as soon as its
//               softmax has read the current ones, so the tensor pipe works on
//               one tile while the other tile's softmax runs.
//   warps 2-17  softmax: two warpgroups per tile, one per half of the 128 keys
//               of a block; thread = one query row (warp w reads TMEM lanes
//               32 (w % 4) .. +31).  Each reads the row's 128 scores in two
//               64-column rounds (the other half's for the maximum only, then
//               its own, kept in registers), applies the mask, updates the
//               running max (rescaling its half of O in tensor memory only
//               when the max grows by more than 2^8, which keeps every
//               probability <= 256 and the result exact), writes its half's
//               probabilities as bf16 to shared memory for the P V product,
//               and at the end of the item divides O by the row sum and stores
//               it.
// Tensor memory: O_0, O_1, S_0, S_1, 128 fp32 columns each (512 columns).
// Shared memory: Q_0, Q_1, P_0, P_1 (32 KB each) and the K/V ring (96 KB).
// Every wait is bounded as in pipeline.cuh.
#pragma once

#include <cuda_bf16.h>

#include "pipeline.cuh"

namespace tspmlp {

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// The largest of three floats (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Two floats as one 64-bit register pair (the operand of the packed f32x2
// instructions of sm_100).
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

// (d0, d1) = (a0, a1) * b + c, b and c packed pairs: one fma.rn.f32x2 (each
// lane rounded once, as fmaf).
__device__ __forceinline__ void fma_f32x2(float a0, float a1, uint64_t b, uint64_t c, float& d0,
                                          float& d1) {
    asm("{\n\t.reg .b64 va, vd;\n\t"
        "mov.b64 va, {%2, %3};\n\t"
        "fma.rn.f32x2 vd, va, %4, %5;\n\t"
        "mov.b64 {%0, %1}, vd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "l"(b), "l"(c));
}

// (s0, s1) += (b0, b1): one add.rn.f32x2.
__device__ __forceinline__ void add_f32x2(float& s0, float& s1, float b0, float b1) {
    asm("{\n\t.reg .b64 vs, vb;\n\t"
        "mov.b64 vs, {%0, %1};\n\t"
        "mov.b64 vb, {%2, %3};\n\t"
        "add.rn.f32x2 vs, vs, vb;\n\t"
        "mov.b64 {%0, %1}, vs;\n\t}"
        : "+f"(s0), "+f"(s1)
        : "f"(b0), "f"(b1));
}

// 2^x on the special-function unit (the ex2 instruction; -inf gives +0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

struct AttnParams {
    CUtensorMap tmQ, tmK, tmV;  // [n][heads * 128] (Q, K bf16 or fp16; V bf16), box {64, 128},
                                // 128-byte swizzle
    __nv_bfloat16* O;           // [n][ldo] bf16
    long long ldo;
    int n;       // tokens
    int heads;
    int P;       // sequence shards
    int ns;      // tokens per sequence shard (n / P)
    int nb;      // key blocks per shard: ceil(ns / 128)
    int npr;     // query-tile pairs per shard: ceil(ns / 256)
    int causal;
    int items;   // heads * P * npr
    float sl2;   // log2(e) / sqrt(128): scores to base-2 exponents
};

// A work item: 256 query rows (two tiles) of one head inside one sequence
// shard, and the key blocks they visit.
struct AttnItem {
    int h, s, q0;
    int qlast;  // last query row of the item inside its shard
    int idiag;  // causal: last block of shard s with a key <= qlast
    int nkv;    // key blocks visited
};

struct AttnCore {
    static constexpr int kThreads = 576;
    static constexpr int kTileBytes = 128 * 128 * 2;  // a 128 x 128 bf16 tile (two 64-column boxes)
    static constexpr int kStages = 3;
    static constexpr int kQOff = 0, kPOff = 2 * kTileBytes, kKVOff = 4 * kTileBytes;
    static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
    static constexpr int kSmemBytes = kBarOff + 512 + 1024;
    // Q K^T in fp16 (the block's projections store Q and K as fp16: three more
    // mantissa bits than bf16 where the scores' rounding matters most) or bf16
    static constexpr uint32_t kIdescSf16 = make_idesc_f16(128, 128, false, false);
    static constexpr uint32_t kIdescSbf16 = make_idesc_bf16(128, 128, false, false);
    static constexpr uint32_t kIdescPV = make_idesc_bf16(128, 128, false, true);
    // the running max is moved (and O rescaled) only when a block's max
    // exceeds it by more than this many powers of two
    static constexpr float kRescaleLog2 = 8.0f;

    // Items in head-major order (concurrent items share their head's keys and
    // values in L2); with the causal mask each head's items run from the
    // most key blocks to the fewest.
    __device__ static AttnItem item(const AttnParams& p, int k) {
        const int per_head = p.P * p.npr;
        AttnItem it;
        it.h = k / per_head;
        int r = k - it.h * per_head;
        if (p.causal) r = per_head - 1 - r;
        it.s = r / p.npr;
        const int i = r - it.s * p.npr;
        it.q0 = it.s * p.ns + i * 256;
        const int shard_end = (it.s + 1) * p.ns;
        it.qlast = min(it.q0 + 255, shard_end - 1);
        it.idiag = (it.qlast - it.s * p.ns) >> 7;
        it.nkv = p.causal ? it.idiag + 1 + it.s * p.nb : p.P * p.nb;
        return it;
    }
    // The item CTA `cta` takes at round `it` (snake order, so that with the
    // causal mask every CTA gets a long and a short item in turn); -1 if none.
    __device__ static int item_index(const AttnParams& p, int it, int cta, int G) {
        const int k = it * G + ((it & 1) ? G - 1 - cta : cta);
        return k < p.items ? k : -1;
    }
    // First key and valid keys of block t of an item: the ring order s, s+1,
    // ... (mod P), every shard in blocks of 128 keys; with the causal mask
    // shard s up to the diagonal, then shards 0 .. s-1.
    __device__ static void block(const AttnParams& p, const AttnItem& it, int t, int* kstart,
                                 int* kvalid) {
        int u, ib;
        if (!p.causal) {
            const int q = t / p.nb;
            u = it.s + q;
            if (u >= p.P) u -= p.P;
            ib = t - q * p.nb;
        } else if (t <= it.idiag) {
            u = it.s;
            ib = t;
        } else {
            const int t2 = t - it.idiag - 1;
            u = t2 / p.nb;
            ib = t2 - u * p.nb;
        }
        *kstart = u * p.ns + ib * 128;
        *kvalid = min(128, p.ns - ib * 128);
    }
};

template <bool QK_F16>
__global__ void __launch_bounds__(AttnCore::kThreads, 1)
    attn_core_kernel(const __grid_constant__ AttnParams p) {
    using C = AttnCore;
    constexpr uint32_t kIdescS = QK_F16 ? C::kIdescSf16 : C::kIdescSbf16;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = smem_raw + (base - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(base_ptr + C::kBarOff);
    const uint32_t bar0 = smem_u32(bars);
    const uint32_t q_full = bar0, q_empty = bar0 + 8;
    auto kv_full = [&](int s) { return bar0 + 16u + 8u * s; };
    auto kv_empty = [&](int s) { return bar0 + 16u + 8u * (S + s); };
    auto s_full = [&](int a) { return bar0 + 16u + 8u * (2 * S + a); };
    auto s_empty = [&](int a) { return bar0 + 16u + 8u * (2 * S + 2 + a); };
    auto p_full = [&](int a) { return bar0 + 16u + 8u * (2 * S + 4 + a); };
    auto pv_done = [&](int a) { return bar0 + 16u + 8u * (2 * S + 6 + a); };
    const uint32_t drain_bar = bar0 + 16u + 8u * (2 * S + 8);
    // the two warps holding rows 32 q .. 32 q + 31 of tile a meet at the end of
    // an item: their row sums are published (x_full), then read (x_read)
    auto x_full = [&](int a, int q) { return bar0 + 16u + 8u * (2 * S + 9 + 4 * a + q); };
    auto x_read = [&](int a, int q) { return bar0 + 16u + 8u * (2 * S + 17 + 4 * a + q); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 + 2 * S + 25);
    static_assert(8 * (2 + 2 * S + 25) + 8 <= 512, "barrier area");
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < S; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(s_full(a), 1);
            mbar_init(s_empty(a), 8);
            mbar_init(p_full(a), 8);
            mbar_init(pv_done(a), 1);
        }
        mbar_init(drain_bar, 1);
        for (int a = 0; a < 2; ++a)
            for (int q = 0; q < 4; ++q) {
                mbar_init(x_full(a, q), 2);
                mbar_init(x_read(a, q), 2);
            }
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.tmQ);
        tma_prefetch_desc(&p.tmK);
        tma_prefetch_desc(&p.tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int G = static_cast<int>(gridDim.x);
    const int cta = static_cast<int>(blockIdx.x);
    const int rounds = (p.items + G - 1) / G;
    const uint32_t qs = base + C::kQOff, ps = base + C::kPOff, kvs = base + C::kKVOff;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            int stage = 0, done = 0;
            uint32_t phase = 0, armed = 0, armed_par = 0;
            bool q_armed = false;
            uint32_t q_par = 0;
            bool ok = true;
            for (int r = 0; r < rounds && ok; ++r) {
                const int k = C::item_index(p, r, cta, G);
                if (k < 0) continue;
                const AttnItem it = C::item(p, k);
                const int col = it.h * 128;
                if (done > 0 && !mbar_wait(q_empty, (done - 1) & 1, abort_flag)) break;
                mbar_arrive_expect_tx(q_full, 2 * C::kTileBytes);
                for (int a = 0; a < 2; ++a) {
                    tma_load_2d(qs + a * C::kTileBytes, &p.tmQ, q_full, col, it.q0 + 128 * a);
                    tma_load_2d(qs + a * C::kTileBytes + 16384, &p.tmQ, q_full, col + 64,
                                it.q0 + 128 * a);
                }
                q_armed = true;
                q_par = done & 1;
                // K_0, then K_{t+1} ahead of V_t: a key block's stage is the one
                // the value block two blocks back used, so the keys of the next
                // block load a whole block before the scores need them
                auto load_block = [&](bool is_v, int t) {
                    int kst, kval;
                    C::block(p, it, t, &kst, &kval);
                    if (!mbar_wait(kv_empty(stage), phase ^ 1u, abort_flag)) return false;
                    const CUtensorMap* m = is_v ? &p.tmV : &p.tmK;
                    const uint32_t dst = kvs + stage * C::kTileBytes;
                    mbar_arrive_expect_tx(kv_full(stage), C::kTileBytes);
                    tma_load_2d(dst, m, kv_full(stage), col, kst);
                    tma_load_2d(dst + 16384, m, kv_full(stage), col + 64, kst);
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    return true;
                };
                ok = load_block(false, 0);
                for (int t = 0; t < it.nkv && ok; ++t) {
                    if (t + 1 < it.nkv && !load_block(false, t + 1)) ok = false;
                    else if (!load_block(true, t)) ok = false;
                }
                ++done;
            }
            // every load must land before shared memory goes away
            for (int s = 0; s < S; ++s)
                if (armed & (1u << s)) mbar_wait_drain(kv_full(s), (armed_par >> s) & 1u);
            if (q_armed) mbar_wait_drain(q_full, q_par);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0, done = 0;
            uint32_t phase = 0;
            uint32_t s_cnt[2] = {0, 0}, p_cnt[2] = {0, 0};
            bool ok = true;
            auto wait_kv = [&](int* st) {
                if (!mbar_wait(kv_full(stage), phase, abort_flag)) return false;
                *st = stage;
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
                return true;
            };
            // S_a = Q_a K^T: A = Q (K-major over dh), B = K block (K-major over dh)
            auto issue_s = [&](int a, int kst) {
                const uint32_t qa = qs + a * C::kTileBytes, kb = kvs + kst * C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + 32 * (kk & 3);
                    umma_bf16(tmem + 256 + 128 * a, make_smem_desc(qa + off, 16, 1024, kLayoutSW128),
                              make_smem_desc(kb + off, 16, 1024, kLayoutSW128), kIdescS,
                              kk != 0 ? 1u : 0u);
                }
                umma_commit(s_full(a));
            };
            // O_a (+)= P_a V: A = P (K-major over keys), B = V block (MN-major)
            auto issue_pv = [&](int a, int vst, bool acc) {
                const uint32_t pa = ps + a * C::kTileBytes, vb = kvs + vst * C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + 32 * (kk & 3);
                    umma_bf16(tmem + 128 * a, make_smem_desc(pa + off, 16, 1024, kLayoutSW128),
                              make_smem_desc(vb + 2048 * kk, 16384, 1024, kLayoutSW128), C::kIdescPV,
                              (acc || kk != 0) ? 1u : 0u);
                }
                umma_commit(pv_done(a));
            };
            for (int r = 0; r < rounds && ok; ++r) {
                const int k = C::item_index(p, r, cta, G);
                if (k < 0) continue;
                const AttnItem it = C::item(p, k);
                if (!mbar_wait(q_full, done & 1, abort_flag)) break;
                tc_fence_after();
                int kst = 0, vst = 0;
                if (!wait_kv(&kst)) break;
                tc_fence_after();
#pragma unroll
                for (int a = 0; a < 2 && ok; ++a) {
                    if (!mbar_wait(s_empty(a), (s_cnt[a] & 1u) ^ 1u, abort_flag)) ok = false;
                    else {
                        tc_fence_after();
                        issue_s(a, kst);
                        ++s_cnt[a];
                    }
                }
                if (!ok) break;
                umma_commit(kv_empty(kst));
                // Q is free once the item's last Q K^T is done: the next item's
                // query tiles load while this item's last blocks finish
                if (it.nkv == 1) umma_commit(q_empty);
                // per block j and tile a: S_{a, j+1} as soon as the softmax has
                // read S_{a, j} (it reads S first), then O_a += P_{a, j} V_j once
                // the probabilities are in shared memory; the next block's
                // scores are then ready when the softmax finishes this one
                for (int j = 0; j < it.nkv && ok; ++j) {
                    // the producer's order: K_{j+1}, then V_j (waited for only
                    // once the first tile's next scores are issued)
                    const bool more = j + 1 < it.nkv;
                    if (more && !wait_kv(&kst)) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int a = 0; a < 2; ++a) {
                        if (more) {
                            if (!mbar_wait(s_empty(a), (s_cnt[a] & 1u) ^ 1u, abort_flag)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            issue_s(a, kst);
                            ++s_cnt[a];
                            if (a == 1) {
                                umma_commit(kv_empty(kst));
                                if (j + 2 == it.nkv) umma_commit(q_empty);
                            }
                        }
                        if (a == 0 && !wait_kv(&vst)) {
                            ok = false;
                            break;
                        }
                        if (!mbar_wait(p_full(a), p_cnt[a] & 1u, abort_flag)) {
                            ok = false;
                            break;
                        }
                        ++p_cnt[a];
                        tc_fence_after();
                        issue_pv(a, vst, j > 0);
                        if (a == 1) umma_commit(kv_empty(vst));
                    }
                }
                if (!ok) break;
                ++done;
            }
            umma_commit(drain_bar);
            mbar_wait_drain(drain_bar, 0);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax (four warpgroups)
        // Two warpgroups per tile: both read the whole score row for its
        // maximum, and each exponentiates, sums and writes P for one half of
        // the 128 keys, and owns that half of O's columns.
        const int sw = warp - 2;
        const int a = sw >> 3;                    // tile of this warpgroup
        const int hf = (sw >> 2) & 1;             // key half [64 hf, 64 hf + 64)
        const int q = warp & 3;                   // TMEM lane quarter
        const int r = q * 32 + lane;              // row of the tile
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t s_tm = tmem + 256 + 128 * a + lane_off;
        const uint32_t o_tm = tmem + 128 * a + 64 * hf + lane_off;
        const uint32_t p_box = ps + a * C::kTileBytes + hf * 16384;  // this half's P box
        const uint32_t p_row = p_box + r * 128;
        const uint32_t p_row_other = ps + a * C::kTileBytes + (1 - hf) * 16384 + r * 128;
        const uint32_t swz = static_cast<uint32_t>(r & 7);
        uint32_t s_cnt = 0, pv_cnt = 0, xn = 0;  // xn: end-of-item meetings so far
        bool ok = true;
        for (int rd = 0; rd < rounds && ok; ++rd) {
            const int k = C::item_index(p, rd, cta, G);
            if (k < 0) continue;
            const AttnItem it = C::item(p, k);
            const int t0 = it.q0 + 128 * a;   // first row of this tile
            const int qrow = t0 + r;
            float m_run = -INFINITY, lsum = 0.f;
            for (int j = 0; j < it.nkv; ++j) {
                int kst, kval;
                C::block(p, it, j, &kst, &kval);
                int w = 0;
                if (lane == 0) w = mbar_wait(s_full(a), s_cnt & 1u, abort_flag) ? 1 : 0;
                ++s_cnt;
                if (!__shfl_sync(0xffffffffu, w, 0)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // keys at column >= lim are masked: past the shard's end, or
                // (causal) after this row's own position
                int lim = 128;
                if (kval < 128 || (p.causal && kst + 127 > t0)) {
                    lim = kval;
                    if (p.causal) lim = min(lim, qrow - kst + 1);
                }
                const bool masked = lim < 128;
                // The row maximum over all 128 keys (both warpgroups of the tile
                // compute it, identically) in two TMEM rounds of 64 columns: the
                // other half's keys first, then this half's, which stay in
                // registers for the probabilities.
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                uint32_t v[2][32];
#pragma unroll
                for (int round = 0; round < 2; ++round) {
                    const int h = round == 0 ? 1 - hf : hf;
                    tmem_ld_32x32b_x32(s_tm + 64 * h, v[0]);
                    tmem_ld_32x32b_x32(s_tm + 64 * h + 32, v[1]);
                    tmem_ld_wait();
                    if (masked) {
#pragma unroll
                        for (int c = 0; c < 2; ++c)
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (64 * h + 32 * c + e >= lim) v[c][e] = __float_as_uint(-INFINITY);
                    }
#pragma unroll
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            m4[0] = fmax3(m4[0], __uint_as_float(v[c][e]), __uint_as_float(v[c][e + 1]));
                            m4[1] = fmax3(m4[1], __uint_as_float(v[c][e + 2]), __uint_as_float(v[c][e + 3]));
                            m4[2] = fmax3(m4[2], __uint_as_float(v[c][e + 4]), __uint_as_float(v[c][e + 5]));
                            m4[3] = fmax3(m4[3], __uint_as_float(v[c][e + 6]), __uint_as_float(v[c][e + 7]));
                        }
                }
                // S_a is no longer read: the next block's Q K^T may overwrite it
                // while these probabilities are computed
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(s_empty(a));
                const float mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
                const float mb = __fmul_rn(mx, p.sl2);
                float alpha = 1.f;
                bool resc = false;
                if (mb > m_run + C::kRescaleLog2) {
                    alpha = ex2_approx(m_run - mb);  // 0 while nothing has been seen
                    m_run = mb;
                    resc = true;
                }
                const float moff = m_run == -INFINITY ? 0.f : m_run;
                // probabilities 2^(s log2(e)/sqrt(128) - m) of this half's 64
                // keys and their sum, packed as bf16 pairs in place (pair e, e + 1
                // into word e / 2, already read).  The exponent is one fused
                // multiply-add: for the row's maximum it leaves only m's own
                // rounding error, below 2^-12 while |m| < 4096.  Larger m
                // (saturated inputs) take the product rounded first, as m was, so
                // the maximum gives exactly 2^0.
                const bool exact_max = fabsf(moff) >= 4096.f;
                // eight partial sums, kept and added in pairs
                float ls8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                const uint64_t sl2x2 = f32x2(p.sl2, p.sl2), negm2 = f32x2(-moff, -moff);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t(&w)[32] = v[c];
                    if (!exact_max) {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            float x0, x1;
                            fma_f32x2(__uint_as_float(w[e]), __uint_as_float(w[e + 1]), sl2x2, negm2, x0, x1);
                            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                            const int g = 2 * ((e >> 1) & 3);
                            add_f32x2(ls8[g], ls8[g + 1], p0, p1);
                            w[e >> 1] = pack_bf16x2(p0, p1);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float p0 = ex2_approx(__fmul_rn(__uint_as_float(w[e]), p.sl2) - moff);
                            const float p1 = ex2_approx(__fmul_rn(__uint_as_float(w[e + 1]), p.sl2) - moff);
                            const int g = 2 * ((e >> 1) & 3);
                            add_f32x2(ls8[g], ls8[g + 1], p0, p1);
                            w[e >> 1] = pack_bf16x2(p0, p1);
                        }
                    }
                }
                if (j > 0) {
                    // P_a and O_a are free once the previous block's P V is done
                    int w2 = 0;
                    if (lane == 0) w2 = mbar_wait(pv_done(a), pv_cnt & 1u, abort_flag) ? 1 : 0;
                    ++pv_cnt;
                    if (!__shfl_sync(0xffffffffu, w2, 0)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                // P in the 128-byte-swizzled K-major layout (box hf; 16-byte chunk
                // k of row r at chunk k ^ (r % 8))
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t chunk = static_cast<uint32_t>(c * 4 + kk);
                        st_shared_v4(p_row + ((chunk ^ swz) << 4), v[c][4 * kk], v[c][4 * kk + 1],
                                     v[c][4 * kk + 2], v[c][4 * kk + 3]);
                    }
                // O_a is rescaled (rarely) with the scores' registers free
                if (j > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
                    for (int c = 0; c < 2; ++c) {
                        uint32_t o[32];
                        tmem_ld_32x32b_x32(o_tm + 32 * c, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st_32x32b_x32(o_tm + 32 * c, o);
                    }
                    tmem_st_wait();
                }
                add_f32x2(ls8[0], ls8[1], ls8[2], ls8[3]);
                add_f32x2(ls8[4], ls8[5], ls8[6], ls8[7]);
                add_f32x2(ls8[0], ls8[1], ls8[4], ls8[5]);
                lsum = lsum * alpha + (ls8[0] + ls8[1]);
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full(a));
            }
            if (!ok) break;
            // epilogue: the row sum of both halves, then this half's columns of
            // O / l in bf16
            int w3 = 0;
            if (lane == 0) w3 = mbar_wait(pv_done(a), pv_cnt & 1u, abort_flag) ? 1 : 0;
            ++pv_cnt;
            if (!__shfl_sync(0xffffffffu, w3, 0)) break;
            tc_fence_after();
            // the last P V has read P: each half leaves its partial sum in its
            // own P row, the row's two warps meet, read the other's, and meet
            // again before either writes P of the next item there
            // (bounded meetings on mbarriers, so that a partner which left on a
            // timeout cannot hold the other warp)
            auto meet = [&](uint32_t bar) {
                __syncwarp();
                int wm = 0;
                if (lane == 0) {
                    mbar_arrive(bar);
                    wm = mbar_wait(bar, xn & 1u, abort_flag) ? 1 : 0;
                }
                wm = __shfl_sync(0xffffffffu, wm, 0);
                __syncwarp();
                return wm != 0;
            };
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(p_row), "f"(lsum) : "memory");
            if (!meet(x_full(a, q))) break;
            float lo;
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(lo) : "r"(p_row_other) : "memory");
            if (!meet(x_read(a, q))) break;
            ++xn;
            const float inv = 1.f / (hf == 0 ? lsum + lo : lo + lsum);
            const bool row_ok = qrow <= it.qlast;
            __nv_bfloat16* orow = p.O + static_cast<long long>(qrow) * p.ldo + it.h * 128 + 64 * hf;
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                uint32_t o[32];
                tmem_ld_32x32b_x32(o_tm + 32 * c, o);
                tmem_ld_wait();
                if (row_ok) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[e] = make_uint4(
                            pack_bf16x2(__uint_as_float(o[8 * e]) * inv, __uint_as_float(o[8 * e + 1]) * inv),
                            pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv),
                            pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv),
                            pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv));
                }
            }
            tc_fence_before();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tspmlp
