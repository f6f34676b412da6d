// recipes.cuh -- the tile recipes run by the tcgen05 pipeline (pipeline.cuh).
//
// Shapes: UMMA M = 128 (tile rows = tokens, or weight rows for the weight
// gradients), N = 128 or 256, K = 16 per instruction; bf16 operands, fp32
// accumulators in tensor memory.  Operand tiles are staged by TMA with the
// 128-byte swizzle (64-byte for the K = 32 stages of the backward kernel):
//   K-major operand, BK = 64: one box {64 k, rows}; 8-row groups 1024 B apart
//       (SBO); the K = 16 sub-steps advance the start address by 32 B.
//   K-major operand, BK = 32: one box {32 k, rows} with the 64-byte swizzle;
//       8-row groups 512 B apart; sub-steps advance by 32 B.
//   MN-major operand: boxes {64 mn, BK k} side by side; a box is BK rows of
//       128 B, 8-row groups 1024 B apart (SBO), neighbouring 64-wide MN blocks
//       BK*128 B apart (LBO); the K = 16 sub-steps advance by 2048 B.
//
// Row segments (SegGeom) let one launch cover several independent row blocks,
// each paired with its own weight shard: the weight-shard schedule uses one
// segment of all tokens; the folded tensor-and-sequence ring uses one segment
// per sequence shard, segment s meeting weight shard (s + t) mod P at ring
// step t ("Folding Tensor and Sequence Parallelism for Memory-Efficient
// Transformer Training & Inference", Abstract).
#pragma once

#include <cuda_bf16.h>

#include "pipeline.cuh"

namespace tspmlp {

struct SegGeom {
    int seg_rows;   // rows per segment
    int num_segs;   // segments in this launch
    int seg_begin;  // global index of the launch's first segment
    int ring;       // 1: segment sg uses weight shard (sg + ring_step) mod P
    int ring_step;
    int P;
    int fs;         // hidden columns per weight shard
    int col_base;   // hidden column base when ring == 0
    __host__ __device__ __forceinline__ int mtiles() const { return (seg_rows + 127) >> 7; }
    __host__ __device__ __forceinline__ int shard_col(int s) const {
        return ring ? ((seg_begin + s + ring_step) % P) * fs : col_base;
    }
};

// ----------------------------------------------------------------------------
// epilogue helpers (one thread = one tile row)

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

__device__ __forceinline__ float gelu_f(float z) {
    return 0.5f * z * (1.0f + erff(z * 0.70710678118654752440f));
}

// 32 bf16 (16 packed words) to dst[0..valid), vectorised when the whole run fits.
__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const uint32_t (&pk)[16],
                                              int valid) {
    if (valid >= 32) {
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    } else {
        // unrolled with constant indices, so pk stays in registers (a
        // run-time index would put it on the stack for every call)
        uint16_t* d16 = reinterpret_cast<uint16_t*>(dst);
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (i < valid)
                d16[i] = static_cast<uint16_t>((i & 1) ? (pk[i >> 1] >> 16) : (pk[i >> 1] & 0xFFFFu));
    }
}

__device__ __forceinline__ void store_f32x32(float* dst, const uint32_t (&v)[32], int valid) {
    if (valid >= 32) {
        float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            d4[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (i < valid) dst[i] = __uint_as_float(v[i]);
    }
}

// ----------------------------------------------------------------------------
// warp-staged stores (coalesced): in the epilogues a thread owns one tile row,
// so a plain vector store of a warp writes 16 bytes into each of 32 rows.
// These helpers pass a warp's 32 rows x 32 columns through a per-warp buffer
// in shared memory (4 KB) and write it out row after row: every store
// instruction then covers whole 128-byte (fp32) or 64-byte (16-bit) row pieces
// of 4 or 8 consecutive rows.  Warp-collective: every lane calls, with the
// warp's common destination base, row pitch and valid column count; rows at
// or past `nrows` are not written.

__device__ __forceinline__ void sts_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// Flags between CTAs of one persistent grid (all resident): a release store,
// and a bounded acquire wait for the value 1 (about two seconds of
// %globaltimer; on expiry the device error word records a timeout and the
// caller goes on).
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void wait_flag_gpu(const int* p) {
    auto ld = [p]() {
        int v;
        asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
        return v;
    };
    if (ld() == 1) return;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
        asm volatile("nanosleep.u32 %0;" ::"r"(64u));
        if (ld() == 1) return;
        if ((i & 15u) == 0u && global_timer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_device_error, kDevErrTimeout);
            return;
        }
    }
}

// Lane t holds v[0..32) for row t: base + t * ld + [0, valid).  Staged with
// row t at stg + 128 t and its 16-byte chunk i at chunk i ^ (t % 8) (no bank
// conflicts either way); written 4 rows an instruction, 8 lanes a row.
__device__ __forceinline__ void warp_store_f32x32(uint32_t stg, float* base, long long ld, int nrows,
                                                  const uint32_t (&v)[32], int valid, int lane) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
        sts_v4(stg + lane * 128 + ((static_cast<uint32_t>(i) ^ (lane & 7)) << 4), v[4 * i],
               v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    __syncwarp();
    const int j = lane & 7, c = 4 * j;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        const int r = 4 * it + (lane >> 3);
        const uint4 x = lds_v4(stg + r * 128 + ((static_cast<uint32_t>(j) ^ (r & 7)) << 4));
        if (r < nrows) {
            float* d = base + r * ld + c;
            if (c + 4 <= valid) {
                *reinterpret_cast<uint4*>(d) = x;
            } else {
                if (c < valid) d[0] = __uint_as_float(x.x);
                if (c + 1 < valid) d[1] = __uint_as_float(x.y);
                if (c + 2 < valid) d[2] = __uint_as_float(x.z);
            }
        }
    }
    __syncwarp();
}

// Lane t holds the packed pairs pk[0..16) (32 16-bit values) for row t:
// base + t * ld + [0, valid).  Staged with row t at stg + 64 t and its 16-byte
// chunk i at chunk i ^ ((t / 2) % 4); written 8 rows an instruction, 4 lanes a
// row.  The values are moved as 16-bit words, whatever their format.
__device__ __forceinline__ void warp_store_16x32(uint32_t stg, void* base, long long ld, int nrows,
                                                 const uint32_t (&pk)[16], int valid, int lane) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
        sts_v4(stg + lane * 64 + ((static_cast<uint32_t>(i) ^ ((lane >> 1) & 3)) << 4), pk[4 * i],
               pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    __syncwarp();
    const int j = lane & 3, c = 8 * j;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int r = 8 * it + (lane >> 2);
        const uint4 x = lds_v4(stg + r * 64 + ((static_cast<uint32_t>(j) ^ ((r >> 1) & 3)) << 4));
        if (r < nrows) {
            uint16_t* d = static_cast<uint16_t*>(base) + r * ld + c;
            if (c + 8 <= valid) {
                *reinterpret_cast<uint4*>(d) = x;
            } else {
                const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 7; ++e)
                    if (c + e < valid)
                        d[e] = static_cast<uint16_t>((e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu));
            }
        }
    }
    __syncwarp();
}

// ============================================================================
// K1: column-split gate/up projection with the activation fused.
//   SwiGLU: H[:, j] = SiLU(X.W_gate[:, c+j]) * (X.W_up[:, c+j]), 128 columns a
//           tile; one N = 256 UMMA per K-step computes gate (TMEM columns
//           0-127) and up (128-255) from the same X tile.
//   GeLU:   H[:, j] = GeLU(X.A[:, c+j]), 256 columns a tile.
// "Tensor Parallelism: Splitting the Math", steps 2-3: each shard's hidden
// columns need only X and its own columns of A.
template <int ACT>  // 0 = GeLU, 1 = SwiGLU
struct FwdHidden {
    struct Params {
        CUtensorMap tmX;  // X [n][d], box {64, 128}
        CUtensorMap tmG;  // W_gate / A [d][f], box {64, 64}
        CUtensorMap tmU;  // W_up [d][f], box {64, 64} (SwiGLU)
        SegGeom g;
        int d;            // contraction (d_model)
        int width;        // hidden columns per segment in this launch
        __nv_bfloat16* H; // [num_segs * seg_rows][width]
        long long ldh;
    };
    static constexpr const char* kName = ACT == 1 ? "fwd_hidden_swiglu" : "fwd_hidden_gelu";
    static constexpr int kBK = 64;
    static constexpr int kOut = ACT == 1 ? 128 : 256;
    static constexpr int kABytes = 128 * kBK * 2;
    static constexpr int kBBytes = 256 * kBK * 2;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = 4;
    static constexpr int kAccCols = 256, kAccBufs = 2, kTmemCols = 512;
    static constexpr uint32_t kIdesc = make_idesc_bf16(128, 256, false, true);
    struct Tile {
        int s, mi, nj;
    };
    __host__ __device__ static int ntiles_n(const Params& p) { return (p.width + kOut - 1) / kOut; }
    __host__ __device__ static int num_tiles(const Params& p) {
        return p.g.num_segs * p.g.mtiles() * ntiles_n(p);
    }
    // segment-major, then output slab, then row tile (row tiles fastest): one
    // sequence segment's rows and weight shard at a time stay in L2
    __device__ static Tile tile(const Params& p, int t) {
        const int mt = p.g.mtiles(), per_seg = mt * ntiles_n(p);
        const int s = t / per_seg, r = t - s * per_seg;
        return Tile{s, r % mt, r / mt};
    }
    __device__ static int num_kb(const Params& p, const Tile&) { return (p.d + kBK - 1) / kBK; }
    __device__ static void prefetch(const Params& p) {
        tma_prefetch_desc(&p.tmX);
        tma_prefetch_desc(&p.tmG);
        if (ACT == 1) tma_prefetch_desc(&p.tmU);
    }
    __device__ static uint32_t load_bytes(const Params&, const Tile&, int) { return kStageBytes; }
    __device__ static void load(const Params& p, const Tile& ti, int kb, uint32_t st, uint32_t bar) {
        const int k0 = kb * kBK;
        tma_load_2d(st, &p.tmX, bar, k0, (p.g.seg_begin + ti.s) * p.g.seg_rows + ti.mi * 128);
        const int c = p.g.shard_col(ti.s) + ti.nj * kOut;
        const uint32_t b = st + kABytes;
        if (ACT == 1) {
            tma_load_2d(b, &p.tmG, bar, c, k0);
            tma_load_2d(b + 8192, &p.tmG, bar, c + 64, k0);
            tma_load_2d(b + 16384, &p.tmU, bar, c, k0);
            tma_load_2d(b + 24576, &p.tmU, bar, c + 64, k0);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) tma_load_2d(b + 8192 * i, &p.tmG, bar, c + 64 * i, k0);
        }
    }
    __device__ static void mma(const Tile&, int kb, uint32_t st, uint32_t acc) {
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t a = make_smem_desc(st + 32 * kk, 16, 1024, kLayoutSW128);
            const uint64_t b = make_smem_desc(st + kABytes + 2048 * kk, 8192, 1024, kLayoutSW128);
            umma_bf16(acc, a, b, kIdesc, (kb | kk) != 0 ? 1u : 0u);
        }
    }
    __device__ static void epilogue(const Params& p, const Tile& ti, uint32_t acc, int q, int lane,
                                    uint32_t stg) {
        const int wr0 = ti.mi * 128 + q * 32;  // the warp's first tile row
        const int nrows = min(32, p.g.seg_rows - wr0);
        __nv_bfloat16* hbase = p.H + static_cast<long long>(ti.s * p.g.seg_rows + wr0) * p.ldh;
        const uint32_t t0 = acc + (static_cast<uint32_t>(q * 32) << 16);
        if (ACT == 1) {
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t g[32], u[32], pk[16];
                tmem_ld_32x32b_x32(t0 + 32 * cc, g);
                tmem_ld_32x32b_x32(t0 + 128 + 32 * cc, u);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float h0 = silu_f(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
                    const float h1 =
                        silu_f(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
                    pk[i] = pack_bf16x2(h0, h1);
                }
                const int c0 = ti.nj * 128 + 32 * cc;
                if (c0 < p.width) warp_store_16x32(stg, hbase + c0, p.ldh, nrows, pk, p.width - c0, lane);
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
                const int c0 = ti.nj * 256 + 32 * cc;
                if (c0 < p.width) warp_store_16x32(stg, hbase + c0, p.ldh, nrows, pk, p.width - c0, lane);
            }
        }
    }
};

// ============================================================================
// K2 / K5: row-split down projection with the partial output added into an
// fp32 accumulator in place ("Tensor Parallelism: Splitting the Math", steps
// 4-6: B split by rows to match A's columns, partial outputs summed -- here a
// local read-modify-write in shard order instead of an all-reduce).
//   out[rows][0..n_out) (+)= sum over K-segments of A_seg . B_seg
// A is K-major (hidden activations, [rows][kdim]); B is MN-major (W_down
// [f][d], forward) or K-major (W_gate / W_up [d][f], input gradient).
// Modes: 0 store fp32, 1 add into fp32, 2 bf16(acc + tile) to out, 3 bf16(tile),
// 4 fp16(tile) to out (magnitudes above 65504 saturate and raise kDevErrRange).
// This struct holds the launch parameters and the per-row epilogue; the
// paired kernel (DownAccumPair in pipeline2.cuh) does the loads and MMAs.
template <bool B_MN, int NSEG>
struct DownAccum {
    struct Params {
        CUtensorMap tmA0, tmB0, tmA1, tmB1;
        SegGeom g;        // shard_col(s): hidden index base of segment s in B
        int kdim;         // hidden columns per K-segment
        int n_out;        // output columns
        int mode;
        int rot_P;        // > 0 (paired kernel): K covers all rot_P shards of g.fs columns,
                          // segment s starting at shard (seg_begin + s) mod rot_P
        float* acc;       // [rows][n_out] fp32 accumulator (global rows)
        long long ldacc;
        __nv_bfloat16* out;  // [rows][n_out] bf16 (global rows)
        long long ldo;
        // Tail split (paired kernel, mode 3 only): the tiles from split_from on
        // -- fewer than half a wave -- each run as two halves of their K loop
        // on two pairs; the first half leaves its fp32 sum in `part` and raises
        // one flag per epilogue warp, the second adds it before rounding.
        // split_from == 0: no split.
        int split_from;
        float* part;  // [split tiles][256][256] fp32
        int* flags;   // [split tiles][8], zeroed before the launch
    };
    static constexpr const char* kName =
        B_MN ? "down_accum_fwd" : (NSEG == 2 ? "dgrad_accum_swiglu" : "dgrad_accum_gelu");
    __device__ static void prefetch(const Params& p) {
        tma_prefetch_desc(&p.tmA0);
        tma_prefetch_desc(&p.tmB0);
        if (NSEG > 1) {
            tma_prefetch_desc(&p.tmA1);
            tma_prefetch_desc(&p.tmB1);
        }
    }
    // A warp's 32 accumulator rows (tile rows wr0 .. wr0 + 31 of segment s,
    // this thread's row wr0 + lane) over NCHUNK x 32 columns starting at output
    // column col0, applied in the launch's mode.  The plain stores (modes 0, 3,
    // 4) go through the warp's staging buffer; the read-modify-write modes
    // (1, 2) keep one row a thread.
    template <int NCHUNK>
    __device__ static void store_rows(const Params& p, int s, int wr0, int lane, int col0,
                                      uint32_t t0, uint32_t stg) {
        const int rl = wr0 + lane;
        const bool row_ok = rl < p.g.seg_rows;
        const int nrows = min(32, p.g.seg_rows - wr0);
        const long long row0 = static_cast<long long>(p.g.seg_begin + s) * p.g.seg_rows + wr0;
        const long long row = row0 + lane;
#pragma unroll 1
        for (int cc = 0; cc < NCHUNK; ++cc) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(t0 + 32 * cc, v);
            tmem_ld_wait();
            const int c0 = col0 + 32 * cc;
            const int valid = p.n_out - c0;
            if (valid <= 0) continue;  // the same for the whole warp
            if (p.mode == 0) {
                warp_store_f32x32(stg, p.acc + row0 * p.ldacc + c0, p.ldacc, nrows, v, valid, lane);
                continue;
            }
            if (p.mode == 3 || p.mode == 4) {
                uint32_t pk[16];
                if (p.mode == 3) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                } else {
                    bool big = false;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float x0 = __uint_as_float(v[2 * i]), x1 = __uint_as_float(v[2 * i + 1]);
                        big |= row_ok && (fabsf(x0) > 65504.f || fabsf(x1) > 65504.f);
                        pk[i] = pack_f16x2_sat(x0, x1);
                    }
                    if (big) atomicOr(&g_device_error, kDevErrRange);
                }
                warp_store_16x32(stg, p.out + row0 * p.ldo + c0, p.ldo, nrows, pk, valid, lane);
                continue;
            }
            if (!row_ok) continue;
            if (p.mode == 1) {
                float* a = p.acc + row * p.ldacc + c0;
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
            } else {  // mode 2: bf16(acc + tile)
                uint32_t pk[16];
                {
                    const float* a = p.acc + row * p.ldacc + c0;
                    if (valid >= 32) {
                        const float4* a4 = reinterpret_cast<const float4*>(a);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float4 o = a4[i];
                            pk[2 * i] = pack_bf16x2(o.x + __uint_as_float(v[4 * i]),
                                                    o.y + __uint_as_float(v[4 * i + 1]));
                            pk[2 * i + 1] = pack_bf16x2(o.z + __uint_as_float(v[4 * i + 2]),
                                                        o.w + __uint_as_float(v[4 * i + 3]));
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float x0 = (2 * i < valid ? a[2 * i] : 0.f) + __uint_as_float(v[2 * i]);
                            const float x1 = (2 * i + 1 < valid ? a[2 * i + 1] : 0.f) +
                                             __uint_as_float(v[2 * i + 1]);
                            pk[i] = pack_bf16x2(x0, x1);
                        }
                    }
                }
                store_bf16x32(p.out + row * p.ldo + c0, pk, valid);
            }
        }
    }
};

// ============================================================================
// K4: weight gradients, contraction over tokens.  Both operands MN-major.
//   out[r][c] = sum_tok A[tok][a_col0 + r] * B[tok][b_col0 + c]
// SPLIT: B is two 128-column sources (dG | dU) written to out0 | out1
// (dW_gate, dW_up share the X operand); otherwise one source of NCOLS.
// This struct holds the launch parameters and the per-row epilogue; the
// paired kernel (WgradPair in bwd_pair.cuh) does the loads and MMAs.
template <int NCOLS, bool SPLIT>
struct Wgrad {
    struct Params {
        CUtensorMap tmA, tmB0, tmB1;  // [ntok][*] bf16, box {64, 64}
        int ntok;
        int m_valid, n_valid;         // rows / columns of the output block
        int a_col0, b_col0;
        float* out0;
        float* out1;
        long long ldo;
        int out_row0, out_col0;
    };
    static constexpr const char* kName =
        SPLIT ? "wgrad_gate_up" : (NCOLS == 256 ? "wgrad_down" : "wgrad_gelu_a");
    static constexpr int kTileCols = SPLIT ? NCOLS / 2 : NCOLS;
    struct Tile {
        int mi, nj;  // 128-row block of the output, NCOLS-column block
    };
    __device__ static void prefetch(const Params& p) {
        tma_prefetch_desc(&p.tmA);
        tma_prefetch_desc(&p.tmB0);
        if (SPLIT) tma_prefetch_desc(&p.tmB1);
    }
    __device__ static void epilogue(const Params& p, const Tile& ti, uint32_t acc, int q, int lane,
                                    uint32_t stg) {
        const int wr0 = ti.mi * 128 + q * 32;  // the warp's first output row
        const int nrows = min(32, p.m_valid - wr0);
        const long long row0 = static_cast<long long>(p.out_row0 + wr0);
        const uint32_t t0 = acc + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
        for (int cc = 0; cc < NCOLS / 32; ++cc) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(t0 + 32 * cc, v);
            tmem_ld_wait();
            const int which = SPLIT ? cc / (NCOLS / 64) : 0;
            const int cl = ti.nj * kTileCols + 32 * (SPLIT ? cc % (NCOLS / 64) : cc);
            float* o = which ? p.out1 : p.out0;
            if (cl < p.n_valid)
                warp_store_f32x32(stg, o + row0 * p.ldo + p.out_col0 + cl, p.ldo, nrows, v,
                                  p.n_valid - cl, lane);
        }
    }
};

}  // namespace tspmlp
