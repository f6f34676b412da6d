// bwd_pair.cuh -- the backward's paired recipes for the pipeline of
// pipeline2.cuh: the weight gradients (WgradPair) and the hidden layer's
// backward as two GEMMs (BwdGateUpPair, DhPair).  The input gradient reuses
// DownAccumPair with K-major weights.
#pragma once

#include "pipeline2.cuh"

namespace tspmlp {

// Derivative factors of the activations, with every rounding written out (no
// multiply-add left for the compiler to fuse or not), so that the recompute
// backward here and the training forward (train_pair.cuh) get the same bits.
//   sigmoid(g) = 1 / (1 + exp(-g))
//   SiLU'(g) u = u s (1 + g (1 - s)),  s = sigmoid(g)
//   GeLU'(z)   = Phi(z) + z phi(z),  Phi(z) = (1 + erf(z / sqrt 2)) / 2,
//                phi(z) = exp(-z^2 / 2) / sqrt(2 pi)
__device__ __forceinline__ float sigmoid_rn(float g) {
    return __fdiv_rn(1.0f, __fadd_rn(1.0f, __expf(-g)));
}
__device__ __forceinline__ float swiglu_gate_factor(float g, float u, float s) {
    return __fmul_rn(__fmul_rn(u, s), __fmaf_rn(g, __fsub_rn(1.0f, s), 1.0f));
}
__device__ __forceinline__ float gelu_cdf_rn(float z) {
    return __fmul_rn(0.5f, __fadd_rn(1.0f, erff(__fmul_rn(z, 0.70710678118654752440f))));
}
__device__ __forceinline__ float gelu_grad_rn(float z, float cdf) {
    const float pdf = __fmul_rn(0.39894228040143267794f, __expf(__fmul_rn(__fmul_rn(-0.5f, z), z)));
    return __fmaf_rn(z, pdf, cdf);
}
// A factor as both backward paths use it: rounded to bf16 (nearest even, the
// rounding of pack_bf16x2, which stores the training forward's factors) and
// widened back to float.
__device__ __forceinline__ float bf16_round(float x) { return __uint_as_float(pack_bf16x2(x, 0.0f) << 16); }

// ============================================================================
// Paired weight gradients (see Wgrad): both operands MN-major, K = tokens.
// Tile = 256 output rows x NCOLS output columns; CTA r stages 128 of the rows
// (A) and NCOLS/2 of the columns (B).  SPLIT: CTA 0 stages dG, CTA 1 dU, so
// TMEM columns 0-127 hold dW_gate and 128-255 dW_up.
template <int NCOLS, bool SPLIT>
struct WgradPair {
    using Base = Wgrad<NCOLS, SPLIT>;
    using Params = typename Base::Params;
    static constexpr const char* kName = Base::kName;
    // 64-deep k-blocks (tokens): 128-deep ones measured the same within noise
    static constexpr int kBK = 64;
    static constexpr int kABytes = 128 * kBK * 2;
    static constexpr int kStageBytes = kABytes + (NCOLS / 2) * kBK * 2;
    static constexpr int kStages = kStageBytes <= 24576 ? 8 : 6;
    static constexpr int kAccCols = 256, kAccBufs = 2;
    static constexpr int kTileCols = Base::kTileCols;
    static constexpr uint32_t kIdesc = make_idesc_bf16(256, NCOLS, true, true);
    struct Tile {
        int mi, nj;
    };
    __host__ __device__ static int num_tiles(const Params& p) {
        return ((p.m_valid + 255) / 256) * ((p.n_valid + kTileCols - 1) / kTileCols);
    }
    // Both operands span all K = tokens, so a wave of concurrent tiles re-reads
    // every block of the operand whose index varies fastest.  That index runs
    // over the operand with fewer blocks (X or dY: n x d_model, which L2
    // holds), so the larger one (H, dG/dU: n x d_ff) streams from HBM once.
    __device__ static Tile tile(const Params& p, int t) {
        const int mt = (p.m_valid + 255) / 256;
        const int nt = (p.n_valid + kTileCols - 1) / kTileCols;
        if (mt <= nt) return Tile{t % mt, t / mt};
        return Tile{t / nt, t % nt};
    }
    __device__ static int num_kb(const Params& p, const Tile&) { return (p.ntok + kBK - 1) / kBK; }
    __device__ static void prefetch(const Params& p) { Base::prefetch(p); }
    __device__ static void load(const Params& p, const Tile& ti, int kb, uint32_t rank, uint32_t st,
                                uint32_t bar) {
        const int k0 = kb * kBK;
        const int a = p.a_col0 + ti.mi * 256 + static_cast<int>(rank) * 128;
        tma_load_2d_pair(st, &p.tmA, bar, a, k0);
        tma_load_2d_pair(st + 8192, &p.tmA, bar, a + 64, k0);
        const uint32_t b = st + kABytes;
        if (SPLIT) {
            const int c = p.b_col0 + ti.nj * kTileCols;
            const CUtensorMap* src = rank == 0 ? &p.tmB0 : &p.tmB1;
#pragma unroll
            for (int i = 0; i < NCOLS / 128; ++i) tma_load_2d_pair(b + 8192 * i, src, bar, c + 64 * i, k0);
        } else {
            const int c = p.b_col0 + ti.nj * NCOLS + static_cast<int>(rank) * (NCOLS / 2);
#pragma unroll
            for (int i = 0; i < NCOLS / 128; ++i) tma_load_2d_pair(b + 8192 * i, &p.tmB0, bar, c + 64 * i, k0);
        }
    }
    __device__ static void mma(const Tile&, int kb, uint32_t st, uint32_t acc) {
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
            // MN-major: 2 KB a K16 step; the next 64-column box 8 KB on
            const uint64_t a = make_smem_desc(st + 2048 * kk, 8192, 1024, kLayoutSW128);
            const uint64_t b = make_smem_desc(st + kABytes + 2048 * kk, 8192, 1024, kLayoutSW128);
            umma_bf16_pair(acc, a, b, kIdesc, (kb | kk) != 0 ? 1u : 0u);
        }
    }
    __device__ static void epilogue(const Params& p, const Tile& ti, uint32_t rank, uint32_t acc,
                                    int q, int lane, uint32_t stg) {
        typename Base::Tile t1{2 * ti.mi + static_cast<int>(rank), ti.nj};
        Base::epilogue(p, t1, acc, q, lane, stg);
    }
};

// ============================================================================
// Backward of the hidden layer as two double-buffered paired GEMMs.
//
// DhPair: dH = dY . W_down[c..]^T (K = d_model, both operands K-major); the
// epilogue stores dH in fp32 (the accumulator as it is).
// BwdGateUpPair: the recomputed gate/up projection (as FwdHiddenPair, K =
// d_model) whose epilogue reads dH and writes, per hidden unit,
//   SwiGLU: H = SiLU(G) U,  dU = dH SiLU(G),  dG = dH U SiLU'(G)   (bf16)
//   GeLU:   H = GeLU(G),    dG = dH GeLU'(G)                        (bf16)
// with SiLU'(g) = s (1 + g (1 - s)), s = sigmoid(g), and GeLU'(z) = Phi(z) +
// z phi(z): the derivatives of the forward definition (helpers above).  dH stays
// fp32; the factors SiLU(G), U SiLU'(G) and GeLU'(G) are rounded to bf16 before
// the products, as the training forward saves them (train_pair.cuh), and H,
// dG and dU are rounded to bf16.
struct DhParams {
    CUtensorMap tmDY;  // dY [n][d], box {64, 128}
    CUtensorMap tmD;   // W_down / B [f][d], box {64, 128} (K-major: rows are hidden units)
    int n, d, col_base, width;
    float* dH;         // [n][width] fp32
    long long ld;
};

template <int ACT>
struct DhPair {
    using Params = DhParams;
    static constexpr const char* kName = ACT == 1 ? "bwd_dh_swiglu" : "bwd_dh_gelu";
    // 64-deep k-blocks: 128-deep ones measured the same within noise
    static constexpr int kBK = 64;
    static constexpr int kABytes = 128 * kBK * 2;
    static constexpr int kStageBytes = kABytes + 128 * kBK * 2;
    static constexpr int kStages = 6;
    static constexpr int kAccCols = 256, kAccBufs = 2;
    static constexpr uint32_t kIdesc = make_idesc_bf16(256, 256, false, false);
    struct Tile {
        int mi, nj;
    };
    __host__ __device__ static int num_tiles(const Params& p) {
        return ((p.n + 255) / 256) * ((p.width + 255) / 256);
    }
    __device__ static Tile tile(const Params& p, int t) {
        const int mt = (p.n + 255) / 256;
        return Tile{t % mt, t / mt};
    }
    __device__ static int num_kb(const Params& p, const Tile&) { return (p.d + kBK - 1) / kBK; }
    __device__ static void prefetch(const Params& p) {
        tma_prefetch_desc(&p.tmDY);
        tma_prefetch_desc(&p.tmD);
    }
    __device__ static void load(const Params& p, const Tile& ti, int kb, uint32_t rank, uint32_t st,
                                uint32_t bar) {
        const int k0 = kb * kBK;
        tma_load_2d_pair(st, &p.tmDY, bar, k0, ti.mi * 256 + static_cast<int>(rank) * 128);
        tma_load_2d_pair(st + kABytes, &p.tmD, bar, k0,
                         p.col_base + ti.nj * 256 + static_cast<int>(rank) * 128);
    }
    __device__ static void mma(const Tile&, int kb, uint32_t st, uint32_t acc) {
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t a = make_smem_desc(st + 32 * kk, 16, 1024, kLayoutSW128);
            const uint64_t b = make_smem_desc(st + kABytes + 32 * kk, 16, 1024, kLayoutSW128);
            umma_bf16_pair(acc, a, b, kIdesc, (kb | kk) != 0 ? 1u : 0u);
        }
    }
    __device__ static void epilogue(const Params& p, const Tile& ti, uint32_t rank, uint32_t acc,
                                    int q, int lane, uint32_t stg) {
        const int wr0 = ti.mi * 256 + static_cast<int>(rank) * 128 + q * 32;  // warp's first row
        const int nrows = min(32, p.n - wr0);
        float* base = p.dH + static_cast<long long>(wr0) * p.ld;
        const uint32_t t0 = acc + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
            uint32_t dh[32];
            tmem_ld_32x32b_x32(t0 + 32 * cc, dh);
            tmem_ld_wait();
            const int c0 = ti.nj * 256 + 32 * cc;
            if (c0 < p.width) warp_store_f32x32(stg, base + c0, p.ld, nrows, dh, p.width - c0, lane);
        }
    }
};

struct BwdGateUpParams {
    CUtensorMap tmX;  // X [n][d], box {64, 128}
    CUtensorMap tmG;  // W_gate / A [d][f], box {64, 64}
    CUtensorMap tmU;  // W_up [d][f], box {64, 64} (SwiGLU)
    int n, d, col_base, width;
    const float* dH;     // [n][width] fp32, from DhPair
    __nv_bfloat16* H;    // [n][width]
    __nv_bfloat16* dG;   // [n][width]
    __nv_bfloat16* dU;   // [n][width] (SwiGLU)
    long long ld;
};

template <int ACT>
struct BwdGateUpPair {
    using Params = BwdGateUpParams;
    static constexpr const char* kName = ACT == 1 ? "bwd_gate_up_swiglu" : "bwd_gate_up_gelu";
    // 128-deep k-blocks as FwdHiddenPair
    static constexpr int kBK = 128;
    static constexpr int kOut = ACT == 1 ? 128 : 256;
    static constexpr int kABytes = 128 * kBK * 2;
    static constexpr int kStageBytes = kABytes + 128 * kBK * 2;
    static constexpr int kStages = 3;
    static constexpr int kAccCols = 256, kAccBufs = 2;
    static constexpr uint32_t kIdesc = make_idesc_bf16(256, 256, false, true);
    struct Tile {
        int mi, nj;
    };
    __host__ __device__ static int num_tiles(const Params& p) {
        return ((p.n + 255) / 256) * ((p.width + kOut - 1) / kOut);
    }
    __device__ static Tile tile(const Params& p, int t) {
        const int mt = (p.n + 255) / 256;
        return Tile{t % mt, t / mt};
    }
    __device__ static int num_kb(const Params& p, const Tile&) { return (p.d + kBK - 1) / kBK; }
    __device__ static void prefetch(const Params& p) {
        tma_prefetch_desc(&p.tmX);
        tma_prefetch_desc(&p.tmG);
        if (ACT == 1) tma_prefetch_desc(&p.tmU);
    }
    __device__ static void load(const Params& p, const Tile& ti, int kb, uint32_t rank, uint32_t st,
                                uint32_t bar) {
        const int k0 = kb * kBK;
        const int xr = ti.mi * 256 + static_cast<int>(rank) * 128;
        tma_load_2d_pair(st, &p.tmX, bar, k0, xr);
        tma_load_2d_pair(st + 16384, &p.tmX, bar, k0 + 64, xr);
        const int c = p.col_base + ti.nj * kOut;
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
            const uint64_t a =
                make_smem_desc(st + (kk >> 2) * 16384 + 32 * (kk & 3), 16, 1024, kLayoutSW128);
            const uint64_t b = make_smem_desc(st + kABytes + 2048 * kk, 16384, 1024, kLayoutSW128);
            umma_bf16_pair(acc, a, b, kIdesc, (kb | kk) != 0 ? 1u : 0u);
        }
    }
    // 32 fp32 values of dH from src[0..valid) (zero beyond)
    __device__ static void load_dh(const float* src, int valid, float (&v)[32]) {
        if (valid >= 32) {
            const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 x = s4[i];
                v[4 * i] = x.x;
                v[4 * i + 1] = x.y;
                v[4 * i + 2] = x.z;
                v[4 * i + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = i < valid ? src[i] : 0.0f;
        }
    }
    __device__ static void epilogue(const Params& p, const Tile& ti, uint32_t rank, uint32_t acc,
                                    int q, int lane, uint32_t stg) {
        const int wr0 = ti.mi * 256 + static_cast<int>(rank) * 128 + q * 32;  // warp's first row
        const int row = wr0 + lane;
        const bool row_ok = row < p.n;
        const int nrows = min(32, p.n - wr0);
        const long long off = static_cast<long long>(row) * p.ld;
        const long long off0 = static_cast<long long>(wr0) * p.ld;
        const uint32_t t0 = acc + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
        for (int cc = 0; cc < (ACT == 1 ? 4 : 8); ++cc) {
            const int c0 = ti.nj * kOut + 32 * cc;
            const int valid = p.width - c0;
            const bool live = row_ok && valid > 0;
            float dh[32];
            if (live) {
                load_dh(p.dH + off + c0, valid, dh);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) dh[i] = 0.0f;
            }
            uint32_t g[32], ph[16], pg[16], pu[16];
            tmem_ld_32x32b_x32(t0 + 32 * cc, g);
            if (ACT == 1) {
                uint32_t u[32];
                tmem_ld_32x32b_x32(t0 + 128 + 32 * cc, u);
                tmem_ld_wait();
                if (valid <= 0) continue;  // the same for the whole warp
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float h[2], dgv[2], duv[2];
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const float gv = __uint_as_float(g[2 * i + j]), uv = __uint_as_float(u[2 * i + j]);
                        const float sg = sigmoid_rn(gv);
                        const float si = __fmul_rn(gv, sg);
                        h[j] = si * uv;
                        // the factors rounded to bf16, as the training forward saves them
                        duv[j] = dh[2 * i + j] * bf16_round(si);
                        dgv[j] = dh[2 * i + j] * bf16_round(swiglu_gate_factor(gv, uv, sg));
                    }
                    ph[i] = pack_bf16x2(h[0], h[1]);
                    pg[i] = pack_bf16x2(dgv[0], dgv[1]);
                    pu[i] = pack_bf16x2(duv[0], duv[1]);
                }
                warp_store_16x32(stg, p.dU + off0 + c0, p.ld, nrows, pu, valid, lane);
            } else {
                tmem_ld_wait();
                if (valid <= 0) continue;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float h[2], dgv[2];
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const float z = __uint_as_float(g[2 * i + j]);
                        const float cdf = gelu_cdf_rn(z);
                        h[j] = z * cdf;
                        dgv[j] = dh[2 * i + j] * bf16_round(gelu_grad_rn(z, cdf));
                    }
                    ph[i] = pack_bf16x2(h[0], h[1]);
                    pg[i] = pack_bf16x2(dgv[0], dgv[1]);
                }
            }
            warp_store_16x32(stg, p.H + off0 + c0, p.ld, nrows, ph, valid, lane);
            warp_store_16x32(stg, p.dG + off0 + c0, p.ld, nrows, pg, valid, lane);
        }
    }
};

}  // namespace tspmlp
