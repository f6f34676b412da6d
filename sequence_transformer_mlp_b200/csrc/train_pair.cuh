// train_pair.cuh -- the training forward that keeps what the backward needs,
// and the backward's first GEMM that reads it.
//
// The recompute backward (bwd_pair.cuh) runs the gate/up projection a second
// time to get G and U back.  Here the forward's gate/up epilogue, which has G
// and U in tensor memory anyway, also writes the activation's derivative
// factors, rounded to bf16 like the other saved activation H, and the dH
// GEMM's epilogue turns dH into dG (and dU) with them directly:
//   SwiGLU: S1 = SiLU(G),  S2 = U SiLU'(G)   dU = dH S1,  dG = dH S2
//   GeLU:   S1 = GeLU'(Z)                     dG = dH S1
// with SiLU'(g) = s (1 + g (1 - s)), s = sigmoid(g), GeLU'(z) = Phi(z) +
// z phi(z) -- the derivatives of the forward definition, evaluated in fp32
// by the recompute backward's own helpers (bwd_pair.cuh, every rounding
// explicit) and rounded to bf16 there too, so dG and dU come out bit for bit
// the same.  dH itself is never stored.
//
// The factors are private to this pair, so their layout follows the
// epilogues' access, where a thread owns a row and a warp 32 consecutive rows:
// the pair of factors (r, c), (r, c + 1) (c even) is one bf16x2 word, at word
// ((r / 32) * ld / 2 + c / 2) * 32 + r % 32 -- each 32-row block interleaved
// by column pairs.  A warp then reads or writes two columns of its 32 rows as
// 128 contiguous bytes, instead of 32 rows' 4-byte pieces.
#pragma once

#include "bwd_pair.cuh"

namespace tspmlp {

// ============================================================================
// Gate/up projection (as FwdHiddenPair) whose epilogue also keeps S1 (S2).
template <int ACT>
struct FwdHiddenSaveParams : FwdHidden<ACT>::Params {
    uint32_t* S1;  // bf16x2 words, 32-row blocks of ldh columns, interleaved by column pairs
    uint32_t* S2;  // (SwiGLU)
};

// Word of the factor pair (r, c), (r, c + 1), c even, in the 32-row-block
// layout with ld (even) columns.
__device__ __forceinline__ long long factor_word(int r, int c, long long ld) {
    return (static_cast<long long>(r >> 5) * (ld >> 1) + (c >> 1)) * 32 + (r & 31);
}

template <int ACT>
struct FwdHiddenSavePair : FwdHiddenPair<ACT> {
    using Base = FwdHiddenPair<ACT>;
    using Params = FwdHiddenSaveParams<ACT>;
    using Tile = typename Base::Tile;
    static constexpr const char* kName = ACT == 1 ? "fwd_hidden_swiglu_save" : "fwd_hidden_gelu_save";

    // the thread's 32 consecutive factors of one row (fp32 bits), rounded to
    // bf16 in pairs: a column pair 32 words apart
    __device__ static void store_factors(uint32_t* dst, const uint32_t (&v)[32], int valid) {
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (2 * i < valid)
                dst[32 * i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
    }

    __device__ static void epilogue(const Params& p, const Tile& ti, uint32_t rank, uint32_t acc,
                                    int q, int lane, uint32_t stg) {
        const int wr0 = (2 * ti.mi + static_cast<int>(rank)) * 128 + q * 32;  // warp's first row
        const int rl = wr0 + lane;
        const bool row_ok = rl < p.g.seg_rows;
        const int nrows = min(32, p.g.seg_rows - wr0);
        const int r = ti.s * p.g.seg_rows + rl;
        const long long off0 = static_cast<long long>(ti.s * p.g.seg_rows + wr0) * p.ldh;
        const uint32_t t0 = acc + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
        for (int cc = 0; cc < Base::kOut / 32; ++cc) {
            const int c0 = ti.nj * Base::kOut + 32 * cc;
            const int valid = p.width - c0;
            uint32_t g[32];
            tmem_ld_32x32b_x32(t0 + 32 * cc, g);
            if (ACT == 1) {
                uint32_t u[32];
                tmem_ld_32x32b_x32(t0 + 128 + 32 * cc, u);
                tmem_ld_wait();
                if (valid <= 0) continue;  // the same for the whole warp
                uint32_t pk[16], s1[32], s2[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float gv = __uint_as_float(g[i]), uv = __uint_as_float(u[i]);
                    const float sg = sigmoid_rn(gv);
                    s1[i] = __float_as_uint(__fmul_rn(gv, sg));
                    s2[i] = __float_as_uint(swiglu_gate_factor(gv, uv, sg));
                    g[i] = __float_as_uint(silu_f(gv) * uv);  // H, as the inference forward
                }
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(g[2 * i]), __uint_as_float(g[2 * i + 1]));
                warp_store_16x32(stg, p.H + off0 + c0, p.ldh, nrows, pk, valid, lane);
                if (row_ok) {
                    store_factors(p.S1 + factor_word(r, c0, p.ldh), s1, valid);
                    store_factors(p.S2 + factor_word(r, c0, p.ldh), s2, valid);
                }
            } else {
                tmem_ld_wait();
                if (valid <= 0) continue;
                uint32_t pk[16], s1[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float z = __uint_as_float(g[i]);
                    s1[i] = __float_as_uint(gelu_grad_rn(z, gelu_cdf_rn(z)));
                    g[i] = __float_as_uint(gelu_f(z));
                }
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(g[2 * i]), __uint_as_float(g[2 * i + 1]));
                warp_store_16x32(stg, p.H + off0 + c0, p.ldh, nrows, pk, valid, lane);
                if (row_ok) store_factors(p.S1 + factor_word(r, c0, p.ldh), s1, valid);
            }
        }
    }
};

// ============================================================================
// dH = dY . W_down[c..]^T (as DhPair), whose epilogue applies the saved
// factors and writes dG (dU) in bf16 instead of storing dH.
struct DhFactorParams : DhParams {
    const uint32_t* S1;  // saved factors (bf16x2 words, 32-row-block layout) from the chunk's first column
    const uint32_t* S2;  // (SwiGLU)
    long long lds;       // columns of the saved layout (d_ff, even)
    __nv_bfloat16* dG;  // [n][width] at pitch ld
    __nv_bfloat16* dU;  // [n][width] (SwiGLU)
};

template <int ACT>
struct DhFactorPair : DhPair<ACT> {
    using Base = DhPair<ACT>;
    using Params = DhFactorParams;
    using Tile = typename Base::Tile;
    static constexpr const char* kName = ACT == 1 ? "bwd_dh_factor_swiglu" : "bwd_dh_factor_gelu";

    // the thread's 32 consecutive factors of one row (a column pair 32 words
    // apart), widened to float; zero from the first pair beyond valid
    __device__ static void load_factors(const uint32_t* src, int valid, float (&v)[32]) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t w = 2 * i < valid ? src[32 * i] : 0u;
            v[2 * i] = __uint_as_float(w << 16);
            v[2 * i + 1] = __uint_as_float(w & 0xffff0000u);
        }
    }

    __device__ static void epilogue(const Params& p, const Tile& ti, uint32_t rank, uint32_t acc,
                                    int q, int lane, uint32_t stg) {
        const int wr0 = ti.mi * 256 + static_cast<int>(rank) * 128 + q * 32;  // warp's first row
        const int row = wr0 + lane;
        const bool row_ok = row < p.n;
        const int nrows = min(32, p.n - wr0);
        const long long off0 = static_cast<long long>(wr0) * p.ld;
        const uint32_t t0 = acc + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
            const int c0 = ti.nj * 256 + 32 * cc;
            const int valid = p.width - c0;
            const bool live = row_ok && valid > 0;
            float s1[32], s2[32];
            if (live) {
                const long long so = factor_word(row, c0, p.lds);
                load_factors(p.S1 + so, valid, s1);
                if (ACT == 1) load_factors(p.S2 + so, valid, s2);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) s1[i] = s2[i] = 0.0f;
            }
            uint32_t dh[32], pk[16];
            tmem_ld_32x32b_x32(t0 + 32 * cc, dh);
            tmem_ld_wait();
            if (valid <= 0) continue;  // the same for the whole warp
            if (ACT == 1) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(dh[2 * i]) * s1[2 * i],
                                        __uint_as_float(dh[2 * i + 1]) * s1[2 * i + 1]);
                warp_store_16x32(stg, p.dU + off0 + c0, p.ld, nrows, pk, valid, lane);
            }
            const float(&sg)[32] = ACT == 1 ? s2 : s1;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(__uint_as_float(dh[2 * i]) * sg[2 * i],
                                    __uint_as_float(dh[2 * i + 1]) * sg[2 * i + 1]);
            warp_store_16x32(stg, p.dG + off0 + c0, p.ld, nrows, pk, valid, lane);
        }
    }
};

}  // namespace tspmlp
