// grad_pair.cuh -- the last two GEMMs of the SwiGLU backward in one
// persistent launch: the input gradient dX = dG.W_gate^T + dU.W_up^T
// (DownAccumPair<false, 2, 256>) and the gate/up weight gradients
// [dW_gate | dW_up] = X^T [dG | dU] (as WgradPair<256, true>, with 128-deep
// k-blocks so both kinds of tile fill the same 64 KB stages).
//
// Why one launch: the input gradient has few, long tiles (256 of them, K =
// 2 d_ff), which leave the last of their 3.46 waves half empty; the weight
// gradients have many short ones (1792, K = tokens).  Each pair takes its
// round-robin share of the long tiles first; the short ones go out in index
// order, first to the pairs with one long tile fewer, so that every pair's
// total work (in k-blocks) is the same within one short tile.  The pair-level arithmetic of each tile is that of
// the separate kernels, in the same order, so the results are bit-identical.
#pragma once

#include "train_pair.cuh"

namespace tspmlp {

struct DgradWgradParams {
    DownAccum<false, 2>::Params d;  // input gradient
    Wgrad<256, true>::Params w;     // gate/up weight gradients (tensor maps with 128-row boxes)
};

struct DgradWgradPair {
    using D = DownAccumPair<false, 2, 256>;
    using W = Wgrad<256, true>;
    using Params = DgradWgradParams;
    static constexpr const char* kName = "dgrad_wgrad_swiglu";
    static constexpr int kBK = 128;
    static constexpr int kABytes = 128 * kBK * 2;
    static constexpr int kStageBytes = D::kStageBytes;
    static_assert(kStageBytes == kABytes + 128 * kBK * 2, "both kinds stage 64 KB a k-block");
    static constexpr int kStages = D::kStages;
    static constexpr int kAccCols = 256, kAccBufs = 2;
    static constexpr int kWCols = W::kTileCols;  // 128 columns of dW_gate and of dW_up a tile
    static constexpr uint32_t kIdescW = make_idesc_bf16(256, 256, true, true);

    enum : int { kDgrad = 0, kWgrad = 1, kNone = 2 };
    struct Tile {
        int kind;
        D::Tile d;
        int wmi, wnj;
    };

    __host__ __device__ static int n_dgrad(const Params& p) { return D::num_tiles(p.d); }
    __host__ __device__ static int w_mtiles(const Params& p) { return (p.w.m_valid + 255) / 256; }
    __host__ __device__ static int w_ntiles(const Params& p) { return (p.w.n_valid + kWCols - 1) / kWCols; }
    __host__ __device__ static int n_wgrad(const Params& p) { return w_mtiles(p) * w_ntiles(p); }
    // an input-gradient tile's k-blocks, counted exactly as D::num_kb counts
    // them (two K segments of ceil(kdim / D::kBK) blocks), for any chunk width
    static_assert(D::kBK == kBK, "both kinds of tile use the same k-block depth");
    __host__ __device__ static int kb_dgrad(const Params& p) { return 2 * ((p.d.kdim + D::kBK - 1) / D::kBK); }
    __host__ __device__ static int kb_wgrad(const Params& p) { return (p.w.ntok + kBK - 1) / kBK; }

    // Schedule over np pairs.  Pair q first runs input-gradient tiles q,
    // q + np, ... (dcount(q): one more for the first nd % np pairs).  The
    // weight-gradient tiles then go out in index order, so that the tiles in
    // flight at any time are neighbours and share their operand panels in L2:
    //   phase 1: while the first nd % np pairs finish their extra long tile,
    //            the others take tiles 0 .. n1-1 round-robin, about one long
    //            tile's worth (cd / cw) each;
    //   phase 2: every pair takes the rest round-robin.
    struct Split {
        int dq, dr;  // input-gradient tiles: dq each, one more for pairs < dr
        int nb;      // pairs in phase 1 (np - dr)
        int n1, n2;  // weight-gradient tiles of phase 1 and phase 2
    };
    __host__ __device__ static Split split(const Params& p, int np) {
        Split s;
        const int nd = n_dgrad(p), nw = n_wgrad(p), cd = kb_dgrad(p), cw = kb_wgrad(p);
        s.dq = nd / np;
        s.dr = nd % np;
        s.nb = np - s.dr;
        const int r1 = s.dr > 0 ? (cd + cw / 2) / (cw > 0 ? cw : 1) : 0;
        const long long n1 = static_cast<long long>(s.nb) * r1;
        s.n1 = static_cast<int>(n1 < nw ? n1 : nw);
        s.n2 = nw - s.n1;
        return s;
    }
    __host__ __device__ static int dcount(const Split& s, int q) { return s.dq + (q < s.dr ? 1 : 0); }
    __host__ __device__ static int count1(const Split& s, int q) {
        const int i = q - s.dr;
        return (i >= 0 && s.n1 > i) ? (s.n1 - 1 - i) / s.nb + 1 : 0;
    }
    __host__ __device__ static int count2(const Split& s, int np, int q) {
        return s.n2 > q ? (s.n2 - 1 - q) / np + 1 : 0;
    }
    // Tile slots the kernel walks: np x the largest pair's count (a pair's
    // slots past its own work are empty).  On the host, before the pair count
    // is known, the number of real tiles (enough to size the grid).
    __host__ __device__ static int num_tiles(const Params& p) {
#ifdef __CUDA_ARCH__
        const int np = static_cast<int>(num_clusters_x());
        const Split s = split(p, np);
        int mx = 0;
        for (int q = 0; q < np; ++q) {
            const int c = dcount(s, q) + count1(s, q) + count2(s, np, q);
            mx = c > mx ? c : mx;
        }
        return np * mx;
#else
        return n_dgrad(p) + n_wgrad(p);
#endif
    }
    __device__ static Tile tile(const Params& p, int t) {
        const int np = static_cast<int>(num_clusters_x());
        const int q = t % np, k = t / np;
        const Split s = split(p, np);
        Tile ti{};
        const int dc = dcount(s, q);
        if (k < dc) {
            ti.kind = kDgrad;
            ti.d = D::tile(p.d, q + k * np);
            return ti;
        }
        const int k1 = k - dc, c1 = count1(s, q);
        int wi;
        if (k1 < c1) {
            wi = (q - s.dr) + k1 * s.nb;
        } else if (k1 - c1 < count2(s, np, q)) {
            wi = s.n1 + q + (k1 - c1) * np;
        } else {
            ti.kind = kNone;
            return ti;
        }
        // the weight gradients' order: the index over the smaller block count
        // runs fastest (see WgradPair)
        ti.kind = kWgrad;
        const int mt = w_mtiles(p), nt = w_ntiles(p);
        if (mt <= nt) {
            ti.wmi = wi % mt;
            ti.wnj = wi / mt;
        } else {
            ti.wmi = wi / nt;
            ti.wnj = wi % nt;
        }
        return ti;
    }
    __device__ static int num_kb(const Params& p, const Tile& ti) {
        return ti.kind == kDgrad ? D::num_kb(p.d, ti.d) : (ti.kind == kWgrad ? kb_wgrad(p) : 0);
    }
    __device__ static void prefetch(const Params& p) {
        D::prefetch(p.d);
        W::prefetch(p.w);
    }
    __device__ static void load(const Params& p, const Tile& ti, int kb, uint32_t rank, uint32_t st,
                                uint32_t bar) {
        if (ti.kind == kDgrad) {
            D::load(p.d, ti.d, kb, rank, st, bar);
            return;
        }
        // weight gradients, both operands MN-major: {64 columns, 128 tokens} boxes
        const int k0 = kb * kBK;
        const int a = p.w.a_col0 + ti.wmi * 256 + static_cast<int>(rank) * 128;
        tma_load_2d_pair(st, &p.w.tmA, bar, a, k0);
        tma_load_2d_pair(st + 16384, &p.w.tmA, bar, a + 64, k0);
        const int c = p.w.b_col0 + ti.wnj * kWCols;
        const CUtensorMap* src = rank == 0 ? &p.w.tmB0 : &p.w.tmB1;
        tma_load_2d_pair(st + kABytes, src, bar, c, k0);
        tma_load_2d_pair(st + kABytes + 16384, src, bar, c + 64, k0);
    }
    __device__ static void mma(const Tile& ti, int kb, uint32_t st, uint32_t acc) {
        if (ti.kind == kDgrad) {
            D::mma(ti.d, kb, st, acc);
            return;
        }
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
            // MN-major: 2 KB a K16 step; the next 64-column box 16 KB on
            const uint64_t a = make_smem_desc(st + 2048 * kk, 16384, 1024, kLayoutSW128);
            const uint64_t b = make_smem_desc(st + kABytes + 2048 * kk, 16384, 1024, kLayoutSW128);
            umma_bf16_pair(acc, a, b, kIdescW, (kb | kk) != 0 ? 1u : 0u);
        }
    }
    __device__ static void epilogue(const Params& p, const Tile& ti, uint32_t rank, uint32_t acc,
                                    int q, int lane, uint32_t stg) {
        if (ti.kind == kDgrad) {
            D::epilogue(p.d, ti.d, rank, acc, q, lane, stg);
        } else if (ti.kind == kWgrad) {
            typename W::Tile t1{2 * ti.wmi + static_cast<int>(rank), ti.wnj};
            W::epilogue(p.w, t1, acc, q, lane, stg);
        }
    }
};

}  // namespace tspmlp
