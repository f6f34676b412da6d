// Host-side check of the fused forward kernel's tile list (fused.cuh):
// for many geometries, the list visits every gate/up and down tile exactly
// once, and every dependency a producer waits for (down tile -> all gate/up
// tiles of its row block; gate/up tile -> all down tiles of the row block R
// earlier, whose H-ring slot it reuses) sits earlier in the list.  Tiles are
// handed out in list order, so this is what makes every wait end.
#include <algorithm>
#include <cstdio>
#include <vector>

#include "../sequence_transformer_mlp_b200/csrc/fused2.cuh"

using tspmlp::FusedFwdParams;
using tspmlp::FusedTile;

static int check(int MB, int nJ, int nC, int GM, int head, int R) {
    FusedFwdParams p{};
    p.MB = MB;
    p.nJ = nJ;
    p.nC = nC;
    p.GM = GM;
    p.G = (MB + GM - 1) / GM;
    p.head = head;
    p.R = R;
    p.total = MB * (nJ + nC);
    std::vector<int> pos_up(MB * nJ, -1), pos_dn(MB * nC, -1);
    for (int t = 0; t < p.total; ++t) {
        const FusedTile ti = tspmlp::fused_tile(p, t);
        if (ti.mb < 0 || ti.mb >= MB) return printf("bad row block %d at %d\n", ti.mb, t), 1;
        if (ti.type == tspmlp::kFusedGateUp) {
            if (ti.j < 0 || ti.j >= nJ || pos_up[ti.mb * nJ + ti.j] >= 0)
                return printf("bad/dup gate-up tile (%d,%d) at %d\n", ti.mb, ti.j, t), 1;
            pos_up[ti.mb * nJ + ti.j] = t;
        } else {
            if (ti.j < 0 || ti.j >= nC || pos_dn[ti.mb * nC + ti.j] >= 0)
                return printf("bad/dup down tile (%d,%d) at %d\n", ti.mb, ti.j, t), 1;
            pos_dn[ti.mb * nC + ti.j] = t;
        }
    }
    for (int m = 0; m < MB; ++m) {
        int last_up = -1, first_dn = p.total, last_dn = -1;
        for (int j = 0; j < nJ; ++j) last_up = pos_up[m * nJ + j] > last_up ? pos_up[m * nJ + j] : last_up;
        for (int c = 0; c < nC; ++c) {
            const int q = pos_dn[m * nC + c];
            first_dn = q < first_dn ? q : first_dn;
            last_dn = q > last_dn ? q : last_dn;
        }
        if (last_up < 0 || last_dn < 0) return printf("missing tiles of row block %d\n", m), 1;
        if (last_up >= first_dn) return printf("down before gate/up in row block %d\n", m), 1;
        if (m + R < MB)
            for (int j = 0; j < nJ; ++j)
                if (pos_up[(m + R) * nJ + j] <= last_dn)
                    return printf("slot reuse before row block %d is read\n", m), 1;
    }
    return 0;
}

// The one-launch pass schedule (fused2.cuh): chunk c's down tiles of row pair
// m after all its gate/up tiles and after all down tiles of chunk c-1 (the
// accumulator), and chunk c's gate/up tiles after all down tiles of chunk c-2
// (H is double-buffered).
template <int KOUT>
static int check_passes(int MP, int C, int nN, int head, const int* widths) {
    tspmlp::FusedPassesParams p{};
    p.MP = MP;
    p.C = C;
    p.nN = nN;
    p.head = head;
    int total = 0;
    for (int c = 0; c < C; ++c) {
        p.cw[c] = widths[c];
        total += tspmlp::pass_nj<KOUT>(p, c) * MP + nN * MP;
    }
    p.total = total;
    // first/last list positions per (type, chunk, row pair), and a full count
    std::vector<int> first(2 * C * MP, total), last(2 * C * MP, -1), cnt(2 * C * MP, 0);
    std::vector<int> seen_up, seen_dn;
    for (int c = 0; c < C; ++c) {
        seen_up.push_back(0);
        seen_dn.push_back(0);
    }
    std::vector<char> hit;
    int maxj = 0;
    for (int c = 0; c < C; ++c) maxj = std::max(maxj, tspmlp::pass_nj<KOUT>(p, c));
    maxj = std::max(maxj, nN);
    hit.assign(static_cast<size_t>(2) * C * MP * maxj, 0);
    for (int t = 0; t < total; ++t) {
        const tspmlp::PassTile ti = tspmlp::pass_tile<KOUT>(p, t);
        if (ti.c < 0 || ti.c >= C || ti.m < 0 || ti.m >= MP) return printf("bad tile at %d\n", t), 1;
        const int lim = ti.type == 0 ? tspmlp::pass_nj<KOUT>(p, ti.c) : nN;
        if (ti.j < 0 || ti.j >= lim) return printf("bad j at %d\n", t), 1;
        const size_t key = ((static_cast<size_t>(ti.type) * C + ti.c) * MP + ti.m) * maxj + ti.j;
        if (hit[key]) return printf("duplicate tile at %d\n", t), 1;
        hit[key] = 1;
        const int g = (ti.type * C + ti.c) * MP + ti.m;
        first[g] = std::min(first[g], t);
        last[g] = std::max(last[g], t);
        ++cnt[g];
    }
    for (int c = 0; c < C; ++c)
        for (int m = 0; m < MP; ++m) {
            const int up = (0 * C + c) * MP + m, dn = (1 * C + c) * MP + m;
            if (cnt[up] != tspmlp::pass_nj<KOUT>(p, c) || cnt[dn] != nN)
                return printf("missing tiles c=%d m=%d\n", c, m), 1;
            if (last[up] >= first[dn]) return printf("down before gate/up c=%d m=%d\n", c, m), 1;
            if (c > 0 && last[(1 * C + c - 1) * MP + m] >= first[dn])
                return printf("down before previous chunk's down c=%d m=%d\n", c, m), 1;
            if (c > 1 && last[(1 * C + c - 2) * MP + m] >= first[up])
                return printf("H buffer reused too early c=%d m=%d\n", c, m), 1;
        }
    return 0;
}

int main() {
    int bad = 0, cases = 0;
    const int heads[] = {1, 37, 148};
    for (int MB = 1; MB <= 70; MB += (MB < 12 ? 1 : 7))
        for (int GM = 1; GM <= 9; ++GM)
            for (int nJ : {1, 3, 112})
                for (int nC : {1, 2, 16})
                    for (int head : heads) {
                        const int R = (3 * GM < MB) ? 3 * GM : MB;
                        bad += check(MB, nJ, nC, GM, head, R);
                        ++cases;
                    }
    for (int MP = 1; MP <= 40; MP += 3)
        for (int C = 1; C <= 9; ++C)
            for (int nN : {1, 4, 16})
                for (int head : {1, 74}) {
                    int w[tspmlp::kFusedMaxChunks];
                    for (int c = 0; c < C; ++c) w[c] = 64 * (1 + (c * 7 + MP) % 40);
                    bad += check_passes<128>(MP, C, nN, head, w);
                    bad += check_passes<256>(MP, C, nN, head, w);
                    cases += 2;
                }
    printf("%d cases, %d failed\n", cases, bad);
    return bad ? 1 : 0;
}
