// Host-side check of the fused forward kernel's tile list (fused.cuh):
// for many geometries, the list visits every gate/up and down tile exactly
// once, and every dependency a producer waits for (down tile -> all gate/up
// tiles of its row block; gate/up tile -> all down tiles of the row block R
// earlier, whose H-ring slot it reuses) sits earlier in the list.  Tiles are
// handed out in list order, so this is what makes every wait end.
#include <cstdio>
#include <vector>

#include "../sequence_transformer_mlp_b200/csrc/fused.cuh"

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
    printf("%d cases, %d failed\n", cases, bad);
    return bad ? 1 : 0;
}
