// Host harness for the library's mask range functions (common.cuh), built and run
// by tests/test_mask_ranges.py.  Reads one mask from stdin:
//   Tq Tk q_off k_off causal num_docs cu[0] .. cu[num_docs]   (num_docs = 0: no documents)
// and prints, one line each,
//   R t cls lo hi          row_interval for every row t
//   Q t0 t1 kbeg kend      rows_key_range for rows [t0, t1] (several tile lengths)
//   K k0 k1 tbeg tend      keys_row_range for keys [k0, k1] (several tile lengths)
//   S s ta tb              key_rows for every key s in [-1, Tk]
//   G nt np lin tile pair  heavy_first over grids of nt tiles x np (batch, head) pairs
#include <cstdio>
#include <vector>

#include "../online_softmax_merge_eagle_b200/csrc/common.cuh"

int main() {
    long long tq, tk, qo, ko;
    int causal, nd;
    if (scanf("%lld %lld %lld %lld %d %d", &tq, &tk, &qo, &ko, &causal, &nd) != 6) return 2;
    std::vector<int32_t> cu(nd + 1);
    if (nd > 0)
        for (int i = 0; i <= nd; ++i)
            if (scanf("%d", &cu[i]) != 1) return 2;
    eagle::MaskDesc m;
    m.cu = nd > 0 ? cu.data() : nullptr;
    m.num_docs = nd;
    m.q_off = qo;
    m.k_off = ko;
    m.causal = causal;
    m.Tq = (int)tq;
    m.Tk = (int)tk;
    for (int t = 0; t < m.Tq; ++t) {
        int lo, hi;
        const int c = eagle::row_interval(m, t, lo, hi);
        printf("R %d %d %d %d\n", t, c, lo, hi);
    }
    const int lens[4] = {1, 7, 128, 300};
    for (int li = 0; li < 4; ++li) {
        for (int t0 = 0; t0 < m.Tq; t0 += (lens[li] > 64 ? 61 : 13)) {
            const int t1 = t0 + lens[li] - 1 < m.Tq ? t0 + lens[li] - 1 : m.Tq - 1;
            int a, b;
            eagle::rows_key_range(m, t0, t1, a, b);
            printf("Q %d %d %d %d\n", t0, t1, a, b);
        }
        for (int k0 = 0; k0 < m.Tk; k0 += (lens[li] > 64 ? 61 : 13)) {
            const int k1 = k0 + lens[li] - 1 < m.Tk ? k0 + lens[li] - 1 : m.Tk - 1;
            int a, b;
            eagle::keys_row_range(m, k0, k1, a, b);
            printf("K %d %d %d %d\n", k0, k1, a, b);
        }
    }
    for (int s = -1; s <= m.Tk; ++s) {
        int a, b;
        eagle::key_rows(m, s, a, b);
        printf("S %d %d %d\n", s, a, b);
    }
    const int grids[6][2] = {{1, 1}, {5, 19}, {64, 64}, {3, 8}, {7, 9}, {2, 17}};
    for (int g = 0; g < 6; ++g)
        for (int lin = 0; lin < grids[g][0] * grids[g][1]; ++lin) {
            int tile, pair;
            eagle::heavy_first(lin, grids[g][0], grids[g][1], tile, pair);
            printf("G %d %d %d %d %d\n", grids[g][0], grids[g][1], lin, tile, pair);
        }
    return 0;
}
