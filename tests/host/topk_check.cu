// Host-side check of the top-k selection list used by the router epilogue
// and by the permutation's warp merge (csrc/topk.cuh): random logits with
// ties, NaN and -inf against a brute-force selection (sort by value
// descending, then index ascending, NaN left out; slots only NaN could fill
// take the lowest indices not taken yet).  Prints "OK <cases>" or the first
// mismatch.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <random>
#include <vector>

#include "topk.cuh"

using l4moe::TopK;
using l4moe::kMaxTopK;

struct Ref {
    std::vector<int> idx;      // k selected
    std::vector<float> val;    // their values (-inf for NaN fills)
    float next;                // the best value left out (-inf if none)
};

static Ref brute(const std::vector<float>& l, int k) {
    std::vector<int> order;
    for (int e = 0; e < (int)l.size(); ++e)
        if (!std::isnan(l[e])) order.push_back(e);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return l[a] > l[b]; });
    Ref r;
    for (int j = 0; j < k && j < (int)order.size(); ++j) {
        r.idx.push_back(order[j]);
        r.val.push_back(l[order[j]]);
    }
    while ((int)r.idx.size() < k) {  // only NaN left: lowest untaken index
        int e = 0;
        while (std::find(r.idx.begin(), r.idx.end(), e) != r.idx.end()) ++e;
        r.idx.push_back(e);
        r.val.push_back(-INFINITY);
    }
    r.next = (int)order.size() > k ? l[order[k]] : -INFINITY;
    return r;
}

// The warp merge of the permutation kernel, one lane after another: lane
// owns experts lane, lane + 32, ...; k + 1 rounds each take the first head
// in (value, index) order.
static TopK merged(const std::vector<float>& l, int k) {
    TopK lane[32];
    int pos[32];
    for (int q = 0; q < 32; ++q) {
        lane[q].init();
        pos[q] = 0;
        for (int e = q; e < (int)l.size(); e += 32) lane[q].offer(l[e], e);
    }
    TopK out;
    out.init();
    for (int j = 0; j <= kMaxTopK; ++j) {
        float hv = lane[0].value(pos[0]);
        int hi = pos[0] <= kMaxTopK ? lane[0].index(pos[0]) : -1, hl = 0;
        for (int q = 1; q < 32; ++q) {
            const float ov = lane[q].value(pos[q]);
            const int oi = pos[q] <= kMaxTopK ? lane[q].index(pos[q]) : -1;
            if (l4moe::topk_before(ov, oi, hv, hi)) hv = ov, hi = oi, hl = q;
        }
        out.set(j, hv, hi);
        if (hi >= 0) ++pos[hl];
    }
    out.fill_empty(k);
    return out;
}

static bool same(float a, float b) { return a == b || (std::isnan(a) && std::isnan(b)); }

static bool check(const TopK& t, const Ref& r, int k, const char* what, int c) {
    for (int j = 0; j < k; ++j)
        if (t.index(j) != r.idx[j] || !same(t.value(j), r.val[j])) {
            printf("MISMATCH %s case %d slot %d: got (%d, %g) want (%d, %g)\n", what, c, j, t.index(j),
                   t.value(j), r.idx[j], r.val[j]);
            return false;
        }
    const float margin = t.value(k - 1) - t.value(k), want = r.val[k - 1] - r.next;
    if (!same(margin, want)) {
        printf("MISMATCH %s case %d margin: got %g want %g\n", what, c, margin, want);
        return false;
    }
    return true;
}

int main() {
    std::mt19937 rng(12345);
    const float pool[] = {0.f, 1.f, -1.f, 2.5f, 2.5f, -INFINITY, NAN, 7.f, -3.f, 1.f};
    int cases = 0;
    for (int c = 0; c < 20000; ++c) {
        const int E = 1 + (int)(rng() % 80);
        const int k = 1 + (int)(rng() % std::min(kMaxTopK, E));
        std::vector<float> l(E);
        const int mode = c % 4;
        for (int e = 0; e < E; ++e) {
            if (mode == 0)
                l[e] = pool[rng() % 10];  // heavy ties, NaN, -inf
            else if (mode == 1)
                l[e] = (float)((int)(rng() % 2001) - 1000) / 100.f;
            else if (mode == 2)
                l[e] = (rng() % 3 == 0) ? (float)(rng() % 5) : NAN;  // mostly NaN
            else
                l[e] = (float)(rng() % 7);
        }
        const Ref r = brute(l, k);
        TopK t;
        t.init();
        for (int e = 0; e < E; ++e) t.offer(l[e], e);
        t.fill_empty(k);
        if (!check(t, r, k, "sequential", c)) return 1;
        if (!check(merged(l, k), r, k, "warp-merge", c)) return 1;
        ++cases;
    }
    printf("OK %d\n", cases);
    return 0;
}
