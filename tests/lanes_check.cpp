// Host-side check of the lane plan (lanes.h) and of the item order the packed-sequence kernels
// build from it.  For random offsets: the lanes are runs of whole sequences covering all of them
// in order, their chunk counts add up, every lane after the first starts at a sequence with
// chunks, P <= min(64, sequences with chunks), NTL is the longest lane.  The item order -- each
// (unit, chunk) pair at base(group) + sum over the group's units of min(count, c) + the group's
// units before it that have chunk c, as the table kernel places it -- is a permutation of all
// pairs, keeps each unit's chunks in order, and equals the batched work order (head groups,
// chunk-major inside a group) when all lanes are equally long.
#include <cstdio>
#include <cstdlib>
#include <random>
#include <vector>

#include "lanes.h"

using namespace ckda;

static int item_pos(const LanePlan& lp, int H, int group, int u, int c) {
    auto cnt = [&](int l) { return lp.cbase[l + 1] - lp.cbase[l]; };
    const int BH = lp.P * H, l = u / H;
    const int g0 = u - u % group, g1 = g0 + group < BH ? g0 + group : BH;
    const int la = g0 / H, lb = (g1 - 1) / H;
    long long pos = (long long)H * lp.cbase[la] + (long long)(g0 - la * H) * cnt(la);
    pos += u - (g0 > l * H ? g0 : l * H);
    for (int c2 = 0; c2 <= c; ++c2)
        for (int l2 = la; l2 <= lb; ++l2) {
            const int m = (g1 < (l2 + 1) * H ? g1 : (l2 + 1) * H) - (g0 > l2 * H ? g0 : l2 * H);
            if (cnt(l2) > c2 && (c2 < c || l2 < l)) pos += m;
        }
    return (int)pos;
}

int main() {
    std::mt19937 rng(12345);
    int failures = 0, cases = 0;
    for (int trial = 0; trial < 400; ++trial) {
        const int n = 1 + rng() % 300, H = 1 + rng() % 12, chunk = 64;
        const bool equal = trial % 5 == 0;
        std::vector<int> cu(n + 1, 0);
        const int fixed = 64 * (1 + rng() % 8);
        for (int s = 0; s < n; ++s) {
            int len = equal ? fixed : (rng() % 10 < 3 ? 0 : (int)(rng() % 500));
            cu[s + 1] = cu[s] + len;
        }
        const LanePlan lp = plan_lanes(cu.data(), n, chunk);
        if (lp.total == 0) continue;
        ++cases;
        int nonempty = 0, total = 0;
        for (int s = 0; s < n; ++s) {
            nonempty += cu[s + 1] > cu[s];
            total += (cu[s + 1] - cu[s] + chunk - 1) / chunk;
        }
        bool ok = lp.P >= 1 && lp.P <= kMaxLanes && lp.P <= nonempty && lp.total == total &&
                  lp.seq0[0] == 0 && lp.seq0[lp.P] == n && lp.cbase[0] == 0 &&
                  lp.cbase[lp.P] == total;
        int longest = 0;
        for (int l = 0; ok && l < lp.P; ++l) {
            int c = 0;
            for (int s = lp.seq0[l]; s < lp.seq0[l + 1]; ++s) c += (cu[s + 1] - cu[s] + chunk - 1) / chunk;
            ok = ok && lp.seq0[l] < lp.seq0[l + 1] && c == lp.cbase[l + 1] - lp.cbase[l];
            if (l > 0) ok = ok && cu[lp.seq0[l] + 1] > cu[lp.seq0[l]];
            if (c > longest) longest = c;
        }
        ok = ok && lp.NTL == longest;
        // the item order
        const int BH = lp.P * H, items = H * lp.total;
        const int groups[] = {1, 3, 7, 32, BH, 1 + (int)(rng() % BH)};
        for (int group : groups) {
            std::vector<int> seen(items, -1);
            std::vector<int> last(BH, -1);
            for (int u = 0; ok && u < BH; ++u)
                for (int c = 0; ok && c < lp.cbase[u / H + 1] - lp.cbase[u / H]; ++c) {
                    const int p = item_pos(lp, H, group, u, c);
                    ok = p >= 0 && p < items && seen[p] < 0;
                    if (ok) seen[p] = u * 4096 + c;
                }
            for (int p = 0; ok && p < items; ++p) {
                const int u = seen[p] / 4096, c = seen[p] % 4096;
                ok = seen[p] >= 0 && last[u] == c - 1;
                last[u] = c;
                if (ok && equal && lp.NTL * lp.P == lp.total) {   // the batched work order
                    const int NT = lp.NTL, lastg = (BH - 1) / group;
                    const int g = p / (group * NT), r = p % (group * NT);
                    const int gs = g == lastg ? BH - lastg * group : group;
                    ok = u == g * group + (r - (r / gs) * gs) && c == r / gs;
                }
            }
        }
        if (!ok) {
            ++failures;
            std::printf("failure: trial %d n %d H %d P %d\n", trial, n, H, lp.P);
        }
    }
    std::printf("cases %d failures %d\n", cases, failures);
    return failures ? 1 : 0;
}
