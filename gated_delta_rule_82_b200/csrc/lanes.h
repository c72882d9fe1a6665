// lanes.h -- how packed sequences of different lengths are dealt to lanes: runs of whole
// sequences, in order, that stand in for batch rows of the chunked forward (a lane's chunks are
// the chunks of its sequences in turn, and one chain per lane and head walks through them).
// Lanes of about kLaneChunks chunks let P x H chains run where one chain per head would walk
// through every sequence.  A lane is closed once it holds at least its share of the chunks and
// the next sequence has chunks (a sequence's chunks must stay in one chain).
//
// Plain C++ (no CUDA types): the host plans with it, the kernels take the plan by value, and a
// host-side test checks it.
#pragma once

#include <string.h>

namespace ckda {

constexpr int kMaxLanes = 64;
constexpr int kLaneChunks = 32;

struct LanePlan {
    int P;                      // lanes
    int NTL;                    // chunks of the longest lane (the NT of the launch)
    int total;                  // chunks of all sequences (per head)
    int seq0[kMaxLanes + 1];    // first sequence of each lane; seq0[P] = number of sequences
    int cbase[kMaxLanes + 1];   // chunks before each lane; cbase[P] = total
};

// n sequences with token offsets cu_host[0..n] (cu_host[0] = 0, non-decreasing), chunks of
// `chunk` tokens (a sequence of len tokens has ceil(len / chunk) of them).
inline LanePlan plan_lanes(const int* cu_host, int n, int chunk) {
    LanePlan lp;
    memset(&lp, 0, sizeof(lp));
    long long total = 0;
    int nonempty = 0;
    for (int s = 0; s < n; ++s) {
        total += (cu_host[s + 1] - cu_host[s] + chunk - 1) / chunk;
        nonempty += cu_host[s + 1] > cu_host[s];
    }
    int P = (int)((total + kLaneChunks / 2) / kLaneChunks);
    P = P < 1 ? 1 : P;
    P = P > kMaxLanes ? kMaxLanes : P;
    P = P > nonempty ? (nonempty > 0 ? nonempty : 1) : P;
    const long long share = (total + P - 1) / P;
    int l = 0;
    long long in_lane = 0, seen = 0;
    lp.seq0[0] = 0;
    lp.cbase[0] = 0;
    for (int s = 0; s < n; ++s) {
        const long long nch = (cu_host[s + 1] - cu_host[s] + chunk - 1) / chunk;
        if (nch > 0 && in_lane >= share && l < P - 1) {
            ++l;
            lp.seq0[l] = s;
            lp.cbase[l] = (int)seen;
            in_lane = 0;
        }
        in_lane += nch;
        seen += nch;
    }
    lp.P = l + 1;
    lp.seq0[lp.P] = n;
    lp.cbase[lp.P] = (int)total;
    lp.total = (int)total;
    lp.NTL = 0;
    for (int i = 0; i < lp.P; ++i)
        if (lp.cbase[i + 1] - lp.cbase[i] > lp.NTL) lp.NTL = lp.cbase[i + 1] - lp.cbase[i];
    return lp;
}

}  // namespace ckda
