// policy.cu -- HyLRA's offline reuse policy over the layer similarity matrix (host code).
//
// "HyLRA: Hybrid Layer Reuse Attention", sec. 2.2: the layer configuration is a
// path search on the similarity matrix M.  A state (i, j) means layer j runs on
// the top-k indices of source layer i.  A reset jump to (j, j) runs layer j in
// full attention, which refreshes the indices; a vertical move (i, j) -> (i, j+1)
// reuses layer i's indices for layer j+1 and is allowed only when M[j+1][i]
// exceeds the threshold theta.  The policy minimises the number of full layers,
// then maximises the summed similarity of the reused layers.
//
// Dynamic programming over the layers, O(L^2): the states alive after layer j
// are the sources i <= j whose run of reuses is still allowed.  A state (i, j)
// with i < j has one history past layer i (layers i..j all on source i), so the
// only choice is the predecessor of each reset, kept in parent[].  Among equal
// (full count, similarity) the smaller source wins; comparing whole policies,
// that is the smallest source sequence read from the last layer backwards.
#include <cmath>
#include <cstdint>
#include <vector>

#include "tsa.h"

namespace tsa {
void set_error_message(const char* msg);
}

namespace {

struct Cost {
    int32_t full;
    double sim;
};

// a before b: fewer full layers, then more similarity (ties: the caller's order)
bool better(const Cost& a, const Cost& b) { return a.full != b.full ? a.full < b.full : a.sim > b.sim; }

}  // namespace

extern "C" tsa_status tsa_reuse_policy(const double* M, int32_t n_layers, double theta, const uint8_t* force_full,
                                       int32_t* source, int32_t* n_full, double* total_sim) {
    if (n_layers < 1 || n_layers > 4096) {
        tsa::set_error_message("tsa_reuse_policy: n_layers must be in [1, 4096]");
        return TSA_ERR_INVALID_ARG;
    }
    if (!M || !source) {
        tsa::set_error_message("tsa_reuse_policy: NULL pointer (M or source)");
        return TSA_ERR_INVALID_ARG;
    }
    if (std::isnan(theta)) {
        tsa::set_error_message("tsa_reuse_policy: theta is NaN");
        return TSA_ERR_INVALID_ARG;
    }
    const int L = n_layers;
    std::vector<Cost> cost(L);
    std::vector<uint8_t> alive(L, 0);
    std::vector<int32_t> parent(L, -1);
    cost[0] = {1, 0.0};  // layer 0 has no earlier indices: a full layer
    alive[0] = 1;
    for (int j = 1; j < L; ++j) {
        // reset at j: the best state after layer j - 1 (smallest source on ties)
        int best = -1;
        for (int i = 0; i < j; ++i)
            if (alive[i] && (best < 0 || better(cost[i], cost[best]))) best = i;
        const Cost reset = {cost[best].full + 1, cost[best].sim};
        parent[j] = best;
        // vertical moves: source i carries on to layer j when M[j][i] > theta
        const bool forced = force_full && force_full[j];
        for (int i = 0; i < j; ++i) {
            if (!alive[i]) continue;
            const double m = M[(size_t)j * L + i];
            if (!forced && m > theta)
                cost[i].sim += m;
            else
                alive[i] = 0;
        }
        cost[j] = reset;
        alive[j] = 1;
    }
    int end = -1;
    for (int i = 0; i < L; ++i)
        if (alive[i] && (end < 0 || better(cost[i], cost[end]))) end = i;
    // layers end..L-1 run on source `end`; the run before it ends at parent[end] - 1 ...
    for (int hi = L - 1, i = end; i >= 0; hi = i - 1, i = parent[i]) {
        for (int j = i; j <= hi; ++j) source[j] = i;
        if (i == 0) break;
    }
    if (n_full) *n_full = cost[end].full;
    if (total_sim) *total_sim = cost[end].sim;
    return TSA_OK;
}
