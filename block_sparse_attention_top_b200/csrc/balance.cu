// Runtime load balancing by head migration, host-side planner (FVAttn review,
// section 3 "Stage 2: Runtime Load Balancing", Eqs. 1-6, section 3.2 and the
// RLB algorithm flow of section 5).  Every rank runs this search on the same
// all-gathered head workloads and gets the same plan, so no rank has to solve
// and broadcast.
//
// Plans: disjoint pairs of ranks, each pair swapping one head of each side
// (one send and one receive per rank, at most one local head moved -- the
// pages' S_20% with "pair topologies"); the empty plan is allowed.
// Objective (Eq. 6): lexicographic minimum of (max_r L_r_new, Var_r L_r_new).
// For a fixed set of pairs the optimum decomposes exactly: the global maximum
// is the larger of the unpaired loads and each pair's smallest achievable
// maximum, and then each pair independently takes its least sum of squares
// among the swaps that stay under that maximum (the total load is invariant,
// so Var orders like the sum of squares).  All sets of pairs are enumerated.
#include <algorithm>
#include <cmath>
#include <vector>

#include "bsa_internal.cuh"

namespace {

struct Planner {
    int R;
    std::vector<double> L;                       // rank loads
    std::vector<std::vector<int>> heads;         // heads of each rank
    const float* Lh;
    // best plan so far
    double best_max = INFINITY, best_ss = INFINITY;
    std::vector<int> best_moves;                 // triples
    // current matching
    std::vector<std::pair<int, int>> pairs;

    // Smallest max over swaps of pair (a, b); the empty set if a rank has no head.
    double pair_min_max(int a, int b) const {
        double m = INFINITY;
        for (int ha : heads[a])
            for (int hb : heads[b]) {
                const double la = L[a] - Lh[ha] + Lh[hb], lb = L[b] - Lh[hb] + Lh[ha];
                m = std::min(m, std::max(la, lb));
            }
        return m;
    }

    void evaluate() {
        std::vector<char> paired(R, 0);
        double M = -INFINITY;
        for (auto& pr : pairs) {
            paired[pr.first] = paired[pr.second] = 1;
            M = std::max(M, pair_min_max(pr.first, pr.second));
        }
        double ss = 0.0;
        for (int r = 0; r < R; ++r)
            if (!paired[r]) { M = std::max(M, L[r]); ss += L[r] * L[r]; }
        if (!(M <= best_max)) return;            // also rejects pairs without any swap (M = inf)
        std::vector<int> moves;
        for (auto& pr : pairs) {
            const int a = pr.first, b = pr.second;
            double bss = INFINITY;
            int bha = -1, bhb = -1;
            for (int ha : heads[a])
                for (int hb : heads[b]) {
                    const double la = L[a] - Lh[ha] + Lh[hb], lb = L[b] - Lh[hb] + Lh[ha];
                    if (std::max(la, lb) > M) continue;
                    const double s = la * la + lb * lb;
                    if (s < bss) { bss = s; bha = ha; bhb = hb; }
                }
            ss += bss;
            moves.insert(moves.end(), {a, b, bha, b, a, bhb});
        }
        if (M < best_max || (M == best_max && ss < best_ss)) {
            best_max = M;
            best_ss = ss;
            best_moves = moves;
        }
    }

    void enumerate(std::vector<int>& free_ranks, size_t pos) {
        if (pos == free_ranks.size()) { evaluate(); return; }
        const int first = free_ranks[pos];
        if (first < 0) { enumerate(free_ranks, pos + 1); return; }
        // `first` stays unpaired
        free_ranks[pos] = -1;
        enumerate(free_ranks, pos + 1);
        // or pairs with a later free rank
        for (size_t i = pos + 1; i < free_ranks.size(); ++i) {
            const int other = free_ranks[i];
            if (other < 0) continue;
            free_ranks[i] = -1;
            pairs.emplace_back(first, other);
            enumerate(free_ranks, pos + 1);
            pairs.pop_back();
            free_ranks[i] = other;
        }
        free_ranks[pos] = first;
    }
};

}  // namespace

extern "C" {

int bsa_rlb_plan(int R, int n_heads, const int32_t* head_rank, const float* L_h, int32_t* moves, int* n_moves,
                 float* L_r_new, float* rho_before, float* rho_after) {
    if (R < 1 || n_heads < 0 || (n_heads > 0 && (!head_rank || !L_h)) || !moves || !n_moves || !L_r_new)
        return BSA_EINVAL;
    if (R > 12) return BSA_EUNSUPPORTED;         // the enumeration grows like the involution numbers
    Planner pl;
    pl.R = R;
    pl.L.assign(R, 0.0);
    pl.heads.assign(R, {});
    pl.Lh = L_h;
    for (int h = 0; h < n_heads; ++h) {
        const int r = head_rank[h];
        if (r < 0 || r >= R || !(L_h[h] >= 0.0f)) return BSA_EINVAL;
        pl.L[r] += L_h[h];
        pl.heads[r].push_back(h);
    }
    std::vector<int> free_ranks(R);
    for (int r = 0; r < R; ++r) free_ranks[r] = r;
    pl.enumerate(free_ranks, 0);
    std::vector<double> Ln = pl.L;
    const int n = (int)pl.best_moves.size() / 3;
    for (int m = 0; m < n; ++m) {
        const int src = pl.best_moves[3 * m], dst = pl.best_moves[3 * m + 1], h = pl.best_moves[3 * m + 2];
        moves[3 * m] = src;
        moves[3 * m + 1] = dst;
        moves[3 * m + 2] = h;
        Ln[src] -= L_h[h];
        Ln[dst] += L_h[h];
    }
    *n_moves = n;
    double s0 = 0.0, m0 = 0.0, s1 = 0.0, m1 = 0.0;
    for (int r = 0; r < R; ++r) {
        L_r_new[r] = (float)Ln[r];
        s0 += pl.L[r]; m0 = std::max(m0, pl.L[r]);
        s1 += Ln[r];   m1 = std::max(m1, Ln[r]);
    }
    if (rho_before) *rho_before = s0 > 0 ? (float)(m0 / (s0 / R)) : 1.0f;
    if (rho_after) *rho_after = s1 > 0 ? (float)(m1 / (s1 / R)) : 1.0f;
    return BSA_OK;
}

int bsa_rank_loads(int R, int n_heads, const int32_t* head_rank, const float* L_h, float* L_r, float* rho,
                   int32_t* heads_per_rank) {
    if (R < 1 || n_heads < 0 || (n_heads > 0 && (!head_rank || !L_h)) || !L_r) return BSA_EINVAL;
    std::vector<double> L(R, 0.0);
    std::vector<int32_t> cnt(R, 0);
    for (int h = 0; h < n_heads; ++h) {
        const int r = head_rank[h];
        if (r < 0 || r >= R || !(L_h[h] >= 0.0f)) return BSA_EINVAL;
        L[r] += L_h[h];                           // Eq. 1: a rank's load is the sum of its heads' loads
        ++cnt[r];
    }
    double s = 0.0, m = 0.0;
    for (int r = 0; r < R; ++r) {
        L_r[r] = (float)L[r];
        s += L[r];
        m = std::max(m, L[r]);
        if (heads_per_rank) heads_per_rank[r] = cnt[r];
    }
    if (rho) *rho = s > 0 ? (float)(m / (s / R)) : 1.0f;   // Eq. 2
    return BSA_OK;
}

int bsa_rlb_gain(int R, const float* L_r, const float* L_r_new, double c, double P, double C, double A,
                 double* K, double* G) {
    if (R < 1 || !L_r || !L_r_new || !K || !G) return BSA_EINVAL;
    double before = -INFINITY, after = -INFINITY;
    for (int r = 0; r < R; ++r) {
        if (!(L_r[r] >= 0.0f) || !(L_r_new[r] >= 0.0f)) return BSA_EINVAL;
        before = std::max(before, (double)L_r[r]);
        after = std::max(after, (double)L_r_new[r]);
    }
    *K = c * (before - after);
    *G = *K - P - C - A;
    return BSA_OK;
}

int bsa_balance_policy(float rho, float k1, float k2) {
    if (!(rho >= 0.0f) || !(k1 <= k2)) return BSA_EINVAL;
    return rho < k1 ? 0 : (rho < k2 ? 1 : 2);
}

}  // extern "C"
