// plan_search.cu -- offline plan search of LoopKV (host code only).
//
// LoopKV paper §3.1 "Allocation": given the per-cell damage of each storage option (the
// profile), choose one option per cell that minimizes the bytes read per token under a
// damage budget and, optionally, a storage budget (the read-optimized plan LoopKV-R uses
// the damage budget alone; the memory-optimized plan LoopKV-M both).  Damages add up over
// cells (§2.4, §3.1: summed single-cell damages predict a plan's KL).
//
// Options per cell of loops 0 .. n_loops-2: 4-bit codes, 2-bit codes, or sharing the final
// loop's cell of the same layer (§3.2: stores nothing, reads the source's INT4 pages like an
// own INT4 cell).  Final-loop cells keep 4-bit codes (the paper's plans choose among the 72
// cells of loops 1-3).  Bytes per token and head, in units of D/4 bytes: 4-bit stores and
// reads 5 (K codes D/2, K meta D/8, V meta D/8, hi D/4, lo D/4), 2-bit 3, a share cell
// stores 0 and reads 5.  Reads count every lo plane (the plan is made before any score is
// known).
//
// Exact solution: a dynamic program over the choosable cells whose state is (read units,
// stored units) and whose value is the least damage reaching that state; the answer is
// the least read total whose state has damage <= budget and storage <= budget, then the
// least damage, then the least storage.  Work is cells x states x 3, about 6 M steps for
// 72 cells.
#include "loopkv.h"

#include <cmath>
#include <cstdint>
#include <limits>
#include <vector>

namespace {

constexpr int kStore[3] = {5, 3, 0}; // stored units of LOOPKV_CELL_4B, _2B, _SHARE (reads: 5, 3, 5)

}  // namespace

extern "C" int loopkv_plan_search(const loopkv_config *cfg, const double *damage, double damage_budget,
                                  double storage_budget, uint8_t *modes_out, loopkv_plan_search_report *report)
{
    if (!cfg || !damage || !modes_out || cfg->n_layers <= 0 || cfg->n_loops <= 0 || cfg->n_heads <= 0 ||
        (cfg->head_dim != 64 && cfg->head_dim != 128) || !(damage_budget >= 0.0) || std::isnan(storage_budget))
        return LOOPKV_ERR_INVALID_ARG;
    const int L = cfg->n_layers, n_cells = cfg->n_loops * L;
    const int M = (cfg->n_loops - 1) * L; // choosable cells: loops 0 .. n_loops-2, loop-major
    for (int c = 0; c < n_cells; ++c)
        for (int o = 0; o < 3; ++o) {
            const double d = damage[3 * c + o];
            const bool used = c < M || o == LOOPKV_CELL_4B;
            if (used && !(d >= 0.0 && std::isfinite(d)))
                return LOOPKV_ERR_INVALID_ARG;
        }
    const double unit = (double)cfg->n_heads * cfg->head_dim / 4.0; // bytes per token of one unit
    // final loop: fixed 4-bit cells
    double fixed_damage = 0.0;
    for (int c = M; c < n_cells; ++c)
        fixed_damage += damage[3 * c + LOOPKV_CELL_4B];
    const int fixed_units = 5 * L;
    // storage budget in units for the choosable cells (no budget: any storage)
    int store_cap = 5 * M;
    if (storage_budget > 0.0) {
        const double cap = std::floor(storage_budget / unit + 1e-9) - fixed_units;
        if (cap < 0.0)
            return LOOPKV_ERR_INFEASIBLE;
        store_cap = cap < 5.0 * M ? (int)cap : 5 * M;
    }

    // read total = 5M - 2 * (#2-bit cells): index the state by k = #2-bit cells (0..M)
    // and s = stored units (0..5M)
    const int NS = 5 * M + 1, NK = M + 1;
    const double INF = std::numeric_limits<double>::infinity();
    std::vector<double> best((size_t)NK * NS, INF), next((size_t)NK * NS, INF);
    std::vector<uint8_t> choice((size_t)M * NK * NS, 0xFF); // option that reached (k, s) at cell c
    best[0] = 0.0;
    for (int c = 0; c < M; ++c) {
        std::fill(next.begin(), next.end(), INF);
        uint8_t *ch = choice.data() + (size_t)c * NK * NS;
        for (int k = 0; k <= c; ++k)
            for (int s = 0; s <= 5 * c; ++s) {
                const double d0 = best[(size_t)k * NS + s];
                if (d0 == INF)
                    continue;
                for (int o = 0; o < 3; ++o) {
                    const int k1 = k + (o == LOOPKV_CELL_2B), s1 = s + kStore[o];
                    const double d1 = d0 + damage[3 * c + o];
                    double &slot = next[(size_t)k1 * NS + s1];
                    if (d1 < slot) { // strict: ties keep the earlier option (deterministic)
                        slot = d1;
                        ch[(size_t)k1 * NS + s1] = (uint8_t)o;
                    }
                }
            }
        best.swap(next);
    }
    // fewest reads = most 2-bit cells; then least damage; then least storage
    int bk = -1, bs = -1;
    double bd = INF;
    for (int k = M; k >= 0 && bk < 0; --k)
        for (int s = 0; s <= store_cap; ++s) {
            const double d = best[(size_t)k * NS + s];
            if (d != INF && d + fixed_damage <= damage_budget && d < bd) {
                bd = d;
                bk = k;
                bs = s;
            }
        }
    if (bk < 0)
        return LOOPKV_ERR_INFEASIBLE;
    // walk the choices back
    for (int c = M - 1, k = bk, s = bs; c >= 0; --c) {
        const int o = choice[((size_t)c * NK + k) * NS + s];
        modes_out[c] = (uint8_t)o;
        k -= (o == LOOPKV_CELL_2B);
        s -= kStore[o];
    }
    for (int c = M; c < n_cells; ++c)
        modes_out[c] = LOOPKV_CELL_4B;
    if (report) {
        report->read_bytes_per_token = unit * (5.0 * M - 2.0 * bk + fixed_units);
        report->stored_bytes_per_token = unit * (bs + fixed_units);
        report->damage = bd + fixed_damage;
    }
    return LOOPKV_OK;
}
