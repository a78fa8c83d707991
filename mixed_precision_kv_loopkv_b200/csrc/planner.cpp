// Offline precision planner over synthetic damage tables (host code).
//
// LoopKV: Loop-Aware KV Cache Compression for Serving Looped Transformers,
// Abstract: a one-time profile gives every (loop, layer) cell a damage for
// each choice (4-bit, 2-bit, reuse of the final loop's cell), damages add up
// over cells, and the planner picks the choices that minimise the bytes read
// per decoded token under budgets on predicted damage and storage.  The
// pages give no formulation; this is the library's reading:
//   * choice of cell c: 4-bit, 2-bit, or reuse (not in the final loop);
//   * damage: sum over cells of damage[c][choice] <= damage_budget;
//   * storage (32-byte units per token-head): 4-bit 5, 2-bit 3, reuse 0;
//     sum <= storage_budget;
//   * reads per token-head: 4-bit q4_read_bytes (128 plus the expected
//     low-plane share), 2-bit 96, reuse the reads of its source, the final
//     loop's cell of the same layer;
//   * objective: minimise total reads; among plans of equal reads, one with
//     the least damage, and among those one with the least storage.
// The problem separates by layer once the final loop's choice of that layer
// is fixed, so an exact dynamic program runs over layers with (damage,
// storage) as state and, per layer, every combination of its L choices.
#include <stdint.h>

#include <algorithm>
#include <limits>
#include <vector>

#include "loopkv.h"

namespace {

constexpr int kChoices = 3;  // 0: 4-bit, 1: 2-bit, 2: reuse (plan codes 0, 1, 2)
constexpr int kStorage[kChoices] = {5, 3, 0};
constexpr int kMaxLoops = 6;
constexpr long kMaxStates = 1L << 25;  // (damage, storage) states times layers

struct Combo {
  int64_t damage;
  int storage;
  int64_t reads;
  int code;  // base-3 digits: choice of loop l at 3^l
};

}  // namespace

extern "C" {

loopkv_status loopkv_plan_cells(int32_t num_loops, int32_t num_layers, const int32_t* damage,
                                int32_t damage_budget, int32_t storage_budget, int32_t q4_read_bytes,
                                uint8_t* plan_out, int64_t* reads_out) {
  const int L = num_loops, N = num_layers;
  if (L <= 0 || L > kMaxLoops || N <= 0 || !damage || !plan_out || damage_budget < 0 || storage_budget < 0 ||
      q4_read_bytes < 0)
    return LOOPKV_ERR_INVALID_ARG;
  for (int c = 0; c < L * N * kChoices; ++c)
    if (damage[c] < 0) return LOOPKV_ERR_INVALID_ARG;
  const int D = damage_budget, S = std::min(storage_budget, kStorage[0] * L * N);
  if (static_cast<long>(D + 1) * (S + 1) * N > kMaxStates) return LOOPKV_ERR_UNSUPPORTED;

  // every admissible choice combination of each layer
  int pow3 = 1;
  for (int l = 0; l < L; ++l) pow3 *= kChoices;
  std::vector<std::vector<Combo>> combos(N);
  for (int j = 0; j < N; ++j) {
    for (int code = 0; code < pow3; ++code) {
      int ch[kMaxLoops];
      for (int l = 0, x = code; l < L; ++l, x /= kChoices) ch[l] = x % kChoices;
      if (ch[L - 1] == 2) continue;  // the final loop stores its own cache
      const int64_t src_reads = ch[L - 1] == 0 ? q4_read_bytes : 96;
      Combo cb{0, 0, 0, code};
      for (int l = 0; l < L; ++l) {
        const int cell = l * N + j;
        cb.damage += damage[cell * kChoices + ch[l]];
        cb.storage += kStorage[ch[l]];
        cb.reads += ch[l] == 0 ? q4_read_bytes : ch[l] == 1 ? 96 : src_reads;
      }
      if (cb.damage <= D && cb.storage <= S) combos[j].push_back(cb);
    }
    if (combos[j].empty()) return LOOPKV_ERR_BAD_PLAN;
  }

  // best[d][s]: minimal (reads, damage, storage) reaching exactly (d, s)
  // after the layers processed so far; choice[j][d][s]: combo index used
  const int64_t kInf = std::numeric_limits<int64_t>::max();
  const size_t states = static_cast<size_t>(D + 1) * (S + 1);
  std::vector<int64_t> best(states, kInf), next(states);
  std::vector<std::vector<int16_t>> choice(N, std::vector<int16_t>(states, -1));
  best[0] = 0;
  for (int j = 0; j < N; ++j) {
    std::fill(next.begin(), next.end(), kInf);
    for (int d = 0; d <= D; ++d)
      for (int s = 0; s <= S; ++s) {
        const int64_t r = best[static_cast<size_t>(d) * (S + 1) + s];
        if (r == kInf) continue;
        for (size_t i = 0; i < combos[j].size(); ++i) {
          const Combo& cb = combos[j][i];
          const int d2 = d + static_cast<int>(cb.damage), s2 = s + cb.storage;
          if (d2 > D || s2 > S) continue;
          const size_t k = static_cast<size_t>(d2) * (S + 1) + s2;
          if (r + cb.reads < next[k]) {
            next[k] = r + cb.reads;
            choice[j][k] = static_cast<int16_t>(i);
          }
        }
      }
    best.swap(next);
  }
  // cheapest end state; ties: less damage, then less storage (scan order)
  int64_t best_r = kInf;
  int bd = -1, bs = -1;
  for (int d = 0; d <= D; ++d)
    for (int s = 0; s <= S; ++s) {
      const int64_t r = best[static_cast<size_t>(d) * (S + 1) + s];
      if (r < best_r) {
        best_r = r;
        bd = d;
        bs = s;
      }
    }
  if (best_r == kInf) return LOOPKV_ERR_BAD_PLAN;  // budgets admit no plan
  // walk back
  int d = bd, s = bs;
  for (int j = N - 1; j >= 0; --j) {
    const int i = choice[j][static_cast<size_t>(d) * (S + 1) + s];
    const Combo& cb = combos[j][i];
    for (int l = 0, x = cb.code; l < L; ++l, x /= kChoices) plan_out[l * N + j] = static_cast<uint8_t>(x % kChoices);
    d -= static_cast<int>(cb.damage);
    s -= cb.storage;
  }
  if (reads_out) *reads_out = best_r;
  return LOOPKV_OK;
}

}  // extern "C"
