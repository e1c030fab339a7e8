// Host check of the fused decode step's work-item order (csrc/prr_schedule.h, the
// definitions the kernel itself uses).  For a sweep of shapes and grid sizes:
//   - every item (SEL chunk, FIN, EMA, SPEC slot, REPAIR item, COMBINE head) is handed
//     out exactly once, with its unit and index in range;
//   - every item comes after every item it waits for (FIN after its unit's chunks; EMA
//     and REPAIR after FIN; COMBINE after FIN and all of its unit's SPEC and REPAIR
//     items), which is what makes the persistent grid free of deadlock;
//   - a unit's first dependent ticket trails its last SPEC ticket by the intended lag;
//   - a simulated grid that takes tickets the way the kernel does (SEL, SPEC and REPAIR
//     items take their CTA's next ticket as they start; a dependent item blocks its CTA
//     until its inputs exist) finishes, in random interleavings, also when fewer CTAs
//     are resident than the grid has.
// Built with -DSIMULATION_ONLY it skips the order and lag checks, so that a test can see
// the simulation alone catch a mis-ordered header.
// With the argument "items" it prints the item counts of the listed shapes instead, one
// line per shape read from stdin ("U maxnb P K G" -> "sel fin ema spec rep comb").
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <random>
#include <vector>

#include "prr_schedule.h"

namespace {

enum Kind { kSel = 1, kSpec = 2, kRepair = 3, kEma = 4, kCombine = 5, kFin = 6 };

struct Item {
  int kind, unit, idx;
};

struct Layout {
  int U, F, P, R, G, dep_lag;
  long long total;
};

int g_failures = 0;
#define CHECK(cond, ...)                       \
  do {                                         \
    if (!(cond)) {                             \
      if (g_failures++ < 20) {                 \
        std::printf("FAIL ");                  \
        std::printf(__VA_ARGS__);              \
        std::printf("\n");                     \
      }                                        \
    }                                          \
  } while (0)

Layout make_layout(int U, int maxnb, int P, int K, int G, long long resident) {
  Layout L{};
  L.U = U;
  const int cb = prr::fused_chunk_blocks(U, maxnb);
  L.F = (maxnb + cb - 1) / cb;
  L.P = P;
  L.R = prr::fused_rep_items(U, K);
  L.G = G;
  L.total = prr::fused_total_items(U, L.F, P, L.R, G);
  const long long grid = resident < L.total ? resident : L.total;  // as the launcher sizes it
  L.dep_lag = prr::fused_dep_lag(grid, P, U);
  return L;
}

// The item of ticket t, following the kernel's ranges.
Item item_of(const Layout& L, int t) {
  if (t < L.U * L.F) return {kSel, t / L.F, t % L.F};
  t -= L.U * L.F;
  if (t < L.U) return {kFin, t, 0};
  t -= L.U;
  if (t < L.U) return {kEma, t, 0};
  t -= L.U;
  int idx = -1, kind = 0;
  if (!prr::decode_tail(L.P, L.G, L.dep_lag, t, L.U, L.R, &idx, &kind)) return {kSpec, idx / L.P, idx % L.P};
  if (kind == 3) return {kRepair, idx / L.R, idx % L.R};
  return {kCombine, idx / L.G, idx % L.G};
}

struct Tickets {  // ticket of every item, -1 until seen
  std::vector<long long> sel, fin, ema, spec, rep, comb;
  explicit Tickets(const Layout& L)
      : sel(static_cast<size_t>(L.U) * L.F, -1), fin(L.U, -1), ema(L.U, -1),
        spec(static_cast<size_t>(L.U) * L.P, -1), rep(static_cast<size_t>(L.U) * L.R, -1),
        comb(static_cast<size_t>(L.U) * L.G, -1) {}
};

// Tickets that item `it` waits for (the kernel's waits: sel_cnt, sel_done, spec_done,
// rep_done and the repair descriptors, which the finisher publishes).
void deps_of(const Layout& L, const Tickets& T, const Item& it, std::vector<long long>* out) {
  out->clear();
  const int u = it.unit;
  switch (it.kind) {
    case kFin:
      for (int c = 0; c < L.F; ++c) out->push_back(T.sel[static_cast<size_t>(u) * L.F + c]);
      break;
    case kEma:
    case kRepair:
      out->push_back(T.fin[u]);
      break;
    case kCombine:
      out->push_back(T.fin[u]);
      for (int j = 0; j < L.P; ++j) out->push_back(T.spec[static_cast<size_t>(u) * L.P + j]);
      for (int r = 0; r < L.R; ++r) out->push_back(T.rep[static_cast<size_t>(u) * L.R + r]);
      break;
    default:
      break;  // SEL and SPEC wait for nothing
  }
}

const char* kind_name(int k) {
  switch (k) {
    case kSel: return "SEL";
    case kSpec: return "SPEC";
    case kRepair: return "REPAIR";
    case kEma: return "EMA";
    case kCombine: return "COMBINE";
    default: return "FIN";
  }
}

// Every item exactly once, in range; every dependency earlier; the lag.  Fills T.
void check_order(const Layout& L, Tickets* T, const char* tag) {
  for (long long t = 0; t < L.total; ++t) {
    const Item it = item_of(L, static_cast<int>(t));
    CHECK(it.unit >= 0 && it.unit < L.U, "%s t %lld: %s unit %d out of range", tag, t, kind_name(it.kind), it.unit);
    if (it.unit < 0 || it.unit >= L.U) continue;
    long long* slot = nullptr;
    const int u = it.unit;
    switch (it.kind) {
      case kSel: slot = it.idx >= 0 && it.idx < L.F ? &T->sel[static_cast<size_t>(u) * L.F + it.idx] : nullptr; break;
      case kFin: slot = &T->fin[u]; break;
      case kEma: slot = &T->ema[u]; break;
      case kSpec: slot = it.idx >= 0 && it.idx < L.P ? &T->spec[static_cast<size_t>(u) * L.P + it.idx] : nullptr; break;
      case kRepair: slot = it.idx >= 0 && it.idx < L.R ? &T->rep[static_cast<size_t>(u) * L.R + it.idx] : nullptr; break;
      case kCombine: slot = it.idx >= 0 && it.idx < L.G ? &T->comb[static_cast<size_t>(u) * L.G + it.idx] : nullptr; break;
    }
    CHECK(slot != nullptr, "%s t %lld: %s index %d out of range", tag, t, kind_name(it.kind), it.idx);
    if (!slot) continue;
    CHECK(*slot < 0, "%s t %lld: %s (%d, %d) handed out twice (first at %lld)", tag, t, kind_name(it.kind), u, it.idx,
          *slot);
    *slot = t;
  }
  const std::vector<long long>* all[6] = {&T->sel, &T->fin, &T->ema, &T->spec, &T->rep, &T->comb};
  for (const auto* v : all)
    for (size_t i = 0; i < v->size(); ++i) CHECK((*v)[i] >= 0, "%s: an item (index %zu) is never handed out", tag, i);

#ifdef SIMULATION_ONLY  // built so, only the grid simulation judges the dependency order
  return;
#endif
  std::vector<long long> deps;
  for (long long t = 0; t < L.total; ++t) {
    const Item it = item_of(L, static_cast<int>(t));
    deps_of(L, *T, it, &deps);
    for (long long d : deps)
      CHECK(d >= 0 && d < t, "%s t %lld: %s of unit %d waits for ticket %lld", tag, t, kind_name(it.kind), it.unit, d);
  }

  // a unit's first dependent ticket trails its last SPEC ticket by at least
  // min(Lc, U - 1 - u) units' SPEC tickets, and Lc units hold two grid rounds
  if (L.P > 0) {
    const int Lc = L.dep_lag < L.U ? L.dep_lag : L.U;
    for (int u = 0; u < L.U; ++u) {
      long long last_spec = -1, first_dep = L.total;
      for (int j = 0; j < L.P; ++j) last_spec = std::max(last_spec, T->spec[static_cast<size_t>(u) * L.P + j]);
      for (int r = 0; r < L.R; ++r) first_dep = std::min(first_dep, T->rep[static_cast<size_t>(u) * L.R + r]);
      for (int h = 0; h < L.G; ++h) first_dep = std::min(first_dep, T->comb[static_cast<size_t>(u) * L.G + h]);
      const long long want = static_cast<long long>(std::min(Lc, L.U - 1 - u)) * L.P;
      CHECK(first_dep - last_spec - 1 >= want, "%s unit %d: %lld tickets between its last SPEC and first dependent, want %lld",
            tag, u, first_dep - last_spec - 1, want);
    }
  }
}

// The grid as the kernel runs it.  `grid` CTAs, at most `resident` of them running at
// once (a CTA starts when a running one exits); a round lets each running CTA try one
// step with probability 1/2.  Returns false on a deadlock (no CTA can move).
bool simulate(const Layout& L, const Tickets& T, long long grid, long long resident, unsigned seed) {
  struct Cta {
    long long cur = -1, next = -1;
    bool started = false, exited = false;
  };
  std::vector<Cta> ctas(static_cast<size_t>(grid));
  std::vector<char> done(static_cast<size_t>(L.total), 0);
  std::mt19937 rng(seed);
  long long counter = 0, finished = 0, running = 0, launched = 0;
  std::vector<long long> deps;
  auto launch_more = [&] {
    while (running < resident && launched < grid) {
      ctas[static_cast<size_t>(launched++)].started = true;
      ++running;
    }
  };
  // One step of CTA c; true if it moved.
  auto step = [&](Cta& c) -> bool {
    if (c.cur < 0) {  // take a ticket (the prefetched one first)
      c.cur = c.next >= 0 ? c.next : counter++;
      c.next = -1;
      if (c.cur >= L.total) {
        c.exited = true;
        --running;
        return true;
      }
      const int k = item_of(L, static_cast<int>(c.cur)).kind;
      if (k == kSel || k == kSpec || k == kRepair) c.next = counter++;
      return true;
    }
    deps_of(L, T, item_of(L, static_cast<int>(c.cur)), &deps);
    for (long long d : deps)
      if (!done[static_cast<size_t>(d)]) return false;
    done[static_cast<size_t>(c.cur)] = 1;
    ++finished;
    c.cur = -1;
    return true;
  };
  launch_more();
  while (finished < L.total || running > 0) {
    bool moved = false;
    for (auto& c : ctas)
      if (c.started && !c.exited && (rng() & 1u)) moved |= step(c);
    if (!moved)
      for (auto& c : ctas)
        if (c.started && !c.exited) moved |= step(c);
    launch_more();
    if (!moved && running > 0) return false;
    if (running == 0 && launched == grid) break;
  }
  return finished == L.total;
}

int run_checks() {
  const int Us[] = {1, 2, 3, 7, 32, 128, 300};
  const int maxnbs[] = {1, 33, 513, 1025, 4100};
  const int Ps[] = {0, 1, 5, 32, 64};
  const int Ks[] = {1, 3, 32, 64};
  const int Gs[] = {1, 4, 8};
  const long long grids[] = {1, 5, 148, 444};
  long long shapes = 0, sims = 0;
  unsigned seed = 1;
  for (int U : Us)
    for (int maxnb : maxnbs)
      for (int P : Ps)
        for (int K : Ks)
          for (int G : Gs)
            for (long long g : grids) {
              const Layout L = make_layout(U, maxnb, P, K, G, g);
              char tag[128];
              std::snprintf(tag, sizeof(tag), "[U %d nb %d P %d K %d G %d grid %lld]", U, maxnb, P, K, G, g);
              Tickets T(L);
              check_order(L, &T, tag);
              ++shapes;
              if (g_failures) goto out;  // one failing shape is enough
              if (P > 0 && L.dep_lag < L.U)
                CHECK(static_cast<long long>(L.dep_lag) * P >= 2 * std::min(g, L.total),
                      "%s: lag of %d units is under two grid rounds", tag, L.dep_lag);
              // simulate the grid on the smaller shapes, fully resident and with a
              // third of it resident
              if (L.total <= 20000 && (U <= 32 || maxnb <= 513)) {
                const long long grid = std::min(g, L.total);
                const long long res[2] = {grid, std::max(1LL, grid / 3)};
                for (long long r : res)
                  for (int s = 0; s < 2; ++s) {
                    CHECK(simulate(L, T, grid, r, seed++), "%s: the simulated grid (%lld resident) deadlocked", tag, r);
                    ++sims;
                  }
              }
              if (g_failures) goto out;
            }
out:
  std::printf("shapes %lld simulations %lld failures %d\n", shapes, sims, g_failures);
  return g_failures == 0 ? 0 : 1;
}

int print_items() {
  int U, maxnb, P, K, G;
  while (std::scanf("%d %d %d %d %d", &U, &maxnb, &P, &K, &G) == 5) {
    const Layout L = make_layout(U, maxnb, P, K, G, 1);
    std::printf("%lld %d %d %lld %lld %lld\n", static_cast<long long>(U) * L.F, U, U, static_cast<long long>(U) * P,
                static_cast<long long>(U) * L.R, static_cast<long long>(U) * G);
  }
  return 0;
}

}  // namespace

int main(int argc, char** argv) {
  if (argc > 1 && std::strcmp(argv[1], "items") == 0) return print_items();
  return run_checks();
}
