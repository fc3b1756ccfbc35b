// Executable models of the expert kernels' synchronisation: the decode
// kernel (decode_tc_kernel: its fused form, gate/up tiles then down tiles in
// one grid, and its two-kernel form) and the prefill grouped GEMM
// (prefill_gemm_kernel), on a run that completes and on a run that aborts.
//
// Every role of every CTA is an actor running the sequence of barrier
// operations that the kernel's code for that role unfolds to.  Copies land,
// and tensor-core commits complete (in issue order, per CTA), as separate
// events.  A scheduler picks one runnable actor or event at random, with a
// random weight per actor per run so that some roles lag far behind.
//
// Barriers are modelled with exact phase numbers; the kernels wait on
// parities.  The model flags any state in which a parity wait would read
// wrongly: a barrier completing phase k + 2 before a waiter has passed its
// wait for phase k (the waiter would miss it), a waiter reaching its wait for
// phase k while the barrier has completed only k - 1 phases (the parity would
// read as complete), and an arrival meant for another phase than the open
// one.  A run ends complete (every actor done, every counter full), in a
// deadlock (nothing runnable), or on such a hazard.
//
// Fused decode, per CTA over its tile list from the real dealing (deal.h):
//   producer   per chunk: wait for the stage's release, start its copy;
//              per down tile: wait for the scale buffer, start the scale
//              copy, then every weight chunk of the tile, then (a new
//              expert) wait for the expert's gate/up counter and a free h
//              buffer and start the h copy
//   decoder g  per down tile: wait for the scales; per chunk of the group:
//              wait for the stage, release it, wait for the chunk's tensor-
//              memory stage, fill it; per down tile: release the scales
//   MMA        per down tile of a new expert: wait for its h; per tile: wait
//              for a free accumulator; per chunk: wait for the filled stage,
//              MMA, commit its release; commit the accumulator; after an
//              expert's last down tile commit its h buffer's release
//   epilogue   per tile: wait for the accumulator, release it; gate/up
//              tiles count themselves in the expert's counter
// The decoders step their shared-memory stage by the group count, which
// equals the chunk index modulo the stage count only when the stage count is
// a multiple of the group count (the kernel's layout guarantees it); the
// model takes the chunk index modulo the stage count, so it covers those
// stage counts only.  The two-kernel form runs the same roles over gate/up
// tiles alone (round robin, no counters), then down tiles alone (a
// contiguous range; h comes from the grid before, and the first tile's
// chunks up to the stage count go out before its h copy).
//
// Prefill, one CTA over its units (chunks j of 64 K in one flat sequence):
//   producer group g (chunks j = g, g + 2, ...): wait for the stage's
//              release, start the B tile copy, wait for the chunk's code
//              stage, fill the A tile, mark the stage full; after its last
//              chunk of a code stage, release the code stage
//   code warp  per code stage: wait for its release, start its copy
//   MMA        per unit: wait for a free accumulator; per chunk: wait for
//              the stage (producers and B copy), MMA, commit its release;
//              commit the accumulator
//   epilogue   per unit: wait for the accumulator, release it
//
// Abort.  Every wait is bounded; once one gives up, the CTA's abort flag
// makes every later wait that is not already satisfied give up at once.
// From then on a wait takes the parity test as the hardware does (phases
// can run ahead of roles that gave up), and only the consequences are
// checked.  A
// role then does what its code does with a failed wait: the decode producer,
// the prefill producers' stage wait and the prefill code warp stop issuing;
// the prefill MMA warp finishes the chunk in hand (as the kernel's loop
// does), commits its accumulator and stops; every other wait is ignored and
// the role carries on.  At the end the kernel drains: for each barrier a
// copy completes, it waits (bounded, not cut short by the flag) for the last
// phase it computes the producer armed there, so that no copy is still
// landing when the CTA exits.  An abort run injects the abort at a random
// step and then checks that a copy never starts into a buffer whose last
// copy is still in flight, that every drain wait is for a phase a copy
// completes, and that no copy is in flight when the CTA's drain ends.
// Releases can be guarded: a consumer releases no buffer a copy refills
// once any of its waits has given up (and the prefill MMA issues nothing
// for a chunk whose stage wait gave up).  Guarding only the release that
// follows the failed wait is not enough: a later wait of the same role can
// pass on a parity that phases running ahead make look complete, and its
// release then frees a buffer whose copy is still in flight.
//
// main() checks the decode model, for many shapes, grids and active-expert
// counts, with the kernel's group and stage counts: every fused run completes
// exactly when stages + 2 x groups >= chunks per down tile (the fused form's
// in-flight capacity condition) and deadlocks otherwise; every run of both
// grids of the two-kernel form completes; four decoder groups sharing three
// tensor-memory stages is flagged as a hazard.  It checks the prefill model
// complete for both code widths over K sizes and unit counts.  Abort runs of
// both kernels must stay clean with guarded releases; without them (the
// consumers' code as it stands) some abort run must show a second copy into
// a buffer that is still filling.  Prints "ok <runs>" or the first failure
// and exits non-zero on a failure.
#include <algorithm>
#include <cstdio>
#include <deque>
#include <functional>
#include <memory>
#include <random>
#include <string>
#include <utility>
#include <vector>

#include "deal.h"

using namespace strata;

namespace {

enum Kind { WAIT, ARRIVE, COPY, COMMIT, CWAIT, CADD, EXIT };
constexpr int kContinue = -1;  // a failed wait: carry on
constexpr int kStop = -2;      // a failed wait: the role ends
constexpr int kNever = -3;     // a drain wait: bounded, not cut short by the abort flag

struct Op {
  Kind k;
  int bar;  // barrier (CWAIT/CADD: counter; EXIT: CTA)
  int ph;   // WAIT: phase awaited; ARRIVE/COPY/COMMIT: phase contributed to; CWAIT: target
  int fail = kContinue;  // WAIT/CWAIT: what a failed wait does (>= 0: run that tail)
  bool gated = false;    // ARRIVE/COMMIT: skipped once any wait of the role gave up
  int cls = -1;          // COPY: the copy's class, for the drain's counts
};

Op W(int b, int ph, int fail = kContinue) { return Op{WAIT, b, ph, fail}; }
Op A(int b, int ph, bool gated = false) { return Op{ARRIVE, b, ph, kContinue, gated}; }
Op M(int b, int ph, bool gated = false) { return Op{COMMIT, b, ph, kContinue, gated}; }
Op C(int b, int ph, int cls) { return Op{COPY, b, ph, kContinue, false, cls}; }

enum Outcome { COMPLETE, DEADLOCK, HAZARD };

const char* outcome_name(Outcome o) {
  return o == COMPLETE ? "complete" : o == DEADLOCK ? "deadlock" : "hazard";
}

// Barriers, counters, actors and the random scheduler.
struct Sim {
  struct Actor {
    Actor(int q, std::string nm) : queue(q), name(std::move(nm)) {}
    int queue;  // the CTA: its commits complete in order
    std::string name;
    std::vector<Op> prog;
    std::vector<std::vector<Op>> tails;  // what a failed wait leads to
    size_t pc = 0, tpc = 0;
    int tail = -1;
    bool stopped = false;
    bool gave_up = false;  // one of its waits gave up
    double w = 1.0;
    // per barrier this actor waits on: the (pc, phase) of each of its waits
    std::vector<std::pair<int, std::vector<std::pair<int, int>>>> waits;
    const Op* cur() const {
      if (stopped) return nullptr;
      if (tail >= 0) return tpc < tails[tail].size() ? &tails[tail][tpc] : nullptr;
      return pc < prog.size() ? &prog[pc] : nullptr;
    }
    bool in_prog() const { return !stopped && tail < 0; }
  };
  std::vector<int> n, arr, cnt, bar_cta, in_flight;
  std::vector<std::string> bar_name;
  std::vector<int> counter, counter_final;
  std::vector<Actor> actors;
  std::vector<std::vector<int>> waiters;                 // barrier -> actors that wait on it
  std::vector<std::deque<std::pair<int, int>>> commits;  // per CTA: (barrier, phase)
  std::vector<std::pair<int, int>> copies;               // in flight: (barrier, phase)
  std::vector<std::vector<int>> issued;                  // per CTA, per class: copies started
  bool aborted = false;
  // called once, after every role has ended in an abort run: adds the drains
  std::function<void(Sim&)> add_drains;
  std::string why;

  int barrier(int cta, const std::string& name, int count) {
    n.push_back(0);
    arr.push_back(0);
    cnt.push_back(count);
    bar_cta.push_back(cta);
    in_flight.push_back(0);
    bar_name.push_back(name);
    waiters.emplace_back();
    return (int)n.size() - 1;
  }
  Actor& actor(int queue, const std::string& name) {
    if ((int)commits.size() <= queue) commits.resize(queue + 1);
    if ((int)issued.size() <= queue) issued.resize(queue + 1, std::vector<int>(8, 0));
    actors.emplace_back(queue, name);
    return actors.back();
  }

  void index_waits(size_t from) {
    for (size_t a = from; a < actors.size(); ++a) {
      Actor& x = actors[a];
      for (size_t pc = 0; pc < x.prog.size(); ++pc) {
        const Op& o = x.prog[pc];
        if (o.k != WAIT) continue;
        auto it = std::find_if(x.waits.begin(), x.waits.end(),
                               [&](const auto& e) { return e.first == o.bar; });
        if (it == x.waits.end()) {
          x.waits.push_back({o.bar, {}});
          it = x.waits.end() - 1;
          waiters[o.bar].push_back((int)a);
        }
        it->second.push_back({(int)pc, o.ph});
      }
    }
  }

  // Before an abort the checks below keep every wait's parity exact, so a
  // wait for phase k passes once k + 1 phases are complete.  After an abort
  // phases can run ahead of waiters that gave up, so the wait takes the
  // hardware's parity test as it is: it passes when the completed-phase
  // count and k differ by an odd number.
  bool satisfied(const Op& o) const {
    if (o.k == WAIT) return aborted ? ((n[o.bar] - o.ph) & 1) != 0 : n[o.bar] >= o.ph + 1;
    if (o.k == CWAIT) return counter[o.bar] >= o.ph;
    return true;
  }
  bool runnable(const Actor& a) const {
    const Op* o = a.cur();
    if (!o) return false;
    if (satisfied(*o)) return true;
    // after an abort a wait gives up at once, except the drain's
    return aborted && o->fail != kNever;
  }

  // An actor standing at a wait for phase k while the barrier has completed
  // k - 1 phases would read the parity as complete.
  bool check_at(const Actor& a) {
    const Op* o = a.cur();
    if (aborted || !o || o->k != WAIT) return true;
    if (n[o->bar] == o->ph - 1) {
      why = a.name + " waits for phase " + std::to_string(o->ph) + " of " + bar_name[o->bar] +
            " with " + std::to_string(n[o->bar]) + " complete: parity reads as complete";
      return false;
    }
    return true;
  }

  // Barrier b has just completed a phase: no waiter still to pass a wait on
  // it may be two behind.
  bool on_complete(int b) {
    if (aborted) return true;
    for (int ai : waiters[b]) {
      const Actor& a = actors[ai];
      if (!a.in_prog()) continue;
      for (const auto& e : a.waits) {
        if (e.first != b) continue;
        auto it = std::lower_bound(e.second.begin(), e.second.end(),
                                   std::make_pair((int)a.pc, -1000000));
        if (it != e.second.end() && n[b] >= it->second + 2) {
          why = bar_name[b] + " completed phase " + std::to_string(n[b] - 1) + " before " +
                a.name + " passed its wait for phase " + std::to_string(it->second);
          return false;
        }
      }
      if (!check_at(a)) return false;
    }
    return true;
  }

  // After an abort an arrival counts toward whatever phase is open.
  bool arrive(int b, int ph) {
    if (!aborted && ph != n[b]) {
      why = "arrival on " + bar_name[b] + " for phase " + std::to_string(ph) + " while phase " +
            std::to_string(n[b]) + " is open";
      return false;
    }
    if (++arr[b] == cnt[b]) {
      arr[b] = 0;
      ++n[b];
      return on_complete(b);
    }
    return true;
  }

  void advance(Actor& a) {
    if (a.tail >= 0) {
      if (++a.tpc >= a.tails[a.tail].size()) a.stopped = true;
    } else {
      ++a.pc;
    }
  }

  // One step of actor a.
  bool step(Actor& a) {
    const Op o = *a.cur();
    switch (o.k) {
      case WAIT:
      case CWAIT:
        if (satisfied(o)) {
          advance(a);
          break;
        }
        a.gave_up = true;
        if (o.fail == kContinue) {
          advance(a);
        } else if (o.fail == kStop) {
          a.stopped = true;
        } else {
          a.tail = o.fail;
          a.tpc = 0;
          if (a.tails[a.tail].empty()) a.stopped = true;
        }
        break;
      case ARRIVE:
      case COMMIT: {
        advance(a);
        if (o.gated && a.gave_up) break;
        if (o.k == COMMIT)
          commits[a.queue].push_back({o.bar, o.ph});
        else if (!arrive(o.bar, o.ph))
          return false;
        break;
      }
      case COPY:
        if (in_flight[o.bar] > 0) {
          why = "a copy into " + bar_name[o.bar] + " (phase " + std::to_string(o.ph) +
                ") starts while the previous one is still in flight";
          return false;
        }
        ++in_flight[o.bar];
        copies.push_back({o.bar, o.ph});
        ++issued[a.queue][o.cls];
        advance(a);
        break;
      case CADD:
        ++counter[o.bar];
        advance(a);
        break;
      case EXIT:
        for (size_t b = 0; b < in_flight.size(); ++b)
          if (bar_cta[b] == o.bar && in_flight[b] > 0) {
            why = "CTA " + std::to_string(o.bar) + " ends its drain with a copy into " +
                  bar_name[b] + " in flight";
            return false;
          }
        advance(a);
        break;
    }
    return check_at(a);
  }

  // abort_at < 0: no abort; else the abort is raised after that many steps.
  Outcome run(unsigned long long seed, long abort_at) {
    index_waits(0);
    std::mt19937_64 rng(seed);
    std::uniform_real_distribution<double> U01(0.0, 1.0);
    for (auto& a : actors) a.w = 0.02 + U01(rng);
    const double w_copy = 0.02 + U01(rng), w_commit = 0.02 + U01(rng);
    std::vector<int> cand;
    std::vector<double> wt;
    bool drains = false;
    for (long steps = 0;; ++steps) {
      if (abort_at >= 0 && steps == abort_at) aborted = true;
      if (aborted && !drains && add_drains) {
        // the drains start once every role has ended (the kernel's
        // __syncthreads); commits and copies may still be completing
        bool roles_done = true;
        for (const auto& a : actors) roles_done = roles_done && !a.cur();
        if (roles_done) {
          drains = true;
          const size_t from = actors.size();
          add_drains(*this);
          index_waits(from);
          for (size_t a = from; a < actors.size(); ++a) actors[a].w = 0.02 + U01(rng);
        }
      }
      cand.clear();
      wt.clear();
      for (size_t a = 0; a < actors.size(); ++a)
        if (runnable(actors[a])) {
          cand.push_back((int)a);
          wt.push_back(actors[a].w);
        }
      if (!copies.empty()) {
        cand.push_back(-1);
        wt.push_back(w_copy);
      }
      for (size_t c = 0; c < commits.size(); ++c)
        if (!commits[c].empty()) {
          cand.push_back(-2 - (int)c);
          wt.push_back(w_commit);
        }
      if (cand.empty()) break;
      double tot = 0;
      for (double w : wt) tot += w;
      double r = U01(rng) * tot;
      size_t pick = 0;
      while (pick + 1 < cand.size() && r >= wt[pick]) r -= wt[pick++];
      const int who = cand[pick];
      if (who == -1) {  // one copy in flight lands
        const size_t j = (size_t)(U01(rng) * copies.size()) % copies.size();
        const auto c = copies[j];
        copies[j] = copies.back();
        copies.pop_back();
        --in_flight[c.first];
        if (!arrive(c.first, c.second)) return HAZARD;
        continue;
      }
      if (who <= -2) {  // the oldest commit of a CTA completes
        auto& q = commits[-2 - who];
        const auto c = q.front();
        q.pop_front();
        if (!arrive(c.first, c.second)) return HAZARD;
        continue;
      }
      if (!step(actors[who])) return HAZARD;
    }
    for (const auto& a : actors)
      if (const Op* o = a.cur()) {
        if (o->fail == kNever) {
          why = a.name + " waits for phase " + std::to_string(o->ph) + " of " +
                bar_name[o->bar] + ", which no copy completes";
          return HAZARD;
        }
        why = a.name + " stuck at " +
              (o->k == CWAIT ? "counter " + std::to_string(o->bar)
                             : "phase " + std::to_string(o->ph) + " of " + bar_name[o->bar]);
        return DEADLOCK;
      }
    if (!aborted)
      for (size_t u = 0; u < counter.size(); ++u)
        if (counter[u] != counter_final[u]) {
          why = "counter " + std::to_string(u) + " ends at " + std::to_string(counter[u]);
          return HAZARD;
        }
    return COMPLETE;
  }

  size_t total_ops() const {
    size_t t = 0;
    for (const auto& a : actors) t += a.prog.size();
    return t;
  }
};

// ---------------------------------------------------------------- decode
struct DecodeParams {
  int G, U, H, I, S, groups, TS, KC;
  int mode;      // 2 fused; 0 gate/up alone, 1 down alone (h from the grid before)
  bool guarded;  // no buffer released once a wait of the role gave up
};

enum { kClsChunk, kClsScale, kClsH, kClsCode, kClsB0, kClsB1 };

void build_decode(Sim& m, const DecodeParams& p) {
  const int nchA = p.H / p.KC, nchB = (p.I + p.KC - 1) / p.KC;
  const int tpeA = p.I / 64, tpeB = p.H / 128;
  m.counter.assign(p.U, 0);
  m.counter_final.assign(p.U, p.mode == 2 ? tpeA : 0);
  const TcDeal d = tc_deal(p.G, p.U, p.H, p.I);
  std::vector<int> bcnt(p.G);
  for (int c = 0; c < p.G; ++c) bcnt[c] = tc_deal_bstart(d, c + 1) - tc_deal_bstart(d, c);
  struct Bars {
    std::vector<int> full, bfull, sfull;
  };
  auto bars = std::make_shared<std::vector<Bars>>(p.G);
  for (int cta = 0; cta < p.G; ++cta) {
    const std::string cn = "CTA " + std::to_string(cta) + " ";
    auto ring = [&](const char* name, int k, int count) {
      std::vector<int> v;
      for (int i = 0; i < k; ++i)
        v.push_back(m.barrier(cta, cn + name + "[" + std::to_string(i) + "]", count));
      return v;
    };
    const auto full = ring("full", p.S, 1), empty = ring("empty", p.S, 1);
    const auto tfull = ring("tfull", p.TS, 1), tempty = ring("tempty", p.TS, 1);
    const auto afull = ring("afull", 2, 1), aempty = ring("aempty", 2, 1);
    const auto sfull = ring("sfull", 2, 1), sempty = ring("sempty", 2, p.groups);
    const auto bfull = ring("bfull", 2, 1), bempty = ring("bempty", 2, 1);
    (*bars)[cta] = Bars{full, bfull, sfull};

    // the CTA's tiles: (gate/up?, active expert).  Fused: the dealing;
    // gate/up alone: round robin; down alone: a contiguous range.
    std::vector<std::pair<bool, int>> tiles;
    int nA = 0;
    if (p.mode == 2) {
      nA = d.q + (cta < d.r ? 1 : 0);
      for (int i = 0; i < nA; ++i) tiles.push_back({true, (cta + i * p.G) / tpeA});
      for (int kk = 0; kk < bcnt[cta]; ++kk)
        tiles.push_back({false, tc_deal_down_tile(d, bcnt.data(), cta, kk) / tpeB});
    } else if (p.mode == 0) {
      for (int j = cta; j < d.ntA; j += p.G) tiles.push_back({true, j / tpeA});
      nA = (int)tiles.size();
    } else {
      const int b0 = (int)((long long)d.ntB * cta / p.G);
      const int b1 = (int)((long long)d.ntB * (cta + 1) / p.G);
      for (int j = b0; j < b1; ++j) tiles.push_back({false, j / tpeB});
    }
    const int T = (int)tiles.size();

    {  // producer: stops at its first failed wait
      auto& prog = m.actor(cta, cn + "producer").prog;
      int gc = 0, bseq = -1, prev = -1, ib = 0;
      auto chunk = [&]() {
        prog.push_back(W(empty[gc % p.S], gc / p.S - 1, kStop));
        prog.push_back(C(full[gc % p.S], gc / p.S, kClsChunk));
        ++gc;
      };
      for (int i = 0; i < T; ++i) {
        if (tiles[i].first) {
          for (int c = 0; c < nchA; ++c) chunk();
          continue;
        }
        const int u = tiles[i].second;
        prog.push_back(W(sempty[ib & 1], (ib >> 1) - 1, kStop));
        prog.push_back(C(sfull[ib & 1], ib >> 1, kClsScale));
        auto load_h = [&]() {
          prog.push_back(W(bempty[(bseq + 1) & 1], ((bseq + 1) >> 1) - 1, kStop));
          ++bseq;
          prog.push_back(C(bfull[bseq & 1], bseq >> 1, kClsH));
        };
        const bool new_h = ib == 0 || u != prev;
        if (p.mode == 1) {
          // the first tile's chunks up to the stage count go out before h
          const int pre = ib == 0 ? std::min(nchB, p.S) : 0;
          for (int c = 0; c < pre; ++c) chunk();
          if (new_h) load_h();
          for (int c = pre; c < nchB; ++c) chunk();
        } else {
          for (int c = 0; c < nchB; ++c) chunk();
          if (new_h) {
            prog.push_back(Op{CWAIT, u, tpeA, kStop});
            load_h();
          }
        }
        prev = u;
        ++ib;
      }
    }
    for (int g = 0; g < p.groups; ++g) {  // decoders: carry on past failed waits
      auto& prog = m.actor(cta, cn + "decoder group " + std::to_string(g)).prog;
      int gc = 0, ib = 0;
      for (int i = 0; i < T; ++i) {
        const bool isA = tiles[i].first;
        const int nch = isA ? nchA : nchB;
        if (!isA) prog.push_back(W(sfull[ib & 1], ib >> 1));
        for (int c = 0; c < nch; ++c) {
          const int x = gc + c;
          if (x % p.groups != g) continue;
          prog.push_back(W(full[x % p.S], x / p.S));
          prog.push_back(A(empty[x % p.S], x / p.S, p.guarded));
          prog.push_back(W(tempty[x % p.TS], x / p.TS - 1));
          prog.push_back(A(tfull[x % p.TS], x / p.TS));
        }
        gc += nch;
        if (!isA) {
          prog.push_back(A(sempty[ib & 1], ib >> 1, p.guarded));
          ++ib;
        }
      }
    }
    {  // MMA: carries on past failed waits
      auto& prog = m.actor(cta, cn + "MMA").prog;
      int gc = 0, bseq = -1, prev = -1;
      for (int i = 0; i < T; ++i) {
        const bool isA = tiles[i].first;
        const int u = tiles[i].second;
        if (!isA) {
          if (i == nA || u != prev) {
            ++bseq;
            prog.push_back(W(bfull[bseq & 1], bseq >> 1));
          }
          prev = u;
        }
        prog.push_back(W(aempty[i & 1], (i >> 1) - 1));
        const int nch = isA ? nchA : nchB;
        for (int c = 0; c < nch; ++c, ++gc) {
          prog.push_back(W(tfull[gc % p.TS], gc / p.TS));
          prog.push_back(M(tempty[gc % p.TS], gc / p.TS));
        }
        prog.push_back(M(afull[i & 1], i >> 1));
        if (!isA && (i + 1 == T || tiles[i + 1].second != u))
          prog.push_back(M(bempty[bseq & 1], bseq >> 1, p.guarded));
      }
    }
    {  // epilogue: carries on past failed waits
      auto& prog = m.actor(cta, cn + "epilogue").prog;
      for (int i = 0; i < T; ++i) {
        prog.push_back(W(afull[i & 1], i >> 1));
        prog.push_back(A(aempty[i & 1], i >> 1));
        if (p.mode == 2 && tiles[i].first) prog.push_back(Op{CADD, tiles[i].second, 1});
      }
    }
  }
  // The drain: the last armed phase of every stage, h buffer and scale
  // buffer, from the producer's counts, as the kernel computes it.
  const int S = p.S;
  m.add_drains = [bars, S](Sim& s) {
    for (int cta = 0; cta < (int)bars->size(); ++cta) {
      const Bars& b = (*bars)[cta];
      const int gc = s.issued[cta][kClsChunk], nh = s.issued[cta][kClsH],
                nsc = s.issued[cta][kClsScale];
      auto& prog = s.actor(cta, "CTA " + std::to_string(cta) + " drain").prog;
      for (int st = 0; st < S && st < gc; ++st) {
        const int ph = (gc - 1 - st) / S;
        if (last_armed_parity(gc, S, st) != (ph & 1)) std::printf("drain parity mismatch\n");
        prog.push_back(W(b.full[st], ph, kNever));
      }
      for (int x = 0; x < 2 && x < nh; ++x)
        prog.push_back(W(b.bfull[x], last_item_of_buffer(nh, x) >> 1, kNever));
      for (int x = 0; x < 2 && x < nsc; ++x)
        prog.push_back(W(b.sfull[x], last_item_of_buffer(nsc, x) >> 1, kNever));
      prog.push_back(Op{EXIT, cta, 0});
    }
  };
}

// ---------------------------------------------------------------- prefill
struct PrefillParams {
  int units, K, CPC, S, CSN;  // units of this CTA, K, chunks per code stage, stages
  bool guarded;
};

void build_prefill(Sim& m, const PrefillParams& p) {
  const int KC = p.K / 64, CSU = (KC + p.CPC - 1) / p.CPC, nchunks = p.units * KC;
  auto ring = [&](const char* name, int k, int count) {
    std::vector<int> v;
    for (int i = 0; i < k; ++i)
      v.push_back(m.barrier(0, std::string(name) + "[" + std::to_string(i) + "]", count));
    return v;
  };
  // arrivals per phase: full one producer group, cempty both groups, tempty
  // the epilogue; the rest one copy or one commit
  const auto full = ring("full", p.S, 1), empty = ring("empty", p.S, 1);
  const auto bfull = ring("bfull", p.S, 1);
  const auto tfull = ring("tfull", 2, 1), tempty = ring("tempty", 2, 1);
  const auto cfull = ring("cfull", p.CSN, 1), cempty = ring("cempty", p.CSN, 2);
  for (int g = 0; g < 2; ++g) {
    // a producer group stops when its stage wait gives up, carries on past a
    // failed code-stage wait
    auto& prog = m.actor(0, "producer group " + std::to_string(g)).prog;
    for (int j = g; j < nchunks; j += 2) {
      const int ui = j / KC, kc = j % KC, s = j % p.S;
      prog.push_back(W(empty[s], j / p.S - 1, kStop));
      prog.push_back(C(bfull[s], j / p.S, g == 0 ? kClsB0 : kClsB1));
      const int gcs = ui * CSU + kc / p.CPC, slot = kc % p.CPC, ci = gcs % p.CSN;
      prog.push_back(W(cfull[ci], gcs / p.CSN));
      prog.push_back(A(full[s], j / p.S));
      const int in_cs = std::min(p.CPC, KC - (kc / p.CPC) * p.CPC);
      if (slot + 2 >= in_cs) prog.push_back(A(cempty[ci], gcs / p.CSN, p.guarded));
    }
  }
  {  // the code warp stops at its first failed wait
    auto& prog = m.actor(0, "code warp").prog;
    for (int gcs = 0; gcs < p.units * CSU; ++gcs) {
      prog.push_back(W(cempty[gcs % p.CSN], gcs / p.CSN - 1, kStop));
      prog.push_back(C(cfull[gcs % p.CSN], gcs / p.CSN, kClsCode));
    }
  }
  {
    // MMA: a failed accumulator wait skips the unit's chunks; a failed stage
    // wait finishes that chunk (MMA, release; guarded: neither); both then
    // commit the accumulator and end the loop
    auto& a = m.actor(0, "MMA");
    auto& prog = a.prog;
    int it_k = 0;
    for (int it = 0; it < p.units; ++it) {
      a.tails.push_back({M(tfull[it & 1], it >> 1)});
      const int t_acc = (int)a.tails.size() - 1;
      prog.push_back(W(tempty[it & 1], (it >> 1) - 1, t_acc));
      for (int kc = 0; kc < KC; ++kc, ++it_k) {
        const int s = it_k % p.S;
        if (p.guarded)
          a.tails.push_back({M(tfull[it & 1], it >> 1)});
        else
          a.tails.push_back({M(empty[s], it_k / p.S), M(tfull[it & 1], it >> 1)});
        const int t_chunk = (int)a.tails.size() - 1;
        prog.push_back(W(full[s], it_k / p.S, t_chunk));
        prog.push_back(W(bfull[s], it_k / p.S, t_chunk));
        prog.push_back(M(empty[s], it_k / p.S));
      }
      prog.push_back(M(tfull[it & 1], it >> 1));
    }
  }
  {  // epilogue: carries on past failed waits
    auto& prog = m.actor(0, "epilogue").prog;
    for (int it = 0; it < p.units; ++it) {
      prog.push_back(W(tfull[it & 1], it >> 1));
      prog.push_back(A(tempty[it & 1], it >> 1));
    }
  }
  // The drain: each producer group's last S / 2 B copies (its stages), and
  // the last armed phase of every code stage.
  const int S = p.S, CSN = p.CSN;
  m.add_drains = [bfull, cfull, S, CSN](Sim& s) {
    auto& prog = s.actor(0, "drain").prog;
    for (int g = 0; g < 2; ++g) {
      const int nb = s.issued[0][g == 0 ? kClsB0 : kClsB1];
      for (int i = nb - 1; i >= 0 && i >= nb - S / 2; --i) {
        const int j = g + 2 * i;
        prog.push_back(W(bfull[j % S], j / S, kNever));
      }
    }
    const int ncs = s.issued[0][kClsCode];
    for (int c = 0; c < CSN && c < ncs; ++c) {
      const int ph = (ncs - 1 - c) / CSN;
      if (last_armed_parity(ncs, CSN, c) != (ph & 1)) std::printf("drain parity mismatch\n");
      prog.push_back(W(cfull[c], ph, kNever));
    }
    prog.push_back(Op{EXIT, 0, 0});
  };
}

template <typename P, typename B>
Outcome run_model(const P& p, B build, unsigned long long seed, bool abort, std::string* why) {
  Sim m;
  build(m, p);
  long at = -1;
  if (abort) {
    std::mt19937_64 r(seed ^ 0x9e3779b97f4a7c15ull);
    at = (long)(r() % (2 * m.total_ops() + 1));
  }
  const Outcome o = m.run(seed, at);
  *why = m.why;
  return o;
}

Outcome run_decode(const DecodeParams& p, unsigned long long seed, std::string* why,
                   bool abort = false) {
  return run_model(p, build_decode, seed, abort, why);
}
Outcome run_prefill(const PrefillParams& p, unsigned long long seed, std::string* why,
                    bool abort = false) {
  return run_model(p, build_prefill, seed, abort, why);
}

}  // namespace

int main() {
  long runs = 0;
  std::string why;
  // Fused decode with the kernel's counts: three decoder groups of four
  // warps, one tensor-memory A stage per group, 256-K chunks, shared-memory
  // stages a multiple of the group count up to 16.
  const int groups = 3, TS = 3, KC = 256;
  const int shapes[][2] = {{256, 128}, {512, 384}, {1024, 640}, {2560, 640},
                           {2048, 1408}, {4096, 2048}, {512, 3072}, {256, 4096}};
  const int grids[] = {1, 2, 3, 5, 8};
  const int actives[] = {1, 2, 3, 7};
  for (const auto& s : shapes)
    for (int G : grids)
      for (int U : actives)
        for (int S = groups; S <= 15; S += groups) {
          const DecodeParams p{G, U, s[0], s[1], S, groups, TS, KC, 2, false};
          const int nchB = (s[1] + KC - 1) / KC;
          // U >= 1 active experts: some CTA has a down tile
          const bool fits = S + 2 * groups >= nchB;
          const int seeds = (s[0] >= 2048 || s[1] >= 2048) ? 2 : 4;
          for (int k = 0; k < seeds; ++k) {
            const Outcome o = run_decode(p, 1000003ull * (unsigned long long)runs + 17, &why);
            ++runs;
            if (o != (fits ? COMPLETE : DEADLOCK)) {
              std::printf("FAIL decode G=%d U=%d H=%d I=%d S=%d: %s, expected %s (%s)\n", G, U,
                          s[0], s[1], S, outcome_name(o), fits ? "complete" : "deadlock",
                          why.c_str());
              return 1;
            }
          }
        }
  // Four decoder groups over three tensor-memory stages: a group can reach a
  // stage's barrier two phases ahead.  Some random schedule must show it.
  {
    bool seen = false;
    for (int k = 0; k < 200 && !seen; ++k) {
      const DecodeParams p{2, 3, 2560, 640, 12, 4, 3, KC, 2, false};
      seen = run_decode(p, 77 + k, &why) == HAZARD;
      ++runs;
    }
    if (!seen) {
      std::printf("FAIL decode: four groups on three tensor-memory stages never flagged\n");
      return 1;
    }
    std::printf("flagged as expected: %s\n", why.c_str());
  }
  // The two-kernel form (where the fused one does not fit): both grids
  // complete for every stage count.
  for (const auto& s : shapes)
    for (int G : {1, 3, 8})
      for (int U : {1, 3, 7})
        for (int S = groups; S <= 15; S += groups)
          for (int mode = 0; mode < 2; ++mode) {
            const DecodeParams p{G, U, s[0], s[1], S, groups, TS, KC, mode, false};
            const Outcome o = run_decode(p, 3000017ull * (unsigned long long)runs + 3, &why);
            ++runs;
            if (o != COMPLETE) {
              std::printf("FAIL decode mode %d G=%d U=%d H=%d I=%d S=%d: %s (%s)\n", mode, G, U,
                          s[0], s[1], S, outcome_name(o), why.c_str());
              return 1;
            }
          }
  // Prefill with the kernel's counts: four A/B stages, three code stages,
  // two producer groups; 4 chunks per code stage for 2-bit codes, 2 for
  // 4-bit; K a multiple of 128 (H and I are).
  const int Ks[] = {128, 256, 384, 640, 2048, 2560, 4096};
  const int unit_counts[] = {1, 2, 3, 5, 8};
  for (int K : Ks)
    for (int CPC : {2, 4})
      for (int units : unit_counts)
        for (int k = 0; k < 6; ++k) {
          const PrefillParams p{units, K, CPC, 4, 3, false};
          const Outcome o = run_prefill(p, 2000003ull * (unsigned long long)runs + 5, &why);
          ++runs;
          if (o != COMPLETE) {
            std::printf("FAIL prefill K=%d CPC=%d units=%d: %s (%s)\n", K, CPC, units,
                        outcome_name(o), why.c_str());
            return 1;
          }
        }
  // Aborts.  Guarded releases: every abort run of both kernels stays clean.
  // As the consumers' code stands (releases after a failed wait), some abort
  // run starts a copy into a buffer that is still filling.
  for (bool guarded : {true, false}) {
    long bad = 0, n_abort = 0;
    std::string first;
    for (const auto& s : shapes)
      for (int G : {1, 3})
        for (int U : {1, 3})
          for (int S : {3, 6, 12})
            for (int mode : {2, 0, 1}) {
              const int nchB = (s[1] + KC - 1) / KC;
              if (mode == 2 && S + 2 * groups < nchB) continue;  // not a fused shape
              const DecodeParams p{G, U, s[0], s[1], S, groups, TS, KC, mode, guarded};
              for (int k = 0; k < 4; ++k) {
                const Outcome o =
                    run_decode(p, 4000037ull * (unsigned long long)runs + 11, &why, true);
                ++runs;
                ++n_abort;
                if (o != COMPLETE && !bad++)
                  first = "decode mode " + std::to_string(mode) + " H=" + std::to_string(s[0]) +
                          " I=" + std::to_string(s[1]) + " S=" + std::to_string(S) + ": " +
                          outcome_name(o) + " (" + why + ")";
              }
            }
    for (int K : Ks)
      for (int CPC : {2, 4})
        for (int units : {1, 2, 5})
          for (int k = 0; k < 8; ++k) {
            const PrefillParams p{units, K, CPC, 4, 3, guarded};
            const Outcome o =
                run_prefill(p, 5000011ull * (unsigned long long)runs + 7, &why, true);
            ++runs;
            ++n_abort;
            if (o != COMPLETE && !bad++)
              first = "prefill K=" + std::to_string(K) + " CPC=" + std::to_string(CPC) +
                      " units=" + std::to_string(units) + ": " + outcome_name(o) + " (" + why +
                      ")";
          }
    if (guarded && bad) {
      std::printf("FAIL abort with guarded releases: %ld of %ld runs, first %s\n", bad, n_abort,
                  first.c_str());
      return 1;
    }
    if (!guarded) {
      if (!bad) {
        std::printf("FAIL abort with unguarded releases: no run flagged\n");
        return 1;
      }
      std::printf("unguarded releases after an abort: %ld of %ld runs flagged, first %s\n", bad,
                  n_abort, first.c_str());
    }
  }
  std::printf("ok %ld\n", runs);
  return 0;
}
