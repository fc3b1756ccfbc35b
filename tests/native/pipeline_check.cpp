// Executable models of the expert kernels' synchronisation: the decode
// kernel (decode_tc_kernel: its fused form, gate/up tiles then down tiles in
// one grid, and its two-kernel form) and the prefill grouped GEMM
// (prefill_gemm_kernel).
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
// stage counts only.
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
// The decode kernel's two-kernel form runs the same roles over gate/up tiles
// alone (round robin, no counters), then down tiles alone (a contiguous
// range; h comes from the grid before, and the first tile's chunks up to the
// stage count go out before its h copy).
//
// main() checks the decode model, for many shapes, grids and active-expert
// counts, with the kernel's group and stage counts: every fused run completes
// exactly when stages + 2 x groups >= chunks per down tile (the fused form's
// in-flight capacity condition) and deadlocks otherwise; every run of both
// grids of the two-kernel form completes; four decoder groups sharing three
// tensor-memory stages is flagged as a hazard.  It checks the prefill model
// complete for both code widths over K sizes and unit counts.
// Prints "ok <runs>" or the first failure and exits non-zero on a failure.
#include <algorithm>
#include <cstdio>
#include <deque>
#include <random>
#include <string>
#include <utility>
#include <vector>

#include "deal.h"

using namespace strata;

namespace {

enum Kind { WAIT, ARRIVE, COPY, COMMIT, CWAIT, CADD };
struct Op {
  Kind k;
  int bar;  // barrier (CWAIT/CADD: counter)
  int ph;   // WAIT: phase awaited; ARRIVE/COPY/COMMIT: phase contributed to; CWAIT: target
};

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
    size_t pc = 0;
    double w = 1.0;
    // per barrier this actor waits on: the (pc, phase) of each of its waits
    std::vector<std::pair<int, std::vector<std::pair<int, int>>>> waits;
  };
  std::vector<int> n, arr, cnt;  // per barrier: phases completed, arrivals, arrivals per phase
  std::vector<std::string> bar_name;
  std::vector<int> counter, counter_final;
  std::vector<Actor> actors;
  std::vector<std::vector<int>> waiters;                 // barrier -> actors that wait on it
  std::vector<std::deque<std::pair<int, int>>> commits;  // per CTA: (barrier, phase)
  std::vector<std::pair<int, int>> copies;               // in flight: (barrier, phase)
  std::string why;

  int barrier(const std::string& name, int count) {
    n.push_back(0);
    arr.push_back(0);
    cnt.push_back(count);
    bar_name.push_back(name);
    waiters.emplace_back();
    return (int)n.size() - 1;
  }
  Actor& actor(int queue, const std::string& name) {
    if ((int)commits.size() <= queue) commits.resize(queue + 1);
    actors.emplace_back(queue, name);
    return actors.back();
  }

  void index_waits() {
    for (size_t a = 0; a < actors.size(); ++a) {
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

  bool runnable(const Actor& a) const {
    if (a.pc >= a.prog.size()) return false;
    const Op& o = a.prog[a.pc];
    if (o.k == WAIT) return n[o.bar] >= o.ph + 1;
    if (o.k == CWAIT) return counter[o.bar] >= o.ph;
    return true;
  }

  // An actor standing at a wait for phase k while the barrier has completed
  // k - 1 phases would read the parity as complete.
  bool check_at(const Actor& a) {
    if (a.pc >= a.prog.size()) return true;
    const Op& o = a.prog[a.pc];
    if (o.k == WAIT && n[o.bar] == o.ph - 1) {
      why = a.name + " waits for phase " + std::to_string(o.ph) + " of " + bar_name[o.bar] +
            " with " + std::to_string(n[o.bar]) + " complete: parity reads as complete";
      return false;
    }
    return true;
  }

  // Barrier b has just completed a phase: no waiter may be two behind.
  bool on_complete(int b) {
    for (int ai : waiters[b]) {
      const Actor& a = actors[ai];
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

  bool arrive(int b, int ph) {
    if (ph != n[b]) {
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

  Outcome run(unsigned long long seed) {
    index_waits();
    std::mt19937_64 rng(seed);
    std::uniform_real_distribution<double> U01(0.0, 1.0);
    for (auto& a : actors) a.w = 0.02 + U01(rng);
    const double w_copy = 0.02 + U01(rng), w_commit = 0.02 + U01(rng);
    std::vector<int> cand;
    std::vector<double> wt;
    for (;;) {
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
      Actor& a = actors[who];
      const Op o = a.prog[a.pc++];
      switch (o.k) {
        case WAIT:
        case CWAIT:
          break;
        case ARRIVE:
          if (!arrive(o.bar, o.ph)) return HAZARD;
          break;
        case COPY:
          copies.push_back({o.bar, o.ph});
          break;
        case COMMIT:
          commits[a.queue].push_back({o.bar, o.ph});
          break;
        case CADD:
          ++counter[o.bar];
          break;
      }
      if (!check_at(a)) return HAZARD;
    }
    for (const auto& a : actors)
      if (a.pc < a.prog.size()) {
        const Op& o = a.prog[a.pc];
        why = a.name + " stuck at " +
              (o.k == CWAIT ? "counter " + std::to_string(o.bar)
                            : "phase " + std::to_string(o.ph) + " of " + bar_name[o.bar]);
        return DEADLOCK;
      }
    for (size_t u = 0; u < counter.size(); ++u)
      if (counter[u] != counter_final[u]) {
        why = "counter " + std::to_string(u) + " ends at " + std::to_string(counter[u]);
        return HAZARD;
      }
    return COMPLETE;
  }
};

// ---------------------------------------------------------------- fused decode
struct DecodeParams {
  int G, U, H, I, S, groups, TS, KC;
  int mode;  // 2 fused; 0 gate/up alone, 1 down alone (h from the grid before)
};

void build_decode(Sim& m, const DecodeParams& p) {
  const int nchA = p.H / p.KC, nchB = (p.I + p.KC - 1) / p.KC;
  const int tpeA = p.I / 64, tpeB = p.H / 128;
  m.counter.assign(p.U, 0);
  m.counter_final.assign(p.U, p.mode == 2 ? tpeA : 0);
  const TcDeal d = tc_deal(p.G, p.U, p.H, p.I);
  std::vector<int> bcnt(p.G);
  for (int c = 0; c < p.G; ++c) bcnt[c] = tc_deal_bstart(d, c + 1) - tc_deal_bstart(d, c);
  for (int cta = 0; cta < p.G; ++cta) {
    const std::string cn = "CTA " + std::to_string(cta) + " ";
    auto ring = [&](const char* name, int k, int count) {
      std::vector<int> v;
      for (int i = 0; i < k; ++i)
        v.push_back(m.barrier(cn + name + "[" + std::to_string(i) + "]", count));
      return v;
    };
    const auto full = ring("full", p.S, 1), empty = ring("empty", p.S, 1);
    const auto tfull = ring("tfull", p.TS, 1), tempty = ring("tempty", p.TS, 1);
    const auto afull = ring("afull", 2, 1), aempty = ring("aempty", 2, 1);
    const auto sfull = ring("sfull", 2, 1), sempty = ring("sempty", 2, p.groups);
    const auto bfull = ring("bfull", 2, 1), bempty = ring("bempty", 2, 1);

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

    {
      auto& prog = m.actor(cta, cn + "producer").prog;
      int gc = 0, bseq = -1, prev = -1, ib = 0;
      auto chunk = [&]() {
        prog.push_back({WAIT, empty[gc % p.S], gc / p.S - 1});
        prog.push_back({COPY, full[gc % p.S], gc / p.S});
        ++gc;
      };
      for (int i = 0; i < T; ++i) {
        if (tiles[i].first) {
          for (int c = 0; c < nchA; ++c) chunk();
          continue;
        }
        const int u = tiles[i].second;
        prog.push_back({WAIT, sempty[ib & 1], (ib >> 1) - 1});
        prog.push_back({COPY, sfull[ib & 1], ib >> 1});
        auto load_h = [&]() {
          prog.push_back({WAIT, bempty[(bseq + 1) & 1], ((bseq + 1) >> 1) - 1});
          ++bseq;
          prog.push_back({COPY, bfull[bseq & 1], bseq >> 1});
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
            prog.push_back({CWAIT, u, tpeA});
            load_h();
          }
        }
        prev = u;
        ++ib;
      }
    }
    for (int g = 0; g < p.groups; ++g) {
      auto& prog = m.actor(cta, cn + "decoder group " + std::to_string(g)).prog;
      int gc = 0, ib = 0;
      for (int i = 0; i < T; ++i) {
        const bool isA = tiles[i].first;
        const int nch = isA ? nchA : nchB;
        if (!isA) prog.push_back({WAIT, sfull[ib & 1], ib >> 1});
        for (int c = 0; c < nch; ++c) {
          const int x = gc + c;
          if (x % p.groups != g) continue;
          prog.push_back({WAIT, full[x % p.S], x / p.S});
          prog.push_back({ARRIVE, empty[x % p.S], x / p.S});
          prog.push_back({WAIT, tempty[x % p.TS], x / p.TS - 1});
          prog.push_back({ARRIVE, tfull[x % p.TS], x / p.TS});
        }
        gc += nch;
        if (!isA) {
          prog.push_back({ARRIVE, sempty[ib & 1], ib >> 1});
          ++ib;
        }
      }
    }
    {
      auto& prog = m.actor(cta, cn + "MMA").prog;
      int gc = 0, bseq = -1, prev = -1;
      for (int i = 0; i < T; ++i) {
        const bool isA = tiles[i].first;
        const int u = tiles[i].second;
        if (!isA) {
          if (i == nA || u != prev) {
            ++bseq;
            prog.push_back({WAIT, bfull[bseq & 1], bseq >> 1});
          }
          prev = u;
        }
        prog.push_back({WAIT, aempty[i & 1], (i >> 1) - 1});
        const int nch = isA ? nchA : nchB;
        for (int c = 0; c < nch; ++c, ++gc) {
          prog.push_back({WAIT, tfull[gc % p.TS], gc / p.TS});
          prog.push_back({COMMIT, tempty[gc % p.TS], gc / p.TS});
        }
        prog.push_back({COMMIT, afull[i & 1], i >> 1});
        if (!isA && (i + 1 == T || tiles[i + 1].second != u))
          prog.push_back({COMMIT, bempty[bseq & 1], bseq >> 1});
      }
    }
    {
      auto& prog = m.actor(cta, cn + "epilogue").prog;
      for (int i = 0; i < T; ++i) {
        prog.push_back({WAIT, afull[i & 1], i >> 1});
        prog.push_back({ARRIVE, aempty[i & 1], i >> 1});
        if (p.mode == 2 && tiles[i].first) prog.push_back({CADD, tiles[i].second, 1});
      }
    }
  }
}

Outcome run_decode(const DecodeParams& p, unsigned long long seed, std::string* why) {
  Sim m;
  build_decode(m, p);
  const Outcome o = m.run(seed);
  *why = m.why;
  return o;
}

// ---------------------------------------------------------------- prefill
struct PrefillParams {
  int units, K, CPC, S, CSN;  // units of this CTA, K, chunks per code stage, stages
};

void build_prefill(Sim& m, const PrefillParams& p) {
  const int KC = p.K / 64, CSU = (KC + p.CPC - 1) / p.CPC, nchunks = p.units * KC;
  auto ring = [&](const char* name, int k, int count) {
    std::vector<int> v;
    for (int i = 0; i < k; ++i)
      v.push_back(m.barrier(std::string(name) + "[" + std::to_string(i) + "]", count));
    return v;
  };
  // arrivals per phase: full one producer group, cempty both groups, tempty
  // the epilogue; the rest one copy or one commit
  const auto full = ring("full", p.S, 1), empty = ring("empty", p.S, 1);
  const auto bfull = ring("bfull", p.S, 1);
  const auto tfull = ring("tfull", 2, 1), tempty = ring("tempty", 2, 1);
  const auto cfull = ring("cfull", p.CSN, 1), cempty = ring("cempty", p.CSN, 2);
  for (int g = 0; g < 2; ++g) {
    auto& prog = m.actor(0, "producer group " + std::to_string(g)).prog;
    for (int j = g; j < nchunks; j += 2) {
      const int ui = j / KC, kc = j % KC, s = j % p.S;
      prog.push_back({WAIT, empty[s], j / p.S - 1});
      prog.push_back({COPY, bfull[s], j / p.S});
      const int gcs = ui * CSU + kc / p.CPC, slot = kc % p.CPC, ci = gcs % p.CSN;
      prog.push_back({WAIT, cfull[ci], gcs / p.CSN});
      prog.push_back({ARRIVE, full[s], j / p.S});
      const int in_cs = std::min(p.CPC, KC - (kc / p.CPC) * p.CPC);
      if (slot + 2 >= in_cs) prog.push_back({ARRIVE, cempty[ci], gcs / p.CSN});
    }
  }
  {
    auto& prog = m.actor(0, "code warp").prog;
    for (int gcs = 0; gcs < p.units * CSU; ++gcs) {
      prog.push_back({WAIT, cempty[gcs % p.CSN], gcs / p.CSN - 1});
      prog.push_back({COPY, cfull[gcs % p.CSN], gcs / p.CSN});
    }
  }
  {
    auto& prog = m.actor(0, "MMA").prog;
    int it_k = 0;
    for (int it = 0; it < p.units; ++it) {
      prog.push_back({WAIT, tempty[it & 1], (it >> 1) - 1});
      for (int kc = 0; kc < KC; ++kc, ++it_k) {
        prog.push_back({WAIT, full[it_k % p.S], it_k / p.S});
        prog.push_back({WAIT, bfull[it_k % p.S], it_k / p.S});
        prog.push_back({COMMIT, empty[it_k % p.S], it_k / p.S});
      }
      prog.push_back({COMMIT, tfull[it & 1], it >> 1});
    }
  }
  {
    auto& prog = m.actor(0, "epilogue").prog;
    for (int it = 0; it < p.units; ++it) {
      prog.push_back({WAIT, tfull[it & 1], it >> 1});
      prog.push_back({ARRIVE, tempty[it & 1], it >> 1});
    }
  }
}

Outcome run_prefill(const PrefillParams& p, unsigned long long seed, std::string* why) {
  Sim m;
  build_prefill(m, p);
  const Outcome o = m.run(seed);
  *why = m.why;
  return o;
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
          const DecodeParams p{G, U, s[0], s[1], S, groups, TS, KC, 2};
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
      const DecodeParams p{2, 3, 2560, 640, 12, 4, 3, KC, 2};
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
            const DecodeParams p{G, U, s[0], s[1], S, groups, TS, KC, mode};
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
          const PrefillParams p{units, K, CPC, 4, 3};
          const Outcome o = run_prefill(p, 2000003ull * (unsigned long long)runs + 5, &why);
          ++runs;
          if (o != COMPLETE) {
            std::printf("FAIL prefill K=%d CPC=%d units=%d: %s (%s)\n", K, CPC, units,
                        outcome_name(o), why.c_str());
            return 1;
          }
        }
  std::printf("ok %ld\n", runs);
  return 0;
}
