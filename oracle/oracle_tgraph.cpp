// CPU oracle for the SM-level task graph (tGraph) of one decode step.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
// cpu_baseline leg of bench.py may load this code.  The GPU library has its
// own, independently written builder; the two share no code.
//
// The pipeline follows the one sentence the pages give on the tGraph
// algorithm (MPK review by zhaifeiyue, §2.4 "incremental vs truly novel"):
// event fusion, then normalisation so that each task has at most one
// dependency event and at most one trigger event, then BFS linearisation so
// that the tasks an event releases form one contiguous [first, last] range.
// The MPK abstract supplies the rest of the framing: operators are split into
// SM-sized tasks and dependencies are tracked per task.  Everything below that
// the pages leave open is one plain reading, stated where it is used:
//
//   tiling      GEMV ops: rows per task n = align_up(ceil(N / W), col_align).
//               QKV: the smallest multiple of col_align that divides one kv
//               group's rows G = (Hq/Hkv + 2) * D and gives ceil(N/n) <= W
//               (else n = G), so no task spans two kv groups.
//               ATTN: S' = max(1, floor(apw * W / (B * Hkv))) (at most
//               apw tasks per worker),
//               chunk = max(min_chunk, align_up(ceil(Lcap / S'), 64)),
//               S = ceil(Lcap / chunk).  Every split writes its partial
//               and may write the merged head block: the split of (b, g) that
//               finishes last merges the partials (no separate merge op).
//               JIT attention (data-dependent ranges resolved at run time,
//               MPK review "Direction 4"): apw * W tasks per layer, each
//               reading all of the layer's q/k/v and the KV lengths and
//               writing all partials and heads; partial slots per (b, g):
//               S = ceil(apw * W / (B * Hkv)) + 2; chunk = 0.
//   regions     each task reads and writes rectangles of named buffers;
//               activations are single-assignment (one buffer per layer/op).
//   raw events  task a -> task c when op(a) < op(c) and a region of a and a
//               region of c on the same buffer overlap with at least one
//               write.  One raw event per (c, producer op).
//   fusion      events with identical trigger sets are merged; after the
//               reduction, events with identical dependent sets are merged;
//               both repeated to a fixpoint.
//   reduction   a dependency event e of task c is dropped when another of
//               c's dependency events e' already guarantees it: every trigger
//               of e is in Done(e'), the set of tasks certainly finished once
//               e' has fired.
//   normalise   k >= 2 dependency events: k empty tasks (dep e_i, trigger
//               e*) feed a new event e* that c waits on.  k >= 2 trigger
//               events: c triggers a new e+, and k empty tasks (dep e+,
//               trigger e_i) replace c among the triggers of the old events.
//   BFS         roots first, in key order; an event enters the FIFO when its
//               last trigger is placed; visiting it places its dependents in
//               key order.  Event ids = FIFO order, task ids = placement order.
//   key         (op, sub, idx): sub 0 = empty tasks that gather
//               dependencies, 1 = real tasks, 2 = empty tasks that fan out
//               triggers; idx of an empty task = its creation number.
#include <algorithm>
#include <cstdint>
#include <deque>
#include <map>
#include <set>
#include <vector>

extern "C" {
struct OracleCfg {
  int32_t n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab, tied;
  float eps;
  int32_t pad0;
  double theta;
  int32_t batch, kv_capacity;
};
}

namespace {

enum { T_GENERIC = 0, T_EMBED = 1, T_QKV, T_ATTN, T_MERGE, T_OPROJ, T_GATEUP, T_DOWN,
       T_LMHEAD, T_ARGMAX, T_EMPTY };

struct Rect {
  int buf, r0, r1, c0, c1;
  bool write;
};

struct Task {
  int type, op, layer, sub, idx;
  std::vector<Rect> regs;
};

struct Event {
  std::vector<int> trig;  // sorted task indices
  std::vector<int> dep;   // sorted task indices
  bool alive = true;
};

struct Graph {
  std::vector<int> t_type, t_op, t_layer, t_idx, t_dep, t_trig;  // final order
  std::vector<int> e_count, e_first, e_last;
  std::vector<int> edge_src, edge_dst;  // raw edges, final task ids
  int qkv_rows = 0, o_rows = 0, gu_rows = 0, down_rows = 0, lm_rows = 0, splits = 0,
      chunk = 0;
};

bool key_less(const Task &a, const Task &b) {
  if (a.op != b.op) return a.op < b.op;
  if (a.sub != b.sub) return a.sub < b.sub;
  return a.idx < b.idx;
}

int ceil_div(long a, long b) { return (int)((a + b - 1) / b); }
int align_up(long a, long b) { return (int)(((a + b - 1) / b) * b); }

bool overlap(const Rect &a, const Rect &b) {
  return a.buf == b.buf && a.r0 < b.r1 && b.r0 < a.r1 && a.c0 < b.c1 && b.c0 < a.c1;
}

bool subset(const std::vector<int> &small, const std::vector<uint64_t> &bits) {
  for (int t : small)
    if (!((bits[t >> 6] >> (t & 63)) & 1)) return false;
  return true;
}

// Lexicographic order of events: trigger list, then dependent list.
bool event_less(const Event &a, const Event &b) {
  if (a.trig != b.trig) return a.trig < b.trig;
  return a.dep < b.dep;
}

// The core pipeline on tasks already sorted by key.  preds[c] = list of
// predecessor task indices of c (any order).
Graph run_pipeline(std::vector<Task> tasks, const std::vector<std::set<int>> &preds) {
  int n = (int)tasks.size();
  Graph out;
  std::vector<std::pair<int, int>> raw_edges;
  for (int c = 0; c < n; ++c)
    for (int a : preds[c]) raw_edges.push_back({a, c});

  // Raw events: one per (consumer, producer op).
  std::vector<Event> ev;
  for (int c = 0; c < n; ++c) {
    std::map<int, std::vector<int>> by_op;
    for (int a : preds[c]) by_op[tasks[a].op].push_back(a);
    for (auto &kv : by_op) {
      Event e;
      e.trig = kv.second;
      std::sort(e.trig.begin(), e.trig.end());
      e.dep = {c};
      ev.push_back(e);
    }
  }

  // Fusion by identical trigger sets.
  auto fuse_by_trig = [&](std::vector<Event> &in) {
    std::map<std::vector<int>, std::set<int>> m;
    for (auto &e : in)
      if (e.alive) m[e.trig].insert(e.dep.begin(), e.dep.end());
    std::vector<Event> res;
    for (auto &kv : m) {
      Event e;
      e.trig = kv.first;
      e.dep.assign(kv.second.begin(), kv.second.end());
      res.push_back(e);
    }
    bool changed = res.size() != in.size();
    in = res;
    return changed;
  };
  auto fuse_by_dep = [&](std::vector<Event> &in) {
    std::map<std::vector<int>, std::set<int>> m;
    for (auto &e : in)
      if (e.alive) m[e.dep].insert(e.trig.begin(), e.trig.end());
    std::vector<Event> res;
    for (auto &kv : m) {
      Event e;
      e.dep = kv.first;
      e.trig.assign(kv.second.begin(), kv.second.end());
      res.push_back(e);
    }
    std::sort(res.begin(), res.end(), event_less);
    bool changed = res.size() != in.size();
    in = res;
    return changed;
  };
  fuse_by_trig(ev);

  // Done(e): tasks certainly finished once e fired.
  int ne = (int)ev.size();
  int words = (n + 63) / 64;
  std::vector<std::vector<int>> deps_of(n);  // event indices each task waits on
  for (int e = 0; e < ne; ++e)
    for (int c : ev[e].dep) deps_of[c].push_back(e);
  std::vector<std::vector<uint64_t>> done(ne);
  std::vector<char> have(ne, 0);
  // After trigger fusion every event's triggers belong to one op, and the
  // events their triggers wait on have triggers in earlier ops: process by op.
  std::vector<int> order(ne);
  for (int e = 0; e < ne; ++e) order[e] = e;
  std::sort(order.begin(), order.end(), [&](int a, int b) {
    return tasks[ev[a].trig[0]].op < tasks[ev[b].trig[0]].op;
  });
  for (int e : order) {
    std::vector<uint64_t> bits(words, 0);
    for (int a : ev[e].trig) {
      bits[a >> 6] |= 1ULL << (a & 63);
      for (int d : deps_of[a]) {
        for (int w = 0; w < words; ++w) bits[w] |= done[d][w];
      }
    }
    done[e] = bits;
    have[e] = 1;
  }

  // Reduction.
  for (int c = 0; c < n; ++c) {
    std::vector<int> ds = deps_of[c];
    if (ds.size() < 2) continue;
    std::sort(ds.begin(), ds.end(), [&](int a, int b) { return event_less(ev[a], ev[b]); });
    std::vector<int> keep = ds;
    for (int e : ds) {
      bool implied = false;
      for (int e2 : keep) {
        if (e2 == e) continue;
        if (subset(ev[e].trig, done[e2])) {
          implied = true;
          break;
        }
      }
      if (implied) keep.erase(std::find(keep.begin(), keep.end(), e));
    }
    for (int e : ds) {
      if (std::find(keep.begin(), keep.end(), e) != keep.end()) continue;
      auto &dl = ev[e].dep;
      dl.erase(std::find(dl.begin(), dl.end(), c));
    }
  }
  for (auto &e : ev)
    if (e.dep.empty()) e.alive = false;
  {
    std::vector<Event> live;
    for (auto &e : ev)
      if (e.alive) live.push_back(e);
    ev = live;
  }
  // Fusion to a fixpoint.
  for (;;) {
    bool a = fuse_by_trig(ev);
    bool b = fuse_by_dep(ev);
    if (!a && !b) break;
  }
  std::sort(ev.begin(), ev.end(), event_less);

  // Normalisation.
  int empty_counter = 0;
  auto dep_lists = [&]() {
    std::vector<std::vector<int>> d(tasks.size());
    for (int e = 0; e < (int)ev.size(); ++e)
      for (int c : ev[e].dep) d[c].push_back(e);
    return d;
  };
  auto trig_lists = [&]() {
    std::vector<std::vector<int>> d(tasks.size());
    for (int e = 0; e < (int)ev.size(); ++e)
      for (int c : ev[e].trig) d[c].push_back(e);
    return d;
  };
  // Tasks are indexed in key order; new empty tasks are appended and a final
  // sort by key happens implicitly in BFS (which orders by key).
  {
    auto dl = dep_lists();
    int n0 = (int)tasks.size();
    for (int c = 0; c < n0; ++c) {
      if (dl[c].size() < 2) continue;
      // Events are ranked by their index: the fused events were sorted by
      // (trigger list, dependent list); events made here rank after them in
      // creation order.
      std::vector<int> ds = dl[c];
      std::sort(ds.begin(), ds.end());
      Event star;
      star.dep = {c};
      std::vector<int> empties;
      for (int e : ds) {
        Task t;
        t.type = T_EMPTY;
        t.op = tasks[c].op;
        t.layer = tasks[c].layer;
        t.sub = 0;
        t.idx = empty_counter++;
        tasks.push_back(t);
        int ti = (int)tasks.size() - 1;
        empties.push_back(ti);
        auto &d = ev[e].dep;
        *std::find(d.begin(), d.end(), c) = ti;
      }
      star.trig = empties;
      ev.push_back(star);
    }
  }
  {
    auto tl = trig_lists();
    int n1 = (int)tasks.size();
    // visit tasks in key order
    std::vector<int> ord(n1);
    for (int i = 0; i < n1; ++i) ord[i] = i;
    std::sort(ord.begin(), ord.end(), [&](int a, int b) { return key_less(tasks[a], tasks[b]); });
    for (int c : ord) {
      if (tl[c].size() < 2) continue;
      std::vector<int> ts = tl[c];
      std::sort(ts.begin(), ts.end());
      Event plus;
      plus.trig = {c};
      std::vector<int> empties;
      for (int e : ts) {
        Task t;
        t.type = T_EMPTY;
        t.op = tasks[c].op;
        t.layer = tasks[c].layer;
        t.sub = 2;
        t.idx = empty_counter++;
        tasks.push_back(t);
        int ti = (int)tasks.size() - 1;
        empties.push_back(ti);
        auto &tr = ev[e].trig;
        *std::find(tr.begin(), tr.end(), c) = ti;
      }
      plus.dep = empties;
      ev.push_back(plus);
    }
  }

  // BFS linearisation.
  int nt = (int)tasks.size(), nev = (int)ev.size();
  auto dl = dep_lists();
  auto tl = trig_lists();
  auto by_key = [&](std::vector<int> v) {
    std::sort(v.begin(), v.end(), [&](int a, int b) { return key_less(tasks[a], tasks[b]); });
    return v;
  };
  std::vector<int> remaining(nev), ev_id(nev, -1), task_id(nt, -1), placed;
  for (int e = 0; e < nev; ++e) remaining[e] = (int)ev[e].trig.size();
  std::deque<int> fifo;
  std::vector<int> ev_order;
  auto place = [&](int t) {
    task_id[t] = (int)placed.size();
    placed.push_back(t);
    for (int e : tl[t]) {
      if (--remaining[e] == 0) {
        ev_id[e] = (int)ev_order.size();
        ev_order.push_back(e);
        fifo.push_back(e);
      }
    }
  };
  std::vector<int> roots;
  for (int t = 0; t < nt; ++t)
    if (dl[t].empty()) roots.push_back(t);
  for (int t : by_key(roots)) place(t);
  std::vector<int> first(nev, -1), last(nev, -1);
  while (!fifo.empty()) {
    int e = fifo.front();
    fifo.pop_front();
    std::vector<int> ds = by_key(ev[e].dep);
    first[e] = (int)placed.size();
    for (int t : ds) place(t);
    last[e] = (int)placed.size() - 1;
  }

  if ((int)placed.size() != nt) {
    out.t_type.clear();
    return out;  // a cycle: caller reports the error
  }
  out.t_type.resize(placed.size());
  out.t_op.resize(placed.size());
  out.t_layer.resize(placed.size());
  out.t_idx.resize(placed.size());
  out.t_dep.resize(placed.size());
  out.t_trig.resize(placed.size());
  for (size_t i = 0; i < placed.size(); ++i) {
    const Task &t = tasks[placed[i]];
    out.t_type[i] = t.type;
    out.t_op[i] = t.op;
    out.t_layer[i] = t.layer;
    out.t_idx[i] = t.idx;
    out.t_dep[i] = dl[placed[i]].empty() ? -1 : ev_id[dl[placed[i]][0]];
    out.t_trig[i] = tl[placed[i]].empty() ? -1 : ev_id[tl[placed[i]][0]];
  }
  out.e_count.resize(ev_order.size());
  out.e_first.resize(ev_order.size());
  out.e_last.resize(ev_order.size());
  for (size_t i = 0; i < ev_order.size(); ++i) {
    int e = ev_order[i];
    out.e_count[i] = (int)ev[e].trig.size();
    out.e_first[i] = first[e];
    out.e_last[i] = last[e];
  }
  for (auto &pr : raw_edges) {
    out.edge_src.push_back(task_id[pr.first]);
    out.edge_dst.push_back(task_id[pr.second]);
  }
  return out;
}

// Build the decode-step tasks with their regions (op order = vector order).
struct Lowered {
  std::vector<Task> tasks;
  int qkv_rows, o_rows, gu_rows, down_rows, lm_rows, splits, chunk;
};

Lowered lower_decode(const OracleCfg &c, int W, int col_align, int apw, int min_chunk, int jit) {
  Lowered L;
  const int Ly = c.n_layers, H = c.hidden, Hq = c.n_q_heads, Hkv = c.n_kv_heads, D = c.head_dim;
  const int F = c.ffn, V = c.vocab, B = c.batch, Lcap = c.kv_capacity, rep = Hq / Hkv;
  const int G = (rep + 2) * D, Nqkv = Hkv * G, qd = Hq * D;
  auto gemv_rows = [&](int N) { return align_up(ceil_div(N, W), col_align); };
  int qkv_rows = G;
  for (int m = col_align; m <= G; m += col_align) {
    if (G % m == 0 && ceil_div(Nqkv, m) <= W) {
      qkv_rows = m;
      break;
    }
  }
  int S, chunk, n_jit = 0;
  if (jit) {
    n_jit = std::max(1, apw * W);
    S = ceil_div(n_jit, (long)B * Hkv) + 2;
    chunk = 0;
  } else {
    int sp = (int)std::max(1L, (long)apw * W / ((long)B * Hkv));
    chunk = std::max(min_chunk, align_up(ceil_div(Lcap, sp), 64));
    S = ceil_div(Lcap, chunk);
  }
  L.qkv_rows = qkv_rows;
  L.o_rows = gemv_rows(H);
  L.gu_rows = gemv_rows(F);
  L.down_rows = gemv_rows(H);
  L.lm_rows = gemv_rows(V);
  L.splits = S;
  L.chunk = chunk;

  // Buffer ids.
  const int B_TOK = 0, B_KVLEN = 1, B_LMP = 2;
  auto B_X = [&](int l) { return 3 + l; };  // l = 0..Ly
  auto lb = [&](int l, int k) { return 4 + Ly + l * 5 + k; };
  auto B_QKV = [&](int l) { return lb(l, 0); };
  auto B_PART = [&](int l) { return lb(l, 1); };
  auto B_ATT = [&](int l) { return lb(l, 2); };
  auto B_XM = [&](int l) { return lb(l, 3); };
  auto B_H = [&](int l) { return lb(l, 4); };

  int op = 0;
  auto add = [&](int type, int layer, int idx, std::vector<Rect> regs) {
    Task t;
    t.type = type;
    t.op = op;
    t.layer = layer;
    t.sub = 1;
    t.idx = idx;
    t.regs = regs;
    L.tasks.push_back(t);
  };
  auto R = [](int buf, int r0, int r1, int c0, int c1) { return Rect{buf, r0, r1, c0, c1, false}; };
  auto Wr = [](int buf, int r0, int r1, int c0, int c1) { return Rect{buf, r0, r1, c0, c1, true}; };

  add(T_EMBED, -1, 0, {R(B_TOK, 0, B, 0, 1), Wr(B_X(0), 0, B, 0, H)});
  ++op;
  for (int l = 0; l < Ly; ++l) {
    for (int j = 0; j * qkv_rows < Nqkv; ++j)
      add(T_QKV, l, j, {R(B_X(l), 0, B, 0, H),
                        Wr(B_QKV(l), 0, B, j * qkv_rows, std::min(Nqkv, (j + 1) * qkv_rows))});
    ++op;
    for (int a = 0; a < n_jit; ++a)
      add(T_ATTN, l, a, {R(B_QKV(l), 0, B, 0, Nqkv), R(B_KVLEN, 0, B, 0, 1),
                         Wr(B_PART(l), 0, B, 0, Hkv * S), Wr(B_ATT(l), 0, B, 0, qd)});
    for (int b = 0; b < (jit ? 0 : B); ++b)
      for (int g = 0; g < Hkv; ++g)
        for (int s = 0; s < S; ++s) {
          std::vector<Rect> regs = {R(B_QKV(l), b, b + 1, g * G, (g + 1) * G),
                                    R(B_KVLEN, b, b + 1, 0, 1)};
          // every split may produce the merged head block: the split that
          // finishes last merges all partials of (b, g)
          if (S > 1) regs.push_back(Wr(B_PART(l), b, b + 1, g * S + s, g * S + s + 1));
          regs.push_back(Wr(B_ATT(l), b, b + 1, g * rep * D, (g + 1) * rep * D));
          add(T_ATTN, l, (b * Hkv + g) * S + s, regs);
        }
    ++op;
    for (int j = 0; j * L.o_rows < H; ++j) {
      int c0 = j * L.o_rows, c1 = std::min(H, c0 + L.o_rows);
      add(T_OPROJ, l, j, {R(B_ATT(l), 0, B, 0, qd), R(B_X(l), 0, B, c0, c1),
                          Wr(B_XM(l), 0, B, c0, c1)});
    }
    ++op;
    for (int j = 0; j * L.gu_rows < F; ++j) {
      int c0 = j * L.gu_rows, c1 = std::min(F, c0 + L.gu_rows);
      add(T_GATEUP, l, j, {R(B_XM(l), 0, B, 0, H), Wr(B_H(l), 0, B, c0, c1)});
    }
    ++op;
    for (int j = 0; j * L.down_rows < H; ++j) {
      int c0 = j * L.down_rows, c1 = std::min(H, c0 + L.down_rows);
      add(T_DOWN, l, j, {R(B_H(l), 0, B, 0, F), R(B_XM(l), 0, B, c0, c1),
                         Wr(B_X(l + 1), 0, B, c0, c1)});
    }
    ++op;
  }
  int n_lm = 0;
  for (int j = 0; j * L.lm_rows < V; ++j, ++n_lm)
    add(T_LMHEAD, -1, j, {R(B_X(Ly), 0, B, 0, H), Wr(B_LMP, 0, B, j, j + 1)});
  ++op;
  add(T_ARGMAX, -1, 0, {R(B_LMP, 0, B, 0, n_lm), Wr(B_TOK, 0, B, 0, 1), Wr(B_KVLEN, 0, B, 0, 1)});
  return L;
}

std::vector<std::set<int>> region_preds(const std::vector<Task> &tasks) {
  // Plain scan: every pair of tasks in different ops.
  int n = (int)tasks.size();
  std::map<int, std::vector<std::pair<int, Rect>>> by_buf;
  for (int t = 0; t < n; ++t)
    for (auto &r : tasks[t].regs) by_buf[r.buf].push_back({t, r});
  std::vector<std::set<int>> preds(n);
  for (int c = 0; c < n; ++c)
    for (auto &rc : tasks[c].regs)
      for (auto &pr : by_buf[rc.buf]) {
        int a = pr.first;
        if (tasks[a].op >= tasks[c].op) continue;
        if (!(pr.second.write || rc.write)) continue;
        if (overlap(pr.second, rc)) preds[c].insert(a);
      }
  return preds;
}

}  // namespace

extern "C" {

int oracle_tgraph_decode(const OracleCfg *cfg, int num_workers, int col_align,
                         int attn_tasks_per_worker, int attn_min_chunk, int attn_jit, void **out) {
  if (!cfg || !out || num_workers < 1 || col_align < 1 || attn_tasks_per_worker < 1 ||
      attn_min_chunk < 1)
    return -1;
  if (cfg->n_kv_heads < 1 || cfg->n_q_heads % cfg->n_kv_heads) return -1;
  Lowered L = lower_decode(*cfg, num_workers, col_align, attn_tasks_per_worker, attn_min_chunk,
                           attn_jit);
  auto preds = region_preds(L.tasks);
  Graph *g = new Graph(run_pipeline(L.tasks, preds));
  if (g->t_type.empty()) {
    delete g;
    return -2;
  }
  g->qkv_rows = L.qkv_rows;
  g->o_rows = L.o_rows;
  g->gu_rows = L.gu_rows;
  g->down_rows = L.down_rows;
  g->lm_rows = L.lm_rows;
  g->splits = L.splits;
  g->chunk = L.chunk;
  *out = g;
  return 0;
}

// Generic entry for property tests: n tasks with (op, idx) keys and an edge
// list over them (src must be in an earlier op than dst).
int oracle_tgraph_from_edges(int n, const int32_t *task_op, const int32_t *task_idx, int n_edges,
                             const int32_t *src, const int32_t *dst, void **out) {
  std::vector<Task> tasks(n);
  for (int i = 0; i < n; ++i) {
    tasks[i].type = T_GENERIC;
    tasks[i].op = task_op[i];
    tasks[i].layer = -1;
    tasks[i].sub = 1;
    tasks[i].idx = task_idx[i];
  }
  for (int e = 0; e < n_edges; ++e)
    if (src[e] < 0 || src[e] >= n || dst[e] < 0 || dst[e] >= n ||
        task_op[src[e]] >= task_op[dst[e]])
      return -1;
  // sort by key; remap edges
  std::vector<int> ord(n);
  for (int i = 0; i < n; ++i) ord[i] = i;
  std::sort(ord.begin(), ord.end(), [&](int a, int b) { return key_less(tasks[a], tasks[b]); });
  for (int i = 1; i < n; ++i)
    if (!key_less(tasks[ord[i - 1]], tasks[ord[i]])) return -1;  // duplicate key
  std::vector<int> pos(n);
  std::vector<Task> sorted(n);
  for (int i = 0; i < n; ++i) {
    pos[ord[i]] = i;
    sorted[i] = tasks[ord[i]];
  }
  std::vector<std::set<int>> preds(n);
  for (int e = 0; e < n_edges; ++e) preds[pos[dst[e]]].insert(pos[src[e]]);
  Graph *g = new Graph(run_pipeline(sorted, preds));
  if (n > 0 && g->t_type.empty()) {
    delete g;
    return -2;
  }
  *out = g;
  return 0;
}

void oracle_tgraph_sizes(const void *g, int32_t *n_tasks, int32_t *n_events, int32_t *n_edges) {
  const Graph *G = (const Graph *)g;
  *n_tasks = (int32_t)G->t_type.size();
  *n_events = (int32_t)G->e_count.size();
  *n_edges = (int32_t)G->edge_src.size();
}

void oracle_tgraph_tiling(const void *g, int32_t *out7) {
  const Graph *G = (const Graph *)g;
  int v[7] = {G->qkv_rows, G->o_rows, G->gu_rows, G->down_rows, G->lm_rows, G->splits, G->chunk};
  for (int i = 0; i < 7; ++i) out7[i] = v[i];
}

void oracle_tgraph_tasks(const void *g, int32_t *type, int32_t *op, int32_t *layer,
                         int32_t *idx, int32_t *dep, int32_t *trig) {
  const Graph *G = (const Graph *)g;
  for (size_t i = 0; i < G->t_type.size(); ++i) {
    type[i] = G->t_type[i];
    op[i] = G->t_op[i];
    layer[i] = G->t_layer[i];
    idx[i] = G->t_idx[i];
    dep[i] = G->t_dep[i];
    trig[i] = G->t_trig[i];
  }
}

void oracle_tgraph_events(const void *g, int32_t *count, int32_t *first, int32_t *last) {
  const Graph *G = (const Graph *)g;
  for (size_t i = 0; i < G->e_count.size(); ++i) {
    count[i] = G->e_count[i];
    first[i] = G->e_first[i];
    last[i] = G->e_last[i];
  }
}

void oracle_tgraph_edges(const void *g, int32_t *src, int32_t *dst) {
  const Graph *G = (const Graph *)g;
  for (size_t i = 0; i < G->edge_src.size(); ++i) {
    src[i] = G->edge_src[i];
    dst[i] = G->edge_dst[i];
  }
}

void oracle_tgraph_free(void *g) { delete (Graph *)g; }

}  // extern "C"
