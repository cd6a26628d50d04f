// Host-side tGraph construction (see tgraph.hpp for the sources of the model).
//
// Pipeline:
//   lower      decode step -> operators -> SM-sized tasks, each declaring the
//              rectangles of named buffers it reads and writes
//   edges      producer -> consumer whenever an earlier operator's access and
//              a later one's overlap with at least one write (RAW/WAR/WAW)
//   raw events one event per (consumer task, producer operator)
//   fuse       merge events with equal trigger sets
//   reduce     drop a dependency event that another dependency event of the
//              same task already implies
//   fuse*      merge equal trigger sets / equal dependent sets to a fixpoint
//   normalise  empty tasks so every task has <= 1 dependency and <= 1 trigger
//   linearise  BFS over events; an event's dependents get one [first,last] range
#include "tgraph.hpp"

#include <algorithm>
#include <cstring>
#include <numeric>
#include <unordered_map>

namespace mk {
namespace {

struct Access {
  int task;
  int op;
  int r0, r1, c0, c1;
  bool write;
};

struct Node {
  int type, op, layer, sub, idx;
};

inline bool node_before(const Node &a, const Node &b) {
  if (a.op != b.op) return a.op < b.op;
  if (a.sub != b.sub) return a.sub < b.sub;
  return a.idx < b.idx;
}

struct VecHash {
  size_t operator()(const std::vector<int> &v) const {
    uint64_t h = 0x9E3779B97F4A7C15ULL ^ v.size();
    for (int x : v) {
      h ^= (uint64_t)(uint32_t)x + 0x9E3779B97F4A7C15ULL + (h << 6) + (h >> 2);
    }
    return (size_t)h;
  }
};

struct Ev {
  std::vector<int> in;   // trigger tasks, ascending
  std::vector<int> out;  // dependent tasks, ascending
};

inline long cdiv(long a, long b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------------------
// Decode lowering
// ---------------------------------------------------------------------------
struct Lowering {
  std::vector<Node> nodes;
  // accesses grouped by buffer
  std::vector<std::vector<Access>> by_buf;
  Tiling tiling;
  int n_ops = 0;
};

std::string lower(const ModelShape &m, const GraphTuning &t, Lowering *L) {
  const int W = t.num_workers;
  const int rep = m.n_q_heads / m.n_kv_heads;
  const int grp = (rep + 2) * m.head_dim;  // rows of one kv group in the QKV output
  const int n_qkv = m.n_kv_heads * grp;
  const int qdim = m.n_q_heads * m.head_dim;
  Tiling &T = L->tiling;

  auto rows_for = [&](int n) { return (int)(cdiv(cdiv(n, W), t.col_align) * t.col_align); };
  T.qkv_rows = grp;
  for (int k = 1; k * t.col_align <= grp; ++k) {
    int cand = k * t.col_align;
    if (grp % cand) continue;
    if (cdiv(n_qkv, cand) <= W) {
      T.qkv_rows = cand;
      break;
    }
  }
  T.o_rows = rows_for(m.hidden);
  T.gu_rows = rows_for(m.ffn);
  T.down_rows = rows_for(m.hidden);
  T.lm_rows = rows_for(m.vocab);
  T.n_qkv = (int)cdiv(n_qkv, T.qkv_rows);
  T.n_o = (int)cdiv(m.hidden, T.o_rows);
  T.n_gu = (int)cdiv(m.ffn, T.gu_rows);
  T.n_down = (int)cdiv(m.hidden, T.down_rows);
  T.n_lm = (int)cdiv(m.vocab, T.lm_rows);
  const long pairs = (long)m.batch * m.n_kv_heads;
  if (t.attn_jit) {
    // JIT: apw * W tasks; each (sequence, kv head) is cut by at most
    // ceil(apw * W / pairs) + 2 of them (the run-time chunk is chosen so)
    T.n_attn = std::max(1, t.attn_tasks_per_worker * W);
    T.attn_splits = (int)(cdiv(T.n_attn, pairs) + 2);
    T.attn_chunk = 0;
  } else {
    // splits per (sequence, kv head): at most attn_tasks_per_worker tasks per worker
    long target = std::max(1L, (long)t.attn_tasks_per_worker * W / pairs);
    long chunk = cdiv(cdiv(m.kv_capacity, target), 64) * 64;
    if (chunk < t.attn_min_chunk) chunk = t.attn_min_chunk;
    T.attn_chunk = (int)chunk;
    T.attn_splits = (int)cdiv(m.kv_capacity, chunk);
    T.n_attn = (int)(pairs * T.attn_splits);
  }
  const int S = T.attn_splits;

  // Buffers: 0 tokens, 1 kv_len, 2 lm partials, then per layer boundary x_l
  // (l = 0..Ly), then per layer {qkv, partials, attn, x_mid, h}.
  enum { kTok = 0, kKvLen = 1, kLmPart = 2 };
  const int x_base = 3, layer_base = 3 + m.n_layers + 1;
  auto xbuf = [&](int l) { return x_base + l; };
  auto lbuf = [&](int l, int which) { return layer_base + 5 * l + which; };
  L->by_buf.assign(layer_base + 5 * m.n_layers, {});

  int op = -1;
  auto new_op = [&]() { ++op; };
  auto task = [&](int type, int layer, int idx) {
    L->nodes.push_back(Node{type, op, layer, 1, idx});
    return (int)L->nodes.size() - 1;
  };
  auto acc = [&](int id, int buf, int r0, int r1, int c0, int c1, bool w) {
    L->by_buf[buf].push_back(Access{id, op, r0, r1, c0, c1, w});
  };
  const int B = m.batch;

  new_op();
  {
    int id = task(kEmbed, -1, 0);
    acc(id, kTok, 0, B, 0, 1, false);
    acc(id, xbuf(0), 0, B, 0, m.hidden, true);
  }
  for (int l = 0; l < m.n_layers; ++l) {
    new_op();
    for (int j = 0; j < T.n_qkv; ++j) {
      int id = task(kQkv, l, j);
      acc(id, xbuf(l), 0, B, 0, m.hidden, false);
      acc(id, lbuf(l, 0), 0, B, j * T.qkv_rows, std::min(n_qkv, (j + 1) * T.qkv_rows), true);
    }
    new_op();
    if (t.attn_jit) {
      // a JIT task may cover any (sequence, kv head): it reads every group's
      // q, k, v and the KV lengths, and may write every partial and head
      for (int a = 0; a < T.n_attn; ++a) {
        int id = task(kAttn, l, a);
        acc(id, lbuf(l, 0), 0, B, 0, n_qkv, false);
        acc(id, kKvLen, 0, B, 0, 1, false);
        acc(id, lbuf(l, 1), 0, B, 0, m.n_kv_heads * S, true);
        acc(id, lbuf(l, 2), 0, B, 0, qdim, true);
      }
    }
    for (int b = 0; b < B && !t.attn_jit; ++b)
      for (int g = 0; g < m.n_kv_heads; ++g)
        for (int s = 0; s < S; ++s) {
          int id = task(kAttn, l, (b * m.n_kv_heads + g) * S + s);
          acc(id, lbuf(l, 0), b, b + 1, g * grp, (g + 1) * grp, false);
          acc(id, kKvLen, b, b + 1, 0, 1, false);
          // the split of (b, g) that finishes last merges the partials of all
          // splits, so every split declares the merged head block as written
          if (S > 1) acc(id, lbuf(l, 1), b, b + 1, g * S + s, g * S + s + 1, true);
          acc(id, lbuf(l, 2), b, b + 1, g * rep * m.head_dim, (g + 1) * rep * m.head_dim, true);
        }
    new_op();
    for (int j = 0; j < T.n_o; ++j) {
      int c0 = j * T.o_rows, c1 = std::min(m.hidden, c0 + T.o_rows);
      int id = task(kOProj, l, j);
      acc(id, lbuf(l, 2), 0, B, 0, qdim, false);
      acc(id, xbuf(l), 0, B, c0, c1, false);
      acc(id, lbuf(l, 3), 0, B, c0, c1, true);
    }
    new_op();
    for (int j = 0; j < T.n_gu; ++j) {
      int c0 = j * T.gu_rows, c1 = std::min(m.ffn, c0 + T.gu_rows);
      int id = task(kGateUp, l, j);
      acc(id, lbuf(l, 3), 0, B, 0, m.hidden, false);
      acc(id, lbuf(l, 4), 0, B, c0, c1, true);
    }
    new_op();
    for (int j = 0; j < T.n_down; ++j) {
      int c0 = j * T.down_rows, c1 = std::min(m.hidden, c0 + T.down_rows);
      int id = task(kDown, l, j);
      acc(id, lbuf(l, 4), 0, B, 0, m.ffn, false);
      acc(id, lbuf(l, 3), 0, B, c0, c1, false);
      acc(id, xbuf(l + 1), 0, B, c0, c1, true);
    }
  }
  new_op();
  for (int j = 0; j < T.n_lm; ++j) {
    int id = task(kLmHead, -1, j);
    acc(id, xbuf(m.n_layers), 0, B, 0, m.hidden, false);
    acc(id, kLmPart, 0, B, j, j + 1, true);
  }
  new_op();
  {
    int id = task(kArgmax, -1, 0);
    acc(id, kLmPart, 0, B, 0, T.n_lm, false);
    acc(id, kTok, 0, B, 0, 1, true);
    acc(id, kKvLen, 0, B, 0, 1, true);
  }
  L->n_ops = op + 1;
  return "";
}

// Predecessors from overlapping accesses.  Accesses of one buffer are sorted
// by their first column; a query scans the prefix whose first column lies
// before the query's end.
std::vector<std::vector<int>> predecessors(const Lowering &L) {
  std::vector<std::vector<int>> preds(L.nodes.size());
  for (const auto &list0 : L.by_buf) {
    if (list0.empty()) continue;
    std::vector<Access> list(list0);
    std::sort(list.begin(), list.end(),
              [](const Access &a, const Access &b) { return a.c0 < b.c0; });
    for (const Access &q : list0) {
      auto end = std::lower_bound(list.begin(), list.end(), q.c1,
                                  [](const Access &a, int c) { return a.c0 < c; });
      for (auto it = list.begin(); it != end; ++it) {
        const Access &a = *it;
        if (a.op >= q.op || a.c1 <= q.c0) continue;
        if (!(a.write || q.write)) continue;
        if (a.r1 <= q.r0 || q.r1 <= a.r0) continue;
        preds[q.task].push_back(a.task);
      }
    }
  }
  for (auto &p : preds) {
    std::sort(p.begin(), p.end());
    p.erase(std::unique(p.begin(), p.end()), p.end());
  }
  return preds;
}

// ---------------------------------------------------------------------------
// Core: events, fusion, reduction, normalisation, linearisation.
// nodes must be sorted by key; preds hold indices into nodes.
// ---------------------------------------------------------------------------
std::string finish(std::vector<Node> nodes, const std::vector<std::vector<int>> &preds,
                   TaskGraph *G, int *status) {
  const int n = (int)nodes.size();

  // raw events (consumer, producer op), fused on the fly by trigger set
  std::vector<Ev> evs;
  {
    std::unordered_map<std::vector<int>, int, VecHash> by_in;
    for (int c = 0; c < n; ++c) {
      const auto &p = preds[c];
      size_t i = 0;
      while (i < p.size()) {
        size_t j = i;
        // predecessors are ascending by index, hence grouped by op
        while (j < p.size() && nodes[p[j]].op == nodes[p[i]].op) ++j;
        std::vector<int> in(p.begin() + i, p.begin() + j);
        auto it = by_in.find(in);
        if (it == by_in.end()) {
          by_in.emplace(in, (int)evs.size());
          evs.push_back(Ev{in, {c}});
        } else {
          evs[it->second].out.push_back(c);
        }
        i = j;
      }
    }
  }
  for (auto &e : evs) std::sort(e.out.begin(), e.out.end());

  // Done(e): tasks certainly complete once e fired = its triggers plus Done of
  // every event those triggers wait on.  Events are visited in order of their
  // triggers' op; the events a trigger waits on come from earlier ops.
  const int ne = (int)evs.size();
  const int words = (n + 63) / 64;
  std::vector<std::vector<int>> waits(n);
  for (int e = 0; e < ne; ++e)
    for (int c : evs[e].out) waits[c].push_back(e);
  std::vector<uint64_t> done((size_t)ne * words, 0);
  {
    std::vector<int> order(ne);
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
      return nodes[evs[a].in.front()].op < nodes[evs[b].in.front()].op;
    });
    std::vector<int> srcs;
    for (int e : order) {
      uint64_t *d = &done[(size_t)e * words];
      srcs.clear();
      for (int a : evs[e].in) {
        d[a >> 6] |= 1ULL << (a & 63);
        srcs.insert(srcs.end(), waits[a].begin(), waits[a].end());
      }
      std::sort(srcs.begin(), srcs.end());
      srcs.erase(std::unique(srcs.begin(), srcs.end()), srcs.end());
      for (int s : srcs) {
        const uint64_t *ds = &done[(size_t)s * words];
        for (int w = 0; w < words; ++w) d[w] |= ds[w];
      }
    }
  }
  auto implied_by = [&](int e, int by) {
    const uint64_t *d = &done[(size_t)by * words];
    for (int a : evs[e].in)
      if (!((d[a >> 6] >> (a & 63)) & 1ULL)) return false;
    return true;
  };
  // events sorted by trigger list == index order after the map above? No:
  // rank them explicitly (trigger list, then dependent list).
  auto ev_less = [&](int a, int b) {
    if (evs[a].in != evs[b].in) return evs[a].in < evs[b].in;
    return evs[a].out < evs[b].out;
  };
  for (int c = 0; c < n; ++c) {
    auto &ws = waits[c];
    if (ws.size() < 2) continue;
    std::sort(ws.begin(), ws.end(), ev_less);
    std::vector<char> dropped(ws.size(), 0);
    for (size_t i = 0; i < ws.size(); ++i) {
      for (size_t j = 0; j < ws.size(); ++j) {
        if (j == i || dropped[j]) continue;
        if (implied_by(ws[i], ws[j])) {
          dropped[i] = 1;
          break;
        }
      }
    }
    for (size_t i = 0; i < ws.size(); ++i) {
      if (!dropped[i]) continue;
      auto &o = evs[ws[i]].out;
      o.erase(std::lower_bound(o.begin(), o.end(), c));
    }
  }
  {
    std::vector<Ev> keep;
    for (auto &e : evs)
      if (!e.out.empty()) keep.push_back(std::move(e));
    evs.swap(keep);
  }

  // fusion to a fixpoint
  auto merge_on = [&](bool by_trigger) {
    std::unordered_map<std::vector<int>, int, VecHash> idx;
    std::vector<Ev> res;
    for (auto &e : evs) {
      const std::vector<int> &key = by_trigger ? e.in : e.out;
      auto it = idx.find(key);
      if (it == idx.end()) {
        idx.emplace(key, (int)res.size());
        res.push_back(e);
      } else {
        Ev &r = res[it->second];
        std::vector<int> &dst = by_trigger ? r.out : r.in;
        const std::vector<int> &add = by_trigger ? e.out : e.in;
        std::vector<int> u;
        std::set_union(dst.begin(), dst.end(), add.begin(), add.end(), std::back_inserter(u));
        dst.swap(u);
      }
    }
    bool changed = res.size() != evs.size();
    evs.swap(res);
    return changed;
  };
  for (;;) {
    bool a = merge_on(true);
    bool b = merge_on(false);
    if (!a && !b) break;
  }
  std::sort(evs.begin(), evs.end(), [](const Ev &a, const Ev &b) {
    if (a.in != b.in) return a.in < b.in;
    return a.out < b.out;
  });

  // normalisation; event rank = position in evs (new events append)
  int made = 0;
  {
    std::vector<std::vector<int>> deps_of(n);
    for (int e = 0; e < (int)evs.size(); ++e)
      for (int c : evs[e].out) deps_of[c].push_back(e);
    for (int c = 0; c < n; ++c) {
      if (deps_of[c].size() < 2) continue;
      Ev gather;
      gather.out = {c};
      for (int e : deps_of[c]) {
        nodes.push_back(Node{kEmpty, nodes[c].op, nodes[c].layer, 0, made++});
        int id = (int)nodes.size() - 1;
        gather.in.push_back(id);
        for (int &x : evs[e].out)
          if (x == c) x = id;
      }
      evs.push_back(gather);
    }
  }
  {
    const int n1 = (int)nodes.size();
    std::vector<std::vector<int>> trig_of(n1);
    for (int e = 0; e < (int)evs.size(); ++e)
      for (int a : evs[e].in) trig_of[a].push_back(e);
    std::vector<int> order(n1);
    std::iota(order.begin(), order.end(), 0);
    std::sort(order.begin(), order.end(),
              [&](int a, int b) { return node_before(nodes[a], nodes[b]); });
    for (int a : order) {
      if (trig_of[a].size() < 2) continue;
      Ev fan;
      fan.in = {a};
      for (int e : trig_of[a]) {
        nodes.push_back(Node{kEmpty, nodes[a].op, nodes[a].layer, 2, made++});
        int id = (int)nodes.size() - 1;
        fan.out.push_back(id);
        for (int &x : evs[e].in)
          if (x == a) x = id;
      }
      evs.push_back(fan);
    }
  }

  // BFS linearisation
  const int nn = (int)nodes.size(), nev = (int)evs.size();
  std::vector<int> dep_ev(nn, -1), trig_ev(nn, -1);
  for (int e = 0; e < nev; ++e) {
    for (int c : evs[e].out) dep_ev[c] = e;
    for (int a : evs[e].in) trig_ev[a] = e;
  }
  auto keyed = [&](std::vector<int> v) {
    std::sort(v.begin(), v.end(), [&](int a, int b) { return node_before(nodes[a], nodes[b]); });
    return v;
  };
  std::vector<int> left(nev), ev_rank(nev, -1), pos(nn, -1), seq;
  for (int e = 0; e < nev; ++e) left[e] = (int)evs[e].in.size();
  std::vector<int> queue;
  size_t head = 0;
  seq.reserve(nn);
  auto put = [&](int t) {
    pos[t] = (int)seq.size();
    seq.push_back(t);
    int e = trig_ev[t];
    if (e >= 0 && --left[e] == 0) {
      ev_rank[e] = (int)queue.size();
      queue.push_back(e);
    }
  };
  {
    std::vector<int> roots;
    for (int t = 0; t < nn; ++t)
      if (dep_ev[t] < 0) roots.push_back(t);
    for (int t : keyed(roots)) put(t);
  }
  std::vector<int> first(nev, -1), last(nev, -1);
  while (head < queue.size()) {
    int e = queue[head++];
    first[e] = (int)seq.size();
    for (int t : keyed(evs[e].out)) put(t);
    last[e] = (int)seq.size() - 1;
  }
  if ((int)seq.size() != nn) {
    *status = -4;
    return "graph has a cycle: not every task became ready";
  }

  G->type.resize(nn);
  G->op.resize(nn);
  G->layer.resize(nn);
  G->idx.resize(nn);
  G->dep.resize(nn);
  G->trig.resize(nn);
  for (int i = 0; i < nn; ++i) {
    const Node &t = nodes[seq[i]];
    G->type[i] = t.type;
    G->op[i] = t.op;
    G->layer[i] = t.layer;
    G->idx[i] = t.idx;
    G->dep[i] = dep_ev[seq[i]] < 0 ? -1 : ev_rank[dep_ev[seq[i]]];
    G->trig[i] = trig_ev[seq[i]] < 0 ? -1 : ev_rank[trig_ev[seq[i]]];
  }
  G->ev_count.assign(nev, 0);
  G->ev_first.assign(nev, 0);
  G->ev_last.assign(nev, 0);
  for (int e = 0; e < nev; ++e) {
    int r = ev_rank[e];
    G->ev_count[r] = (int)evs[e].in.size();
    G->ev_first[r] = first[e];
    G->ev_last[r] = last[e];
  }
  G->edge_src.clear();
  G->edge_dst.clear();
  for (int c = 0; c < n; ++c)
    for (int a : preds[c]) {
      G->edge_src.push_back(pos[a]);
      G->edge_dst.push_back(pos[c]);
    }
  int max_op = -1;
  for (int i = 0; i < nn; ++i) max_op = std::max(max_op, G->op[i]);
  G->n_ops = max_op + 1;
  G->op_tasks.assign(G->n_ops, {});
  for (int i = 0; i < nn; ++i) G->op_tasks[G->op[i]].push_back(i);
  *status = 0;
  return "";
}

}  // namespace

std::string plan_decode_graph(const ModelShape &m, const GraphTuning &t, TaskGraph *out,
                              int *status) {
  *status = -1;
  if (t.num_workers < 1 || t.col_align < 1 || t.attn_tasks_per_worker < 1 ||
      t.attn_min_chunk < 1)
    return "tuning values must be positive";
  if (m.n_layers < 1 || m.hidden < 1 || m.n_q_heads < 1 || m.n_kv_heads < 1 ||
      m.head_dim < 2 || m.ffn < 1 || m.vocab < 1 || m.batch < 1 || m.kv_capacity < 1)
    return "model dimensions must be positive";
  if (m.n_q_heads % m.n_kv_heads) return "n_q_heads must be a multiple of n_kv_heads";
  Lowering L;
  std::string err = lower(m, t, &L);
  if (!err.empty()) return err;
  auto preds = predecessors(L);
  err = finish(L.nodes, preds, out, status);
  if (!err.empty()) return err;
  out->tiling = L.tiling;
  out->num_workers = t.num_workers;
  return "";
}

std::string plan_generic_graph(int n, const int32_t *op, const int32_t *idx, int n_edges,
                               const int32_t *src, const int32_t *dst, TaskGraph *out,
                               int *status) {
  *status = -1;
  if (n < 0 || n_edges < 0) return "negative sizes";
  std::vector<int> perm(n);
  std::iota(perm.begin(), perm.end(), 0);
  std::vector<Node> raw(n);
  for (int i = 0; i < n; ++i) raw[i] = Node{kGeneric, op[i], -1, 1, idx[i]};
  std::sort(perm.begin(), perm.end(),
            [&](int a, int b) { return node_before(raw[a], raw[b]); });
  std::vector<int> where(n);
  std::vector<Node> nodes(n);
  for (int i = 0; i < n; ++i) {
    where[perm[i]] = i;
    nodes[i] = raw[perm[i]];
    if (i && !node_before(nodes[i - 1], nodes[i])) return "task keys (op, idx) must be unique";
  }
  std::vector<std::vector<int>> preds(n);
  for (int e = 0; e < n_edges; ++e) {
    if (src[e] < 0 || src[e] >= n || dst[e] < 0 || dst[e] >= n) return "edge out of range";
    if (op[src[e]] >= op[dst[e]]) return "edges must go from an earlier op to a later one";
    preds[where[dst[e]]].push_back(where[src[e]]);
  }
  for (auto &p : preds) {
    std::sort(p.begin(), p.end());
    p.erase(std::unique(p.begin(), p.end()), p.end());
  }
  std::string err = finish(nodes, preds, out, status);
  out->num_workers = 1;
  return err;
}

}  // namespace mk
