// Host-side construction of the SM-level task graph (tGraph) of one decode step.
//
// The graph model comes from the MPK abstract ("MPK: A Compiler and Runtime for
// Mega-Kernelizing Tensor Programs": dependencies captured per SM-sized task)
// and from the MPK review by zhaifeiyue, section 2.4 (event fusion, then
// normalisation to at most one dependency and one trigger event per task, then
// BFS linearisation so that each event releases a contiguous [first, last]
// range of tasks, which lets the in-kernel runtime schedule with only
// atomicAdd and local state).
#pragma once

#include <cstdint>
#include <string>
#include <vector>

namespace mk {

enum TaskType : int {
  kGeneric = 0, kEmbed = 1, kQkv = 2, kAttn = 3, kMerge = 4, kOProj = 5, kGateUp = 6,
  kDown = 7, kLmHead = 8, kArgmax = 9, kEmpty = 10
};

struct ModelShape {
  int n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab, batch, kv_capacity;
};

struct GraphTuning {
  int num_workers = 1;
  int col_align = 16;
  int attn_tasks_per_worker = 4;
  int attn_min_chunk = 64;
  // 1: attention tasks are resolved at run time (JIT): apw * W tasks per
  // layer, each reading every kv group and writing every head, whose position
  // ranges come from the live KV lengths of the step
  int attn_jit = 0;
};

// Rows per task chosen by the tiling rules.
struct Tiling {
  int qkv_rows = 0, o_rows = 0, gu_rows = 0, down_rows = 0, lm_rows = 0;
  int attn_splits = 0, attn_chunk = 0;  // JIT: partial slots per (sequence, kv head), 0
  int n_qkv = 0, n_o = 0, n_gu = 0, n_down = 0, n_lm = 0;
  int n_attn = 0;  // attention tasks per layer
};

// The finished graph: tasks in linear order, events by id.
struct TaskGraph {
  std::vector<int32_t> type, op, layer, idx, dep, trig;
  std::vector<int32_t> ev_count, ev_first, ev_last;
  std::vector<int32_t> edge_src, edge_dst;
  Tiling tiling;
  int num_workers = 1;
  int n_ops = 0;
  // op id -> task ids of that op in increasing order (for per-operator launches)
  std::vector<std::vector<int32_t>> op_tasks;
};

// Returns an empty string on success, else an error text.  `status` receives
// -1 for argument errors and -4 for graph inconsistencies.
std::string plan_decode_graph(const ModelShape &m, const GraphTuning &t, TaskGraph *out,
                              int *status);

std::string plan_generic_graph(int n, const int32_t *op, const int32_t *idx, int n_edges,
                               const int32_t *src, const int32_t *dst, TaskGraph *out,
                               int *status);

}  // namespace mk
