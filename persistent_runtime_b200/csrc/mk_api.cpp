// C ABI of the decode-step megakernel library (see include/mk.h).
#include "mk.h"

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "runtime.cuh"
#include "tgraph.hpp"

#include "mk_handle.hpp"

using mk::Params;

namespace {

thread_local std::string g_last_error;

mk_status fail(mk_handle *h, mk_status s, const std::string &msg) {
  if (h)
    h->err = msg;
  else
    g_last_error = msg;
  return s;
}

mk_status cuda_fail(mk_handle *h, cudaError_t e, const char *what) {
  return fail(h, MK_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

mk_tuning fill_defaults(const mk_tuning *t, int batch = 1) {
  mk_tuning d{};
  if (t) d = *t;
  // batch 1: 4-row alignment gives every SM a tile of the row operators (e.g.
  // 147 x 28 rows of a 4096-row matrix on 148 SMs instead of 128 x 32);
  // the tensor-core tiles of batch >= 2 need whole 16-row m-tiles
  if (d.col_align <= 0) d.col_align = batch > 1 ? 16 : 4;
  // one round of attention tasks: a second round costs a whole task latency,
  // and more splits mean more partials to merge (measured on Qwen3-8B: bs16
  // 12.65 ms at 4 per worker, 11.36 ms at 1; bs8 7.23 -> 6.38 ms)
  if (d.attn_tasks_per_worker <= 0) d.attn_tasks_per_worker = 1;
  if (d.attn_min_chunk <= 0) d.attn_min_chunk = 64;
  if (d.ring_stages <= 0) d.ring_stages = 4;
  if (d.ring_stage_bytes <= 0) d.ring_stage_bytes = 48 * 1024;
  if (d.wait_timeout_us == 0) d.wait_timeout_us = 2000000u;
  // l2_prefetch_bytes: 0 (default) is resolved by default_l2_prefetch once
  // the worker count is known; negative stays "off" until then
  return d;
}

// Default distance of the attention-window L2 prefetch.  At batch 1, while the
// compute warps wait for an O projection's event (the attention window), the
// producer prefetches up to this many bytes of its following stages into L2.
// Qwen3-8B bs1, one box, us per step: off 3146, 512 KB 3121, 1 MB 3083, 2 MB
// 3064, 4 MB 3064 (the window ends first: about 370 KB per worker and layer
// are prefetched at 2 MB); opening the window also while a worker waits for
// its attention task's event, or at every event wait, prefetches more and
// runs slower (3090, 3126).  It pays only where a layer's weights are large
// per worker: Qwen3-0.6B (0.21 MB per worker and layer against 2.4 MB for 8B)
// runs 892 us off against 909 us with 2 MB (its prefetches run layers ahead
// and leave L2 before use: DRAM reads 1.68x the algorithmic bytes) and
// 894-902 us at 128 KB - 1 MB.  At batch >= 2 attention streams the caches in
// that window.
int default_l2_prefetch(const mk_model_config &c, int workers) {
  if (c.batch > 1) return 0;
  const double rep = (double)c.n_q_heads / c.n_kv_heads;
  const double layer_bytes =
      2.0 * ((double)c.n_kv_heads * (rep + 2.0) * c.head_dim * c.hidden +
             (double)c.hidden * c.n_q_heads * c.head_dim + 3.0 * (double)c.ffn * c.hidden);
  return layer_bytes / workers >= 1024.0 * 1024.0 ? 2 * 1024 * 1024 : 0;
}

// Resolve the defaults that depend on the worker count.
void resolve_worker_defaults(mk_tuning &t, const mk_model_config &c, int workers) {
  if (t.l2_prefetch_bytes == 0) t.l2_prefetch_bytes = default_l2_prefetch(c, workers);
  if (t.l2_prefetch_bytes < 0) t.l2_prefetch_bytes = 0;
}

std::string check_shape(const mk_model_config &c) {
  if (c.n_layers < 1 || c.hidden < 1 || c.n_q_heads < 1 || c.n_kv_heads < 1 || c.ffn < 1 ||
      c.vocab < 1 || c.batch < 1 || c.kv_capacity < 1 || c.head_dim < 2)
    return "model dimensions must be positive";
  if (c.n_q_heads % c.n_kv_heads) return "n_q_heads must be a multiple of n_kv_heads";
  if (!(c.rms_eps >= 0.0f)) return "rms_eps must be >= 0";
  return "";
}

std::string check_gpu_shape(const mk_model_config &c) {
  std::string e = check_shape(c);
  if (!e.empty()) return e;
  const int rep = c.n_q_heads / c.n_kv_heads;
  const int qd = c.n_q_heads * c.head_dim;
  if (c.head_dim != 64 && c.head_dim != 128) return "head_dim must be 64 or 128";
  if (rep > mk::kMaxRep) return "at most 8 q heads per kv head";
  if (c.hidden % 256 || c.ffn % 256 || qd % 256)
    return "hidden, ffn and n_q_heads*head_dim must be multiples of 256";
  if (std::max(std::max(c.hidden, c.ffn), qd) > mk::kMaxCpt * 8 * mk::kComputeThreads)
    return "projection input width above 16384";
  if (c.batch > mk::kMaxBatch) return "batch above 16";
  return "";
}

// Tensor-core tiling of the batched projections (QKV, O, GATE_UP, DOWN,
// LM_HEAD, in that order).  m-tiles per row block: the task's rows up to the
// accumulator limit; k-blocks per ring stage: what a stage holds for that
// many m-tiles, a multiple of 8 (one share per warp), at most
// mma_max_kpw(nn) per warp (the B-fragment registers of one stage).
struct MmaTiling {
  int mb[5], kcb[5];
};

MmaTiling mma_tiling(const mk::Tiling &T, int ring_stage_bytes, int nn) {
  const int units = ring_stage_bytes / 512;
  auto mb_of = [&](int task_rows) { return std::max(1, std::min(mk::kMmaMaxMB, task_rows / 16)); };
  const int rows[5] = {T.qkv_rows, T.o_rows, 2 * T.gu_rows, T.down_rows, T.lm_rows};
  MmaTiling m{};
  for (int i = 0; i < 5; ++i) {
    m.mb[i] = mb_of(rows[i]);
    m.kcb[i] = std::min(8 * mk::mma_max_kpw(nn), units / m.mb[i] / 8 * 8);
  }
  return m;
}

mk::ModelShape shape_of(const mk_model_config &c) {
  return mk::ModelShape{c.n_layers, c.hidden, c.n_q_heads, c.n_kv_heads, c.head_dim,
                        c.ffn,      c.vocab,  c.batch,     c.kv_capacity};
}

// JIT attention: opt-in from batch 2 (the batch-1 kernel's attention keeps
// its splits fixed at build time, see mk_build_graph).  Measured on Qwen3-8B
// (one box): bs8 4413 us per step with it, 4324 us without; bs16 10904 vs
// 8549 us -- the cache stream is bound near 5.7 TB/s either way, so spreading
// it over all SMs gains nothing, and every pair then needs a merge.
bool jit_attention(const mk_model_config &c, const mk_tuning &t) {
  return c.batch > 1 && t.attn_jit > 0;
}

mk_status plan(const mk_model_config *cfg, const mk_tuning &t, int workers, mk_handle *h) {
  mk::GraphTuning gt;
  gt.num_workers = workers;
  gt.col_align = t.col_align;
  gt.attn_tasks_per_worker = t.attn_tasks_per_worker;
  gt.attn_min_chunk = t.attn_min_chunk;
  gt.attn_jit = jit_attention(*cfg, t) ? 1 : 0;
  int st = 0;
  std::string e = mk::plan_decode_graph(shape_of(*cfg), gt, &h->graph, &st);
  if (!e.empty()) return fail(h, st == -4 ? MK_ERR_GRAPH : MK_ERR_ARG, e);
  return MK_OK;
}

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

}  // namespace

extern "C" {

mk_status mk_plan_graph(const mk_model_config *cfg, const mk_tuning *tuning, int num_workers,
                        mk_handle **out) {
  if (!cfg || !out) return fail(nullptr, MK_ERR_ARG, "null argument");
  *out = nullptr;
  std::string e = check_shape(*cfg);
  if (!e.empty()) return fail(nullptr, MK_ERR_ARG, e);
  if (num_workers < 1) return fail(nullptr, MK_ERR_ARG, "num_workers must be >= 1");
  mk_handle *h = new (std::nothrow) mk_handle();
  if (!h) return fail(nullptr, MK_ERR_OOM, "out of host memory");
  h->cfg = *cfg;
  h->tune = fill_defaults(tuning, cfg->batch);
  h->tune.num_workers = num_workers;
  resolve_worker_defaults(h->tune, *cfg, num_workers);
  mk_status s = plan(cfg, h->tune, num_workers, h);
  if (s != MK_OK) {
    g_last_error = h->err;
    delete h;
    return s;
  }
  *out = h;
  return MK_OK;
}

mk_status mk_graph_from_edges(int n_tasks, const int32_t *task_op, const int32_t *task_idx,
                              int n_edges, const int32_t *edge_src, const int32_t *edge_dst,
                              mk_handle **out) {
  if (!out || n_tasks < 0 || n_edges < 0 || (n_tasks && (!task_op || !task_idx)) ||
      (n_edges && (!edge_src || !edge_dst)))
    return fail(nullptr, MK_ERR_ARG, "bad argument");
  *out = nullptr;
  mk_handle *h = new (std::nothrow) mk_handle();
  if (!h) return fail(nullptr, MK_ERR_OOM, "out of host memory");
  int st = 0;
  std::string e =
      mk::plan_generic_graph(n_tasks, task_op, task_idx, n_edges, edge_src, edge_dst, &h->graph,
                             &st);
  if (!e.empty()) {
    delete h;
    return fail(nullptr, st == -4 ? MK_ERR_GRAPH : MK_ERR_ARG, e);
  }
  *out = h;
  return MK_OK;
}

mk_status mk_build_graph(const mk_model_config *cfg, const mk_tuning *tuning, int device,
                         mk_handle **out) {
  if (!cfg || !out) return fail(nullptr, MK_ERR_ARG, "null argument");
  *out = nullptr;
  std::string e = check_gpu_shape(*cfg);
  if (!e.empty()) return fail(nullptr, MK_ERR_ARG, e);
  cudaError_t ce = cudaSetDevice(device);
  if (ce != cudaSuccess) return cuda_fail(nullptr, ce, "cudaSetDevice");
  int sms = 0, coop = 0, smem_optin = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, device);
  cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (!coop) return fail(nullptr, MK_ERR_CUDA, "device does not support cooperative launch");

  mk_handle *h = new (std::nothrow) mk_handle();
  if (!h) return fail(nullptr, MK_ERR_OOM, "out of host memory");
  h->host_only = false;
  h->device = device;
  h->cfg = *cfg;
  h->tune = fill_defaults(tuning, cfg->batch);
  mk_tuning &t = h->tune;
  const mk_model_config &c = *cfg;
  const int D = c.head_dim;
  if (t.ring_stages > 16) {
    delete h;
    return fail(nullptr, MK_ERR_ARG, "at most 16 ring stages");
  }
  if (t.ring_stage_bytes % 1024) {
    delete h;
    return fail(nullptr, MK_ERR_ARG, "ring_stage_bytes must be a multiple of 1024");
  }
  if (c.batch > 1 && t.col_align % 16) {
    delete h;
    return fail(nullptr, MK_ERR_ARG, "batch > 1 needs col_align to be a multiple of 16");
  }
  if (c.batch == 1 && t.attn_jit > 0) {
    delete h;
    return fail(nullptr, MK_ERR_ARG, "JIT attention needs batch >= 2");
  }
  if (t.kv_page_size < 0 || t.kv_page_size % 64) {
    delete h;
    return fail(nullptr, MK_ERR_ARG, "kv_page_size must be 0 or a multiple of 64");
  }
  const int rep0 = c.n_q_heads / c.n_kv_heads;
  // q heads per kv head padded to the attention instantiations (2, 4, 8):
  // the per-warp state scratch is sized by it
  const int rep_p = rep0 <= 2 ? 2 : rep0 <= 4 ? 4 : 8;
  // shared memory: shrink the stage size until the CTA fits
  size_t smem = 0;
  for (;;) {
    const int pps = std::min(256, t.ring_stage_bytes / (4 * D) / 8 * 8);
    smem = mk::worker_smem_bytes(t.ring_stages, t.ring_stage_bytes, pps, D, rep_p);
    if ((int)smem <= smem_optin) break;
    t.ring_stage_bytes -= 1024;
    if (t.ring_stage_bytes < 2 * std::max(std::max(c.hidden, c.ffn), c.n_q_heads * D)) {
      delete h;
      return fail(nullptr, MK_ERR_ARG, "ring does not fit in shared memory");
    }
  }
  h->smem = smem;
  ce = mk::worker_configure(smem);
  if (ce != cudaSuccess) {
    mk_status s = cuda_fail(nullptr, ce, "cudaFuncSetAttribute");
    delete h;
    return s;
  }
  int per_sm = 0;
  mk::worker_max_blocks(&per_sm, smem);
  if (per_sm < 1) {
    delete h;
    return fail(nullptr, MK_ERR_CUDA, "worker kernel cannot be resident");
  }
  // dispatch mode: one CTA of the launch is the scheduler
  const int W = t.num_workers > 0 ? t.num_workers : (t.dispatch > 0 ? sms - 1 : sms);
  if (W < 1 || W + (t.dispatch > 0 ? 1 : 0) > sms * per_sm) {
    delete h;
    return fail(nullptr, MK_ERR_ARG, "more workers than co-resident CTAs");
  }
  t.num_workers = W;
  resolve_worker_defaults(t, c, W);
  mk_status s = plan(cfg, t, W, h);
  if (s != MK_OK) {
    g_last_error = h->err;
    delete h;
    return s;
  }
  const mk::TaskGraph &G = h->graph;
  const mk::Tiling &T = G.tiling;

  // sizes
  const int B = c.batch, H = c.hidden, F = c.ffn, Ly = c.n_layers, V = c.vocab;
  const int rep = c.n_q_heads / c.n_kv_heads, grp = (rep + 2) * D, n_qkv = c.n_kv_heads * grp;
  const int qd = c.n_q_heads * D, S = T.attn_splits;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = up256(off + bytes);
    return o;
  };
  const size_t o_tasks = take(sizeof(mk::DevTask) * G.type.size());
  const size_t o_events = take(sizeof(mk::DevEvent) * std::max<size_t>(1, G.ev_count.size()));
  const size_t o_counters = take(4 * std::max<size_t>(1, G.ev_count.size()));
  const size_t o_arrivals = take(4 * (size_t)c.n_layers * c.batch * c.n_kv_heads);
  const size_t o_epoch = take(4);
  const size_t o_status = take(16);
  const size_t o_layers = take(sizeof(mk::DevLayer) * Ly);
  const size_t o_optasks = take(4 * G.type.size());
  // dispatch mode: per-worker queues (round-robin dealing gives each worker
  // at most ceil(n_tasks / W) tasks, plus the end mark)
  const int q_cap = (int)((G.type.size() + W - 1) / W) + 2;
  const size_t o_qlist = t.dispatch > 0 ? take(4 * (size_t)W * q_cap) : 0;
  const size_t o_qtail = t.dispatch > 0 ? take(4 * (size_t)W) : 0;
  const size_t o_rope = take(4 * (size_t)c.kv_capacity * D);
  const size_t o_lmv = take(4 * (size_t)B * T.n_lm);
  const size_t o_lmi = take(4 * (size_t)B * T.n_lm);
  const size_t act0 = off;
  const size_t o_x = take(4 * (size_t)(Ly + 1) * B * H);
  std::vector<size_t> o_qkv(Ly), o_part(Ly), o_att(Ly), o_xm(Ly), o_h(Ly);
  for (int l = 0; l < Ly; ++l) {
    o_qkv[l] = take(4 * (size_t)B * n_qkv);
    o_part[l] = S > 1 ? take(4 * (size_t)B * c.n_q_heads * S * (D + 2)) : 0;
    o_att[l] = take(4 * (size_t)B * qd);
    o_xm[l] = take(4 * (size_t)B * H);
    o_h[l] = take(4 * (size_t)B * F);
  }
  // batch >= 2: fragment-ordered hi/lo bf16 operands (8 or 16 columns) and
  // the per-16-row sums of squares of the streams that feed an RMSNorm
  const bool mma = B > 1;
  const int nn = B > 8 ? 2 : 1, Bp = 8 * nn, n_parts = H / 16;
  std::vector<size_t> o_xa(Ly + 1), o_ssa(Ly + 1), o_attb(Ly), o_xmb(Ly), o_ssm(Ly), o_hb(Ly);
  if (mma) {
    for (int l = 0; l <= Ly; ++l) {  // entry Ly: the final hidden state (LM head input)
      o_xa[l] = take(4 * (size_t)Bp * H);
      o_ssa[l] = take(4 * (size_t)B * n_parts);
    }
    for (int l = 0; l < Ly; ++l) {
      o_attb[l] = take(4 * (size_t)Bp * qd);
      o_xmb[l] = take(4 * (size_t)Bp * H);
      o_ssm[l] = take(4 * (size_t)B * n_parts);
      o_hb[l] = take(4 * (size_t)Bp * F);
    }
  }
  h->act_bytes = (int64_t)(off - act0);
  h->dev_block_bytes = off;
  ce = cudaMalloc(&h->dev_block, off);
  if (ce != cudaSuccess) {
    delete h;
    return fail(nullptr, MK_ERR_OOM, "cudaMalloc of graph and activation buffers failed");
  }
  char *base = static_cast<char *>(h->dev_block);
  cudaMemset(base, 0, off);

  // tables
  std::vector<mk::DevTask> tasks(G.type.size());
  for (size_t i = 0; i < tasks.size(); ++i) {
    tasks[i].type = (uint8_t)G.type[i];
    tasks[i].pad = 0;
    tasks[i].layer = (uint16_t)(G.layer[i] < 0 ? 0xFFFF : G.layer[i]);
    tasks[i].idx = (uint32_t)G.idx[i];
    tasks[i].dep = G.dep[i];
    tasks[i].trig = G.trig[i];
  }
  std::vector<mk::DevEvent> events(G.ev_count.size());
  for (size_t e = 0; e < events.size(); ++e)
    events[e] = mk::DevEvent{(uint32_t)G.ev_count[e], G.ev_first[e], G.ev_last[e], 0u};
  std::vector<int32_t> op_list;
  h->op_offset.assign(G.n_ops + 1, 0);
  for (int o = 0; o < G.n_ops; ++o) {
    h->op_offset[o] = (int32_t)op_list.size();
    op_list.insert(op_list.end(), G.op_tasks[o].begin(), G.op_tasks[o].end());
  }
  h->op_offset[G.n_ops] = (int32_t)op_list.size();
  std::vector<float> rope((size_t)c.kv_capacity * D);
  for (int pos = 0; pos < c.kv_capacity; ++pos)
    for (int i = 0; i < D / 2; ++i) {
      const double inv_freq = std::pow(c.rope_theta, -(2.0 * i) / (double)D);
      const double ang = (double)pos * inv_freq;
      rope[(size_t)pos * D + 2 * i] = (float)std::cos(ang);
      rope[(size_t)pos * D + 2 * i + 1] = (float)std::sin(ang);
    }
  h->layers.resize(Ly);
  for (int l = 0; l < Ly; ++l) {
    mk::DevLayer &L = h->layers[l];
    std::memset(&L, 0, sizeof(L));
    L.qkv = reinterpret_cast<float *>(base + o_qkv[l]);
    L.part = S > 1 ? reinterpret_cast<float *>(base + o_part[l]) : nullptr;
    L.att = reinterpret_cast<float *>(base + o_att[l]);
    L.xm = reinterpret_cast<float *>(base + o_xm[l]);
    L.h = reinterpret_cast<float *>(base + o_h[l]);
    L.x_in = reinterpret_cast<float *>(base + o_x) + (size_t)l * B * H;
    L.x_out = reinterpret_cast<float *>(base + o_x) + (size_t)(l + 1) * B * H;
    if (mma) {
      L.xa = reinterpret_cast<uint16_t *>(base + o_xa[l]);
      L.ssa = reinterpret_cast<float *>(base + o_ssa[l]);
      L.attb = reinterpret_cast<uint16_t *>(base + o_attb[l]);
      L.xmb = reinterpret_cast<uint16_t *>(base + o_xmb[l]);
      L.ssm = reinterpret_cast<float *>(base + o_ssm[l]);
      L.hb = reinterpret_cast<uint16_t *>(base + o_hb[l]);
      L.xa_next = reinterpret_cast<uint16_t *>(base + o_xa[l + 1]);
      L.ssa_next = reinterpret_cast<float *>(base + o_ssa[l + 1]);
    }
  }
  ce = cudaMemcpy(base + o_tasks, tasks.data(), sizeof(mk::DevTask) * tasks.size(),
                  cudaMemcpyHostToDevice);
  if (ce == cudaSuccess && !events.empty())
    ce = cudaMemcpy(base + o_events, events.data(), sizeof(mk::DevEvent) * events.size(),
                    cudaMemcpyHostToDevice);
  if (ce == cudaSuccess)
    ce = cudaMemcpy(base + o_optasks, op_list.data(), 4 * op_list.size(), cudaMemcpyHostToDevice);
  if (ce == cudaSuccess)
    ce = cudaMemcpy(base + o_rope, rope.data(), 4 * rope.size(), cudaMemcpyHostToDevice);
  if (ce == cudaSuccess)
    ce = cudaMemcpy(base + o_layers, h->layers.data(), sizeof(mk::DevLayer) * Ly,
                    cudaMemcpyHostToDevice);
  if (ce != cudaSuccess) {
    mk_status st = cuda_fail(nullptr, ce, "upload of graph tables");
    mk_destroy(h);
    return st;
  }
  h->d_layers = reinterpret_cast<mk::DevLayer *>(base + o_layers);
  h->d_op_tasks = reinterpret_cast<int32_t *>(base + o_optasks);

  Params &p = h->base;
  std::memset(&p, 0, sizeof(p));
  p.tasks = reinterpret_cast<const mk::DevTask *>(base + o_tasks);
  p.events = reinterpret_cast<const mk::DevEvent *>(base + o_events);
  p.counters = reinterpret_cast<uint32_t *>(base + o_counters);
  p.arrivals = reinterpret_cast<uint32_t *>(base + o_arrivals);
  p.epoch = reinterpret_cast<uint32_t *>(base + o_epoch);
  p.status = reinterpret_cast<int32_t *>(base + o_status);
  p.n_tasks = (int)tasks.size();
  p.n_events = (int)events.size();
  if (t.dispatch > 0) {
    p.dispatch = 1;
    p.n_workers = W;
    p.q_cap = q_cap;
    p.q_list = reinterpret_cast<int32_t *>(base + o_qlist);
    p.q_tail = reinterpret_cast<uint32_t *>(base + o_qtail);
  }
  p.layers = h->d_layers;
  p.x0 = reinterpret_cast<float *>(base + o_x);
  p.x_final = reinterpret_cast<float *>(base + o_x) + (size_t)Ly * B * H;
  p.lm_val = reinterpret_cast<float *>(base + o_lmv);
  p.lm_idx = reinterpret_cast<int32_t *>(base + o_lmi);
  p.rope = reinterpret_cast<const float *>(base + o_rope);
  p.B = B; p.H = H; p.Hq = c.n_q_heads; p.Hkv = c.n_kv_heads; p.D = D; p.F = F; p.V = V;
  p.Ly = Ly; p.Lcap = c.kv_capacity; p.rep = rep; p.grp = grp; p.n_qkv = n_qkv; p.qdim = qd;
  p.rep_p = rep_p;
  p.eps = c.rms_eps;
  p.attn_scale = (float)(1.0 / std::sqrt((double)D));
  p.qkv_rows = T.qkv_rows; p.o_rows = T.o_rows; p.gu_rows = T.gu_rows;
  p.down_rows = T.down_rows; p.lm_rows = T.lm_rows; p.S = S; p.chunk = T.attn_chunk;
  p.n_lm = T.n_lm;
  // GEMV rows per ring stage: a multiple of 8 when at least 8 rows fit,
  // else 6, 4, 2 or 1 (the kernel batches rows 8 or fewer at a time)
  auto rps = [&](int K) {
    const int raw = std::min(mk::kMaxRowsPerStage, t.ring_stage_bytes / (2 * K));
    if (raw >= 8) return raw / 8 * 8;
    for (int r : {6, 4, 2}) if (raw >= r) return r;
    return 1;
  };
  p.rps_qkv = rps(H);
  p.rps_o = rps(qd);
  p.rps_gu = std::max(2, rps(H) & ~1);
  p.rps_down = rps(F);
  p.rps_lm = rps(H);
  // KV positions per stage: K and V of pps rows each, a multiple of 8 (whole
  // 1024-byte swizzle atoms), at most 256 (the TMA box height limit) and, with
  // splits fixed at build time, at most one split (a multiple of 64), so a
  // short split is one exact box
  p.jit = jit_attention(c, t) ? 1 : 0;
  p.n_attn = T.n_attn;
  p.pps = std::min(p.jit ? 256 : std::min(256, T.attn_chunk), t.ring_stage_bytes / (4 * D) / 8 * 8);
  if (t.kv_page_size > 0) {
    // paged pools: a stage must stay inside one page; splits start at
    // multiples of 64 (JIT pieces: stages start at multiples of pps within a
    // pair) and pages hold multiples of 64 rows, so a stage of a divisor of
    // 64 rows never crosses a page
    int q = 64;
    while (q > p.pps) q >>= 1;
    p.pps = q;
    p.page_size = t.kv_page_size;
    p.max_pages = (c.kv_capacity + t.kv_page_size - 1) / t.kv_page_size;
  }
  if (p.pps < 8) {
    mk_destroy(h);
    return fail(nullptr, MK_ERR_ARG, "ring stage smaller than 8 K/V rows");
  }
  if (mma) {
    const MmaTiling mt = mma_tiling(T, t.ring_stage_bytes, nn);
    p.mma = 1;
    p.nn = nn;
    p.n_parts = n_parts;
    p.mb_qkv = mt.mb[0];
    p.mb_o = mt.mb[1];
    p.mb_gu = mt.mb[2];
    p.mb_down = mt.mb[3];
    p.mb_lm = mt.mb[4];
    p.kcb_qkv = mt.kcb[0];
    p.kcb_o = mt.kcb[1];
    p.kcb_gu = mt.kcb[2];
    p.kcb_down = mt.kcb[3];
    p.kcb_lm = mt.kcb[4];
    p.xfb = reinterpret_cast<uint16_t *>(base + o_xa[Ly]);
    p.ssf = reinterpret_cast<float *>(base + o_ssa[Ly]);
    if (std::min({p.kcb_qkv, p.kcb_o, p.kcb_gu, p.kcb_down, p.kcb_lm}) < 8) {
      mk_destroy(h);
      return fail(nullptr, MK_ERR_ARG, "ring stage too small for the tensor-core tiles");
    }
  }
  p.ring_stages = t.ring_stages;
  p.stage_bytes = t.ring_stage_bytes;
  p.l2_prefetch_bytes = t.l2_prefetch_bytes;
  p.evict_first = t.l2_stream_policy >= 0 ? 1 : 0;
  p.timeout_ns = (unsigned long long)t.wait_timeout_us * 1000ull;
  p.trace = nullptr;
  p.n_steps = 1;
  *out = h;
  return MK_OK;
}

mk_status mk_load_weights(mk_handle *h, const mk_weights *w, void *stream) {
  if (!h) return fail(nullptr, MK_ERR_ARG, "null handle");
  if (h->host_only) return fail(h, MK_ERR_ARG, "handle was made by mk_plan_graph");
  if (!w || !w->embed || !w->final_norm || !w->attn_norm || !w->wq || !w->wk || !w->wv ||
      !w->q_norm || !w->k_norm || !w->wo || !w->mlp_norm || !w->w_gate || !w->w_up ||
      !w->w_down)
    return fail(h, MK_ERR_ARG, "missing weight pointer");
  const mk_model_config &c = h->cfg;
  if ((w->lm_head == nullptr) != (c.tied_embeddings != 0))
    return fail(h, MK_ERR_ARG, "lm_head must be NULL exactly when embeddings are tied");
  cudaSetDevice(h->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int H = c.hidden, F = c.ffn, D = c.head_dim, Ly = c.n_layers, V = c.vocab;
  const int rep = c.n_q_heads / c.n_kv_heads, grp = (rep + 2) * D;
  const size_t n_qkv = (size_t)c.n_kv_heads * grp, qd = (size_t)c.n_q_heads * D;
  // arena layout
  size_t off = 0;
  auto take = [&](size_t elems) {
    size_t o = off;
    off = up256(off + 2 * elems);
    return o;
  };
  std::vector<size_t> o_qkv(Ly), o_o(Ly), o_gu(Ly), o_dn(Ly), o_an(Ly), o_qn(Ly), o_kn(Ly),
      o_mn(Ly);
  for (int l = 0; l < Ly; ++l) {
    o_qkv[l] = take(n_qkv * H);
    o_o[l] = take((size_t)H * qd);
    o_gu[l] = take((size_t)2 * F * H);
    o_dn[l] = take((size_t)H * F);
  }
  // batch >= 2: projection matrices in mma.sync fragment order, the LM head
  // padded to whole 16-row m-tiles and kept apart from the (row-major)
  // embedding table even when the two are tied
  const bool mma = h->base.mma != 0;
  const size_t Vp = mma ? ((size_t)V + 15) / 16 * 16 : (size_t)V;
  const bool lm_shares_embed = c.tied_embeddings && !mma;
  const size_t o_lm = lm_shares_embed ? 0 : take(Vp * H);
  const size_t o_emb = take((size_t)V * H);
  for (int l = 0; l < Ly; ++l) {
    o_an[l] = take(H);
    o_qn[l] = take(D);
    o_kn[l] = take(D);
    o_mn[l] = take(H);
  }
  const size_t o_fn = take(H);
  if (!h->arena || h->arena_bytes != off) {
    if (h->arena) cudaFree(h->arena);
    h->arena = nullptr;
    if (cudaMalloc(&h->arena, off) != cudaSuccess) {
      h->arena_bytes = 0;
      return fail(h, MK_ERR_OOM, "cudaMalloc of the weight arena failed");
    }
    h->arena_bytes = off;
  }
  char *A = static_cast<char *>(h->arena);
  cudaError_t e = cudaSuccess;
  auto cpy = [&](char *dst, const void *src, size_t bytes) {
    if (e == cudaSuccess) e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDefault, st);
  };
  auto cp = [&](size_t dst_off, const void *src, size_t bytes) { cpy(A + dst_off, src, bytes); };
  const size_t row = 2 * (size_t)H;
  // Row-major matrices in arena row order, written at dst: QKV group-major,
  // gate/up interleaved.
  auto put_qkv = [&](char *dst, int l) {
    for (int g = 0; g < c.n_kv_heads; ++g) {
      char *d = dst + (size_t)g * grp * row;
      cpy(d, static_cast<const char *>(w->wq[l]) + (size_t)g * rep * D * row, (size_t)rep * D * row);
      cpy(d + (size_t)rep * D * row, static_cast<const char *>(w->wk[l]) + (size_t)g * D * row,
          (size_t)D * row);
      cpy(d + (size_t)(rep + 1) * D * row,
          static_cast<const char *>(w->wv[l]) + (size_t)g * D * row, (size_t)D * row);
    }
  };
  auto put_gu = [&](char *dst, int l) {
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(dst, 2 * row, w->w_gate[l], row, row, F, cudaMemcpyDefault, st);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(dst + row, 2 * row, w->w_up[l], row, row, F, cudaMemcpyDefault, st);
  };
  const void *lm_src = c.tied_embeddings ? w->embed : w->lm_head;
  if (!mma) {
    for (int l = 0; l < Ly; ++l) {
      put_qkv(A + o_qkv[l], l);
      cp(o_o[l], w->wo[l], (size_t)H * qd * 2);
      put_gu(A + o_gu[l], l);
      cp(o_dn[l], w->w_down[l], (size_t)H * F * 2);
    }
    if (!c.tied_embeddings) cp(o_lm, w->lm_head, (size_t)V * H * 2);
  } else {
    // each matrix goes row-major into a staging buffer, then a kernel writes
    // it to the arena in fragment order; the LM head goes in row slabs
    const size_t tmp_bytes =
        2 * std::max({n_qkv * H, (size_t)H * qd, (size_t)2 * F * H, (size_t)H * F});
    void *tmp = nullptr;
    if (cudaMalloc(&tmp, tmp_bytes) != cudaSuccess)
      return fail(h, MK_ERR_OOM, "cudaMalloc of the weight staging buffer failed");
    char *T = static_cast<char *>(tmp);
    auto frag = [&](size_t dst_off, int rows, int K) {
      if (e == cudaSuccess) e = mk::permute_to_fragments(A + dst_off, T, rows, K, st);
    };
    for (int l = 0; l < Ly; ++l) {
      put_qkv(T, l);
      frag(o_qkv[l], (int)n_qkv, H);
      cpy(T, w->wo[l], (size_t)H * qd * 2);
      frag(o_o[l], H, (int)qd);
      put_gu(T, l);
      frag(o_gu[l], 2 * F, H);
      cpy(T, w->w_down[l], (size_t)H * F * 2);
      frag(o_dn[l], H, F);
    }
    const int slab = (int)std::min<size_t>((size_t)V, tmp_bytes / row / 16 * 16);
    for (int r0 = 0; r0 < V; r0 += slab) {
      const int n = std::min(slab, V - r0);
      cpy(T, static_cast<const char *>(lm_src) + (size_t)r0 * row, (size_t)n * row);
      // m-tile r0 / 16 of the padded head: 512-byte blocks, H / 16 per m-tile
      frag(o_lm + (size_t)(r0 / 16) * (H / 16) * 512, n, H);
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);  // the staging buffer is freed next
    cudaFree(tmp);
  }
  for (int l = 0; l < Ly; ++l) {
    cp(o_an[l], w->attn_norm[l], (size_t)H * 2);
    cp(o_qn[l], w->q_norm[l], (size_t)D * 2);
    cp(o_kn[l], w->k_norm[l], (size_t)D * 2);
    cp(o_mn[l], w->mlp_norm[l], (size_t)H * 2);
  }
  cp(o_emb, w->embed, (size_t)V * H * 2);
  cp(o_fn, w->final_norm, (size_t)H * 2);
  if (e != cudaSuccess) return cuda_fail(h, e, "weight copy");
  for (int l = 0; l < Ly; ++l) {
    mk::DevLayer &L = h->layers[l];
    L.w_qkv = reinterpret_cast<const uint16_t *>(A + o_qkv[l]);
    L.w_o = reinterpret_cast<const uint16_t *>(A + o_o[l]);
    L.w_gu = reinterpret_cast<const uint16_t *>(A + o_gu[l]);
    L.w_down = reinterpret_cast<const uint16_t *>(A + o_dn[l]);
    L.attn_norm = reinterpret_cast<const uint16_t *>(A + o_an[l]);
    L.q_norm = reinterpret_cast<const uint16_t *>(A + o_qn[l]);
    L.k_norm = reinterpret_cast<const uint16_t *>(A + o_kn[l]);
    L.mlp_norm = reinterpret_cast<const uint16_t *>(A + o_mn[l]);
    L.gain_next = reinterpret_cast<const uint16_t *>(A + (l + 1 < Ly ? o_an[l + 1] : o_fn));
  }
  e = cudaMemcpyAsync(h->d_layers, h->layers.data(), sizeof(mk::DevLayer) * Ly,
                      cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);  // the host array is reused
  if (e != cudaSuccess) return cuda_fail(h, e, "layer table upload");
  Params &p = h->base;
  p.embed = reinterpret_cast<const uint16_t *>(A + o_emb);
  p.lm_head = reinterpret_cast<const uint16_t *>(A + (lm_shares_embed ? o_emb : o_lm));
  p.final_norm = reinterpret_cast<const uint16_t *>(A + o_fn);
  h->weight_bytes = 0;
  for (int l = 0; l < Ly; ++l)
    h->weight_bytes += 2 * ((int64_t)n_qkv * H + (int64_t)H * qd + 3LL * F * H + 2LL * H + 2LL * D);
  h->weight_bytes += 2 * ((int64_t)(c.tied_embeddings ? 1 : 2) * V * H + H);
  h->loaded = true;
  return MK_OK;
}

}  // extern "C"

namespace {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

}  // namespace

std::string mk::encode_kv_maps(const mk_handle *h, const void *kc, const void *vc, Params *p) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return "cuTensorMapEncodeTiled is not available from the driver";
  const mk_model_config &c = h->cfg;
  if ((reinterpret_cast<uintptr_t>(kc) | reinterpret_cast<uintptr_t>(vc)) & 15)
    return "K/V caches must be 16-byte aligned";
  const cuuint64_t rows =
      p->page_size > 0
          ? (cuuint64_t)p->n_pages * c.n_layers * c.n_kv_heads * p->page_size
          : (cuuint64_t)c.n_layers * c.batch * c.n_kv_heads * c.kv_capacity;
  const cuuint64_t dims[2] = {(cuuint64_t)c.head_dim, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)c.head_dim * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)h->base.pps};
  const cuuint32_t estride[2] = {1u, 1u};
  for (int i = 0; i < 2; ++i) {
    CUresult r = enc(i == 0 ? &p->tmap_k : &p->tmap_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                     const_cast<void *>(i == 0 ? kc : vc), dims, strides, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
      return "cuTensorMapEncodeTiled failed (" + std::to_string((int)r) + ")";
  }
  return "";
}

extern "C" {

static mk_status step_args(mk_handle *h, const int32_t *tin, int32_t *tout, int32_t *kvl,
                           void *kc, void *vc, Params *p, int n_pages = 0,
                           const int32_t *page_table = nullptr) {
  if (!h) return fail(nullptr, MK_ERR_ARG, "null handle");
  if (!h->host_only && (h->base.page_size > 0) != (page_table != nullptr))
    return fail(h, MK_ERR_ARG,
                h->base.page_size > 0 ? "the handle was built for paged K/V: use mk_decode_steps_paged"
                                      : "the handle was built for contiguous K/V caches");
  if (h->host_only) return fail(h, MK_ERR_ARG, "handle was made by mk_plan_graph");
  if (!h->loaded) return fail(h, MK_ERR_NOT_LOADED, "mk_load_weights has not been called");
  if (!tin || !tout || !kvl || !kc || !vc) return fail(h, MK_ERR_ARG, "null buffer");
  // K/V rows are moved by bulk / tensor copies, which need 16-byte alignment
  if ((reinterpret_cast<uintptr_t>(kc) | reinterpret_cast<uintptr_t>(vc)) & 15)
    return fail(h, MK_ERR_ARG, "K/V caches must be 16-byte aligned");
  *p = h->base;
  p->tokens_in = tin;
  p->tokens_out = tout;
  p->kv_len = kvl;
  p->k_cache = static_cast<uint16_t *>(kc);
  p->v_cache = static_cast<uint16_t *>(vc);
  if (page_table) {
    if (n_pages < 1) return fail(h, MK_ERR_ARG, "n_pages must be >= 1");
    p->page_table = page_table;
    p->n_pages = n_pages;
  }
  if (h->base.mma) {  // only the batched kernel reads K/V through tensor maps
    const std::string e = mk::encode_kv_maps(h, kc, vc, p);
    if (!e.empty()) return fail(h, MK_ERR_ARG, e);
  }
  return MK_OK;
}

mk_status mk_decode_step(mk_handle *h, const int32_t *d_tokens_in, int32_t *d_tokens_out,
                         int32_t *d_kv_len, void *d_k_cache, void *d_v_cache, float *d_logits,
                         void *stream) {
  Params p;
  mk_status s = step_args(h, d_tokens_in, d_tokens_out, d_kv_len, d_k_cache, d_v_cache, &p);
  if (s != MK_OK) return s;
  p.logits = d_logits;
  p.persistent = 1;
  if (p.dispatch) {  // the scheduler publishes the queues from zero
    cudaError_t e = cudaMemsetAsync(p.q_tail, 0, 4 * (size_t)p.n_workers,
                                    static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(h, e, "queue reset");
  }
  cudaError_t e = mk::launch_persistent(p, h->tune.num_workers + p.dispatch, h->smem,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(h, e, "persistent launch");
  return MK_OK;
}

mk_status mk_decode_steps(mk_handle *h, int n_steps, const int32_t *d_tokens_in,
                          int32_t *d_tokens_out, int32_t *d_kv_len, void *d_k_cache,
                          void *d_v_cache, float *d_logits, void *stream) {
  if (n_steps < 1) return fail(h, MK_ERR_ARG, "n_steps must be >= 1");
  if (h && h->base.dispatch) {
    if (n_steps > 1) return fail(h, MK_ERR_ARG, "dispatch mode runs one step per launch");
    return mk_decode_step(h, d_tokens_in, d_tokens_out, d_kv_len, d_k_cache, d_v_cache,
                          d_logits, stream);
  }
  Params p;
  mk_status s = step_args(h, d_tokens_in, d_tokens_out, d_kv_len, d_k_cache, d_v_cache, &p);
  if (s != MK_OK) return s;
  p.logits = d_logits;
  p.persistent = 1;
  p.n_steps = n_steps;
  cudaError_t e = mk::launch_persistent(p, h->tune.num_workers, h->smem,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(h, e, "persistent launch");
  return MK_OK;
}

mk_status mk_decode_steps_paged(mk_handle *h, int n_steps, const int32_t *d_tokens_in,
                                int32_t *d_tokens_out, int32_t *d_kv_len, void *d_k_pool,
                                void *d_v_pool, int n_pages, const int32_t *d_page_table,
                                float *d_logits, void *stream) {
  if (n_steps < 1) return fail(h, MK_ERR_ARG, "n_steps must be >= 1");
  if (!d_page_table) return fail(h, MK_ERR_ARG, "null page table");
  if (h && h->base.dispatch) return fail(h, MK_ERR_ARG, "dispatch mode: use mk_decode_step");
  Params p;
  mk_status s = step_args(h, d_tokens_in, d_tokens_out, d_kv_len, d_k_pool, d_v_pool, &p,
                          n_pages, d_page_table);
  if (s != MK_OK) return s;
  p.logits = d_logits;
  p.persistent = 1;
  p.n_steps = n_steps;
  cudaError_t e = mk::launch_persistent(p, h->tune.num_workers, h->smem,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(h, e, "persistent launch");
  return MK_OK;
}

mk_status mk_decode_step_perop(mk_handle *h, const int32_t *d_tokens_in, int32_t *d_tokens_out,
                               int32_t *d_kv_len, void *d_k_cache, void *d_v_cache,
                               float *d_logits, void *stream) {
  Params p;
  mk_status s = step_args(h, d_tokens_in, d_tokens_out, d_kv_len, d_k_cache, d_v_cache, &p);
  if (s != MK_OK) return s;
  p.logits = d_logits;
  p.persistent = 0;
  p.dispatch = 0;
  for (int o = 0; o + 1 < (int)h->op_offset.size(); ++o) {
    const int n = h->op_offset[o + 1] - h->op_offset[o];
    if (n == 0) continue;
    p.task_list = h->d_op_tasks + h->op_offset[o];
    cudaError_t e = mk::launch_tasks(p, n, h->smem, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(h, e, "per-operator launch");
  }
  return MK_OK;
}

mk_status mk_sync_status(mk_handle *h, void *stream, int32_t *detail) {
  if (!h || h->host_only) return fail(h, MK_ERR_ARG, "no device state");
  cudaSetDevice(h->device);
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(h, e, "stream synchronize");
  int32_t st[4] = {0, 0, 0, 0};
  e = cudaMemcpy(st, h->base.status, sizeof(st), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(h, e, "status read");
  if (detail) std::memcpy(detail, st, sizeof(st));
  if (st[0] == mk::kDevTimeout) {
    char buf[160];
    std::snprintf(buf, sizeof(buf), "event wait timed out (task %d, event %d, block %d)", st[1],
                  st[2], st[3]);
    return fail(h, MK_ERR_TIMEOUT, buf);
  }
  if (st[0] != 0) {
    char buf[160];
    std::snprintf(buf, sizeof(buf), "device rejected the step inputs (sequence %d)", st[2]);
    return fail(h, MK_ERR_DEVICE, buf);
  }
  return MK_OK;
}

mk_status mk_reset(mk_handle *h, void *stream) {
  if (!h || h->host_only) return fail(h, MK_ERR_ARG, "no device state");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t ne = std::max<size_t>(1, h->graph.ev_count.size());
  cudaError_t e = cudaMemsetAsync(h->base.counters, 0, 4 * ne, st);
  if (e == cudaSuccess)
    e = cudaMemsetAsync(h->base.arrivals, 0,
                        4 * (size_t)h->cfg.n_layers * h->cfg.batch * h->cfg.n_kv_heads, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->base.epoch, 0, 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->base.status, 0, 16, st);
  if (e != cudaSuccess) return cuda_fail(h, e, "reset");
  return MK_OK;
}

mk_status mk_graph_export(const mk_handle *h, mk_graph_view *out) {
  if (!h || !out) return fail(nullptr, MK_ERR_ARG, "null argument");
  const mk::TaskGraph &G = h->graph;
  std::memset(out, 0, sizeof(*out));
  out->n_tasks = (int32_t)G.type.size();
  out->n_events = (int32_t)G.ev_count.size();
  out->n_edges = (int32_t)G.edge_src.size();
  out->num_workers = G.num_workers;
  out->task_type = G.type.data();
  out->task_op = G.op.data();
  out->task_layer = G.layer.data();
  out->task_idx = G.idx.data();
  out->task_dep = G.dep.data();
  out->task_trig = G.trig.data();
  out->event_count = G.ev_count.data();
  out->event_first = G.ev_first.data();
  out->event_last = G.ev_last.data();
  out->edge_src = G.edge_src.data();
  out->edge_dst = G.edge_dst.data();
  const mk::Tiling &T = G.tiling;
  out->qkv_rows = T.qkv_rows;
  out->o_rows = T.o_rows;
  out->gu_rows = T.gu_rows;
  out->down_rows = T.down_rows;
  out->lm_rows = T.lm_rows;
  out->attn_splits = T.attn_splits;
  out->attn_chunk = T.attn_chunk;
  if (h->cfg.batch > 1 && T.qkv_rows > 0) {
    const MmaTiling mt = mma_tiling(T, h->tune.ring_stage_bytes, (h->cfg.batch + 7) / 8);
    for (int i = 0; i < 5; ++i) {
      out->mma_mb[i] = mt.mb[i];
      out->mma_kcb[i] = mt.kcb[i];
    }
  }
  return MK_OK;
}

mk_status mk_get_info(const mk_handle *h, mk_info *out) {
  if (!h || !out) return fail(nullptr, MK_ERR_ARG, "null argument");
  std::memset(out, 0, sizeof(*out));
  out->device = h->device;
  out->num_workers = h->tune.num_workers;
  out->n_tasks = (int32_t)h->graph.type.size();
  out->n_events = (int32_t)h->graph.ev_count.size();
  out->n_ops = h->graph.n_ops;
  out->smem_bytes = (int32_t)h->smem;
  out->ring_stages = h->tune.ring_stages;
  out->ring_stage_bytes = h->tune.ring_stage_bytes;
  out->weight_bytes = h->weight_bytes;
  out->act_bytes = h->act_bytes;
  return MK_OK;
}

mk_status mk_final_hidden(const mk_handle *h, const float **d_ptr) {
  if (!h || !d_ptr || h->host_only) return fail(nullptr, MK_ERR_ARG, "no device state");
  *d_ptr = h->base.x_final;
  return MK_OK;
}

mk_status mk_debug_set_event_count(mk_handle *h, int event, int count, void *stream) {
  if (!h || h->host_only) return fail(h, MK_ERR_ARG, "no device state");
  if (event < 0 || event >= (int)h->graph.ev_count.size() || count < 0)
    return fail(h, MK_ERR_ARG, "event out of range");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  uint32_t v = (uint32_t)count;
  if (e == cudaSuccess)
    e = cudaMemcpy((char *)h->base.events + sizeof(mk::DevEvent) * event, &v, 4,
                   cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(h, e, "event table write");
  return MK_OK;
}

mk_status mk_set_trace(mk_handle *h, void *d_buf, int64_t bytes) {
  if (!h || h->host_only) return fail(h, MK_ERR_ARG, "no device state");
  if (d_buf && bytes < (int64_t)64 * (int64_t)h->graph.type.size())
    return fail(h, MK_ERR_ARG, "trace buffer smaller than 64 bytes per task");
  h->base.trace = static_cast<unsigned long long *>(d_buf);
  return MK_OK;
}

mk_status mk_set_timeout_us(mk_handle *h, unsigned timeout_us) {
  if (!h || timeout_us == 0) return fail(h, MK_ERR_ARG, "bad argument");
  h->tune.wait_timeout_us = timeout_us;
  h->base.timeout_ns = (unsigned long long)timeout_us * 1000ull;
  return MK_OK;
}

const char *mk_last_error(const mk_handle *h) {
  return h ? h->err.c_str() : g_last_error.c_str();
}

void mk_destroy(mk_handle *h) {
  if (!h) return;
  if (!h->host_only && h->device >= 0) {
    cudaSetDevice(h->device);
    if (h->dev_block) cudaFree(h->dev_block);
    if (h->arena) cudaFree(h->arena);
  }
  delete h;
}

}  // extern "C"
