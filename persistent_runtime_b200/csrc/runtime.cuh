// Structures shared by the host API and the device runtime of the decode-step
// megakernel.  Plain data only, so the host side can include this file
// without nvcc.
#pragma once

#include <cuda.h>  // CUtensorMap (a plain 128-byte descriptor type)

#include <cstdint>

namespace mk {

constexpr int kComputeWarps = 8;
constexpr int kStateSlots = kComputeWarps < 8 ? kComputeWarps : 8;  // attention warp states in smem
constexpr int kComputeThreads = kComputeWarps * 32;  // threads that run task bodies
constexpr int kThreads = kComputeThreads + 32;       // + one producer (TMA) warp
constexpr int kMaxChunks = 8;          // 16-byte weight chunks per thread and row
constexpr int kMaxCpt = (16384 / 8 + kComputeThreads - 1) / kComputeThreads;  // K <= 16384
constexpr int kMaxRowsPerStage = 64;   // GEMV rows in one ring stage
constexpr int kRedRows = 256;          // GEMV rows whose warp partials shared memory holds
constexpr int kMaxRep = 8;             // q heads per kv head
constexpr int kMaxHeadDim = 128;
constexpr int kMaxBatch = 16;
// Tensor-core projections (batch >= 2): mma.sync m16n8k16, bf16 in, fp32 out.
constexpr int kMmaMaxMB = 6;    // 16-row m-tiles per row block (accumulators per warp)
// 16-column k-blocks per warp and ring stage: a stage's B fragments take
// kpw x nn x 4 registers per thread, so one column tile (batch <= 8) affords
// twice as many as two
__host__ __device__ constexpr int mma_max_kpw(int nn) { return nn == 1 ? 6 : 3; }
constexpr int kMmaCredFloats = kComputeWarps * 4 * 16 * 9;  // cross-warp reduction buffer

// Device status words: [0] status code, [1] task, [2] event, [3] block.
enum DeviceStatus : int { kDevOk = 0, kDevTimeout = -6, kDevBadInput = -7 };

struct DevTask {  // 16 bytes
  uint8_t type;
  uint8_t pad;
  uint16_t layer;  // 0xFFFF for EMBED / LM_HEAD / ARGMAX
  uint32_t idx;    // index of the task within its operator
  int32_t dep;     // event this task waits for, -1 = none
  int32_t trig;    // event this task triggers, -1 = none
};

struct DevEvent {  // 16 bytes
  uint32_t count;  // triggers needed per step
  int32_t first, last;
  uint32_t pad;
};

// Per-layer device pointers: weight arena slices and activation buffers.
// With batch >= 2 the four projection matrices are stored in mma.sync
// A-fragment order (see frag_permute_kernel in the worker), not row-major.
struct DevLayer {
  const uint16_t *w_qkv;   // [n_kv_heads * (rep + 2) * D][H], group-major rows
  const uint16_t *w_o;     // [H][Hq * D]
  const uint16_t *w_gu;    // [2F][H], row 2i = gate_i, row 2i+1 = up_i
  const uint16_t *w_down;  // [H][F]
  const uint16_t *attn_norm, *q_norm, *k_norm, *mlp_norm;
  float *qkv;   // [B][n_kv_heads * (rep + 2) * D]
  float *part;  // [B][Hq][S][D + 2]: unnormalised o, running max, running sum
  float *att;   // [B][Hq * D]
  float *xm;    // [B][H]  residual stream after attention
  float *h;     // [B][F]  SiLU(gate) * up
  float *x_in;  // [B][H]  residual stream entering the layer
  float *x_out; // [B][H]  residual stream leaving the layer
  // Batch >= 2 only: the projection inputs as two-term bf16 expansions
  // (x = hi + lo) in mma.sync B-fragment order (see opnd_off in the worker),
  // with the following RMSNorm's gain folded in, and per-16-row sums of
  // squares [B][H / 16] of the streams that feed an RMSNorm.
  uint16_t *xa;    // x_in * attn_norm   (QKV input)
  float *ssa;      // sums of squares of x_in
  uint16_t *attb;  // att                (O input)
  uint16_t *xmb;   // xm * mlp_norm      (GATE_UP input)
  float *ssm;      // sums of squares of xm
  uint16_t *hb;    // h                  (DOWN input)
  uint16_t *xa_next;  // DOWN epilogue targets: next layer's xa / ssa (or the
  float *ssa_next;    // final hidden state's), with the gain of that norm
  const uint16_t *gain_next;
};

struct Params {
  // 2-D tensor maps of the K and V caches seen as [Ly * B * Hkv * Lcap][D]
  // bf16 rows: boxes of 64 dims x pps rows, 128-byte swizzle (encoded on the
  // host for every step, since the caches are step arguments)
  alignas(64) CUtensorMap tmap_k;
  alignas(64) CUtensorMap tmap_v;
  // graph
  const DevTask *tasks;
  const DevEvent *events;
  uint32_t *counters;  // one per event, monotone: count * epoch after each step
  uint32_t *arrivals;  // per (layer, sequence, kv head): attention splits finished this step
  uint32_t *epoch;     // steps completed by the persistent kernel
  int32_t *status;     // 4 words, see DeviceStatus
  int n_tasks;
  int n_events;
  int persistent;       // 1: worker w runs tasks w, w + W, ...; 0: one task per CTA
  const int32_t *task_list;  // per-operator mode: task ids, one per CTA
  // dispatch mode (persistent, one step per launch): CTA n_workers is a
  // scheduler that hands ready tasks to the workers through per-worker queues
  // [n_workers][q_cap] of task ids (-1 ends a queue), q_tail[w] = entries
  // published (zeroed before the launch)
  int dispatch, n_workers, q_cap;
  int32_t *q_list;
  uint32_t *q_tail;
  // model
  const DevLayer *layers;
  const uint16_t *embed, *lm_head, *final_norm;
  float *x0, *x_final;     // residual stream before layer 0 / after the last layer
  float *lm_val;           // [B][n_lm] partial argmax values
  int32_t *lm_idx;         // [B][n_lm] partial argmax indices
  const float *rope;       // [kv_capacity][D/2][2] cos, sin
  // step arguments
  int n_steps;  // steps run by this launch (persistent mode): step s reads the
                // tokens step s - 1 wrote and writes tokens_out[s][B]
  const int32_t *tokens_in;
  int32_t *tokens_out;
  int32_t *kv_len;
  uint16_t *k_cache, *v_cache;  // [Ly][B][Hkv][Lcap][D], or paged pools (below)
  // paged KV (page_size > 0): pools [n_pages][Ly][Hkv][page_size][D]; position
  // pos of sequence b is row pos % page_size of page page_table[b][pos / page_size]
  const int32_t *page_table;    // [B][max_pages]
  int page_size, max_pages, n_pages;
  float *logits;                // [B][V] of the last step, or null
  // shapes
  int B, H, Hq, Hkv, D, F, V, Ly, Lcap, rep, grp, n_qkv, qdim;
  int rep_p;  // rep rounded up to 2, 4 or 8 (the attention instantiations)
  float eps;
  float attn_scale;  // 1 / sqrt(D)
  // tiling
  int qkv_rows, o_rows, gu_rows, down_rows, lm_rows, S, chunk, n_lm;
  // JIT attention (batch >= 2): n_attn tasks per layer cut the live positions
  // of all (sequence, kv head) pairs into equal chunks; S is then the partial
  // slots per pair, chunk 0
  int jit, n_attn;
  int rps_qkv, rps_o, rps_gu, rps_down, rps_lm;  // GEMV rows per ring stage
  int pps;  // KV positions per ring stage (multiple of 8): K then V, D / 64 swizzled boxes each
  // tensor-core projections (batch >= 2)
  int mma;      // 1: projections run on mma.sync with fragment-ordered weights
  int nn;       // 8-sequence column tiles (1 or 2)
  int n_parts;  // H / 16: sum-of-squares partials per sequence
  int mb_qkv, mb_o, mb_gu, mb_down, mb_lm;        // m-tiles per row block
  int kcb_qkv, kcb_o, kcb_gu, kcb_down, kcb_lm;   // k-blocks per ring stage
  uint16_t *xfb;  // operand of the LM head: x_final * final_norm
  float *ssf;     // sums of squares of x_final
  // ring
  int ring_stages, stage_bytes;
  int l2_prefetch_bytes;  // per worker: L2 prefetch distance ahead of the ring
  int evict_first;        // 1: ring copies carry an L2 evict-first cache hint
  unsigned long long timeout_ns;
  // optional task trace: per task id {wait begin, ready, end, worker} (%globaltimer ns)
  unsigned long long *trace;
};

}  // namespace mk
