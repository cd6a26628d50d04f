/*
 * mk.h - C ABI of the decode-step megakernel library (libmk.so).
 *
 * One low-batch decode step of a Qwen3-style decoder runs as ONE persistent
 * kernel launch on one GPU: an SM-level task graph (tGraph) is built on the
 * host once, and a worker kernel with one CTA per SM executes it with event
 * counters and per-SM task queues, with no further launches inside the step.
 *
 * Where the operations come from:
 *   - "MPK: A Compiler and Runtime for Mega-Kernelizing Tensor Programs",
 *     Abstract: an SM-level graph captures data dependencies per SM-sized
 *     task; an in-kernel runtime executes the tasks inside one persistent
 *     kernel with decentralized scheduling across SMs.
 *   - MPK review (zhaifeiyue), section 2.4: event fusion, normalisation so
 *     that every task has at most one dependency event and one trigger event,
 *     BFS linearisation so that an event's fan-out is a [first, last] task
 *     range, scheduling with only atomicAdd and local state.
 *   - "Mirage Persistent Kernel (MPK)" page, section 5.1 (worker kernel with
 *     one resident CTA per worker, dispatch-only scheduler beside it) and
 *     section 5.3 (one call runs the decode; the baseline launches one kernel
 *     per operator and takes the argmax of the logits).
 *
 * Conventions for every call:
 *   - Every function returns mk_status (MK_OK = 0 on success); nothing throws
 *     across the ABI.  mk_last_error(h) gives a text for the last failure on h.
 *   - Pointers named d_* are device pointers on the handle's device; other
 *     pointers are host pointers.  Streams are cudaStream_t passed as void*
 *     (NULL = the legacy default stream).
 *   - bf16 data is IEEE bfloat16 bit patterns (uint16_t); matrices are
 *     row-major [out_features][in_features], the nn.Linear layout.
 *   - Calls on one handle are not thread-safe; use one handle per thread.
 */
#ifndef MK_H
#define MK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct mk_handle mk_handle;

typedef enum {
  MK_OK = 0,
  MK_ERR_ARG = -1,        /* bad argument or unsupported shape */
  MK_ERR_CUDA = -2,       /* a CUDA runtime call failed */
  MK_ERR_OOM = -3,        /* device or host allocation failed */
  MK_ERR_GRAPH = -4,      /* graph construction found an inconsistency (a cycle) */
  MK_ERR_NOT_LOADED = -5, /* mk_decode_step before mk_load_weights */
  MK_ERR_TIMEOUT = -6,    /* a device-side event wait ran out of time */
  MK_ERR_DEVICE = -7      /* device-side check failed (kv_len or token range) */
} mk_status;

/* Task types as stored in the task table (mk_graph_view.task_type). */
enum {
  MK_TASK_GENERIC = 0, /* task of a graph built by mk_graph_from_edges */
  MK_TASK_EMBED = 1,   /* x0[b] = float(E[token_b])                                  */
  MK_TASK_QKV = 2,     /* RMSNorm prologue, q/k/v rows of one kv-group-aligned tile    */
  MK_TASK_ATTN = 3,    /* one (sequence, kv head, KV split) of decode attention; the   */
                       /* split that finishes last merges the splits (online softmax)  */
  MK_TASK_MERGE = 4,   /* reserved (decode graphs merge inside the last ATTN split)    */
  MK_TASK_OPROJ = 5,   /* O projection tile, residual add epilogue                     */
  MK_TASK_GATEUP = 6,  /* RMSNorm prologue, gate/up tile, SiLU(g)*u epilogue           */
  MK_TASK_DOWN = 7,    /* down projection tile, residual add epilogue                  */
  MK_TASK_LMHEAD = 8,  /* final RMSNorm prologue, LM-head tile, partial argmax epilogue */
  MK_TASK_ARGMAX = 9,  /* argmax over the partials, token write, kv_len += 1           */
  MK_TASK_EMPTY = 10   /* normalisation task: waits on one event, triggers another     */
};

/* Shape of the decoder and of the batch state one handle serves. */
typedef struct {
  int n_layers;        /* decoder layers (Ly) */
  int hidden;          /* H, multiple of 256 */
  int n_q_heads;       /* Hq */
  int n_kv_heads;      /* Hkv, divides Hq */
  int head_dim;        /* D: 64 or 128 */
  int ffn;             /* F, multiple of 256 */
  int vocab;           /* V */
  int tied_embeddings; /* 1: the LM head is the embedding matrix */
  float rms_eps;       /* epsilon of every RMSNorm */
  double rope_theta;   /* RoPE base */
  int batch;           /* B sequences advanced per step, 1..16 */
  int kv_capacity;     /* cache rows per (layer, sequence, kv head) */
} mk_model_config;

/* Tuning knobs; pass NULL for defaults.  A zero field also means "default". */
typedef struct {
  int num_workers;           /* worker CTAs W; 0 = one per SM of the device */
  int col_align;             /* rows per GEMV task rounded up to this (4 at batch 1, else 16;
                                batch >= 2 needs a multiple of 16) */
  int attn_tasks_per_worker; /* at most this many attention tasks per worker (1) */
  int attn_min_chunk;        /* smallest KV positions per attention task (64) */
  int ring_stages;           /* shared-memory weight ring depth (4) */
  int ring_stage_bytes;      /* bytes per ring stage, multiple of 1024 (49152) */
  int l2_prefetch_bytes;     /* per-worker L2 prefetch distance ahead of the ring, used while
                                the compute warps wait for an O projection's event (the
                                step's attention window, when HBM is otherwise idle);
                                default at batch 1: 2097152 when one layer's weights
                                exceed 1 MB per worker, else off (the prefetches of small
                                layers run layers ahead and leave L2 before use); off at
                                batch >= 2 (attention streams the caches there);
                                negative = off */
  unsigned wait_timeout_us;  /* device-side bound on one event wait (2,000,000) */
  int kv_page_size;          /* 0: contiguous K/V caches; else positions per page of the
                                paged pools (a multiple of 64), see mk_decode_steps_paged */
  int l2_stream_policy;      /* L2 policy of streamed weights and cached K/V: 0 or 1 =
                                evict-first (default: they are read once per step and
                                must not displace code, activations and counters),
                                -1 = the normal policy */
  int attn_jit;              /* attention tasks resolved at run time (MPK review, "Direction 4":
                                data-dependent operators JIT, the rest ahead of time):
                                attn_tasks_per_worker * W tasks per layer cut the live
                                positions of all (sequence, kv head) pairs into equal
                                chunks, which may cross pairs.  0 = off (default): splits
                                fixed at build time from kv_capacity; 1 = on (batch >= 2
                                only; MK_ERR_ARG at batch 1) */
  int dispatch;              /* 0 = static queues: worker w runs tasks w, w + W, ... and waits
                                on their events itself (default); 1 = a scheduler CTA in the
                                same launch hands ready tasks to the workers (the pages'
                                dispatch design, kept as an ablation): W = SMs - 1 workers
                                unless num_workers is set, one step per launch
                                (mk_decode_step only) */
} mk_tuning;

/* Weights: device pointers, bf16, row-major [out][in].  Per-layer arrays are
 * host arrays of n_layers device pointers.  lm_head must be NULL iff tied. */
typedef struct {
  const void *embed;      /* [vocab][hidden] */
  const void *final_norm; /* [hidden] */
  const void *lm_head;    /* [vocab][hidden] or NULL when tied */
  const void *const *attn_norm; /* [hidden] */
  const void *const *wq;        /* [n_q_heads*head_dim][hidden] */
  const void *const *wk;        /* [n_kv_heads*head_dim][hidden] */
  const void *const *wv;        /* [n_kv_heads*head_dim][hidden] */
  const void *const *q_norm;    /* [head_dim], shared by all q heads */
  const void *const *k_norm;    /* [head_dim], shared by all kv heads */
  const void *const *wo;        /* [hidden][n_q_heads*head_dim] */
  const void *const *mlp_norm;  /* [hidden] */
  const void *const *w_gate;    /* [ffn][hidden] */
  const void *const *w_up;      /* [ffn][hidden] */
  const void *const *w_down;    /* [hidden][ffn] */
} mk_weights;

/* Host copies of the graph tables (owned by the handle, valid until
 * mk_destroy).  Tasks are in linear (BFS) order; task i runs on worker
 * i mod num_workers; worker w runs its tasks in increasing order. */
typedef struct {
  int32_t n_tasks, n_events, n_edges, num_workers;
  const int32_t *task_type, *task_op, *task_layer, *task_idx, *task_dep, *task_trig;
  const int32_t *event_count, *event_first, *event_last;
  const int32_t *edge_src, *edge_dst; /* raw data dependencies, final task ids */
  /* tiling chosen for the decode graph (0 for generic graphs) */
  int32_t qkv_rows, o_rows, gu_rows, down_rows, lm_rows, attn_splits, attn_chunk;
  /* batch >= 2: tensor-core tiles of QKV, O, GATE_UP, DOWN, LM_HEAD (in that
   * order): 16-row m-tiles of a full pass (a task's rows run in passes of at
   * most 256, one TMEM accumulator each) and 16-column k-blocks per ring stage
   * of such a pass, for the handle's ring stage size (0 at batch 1, and a
   * kcb of 0 when a stage cannot hold one k-block: mk_build_graph rejects it) */
  int32_t mma_mb[5], mma_kcb[5];
} mk_graph_view;

/* Sizes and roofline inputs of a built handle. */
typedef struct {
  int32_t device, num_workers, n_tasks, n_events, n_ops;
  int32_t smem_bytes, ring_stages, ring_stage_bytes;
  int64_t weight_bytes;  /* bytes of the weight arena (every weight once) */
  int64_t act_bytes;     /* bytes of the library-owned activation buffers */
} mk_info;

/*
 * mk_plan_graph - build the task graph of one decode step on the host only
 * (no CUDA call).  Tiling, raw events from region overlaps, fusion, reduction,
 * normalisation and BFS linearisation follow the MPK review (zhaifeiyue),
 * section 2.4.  num_workers must be >= 1.  The handle can be inspected with
 * mk_graph_export and must be released with mk_destroy; it cannot run steps.
 * Errors: MK_ERR_ARG (shape unsupported), MK_ERR_GRAPH, MK_ERR_OOM.
 */
mk_status mk_plan_graph(const mk_model_config *cfg, const mk_tuning *tuning, int num_workers,
                        mk_handle **out);

/*
 * mk_graph_from_edges - the same fusion/normalisation/linearisation pipeline
 * on an arbitrary op-ordered task DAG (for property tests).  Task i has key
 * (task_op[i], task_idx[i]) (keys unique); every edge src -> dst must go from
 * an earlier op to a later one.  Host only.  Errors: MK_ERR_ARG, MK_ERR_GRAPH.
 */
mk_status mk_graph_from_edges(int n_tasks, const int32_t *task_op, const int32_t *task_idx,
                              int n_edges, const int32_t *edge_src, const int32_t *edge_dst,
                              mk_handle **out);

/*
 * mk_build_graph - plan the graph for `device` (W = its SM count unless
 * tuning->num_workers is set), upload the task/event tables, and allocate the
 * event counters, the step epoch, the status word and the activation buffers
 * (all owned by the handle).  batch 1 runs the CUDA-core worker kernel;
 * batch 2..16 the tensor-core one (projections on tcgen05.mma: the hi/lo
 * activation operand as the 128-row A matrix, the task's weight rows as N,
 * fp32 accumulators in tensor memory; attention on mma.sync over TMA K/V
 * tiles), which needs col_align to be a multiple of 16.  Errors: MK_ERR_ARG
 * (also for a ring stage too small for one tensor-core k-block), MK_ERR_CUDA,
 * MK_ERR_OOM.
 */
mk_status mk_build_graph(const mk_model_config *cfg, const mk_tuning *tuning, int device,
                         mk_handle **out);

/*
 * mk_load_weights - copy the caller's weights into a library-owned arena laid
 * out in task-stream order: QKV rows group-major (per kv head: its q heads,
 * then k, then v), gate and up rows interleaved, every task's weight tile one
 * contiguous range.  For batch >= 2 handles the projection matrices are then
 * permuted on the device into the tcgen05 operand order of their tasks (per
 * pass of at most 256 task rows, per 16-column k-block, 8-row x 16-byte core
 * matrices) and the LM head is padded to whole 16-row tiles (a separate copy
 * even when tied); this uses a temporary device staging
 * buffer of the largest layer matrix and synchronises `stream`.  Copies are
 * ordered on `stream`; the caller may free its tensors once the stream has
 * passed this call.  May be called again to replace the weights.  Errors:
 * MK_ERR_ARG, MK_ERR_OOM, MK_ERR_CUDA.
 */
mk_status mk_load_weights(mk_handle *h, const mk_weights *w, void *stream);

/*
 * mk_decode_step - advance every sequence b by one token with ONE persistent
 * kernel launch on `stream` (asynchronous, stream ordered):
 *   reads d_tokens_in[b]; appends K/V at row d_kv_len[b] of every layer's
 *   cache; attends over d_kv_len[b] + 1 rows at RoPE position d_kv_len[b];
 *   writes d_tokens_out[b] (greedy argmax, lowest index on ties); increments
 *   d_kv_len[b].
 * Buffers (caller owned, device): d_tokens_in/out int32 [batch] (may be the
 * same buffer); d_kv_len int32 [batch]; d_k_cache, d_v_cache bf16
 * [n_layers][batch][n_kv_heads][kv_capacity][head_dim], 16-byte aligned (for
 * batch >= 2 the call encodes two TMA tensor maps of them on the host);
 * d_logits fp32 [batch][vocab] or NULL (then logits are not stored).
 * Misaligned caches are rejected with MK_ERR_ARG before any launch.
 * Device-side failures (kv_len[b] + 1 > kv_capacity or a token out of range:
 * the step writes nothing; an event wait that times out) are recorded in the
 * handle's status word, make later steps no-ops, and are returned by
 * mk_sync_status.  Errors returned here: MK_ERR_NOT_LOADED, MK_ERR_ARG,
 * MK_ERR_CUDA (for instance when the workers cannot all be co-resident).
 */
mk_status mk_decode_step(mk_handle *h, const int32_t *d_tokens_in, int32_t *d_tokens_out,
                         int32_t *d_kv_len, void *d_k_cache, void *d_v_cache, float *d_logits,
                         void *stream);

/*
 * mk_decode_steps - n_steps decode steps in ONE persistent launch, with the
 * greedy token fed back on the device ("Mirage Persistent Kernel (MPK)" page,
 * section 5.3: one call runs the decode).  Step 0 reads d_tokens_in; step s
 * writes d_tokens_out[s * batch + b] and step s + 1 reads it; every step
 * appends one K/V row per (layer, sequence, kv head) and increments
 * d_kv_len[b].  d_logits [batch][vocab] (or NULL) receives the last step's
 * logits.  Results are bitwise those of n_steps calls of mk_decode_step.
 * Weight streams run ahead across step boundaries; K/V rows of a step are
 * read only after the previous step has completed.  Requires
 * kv_len[b] + n_steps <= kv_capacity (else the launch writes nothing and the
 * status word reports MK_ERR_DEVICE).  n_steps must be >= 1.  Errors as for
 * mk_decode_step.
 */
mk_status mk_decode_steps(mk_handle *h, int n_steps, const int32_t *d_tokens_in,
                          int32_t *d_tokens_out, int32_t *d_kv_len, void *d_k_cache,
                          void *d_v_cache, float *d_logits, void *stream);

/*
 * mk_decode_steps_paged - mk_decode_steps with the K/V caches as pools of
 * pages (MPK review, zhaifeiyue, paradigm-positioning paragraph on adoption:
 * paged attention and page allocation have to run inside the megakernel
 * runtime for it to replace a serving stack).  The handle must
 * have been built with tuning->kv_page_size = P > 0 (a multiple of 64).
 * d_k_pool, d_v_pool: bf16 [n_pages][n_layers][n_kv_heads][P][head_dim],
 * 16-byte aligned.  d_page_table: int32 [batch][ceil(kv_capacity / P)];
 * position pos of sequence b is row pos % P of page
 * d_page_table[b][pos / P].  Pages of one sequence may be anywhere in the
 * pool; two sequences must not share a page they write.  Entries for
 * positions [0, kv_len[b] + n_steps) must lie in [0, n_pages), else the
 * launch writes nothing and the status word reports MK_ERR_DEVICE.  All
 * other semantics and errors as mk_decode_steps; results are bitwise those
 * of the contiguous layout.
 */
mk_status mk_decode_steps_paged(mk_handle *h, int n_steps, const int32_t *d_tokens_in,
                                int32_t *d_tokens_out, int32_t *d_kv_len, void *d_k_pool,
                                void *d_v_pool, int n_pages, const int32_t *d_page_table,
                                float *d_logits, void *stream);

/*
 * mk_decode_step_perop - the comparison path: the same task bodies, launched
 * one grid per operator (one CTA per task, no event waits; kernel boundaries
 * order the operators), as in the kernel-per-operator baseline of the MPK
 * page, section 5.3.  Same arguments and results as mk_decode_step; the call
 * only launches kernels, so it can be captured into a CUDA Graph.
 */
mk_status mk_decode_step_perop(mk_handle *h, const int32_t *d_tokens_in, int32_t *d_tokens_out,
                               int32_t *d_kv_len, void *d_k_cache, void *d_v_cache,
                               float *d_logits, void *stream);

/*
 * mk_decode_step_noalloc - mk_decode_step that allocates nothing and keeps
 * every per-step working buffer (event and arrival counters, step epoch,
 * activations, attention partials, LM-head partials, per-layer pointer table)
 * in one static device region of 16 MiB instead of the handle's own buffers.
 * The pages have no counterpart: this exists for callers that cannot call
 * cudaMalloc when they need another stepping context -- cudaMalloc may
 * synchronise the device and cannot run while a stream is being captured,
 * and some programs hand all device memory out through their own allocator
 * once the model is loaded.  The handle (graph tables, weights, status word)
 * is used as built; its own working buffers, and so mk_final_hidden, are left
 * untouched.  Arguments, results and device-side error reporting
 * (mk_sync_status, mk_reset) are those of mk_decode_step.
 * The region is a file-scope static array: every GPU that loads the library
 * holds it until the process exits.  The first call on a device looks up the
 * region's device address (cudaGetSymbolAddress) with that device current;
 * make that first call before any stream capture.  All calls share the one
 * region and clear its counters first, so calls that overlap on the GPU race:
 * order them on one stream.  Errors: MK_ERR_ARG when the step needs more than
 * 16 MiB of working memory (or for bad arguments), MK_ERR_NOT_LOADED,
 * MK_ERR_CUDA.
 */
mk_status mk_decode_step_noalloc(mk_handle *h, const int32_t *d_tokens_in, int32_t *d_tokens_out,
                                 int32_t *d_kv_len, void *d_k_cache, void *d_v_cache,
                                 float *d_logits, void *stream);

/* mk_sync_status - synchronize `stream`, then return the device status word
 * (MK_OK, MK_ERR_TIMEOUT or MK_ERR_DEVICE).  detail (nullable, 4 ints):
 * {status, task id, event id, block}; an event id of -2 after a failure means
 * that a worker exited with copies into its shared memory still outstanding
 * after its bounded wait for them.  The word stays set until mk_reset. */
mk_status mk_sync_status(mk_handle *h, void *stream, int32_t *detail);

/* mk_reset - stream-ordered: zero the event counters, the step epoch and the
 * status word (needed after a device-side failure). */
mk_status mk_reset(mk_handle *h, void *stream);

/* mk_graph_export - fill *out with host views of the tables (see mk_graph_view). */
mk_status mk_graph_export(const mk_handle *h, mk_graph_view *out);

/* mk_get_info - sizes of a handle built with mk_build_graph. */
mk_status mk_get_info(const mk_handle *h, mk_info *out);

/* mk_final_hidden - device pointer to the fp32 [batch][hidden] residual
 * stream after the last layer (before the final norm) of the latest step. */
mk_status mk_final_hidden(const mk_handle *h, const float **d_ptr);

/* mk_debug_set_event_count - test hook: overwrite one event's trigger count in
 * the device table (stream ordered).  Raising it by one makes every waiter of
 * that event time out, which exercises the bounded-wait error path. */
mk_status mk_debug_set_event_count(mk_handle *h, int event, int count, void *stream);

/* mk_set_trace - record, for every task of later steps, eight uint64 words
 * {wait begin, ready, end, (smid << 32) | worker, prologue done, streaming
 * done, bytes the worker has prefetched into L2 so far, first ring stage
 * available} (%globaltimer ns; the phase marks are 0 for tasks without those
 * phases) into the caller's device buffer d_buf of `bytes` >= 64 * n_tasks
 * bytes (task id order).  d_buf = NULL turns tracing off.  The buffer must outlive the steps
 * that use it.  This is the "--profiling" trace of the MPK page, section 7.2. */
mk_status mk_set_trace(mk_handle *h, void *d_buf, int64_t bytes);

/* mk_set_timeout_us - change the device-side bound on one event wait. */
mk_status mk_set_timeout_us(mk_handle *h, unsigned timeout_us);

/* mk_last_error - text of the last failure on h (or of the last failed
 * constructor call when h is NULL).  Never NULL. */
const char *mk_last_error(const mk_handle *h);

/* mk_destroy - free everything the handle owns.  NULL is allowed. */
void mk_destroy(mk_handle *h);

#ifdef __cplusplus
}
#endif

#endif /* MK_H */
