// Persistent worker kernel for one decode step, sm_100a.
//
// Execution model (MPK abstract; "Mirage Persistent Kernel (MPK)" page,
// section 5.1; MPK review by zhaifeiyue, section 2.4): the step's task graph is
// executed inside ONE kernel.  Each CTA is a worker pinned to one SM.  Worker w
// runs the linearised tasks w, w + W, w + 2W, ... in order.  A task first waits
// until its dependency event has collected `count` triggers in this step, runs
// its body, and then adds one to its trigger event with a release atomic.
// Counters are never reset: in step e (1-based) an event is complete when its
// counter reaches count * e.
//
// CTA layout: 8 compute warps run the task bodies; 1 producer warp streams
// everything a task reads that does not depend on the step's results (weight
// tiles, cached K/V rows) into a shared-memory ring with cp.async.bulk and
// mbarrier transaction counts.  The producer runs ahead across task
// boundaries, so the next task's weights are in flight while the compute
// warps wait for its dependency event.
//
// Every wait is bounded (%globaltimer deadline); on expiry the kernel records
// the error in the status words, stops issuing copies, waits for the copies it
// already issued, and returns.
#include <cuda_runtime.h>

#include <cstdint>

#include "runtime.cuh"

namespace mk {
namespace {

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(uint32_t *p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void compute_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kComputeThreads) : "memory");
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf2f(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

__device__ __forceinline__ uint16_t f2bf(float f) {  // round to nearest even
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float dot8(const uint4 w, const float *x) {
  float a = bf_lo(w.x) * x[0];
  a = fmaf(bf_hi(w.x), x[1], a);
  a = fmaf(bf_lo(w.y), x[2], a);
  a = fmaf(bf_hi(w.y), x[3], a);
  a = fmaf(bf_lo(w.z), x[4], a);
  a = fmaf(bf_hi(w.z), x[5], a);
  a = fmaf(bf_lo(w.w), x[6], a);
  a = fmaf(bf_hi(w.w), x[7], a);
  return a;
}

// ---------------------------------------------------------------------------
// Shared memory layout (identical computation on host: see smem_bytes()).
// ---------------------------------------------------------------------------
enum Ctl { kAbort = 0, kEpoch = 1, kConsumed = 2, kIssued = 3, kCtlWords = 16 };

struct Smem {
  uint8_t *ring;
  uint64_t *full, *empty;
  volatile int *ctl;
  // GEMV scratch
  float *red;   // [2][kMaxRowsPerStage][kComputeWarps]
  float *ss;    // [kComputeWarps]
  float *lmv;   // [kMaxRowsPerStage]
  int *lmi;     // [kMaxRowsPerStage]
  // attention scratch
  float *q;     // [kMaxRep][kMaxHeadDim]
  uint16_t *knew, *vnew;  // [kMaxHeadDim] bf16
  float *sc;    // [kMaxRep][pps]
  float *mls;   // [3][kMaxRep]: running max, running sum, rescale
  float *ored;  // [npg][kMaxRep][kMaxHeadDim]
};

__host__ __device__ inline size_t align_to(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct SmemOffsets {
  size_t full, empty, ctl, red, ss, lmv, lmi, q, knew, vnew, sc, mls, ored, total;
};

__host__ __device__ inline SmemOffsets smem_offsets(int stages, int stage_bytes, int pps,
                                                    int head_dim) {
  SmemOffsets o;
  size_t p = (size_t)stages * stage_bytes;
  o.full = p;
  p += 8 * (size_t)stages;
  o.empty = p;
  p += 8 * (size_t)stages;
  o.ctl = p;
  p += 4 * kCtlWords;
  p = align_to(p, 16);
  // GEMV scratch
  size_t g = p;
  o.red = g;
  g += 4 * 2 * kMaxRowsPerStage * kComputeWarps;
  o.ss = g;
  g += 4 * kComputeWarps;
  o.lmv = g;
  g += 4 * kMaxRowsPerStage;
  o.lmi = g;
  g += 4 * kMaxRowsPerStage;
  // attention scratch (shares the same bytes: a CTA runs one task at a time)
  size_t a = p;
  o.q = a;
  a += 4 * kMaxRep * kMaxHeadDim;
  o.knew = a;
  a += 2 * kMaxHeadDim;
  o.vnew = a;
  a += 2 * kMaxHeadDim;
  o.sc = a;
  a += 4 * (size_t)kMaxRep * pps;
  o.mls = a;
  a += 4 * 3 * kMaxRep;
  a = align_to(a, 16);
  o.ored = a;
  int npg = kComputeThreads / (head_dim / 2);
  a += 4 * (size_t)npg * kMaxRep * head_dim;
  o.total = align_to(g > a ? g : a, 128);
  return o;
}

__device__ __forceinline__ Smem carve(uint8_t *base, const Params &p) {
  SmemOffsets o = smem_offsets(p.ring_stages, p.stage_bytes, p.pps, p.D);
  Smem s;
  s.ring = base;
  s.full = reinterpret_cast<uint64_t *>(base + o.full);
  s.empty = reinterpret_cast<uint64_t *>(base + o.empty);
  s.ctl = reinterpret_cast<volatile int *>(base + o.ctl);
  s.red = reinterpret_cast<float *>(base + o.red);
  s.ss = reinterpret_cast<float *>(base + o.ss);
  s.lmv = reinterpret_cast<float *>(base + o.lmv);
  s.lmi = reinterpret_cast<int *>(base + o.lmi);
  s.q = reinterpret_cast<float *>(base + o.q);
  s.knew = reinterpret_cast<uint16_t *>(base + o.knew);
  s.vnew = reinterpret_cast<uint16_t *>(base + o.vnew);
  s.sc = reinterpret_cast<float *>(base + o.sc);
  s.mls = reinterpret_cast<float *>(base + o.mls);
  s.ored = reinterpret_cast<float *>(base + o.ored);
  return s;
}

__device__ void record_error(const Params &p, int code, int task, int event) {
  if (atomicCAS(p.status, 0, code) == 0) {
    p.status[1] = task;
    p.status[2] = event;
    p.status[3] = (int)blockIdx.x;
    __threadfence();
  }
}

// ---------------------------------------------------------------------------
// What each task streams through the ring.
// ---------------------------------------------------------------------------
struct Gemv {
  const uint16_t *w;  // first row of the operator's weight matrix (arena)
  int K;              // columns
  int row0, row1;     // arena rows of this task
  int rps;            // rows per ring stage
};

__device__ __forceinline__ Gemv gemv_of(const Params &p, int type, int layer, int idx) {
  Gemv g;
  const DevLayer *L = layer < p.Ly ? p.layers + layer : nullptr;
  switch (type) {
    case 2:  // QKV
      g.w = L->w_qkv; g.K = p.H; g.rps = p.rps_qkv;
      g.row0 = idx * p.qkv_rows; g.row1 = min(p.n_qkv, g.row0 + p.qkv_rows);
      break;
    case 5:  // O projection
      g.w = L->w_o; g.K = p.qdim; g.rps = p.rps_o;
      g.row0 = idx * p.o_rows; g.row1 = min(p.H, g.row0 + p.o_rows);
      break;
    case 6:  // gate/up, rows interleaved
      g.w = L->w_gu; g.K = p.H; g.rps = p.rps_gu;
      g.row0 = 2 * idx * p.gu_rows; g.row1 = min(2 * p.F, g.row0 + 2 * p.gu_rows);
      break;
    case 7:  // down
      g.w = L->w_down; g.K = p.F; g.rps = p.rps_down;
      g.row0 = idx * p.down_rows; g.row1 = min(p.H, g.row0 + p.down_rows);
      break;
    default:  // 8: LM head
      g.w = p.lm_head; g.K = p.H; g.rps = p.rps_lm;
      g.row0 = idx * p.lm_rows; g.row1 = min(p.V, g.row0 + p.lm_rows);
      break;
  }
  return g;
}

struct AttnSpan {
  int b, g, s, L;      // sequence, kv head, split, cached rows before the step
  int p0, cached_end;  // cached rows [p0, cached_end) of this split
  bool has_new;        // the split holds position L (the new row)
  bool active;         // the split holds any position
};

__device__ __forceinline__ AttnSpan attn_span(const Params &p, int idx) {
  AttnSpan a;
  a.s = idx % p.S;
  int bg = idx / p.S;
  a.g = bg % p.Hkv;
  a.b = bg / p.Hkv;
  a.L = p.kv_len[a.b];
  a.p0 = a.s * p.chunk;
  int end = a.p0 + p.chunk;
  a.cached_end = min(end, a.L);
  a.has_new = a.L >= a.p0 && a.L < end;
  a.active = a.p0 <= a.L;
  return a;
}

__device__ __forceinline__ size_t kv_row(const Params &p, int layer, int b, int g, int row) {
  return ((((size_t)layer * p.B + b) * p.Hkv + g) * p.Lcap + row) * p.D;
}

// Number of ring stages a task consumes.
__device__ __forceinline__ int task_stages(const Params &p, const DevTask &t) {
  int type = t.type;
  if (type == 2 || (type >= 5 && type <= 8)) {
    Gemv g = gemv_of(p, type, t.layer, (int)t.idx);
    return (g.row1 - g.row0 + g.rps - 1) / g.rps;
  }
  if (type == 3) {
    AttnSpan a = attn_span(p, (int)t.idx);
    int n = a.cached_end - a.p0;
    return n > 0 ? (n + p.pps - 1) / p.pps : 0;
  }
  return 0;
}

// Source ranges of stage `st` of a task: up to two contiguous byte ranges.
struct Copy {
  const void *src0, *src1;
  uint32_t bytes0, bytes1;
};

__device__ __forceinline__ Copy stage_copy(const Params &p, const DevTask &t, int st) {
  Copy c{nullptr, nullptr, 0u, 0u};
  int type = t.type;
  if (type == 3) {
    AttnSpan a = attn_span(p, (int)t.idx);
    int r0 = a.p0 + st * p.pps;
    int n = min(p.pps, a.cached_end - r0);
    size_t off = kv_row(p, t.layer, a.b, a.g, r0);
    c.src0 = p.k_cache + off;
    c.src1 = p.v_cache + off;
    c.bytes0 = c.bytes1 = (uint32_t)(n * p.D * 2);
  } else {
    Gemv g = gemv_of(p, type, t.layer, (int)t.idx);
    int r0 = g.row0 + st * g.rps;
    int n = min(g.rps, g.row1 - r0);
    c.src0 = g.w + (size_t)r0 * g.K;
    c.bytes0 = (uint32_t)((size_t)n * g.K * 2);
  }
  return c;
}

// ---------------------------------------------------------------------------
// Producer: one thread streams every stage of the worker's queue.
// ---------------------------------------------------------------------------
struct Queue {
  int first, stride, count;  // tasks first, first + stride, ... (count of them)
};

__device__ void producer_loop(const Params &p, const Smem &sm, const Queue &q) {
  const int NS = p.ring_stages;
  uint32_t k = 0;
  const uint64_t budget = 4ull * p.timeout_ns + 1000000000ull;
  for (int n = 0; n < q.count; ++n) {
    const DevTask t = p.tasks[q.first + n * q.stride];
    const int ns = task_stages(p, t);
    for (int st = 0; st < ns; ++st) {
      const int slot = (int)(k % NS);
      const uint32_t use = k / NS;
      if (use > 0) {
        const uint32_t par = (use - 1) & 1u;
        uint64_t t0 = 0;
        uint32_t spins = 0;
        while (!mbar_test(&sm.empty[slot], par)) {
          if (sm.ctl[kAbort]) goto out;
          if ((++spins & 255u) == 0) {
            uint64_t now = global_timer();
            if (t0 == 0) t0 = now;
            else if (now - t0 > budget) {
              record_error(p, kDevTimeout, q.first + n * q.stride, -1);
              goto out;
            }
          }
        }
      }
      const Copy c = stage_copy(p, t, st);
      uint8_t *dst = sm.ring + (size_t)slot * p.stage_bytes;
      mbar_arrive_expect_tx(&sm.full[slot], c.bytes0 + c.bytes1);
      bulk_g2s(dst, c.src0, c.bytes0, &sm.full[slot]);
      if (c.bytes1) bulk_g2s(dst + p.stage_bytes / 2, c.src1, c.bytes1, &sm.full[slot]);
      ++k;
    }
  }
out:
  sm.ctl[kIssued] = (int)k;
}

// ---------------------------------------------------------------------------
// Compute side helpers
// ---------------------------------------------------------------------------
// Wait until ring stage k is full; false if the CTA is aborting.
__device__ __forceinline__ bool wait_full(const Params &p, const Smem &sm, uint32_t k, int task) {
  const int slot = (int)(k % p.ring_stages);
  const uint32_t par = (k / p.ring_stages) & 1u;
  if (mbar_test(&sm.full[slot], par)) return true;
  uint64_t t0 = 0;
  uint32_t spins = 0;
  while (!mbar_test(&sm.full[slot], par)) {
    if (sm.ctl[kAbort]) return false;
    if ((++spins & 255u) == 0) {
      uint64_t now = global_timer();
      if (t0 == 0) t0 = now;
      else if (now - t0 > 4ull * p.timeout_ns + 1000000000ull) {
        record_error(p, kDevTimeout, task, -1);
        sm.ctl[kAbort] = 1;
        return false;
      }
    }
  }
  return true;
}

__device__ __forceinline__ void release_stage(const Smem &sm, const Params &p, uint32_t k) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.empty[k % p.ring_stages]);
}

// Thread 0 of the compute group: wait (bounded) until event e reached count*epoch.
__device__ bool wait_event(const Params &p, int e, uint32_t epoch, int task) {
  const uint32_t target = p.events[e].count * epoch;
  const uint32_t *ctr = p.counters + e;
  if ((int32_t)(ld_acquire(ctr) - target) >= 0) return true;
  const uint64_t t0 = global_timer();
  uint32_t spins = 0;
  for (;;) {
    if ((int32_t)(ld_acquire(ctr) - target) >= 0) return true;
    if (++spins > 64) __nanosleep(32);
    if ((spins & 63u) == 0 && global_timer() - t0 > p.timeout_ns) {
      record_error(p, kDevTimeout, task, e);
      return false;
    }
  }
}

// ---------------------------------------------------------------------------
// GEMV task body (batch 1): prologue RMSNorm, weight stream, fused epilogue.
// ---------------------------------------------------------------------------
__device__ bool gemv_task(const Params &p, const Smem &sm, const DevTask &t, uint32_t &k,
                          int task_id) {
  const int type = t.type;
  const int layer = t.layer;
  const Gemv g = gemv_of(p, type, layer, (int)t.idx);
  const DevLayer *L = layer < p.Ly ? p.layers + layer : nullptr;
  const float *act;
  const uint16_t *gain = nullptr;
  switch (type) {
    case 2: act = L->x_in; gain = L->attn_norm; break;
    case 5: act = L->att; break;
    case 6: act = L->xm; gain = L->mlp_norm; break;
    case 7: act = L->h; break;
    default: act = p.x_final; gain = p.final_norm; break;
  }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = g.K, nch = K >> 3;
  const int tpg = nch < kComputeThreads ? nch : kComputeThreads;  // threads per row group
  const int ngroups = kComputeThreads / tpg;
  const int grp = tid / tpg, li = tid - grp * tpg;
  const bool active = grp < ngroups;
  const int wpg = tpg >> 5, wig = li >> 5;  // warps per group, warp index in group
  const int cpt = (nch + tpg - 1) / tpg;

  // activation chunks of this thread
  float x[kMaxChunks][8];
#pragma unroll
  for (int j = 0; j < kMaxChunks; ++j) {
    const int c = li + j * tpg;
    if (active && j < cpt && c < nch) {
      const float4 a = __ldcg(reinterpret_cast<const float4 *>(act + 8 * c));
      const float4 b = __ldcg(reinterpret_cast<const float4 *>(act + 8 * c + 4));
      x[j][0] = a.x; x[j][1] = a.y; x[j][2] = a.z; x[j][3] = a.w;
      x[j][4] = b.x; x[j][5] = b.y; x[j][6] = b.z; x[j][7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[j][i] = 0.f;
    }
  }
  if (gain) {
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxChunks; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(x[j][i], x[j][i], ss);
    ss = warp_sum(ss);
    if (lane == 0) sm.ss[warp] = ss;
    compute_sync();
    float tot = 0.f;
    if (active)
      for (int w = 0; w < wpg; ++w) tot += sm.ss[grp * wpg + w];
    const float inv = rsqrtf(tot / (float)K + p.eps);
#pragma unroll
    for (int j = 0; j < kMaxChunks; ++j) {
      const int c = li + j * tpg;
      if (active && j < cpt && c < nch) {
        const uint4 gw = __ldg(reinterpret_cast<const uint4 *>(gain + 8 * c));
        x[j][0] *= inv * bf_lo(gw.x); x[j][1] *= inv * bf_hi(gw.x);
        x[j][2] *= inv * bf_lo(gw.y); x[j][3] *= inv * bf_hi(gw.y);
        x[j][4] *= inv * bf_lo(gw.z); x[j][5] *= inv * bf_hi(gw.z);
        x[j][6] *= inv * bf_lo(gw.w); x[j][7] *= inv * bf_hi(gw.w);
      }
    }
  }

  const int rows = g.row1 - g.row0;
  const int nst = (rows + g.rps - 1) / g.rps;
  float best_v = -INFINITY;
  int best_i = 0x7fffffff;
  for (int st = 0; st < nst; ++st) {
    const int r_here = min(g.rps, rows - st * g.rps);
    if (!wait_full(p, sm, k, task_id)) {
      sm.ctl[kAbort] = 1;
    }
    if (!sm.ctl[kAbort]) {
      const uint16_t *ws =
          reinterpret_cast<const uint16_t *>(sm.ring + (size_t)(k % p.ring_stages) * p.stage_bytes);
      float *red = sm.red + (st & 1) * kMaxRowsPerStage * kComputeWarps;
      if (active) {
        for (int r = grp; r < r_here; r += ngroups) {
          const uint4 *wr = reinterpret_cast<const uint4 *>(ws + (size_t)r * K);
          float acc = 0.f;
#pragma unroll
          for (int j = 0; j < kMaxChunks; ++j) {
            const int c = li + j * tpg;
            if (j < cpt && c < nch) acc += dot8(wr[c], x[j]);
          }
          acc = warp_sum(acc);
          if (lane == 0) red[r * kComputeWarps + wig] = acc;
        }
      }
    }
    release_stage(sm, p, k);
    ++k;
    compute_sync();
    if (sm.ctl[kAbort]) return false;
    const float *red = sm.red + (st & 1) * kMaxRowsPerStage * kComputeWarps;
    const int n0 = g.row0 + st * g.rps;  // first arena row of the stage
    if (type == 6) {
      if (tid < r_here / 2) {
        float gv = 0.f, uv = 0.f;
        for (int w = 0; w < wpg; ++w) {
          gv += red[(2 * tid) * kComputeWarps + w];
          uv += red[(2 * tid + 1) * kComputeWarps + w];
        }
        const float hv = gv / (1.f + __expf(-gv)) * uv;
        L->h[(n0 >> 1) + tid] = hv;
      }
    } else if (tid < r_here) {
      float v = 0.f;
      for (int w = 0; w < wpg; ++w) v += red[tid * kComputeWarps + w];
      const int n = n0 + tid;
      if (type == 2) {
        L->qkv[n] = v;
      } else if (type == 5) {
        L->xm[n] = __ldcg(L->x_in + n) + v;
      } else if (type == 7) {
        L->x_out[n] = __ldcg(L->xm + n) + v;
      } else {
        if (p.logits) p.logits[n] = v;
        if (v > best_v || (v == best_v && n < best_i)) {
          best_v = v;
          best_i = n;
        }
      }
    }
  }
  if (type == 8) {
    if (tid < kMaxRowsPerStage) {
      sm.lmv[tid] = best_v;
      sm.lmi[tid] = best_i;
    }
    compute_sync();
    if (tid == 0) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
      const int nf = min(g.rps, rows);
      for (int f = 0; f < nf; ++f) {
        const float v = sm.lmv[f];
        const int i = sm.lmi[f];
        if (v > bv || (v == bv && i < bi)) {
          bv = v;
          bi = i;
        }
      }
      if (bi == 0x7fffffff) bi = g.row0;  // all values NaN: keep a valid index
      p.lm_val[(int)t.idx] = bv;
      p.lm_idx[(int)t.idx] = bi;
    }
  }
  return true;
}

// ---------------------------------------------------------------------------
// Attention: one (sequence b, kv head g, split s).
// ---------------------------------------------------------------------------
// Scores, softmax update and PV for n rows of K and V held in shared memory.
__device__ __forceinline__ void attn_block(const Params &p, const Smem &sm, const uint16_t *Ks,
                                           const uint16_t *Vs, int n, const float (&qr)[kMaxRep][4],
                                           float (&o)[kMaxRep][2]) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int D = p.D, rep = p.rep, dpl = D >> 5;
  // 1. scores s[h][j] = q_h . k_j (q already scaled by 1/sqrt(D))
  for (int j = warp; j < n; j += kComputeWarps) {
    float kf[4];
    if (dpl == 4) {
      const uint2 kv = *reinterpret_cast<const uint2 *>(Ks + (size_t)j * D + 4 * lane);
      kf[0] = bf_lo(kv.x); kf[1] = bf_hi(kv.x); kf[2] = bf_lo(kv.y); kf[3] = bf_hi(kv.y);
    } else {
      const uint32_t kv = *reinterpret_cast<const uint32_t *>(Ks + (size_t)j * D + 2 * lane);
      kf[0] = bf_lo(kv); kf[1] = bf_hi(kv); kf[2] = 0.f; kf[3] = 0.f;
    }
    float mine = 0.f;
#pragma unroll
    for (int h = 0; h < kMaxRep; ++h) {
      if (h < rep) {
        float d = qr[h][0] * kf[0];
        d = fmaf(qr[h][1], kf[1], d);
        d = fmaf(qr[h][2], kf[2], d);
        d = fmaf(qr[h][3], kf[3], d);
        d = warp_sum(d);
        if (lane == h) mine = d;
      }
    }
    if (lane < rep) sm.sc[lane * p.pps + j] = mine;
  }
  compute_sync();
  // 2. online softmax update, one warp per head
  if (warp < rep) {
    const int h = warp;
    float *s = sm.sc + h * p.pps;
    const float m_old = sm.mls[h];
    float mx = -INFINITY;
    for (int j = lane; j < n; j += 32) mx = fmaxf(mx, s[j]);
    mx = warp_max(mx);
    const float m_new = fmaxf(m_old, mx);
    float sum = 0.f;
    for (int j = lane; j < n; j += 32) {
      const float e = __expf(s[j] - m_new);
      s[j] = e;
      sum += e;
    }
    sum = warp_sum(sum);
    if (lane == 0) {
      const float alpha = m_old == -INFINITY ? 0.f : __expf(m_old - m_new);
      sm.mls[h] = m_new;
      sm.mls[kMaxRep + h] = sm.mls[kMaxRep + h] * alpha + sum;
      sm.mls[2 * kMaxRep + h] = alpha;
    }
  }
  compute_sync();
  // 3. o = alpha * o + sum_j p_j v_j on (dim pair, position group)
  const int half = D >> 1;
  const int dp = tid % half, pg = tid / half, npg = kComputeThreads / half;
#pragma unroll
  for (int h = 0; h < kMaxRep; ++h) {
    if (h < rep) {
      const float a = sm.mls[2 * kMaxRep + h];
      o[h][0] *= a;
      o[h][1] *= a;
    }
  }
  for (int j = pg; j < n; j += npg) {
    const uint32_t vv = *reinterpret_cast<const uint32_t *>(Vs + (size_t)j * D + 2 * dp);
    const float v0 = bf_lo(vv), v1 = bf_hi(vv);
#pragma unroll
    for (int h = 0; h < kMaxRep; ++h) {
      if (h < rep) {
        const float pj = sm.sc[h * p.pps + j];
        o[h][0] = fmaf(pj, v0, o[h][0]);
        o[h][1] = fmaf(pj, v1, o[h][1]);
      }
    }
  }
  compute_sync();
}

__device__ bool attn_task(const Params &p, const Smem &sm, const DevTask &t, uint32_t &k,
                          int task_id) {
  const AttnSpan a = attn_span(p, (int)t.idx);
  if (!a.active) return true;  // the split starts past the new row: nothing to do
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int D = p.D, rep = p.rep, dpl = D >> 5;
  const DevLayer &L = p.layers[t.layer];
  const float *qkv = L.qkv + (size_t)a.b * p.n_qkv + (size_t)a.g * p.grp;
  const float *rope = p.rope + (size_t)a.L * D;  // [D/2][2]

  // prologue: per-head RMSNorm + RoPE of q (and of the new k when this split
  // holds position L; v is only rounded)
  for (int row = warp; row < rep + 2; row += kComputeWarps) {
    if (row >= rep && !a.has_new) continue;
    float v[4];
    for (int i = 0; i < dpl; ++i) v[i] = __ldcg(qkv + row * D + lane + 32 * i);
    if (row <= rep) {  // q heads and k
      const uint16_t *gain = row < rep ? L.q_norm : L.k_norm;
      float ss = 0.f;
      for (int i = 0; i < dpl; ++i) ss = fmaf(v[i], v[i], ss);
      ss = warp_sum(ss);
      const float inv = rsqrtf(ss / (float)D + p.eps);
      for (int i = 0; i < dpl; ++i) v[i] = v[i] * inv * bf2f(gain[lane + 32 * i]);
      const int hp = dpl >> 1;  // dims lane + 32 i pair with lane + 32 (i + hp)
      for (int i = 0; i < hp; ++i) {
        const int d = lane + 32 * i;
        const float c = rope[2 * d], s = rope[2 * d + 1];
        const float x0 = v[i], x1 = v[i + hp];
        v[i] = x0 * c - x1 * s;
        v[i + hp] = x1 * c + x0 * s;
      }
    }
    if (row < rep) {
      for (int i = 0; i < dpl; ++i) sm.q[row * kMaxHeadDim + lane + 32 * i] = v[i] * p.attn_scale;
    } else {
      uint16_t *cache = row == rep ? p.k_cache : p.v_cache;
      uint16_t *dst = row == rep ? sm.knew : sm.vnew;
      const size_t off = kv_row(p, t.layer, a.b, a.g, a.L);
      for (int i = 0; i < dpl; ++i) {
        const uint16_t hb = f2bf(v[i]);
        cache[off + lane + 32 * i] = hb;
        dst[lane + 32 * i] = hb;
      }
    }
  }
  if (tid < kMaxRep) {
    sm.mls[tid] = -INFINITY;
    sm.mls[kMaxRep + tid] = 0.f;
    sm.mls[2 * kMaxRep + tid] = 1.f;
  }
  compute_sync();
  float qr[kMaxRep][4];
#pragma unroll
  for (int h = 0; h < kMaxRep; ++h)
#pragma unroll
    for (int i = 0; i < 4; ++i)
      qr[h][i] = (h < rep && i < dpl) ? sm.q[h * kMaxHeadDim + dpl * lane + i] : 0.f;
  float o[kMaxRep][2];
#pragma unroll
  for (int h = 0; h < kMaxRep; ++h) o[h][0] = o[h][1] = 0.f;

  const int cached = a.cached_end - a.p0;
  const int nst = cached > 0 ? (cached + p.pps - 1) / p.pps : 0;
  for (int st = 0; st < nst; ++st) {
    const int n = min(p.pps, cached - st * p.pps);
    bool ok = wait_full(p, sm, k, task_id);
    if (!ok) sm.ctl[kAbort] = 1;
    compute_sync();
    if (sm.ctl[kAbort]) {
      release_stage(sm, p, k);
      ++k;
      return false;
    }
    const uint16_t *Ks =
        reinterpret_cast<const uint16_t *>(sm.ring + (size_t)(k % p.ring_stages) * p.stage_bytes);
    const uint16_t *Vs = Ks + p.stage_bytes / 4;  // second half of the stage
    attn_block(p, sm, Ks, Vs, n, qr, o);
    release_stage(sm, p, k);
    ++k;
  }
  if (a.has_new) attn_block(p, sm, sm.knew, sm.vnew, 1, qr, o);

  // reduce the position groups, then write the normalised output (one split)
  // or the unnormalised partial with its running max and sum (several splits)
  const int half = D >> 1;
  const int dp = tid % half, pg = tid / half, npg = kComputeThreads / half;
#pragma unroll
  for (int h = 0; h < kMaxRep; ++h) {
    if (h < rep) {
      sm.ored[(pg * kMaxRep + h) * D + 2 * dp] = o[h][0];
      sm.ored[(pg * kMaxRep + h) * D + 2 * dp + 1] = o[h][1];
    }
  }
  compute_sync();
  for (int oi = tid; oi < rep * D; oi += kComputeThreads) {
    const int h = oi / D, d = oi - h * D;
    float v = 0.f;
    for (int q = 0; q < npg; ++q) v += sm.ored[(q * kMaxRep + h) * D + d];
    const int head = a.g * rep + h;
    if (p.S == 1) {
      L.att[(size_t)a.b * p.qdim + head * D + d] = v / sm.mls[kMaxRep + h];
    } else {
      float *dst = L.part + (((size_t)a.b * p.Hq + head) * p.S + a.s) * (D + 2);
      dst[d] = v;
      if (d == 0) {
        dst[D] = sm.mls[h];
        dst[D + 1] = sm.mls[kMaxRep + h];
      }
    }
  }
  return true;
}

__device__ void merge_task(const Params &p, const DevTask &t) {
  const int b = (int)t.idx / p.Hkv, g = (int)t.idx % p.Hkv;
  const DevLayer &L = p.layers[t.layer];
  const int Lb = p.kv_len[b];
  const int ns = min(p.S, Lb / p.chunk + 1);  // splits that hold any position
  const int D = p.D;
  for (int oi = threadIdx.x; oi < p.rep * D; oi += kComputeThreads) {
    const int h = oi / D, d = oi - h * D;
    const int head = g * p.rep + h;
    const float *base = L.part + ((size_t)b * p.Hq + head) * p.S * (D + 2);
    float M = -INFINITY;
    for (int s = 0; s < ns; ++s) M = fmaxf(M, __ldcg(base + s * (D + 2) + D));
    float den = 0.f, num = 0.f;
    for (int s = 0; s < ns; ++s) {
      const float w = __expf(__ldcg(base + s * (D + 2) + D) - M);
      den = fmaf(w, __ldcg(base + s * (D + 2) + D + 1), den);
      num = fmaf(w, __ldcg(base + s * (D + 2) + d), num);
    }
    L.att[(size_t)b * p.qdim + head * D + d] = num / den;
  }
}

__device__ void embed_task(const Params &p) {
  for (int b = 0; b < p.B; ++b) {
    const uint16_t *e = p.embed + (size_t)p.tokens_in[b] * p.H;
    for (int i = threadIdx.x; i < p.H; i += kComputeThreads) p.x0[(size_t)b * p.H + i] = bf2f(e[i]);
  }
}

__device__ void argmax_task(const Params &p, uint32_t epoch) {
  const int b = threadIdx.x;
  if (b < p.B) {
    float bv = -INFINITY;
    int bi = 0;
    bool any = false;
    for (int j = 0; j < p.n_lm; ++j) {
      const float v = __ldcg(p.lm_val + (size_t)b * p.n_lm + j);
      if (!any || v > bv) {
        bv = v;
        bi = __ldcg(p.lm_idx + (size_t)b * p.n_lm + j);
        any = true;
      }
    }
    p.tokens_out[b] = bi;
    p.kv_len[b] = p.kv_len[b] + 1;
  }
  if (threadIdx.x == 0 && p.persistent) *p.epoch = epoch;
}

// ---------------------------------------------------------------------------
// The worker kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) mk_worker_kernel(const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const Smem sm = carve(smem_raw, p);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;

  Queue q;
  if (p.persistent) {
    q.first = blockIdx.x;
    q.stride = gridDim.x;
    q.count = q.first < p.n_tasks ? (p.n_tasks - q.first + q.stride - 1) / q.stride : 0;
  } else {
    q.first = p.task_list[blockIdx.x];
    q.stride = 1;
    q.count = 1;
  }
  if (q.count == 0) return;

  if (tid == 0) {
    for (int s = 0; s < p.ring_stages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kComputeWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    int bad = 0;
    if (*(volatile int32_t *)p.status != 0) bad = 1;  // an earlier step failed: no-op
    for (int b = 0; b < p.B && !bad; ++b) {
      const int L = p.kv_len[b], tok = p.tokens_in[b];
      if (L < 0 || L + 1 > p.Lcap || tok < 0 || tok >= p.V) {
        record_error(p, kDevBadInput, -1, b);
        bad = 1;
      }
    }
    sm.ctl[kAbort] = bad;
    sm.ctl[kEpoch] = p.persistent ? (int)(*(volatile uint32_t *)p.epoch + 1u) : 0;
    sm.ctl[kConsumed] = 0;
    sm.ctl[kIssued] = 0;
  }
  __syncthreads();
  if (sm.ctl[kAbort]) return;  // nothing issued yet

  if (warp == kComputeWarps) {
    if ((tid & 31) == 0) producer_loop(p, sm, q);
    __syncwarp();
  } else {
    const uint32_t epoch = (uint32_t)sm.ctl[kEpoch];
    uint32_t k = 0;
    for (int n = 0; n < q.count; ++n) {
      const int id = q.first + n * q.stride;
      const DevTask t = p.tasks[id];
      if (p.persistent && t.dep >= 0 && tid == 0) {
        if (!wait_event(p, t.dep, epoch, id)) sm.ctl[kAbort] = 1;
      }
      compute_sync();
      if (sm.ctl[kAbort]) break;
      bool ok = true;
      switch (t.type) {
        case 1: embed_task(p); break;
        case 2: case 5: case 6: case 7: case 8: ok = gemv_task(p, sm, t, k, id); break;
        case 3: ok = attn_task(p, sm, t, k, id); break;
        case 4: merge_task(p, t); break;
        case 9: argmax_task(p, epoch); break;
        default: break;  // empty task
      }
      if (!ok) break;
      compute_sync();
      if (p.persistent && t.trig >= 0 && tid == 0) {
        __threadfence();
        red_release_add(p.counters + t.trig, 1u);
      }
    }
    if (tid == 0) sm.ctl[kConsumed] = (int)k;
  }
  __syncthreads();
  if (sm.ctl[kAbort] && warp == kComputeWarps && (tid & 31) == 0) {
    // wait for every copy issued but not consumed before the CTA exits
    const uint32_t from = (uint32_t)sm.ctl[kConsumed], to = (uint32_t)sm.ctl[kIssued];
    for (uint32_t kk = from; kk < to; ++kk) {
      const int slot = (int)(kk % p.ring_stages);
      const uint32_t par = (kk / p.ring_stages) & 1u;
      const uint64_t t0 = global_timer();
      while (!mbar_test(&sm.full[slot], par)) {
        if (global_timer() - t0 > 1000000000ull) break;
      }
    }
  }
}

}  // namespace

size_t worker_smem_bytes(int stages, int stage_bytes, int pps, int head_dim) {
  return smem_offsets(stages, stage_bytes, pps, head_dim).total;
}

cudaError_t worker_configure(size_t smem) {
  return cudaFuncSetAttribute(mk_worker_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)smem);
}

cudaError_t worker_max_blocks(int *blocks, size_t smem) {
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, mk_worker_kernel, kThreads, smem);
}

// Persistent launch: one cooperative grid of `workers` CTAs.
cudaError_t launch_persistent(const Params &p, int workers, size_t smem, cudaStream_t stream) {
  void *args[] = {const_cast<Params *>(&p)};
  return cudaLaunchCooperativeKernel((const void *)mk_worker_kernel, dim3(workers), dim3(kThreads),
                                     args, smem, stream);
}

// Per-operator launch: one CTA per task of the operator.
cudaError_t launch_tasks(const Params &p, int n_ctas, size_t smem, cudaStream_t stream) {
  mk_worker_kernel<<<n_ctas, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mk
