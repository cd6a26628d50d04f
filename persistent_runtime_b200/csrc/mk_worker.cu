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

// Order this thread's earlier (acquire-synchronised) view of global memory
// before its later async-proxy (bulk / tensor copy) reads.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
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

// Global -> shared bulk copy completing on an mbarrier, with an L2 cache
// policy (createpolicy) for the source lines.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// 2-D tiled TMA load of the box at (x, y) of a tensor map (kernel parameter
// space) into shared memory, completing on an mbarrier.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// L2 policy for data read once per step: evict first (or the normal policy).
__device__ __forceinline__ uint64_t stream_policy(bool evict_first) {
  uint64_t pol;
  if (evict_first)
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  else
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
  return pol;
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

__device__ __forceinline__ uint32_t atom_acq_rel_add(uint32_t *p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
               : "memory");
  return old;
}

__device__ __forceinline__ void st_release(uint32_t *p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
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

// (a0, a1) += (w0, w1) * (x0, x1) as one packed fp32x2 FMA (sm_100).
__device__ __forceinline__ void ffma2(float &a0, float &a1, float w0, float w1, float x0,
                                      float x1) {
  asm("{\n\t.reg .b64 A, W, X;\n\t"
      "mov.b64 A, {%0, %1};\n\t"
      "mov.b64 W, {%2, %3};\n\t"
      "mov.b64 X, {%4, %5};\n\t"
      "fma.rn.f32x2 A, W, X, A;\n\t"
      "mov.b64 {%0, %1}, A;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(w0), "f"(w1), "f"(x0), "f"(x1));
}

// acc (even, odd element partial sums) += w (8 bf16) . x (8 fp32)
__device__ __forceinline__ void dot8_acc(const uint4 w, const float *x, float (&acc)[2]) {
  ffma2(acc[0], acc[1], bf_lo(w.x), bf_hi(w.x), x[0], x[1]);
  ffma2(acc[0], acc[1], bf_lo(w.y), bf_hi(w.y), x[2], x[3]);
  ffma2(acc[0], acc[1], bf_lo(w.z), bf_hi(w.z), x[4], x[5]);
  ffma2(acc[0], acc[1], bf_lo(w.w), bf_hi(w.w), x[6], x[7]);
}

// One step of a transposed warp reduction: lanes that differ in bit OFF swap
// halves of their value arrays, so each lane keeps HALF partial sums.  After
// the steps for every lane bit, each lane holds the full warp sum of one of
// the original values (which one follows from its lane bits).
template <int HALF, int OFF>
__device__ __forceinline__ void transpose_step(float *v, int lane) {
  const bool up = (lane & OFF) != 0;
#pragma unroll
  for (int i = 0; i < HALF; ++i) {
    const float send = up ? v[i] : v[i + HALF];
    const float keep = up ? v[i + HALF] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
  }
}

// Warp sums of 8 values with 9 shuffles; lane 4*i returns the sum of v[i].
__device__ __forceinline__ float warp_sum8(float (&v)[8], int lane) {
  transpose_step<4, 16>(v, lane);
  transpose_step<2, 8>(v, lane);
  transpose_step<1, 4>(v, lane);
  float r = v[0];
  r += __shfl_xor_sync(0xffffffffu, r, 2);
  r += __shfl_xor_sync(0xffffffffu, r, 1);
  return r;
}

// Warp sums of 32 values with 31 shuffles; lane i returns the sum of v[i].
__device__ __forceinline__ float warp_sum32(float (&v)[32], int lane) {
  transpose_step<16, 16>(v, lane);
  transpose_step<8, 8>(v, lane);
  transpose_step<4, 4>(v, lane);
  transpose_step<2, 2>(v, lane);
  transpose_step<1, 1>(v, lane);
  return v[0];
}

// ---------------------------------------------------------------------------
// Tensor cores (batch >= 2): mma.sync.m16n8k16, A = weights (16 rows x 16 k,
// row major), B = activations (16 k x 8 sequences), fp32 accumulators.
// Fragment ownership (PTX ISA, "Matrix Fragments for mma.m16n8k16"), lane l,
// g = l / 4, t = l % 4:  A regs {(g, 2t..2t+1), (g+8, 2t..), (g, 2t+8..),
// (g+8, 2t+8..)};  B regs {(2t..2t+1, g), (2t+8..2t+9, g)};  C {(g, 2t),
// (g, 2t+1), (g+8, 2t), (g+8, 2t+1)}.  Weights and activations are stored in
// exactly this order, so each lane fetches its fragment with one 16-byte
// (A) or 8-byte (B) load.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint4 &a, const uint2 &b) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y));
}

// m16n8k8 variant (A 16 x 8: two registers, B 8 x 8: one register).
__device__ __forceinline__ void mma_bf16_k8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5}, {%6}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b));
}

// Four 8 x 8 b16 matrices from shared memory; lanes 8i..8i+7 give the row
// addresses of matrix i.  Plain: thread l receives row l / 4, columns
// 2 (l % 4) and 2 (l % 4) + 1; .trans: rows 2 (l % 4), 2 (l % 4) + 1 of
// column l / 4.
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Activation operands are two-term bf16 expansions x = hi + lo, hi = bf16(x),
// lo = bf16(x - hi): about 16 significant bits, so W x = W hi + W lo (two MMAs
// into one fp32 accumulator) keeps the projection inputs close to fp32 while
// the weights stay exactly bf16.  A single bf16 rounding of every input would
// cost ~0.4 % of the residual stream per layer.
//
// Element (k, sequence b) of an operand with nn 8-column tiles, in bf16
// units: 512-byte blocks per (16-row k-block, column tile), 16 bytes per lane
// inside a block: {hi b0, hi b1, lo b0, lo b1} of the lane's B fragment.
// Returns the position of hi; lo is 4 elements further.
__device__ __forceinline__ size_t opnd_off(int k, int b, int nn) {
  const int kk = k & 15;
  return ((size_t)(k >> 4) * nn + (b >> 3)) * 256 + ((b & 7) * 4 + ((kk & 7) >> 1)) * 8 +
         (kk >> 3) * 2 + (kk & 1);
}

__device__ __forceinline__ void put_opnd(uint16_t *buf, int k, int b, int nn, float x) {
  const size_t o = opnd_off(k, b, nn);
  const uint16_t hi = f2bf(x);
  buf[o] = hi;
  buf[o + 4] = f2bf(x - bf2f(hi));
}

// JIT attention (MPK review, "Direction 4": the data-dependent operator is
// resolved at run time).  The pairs p = b * Hkv + g, each with n_b = L_b + 1
// positions (its cached rows and the new one), lie end to end on one line of
// T positions; task a takes positions [a C, (a + 1) C) of it, so the tasks of
// a layer carry equal work whatever the KV lengths, and a task may cover the
// end of one pair and the start of the next.  C = the larger of ceil(T / A)
// and ceil(max n_b / (S - 1)), rounded up to 16: at most S tasks touch a pair
// (S = the partial slots per pair).  Every task and its producer derive the
// same pieces from kv_len, which no task of the step changes before ARGMAX.
struct JitPart {
  int C, T;
  const int *n;  // positions of each sequence's pairs (kv_len + 1), in shared memory
};

// Reads kv_len once (independent loads) into `lens` (kMaxBatch ints of
// shared memory owned by the calling thread) and derives C and T.
__device__ __forceinline__ JitPart jit_part(const Params &p, int *lens) {
  int T = 0, nmax = 0;
  for (int b = 0; b < p.B; ++b) lens[b] = __ldcg(p.kv_len + b) + 1;
  for (int b = 0; b < p.B; ++b) {
    T += lens[b] * p.Hkv;
    nmax = max(nmax, lens[b]);
  }
  int C = (T + p.n_attn - 1) / p.n_attn;
  C = max(C, (nmax + p.S - 2) / (p.S - 1));
  return JitPart{(C + 15) & ~15, T, lens};
}

// One piece of an attention task: cached rows [c0, c1) of pair (b, g)
// streamed in stages at origin o (stage st covers [o + st pps, o + (st + 1)
// pps), clipped to [c0, c1)), the new row (position L) if has_new; the
// piece's result is partial slot `slot` of the `expect` tasks that complete
// the pair (expect == 1: written straight to att), and the last of them
// merges `nmerge` partials.
struct AttnSeg {
  int b, g, L;
  int c0, c1, o;
  bool has_new;
  int slot, expect, nmerge;
};

__device__ __forceinline__ int seg_stages(const Params &p, const AttnSeg &s) {
  return s.c1 > s.c0 ? (s.c1 - 1 - s.o) / p.pps + 1 : 0;
}

// The pieces of JIT task a, in line order (no memory reads: the lengths
// come with the partition).
struct JitCursor {
  int a, C, x, x1, b, g, r, n;
  const int *len;
  __device__ __forceinline__ void start(const Params &p, int task, const JitPart &jp) {
    len = jp.n;
    a = task;
    C = jp.C;
    x = min(a * C, jp.T);
    x1 = min(x + C, jp.T);
    int rest = x;
    b = 0;
    g = 0;
    r = 0;
    n = 1;
    for (; b < p.B; ++b) {
      n = len[b];
      if (rest < n * p.Hkv) {
        g = rest / n;
        r = rest - g * n;
        break;
      }
      rest -= n * p.Hkv;
    }
  }
  __device__ __forceinline__ bool next(const Params &p, AttnSeg &s) {
    if (x >= x1) return false;
    const int len_here = min(n - r, x1 - x);
    const int pp = x - r;  // line position of the pair's row 0
    s.b = b;
    s.g = g;
    s.L = n - 1;
    s.c0 = r;
    s.c1 = min(r + len_here, s.L);
    s.o = r / p.pps * p.pps;
    s.has_new = r + len_here == n;
    s.slot = a - pp / C;
    s.expect = (pp + n - 1) / C - pp / C + 1;
    s.nmerge = s.expect;
    x += len_here;
    r += len_here;
    if (r == n) {
      r = 0;
      if (++g == p.Hkv) {
        g = 0;
        if (++b < p.B) n = len[b];
      }
    }
    return true;
  }
};

// JIT attention state kept in shared memory rather than registers: the
// producer's lengths, and the compute side's lengths, cursor and current
// piece (thread 0 advances the cursor; every compute thread reads the piece).
struct JitShared {
  int lens_p[kMaxBatch];
  int lens_c[kMaxBatch];
  JitCursor cur;
  AttnSeg seg;
  int more;
};

// ---------------------------------------------------------------------------
// Shared memory layout (identical computation on host: see smem_bytes()).
// ---------------------------------------------------------------------------
enum Ctl { kAbort = 0, kEpoch = 1, kConsumed = 2, kIssued = 3, kLast = 4, kLogits = 5, kWindow = 6,
           kCtlWords = 16 };

struct Smem {
  uint8_t *ring;
  uint64_t *full, *empty;
  volatile int *ctl;
  unsigned long long *tmark;  // [8] trace marks: prologue done, streaming done, ready,
                              // L2 prefetch bytes, first ring stage available
  JitShared *jit;             // JIT attention state
  // GEMV scratch
  float *red;   // [kRedRows][kComputeWarps] warp partial sums of tile rows
  float *ss;    // [kComputeWarps]
  float *lmv;   // [kComputeWarps] partial argmax values (LM head)
  int *lmi;     // [kComputeWarps] partial argmax indices
  // attention scratch
  float *q;     // [kMaxRep][kMaxHeadDim]
  uint16_t *knew, *vnew;  // [kMaxHeadDim] bf16
  float *sc;    // per warp: [32] probabilities, [kMaxRep] rescale factors
  float *mls;   // [3][kMaxRep]
  float *ored;  // per warp and head: [D] output, running max, running sum (merge: weights)
  // tensor-core projection scratch
  float *cred;  // [warp][m-tile of the pass][16 rows][8 nn + 1] accumulator partials
  float *minv;  // [kMaxBatch] 1 / rms of each sequence's input
  float *mlv;   // [16] partial argmax values (LM head)
  int *mli;     // [16] partial argmax indices
};

__host__ __device__ inline size_t align_to(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct SmemOffsets {
  size_t full, empty, ctl, tmark, jit, red, ss, lmv, lmi, q, knew, vnew, sc, mls, ored, cred, minv,
      mlv, mli, total;
};

__host__ __device__ inline SmemOffsets smem_offsets(int stages, int stage_bytes, int pps,
                                                    int head_dim, int rep_p) {
  SmemOffsets o;
  size_t p = (size_t)stages * stage_bytes;
  o.full = p;
  p += 8 * (size_t)stages;
  o.empty = p;
  p += 8 * (size_t)stages;
  o.ctl = p;
  p += 4 * kCtlWords;
  p = align_to(p, 16);
  o.tmark = p;
  p += 64;
  o.jit = p;
  p += align_to(sizeof(JitShared), 16);
  // GEMV scratch
  size_t g = p;
  o.red = g;
  g += 4 * kRedRows * kComputeWarps;
  o.ss = g;
  g += 4 * kComputeWarps;
  o.lmv = g;
  g += 4 * kComputeWarps;
  o.lmi = g;
  g += 4 * kComputeWarps;
  // attention scratch (shares the same bytes: a CTA runs one task at a time)
  size_t a = p;
  o.q = a;
  a += 4 * kMaxRep * kMaxHeadDim;
  o.knew = a;
  a += 2 * kMaxHeadDim;
  o.vnew = a;
  a += 2 * kMaxHeadDim;
  o.sc = a;  // per warp: 32 probabilities + kMaxRep rescale factors
  a += 4 * (size_t)kComputeWarps * (32 + kMaxRep);
  o.mls = a;
  a += 4 * 3 * kMaxRep;
  a = align_to(a, 16);
  o.ored = a;  // per warp and head: o[D], running max, running sum
  a += 4 * (size_t)kStateSlots * rep_p * (head_dim + 2);
  // tensor-core projection scratch (same bytes again)
  size_t m = p;
  o.cred = m;
  m += 4 * (size_t)kMmaCredFloats;
  o.minv = m;
  m += 4 * kMaxBatch;
  o.mlv = m;
  m += 4 * 16;
  o.mli = m;
  m += 4 * 16;
  size_t top = g > a ? g : a;
  top = top > m ? top : m;
  o.total = align_to(top, 128);
  return o;
}

__device__ __forceinline__ Smem carve(uint8_t *base, const Params &p) {
  SmemOffsets o = smem_offsets(p.ring_stages, p.stage_bytes, p.pps, p.D, p.rep_p);
  Smem s;
  s.ring = base;
  s.full = reinterpret_cast<uint64_t *>(base + o.full);
  s.empty = reinterpret_cast<uint64_t *>(base + o.empty);
  s.ctl = reinterpret_cast<volatile int *>(base + o.ctl);
  s.tmark = reinterpret_cast<unsigned long long *>(base + o.tmark);
  s.jit = reinterpret_cast<JitShared *>(base + o.jit);
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
  s.cred = reinterpret_cast<float *>(base + o.cred);
  s.minv = reinterpret_cast<float *>(base + o.minv);
  s.mlv = reinterpret_cast<float *>(base + o.mlv);
  s.mli = reinterpret_cast<int *>(base + o.mli);
  return s;
}

// Trace mark i (0: prologue done, 1: streaming done) of the running task.
__device__ __forceinline__ void trace_mark(const Params &p, const Smem &sm, int i) {
  if (p.trace && threadIdx.x == 0) sm.tmark[i] = global_timer();
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

// A projection task on tensor cores: its m-tiles [mt0, mt1) of the
// fragment-ordered matrix are streamed as row blocks of mb m-tiles, each row
// block as nkc ring stages of (up to) kcb k-blocks.  Every (m-tile, k-block)
// is one 512-byte fragment block; stage (rb, kc) packs the blocks of its
// m-tiles as [m-tile][k-block].
struct MmaTile {
  const uint16_t *w;  // the operator's matrix, fragment order
  int KB;             // k-blocks per row (K / 16)
  int mt0, mt1;       // m-tiles of this task
  int mb, kcb, nkc, nrb;
};

__device__ __forceinline__ MmaTile mma_tile(const Params &p, int type, int layer, int idx) {
  const Gemv g = gemv_of(p, type, layer, idx);
  MmaTile m;
  m.w = g.w;
  m.KB = g.K >> 4;
  m.mt0 = g.row0 >> 4;
  m.mt1 = (g.row1 + 15) >> 4;  // the LM head's last m-tile may hold zero padding rows
  switch (type) {
    case 2: m.mb = p.mb_qkv; m.kcb = p.kcb_qkv; break;
    case 5: m.mb = p.mb_o; m.kcb = p.kcb_o; break;
    case 6: m.mb = p.mb_gu; m.kcb = p.kcb_gu; break;
    case 7: m.mb = p.mb_down; m.kcb = p.kcb_down; break;
    default: m.mb = p.mb_lm; m.kcb = p.kcb_lm; break;
  }
  m.nkc = (m.KB + m.kcb - 1) / m.kcb;
  m.nrb = (m.mt1 - m.mt0 + m.mb - 1) / m.mb;
  return m;
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
  a.L = __ldcg(p.kv_len + a.b);  // updated by every step's ARGMAX: read through L2
  a.p0 = a.s * p.chunk;
  int end = a.p0 + p.chunk;
  a.cached_end = min(end, a.L);
  a.has_new = a.L >= a.p0 && a.L < end;
  a.active = a.p0 <= a.L;
  return a;
}

// Element offset of cache row `row` of (layer, sequence b, kv head g): the
// contiguous layout, or row % P of the sequence's page of the paged pools.
__device__ __forceinline__ size_t kv_row(const Params &p, int layer, int b, int g, int row) {
  if (p.page_size > 0) {
    const int page = __ldg(p.page_table + (size_t)b * p.max_pages + row / p.page_size);
    return ((((size_t)page * p.Ly + layer) * p.Hkv + g) * p.page_size + row % p.page_size) * p.D;
  }
  return ((((size_t)layer * p.B + b) * p.Hkv + g) * p.Lcap + row) * p.D;
}

// Everything the producer needs to stream one task, computed once per task so
// that issuing a stage is pure address arithmetic (no dependent loads).
struct Stream {
  const uint8_t *src0 = nullptr;  // stage 0 source (weights)
  uint32_t bytes = 0, last_bytes = 0;  // bytes of a full / of the last stage
  uint32_t stride = 0;            // bytes between consecutive stages
  int nst = 0;                    // stages
  // tensor-core projections: stage st = (row block st / nkc, k chunk st % nkc)
  int nkc = 0;                    // 0 for the other streams
  int KB = 0, mt0 = 0, mt1 = 0, mb = 0, kcb = 0;
  // attention: K/V rows y0 + st * pps .. of the 2-D cache tensor maps (paged
  // pools: stage st starts at position kv_p0 + st * pps of (layer, b, g);
  // a stage never crosses a page)
  int kv = 0;
  int y0 = 0;
  int kv_l = 0, kv_b = 0, kv_g = 0, kv_p0 = 0;
  // JIT attention: the pieces of task ja (see JitCursor), stages in piece order
  int jit = 0, ja = 0;
  JitPart jp{0, 0, nullptr};
};

// First cache row (in rows of D elements) of K/V stage st of stream s.
template <bool kExt>
__device__ __forceinline__ int kv_stage_row(const Params &p, const Stream &s, int st) {
  if (kExt && s.jit) {  // the piece holding stage st; the stage starts at its first row
    JitCursor cur;
    cur.start(p, s.ja, s.jp);
    AttnSeg sg;
    while (cur.next(p, sg)) {
      const int n = seg_stages(p, sg);
      if (st < n)
        return (int)(kv_row(p, s.kv_l, sg.b, sg.g, max(sg.c0, sg.o + st * p.pps)) / p.D);
      st -= n;
    }
    return 0;  // not reached: st < the task's stage count
  }
  if (p.page_size > 0) return (int)(kv_row(p, s.kv_l, s.kv_b, s.kv_g, s.kv_p0 + st * p.pps) / p.D);
  return s.y0 + st * p.pps;
}

// kMma: the batched kernel (tensor-core tiles, swizzled TMA K/V boxes);
// kExt: the extended kernels (JIT attention, dispatch mode).
template <bool kMma, bool kExt>
__device__ __forceinline__ Stream task_stream(const Params &p, const DevTask &t, int *jit_lens) {
  Stream s{};
  const int type = t.type;
  if (kMma && (type == 2 || (type >= 5 && type <= 8))) {
    const MmaTile m = mma_tile(p, type, t.layer, (int)t.idx);
    s.src0 = reinterpret_cast<const uint8_t *>(m.w);
    s.nst = m.nrb * m.nkc;
    s.nkc = m.nkc;
    s.KB = m.KB;
    s.mt0 = m.mt0;
    s.mt1 = m.mt1;
    s.mb = m.mb;
    s.kcb = m.kcb;
    return s;
  }

  if (kMma && kExt && type == 3 && p.jit) {
    // whole boxes of pps rows from each stage's first row (masked past its end)
    s.jp = jit_part(p, jit_lens);
    s.ja = (int)t.idx;
    s.jit = 1;
    s.kv = 1;
    s.kv_l = t.layer;
    JitCursor cur;
    cur.start(p, s.ja, s.jp);
    AttnSeg sg;
    while (cur.next(p, sg)) s.nst += seg_stages(p, sg);
    s.bytes = s.last_bytes = (uint32_t)(p.pps * p.D * 2);
    return s;
  }
  if (type == 3) {
    // whole boxes of pps rows (the last stage reads past the split: masked)
    const AttnSpan a = attn_span(p, (int)t.idx);
    const int n = a.cached_end - a.p0;
    if (n <= 0) return s;
    s.nst = (n + p.pps - 1) / p.pps;
    s.kv = 1;
    s.kv_l = t.layer;
    s.kv_b = a.b;
    s.kv_g = a.g;
    s.kv_p0 = a.p0;
    s.y0 = (int)(kv_row(p, t.layer, a.b, a.g, a.p0) / p.D);
    s.bytes = s.last_bytes = (uint32_t)(p.pps * p.D * 2);
    // batch 1: plain row copies of exactly the cached rows
    if (!kMma) s.last_bytes = (uint32_t)((n - (s.nst - 1) * p.pps) * p.D * 2);
  } else if (type == 2 || (type >= 5 && type <= 8)) {
    const Gemv g = gemv_of(p, type, t.layer, (int)t.idx);
    const int rows = g.row1 - g.row0;
    s.nst = (rows + g.rps - 1) / g.rps;
    s.src0 = reinterpret_cast<const uint8_t *>(g.w + (size_t)g.row0 * g.K);
    s.stride = s.bytes = (uint32_t)((size_t)g.rps * g.K * 2);
    s.last_bytes = (uint32_t)((size_t)(rows - (s.nst - 1) * g.rps) * g.K * 2);
  }
  return s;
}

// Bytes that stage st of stream s lands in the ring.
template <bool kMma>
__device__ __forceinline__ uint32_t stage_bytes_of(const Stream &s, int st) {
  if (kMma && s.nkc > 0) {
    const int rb = st / s.nkc, kc = st - rb * s.nkc;
    const int nm = min(s.mb, s.mt1 - (s.mt0 + rb * s.mb));
    const int nkb = min(s.kcb, s.KB - kc * s.kcb);
    return (uint32_t)(nm * nkb * 512);
  }
  if (s.kv) return 2 * (st == s.nst - 1 ? s.last_bytes : s.bytes);  // K and V
  return st == s.nst - 1 ? s.last_bytes : s.bytes;
}

// Issue the copies of stage st of stream s into ring slot dst (the full
// barrier already expects stage_bytes_of(s, st) bytes).
template <bool kMma, bool kExt>
__device__ __forceinline__ void issue_stage(const Params &p, const Stream &s, int st, uint8_t *dst,
                                            uint64_t *bar, uint64_t pol) {
  if (s.kv) {
    const int y = kv_stage_row<kExt>(p, s, st);
    if (!kMma) {  // plain rows: K at dst, V pps rows further
      const uint32_t nb = st == s.nst - 1 ? s.last_bytes : s.bytes;
      bulk_g2s(dst, p.k_cache + (size_t)y * p.D, nb, bar, pol);
      bulk_g2s(dst + s.bytes, p.v_cache + (size_t)y * p.D, nb, bar, pol);
      return;
    }
    // K boxes (64 dims x pps rows, 128-byte swizzle) at dst, V boxes after them
    const uint32_t box = (uint32_t)p.pps * 128u;
    for (int h = 0; h < (p.D >> 6); ++h) {
      tma_load_2d(dst + h * box, &p.tmap_k, 64 * h, y, bar, pol);
      tma_load_2d(dst + s.bytes + h * box, &p.tmap_v, 64 * h, y, bar, pol);
    }
    return;
  }
  if (kMma && s.nkc > 0) {
    const int rb = st / s.nkc, kc = st - rb * s.nkc;
    const int m0 = s.mt0 + rb * s.mb, nm = min(s.mb, s.mt1 - m0);
    const int kb0 = kc * s.kcb, nkb = min(s.kcb, s.KB - kb0);
    const uint32_t cb = (uint32_t)nkb * 512u;
    for (int i = 0; i < nm; ++i)
      bulk_g2s(dst + (size_t)i * cb, s.src0 + ((size_t)(m0 + i) * s.KB + kb0) * 512, cb, bar,
               pol);
    return;
  }
  const uint32_t nb = st == s.nst - 1 ? s.last_bytes : s.bytes;
  bulk_g2s(dst, s.src0 + (size_t)st * s.stride, nb, bar, pol);
}

// Prefetch stage st of stream s into L2; returns the bytes requested.
template <bool kMma>
__device__ __forceinline__ uint32_t prefetch_stage(const Stream &s, int st) {
  if (kMma && s.nkc > 0) {
    const int rb = st / s.nkc, kc = st - rb * s.nkc;
    const int m0 = s.mt0 + rb * s.mb, nm = min(s.mb, s.mt1 - m0);
    const int kb0 = kc * s.kcb, nkb = min(s.kcb, s.KB - kb0);
    const uint32_t cb = (uint32_t)nkb * 512u;
    for (int i = 0; i < nm; ++i) prefetch_l2(s.src0 + ((size_t)(m0 + i) * s.KB + kb0) * 512, cb);
    return cb * (uint32_t)nm;
  }
  if (s.kv) return 0u;  // K/V tiles are not prefetched
  const uint32_t pb = st == s.nst - 1 ? s.last_bytes : s.bytes;
  prefetch_l2(s.src0 + (size_t)st * s.stride, pb);
  return pb;
}

// ---------------------------------------------------------------------------
// Producer: one thread streams every stage of the worker's queue.
// ---------------------------------------------------------------------------
struct Queue {
  int first, stride, count;  // tasks first, first + stride, ... (count of them)
  // dispatch mode: the entries the scheduler publishes for this worker
  const int32_t *list = nullptr;
  const uint32_t *tail = nullptr;
};

// Task id of entry n of the worker's queue, or -1 past its end (static
// queues) / at the scheduler's end mark.  In dispatch mode the entry is
// waited for (bounded); -1 also when the CTA aborts or the wait runs out.
template <bool kExt>
__device__ __forceinline__ int queue_task(const Params &p, const Smem &sm, const Queue &q, int n) {
  if (!kExt || !q.list) return n < q.count ? q.first + n * q.stride : -1;
  if ((int32_t)(ld_acquire(q.tail) - (uint32_t)n) <= 0) {
    const uint64_t t0 = global_timer();
    uint32_t spins = 0;
    while ((int32_t)(ld_acquire(q.tail) - (uint32_t)n) <= 0) {
      if (sm.ctl[kAbort]) return -1;
      if (++spins > 16) __nanosleep(64);
      if ((spins & 63u) == 0 && global_timer() - t0 > 4ull * p.timeout_ns + 1000000000ull) {
        record_error(p, kDevTimeout, -1, -3);
        sm.ctl[kAbort] = 1;
        return -1;
      }
    }
  }
  return __ldcg(q.list + n);
}

template <bool kMma, bool kExt>
__device__ void producer_loop(const Params &p, const Smem &sm, const Queue &q) {
  const int NS = p.ring_stages;
  uint32_t k = 0;
  const uint64_t budget = 4ull * p.timeout_ns + 1000000000ull;
  // L2 prefetch cursor (task pf_n, stage pf_st, global stage index pf_k) in
  // the worker's stream of stages, across task boundaries.  While the ring is
  // full and the compute warps wait for an O projection's event
  // (sm.ctl[kWindow]), the step is in its attention window: attention moves
  // little data and no operator streams weights, so every SM has spare HBM
  // bandwidth.  The producer then prefetches its next stages into L2, one per
  // poll of the ring, up to l2_prefetch_bytes ahead of it.  (Prefetching
  // whenever the ring stalls takes bandwidth from SMs still streaming the
  // current operator; a burst from every SM while attention runs slows the
  // attention tasks on the critical path.  Qwen3-8B at batch 1, one box:
  // 3079 us per step with this window, 3130 us with the stall-gated rule,
  // 3141 us with back-to-back prefetches during attention.)
  // (dispatch mode: the queue holds only tasks that are ready, no lookahead)
  const long long dist = q.list ? 0 : p.l2_prefetch_bytes;
  const uint64_t pol = stream_policy(p.evict_first != 0);
  int pf_n = 0, pf_st = 0;
  Stream pfs{};
  pfs.nst = -1;
  uint32_t pf_k = 0;
  long long ahead = 0;
  const uint32_t epoch0 = (uint32_t)sm.ctl[kEpoch];
  int *jl = sm.jit->lens_p;
  for (int s = 0; s < p.n_steps; ++s) {
  // K/V rows of step s > 0 include the rows step s - 1 appended (possibly on
  // another SM), and the stream's extent depends on kv_len: the first K/V
  // stream of a step waits until the previous step has completed.  Weight
  // streams are never gated, so they run ahead across the step boundary.
  bool kv_open = s == 0;
  // the prefetch cursor walks this step's queue from its first task
  pf_n = 0;
  pf_st = 0;
  pfs.nst = -1;
  pf_k = k;
  ahead = 0;
  for (int n = 0; n < q.count; ++n) {
    const int tid_n = queue_task<kExt>(p, sm, q, n);
    if (tid_n < 0) break;
    const DevTask tk = p.tasks[tid_n];
    if (tk.type == 3 && !kv_open) {
      const uint64_t t0 = global_timer();
      uint32_t spins = 0;
      while ((int32_t)(ld_acquire(p.epoch) - (epoch0 + (uint32_t)s - 1u)) < 0) {
        if (sm.ctl[kAbort]) goto out;
        if ((++spins & 63u) == 0 && global_timer() - t0 > budget) {
          record_error(p, kDevTimeout, tid_n, -1);
          goto out;
        }
      }
      fence_proxy_async_global();  // the appended rows are read by bulk / tensor copies
      kv_open = true;
    }
    const Stream ts = task_stream<kMma, kExt>(p, tk, jl);
    for (int st = 0; st < ts.nst; ++st) {
      const uint32_t nb = stage_bytes_of<kMma>(ts, st);
      if (dist > 0) {
        // stages before k were issued without a prefetch: move the cursor on
        while (pf_k < k && pf_n < q.count) {
          if (pfs.nst < 0) pfs = task_stream<kMma, kExt>(p, p.tasks[q.first + pf_n * q.stride], jl);
          if (pf_st >= pfs.nst) {
            ++pf_n;
            pf_st = 0;
            pfs.nst = -1;
            continue;
          }
          ++pf_st;
          ++pf_k;
        }
        if (pf_k <= k) ahead = 0;
      }
      const int slot = (int)(k % NS);
      const uint32_t use = k / NS;
      if (use > 0) {
        const uint32_t par = (use - 1) & 1u;
        uint64_t t0 = 0;
        uint32_t spins = 0;
        while (!mbar_test(&sm.empty[slot], par)) {
          if (sm.ctl[kAbort]) goto out;
          ++spins;
          if (dist > 0 && ahead < dist && pf_n < q.count && sm.ctl[kWindow]) {
            if (pfs.nst < 0) pfs = task_stream<kMma, kExt>(p, p.tasks[q.first + pf_n * q.stride], jl);
            if (pf_st >= pfs.nst) {
              ++pf_n;
              pf_st = 0;
              pfs.nst = -1;
            } else {
              const uint32_t pb = prefetch_stage<kMma>(pfs, pf_st);
              ahead += pb;
              if (p.trace) sm.tmark[3] += pb;
              ++pf_st;
              ++pf_k;
            }
          }
          if ((spins & 255u) == 0) {
            uint64_t now = global_timer();
            if (t0 == 0) t0 = now;
            else if (now - t0 > budget) {
              record_error(p, kDevTimeout, tid_n, -1);
              goto out;
            }
          }
        }
      }
      uint8_t *dst = sm.ring + (size_t)slot * p.stage_bytes;
      mbar_arrive_expect_tx(&sm.full[slot], nb);
      issue_stage<kMma, kExt>(p, ts, st, dst, &sm.full[slot], pol);
      if (dist > 0 && pf_k > k) ahead -= nb;  // stage k was prefetched
      ++k;
    }
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

// Trace mark 4: the running task's first ring stage is available.
__device__ __forceinline__ void trace_first_stage(const Params &p, const Smem &sm, int st) {
  if (p.trace && st == 0 && threadIdx.x == 0) sm.tmark[4] = global_timer();
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

// Thread 0: wait (bounded) until the device step epoch reached `target`.
__device__ bool wait_epoch(const Params &p, uint32_t target, int task) {
  const uint64_t t0 = global_timer();
  uint32_t spins = 0;
  while ((int32_t)(ld_acquire(p.epoch) - target) < 0) {
    if (++spins > 64) __nanosleep(32);
    if ((spins & 63u) == 0 && global_timer() - t0 > p.timeout_ns) {
      record_error(p, kDevTimeout, task, -1);
      return false;
    }
  }
  return true;
}

// The wait for a task's dependency event.  Task bodies first issue the loads
// that do not depend on this step's results (gains, RoPE factors), then call
// this; every compute thread calls it exactly once per task.
struct DepWait {
  const Params &p;
  const Smem &sm;
  int dep;
  uint32_t epoch;
  int task;
  int type;
  __device__ __forceinline__ bool operator()() const {
    // (dispatch mode: the scheduler hands out a task once its event fired)
    if (p.persistent && !p.dispatch && dep >= 0 && threadIdx.x == 0) {
      // the wait of an O projection is the step's attention window (see producer_loop)
      sm.ctl[kWindow] = type == 5;
      if (!wait_event(p, dep, epoch, task)) sm.ctl[kAbort] = 1;
      sm.ctl[kWindow] = 0;
    }
    compute_sync();
    if (p.trace && threadIdx.x == 0) sm.tmark[2] = global_timer();
    return !sm.ctl[kAbort];
  }
};

// ---------------------------------------------------------------------------
// GEMV task body (batch 1): prologue RMSNorm, weight stream, fused epilogue.
// ---------------------------------------------------------------------------
// Epilogue of `n` finished tile rows whose warp partials sit in sm.red, the
// first of them at arena row `row0`.  Runs on all compute threads.
__device__ __forceinline__ void gemv_finish(const Params &p, const Smem &sm, int type,
                                            const DevLayer *L, int row0, int n, int wpg,
                                            float res, float &best_v, int &best_i) {
  const int tid = threadIdx.x;
  if (type == 6) {  // rows (2i, 2i+1) = (gate_i, up_i): h_i = silu(g) * u
    for (int f = tid; f < n / 2; f += kComputeThreads) {
      float gv = 0.f, uv = 0.f;
      for (int w = 0; w < wpg; ++w) {
        gv += sm.red[(2 * f) * kComputeWarps + w];
        uv += sm.red[(2 * f + 1) * kComputeWarps + w];
      }
      L->h[(row0 >> 1) + f] = gv / (1.f + __expf(-gv)) * uv;
    }
    return;
  }
  for (int f = tid; f < n; f += kComputeThreads) {
    float v = 0.f;
    for (int w = 0; w < wpg; ++w) v += sm.red[f * kComputeWarps + w];
    const int r = row0 + f;
    if (type == 2) {
      L->qkv[r] = v;
    } else if (type == 5) {
      L->xm[r] = (f == tid ? res : __ldcg(L->x_in + r)) + v;
    } else if (type == 7) {
      L->x_out[r] = (f == tid ? res : __ldcg(L->xm + r)) + v;
    } else {
      if (p.logits && sm.ctl[kLogits]) p.logits[r] = v;
      if (v > best_v || (v == best_v && r < best_i)) {
        best_v = v;
        best_i = r;
      }
    }
  }
}

// GEMV task (batch 1).  Prologue: the input vector in registers, RMSNorm
// applied when the operator has one.  Main loop: every warp walks the ring
// stages on its own (wait full, accumulate, release its share), writing warp
// partial sums of each row to shared memory; no CTA barrier per stage.  The
// epilogue runs once per task (or per kRedRows rows) on all threads.
template <int CPT, int NR>
__device__ __forceinline__ bool gemv_task(const Params &p, const Smem &sm, const DevTask &t,
                                          uint32_t &k, int task_id, const DepWait &dep_wait) {
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

  // norm gains of this thread's chunks: weights, so loaded before the wait
  uint4 gw[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int c = li + j * tpg;
    gw[j] = (gain && active && c < nch) ? __ldg(reinterpret_cast<const uint4 *>(gain + 8 * c))
                                        : make_uint4(0u, 0u, 0u, 0u);
  }
  if (!dep_wait()) return false;
  // activation chunks of this thread
  float x[CPT][8];
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int c = li + j * tpg;
    if (active && c < nch) {
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
    for (int j = 0; j < CPT; ++j)
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
    for (int j = 0; j < CPT; ++j) {
      const int c = li + j * tpg;
      if (active && c < nch) {
        x[j][0] *= inv * bf_lo(gw[j].x); x[j][1] *= inv * bf_hi(gw[j].x);
        x[j][2] *= inv * bf_lo(gw[j].y); x[j][3] *= inv * bf_hi(gw[j].y);
        x[j][4] *= inv * bf_lo(gw[j].z); x[j][5] *= inv * bf_hi(gw[j].z);
        x[j][6] *= inv * bf_lo(gw[j].w); x[j][7] *= inv * bf_hi(gw[j].w);
      }
    }
  }

  const int rows = g.row1 - g.row0;
  const int nst = (rows + g.rps - 1) / g.rps;
  const int row16 = K >> 3;  // 16-byte chunks per row
  // residual of the row this thread finishes, loaded now to hide its latency
  float res = 0.f;
  if (tid < rows && (type == 5 || type == 7))
    res = __ldcg((type == 5 ? L->x_in : L->xm) + g.row0 + tid);
  float best_v = -INFINITY;
  int best_i = 0x7fffffff;
  int buf0 = 0;  // first tile row whose partials sm.red holds
  trace_mark(p, sm, 0);
  for (int st = 0; st < nst; ++st) {
    const int r0 = st * g.rps;
    const int r_here = min(g.rps, rows - r0);
    if (r0 + r_here - buf0 > kRedRows) {  // shared partials full: finish them
      compute_sync();
      if (!sm.ctl[kAbort]) gemv_finish(p, sm, type, L, g.row0 + buf0, r0 - buf0, wpg, res, best_v, best_i);
      compute_sync();
      buf0 = r0;
    }
    const bool got = sm.ctl[kAbort] ? false : wait_full(p, sm, k, task_id);
    if (got) {
      trace_first_stage(p, sm, st);
      const uint16_t *ws =
          reinterpret_cast<const uint16_t *>(sm.ring + (size_t)(k % p.ring_stages) * p.stage_bytes);
      if (active) {
        // NR rows at a time: NR independent (even, odd) accumulator pairs per
        // thread fed by packed FMAs, then one transposed warp reduction
        for (int rb = grp * NR; rb < r_here; rb += ngroups * NR) {
          const int nr = min(NR, r_here - rb);
          const uint4 *wr = reinterpret_cast<const uint4 *>(ws + (size_t)rb * K);
          // few rows per batch: spread the chunks over AS accumulator sets so
          // every thread still has >= 8 independent FMA chains
          constexpr int AS = NR >= 4 ? 1 : (CPT >= 3 ? 3 : CPT);
          float acc[NR][AS][2];
#pragma unroll
          for (int i = 0; i < NR; ++i)
#pragma unroll
            for (int a = 0; a < AS; ++a) acc[i][a][0] = acc[i][a][1] = 0.f;
          // a partial last batch still reads NR rows: rb + NR <= rps keeps them
          // inside the slot, and rows >= nr (stale data) are never stored
#pragma unroll
          for (int j = 0; j < CPT; ++j) {
            const int c = li + j * tpg;
            if (c < nch) {
              uint4 w[NR];
#pragma unroll
              for (int i = 0; i < NR; ++i) w[i] = wr[i * row16 + c];
#pragma unroll
              for (int i = 0; i < NR; ++i) dot8_acc(w[i], x[j], acc[i][j % AS]);
            }
          }
          float v8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float v = 0.f;
            if (i < NR) {
#pragma unroll
              for (int a = 0; a < AS; ++a) v += acc[i][a][0] + acc[i][a][1];
            }
            v8[i] = v;
          }
          const float v = warp_sum8(v8, lane);
          if ((lane & 3) == 0 && (lane >> 2) < nr)
            sm.red[(r0 - buf0 + rb + (lane >> 2)) * kComputeWarps + wig] = v;
        }
      }
      release_stage(sm, p, k);
      ++k;
    }
  }
  trace_mark(p, sm, 1);
  compute_sync();
  if (sm.ctl[kAbort]) return false;
  gemv_finish(p, sm, type, L, g.row0 + buf0, rows - buf0, wpg, res, best_v, best_i);
  if (type == 8) {
    // (max, lowest index) over the threads: warp shuffles, then warp 0
    float bv = best_v;
    int bi = best_i;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) {
      sm.lmv[warp] = bv;
      sm.lmi[warp] = bi;
    }
    compute_sync();
    if (warp == 0) {
      bv = lane < kComputeWarps ? sm.lmv[lane] : -INFINITY;
      bi = lane < kComputeWarps ? sm.lmi[lane] : 0x7fffffff;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
      if (lane == 0) {
        if (bi == 0x7fffffff) bi = g.row0;  // all values NaN: keep a valid index
        p.lm_val[(int)t.idx] = bv;
        p.lm_idx[(int)t.idx] = bi;
      }
    }
  }
  return true;
}

// ---------------------------------------------------------------------------
// Projection task on tensor cores (batch >= 2).
// ---------------------------------------------------------------------------
// B fragments of k-blocks kb0 + warp + 8 j (j < kpw) of the operand xb: the
// activations are written earlier in this step by other SMs, so they are read
// through L2 (never from a possibly stale L1 line).
template <int NN>
__device__ __forceinline__ void load_bfrag(uint4 (&bf)[mma_max_kpw(NN)][NN], const uint16_t *xb,
                                           int kb0, int kpw, int warp, int lane) {
#pragma unroll
  for (int j = 0; j < mma_max_kpw(NN); ++j) {
    if (j < kpw) {
#pragma unroll
      for (int n = 0; n < NN; ++n)
        bf[j][n] = __ldcg(reinterpret_cast<const uint4 *>(
                              xb + ((size_t)(kb0 + warp + 8 * j) * NN + n) * 256) + lane);
    }
  }
}

// One ring stage of a projection with compile-time tile counts (MBF m-tiles,
// KPWF k-blocks per warp): the common cases, with no per-tile guards, so the
// A fragments of a k-block are loaded before its MMAs.  The B fragments of
// the next stage's first kpw_n k-blocks are refilled after their last use.
template <int NN, int MBF, int KPWF, bool kGuard>
__device__ __forceinline__ void mma_stage_fixed(float (&acc)[kMmaMaxMB][NN][4],
                                                uint4 (&bc)[mma_max_kpw(NN)][NN], const uint8_t *slot,
                                                const uint16_t *xn, int kpw_n, int warp, int lane) {
  constexpr int NKB = 8 * KPWF;
#pragma unroll
  for (int j = 0; j < KPWF; ++j) {
    const uint8_t *blk = slot + (size_t)(warp + 8 * j) * 512 + lane * 16;
    uint4 a[MBF];
#pragma unroll
    for (int m = 0; m < MBF; ++m) a[m] = *reinterpret_cast<const uint4 *>(blk + m * NKB * 512);
#pragma unroll
    for (int m = 0; m < MBF; ++m)
#pragma unroll
      for (int n = 0; n < NN; ++n) {
        mma_bf16(acc[m][n], a[m], make_uint2(bc[j][n].x, bc[j][n].y));  // W hi
        mma_bf16(acc[m][n], a[m], make_uint2(bc[j][n].z, bc[j][n].w));  // W lo
      }
    if (!kGuard || j < kpw_n) {
#pragma unroll
      for (int n = 0; n < NN; ++n)
        bc[j][n] = __ldcg(reinterpret_cast<const uint4 *>(xn + ((size_t)(8 * j) * NN + n) * 256) + lane);
    }
  }
  // a next stage with more k-blocks (the first chunk after a short last one)
#pragma unroll
  for (int j = KPWF; j < (kGuard ? mma_max_kpw(NN) : 0); ++j) {
    if (j < kpw_n) {
#pragma unroll
      for (int n = 0; n < NN; ++n)
        bc[j][n] = __ldcg(reinterpret_cast<const uint4 *>(xn + ((size_t)(8 * j) * NN + n) * 256) + lane);
    }
  }
}

// Sum over the 16 lanes of a half warp (lanes that share a sequence column).
__device__ __forceinline__ float half_warp_sum(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The batched projection y[b][r] = sum_k W[r][k] x̂[b][k] of one task on
// mma.sync.  The input arrives as a hi/lo bf16 operand of x[b][k] * gain[k]
// written by the producing task's epilogue, with per-16-row sums of squares;
// the RMSNorm's per-sequence factor 1 / rms(x_b) is applied to the fp32
// accumulators in the epilogue (it factors out of the sum over k).
//
// Work split: for each ring stage (row block x k chunk) warp w takes the
// k-blocks w, w + 8, ... of the chunk for every m-tile of the row block, so
// every B fragment is loaded by one warp, once per row block.  The warps'
// partial sums of a row block are added in shared memory in a fixed order
// (deterministic), PM m-tiles per pass, and the fused epilogue of the
// operator runs on the sums: thread (row = tid % 16, sequence = tid / 16 % 8nn).
template <int NN>
__device__ __forceinline__ bool mma_task(const Params &p, const Smem &sm, const DevTask &t,
                                         uint32_t &k, int task_id, const DepWait &dep_wait) {
  constexpr int NC = 8 * NN;          // operand columns (sequences, zero padded)
  constexpr int PM = NN == 2 ? 2 : 4; // m-tiles per reduction pass
  constexpr int CS = NC + 1;          // row stride of the reduction buffer (floats)
  static_assert(kComputeWarps * PM * 16 * CS <= kMmaCredFloats, "reduction buffer");
  const int type = t.type;
  const int layer = t.layer;
  const DevLayer *L = layer < p.Ly ? p.layers + layer : nullptr;
  const MmaTile mt = mma_tile(p, type, layer, (int)t.idx);
  const uint16_t *xb;
  const float *ssp = nullptr;
  switch (type) {
    case 2: xb = L->xa; ssp = L->ssa; break;
    case 5: xb = L->attb; break;
    case 6: xb = L->xmb; ssp = L->ssm; break;
    case 7: xb = L->hb; break;
    default: xb = p.xfb; ssp = p.ssf; break;
  }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = tid & 15;          // row of an m-tile this thread finishes
  const int col = (tid >> 4) % NC;   // sequence this thread finishes
  const bool col_ok = col < p.B;
  const int N = type == 2 ? p.n_qkv : type == 6 ? 2 * p.F : type == 8 ? p.V : p.H;

  if (!dep_wait()) return false;
  uint4 bc[mma_max_kpw(NN)][NN];
  load_bfrag<NN>(bc, xb, 0, min(mt.kcb, mt.KB) >> 3, warp, lane);
  float inv = 1.f;
  if (ssp) {
    for (int b = warp; b < p.B; b += kComputeWarps) {
      float s = 0.f;
      for (int j = lane; j < p.n_parts; j += 32) s += __ldcg(ssp + (size_t)b * p.n_parts + j);
      s = warp_sum(s);
      if (lane == 0) sm.minv[b] = rsqrtf(s / (float)p.H + p.eps);
    }
    compute_sync();
    inv = col_ok ? sm.minv[col] : 0.f;
  }

  float acc[kMmaMaxMB][NN][4];
#pragma unroll
  for (int m = 0; m < kMmaMaxMB; ++m)
#pragma unroll
    for (int n = 0; n < NN; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[m][n][i] = 0.f;
  float best_v = -INFINITY;
  int best_i = 0x7fffffff;
  trace_mark(p, sm, 0);
  const int nst = mt.nrb * mt.nkc;
  for (int st = 0; st < nst; ++st) {
    const int rb = st / mt.nkc, kc = st - rb * mt.nkc;
    const int m0 = mt.mt0 + rb * mt.mb, nm = min(mt.mb, mt.mt1 - m0);
    const int nkb = min(mt.kcb, mt.KB - kc * mt.kcb), kpw = nkb >> 3;
    // the next stage's k chunk (the same chunks repeat for every row block):
    // each B fragment register is refilled for it right after its last use
    const int kn = kc + 1 == mt.nkc ? 0 : kc + 1;
    const int kpw_n = st + 1 < nst ? min(mt.kcb, mt.KB - kn * mt.kcb) >> 3 : 0;
    const uint16_t *xn = xb + ((size_t)(kn * mt.kcb + warp) * NN) * 256;
    const bool got = sm.ctl[kAbort] ? false : wait_full(p, sm, k, task_id);
    if (got) {
      trace_first_stage(p, sm, st);
      const uint8_t *slot = sm.ring + (size_t)(k % p.ring_stages) * p.stage_bytes;
      const bool same = kpw_n == kpw;  // the next stage refills every fragment
      if (NN == 1 && same && kpw == 6 && nm == 2) {
        mma_stage_fixed<NN, 2, (NN == 1 ? 6 : 3), false>(acc, bc, slot, xn, kpw_n, warp, lane);
      } else if (NN == 1 && same && kpw == 4 && nm == 3) {
        mma_stage_fixed<NN, 3, (NN == 1 ? 4 : 3), false>(acc, bc, slot, xn, kpw_n, warp, lane);
      } else if (NN == 1 && kpw == 6 && nm == 2) {
        mma_stage_fixed<NN, 2, (NN == 1 ? 6 : 3), true>(acc, bc, slot, xn, kpw_n, warp, lane);
      } else if (NN == 1 && kpw == 4 && nm == 3) {
        mma_stage_fixed<NN, 3, (NN == 1 ? 4 : 3), true>(acc, bc, slot, xn, kpw_n, warp, lane);
      } else if (same && kpw == 3 && nm == 2) {
        mma_stage_fixed<NN, 2, 3, false>(acc, bc, slot, xn, kpw_n, warp, lane);
      } else if (same && kpw == 3 && nm == 3) {
        mma_stage_fixed<NN, 3, 3, false>(acc, bc, slot, xn, kpw_n, warp, lane);
      } else if (same && kpw == 2 && nm == 6) {
        mma_stage_fixed<NN, 6, 2, false>(acc, bc, slot, xn, kpw_n, warp, lane);
      } else if (kpw == 3 && nm == 2) {
        mma_stage_fixed<NN, 2, 3, true>(acc, bc, slot, xn, kpw_n, warp, lane);
      } else if (kpw == 3 && nm == 3) {
        mma_stage_fixed<NN, 3, 3, true>(acc, bc, slot, xn, kpw_n, warp, lane);
      } else if (kpw == 2 && nm == 2) {
        mma_stage_fixed<NN, 2, 2, true>(acc, bc, slot, xn, kpw_n, warp, lane);
      } else if (kpw == 2 && nm == 3) {
        mma_stage_fixed<NN, 3, 2, true>(acc, bc, slot, xn, kpw_n, warp, lane);
      } else {
#pragma unroll
      for (int j = 0; j < mma_max_kpw(NN); ++j) {
        if (j < kpw) {
          const uint8_t *blk = slot + (size_t)(warp + 8 * j) * 512 + lane * 16;
#pragma unroll
          for (int m = 0; m < kMmaMaxMB; ++m) {
            if (m < nm) {
              const uint4 a = *reinterpret_cast<const uint4 *>(blk + (size_t)m * nkb * 512);
#pragma unroll
              for (int n = 0; n < NN; ++n) {
                mma_bf16(acc[m][n], a, make_uint2(bc[j][n].x, bc[j][n].y));  // W hi
                mma_bf16(acc[m][n], a, make_uint2(bc[j][n].z, bc[j][n].w));  // W lo
              }
            }
          }
        }
        if (j < kpw_n) {
#pragma unroll
          for (int n = 0; n < NN; ++n)
            bc[j][n] = __ldcg(reinterpret_cast<const uint4 *>(
                                  xn + ((size_t)(8 * j) * NN + n) * 256) + lane);
        }
      }
      }
      release_stage(sm, p, k);
      ++k;
    }
    if (kc + 1 < mt.nkc) continue;

    // row block done: cross-warp sums and the fused epilogue, PM m-tiles per pass
#pragma unroll
    for (int q0 = 0; q0 < kMmaMaxMB; q0 += PM) {
      if (q0 >= nm) break;  // uniform over the CTA
      {
        const int g = lane >> 2, tq = lane & 3;
#pragma unroll
        for (int ml = 0; ml < PM; ++ml) {
          const int m = q0 + ml;
          if (m < kMmaMaxMB && m < nm) {
            float *cw = sm.cred + (size_t)(warp * PM + ml) * 16 * CS;
#pragma unroll
            for (int n = 0; n < NN; ++n) {
              const int c = n * 8 + 2 * tq;
              cw[g * CS + c] = acc[m][n][0];
              cw[g * CS + c + 1] = acc[m][n][1];
              cw[(g + 8) * CS + c] = acc[m][n][2];
              cw[(g + 8) * CS + c + 1] = acc[m][n][3];
            }
          }
        }
      }
      compute_sync();
      if (!sm.ctl[kAbort]) {
#pragma unroll
        for (int it = 0; it < PM * NC / 16; ++it) {
          const int ml = (tid + kComputeThreads * it) / (16 * NC);  // uniform per warp
          const bool m_ok = q0 + ml < nm;
          float v = 0.f;
          if (m_ok) {
#pragma unroll
            for (int w = 0; w < kComputeWarps; ++w)
              v += sm.cred[((size_t)(w * PM + ml) * 16 + row) * CS + col];
          }
          const int r = (m0 + q0 + ml) * 16 + row;  // row of the operator's output
          const bool store = m_ok && col_ok && r < N;
          const size_t bH = (size_t)col * p.H;
          if (type == 2) {
            if (store) L->qkv[(size_t)col * p.n_qkv + r] = v * inv;
          } else if (type == 5 || type == 7) {
            // residual add, next operand (gain of the following norm), 16-row ss
            float x = 0.f;
            if (store) {
              x = __ldcg((type == 5 ? L->x_in : L->xm) + bH + r) + v;
              (type == 5 ? L->xm : L->x_out)[bH + r] = x;
              const uint16_t *gn = type == 5 ? L->mlp_norm : L->gain_next;
              put_opnd(type == 5 ? L->xmb : L->xa_next, r, col, NN, x * bf2f(gn[r]));
            }
            const float s2 = half_warp_sum(x * x);
            if (store && row == 0)
              (type == 5 ? L->ssm : L->ssa_next)[(size_t)col * p.n_parts + (r >> 4)] = s2;
          } else if (type == 6) {
            // rows (2i, 2i + 1) = (gate_i, up_i) sit on neighbouring lanes
            const float gv = v * inv;
            const float uv = __shfl_xor_sync(0xffffffffu, gv, 1);
            if (store && !(row & 1)) {
              const int i = r >> 1;
              const float hv = gv / (1.f + __expf(-gv)) * uv;
              L->h[(size_t)col * p.F + i] = hv;
              put_opnd(L->hb, i, col, NN, hv);
            }
          } else {
            const float lv = v * inv;
            if (store) {
              if (p.logits && sm.ctl[kLogits]) p.logits[(size_t)col * p.V + r] = lv;
              if (lv > best_v || (lv == best_v && r < best_i)) {
                best_v = lv;
                best_i = r;
              }
            }
          }
        }
      }
      compute_sync();
    }
#pragma unroll
    for (int m = 0; m < kMmaMaxMB; ++m)
#pragma unroll
      for (int n = 0; n < NN; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[m][n][i] = 0.f;
  }
  trace_mark(p, sm, 1);
  if (sm.ctl[kAbort]) return false;
  if (type == 8) {
    // (max, lowest index) per sequence: the 16 lanes of a half warp share a
    // column, then the 16 / NC half warps of each column
    float bv = best_v;
    int bi = best_i;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (row == 0) {
      sm.mlv[tid >> 4] = bv;
      sm.mli[tid >> 4] = bi;
    }
    compute_sync();
    if (tid < p.B) {
      bv = -INFINITY;
      bi = 0x7fffffff;
      for (int h = tid; h < 16; h += NC) {
        const float ov = sm.mlv[h];
        const int oi = sm.mli[h];
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
      if (bi == 0x7fffffff) bi = mt.mt0 * 16;  // all values NaN: keep a valid index
      p.lm_val[(size_t)tid * p.n_lm + t.idx] = bv;
      p.lm_idx[(size_t)tid * p.n_lm + t.idx] = bi;
    }
  }
  return true;
}

// ---------------------------------------------------------------------------
// Attention: one (sequence b, kv head g, split s).
// ---------------------------------------------------------------------------
// Split-KV attention: after writing its partial, a split arrives on the
// (layer, sequence, kv head) counter; the split that arrives last merges all
// partials (online softmax:  M = max_s m_s,  w_s = exp(m_s - M),
// o = sum_s w_s o_s / sum_s w_s l_s) into the head block of att and resets the
// counter, so no separate merge task (and no extra event) is needed.  The
// acquire-release atomic orders every split's partial before the merge reads.
// Each warp owns (head, 64 dims) slices and issues a pass of kPass splits'
// loads at once; passes combine online.
// expect: the arrivals that complete (b, g); ns: the partial slots 0 .. ns - 1
// to merge.
__device__ __forceinline__ bool attn_arrive_and_merge(const Params &p, const Smem &sm, int layer,
                                                      int b, int g, int expect, int ns) {
  constexpr int kPass = 24;  // splits merged per round trip
  compute_sync();  // every thread's partial stores precede the arrival
  uint32_t *ctr = p.arrivals + ((size_t)layer * p.B + b) * p.Hkv + g;
  if (threadIdx.x == 0) {
    const uint32_t old = atom_acq_rel_add(ctr, 1u);
    sm.ctl[kLast] = old + 1u == (uint32_t)expect;
  }
  compute_sync();
  if (!sm.ctl[kLast]) return true;
  if (threadIdx.x == 0) *ctr = 0u;  // every split of this step has arrived
  const DevLayer &L = p.layers[layer];
  const int D = p.D, rep = p.rep;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int per_head = D / 64;  // warps per head (64 dims each, 2 per lane)
  for (int slice = warp; slice < rep * per_head; slice += kComputeWarps) {
    const int h = slice / per_head;
    const int d0 = (slice % per_head) * 64 + lane;
    const float *src = L.part + (((size_t)b * p.Hq + g * rep + h) * p.S) * (D + 2);
    float M = -INFINITY, den = 0.f, n0 = 0.f, n1 = 0.f;
    for (int s0 = 0; s0 < ns; s0 += kPass) {
      // every load of the pass is issued before any is used: lane i holds
      // split s0 + i's running max and sum, every lane its two dims of
      // each split
      const bool mine = lane < kPass && s0 + lane < ns;
      const float *pl = src + (size_t)(s0 + lane) * (D + 2);
      const float ml = mine ? __ldcg(pl + D) : -INFINITY;
      const float ll = mine ? __ldcg(pl + D + 1) : 0.f;
      float o0[kPass], o1[kPass];
#pragma unroll
      for (int i = 0; i < kPass; ++i) {
        const bool ok = s0 + i < ns;
        const float *ps = src + (size_t)(s0 + i) * (D + 2);
        o0[i] = ok ? __ldcg(ps + d0) : 0.f;
        o1[i] = ok ? __ldcg(ps + d0 + 32) : 0.f;
      }
      const float Mp = fmaxf(M, warp_max(ml));
      const float r = M == -INFINITY ? 0.f : __expf(M - Mp);
      const float wl = ml == -INFINITY ? 0.f : __expf(ml - Mp);
      den = den * r + warp_sum(wl * ll);
      n0 *= r;
      n1 *= r;
#pragma unroll
      for (int i = 0; i < kPass; ++i) {
        const float w = __shfl_sync(0xffffffffu, wl, i);
        n0 = fmaf(w, o0[i], n0);
        n1 = fmaf(w, o1[i], n1);
      }
      M = Mp;
    }
    const int c0 = (g * rep + h) * D + d0;
    float *dst = L.att + (size_t)b * p.qdim;
    const float inv = 1.f / den;
    dst[c0] = n0 * inv;
    dst[c0 + 32] = n1 * inv;
    if (p.mma) {
      put_opnd(L.attb, c0, b, p.nn, n0 * inv);
      put_opnd(L.attb, c0 + 32, b, p.nn, n1 * inv);
    }
  }
  return true;
}

// bf16 pair (lo element in the low half) and its rounding remainder pair:
// x = hi + lo to about 16 significant bits (see opnd_off).
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  const uint16_t h0 = f2bf(x0), h1 = f2bf(x1);
  hi = (uint32_t)h0 | ((uint32_t)h1 << 16);
  lo = (uint32_t)f2bf(x0 - bf2f(h0)) | ((uint32_t)f2bf(x1 - bf2f(h1)) << 16);
}

// One block of 8 positions [j0, j0 + 8) of a K/V tile (rows of D bf16) for
// one warp, on tensor cores.  Query heads are the rows of the MMA, positions
// its columns:
//   S  = Q K^T        m16n8k16; rows g < 8 hold q head g's hi bf16 term and
//                     rows g + 8 its lo term, so lane (g, t) receives both
//                     halves of head g's scores at positions 2t, 2t + 1 and
//                     adds them (one MMA per k-step for both terms)
//   P  = exp(S - m)   online softmax on the accumulator fragments: head g's 8
//                     scores sit in the 4 lanes of quad g (2 each)
//   O^T += V^T P^T    m16n8k8, V fragments by ldmatrix.trans; the B fragment
//                     of P^T is the lane's own pair of probabilities.  pk (at
//                     most 4 heads): P's hi term in columns h < 4 and its lo
//                     term in columns h + 4 of the same MMA, added once at the
//                     end of the task; else one MMA per term.
// K and V are exact bf16.  Positions >= n are masked; their rows are read
// from position n - 1 so every value stays finite.  Lane (g, t) keeps head
// g's running max and sum (m_run, l_run) and o[j] = O^T rows (16 j + g,
// 16 j + g + 8), columns (2 t, 2 t + 1).
// Byte offset of (row r, 16-byte chunk c16 of the head dims) in a K or V
// tile.  SWZ: D / 64 TMA boxes of 64 dims x `rows` rows with the 128-byte
// swizzle (chunk c of row r stored at chunk c ^ (r mod 8) of its 128-byte
// line; conflict-free for 8 consecutive rows); else plain row-major rows.
template <int D, bool SWZ>
__device__ __forceinline__ uint32_t kv_off(int r, int c16, int rows) {
  if (!SWZ) return (uint32_t)(r * D * 2 + c16 * 16);
  return (uint32_t)((c16 >> 3) * rows * 128 + r * 128 + (((c16 & 7) ^ (r & 7)) << 4));
}

template <int D, bool SWZ>
__device__ __forceinline__ void attn_block_mma(uint32_t kbase, uint32_t vbase, int rows, int j0,
                                               int n, bool pk, const uint32_t (&qh)[D / 16][2],
                                               const uint32_t (&ql)[D / 16][2], float &m_run,
                                               float &l_run, float (&o)[D / 16][4]) {
  const int lane = threadIdx.x & 31, t = lane & 3;
  // ldmatrix rows: 8 consecutive positions (distinct r mod 8: no bank conflicts)
  const int pos = min(j0 + (lane & 7), n - 1);
  const int mat = lane >> 3;  // the 8 x 8 matrix this lane addresses
  // two independent accumulation chains (even / odd k-step), summed
  float sa[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i) sa[i][0] = sa[i][1] = sa[i][2] = sa[i][3] = 0.f;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {  // 32 dims (two k-steps) per ldmatrix.x4
    uint32_t b[4];
    ldmatrix_x4(b, kbase + kv_off<D, SWZ>(pos, 4 * c + mat, rows));
    mma_bf16(sa[0], make_uint4(qh[2 * c][0], ql[2 * c][0], qh[2 * c][1], ql[2 * c][1]),
             make_uint2(b[0], b[1]));
    mma_bf16(sa[1], make_uint4(qh[2 * c + 1][0], ql[2 * c + 1][0], qh[2 * c + 1][1], ql[2 * c + 1][1]),
             make_uint2(b[2], b[3]));
  }
  float s[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) s[i] = (sa[0][i] + sa[1][i]) + (sa[0][i + 2] + sa[1][i + 2]);
  const bool v0 = j0 + 2 * t < n, v1 = j0 + 2 * t + 1 < n;
  const float s0 = v0 ? s[0] : -INFINITY, s1 = v1 ? s[1] : -INFINITY;
  float mx = fmaxf(s0, s1);
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  const float m_new = fmaxf(m_run, mx);  // finite: position j0 < n is valid
  const float alpha = m_run == -INFINITY ? 0.f : __expf(m_run - m_new);
  const float p0 = v0 ? __expf(s0 - m_new) : 0.f, p1 = v1 ? __expf(s1 - m_new) : 0.f;
  float sum = p0 + p1;
  sum += __shfl_xor_sync(0xffffffffu, sum, 1);
  sum += __shfl_xor_sync(0xffffffffu, sum, 2);
  l_run = l_run * alpha + sum;
  m_run = m_new;
  uint32_t ph, pl;
  split_pair(p0, p1, ph, pl);
  // rescale factors of the heads of columns 2t, 2t + 1 (column c is head
  // c & 3 when P is packed)
  const int c0 = pk ? (2 * t) & 3 : 2 * t;
  const float a0 = __shfl_sync(0xffffffffu, alpha, 4 * c0);
  const float a1 = __shfl_sync(0xffffffffu, alpha, 4 * c0 + 4);
#pragma unroll
  for (int j = 0; j < D / 16; ++j) {
    o[j][0] *= a0;
    o[j][1] *= a1;
    o[j][2] *= a0;
    o[j][3] *= a1;
  }
  // packed: lanes of quads 4..7 supply the lo term of head g - 4
  const uint32_t pl_up = __shfl_xor_sync(0xffffffffu, pl, 16);
  const uint32_t pb = (lane >> 2) < 4 ? ph : pl_up;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {  // two 16-dim m-tiles per ldmatrix.x4.trans
    uint32_t v[4];
    ldmatrix_x4_trans(v, vbase + kv_off<D, SWZ>(pos, 4 * c + mat, rows));
    if (pk) {
      mma_bf16_k8(o[2 * c], v[0], v[1], pb);
      mma_bf16_k8(o[2 * c + 1], v[2], v[3], pb);
    } else {
      mma_bf16_k8(o[2 * c], v[0], v[1], ph);
      mma_bf16_k8(o[2 * c], v[0], v[1], pl);
      mma_bf16_k8(o[2 * c + 1], v[2], v[3], ph);
      mma_bf16_k8(o[2 * c + 1], v[2], v[3], pl);
    }
  }
}

// Two 8-position tiles [j0, j0 + 8) and [j0 + 8, j0 + 16) at once: the same
// S and softmax steps on both (independent MMA chains), one rescale of o,
// and O^T += V^T P^T as m16n8k16 over the 16 positions (the B fragment of
// P^T is the lane's own probabilities of both tiles).
template <int D, bool SWZ>
__device__ __forceinline__ void attn_block16_mma(uint32_t kbase, uint32_t vbase, int rows, int j0,
                                                 int n, bool pk, const uint32_t (&qh)[D / 16][2],
                                                 const uint32_t (&ql)[D / 16][2], float &m_run,
                                                 float &l_run, float (&o)[D / 16][4]) {
  const int lane = threadIdx.x & 31, t = lane & 3;
  const int pa = min(j0 + (lane & 7), n - 1), pb = min(j0 + 8 + (lane & 7), n - 1);
  const int mat = lane >> 3;
  float sa[2][4], sb[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int r = 0; r < 4; ++r) sa[i][r] = sb[i][r] = 0.f;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t ka[4], kb[4];
    ldmatrix_x4(ka, kbase + kv_off<D, SWZ>(pa, 4 * c + mat, rows));
    ldmatrix_x4(kb, kbase + kv_off<D, SWZ>(pb, 4 * c + mat, rows));
    const uint4 q0 = make_uint4(qh[2 * c][0], ql[2 * c][0], qh[2 * c][1], ql[2 * c][1]);
    const uint4 q1 = make_uint4(qh[2 * c + 1][0], ql[2 * c + 1][0], qh[2 * c + 1][1], ql[2 * c + 1][1]);
    mma_bf16(sa[0], q0, make_uint2(ka[0], ka[1]));
    mma_bf16(sb[0], q0, make_uint2(kb[0], kb[1]));
    mma_bf16(sa[1], q1, make_uint2(ka[2], ka[3]));
    mma_bf16(sb[1], q1, make_uint2(kb[2], kb[3]));
  }
  float sv[4];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    sv[i] = (sa[0][i] + sa[1][i]) + (sa[0][i + 2] + sa[1][i + 2]);
    sv[i + 2] = (sb[0][i] + sb[1][i]) + (sb[0][i + 2] + sb[1][i + 2]);
  }
  bool ok[4];
  ok[0] = j0 + 2 * t < n;
  ok[1] = j0 + 2 * t + 1 < n;
  ok[2] = j0 + 8 + 2 * t < n;
  ok[3] = j0 + 9 + 2 * t < n;
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    sv[i] = ok[i] ? sv[i] : -INFINITY;
    mx = fmaxf(mx, sv[i]);
  }
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  const float m_new = fmaxf(m_run, mx);  // finite: position j0 < n is valid
  const float alpha = m_run == -INFINITY ? 0.f : __expf(m_run - m_new);
  float pr[4], sum = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    pr[i] = ok[i] ? __expf(sv[i] - m_new) : 0.f;
    sum += pr[i];
  }
  sum += __shfl_xor_sync(0xffffffffu, sum, 1);
  sum += __shfl_xor_sync(0xffffffffu, sum, 2);
  l_run = l_run * alpha + sum;
  m_run = m_new;
  uint32_t pha, pla, phb, plb;
  split_pair(pr[0], pr[1], pha, pla);
  split_pair(pr[2], pr[3], phb, plb);
  const int c0 = pk ? (2 * t) & 3 : 2 * t;
  const float a0 = __shfl_sync(0xffffffffu, alpha, 4 * c0);
  const float a1 = __shfl_sync(0xffffffffu, alpha, 4 * c0 + 4);
#pragma unroll
  for (int j = 0; j < D / 16; ++j) {
    o[j][0] *= a0;
    o[j][1] *= a1;
    o[j][2] *= a0;
    o[j][3] *= a1;
  }
  const bool upper = (lane >> 2) < 4;
  const uint32_t pla_up = __shfl_xor_sync(0xffffffffu, pla, 16);
  const uint32_t plb_up = __shfl_xor_sync(0xffffffffu, plb, 16);
  const uint2 bp = make_uint2(upper ? pha : pla_up, upper ? phb : plb_up);
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t va[4], vb[4];
    ldmatrix_x4_trans(va, vbase + kv_off<D, SWZ>(pa, 4 * c + mat, rows));
    ldmatrix_x4_trans(vb, vbase + kv_off<D, SWZ>(pb, 4 * c + mat, rows));
    const uint4 v0 = make_uint4(va[0], va[1], vb[0], vb[1]);
    const uint4 v1 = make_uint4(va[2], va[3], vb[2], vb[3]);
    if (pk) {
      mma_bf16(o[2 * c], v0, bp);
      mma_bf16(o[2 * c + 1], v1, bp);
    } else {
      mma_bf16(o[2 * c], v0, make_uint2(pha, phb));
      mma_bf16(o[2 * c], v0, make_uint2(pla, plb));
      mma_bf16(o[2 * c + 1], v1, make_uint2(pha, phb));
      mma_bf16(o[2 * c + 1], v1, make_uint2(pla, plb));
    }
  }
}

// Decode attention for one (sequence b, kv head g, split s), splits fixed at
// build time (the default kernels): q/k RMSNorm and RoPE prologue, K/V
// append, then every warp runs flash-decoding style over
// its own 8-position blocks on tensor cores (no CTA barrier inside the loop)
// and the warps' states are merged once at the end.  D: head dim (64, 128);
// SWZ: the K/V tiles arrive as swizzled TMA boxes (else as plain rows).
template <int D, bool SWZ>
__device__ __forceinline__ bool attn_task_fixed(const Params &p, const Smem &sm, const DevTask &t,
                                                uint32_t &k, int task_id,
                                                const DepWait &dep_wait) {
  constexpr int NP = 8;  // positions per warp block
  // the span read before the wait is exact when the launch runs one step
  // (kv_len is fixed during it); a multi-step launch re-reads it after the wait
  const AttnSpan a0 = attn_span(p, (int)t.idx);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rep = p.rep;
  constexpr int dpl = D >> 5;
  const DevLayer &L = p.layers[t.layer];
  const float *qkv = L.qkv + (size_t)a0.b * p.n_qkv + (size_t)a0.g * p.grp;
  // gains and RoPE factors of this lane's dims (the RoPE position is the
  // speculative one above): loaded before the wait
  float gq[4], gk[4], rc[2], rs[2];
  for (int i = 0; i < dpl; ++i) {
    gq[i] = bf2f(L.q_norm[lane + 32 * i]);
    gk[i] = bf2f(L.k_norm[lane + 32 * i]);
  }
  auto load_rope = [&](int pos) {  // [D/2][2] cos, sin of position pos
    const float *rope = p.rope + (size_t)pos * D;
    for (int i = 0; i < (dpl >> 1); ++i) {
      rc[i] = rope[2 * (lane + 32 * i)];
      rs[i] = rope[2 * (lane + 32 * i) + 1];
    }
  };
  load_rope(a0.L);
  if (!dep_wait()) return false;
  AttnSpan a = a0;
  if (p.n_steps > 1) {  // kv_len advanced by the previous step of this launch
    a = attn_span(p, (int)t.idx);
    if (a.L != a0.L) load_rope(a.L);
  }
  const int nmerge = min(p.S, a.L / p.chunk + 1);  // splits that hold any position
  if (!a.active)  // the split starts past the new row: it only arrives
    return attn_arrive_and_merge(p, sm, t.layer, a.b, a.g, p.S, nmerge);

  // prologue: per-head RMSNorm + RoPE of q (and of the new k when this split
  // holds position L; v is only rounded)
  for (int row = warp; row < rep + 2; row += kComputeWarps) {
    if (row >= rep && !a.has_new) continue;
    float v[4];
    for (int i = 0; i < dpl; ++i) v[i] = __ldcg(qkv + row * D + lane + 32 * i);
    if (row <= rep) {  // q heads and k
      float ss = 0.f;
      for (int i = 0; i < dpl; ++i) ss = fmaf(v[i], v[i], ss);
      ss = warp_sum(ss);
      const float inv = rsqrtf(ss / (float)D + p.eps);
      for (int i = 0; i < dpl; ++i) v[i] = v[i] * inv * (row < rep ? gq[i] : gk[i]);
      const int hp = dpl >> 1;  // dims lane + 32 i pair with lane + 32 (i + hp)
      for (int i = 0; i < hp; ++i) {
        const float c = rc[i], s = rs[i];
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
  compute_sync();
  // Q fragments (rows = heads, zero from rep on) as hi/lo bf16 pairs
  const int gq_row = lane >> 2, tq = lane & 3;
  uint32_t qh[D / 16][2], ql[D / 16][2];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int c = 16 * kk + 2 * tq + 8 * half;
      const bool ok = gq_row < rep;
      const float x0 = ok ? sm.q[gq_row * kMaxHeadDim + c] : 0.f;
      const float x1 = ok ? sm.q[gq_row * kMaxHeadDim + c + 1] : 0.f;
      split_pair(x0, x1, qh[kk][half], ql[kk][half]);
    }
  }
  float o[D / 16][4];
#pragma unroll
  for (int j = 0; j < D / 16; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) o[j][i] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  const bool pk = rep <= 4;  // P's hi and lo terms share one MMA
  // 16-position blocks when the stages hold whole ones (8-position otherwise)
  const bool np16 = p.pps % (2 * NP) == 0;
  trace_mark(p, sm, 0);

  const int cached = a.cached_end - a.p0;
  const int nst = cached > 0 ? (cached + p.pps - 1) / p.pps : 0;
  for (int st = 0; st < nst; ++st) {
    const int n = min(p.pps, cached - st * p.pps);
    const bool got = sm.ctl[kAbort] ? false : wait_full(p, sm, k, task_id);
    if (!got) continue;
    trace_first_stage(p, sm, st);
    const uint32_t kb = smem_u32(sm.ring + (size_t)(k % p.ring_stages) * p.stage_bytes);
    const uint32_t vb = kb + (uint32_t)(p.pps * D * 2);  // V boxes follow the K boxes
    // blocks are numbered across the split's stages and dealt round-robin
    // (warp w takes global blocks w, w + 8, ...), so a stage whose block
    // count is not a multiple of 8 does not leave the same warps idle every
    // time; warps drift apart by at most the ring depth
    if (np16) {
      const int base = st * (p.pps / (2 * NP));
      for (int j0 = ((warp - base) % kComputeWarps + kComputeWarps) % kComputeWarps * 2 * NP;
           j0 < n; j0 += kComputeWarps * 2 * NP)
        attn_block16_mma<D, SWZ>(kb, vb, p.pps, j0, n, pk, qh, ql, m_run, l_run, o);
    } else {
      const int base = st * (p.pps / NP);
      for (int j0 = ((warp - base) % kComputeWarps + kComputeWarps) % kComputeWarps * NP; j0 < n;
           j0 += kComputeWarps * NP)
        attn_block_mma<D, SWZ>(kb, vb, p.pps, j0, n, pk, qh, ql, m_run, l_run, o);
    }
    release_stage(sm, p, k);
    ++k;
  }
  // the new row: one more block, on the warp after the last cached block
  const int blk = np16 ? 2 * NP : NP;
  if (a.has_new && warp == ((cached + blk - 1) / blk) % kComputeWarps)
    attn_block_mma<D, false>(smem_u32(sm.knew), smem_u32(sm.vnew), 0, 0, 1, pk, qh, ql, m_run, l_run,
                             o);

  trace_mark(p, sm, 1);
  if (pk) {  // add the lo-term columns h + 4 into the columns h of lanes tq < 2
#pragma unroll
    for (int j = 0; j < D / 16; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[j][i] += __shfl_down_sync(0xffffffffu, o[j][i], 2);
  }
  // every warp's state to shared memory: o (heads 2 tq, 2 tq + 1), then the
  // running max and sum of head gq_row
  static_assert(kStateSlots == kComputeWarps, "one state slot per warp");
  const int stride = D + 2;
  {
    float *st_w = sm.ored + (size_t)warp * p.rep_p * stride;
    const int h0 = 2 * tq, h1 = 2 * tq + 1;
#pragma unroll
    for (int j = 0; j < D / 16; ++j) {
      const int d = 16 * j + gq_row;
      if (h0 < rep) {
        st_w[h0 * stride + d] = o[j][0];
        st_w[h0 * stride + d + 8] = o[j][2];
      }
      if (h1 < rep) {
        st_w[h1 * stride + d] = o[j][1];
        st_w[h1 * stride + d + 8] = o[j][3];
      }
    }
    if (tq == 0 && gq_row < rep) {
      st_w[gq_row * stride + D] = m_run;
      st_w[gq_row * stride + D + 1] = l_run;
    }
  }
  compute_sync();
  if (sm.ctl[kAbort]) return false;
  for (int oi = tid; oi < rep * D; oi += kComputeThreads) {
    const int h = oi / D, d = oi - h * D;
    float M = -INFINITY;
    for (int w = 0; w < kStateSlots; ++w)
      M = fmaxf(M, sm.ored[((size_t)w * p.rep_p + h) * stride + D]);
    float num = 0.f, den = 0.f;
    for (int w = 0; w < kStateSlots; ++w) {
      const float *sw = sm.ored + ((size_t)w * p.rep_p + h) * stride;
      const float mw = sw[D];
      const float e = mw == -INFINITY ? 0.f : __expf(mw - M);
      den = fmaf(e, sw[D + 1], den);
      num = fmaf(e, sw[d], num);
    }
    const int head = a.g * rep + h;
    if (p.S == 1) {
      L.att[(size_t)a.b * p.qdim + head * D + d] = num / den;
      if (p.mma) put_opnd(L.attb, head * D + d, a.b, p.nn, num / den);
    } else {
      float *dst = L.part + (((size_t)a.b * p.Hq + head) * p.S + a.s) * (D + 2);
      dst[d] = num;
      if (d == 0) {
        dst[D] = M;
        dst[D + 1] = den;
      }
    }
  }
  if (p.S == 1) return true;
  return attn_arrive_and_merge(p, sm, t.layer, a.b, a.g, p.S, nmerge);
}

// Decode attention of one piece (see AttnSeg) on tensor cores: q/k RMSNorm
// and RoPE prologue, K/V append when the piece holds the new row, then every
// warp runs flash-decoding style over its own position blocks of the piece's
// stages (no CTA barrier inside the loop), the warps' states are merged once,
// and the piece's result goes to att (a piece that completes its pair alone)
// or to its partial slot, the last arriving piece of the pair merging.
// D: head dim (64, 128); SWZ: the K/V tiles arrive as swizzled TMA boxes
// (else as plain rows).  gq, gk: this lane's q/k norm gains.
template <int D, bool SWZ>
__device__ __forceinline__ bool attn_piece(const Params &p, const Smem &sm, int layer,
                                           const AttnSeg &sg, const float (&gq)[4],
                                           const float (&gk)[4], uint32_t &k, int task_id) {
  constexpr int NP = 8;  // positions per warp block
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rep = p.rep;
  constexpr int dpl = D >> 5;
  const DevLayer &L = p.layers[layer];
  const float *qkv = L.qkv + (size_t)sg.b * p.n_qkv + (size_t)sg.g * p.grp;
  float rc[2], rs[2];
  {
    const float *rope = p.rope + (size_t)sg.L * D;  // [D/2][2] cos, sin of position L
    for (int i = 0; i < (dpl >> 1); ++i) {
      rc[i] = rope[2 * (lane + 32 * i)];
      rs[i] = rope[2 * (lane + 32 * i) + 1];
    }
  }
  // every warp's state slots of the previous piece have been read
  compute_sync();
  // prologue: per-head RMSNorm + RoPE of q (and of the new k when this piece
  // holds position L; v is only rounded)
  for (int row = warp; row < rep + 2; row += kComputeWarps) {
    if (row >= rep && !sg.has_new) continue;
    float v[4];
    for (int i = 0; i < dpl; ++i) v[i] = __ldcg(qkv + row * D + lane + 32 * i);
    if (row <= rep) {  // q heads and k
      float ss = 0.f;
      for (int i = 0; i < dpl; ++i) ss = fmaf(v[i], v[i], ss);
      ss = warp_sum(ss);
      const float inv = rsqrtf(ss / (float)D + p.eps);
      for (int i = 0; i < dpl; ++i) v[i] = v[i] * inv * (row < rep ? gq[i] : gk[i]);
      const int hp = dpl >> 1;  // dims lane + 32 i pair with lane + 32 (i + hp)
      for (int i = 0; i < hp; ++i) {
        const float c = rc[i], s = rs[i];
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
      const size_t off = kv_row(p, layer, sg.b, sg.g, sg.L);
      for (int i = 0; i < dpl; ++i) {
        const uint16_t hb = f2bf(v[i]);
        cache[off + lane + 32 * i] = hb;
        dst[lane + 32 * i] = hb;
      }
    }
  }
  compute_sync();
  // Q fragments (rows = heads, zero from rep on) as hi/lo bf16 pairs
  const int gq_row = lane >> 2, tq = lane & 3;
  uint32_t qh[D / 16][2], ql[D / 16][2];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int c = 16 * kk + 2 * tq + 8 * half;
      const bool ok = gq_row < rep;
      const float x0 = ok ? sm.q[gq_row * kMaxHeadDim + c] : 0.f;
      const float x1 = ok ? sm.q[gq_row * kMaxHeadDim + c + 1] : 0.f;
      split_pair(x0, x1, qh[kk][half], ql[kk][half]);
    }
  }
  float o[D / 16][4];
#pragma unroll
  for (int j = 0; j < D / 16; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) o[j][i] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  const bool pk = rep <= 4;  // P's hi and lo terms share one MMA
  // 16-position blocks when the stages hold whole ones (8-position otherwise)
  const bool np16 = p.pps % (2 * NP) == 0;
  trace_mark(p, sm, 0);

  const int nst = seg_stages(p, sg);
  for (int st = 0; st < nst; ++st) {
    const int r0 = max(sg.c0, sg.o + st * p.pps);
    const int n = min(sg.c1, sg.o + (st + 1) * p.pps) - r0;  // rows of the box that count
    const bool got = sm.ctl[kAbort] ? false : wait_full(p, sm, k, task_id);
    if (!got) continue;
    trace_first_stage(p, sm, st);
    const uint32_t kb = smem_u32(sm.ring + (size_t)(k % p.ring_stages) * p.stage_bytes);
    const uint32_t vb = kb + (uint32_t)(p.pps * D * 2);  // V boxes follow the K boxes
    // blocks are numbered across the piece's stages and dealt round-robin
    // (warp w takes global blocks w, w + 8, ...), so a stage whose block
    // count is not a multiple of 8 does not leave the same warps idle every
    // time; warps drift apart by at most the ring depth
    if (np16) {
      const int base = st * (p.pps / (2 * NP));
      for (int j0 = ((warp - base) % kComputeWarps + kComputeWarps) % kComputeWarps * 2 * NP;
           j0 < n; j0 += kComputeWarps * 2 * NP)
        attn_block16_mma<D, SWZ>(kb, vb, p.pps, j0, n, pk, qh, ql, m_run, l_run, o);
    } else {
      const int base = st * (p.pps / NP);
      for (int j0 = ((warp - base) % kComputeWarps + kComputeWarps) % kComputeWarps * NP; j0 < n;
           j0 += kComputeWarps * NP)
        attn_block_mma<D, SWZ>(kb, vb, p.pps, j0, n, pk, qh, ql, m_run, l_run, o);
    }
    release_stage(sm, p, k);
    ++k;
  }
  // the new row: one more block, on the warp after the last cached block
  const int cached = max(0, sg.c1 - sg.c0);
  const int blk = np16 ? 2 * NP : NP;
  if (sg.has_new && warp == ((cached + blk - 1) / blk) % kComputeWarps)
    attn_block_mma<D, false>(smem_u32(sm.knew), smem_u32(sm.vnew), 0, 0, 1, pk, qh, ql, m_run, l_run,
                             o);

  trace_mark(p, sm, 1);
  if (pk) {  // add the lo-term columns h + 4 into the columns h of lanes tq < 2
#pragma unroll
    for (int j = 0; j < D / 16; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[j][i] += __shfl_down_sync(0xffffffffu, o[j][i], 2);
  }
  // every warp's state to shared memory: o (heads 2 tq, 2 tq + 1), then the
  // running max and sum of head gq_row
  static_assert(kStateSlots == kComputeWarps, "one state slot per warp");
  const int stride = D + 2;
  {
    float *st_w = sm.ored + (size_t)warp * p.rep_p * stride;
    const int h0 = 2 * tq, h1 = 2 * tq + 1;
#pragma unroll
    for (int j = 0; j < D / 16; ++j) {
      const int d = 16 * j + gq_row;
      if (h0 < rep) {
        st_w[h0 * stride + d] = o[j][0];
        st_w[h0 * stride + d + 8] = o[j][2];
      }
      if (h1 < rep) {
        st_w[h1 * stride + d] = o[j][1];
        st_w[h1 * stride + d + 8] = o[j][3];
      }
    }
    if (tq == 0 && gq_row < rep) {
      st_w[gq_row * stride + D] = m_run;
      st_w[gq_row * stride + D + 1] = l_run;
    }
  }
  compute_sync();
  if (sm.ctl[kAbort]) return false;
  for (int oi = tid; oi < rep * D; oi += kComputeThreads) {
    const int h = oi / D, d = oi - h * D;
    float M = -INFINITY;
    for (int w = 0; w < kStateSlots; ++w)
      M = fmaxf(M, sm.ored[((size_t)w * p.rep_p + h) * stride + D]);
    float num = 0.f, den = 0.f;
    for (int w = 0; w < kStateSlots; ++w) {
      const float *sw = sm.ored + ((size_t)w * p.rep_p + h) * stride;
      const float mw = sw[D];
      const float e = mw == -INFINITY ? 0.f : __expf(mw - M);
      den = fmaf(e, sw[D + 1], den);
      num = fmaf(e, sw[d], num);
    }
    const int head = sg.g * rep + h;
    if (sg.expect == 1) {
      L.att[(size_t)sg.b * p.qdim + head * D + d] = num / den;
      put_opnd(L.attb, head * D + d, sg.b, p.nn, num / den);
    } else {
      float *dst = L.part + (((size_t)sg.b * p.Hq + head) * p.S + sg.slot) * (D + 2);
      dst[d] = num;
      if (d == 0) {
        dst[D] = M;
        dst[D + 1] = den;
      }
    }
  }
  if (sg.expect == 1) return true;
  return attn_arrive_and_merge(p, sm, layer, sg.b, sg.g, sg.expect, sg.nmerge);
}

// Decode attention task of the extended batched kernels (JIT attention or
// dispatch mode): one (sequence b, kv head g, split s) piece when the splits
// are fixed at build time, else the pieces of JIT task t.idx (see JitCursor).
template <int D, bool SWZ>
__device__ __forceinline__ bool attn_task(const Params &p, const Smem &sm, const DevTask &t,
                                          uint32_t &k, int task_id, const DepWait &dep_wait) {
  const int lane = threadIdx.x & 31;
  constexpr int dpl = D >> 5;
  const DevLayer &L = p.layers[t.layer];
  // the norm gains of this lane's dims: weights, loaded before the wait
  float gq[4], gk[4];
  for (int i = 0; i < dpl; ++i) {
    gq[i] = bf2f(L.q_norm[lane + 32 * i]);
    gk[i] = bf2f(L.k_norm[lane + 32 * i]);
  }
  if (!dep_wait()) return false;
  if (p.jit) {
    JitShared &js = *sm.jit;
    if (threadIdx.x == 0) js.cur.start(p, (int)t.idx, jit_part(p, js.lens_c));
    for (;;) {
      if (threadIdx.x == 0) js.more = js.cur.next(p, js.seg);
      compute_sync();
      if (!js.more) return true;
      const AttnSeg sg = js.seg;
      if (!attn_piece<D, SWZ>(p, sm, t.layer, sg, gq, gk, k, task_id)) return false;
    }
  }
  // splits fixed at build time; kv_len is read after the wait (a multi-step
  // launch advances it between steps)
  const AttnSpan a = attn_span(p, (int)t.idx);
  const int nmerge = min(p.S, a.L / p.chunk + 1);  // splits that hold any position
  if (!a.active)  // the split starts past the new row: it only arrives
    return attn_arrive_and_merge(p, sm, t.layer, a.b, a.g, p.S, nmerge);
  AttnSeg sg;
  sg.b = a.b;
  sg.g = a.g;
  sg.L = a.L;
  sg.c0 = a.p0;
  sg.c1 = a.cached_end;
  sg.o = a.p0;
  sg.has_new = a.has_new;
  sg.slot = a.s;
  sg.expect = p.S;
  sg.nmerge = nmerge;
  return attn_piece<D, SWZ>(p, sm, t.layer, sg, gq, gk, k, task_id);
}

// One block of up to NP = 32 / RP positions for one warp: scores, online
// softmax update of the warp's running state, and PV.  RP = q heads per kv head
// rounded up to a power of two (heads >= rep are padding).  Lane l covers dims
// [dpl*l, dpl*l + dpl) of every head; after the transposed score reduction lane
// l holds the score of head l / NP at position l % NP, and keeps the running
// max and sum of that head.  pw / aw: the warp's probability / rescale scratch.
template <int RP>
__device__ __forceinline__ void attn_block(const Params &p, float *pw, float *aw,
                                           const uint16_t *Ks, const uint16_t *Vs, int j0, int n,
                                           const float (&qr)[RP][4], float &m_run, float &l_run,
                                           float (&o)[RP][4]) {
  constexpr int NP = 32 / RP;
  const int lane = threadIdx.x & 31;
  const int D = p.D, dpl = D >> 5;
  float v[32];
#pragma unroll
  for (int jj = 0; jj < NP; ++jj) {
    float kf[4] = {0.f, 0.f, 0.f, 0.f};
    if (j0 + jj < n) {
      if (dpl == 4) {
        const uint2 kv = *reinterpret_cast<const uint2 *>(Ks + (size_t)(j0 + jj) * D + 4 * lane);
        kf[0] = bf_lo(kv.x); kf[1] = bf_hi(kv.x); kf[2] = bf_lo(kv.y); kf[3] = bf_hi(kv.y);
      } else {
        const uint32_t kv = *reinterpret_cast<const uint32_t *>(Ks + (size_t)(j0 + jj) * D + 2 * lane);
        kf[0] = bf_lo(kv); kf[1] = bf_hi(kv);
      }
    }
#pragma unroll
    for (int h = 0; h < RP; ++h) {
      float d = qr[h][0] * kf[0];
      d = fmaf(qr[h][1], kf[1], d);
      d = fmaf(qr[h][2], kf[2], d);
      d = fmaf(qr[h][3], kf[3], d);
      v[h * NP + jj] = d;
    }
  }
  float sc = warp_sum32(v, lane);
  const int h = lane / NP, jj = lane % NP;
  const bool valid = h < p.rep && j0 + jj < n;
  sc = valid ? sc : -INFINITY;
  float mx = sc;
#pragma unroll
  for (int off = NP / 2; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  const float m_new = fmaxf(m_run, mx);
  const float pj = valid ? __expf(sc - m_new) : 0.f;
  float sum = pj;
#pragma unroll
  for (int off = NP / 2; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float alpha = m_run == -INFINITY ? 0.f : __expf(m_run - m_new);
  l_run = l_run * alpha + sum;
  m_run = m_new;
  pw[jj * RP + h] = pj;
  if (jj == 0) aw[h] = alpha;
  __syncwarp();
#pragma unroll
  for (int hh = 0; hh < RP; ++hh) {
    const float a = aw[hh];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[hh][i] *= a;
  }
#pragma unroll
  for (int t = 0; t < NP; ++t) {
    if (j0 + t < n) {
      float vf[4] = {0.f, 0.f, 0.f, 0.f};
      if (dpl == 4) {
        const uint2 vv = *reinterpret_cast<const uint2 *>(Vs + (size_t)(j0 + t) * D + 4 * lane);
        vf[0] = bf_lo(vv.x); vf[1] = bf_hi(vv.x); vf[2] = bf_lo(vv.y); vf[3] = bf_hi(vv.y);
      } else {
        const uint32_t vv = *reinterpret_cast<const uint32_t *>(Vs + (size_t)(j0 + t) * D + 2 * lane);
        vf[0] = bf_lo(vv); vf[1] = bf_hi(vv);
      }
      float pr[RP];
      if constexpr (RP >= 4) {
#pragma unroll
        for (int q = 0; q < RP; q += 4) {
          const float4 p4 = *reinterpret_cast<const float4 *>(pw + t * RP + q);
          pr[q] = p4.x; pr[q + 1] = p4.y; pr[q + 2] = p4.z; pr[q + 3] = p4.w;
        }
      } else {
#pragma unroll
        for (int q = 0; q < RP; ++q) pr[q] = pw[t * RP + q];
      }
#pragma unroll
      for (int hh = 0; hh < RP; ++hh)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[hh][i] = fmaf(pr[hh], vf[i], o[hh][i]);
    }
  }
  __syncwarp();
}

// Decode attention for one (sequence b, kv head g, split s) on CUDA cores
// (the batch-1 kernel): q/k RMSNorm and RoPE prologue, K/V append, then every
// warp runs flash-decoding style over its own positions (no CTA barrier
// inside the loop) and the warps' states are merged once at the end.  At
// batch 1 a split is one 8-position block per warp and the step is bound by
// the weight stream; this body keeps the batch-1 kernel's register budget.
template <int RP>
__device__ __forceinline__ bool attn_task_cc(const Params &p, const Smem &sm, const DevTask &t,
                                          uint32_t &k, int task_id, const DepWait &dep_wait) {
  constexpr int NP = 32 / RP;
  // the span read before the wait is exact when the launch runs one step
  // (kv_len is fixed during it); a multi-step launch re-reads it after the wait
  const AttnSpan a0 = attn_span(p, (int)t.idx);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int D = p.D, rep = p.rep, dpl = D >> 5;
  const DevLayer &L = p.layers[t.layer];
  const float *qkv = L.qkv + (size_t)a0.b * p.n_qkv + (size_t)a0.g * p.grp;
  // gains and RoPE factors of this lane's dims (the RoPE position is the
  // speculative one above): loaded before the wait
  float gq[4], gk[4], rc[2], rs[2];
  for (int i = 0; i < dpl; ++i) {
    gq[i] = bf2f(L.q_norm[lane + 32 * i]);
    gk[i] = bf2f(L.k_norm[lane + 32 * i]);
  }
  auto load_rope = [&](int pos) {  // [D/2][2] cos, sin of position pos
    const float *rope = p.rope + (size_t)pos * D;
    for (int i = 0; i < (dpl >> 1); ++i) {
      rc[i] = rope[2 * (lane + 32 * i)];
      rs[i] = rope[2 * (lane + 32 * i) + 1];
    }
  };
  load_rope(a0.L);
  if (!dep_wait()) return false;
  AttnSpan a = a0;
  if (p.n_steps > 1) {  // kv_len advanced by the previous step of this launch
    a = attn_span(p, (int)t.idx);
    if (a.L != a0.L) load_rope(a.L);
  }
  const int nmerge = min(p.S, a.L / p.chunk + 1);  // splits that hold any position
  if (!a.active)  // the split starts past the new row: it only arrives
    return attn_arrive_and_merge(p, sm, t.layer, a.b, a.g, p.S, nmerge);

  // prologue: per-head RMSNorm + RoPE of q (and of the new k when this split
  // holds position L; v is only rounded)
  for (int row = warp; row < rep + 2; row += kComputeWarps) {
    if (row >= rep && !a.has_new) continue;
    float v[4];
    for (int i = 0; i < dpl; ++i) v[i] = __ldcg(qkv + row * D + lane + 32 * i);
    if (row <= rep) {  // q heads and k
      float ss = 0.f;
      for (int i = 0; i < dpl; ++i) ss = fmaf(v[i], v[i], ss);
      ss = warp_sum(ss);
      const float inv = rsqrtf(ss / (float)D + p.eps);
      for (int i = 0; i < dpl; ++i) v[i] = v[i] * inv * (row < rep ? gq[i] : gk[i]);
      const int hp = dpl >> 1;  // dims lane + 32 i pair with lane + 32 (i + hp)
      for (int i = 0; i < hp; ++i) {
        const float c = rc[i], s = rs[i];
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
  compute_sync();
  float qr[RP][4];
#pragma unroll
  for (int h = 0; h < RP; ++h)
#pragma unroll
    for (int i = 0; i < 4; ++i)
      qr[h][i] = (h < rep && i < dpl) ? sm.q[h * kMaxHeadDim + dpl * lane + i] : 0.f;
  float o[RP][4];
#pragma unroll
  for (int h = 0; h < RP; ++h)
#pragma unroll
    for (int i = 0; i < 4; ++i) o[h][i] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  trace_mark(p, sm, 0);
  float *pw = sm.sc + warp * (32 + kMaxRep);
  float *aw = pw + 32;

  const int cached = a.cached_end - a.p0;
  const int nst = cached > 0 ? (cached + p.pps - 1) / p.pps : 0;
  for (int st = 0; st < nst; ++st) {
    const int n = min(p.pps, cached - st * p.pps);
    const bool got = sm.ctl[kAbort] ? false : wait_full(p, sm, k, task_id);
    if (!got) continue;
    trace_first_stage(p, sm, st);
    const uint16_t *Ks =
        reinterpret_cast<const uint16_t *>(sm.ring + (size_t)(k % p.ring_stages) * p.stage_bytes);
    const uint16_t *Vs = Ks + (size_t)p.pps * p.D;  // V rows follow the pps K rows
    for (int j0 = warp * NP; j0 < n; j0 += kComputeWarps * NP)
      attn_block<RP>(p, pw, aw, Ks, Vs, j0, n, qr, m_run, l_run, o);
    release_stage(sm, p, k);
    ++k;
  }
  // the new row: one more block, on the warp after the last cached block
  if (a.has_new && warp == ((cached + NP - 1) / NP) % kComputeWarps)
    attn_block<RP>(p, pw, aw, sm.knew, sm.vnew, 0, 1, qr, m_run, l_run, o);

  trace_mark(p, sm, 1);
  // merge the warps' states: warps >= kStateSlots first fold into warp
  // (w - kStateSlots), then the kStateSlots states are combined per output
  const int stride = D + 2;
  if (kComputeWarps > kStateSlots) {
    if (warp >= kStateSlots) {
      float *st_w = sm.ored + (size_t)(warp - kStateSlots) * RP * stride;
#pragma unroll
      for (int h = 0; h < RP; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (i < dpl) st_w[h * stride + dpl * lane + i] = o[h][i];
      if (lane % NP == 0) {
        st_w[(lane / NP) * stride + D] = m_run;
        st_w[(lane / NP) * stride + D + 1] = l_run;
      }
    }
    compute_sync();
    if (warp < kStateSlots) {
      const float *st_p = sm.ored + (size_t)warp * RP * stride;
#pragma unroll
      for (int h = 0; h < RP; ++h) {
        const float m_me = __shfl_sync(0xffffffffu, m_run, h * NP);
        const float m_pa = st_p[h * stride + D];
        const float M = fmaxf(m_me, m_pa);
        const float a = m_me == -INFINITY ? 0.f : __expf(m_me - M);
        const float b = m_pa == -INFINITY ? 0.f : __expf(m_pa - M);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (i < dpl) o[h][i] = a * o[h][i] + b * st_p[h * stride + dpl * lane + i];
        if (lane / NP == h) {
          l_run = a * l_run + b * st_p[h * stride + D + 1];
          m_run = M;
        }
      }
    }
    compute_sync();
  }
  if (warp < kStateSlots) {
    float *st_w = sm.ored + (size_t)warp * RP * stride;
#pragma unroll
    for (int h = 0; h < RP; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (i < dpl) st_w[h * stride + dpl * lane + i] = o[h][i];
    if (lane % NP == 0) {
      const int h = lane / NP;
      st_w[h * stride + D] = m_run;
      st_w[h * stride + D + 1] = l_run;
    }
  }
  compute_sync();
  if (sm.ctl[kAbort]) return false;
  for (int oi = tid; oi < rep * D; oi += kComputeThreads) {
    const int h = oi / D, d = oi - h * D;
    float M = -INFINITY;
    for (int w = 0; w < kStateSlots; ++w) M = fmaxf(M, sm.ored[((size_t)w * RP + h) * stride + D]);
    float num = 0.f, den = 0.f;
    for (int w = 0; w < kStateSlots; ++w) {
      const float *sw = sm.ored + ((size_t)w * RP + h) * stride;
      const float mw = sw[D];
      const float e = mw == -INFINITY ? 0.f : __expf(mw - M);
      den = fmaf(e, sw[D + 1], den);
      num = fmaf(e, sw[d], num);
    }
    const int head = a.g * rep + h;
    if (p.S == 1) {
      L.att[(size_t)a.b * p.qdim + head * D + d] = num / den;
      if (p.mma) put_opnd(L.attb, head * D + d, a.b, p.nn, num / den);
    } else {
      float *dst = L.part + (((size_t)a.b * p.Hq + head) * p.S + a.s) * (D + 2);
      dst[d] = num;
      if (d == 0) {
        dst[D] = M;
        dst[D + 1] = den;
      }
    }
  }
  if (p.S == 1) return true;
  return attn_arrive_and_merge(p, sm, t.layer, a.b, a.g, p.S, nmerge);
}

// Batch >= 2 EMBED: kept out of line so its load batches do not raise the
// register demand of the worker loop.
// tok: this step's input tokens (read through L2: the previous step of the
// same launch may have written them).
__device__ __noinline__ void embed_batch(const Params &p, const int32_t *tok) {
  // One item per (k-block kb, sequence b < 8 nn): its 16 embedding elements
  // 16 kb .. 16 kb + 15 (two 16-byte loads) become the fp32 row slice, the
  // sum of squares of the 16-row part, and the 4 lane units of layer 0's
  // QKV operand: unit (kb, column tile b / 8, lane (b % 8, t)) holds
  // elements 16 kb + {2t, 2t + 1, 2t + 8, 2t + 9} times the attention-norm
  // gains as hi, then lo, bf16 pairs (zeros for padded sequences).  One CTA
  // does it all, so each thread keeps kU items' loads in flight before it
  // uses any.
  constexpr int kU = 4;
  const DevLayer &L0 = p.layers[0];
  const int nb8 = 8 * p.nn, items = (p.H >> 4) * nb8;
  const uint4 *gn = reinterpret_cast<const uint4 *>(L0.attn_norm);
  uint4 *xa = reinterpret_cast<uint4 *>(L0.xa);
  for (int i0 = threadIdx.x; i0 < items; i0 += kU * kComputeThreads) {
    uint4 e[kU][2], gw[kU][2];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int it = i0 + u * kComputeThreads;
      const int kb = it / nb8, b = it - kb * nb8;
      e[u][0] = e[u][1] = gw[u][0] = gw[u][1] = make_uint4(0u, 0u, 0u, 0u);
      if (it < items && b < p.B) {
        const uint4 *er = reinterpret_cast<const uint4 *>(p.embed + (size_t)__ldcg(tok + b) * p.H);
        e[u][0] = __ldg(er + 2 * kb);
        e[u][1] = __ldg(er + 2 * kb + 1);
        gw[u][0] = __ldg(gn + 2 * kb);
        gw[u][1] = __ldg(gn + 2 * kb + 1);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int it = i0 + u * kComputeThreads;
      if (it >= items) break;
      const int kb = it / nb8, b = it - kb * nb8;
      const uint32_t ew[8] = {e[u][0].x, e[u][0].y, e[u][0].z, e[u][0].w,
                              e[u][1].x, e[u][1].y, e[u][1].z, e[u][1].w};
      const uint32_t gv[8] = {gw[u][0].x, gw[u][0].y, gw[u][0].z, gw[u][0].w,
                              gw[u][1].x, gw[u][1].y, gw[u][1].z, gw[u][1].w};
      float x[16], y[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        x[2 * i] = bf_lo(ew[i]);
        x[2 * i + 1] = bf_hi(ew[i]);
        y[2 * i] = x[2 * i] * bf_lo(gv[i]);
        y[2 * i + 1] = x[2 * i + 1] * bf_hi(gv[i]);
      }
      float st[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float a0 = x[2 * t], a1 = x[2 * t + 1], a8 = x[2 * t + 8], a9 = x[2 * t + 9];
        st[t] = fmaf(a0, a0, fmaf(a1, a1, fmaf(a8, a8, a9 * a9)));
        const uint16_t h0 = f2bf(y[2 * t]), h1 = f2bf(y[2 * t + 1]);
        const uint16_t h8 = f2bf(y[2 * t + 8]), h9 = f2bf(y[2 * t + 9]);
        uint4 o;
        o.x = (uint32_t)h0 | ((uint32_t)h1 << 16);
        o.y = (uint32_t)h8 | ((uint32_t)h9 << 16);
        o.z = (uint32_t)f2bf(y[2 * t] - bf2f(h0)) | ((uint32_t)f2bf(y[2 * t + 1] - bf2f(h1)) << 16);
        o.w = (uint32_t)f2bf(y[2 * t + 8] - bf2f(h8)) | ((uint32_t)f2bf(y[2 * t + 9] - bf2f(h9)) << 16);
        xa[((size_t)kb * p.nn + (b >> 3)) * 32 + (b & 7) * 4 + t] = o;
      }
      if (b < p.B) {
        // the sum in the order of a quad's two butterfly steps
        L0.ssa[(size_t)b * p.n_parts + kb] = (st[0] + st[1]) + (st[2] + st[3]);
        float4 *dst = reinterpret_cast<float4 *>(p.x0 + (size_t)b * p.H + 16 * kb);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
      }
    }
  }
}

template <bool kMma>
__device__ void embed_task(const Params &p, const int32_t *tok) {
  if (kMma) {
    embed_batch(p, tok);
    return;
  }
  // 8 elements per 16-byte load (H is a multiple of 256: H / 2048 loads
  // per thread)
  const int nch = p.H >> 3;
  for (int b = 0; b < p.B; ++b) {
    const uint4 *e = reinterpret_cast<const uint4 *>(p.embed + (size_t)__ldcg(tok + b) * p.H);
    float4 *dst = reinterpret_cast<float4 *>(p.x0 + (size_t)b * p.H);
    for (int c = threadIdx.x; c < nch; c += kComputeThreads) {
      const uint4 w = __ldg(e + c);
      dst[2 * c] = make_float4(bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y));
      dst[2 * c + 1] = make_float4(bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w));
    }
  }
}

// (value, index) a beats b: larger value, lower index on ties; NaN never
// beats a number (all-NaN partials give the lowest index).
__device__ __forceinline__ bool beats(float av, int ai, float bv, int bi) {
  if (av > bv) return true;
  if (av == bv) return ai < bi;
  return isnan(bv) && (!isnan(av) || ai < bi);
}

// One warp per sequence: lanes scan the LM-head partials (task order), then a
// shuffle reduction with the same total order.
// tok_out: this step's output tokens.
__device__ __noinline__ void argmax_task(const Params &p, int32_t *tok_out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int b = warp; b < p.B; b += kComputeWarps) {
    float bv = NAN;
    int bi = 0x7fffffff;
    for (int j = lane; j < p.n_lm; j += 32) {
      const float v = __ldcg(p.lm_val + (size_t)b * p.n_lm + j);
      const int i = __ldcg(p.lm_idx + (size_t)b * p.n_lm + j);
      if (beats(v, i, bv, bi)) {
        bv = v;
        bi = i;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (beats(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) {
      tok_out[b] = bi;
      p.kv_len[b] = __ldcg(p.kv_len + b) + 1;
    }
  }
}

// ---------------------------------------------------------------------------
// Dispatch mode: a scheduler CTA beside the workers ("Mirage Persistent
// Kernel (MPK)" page, section 5.1: scheduler CTAs hand tasks to the workers).
// One warp polls the events in a window of 32 from the lowest one not yet
// handled; when an event has collected its triggers for this step, its
// dependents [first, last] (a contiguous range of the linearised graph) are
// dealt round-robin to the workers' queues; the tasks without a dependency
// (the linear order's prefix) go out first, and every queue ends with -1.
// The workers run their queue in order without waiting on events.  Every
// wait is bounded; on a timeout or an abort the queues are closed at once.
// ---------------------------------------------------------------------------
__device__ void scheduler_loop(const Params &p, const Smem &sm) {
  const int lane = threadIdx.x & 31;
  const int W = p.n_workers;
  uint32_t *cnt = reinterpret_cast<uint32_t *>(sm.ring);       // [W] entries per queue
  uint32_t *done = cnt + ((W + 31) & ~31);                      // [n_events / 32] handled
  const int nw32 = (p.n_events + 31) >> 5;
  for (int i = lane; i < W; i += 32) cnt[i] = 0u;
  for (int i = lane; i < nw32; i += 32) done[i] = 0u;
  __syncwarp();
  const uint32_t epoch = *(volatile uint32_t *)p.epoch + 1u;
  int rr = 0;  // round-robin cursor over the workers
  // deal tasks [t0, t1) to the queues: task t0 + i to worker (rr + i) % W
  auto deal = [&](int t0, int t1) {
    const int m = t1 - t0;
    for (int i = lane; i < m; i += 32) {
      const int g = rr + i, w = g % W;
      const int g1 = rr + ((w - rr % W) % W + W) % W;  // first slot of this deal for worker w
      const uint32_t pos = cnt[w] + (uint32_t)((g - g1) / W);
      if (pos < (uint32_t)p.q_cap - 1u) p.q_list[(size_t)w * p.q_cap + pos] = t0 + i;
    }
    __threadfence();
    __syncwarp();
    for (int w = lane; w < W; w += 32) {
      // entries of this deal for worker w
      const int first = ((w - rr % W) % W + W) % W;
      const int k = m > first ? (m - first + W - 1) / W : 0;
      if (k > 0) {
        cnt[w] += (uint32_t)k;
        st_release(p.q_tail + w, cnt[w]);
      }
    }
    __syncwarp();
    rr = (rr + m) % W;
  };
  // the roots: the prefix of the linear order without a dependency event
  int n_roots = 0;
  while (n_roots < p.n_tasks && p.tasks[n_roots].dep < 0) ++n_roots;
  deal(0, n_roots);
  int head = 0;  // lowest event not yet handled
  const uint64_t t0 = global_timer();
  uint32_t spins = 0;
  while (head < p.n_events) {
    const int e = head + lane;
    bool ready = false;
    if (e < p.n_events && !((done[e >> 5] >> (e & 31)) & 1u)) {
      const uint32_t target = p.events[e].count * epoch;
      ready = (int32_t)(ld_acquire(p.counters + e) - target) >= 0;
    }
    uint32_t mask = __ballot_sync(0xffffffffu, ready);
    while (mask) {  // in event order
      const int b = __ffs(mask) - 1;
      mask &= mask - 1u;
      const int ev = head + b;
      deal(p.events[ev].first, p.events[ev].last + 1);
      if (lane == 0) done[ev >> 5] |= 1u << (ev & 31);
      __syncwarp();
    }
    while (head < p.n_events && ((done[head >> 5] >> (head & 31)) & 1u)) ++head;
    if (*(volatile int32_t *)p.status != 0) break;
    if (++spins > 16) __nanosleep(64);
    if ((spins & 63u) == 0 && global_timer() - t0 > 4ull * p.timeout_ns + 1000000000ull) {
      if (lane == 0) record_error(p, kDevTimeout, -1, head);
      break;
    }
  }
  // close every queue (an abort closes them where they stand)
  for (int w = lane; w < W; w += 32) {
    const uint32_t pos = cnt[w] < (uint32_t)p.q_cap ? cnt[w] : (uint32_t)p.q_cap - 1u;
    p.q_list[(size_t)w * p.q_cap + pos] = -1;
    __threadfence();
    st_release(p.q_tail + w, pos + 1u);
  }
}

// ---------------------------------------------------------------------------
// The worker kernel
// ---------------------------------------------------------------------------
// kMma: projections on tensor cores (batch >= 2) instead of the CUDA-core
// GEMV; kNN: the operand's 8-column tiles (1 or 2) of the tensor-core
// projections (0 at batch 1); kExt: the extended kernels (JIT attention and
// dispatch mode), kept apart so that their code does not raise the register
// demand of the default kernels.  Each mode is its own instantiation so that
// each gets its own register allocation.
template <bool kMma, int kNN, bool kExt>
__global__ void __launch_bounds__(kThreads, 1) mk_worker_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const Smem sm = carve(smem_raw, p);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;

  Queue q;
  if (kExt && p.dispatch) {
    if ((int)blockIdx.x == p.n_workers) {  // the scheduler CTA
      if (tid < 32) scheduler_loop(p, sm);
      return;
    }
    q.first = 0;
    q.stride = 0;
    q.count = p.q_cap;
    q.list = p.q_list + (size_t)blockIdx.x * p.q_cap;
    q.tail = p.q_tail + blockIdx.x;
  } else if (p.persistent) {
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
      if (L < 0 || L + p.n_steps > p.Lcap || tok < 0 || tok >= p.V) {
        record_error(p, kDevBadInput, -1, b);
        bad = 1;
      }
    }
    sm.ctl[kAbort] = bad;
    sm.ctl[kEpoch] = p.persistent ? (int)(*(volatile uint32_t *)p.epoch + 1u) : 0;
    sm.ctl[kConsumed] = 0;
    sm.ctl[kIssued] = 0;
    sm.ctl[kWindow] = 0;
    sm.tmark[3] = 0;
  }
  __syncthreads();
  if (p.page_size > 0 && !sm.ctl[kAbort]) {
    // every page a sequence touches in this launch must be in the pools
    int badp = 0;
    for (int i = tid; i < p.B * p.max_pages; i += kThreads) {
      const int b = i / p.max_pages, j = i - b * p.max_pages;
      const int rows = min(p.kv_len[b] + p.n_steps, p.Lcap);
      if (j * p.page_size < rows) {
        const int pg = p.page_table[i];
        if (pg < 0 || pg >= p.n_pages) badp = 1;
      }
    }
    if (__syncthreads_or(badp)) {
      if (tid == 0) record_error(p, kDevBadInput, -1, -1);
      return;  // nothing issued yet
    }
  }
  if (sm.ctl[kAbort]) return;  // nothing issued yet
  if (warp == kComputeWarps) {
    if ((tid & 31) == 0) producer_loop<kMma, kExt>(p, sm, q);
    __syncwarp();
  } else {
    const uint32_t epoch0 = (uint32_t)sm.ctl[kEpoch];  // step 0's epoch
    uint32_t k = 0;
    bool run = true;
    for (int s = 0; s < p.n_steps && run; ++s) {
    const uint32_t epoch = epoch0 + (uint32_t)s;
    if (tid == 0) sm.ctl[kLogits] = s == p.n_steps - 1;  // seen after the next barrier
    for (int n = 0; n < q.count; ++n) {
      const int id = queue_task<kExt>(p, sm, q, n);
      if (id < 0) break;
      const DevTask t = p.tasks[id];
      uint64_t t_wait = 0;
      if (p.trace && tid == 0) {
        t_wait = global_timer();
        sm.tmark[0] = sm.tmark[1] = sm.tmark[2] = sm.tmark[4] = 0;  // tmark[3] accumulates
      }
      const DepWait dw{p, sm, t.dep, epoch, id, (int)t.type};
      bool ok = true;
      switch (t.type) {
        case 1:
          ok = dw();
          // step s > 0 reads the tokens step s - 1 wrote: wait until that
          // step's ARGMAX has published its epoch (every task of step s
          // descends from this EMBED)
          if (ok && s > 0) {
            if (tid == 0 && !wait_epoch(p, epoch - 1u, id)) sm.ctl[kAbort] = 1;
            compute_sync();
            ok = !sm.ctl[kAbort];
          }
          if (ok) embed_task<kMma>(p, s == 0 ? p.tokens_in : p.tokens_out + (size_t)(s - 1) * p.B);
          break;
        case 2: case 5: case 6: case 7: case 8: {
          if constexpr (kMma) {
            ok = mma_task<kNN == 2 ? 2 : 1>(p, sm, t, k, id, dw);
          } else {
            const int K = t.type == 5 ? p.qdim : t.type == 7 ? p.F : p.H;
            const int nch = K >> 3;
            const int cpt =
                nch <= kComputeThreads ? 1 : (nch + kComputeThreads - 1) / kComputeThreads;
            const int rps = t.type == 2 ? p.rps_qkv : t.type == 5 ? p.rps_o
                          : t.type == 6 ? p.rps_gu : t.type == 7 ? p.rps_down : p.rps_lm;
            if (cpt == 1 && rps >= 8) ok = gemv_task<1, 8>(p, sm, t, k, id, dw);
            else if (cpt == 2 && rps == 6) ok = gemv_task<2, 6>(p, sm, t, k, id, dw);
            else if (cpt == 2 && rps >= 8) ok = gemv_task<2, 8>(p, sm, t, k, id, dw);
            else if (cpt <= 6 && rps == 2) ok = gemv_task<6, 2>(p, sm, t, k, id, dw);
            else ok = gemv_task<kMaxCpt, 8>(p, sm, t, k, id, dw);
          }
          break;
        }
        case 3:
          if constexpr (kMma) {
            if constexpr (kExt)
              ok = p.D == 128 ? attn_task<128, true>(p, sm, t, k, id, dw)
                              : attn_task<64, true>(p, sm, t, k, id, dw);
            else
              ok = p.D == 128 ? attn_task_fixed<128, true>(p, sm, t, k, id, dw)
                              : attn_task_fixed<64, true>(p, sm, t, k, id, dw);
          } else {
            const int rp = p.rep_p;
            ok = rp <= 2 ? attn_task_cc<2>(p, sm, t, k, id, dw)
               : rp == 4 ? attn_task_cc<4>(p, sm, t, k, id, dw)
                         : attn_task_cc<8>(p, sm, t, k, id, dw);
          }
          break;
        case 9: ok = dw(); if (ok) argmax_task(p, p.tokens_out + (size_t)s * p.B); break;
        default: ok = dw(); break;  // empty task
      }
      if (!ok) {
        run = false;
        break;
      }
      compute_sync();
      if (tid == 0) {
        // bar.sync above orders every compute thread's stores before this
        // release, which is cumulative at gpu scope
        if (p.persistent && t.trig >= 0) red_release_add(p.counters + t.trig, 1u);
        // the step is complete once its ARGMAX has run: publish the epoch
        if (p.persistent && t.type == 9) st_release(p.epoch, epoch);
        if (p.trace) {
          uint32_t smid;
          asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
          unsigned long long *tr = p.trace + 8 * (size_t)id;
          tr[0] = t_wait;
          tr[1] = sm.tmark[2];
          tr[2] = global_timer();
          tr[3] = ((unsigned long long)smid << 32) | blockIdx.x;
          tr[4] = sm.tmark[0];
          tr[5] = sm.tmark[1];
          tr[6] = sm.tmark[3];  // bytes this worker has prefetched into L2 so far
          tr[7] = sm.tmark[4];  // the task's first ring stage was available
        }
      }
    }
    }
    if (tid == 0) sm.ctl[kConsumed] = (int)k;
  }
  __syncthreads();
  if (sm.ctl[kAbort] && warp == kComputeWarps && (tid & 31) == 0) {
    // Copies into this CTA's shared memory must land before it exits.  Only
    // the last ring_stages issued stages can still be in flight (each is the
    // latest use of its slot, so its phase parity is unambiguous).  The wait
    // has the kernel's timeout budget; if it runs out, the status words' event
    // field is set to -2 to say that the CTA exited with copies outstanding.
    const uint32_t to = (uint32_t)sm.ctl[kIssued];
    const uint32_t from = to > (uint32_t)p.ring_stages ? to - (uint32_t)p.ring_stages : 0u;
    const uint64_t budget = 4ull * p.timeout_ns + 1000000000ull;
    const uint64_t t0 = global_timer();
    bool late = false;
    for (uint32_t kk = from; kk < to && !late; ++kk) {
      const int slot = (int)(kk % p.ring_stages);
      const uint32_t par = (kk / p.ring_stages) & 1u;
      while (!mbar_test(&sm.full[slot], par)) {
        if (global_timer() - t0 > budget) {
          late = true;
          break;
        }
      }
    }
    if (late) {
      p.status[2] = -2;
      __threadfence();
    }
  }
}

// Weight layout for the tensor-core path: a row-major [rows][K] bf16 matrix
// to mma.sync A-fragment order.  Item (m-tile mt, k-block kb, lane) holds the
// lane's 8 elements, so stage copies and fragment loads are 16 bytes per lane.
// Rows >= rows (the last m-tile's padding) are zero.
__global__ void frag_permute_kernel(uint4 *dst, const uint32_t *src, int rows, int K,
                                    long long n_items) {
  const long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= n_items) return;
  const int lane = (int)(item & 31);
  const long long blk = item >> 5;
  const int KB = K >> 4;
  const int mt = (int)(blk / KB), kb = (int)(blk - (long long)mt * KB);
  const int r0 = mt * 16 + (lane >> 2), r1 = r0 + 8;
  const int c = kb * 16 + 2 * (lane & 3);  // even: one 32-bit word holds (c, c + 1)
  const size_t w = (size_t)K / 2;
  uint4 o;
  o.x = r0 < rows ? src[(size_t)r0 * w + c / 2] : 0u;
  o.y = r1 < rows ? src[(size_t)r1 * w + c / 2] : 0u;
  o.z = r0 < rows ? src[(size_t)r0 * w + c / 2 + 4] : 0u;
  o.w = r1 < rows ? src[(size_t)r1 * w + c / 2 + 4] : 0u;
  dst[item] = o;
}

}  // namespace

// dst receives ceil(rows / 16) m-tiles of K / 16 fragment blocks (512 bytes each).
cudaError_t permute_to_fragments(void *dst, const void *src, int rows, int K,
                                 cudaStream_t stream) {
  const long long n_items = (long long)((rows + 15) / 16) * (K / 16) * 32;
  if (n_items == 0) return cudaSuccess;
  const int threads = 256;
  const long long blocks = (n_items + threads - 1) / threads;
  frag_permute_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
      static_cast<uint4 *>(dst), static_cast<const uint32_t *>(src), rows, K, n_items);
  return cudaGetLastError();
}

size_t worker_smem_bytes(int stages, int stage_bytes, int pps, int head_dim, int rep_p) {
  return smem_offsets(stages, stage_bytes, pps, head_dim, rep_p).total;
}

// The instantiation for a parameter block's mode.
static const void *worker_fn(const Params &p) {
  const bool ext = p.jit || p.dispatch;
  if (!p.mma)
    return ext ? (const void *)mk_worker_kernel<false, 0, true> : (const void *)mk_worker_kernel<false, 0, false>;
  if (p.nn == 2)
    return ext ? (const void *)mk_worker_kernel<true, 2, true> : (const void *)mk_worker_kernel<true, 2, false>;
  return ext ? (const void *)mk_worker_kernel<true, 1, true> : (const void *)mk_worker_kernel<true, 1, false>;
}

static const void *const kWorkerFns[] = {
    (const void *)mk_worker_kernel<false, 0, false>, (const void *)mk_worker_kernel<true, 1, false>,
    (const void *)mk_worker_kernel<true, 2, false>,  (const void *)mk_worker_kernel<false, 0, true>,
    (const void *)mk_worker_kernel<true, 1, true>,   (const void *)mk_worker_kernel<true, 2, true>};

cudaError_t worker_configure(size_t smem) {
  for (const void *fn : kWorkerFns) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t worker_max_blocks(int *blocks, size_t smem) {
  int lo = 1 << 30;
  for (const void *fn : kWorkerFns) {
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kThreads, smem);
    if (e != cudaSuccess) return e;
    lo = n < lo ? n : lo;
  }
  *blocks = lo;
  return cudaSuccess;
}

// Persistent launch: one cooperative grid of `workers` CTAs.
cudaError_t launch_persistent(const Params &p, int workers, size_t smem, cudaStream_t stream) {
  void *args[] = {const_cast<Params *>(&p)};
  return cudaLaunchCooperativeKernel(worker_fn(p), dim3(workers), dim3(kThreads), args, smem, stream);
}

// Per-operator launch: one CTA per task of the operator.
cudaError_t launch_tasks(const Params &p, int n_ctas, size_t smem, cudaStream_t stream) {
  void *args[] = {const_cast<Params *>(&p)};
  return cudaLaunchKernel(worker_fn(p), dim3(n_ctas), dim3(kThreads), args, smem, stream);
}

}  // namespace mk
