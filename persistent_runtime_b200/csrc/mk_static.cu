// mk_decode_step_noalloc: the decode step with its working buffers in a fixed,
// statically allocated device region instead of the handle's own buffers.
//
// Some callers cannot call cudaMalloc at the moment they need another
// stepping context: cudaMalloc may synchronise the whole device and is not
// allowed while a stream is being captured, and some host programs hand out
// all device memory through their own allocator once the model is loaded.
// This entry point allocates nothing: every per-step working buffer (event
// and arrival counters, step epoch, activations, attention partials, LM-head
// partials and the per-layer pointer table) lives in g_step_scratch below,
// a file-scope static array that every GPU loading the library holds until
// the process exits.  The handle's graph tables, weights and status word are
// used as they are; the handle's own working buffers are left untouched.
// Each call issues, on the caller's stream: one memset of the counters, one
// small kernel that writes the per-layer pointer table into the region (from
// the handle's device table and the region's layout, passed by value), and
// the worker launch.  No host buffer is read by a copy.
//
// Batched handles pad the tensor-core operands to 8 or 16 sequence columns.
// The region is not cleared between calls, so the padding columns hold what
// an earlier call left there; they cannot reach the outputs: a column of an
// MMA's result depends only on the same column of its operand, and only the
// batch's columns are ever stored.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <string>

#include "mk_handle.hpp"

namespace {

// Maximum bytes of per-step working memory; a Qwen3-8B-shaped decoder at
// batch 1 (about 14.5 MiB) fits.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_step_scratch[kStaticScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

// Offsets in the region.  Per-layer buffers sit in equal blocks, so layer l's
// buffer is its layer-0 offset plus l times the block size.
struct Layout {
  size_t counters, arrivals, epoch, status, layers, lm_val, lm_idx, x, total;
  // per layer: offsets within layer 0's block, block size
  size_t qkv, part, att, xm, h, lstride;
  // batch >= 2: operand and sum-of-squares blocks; xa / ssa have n_layers + 1
  // entries (the last: the final hidden state, input of the LM head)
  size_t xa, ssa, xstride, attb, xmb, ssm, hb, bstride;
};

Layout layout_of(const mk_model_config &c, const mk::TaskGraph &g) {
  Layout L{};
  const int B = c.batch, H = c.hidden, F = c.ffn, Ly = c.n_layers, D = c.head_dim;
  const int rep = c.n_q_heads / c.n_kv_heads;
  const size_t n_qkv = (size_t)c.n_kv_heads * (rep + 2) * D, qd = (size_t)c.n_q_heads * D;
  const int S = g.tiling.attn_splits, n_lm = g.tiling.n_lm;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = up256(off + bytes);
    return o;
  };
  // the counters, arrival counters and epoch are contiguous: one memset clears them
  L.counters = take(4 * std::max<size_t>(1, g.ev_count.size()));
  L.arrivals = take(4 * (size_t)Ly * B * c.n_kv_heads);
  L.epoch = take(4);
  L.status = take(16);
  L.layers = take(sizeof(mk::DevLayer) * Ly);
  L.lm_val = take(4 * (size_t)B * n_lm);
  L.lm_idx = take(4 * (size_t)B * n_lm);
  L.x = take(4 * (size_t)(Ly + 1) * B * H);
  // one block per layer: qkv, split partials, att, x_mid, h
  {
    size_t o = 0;
    auto sub = [&](size_t bytes) {
      size_t r = o;
      o = up256(o + bytes);
      return r;
    };
    L.qkv = sub(4 * (size_t)B * n_qkv);
    L.part = S > 1 ? sub(4 * (size_t)B * c.n_q_heads * S * (D + 2)) : 0;
    L.att = sub(4 * (size_t)B * qd);
    L.xm = sub(4 * (size_t)B * H);
    L.h = sub(4 * (size_t)B * F);
    L.lstride = o;
    const size_t base = take(o * Ly);
    L.qkv += base; L.att += base; L.xm += base; L.h += base;
    if (S > 1) L.part += base;
  }
  if (B > 1) {
    const int Bp = B > 8 ? 16 : 8, n_parts = H / 16;
    size_t o = 0;
    auto sub = [&](size_t bytes) {
      size_t r = o;
      o = up256(o + bytes);
      return r;
    };
    L.xa = sub(4 * (size_t)Bp * H);
    L.ssa = sub(4 * (size_t)B * n_parts);
    L.xstride = o;
    size_t base = take(o * (Ly + 1));
    L.xa += base; L.ssa += base;
    o = 0;
    L.attb = sub(4 * (size_t)Bp * qd);
    L.xmb = sub(4 * (size_t)Bp * H);
    L.ssm = sub(4 * (size_t)B * n_parts);
    L.hb = sub(4 * (size_t)Bp * F);
    L.bstride = o;
    base = take(o * Ly);
    L.attb += base; L.xmb += base; L.ssm += base; L.hb += base;
  }
  L.total = off;
  return L;
}

// By-value description of the region for the pointer-table kernel.
struct StaticLayers {
  char *base;
  Layout lay;
  int B, H, Ly, has_part, batched;
};

// Layer l's entry of the region's pointer table: the handle's entry (weights
// and gains) with every activation pointer moved into the region.
__global__ void static_layers_kernel(const mk::DevLayer *src, mk::DevLayer *dst, StaticLayers s) {
  const int l = blockIdx.x * blockDim.x + threadIdx.x;
  if (l >= s.Ly) return;
  const Layout &y = s.lay;
  char *b = s.base;
  mk::DevLayer d = src[l];
  const size_t lo = (size_t)l * y.lstride;
  float *x = reinterpret_cast<float *>(b + y.x);
  d.qkv = reinterpret_cast<float *>(b + y.qkv + lo);
  d.part = s.has_part ? reinterpret_cast<float *>(b + y.part + lo) : nullptr;
  d.att = reinterpret_cast<float *>(b + y.att + lo);
  d.xm = reinterpret_cast<float *>(b + y.xm + lo);
  d.h = reinterpret_cast<float *>(b + y.h + lo);
  d.x_in = x + (size_t)l * s.B * s.H;
  d.x_out = x + (size_t)(l + 1) * s.B * s.H;
  if (s.batched) {
    const size_t xo = (size_t)l * y.xstride, bo = (size_t)l * y.bstride;
    d.xa = reinterpret_cast<uint16_t *>(b + y.xa + xo);
    d.ssa = reinterpret_cast<float *>(b + y.ssa + xo);
    d.xa_next = reinterpret_cast<uint16_t *>(b + y.xa + xo + y.xstride);
    d.ssa_next = reinterpret_cast<float *>(b + y.ssa + xo + y.xstride);
    d.attb = reinterpret_cast<uint16_t *>(b + y.attb + bo);
    d.xmb = reinterpret_cast<uint16_t *>(b + y.xmb + bo);
    d.ssm = reinterpret_cast<float *>(b + y.ssm + bo);
    d.hb = reinterpret_cast<uint16_t *>(b + y.hb + bo);
  }
  dst[l] = d;
}

// Device address of g_step_scratch on `device`, looked up once per device
// with that device current.
cudaError_t scratch_address(int device, void **out) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!g_scratch_ptr[device]) {
    int prev = 0;
    cudaError_t e = cudaGetDevice(&prev);
    if (e != cudaSuccess) return e;
    e = cudaSetDevice(device);
    if (e != cudaSuccess) return e;
    void *ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_step_scratch);
    cudaSetDevice(prev);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[device] = ptr;
  }
  *out = g_scratch_ptr[device];
  return cudaSuccess;
}

}  // namespace

extern "C" mk_status mk_decode_step_noalloc(mk_handle *h, const int32_t *d_tokens_in,
                                            int32_t *d_tokens_out, int32_t *d_kv_len,
                                            void *d_k_cache, void *d_v_cache, float *d_logits,
                                            void *stream) {
  if (!h) return MK_ERR_ARG;
  if (h->host_only) {
    h->err = "handle was made by mk_plan_graph";
    return MK_ERR_ARG;
  }
  if (h->base.page_size > 0) {
    h->err = "the handle was built for paged K/V: use mk_decode_steps_paged";
    return MK_ERR_ARG;
  }
  if (h->base.dispatch) {
    h->err = "the handle was built for dispatch mode: use mk_decode_step";
    return MK_ERR_ARG;
  }
  const Layout L = layout_of(h->cfg, h->graph);
  if (L.total > kStaticScratchBytes) {
    h->err = "step working memory of " + std::to_string(L.total) +
             " bytes exceeds the static region of " + std::to_string(kStaticScratchBytes) +
             " bytes";
    return MK_ERR_ARG;
  }
  if (!h->loaded) {
    h->err = "mk_load_weights has not been called";
    return MK_ERR_NOT_LOADED;
  }
  if (!d_tokens_in || !d_tokens_out || !d_kv_len || !d_k_cache || !d_v_cache) {
    h->err = "null buffer";
    return MK_ERR_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(d_k_cache) | reinterpret_cast<uintptr_t>(d_v_cache)) & 15) {
    h->err = "K/V caches must be 16-byte aligned";
    return MK_ERR_ARG;
  }
  void *base_v = nullptr;
  cudaError_t e = scratch_address(h->device, &base_v);
  if (e != cudaSuccess) {
    h->err = std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e);
    return MK_ERR_CUDA;
  }
  e = cudaSetDevice(h->device);
  if (e != cudaSuccess) {
    h->err = std::string("cudaSetDevice: ") + cudaGetErrorString(e);
    return MK_ERR_CUDA;
  }
  char *base = static_cast<char *>(base_v);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const mk_model_config &c = h->cfg;
  const int B = c.batch, H = c.hidden, Ly = c.n_layers;

  float *x = reinterpret_cast<float *>(base + L.x);
  mk::Params p = h->base;
  p.counters = reinterpret_cast<uint32_t *>(base + L.counters);
  p.arrivals = reinterpret_cast<uint32_t *>(base + L.arrivals);
  p.epoch = reinterpret_cast<uint32_t *>(base + L.epoch);
  // device-side failures are reported through the handle's status word, so
  // mk_sync_status / mk_reset apply to this entry point as well
  p.layers = reinterpret_cast<const mk::DevLayer *>(base + L.layers);
  p.x0 = x;
  p.x_final = x + (size_t)Ly * B * H;
  p.lm_val = reinterpret_cast<float *>(base + L.lm_val);
  p.lm_idx = reinterpret_cast<int32_t *>(base + L.lm_idx);
  if (B > 1) {
    p.xfb = reinterpret_cast<uint16_t *>(base + L.xa + (size_t)Ly * L.xstride);
    p.ssf = reinterpret_cast<float *>(base + L.ssa + (size_t)Ly * L.xstride);
  }
  p.trace = nullptr;
  p.tokens_in = d_tokens_in;
  p.tokens_out = d_tokens_out;
  p.kv_len = d_kv_len;
  p.k_cache = static_cast<uint16_t *>(d_k_cache);
  p.v_cache = static_cast<uint16_t *>(d_v_cache);
  const std::string me = p.mma ? mk::encode_kv_maps(h, d_k_cache, d_v_cache, &p) : "";
  if (!me.empty()) {
    h->err = me;
    return MK_ERR_ARG;
  }
  // The region keeps the previous call's contents: counters, arrival counters
  // and the epoch must start at zero (activations are fully rewritten).
  e = cudaMemsetAsync(base + L.counters, 0, L.status - L.counters, st);
  if (e == cudaSuccess) {
    StaticLayers sl{base, L, B, H, Ly, h->graph.tiling.attn_splits > 1, B > 1};
    static_layers_kernel<<<(Ly + 63) / 64, 64, 0, st>>>(
        h->d_layers, reinterpret_cast<mk::DevLayer *>(base + L.layers), sl);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    h->err = std::string("static region set-up: ") + cudaGetErrorString(e);
    return MK_ERR_CUDA;
  }
  p.logits = d_logits;
  p.persistent = 1;
  e = mk::launch_persistent(p, h->tune.num_workers, h->smem, st);
  if (e != cudaSuccess) {
    h->err = std::string("persistent launch: ") + cudaGetErrorString(e);
    return MK_ERR_CUDA;
  }
  return MK_OK;
}
