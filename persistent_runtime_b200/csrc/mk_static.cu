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
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

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

struct Layout {
  size_t counters, arrivals, epoch, status, layers, lm_val, lm_idx, x, total;
  std::vector<size_t> qkv, part, att, xm, h;
  // batch >= 2: operands and sums of squares (index n_layers of xa / ssa: the
  // final hidden state)
  std::vector<size_t> xa, ssa, attb, xmb, ssm, hb;
};

Layout layout_of(const mk_model_config &c, const mk::TaskGraph &g) {
  Layout L;
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
  for (int l = 0; l < Ly; ++l) {
    L.qkv.push_back(take(4 * (size_t)B * n_qkv));
    L.part.push_back(S > 1 ? take(4 * (size_t)B * c.n_q_heads * S * (D + 2)) : 0);
    L.att.push_back(take(4 * (size_t)B * qd));
    L.xm.push_back(take(4 * (size_t)B * H));
    L.h.push_back(take(4 * (size_t)B * F));
  }
  if (B > 1) {
    const int Bp = B > 8 ? 16 : 8, n_parts = H / 16;
    for (int l = 0; l <= Ly; ++l) {
      L.xa.push_back(take(4 * (size_t)Bp * H));
      L.ssa.push_back(take(4 * (size_t)B * n_parts));
    }
    for (int l = 0; l < Ly; ++l) {
      L.attb.push_back(take(4 * (size_t)Bp * qd));
      L.xmb.push_back(take(4 * (size_t)Bp * H));
      L.ssm.push_back(take(4 * (size_t)B * n_parts));
      L.hb.push_back(take(4 * (size_t)Bp * F));
    }
  }
  L.total = off;
  return L;
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

  // per-layer pointer table: the handle's weights, the static activations
  std::vector<mk::DevLayer> layers(h->layers);
  float *x = reinterpret_cast<float *>(base + L.x);
  for (int l = 0; l < Ly; ++l) {
    mk::DevLayer &d = layers[l];
    d.qkv = reinterpret_cast<float *>(base + L.qkv[l]);
    d.part = L.part[l] ? reinterpret_cast<float *>(base + L.part[l]) : nullptr;
    d.att = reinterpret_cast<float *>(base + L.att[l]);
    d.xm = reinterpret_cast<float *>(base + L.xm[l]);
    d.h = reinterpret_cast<float *>(base + L.h[l]);
    d.x_in = x + (size_t)l * B * H;
    d.x_out = x + (size_t)(l + 1) * B * H;
    if (B > 1) {
      d.xa = reinterpret_cast<uint16_t *>(base + L.xa[l]);
      d.ssa = reinterpret_cast<float *>(base + L.ssa[l]);
      d.attb = reinterpret_cast<uint16_t *>(base + L.attb[l]);
      d.xmb = reinterpret_cast<uint16_t *>(base + L.xmb[l]);
      d.ssm = reinterpret_cast<float *>(base + L.ssm[l]);
      d.hb = reinterpret_cast<uint16_t *>(base + L.hb[l]);
      d.xa_next = reinterpret_cast<uint16_t *>(base + L.xa[l + 1]);
      d.ssa_next = reinterpret_cast<float *>(base + L.ssa[l + 1]);
    }
  }
  // The region keeps the previous call's contents: counters, arrival counters
  // and the epoch must start at zero (activations are fully rewritten).
  e = cudaMemsetAsync(base + L.counters, 0, L.status - L.counters, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(base + L.layers, layers.data(), sizeof(mk::DevLayer) * Ly,
                        cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) {
    h->err = std::string("static region set-up: ") + cudaGetErrorString(e);
    return MK_ERR_CUDA;
  }
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
    p.xfb = reinterpret_cast<uint16_t *>(base + L.xa[Ly]);
    p.ssf = reinterpret_cast<float *>(base + L.ssa[Ly]);
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
  p.logits = d_logits;
  p.persistent = 1;
  e = mk::launch_persistent(p, h->tune.num_workers, h->smem, st);
  if (e != cudaSuccess) {
    h->err = std::string("persistent launch: ") + cudaGetErrorString(e);
    return MK_ERR_CUDA;
  }
  return MK_OK;
}
