// CPU oracle for one decode step of a Qwen3-style decoder.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
// cpu_baseline leg of bench.py may load this code.  The GPU library shares no
// code with it: no headers, helpers, tables or constants.
//
// What it computes is the ordinary transformer decode step; MPK changes only
// how the step is scheduled, not what it computes ("Mirage Persistent Kernel
// (MPK)" page, §2.1 and §7.1: the megakernel removes launches and activation
// round trips and still streams every weight once).  The operator list is the
// one the MPK abstract's tensor programs lower (embedding, RMSNorm, QKV
// projection, per-head q/k RMSNorm, RoPE, GQA attention over the KV cache, O
// projection, residual add, gate/up projection, SiLU*mul, down projection,
// final norm, LM head, argmax).
//
// Precision: single thread, fp32 arithmetic, every sum accumulated
// sequentially in index order, compiled with -ffp-contract=off (no fused
// multiply-add).  Weights, gains and cached K/V are bf16 bit patterns.
//
// Readings taken where the pages are silent:
//   * RMSNorm: y_i = g_i * (x_i / sqrt(mean(x^2) + eps)), gain multiplied
//     directly; the same eps for every norm.
//   * q/k norm: one head_dim-sized gain shared by all heads, applied per head
//     before RoPE.
//   * RoPE: rotate-half pairs (i, i + D/2), inv_freq_i = theta^(-2i/D),
//     angle = pos * inv_freq_i with cos/sin taken in double and rounded to
//     float.
//   * GQA: q head h reads kv head floor(h / (Hq / Hkv)).
//   * KV length L: L rows are cached; the new token has position L, its K
//     (normed, roped) and V are rounded to bf16, stored at row L, and the
//     rounded values take part in this step's attention over L + 1 rows.
//   * argmax: lowest index on ties.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

float bf(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

uint16_t to_bf16(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

}  // namespace

extern "C" {

struct OracleCfg {
  int32_t n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab, tied;
  float eps;
  int32_t pad0;
  double theta;
  int32_t batch, kv_capacity;
};

struct OracleLayer {
  const uint16_t *attn_norm, *wq, *wk, *wv, *q_norm, *k_norm, *wo, *mlp_norm, *w_gate,
      *w_up, *w_down;
};

struct OracleWeights {
  const uint16_t *embed, *lm_head, *final_norm;
  const OracleLayer *layers;
};

// RMSNorm of n values with a bf16 gain.
void oracle_rmsnorm(const float *x, const uint16_t *gain, int n, float eps, float *out) {
  float ss = 0.0f;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  float mean = ss / (float)n;
  float r = std::sqrt(mean + eps);
  for (int i = 0; i < n; ++i) out[i] = bf(gain[i]) * (x[i] / r);
}

// y[n] = sum_k W[n][k] * x[k] for a bf16 row-major [N][K] matrix.
void oracle_gemv(const uint16_t *w, int n_rows, int k_cols, const float *x, float *y) {
  for (int n = 0; n < n_rows; ++n) {
    const uint16_t *row = w + (size_t)n * k_cols;
    float acc = 0.0f;
    for (int k = 0; k < k_cols; ++k) acc += bf(row[k]) * x[k];
    y[n] = acc;
  }
}

// Rotary embedding of one head vector in place (rotate-half pairing).
void oracle_rope(float *v, int d, int pos, double theta) {
  int half = d / 2;
  for (int i = 0; i < half; ++i) {
    double inv_freq = std::pow(theta, -(2.0 * i) / (double)d);
    double ang = (double)pos * inv_freq;
    float c = (float)std::cos(ang), s = (float)std::sin(ang);
    float a = v[i], b = v[i + half];
    v[i] = a * c - b * s;
    v[i + half] = b * c + a * s;
  }
}

float oracle_silu(float x) { return x / (1.0f + std::exp(-x)); }

// Decode attention of n_heads query heads against n_pos cached rows of one kv
// head.  q: [n_heads][d] (already normed and roped); k, v: bf16 [n_pos][d].
// out: [n_heads][d].  probs (nullable): [n_heads][n_pos].
void oracle_attention(const float *q, const uint16_t *k, const uint16_t *v, int n_pos,
                      int n_heads, int d, float *out, float *probs) {
  std::vector<float> s(n_pos > 0 ? n_pos : 1);
  float scale_div = std::sqrt((float)d);
  for (int h = 0; h < n_heads; ++h) {
    const float *qh = q + (size_t)h * d;
    float m = -INFINITY;
    for (int j = 0; j < n_pos; ++j) {
      float dot = 0.0f;
      for (int i = 0; i < d; ++i) dot += qh[i] * bf(k[(size_t)j * d + i]);
      s[j] = dot / scale_div;
      if (s[j] > m) m = s[j];
    }
    float l = 0.0f;
    for (int j = 0; j < n_pos; ++j) {
      s[j] = std::exp(s[j] - m);
      l += s[j];
    }
    for (int j = 0; j < n_pos; ++j) s[j] = s[j] / l;
    if (probs)
      for (int j = 0; j < n_pos; ++j) probs[(size_t)h * n_pos + j] = s[j];
    float *oh = out + (size_t)h * d;
    for (int i = 0; i < d; ++i) {
      float acc = 0.0f;
      for (int j = 0; j < n_pos; ++j) acc += s[j] * bf(v[(size_t)j * d + i]);
      oh[i] = acc;
    }
  }
}

// Index of the largest value; lowest index on ties.
int32_t oracle_argmax(const float *v, int n) {
  int32_t best = 0;
  for (int i = 1; i < n; ++i)
    if (v[i] > v[best]) best = i;
  return best;
}

uint16_t oracle_round_bf16(float f) { return to_bf16(f); }

// One decode step.  For every sequence b with seq_mask == NULL or
// seq_mask[b] != 0: reads tokens_in[b], appends K/V at row kv_len[b] of each
// layer's cache, attends over kv_len[b] + 1 rows at RoPE position kv_len[b],
// writes tokens_out[b] and increments kv_len[b].
//
// Caches: bf16 [n_layers][batch][n_kv_heads][kv_capacity][head_dim], updated
// in place.  logits (nullable): fp32 [batch][vocab].  hidden (nullable): fp32
// [batch][hidden], the residual stream after the last layer (pre final norm).
//
// layers_run / vocab_run < 0 mean "all".  Smaller values run only a prefix of
// the layers and of the LM-head rows; that is used for timing samples only and
// then the outputs are not a decode step.
//
// Returns 0, or -1 when a kv_len would exceed kv_capacity or a token is out of
// range (nothing is written in that case).
int oracle_decode_step_ex(const OracleCfg *cfg, const OracleWeights *w,
                          const int32_t *tokens_in, int32_t *tokens_out, int32_t *kv_len,
                          uint16_t *k_cache, uint16_t *v_cache, float *logits, float *hidden,
                          const uint8_t *seq_mask, int layers_run, int vocab_run) {
  const int Ly = cfg->n_layers, H = cfg->hidden, Hq = cfg->n_q_heads, Hkv = cfg->n_kv_heads;
  const int D = cfg->head_dim, F = cfg->ffn, V = cfg->vocab, B = cfg->batch;
  const int Lcap = cfg->kv_capacity, rep = Hq / Hkv;
  const int qd = Hq * D, kvd = Hkv * D;
  if (layers_run < 0 || layers_run > Ly) layers_run = Ly;
  if (vocab_run < 0 || vocab_run > V) vocab_run = V;
  for (int b = 0; b < B; ++b) {
    if (seq_mask && !seq_mask[b]) continue;
    if (kv_len[b] < 0 || kv_len[b] + 1 > Lcap) return -1;
    if (tokens_in[b] < 0 || tokens_in[b] >= V) return -1;
  }
  const uint16_t *lm = cfg->tied ? w->embed : w->lm_head;

  std::vector<float> x(H), xn(H), q(qd), k(kvd), v(kvd), o(qd), y(H), g(F), u(F), hh(F);
  std::vector<float> tmp(D), lg(V);
  std::vector<uint16_t> krow(D), vrow(D);
  for (int b = 0; b < B; ++b) {
    if (seq_mask && !seq_mask[b]) continue;
    const int pos = kv_len[b];
    const uint16_t *e = w->embed + (size_t)tokens_in[b] * H;
    for (int i = 0; i < H; ++i) x[i] = bf(e[i]);

    for (int l = 0; l < layers_run; ++l) {
      const OracleLayer &L = w->layers[l];
      oracle_rmsnorm(x.data(), L.attn_norm, H, cfg->eps, xn.data());
      oracle_gemv(L.wq, qd, H, xn.data(), q.data());
      oracle_gemv(L.wk, kvd, H, xn.data(), k.data());
      oracle_gemv(L.wv, kvd, H, xn.data(), v.data());
      for (int h = 0; h < Hq; ++h) {
        oracle_rmsnorm(&q[(size_t)h * D], L.q_norm, D, cfg->eps, tmp.data());
        std::memcpy(&q[(size_t)h * D], tmp.data(), sizeof(float) * D);
        oracle_rope(&q[(size_t)h * D], D, pos, cfg->theta);
      }
      for (int gi = 0; gi < Hkv; ++gi) {
        oracle_rmsnorm(&k[(size_t)gi * D], L.k_norm, D, cfg->eps, tmp.data());
        std::memcpy(&k[(size_t)gi * D], tmp.data(), sizeof(float) * D);
        oracle_rope(&k[(size_t)gi * D], D, pos, cfg->theta);
      }
      for (int gi = 0; gi < Hkv; ++gi) {
        size_t slab = (((size_t)l * B + b) * Hkv + gi) * (size_t)Lcap * D;
        uint16_t *kc = k_cache + slab;
        uint16_t *vc = v_cache + slab;
        for (int i = 0; i < D; ++i) {
          kc[(size_t)pos * D + i] = to_bf16(k[(size_t)gi * D + i]);
          vc[(size_t)pos * D + i] = to_bf16(v[(size_t)gi * D + i]);
        }
        oracle_attention(&q[(size_t)gi * rep * D], kc, vc, pos + 1, rep, D,
                         &o[(size_t)gi * rep * D], nullptr);
      }
      oracle_gemv(L.wo, H, qd, o.data(), y.data());
      for (int i = 0; i < H; ++i) x[i] = x[i] + y[i];

      oracle_rmsnorm(x.data(), L.mlp_norm, H, cfg->eps, xn.data());
      oracle_gemv(L.w_gate, F, H, xn.data(), g.data());
      oracle_gemv(L.w_up, F, H, xn.data(), u.data());
      for (int i = 0; i < F; ++i) hh[i] = oracle_silu(g[i]) * u[i];
      oracle_gemv(L.w_down, H, F, hh.data(), y.data());
      for (int i = 0; i < H; ++i) x[i] = x[i] + y[i];
    }
    if (hidden) std::memcpy(hidden + (size_t)b * H, x.data(), sizeof(float) * H);
    oracle_rmsnorm(x.data(), w->final_norm, H, cfg->eps, xn.data());
    oracle_gemv(lm, vocab_run, H, xn.data(), lg.data());
    if (logits) std::memcpy(logits + (size_t)b * V, lg.data(), sizeof(float) * vocab_run);
    tokens_out[b] = oracle_argmax(lg.data(), vocab_run);
  }
  for (int b = 0; b < B; ++b) {
    if (seq_mask && !seq_mask[b]) continue;
    kv_len[b] += 1;
  }
  return 0;
}

int oracle_decode_step(const OracleCfg *cfg, const OracleWeights *w, const int32_t *tokens_in,
                       int32_t *tokens_out, int32_t *kv_len, uint16_t *k_cache,
                       uint16_t *v_cache, float *logits, float *hidden,
                       const uint8_t *seq_mask) {
  return oracle_decode_step_ex(cfg, w, tokens_in, tokens_out, kv_len, k_cache, v_cache, logits,
                               hidden, seq_mask, -1, -1);
}

}  // extern "C"
