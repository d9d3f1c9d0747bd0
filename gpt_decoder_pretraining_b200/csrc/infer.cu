// Forward-only inference with a key/value cache: prefill of a prompt batch and decode of one token
// per sequence ("supa beginna nanochat", notes on each stage: the engine that samples from the
// trained model keeps a KV cache).  The model is the training step's forward pass: the same
// kernels (RMSNorm, the QKV projection with RoPE + QK-norm, tcgen05 attention, the fused-epilogue
// GEMMs), with k̃ and v written straight into the cache by the QKV projection's epilogue and the
// lm-head applied to the last position of each sequence only.
//
// Cache layout (bf16, caller-owned): [depth][2][max_batch][n_kv_heads][max_len][head_dim] — k̃ then
// v of every layer; position t of sequence b is written when that token is processed.  All
// sequences of a call share one length: prefill processes positions 0 .. T−1, decode position
// `pos` and attends to positions 0 .. pos.

#include <algorithm>
#include <new>
#include <vector>

#include "common.cuh"
#include "host.h"

namespace gpt {

gpt_status rmsnorm_fwd(const void* x, void* y, float* rho, int rows, int d, cudaStream_t s);
gpt_status rope_table(float* cs, int T, int Dh, cudaStream_t s);
gpt_status embedding_fwd(const int32_t* tok, const void* wte, void* x, int M, int d, int V,
                         int* status, cudaStream_t s);
gpt_status attention_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int Hkv, int T, int Dh, int window, HeadLayout lq, HeadLayout lkv,
                         HeadLayout lo, int* status, cudaStream_t stream, float* kmax_scratch,
                         int Tk, int q_off);

namespace {

inline size_t al256i(size_t b) { return (b + 255) & ~(size_t)255; }

struct InferPlan {
  size_t status, rope, x, r, rho, q, o, h, lse, xf, sk, total;
};

}  // namespace
}  // namespace gpt

struct gpt_infer {
  gpt_config cfg;
  std::vector<int32_t> window;
  std::vector<size_t> off;  // parameter offsets (gpt_param_layout)
  int max_batch, max_len;
  gpt::InferPlan plan;
};

namespace gpt {
namespace {

int kv_heads_of(const gpt_config& c) { return c.n_kv_heads > 0 ? c.n_kv_heads : c.n_heads; }

InferPlan make_infer_plan(const gpt_config& c, int Bm, int Tm) {
  InferPlan p{};
  const size_t M = (size_t)Bm * Tm, d = c.d_model, F = c.d_mlp;
  size_t pos = 0;
  auto take = [&](size_t bytes) { size_t o = pos; pos += al256i(bytes); return o; };
  p.status = take(256);
  p.rope = take((size_t)Tm * c.head_dim * sizeof(float));
  p.x = take(M * d * 2);
  p.r = take(M * d * 2);
  p.rho = take(M * 4);
  p.q = take(M * d * 2);
  p.o = take(M * d * 2);
  p.h = take(M * F * 2);
  p.lse = take(M * (size_t)c.n_heads * 4);
  p.xf = take(M * d * 2);
  p.sk = take(gemm_sk_scratch_bytes());
  p.total = pos;
  return p;
}

// The forward of `T` new positions per sequence (first position `t0`) for `B` sequences, k̃ and v
// of each layer written into the cache; logits [B, V] of the last new position.
gpt_status infer_forward(gpt_infer* st, const void* params, const int32_t* tokens, int B, int T,
                         int t0, float* logits, void* kv_cache, uint8_t* ws, cudaStream_t s) {
  const gpt_config& c = st->cfg;
  const InferPlan& p = st->plan;
  const int M = B * T, d = c.d_model, F = c.d_mlp, V = c.vocab, H = c.n_heads, Dh = c.head_dim;
  const int Hkv = kv_heads_of(c), Tm = st->max_len, Bm = st->max_batch;
  const uint16_t* P = reinterpret_cast<const uint16_t*>(params);
  auto W = [&](int idx) { return P + st->off[idx]; };
  int* status = reinterpret_cast<int*>(ws + p.status);
  float* rope = reinterpret_cast<float*>(ws + p.rope);
  uint16_t* x = reinterpret_cast<uint16_t*>(ws + p.x);
  uint16_t* r = reinterpret_cast<uint16_t*>(ws + p.r);
  float* rho = reinterpret_cast<float*>(ws + p.rho);
  uint16_t* q = reinterpret_cast<uint16_t*>(ws + p.q);
  uint16_t* o = reinterpret_cast<uint16_t*>(ws + p.o);
  uint16_t* hbuf = reinterpret_cast<uint16_t*>(ws + p.h);
  float* lse = reinterpret_cast<float*>(ws + p.lse);
  uint16_t* xf = reinterpret_cast<uint16_t*>(ws + p.xf);
  void* sk = ws + p.sk;
  GPT_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int), s));
  GPT_CUDA_TRY(cudaMemsetAsync(sk, 0, GEMM_SK_COUNTER_BYTES, s));
  GPT_TRY(rope_table(rope, Tm, Dh, s));
  GPT_TRY(embedding_fwd(tokens, W(0), x, M, d, V, status, s));
  const size_t layer_cache = (size_t)2 * Bm * Hkv * Tm * Dh;  // elements per layer
  const HeadLayout lq{(long long)H * T * Dh, (long long)T * Dh, Dh};
  const HeadLayout lkv{(long long)Hkv * Tm * Dh, (long long)Tm * Dh, Dh};
  const HeadLayout lo{(long long)T * d, Dh, d};
  for (int l = 0; l < c.depth; ++l) {
    const int wq = 1 + 4 * l;
    uint16_t* kc = reinterpret_cast<uint16_t*>(kv_cache) + l * layer_cache;
    uint16_t* vc = kc + (size_t)Bm * Hkv * Tm * Dh;
    GPT_TRY(rmsnorm_fwd(x, r, rho, M, d, s));
    QkvDest dest{q, kc, vc, T, Tm, t0};
    GPT_TRY(gemm_qkv_rope_launch(M, d, r, W(wq), nullptr, nullptr, nullptr, rope, T, H, Dh, status, s,
                                 Hkv, &dest));
    GPT_TRY(attention_fwd(q, kc, vc, o, lse, B, H, Hkv, T, Dh, st->window[l], lq, lkv, lo, status, s,
                          nullptr, t0 + T, t0));
    GPT_TRY(gemm_launch(GPT_GEMM_NT, GPT_EPI_RESID, M, d, d, o, d, W(wq + 1), d, x, d, nullptr, nullptr,
                        0, status, s, sk));
    GPT_TRY(rmsnorm_fwd(x, r, rho, M, d, s));
    GPT_TRY(gemm_launch(GPT_GEMM_NT, GPT_EPI_RELU2, M, F, d, r, d, W(wq + 2), d, hbuf, F, nullptr,
                        nullptr, 0, status, s, sk));
    GPT_TRY(gemm_launch(GPT_GEMM_NT, GPT_EPI_RESID, M, d, F, hbuf, F, W(wq + 3), F, x, d, nullptr,
                        nullptr, 0, status, s, sk));
  }
  GPT_TRY(rmsnorm_fwd(x, xf, rho, M, d, s));
  // lm-head on the last position of every sequence: rows T−1, 2T−1, … (row stride T·d)
  return gemm_launch(GPT_GEMM_NT, GPT_EPI_F32, B, V, d, xf + (size_t)(T - 1) * d, T * d,
                     W(1 + 4 * c.depth), d, logits, V, nullptr, nullptr, 0, status, s, sk);
}

gpt_status check_call(const gpt_infer* st, const void* params, const int32_t* tokens, int B,
                      float* logits, void* kv_cache, void* ws, size_t ws_bytes) {
  if (!st || !params || !tokens || !logits || !kv_cache || !ws) return GPT_ERR_INVALID_ARG;
  if (B <= 0 || B > st->max_batch) return GPT_ERR_INVALID_ARG;
  if (ws_bytes < st->plan.total) return GPT_ERR_WORKSPACE_TOO_SMALL;
  if ((reinterpret_cast<uintptr_t>(ws) & 255) || (reinterpret_cast<uintptr_t>(kv_cache) & 15) ||
      (reinterpret_cast<uintptr_t>(params) & 15) || (reinterpret_cast<uintptr_t>(logits) & 15))
    return GPT_ERR_UNSUPPORTED_SHAPE;
  return GPT_OK;
}

}  // namespace
}  // namespace gpt

extern "C" {

gpt_status gpt_infer_create(const gpt_config* cfg, int max_batch, int max_len, gpt_infer** out) {
  if (!out) return GPT_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg || max_batch <= 0 || max_len <= 0) return GPT_ERR_INVALID_ARG;
  size_t total = 0;
  std::vector<size_t> off(2 + 4 * (size_t)std::max(0, cfg->depth));
  GPT_TRY(gpt_param_layout(cfg, off.data(), &total));
  if (cfg->param_dtype != GPT_DTYPE_BF16) return GPT_ERR_UNSUPPORTED_SHAPE;
  if (cfg->head_dim != 64 && cfg->head_dim != 128) return GPT_ERR_UNSUPPORTED_SHAPE;
  if ((long long)max_batch * max_len > (1ll << 26)) return GPT_ERR_UNSUPPORTED_SHAPE;
  gpt_infer* st = new (std::nothrow) gpt_infer();
  if (!st) return GPT_ERR_INVALID_ARG;
  st->cfg = *cfg;
  st->window.assign(cfg->depth, 0);
  if (cfg->window)
    for (int l = 0; l < cfg->depth; ++l) st->window[l] = cfg->window[l];
  st->cfg.window = nullptr;
  st->off = off;
  st->max_batch = max_batch;
  st->max_len = max_len;
  st->plan = gpt::make_infer_plan(st->cfg, max_batch, max_len);
  *out = st;
  return GPT_OK;
}

void gpt_infer_destroy(gpt_infer* st) { delete st; }

gpt_status gpt_infer_workspace_bytes(const gpt_infer* st, size_t* bytes) {
  if (!st || !bytes) return GPT_ERR_INVALID_ARG;
  *bytes = st->plan.total;
  return GPT_OK;
}

size_t gpt_infer_kv_cache_bytes(const gpt_infer* st) {
  if (!st) return 0;
  const int Hkv = st->cfg.n_kv_heads > 0 ? st->cfg.n_kv_heads : st->cfg.n_heads;
  return (size_t)st->cfg.depth * 2 * st->max_batch * Hkv * st->max_len * st->cfg.head_dim * 2;
}

gpt_status gpt_prefill(gpt_infer* st, const void* params, const int32_t* tokens, int batch, int T,
                       float* logits, void* kv_cache, void* workspace, size_t workspace_bytes,
                       void* stream) {
  GPT_TRY(gpt::check_call(st, params, tokens, batch, logits, kv_cache, workspace, workspace_bytes));
  if (T <= 0 || T > st->max_len) return GPT_ERR_INVALID_ARG;
  int sms = 0;
  GPT_TRY(gpt::device_info(&sms));
  return gpt::infer_forward(st, params, tokens, batch, T, 0, logits, kv_cache,
                            reinterpret_cast<uint8_t*>(workspace), gpt::as_stream(stream));
}

gpt_status gpt_decode(gpt_infer* st, const void* params, const int32_t* tokens, int batch, int pos,
                      float* logits, void* kv_cache, void* workspace, size_t workspace_bytes,
                      void* stream) {
  GPT_TRY(gpt::check_call(st, params, tokens, batch, logits, kv_cache, workspace, workspace_bytes));
  if (pos < 0 || pos >= st->max_len) return GPT_ERR_INVALID_ARG;
  int sms = 0;
  GPT_TRY(gpt::device_info(&sms));
  return gpt::infer_forward(st, params, tokens, batch, 1, pos, logits, kv_cache,
                            reinterpret_cast<uint8_t*>(workspace), gpt::as_stream(stream));
}

gpt_status gpt_infer_status(const gpt_infer* st, const void* workspace, void* stream) {
  if (!st || !workspace) return GPT_ERR_INVALID_ARG;
  cudaStream_t s = gpt::as_stream(stream);
  int* dst = reinterpret_cast<int*>(const_cast<void*>(workspace)) + st->plan.status / sizeof(int);
  int host = 0;
  if (cudaMemcpyAsync(&host, dst, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return GPT_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GPT_ERR_CUDA;
  return static_cast<gpt_status>(host);
}

}  // extern "C"
