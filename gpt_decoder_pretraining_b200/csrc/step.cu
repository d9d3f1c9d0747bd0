// The training-step orchestrator behind the C ABI: parameter packing, workspace plan, and the
// launch sequence of one forward + backward pass of the nanochat GPT decoder.
//
// Forward, per layer ("nanochat User Guide" §10; "Introducing nanochat", Pretraining):
//   r1 = RMS(x) → qkv = r1·W_qkvᵀ → RoPE + QK-norm (in place) → o = attention(q̃, k̃, v)
//   → x += o·W_oᵀ (residual epilogue) → r2 = RMS(x) → a = relu(r2·W_fcᵀ), h = a² (epilogue)
//   → x += h·W_projᵀ (residual epilogue)
// then x_f = RMS(x) and the fused lm-head + cross-entropy ("supa beginna nanochat",
// Troubleshooting: mean over targets ≠ −1).  The backward pass runs the same chain in reverse with
// an fp32 residual gradient and its bf16 copy as the GEMM operand; every weight gradient is an
// fp32 GEMM output written straight into the caller's gradient buffer.

#include <algorithm>
#include <new>
#include <vector>

#include "common.cuh"
#include "host.h"

namespace gpt {

gpt_status rmsnorm_fwd(const void* x, void* y, float* rho, int rows, int d, cudaStream_t s);
gpt_status rmsnorm_bwd(const void* dy, int dy_f32, const void* y, const float* rho, float* gx,
                       void* gx_bf16, int accumulate, int rows, int d, cudaStream_t s);
gpt_status rope_table(float* cs, int T, int Dh, cudaStream_t s);
gpt_status rope_qknorm_fwd(void* qkv, float* rq, float* rk, const float* cs, int B, int T, int H,
                           int Dh, cudaStream_t s);
gpt_status rope_qknorm_bwd(void* dqkv, const void* qkv, const float* rq, const float* rk,
                           const float* cs, int B, int T, int H, int Dh, cudaStream_t s);
gpt_status rope_qknorm_bwd_heads(void* dqkv, const void* y_heads, const float* rq, const float* rk,
                                 const float* cs, int B, int T, int H, int Dh, cudaStream_t s);
gpt_status embedding_fwd(const int32_t* tok, const void* wte, void* x, int M, int d, int V,
                         int* status, cudaStream_t s);
size_t embedding_bwd_scratch_bytes(int M, int d, int V);
size_t attention_bwd_scratch_bytes(int B, int H, int T, bool store_ds);
gpt_status embedding_bwd(const int32_t* tok, const float* gx, float* dwte, int M, int d, int V,
                         void* scratch, cudaStream_t s);
gpt_status ce_rows(const float2* stats, int ntiles, const float* zt, const int32_t* targets, int M,
                   int V, float* lse, float* ell, int* status, cudaStream_t s);
gpt_status ce_finalize(const float* ell, const int32_t* targets, int M, int V, float* loss,
                       float* inv_n, cudaStream_t s);
gpt_status cast_f32_bf16(const float* src, void* dst, size_t n, cudaStream_t s);
gpt_status add_f32(float* dst, const float* src, size_t n, cudaStream_t s);
gpt_status attention_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int Hkv, int T, int Dh, int window, HeadLayout lq, HeadLayout lkv,
                         HeadLayout lo, int* status, cudaStream_t stream, float* kmax_scratch,
                         int Tk, int q_off);
gpt_status attention_bwd(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, float* delta, void* dq, void* dk,
                         void* dv, int B, int H, int Hkv, int T, int Dh, int window, HeadLayout lq,
                         HeadLayout lkv, HeadLayout ldq, HeadLayout ldkv, HeadLayout lo,
                         HeadLayout ldo, int* status, cudaStream_t stream, const float* rho_q,
                         const float* rho_k, const float* cos_sin, bool store_ds, bool delta_ready);

static inline size_t al256(size_t b) { return (b + 255) & ~(size_t)255; }

// Key/value heads (grouped-query attention; n_kv_heads = 0 means one per query head) and width.
static inline int kv_heads(const gpt_config& c) { return c.n_kv_heads > 0 ? c.n_kv_heads : c.n_heads; }
static inline int kv_dim(const gpt_config& c) { return kv_heads(c) * c.head_dim; }

// ------------------------------------------------------------------------------------------------
// configuration and packing
// ------------------------------------------------------------------------------------------------
static gpt_status validate(const gpt_config* c) {
  if (!c) return GPT_ERR_INVALID_ARG;
  if (c->depth < 0 || c->d_model <= 0 || c->n_heads <= 0 || c->head_dim <= 0 || c->d_mlp <= 0 ||
      c->vocab <= 0 || c->seq_len <= 0 || c->batch <= 0)
    return GPT_ERR_INVALID_ARG;
  if (c->param_dtype != GPT_DTYPE_BF16 && c->param_dtype != GPT_DTYPE_F32) return GPT_ERR_INVALID_ARG;
  if (c->n_heads * c->head_dim != c->d_model) return GPT_ERR_INVALID_ARG;
  if (c->n_kv_heads < 0 || (c->n_kv_heads > 0 && c->n_heads % c->n_kv_heads)) return GPT_ERR_INVALID_ARG;
  // the head_dim-32 attention path handles one query head per key/value head only
  if (c->head_dim == 32 && c->n_kv_heads > 0 && c->n_kv_heads != c->n_heads) return GPT_ERR_UNSUPPORTED_SHAPE;
  if (c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128) return GPT_ERR_UNSUPPORTED_SHAPE;
  if ((c->d_model % 64) || (c->d_mlp % 64) || (c->vocab % 64)) return GPT_ERR_UNSUPPORTED_SHAPE;
  if (c->vocab > 65536) return GPT_ERR_UNSUPPORTED_SHAPE;
  const long long M = (long long)c->batch * c->seq_len;
  if (M > (1ll << 30)) return GPT_ERR_UNSUPPORTED_SHAPE;
  return GPT_OK;
}

struct Layout {
  std::vector<size_t> off;  // 2 + 4·depth
  size_t total = 0;
};

static Layout make_layout(const gpt_config& c) {
  Layout L;
  const size_t d = c.d_model, F = c.d_mlp, V = c.vocab;
  size_t pos = 0;
  L.off.push_back(pos); pos += V * d;
  for (int l = 0; l < c.depth; ++l) {
    L.off.push_back(pos); pos += (d + 2 * kv_dim(c)) * d;
    L.off.push_back(pos); pos += d * d;
    L.off.push_back(pos); pos += F * d;
    L.off.push_back(pos); pos += d * F;
  }
  L.off.push_back(pos); pos += V * d;
  L.total = pos;
  return L;
}

// ------------------------------------------------------------------------------------------------
// workspace plan
// ------------------------------------------------------------------------------------------------
struct Plan {
  size_t status, rope, pshadow;
  size_t x, xf, rhof;
  // per layer (base + l·stride)
  size_t r1, rho1, qkv, rq, rk, lse, o, r2, rho2, hsq, layer_stride;
  // CE
  size_t stats, zt, lse_ce, ell, inv_n, dz, dxf;
  // backward transients
  size_t gx, gxb, gxb2, du, dr, dO, dqkv, delta, emb, sk;
  size_t gacc;  // this micro-batch's gradients when the call accumulates into the caller's
  size_t total;
  int vc;  // vocabulary chunk of the backward lm-head
};

}  // namespace gpt

namespace gpt {
// Optional per-launch CUDA-event timing, by kernel class (see gpt_step_profile).
struct Profiler {
  struct Rec {
    int cls;
    double flops, bytes;
    cudaEvent_t a, b;
  };
  bool on = false;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  std::vector<Rec> recs;
  cudaEvent_t get() {
    if (used < pool.size()) return pool[used++];
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    pool.push_back(e);
    ++used;
    return e;
  }
  ~Profiler() {
    for (cudaEvent_t e : pool) cudaEventDestroy(e);
  }
};
}  // namespace gpt

struct gpt_step {
  gpt_config cfg;
  std::vector<int32_t> window;
  gpt::Layout layout;
  gpt::Plan plan;
  int64_t last_launches = 0;
  gpt::Profiler prof;
  // gradient buckets (W_lm, layers depth−1 .. 0, wte) and the events recorded when each is final
  std::vector<cudaEvent_t> grad_events;
  bool record_in_step = true;  // false while a call accumulates: events follow the final add
  ~gpt_step() {
    for (cudaEvent_t e : grad_events) cudaEventDestroy(e);
  }
};

namespace gpt {

static Plan make_plan(const gpt_config& c, size_t n_params) {
  Plan p{};
  const size_t M = (size_t)c.batch * c.seq_len, d = c.d_model, F = c.d_mlp, V = c.vocab,
               H = c.n_heads;
  size_t pos = 0;
  auto take = [&](size_t bytes) { size_t o = pos; pos += al256(bytes); return o; };
  p.status = take(256);
  p.rope = take((size_t)c.seq_len * c.head_dim * sizeof(float));
  p.pshadow = (c.param_dtype == GPT_DTYPE_F32) ? take(n_params * 2) : 0;
  p.x = take(M * d * 2);
  p.xf = take(M * d * 2);
  p.rhof = take(M * 4);
  // per-layer saved activations
  const size_t layer0 = pos;
  p.r1 = take(M * d * 2) - layer0;
  p.rho1 = take(M * 4) - layer0;
  p.qkv = take(M * (d + 2 * kv_dim(c)) * 2) - layer0;
  p.rq = take(M * H * 4) - layer0;
  p.rk = take(M * kv_heads(c) * 4) - layer0;
  p.lse = take(M * H * 4) - layer0;
  p.o = take(M * d * 2) - layer0;
  p.r2 = take(M * d * 2) - layer0;
  p.rho2 = take(M * 4) - layer0;
  p.hsq = take(M * F * 2) - layer0;
  p.layer_stride = pos - layer0;
  pos = layer0 + p.layer_stride * (size_t)c.depth;
  // make the per-layer offsets absolute for layer 0
  p.r1 += layer0; p.rho1 += layer0; p.qkv += layer0; p.rq += layer0; p.rk += layer0;
  p.lse += layer0; p.o += layer0; p.r2 += layer0; p.rho2 += layer0; p.hsq += layer0;
  // cross-entropy
  const int tiles = (int)((V + gemm_ce_tile_n() - 1) / gemm_ce_tile_n());
  p.stats = take(M * tiles * sizeof(float2));
  p.zt = take(M * 4);
  p.lse_ce = take(M * 4);
  p.ell = take(M * 4);
  p.inv_n = take(256);
  int vc = (int)V;
  while ((size_t)vc * M * 2 > ((size_t)1 << 29) && vc % 128 == 0 && vc > 256) vc /= 2;
  p.vc = vc;
  p.dz = take(M * (size_t)vc * 2);
  p.dxf = take(M * d * 4);
  // backward transients
  p.gx = take(M * d * 4);
  p.gxb = take(M * d * 2);
  p.gxb2 = take(M * d * 2);
  p.du = take(M * F * 2);
  p.dr = take(M * d * 2);
  p.dO = take(M * d * 2);
  p.dqkv = take(M * (d + 2 * kv_dim(c)) * 2);
  p.delta = take(attention_bwd_scratch_bytes(c.batch, H, c.seq_len, true));
  p.emb = take(embedding_bwd_scratch_bytes((int)M, (int)d, (int)V));
  p.sk = take(gemm_sk_scratch_bytes());
  p.gacc = take(n_params * 4);
  p.total = pos;
  return p;
}

// ------------------------------------------------------------------------------------------------
// the step
// ------------------------------------------------------------------------------------------------
// Kernel classes reported by gpt_step_profile.
enum { PROF_GEMM = 0, PROF_ATTN_FWD, PROF_ATTN_BWD, PROF_NORM, PROF_ROPE, PROF_EMBED, PROF_CE, PROF_N };

// Run `expr` (a launcher returning gpt_status); when profiling, bracket it with CUDA events on
// the step's stream and record its class and algorithmic FLOPs / bytes.
#define PROF(cls, fl, by, expr)                                                          \
  do {                                                                                   \
    cudaEvent_t e0_ = nullptr, e1_ = nullptr;                                            \
    if (st->prof.on) {                                                                   \
      e0_ = st->prof.get();                                                              \
      e1_ = st->prof.get();                                                              \
      if (e0_) cudaEventRecord(e0_, s);                                                  \
    }                                                                                    \
    GPT_TRY(expr);                                                                       \
    if (e0_ && e1_) {                                                                    \
      cudaEventRecord(e1_, s);                                                           \
      st->prof.recs.push_back({(cls), (double)(fl), (double)(by), e0_, e1_});            \
    }                                                                                    \
  } while (0)

static double gemm_flops(double M, double N, double K) { return 2.0 * M * N * K; }

// Σ over query rows of the keys each one attends to (causal band of width w).
static double attn_pairs(int T, int w) {
  const double W = (w > 0 && w < T) ? w : T;
  double full = 0;
  // rows t < W see t+1 keys, rows t ≥ W see W keys
  const double a = std::min<double>(W, T);
  full += a * (a + 1) / 2;
  full += (T - a) * W;
  return full;
}

static gpt_status run_step(gpt_step* st, const void* params, const int32_t* tokens,
                           const int32_t* targets, float* loss, float* grads, uint8_t* ws,
                           cudaStream_t s) {
  const gpt_config& c = st->cfg;
  const Plan& p = st->plan;
  const Layout& L = st->layout;
  const int B = c.batch, T = c.seq_len, M = B * T, d = c.d_model, F = c.d_mlp, V = c.vocab,
            H = c.n_heads, Dh = c.head_dim;
  int* status = reinterpret_cast<int*>(ws + p.status);
  float* rope = reinterpret_cast<float*>(ws + p.rope);
  GPT_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int), s));
  // arrival counters of the GEMMs' split tiles: zero here, and every GEMM leaves them at zero
  void* sk = ws + p.sk;
  GPT_CUDA_TRY(cudaMemsetAsync(sk, 0, GEMM_SK_COUNTER_BYTES, s));
  const uint16_t* P = reinterpret_cast<const uint16_t*>(params);
  if (c.param_dtype == GPT_DTYPE_F32) {
    PROF(PROF_CE, 0, 6.0 * L.total, cast_f32_bf16(reinterpret_cast<const float*>(params), ws + p.pshadow, L.total, s));
    P = reinterpret_cast<const uint16_t*>(ws + p.pshadow);
  }
  auto W = [&](int idx) { return P + L.off[idx]; };
  auto G = [&](int idx) { return grads + L.off[idx]; };
  auto at = [&](size_t off, int l) { return ws + off + (size_t)l * p.layer_stride; };
  uint16_t* x = reinterpret_cast<uint16_t*>(ws + p.x);
  uint16_t* xf = reinterpret_cast<uint16_t*>(ws + p.xf);
  float* rhof = reinterpret_cast<float*>(ws + p.rhof);
  const int Hkv = kv_heads(c), dkv = kv_dim(c), nqkv = d + 2 * dkv;  // q | k | v widths
  const long long qs_b = (long long)T * nqkv, qs_h = Dh, qs_t = nqkv;  // dq/dk/dv inside dqkv
  const long long os_b = (long long)T * d, os_h = Dh, os_t = d;          // o (token-major)
  const long long hs_b = (long long)H * T * Dh, hs_h = (long long)T * Dh, hs_t = Dh;  // head-major
  const long long bhtd = (long long)B * H * T * Dh, bhktd = (long long)B * Hkv * T * Dh;
  const HeadLayout lay_q{hs_b, hs_h, hs_t};                            // q̃ head-major
  const HeadLayout lay_kv{(long long)Hkv * T * Dh, hs_h, hs_t};       // k̃, v head-major
  const HeadLayout lay_o{os_b, os_h, os_t};                            // o token-major
  const HeadLayout lay_dqkv{qs_b, qs_h, qs_t};                         // dq, dk, dv in dqkv

  // bucket b of the gradient is final: b = 0 W_lm, 1 + (depth − 1 − l) layer l, depth + 1 wte
  auto bucket_done = [&](int b) -> gpt_status {
    if (!st->grad_events.empty() && st->record_in_step)
      GPT_CUDA_TRY(cudaEventRecord(st->grad_events[b], s));
    return GPT_OK;
  };
  PROF(PROF_ROPE, 0, (double)T * Dh * 4, rope_table(rope, T, Dh, s));
  PROF(PROF_EMBED, 0, 4.0 * (double)M * d, embedding_fwd(tokens, W(0), x, M, d, V, status, s));

  // ---------------- forward ----------------
  for (int l = 0; l < c.depth; ++l) {
    const int wq = 1 + 4 * l;
    uint16_t* r1 = reinterpret_cast<uint16_t*>(at(p.r1, l));
    float* rho1 = reinterpret_cast<float*>(at(p.rho1, l));
    uint16_t* qkv = reinterpret_cast<uint16_t*>(at(p.qkv, l));
    float* rq = reinterpret_cast<float*>(at(p.rq, l));
    float* rk = reinterpret_cast<float*>(at(p.rk, l));
    float* lse = reinterpret_cast<float*>(at(p.lse, l));
    uint16_t* o = reinterpret_cast<uint16_t*>(at(p.o, l));
    uint16_t* r2 = reinterpret_cast<uint16_t*>(at(p.r2, l));
    float* rho2 = reinterpret_cast<float*>(at(p.rho2, l));
    uint16_t* hsq = reinterpret_cast<uint16_t*>(at(p.hsq, l));
    PROF(PROF_NORM, 0, 4.0 * (double)M * d + 4.0 * M, rmsnorm_fwd(x, r1, rho1, M, d, s));
    // q̃ [B][H][T][Dh], k̃ and v [B][Hkv][T][Dh] head-major; RoPE + QK-norm fused into the
    // projection epilogue
    PROF(PROF_GEMM, gemm_flops(M, (double)nqkv, d), 0,
         gemm_qkv_rope_launch(M, d, r1, W(wq), qkv, rq, rk, rope, T, H, Dh, status, s, Hkv));
    PROF(PROF_ATTN_FWD, 4.0 * Dh * H * B * attn_pairs(T, st->window[l]), 0,
         attention_fwd(qkv, qkv + bhtd, qkv + bhtd + bhktd, o, lse, B, H, Hkv, T, Dh,
                       st->window[l], lay_q, lay_kv, lay_o, status, s, nullptr, T, 0));
    PROF(PROF_GEMM, gemm_flops(M, d, d), 0, gemm_launch(GPT_GEMM_NT, GPT_EPI_RESID, M, d, d, o, d, W(wq + 1), d, x, d, nullptr,
                        nullptr, 0, status, s, sk));
    PROF(PROF_NORM, 0, 4.0 * (double)M * d + 4.0 * M, rmsnorm_fwd(x, r2, rho2, M, d, s));
    PROF(PROF_GEMM, gemm_flops(M, F, d), 0, gemm_launch(GPT_GEMM_NT, GPT_EPI_RELU2, M, F, d, r2, d, W(wq + 2), d, hsq, F, nullptr,
                        nullptr, 0, status, s, sk));
    PROF(PROF_GEMM, gemm_flops(M, d, F), 0, gemm_launch(GPT_GEMM_NT, GPT_EPI_RESID, M, d, F, hsq, F, W(wq + 3), F, x, d, nullptr,
                        nullptr, 0, status, s, sk));
  }
  PROF(PROF_NORM, 0, 4.0 * (double)M * d + 4.0 * M, rmsnorm_fwd(x, xf, rhof, M, d, s));

  // ---------------- lm-head + cross-entropy ----------------
  const int wlm = 1 + 4 * c.depth;
  const int tiles = (V + gemm_ce_tile_n() - 1) / gemm_ce_tile_n();
  CeArgs ce{};
  ce.targets = targets;
  ce.lse = reinterpret_cast<float*>(ws + p.lse_ce);
  ce.inv_n = reinterpret_cast<float*>(ws + p.inv_n);
  ce.stats = reinterpret_cast<float2*>(ws + p.stats);
  ce.stats_ld = tiles;
  ce.ztarget = reinterpret_cast<float*>(ws + p.zt);
  ce.n_offset = 0;
  ce.stats_col0 = 0;
  PROF(PROF_GEMM, gemm_flops(M, V, d), 0, gemm_ce_launch(false, M, V, d, xf, d, W(wlm), d, nullptr, 0, ce, status, s));
  PROF(PROF_CE, 0, (double)M * tiles * 8, ce_rows(ce.stats, tiles, ce.ztarget, targets, M, V, const_cast<float*>(ce.lse),
                  reinterpret_cast<float*>(ws + p.ell), status, s));
  PROF(PROF_CE, 0, 8.0 * M, ce_finalize(reinterpret_cast<float*>(ws + p.ell), targets, M, V, loss,
                      const_cast<float*>(ce.inv_n), s));
  uint16_t* dz = reinterpret_cast<uint16_t*>(ws + p.dz);
  float* dxf = reinterpret_cast<float*>(ws + p.dxf);
  for (int c0 = 0; c0 < V; c0 += p.vc) {
    const int n = std::min(p.vc, V - c0);
    ce.n_offset = c0;
    PROF(PROF_GEMM, gemm_flops(M, n, d), 0, gemm_ce_launch(true, M, n, d, xf, d, W(wlm) + (size_t)c0 * d, d, dz, n, ce, status, s));
    PROF(PROF_GEMM, gemm_flops(n, d, M), 0, gemm_launch(GPT_GEMM_TN, GPT_EPI_F32, n, d, M, dz, n, xf, d, G(wlm) + (size_t)c0 * d, d,
                        nullptr, nullptr, 0, status, s, sk));
    PROF(PROF_GEMM, gemm_flops(M, d, n), 0, gemm_launch(GPT_GEMM_NN, c0 == 0 ? GPT_EPI_F32 : GPT_EPI_F32_ADD, M, d, n, dz, n,
                        W(wlm) + (size_t)c0 * d, d, dxf, d, nullptr, nullptr, 0, status, s, sk));
  }
  float* gx = reinterpret_cast<float*>(ws + p.gx);
  uint16_t* gxb = reinterpret_cast<uint16_t*>(ws + p.gxb);
  GPT_TRY(bucket_done(0));
  PROF(PROF_NORM, 0, 12.0 * (double)M * d, rmsnorm_bwd(dxf, 1, xf, rhof, gx, gxb, 0, M, d, s));

  // ---------------- backward ----------------
  uint16_t* du = reinterpret_cast<uint16_t*>(ws + p.du);
  uint16_t* dr = reinterpret_cast<uint16_t*>(ws + p.dr);
  uint16_t* gxb2 = reinterpret_cast<uint16_t*>(ws + p.gxb2);  // bf16 residual gradient at the attention branch
  uint16_t* dO = reinterpret_cast<uint16_t*>(ws + p.dO);
  uint16_t* dqkv = reinterpret_cast<uint16_t*>(ws + p.dqkv);
  float* delta = reinterpret_cast<float*>(ws + p.delta);
  // the delta rows come from the dO GEMM's epilogue when no row of the scratch is padding
  const bool fuse_delta = (T % 64) == 0;
  for (int l = c.depth - 1; l >= 0; --l) {
    const int wq = 1 + 4 * l;
    uint16_t* r1 = reinterpret_cast<uint16_t*>(at(p.r1, l));
    float* rho1 = reinterpret_cast<float*>(at(p.rho1, l));
    uint16_t* qkv = reinterpret_cast<uint16_t*>(at(p.qkv, l));
    float* rq = reinterpret_cast<float*>(at(p.rq, l));
    float* rk = reinterpret_cast<float*>(at(p.rk, l));
    float* lse = reinterpret_cast<float*>(at(p.lse, l));
    uint16_t* o = reinterpret_cast<uint16_t*>(at(p.o, l));
    uint16_t* r2 = reinterpret_cast<uint16_t*>(at(p.r2, l));
    float* rho2 = reinterpret_cast<float*>(at(p.rho2, l));
    uint16_t* hsq = reinterpret_cast<uint16_t*>(at(p.hsq, l));
    // MLP (its weight gradients are formed with the attention ones, below)
    PROF(PROF_GEMM, gemm_flops(M, F, d), 0, gemm_launch(GPT_GEMM_NN, GPT_EPI_DRELU2, M, F, d, gxb, d, W(wq + 3), F, du, F, nullptr,
                        hsq, F, status, s, sk));
    PROF(PROF_GEMM, gemm_flops(M, d, F), 0, gemm_launch(GPT_GEMM_NN, GPT_EPI_BF16, M, d, F, du, F, W(wq + 2), d, dr, d, nullptr,
                        nullptr, 0, status, s, sk));
    PROF(PROF_NORM, 0, 14.0 * (double)M * d, rmsnorm_bwd(dr, 0, r2, rho2, gx, gxb2, 1, M, d, s));
    // attention
    // dO head-major; its epilogue also forms the attention backward's delta rows (T % 64 == 0)
    AttnDeltaFusion fuse{o, os_b, os_t, lse, delta, T};
    PROF(PROF_GEMM, gemm_flops(M, d, d), 0,
         gemm_heads_launch(GPT_GEMM_NN, M, d, d, gxb2, d, W(wq + 1), d, dO, T, H, Dh, status, s,
                           fuse_delta ? &fuse : nullptr));
    PROF(PROF_ATTN_BWD, 8.0 * Dh * H * B * attn_pairs(T, st->window[l]), 0,
         attention_bwd(qkv, qkv + bhtd, qkv + bhtd + bhktd, o, dO, lse, delta, dqkv, dqkv + d,
                       dqkv + d + dkv, B, H, Hkv, T, Dh, st->window[l], lay_q, lay_kv, lay_dqkv,
                       lay_dqkv, lay_o, lay_q, status, s, Dh == 32 ? nullptr : rq, rk, rope,
                       true, fuse_delta));
    if (Dh == 32) {  // the mma.sync path for head_dim 32 has no fused QK-norm/RoPE backward
      PROF(PROF_ROPE, 0, 12.0 * (double)M * d,
           rope_qknorm_bwd_heads(dqkv, qkv, rq, rk, rope, B, T, H, Dh, s));
    }
    // the layer's four weight gradients in one launch: dW_proj = dyᵀ·h, dW_fc = duᵀ·r₂,
    // dW_o = dyᵀ·o, dW_qkv = dqkvᵀ·r₁ (their tiles share whole waves instead of four partly
    // empty last ones)
    {
      const GemmTnProblem wg[4] = {{(int)d, (int)F, gxb, (int)d, hsq, (int)F, G(wq + 3), (int)F},
                                   {(int)F, (int)d, du, (int)F, r2, (int)d, G(wq + 2), (int)d},
                                   {(int)d, (int)d, gxb2, (int)d, o, (int)d, G(wq + 1), (int)d},
                                   {(int)nqkv, (int)d, dqkv, (int)nqkv, r1, (int)d, G(wq), (int)d}};
      PROF(PROF_GEMM, gemm_flops(d, F, M) + gemm_flops(F, d, M) + gemm_flops(d, d, M) + gemm_flops((double)nqkv, d, M), 0,
           gemm_group_tn_launch(4, wg, (int)M, GPT_EPI_F32, status, s, sk));
    }
    GPT_TRY(bucket_done(1 + (c.depth - 1 - l)));
    PROF(PROF_GEMM, gemm_flops(M, d, (double)nqkv), 0, gemm_launch(GPT_GEMM_NN, GPT_EPI_BF16, M, d, nqkv, dqkv, nqkv, W(wq), d, dr, d,
                        nullptr, nullptr, 0, status, s, sk));
    PROF(PROF_NORM, 0, 14.0 * (double)M * d, rmsnorm_bwd(dr, 0, r1, rho1, gx, gxb, 1, M, d, s));
  }
  PROF(PROF_EMBED, 0, 4.0 * (double)M * d + 8.0 * V * d, embedding_bwd(tokens, gx, G(0), M, d, V, ws + p.emb, s));
  GPT_TRY(bucket_done(c.depth + 1));
  return GPT_OK;
}

}  // namespace gpt

// ================================================================================================
// C ABI
// ================================================================================================
extern "C" {

gpt_status gpt_param_layout(const gpt_config* cfg, size_t* offsets, size_t* total) {
  gpt_status v = gpt::validate(cfg);
  if (v != GPT_OK) return v;
  if (!total) return GPT_ERR_INVALID_ARG;
  gpt::Layout L = gpt::make_layout(*cfg);
  if (offsets)
    for (size_t i = 0; i < L.off.size(); ++i) offsets[i] = L.off[i];
  *total = L.total;
  return GPT_OK;
}

gpt_status gpt_step_create(const gpt_config* cfg, gpt_step** out) {
  if (!out) return GPT_ERR_INVALID_ARG;
  *out = nullptr;
  gpt_status v = gpt::validate(cfg);
  if (v != GPT_OK) return v;
  gpt_step* st = new (std::nothrow) gpt_step();
  if (!st) return GPT_ERR_INVALID_ARG;
  st->cfg = *cfg;
  st->window.assign(cfg->depth, 0);
  if (cfg->window)
    for (int l = 0; l < cfg->depth; ++l) st->window[l] = cfg->window[l];
  st->cfg.window = nullptr;  // the copy in st->window is the one used
  st->layout = gpt::make_layout(*cfg);
  st->plan = gpt::make_plan(*cfg, st->layout.total);
  *out = st;
  return GPT_OK;
}

void gpt_step_destroy(gpt_step* step) { delete step; }

int gpt_step_grad_buckets(const gpt_step* step) { return step ? step->cfg.depth + 2 : -1; }

gpt_status gpt_step_grad_bucket(const gpt_step* step, int i, size_t* begin, size_t* end) {
  if (!step || !begin || !end) return GPT_ERR_INVALID_ARG;
  const int L = step->cfg.depth;
  if (i < 0 || i > L + 1) return GPT_ERR_INVALID_ARG;
  const auto& off = step->layout.off;
  const size_t vd = (size_t)step->cfg.vocab * step->cfg.d_model;
  if (i == 0) {
    *begin = off[1 + 4 * (size_t)L];
    *end = *begin + vd;
  } else if (i == L + 1) {
    *begin = 0;
    *end = vd;
  } else {
    const int l = L - i;  // bucket 1 is the last layer
    *begin = off[1 + 4 * (size_t)l];
    *end = off[1 + 4 * (size_t)l + 4];
  }
  return GPT_OK;
}

gpt_status gpt_step_enable_grad_events(gpt_step* step, int enable) {
  if (!step) return GPT_ERR_INVALID_ARG;
  for (cudaEvent_t e : step->grad_events) cudaEventDestroy(e);
  step->grad_events.clear();
  if (!enable) return GPT_OK;
  int sms = 0;
  GPT_TRY(gpt::device_info(&sms));
  for (int i = 0; i < step->cfg.depth + 2; ++i) {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      for (cudaEvent_t x : step->grad_events) cudaEventDestroy(x);
      step->grad_events.clear();
      return GPT_ERR_CUDA;
    }
    step->grad_events.push_back(e);
  }
  return GPT_OK;
}

gpt_status gpt_step_wait_grad_bucket(const gpt_step* step, int i, void* stream) {
  if (!step || i < 0 || i >= (int)step->grad_events.size()) return GPT_ERR_INVALID_ARG;
  GPT_CUDA_TRY(cudaStreamWaitEvent(gpt::as_stream(stream), step->grad_events[i], 0));
  return GPT_OK;
}

gpt_status gpt_step_workspace_bytes(const gpt_step* step, size_t* bytes) {
  if (!step || !bytes) return GPT_ERR_INVALID_ARG;
  *bytes = step->plan.total;
  return GPT_OK;
}

int64_t gpt_step_last_launch_count(const gpt_step* step) { return step ? step->last_launches : -1; }

gpt_status gpt_step_set_profiling(gpt_step* step, int enable) {
  if (!step) return GPT_ERR_INVALID_ARG;
  step->prof.on = enable != 0;
  return GPT_OK;
}

gpt_status gpt_step_profile(gpt_step* step, double* ms, int64_t* calls, double* flops, double* bytes,
                            int n_classes) {
  if (!step || n_classes <= 0) return GPT_ERR_INVALID_ARG;
  for (int c = 0; c < n_classes; ++c) {
    if (ms) ms[c] = 0;
    if (calls) calls[c] = 0;
    if (flops) flops[c] = 0;
    if (bytes) bytes[c] = 0;
  }
  gpt::Profiler& P = step->prof;
  gpt_status r = GPT_OK;
  for (const auto& rec : P.recs) {
    float t = 0.f;
    if (cudaEventSynchronize(rec.b) != cudaSuccess || cudaEventElapsedTime(&t, rec.a, rec.b) != cudaSuccess) {
      r = GPT_ERR_CUDA;
      continue;
    }
    if (rec.cls < n_classes) {
      if (ms) ms[rec.cls] += t;
      if (calls) calls[rec.cls] += 1;
      if (flops) flops[rec.cls] += rec.flops;
      if (bytes) bytes[rec.cls] += rec.bytes;
    }
  }
  P.recs.clear();
  P.used = 0;
  return r;
}

gpt_status gpt_step_fwd_bwd(gpt_step* step, const void* params, const int32_t* tokens,
                            const int32_t* targets, float* loss, float* grads, void* workspace,
                            size_t workspace_bytes, int accumulate, void* stream) {
  if (!step || !params || !tokens || !targets || !loss || !grads || !workspace)
    return GPT_ERR_INVALID_ARG;
  if (accumulate != 0 && accumulate != 1) return GPT_ERR_INVALID_ARG;
  if (workspace_bytes < step->plan.total) return GPT_ERR_WORKSPACE_TOO_SMALL;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) || (reinterpret_cast<uintptr_t>(params) & 15) ||
      (reinterpret_cast<uintptr_t>(grads) & 15))
    return GPT_ERR_UNSUPPORTED_SHAPE;
  int sms = 0;
  gpt_status dv = gpt::device_info(&sms);
  if (dv != GPT_OK) return dv;
  const int64_t before = gpt::g_launch_count;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  // accumulate = 1: the step's gradients go to workspace scratch and are then added to `grads`
  // element by element (one fp32 add per element, so the result does not depend on scheduling)
  float* g = accumulate ? reinterpret_cast<float*>(ws + step->plan.gacc) : grads;
  step->record_in_step = !accumulate;
  gpt_status r = gpt::run_step(step, params, tokens, targets, loss, g, ws, gpt::as_stream(stream));
  if (r == GPT_OK && accumulate)
    r = gpt::add_f32(grads, g, step->layout.total, gpt::as_stream(stream));
  if (r == GPT_OK && accumulate) {
    for (cudaEvent_t e : step->grad_events)
      if (cudaEventRecord(e, gpt::as_stream(stream)) != cudaSuccess) r = GPT_ERR_CUDA;
  }
  step->record_in_step = true;
  step->last_launches = gpt::g_launch_count - before;
  return r;
}

gpt_status gpt_step_status(const gpt_step* step, const void* workspace, void* stream) {
  if (!step || !workspace) return GPT_ERR_INVALID_ARG;
  cudaStream_t s = gpt::as_stream(stream);
  int* dst = reinterpret_cast<int*>(const_cast<void*>(workspace)) + step->plan.status / sizeof(int);
  int host = 0;
  if (cudaMemcpyAsync(&host, dst, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return GPT_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GPT_ERR_CUDA;
  if (host != 0) {
    if (cudaMemsetAsync(dst, 0, sizeof(int), s) != cudaSuccess) return GPT_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GPT_ERR_CUDA;
  }
  return static_cast<gpt_status>(host);
}

size_t gpt_lmhead_ce_scratch_bytes(int M, int d, int V) {
  (void)d;
  const size_t tiles = (size_t)(V + gpt::gemm_ce_tile_n() - 1) / gpt::gemm_ce_tile_n();
  return gpt::al256((size_t)M * tiles * 8) + 4 * gpt::al256((size_t)M * 4) + 256 +
         gpt::al256((size_t)M * V * 2);
}

gpt_status gpt_lmhead_ce_fwd_bwd(const void* xf, const void* wlm, const int32_t* targets, int M,
                                 int d, int V, float* loss, float* lse, float* dx, float* dW,
                                 void* scratch, int* status, void* stream) {
  if (!xf || !wlm || !targets || !loss || !lse || !dx || !dW || !scratch) return GPT_ERR_INVALID_ARG;
  if (M <= 0 || d <= 0 || V <= 0) return GPT_ERR_INVALID_ARG;
  if ((d % 64) || (V % 64)) return GPT_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t s = gpt::as_stream(stream);
  uint8_t* p = reinterpret_cast<uint8_t*>(scratch);
  const int tiles = (V + gpt::gemm_ce_tile_n() - 1) / gpt::gemm_ce_tile_n();
  gpt::CeArgs ce{};
  ce.targets = targets;
  ce.stats = reinterpret_cast<float2*>(p);
  p += gpt::al256((size_t)M * tiles * 8);
  ce.ztarget = reinterpret_cast<float*>(p); p += gpt::al256((size_t)M * 4);
  float* ell = reinterpret_cast<float*>(p); p += gpt::al256((size_t)M * 4);
  p += 2 * gpt::al256((size_t)M * 4);
  ce.inv_n = reinterpret_cast<float*>(p); p += 256;
  uint16_t* dz = reinterpret_cast<uint16_t*>(p);
  ce.lse = lse;
  ce.stats_ld = tiles;
  GPT_TRY(gpt::gemm_ce_launch(false, M, V, d, xf, d, wlm, d, nullptr, 0, ce, status, s));
  GPT_TRY(gpt::ce_rows(ce.stats, tiles, ce.ztarget, targets, M, V, lse, ell, status, s));
  GPT_TRY(gpt::ce_finalize(ell, targets, M, V, loss, const_cast<float*>(ce.inv_n), s));
  GPT_TRY(gpt::gemm_ce_launch(true, M, V, d, xf, d, wlm, d, dz, V, ce, status, s));
  GPT_TRY(gpt::gemm_launch(GPT_GEMM_TN, GPT_EPI_F32, V, d, M, dz, V, xf, d, dW, d, nullptr, nullptr,
                           0, status, s));
  GPT_TRY(gpt::gemm_launch(GPT_GEMM_NN, GPT_EPI_F32, M, d, V, dz, V, wlm, d, dx, d, nullptr,
                           nullptr, 0, status, s));
  return GPT_OK;
}

}  // extern "C"
