// The optimizer step that follows the training step: Muon for the block matrices, AdamW for the
// embedding and the lm-head ("Introducing nanochat", Pretraining log: Muon groups the matrices by
// shape; the AdamW learning rates are scaled by 1/√(d/768)).
//
// Muon, per matrix W with gradient g and momentum buffer b (the published method, every
// hyperparameter an argument):
//   b ← μ·b + g;  u = g + μ·b (Nesterov) or b;  X = u / (‖u‖_F + 1e-7)
//   ns_steps times:  A = X·Xᵀ;  X ← a·X + (b_ns·A + c_ns·A·A)·X     (a tall matrix is iterated as
//                                                                   its transpose)
//   W ← W − lr·√max(1, rows/cols)·X
// The matrices of one shape are processed together: the momentum / normalisation / update passes
// are elementwise kernels over all of them, and each Newton–Schulz product is one batched tcgen05
// GEMM over the whole group (bf16 operands, fp32 accumulation, bf16 result with the a·X and
// b_ns·A terms folded into the epilogue), so an iteration is three launches for the group.
// A tall matrix U (rows > cols) is kept in its own layout: A = UᵀU is a TN product and the update
// U·B an NN product, which is the transposed iteration without any transposed copy.
//
// AdamW (decoupled weight decay), elementwise over fp32 master weights:
//   m ← β1·m + (1−β1)·g;  v ← β2·v + (1−β2)·g²;  m̂ = m/(1−β1^t);  v̂ = v/(1−β2^t)
//   W ← W·(1 − lr·wd) − lr·m̂/(√v̂ + ε)
// Both write the new weights to the fp32 master copy and, when given, to the parameter buffer the
// training step reads (rounded to bf16, or copied for fp32 parameters).

#include <algorithm>
#include <cmath>
#include <vector>

#include "common.cuh"
#include "host.h"

namespace gpt {

namespace {

constexpr int OPT_THREADS = 256;
constexpr int MUON_CHUNK = 8192;  // elements of one matrix per block in the elementwise passes

// Offset of element e of matrix i when matrices come in `groups` groups of `per` contiguous
// matrices of `mat` elements, consecutive groups `gstride` elements apart.
__device__ __forceinline__ long long mat_off(int i, int per, long long gstride, long long mat) {
  return (long long)(i / per) * gstride + (long long)(i % per) * mat;
}

template <bool BF16>
__device__ __forceinline__ void store_param(void* p, long long idx, float w) {
  if (BF16) reinterpret_cast<uint16_t*>(p)[idx] = f2bf(w);
  else reinterpret_cast<float*>(p)[idx] = w;
}

// ---------------------------------------------------------------------------------------------
// AdamW
// ---------------------------------------------------------------------------------------------
template <int PDT>  // 0: no parameter copy, 1: bf16 copy, 2: fp32 copy
__global__ void __launch_bounds__(OPT_THREADS) adamw_kernel(float* __restrict__ w, void* __restrict__ p,
                                                            const float* __restrict__ g,
                                                            float* __restrict__ m, float* __restrict__ v,
                                                            long long n, float lr, float b1, float b2,
                                                            float eps, float decay, float inv_bc1,
                                                            float inv_bc2) {
  const long long n4 = n / 4;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 gw = reinterpret_cast<const float4*>(g)[i];
    float4 mw = reinterpret_cast<float4*>(m)[i];
    float4 vw = reinterpret_cast<float4*>(v)[i];
    float4 ww = reinterpret_cast<float4*>(w)[i];
    float gg[4] = {gw.x, gw.y, gw.z, gw.w}, mm[4] = {mw.x, mw.y, mw.z, mw.w};
    float vv[4] = {vw.x, vw.y, vw.z, vw.w}, wv[4] = {ww.x, ww.y, ww.z, ww.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      mm[e] = b1 * mm[e] + (1.f - b1) * gg[e];
      vv[e] = b2 * vv[e] + (1.f - b2) * gg[e] * gg[e];
      const float mh = mm[e] * inv_bc1, vh = vv[e] * inv_bc2;
      wv[e] = wv[e] * decay - lr * mh / (sqrtf(vh) + eps);
    }
    reinterpret_cast<float4*>(m)[i] = make_float4(mm[0], mm[1], mm[2], mm[3]);
    reinterpret_cast<float4*>(v)[i] = make_float4(vv[0], vv[1], vv[2], vv[3]);
    reinterpret_cast<float4*>(w)[i] = make_float4(wv[0], wv[1], wv[2], wv[3]);
    if (PDT == 1) {
      reinterpret_cast<uint2*>(p)[i] = make_uint2(pack_bf2(wv[0], wv[1]), pack_bf2(wv[2], wv[3]));
    } else if (PDT == 2) {
      reinterpret_cast<float4*>(p)[i] = make_float4(wv[0], wv[1], wv[2], wv[3]);
    }
  }
  // tail (n not a multiple of 4)
  for (long long i = 4 * n4 + (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const float gg = g[i];
    const float mm = b1 * m[i] + (1.f - b1) * gg;
    const float vv = b2 * v[i] + (1.f - b2) * gg * gg;
    const float wv = w[i] * decay - lr * (mm * inv_bc1) / (sqrtf(vv * inv_bc2) + eps);
    m[i] = mm;
    v[i] = vv;
    w[i] = wv;
    if (PDT == 1) store_param<true>(p, i, wv);
    if (PDT == 2) store_param<false>(p, i, wv);
  }
}

// ---------------------------------------------------------------------------------------------
// Muon elementwise passes
// ---------------------------------------------------------------------------------------------
// Fixed-order block sum of one float per thread (deterministic).
__device__ __forceinline__ float block_sum(float x, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = x;
  __syncthreads();
  float t = 0.f;
  if (threadIdx.x == 0) {
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
  }
  __syncthreads();
  return t;  // valid in thread 0
}

// b ← μ·b + g and the partial Σu² of this block's chunk of matrix blockIdx.y, u = g + μ·b
// (Nesterov) or b.  partial: [nb][gridDim.x].
__global__ void __launch_bounds__(OPT_THREADS) muon_momentum_kernel(const float* __restrict__ g,
                                                                    float* __restrict__ buf, int per,
                                                                    long long gstride, long long mat,
                                                                    float mu, int nesterov,
                                                                    float* __restrict__ partial) {
  __shared__ float red[OPT_THREADS / 32];
  const int i = blockIdx.y;
  const long long base = mat_off(i, per, gstride, mat);
  const long long e0 = (long long)blockIdx.x * MUON_CHUNK;
  const long long e1 = min(mat, e0 + MUON_CHUNK);
  float ss = 0.f;
  for (long long e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const float gg = g[base + e];
    const float bb = mu * buf[base + e] + gg;
    buf[base + e] = bb;
    const float u = nesterov ? gg + mu * bb : bb;
    ss += u * u;
  }
  const float t = block_sum(ss, red);
  if (threadIdx.x == 0) partial[(long long)i * gridDim.x + blockIdx.x] = t;
}

// X = bf16(u / (‖u‖_F + 1e-7)) into x [nb][mat] (contiguous), ‖u‖² summed from the partials in
// block order.
__global__ void __launch_bounds__(OPT_THREADS) muon_normalize_kernel(const float* __restrict__ g,
                                                                     const float* __restrict__ buf,
                                                                     int per, long long gstride,
                                                                     long long mat, float mu,
                                                                     int nesterov,
                                                                     const float* __restrict__ partial,
                                                                     uint16_t* __restrict__ x) {
  __shared__ float s_inv;
  const int i = blockIdx.y;
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int j = 0; j < (int)gridDim.x; ++j) t += partial[(long long)i * gridDim.x + j];
    s_inv = 1.f / (sqrtf(t) + 1e-7f);
  }
  __syncthreads();
  const float inv = s_inv;
  const long long base = mat_off(i, per, gstride, mat);
  const long long e0 = (long long)blockIdx.x * MUON_CHUNK;
  const long long e1 = min(mat, e0 + MUON_CHUNK);
  uint16_t* xi = x + (long long)i * mat;
  for (long long e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const float gg = g[base + e];
    const float bb = buf[base + e];
    const float u = nesterov ? gg + mu * bb : bb;
    xi[e] = f2bf(u * inv);
  }
}

// W ← W − step·X, and the parameter copy.
template <int PDT>
__global__ void __launch_bounds__(OPT_THREADS) muon_apply_kernel(float* __restrict__ w, void* __restrict__ p,
                                                                 int per, long long gstride,
                                                                 long long mat,
                                                                 const uint16_t* __restrict__ x,
                                                                 float step) {
  const int i = blockIdx.y;
  const long long base = mat_off(i, per, gstride, mat);
  const long long e0 = (long long)blockIdx.x * MUON_CHUNK;
  const long long e1 = min(mat, e0 + MUON_CHUNK);
  const uint16_t* xi = x + (long long)i * mat;
  for (long long e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const float wv = w[base + e] - step * bf2f(xi[e]);
    w[base + e] = wv;
    if (PDT == 1) store_param<true>(p, base + e, wv);
    if (PDT == 2) store_param<false>(p, base + e, wv);
  }
}

struct MuonScratch {
  uint16_t *x0, *x1, *gm, *bm;
  float* partial;
};

size_t muon_scratch_layout(int nb, int rows, int cols, uint8_t* base, MuonScratch* out) {
  const long long mat = (long long)rows * cols;
  const long long r = std::min(rows, cols);
  const int blocks = (int)((mat + MUON_CHUNK - 1) / MUON_CHUNK);
  size_t pos = 0;
  auto take = [&](size_t bytes) {
    const size_t o = pos;
    pos += (bytes + 255) & ~(size_t)255;
    return o;
  };
  const size_t ox0 = take((size_t)nb * mat * 2), ox1 = take((size_t)nb * mat * 2);
  const size_t og = take((size_t)nb * r * r * 2), ob = take((size_t)nb * r * r * 2);
  const size_t op = take((size_t)nb * blocks * 4);
  if (out && base) {
    out->x0 = reinterpret_cast<uint16_t*>(base + ox0);
    out->x1 = reinterpret_cast<uint16_t*>(base + ox1);
    out->gm = reinterpret_cast<uint16_t*>(base + og);
    out->bm = reinterpret_cast<uint16_t*>(base + ob);
    out->partial = reinterpret_cast<float*>(base + op);
  }
  return pos;
}

int grid_for(long long n4) {
  int sms = 148;
  device_info(&sms);
  const long long want = (n4 + OPT_THREADS - 1) / OPT_THREADS;
  return (int)std::max<long long>(1, std::min<long long>(want, (long long)sms * 8));
}

}  // namespace

size_t muon_scratch_bytes(int nb, int rows, int cols) {
  if (nb <= 0 || rows <= 0 || cols <= 0) return 0;
  return muon_scratch_layout(nb, rows, cols, nullptr, nullptr);
}

gpt_status muon_step(float* w, void* params, int param_dtype, const float* g, float* buf, int groups,
                     int per, long long gstride, int rows, int cols, float lr, float mu, int nesterov,
                     int ns_steps, float na, float nb_, float nc, void* scratch, size_t scratch_bytes,
                     int* status, cudaStream_t s) {
  if (!w || !g || !buf || !scratch) return GPT_ERR_INVALID_ARG;
  if (groups <= 0 || per <= 0 || rows <= 0 || cols <= 0 || ns_steps < 0) return GPT_ERR_INVALID_ARG;
  if (param_dtype != GPT_DTYPE_BF16 && param_dtype != GPT_DTYPE_F32) return GPT_ERR_INVALID_ARG;
  const long long mat = (long long)rows * cols;
  if (groups > 1 && gstride < per * mat) return GPT_ERR_INVALID_ARG;  // groups must not overlap
  if ((rows % 8) || (cols % 8)) return GPT_ERR_UNSUPPORTED_SHAPE;  // 16-byte rows for TMA
  const int nb = groups * per;
  if (scratch_bytes < muon_scratch_bytes(nb, rows, cols)) return GPT_ERR_WORKSPACE_TOO_SMALL;
  if (reinterpret_cast<uintptr_t>(scratch) & 255) return GPT_ERR_UNSUPPORTED_SHAPE;
  int sms = 0;
  GPT_TRY(device_info(&sms));
  MuonScratch sc;
  muon_scratch_layout(nb, rows, cols, reinterpret_cast<uint8_t*>(scratch), &sc);
  const int blocks = (int)((mat + MUON_CHUNK - 1) / MUON_CHUNK);
  const dim3 grid(blocks, nb);
  muon_momentum_kernel<<<grid, OPT_THREADS, 0, s>>>(g, buf, per, gstride, mat, mu, nesterov, sc.partial);
  count_launch();
  GPT_CUDA_TRY(cudaGetLastError());
  muon_normalize_kernel<<<grid, OPT_THREADS, 0, s>>>(g, buf, per, gstride, mat, mu, nesterov,
                                                     sc.partial, sc.x0);
  count_launch();
  GPT_CUDA_TRY(cudaGetLastError());
  // Newton–Schulz on the group: three batched GEMMs per step
  const bool tall = rows > cols;
  const int r = std::min(rows, cols);
  uint16_t* x = sc.x0;
  uint16_t* xn = sc.x1;
  for (int it = 0; it < ns_steps; ++it) {
    GemmBatch gA{};  // A = X·Xᵀ (wide) or UᵀU (tall): [r, r]
    gA.op = tall ? GPT_GEMM_TN : GPT_GEMM_NT;
    gA.epi = GPT_EPI_BF16;
    gA.M = r; gA.N = r; gA.K = tall ? rows : cols; gA.batch = nb;
    gA.A = x; gA.lda = cols; gA.a_bstride = mat;
    gA.B = x; gA.ldb = cols; gA.b_bstride = mat;
    gA.C = sc.gm; gA.ldc = r; gA.c_bstride = (long long)r * r;
    gA.alpha = 1.f; gA.beta = 0.f; gA.status = status;
    GPT_TRY(gemm_launch_batched(gA, s, nullptr));
    GemmBatch gB{};  // B = b_ns·A + c_ns·A·A (A symmetric, so A·A = A·Aᵀ)
    gB.op = GPT_GEMM_NT;
    gB.epi = GPT_EPI_AXPBY;
    gB.M = r; gB.N = r; gB.K = r; gB.batch = nb;
    gB.A = sc.gm; gB.lda = r; gB.a_bstride = (long long)r * r;
    gB.B = sc.gm; gB.ldb = r; gB.b_bstride = (long long)r * r;
    gB.C = sc.bm; gB.ldc = r; gB.c_bstride = (long long)r * r;
    gB.aux = sc.gm; gB.ldaux = r; gB.aux_bstride = (long long)r * r;
    gB.alpha = nc; gB.beta = nb_; gB.status = status;
    GPT_TRY(gemm_launch_batched(gB, s, nullptr));
    GemmBatch gX{};  // X ← a·X + B·X (wide) or U ← a·U + U·B (tall)
    gX.op = GPT_GEMM_NN;
    gX.epi = GPT_EPI_AXPBY;
    gX.M = rows; gX.N = cols; gX.K = r; gX.batch = nb;
    if (!tall) {
      gX.A = sc.bm; gX.lda = r; gX.a_bstride = (long long)r * r;
      gX.B = x; gX.ldb = cols; gX.b_bstride = mat;
    } else {
      gX.A = x; gX.lda = cols; gX.a_bstride = mat;
      gX.B = sc.bm; gX.ldb = r; gX.b_bstride = (long long)r * r;
    }
    gX.C = xn; gX.ldc = cols; gX.c_bstride = mat;
    gX.aux = x; gX.ldaux = cols; gX.aux_bstride = mat;
    gX.alpha = 1.f; gX.beta = na; gX.status = status;
    GPT_TRY(gemm_launch_batched(gX, s, nullptr));
    std::swap(x, xn);
  }
  const float step = lr * std::sqrt(std::max(1.f, (float)rows / (float)cols));
  if (!params || params == w) {
    muon_apply_kernel<0><<<grid, OPT_THREADS, 0, s>>>(w, nullptr, per, gstride, mat, x, step);
  } else if (param_dtype == GPT_DTYPE_BF16) {
    muon_apply_kernel<1><<<grid, OPT_THREADS, 0, s>>>(w, params, per, gstride, mat, x, step);
  } else {
    muon_apply_kernel<2><<<grid, OPT_THREADS, 0, s>>>(w, params, per, gstride, mat, x, step);
  }
  count_launch();
  GPT_CUDA_TRY(cudaGetLastError());
  return GPT_OK;
}

gpt_status adamw_step(float* w, void* params, int param_dtype, const float* g, float* m, float* v,
                      long long n, int t, float lr, float beta1, float beta2, float eps, float wd,
                      cudaStream_t s) {
  if (!w || !g || !m || !v || n <= 0 || t < 1) return GPT_ERR_INVALID_ARG;
  if (param_dtype != GPT_DTYPE_BF16 && param_dtype != GPT_DTYPE_F32) return GPT_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(g) |
       reinterpret_cast<uintptr_t>(m) | reinterpret_cast<uintptr_t>(v)) & 15)
    return GPT_ERR_UNSUPPORTED_SHAPE;
  if (params && params != w && (reinterpret_cast<uintptr_t>(params) & 15)) return GPT_ERR_UNSUPPORTED_SHAPE;
  int sms = 0;
  GPT_TRY(device_info(&sms));
  // bias corrections in double on the host
  const float inv_bc1 = (float)(1.0 / (1.0 - std::pow((double)beta1, (double)t)));
  const float inv_bc2 = (float)(1.0 / (1.0 - std::pow((double)beta2, (double)t)));
  const float decay = 1.f - lr * wd;
  const int grid = grid_for(std::max<long long>(1, n / 4));
  if (!params || params == w) {
    adamw_kernel<0><<<grid, OPT_THREADS, 0, s>>>(w, nullptr, g, m, v, n, lr, beta1, beta2, eps, decay,
                                                 inv_bc1, inv_bc2);
  } else if (param_dtype == GPT_DTYPE_BF16) {
    adamw_kernel<1><<<grid, OPT_THREADS, 0, s>>>(w, params, g, m, v, n, lr, beta1, beta2, eps, decay,
                                                 inv_bc1, inv_bc2);
  } else {
    adamw_kernel<2><<<grid, OPT_THREADS, 0, s>>>(w, params, g, m, v, n, lr, beta1, beta2, eps, decay,
                                                 inv_bc1, inv_bc2);
  }
  count_launch();
  GPT_CUDA_TRY(cudaGetLastError());
  return GPT_OK;
}

}  // namespace gpt

// =================================================================================================
// C ABI
// =================================================================================================
namespace {

struct MuonGroup {
  size_t off;
  int groups, per;
  long long gstride;
  int rows, cols;
};

// The pages' grouping: per layer the q, k, v row blocks of W_qkv and W_o (four d×d matrices, each
// layer's four contiguous), then every W_fc (F×d), then every W_proj (d×F).  With grouped
// key/value heads, k and v are (n_kv_heads·Dh)×d: q, the k/v pair and W_o form three groups.
std::vector<MuonGroup> muon_groups(const gpt_config* cfg, const size_t* off) {
  std::vector<MuonGroup> out;
  const int L = cfg->depth;
  if (L <= 0) return out;
  const long long stride = L > 1 ? (long long)(off[1 + 4] - off[1]) : 0;
  const int d = cfg->d_model, F = cfg->d_mlp;
  const int kv = (cfg->n_kv_heads > 0 ? cfg->n_kv_heads : cfg->n_heads) * cfg->head_dim;
  if (kv == d) {
    out.push_back({off[1], L, 4, stride, d, d});
  } else {
    out.push_back({off[1], L, 1, stride, d, d});
    out.push_back({off[1] + (size_t)d * d, L, 2, stride, kv, d});
    out.push_back({off[1 + 1], L, 1, stride, d, d});
  }
  out.push_back({off[1 + 2], L, 1, stride, F, d});
  out.push_back({off[1 + 3], L, 1, stride, d, F});
  return out;
}

}  // namespace

extern "C" {

gpt_status gpt_adamw_step(float* master, void* params, int param_dtype, const float* grads,
                          float* m, float* v, long long n, int t, float lr, float beta1, float beta2,
                          float eps, float weight_decay, void* stream) {
  return gpt::adamw_step(master, params, param_dtype, grads, m, v, n, t, lr, beta1, beta2, eps,
                         weight_decay, gpt::as_stream(stream));
}

size_t gpt_muon_scratch_bytes(int n_matrices, int rows, int cols) {
  return gpt::muon_scratch_bytes(n_matrices, rows, cols);
}

gpt_status gpt_muon_step(float* master, void* params, int param_dtype, const float* grads,
                         float* momentum_buf, int groups, int per_group, long long group_stride,
                         int rows, int cols, float lr, float momentum, int nesterov, int ns_steps,
                         float ns_a, float ns_b, float ns_c, void* scratch, size_t scratch_bytes,
                         int* status, void* stream) {
  return gpt::muon_step(master, params, param_dtype, grads, momentum_buf, groups, per_group,
                        group_stride, rows, cols, lr, momentum, nesterov, ns_steps, ns_a, ns_b, ns_c,
                        scratch, scratch_bytes, status, gpt::as_stream(stream));
}

size_t gpt_optim_scratch_bytes(const gpt_config* cfg) {
  if (!cfg || cfg->depth <= 0) return 0;
  std::vector<size_t> off(2 + 4 * (size_t)cfg->depth);
  size_t total = 0;
  if (gpt_param_layout(cfg, off.data(), &total) != GPT_OK) return 0;
  size_t need = 0;
  for (const auto& g : muon_groups(cfg, off.data()))
    need = std::max(need, gpt::muon_scratch_bytes(g.groups * g.per, g.rows, g.cols));
  return need;
}

gpt_status gpt_optim_step(const gpt_config* cfg, float* master, void* params, const float* grads,
                          float* state_m, float* state_v, int t, const gpt_optim_hparams* hp,
                          void* scratch, size_t scratch_bytes, int* status, void* stream) {
  if (!cfg || !master || !grads || !state_m || !state_v || !hp || t < 1) return GPT_ERR_INVALID_ARG;
  std::vector<size_t> off(2 + 4 * (size_t)std::max(0, cfg->depth));
  size_t total = 0;
  GPT_TRY(gpt_param_layout(cfg, off.data(), &total));
  if (cfg->depth > 0 && (!scratch || scratch_bytes < gpt_optim_scratch_bytes(cfg)))
    return GPT_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = gpt::as_stream(stream);
  const int pdt = cfg->param_dtype;
  auto P = [&](size_t o) -> void* {
    if (!params) return nullptr;
    return pdt == GPT_DTYPE_BF16 ? (void*)(reinterpret_cast<uint16_t*>(params) + o)
                                 : (void*)(reinterpret_cast<float*>(params) + o);
  };
  for (const auto& g : muon_groups(cfg, off.data())) {
    GPT_TRY(gpt::muon_step(master + g.off, P(g.off), pdt, grads + g.off, state_m + g.off, g.groups,
                           g.per, g.gstride, g.rows, g.cols, hp->muon_lr, hp->muon_momentum,
                           hp->muon_nesterov, hp->ns_steps, hp->ns_a, hp->ns_b, hp->ns_c, scratch,
                           scratch_bytes, status, s));
  }
  const float scale = 1.f / std::sqrt((float)cfg->d_model / 768.f);
  const size_t nvd = (size_t)cfg->vocab * cfg->d_model;
  const size_t emb[2] = {off[0], off[1 + 4 * (size_t)cfg->depth]};
  const float lrs[2] = {hp->adam_lr_wte * scale, hp->adam_lr_lm * scale};
  for (int i = 0; i < 2; ++i) {
    GPT_TRY(gpt::adamw_step(master + emb[i], P(emb[i]), pdt, grads + emb[i], state_m + emb[i],
                            state_v + emb[i], (long long)nvd, t, lrs[i], hp->beta1, hp->beta2,
                            hp->eps, hp->weight_decay, s));
  }
  return GPT_OK;
}

}  // extern "C"
