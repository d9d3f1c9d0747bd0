// Memory-bound kernels of the training step: RMSNorm, RoPE + QK-norm, embedding gather and
// deterministic scatter, cross-entropy reductions, parameter cast.  Each is one pass over its
// operands with 16-byte vector accesses and one warp per row.
//
// RMSNorm has no gain ("Introducing nanochat", Pretraining: no RMSNorm parameters):
//   y = x·rho, rho = 1/sqrt(mean(x²) + 1e-6);  backward dx = rho·(dy − y·mean(y·dy)).
// RoPE ("nanochat User Guide" §10: rotary positional embeddings) rotates the pairs (i, i+Dh/2) by
// t·10000^(−2i/Dh); QK-norm (same section) is the parameter-free RMSNorm over each head.

#include <algorithm>

#include "common.cuh"
#include "host.h"

namespace gpt {

constexpr float NORM_EPS = 1e-6f;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
  return v;
}

// ------------------------------------------------------------------------------------------------
// RMSNorm
// ------------------------------------------------------------------------------------------------
__global__ void rmsnorm_fwd_kernel(const uint16_t* __restrict__ x, uint16_t* __restrict__ y,
                                   float* __restrict__ rho, int rows, int d) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)row * d);
  uint4* yr = reinterpret_cast<uint4*>(y + (size_t)row * d);
  const int nv = d >> 3;
  float ss = 0.f;
  for (int i = lane; i < nv; i += 32) {
    const uint4 v = xr[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) ss += bf_lo(w[e]) * bf_lo(w[e]) + bf_hi(w[e]) * bf_hi(w[e]);
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)d + NORM_EPS);
  for (int i = lane; i < nv; i += 32) {
    const uint4 v = xr[i];
    uint4 o;
    o.x = pack_bf2(bf_lo(v.x) * r, bf_hi(v.x) * r);
    o.y = pack_bf2(bf_lo(v.y) * r, bf_hi(v.y) * r);
    o.z = pack_bf2(bf_lo(v.z) * r, bf_hi(v.z) * r);
    o.w = pack_bf2(bf_lo(v.w) * r, bf_hi(v.w) * r);
    yr[i] = o;
  }
  if (lane == 0) rho[row] = r;
}

template <bool DY_F32>
__device__ __forceinline__ void load8(const void* p, size_t idx, float (&v)[8]) {
  if (DY_F32) {
    const float4* f = reinterpret_cast<const float4*>(p) + idx * 2;
    const float4 a = f[0], b = f[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 u = reinterpret_cast<const uint4*>(p)[idx];
    v[0] = bf_lo(u.x); v[1] = bf_hi(u.x); v[2] = bf_lo(u.y); v[3] = bf_hi(u.y);
    v[4] = bf_lo(u.z); v[5] = bf_hi(u.z); v[6] = bf_lo(u.w); v[7] = bf_hi(u.w);
  }
}

template <bool DY_F32>
__global__ void rmsnorm_bwd_kernel(const void* __restrict__ dy, const uint16_t* __restrict__ y,
                                   const float* __restrict__ rho, float* __restrict__ gx,
                                   uint16_t* __restrict__ gx_bf16, int accumulate, int rows, int d) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int nv = d >> 3;
  const size_t base = (size_t)row * nv;
  float dot = 0.f;
  for (int i = lane; i < nv; i += 32) {
    float a[8], b[8];
    load8<DY_F32>(dy, base + i, a);
    load8<false>(y, base + i, b);
#pragma unroll
    for (int e = 0; e < 8; ++e) dot += a[e] * b[e];
  }
  dot = warp_sum(dot) / (float)d;
  const float r = rho[row];
  for (int i = lane; i < nv; i += 32) {
    float a[8], b[8];
    load8<DY_F32>(dy, base + i, a);
    load8<false>(y, base + i, b);
    float4* g = reinterpret_cast<float4*>(gx) + (base + i) * 2;
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = r * (a[e] - b[e] * dot);
    if (accumulate) {
      const float4 p0 = g[0], p1 = g[1];
      o[0] += p0.x; o[1] += p0.y; o[2] += p0.z; o[3] += p0.w;
      o[4] += p1.x; o[5] += p1.y; o[6] += p1.z; o[7] += p1.w;
    }
    g[0] = make_float4(o[0], o[1], o[2], o[3]);
    g[1] = make_float4(o[4], o[5], o[6], o[7]);
    if (gx_bf16) {
      uint4 u;
      u.x = pack_bf2(o[0], o[1]); u.y = pack_bf2(o[2], o[3]);
      u.z = pack_bf2(o[4], o[5]); u.w = pack_bf2(o[6], o[7]);
      reinterpret_cast<uint4*>(gx_bf16)[base + i] = u;
    }
  }
}

// ------------------------------------------------------------------------------------------------
// RoPE + QK-norm
// ------------------------------------------------------------------------------------------------
__global__ void rope_table_kernel(float* __restrict__ cs, int T, int half, int Dh) {
  pdl_wait();
  pdl_trigger();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= T * half) return;
  const int t = idx / half, i = idx % half;
  const double inv_freq = pow(10000.0, -2.0 * (double)i / (double)Dh);
  const double phi = (double)t * inv_freq;
  cs[2 * idx] = (float)cos(phi);
  cs[2 * idx + 1] = (float)sin(phi);
}

// One warp per token: it walks the 2H (part ∈ {q, k}, head) units of the token in batches of 8,
// issuing all loads of a batch before using them.  Lane l holds the pairs i = 2l, 2l+1 (+64 per
// further round) of the first half of each head and their partners i + Dh/2; the cos/sin of those
// pairs at position t are loaded once per token.
constexpr int ROPE_BATCH = 8;

template <int ROUNDS>
__global__ void __launch_bounds__(256) rope_qknorm_fwd_kernel(uint16_t* __restrict__ qkv, float* __restrict__ rho_q,
                                                              float* __restrict__ rho_k, const float* __restrict__ cs,
                                                              int M, int T, int H, int Dh) {
  pdl_wait();
  pdl_trigger();
  const long long m = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  const int t = (int)(m % T), half = Dh >> 1, d = H * Dh;
  bool act[ROUNDS];
  float4 cw[ROUNDS];  // cos_i, sin_i, cos_{i+1}, sin_{i+1}
#pragma unroll
  for (int rr = 0; rr < ROUNDS; ++rr) {
    const int i = 2 * lane + 64 * rr;
    act[rr] = i < half;
    if (act[rr]) cw[rr] = *reinterpret_cast<const float4*>(cs + 2 * ((size_t)t * half + i));
  }
  uint16_t* row = qkv + m * 3 * d;
  for (int u0 = 0; u0 < 2 * H; u0 += ROPE_BATCH) {
    uint32_t ua[ROPE_BATCH][ROUNDS], ub[ROPE_BATCH][ROUNDS];
#pragma unroll
    for (int k = 0; k < ROPE_BATCH; ++k) {
      const int u = u0 + k;
#pragma unroll
      for (int rr = 0; rr < ROUNDS; ++rr) {
        ua[k][rr] = ub[k][rr] = 0;
        if (u < 2 * H && act[rr]) {
          const uint16_t* p = row + (u / H) * d + (u % H) * Dh + 2 * lane + 64 * rr;
          ua[k][rr] = *reinterpret_cast<const uint32_t*>(p);
          ub[k][rr] = *reinterpret_cast<const uint32_t*>(p + half);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < ROPE_BATCH; ++k) {
      const int u = u0 + k;
      if (u >= 2 * H) break;  // warp-uniform
      float a0[ROUNDS], a1[ROUNDS], b0[ROUNDS], b1[ROUNDS];
      float ss = 0.f;
#pragma unroll
      for (int rr = 0; rr < ROUNDS; ++rr) {
        const float x0 = bf_lo(ua[k][rr]), x1 = bf_hi(ua[k][rr]);
        const float y0 = bf_lo(ub[k][rr]), y1 = bf_hi(ub[k][rr]);
        const float4 c = cw[rr];
        a0[rr] = x0 * c.x - y0 * c.y;
        b0[rr] = x0 * c.y + y0 * c.x;
        a1[rr] = x1 * c.z - y1 * c.w;
        b1[rr] = x1 * c.w + y1 * c.z;
        if (act[rr]) ss += a0[rr] * a0[rr] + a1[rr] * a1[rr] + b0[rr] * b0[rr] + b1[rr] * b1[rr];
      }
      ss = warp_sum(ss);
      const float r = rsqrtf(ss / (float)Dh + NORM_EPS);
      uint16_t* p = row + (u / H) * d + (u % H) * Dh + 2 * lane;
#pragma unroll
      for (int rr = 0; rr < ROUNDS; ++rr) {
        if (act[rr]) {
          *reinterpret_cast<uint32_t*>(p + 64 * rr) = pack_bf2(a0[rr] * r, a1[rr] * r);
          *reinterpret_cast<uint32_t*>(p + 64 * rr + half) = pack_bf2(b0[rr] * r, b1[rr] * r);
        }
      }
      if (lane == 0) ((u < H) ? rho_q : rho_k)[m * H + (u % H)] = r;
    }
  }
}

// Backward: g = rho·(dŷ − ŷ·mean(ŷ·dŷ)) with ŷ the stored forward output, then the inverse
// rotation (a, b) → (a cos + b sin, −a sin + b cos).  Same work split as the forward.
// Y_HEADS: the forward output ŷ is read head-major, y[part][b][h][t][j], instead of from the
// token-major [M, 3d] rows.
template <int ROUNDS, bool Y_HEADS>
__global__ void __launch_bounds__(256) rope_qknorm_bwd_kernel(uint16_t* __restrict__ dqkv, const uint16_t* __restrict__ qkv,
                                                              const float* __restrict__ rho_q, const float* __restrict__ rho_k,
                                                              const float* __restrict__ cs, int M, int T, int H, int Dh) {
  pdl_wait();
  pdl_trigger();
  const long long m = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  const int t = (int)(m % T), half = Dh >> 1, d = H * Dh;
  bool act[ROUNDS];
  float4 cw[ROUNDS];
#pragma unroll
  for (int rr = 0; rr < ROUNDS; ++rr) {
    const int i = 2 * lane + 64 * rr;
    act[rr] = i < half;
    if (act[rr]) cw[rr] = *reinterpret_cast<const float4*>(cs + 2 * ((size_t)t * half + i));
  }
  uint16_t* grow = dqkv + m * 3 * d;
  const uint16_t* yrow = qkv + m * 3 * d;
  for (int u0 = 0; u0 < 2 * H; u0 += ROPE_BATCH) {
    uint32_t ga[ROPE_BATCH][ROUNDS], gb[ROPE_BATCH][ROUNDS], ya[ROPE_BATCH][ROUNDS], yb[ROPE_BATCH][ROUNDS];
    float rh[ROPE_BATCH];
#pragma unroll
    for (int k = 0; k < ROPE_BATCH; ++k) {
      const int u = u0 + k;
      rh[k] = 0.f;
      if (u < 2 * H) rh[k] = ((u < H) ? rho_q : rho_k)[m * H + (u % H)];
#pragma unroll
      for (int rr = 0; rr < ROUNDS; ++rr) {
        ga[k][rr] = gb[k][rr] = ya[k][rr] = yb[k][rr] = 0;
        if (u < 2 * H && act[rr]) {
          const size_t off = (u / H) * d + (u % H) * Dh + 2 * lane + 64 * rr;
          ga[k][rr] = *reinterpret_cast<const uint32_t*>(grow + off);
          gb[k][rr] = *reinterpret_cast<const uint32_t*>(grow + off + half);
          const uint16_t* yp;
          if (Y_HEADS) {
            const long long b = m / T;
            yp = qkv + (long long)(u / H) * M * d + ((b * H + (u % H)) * T + t) * Dh + 2 * lane + 64 * rr;
          } else {
            yp = yrow + off;
          }
          ya[k][rr] = *reinterpret_cast<const uint32_t*>(yp);
          yb[k][rr] = *reinterpret_cast<const uint32_t*>(yp + half);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < ROPE_BATCH; ++k) {
      const int u = u0 + k;
      if (u >= 2 * H) break;
      float dot = 0.f;
#pragma unroll
      for (int rr = 0; rr < ROUNDS; ++rr)
        dot += bf_lo(ga[k][rr]) * bf_lo(ya[k][rr]) + bf_hi(ga[k][rr]) * bf_hi(ya[k][rr]) +
               bf_lo(gb[k][rr]) * bf_lo(yb[k][rr]) + bf_hi(gb[k][rr]) * bf_hi(yb[k][rr]);
      dot = warp_sum(dot) / (float)Dh;
      const float r = rh[k];
      uint16_t* p = grow + (u / H) * d + (u % H) * Dh + 2 * lane;
#pragma unroll
      for (int rr = 0; rr < ROUNDS; ++rr) {
        if (!act[rr]) continue;
        const float4 c = cw[rr];
        const float na0 = r * (bf_lo(ga[k][rr]) - bf_lo(ya[k][rr]) * dot);
        const float na1 = r * (bf_hi(ga[k][rr]) - bf_hi(ya[k][rr]) * dot);
        const float nb0 = r * (bf_lo(gb[k][rr]) - bf_lo(yb[k][rr]) * dot);
        const float nb1 = r * (bf_hi(gb[k][rr]) - bf_hi(yb[k][rr]) * dot);
        *reinterpret_cast<uint32_t*>(p + 64 * rr) =
            pack_bf2(na0 * c.x + nb0 * c.y, na1 * c.z + nb1 * c.w);
        *reinterpret_cast<uint32_t*>(p + 64 * rr + half) =
            pack_bf2(-na0 * c.y + nb0 * c.x, -na1 * c.w + nb1 * c.z);
      }
    }
  }
}

// ------------------------------------------------------------------------------------------------
// embedding
// ------------------------------------------------------------------------------------------------
__global__ void embedding_fwd_kernel(const int32_t* __restrict__ tok, const uint16_t* __restrict__ wte,
                                     uint16_t* __restrict__ x, int M, int d, int V, int* status) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= M) return;
  int id = tok[row];
  if (id < 0 || id >= V) {
    if (lane == 0) set_status(status, GPT_ERR_TOKEN_OUT_OF_RANGE);
    id = min(max(id, 0), V - 1);
  }
  const uint4* src = reinterpret_cast<const uint4*>(wte + (size_t)id * d);
  uint4* dst = reinterpret_cast<uint4*>(x + (size_t)row * d);
  for (int i = lane; i < (d >> 3); i += 32) dst[i] = src[i];
}

// Single-CTA stable sort of the keys (id << 16 | local index) of one segment of ≤ 32768 tokens by
// id: a least-significant-digit radix sort over the 16 id bits in four 4-bit passes.  Thread t owns
// the 32 keys at positions 32t .. 32t+31 of the current order; per pass it counts its digits, a
// block-wide exclusive scan over (digit, thread) gives every thread its first slot per digit, and
// the thread writes its keys there in order — so equal ids keep their position order (stable), and
// since positions start in increasing order the keys end sorted by (id, position).  Then the run
// heads (first position of every distinct id) are compacted in ascending order.
// Outputs: sorted keys [n], run starts [nruns + 1] (last = n), *nruns.
constexpr int EMB_SEG = 32768;
constexpr int EMB_SORT_THREADS = 1024;
constexpr int EMB_SORT_PER_THREAD = EMB_SEG / EMB_SORT_THREADS;                     // 32
constexpr int EMB_SORT_SMEM = EMB_SEG * 4 + 16 * EMB_SORT_THREADS * 4;                // keys + counts
__global__ void __launch_bounds__(EMB_SORT_THREADS) embedding_sort_kernel(const int32_t* __restrict__ tok, int n,
                                                                          int V, uint32_t* __restrict__ keys_out,
                                                                          int* __restrict__ run_start,
                                                                          int* __restrict__ nruns) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint32_t sk[];                  // [EMB_SEG] keys
  int* cnt = reinterpret_cast<int*>(sk + EMB_SEG);  // [16][EMB_SORT_THREADS] digit counts, then offsets
  __shared__ int warp_sum[EMB_SORT_THREADS / 32];
  const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
  uint32_t key[EMB_SORT_PER_THREAD];
#pragma unroll
  for (int j = 0; j < EMB_SORT_PER_THREAD; ++j) {
    const int i = t * EMB_SORT_PER_THREAD + j;
    if (i < n) {
      int id = tok[i];
      id = min(max(id, 0), V - 1);
      key[j] = ((uint32_t)id << 16) | (uint32_t)i;
    } else {
      key[j] = 0xFFFFFFFFu;  // after every real key of id 0xFFFF too: it starts later and the sort is stable
    }
  }
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 16 + 4 * pass;
    int c[16];
#pragma unroll
    for (int dg = 0; dg < 16; ++dg) c[dg] = 0;
#pragma unroll
    for (int j = 0; j < EMB_SORT_PER_THREAD; ++j) {
      const int dg = (key[j] >> shift) & 15;
#pragma unroll
      for (int e = 0; e < 16; ++e) c[e] += (dg == e);
    }
#pragma unroll
    for (int dg = 0; dg < 16; ++dg) cnt[dg * EMB_SORT_THREADS + t] = c[dg];
    __syncthreads();
    // exclusive scan of cnt in (digit, thread) order: thread t scans elements 16t .. 16t+15
    int local[16], sum = 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      local[e] = sum;
      sum += cnt[16 * t + e];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sum[wid] = incl;
    __syncthreads();
    int base = incl - sum;
    for (int w = 0; w < wid; ++w) base += warp_sum[w];
#pragma unroll
    for (int e = 0; e < 16; ++e) cnt[16 * t + e] = base + local[e];
    __syncthreads();
    // scatter this thread's keys, in order, from its first slot per digit
    int off[16];
#pragma unroll
    for (int dg = 0; dg < 16; ++dg) off[dg] = cnt[dg * EMB_SORT_THREADS + t];
#pragma unroll
    for (int j = 0; j < EMB_SORT_PER_THREAD; ++j) {
      const int dg = (key[j] >> shift) & 15;
      int slot = 0;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        if (dg == e) { slot = off[e]; off[e] = slot + 1; }
      }
      sk[slot] = key[j];
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < EMB_SORT_PER_THREAD; ++j) key[j] = sk[t * EMB_SORT_PER_THREAD + j];
    __syncthreads();
  }
  for (int i = t; i < n; i += blockDim.x) keys_out[i] = sk[i];
  __syncthreads();
  // run heads: a stable compaction with a block-wide scan over chunks of blockDim.x
  __shared__ int warp_tot[32];
  __shared__ int base_s;
  if (threadIdx.x == 0) base_s = 0;
  __syncthreads();
  for (int c0 = 0; c0 < n; c0 += blockDim.x) {
    const int i = c0 + threadIdx.x;
    const int head = (i < n) && (i == 0 || (sk[i] >> 16) != (sk[i - 1] >> 16));
    const unsigned mask = __ballot_sync(0xffffffffu, head);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int before = __popc(mask & ((1u << lane) - 1));
    if (lane == 0) warp_tot[wid] = __popc(mask);
    __syncthreads();
    int off = 0;
    for (int w = 0; w < wid; ++w) off += warp_tot[w];
    if (head) run_start[base_s + off + before] = i;
    __syncthreads();
    if (threadIdx.x == 0) {
      int tot = 0;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += warp_tot[w];
      base_s += tot;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    run_start[base_s] = n;
    *nruns = base_s;
  }
}

// Deterministic accumulation over the sorted (id, position) keys in fixed pieces of EMB_PIECE
// consecutive keys, so that a frequent id (Zipf-hot rows) is spread over many CTAs:
//   piece kernel  one CTA per piece; threads cover the columns (4 floats each) and walk the piece's
//                 rows in order.  A run (equal ids) lying wholly inside the piece is written to
//                 dwte directly; a run that crosses the piece's start goes to partial slot 0, one
//                 that continues past its end to slot 1 (a run crossing both: slot 0).
//   fix-up kernel one CTA per run that spans several pieces: sums slot 1 of its first piece,
//                 slot 0 of the pieces after it, in piece order, into dwte[id].
constexpr int EMB_PIECE = 64;

__global__ void embedding_piece_kernel(const uint32_t* __restrict__ keys, int n, const float* __restrict__ gx,
                                       float* __restrict__ dwte, float* __restrict__ partial, int seg0, int d,
                                       int accumulate) {
  pdl_wait();
  pdl_trigger();
  const int p = blockIdx.x;
  const int s = p * EMB_PIECE, e = min(n, s + EMB_PIECE);
  const int idx_before = (s > 0) ? (int)(keys[s - 1] >> 16) : -1;
  const int idx_after = (e < n) ? (int)(keys[e] >> 16) : -1;
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int i = s;
    while (i < e) {
      const int id = (int)(keys[i] >> 16);
      int j = i;
      acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (; j < e && (int)(keys[j] >> 16) == id; ++j) {
        const int m = seg0 + (int)(keys[j] & 0xFFFFu);
        const float4 v = *reinterpret_cast<const float4*>(gx + (size_t)m * d + c);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
      const bool from_before = (i == s) && (id == idx_before);
      const bool to_after = (j == e) && (id == idx_after);
      if (!from_before && !to_after) {
        float4* dst = reinterpret_cast<float4*>(dwte + (size_t)id * d + c);
        if (accumulate) {
          const float4 o = *dst;
          acc.x += o.x; acc.y += o.y; acc.z += o.z; acc.w += o.w;
        }
        *dst = acc;
      } else {
        const int slot = from_before ? 0 : 1;
        *reinterpret_cast<float4*>(partial + ((size_t)p * 2 + slot) * d + c) = acc;
      }
      i = j;
    }
  }
}

__global__ void embedding_fixup_kernel(const uint32_t* __restrict__ keys, const int* __restrict__ run_start,
                                       const int* __restrict__ nruns, const float* __restrict__ partial,
                                       float* __restrict__ dwte, int d, int accumulate) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  if (r >= *nruns) return;
  const int s = run_start[r], e = run_start[r + 1];
  const int ps = s / EMB_PIECE, pe = (e - 1) / EMB_PIECE;
  if (ps == pe) return;  // written by its piece
  const int id = (int)(keys[s] >> 16);
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
    // the first piece holds the run's head in slot 1 (slot 0 if the run starts the piece at its
    // first key and the previous key has another id, which makes it "not from before")
    float4 acc = *reinterpret_cast<const float4*>(partial + ((size_t)ps * 2 + 1) * d + c);
    for (int p = ps + 1; p <= pe; ++p) {
      const float4 v = *reinterpret_cast<const float4*>(partial + ((size_t)p * 2 + 0) * d + c);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    float4* dst = reinterpret_cast<float4*>(dwte + (size_t)id * d + c);
    if (accumulate) {
      const float4 o = *dst;
      acc.x += o.x; acc.y += o.y; acc.z += o.z; acc.w += o.w;
    }
    *dst = acc;
  }
}

// ------------------------------------------------------------------------------------------------
// cross-entropy reductions
// ------------------------------------------------------------------------------------------------
// Per row: lse = logsumexp over the vocabulary tiles' (max, Σexp) pairs; ℓ = lse − z[target]
// (0 for ignored rows).  One warp per row.
__global__ void ce_rows_kernel(const float2* __restrict__ stats, int ntiles, const float* __restrict__ zt,
                               const int32_t* __restrict__ targets, int M, int V, float* __restrict__ lse,
                               float* __restrict__ ell, int* status) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= M) return;
  const float2* s = stats + (size_t)row * ntiles;
  float mx = -INFINITY;
  for (int i = lane; i < ntiles; i += 32) mx = fmaxf(mx, s[i].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
  for (int i = lane; i < ntiles; i += 32) sum += s[i].y * __expf(s[i].x - mx);
  sum = warp_sum(sum);
  if (lane == 0) {
    const float l = mx + logf(sum);
    lse[row] = l;
    const int t = targets[row];
    if (t < -1 || t >= V) set_status(status, GPT_ERR_TOKEN_OUT_OF_RANGE);
    ell[row] = (t >= 0 && t < V) ? (l - zt[row]) : 0.f;
  }
}

// Single CTA: loss = Σ ℓ / n_valid in a fixed order (0 when n_valid = 0); inv_n = 1/n_valid.
__global__ void __launch_bounds__(1024) ce_finalize_kernel(const float* __restrict__ ell,
                                                           const int32_t* __restrict__ targets, int M,
                                                           int V, float* __restrict__ loss,
                                                           float* __restrict__ inv_n) {
  pdl_wait();
  pdl_trigger();
  __shared__ double ssum[1024];
  __shared__ int scnt[1024];
  double acc = 0.0;
  int cnt = 0;
  for (int i = threadIdx.x; i < M; i += blockDim.x) {
    const int t = targets[i];
    if (t >= 0 && t < V) { acc += (double)ell[i]; ++cnt; }
  }
  ssum[threadIdx.x] = acc;
  scnt[threadIdx.x] = cnt;
  __syncthreads();
  for (int s = blockDim.x >> 1; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) {
      ssum[threadIdx.x] += ssum[threadIdx.x + s];
      scnt[threadIdx.x] += scnt[threadIdx.x + s];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int n = scnt[0];
    *loss = n ? (float)(ssum[0] / (double)n) : 0.f;
    *inv_n = n ? 1.f / (float)n : 0.f;
  }
}

__global__ void cast_f32_bf16_kernel(const float* __restrict__ src, uint16_t* __restrict__ dst, size_t n) {
  pdl_wait();
  pdl_trigger();
  const size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i + 4 <= n) {
    const float4 v = *reinterpret_cast<const float4*>(src + i);
    uint2 o;
    o.x = pack_bf2(v.x, v.y);
    o.y = pack_bf2(v.z, v.w);
    *reinterpret_cast<uint2*>(dst + i) = o;
  } else {
    for (size_t j = i; j < n; ++j) dst[j] = f2bf(src[j]);
  }
}

// dst[i] += src[i] (gradient accumulation across micro-batches), four floats per thread
__global__ void add_f32_kernel(float* __restrict__ dst, const float* __restrict__ src, size_t n) {
  pdl_wait();
  pdl_trigger();
  const size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i + 4 <= n) {
    float4 a = *reinterpret_cast<const float4*>(dst + i);
    const float4 b = *reinterpret_cast<const float4*>(src + i);
    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    *reinterpret_cast<float4*>(dst + i) = a;
  } else {
    for (size_t j = i; j < n; ++j) dst[j] += src[j];
  }
}

// ------------------------------------------------------------------------------------------------
// launchers
// ------------------------------------------------------------------------------------------------
static inline unsigned blocks_for_warps(long long warps, int threads) {
  return (unsigned)((warps * 32 + threads - 1) / threads);
}

gpt_status rmsnorm_fwd(const void* x, void* y, float* rho, int rows, int d, cudaStream_t s) {
  if (!x || !y || !rho || rows <= 0 || d <= 0) return GPT_ERR_INVALID_ARG;
  if (d % 8) return GPT_ERR_UNSUPPORTED_SHAPE;
  return launch_kernel(rmsnorm_fwd_kernel, dim3(blocks_for_warps(rows, 256)), dim3(256), 0, s,
                       reinterpret_cast<const uint16_t*>(x), reinterpret_cast<uint16_t*>(y), rho, rows, d);
}

gpt_status rmsnorm_bwd(const void* dy, int dy_f32, const void* y, const float* rho, float* gx,
                       void* gx_bf16, int accumulate, int rows, int d, cudaStream_t s) {
  if (!dy || !y || !rho || !gx || rows <= 0 || d <= 0) return GPT_ERR_INVALID_ARG;
  if (d % 8) return GPT_ERR_UNSUPPORTED_SHAPE;
  const unsigned nb = blocks_for_warps(rows, 256);
  if (dy_f32)
    return launch_kernel(rmsnorm_bwd_kernel<true>, dim3(nb), dim3(256), 0, s, dy,
                         reinterpret_cast<const uint16_t*>(y), rho, gx,
                         reinterpret_cast<uint16_t*>(gx_bf16), accumulate, rows, d);
  return launch_kernel(rmsnorm_bwd_kernel<false>, dim3(nb), dim3(256), 0, s, dy,
                       reinterpret_cast<const uint16_t*>(y), rho, gx,
                       reinterpret_cast<uint16_t*>(gx_bf16), accumulate, rows, d);
}

gpt_status rope_table(float* cs, int T, int Dh, cudaStream_t s) {
  if (!cs || T <= 0 || Dh <= 0 || (Dh % 4)) return GPT_ERR_INVALID_ARG;
  const int n = T * (Dh / 2);
  return launch_kernel(rope_table_kernel, dim3((n + 255) / 256), dim3(256), 0, s, cs, T, Dh / 2, Dh);
}

static gpt_status check_rope(int B, int T, int H, int Dh) {
  if (B <= 0 || T <= 0 || H <= 0) return GPT_ERR_INVALID_ARG;
  if (Dh != 32 && Dh != 64 && Dh != 128 && Dh != 256) return GPT_ERR_UNSUPPORTED_SHAPE;
  return GPT_OK;
}

gpt_status rope_qknorm_fwd(void* qkv, float* rq, float* rk, const float* cs, int B, int T, int H,
                           int Dh, cudaStream_t s) {
  if (!qkv || !rq || !rk || !cs) return GPT_ERR_INVALID_ARG;
  GPT_TRY(check_rope(B, T, H, Dh));
  const long long warps = (long long)B * T;
  if (Dh > 128)
    rope_qknorm_fwd_kernel<2><<<blocks_for_warps(warps, 256), 256, 0, s>>>(
        reinterpret_cast<uint16_t*>(qkv), rq, rk, cs, B * T, T, H, Dh);
  else
    rope_qknorm_fwd_kernel<1><<<blocks_for_warps(warps, 256), 256, 0, s>>>(
        reinterpret_cast<uint16_t*>(qkv), rq, rk, cs, B * T, T, H, Dh);
  count_launch();
  GPT_CUDA_TRY(cudaGetLastError());
  return GPT_OK;
}

template <bool Y_HEADS>
static void launch_rope_bwd(void* dqkv, const void* y, const float* rq, const float* rk,
                            const float* cs, int B, int T, int H, int Dh, cudaStream_t s) {
  const long long warps = (long long)B * T;
  if (Dh > 128)
    rope_qknorm_bwd_kernel<2, Y_HEADS><<<blocks_for_warps(warps, 256), 256, 0, s>>>(
        reinterpret_cast<uint16_t*>(dqkv), reinterpret_cast<const uint16_t*>(y), rq, rk, cs, B * T,
        T, H, Dh);
  else
    rope_qknorm_bwd_kernel<1, Y_HEADS><<<blocks_for_warps(warps, 256), 256, 0, s>>>(
        reinterpret_cast<uint16_t*>(dqkv), reinterpret_cast<const uint16_t*>(y), rq, rk, cs, B * T,
        T, H, Dh);
}

// y_heads: the forward output is stored head-major [2][B][H][T][Dh] (q̃ then k̃).
gpt_status rope_qknorm_bwd_heads(void* dqkv, const void* y_heads, const float* rq, const float* rk,
                                 const float* cs, int B, int T, int H, int Dh, cudaStream_t s) {
  if (!dqkv || !y_heads || !rq || !rk || !cs) return GPT_ERR_INVALID_ARG;
  GPT_TRY(check_rope(B, T, H, Dh));
  launch_rope_bwd<true>(dqkv, y_heads, rq, rk, cs, B, T, H, Dh, s);
  count_launch();
  GPT_CUDA_TRY(cudaGetLastError());
  return GPT_OK;
}

gpt_status rope_qknorm_bwd(void* dqkv, const void* qkv, const float* rq, const float* rk,
                           const float* cs, int B, int T, int H, int Dh, cudaStream_t s) {
  if (!dqkv || !qkv || !rq || !rk || !cs) return GPT_ERR_INVALID_ARG;
  GPT_TRY(check_rope(B, T, H, Dh));
  launch_rope_bwd<false>(dqkv, qkv, rq, rk, cs, B, T, H, Dh, s);
  count_launch();
  GPT_CUDA_TRY(cudaGetLastError());
  return GPT_OK;
}

gpt_status embedding_fwd(const int32_t* tok, const void* wte, void* x, int M, int d, int V,
                         int* status, cudaStream_t s) {
  if (!tok || !wte || !x || M <= 0 || d <= 0 || V <= 0) return GPT_ERR_INVALID_ARG;
  if (d % 8) return GPT_ERR_UNSUPPORTED_SHAPE;
  return launch_kernel(embedding_fwd_kernel, dim3(blocks_for_warps(M, 256)), dim3(256), 0, s, tok,
                       reinterpret_cast<const uint16_t*>(wte), reinterpret_cast<uint16_t*>(x), M, d, V,
                       status);
}

size_t embedding_bwd_scratch_bytes(int M, int d, int V) {
  (void)V;
  const int seg = std::min(M, EMB_SEG);
  const size_t pieces = (seg + EMB_PIECE - 1) / EMB_PIECE;
  // keys [seg], run starts [seg + 1], nruns, partial sums [pieces][2][d]
  auto al = [](size_t b) { return (b + 255) & ~(size_t)255; };
  return al((size_t)seg * 4) + al((size_t)(seg + 1) * 4) + al(4) + al(pieces * 2 * (size_t)d * 4);
}

gpt_status embedding_bwd(const int32_t* tok, const float* gx, float* dwte, int M, int d, int V,
                         void* scratch, cudaStream_t s) {
  if (!tok || !gx || !dwte || !scratch || M <= 0 || d <= 0 || V <= 0) return GPT_ERR_INVALID_ARG;
  if ((d % 4) || V > 65536) return GPT_ERR_UNSUPPORTED_SHAPE;
  auto al = [](size_t b) { return (b + 255) & ~(size_t)255; };
  const int seg = std::min(M, EMB_SEG);
  uint8_t* p = reinterpret_cast<uint8_t*>(scratch);
  uint32_t* keys = reinterpret_cast<uint32_t*>(p);
  int* run_start = reinterpret_cast<int*>(p + al((size_t)seg * 4));
  int* nruns = reinterpret_cast<int*>(p + al((size_t)seg * 4) + al((size_t)(seg + 1) * 4));
  float* partial = reinterpret_cast<float*>(p + al((size_t)seg * 4) + al((size_t)(seg + 1) * 4) + al(4));
  GPT_CUDA_TRY(cudaMemsetAsync(dwte, 0, (size_t)V * d * sizeof(float), s));
  GPT_TRY(ensure_smem(embedding_sort_kernel, EMB_SORT_SMEM));
  const int threads = std::min(512, std::max(32, ((d / 4) + 31) / 32 * 32));
  for (int s0 = 0; s0 < M; s0 += EMB_SEG) {
    const int n = std::min(EMB_SEG, M - s0);
    embedding_sort_kernel<<<1, EMB_SORT_THREADS, EMB_SORT_SMEM, s>>>(tok + s0, n, V, keys, run_start, nruns);
    count_launch();
    GPT_CUDA_TRY(cudaGetLastError());
    const int pieces = (n + EMB_PIECE - 1) / EMB_PIECE;
    // segments after the first add onto the rows earlier segments wrote
    const int acc = (s0 > 0) ? 1 : 0;
    embedding_piece_kernel<<<pieces, threads, 0, s>>>(keys, n, gx, dwte, partial, s0, d, acc);
    count_launch();
    GPT_CUDA_TRY(cudaGetLastError());
    embedding_fixup_kernel<<<n, threads, 0, s>>>(keys, run_start, nruns, partial, dwte, d, acc);
    count_launch();
    GPT_CUDA_TRY(cudaGetLastError());
  }
  return GPT_OK;
}

gpt_status ce_rows(const float2* stats, int ntiles, const float* zt, const int32_t* targets, int M,
                   int V, float* lse, float* ell, int* status, cudaStream_t s) {
  return launch_kernel(ce_rows_kernel, dim3(blocks_for_warps(M, 256)), dim3(256), 0, s, stats, ntiles, zt,
                       targets, M, V, lse, ell, status);
}

gpt_status ce_finalize(const float* ell, const int32_t* targets, int M, int V, float* loss,
                       float* inv_n, cudaStream_t s) {
  return launch_kernel(ce_finalize_kernel, dim3(1), dim3(1024), 0, s, ell, targets, M, V, loss, inv_n);
}

gpt_status add_f32(float* dst, const float* src, size_t n, cudaStream_t s) {
  const size_t threads = 256, per = 4;
  const size_t blocks = (n + threads * per - 1) / (threads * per);
  return launch_kernel(add_f32_kernel, dim3((unsigned)blocks), dim3((unsigned)threads), 0, s, dst, src, n);
}

gpt_status cast_f32_bf16(const float* src, void* dst, size_t n, cudaStream_t s) {
  const size_t threads = 256, per = 4;
  const size_t blocks = (n + threads * per - 1) / (threads * per);
  return launch_kernel(cast_f32_bf16_kernel, dim3((unsigned)blocks), dim3((unsigned)threads), 0, s, src,
                       reinterpret_cast<uint16_t*>(dst), n);
}

}  // namespace gpt

extern "C" {
gpt_status gpt_rmsnorm_fwd(const void* x, void* y, float* rho, int rows, int d, void* stream) {
  return gpt::rmsnorm_fwd(x, y, rho, rows, d, gpt::as_stream(stream));
}
gpt_status gpt_rmsnorm_bwd(const void* dy, int dy_f32, const void* y, const float* rho, float* gx,
                           void* gx_bf16, int accumulate, int rows, int d, void* stream) {
  return gpt::rmsnorm_bwd(dy, dy_f32, y, rho, gx, gx_bf16, accumulate, rows, d, gpt::as_stream(stream));
}
gpt_status gpt_rope_table(float* cos_sin, int T, int Dh, void* stream) {
  return gpt::rope_table(cos_sin, T, Dh, gpt::as_stream(stream));
}
gpt_status gpt_rope_qknorm_fwd(void* qkv, float* rho_q, float* rho_k, const float* cos_sin, int B,
                               int T, int H, int Dh, void* stream) {
  return gpt::rope_qknorm_fwd(qkv, rho_q, rho_k, cos_sin, B, T, H, Dh, gpt::as_stream(stream));
}
gpt_status gpt_rope_qknorm_bwd(void* dqkv, const void* qkv, const float* rho_q, const float* rho_k,
                               const float* cos_sin, int B, int T, int H, int Dh, void* stream) {
  return gpt::rope_qknorm_bwd(dqkv, qkv, rho_q, rho_k, cos_sin, B, T, H, Dh, gpt::as_stream(stream));
}
gpt_status gpt_embedding_fwd(const int32_t* tokens, const void* wte, void* x, int M, int d, int V,
                             int* status, void* stream) {
  return gpt::embedding_fwd(tokens, wte, x, M, d, V, status, gpt::as_stream(stream));
}
size_t gpt_embedding_bwd_scratch_bytes(int M, int d, int V) {
  return gpt::embedding_bwd_scratch_bytes(M, d, V);
}
gpt_status gpt_embedding_bwd(const int32_t* tokens, const float* gx, float* dwte, int M, int d,
                             int V, void* scratch, void* stream) {
  return gpt::embedding_bwd(tokens, gx, dwte, M, d, V, scratch, gpt::as_stream(stream));
}
}
