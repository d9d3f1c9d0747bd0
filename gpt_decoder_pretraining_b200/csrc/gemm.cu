// Persistent, warp-specialised bf16 GEMM on the sm_100a tcgen05 tensor cores, run by CTA pairs.
//
// A cluster of two CTAs (one per SM) computes 256×256 output tiles with one `cta_group::2` MMA
// stream: each CTA stages its own 128 rows of A and its own 128 rows (columns of C) of B, the even
// CTA issues the MMAs, and each CTA's tensor memory receives its 128 accumulator rows.  Per SM this
// halves the B traffic of a 128×256 single-CTA tile and leaves room for a 6-deep TMA ring.
//
//   warp 0      TMA producer (both CTAs): 128×64 A and 128×64 B tiles (128-byte swizzle) into the
//               ring; every load counts its bytes on the leader CTA's "full" barrier.
//   warp 1      MMA issuer (leader CTA only; the warp runs the loop, one elected lane issues):
//               tcgen05.mma 256×256×16 into a double-buffered accumulator; commits free the ring
//               stage and publish the tile in both CTAs.
//   warps 2..   epilogue (both CTAs): 4 warps per column group (one per tensor-memory lane
//               quarter; two groups split the 256 columns, one for the QKV + RoPE epilogue);
//               tcgen05.ld one accumulator row per thread, fused epilogue (bf16 cast, residual add,
//               ReLU², dReLU², fp32 store / add, axpby, head-major stores, QKV + RoPE + QK-norm, or the
//               cross-entropy statistics / gradient of the fused lm-head), global store; then
//               release the accumulator buffer to the leader.
// Tiles are distributed persistently over the CTA pairs.  When the tile count leaves the last wave
// partly empty, each tail tile is split along K into equal ranges that start together on several
// pairs (the whole waves before them keep every pair's K in step, so operands shared by
// concurrent tiles come from L2); a tile whose K range is split is summed from its pieces, in
// ascending K order, by the piece that finishes last (no waiting, no atomics on the output,
// bitwise reproducible).
//
// Operand majors: A and B may each be K-contiguous ("K-major") or M/N-contiguous ("MN-major"),
// which covers y = x·Wᵀ (forward), dx = dy·W (activation gradient) and dW = dyᵀ·x (weight
// gradient) without any transposed copy.

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "host.h"

namespace gpt {

gpt_status wait_limit_set_gemm(long long cycles) { return set_wait_limit_here(cycles); }

constexpr int BM = 128;   // rows per CTA (the pair covers 256)
constexpr int BN = 256;   // columns per tile (each CTA stages 128 rows of B)
constexpr int BK = 64;

enum : int {
  EPI_CE_STATS = 100,
  EPI_CE_GRAD = 101,
  EPI_BF16_HEADS = 103,   // bf16 store with row m = b·T + t, column n = h·Dh + j sent to [B, H, T, Dh]
  EPI_QKV_ROPE = 200      // + Dh: RoPE + QK-norm of the q and k heads, all three to [3][B][H][T][Dh]
};

// TMA warp, MMA warp, then 4 epilogue warps per column group (one per TMEM lane quarter).  Two
// column groups halve the epilogue time of a tile.
template <int EPI>
constexpr int gemm_col_groups() { return 2; }
template <int EPI>
constexpr int gemm_threads() { return 64 + 128 * gemm_col_groups<EPI>(); }

// Persistent schedule over the CTA pairs.  Output tiles 0 .. dp_tiles−1 are dealt round-robin and
// computed whole; dp_tiles is a whole number of waves, so every pair walks K in step with the others
// and the operand rows / columns that tiles of one wave share are read from L2, not HBM.  The
// sk_tiles after them (the last, partly empty wave) are each cut along K into sk_split equal
// pieces, all starting together: pair p takes piece p mod sk_split of tail tile p / sk_split,
// k-tiles [⌊j·k_tiles/sk_split⌋, ⌊(j+1)·k_tiles/sk_split⌋).  At any moment the tail pieces sit at
// sk_split K offsets, so L2 reuse across the tail tiles survives the split.
struct Sched {
  int num_pairs, k_tiles;
  int dp_tiles, sk_tiles;
  int sk_split;  // pieces per tail tile (1: no split)
};

// One unit of a pair's work: k-tiles [k0, k1) of output tile `tile`; `piece` is the piece index of
// a split tail tile, −1 for a whole tile.
struct Work {
  int tile, k0, k1, piece;
};
struct WorkIter {
  int dp_next;
  bool tail_done;
  __device__ WorkIter(const Sched& s, int p) : dp_next(p), tail_done(false) {}
  __device__ bool next(const Sched& s, Work& w) {
    if (dp_next < s.dp_tiles) {
      w.tile = dp_next;
      w.k0 = 0;
      w.k1 = s.k_tiles;
      w.piece = -1;
      dp_next += s.num_pairs;
      return true;
    }
    const int p = dp_next - s.dp_tiles;  // this pair's index in the tail phase
    if (!tail_done && p < s.sk_tiles * s.sk_split) {
      tail_done = true;
      const int j = p % s.sk_split;
      w.tile = s.dp_tiles + p / s.sk_split;
      w.k0 = (int)((long long)j * s.k_tiles / s.sk_split);
      w.k1 = (int)((long long)(j + 1) * s.k_tiles / s.sk_split);
      w.piece = s.sk_split > 1 ? j : -1;
      return true;
    }
    return false;
  }
};

// Output tile order within one matrix: groups of `group` row tiles, column by column inside a
// group (group 1: row by row).  With groups of 8 the tiles that run at the same time share a few row
// blocks of A and the column blocks of B they read, so a B larger than L2 (the lm-head's vocabulary
// matrix) is streamed once per group of row tiles instead of once per row tile.  Any order gives the
// same results: every tile is computed whole (or by its own pieces) and written once.
__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int group, int& tm, int& tn) {
  const int per_group = group * tiles_n;
  const int g = t / per_group, r = t - g * per_group;
  const int rows = min(group, tiles_m - g * group);
  tm = g * group + r % rows;
  tn = r / rows;
}
// Row-by-row order everywhere except the lm-head's NT products against the vocabulary matrix (its
// B, 100–168 MB, does not fit in L2); the projection weights (≤ 19 MB at d24) stay in L2 either way.
constexpr long long RASTER_B_BYTES = 32ll << 20;
inline int raster_for(int op, int N, int K) {
  return (op == GPT_GEMM_NT && (long long)N * K * 2 > RASTER_B_BYTES) ? 8 : 1;
}

// Piece exchange of a split tail tile: each piece writes its fp32 partial tile to its own slot
// (256 × 256 floats, slot = tail tile·sk_split + piece), then counts itself in one counter per
// epilogue warp (32 rows × 128 columns: 16 per tile).
constexpr int SK_WARPS_PER_TILE = 16;
constexpr int SK_MAX_TILES = 320;
constexpr int SK_MAX_SLOTS = 320;
constexpr size_t SK_SLOT_FLOATS = 256 * 256;
static_assert(GEMM_SK_COUNTER_BYTES == (size_t)SK_MAX_TILES * SK_WARPS_PER_TILE * sizeof(int),
              "counter region size");

struct GemmArgs {
  int M, N, K;
  int tiles_m, tiles_n, k_tiles;  // tiles_m counts 256-row pair tiles
  int raster;                     // row tiles per group of the tile order (tile_coords)
  Sched sched;
  float* sk_part;                  // [sk_tiles·sk_split][256][256] partial tiles
  int* sk_cnt;                     // [sk_tiles·16] arrival counters, zero between launches
  int batch;                       // independent matrices; tile t belongs to matrix t / (tiles_m·tiles_n)
  // grouped launch (groups > 1, a kernel built for that): tiles g_tile0[g] .. g_tile0[g+1]−1 belong
  // to problem g — its own operand maps, output g_C[g] (row stride g_ldc[g]) of g_M[g] × g_N[g] in
  // g_tiles_m[g] × g_tiles_n[g] tiles; every problem has the same K
  int groups;
  int g_tile0[GEMM_MAX_GROUPS + 1];
  int g_M[GEMM_MAX_GROUPS], g_N[GEMM_MAX_GROUPS], g_tiles_m[GEMM_MAX_GROUPS], g_tiles_n[GEMM_MAX_GROUPS];
  int g_ldc[GEMM_MAX_GROUPS];
  void* g_C[GEMM_MAX_GROUPS];
  long long c_bstride, aux_bstride;  // elements between consecutive matrices of C and aux
  float alpha, beta;               // GPT_EPI_AXPBY
  const float* dq_a;               // e4m3 operands: device dequantisation factors (else null)
  const float* dq_b;
  void* C;
  int ldc;
  void* C2;
  const uint16_t* aux;
  int ldaux;
  int* status;
  CeArgs ce;
  // head-major outputs (EPI_BF16_HEADS, EPI_QKV_ROPE + Dh); Hkv key/value heads (QKV)
  int T, H, Dh, d, Hkv;
  // QKV: destination of q, k, v — [B][heads][ts][Dh]; row m = b·T + t has RoPE position t + t_off,
  // q is written at position t (q_ts ≥ T), k and v at t + t_off (kv_ts ≥ T + t_off: a cache)
  uint16_t* qkv_dst[3];
  int qkv_ts[3];
  int t_off;
  const float* cs;        // [T, Dh/2, 2] cos / sin
  float* rho_q;           // [M, H]
  float* rho_k;
  // EPI_BF16_HEADS (optional, dl_pad != null): the attention backward's per-row scratch for the
  // dO just stored — delta = rowsum(dO∘O) from the bf16-rounded dO and LSE·log2 e — at row
  // (b·H + h)·Tpad + t of [2][B·H·Tpad]
  const uint16_t* dl_o;   // o, token-major: (b, h, t, j) at b·dl_sb + h·Dh + t·dl_st + j
  long long dl_sb, dl_st;
  const float* dl_lse;    // [B, H, T]
  float* dl_pad;
  int dl_Tpad;
  long long dl_rows;      // B·H·Tpad
};

// Operand maps of the NG problems of one launch (NG = 1: an ordinary or batched GEMM).
template <int NG>
struct GemmMaps {
  CUtensorMap a[NG];
  CUtensorMap b[NG];
};

// Output tile t of the launch → problem g, matrix bb of a batch, pair-tile row tm and column tn.
template <int NG>
__device__ __forceinline__ void decode_tile(const GemmArgs& a, int t, int& g, int& bb, int& tm, int& tn) {
  if constexpr (NG == 1) {
    const int per_mat = a.tiles_m * a.tiles_n;
    g = 0;
    bb = t / per_mat;
    tile_coords(t - bb * per_mat, a.tiles_m, a.tiles_n, a.raster, tm, tn);
  } else {
    g = 0;
#pragma unroll
    for (int i = 1; i < NG; ++i) g += (i < a.groups && t >= a.g_tile0[i]) ? 1 : 0;
    bb = 0;
    tile_coords(t - a.g_tile0[g], a.g_tiles_m[g], a.g_tiles_n[g], 1, tm, tn);
  }
}

struct GemmShape {
  static constexpr int A_BYTES = BM * BK * 2;        // 16 KB
  static constexpr int B_BYTES = (BN / 2) * BK * 2;  // 16 KB
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = 6;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
};

__device__ __forceinline__ bool j0_end_of_head(int n0, int Dh) { return (n0 % Dh) + 32 == Dh; }

// ------------------------------------------------------------------------------------------------
// epilogue: one thread owns row m, columns n0 .. n0+31 of the tile (32 fp32 values in v)
// ------------------------------------------------------------------------------------------------
// With use_pre, `pre` holds the 32 bf16 values of the residual (RESID) or of the saved activation
// (DRELU2) at (m, n0 ..), loaded ahead of the accumulator; otherwise they are loaded here.
template <int EPI>
__device__ __forceinline__ void epilogue_store(const GemmArgs& a, int b, int m, int n0, const float* v,
                                               bool use_pre, const uint4 (&pre)[4]) {
  const bool full = (n0 + 32 <= a.N);
  if (EPI == GPT_EPI_AXPBY) {
    // C = alpha·acc + beta·aux (bf16); aux is not read when beta = 0
    uint16_t* c = reinterpret_cast<uint16_t*>(a.C) + b * a.c_bstride + (size_t)m * a.ldc + n0;
    const uint16_t* x = a.aux + b * a.aux_bstride + (size_t)m * a.ldaux + n0;
    const bool rd = a.beta != 0.f;
    // 8-bit operands: the accumulator is in units of (1/scale_a)·(1/scale_b)
    const float al = a.dq_a ? a.alpha * (*a.dq_a) * (*a.dq_b) : a.alpha;
    if (full) {
#pragma unroll
      for (int j = 0; j < 32; j += 8) {
        float w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = al * v[j + e];
        if (rd) {
          const uint4 p = *reinterpret_cast<const uint4*>(x + j);
          const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            w[2 * e] = fmaf(a.beta, bf_lo(pw[e]), w[2 * e]);
            w[2 * e + 1] = fmaf(a.beta, bf_hi(pw[e]), w[2 * e + 1]);
          }
        }
        uint4 o;
        o.x = pack_bf2(w[0], w[1]); o.y = pack_bf2(w[2], w[3]);
        o.z = pack_bf2(w[4], w[5]); o.w = pack_bf2(w[6], w[7]);
        *reinterpret_cast<uint4*>(c + j) = o;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (n0 + j >= a.N) continue;
        float w = al * v[j];
        if (rd) w = fmaf(a.beta, bf2f(x[j]), w);
        c[j] = f2bf(w);
      }
    }
    return;
  }
  if (EPI == GPT_EPI_F32 || EPI == GPT_EPI_F32_ADD) {
    float* c = reinterpret_cast<float*>(a.C) + b * a.c_bstride + (size_t)m * a.ldc + n0;
    if (full) {
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        float4 o = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        if (EPI == GPT_EPI_F32_ADD) {
          float4 p = *reinterpret_cast<const float4*>(c + j);
          o.x += p.x; o.y += p.y; o.z += p.z; o.w += p.w;
        }
        *reinterpret_cast<float4*>(c + j) = o;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (n0 + j < a.N) c[j] = (EPI == GPT_EPI_F32_ADD) ? c[j] + v[j] : v[j];
    }
    return;
  }
  uint16_t* c = reinterpret_cast<uint16_t*>(a.C) + b * a.c_bstride + (size_t)m * a.ldc + n0;
  if (EPI == GPT_EPI_BF16 || EPI == GPT_EPI_RESID || EPI == GPT_EPI_DRELU2) {
    const uint16_t* x = nullptr;
    if (EPI == GPT_EPI_RESID) x = c;
    if (EPI == GPT_EPI_DRELU2) x = a.aux + b * a.aux_bstride + (size_t)m * a.ldaux + n0;
    if (full) {
#pragma unroll
      for (int j = 0; j < 32; j += 8) {
        float w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = v[j + e];
        if (EPI != GPT_EPI_BF16) {
          const uint4 p = use_pre ? pre[j / 8] : *reinterpret_cast<const uint4*>(x + j);
          const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float lo = bf_lo(pw[e]), hi = bf_hi(pw[e]);
            if (EPI == GPT_EPI_RESID) { w[2 * e] += lo; w[2 * e + 1] += hi; }
            else { w[2 * e] *= 2.f * sqrt_approx(lo); w[2 * e + 1] *= 2.f * sqrt_approx(hi); }
          }
        }
        uint4 o;
        o.x = pack_bf2(w[0], w[1]); o.y = pack_bf2(w[2], w[3]);
        o.z = pack_bf2(w[4], w[5]); o.w = pack_bf2(w[6], w[7]);
        *reinterpret_cast<uint4*>(c + j) = o;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (n0 + j >= a.N) continue;
        float w = v[j];
        if (EPI == GPT_EPI_RESID) w += bf2f(x[j]);
        if (EPI == GPT_EPI_DRELU2) w *= 2.f * sqrt_approx(bf2f(x[j]));
        c[j] = f2bf(w);
      }
    }
    return;
  }
  if (EPI == GPT_EPI_RELU2) {
    // only h = max(u,0)² is stored: the next GEMM's operand, and (as √h = max(u,0)) all the
    // backward needs
    if (full) {
#pragma unroll
      for (int j = 0; j < 32; j += 8) {
        float r[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = fmaxf(v[j + e], 0.f);
        uint4 o;
        o.x = pack_bf2(r[0] * r[0], r[1] * r[1]); o.y = pack_bf2(r[2] * r[2], r[3] * r[3]);
        o.z = pack_bf2(r[4] * r[4], r[5] * r[5]); o.w = pack_bf2(r[6] * r[6], r[7] * r[7]);
        *reinterpret_cast<uint4*>(c + j) = o;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (n0 + j >= a.N) continue;
        const float r = fmaxf(v[j], 0.f);
        c[j] = f2bf(r * r);
      }
    }
  }
}

template <int EPI>
__device__ __forceinline__ void epilogue_store(const GemmArgs& a, int b, int m, int n0, const float* v) {
  const uint4 none[4] = {};
  epilogue_store<EPI>(a, b, m, n0, v, false, none);
}

// Epilogues that write each accumulator element on its own (bf16 cast, residual add, ReLU²,
// dReLU², fp32 store / add, axpby): these are the ones whose tiles may be split along K.
template <int EPI>
constexpr bool epi_plain() {
  return EPI == GPT_EPI_BF16 || EPI == GPT_EPI_RESID || EPI == GPT_EPI_RELU2 ||
         EPI == GPT_EPI_DRELU2 || EPI == GPT_EPI_F32 || EPI == GPT_EPI_F32_ADD || EPI == GPT_EPI_AXPBY;
}

// One epilogue warp's share of a work unit: rows 32q .. 32q+31 of this CTA's 128, columns
// 128·half .. +127 of the tile.  Waits for the accumulator (`tfull`), then either stores the tile
// (a whole-K unit) or, for a piece of a split tile, publishes its partial sums and — if it is the last
// piece of the tile to arrive — adds all pieces in ascending K order and stores the sum.
// Returns false if the wait gave up.
template <int EPI>
__device__ __forceinline__ bool plain_epilogue(const GemmArgs& a, const Work& w, int bb, int m, int tn,
                                               uint32_t tm_addr, uint32_t rank, int q, int half,
                                               int lane, uint64_t* tfull, uint32_t parity,
                                               volatile int* abort_flag) {
  constexpr int NC = BN / 32 / 2;  // 32-column chunks per thread
  const Sched& sch = a.sched;
  const bool piece = w.piece >= 0;
  const int nbase = tn * BN + half * (BN / 2);
  constexpr bool kPre = (EPI == GPT_EPI_RESID || EPI == GPT_EPI_DRELU2);
  // The residual / saved activation does not depend on the accumulator: chunk 0 is fetched before
  // the wait for the tile, and chunk c+1 before chunk c is read from tensor memory, so that one
  // 64-byte row segment per thread is always in flight (within the epilogue warps' registers).  Two
  // buffers alternate, chunk pairs per loop trip, so no register copy waits on a load in flight.
  const bool pre_ok = kPre && !piece && m < a.M;
  uint4 bufa[4], bufb[4];
  auto fetch = [&](int c, uint4 (&dst)[4]) {
    const int n0 = nbase + 32 * c;
    if (pre_ok && n0 + 32 <= a.N) {
      const uint16_t* src = (EPI == GPT_EPI_RESID)
                                ? reinterpret_cast<const uint16_t*>(a.C) + bb * a.c_bstride + (size_t)m * a.ldc + n0
                                : a.aux + bb * a.aux_bstride + (size_t)m * a.ldaux + n0;
#pragma unroll
      for (int e = 0; e < 4; ++e) dst[e] = *reinterpret_cast<const uint4*>(src + 8 * e);
    }
  };
  if (kPre) fetch(0, bufa);
  if (!mbar_wait_warp(tfull, parity, abort_flag, a.status)) return false;
  tc_fence_after();
  const uint32_t t0 = tm_addr + half * (BN / 2);
  if (!piece) {
    auto chunk = [&](int c, const uint4 (&pre)[4]) {
      uint32_t r[32];
      tmem_ld32(t0 + 32 * c, r);
      tmem_ld_wait();
      const int n0 = nbase + 32 * c;
      const bool use_pre = pre_ok && n0 + 32 <= a.N;
      if (m < a.M && n0 < a.N)
        epilogue_store<EPI>(a, bb, m, n0, reinterpret_cast<const float*>(r), use_pre, pre);
    };
    static_assert(NC % 2 == 0, "chunk pairs");
#pragma unroll 1
    for (int c = 0; c < NC; c += 2) {
      if (kPre) fetch(c + 1, bufb);
      chunk(c, bufa);
      if (kPre && c + 2 < NC) fetch(c + 2, bufa);
      chunk(c + 1, bufb);
    }
    return true;
  }
  // ---- piece of a split tile ----
  const int st = w.tile - sch.dp_tiles;
  const int nseg = sch.sk_split, seg = w.piece;
  const size_t row_off = (size_t)(rank * BM + q * 32 + lane) * BN + half * (BN / 2);
  float* mine = a.sk_part + (size_t)(st * nseg + seg) * SK_SLOT_FLOATS + row_off;
#pragma unroll 1
  for (int c = 0; c < NC; ++c) {
    uint32_t r[32];
    tmem_ld32(t0 + 32 * c, r);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      *reinterpret_cast<uint4*>(mine + 32 * c + j) = make_uint4(r[j], r[j + 1], r[j + 2], r[j + 3]);
  }
  __threadfence();
  __syncwarp();
  int* cnt = a.sk_cnt + st * SK_WARPS_PER_TILE + (int)rank * 8 + half * 4 + q;
  int old = 0;
  if (lane == 0) old = atomicAdd(cnt, 1);
  old = __shfl_sync(0xffffffffu, old, 0);
  if (old != nseg - 1) return true;
  // last piece: every other piece's partial is visible; sum in ascending K (= slot) order
  __threadfence();
  const float* slot0 = a.sk_part + (size_t)st * nseg * SK_SLOT_FLOATS + row_off;
#pragma unroll 1
  for (int c = 0; c < NC; ++c) {
    uint32_t r[32];
    tmem_ld32(t0 + 32 * c, r);
    tmem_ld_wait();
    float v[32];
#pragma unroll 1
    for (int sgi = 0; sgi < nseg; ++sgi) {
      if (sgi == seg) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = (sgi == 0) ? __uint_as_float(r[j]) : v[j] + __uint_as_float(r[j]);
      } else {
        const float4* src = reinterpret_cast<const float4*>(slot0 + (size_t)sgi * SK_SLOT_FLOATS + 32 * c);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 p = __ldcg(src + j);
          if (sgi == 0) {
            v[4 * j] = p.x; v[4 * j + 1] = p.y; v[4 * j + 2] = p.z; v[4 * j + 3] = p.w;
          } else {
            v[4 * j] += p.x; v[4 * j + 1] += p.y; v[4 * j + 2] += p.z; v[4 * j + 3] += p.w;
          }
        }
      }
    }
    const int n0 = nbase + 32 * c;
    if (m < a.M && n0 < a.N) epilogue_store<EPI>(a, bb, m, n0, v);
  }
  if (lane == 0) atomicExch(cnt, 0);  // ready for the next launch
  return true;
}

// ------------------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------------------
// F8: A and B are e4m3 (one byte per element): a k-tile is 128 elements (the same 128-byte rows as
// 64 bf16), one MMA instruction covers K = 32, and the accumulator is scaled in the epilogue.
// NG > 1: a grouped launch of NG problems (plain epilogues only), see GemmArgs::groups.
template <bool A_MN, bool B_MN, int EPI, bool F8 = false, int NG = 1>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(gemm_threads<EPI>(), 1)
    gemm_kernel(const __grid_constant__ GemmMaps<NG> maps, const GemmArgs args) {
  static_assert(NG == 1 || epi_plain<EPI>(), "grouped launches use the plain epilogues");
  constexpr int KE = F8 ? 2 * BK : BK;  // elements per k-tile
  using S = GemmShape;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::STAGES * S::STAGE_BYTES);
  uint64_t* empty = full + S::STAGES;
  uint64_t* tfull = empty + S::STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();  // 0 = leader (issues the MMAs), 1 = peer
  const bool leader = (rank == 0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * 128 * gemm_col_groups<EPI>());  // epilogue threads of both CTAs
    }
    *abort_flag = 0;
    fence_mbar_init();
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      tma_prefetch_desc(&maps.a[g]);
      tma_prefetch_desc(&maps.b[g]);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, S::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // inputs written by the preceding kernel are visible from here on
  pdl_trigger();

  const int pair = blockIdx.x >> 1;
  const Sched& sch = args.sched;

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      WorkIter it(sch, pair);
      Work w;
      while (it.next(sch, w)) {
        int g, bb, tm, tn;
        decode_tile<NG>(args, w.tile, g, bb, tm, tn);
        const CUtensorMap* tmA = &maps.a[g];
        const CUtensorMap* tmB = &maps.b[g];
        const int kt0 = w.k0, kt1 = w.k1;
        const int arow = tm * 2 * BM + rank * BM;        // this CTA's 128 rows of A
        const int brow = tn * BN + rank * (BN / 2);      // this CTA's 128 rows of B
        bool ok = true;
        for (int kt = kt0; kt < kt1; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, args.status)) { ok = false; break; }
          uint8_t* sa = smem + stage * S::STAGE_BYTES;
          uint8_t* sb = sa + S::A_BYTES;
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * S::STAGE_BYTES);
          const int k0 = kt * KE;
          if (!A_MN) {
            tma_load_3d_pair(sa, tmA, &full[stage], k0, arow, bb);
          } else {
#pragma unroll
            for (int c = 0; c < BM / 64; ++c)
              tma_load_3d_pair(sa + c * 8192, tmA, &full[stage], arow + c * 64, k0, bb);
          }
          if (!B_MN) {
            tma_load_3d_pair(sb, tmB, &full[stage], k0, brow, bb);
          } else {
#pragma unroll
            for (int c = 0; c < (BN / 2) / 64; ++c)
              tma_load_3d_pair(sb + c * 8192, tmB, &full[stage], brow + c * 64, k0, bb);
          }
          if (++stage == S::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader CTA): the warp runs the loop, one elected lane issues ----------------
    if (leader) {
      constexpr uint32_t idesc = F8 ? idesc_e4m3(2 * BM, BN) : idesc_bf16(2 * BM, BN, A_MN, B_MN);
      // stage-0 descriptors; stage s and slice kk are constant byte offsets from them
      const uint32_t s0 = smem_u32(smem);
      const uint64_t a_desc0 = A_MN ? sdesc_sw128(s0, 8192, 1024) : sdesc_sw128(s0, 16, 1024);
      const uint64_t b_desc0 = B_MN ? sdesc_sw128(s0 + S::A_BYTES, 8192, 1024)
                                    : sdesc_sw128(s0 + S::A_BYTES, 16, 1024);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      WorkIter it(sch, pair);
      Work w;
      while (it.next(sch, w)) {
        const int kt0 = w.k0, kt1 = w.k1;
        if (!mbar_wait_warp(&tempty[acc], acc_phase ^ 1, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        bool ok = true;
        for (int kt = kt0; kt < kt1; ++kt) {
          if (!mbar_wait_warp(&full[stage], phase, abort_flag, args.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = sdesc_add(a_desc0, stage * S::STAGE_BYTES);
          const uint64_t bd = sdesc_add(b_desc0, stage * S::STAGE_BYTES);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              if constexpr (F8) {
                mma_e4m3_pair(d_tmem, sdesc_add(ad, kk * 32), sdesc_add(bd, kk * 32), idesc,
                              (kt > kt0 || kk > 0) ? 1u : 0u);
              } else {
                mma_bf16_pair(d_tmem, sdesc_add(ad, A_MN ? kk * 2048 : kk * 32),
                              sdesc_add(bd, B_MN ? kk * 2048 : kk * 32), idesc,
                              (kt > kt0 || kk > 0) ? 1u : 0u);
              }
            }
            tc_commit_pair(&empty[stage], 0x3);
          }
          __syncwarp();
          if (++stage == S::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (elect_one()) tc_commit_pair(&tfull[acc], 0x3);
        __syncwarp();
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
    }
  } else {
    // ---------------- epilogue warps (both CTAs): lane quarter q, column half `half` ----------------
    const int q = warp & 3;
    constexpr int G = gemm_col_groups<EPI>();
    const int half = (warp - 2) >> 2;  // column group
    const int row_in_tile = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    WorkIter it(sch, pair);
    Work w;
    while (it.next(sch, w)) {
      int g, bb, tm, tn;
      decode_tile<NG>(args, w.tile, g, bb, tm, tn);
      const int m = tm * 2 * BM + rank * BM + row_in_tile;
      if constexpr (epi_plain<EPI>()) {
        bool ok_tile;
        if constexpr (NG == 1) {
          ok_tile = plain_epilogue<EPI>(args, w, bb, m, tn, tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN,
                                        rank, q, half, lane, &tfull[acc], acc_phase, abort_flag);
        } else {
          GemmArgs ga = args;  // problem g's output
          ga.M = args.g_M[g];
          ga.N = args.g_N[g];
          ga.C = args.g_C[g];
          ga.ldc = args.g_ldc[g];
          ok_tile = plain_epilogue<EPI>(ga, w, 0, m, tn, tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN,
                                        rank, q, half, lane, &tfull[acc], acc_phase, abort_flag);
        }
        if (!ok_tile) break;
        tc_fence_before();
        mbar_arrive_leader(&tempty[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
        continue;
      }
      if (!mbar_wait_warp(&tfull[acc], acc_phase, abort_flag, args.status)) break;
      tc_fence_after();
      float run_max = -INFINITY, run_sum = 0.f;
      int tgt = -1;
      float lse_m = 0.f, scale = 0.f;
      if (EPI == EPI_CE_STATS || EPI == EPI_CE_GRAD) {
        if (m < args.M) {
          tgt = args.ce.targets[m] - args.ce.n_offset;
          if (EPI == EPI_CE_GRAD) {
            lse_m = args.ce.lse[m];
            scale = (args.ce.targets[m] >= 0) ? *args.ce.inv_n : 0.f;
          }
        }
      }
      if constexpr (EPI > EPI_QKV_ROPE) {
        // one head (DH columns) at a time: q and k heads get RoPE + QK-norm, v heads a plain cast.
        // Two passes over tensor memory keep at most 64 values per thread in registers: the sum of
        // squares first (rotation preserves it), then the rotation pairs (j, j + DH/2) 32 at a time.
        constexpr int DH = EPI - EPI_QKV_ROPE, HALF = DH / 2;
        const int dkv = args.Hkv * DH;
        const int b = m / args.T, tl = m % args.T, t = tl + args.t_off;  // local row, position
        const bool row_ok = m < args.M;
#pragma unroll 1
        for (int hh = half * (BN / DH / G); hh < (half + 1) * (BN / DH / G); ++hh) {
          const int n_head = tn * BN + hh * DH;
          if (n_head >= args.N) continue;  // the same for every lane of the warp
          const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + hh * DH;
          // columns: q (H heads) | k (Hkv heads) | v (Hkv heads)
          const int region = n_head < args.d ? 0 : (n_head < args.d + dkv ? 1 : 2);
          const int h = (n_head - (region == 0 ? 0 : args.d + (region - 1) * dkv)) / DH;
          const int nh = region == 0 ? args.H : args.Hkv;  // heads of this region
          uint16_t* dst = args.qkv_dst[region] +
                          (((long long)b * nh + h) * args.qkv_ts[region] + (region == 0 ? tl : t)) * DH;
          auto store32 = [&](int col, const float* w) {
            if (!row_ok) return;
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              uint4 o;
              o.x = pack_bf2(w[j], w[j + 1]);
              o.y = pack_bf2(w[j + 2], w[j + 3]);
              o.z = pack_bf2(w[j + 4], w[j + 5]);
              o.w = pack_bf2(w[j + 6], w[j + 7]);
              *reinterpret_cast<uint4*>(dst + col + j) = o;
            }
          };
          if (region == 2) {
#pragma unroll 1
            for (int c = 0; c < DH / 32; ++c) {
              uint32_t r[32];
              tmem_ld32(tb + 32 * c, r);
              tmem_ld_wait();
              store32(32 * c, reinterpret_cast<const float*>(r));
            }
            continue;
          }
          float ss = 0.f;
#pragma unroll 1
          for (int c = 0; c < DH / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tb + 32 * c, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) ss = fmaf(__uint_as_float(r[j]), __uint_as_float(r[j]), ss);
          }
          const float rr = rsqrtf(ss / (float)DH + 1e-6f);
          float* rho = region == 0 ? args.rho_q : args.rho_k;
          if (row_ok && rho) rho[(size_t)m * nh + h] = rr;
          const float4* cs4 = reinterpret_cast<const float4*>(args.cs + (size_t)(row_ok ? t : 0) * DH);
          constexpr int PC = HALF < 32 ? HALF : 32;  // rotation pairs per pass
#pragma unroll 1
          for (int p0 = 0; p0 < HALF; p0 += PC) {
            uint32_t ra[32], rb[32];
            float wa[32], wb[32];
            if constexpr (HALF >= 32) {
              tmem_ld32(tb + p0, ra);
              tmem_ld32(tb + HALF + p0, rb);
            } else {
              tmem_ld32(tb, ra);  // DH = 32: one load holds both halves
#pragma unroll
              for (int j = 0; j < PC; ++j) rb[j] = ra[HALF + j];
            }
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < PC; j += 2) {
              const float4 w = cs4[(p0 + j) / 2];  // cos_j, sin_j, cos_{j+1}, sin_{j+1}
              const float a0 = __uint_as_float(ra[j]), b0 = __uint_as_float(rb[j]);
              const float a1 = __uint_as_float(ra[j + 1]), b1 = __uint_as_float(rb[j + 1]);
              wa[j] = (a0 * w.x - b0 * w.y) * rr;
              wb[j] = (a0 * w.y + b0 * w.x) * rr;
              wa[j + 1] = (a1 * w.z - b1 * w.w) * rr;
              wb[j + 1] = (a1 * w.w + b1 * w.z) * rr;
            }
            if constexpr (HALF >= 32) {
              store32(p0, wa);
              store32(HALF + p0, wb);
            } else {
              float wf[32];
#pragma unroll
              for (int j = 0; j < PC; ++j) {
                wf[j] = wa[j];
                wf[HALF + j] = wb[j];
              }
              store32(0, wf);
            }
          }
        }
      } else {
      float dl_dot = 0.f;  // EPI_BF16_HEADS with the fused delta: rowsum(dO∘O) of the current head
#pragma unroll 1
      for (int c = half * (BN / 32 / G); c < (half + 1) * (BN / 32 / G); ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + c * 32, r);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        const int n0 = tn * BN + c * 32;
        if (EPI == EPI_CE_STATS) {
          if (m < args.M) {
            float cm = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n0 + j < args.N) cm = fmaxf(cm, v[j]);
            const float nm = fmaxf(run_max, cm);
            float sacc = (run_max == -INFINITY) ? 0.f : run_sum * __expf(run_max - nm);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n0 + j < args.N) sacc += __expf(v[j] - nm);
            run_max = nm;
            run_sum = sacc;
            if (tgt >= n0 && tgt < n0 + 32 && tgt < args.N) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (n0 + j == tgt) args.ce.ztarget[m] = v[j];
            }
          }
        } else if (EPI == EPI_CE_GRAD) {
          if (m < args.M && n0 < args.N) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float p = __expf(v[j] - lse_m);
              v[j] = (p - ((n0 + j == tgt) ? 1.f : 0.f)) * scale;
            }
            epilogue_store<GPT_EPI_BF16>(args, 0, m, n0, v);
          }
        } else if (EPI == EPI_BF16_HEADS) {
          if (m < args.M && n0 < args.N) {
            const int b = m / args.T, t = m % args.T, h = n0 / args.Dh, j0 = n0 % args.Dh;
            uint16_t* dst = reinterpret_cast<uint16_t*>(args.C) +
                            (((long long)b * args.H + h) * args.T + t) * args.Dh + j0;
            const uint16_t* orow = args.dl_pad ? args.dl_o + b * args.dl_sb + (long long)h * args.Dh +
                                                     (long long)t * args.dl_st + j0
                                               : nullptr;
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              uint4 o;
              o.x = pack_bf2(v[j], v[j + 1]);
              o.y = pack_bf2(v[j + 2], v[j + 3]);
              o.z = pack_bf2(v[j + 4], v[j + 5]);
              o.w = pack_bf2(v[j + 6], v[j + 7]);
              *reinterpret_cast<uint4*>(dst + j) = o;
              if (orow) {  // delta from the dO values as stored
                const uint4 x = *reinterpret_cast<const uint4*>(orow + j);
                dl_dot += bf_lo(o.x) * bf_lo(x.x) + bf_hi(o.x) * bf_hi(x.x) + bf_lo(o.y) * bf_lo(x.y) +
                          bf_hi(o.y) * bf_hi(x.y) + bf_lo(o.z) * bf_lo(x.z) + bf_hi(o.z) * bf_hi(x.z) +
                          bf_lo(o.w) * bf_lo(x.w) + bf_hi(o.w) * bf_hi(x.w);
              }
            }
            if (orow && j0 + 32 == args.Dh) {  // the head's last chunk: its scratch row
              const long long r = ((long long)b * args.H + h) * args.dl_Tpad + t;
              const float l = args.dl_lse[((long long)b * args.H + h) * args.T + t];
              args.dl_pad[r] = l * 1.4426950408889634f;
              args.dl_pad[args.dl_rows + r] = dl_dot;
            }
          }
          if (j0_end_of_head(n0, args.Dh)) dl_dot = 0.f;
        } else {
          if (m < args.M && n0 < args.N) epilogue_store<EPI>(args, 0, m, n0, v);
        }
      }
      }
      if (EPI == EPI_CE_STATS && m < args.M && tn * BN + half * (BN / G) < args.N) {
        args.ce.stats[(size_t)m * args.ce.stats_ld + args.ce.stats_col0 + G * tn + half] =
            make_float2(run_max, run_sum);
      }
      tc_fence_before();
      mbar_arrive_leader(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  __syncwarp();
  // After an expired wait, give copies and MMAs already in flight time to land before the shared
  // and tensor memory they target is released.
  if (*abort_flag && threadIdx.x == 0) {
    for (int i = 0; i < 2000; ++i) __nanosleep(1000);
  }
  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its partner may still signal or read it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
}

// ------------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------------
template <bool A_MN, bool B_MN, int EPI, bool F8 = false>
static gpt_status launch_inst(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& a,
                              cudaStream_t stream) {
  using S = GemmShape;
  auto kern = gemm_kernel<A_MN, B_MN, EPI, F8, 1>;
  GPT_TRY(ensure_smem(kern, S::SMEM_BYTES));
  GemmMaps<1> maps;
  maps.a[0] = ma;
  maps.b[0] = mb;
  return launch_kernel(kern, dim3(2 * a.sched.num_pairs), dim3(gemm_threads<EPI>()), S::SMEM_BYTES,
                       stream, maps, a);
}

template <bool A_MN, bool B_MN>
static gpt_status dispatch_epi(int epi, const CUtensorMap& ma, const CUtensorMap& mb,
                               const GemmArgs& a, cudaStream_t s) {
  switch (epi) {
    case GPT_EPI_BF16: return launch_inst<A_MN, B_MN, GPT_EPI_BF16>(ma, mb, a, s);
    case GPT_EPI_RESID: return launch_inst<A_MN, B_MN, GPT_EPI_RESID>(ma, mb, a, s);
    case GPT_EPI_RELU2: return launch_inst<A_MN, B_MN, GPT_EPI_RELU2>(ma, mb, a, s);
    case GPT_EPI_DRELU2: return launch_inst<A_MN, B_MN, GPT_EPI_DRELU2>(ma, mb, a, s);
    case GPT_EPI_F32: return launch_inst<A_MN, B_MN, GPT_EPI_F32>(ma, mb, a, s);
    case GPT_EPI_F32_ADD: return launch_inst<A_MN, B_MN, GPT_EPI_F32_ADD>(ma, mb, a, s);
    case GPT_EPI_AXPBY: return launch_inst<A_MN, B_MN, GPT_EPI_AXPBY>(ma, mb, a, s);
    default: return GPT_ERR_INVALID_ARG;
  }
}

// Operand map for one CTA's half of a pair tile, over `batch` matrices `bstride` elements apart
// (third map dimension): K-major [rows, K] with box {64, 128, 1}; MN-major [K rows, MN cols] with
// box {64, 64, 1}.
static bool make_operand_map(CUtensorMap* map, const void* base, bool mn_major, int mn, int K,
                             int ld, int batch = 1, long long bstride = 0) {
  uint64_t dims[3], strides[2];
  uint32_t box[3];
  strides[0] = (uint64_t)ld * 2;
  const uint64_t outer = mn_major ? (uint64_t)K : (uint64_t)mn;
  // a single matrix still gets a valid (unused) stride for the third dimension
  strides[1] = batch > 1 ? (uint64_t)bstride * 2 : ((strides[0] * outer + 15) & ~(uint64_t)15);
  if (!mn_major) {
    dims[0] = (uint64_t)K; dims[1] = (uint64_t)mn;
    box[0] = 64; box[1] = 128;
  } else {
    dims[0] = (uint64_t)mn; dims[1] = (uint64_t)K;
    box[0] = 64; box[1] = 64;
  }
  dims[2] = (uint64_t)batch;
  box[2] = 1;
  return encode_map_bf16(map, base, 3, dims, strides, box, true);
}

static gpt_status check_gemm_args(int op, int M, int N, int K, const void* A, int lda, const void* B,
                                  int ldb, void* C, int ldc) {
  if (!A || !B || !C) return GPT_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return GPT_ERR_INVALID_ARG;
  if (op < GPT_GEMM_NT || op > GPT_GEMM_TN) return GPT_ERR_INVALID_ARG;
  const int a_inner = (op == GPT_GEMM_TN) ? M : K;
  const int b_inner = (op == GPT_GEMM_NT) ? K : N;
  if (lda < a_inner || ldb < b_inner || ldc < N) return GPT_ERR_INVALID_ARG;
  if ((lda % 8) || (ldb % 8) || (ldc % 8)) return GPT_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B) |
       reinterpret_cast<uintptr_t>(C)) & 15)
    return GPT_ERR_UNSUPPORTED_SHAPE;
  return GPT_OK;
}

// Tiles and the plain round-robin schedule (every tile whole, one CTA pair per tile up to the SM
// count).
static gpt_status fill_args(GemmArgs& a, int M, int N, int K, int batch = 1, int k_per_tile = BK) {
  int sms = 0;
  GPT_TRY(device_info(&sms));
  a.M = M; a.N = N; a.K = K;
  a.tiles_m = (M + 2 * BM - 1) / (2 * BM);
  a.tiles_n = (N + BN - 1) / BN;
  a.k_tiles = (K + k_per_tile - 1) / k_per_tile;
  a.raster = 1;
  a.batch = batch;
  a.alpha = 1.f;
  a.beta = 0.f;
  const long long tiles_ll = (long long)a.tiles_m * a.tiles_n * batch;
  if (tiles_ll > (1ll << 30)) return GPT_ERR_UNSUPPORTED_SHAPE;
  const int tiles = (int)tiles_ll;
  Sched& s = a.sched;
  s = Sched{};
  s.num_pairs = std::max(1, std::min(tiles, sms / 2));
  s.k_tiles = a.k_tiles;
  s.dp_tiles = tiles;
  return GPT_OK;
}

// Split plan for the tail of the tile list, or false when the round-robin schedule is as good.
// Cost model, in k-step times of one CTA pair: round robin takes ⌈tiles/P⌉·k_tiles; the split takes
// ⌊tiles/P⌋·k_tiles + ⌈k_tiles/s⌉ plus the piece exchange, ≈ 8 k-steps per extra piece that the
// last piece reads back (a 128 KB partial per CTA) + 4 for writing its own.  s ≤ P / tail tiles,
// and the split must save at least 5%.
bool plan_stream_k(int tiles, int k_tiles, int pairs, Sched* out) {
  if (pairs < 2 || tiles <= 0 || k_tiles < 2 || tiles % pairs == 0) return false;
  const int waves = tiles / pairs, tail = tiles % pairs;
  const long long rr_cost = (long long)(waves + 1) * k_tiles;
  int best_s = 1;
  long long best = k_tiles;
  for (int sp = 2; sp <= pairs / tail && sp <= k_tiles; ++sp) {
    if (tail > SK_MAX_TILES || (long long)tail * sp > SK_MAX_SLOTS) break;
    const long long c = (k_tiles + sp - 1) / sp + 8 * (sp - 1) + 4;
    if (c < best) { best = c; best_s = sp; }
  }
  if (best_s == 1) return false;
  const long long cost = (long long)waves * k_tiles + best;
  if (100 * cost > 95 * rr_cost) return false;
  Sched s{};
  s.num_pairs = waves > 0 ? pairs : tail * best_s;  // with no whole wave, launch only the pieces
  s.k_tiles = k_tiles;
  s.dp_tiles = waves * pairs;
  s.sk_tiles = tail;
  s.sk_split = best_s;
  *out = s;
  return true;
}

size_t gemm_sk_scratch_bytes() {
  return ((GEMM_SK_COUNTER_BYTES + 255) & ~(size_t)255) +
         (size_t)SK_MAX_SLOTS * SK_SLOT_FLOATS * sizeof(float);
}

gpt_status gemm_launch_batched(const GemmBatch& g, cudaStream_t stream, void* sk_scratch) {
  const int op = g.op, M = g.M, N = g.N, K = g.K;
  int epi = g.epi;
  GPT_TRY(check_gemm_args(op, M, N, K, g.A, g.lda, g.B, g.ldb, g.C, g.ldc));
  if (epi < GPT_EPI_BF16 || epi > GPT_EPI_AXPBY) return GPT_ERR_INVALID_ARG;
  if (epi == GPT_EPI_DRELU2 && (!g.aux || g.ldaux < N || (g.ldaux % 8))) return GPT_ERR_INVALID_ARG;
  if (epi == GPT_EPI_AXPBY && g.beta != 0.f && (!g.aux || g.ldaux < N || (g.ldaux % 8) ||
                                                (reinterpret_cast<uintptr_t>(g.aux) & 15)))
    return GPT_ERR_INVALID_ARG;
  if (g.batch < 1) return GPT_ERR_INVALID_ARG;
  if (g.batch > 1) {
    // matrices must not overlap and their starts must keep 16-byte alignment (TMA)
    const long long a_rows = (op == GPT_GEMM_TN) ? K : M, b_rows = (op == GPT_GEMM_NT) ? N : K;
    if (g.a_bstride < a_rows * g.lda || g.b_bstride < b_rows * g.ldb || g.c_bstride < (long long)M * g.ldc)
      return GPT_ERR_INVALID_ARG;
    if ((g.a_bstride % 8) || (g.b_bstride % 8) || (g.c_bstride % 8)) return GPT_ERR_UNSUPPORTED_SHAPE;
    if (g.aux && ((g.aux_bstride % 8) || g.aux_bstride < (long long)M * g.ldaux)) return GPT_ERR_INVALID_ARG;
  }
  if (reinterpret_cast<uintptr_t>(sk_scratch) & 255) return GPT_ERR_UNSUPPORTED_SHAPE;
  const bool a_mn = (op == GPT_GEMM_TN);
  const bool b_mn = (op != GPT_GEMM_NT);
  CUtensorMap ma, mb;
  if (!make_operand_map(&ma, g.A, a_mn, M, K, g.lda, g.batch, g.a_bstride)) return GPT_ERR_UNSUPPORTED_SHAPE;
  if (!make_operand_map(&mb, g.B, b_mn, N, K, g.ldb, g.batch, g.b_bstride)) return GPT_ERR_UNSUPPORTED_SHAPE;
  GemmArgs a{};
  GPT_TRY(fill_args(a, M, N, K, g.batch));
  a.raster = raster_for(op, N, K);
  a.C = g.C; a.ldc = g.ldc; a.C2 = nullptr;
  a.aux = reinterpret_cast<const uint16_t*>(g.aux); a.ldaux = g.ldaux;
  a.c_bstride = g.batch > 1 ? g.c_bstride : 0;
  a.aux_bstride = g.batch > 1 ? g.aux_bstride : 0;
  a.alpha = g.alpha;
  a.beta = g.beta;
  a.status = g.status;
  if (sk_scratch) {
    int sms = 0;
    GPT_TRY(device_info(&sms));
    Sched sk;
    if (plan_stream_k(a.tiles_m * a.tiles_n * g.batch, a.k_tiles, std::max(1, sms / 2), &sk)) {
      a.sched = sk;
      a.sk_cnt = reinterpret_cast<int*>(sk_scratch);
      a.sk_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sk_scratch) +
                                           ((GEMM_SK_COUNTER_BYTES + 255) & ~(size_t)255));
    }
  }
  if (op == GPT_GEMM_NT) return dispatch_epi<false, false>(epi, ma, mb, a, stream);
  if (op == GPT_GEMM_NN) return dispatch_epi<false, true>(epi, ma, mb, a, stream);
  return dispatch_epi<true, true>(epi, ma, mb, a, stream);
}

gpt_status gemm_group_tn_launch(int n, const GemmTnProblem* p, int K, int epi, int* status,
                                cudaStream_t stream, void* sk_scratch) {
  if (n < 1 || n > GEMM_MAX_GROUPS || !p) return GPT_ERR_INVALID_ARG;
  if (epi != GPT_EPI_F32 && epi != GPT_EPI_F32_ADD) return GPT_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(sk_scratch) & 255) return GPT_ERR_UNSUPPORTED_SHAPE;
  GemmMaps<GEMM_MAX_GROUPS> maps;
  GemmArgs a{};
  long long tiles = 0;
  for (int g = 0; g < n; ++g)  // every argument is checked before any map is encoded
    GPT_TRY(check_gemm_args(GPT_GEMM_TN, p[g].M, p[g].N, K, p[g].A, p[g].lda, p[g].B, p[g].ldb, p[g].C,
                            p[g].ldc));
  for (int g = 0; g < n; ++g) {
    const GemmTnProblem& q = p[g];
    if (!make_operand_map(&maps.a[g], q.A, true, q.M, K, q.lda) ||
        !make_operand_map(&maps.b[g], q.B, true, q.N, K, q.ldb))
      return GPT_ERR_UNSUPPORTED_SHAPE;
    a.g_tile0[g] = (int)tiles;
    a.g_M[g] = q.M;
    a.g_N[g] = q.N;
    a.g_tiles_m[g] = (q.M + 2 * BM - 1) / (2 * BM);
    a.g_tiles_n[g] = (q.N + BN - 1) / BN;
    a.g_C[g] = q.C;
    a.g_ldc[g] = q.ldc;
    tiles += (long long)a.g_tiles_m[g] * a.g_tiles_n[g];
  }
  for (int g = n; g < GEMM_MAX_GROUPS; ++g) maps.a[g] = maps.b[g] = maps.a[0];  // never read
  if (tiles > (1 << 30)) return GPT_ERR_UNSUPPORTED_SHAPE;
  a.g_tile0[n] = (int)tiles;
  a.groups = n;
  int sms = 0;
  GPT_TRY(device_info(&sms));
  // one schedule over the whole tile list (tiles_m / tiles_n / M / N are per problem here)
  a.M = p[0].M; a.N = p[0].N; a.K = K;
  a.tiles_m = a.tiles_n = 1;
  a.k_tiles = (K + BK - 1) / BK;
  a.raster = 1;
  a.batch = 1;
  a.alpha = 1.f;
  a.beta = 0.f;
  a.sched = Sched{};
  a.sched.num_pairs = std::max(1, std::min((int)tiles, sms / 2));
  a.sched.k_tiles = a.k_tiles;
  a.sched.dp_tiles = (int)tiles;
  a.status = status;
  if (sk_scratch) {
    Sched sk;
    if (plan_stream_k((int)tiles, a.k_tiles, std::max(1, sms / 2), &sk)) {
      a.sched = sk;
      a.sk_cnt = reinterpret_cast<int*>(sk_scratch);
      a.sk_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sk_scratch) +
                                           ((GEMM_SK_COUNTER_BYTES + 255) & ~(size_t)255));
    }
  }
  using S = GemmShape;
  auto kern = (epi == GPT_EPI_F32) ? gemm_kernel<true, true, GPT_EPI_F32, false, GEMM_MAX_GROUPS>
                                   : gemm_kernel<true, true, GPT_EPI_F32_ADD, false, GEMM_MAX_GROUPS>;
  GPT_TRY(ensure_smem(kern, S::SMEM_BYTES));
  return launch_kernel(kern, dim3(2 * a.sched.num_pairs), dim3(gemm_threads<GPT_EPI_F32>()),
                       S::SMEM_BYTES, stream, maps, a);
}

gpt_status gemm_launch(int op, int epi, int M, int N, int K, const void* A, int lda, const void* B,
                       int ldb, void* C, int ldc, void* C2, const void* aux, int ldaux, int* status,
                       cudaStream_t stream, void* sk_scratch) {
  (void)C2;
  GemmBatch g{};
  g.op = op; g.epi = epi; g.M = M; g.N = N; g.K = K; g.batch = 1;
  g.A = A; g.lda = lda; g.B = B; g.ldb = ldb; g.C = C; g.ldc = ldc;
  g.aux = aux; g.ldaux = ldaux; g.alpha = 1.f; g.beta = 0.f; g.status = status;
  return gemm_launch_batched(g, stream, sk_scratch);
}

// C[M,N] (bf16) = alpha·dq_a·dq_b·(A·Bᵀ) with A [M,K] and B [N,K] e4m3, K-contiguous (NT).
gpt_status gemm_e4m3_launch(int M, int N, int K, const void* A, int lda, const void* B, int ldb,
                            void* C, int ldc, const float* dq_a, const float* dq_b, float alpha,
                            int* status, cudaStream_t stream, void* sk_scratch) {
  if (!A || !B || !C || !dq_a || !dq_b) return GPT_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || lda < K || ldb < K || ldc < N) return GPT_ERR_INVALID_ARG;
  if ((lda % 16) || (ldb % 16) || (ldc % 8)) return GPT_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B) |
       reinterpret_cast<uintptr_t>(C)) & 15)
    return GPT_ERR_UNSUPPORTED_SHAPE;
  if (reinterpret_cast<uintptr_t>(sk_scratch) & 255) return GPT_ERR_UNSUPPORTED_SHAPE;
  CUtensorMap ma, mb;
  {
    const uint64_t da[3] = {(uint64_t)K, (uint64_t)M, 1}, db[3] = {(uint64_t)K, (uint64_t)N, 1};
    const uint64_t sa[2] = {(uint64_t)lda, ((uint64_t)lda * M + 15) & ~(uint64_t)15};
    const uint64_t sb[2] = {(uint64_t)ldb, ((uint64_t)ldb * N + 15) & ~(uint64_t)15};
    const uint32_t box[3] = {128, 128, 1};
    if (!encode_map_u8(&ma, A, 3, da, sa, box) || !encode_map_u8(&mb, B, 3, db, sb, box))
      return GPT_ERR_UNSUPPORTED_SHAPE;
  }
  GemmArgs a{};
  GPT_TRY(fill_args(a, M, N, K, 1, 2 * BK));
  a.C = C; a.ldc = ldc;
  a.alpha = alpha; a.beta = 0.f;
  a.dq_a = dq_a; a.dq_b = dq_b;
  a.status = status;
  if (sk_scratch) {
    int sms = 0;
    GPT_TRY(device_info(&sms));
    Sched sk;
    if (plan_stream_k(a.tiles_m * a.tiles_n, a.k_tiles, std::max(1, sms / 2), &sk)) {
      a.sched = sk;
      a.sk_cnt = reinterpret_cast<int*>(sk_scratch);
      a.sk_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sk_scratch) +
                                           ((GEMM_SK_COUNTER_BYTES + 255) & ~(size_t)255));
    }
  }
  return launch_inst<false, false, GPT_EPI_AXPBY, true>(ma, mb, a, stream);
}

gpt_status gemm_heads_launch(int op, int M, int N, int K, const void* A, int lda, const void* B,
                             int ldb, void* heads, int T, int H, int Dh, int* status,
                             cudaStream_t stream, const AttnDeltaFusion* fuse) {
  GPT_TRY(check_gemm_args(op, M, N, K, A, lda, B, ldb, heads, N));
  if (T <= 0 || H <= 0 || Dh <= 0 || (Dh % 32) || H * Dh != N || (M % T)) return GPT_ERR_INVALID_ARG;
  const bool a_mn = (op == GPT_GEMM_TN), b_mn = (op != GPT_GEMM_NT);
  CUtensorMap ma, mb;
  if (!make_operand_map(&ma, A, a_mn, M, K, lda)) return GPT_ERR_UNSUPPORTED_SHAPE;
  if (!make_operand_map(&mb, B, b_mn, N, K, ldb)) return GPT_ERR_UNSUPPORTED_SHAPE;
  GemmArgs a{};
  GPT_TRY(fill_args(a, M, N, K));
  a.C = heads; a.ldc = N; a.status = status;
  a.T = T; a.H = H; a.Dh = Dh;
  if (fuse) {
    if (!fuse->o || !fuse->lse || !fuse->pad || fuse->Tpad < T) return GPT_ERR_INVALID_ARG;
    a.dl_o = reinterpret_cast<const uint16_t*>(fuse->o);
    a.dl_sb = fuse->sb_o; a.dl_st = fuse->st_o;
    a.dl_lse = fuse->lse; a.dl_pad = fuse->pad;
    a.dl_Tpad = fuse->Tpad; a.dl_rows = (long long)(M / T) * H * fuse->Tpad;
  }
  if (op == GPT_GEMM_NT) return launch_inst<false, false, EPI_BF16_HEADS>(ma, mb, a, stream);
  if (op == GPT_GEMM_NN) return launch_inst<false, true, EPI_BF16_HEADS>(ma, mb, a, stream);
  return launch_inst<true, true, EPI_BF16_HEADS>(ma, mb, a, stream);
}

gpt_status gemm_qkv_rope_launch(int M, int d, const void* A, const void* Wqkv, void* heads,
                                float* rho_q, float* rho_k, const float* cs, int T, int H, int Dh,
                                int* status, cudaStream_t stream, int Hkv, const QkvDest* dest) {
  if (Hkv <= 0) Hkv = H;
  if (H % Hkv) return GPT_ERR_INVALID_ARG;
  const int N = d + 2 * Hkv * Dh, K = d;
  GPT_TRY(check_gemm_args(GPT_GEMM_NT, M, N, K, A, K, Wqkv, K, dest ? dest->q : heads, N));
  if ((!dest && (!rho_q || !rho_k)) || !cs || T <= 0 || H * Dh != d || (M % T))
    return GPT_ERR_INVALID_ARG;
  if (Dh != 32 && Dh != 64 && Dh != 128) return GPT_ERR_UNSUPPORTED_SHAPE;
  CUtensorMap ma, mb;
  if (!make_operand_map(&ma, A, false, M, K, K)) return GPT_ERR_UNSUPPORTED_SHAPE;
  if (!make_operand_map(&mb, Wqkv, false, N, K, K)) return GPT_ERR_UNSUPPORTED_SHAPE;
  GemmArgs a{};
  GPT_TRY(fill_args(a, M, N, K));
  a.C = heads; a.ldc = N; a.status = status;
  a.T = T; a.H = H; a.Dh = Dh; a.d = d; a.Hkv = Hkv; a.cs = cs; a.rho_q = rho_q; a.rho_k = rho_k;
  if (dest) {
    if (!dest->k || !dest->v || dest->q_ts < T || dest->kv_ts < T + dest->t_off ||
        dest->t_off < 0)
      return GPT_ERR_INVALID_ARG;
    a.qkv_dst[0] = reinterpret_cast<uint16_t*>(dest->q);
    a.qkv_dst[1] = reinterpret_cast<uint16_t*>(dest->k);
    a.qkv_dst[2] = reinterpret_cast<uint16_t*>(dest->v);
    a.qkv_ts[0] = dest->q_ts;
    a.qkv_ts[1] = a.qkv_ts[2] = dest->kv_ts;
    a.t_off = dest->t_off;
  } else {  // q̃, k̃, v one after the other in `heads`
    const long long btd = (long long)(M / T) * T * Dh;
    uint16_t* h0 = reinterpret_cast<uint16_t*>(heads);
    a.qkv_dst[0] = h0;
    a.qkv_dst[1] = h0 + btd * H;
    a.qkv_dst[2] = h0 + btd * (H + Hkv);
    a.qkv_ts[0] = a.qkv_ts[1] = a.qkv_ts[2] = T;
    a.t_off = 0;
  }
  if (Dh == 128) return launch_inst<false, false, EPI_QKV_ROPE + 128>(ma, mb, a, stream);
  if (Dh == 64) return launch_inst<false, false, EPI_QKV_ROPE + 64>(ma, mb, a, stream);
  return launch_inst<false, false, EPI_QKV_ROPE + 32>(ma, mb, a, stream);
}

int gemm_ce_tile_n() { return BN / gemm_col_groups<EPI_CE_STATS>(); }

gpt_status gemm_ce_launch(bool grad, int M, int N, int K, const void* A, int lda, const void* B,
                          int ldb, void* C, int ldc, const CeArgs& ce, int* status,
                          cudaStream_t stream) {
  GPT_TRY(check_gemm_args(GPT_GEMM_NT, M, N, K, A, lda, B, ldb, grad ? C : (void*)A, grad ? ldc : N));
  CUtensorMap ma, mb;
  if (!make_operand_map(&ma, A, false, M, K, lda)) return GPT_ERR_UNSUPPORTED_SHAPE;
  if (!make_operand_map(&mb, B, false, N, K, ldb)) return GPT_ERR_UNSUPPORTED_SHAPE;
  GemmArgs a{};
  GPT_TRY(fill_args(a, M, N, K));
  a.raster = raster_for(GPT_GEMM_NT, N, K);
  a.C = C; a.ldc = ldc;
  a.status = status;
  a.ce = ce;
  if (grad) return launch_inst<false, false, EPI_CE_GRAD>(ma, mb, a, stream);
  return launch_inst<false, false, EPI_CE_STATS>(ma, mb, a, stream);
}

}  // namespace gpt

extern "C" gpt_status gpt_qkv_proj_rope(const void* r, const void* w_qkv, void* heads, float* rho_q,
                                        float* rho_k, const float* cos_sin, int B, int T, int H,
                                        int H_kv, int Dh, int* status, void* stream) {
  if (B <= 0 || T <= 0 || H <= 0 || Dh <= 0 || H_kv <= 0) return GPT_ERR_INVALID_ARG;
  return gpt::gemm_qkv_rope_launch(B * T, H * Dh, r, w_qkv, heads, rho_q, rho_k, cos_sin, T, H, Dh,
                                   status, gpt::as_stream(stream), H_kv);
}

extern "C" size_t gpt_gemm_scratch_bytes(void) { return gpt::gemm_sk_scratch_bytes(); }

extern "C" gpt_status gpt_gemm_e4m3(int M, int N, int K, const void* A, int lda, const void* B,
                                    int ldb, void* C, int ldc, const float* dq_a, const float* dq_b,
                                    float alpha, void* scratch, int* status, void* stream) {
  cudaStream_t s = gpt::as_stream(stream);
  if (scratch) {
    if (reinterpret_cast<uintptr_t>(scratch) & 255) return GPT_ERR_UNSUPPORTED_SHAPE;
    GPT_CUDA_TRY(cudaMemsetAsync(scratch, 0, gpt::GEMM_SK_COUNTER_BYTES, s));
  }
  return gpt::gemm_e4m3_launch(M, N, K, A, lda, B, ldb, C, ldc, dq_a, dq_b, alpha, status, s,
                               scratch);
}

extern "C" gpt_status gpt_gemm_batched(int op, int epilogue, int batch, int M, int N, int K,
                                       const void* A, int lda, long long a_bstride, const void* B,
                                       int ldb, long long b_bstride, void* C, int ldc,
                                       long long c_bstride, const void* aux, int ldaux,
                                       long long aux_bstride, float alpha, float beta,
                                       int* status, void* stream) {
  gpt::GemmBatch g{};
  g.op = op; g.epi = epilogue; g.M = M; g.N = N; g.K = K; g.batch = batch;
  g.A = A; g.lda = lda; g.a_bstride = a_bstride;
  g.B = B; g.ldb = ldb; g.b_bstride = b_bstride;
  g.C = C; g.ldc = ldc; g.c_bstride = c_bstride;
  g.aux = aux; g.ldaux = ldaux; g.aux_bstride = aux_bstride;
  g.alpha = alpha; g.beta = beta; g.status = status;
  if (epilogue != GPT_EPI_AXPBY) { g.alpha = 1.f; g.beta = 0.f; }
  return gpt::gemm_launch_batched(g, gpt::as_stream(stream), nullptr);
}

extern "C" gpt_status gpt_gemm_group_tn(int n, const gpt_gemm_tn_problem* problems, int K, int epilogue,
                                        void* scratch, int* status, void* stream) {
  if (n < 1 || n > gpt::GEMM_MAX_GROUPS || !problems) return GPT_ERR_INVALID_ARG;
  gpt::GemmTnProblem p[gpt::GEMM_MAX_GROUPS];
  for (int g = 0; g < n; ++g) {
    const gpt_gemm_tn_problem& q = problems[g];
    p[g] = gpt::GemmTnProblem{q.M, q.N, q.A, q.lda, q.B, q.ldb, q.C, q.ldc};
  }
  cudaStream_t s = gpt::as_stream(stream);
  if (scratch) {
    if (reinterpret_cast<uintptr_t>(scratch) & 255) return GPT_ERR_UNSUPPORTED_SHAPE;
    GPT_CUDA_TRY(cudaMemsetAsync(scratch, 0, gpt::GEMM_SK_COUNTER_BYTES, s));
  }
  return gpt::gemm_group_tn_launch(n, p, K, epilogue, status, s, scratch);
}

extern "C" gpt_status gpt_gemm(int op, int epilogue, int M, int N, int K, const void* A, int lda,
                               const void* B, int ldb, void* C, int ldc, void* C2,
                               const void* aux, int ldaux, void* scratch, int* status,
                               void* stream) {
  cudaStream_t s = gpt::as_stream(stream);
  if (scratch) {
    // the arrival counters start at zero; every launch leaves them at zero again
    if (reinterpret_cast<uintptr_t>(scratch) & 255) return GPT_ERR_UNSUPPORTED_SHAPE;
    GPT_CUDA_TRY(cudaMemsetAsync(scratch, 0, gpt::GEMM_SK_COUNTER_BYTES, s));
  }
  return gpt::gemm_launch(op, epilogue, M, N, K, A, lda, B, ldb, C, ldc, C2, aux, ldaux, status, s,
                          scratch);
}
