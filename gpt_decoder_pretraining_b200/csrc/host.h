// Host-side helpers shared by the .cu files: CUDA error mapping, device properties, TMA tensor-map
// encoding (through the runtime's driver entry point, so the library does not link libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/gptstep.h"

namespace gpt {

// The CUDA error behind the last GPT_ERR_CUDA of this thread (gpt_last_cuda_error reports it).
void note_cuda_error(cudaError_t e);

#define GPT_CUDA_TRY(expr)                           \
  do {                                               \
    cudaError_t e_ = (expr);                         \
    if (e_ != cudaSuccess) {                         \
      ::gpt::note_cuda_error(e_);                    \
      return GPT_ERR_CUDA;                           \
    }                                                \
  } while (0)

#define GPT_TRY(expr)                                \
  do {                                               \
    gpt_status s_ = (expr);                          \
    if (s_ != GPT_OK) return s_;                     \
  } while (0)

// Multiprocessor count and sm_100 check of the current device (cached per device).
gpt_status device_info(int* num_sms);

// Encode a tiled TMA map over a bf16 tensor of `rank` dims (dims[0] contiguous).  strides_bytes
// has rank-1 entries (byte stride of dims 1..rank-1).  128-byte swizzle when swizzle128 is set.
// Returns false if the driver rejects the map (alignment, box size).
bool encode_map_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box, bool swizzle128);
// Same for a tensor of bytes (e4m3), 128-byte swizzle.
bool encode_map_u8(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                   const uint64_t* strides_bytes, const uint32_t* box);
// Same for an fp32 tensor, no swizzle.
bool encode_map_f32(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box);

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Raise a kernel's dynamic shared-memory limit to `bytes` on the current device, once per
// (kernel, device); safe to call from several host threads.
gpt_status ensure_smem_limit(const void* kernel, int bytes);
template <typename K>
inline gpt_status ensure_smem(K kernel, int bytes) {
  return ensure_smem_limit(reinterpret_cast<const void*>(kernel), bytes);
}

// Kernel-launch counter for reporting how many of this library's kernels a step enqueued.
extern thread_local int64_t g_launch_count;
inline void count_launch(int n = 1) { g_launch_count += n; }

// Whether kernels are launched with programmatic stream serialization (default on; the environment
// variable GPTSTEP_PDL=0 turns it off for comparison).
bool pdl_enabled();

// Launch `kern` on `s` with programmatic dependent launch allowed (see pdl_wait in common.cuh) and
// count it.  Launch errors are reported as GPT_ERR_CUDA.
template <typename... KArgs, typename... Args>
inline gpt_status launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (e != cudaSuccess) {
    note_cuda_error(e);
    return GPT_ERR_CUDA;
  }
  count_launch();
  return GPT_OK;
}

// Set the bounded-wait limit of the kernels of one translation unit on the current device.
gpt_status wait_limit_set_gemm(long long cycles);
gpt_status wait_limit_set_attention(long long cycles);
gpt_status wait_limit_set_diag(long long cycles);

// Element strides of a [B, heads, T, Dh] tensor: batch, head, position (Dh contiguous).
struct HeadLayout {
  long long sb, sh, st;
};

// Kernel-level launchers used by the step orchestrator (same semantics as the C entry points).
// sk_scratch (may be null): gemm_sk_scratch_bytes() bytes, 256-byte aligned, whose leading
// arrival counters are zero; with it, tiles of a partly empty last wave may be split along K.
gpt_status gemm_launch(int op, int epi, int M, int N, int K, const void* A, int lda, const void* B,
                       int ldb, void* C, int ldc, void* C2, const void* aux, int ldaux, int* status,
                       cudaStream_t stream, void* sk_scratch = nullptr);
size_t gemm_sk_scratch_bytes();
// A batch of independent GEMMs of one shape: matrix i of each operand starts `*_bstride` elements
// after matrix i−1 (ignored for batch = 1).  GPT_EPI_AXPBY writes bf16(alpha·acc + beta·aux).
struct GemmBatch {
  int op, epi, M, N, K, batch;
  const void* A; int lda; long long a_bstride;
  const void* B; int ldb; long long b_bstride;
  void* C; int ldc; long long c_bstride;
  const void* aux; int ldaux; long long aux_bstride;
  float alpha, beta;
  int* status;
};
gpt_status gemm_launch_batched(const GemmBatch& g, cudaStream_t stream, void* sk_scratch);
// Bytes at the start of the split-tile scratch holding the arrival counters (zeroed per step).
constexpr size_t GEMM_SK_COUNTER_BYTES = 320 * 16 * sizeof(int);
// Grouped weight gradients: up to GEMM_MAX_GROUPS products C_g[M_g, N_g] = A_gᵀ·B_g with one K
// (A_g [K, M_g] and B_g [K, N_g] bf16, rows lda / ldb apart; C_g fp32, rows ldc apart) in one
// launch, their tiles dealt over the CTA pairs as one list, so that a layer's small weight
// gradients share whole waves instead of each ending in a partly empty one.  epi: GPT_EPI_F32 or
// GPT_EPI_F32_ADD.
constexpr int GEMM_MAX_GROUPS = 4;
struct GemmTnProblem {
  int M, N;
  const void* A; int lda;
  const void* B; int ldb;
  float* C; int ldc;
};
gpt_status gemm_group_tn_launch(int n, const GemmTnProblem* p, int K, int epi, int* status,
                                cudaStream_t stream, void* sk_scratch);

struct CeArgs {
  const int32_t* targets;
  int n_offset;         // vocabulary index of column 0 of this launch
  const float* lse;     // [M]
  const float* inv_n;   // device scalar: 1 / n_valid (0 if none)
  float2* stats;        // [M, stats_ld] (max, sum exp) per vocabulary tile
  int stats_ld;
  int stats_col0;       // tile index of column 0 of this launch
  float* ztarget;       // [M] logit of the target
};
// z = A·Bᵀ (A = x_f [M,K], B = W_lm rows [N,K]); CE statistics (stats/ztarget) or CE gradient
// dz = (softmax − onehot)·inv_n stored bf16 into C [M, ldc].
gpt_status gemm_ce_launch(bool grad, int M, int N, int K, const void* A, int lda, const void* B,
                          int ldb, void* C, int ldc, const CeArgs& ce, int* status,
                          cudaStream_t stream);
int gemm_ce_tile_n();  // vocabulary columns per CE statistics tile

// The attention backward's per-row scratch, computed in the epilogue of the GEMM that produces dO
// (so that the backward skips its own pass over O and dO): o token-major (b, h, t, j) at
// b·sb_o + h·Dh + t·st_o + j; lse [B, H, T]; pad = the scratch (fp32 [2][B·H·Tpad]).  Only for T a
// multiple of 64 (no zero-padded rows to fill).
struct AttnDeltaFusion {
  const void* o;
  long long sb_o, st_o;
  const float* lse;
  float* pad;
  int Tpad;
};
// C (row m = b·T + t, column n = h·Dh + j) stored bf16 head-major at heads[((b·H + h)·T + t)·Dh + j].
gpt_status gemm_heads_launch(int op, int M, int N, int K, const void* A, int lda, const void* B,
                             int ldb, void* heads, int T, int H, int Dh, int* status,
                             cudaStream_t stream, const AttnDeltaFusion* fuse = nullptr);
// [q|k|v] = A·W_qkvᵀ with RoPE + QK-norm applied to q and k, stored head-major: q [B][H][T][Dh],
// then k and v [B][Hkv][T][Dh] (Hkv ≤ 0: H); rho_q [M, H] / rho_k [M, Hkv] receive the norm factors.
// Optional destination of the QKV projection for inference: q̃ [B][H][q_ts][Dh] and k̃, v
// [B][Hkv][kv_ts][Dh] (a key/value cache), row m = b·T + t written at position t + t_off, which is
// also its RoPE position.  rho_q / rho_k may then be null.
struct QkvDest {
  void* q;
  void* k;
  void* v;
  int q_ts, kv_ts, t_off;
};
gpt_status gemm_qkv_rope_launch(int M, int d, const void* A, const void* Wqkv, void* heads,
                                float* rho_q, float* rho_k, const float* cs, int T, int H, int Dh,
                                int* status, cudaStream_t stream, int Hkv = 0,
                                const QkvDest* dest = nullptr);

}  // namespace gpt
