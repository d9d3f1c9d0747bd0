/*
 * gptstep.h — C ABI of libgptstep.so: one training step (forward + backward to parameter
 * gradients) of a nanochat-style GPT decoder, computed by hand-written sm_100a CUDA kernels.
 *
 * The model (nanochat User Guide, §10 "How It Works"; Introducing nanochat, Pretraining section):
 *   x0 = wte[tok]                                     (no norm after the embedding)
 *   per layer l:  r1 = RMS(x);  [q|k|v] = r1·W_qkvᵀ;  q̃,k̃ = RMS_Dh(RoPE(q)), RMS_Dh(RoPE(k)) per head
 *                 o = softmax(q̃k̃ᵀ/√Dh + causal/window mask)·v;   x += o·W_oᵀ
 *                 r2 = RMS(x);  x += relu(r2·W_fcᵀ)²·W_projᵀ
 *   x_f = RMS(x);  z = x_f·W_lmᵀ;  loss = mean over valid targets of (logsumexp(z) − z[target])
 * RMS(x) = x/sqrt(mean(x²) + 1e-6) with no gain; RoPE base 10000 on the pairs (i, i + Dh/2);
 * window w keeps keys t−w < j ≤ t (w ≤ 0 or w ≥ T: full causal); targets equal to −1 are ignored
 * (supa beginna nanochat, Troubleshooting: cross_entropy with ignore_index=−1, mean reduction).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers unless a parameter says "host".  The caller owns every
 *     buffer, including the workspace.  The library never calls cudaMalloc on the step path and keeps
 *     no pointer after a call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Kernels are
 *     enqueued on it; results are ready when the stream reaches that point.
 *   - bf16 tensors are raw IEEE bfloat16 (uint16 storage).  Matrices are row-major.  A weight is
 *     stored [out, in] and applied as y = x·Wᵀ.
 *   - Every call returns a gpt_status.  Argument errors are reported before anything is enqueued.
 *     Nothing aborts, throws across the ABI or traps on the device.  Problems found on the device
 *     (token id out of range, a bounded wait that expired) are written to a status word that
 *     gpt_step_status() / the `status` argument of the kernel-level calls report.
 */
#ifndef GPTSTEP_H
#define GPTSTEP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gpt_status {
  GPT_OK = 0,
  GPT_ERR_INVALID_ARG = -1,        /* null pointer, non-positive size, bad enum */
  GPT_ERR_UNSUPPORTED_SHAPE = -2,  /* a size the library cannot tile (see each call) */
  GPT_ERR_WORKSPACE_TOO_SMALL = -3,
  GPT_ERR_CUDA = -4,               /* a CUDA runtime call or kernel launch failed */
  GPT_ERR_DEVICE_TIMEOUT = -5,     /* a bounded device-side wait expired; results are invalid */
  GPT_ERR_TOKEN_OUT_OF_RANGE = -6, /* a token id outside [0, V) (or a target outside [-1, V)) */
  GPT_ERR_NO_DEVICE = -7,          /* no sm_100 device is current */
  GPT_ERR_NUMERIC_RANGE = -8       /* attention: some ‖q‖·‖k‖/√Dh exceeds 40 (see gpt_attention_fwd) */
} gpt_status;

enum { GPT_DTYPE_BF16 = 0, GPT_DTYPE_F32 = 1 };

/* Model and batch shape.  d_model = n_heads·head_dim.  head_dim ∈ {32, 64, 128}; d_model, d_mlp and
 * vocab multiples of 64; seq_len ≥ 1; batch ≥ 1.  `window` is a HOST array of `depth` entries
 * (copied by gpt_step_create; may be NULL = every layer full causal).  param_dtype selects the
 * parameter storage: BF16 is used as is, F32 is rounded to a bf16 copy inside the workspace at every
 * step (weights live in one dtype and are cast on the fly, nanochat User Guide "Precision"). */
typedef struct gpt_config {
  int32_t depth, d_model, n_heads, head_dim, d_mlp, vocab, seq_len, batch;
  const int32_t* window;
  int32_t param_dtype;
  int32_t n_kv_heads;  /* grouped-query attention: key/value heads, a divisor of n_heads; query
                          head h reads key/value head h / (n_heads/n_kv_heads) (nanochat User
                          Guide §10, group-query attention); 0 = n_heads.  head_dim 32 needs 0. */
} gpt_config;

typedef struct gpt_step gpt_step; /* opaque host-side plan; owns no device memory */

/* Flat parameter packing (element offsets, each a multiple of 64).  The tensors are the ones the
 * pages count (Introducing nanochat, Pretraining: the parameter count 560,988,160 at depth 20 is
 * 2·V·d for the untied embedding and lm-head plus 12·d² per layer; nanochat User Guide §10: untied
 * embedding/unembedding, no biases); the order is this library's:
 *   offsets[0]            wte   [V, d]
 *   offsets[1 + 4l + 0]   W_qkv [d + 2·dkv, d]   rows q (d) | k (dkv) | v (dkv), dkv = n_kv_heads·Dh
 *                                        (3d without grouping); head h's rows start at h·Dh of
 *                                        its block
 *   offsets[1 + 4l + 1]   W_o   [d, d]
 *   offsets[1 + 4l + 2]   W_fc  [F, d]
 *   offsets[1 + 4l + 3]   W_proj[d, F]
 *   offsets[1 + 4·depth]  W_lm  [V, d]
 * `offsets` is a HOST array of 2 + 4·depth entries (may be NULL); *total gets the element count.
 * Gradients use the same packing in fp32.  Host-only; needs no GPU. */
gpt_status gpt_param_layout(const gpt_config* cfg, size_t* offsets, size_t* total);

/* Validate cfg and build the host plan (the window pattern of nanochat User Guide §10 is given
 * per layer in cfg.window).  Host-only; needs no GPU. */
gpt_status gpt_step_create(const gpt_config* cfg, gpt_step** out);
void gpt_step_destroy(gpt_step* step);

/* Bytes of device workspace gpt_step_fwd_bwd needs (activations kept for the backward pass,
 * gradient scratch, statistics).  The pages give no memory plan; the caller allocates this once
 * and the library keeps no pointer into it past a call (Porting nanochat to a TPU, §4, the first
 * lesson: a buffer reused after it was captured corrupted every batch).  Host-only. */
gpt_status gpt_step_workspace_bytes(const gpt_step* step, size_t* bytes);

/* One training step: the forward pass of the model above (nanochat User Guide §10, How It Works),
 * the mean cross-entropy over targets ≠ −1 (supa beginna nanochat, Troubleshooting) and the backward
 * pass to the gradients of every parameter (the step whose throughput the pages report as tok/sec and
 * MFU, Introducing nanochat, Pretraining log).
 *   params    [n_params] bf16 or fp32 (cfg.param_dtype), packing as above
 *   tokens    [batch, seq_len] int32 in [0, V)
 *   targets   [batch, seq_len] int32 in [0, V) or −1 (ignored)
 *   loss      1 float: Σ_valid ℓ / n_valid, or 0 when no target is valid (grads are then 0 too)
 *   grads     [n_params] fp32: overwritten (accumulate = 0) or added to (accumulate = 1: the
 *             step's own gradients go to workspace scratch first and are then added element by
 *             element, so micro-batches accumulate deterministically; loss is this call's alone)
 *   workspace ≥ gpt_step_workspace_bytes, 256-byte aligned
 * Out-of-range ids are clamped for memory safety and flagged in the device status word. */
gpt_status gpt_step_fwd_bwd(gpt_step* step, const void* params, const int32_t* tokens,
                            const int32_t* targets, float* loss, float* grads, void* workspace,
                            size_t workspace_bytes, int accumulate, void* stream);

/* Synchronize `stream`, read and clear the device status word that the last step on `workspace`
 * wrote.  Returns GPT_OK, GPT_ERR_TOKEN_OUT_OF_RANGE or GPT_ERR_DEVICE_TIMEOUT (or GPT_ERR_CUDA).
 * The pages have no counterpart (errors found on the device instead of a trap or a hang). */
gpt_status gpt_step_status(const gpt_step* step, const void* workspace, void* stream);

/* A short English description of a status code ("unknown status" for others).  No page
 * counterpart. */
const char* gpt_strerror(int status);
/* The name and text of the CUDA error behind this thread's last GPT_ERR_CUDA (a per-thread buffer,
 * valid until the next call on the thread; "cudaSuccess: …" when there was none). */
const char* gpt_last_cuda_error(void);

/* Number of kernel launches the last gpt_step_fwd_bwd enqueued (host counter, for reporting; the
 * pages trace idle gaps between device programs, Porting nanochat to a TPU, §4). */
int64_t gpt_step_last_launch_count(const gpt_step* step);

/* Gradient buckets, for a data-parallel exchange that overlaps the backward pass.  The gradient
 * buffer splits into depth + 2 buckets in the order the backward pass finishes them: bucket 0 is
 * W_lm, bucket 1 + (depth − 1 − l) is layer l's W_qkv, W_o, W_fc, W_proj (contiguous in the
 * packing), bucket depth + 1 is wte.  gpt_step_grad_bucket gives bucket i's element range
 * [*begin, *end) (host-only).  With events enabled (created on the current device, owned by the
 * step), every gpt_step_fwd_bwd records one event per bucket on its stream as soon as that bucket
 * is final (with accumulate = 1, after the final addition); gpt_step_wait_grad_bucket makes
 * `stream` wait for bucket i of the last enqueued step, so that a collective on another stream
 * can start on it while the rest of the backward pass runs (Introducing nanochat: the 8-GPU run;
 * alpha-nanochat-d24, The run: the sharded optimizer exchanges gradients across ranks). */
int gpt_step_grad_buckets(const gpt_step* step);
gpt_status gpt_step_grad_bucket(const gpt_step* step, int i, size_t* begin, size_t* end);
gpt_status gpt_step_enable_grad_events(gpt_step* step, int enable);
gpt_status gpt_step_wait_grad_bucket(const gpt_step* step, int i, void* stream);

/* Per-kernel-class timing.  While enabled, every launcher call of gpt_step_fwd_bwd is bracketed
 * by two CUDA events recorded on the step's stream.  gpt_step_profile waits for those events and
 * returns, for each class c < n_classes, the summed milliseconds, number of calls, algorithmic
 * FLOPs (2·M·N·K per GEMM; 4·Dh per visible query-key pair for attention forward, twice that
 * backward) and algorithmic bytes (memory-bound kernels), then clears the record.  Classes:
 * 0 GEMM (all projections, MLP and lm-head GEMMs), 1 attention forward, 2 attention backward,
 * 3 RMSNorm, 4 RoPE + QK-norm, 5 embedding, 6 cross-entropy reductions and parameter cast.
 * Any output pointer may be NULL. */
gpt_status gpt_step_set_profiling(gpt_step* step, int enable);
gpt_status gpt_step_profile(gpt_step* step, double* ms, int64_t* calls, double* flops,
                            double* bytes, int n_classes);

/* ---------------------------------------------------------------------------------------------
 * Kernel-level entry points.  The step is built from these; they are exported for unit parity
 * tests and for the attention-only workload.  `status` (device int, may be NULL) receives a
 * device-side error code (0 = fine); it is only ever written with a nonzero code.
 * --------------------------------------------------------------------------------------------- */

/* Dense bf16 GEMM on the tcgen05 tensor cores, fp32 accumulation in tensor memory.
 *   op = GPT_GEMM_NT : C[M,N] = A[M,K]·B[N,K]ᵀ      (forward projections; A, B K-contiguous)
 *   op = GPT_GEMM_NN : C[M,N] = A[M,K]·B[K,N]       (activation gradient; B N-contiguous)
 *   op = GPT_GEMM_TN : C[M,N] = A[K,M]ᵀ·B[K,N]      (weight gradient; A, B M/N-contiguous)
 * lda/ldb/ldc/ldaux are row strides in elements (multiples of 8 for bf16, 4 for fp32).
 * epilogue (what is written for each accumulator value acc at (m, n)):
 *   GPT_EPI_BF16    C = bf16(acc)
 *   GPT_EPI_RESID   C = bf16(C + acc)                 (C bf16, residual add in place)
 *   GPT_EPI_RELU2   C = bf16(max(acc,0)²)             (C2 unused)
 *   GPT_EPI_DRELU2  C = bf16(acc · 2 · √aux)          (aux bf16 = max(u,0)² saved by RELU2, so
 *                                                       √aux = max(u,0): the ReLU² derivative)
 *   GPT_EPI_F32     C = acc                           (C fp32)
 *   GPT_EPI_F32_ADD C = C + acc                       (C fp32)
 *   GPT_EPI_AXPBY   C = bf16(alpha·acc + beta·aux)    (aux bf16, not read when beta = 0; only
 *                                                       through gpt_gemm_batched)
 * Sizes: M, N ≥ 1; K ≥ 1 (tails are zero-filled).  Pointers 16-byte aligned.
 * scratch: NULL, or gpt_gemm_scratch_bytes() bytes of device memory (256-byte aligned) that the
 * call may use to split the tiles of a partly empty last wave along K: after the whole waves, each
 * remaining tile is cut into s equal K ranges that run at the same time on s CTA pairs (s chosen
 * by a cost model, at most pairs / tail tiles); the pieces of a split tile are summed in ascending K
 * order by the piece that finishes last, so results are bitwise reproducible and no output is
 * zeroed or updated atomically.  The call zeroes the scratch's counters on `stream`
 * first; concurrent calls need separate scratch buffers.  With NULL every tile is computed whole. */
enum { GPT_GEMM_NT = 0, GPT_GEMM_NN = 1, GPT_GEMM_TN = 2 };
enum {
  GPT_EPI_BF16 = 0, GPT_EPI_RESID = 1, GPT_EPI_RELU2 = 2, GPT_EPI_DRELU2 = 3,
  GPT_EPI_F32 = 4, GPT_EPI_F32_ADD = 5, GPT_EPI_AXPBY = 6
};
size_t gpt_gemm_scratch_bytes(void);
gpt_status gpt_gemm(int op, int epilogue, int M, int N, int K, const void* A, int lda,
                    const void* B, int ldb, void* C, int ldc, void* C2, const void* aux,
                    int ldaux, void* scratch, int* status, void* stream);

/* Grouped weight gradients ("Introducing nanochat", Pretraining: the gradients of every block
 * matrix, which the optimizer then updates): for g < n (1 ≤ n ≤ 4), C_g[M_g, N_g] = A_gᵀ·B_g
 * (epilogue GPT_EPI_F32) or C_g += A_gᵀ·B_g (GPT_EPI_F32_ADD), with A_g [K, M_g] and B_g [K, N_g]
 * bf16 (row strides lda ≥ M_g, ldb ≥ N_g, multiples of 8) and C_g fp32 (ldc ≥ N_g), one K for all.
 * The output tiles of all n products are dealt to the CTA pairs as one list, so the products of one
 * layer (at d20: 75, 25, 100 and 100 tiles) fill whole waves together instead of each ending in a
 * partly empty one.  scratch, status and stream as for gpt_gemm; argument errors return
 * GPT_ERR_INVALID_ARG / GPT_ERR_UNSUPPORTED_SHAPE before anything is launched. */
typedef struct {
  int M, N;
  const void* A;
  int lda;
  const void* B;
  int ldb;
  float* C;
  int ldc;
} gpt_gemm_tn_problem;
gpt_status gpt_gemm_group_tn(int n, const gpt_gemm_tn_problem* problems, int K, int epilogue,
                             void* scratch, int* status, void* stream);

/* `batch` independent GEMMs of one shape and op (as gpt_gemm): matrix i of A, B, C and aux starts
 * i·*_bstride elements after matrix 0 (multiples of 8; the matrices must not overlap).  Any
 * epilogue of gpt_gemm, plus GPT_EPI_AXPBY (alpha, beta are ignored by the others).  One launch
 * covers the whole batch: output tiles of all matrices are dealt to the CTA pairs together.  Used
 * by the Newton–Schulz iterations of Muon (gpt_muon_step), whose matrices come in groups of one
 * shape. */
gpt_status gpt_gemm_batched(int op, int epilogue, int batch, int M, int N, int K, const void* A,
                            int lda, long long a_bstride, const void* B, int ldb,
                            long long b_bstride, void* C, int ldc, long long c_bstride,
                            const void* aux, int ldaux, long long aux_bstride, float alpha,
                            float beta, int* status, void* stream);

/* 8-bit GEMM (the FP8 matrix products of the d24 speedrun, supa beginna nanochat, and of the
 * alpha-nanochat-d24 run): tcgen05 kind::f8f6f4 on e4m3 operands with per-tensor scales.
 *   C[M,N] (bf16) = bf16(alpha · dq_a · dq_b · Σ_k A[m,k]·B[n,k])      (NT: A, B K-contiguous)
 * A, B: e4m3 bytes, lda/ldb multiples of 16; dq_a, dq_b: DEVICE floats (from gpt_quantize_e4m3);
 * fp32 accumulation; scratch as for gpt_gemm (NULL: every tile whole). */
gpt_status gpt_gemm_e4m3(int M, int N, int K, const void* A, int lda, const void* B, int ldb,
                         void* C, int ldc, const float* dq_a, const float* dq_b, float alpha,
                         void* scratch, int* status, void* stream);

/* Per-tensor e4m3 quantisation of n bf16 values: amax = max|x|, scale = 448/amax (1 if amax = 0),
 * q = e4m3(x·scale) (one fp32 multiply, round to nearest even, saturated to ±448), *dq = amax/448
 * (1 if amax = 0) — so x ≈ q·dq.  q: n bytes (8-byte aligned); dq: device float; amax_scratch:
 * one device unsigned int (zeroed by the call).  Deterministic. */
gpt_status gpt_quantize_e4m3(const void* x, long long n, void* q, float* dq,
                             unsigned int* amax_scratch, void* stream);

/* Fused QKV projection with RoPE + QK-norm, the step's forward entry into attention:
 * [q | k | v] = r·W_qkvᵀ (r bf16 [B·T, d], W_qkv bf16 [d + 2·H_kv·Dh, d], d = H·Dh); each q and k
 * head becomes RMS_Dh(RoPE(·, t)) as in gpt_rope_qknorm_fwd; all three are stored head-major in
 * `heads`: q̃ bf16 [B][H][T][Dh], then k̃ and v bf16 [B][H_kv][T][Dh].  rho_q fp32 [B·T, H], rho_k
 * fp32 [B·T, H_kv]; cos_sin from gpt_rope_table.  Dh ∈ {32, 64, 128}; H_kv divides H (H_kv = H:
 * no grouping). */
gpt_status gpt_qkv_proj_rope(const void* r, const void* w_qkv, void* heads, float* rho_q,
                             float* rho_k, const float* cos_sin, int B, int T, int H, int H_kv,
                             int Dh, int* status, void* stream);

/* RMSNorm forward over rows of d (bf16 in/out), y = x·rho, rho = 1/sqrt(mean(x²)+1e-6) (fp32). */
gpt_status gpt_rmsnorm_fwd(const void* x, void* y, float* rho, int rows, int d, void* stream);

/* RMSNorm backward: g = rho·(dy − y·mean(y·dy)).  dy is bf16 (dy_f32 = 0) or fp32 (dy_f32 = 1).
 * gx (fp32 [rows,d]) receives g (accumulate = 0) or gx + g (accumulate = 1); gx_bf16 (may be NULL)
 * receives a bf16 copy of the new gx. */
gpt_status gpt_rmsnorm_bwd(const void* dy, int dy_f32, const void* y, const float* rho, float* gx,
                           void* gx_bf16, int accumulate, int rows, int d, void* stream);

/* RoPE + QK-norm forward on qkv [B·T, 3·H·Dh] (bf16, output of the QKV projection), in place:
 * the q and k blocks of every head become RMS_Dh(RoPE(·, t)); v is untouched.  rho_q, rho_k fp32
 * [B·T, H].  cos_sin: fp32 [T, Dh/2, 2] table from gpt_rope_table. */
gpt_status gpt_rope_qknorm_fwd(void* qkv, float* rho_q, float* rho_k, const float* cos_sin, int B,
                               int T, int H, int Dh, void* stream);
/* Backward of the above, in place on dqkv (q and k blocks hold dq̃, dk̃ on entry, dq, dk on exit);
 * qkv holds the forward output (q̃, k̃). */
gpt_status gpt_rope_qknorm_bwd(void* dqkv, const void* qkv, const float* rho_q, const float* rho_k,
                               const float* cos_sin, int B, int T, int H, int Dh, void* stream);
/* Fill cos_sin [T, Dh/2, 2] with cos/sin of t·10000^(−2i/Dh), angles computed in fp64. */
gpt_status gpt_rope_table(float* cos_sin, int T, int Dh, void* stream);

/* Causal / sliding-window flash attention with grouped-query heads.  q, o, dO, dq have H heads;
 * k, v, dk, dv have H_kv heads (H a multiple of H_kv); query head h attends with key/value head
 * h / (H/H_kv), and dk, dv sum over the query heads of their group (H_kv = H: multi-head
 * attention).  Tensors are bf16, element (b, h, t, j) at base + b·sb + h·sh + t·st + j (strides in
 * elements, j contiguous), one stride set per tensor group: (sb_q, sh_q, st_q) for q and dq,
 * (sb_kv, sh_kv, st_kv) for k, v, dk, dv, (sb_o, sh_o, st_o) for o and dO.  lse: fp32 [B, H, T],
 * the natural-log logsumexp of the scaled scores.  Dh ∈ {32, 64, 128} (32: H_kv = H only).
 * window ≤ 0 or ≥ T = full causal.  delta: backward scratch of at least
 * gpt_attention_bwd_scratch_bytes(B, H, T) bytes, 16-byte aligned; per row (zero-padded to a
 * multiple of 64 rows per (b, h)) the backward stores LSE·log2(e) and rowsum(dO∘O) in fp32; after
 * these rows, for Dh ≥ 64, the dK/dV kernel stores dS (bf16 [nb·H][T][⌈T/64⌉·64], query rows and
 * key columns, causal band / window only) for a chunk of nb batches and the dQ kernel contracts it
 * with K, chunk after chunk; nb is the largest count whose dS fits GPT_ATTN_BWD_DS_MAX_BYTES, and
 * when not even one batch fits, dS is not stored and the dQ kernel recomputes the scores.
 * The forward shifts each row's exponentials by the Cauchy–Schwarz bound c_t = ‖q_t‖·max_j‖k_j‖/√Dh
 * instead of a running maximum (softmax is invariant to the shift, so the result is exact); this
 * needs c_t ≤ 40 so that no row underflows, which always holds after QK-norm (c_t ≈ √Dh) — rows
 * beyond it set GPT_ERR_NUMERIC_RANGE in *status. */
/* kmax: device scratch of B·H_kv floats that receives max_t ‖k_t‖ per (b, key/value head), or
 * NULL when every k row is RMS-normalised over Dh (QK-norm), in which case the bound
 * √Dh·(1 + 2⁻⁹) is used. */
gpt_status gpt_attention_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                             float* kmax, int B, int H, int H_kv, int T, int Dh, int window,
                             long long sb_q, long long sh_q, long long st_q, long long sb_kv,
                             long long sh_kv, long long st_kv, long long sb_o, long long sh_o,
                             long long st_o, int* status, void* stream);
/* Bytes of the `delta` scratch that gpt_attention_bwd needs for (B, H, T): 8 bytes per row of
 * R = B·H·⌈T/64⌉·64, plus the dS of one batch chunk, nb·H·T·⌈T/64⌉·64·2 bytes ≤
 * GPT_ATTN_BWD_DS_MAX_BYTES (1.6 GB for B 16 × H 12 at T = 2048, one chunk; 8.6 GB for B 32 × H 8
 * at T = 8192, which runs as four chunks of 8 batches).  Callers short of memory can use, within
 * its row limit, gpt_attention_bwd_noalloc, which recomputes the scores instead.  Returns 0 for a
 * non-positive size. */
#define GPT_ATTN_BWD_DS_MAX_BYTES (8ll << 30)
size_t gpt_attention_bwd_scratch_bytes(int B, int H, int T);
gpt_status gpt_attention_bwd(const void* q, const void* k, const void* v, const void* o,
                             const void* dout, const float* lse, float* delta, void* dq, void* dk,
                             void* dv, int B, int H, int H_kv, int T, int Dh, int window,
                             long long sb_q, long long sh_q, long long st_q, long long sb_kv,
                             long long sh_kv, long long st_kv, long long sb_o, long long sh_o,
                             long long st_o, int* status, void* stream);

/* Attention backward that allocates nothing.  The pages have no counterpart: this is a calling
 * convenience, not part of the method.  Arguments and results are those of gpt_attention_bwd
 * without `delta`, for multi-head attention (H_kv = H, one stride set (sb_qkv, sh_qkv, st_qkv) for
 * q/k/v/dq/dk/dv); the per-row scratch that the backward needs (8 bytes per row of
 * B·H·⌈T/64⌉·64) is kept in a static device array inside this library
 * (GPT_ATTN_BWD_NOALLOC_FLOATS fp32 values = 8 MiB), which every GPU that loads the library holds
 * until the process exits.  dS is not stored: the dQ kernel recomputes the scores instead.
 * It serves callers that cannot obtain device memory where they call the backward — for example
 * code running under a device-memory budget fixed at start-up, or inside a host framework whose own
 * allocator owns all device memory and allows no side allocations — and therefore cannot hand
 * gpt_attention_bwd its scratch buffer.  It calls no cudaMalloc, cudaFree or allocating routine.
 *   - The array holds GPT_ATTN_BWD_NOALLOC_FLOATS fp32 values; at 8 bytes (2 floats) per padded
 *     row it serves B·H·⌈T/64⌉·64 ≤ GPT_ATTN_BWD_NOALLOC_MAX_ROWS rows (1,048,576, itself a
 *     multiple of 64).  Larger shapes return GPT_ERR_UNSUPPORTED_SHAPE before anything is enqueued
 *     or any CUDA call is made.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress, with
 *     that device current); make that first call before any stream capture.
 *   - All calls share the one array.  Each call writes the rows it uses before reading them, so
 *     nothing needs clearing, but calls that overlap on the GPU (unordered streams, several host
 *     threads) race on it and give wrong results: order them on one stream. */
#define GPT_ATTN_BWD_NOALLOC_FLOATS (1ll << 21)
#define GPT_ATTN_BWD_NOALLOC_MAX_ROWS (GPT_ATTN_BWD_NOALLOC_FLOATS / 2)
gpt_status gpt_attention_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                     const void* dout, const float* lse, void* dq, void* dk,
                                     void* dv, int B, int H, int T, int Dh, int window,
                                     long long sb_qkv, long long sh_qkv, long long st_qkv,
                                     long long sb_o, long long sh_o, long long st_o, int* status,
                                     void* stream);

/* Embedding gather x[m] = wte[tok[m]] (bf16 rows of d).  Ids outside [0, V) are clamped and
 * flagged in *status. */
gpt_status gpt_embedding_fwd(const int32_t* tokens, const void* wte, void* x, int M, int d, int V,
                             int* status, void* stream);
/* Embedding backward dwte = Σ_{m: tok[m]=v} gx[m] for every row v (fp32, rows without a token are
 * zeroed).  Duplicate ids are summed in a fixed order (ascending m within pieces of 64 sorted
 * tokens, pieces in order), so the result is deterministic.  scratch: device bytes ≥
 * gpt_embedding_bwd_scratch_bytes(M, d, V). */
size_t gpt_embedding_bwd_scratch_bytes(int M, int d, int V);
gpt_status gpt_embedding_bwd(const int32_t* tokens, const float* gx, float* dwte, int M, int d,
                             int V, void* scratch, void* stream);

/* Fused lm-head + softmax cross-entropy, vocabulary processed in tiles so the [M, V] logits are
 * never stored.  Forward: lse[m] = logsumexp_v(x_f[m]·W_lm[v]), loss = Σ_valid (lse − z[target])
 * / n_valid.  Backward (dz = (softmax − onehot)/n_valid, rows with target −1 get 0):
 * dx (fp32 [M,d]) = dz·W_lm and dW (fp32 [V,d]) = dzᵀ·x_f.  x_f, W_lm bf16.  scratch: device
 * bytes ≥ gpt_lmhead_ce_scratch_bytes(M, d, V). */
size_t gpt_lmhead_ce_scratch_bytes(int M, int d, int V);
gpt_status gpt_lmhead_ce_fwd_bwd(const void* xf, const void* wlm, const int32_t* targets, int M,
                                 int d, int V, float* loss, float* lse, float* dx, float* dW,
                                 void* scratch, int* status, void* stream);

/* ---------------------------------------------------------------------------------------------
 * Forward-only inference with a key/value cache (supa beginna nanochat, notes on each stage: the
 * engine that samples from the trained model keeps a KV cache).  The forward pass is the training
 * step's (same kernels and numerics); the QKV projection writes k̃ = RMS_Dh(RoPE(k)) and v of every
 * layer straight into the cache, and the lm-head runs on the last position of each sequence only.
 *   kv_cache: caller-owned device memory of gpt_infer_kv_cache_bytes() bytes, bf16
 *             [depth][2][max_batch][n_kv_heads][max_len][head_dim] (k̃ then v per layer).
 *   gpt_prefill: tokens [batch, T] (positions 0 .. T−1 of every sequence), fills cache positions
 *             0 .. T−1 and writes logits [batch, V] (fp32) of position T−1.
 *   gpt_decode: tokens [batch] at position `pos` of every sequence (cache positions 0 .. pos−1
 *             already filled), fills position pos and writes logits [batch, V] of it.
 * All sequences of a call share one length.  param_dtype must be BF16 and head_dim 64 or 128.
 * batch ≤ max_batch, T and pos + 1 ≤ max_len.  Token ids outside [0, V) are clamped and flagged in
 * the status word (gpt_infer_status).  Host-only: create, destroy, the byte counts. */
typedef struct gpt_infer gpt_infer;
gpt_status gpt_infer_create(const gpt_config* cfg, int max_batch, int max_len, gpt_infer** out);
void gpt_infer_destroy(gpt_infer* inf);
gpt_status gpt_infer_workspace_bytes(const gpt_infer* inf, size_t* bytes);
size_t gpt_infer_kv_cache_bytes(const gpt_infer* inf);
gpt_status gpt_prefill(gpt_infer* inf, const void* params, const int32_t* tokens, int batch, int T,
                       float* logits, void* kv_cache, void* workspace, size_t workspace_bytes,
                       void* stream);
gpt_status gpt_decode(gpt_infer* inf, const void* params, const int32_t* tokens, int batch, int pos,
                      float* logits, void* kv_cache, void* workspace, size_t workspace_bytes,
                      void* stream);
gpt_status gpt_infer_status(const gpt_infer* inf, const void* workspace, void* stream);

/* ---------------------------------------------------------------------------------------------
 * The optimizer step after the training step (Introducing nanochat, Pretraining log: the block
 * matrices go to Muon, grouped by shape — q, k, v, the output projection, W_fc, W_proj — and the
 * embedding and lm-head to AdamW, whose learning rates are scaled by 1/√(d/768)).  The pages print
 * no hyperparameter values and no Muon internals: the published method is restated below and
 * every value is an argument.  Weights are updated in an fp32 master copy; `params` (may be NULL
 * or equal to the master) receives the new values in the step's parameter dtype (bf16 rounded to
 * nearest even, or fp32).  Optimizer state buffers are fp32, caller-owned, zero before step 1.
 * --------------------------------------------------------------------------------------------- */

/* AdamW with decoupled weight decay over n elements (t ≥ 1 counts steps from 1):
 *   m ← β1·m + (1−β1)·g;  v ← β2·v + (1−β2)·g²;  m̂ = m/(1−β1^t);  v̂ = v/(1−β2^t)
 *   W ← W·(1 − lr·weight_decay) − lr·m̂/(√v̂ + eps)
 * master, grads, m, v (and params) 16-byte aligned.  One fused elementwise kernel. */
gpt_status gpt_adamw_step(float* master, void* params, int param_dtype, const float* grads,
                          float* m, float* v, long long n, int t, float lr, float beta1,
                          float beta2, float eps, float weight_decay, void* stream);

/* Muon on a group of n = groups·per_group matrices of shape rows × cols: matrix i starts at
 * element (i / per_group)·group_stride + (i % per_group)·rows·cols of master, grads and
 * momentum_buf (the packing of the flat parameter buffer: per layer q, k, v, o are four contiguous
 * d×d matrices, layers one stride apart).  Per matrix:
 *   buf ← momentum·buf + g;  u = g + momentum·buf (nesterov ≠ 0) or buf;  X = u/(‖u‖_F + 1e-7)
 *   ns_steps times: A = X·Xᵀ;  X ← ns_a·X + (ns_b·A + ns_c·A·A)·X  (tall matrices iterated as their
 *   transpose; the published quintic is (3.4445, −4.7750, 2.0315) for 5 steps)
 *   W ← W − lr·√max(1, rows/cols)·X
 * The Newton–Schulz products are batched tcgen05 GEMMs over the group in bf16 with fp32
 * accumulation (the precision the method is published with); ‖u‖ is summed in a fixed order.
 * rows, cols multiples of 8; with groups > 1, group_stride ≥ per_group·rows·cols (ignored for one
 * group).  scratch ≥ gpt_muon_scratch_bytes(n, rows, cols), 256-byte aligned. */
size_t gpt_muon_scratch_bytes(int n_matrices, int rows, int cols);
gpt_status gpt_muon_step(float* master, void* params, int param_dtype, const float* grads,
                         float* momentum_buf, int groups, int per_group, long long group_stride,
                         int rows, int cols, float lr, float momentum, int nesterov, int ns_steps,
                         float ns_a, float ns_b, float ns_c, void* scratch, size_t scratch_bytes,
                         int* status, void* stream);

typedef struct gpt_optim_hparams {
  float muon_lr, muon_momentum;
  int32_t muon_nesterov, ns_steps;
  float ns_a, ns_b, ns_c;
  float adam_lr_wte, adam_lr_lm;  /* before the 1/√(d_model/768) scale */
  float beta1, beta2, eps, weight_decay;
} gpt_optim_hparams;

/* The whole optimizer step over the flat packing of cfg: Muon on every layer's q, k, v, o (one
 * group), W_fc (one group), W_proj (one group); AdamW on wte and W_lm with learning rates
 * adam_lr_* · 1/√(d_model/768).  state_m holds Muon's momentum buffers and AdamW's first moments,
 * state_v AdamW's second moments, both fp32 [n_params] in the same packing.  scratch ≥
 * gpt_optim_scratch_bytes(cfg). */
size_t gpt_optim_scratch_bytes(const gpt_config* cfg);
gpt_status gpt_optim_step(const gpt_config* cfg, float* master, void* params, const float* grads,
                          float* state_m, float* state_v, int t, const gpt_optim_hparams* hp,
                          void* scratch, size_t scratch_bytes, int* status, void* stream);

/* ---------------------------------------------------------------------------------------------
 * Diagnostics.  Not part of the method: they exist so that the failure handling of the kernels and
 * the accuracy of one of their approximations can be tested on a GPU without faulting it.
 * --------------------------------------------------------------------------------------------- */

/* Every mbarrier wait inside the GEMM and attention kernels gives up after a limit (SM clock
 * cycles, default 4e9 ≈ 2 s): it then records GPT_ERR_DEVICE_TIMEOUT in the call's status word,
 * makes the CTA's other roles stop waiting, lets copies already in flight land, frees its tensor
 * memory and returns; nothing traps.  This sets the limit for kernels launched afterwards on the
 * CURRENT device (cycles ≤ 0 restores the default).  It is a blocking copy to device memory: call it
 * between launches, not while kernels of this library run.  A small limit makes ordinary waits
 * (a TMA load in flight) run out, which is how the tests exercise the timeout path. */
gpt_status gpt_set_wait_limit(long long cycles);

/* Launch one CTA that waits, with the bounded wait of the kernels above, on an mbarrier that
 * nothing ever completes.  The wait runs out after the current limit and *status (device int)
 * receives GPT_ERR_DEVICE_TIMEOUT; the kernel then returns and the context stays usable. */
gpt_status gpt_debug_wait_probe(int* status, void* stream);

/* y[i] = 2^x[i] computed as the attention forward computes a quarter of its softmax weights on the
 * FMA pipe: x clamped to ≥ −126, x = n + f with n = round(x), 2^f by a fitted cubic on [−1/2, 1/2]
 * (relative error ≤ 7.5e-5), n added to the exponent field.  x, y: device fp32 arrays of n. */
gpt_status gpt_debug_exp2_poly2(const float* x, float* y, int n, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* GPTSTEP_H */
