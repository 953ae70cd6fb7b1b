/*
 * samba.h - C ABI of the B200 (sm_100a) Samba block library (libsamba.so).
 *
 * What is computed follows the page "Samba: Simple Hybrid State Space Models
 * for Efficient Unlimited Context Language Modeling" (a long-form summary of
 * arXiv 2406.07522), cited as [Samba <section>, <sub-heading>].  The block is
 * Mamba -> SwiGLU MLP -> sliding-window attention -> SwiGLU MLP, every layer
 * pre-RMSNorm with a residual add [Samba 3.2 "Big-Picture Architecture"].
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *     aligned, contiguous row-major with the innermost dimension last, unless an
 *     argument says otherwise.  The library allocates no device memory: scratch
 *     space comes from the caller through (workspace, workspace_bytes), sized by
 *     the matching *_workspace_size query.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  The return value reports argument validation and launch errors
 *     only.  Errors detected on the device (a bounded wait that gave up, a
 *     failed device-side check) are latched in a device error word that
 *     samba_get_error() reads.
 *   - Activations and weight matrices are `samba_dtype` (fp32 or bf16); per-channel
 *     parameters (norm gains, conv taps, dt bias, A_log, D) and the SSM state are
 *     fp32.  Arithmetic is fp32 (fp32 accumulation on the tensor cores).
 *   - Weight matrices are stored [out_features, in_features] row-major, i.e. the
 *     transpose of the pages' X W notation.
 *   - No exception, C++ type or torch type crosses this boundary; the library is
 *     stateless apart from the device error word and is reentrant.
 *   - Size limits of the launch grids: a batch B (and a head count) of at most
 *     65535, and at most 65535 * 32 = 2,097,120 tokens per sequence in one call
 *     of an entry point that runs the causal conv (longer prompts go through
 *     samba_block_fwd_chunk).  Larger shapes return SAMBA_ERR_UNSUPPORTED before
 *     anything is launched.
 */
#ifndef SAMBA_H_
#define SAMBA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SAMBA_OK = 0,
  SAMBA_ERR_INVALID_ARG = 1,  /* NULL where data is required, bad size, workspace too small */
  SAMBA_ERR_UNSUPPORTED = 2,  /* valid but not handled by these kernels (misaligned, N != 16, ...) */
  SAMBA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed (launch, tensor-map encode) */
  SAMBA_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up (from samba_get_error) */
  SAMBA_ERR_DEVICE = 5,       /* a device-side check failed (from samba_get_error) */
  SAMBA_ERR_BOUNDS = 6        /* debug-check build: an index bounds check or a workspace
                                 guard band failed (from samba_get_error) */
} samba_status;

typedef enum { SAMBA_F32 = 0, SAMBA_BF16 = 1 } samba_dtype;

typedef void* samba_stream; /* cudaStream_t */

/* Human-readable name of a status code (static string). */
const char* samba_status_string(samba_status s);

/* Library version string (static). */
const char* samba_version(void);

/* The CUDA error behind the calling thread's last SAMBA_ERR_CUDA return ("where:
 * message (code)"), or "" if none was recorded.  Owned by the library; valid
 * until the thread's next failing call. */
const char* samba_last_cuda_error(void);

/* Measurement hook for benchmarks and profilers (no effect unless installed).
 * While installed, every launch of a projection with epilogue kind `epi` (the
 * samba_linear kinds: 0 none, 1 residual, 2 SwiGLU, 3 softplus + bias; 4 the
 * Q/K/V projection with RoPE inside the block) records start_events[i] on its
 * stream immediately before the kernel and stop_events[i] immediately after it,
 * i = 0, 1, ... in launch order; launches past `capacity` are not recorded.
 * Events are cudaEvent_t created by the caller with timing enabled and must
 * outlive the hook.  epi < 0 removes the hook (the arrays may then be NULL).
 * Installing or removing the hook resets the launch count; it is process-wide,
 * so install it only while one host thread launches.  Returns
 * SAMBA_ERR_INVALID_ARG for NULL arrays or entries, capacity < 1 or epi > 4. */
samba_status samba_set_gemm_timing(int epi, void* const* start_events, void* const* stop_events, int capacity);

/* Launches recorded by the hook since it was installed. */
int samba_gemm_timing_count(void);

/* Failure-detection test hook (the paper has no counterpart).  While set
 * (stop_after_chunks >= 0), every selective-scan launch stops issuing its
 * input loads after that many 64-token chunks, and its bounded waits give up
 * after wait_limit_ns (1 ms .. 2 s) instead of 2 s: the wait for the next chunk
 * then runs out, the kernel latches SAMBA_ERR_TIMEOUT in the device error word,
 * waits for its own output stores and returns, leaving the context usable.
 * Outputs past the stop are unspecified.  stop_after_chunks = -1 clears the hook
 * (wait_limit_ns is then ignored).  Process-wide; the scan reads it at each
 * launch on the host.  SAMBA_ERR_INVALID_ARG for stop_after_chunks < -1 or a
 * limit outside the range. */
samba_status samba_debug_scan_stall(int stop_after_chunks, uint64_t wait_limit_ns);

/* Synchronises `stream`, returns and clears the device error word of the
 * current device: SAMBA_OK, SAMBA_ERR_TIMEOUT, SAMBA_ERR_DEVICE or (debug-check
 * build) SAMBA_ERR_BOUNDS, or SAMBA_ERR_CUDA if the synchronisation itself
 * failed.  The word keeps the first error latched since it was last read. */
samba_status samba_get_error(samba_stream stream);

/* ------------------------------------------------------------------------
 * Debug-check build.  libsamba_debug.so is the same library compiled with
 * SAMBA_DEBUG_CHECKS=1 (same symbols, same results):
 *   - device index checks: before the accesses they guard (tile and chunk
 *     coordinates, ring slots, key ranges, reduction slots, output rows), the
 *     kernels check the index against the extent it must stay in; a failed
 *     check skips the access and latches SAMBA_ERR_BOUNDS with its site, and the
 *     kernel runs on (no trap, no assert);
 *   - workspace guard bands: every sub-buffer the library carves from a
 *     workspace is followed by a 4 KiB band that is filled with a pattern
 *     before the call's kernels and verified after them; the workspace-size
 *     queries include the bands.
 * ---------------------------------------------------------------------- */

/* 1 in the debug-check build, 0 in the release build. */
int samba_debug_checks_enabled(void);

/* Where the check behind the calling thread's last SAMBA_ERR_BOUNDS from
 * samba_get_error failed ("file.cu:line", or "workspace guard band <i>
 * overwritten"); "" if none.  Owned by the library, per thread. */
const char* samba_last_check_site(void);

/* Self-test of the debug checks; makes no out-of-bounds access of any kind.
 * kind 0: a kernel evaluates one device check on an index the host chose out
 *         of range and skips the access it guards;
 * kind 1: two sub-buffers of 4 KiB are carved from `workspace` with their guard
 *         bands, one byte inside the first band (memory of the caller's
 *         workspace) is changed between the fill and the verification.
 * Both then latch SAMBA_ERR_BOUNDS for samba_get_error.  Returns
 * SAMBA_ERR_UNSUPPORTED in the release build, SAMBA_ERR_INVALID_ARG for another
 * kind or (kind 1) a workspace smaller than samba_debug_selftest_workspace_size(). */
size_t samba_debug_selftest_workspace_size(void);
samba_status samba_debug_check_selftest(int kind, void* workspace, size_t workspace_bytes, samba_stream stream);

/* ------------------------------------------------------------------------
 * Selective scan (S6)  [Samba 3.4 "The State Space Model Update (S6)",
 *                        "Input-Dependent Selective Gating", "Gated Output"]
 *
 *   Delta_t = dt_softplus ? log(1 + exp(dt_t + dt_bias)) : dt_t (+ dt_bias)
 *   h_t     = exp(Delta_t * A) (.) h_{t-1} + (Delta_t * u_t) * B_t,  A = -exp(A_log)
 *   y_t     = <C_t, h_t> + Dskip * u_t,  then  y_t *= SiLU(z_t)  if z != NULL
 *
 *   u, dt, z, y : [B, L, D] dtype        Bm, Cm : [B, L, N] dtype
 *   A_log       : [D, N] fp32            dt_bias, Dskip : [D] fp32 or NULL (0)
 *   h0          : [B, D, N] fp32 initial state or NULL (zeros)
 *   hT          : [B, D, N] fp32 state after the last token, or NULL
 * Requirements: N == 16, D % 32 == 0, B >= 1, L >= 0.  L == 0 copies h0 (or
 * zeros) into hT.  The state is kept in fp32 throughout.
 * ---------------------------------------------------------------------- */
size_t samba_selective_scan_workspace_size(int B, int L, int D, int N);

samba_status samba_selective_scan(const void* u, const void* dt, const float* dt_bias, int dt_softplus,
                                  const float* A_log, const void* Bm, const void* Cm, const float* Dskip,
                                  const void* z, const float* h0, float* hT, void* y, int B, int L, int D,
                                  int N, samba_dtype dtype, void* workspace, size_t workspace_bytes,
                                  samba_stream stream);

/* ------------------------------------------------------------------------
 * The selective scan with the dt projection folded in, on the x_proj output
 * of a Mamba layer [Samba §3.4 "Input-Dependent Selective Gating (The Delta
 * Parameter)": Delta = softplus(dt_low W_dt^T + dt_bias), the low-rank
 * bottleneck dt_low being the first dt_rank columns of x W_x^T; then "The
 * State Space Model Update (S6)" and "Gated Output" as samba_selective_scan].
 *
 * x_dbl: [B, L, dt_rank + 2*N] dtype, row-major: dt_low | B_t | C_t per token.
 * W_dt: [D, dt_rank] dtype.  dt_bias: [D] fp32 (may be NULL).  u, z, y:
 * [B, L, D] dtype (z may be NULL).  A_log, Dskip, h0, hT as samba_selective_scan.
 * Delta is formed inside the scan kernel in fp32 and never written to memory.
 * Supported: bf16, N == 16, D % 16 == 0, dt_rank a multiple of 16 and at most
 * 128, 16-byte aligned arrays; otherwise SAMBA_ERR_UNSUPPORTED (use
 * samba_linear with the softplus epilogue and samba_selective_scan).
 * ---------------------------------------------------------------------- */
samba_status samba_selective_scan_xdbl(const void* u, const void* x_dbl, int dt_rank, const void* W_dt,
                                       const float* dt_bias, const float* A_log, const float* Dskip, const void* z,
                                       const float* h0, float* hT, void* y, int B, int L, int D, int N,
                                       samba_dtype dtype, samba_stream stream);

/* ------------------------------------------------------------------------
 * Causal sliding-window attention with grouped-query heads and RoPE
 *   [Samba 3.4 "Window Specification", "Positional Encoding", "Implementation"]
 *
 *   qr = RoPE(q, pos0 + t), kr = RoPE(k, pos0 + t)   (rope_base == 0: no rotation)
 *   o[b,t,h] = sum_{s = max(0, t-window+1)}^{t} softmax_s(scale * qr[b,t,h] . kr[b,s,g(h)]) v[b,s,g(h)]
 *   g(h) = h / (Hq / Hkv);  scale = softmax_scale > 0 ? softmax_scale : 1/sqrt(head_dim)
 *
 *   q, o : [B, L, Hq, head_dim] dtype      k, v : [B, L, Hkv, head_dim] dtype
 * RoPE pairs channel i with i + head_dim/2 and uses theta_i = rope_base^(-2i/head_dim);
 * angles are formed from fp64 tables so that positions up to 2^30 keep ~1e-7 rad.
 * Requirements: Hq % Hkv == 0, head_dim in {16, 32, 64} (any dtype) or 256 (bf16), window >= 1,
 * pos0 >= 0, pos0 + L <= 2^30.  With rope_base != 0 the rotated copies of q and k
 * live in the workspace.
 * ---------------------------------------------------------------------- */
size_t samba_swa_workspace_size(int B, int L, int Hq, int Hkv, int head_dim, float rope_base,
                                samba_dtype dtype);

samba_status samba_swa_fwd(const void* q, const void* k, const void* v, void* o, int B, int L, int Hq, int Hkv,
                           int head_dim, int window, float rope_base, int64_t pos0, float softmax_scale,
                           samba_dtype dtype, void* workspace, size_t workspace_bytes, samba_stream stream);

/* Same computation and arguments as samba_swa_fwd, for callers that cannot
 * allocate device memory: for instance a plugin running inside a host
 * application that owns all device memory and gives the plugin no allocator, so
 * it has no way to obtain a workspace.  The paper has no counterpart: this is a
 * library convenience.
 * The scratch it needs with rope_base != 0 (the rotation table and rotated copies
 * of q and k) lives in a fixed 16 MiB device array inside the library, held on
 * every GPU that loads the library until the process exits.  It fits when
 *   round256(3*1024*(head_dim/2)*8) + round256(B*L*Hq*head_dim*esize)
 *                                   + round256(B*L*Hkv*head_dim*esize) <= 16 MiB
 * (esize 2 for bf16, 4 for fp32); larger calls return SAMBA_ERR_UNSUPPORTED and
 * launch nothing.  No cudaMalloc/cudaFree or other allocation is made.
 * The first call on each device looks up the array's device address (set-up),
 * and a call after the device's context was replaced (cudaDeviceReset) looks it
 * up again; make the first call on a device before any stream capture.  Shapes
 * beyond the launch grids (B or Hq > 65535) are rejected before any launch, like
 * the size check above.  All calls share the array and
 * it keeps the last call's contents (each call rewrites what it reads); calls that
 * overlap on the GPU (other streams, other host threads) race on it. */
samba_status samba_swa_fwd_noalloc(const void* q, const void* k, const void* v, void* o, int B, int L, int Hq,
                                   int Hkv, int head_dim, int window, float rope_base, int64_t pos0,
                                   float softmax_scale, samba_dtype dtype, samba_stream stream);

/* ------------------------------------------------------------------------
 * Building blocks of the block (also used by it)
 * ---------------------------------------------------------------------- */

/* RMSNorm [Samba 3.2]: out[r,:] = x[r,:] / sqrt(mean(x[r,:]^2) + eps) * g.
 * x, out: [rows, dim] dtype (may alias); g: [dim] fp32.  dim % 8 == 0. */
samba_status samba_rmsnorm(const void* x, const float* g, void* out, int64_t rows, int dim, float eps,
                           samba_dtype dtype, samba_stream stream);

/* Short convolution [Samba 3.4 "Input Projection and Short Convolution"]:
 *   u[b,t,c] = SiLU( sum_{j<k} w[c,j] * x[b, t-(k-1)+j, c] + bias[c] ),  x before t = 0 is 0.
 * x: [B, L, *] dtype with row stride ld_x elements (>= D); w: [D, k] fp32;
 * bias: [D] fp32 or NULL; u: [B, L, D] dtype; conv_state: [B, D, k-1] dtype
 * receiving the last k-1 inputs (oldest first; zeros where L < k-1), or NULL.
 * Requirements: 2 <= k <= 8, D % 8 == 0. */
samba_status samba_causal_conv1d(const void* x, int64_t ld_x, const float* w, const float* bias, void* u,
                                 void* conv_state, int B, int L, int D, int k, samba_dtype dtype,
                                 samba_stream stream);

typedef enum {
  SAMBA_EPI_NONE = 0,          /* out = x W^T */
  SAMBA_EPI_RESIDUAL = 1,      /* out = resid + x W^T            (resid [M, N] dtype, may alias out) */
  SAMBA_EPI_SWIGLU = 2,        /* out = (x W^T) * SiLU(x W2^T)   [Samba 3.4 "SwiGLU Formulation"] */
  SAMBA_EPI_SOFTPLUS_BIAS = 3  /* out = log(1 + exp(x W^T + bias))  (bias [N] fp32) */
} samba_epilogue;

/* Dense projection out[M, N] = epilogue(x[M, K] W[N, K]^T) with fp32 accumulation.
 * W2 only for SWIGLU ([N, K]); bias only for SOFTPLUS_BIAS; resid only for RESIDUAL.
 * Requirements: K % 8 == 0, N % 8 == 0. */
samba_status samba_linear(const void* x, const void* W, const void* W2, const float* bias, const void* resid,
                          void* out, int64_t M, int N, int K, samba_epilogue epilogue, samba_dtype dtype,
                          samba_stream stream);

/* ------------------------------------------------------------------------
 * The Samba block (prefill)                                  [Samba 3.2, 3.4]
 * ---------------------------------------------------------------------- */
typedef struct {
  int d_model;   /* model width d_m */
  int d_inner;   /* Mamba expanded width d_e (2 d_m in the pages) */
  int d_state;   /* SSM state size d_s (16) */
  int d_conv;    /* short-conv kernel size k (4) */
  int dt_rank;   /* low-rank Delta bottleneck d_r (d_m / 16) */
  int n_q;       /* query heads */
  int n_kv;      /* key/value heads (GQA groups) */
  int head_dim;  /* per-head width */
  int window;    /* sliding window w (keys t-w+1 .. t) */
  int d_ff;      /* SwiGLU hidden width d_p */
  float rope_base; /* RoPE base (10000); 0 disables RoPE */
  float norm_eps;  /* RMSNorm epsilon */
  samba_dtype dtype;
} samba_block_config;

typedef struct {
  const float* norm_g[4]; /* [d_model] gains before Mamba, MLP1, SWA, MLP2 */
  const void* W_in;       /* [2*d_inner, d_model]: rows [0,d_inner) = W_in (x branch), rest = W_g (gate z) */
  const float* conv_w;    /* [d_inner, d_conv] */
  const float* conv_b;    /* [d_inner] or NULL */
  const void* W_x;        /* [dt_rank + 2*d_state, d_inner]: rows = W_r | W_b | W_c */
  const void* W_dt;       /* [d_inner, dt_rank]  (W_q of the pages) */
  const float* dt_bias;   /* [d_inner] */
  const float* A_log;     /* [d_inner, d_state]; A = -exp(A_log) */
  const float* Dskip;     /* [d_inner] */
  const void* W_out;      /* [d_model, d_inner] */
  const void* Wq;         /* [n_q*head_dim, d_model] */
  const void* Wk;         /* [n_kv*head_dim, d_model] */
  const void* Wv;         /* [n_kv*head_dim, d_model] */
  const void* Wo;         /* [d_model, n_q*head_dim] */
  const void* mlp1_W1;    /* [d_ff, d_model]  value branch */
  const void* mlp1_W2;    /* [d_ff, d_model]  SiLU gate branch */
  const void* mlp1_W3;    /* [d_model, d_ff] */
  const void* mlp2_W1;
  const void* mlp2_W2;
  const void* mlp2_W3;
} samba_block_weights;

/* Decode state of one block, all caller-owned device buffers. */
typedef struct {
  float* ssm;     /* [B, d_inner, d_state] fp32 recurrent state, 16-byte aligned */
  void* conv;     /* [B, d_inner, d_conv-1] dtype: last d_conv-1 pre-conv inputs, oldest first */
  void* k_ring;   /* [B, window, n_kv, head_dim] dtype: post-RoPE keys, slot = position mod window */
  void* v_ring;   /* [B, window, n_kv, head_dim] dtype */
  int64_t* pos;   /* [B] number of tokens seen so far (the next token's position) */
} samba_decode_state;

/* Optional taps of intermediate results (each NULL or [B, L, d_model] dtype). */
typedef struct {
  void* branch[4]; /* f(RMSNorm(x)) of Mamba, MLP1, SWA, MLP2, before the residual add */
  void* resid[3];  /* residual stream after Mamba, MLP1, SWA (x_out is the fourth) */
} samba_block_taps;

size_t samba_block_workspace_size(const samba_block_config* cfg, int B, int L);

/* One block over a fresh sequence (positions 0..L-1) [Samba §3.2 "Big-Picture
 * Architecture": every layer pre-RMSNorm with a residual add; §3.4 "Detailed,
 * Sentence-Based Technical Breakdown": the Mamba layer per "The Mamba Layer",
 * "Input-Dependent Selective Gating (The Delta Parameter)", "The State Space
 * Model Update (S6)" and "Gated Output"; the SWA layer per "Window
 * Specification" (keys t-w+1..t), "Positional Encoding" (RoPE, base 10,000)
 * and the Llama-3-style GQA heads of the configuration; the MLPs per "The
 * SwiGLU MLP Layer" ("SwiGLU Formulation")]:
 *   x1 = x  + Mamba(RMSNorm(x)); x2 = x1 + MLP1(RMSNorm(x1));
 *   x3 = x2 + SWA(RMSNorm(x2));  x_out = x3 + MLP2(RMSNorm(x3)).
 * x_in, x_out: [B, L, d_model] dtype (must not alias; may be NULL when L == 0).  If st != NULL it is
 * overwritten with the decode state after the last token (SSM state, the last
 * d_conv-1 pre-conv inputs, the last min(L, window) post-RoPE keys/values in
 * their ring slots, pos[b] = L).  taps may be NULL.
 * Requirements: d_state == 16, head_dim in {16, 32, 64} (64 or 256 on the bf16
 * tensor-core path), d_model, d_inner, d_ff multiples of 64, dt_rank a multiple
 * of 8, n_q % n_kv == 0.  samba_step takes the same head dims (at head_dim 256
 * its attention runs on the CUDA-core decode kernel). */
samba_status samba_block_fwd(const samba_block_config* cfg, const samba_block_weights* w, const void* x_in,
                             void* x_out, samba_decode_state* st, const samba_block_taps* taps, int B, int L,
                             void* workspace, size_t workspace_bytes, samba_stream stream);

/* ------------------------------------------------------------------------
 * Chunked prefill: the block over the next L tokens of sequences that have
 * already seen pos0 tokens [blog page "Samba Guide: Hybrid Mamba & Sliding
 * Window Architecture", "Production Deployment & Long-Context Best Practices",
 * item 3 "Chunked Prefilling for 1M-Token Sequences": process a long prompt in
 * chunks, carrying the recurrent state forward, so activation memory is bounded
 * by the chunk].
 *
 * st holds the decode state after pos0 tokens (from samba_block_fwd, an earlier
 * chunk, or samba_step); pos[b] must equal pos0 for every row, which a device
 * check verifies (mismatch: SAMBA_ERR_DEVICE from samba_get_error; outputs and
 * state are then undefined).  The chunk's conv inputs continue the d_conv-1
 * carried inputs, its scan starts from st->ssm, its queries attend to the ring's
 * keys of the min(pos0, window-1) preceding positions and to the chunk's own, and
 * RoPE positions are pos0..pos0+L-1.  On return st holds the state after
 * pos0 + L tokens, so x_out equals rows pos0..pos0+L-1 of samba_block_fwd over
 * the whole prefix (up to rounding).  pos0 == 0 is samba_block_fwd with st.
 * The workspace (samba_block_chunk_workspace_size) depends on B and L only and
 * holds the chunk's activations plus B*(window-1+L) rows of keys and values.
 * Requirements as samba_block_fwd; pos0 + L <= 2^30.
 * ---------------------------------------------------------------------- */
size_t samba_block_chunk_workspace_size(const samba_block_config* cfg, int B, int L);

samba_status samba_block_fwd_chunk(const samba_block_config* cfg, const samba_block_weights* w, const void* x_in,
                                   void* x_out, samba_decode_state* st, int64_t pos0, const samba_block_taps* taps,
                                   int B, int L, void* workspace, size_t workspace_bytes, samba_stream stream);

/* ------------------------------------------------------------------------
 * A language-model stack: token embedding, a sequence of pre-RMSNorm residual
 * sub-layers, final RMSNorm, vocabulary projection [Samba §3.2 "Big-Picture
 * Architecture": token embeddings enter the first layer, the layers repeat
 * Mamba -> MLP -> Mamba -> MLP -> SWA -> MLP (2:1 Mamba to SWA), each preceded
 * by RMSNorm and followed by a residual add, and the last layer's output is
 * projected to vocabulary logits].  The same entry point runs any layout, e.g.
 * a GQA Transformer as (SWA with window >= L, MLP) pairs.
 * ---------------------------------------------------------------------- */
typedef enum { SAMBA_LAYER_MAMBA = 0, SAMBA_LAYER_MLP = 1, SAMBA_LAYER_SWA = 2 } samba_layer_kind;

typedef struct {
  samba_block_config cfg;             /* shapes shared by all layers; window >= L is full causal attention */
  int n_layers;
  const int* kinds;                   /* host [n_layers] samba_layer_kind */
  const samba_block_weights* layers;  /* host [n_layers]; a layer reads only the fields of its kind:
                                         Mamba: norm_g[0], W_in, conv_w, conv_b, W_x, W_dt, dt_bias,
                                         A_log, Dskip, W_out;  MLP: norm_g[1], mlp1_W1..W3;
                                         SWA: norm_g[2], Wq, Wk, Wv, Wo */
  const void* embedding;              /* device [vocab, d_model] dtype */
  const float* final_norm;            /* device [d_model] fp32 gain */
  const void* lm_head;                /* device [vocab, d_model] dtype */
  int vocab;
} samba_model;

size_t samba_model_workspace_size(const samba_model* m, int B, int L);

/* Prompt processing: the logits of the last position of each of B sequences.
 * ids: device int32 [B, L], each in [0, vocab) (an id outside it latches
 * SAMBA_ERR_DEVICE for samba_get_error and embeds as a zero row); logits:
 * device [B, vocab] dtype.  The stack runs layer by layer over all B*L tokens
 * (workspace: one block's activations plus two residual streams). */
samba_status samba_model_prefill(const samba_model* m, const int32_t* ids, void* logits, int B, int L,
                                 void* workspace, size_t workspace_bytes, samba_stream stream);

/* Decode state of one sub-layer of a model: Mamba layers use ssm
 * [B, d_inner, d_state] fp32 and conv [B, d_inner, d_conv-1]; SWA layers k_ring
 * and v_ring [B, cfg.window, n_kv, head_dim] (post-RoPE, slot = position mod
 * window; a window at least the longest sequence is a full KV cache); MLP
 * layers none (their fields are ignored).  A new sequence starts from zeroed
 * states and pos = 0. */
typedef struct {
  float* ssm;
  void* conv;
  void* k_ring;
  void* v_ring;
} samba_layer_state;

size_t samba_model_step_workspace_size(const samba_model* m, int B);

/* One decode step of the stack for one new token per sequence [the same layers
 * at a single t; Samba §5's constant-cost decoding for Mamba, a window-sized
 * ring for SWA]: ids_t device int32 [B]; logits device [B, vocab] dtype;
 * states host [n_layers]; pos device int64 [B], the tokens each sequence has
 * seen (the new token's position), incremented on return.  Feeding tokens
 * t = 0..T-1 one by one gives, at step t, the logits samba_model_prefill gives
 * for the prefix of t+1 tokens (up to rounding).  Rings above 2048 slots
 * (head_dim 64, bf16) use a split attention whose partials live in the
 * workspace.  Positions are read on the device: the call can be captured in a
 * CUDA graph and replayed. */
samba_status samba_model_step(const samba_model* m, const int32_t* ids_t, void* logits, samba_layer_state* states,
                              int64_t* pos, int B, void* workspace, size_t workspace_bytes, samba_stream stream);

/* ------------------------------------------------------------------------
 * The Samba block, one decode step per sequence (constant cost per token):
 * the layers of samba_block_fwd for one new token [Samba §3.4 "The State Space
 * Model Update (S6)": the recurrence advanced by one step from the carried
 * state; "Window Specification": the new query attends to positions
 * t-w+1..t; the decoding-throughput discussion of Figure 2b; the blog page
 * "Samba Guide: Hybrid Mamba & Sliding Window Architecture", "Sliding Window
 * KV Eviction Configuration": a w-slot ring, slot = position mod w]
 *
 * x_t, y_t: [B, d_model] dtype.  For each row b with p = pos[b]: the Mamba layer
 * advances the conv state and the SSM state by one step; the SWA layer writes
 * RoPE(k)/v at ring slot p mod window and attends over the min(p+1, window)
 * most recent slots; pos[b] becomes p + 1.  All state updates are in place and
 * read positions from device memory, so the call can be captured in a CUDA graph
 * and replayed.  On the bf16 tensor-core path (B <= 64) the three RMSNorms after
 * the first are completed inside the projections around them (the producer of a
 * stream row also writes the norm's input and per-8-feature sums of squares, the
 * consumer scales its rows): the same result up to rounding, bit-reproducible
 * from run to run; the environment variable SAMBA_NORM_FOLD=0 launches the norms
 * separately instead.  samba_model_step does the same across its stack.
 * ---------------------------------------------------------------------- */
/* Workspace of samba_step: one block's activations for B tokens (with the norm
 * fold's sums of squares) and, for rings above 2048 slots, the per-slice
 * partials of the decode attention. */
size_t samba_step_workspace_size(const samba_block_config* cfg, int B);

samba_status samba_step(const samba_block_config* cfg, const samba_block_weights* w, const void* x_t, void* y_t,
                        samba_decode_state* st, int B, void* workspace, size_t workspace_bytes,
                        samba_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* SAMBA_H_ */
