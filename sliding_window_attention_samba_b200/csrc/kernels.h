// Internal launcher interfaces of libsamba (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/samba.h"

namespace samba {

// Grid limits the launchers check before launching: batch rows and heads go to
// grid y/z (at most 65535 each); the conv kernel puts 32-token runs on grid y.
constexpr int kMaxGridYZ = 65535;
constexpr int kConvRunTokens = 32;
constexpr int64_t kMaxConvTokens = (int64_t)kMaxGridYZ * kConvRunTokens;

// ---------------- debug-check build: workspace guard bands ----------------
#if defined(SAMBA_DEBUG_CHECKS) && SAMBA_DEBUG_CHECKS
constexpr size_t kGuardBytes = 4096;
#else
constexpr size_t kGuardBytes = 0;
#endif
constexpr int kMaxGuards = 48;
constexpr int kGuardSiteTu = 15;  // site file id that names a guard band (the line is its index)
struct GuardList {
  int n = 0;
  size_t off[kMaxGuards];
};
// Fill each band [base + off[i], + kGuardBytes) with a fixed pattern / verify
// it after the call (a changed band latches kErrBounds naming its index).
samba_status launch_guard_fill(char* base, const GuardList& g, cudaStream_t st);
samba_status launch_guard_check(const char* base, const GuardList& g, cudaStream_t st);
// One device check on an index made out of range on purpose (debug-check self-test).
samba_status launch_dcheck_selftest(cudaStream_t st);

// ---------------- selective scan ----------------
struct ScanArgs {
  const void* u = nullptr;
  const void* dt = nullptr;       // Delta (or dt before softplus); NULL with dt_low below
  // folded dt projection (bf16, dt_rank R <= 128, R % 16 == 0): Delta =
  // softplus(dt_low W_dt^T + dt_bias) formed in the scan from dt_low [B, L, R]
  // (row stride ld_dtl) and W_dt [D, R]
  const void* dt_low = nullptr;
  int64_t ld_dtl = 0;
  int R = 0;
  const void* W_dt = nullptr;
  const void* z = nullptr;
  const void* Bm = nullptr;
  const void* Cm = nullptr;
  void* y = nullptr;
  int64_t ld_u = 0, ld_dt = 0, ld_z = 0, ld_bc = 0, ld_y = 0;  // row strides (elements)
  const float* dt_bias = nullptr;
  const float* A_log = nullptr;
  const float* Dskip = nullptr;
  const float* h0 = nullptr;
  float* hT = nullptr;
  int B = 0, L = 0, D = 0, N = 0;
  bool softplus = true;
  samba_dtype dtype = SAMBA_BF16;
};
samba_status validate_scan(const ScanArgs& a);
bool scan_dt_fold_supported(const ScanArgs& a);
samba_status launch_selective_scan(const ScanArgs& a, cudaStream_t st);

// ---------------- RoPE ----------------
// Table of (cos, sin) pairs: [3][1024][half] float2 for angle p * theta_i with
// p = a*2^20 + b*2^10 + c; entries built in fp64.
constexpr int kRopeLevels = 3;
constexpr int kRopeRadix = 1024;
size_t rope_table_bytes(int head_dim);
samba_status launch_build_rope_table(float2* tab, int head_dim, float base, cudaStream_t st, bool pdl = false);
// out[b,t,h,:] = RoPE(x[b,t,h,:], pos0 + t); x may alias out.
samba_status launch_rope_apply(const void* x, void* out, int B, int L, int H, int head_dim, int64_t pos0,
                               const float2* tab, samba_dtype dt, cudaStream_t st);

// ---------------- token embedding ----------------
// out[t, :] = table[ids[t], :]; ids outside [0, vocab) latch kErrDevice and give zeros.
samba_status launch_embedding(const int32_t* ids, const void* table, void* out, int64_t T, int d_model, int vocab,
                              samba_dtype dt, cudaStream_t st);

// ---------------- RMSNorm ----------------
samba_status launch_rmsnorm(const void* x, int64_t ld_x, const float* g, void* out, int64_t ld_out, int64_t rows,
                            int dim, float eps, samba_dtype dt, cudaStream_t st, bool pdl = false);

// ---------------- causal conv ----------------
struct ConvArgs {
  const void* x = nullptr;
  int64_t ld_x = 0;
  const float* w = nullptr;
  const float* bias = nullptr;
  void* u = nullptr;
  void* state = nullptr;       // out: [B, D, k-1] the last k-1 inputs, oldest first (may be NULL)
  const void* hist = nullptr;  // in: [B, D, k-1] the k-1 inputs before token 0, oldest first; NULL = zeros.
                               // Must not alias `state`.
  int B = 0, L = 0, D = 0, k = 0;
  samba_dtype dtype = SAMBA_BF16;
};
samba_status launch_causal_conv(const ConvArgs& a, cudaStream_t st);

// ---------------- dense projections ----------------
enum GemmEpi : int { kEpiNone = 0, kEpiResid = 1, kEpiSwiglu = 2, kEpiSoftplus = 3, kEpiRope = 4 };

struct GemmSeg {
  const void* W = nullptr;   // [n, K] row-major (row stride K)
  const void* W2 = nullptr;  // SwiGLU gate weights [n, K]
  int n = 0;                 // output columns of this segment
};

struct GemmArgs {
  const void* A = nullptr;  // [M, K], row stride lda
  int64_t lda = 0;
  int nseg = 1;
  GemmSeg seg[3];           // B operand, segments concatenated along N
  int64_t M = 0;
  int N = 0, K = 0;         // N = sum of seg[i].n
  int epi = kEpiNone;
  void* out = nullptr;      // [M, N], row stride ldo
  int64_t ldo = 0;
  const void* resid = nullptr;  // kEpiResid: out = resid + acc
  int64_t ldr = 0;
  void* tap = nullptr;          // kEpiResid: optional copy of acc (before the residual add)
  int64_t ldt = 0;
  const float* bias = nullptr;  // kEpiSoftplus
  // kEpiRope: columns [0, rope_cols) are rotated per head of head_dim;
  // position = pos_dev ? pos_dev[row] : pos0 + row % seq_len.
  int rope_cols = 0, head_dim = 0, seq_len = 1;
  int64_t pos0 = 0;
  const int64_t* pos_dev = nullptr;
  const float2* rope_tab = nullptr;
  // skinny kernel only (see gemm_takes_skinny): rope_tab may be NULL when
  // rope_base > 0, the rotation then evaluated from the position directly
  float rope_base = 0.f;
  // decode (skinny kernel only, see gemm_takes_skinny): also write the key and
  // value columns [ring_k_col, +ring_kvw) and [ring_v_col, +ring_kvw) of row b
  // into slot pos_dev[b] mod ring_window of k_ring / v_ring ([M, window, kvw])
  void* k_ring = nullptr;
  void* v_ring = nullptr;
  int ring_window = 0, ring_k_col = 0, ring_v_col = 0, ring_kvw = 0;
  // decode (skinny kernel only, kEpiNone): columns [0, conv_cols) are the
  // short convolution's new input x; instead of writing them to out, the kernel
  // forms u = SiLU(conv_b + sum_j conv_w[c, j] win_j) over win = [conv_state
  // (d_conv - 1 oldest first), x] into conv_u ([M, conv_cols]) and shifts x
  // into conv_state ([M, conv_cols, d_conv - 1]); d_conv == 4
  const float* conv_w = nullptr;
  const float* conv_b = nullptr;
  void* conv_state = nullptr;
  void* conv_u = nullptr;
  int conv_cols = 0, conv_k = 0;
  // decode norm fold (skinny kernel only).  ss_in != NULL: the A rows are
  // x (.) g of stream rows x, and ss_in[b * norm_dim/8 + j] holds the sum of
  // squares of x[b, 8j .. 8j+8); output row b is scaled by
  // rsqrt(sum_j ss_in[b, j] / norm_dim + norm_eps), which completes
  // RMSNorm(x) W^T.  ss_out != NULL (kEpiResid): also writes bf16(out) (.) g_next
  // to xg_out (row stride ldo) and the sums of squares of every 8 stored
  // features to ss_out[b * N/8 + n/8] -- one writer per slot, summed in a fixed
  // order by the consumer, so the result is deterministic
  const float* ss_in = nullptr;
  int norm_dim = 0;
  float norm_eps = 0.f;
  const float* g_next = nullptr;
  void* xg_out = nullptr;
  float* ss_out = nullptr;
  // decode (skinny kernel only): add 1 to pos_inc[0 .. M) once the kernel's
  // prerequisites have completed (the last projection of a step)
  int64_t* pos_inc = nullptr;
  samba_dtype dtype = SAMBA_BF16;
  bool pdl = false;  // launch as a programmatic dependent of the previous kernel (decode path)
};
samba_status launch_gemm(const GemmArgs& a, cudaStream_t st);       // picks the kernel
// Measurement hook: while installed, launches of epilogue kind `epi` record
// start[i] / stop[i] on their stream around the kernel (i counts the launches).
samba_status gemm_timing_set(int epi, void* const* start, void* const* stop, int capacity);
int gemm_timing_count();
samba_status launch_gemm_simt(const GemmArgs& a, cudaStream_t st);  // CUDA-core fp32 FMA kernel
samba_status launch_gemm_tc(const GemmArgs& a, cudaStream_t st);    // tcgen05 kernel (bf16)
bool gemm_tc_supported(const GemmArgs& a);
samba_status launch_gemm_skinny(const GemmArgs& a, cudaStream_t st);  // M <= 64: swap-AB, cluster split-K
bool gemm_skinny_supported(const GemmArgs& a);
// launch_gemm runs these arguments on the skinny kernel (the only one that
// honours the ring and pos_inc fields)
bool gemm_takes_skinny(const GemmArgs& a);

// ---------------- sliding-window attention ----------------
struct SwaArgs {
  const void* q = nullptr;  // [B, L, Hq, d] rows of stride ld_q elements per token
  const void* k = nullptr;  // [B, L + qoff, Hkv, d]
  const void* v = nullptr;
  void* o = nullptr;        // [B, L, Hq, d]
  int64_t ld_q = 0, ld_k = 0, ld_v = 0, ld_o = 0;  // elements between consecutive tokens
  int B = 0, L = 0, Hq = 0, Hkv = 0, d = 0, window = 0;
  int qoff = 0;             // query row t is key row t + qoff (keys of earlier tokens lead the K/V rows)
  float scale = 0.f;
  samba_dtype dtype = SAMBA_BF16;
};
samba_status launch_swa(const SwaArgs& a, cudaStream_t st);
samba_status launch_swa_simt(const SwaArgs& a, cudaStream_t st);
samba_status launch_swa_tc(const SwaArgs& a, cudaStream_t st);
bool swa_tc_supported(const SwaArgs& a);

}  // namespace samba
