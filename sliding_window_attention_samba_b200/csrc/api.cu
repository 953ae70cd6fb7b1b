// C ABI of libsamba: validation, workspace carving and the launch sequences of
// the Samba block prefill and decode step [Samba 3.2 "Big-Picture
// Architecture"; 3.4 "Detailed, Sentence-Based Technical Breakdown"].
#include <algorithm>
#include <initializer_list>
#include <mutex>
#include <map>
#include <set>
#include <utility>
#include <stdio.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

#define SAMBA_TU_ID 1  // site id of this file in debug-check reports
#include "common.cuh"
#include "decode.h"
#include "kernels.h"

namespace samba {

// NVTX range around an entry point or a sub-layer's launches (host-side
// markers for profilers; inert unless a tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// ---------------------------------------------------------------------------
// Device error word
// ---------------------------------------------------------------------------
__device__ int g_error_word = 0;

// Identity of the calling thread's current CUDA context.  A module-scope
// __device__ variable lives in the context that loaded the module, so a
// device address cached for it is only valid while that context lives: after
// cudaDeviceReset the device gets a new primary context and the address is
// looked up again.
uintptr_t current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  static GetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return 0;
  return reinterpret_cast<uintptr_t>(c);
}

int* device_error_word() {
  static int* addr[64] = {nullptr};
  static uintptr_t ctx[64] = {0};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  const uintptr_t c = current_context_id();  // 0 before the runtime's first call made one current
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev] || ctx[dev] != c) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int*>(p);
    ctx[dev] = c;
  }
  return addr[dev];
}

// ---------------------------------------------------------------------------
// The CUDA error behind the last SAMBA_ERR_CUDA of the calling thread
// ---------------------------------------------------------------------------
static thread_local char g_cuda_err_msg[256] = {0};
samba_status note_cuda_failure(const char* where, int cuda_error) {
  snprintf(g_cuda_err_msg, sizeof(g_cuda_err_msg), "%s: %s (%d)", where,
           cudaGetErrorString((cudaError_t)cuda_error), cuda_error);
  return SAMBA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Site of the last failed debug check read by samba_get_error (calling thread)
// ---------------------------------------------------------------------------
static thread_local char g_check_site[96] = {0};
static void note_check_site(int word) {
  static const char* const files[16] = {"?", "api.cu", "decode.cu", "elementwise.cu", "gemm.cu", "gemm_skinny.cu",
                                        "scan.cu", "swa.cu", "swa_noalloc.cu", "swa_tc.cu", "?", "?", "?", "?",
                                        "?", "workspace guard band"};
  const int tu = (word >> 4) & 15, line = (word >> 8) & 0x7fffff;
  if (tu == kGuardSiteTu)
    snprintf(g_check_site, sizeof(g_check_site), "%s %d overwritten", files[tu], line);
  else
    snprintf(g_check_site, sizeof(g_check_site), "%s:%d", files[tu], line);
}

// ---------------------------------------------------------------------------
// Failure-detection test hook of the selective scan
// ---------------------------------------------------------------------------
static std::mutex g_stall_mu;
static StallHook g_stall = {-1, kWaitLimitNs};
StallHook scan_stall_hook() {
  std::lock_guard<std::mutex> lk(g_stall_mu);
  return g_stall;
}

// ---------------------------------------------------------------------------
// Per-(kernel, device) record of raised shared-memory limits
// ---------------------------------------------------------------------------
static std::mutex g_attr_mu;
static std::map<std::pair<const void*, int>, size_t> g_attr_done;
bool smem_attr_done(const void* kern, int dev, size_t bytes) {
  std::lock_guard<std::mutex> lk(g_attr_mu);
  auto it = g_attr_done.find({kern, dev});
  return it != g_attr_done.end() && it->second >= bytes;
}
void smem_attr_mark(const void* kern, int dev, size_t bytes) {
  std::lock_guard<std::mutex> lk(g_attr_mu);
  size_t& v = g_attr_done[{kern, dev}];
  if (bytes > v) v = bytes;
}

// ---------------------------------------------------------------------------
// Tensor maps through the driver entry point (no link-time libcuda dependency)
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_tmap(CUtensorMap* m, const void* base, samba_dtype dt, int rank, const uint64_t* dims,
               const uint64_t* strides_elems, const uint32_t* box, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  const size_t es = dtype_size(dt);
  cuuint64_t gdim[5], gstride[4];
  cuuint32_t bdim[5], estride[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estride[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gstride[i] = strides_elems[i] * es;
  CUresult r = fn(m, dt == SAMBA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  (cuuint32_t)rank, const_cast<void*>(base), gdim, gstride, bdim, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    snprintf(g_cuda_err_msg, sizeof(g_cuda_err_msg), "cuTensorMapEncodeTiled: CUresult %d", (int)r);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// Workspace carving (256-byte aligned sub-buffers)
// ---------------------------------------------------------------------------
// Workspace carving: 256-byte aligned sub-buffers.  In the debug-check build
// every sub-buffer is followed by a guard band that is filled with a pattern
// before the call's kernels run and verified after them (guards_arm /
// guards_check), so a kernel that writes past the end of its buffer is
// reported as SAMBA_ERR_BOUNDS naming the band.
struct Carve {
  size_t off = 0;
  int nguard = 0;
  size_t guard[kMaxGuards];
  size_t take(size_t bytes) {
    const size_t o = off;
    off = (off + bytes + 255) & ~size_t(255);
    if (kGuardBytes && nguard < kMaxGuards) {
      guard[nguard++] = off;
      off += kGuardBytes;
    }
    return o;
  }
};

static samba_status guards_arm(char* base, const Carve& c, cudaStream_t st) {
  if (!c.nguard) return SAMBA_OK;
  GuardList g;
  g.n = c.nguard;
  for (int i = 0; i < c.nguard; ++i) g.off[i] = c.guard[i];
  return launch_guard_fill(base, g, st);
}
static samba_status guards_check(char* base, const Carve& c, cudaStream_t st) {
  if (!c.nguard) return SAMBA_OK;
  GuardList g;
  g.n = c.nguard;
  for (int i = 0; i < c.nguard; ++i) g.off[i] = c.guard[i];
  return launch_guard_check(base, g, st);
}

struct BlockPlan {
  size_t tab, xn, hz, u, xdbl, dlt, y, x1, x2, x3, hmlp, qkv, o, kx, vx, convh, ss, total;
  int xdw, qkvw;
  Carve cv;  // the carving (guard bands of the debug-check build)
};

// Workspace of one block over T = B*L tokens; a chunked prefill (chunk_B > 0)
// adds the K/V rows of the preceding window and a copy of the conv history.
static BlockPlan plan_block(const samba_block_config& c, int64_t T, int chunk_B = 0) {
  BlockPlan p;
  const size_t es = dtype_size(c.dtype);
  p.xdw = c.dt_rank + 2 * c.d_state;
  p.qkvw = (c.n_q + 2 * c.n_kv) * c.head_dim;
  Carve cv;
  p.tab = cv.take(rope_table_bytes(c.head_dim));
  p.xn = cv.take(T * c.d_model * es);
  p.hz = cv.take(T * 2 * c.d_inner * es);
  p.u = cv.take(T * c.d_inner * es);
  p.xdbl = cv.take(T * p.xdw * es);
  p.dlt = cv.take(T * c.d_inner * es);
  p.y = cv.take(T * c.d_inner * es);
  p.x1 = cv.take(T * c.d_model * es);
  p.x2 = cv.take(T * c.d_model * es);
  p.x3 = cv.take(T * c.d_model * es);
  p.hmlp = cv.take(T * c.d_ff * es);
  p.qkv = cv.take(T * p.qkvw * es);
  p.o = cv.take(T * c.n_q * c.head_dim * es);
  const int64_t kv_rows = chunk_B > 0 ? T + (int64_t)chunk_B * (c.window - 1) : 0;
  p.kx = cv.take(kv_rows * c.n_kv * c.head_dim * es);
  p.vx = cv.take(kv_rows * c.n_kv * c.head_dim * es);
  p.convh = cv.take((int64_t)chunk_B * c.d_inner * (c.d_conv - 1) * es);
  // decode norm fold: partial sums of squares of norms 1..3, d_model/8 per row, for up to 64 rows
  p.ss = cv.take((size_t)3 * std::min<int64_t>(T, 64) * (c.d_model / 8) * sizeof(float));
  p.total = cv.off + 256;  // slack for aligning the caller's base pointer
  p.cv = cv;
  return p;
}

static samba_status validate_cfg(const samba_block_config* c) {
  if (!c) return SAMBA_ERR_INVALID_ARG;
  if (c->d_model <= 0 || c->d_inner <= 0 || c->d_state <= 0 || c->d_conv <= 0 || c->dt_rank <= 0 || c->n_q <= 0 ||
      c->n_kv <= 0 || c->head_dim <= 0 || c->window <= 0 || c->d_ff <= 0)
    return SAMBA_ERR_INVALID_ARG;
  if (c->dtype != SAMBA_F32 && c->dtype != SAMBA_BF16) return SAMBA_ERR_INVALID_ARG;
  if (c->n_q % c->n_kv) return SAMBA_ERR_INVALID_ARG;
  if (c->d_state != 16 || c->d_conv < 2 || c->d_conv > 8) return SAMBA_ERR_UNSUPPORTED;
  // head_dim 256 (the 3.8B shapes) runs on the bf16 tensor-core path only
  if (c->head_dim != 16 && c->head_dim != 32 && c->head_dim != 64 && !(c->head_dim == 256 && c->dtype == SAMBA_BF16))
    return SAMBA_ERR_UNSUPPORTED;
  if (c->d_model % 64 || c->d_inner % 64 || c->d_ff % 64) return SAMBA_ERR_UNSUPPORTED;
  const size_t es = dtype_size(c->dtype);
  if ((c->dt_rank * es) % 16) return SAMBA_ERR_UNSUPPORTED;
  return SAMBA_OK;
}

static samba_status validate_weights(const samba_block_weights* w) {
  if (!w) return SAMBA_ERR_INVALID_ARG;
  const void* req[] = {w->norm_g[0], w->norm_g[1], w->norm_g[2], w->norm_g[3], w->W_in, w->conv_w, w->W_x,
                       w->W_dt, w->dt_bias, w->A_log, w->Dskip, w->W_out, w->Wq, w->Wk, w->Wv, w->Wo,
                       w->mlp1_W1, w->mlp1_W2, w->mlp1_W3, w->mlp2_W1, w->mlp2_W2, w->mlp2_W3};
  for (const void* p : req)
    if (!p) return SAMBA_ERR_INVALID_ARG;
  for (const void* p : req)
    if (!aligned16(p)) return SAMBA_ERR_UNSUPPORTED;
  return SAMBA_OK;
}

#define TRY(x)                            \
  do {                                    \
    samba_status s_ = (x);                \
    if (s_ != SAMBA_OK) return s_;        \
  } while (0)

static GemmArgs gemm1(const void* A, int64_t lda, const void* W, int64_t M, int N, int K, void* out, int64_t ldo,
                      samba_dtype dt) {
  GemmArgs g;
  g.A = A;
  g.lda = lda;
  g.nseg = 1;
  g.seg[0].W = W;
  g.seg[0].n = N;
  g.M = M;
  g.N = N;
  g.K = K;
  g.out = out;
  g.ldo = ldo;
  g.dtype = dt;
  return g;
}

// SwiGLU MLP sub-layer: x_next = x + W3 ((W1 xn) * SiLU(W2 xn))  [Samba 3.4 "SwiGLU Formulation"]
// Decode (pdl): pos_inc / pos_done let the down projection advance the
// positions; ss_in / ss_out / g_next are the norm fold (the up projection
// completes this sub-layer's RMSNorm, the down projection writes the next one's
// input and sums of squares).
static samba_status mlp_sublayer(const samba_block_config& c, const float* g, const void* W1, const void* W2,
                                 const void* W3, const void* x, void* x_next, void* xn, void* hmlp, void* tap,
                                 int64_t T, cudaStream_t st, bool pdl = false, int64_t* pos_inc = nullptr,
                                 bool* pos_done = nullptr, const float* ss_in = nullptr, float* ss_out = nullptr,
                                 const float* g_next = nullptr) {
  NvtxRange nvtx_("samba.mlp");
  // ss_in (decode norm fold): xn already holds x (.) g from the producer of x
  if (!ss_in) TRY(launch_rmsnorm(x, c.d_model, g, xn, c.d_model, T, c.d_model, c.norm_eps, c.dtype, st, pdl));
  GemmArgs up = gemm1(xn, c.d_model, W1, T, c.d_ff, c.d_model, hmlp, c.d_ff, c.dtype);
  up.seg[0].W2 = W2;
  up.epi = kEpiSwiglu;
  up.pdl = pdl;
  up.ss_in = ss_in;
  up.norm_dim = c.d_model;
  up.norm_eps = c.norm_eps;
  TRY(launch_gemm(up, st));
  GemmArgs dn = gemm1(hmlp, c.d_ff, W3, T, c.d_model, c.d_ff, x_next, c.d_model, c.dtype);
  dn.pdl = pdl;
  dn.epi = kEpiResid;
  dn.resid = x;
  dn.ldr = c.d_model;
  dn.tap = tap;
  dn.ldt = c.d_model;
  if (ss_out) {  // the next norm's input and sums of squares
    dn.ss_out = ss_out;
    dn.g_next = g_next;
    dn.xg_out = xn;
  }
  if (pos_inc) {  // decode: the step's last projection also advances the positions
    GemmArgs dp = dn;
    dp.pos_inc = pos_inc;
    if (gemm_takes_skinny(dp)) {
      dn = dp;
      *pos_done = true;
    }
  }
  return launch_gemm(dn, st);
}

}  // namespace samba

using namespace samba;

extern "C" {

const char* samba_status_string(samba_status s) {
  switch (s) {
    case SAMBA_OK: return "SAMBA_OK";
    case SAMBA_ERR_INVALID_ARG: return "SAMBA_ERR_INVALID_ARG";
    case SAMBA_ERR_UNSUPPORTED: return "SAMBA_ERR_UNSUPPORTED";
    case SAMBA_ERR_CUDA: return "SAMBA_ERR_CUDA";
    case SAMBA_ERR_TIMEOUT: return "SAMBA_ERR_TIMEOUT";
    case SAMBA_ERR_DEVICE: return "SAMBA_ERR_DEVICE";
    case SAMBA_ERR_BOUNDS: return "SAMBA_ERR_BOUNDS";
  }
  return "SAMBA_ERR_UNKNOWN";
}

const char* samba_version(void) { return "samba-b200 0.1 (sm_100a)"; }

const char* samba_last_cuda_error(void) { return g_cuda_err_msg; }

samba_status samba_set_gemm_timing(int epi, void* const* start_events, void* const* stop_events, int capacity) {
  return gemm_timing_set(epi, start_events, stop_events, capacity);
}

int samba_gemm_timing_count(void) { return gemm_timing_count(); }

samba_status samba_debug_scan_stall(int stop_after_chunks, uint64_t wait_limit_ns) {
  if (stop_after_chunks < -1) return SAMBA_ERR_INVALID_ARG;
  if (stop_after_chunks >= 0 && (wait_limit_ns < 1000000ull || wait_limit_ns > kWaitLimitNs))
    return SAMBA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_stall_mu);
  g_stall.stop_chunk = stop_after_chunks;
  g_stall.wait_limit_ns = stop_after_chunks >= 0 ? wait_limit_ns : kWaitLimitNs;
  return SAMBA_OK;
}

samba_status samba_get_error(samba_stream stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return SAMBA_ERR_CUDA;
  int* w = device_error_word();
  if (!w) return SAMBA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SAMBA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return SAMBA_ERR_CUDA;
  }
  if ((v & 15) == kErrBounds) {
    note_check_site(v);
    return SAMBA_ERR_BOUNDS;
  }
  return v == kErrTimeout ? SAMBA_ERR_TIMEOUT : (v ? SAMBA_ERR_DEVICE : SAMBA_OK);
}

int samba_debug_checks_enabled(void) { return SAMBA_DEBUG_CHECKS; }

size_t samba_debug_selftest_workspace_size(void) {
  Carve cv;
  cv.take(4096);
  cv.take(4096);
  return cv.off + 256;
}

samba_status samba_debug_check_selftest(int kind, void* workspace, size_t workspace_bytes, samba_stream stream) {
  cudaStream_t st = (cudaStream_t)stream;
  if (kind != 0 && kind != 1) return SAMBA_ERR_INVALID_ARG;
  if (!SAMBA_DEBUG_CHECKS) return SAMBA_ERR_UNSUPPORTED;
  if (kind == 0) return launch_dcheck_selftest(st);
  if (!workspace || workspace_bytes < samba_debug_selftest_workspace_size()) return SAMBA_ERR_INVALID_ARG;
  char* base = (char*)(((uintptr_t)workspace + 255) & ~uintptr_t(255));
  Carve cv;
  cv.take(4096);
  cv.take(4096);
  TRY(guards_arm(base, cv, st));
  // one byte of the first band: inside the caller's workspace, outside every sub-buffer
  if (cudaMemsetAsync(base + cv.guard[0] + 17, 0x11, 1, st) != cudaSuccess)
    return note_cuda_failure("cudaMemsetAsync (guard self-test)", cudaGetLastError());
  return guards_check(base, cv, st);
}

const char* samba_last_check_site(void) { return g_check_site; }

// ------------------------------------------------------------------ scan
size_t samba_selective_scan_workspace_size(int, int, int, int) { return 0; }

samba_status samba_selective_scan(const void* u, const void* dt, const float* dt_bias, int dt_softplus,
                                  const float* A_log, const void* Bm, const void* Cm, const float* Dskip,
                                  const void* z, const float* h0, float* hT, void* y, int B, int L, int D, int N,
                                  samba_dtype dtype, void*, size_t, samba_stream stream) {
  NvtxRange nvtx_("samba_selective_scan");
  if (dtype != SAMBA_F32 && dtype != SAMBA_BF16) return SAMBA_ERR_INVALID_ARG;
  ScanArgs a;
  a.u = u;
  a.dt = dt;
  a.z = z;
  a.Bm = Bm;
  a.Cm = Cm;
  a.y = y;
  a.ld_u = a.ld_dt = a.ld_z = a.ld_y = D;
  a.ld_bc = N;
  a.dt_bias = dt_bias;
  a.A_log = A_log;
  a.Dskip = Dskip;
  a.h0 = h0;
  a.hT = hT;
  a.B = B;
  a.L = L;
  a.D = D;
  a.N = N;
  a.softplus = dt_softplus != 0;
  a.dtype = dtype;
  return launch_selective_scan(a, (cudaStream_t)stream);
}

samba_status samba_selective_scan_xdbl(const void* u, const void* x_dbl, int dt_rank, const void* W_dt,
                                       const float* dt_bias, const float* A_log, const float* Dskip, const void* z,
                                       const float* h0, float* hT, void* y, int B, int L, int D, int N,
                                       samba_dtype dtype, samba_stream stream) {
  NvtxRange nvtx_("samba_selective_scan_xdbl");
  if (dtype != SAMBA_F32 && dtype != SAMBA_BF16) return SAMBA_ERR_INVALID_ARG;
  if (!x_dbl || !W_dt || dt_rank < 1 || N < 1) return SAMBA_ERR_INVALID_ARG;
  ScanArgs a;
  a.u = u;
  a.dt_low = x_dbl;
  a.ld_dtl = (int64_t)dt_rank + 2 * (int64_t)N;
  a.R = dt_rank;
  a.W_dt = W_dt;
  a.z = z;
  a.Bm = (const char*)x_dbl + (size_t)dt_rank * dtype_size(dtype);
  a.Cm = (const char*)x_dbl + (size_t)(dt_rank + N) * dtype_size(dtype);
  a.y = y;
  a.ld_u = a.ld_z = a.ld_y = D;
  a.ld_bc = a.ld_dtl;
  a.dt_bias = dt_bias;
  a.A_log = A_log;
  a.Dskip = Dskip;
  a.h0 = h0;
  a.hT = hT;
  a.B = B;
  a.L = L;
  a.D = D;
  a.N = N;
  a.softplus = true;
  a.dtype = dtype;
  if (!scan_dt_fold_supported(a)) return SAMBA_ERR_UNSUPPORTED;
  return launch_selective_scan(a, (cudaStream_t)stream);
}

// ------------------------------------------------------------------ SWA
size_t samba_swa_workspace_size(int B, int L, int Hq, int Hkv, int head_dim, float rope_base, samba_dtype dtype) {
  if (rope_base == 0.f || B <= 0 || L <= 0) return 0;
  Carve cv;
  const size_t es = dtype_size(dtype);
  cv.take(rope_table_bytes(head_dim));
  cv.take((size_t)B * L * Hq * head_dim * es);
  cv.take((size_t)B * L * Hkv * head_dim * es);
  return cv.off + 256;
}

samba_status samba_swa_fwd(const void* q, const void* k, const void* v, void* o, int B, int L, int Hq, int Hkv,
                           int head_dim, int window, float rope_base, int64_t pos0, float softmax_scale,
                           samba_dtype dtype, void* workspace, size_t workspace_bytes, samba_stream stream) {
  NvtxRange nvtx_("samba_swa_fwd");
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype != SAMBA_F32 && dtype != SAMBA_BF16) return SAMBA_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || B < 1 || L < 0 || Hq < 1 || Hkv < 1 || window < 1 || pos0 < 0 || rope_base < 0.f)
    return SAMBA_ERR_INVALID_ARG;
  if (Hq % Hkv) return SAMBA_ERR_INVALID_ARG;
  if (head_dim != 16 && head_dim != 32 && head_dim != 64 && !(head_dim == 256 && dtype == SAMBA_BF16))
    return SAMBA_ERR_UNSUPPORTED;
  if (pos0 + (int64_t)L > (int64_t(1) << 30)) return SAMBA_ERR_UNSUPPORTED;
  if (B > kMaxGridYZ || Hq > kMaxGridYZ) return SAMBA_ERR_UNSUPPORTED;  // before the RoPE launches
  if (L == 0) return SAMBA_OK;
  SwaArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.ld_q = (int64_t)Hq * head_dim;
  a.ld_k = a.ld_v = (int64_t)Hkv * head_dim;
  a.ld_o = (int64_t)Hq * head_dim;
  a.B = B;
  a.L = L;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = head_dim;
  a.window = window;
  a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)head_dim);
  a.dtype = dtype;
  if (rope_base != 0.f) {
    const size_t need = samba_swa_workspace_size(B, L, Hq, Hkv, head_dim, rope_base, dtype);
    if (!workspace || workspace_bytes < need) return SAMBA_ERR_INVALID_ARG;
    char* base = (char*)(((uintptr_t)workspace + 255) & ~uintptr_t(255));
    Carve cv;
    const size_t es = dtype_size(dtype);
    float2* tab = (float2*)(base + cv.take(rope_table_bytes(head_dim)));
    void* qr = base + cv.take((size_t)B * L * Hq * head_dim * es);
    void* kr = base + cv.take((size_t)B * L * Hkv * head_dim * es);
    TRY(guards_arm(base, cv, st));
    TRY(launch_build_rope_table(tab, head_dim, rope_base, st));
    TRY(launch_rope_apply(q, qr, B, L, Hq, head_dim, pos0, tab, dtype, st));
    TRY(launch_rope_apply(k, kr, B, L, Hkv, head_dim, pos0, tab, dtype, st));
    a.q = qr;
    a.k = kr;
    TRY(launch_swa(a, st));
    return guards_check(base, cv, st);
  }
  return launch_swa(a, st);
}

// ------------------------------------------------------------------ pieces
samba_status samba_rmsnorm(const void* x, const float* g, void* out, int64_t rows, int dim, float eps,
                           samba_dtype dtype, samba_stream stream) {
  return launch_rmsnorm(x, dim, g, out, dim, rows, dim, eps, dtype, (cudaStream_t)stream);
}

samba_status samba_causal_conv1d(const void* x, int64_t ld_x, const float* w, const float* bias, void* u,
                                 void* conv_state, int B, int L, int D, int k, samba_dtype dtype,
                                 samba_stream stream) {
  ConvArgs a;
  a.x = x;
  a.ld_x = ld_x;
  a.w = w;
  a.bias = bias;
  a.u = u;
  a.state = conv_state;
  a.B = B;
  a.L = L;
  a.D = D;
  a.k = k;
  a.dtype = dtype;
  return launch_causal_conv(a, (cudaStream_t)stream);
}

samba_status samba_linear(const void* x, const void* W, const void* W2, const float* bias, const void* resid,
                          void* out, int64_t M, int N, int K, samba_epilogue epilogue, samba_dtype dtype,
                          samba_stream stream) {
  if (K % 8 || N % 8) return SAMBA_ERR_UNSUPPORTED;
  GemmArgs g = gemm1(x, K, W, M, N, K, out, N, dtype);
  switch (epilogue) {
    case SAMBA_EPI_NONE: g.epi = kEpiNone; break;
    case SAMBA_EPI_RESIDUAL: g.epi = kEpiResid; g.resid = resid; g.ldr = N; break;
    case SAMBA_EPI_SWIGLU: g.epi = kEpiSwiglu; g.seg[0].W2 = W2; break;
    case SAMBA_EPI_SOFTPLUS_BIAS: g.epi = kEpiSoftplus; g.bias = bias; break;
    default: return SAMBA_ERR_INVALID_ARG;
  }
  return launch_gemm(g, (cudaStream_t)stream);
}

// ------------------------------------------------------------------ block
size_t samba_block_workspace_size(const samba_block_config* cfg, int B, int L) {
  if (validate_cfg(cfg) != SAMBA_OK || B < 1 || L < 0) return 0;
  return plan_block(*cfg, (int64_t)B * L).total;
}

}  // extern "C"

namespace samba {

// Shapes, workspace plan and stream shared by the sub-layers of one call.
struct LayerCtx {
  const samba_block_config& c;
  const BlockPlan& P;
  char* base;  // workspace, 256-byte aligned
  int B, L;
  int64_t T;
  cudaStream_t st;
};

// Mamba sub-layer over B x L tokens: x_out = x_in + Mamba(RMSNorm(x_in))
// [Samba 3.4 "The Mamba Layer"].  stt: NULL, or the decode state, overwritten
// with the state after the last token (resume: the layer continues from it).
static samba_status mamba_sublayer(const LayerCtx& X, const samba_block_weights* w, const void* x_in, void* x_out,
                                   samba_decode_state* stt, bool resume, void* tap) {
  NvtxRange nvtx_("samba.mamba");
  const samba_block_config& c = X.c;
  const BlockPlan& P = X.P;
  const int B = X.B, L = X.L;
  const int64_t T = X.T;
  cudaStream_t st = X.st;
  const samba_dtype dt = c.dtype;
  auto buf = [&](size_t off) -> void* { return X.base + off; };
  const int Di = c.d_inner, Dm = c.d_model, N = c.d_state, R = c.dt_rank;
  const size_t es = dtype_size(dt);
  void* xn = buf(P.xn);
  char* hz = (char*)buf(P.hz);
  char* xdbl = (char*)buf(P.xdbl);
  TRY(launch_rmsnorm(x_in, Dm, w->norm_g[0], xn, Dm, T, Dm, c.norm_eps, dt, st));
  TRY(launch_gemm(gemm1(xn, Dm, w->W_in, T, 2 * Di, Dm, hz, 2 * Di, dt), st));  // H | X W_g
  {
    ConvArgs ca;
    ca.x = hz;
    ca.ld_x = 2 * Di;
    ca.w = w->conv_w;
    ca.bias = w->conv_b;
    ca.u = buf(P.u);
    ca.state = stt ? stt->conv : nullptr;
    if (resume) {  // the history is read from a copy: the kernel rewrites the state in place
      const size_t bytes = (size_t)B * Di * (c.d_conv - 1) * es;
      if (cudaMemcpyAsync(buf(P.convh), stt->conv, bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return SAMBA_ERR_CUDA;
      ca.hist = buf(P.convh);
    }
    ca.B = B;
    ca.L = L;
    ca.D = Di;
    ca.k = c.d_conv;
    ca.dtype = dt;
    TRY(launch_causal_conv(ca, st));
  }
  TRY(launch_gemm(gemm1(buf(P.u), Di, w->W_x, T, P.xdw, Di, xdbl, P.xdw, dt), st));  // dt_low | B | C
  ScanArgs a;
  // The dt projection can be folded into the scan (bf16, dt_rank <= 128): no
  // Delta buffer and one launch less, but the folded scan measured 7.13 ms
  // against 6.31 ms for projection + scan at L = 131072 (its stages carry
  // dt_low, which halves their depth), so it is opt-in (SAMBA_SCAN_FOLD_DT=1).
  a.dt_low = xdbl;
  a.ld_dtl = P.xdw;
  a.R = R;
  a.W_dt = w->W_dt;
  a.dtype = dt;
  const char* fold_env = getenv("SAMBA_SCAN_FOLD_DT");
  const bool fold = fold_env && fold_env[0] == '1' && scan_dt_fold_supported(a);
  if (!fold) {
    a.dt_low = nullptr;
    a.W_dt = nullptr;
    GemmArgs g = gemm1(xdbl, P.xdw, w->W_dt, T, Di, R, buf(P.dlt), Di, dt);  // Delta = softplus(.. + b)
    g.epi = kEpiSoftplus;
    g.bias = w->dt_bias;
    TRY(launch_gemm(g, st));
  }
  {
    a.u = buf(P.u);
    a.dt = fold ? nullptr : buf(P.dlt);
    a.dt_bias = fold ? w->dt_bias : nullptr;
    a.z = hz + (size_t)Di * es;
    a.Bm = xdbl + (size_t)R * es;
    a.Cm = xdbl + (size_t)(R + N) * es;
    a.y = buf(P.y);
    a.ld_u = a.ld_dt = a.ld_y = Di;
    a.ld_z = 2 * Di;
    a.ld_bc = P.xdw;
    a.A_log = w->A_log;
    a.Dskip = w->Dskip;
    a.h0 = resume ? stt->ssm : nullptr;  // each thread reads its h0 entries before writing hT
    a.hT = stt ? stt->ssm : nullptr;
    a.B = B;
    a.L = L;
    a.D = Di;
    a.N = N;
    a.softplus = fold;
    a.dtype = dt;
    TRY(launch_selective_scan(a, st));
  }
  {
    GemmArgs g = gemm1(buf(P.y), Di, w->W_out, T, Dm, Di, x_out, Dm, dt);
    g.epi = kEpiResid;
    g.resid = x_in;
    g.ldr = Dm;
    g.tap = tap;
    g.ldt = Dm;
    TRY(launch_gemm(g, st));
  }
  return SAMBA_OK;
}

// SWA sub-layer over B x L tokens: x_out = x_in + SWA(RMSNorm(x_in))
// [Samba 3.4 "The Sliding Window Attention (SWA) Layer"]; RoPE positions start
// at pos0.  stt: NULL, or the decode state whose ring receives the last
// min(L, window) keys/values (resume: the ring also supplies the keys of the
// min(pos0, window-1) tokens before this chunk).
static samba_status swa_sublayer(const LayerCtx& X, const samba_block_weights* w, const void* x_in, void* x_out,
                                 samba_decode_state* stt, int64_t pos0, bool resume, void* tap) {
  NvtxRange nvtx_("samba.swa");
  const samba_block_config& c = X.c;
  const BlockPlan& P = X.P;
  const int B = X.B, L = X.L;
  const int64_t T = X.T;
  cudaStream_t st = X.st;
  const samba_dtype dt = c.dtype;
  auto buf = [&](size_t off) -> void* { return X.base + off; };
  const int Dm = c.d_model;
  const size_t es = dtype_size(dt);
  void* xn = buf(P.xn);
  char* qkv = (char*)buf(P.qkv);
  float2* tab = (float2*)buf(P.tab);
  TRY(launch_rmsnorm(x_in, Dm, w->norm_g[2], xn, Dm, T, Dm, c.norm_eps, dt, st));
  const int hd = c.head_dim;
  const int qw = c.n_q * hd, kvw = c.n_kv * hd;
  {
    GemmArgs g = gemm1(xn, Dm, w->Wq, T, P.qkvw, Dm, qkv, P.qkvw, dt);
    g.nseg = 3;
    g.seg[0].W = w->Wq;
    g.seg[0].n = qw;
    g.seg[1].W = w->Wk;
    g.seg[1].n = kvw;
    g.seg[2].W = w->Wv;
    g.seg[2].n = kvw;
    if (c.rope_base != 0.f) {
      TRY(launch_build_rope_table(tab, hd, c.rope_base, st));
      g.epi = kEpiRope;
      g.rope_cols = qw + kvw;
      g.head_dim = hd;
      g.seq_len = L;
      g.pos0 = pos0;
      g.rope_tab = tab;
    }
    TRY(launch_gemm(g, st));
  }
  {
    SwaArgs a;
    a.q = qkv;
    a.k = qkv + (size_t)qw * es;
    a.v = qkv + (size_t)(qw + kvw) * es;
    a.o = buf(P.o);
    a.ld_q = a.ld_k = a.ld_v = P.qkvw;
    a.ld_o = qw;
    a.B = B;
    a.L = L;
    a.Hq = c.n_q;
    a.Hkv = c.n_kv;
    a.d = hd;
    a.window = c.window;
    a.scale = 1.0f / sqrtf((float)hd);
    a.dtype = dt;
    if (resume) {  // keys of the h tokens before the chunk lead the chunk's own K/V rows
      const int h = (int)std::min<int64_t>(pos0, c.window - 1);
      TRY(launch_kv_window_gather(qkv, P.qkvw, qw, qw + kvw, stt->k_ring, stt->v_ring, buf(P.kx), buf(P.vx), B, L,
                                  pos0, h, c.window, kvw, dt, st));
      a.k = buf(P.kx);
      a.v = buf(P.vx);
      a.ld_k = a.ld_v = kvw;
      a.qoff = h;
    }
    TRY(launch_swa(a, st));
  }
  if (stt)
    TRY(launch_ring_fill(qkv, P.qkvw, qw, qw + kvw, stt->k_ring, stt->v_ring, B, L, pos0, c.window, kvw, dt, st));
  {
    GemmArgs g = gemm1(buf(P.o), qw, w->Wo, T, Dm, qw, x_out, Dm, dt);
    g.epi = kEpiResid;
    g.resid = x_in;
    g.ldr = Dm;
    g.tap = tap;
    g.ldt = Dm;
    TRY(launch_gemm(g, st));
  }
  return SAMBA_OK;
}

// Decode step of a Mamba sub-layer for one token per sequence (X.T = B rows):
// conv-state shift, one recurrence step of the fp32 SSM state, gate, residual
// [Samba 3.4 "The Mamba Layer" at a single t].  Every launch of a decode step is
// a programmatic dependent of the one before it: a kernel sets up (and the
// projections fetch their first weight tiles) while its predecessor finishes.
// ss_in / ss_out / g_next: the norm fold (the layer's RMSNorm completed by its
// input projection from the previous producer's sums of squares; its output
// projection writes the next norm's input and sums of squares).
static samba_status mamba_step_layer(const LayerCtx& X, const samba_block_weights* w, const void* x_in, void* x_out,
                                     float* ssm, void* conv, const float* ss_in = nullptr, float* ss_out = nullptr,
                                     const float* g_next = nullptr) {
  NvtxRange nvtx_("samba.mamba_step");
  const samba_block_config& c = X.c;
  const BlockPlan& P = X.P;
  const int B = X.B;
  cudaStream_t st = X.st;
  const samba_dtype dt = c.dtype;
  auto buf = [&](size_t off) -> void* { return X.base + off; };
  const int Di = c.d_inner, Dm = c.d_model, R = c.dt_rank;
  const size_t es = dtype_size(dt);
  void* xn = buf(P.xn);
  char* hz = (char*)buf(P.hz);
  char* xdbl = (char*)buf(P.xdbl);
  auto gemm_pdl = [&](GemmArgs g) {
    g.pdl = true;
    return launch_gemm(g, st);
  };
  if (!ss_in) TRY(launch_rmsnorm(x_in, Dm, w->norm_g[0], xn, Dm, B, Dm, c.norm_eps, dt, st, true));
  {
    GemmArgs g = gemm1(xn, Dm, w->W_in, B, 2 * Di, Dm, hz, 2 * Di, dt);
    g.ss_in = ss_in;
    g.norm_dim = Dm;
    g.norm_eps = c.norm_eps;
    // the skinny projection runs the short convolution step on its x columns itself
    GemmArgs gc = g;
    gc.conv_w = w->conv_w;
    gc.conv_b = w->conv_b;
    gc.conv_state = conv;
    gc.conv_u = buf(P.u);
    gc.conv_cols = Di;
    gc.conv_k = c.d_conv;
    if (gemm_takes_skinny(gc)) {
      TRY(gemm_pdl(gc));
    } else {
      TRY(gemm_pdl(g));
      TRY(launch_conv_step(hz, 2 * Di, w->conv_w, w->conv_b, conv, buf(P.u), B, Di, c.d_conv, dt, st));
    }
  }
  TRY(gemm_pdl(gemm1(buf(P.u), Di, w->W_x, B, P.xdw, Di, xdbl, P.xdw, dt)));
  if (scan_step_dt_supported(R, Di, P.xdw, dt) && aligned16(w->W_dt) && aligned16(w->A_log)) {
    // the dt projection inside the recurrence step
    TRY(launch_scan_step_dt(buf(P.u), hz + (size_t)Di * es, 2 * Di, xdbl, P.xdw, R, w->W_dt, w->dt_bias, w->A_log,
                            w->Dskip, ssm, buf(P.y), B, Di, dt, st));
  } else {
    GemmArgs g = gemm1(xdbl, P.xdw, w->W_dt, B, Di, R, buf(P.dlt), Di, dt);
    g.epi = kEpiSoftplus;
    g.bias = w->dt_bias;
    TRY(gemm_pdl(g));
    TRY(launch_scan_step(buf(P.u), buf(P.dlt), hz + (size_t)Di * es, 2 * Di, xdbl, P.xdw, R, w->A_log, w->Dskip,
                         ssm, buf(P.y), B, Di, dt, st));
  }
  GemmArgs g = gemm1(buf(P.y), Di, w->W_out, B, Dm, Di, x_out, Dm, dt);
  g.epi = kEpiResid;
  g.resid = x_in;
  g.ldr = Dm;
  if (ss_out) {  // the next norm's input and sums of squares
    g.ss_out = ss_out;
    g.g_next = g_next;
    g.xg_out = xn;
  }
  return gemm_pdl(g);
}

// Decode step of an SWA sub-layer: q, k, v of the new token rotated at
// position pos[b], k/v written to ring slot pos[b] mod window, attention over
// the min(pos[b] + 1, window) valid slots, output projection, residual.
// attn_ws: partials of the split attention for rings above 2048 slots.
// ss_in / ss_out / g_next: the norm fold, as for the Mamba step layer.
static samba_status swa_step_layer(const LayerCtx& X, const samba_block_weights* w, const void* x_in, void* x_out,
                                   void* k_ring, void* v_ring, const int64_t* pos, void* attn_ws,
                                   size_t attn_ws_bytes, const float* ss_in = nullptr, float* ss_out = nullptr,
                                   const float* g_next = nullptr) {
  NvtxRange nvtx_("samba.swa_step");
  const samba_block_config& c = X.c;
  const BlockPlan& P = X.P;
  const int B = X.B;
  cudaStream_t st = X.st;
  const samba_dtype dt = c.dtype;
  auto buf = [&](size_t off) -> void* { return X.base + off; };
  const int Dm = c.d_model;
  void* xn = buf(P.xn);
  char* qkv = (char*)buf(P.qkv);
  float2* tab = (float2*)buf(P.tab);
  if (!ss_in) TRY(launch_rmsnorm(x_in, Dm, w->norm_g[2], xn, Dm, B, Dm, c.norm_eps, dt, st, true));
  const int hd = c.head_dim;
  const int qw = c.n_q * hd, kvw = c.n_kv * hd;
  {
    GemmArgs g = gemm1(xn, Dm, w->Wq, B, P.qkvw, Dm, qkv, P.qkvw, dt);
    g.nseg = 3;
    g.seg[0].W = w->Wq;
    g.seg[0].n = qw;
    g.seg[1].W = w->Wk;
    g.seg[1].n = kvw;
    g.seg[2].W = w->Wv;
    g.seg[2].n = kvw;
    g.pdl = true;
    g.ss_in = ss_in;
    g.norm_dim = Dm;
    g.norm_eps = c.norm_eps;
    bool ring_done = false;
    if (c.rope_base != 0.f) {
      g.epi = kEpiRope;
      g.rope_cols = qw + kvw;
      g.head_dim = hd;
      g.pos_dev = pos;
      g.rope_base = c.rope_base;  // the skinny projection evaluates the rotation from the position
      if (!gemm_takes_skinny(g)) {
        TRY(launch_build_rope_table(tab, hd, c.rope_base, st, true));
        g.rope_tab = tab;
      }
      // the skinny projection writes the new token's k, v into the ring itself
      GemmArgs gr = g;
      gr.k_ring = k_ring;
      gr.v_ring = v_ring;
      gr.ring_window = c.window;
      gr.ring_k_col = qw;
      gr.ring_v_col = qw + kvw;
      gr.ring_kvw = kvw;
      if (gemm_takes_skinny(gr)) {
        g = gr;
        ring_done = true;
      }
    }
    TRY(launch_gemm(g, st));
    if (!ring_done)
      TRY(launch_ring_write(qkv, P.qkvw, qw, qw + kvw, pos, k_ring, v_ring, B, c.window, kvw, dt, st));
  }
  TRY(launch_attn_decode(qkv, P.qkvw, pos, k_ring, v_ring, buf(P.o), B, c.n_q, c.n_kv, hd, c.window,
                         1.0f / sqrtf((float)hd), dt, st, attn_ws, attn_ws_bytes));
  GemmArgs g = gemm1(buf(P.o), qw, w->Wo, B, Dm, qw, x_out, Dm, dt);
  g.epi = kEpiResid;
  g.resid = x_in;
  g.ldr = Dm;
  g.pdl = true;
  if (ss_out) {  // the MLP norm's input and sums of squares
    g.ss_out = ss_out;
    g.g_next = g_next;
    g.xg_out = xn;
  }
  return launch_gemm(g, st);
}

// One block over B x L tokens.  pos0 > 0 continues a prefill from the decode
// state `stt` holds after pos0 tokens (chunked prefill): the conv history, the
// SSM state and the ring's last window of K/V are the inputs before token 0,
// RoPE positions start at pos0, and the state is advanced to pos0 + L.
static samba_status block_forward(const samba_block_config* cfg, const samba_block_weights* w, const void* x_in,
                                  void* x_out, samba_decode_state* stt, int64_t pos0, const samba_block_taps* taps,
                                  int B, int L, void* workspace, size_t workspace_bytes, samba_stream stream) {
  NvtxRange nvtx_("samba_block_fwd");
  TRY(validate_cfg(cfg));
  TRY(validate_weights(w));
  if (B < 1 || L < 0 || pos0 < 0) return SAMBA_ERR_INVALID_ARG;
  if (L > 0 && (!x_in || !x_out || x_in == x_out)) return SAMBA_ERR_INVALID_ARG;
  if (stt && (!stt->ssm || !stt->conv || !stt->k_ring || !stt->v_ring || !stt->pos)) return SAMBA_ERR_INVALID_ARG;
  const bool resume = pos0 > 0;
  if (resume && !stt) return SAMBA_ERR_INVALID_ARG;
  if (pos0 + (int64_t)L > (int64_t(1) << 30)) return SAMBA_ERR_UNSUPPORTED;
  if (B > kMaxGridYZ || L > kMaxConvTokens) return SAMBA_ERR_UNSUPPORTED;
  const samba_block_config& c = *cfg;
  const int64_t T = (int64_t)B * L;
  const BlockPlan P = plan_block(c, T, resume ? B : 0);
  if (!workspace || workspace_bytes < P.total) return SAMBA_ERR_INVALID_ARG;
  if (!aligned16(x_in) || !aligned16(x_out)) return SAMBA_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  const samba_dtype dt = c.dtype;
  char* base = (char*)(((uintptr_t)workspace + 255) & ~uintptr_t(255));
  auto buf = [&](size_t off) -> void* { return base + off; };
  const int Di = c.d_inner, N = c.d_state;
  const size_t es = dtype_size(dt);
  void* x1 = (taps && taps->resid[0]) ? taps->resid[0] : buf(P.x1);
  void* x2 = (taps && taps->resid[1]) ? taps->resid[1] : buf(P.x2);
  void* x3 = (taps && taps->resid[2]) ? taps->resid[2] : buf(P.x3);
  void* xn = buf(P.xn);

  if (T == 0 && resume) return launch_pos_check_set(stt->pos, B, pos0, pos0, st);
  if (T == 0) {
    if (stt) {
      TRY(launch_pos_update(stt->pos, B, 0, true, st));
      if (cudaMemsetAsync(stt->ssm, 0, (size_t)B * Di * N * sizeof(float), st) != cudaSuccess ||
          cudaMemsetAsync(stt->conv, 0, (size_t)B * Di * (c.d_conv - 1) * es, st) != cudaSuccess)
        return SAMBA_ERR_CUDA;
    }
    return SAMBA_OK;
  }

  const LayerCtx X{c, P, base, B, L, T, st};
  TRY(guards_arm(base, P.cv, st));
  TRY(mamba_sublayer(X, w, x_in, x1, stt, resume, taps ? taps->branch[0] : nullptr));
  // ---- MLP 1
  TRY(mlp_sublayer(c, w->norm_g[1], w->mlp1_W1, w->mlp1_W2, w->mlp1_W3, x1, x2, xn, buf(P.hmlp),
                   taps ? taps->branch[1] : nullptr, T, st));
  TRY(swa_sublayer(X, w, x2, x3, stt, pos0, resume, taps ? taps->branch[2] : nullptr));
  // ---- MLP 2
  TRY(mlp_sublayer(c, w->norm_g[3], w->mlp2_W1, w->mlp2_W2, w->mlp2_W3, x3, x_out, xn, buf(P.hmlp),
                   taps ? taps->branch[3] : nullptr, T, st));
  TRY(guards_check(base, P.cv, st));
  if (resume) return launch_pos_check_set(stt->pos, B, pos0, pos0 + L, st);
  if (stt) TRY(launch_pos_update(stt->pos, B, L, true, st));
  return SAMBA_OK;
}

}  // namespace samba

extern "C" {

samba_status samba_block_fwd(const samba_block_config* cfg, const samba_block_weights* w, const void* x_in,
                             void* x_out, samba_decode_state* stt, const samba_block_taps* taps, int B, int L,
                             void* workspace, size_t workspace_bytes, samba_stream stream) {
  return block_forward(cfg, w, x_in, x_out, stt, 0, taps, B, L, workspace, workspace_bytes, stream);
}

// ------------------------------------------------------------------ chunked prefill
size_t samba_block_chunk_workspace_size(const samba_block_config* cfg, int B, int L) {
  if (validate_cfg(cfg) != SAMBA_OK || B < 1 || L < 0) return 0;
  return plan_block(*cfg, (int64_t)B * L, B).total;
}

samba_status samba_block_fwd_chunk(const samba_block_config* cfg, const samba_block_weights* w, const void* x_in,
                                   void* x_out, samba_decode_state* stt, int64_t pos0, const samba_block_taps* taps,
                                   int B, int L, void* workspace, size_t workspace_bytes, samba_stream stream) {
  if (!stt) return SAMBA_ERR_INVALID_ARG;
  return block_forward(cfg, w, x_in, x_out, stt, pos0, taps, B, L, workspace, workspace_bytes, stream);
}


// ------------------------------------------------------------------ language-model stack
}  // extern "C"

namespace samba {

struct ModelPlan {
  BlockPlan P;                 // one sub-layer's activations over all B*L tokens
  size_t xa, xb, xl, total;    // two residual streams, the normed last rows
  Carve cv;
};

static ModelPlan plan_model(const samba_block_config& c, int B, int L) {
  ModelPlan m;
  const int64_t T = (int64_t)B * L;
  const size_t es = dtype_size(c.dtype);
  m.P = plan_block(c, T);
  Carve cv = m.P.cv;  // keeps the block's guard bands
  cv.off = m.P.total;
  m.xa = cv.take(T * c.d_model * es);
  m.xb = cv.take(T * c.d_model * es);
  m.xl = cv.take((size_t)B * c.d_model * es);
  m.total = cv.off + 256;
  m.cv = cv;
  return m;
}

static samba_status validate_layer(int kind, const samba_block_weights& w) {
  std::initializer_list<const void*> mamba = {w.norm_g[0], w.W_in, w.conv_w, w.W_x, w.W_dt,
                                              w.dt_bias,   w.A_log, w.Dskip, w.W_out};
  std::initializer_list<const void*> mlp = {w.norm_g[1], w.mlp1_W1, w.mlp1_W2, w.mlp1_W3};
  std::initializer_list<const void*> swa = {w.norm_g[2], w.Wq, w.Wk, w.Wv, w.Wo};
  const std::initializer_list<const void*>* req =
      kind == SAMBA_LAYER_MAMBA ? &mamba : kind == SAMBA_LAYER_MLP ? &mlp : kind == SAMBA_LAYER_SWA ? &swa : nullptr;
  if (!req) return SAMBA_ERR_INVALID_ARG;
  for (const void* p : *req)
    if (!p) return SAMBA_ERR_INVALID_ARG;
  for (const void* p : *req)
    if (!aligned16(p)) return SAMBA_ERR_UNSUPPORTED;
  return SAMBA_OK;
}

}  // namespace samba

extern "C" {

size_t samba_model_workspace_size(const samba_model* m, int B, int L) {
  if (!m || validate_cfg(&m->cfg) != SAMBA_OK || B < 1 || L < 1) return 0;
  return plan_model(m->cfg, B, L).total;
}

samba_status samba_model_prefill(const samba_model* m, const int32_t* ids, void* logits, int B, int L,
                                 void* workspace, size_t workspace_bytes, samba_stream stream) {
  NvtxRange nvtx_("samba_model_prefill");
  if (!m) return SAMBA_ERR_INVALID_ARG;
  TRY(validate_cfg(&m->cfg));
  if (!ids || !logits || B < 1 || L < 1 || m->n_layers < 0 || m->vocab < 1) return SAMBA_ERR_INVALID_ARG;
  if (B > kMaxGridYZ || L > kMaxConvTokens) return SAMBA_ERR_UNSUPPORTED;
  if (m->n_layers > 0 && (!m->kinds || !m->layers)) return SAMBA_ERR_INVALID_ARG;
  if (!m->embedding || !m->final_norm || !m->lm_head) return SAMBA_ERR_INVALID_ARG;
  for (int i = 0; i < m->n_layers; ++i) TRY(validate_layer(m->kinds[i], m->layers[i]));
  if ((int64_t)L > (int64_t(1) << 30)) return SAMBA_ERR_UNSUPPORTED;
  const samba_block_config& c = m->cfg;
  const ModelPlan MP = plan_model(c, B, L);
  if (!workspace || workspace_bytes < MP.total) return SAMBA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const samba_dtype dt = c.dtype;
  const size_t es = dtype_size(dt);
  char* base = (char*)(((uintptr_t)workspace + 255) & ~uintptr_t(255));
  const int64_t T = (int64_t)B * L;
  const int Dm = c.d_model;
  char* cur = base + MP.xa;
  char* nxt = base + MP.xb;
  TRY(guards_arm(base, MP.cv, st));
  TRY(launch_embedding(ids, m->embedding, cur, T, Dm, m->vocab, dt, st));
  const LayerCtx X{c, MP.P, base, B, L, T, st};
  for (int i = 0; i < m->n_layers; ++i) {
    const samba_block_weights& w = m->layers[i];
    switch (m->kinds[i]) {
      case SAMBA_LAYER_MAMBA: TRY(mamba_sublayer(X, &w, cur, nxt, nullptr, false, nullptr)); break;
      case SAMBA_LAYER_SWA: TRY(swa_sublayer(X, &w, cur, nxt, nullptr, 0, false, nullptr)); break;
      default:
        TRY(mlp_sublayer(c, w.norm_g[1], w.mlp1_W1, w.mlp1_W2, w.mlp1_W3, cur, nxt, base + MP.P.xn,
                         base + MP.P.hmlp, nullptr, T, st));
        break;
    }
    std::swap(cur, nxt);
  }
  // final RMSNorm of each sequence's last position, then the vocabulary projection
  TRY(launch_rmsnorm(cur + (size_t)(L - 1) * Dm * es, (int64_t)L * Dm, m->final_norm, base + MP.xl, Dm, B, Dm,
                     c.norm_eps, dt, st));
  TRY(launch_gemm(gemm1(base + MP.xl, Dm, m->lm_head, B, m->vocab, Dm, logits, m->vocab, dt), st));
  return guards_check(base, MP.cv, st);
}

}  // extern "C"

namespace samba {

struct ModelStepPlan {
  BlockPlan P;
  size_t xa, xb, xl, attn, attn_bytes, total;
  Carve cv;
};

static ModelStepPlan plan_model_step(const samba_block_config& c, int B) {
  ModelStepPlan m;
  const size_t es = dtype_size(c.dtype);
  m.P = plan_block(c, B);
  Carve cv = m.P.cv;
  cv.off = m.P.total;
  m.xa = cv.take((size_t)B * c.d_model * es);
  m.xb = cv.take((size_t)B * c.d_model * es);
  m.xl = cv.take((size_t)B * c.d_model * es);
  m.attn_bytes = attn_decode_workspace_bytes(B, c.n_kv, c.window);
  m.attn = cv.take(m.attn_bytes);
  m.total = cv.off + 256;
  m.cv = cv;
  return m;
}

// The decode norm fold: a layer's RMSNorm is completed by its input
// projection(s), which scale their output rows by the RMS from per-8-feature
// sums of squares, and the residual projection before it writes the norm's
// input (the stream row times the norm's gain) and those sums.  Every
// projection involved must run on the skinny kernel: bf16, batch <= 64, K
// multiples of 64, QKV segments on 128-row tile boundaries with RoPE heads of
// at most 128, 16-byte aligned weights and gains.  SAMBA_NORM_FOLD=0 turns it
// off.
static bool fold_dims_ok(const samba_block_config& c, int B) {
  const char* e = getenv("SAMBA_NORM_FOLD");
  if (e && e[0] == '0') return false;
  const char* gk = getenv("SAMBA_GEMM_KERNEL");
  if (gk && gk[0] == 's') return false;
  if (c.dtype != SAMBA_BF16 || B > 64) return false;
  const int hd = c.head_dim, qw = c.n_q * hd, kvw = c.n_kv * hd;
  if (c.d_model % 64 || c.d_inner % 64 || c.d_ff % 64 || qw % 64) return false;
  if (qw % 128 || (qw + kvw) % 128) return false;  // tiles never straddle the Q | K | V segments
  if (c.rope_base != 0.f && (hd < 16 || 128 % hd != 0 || hd / 2 > 64)) return false;
  return true;
}

static bool all_aligned16(std::initializer_list<const void*> ptrs) {
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return false;
  return true;
}

// The weights and input gain of one sub-layer kind the fold touches.
static bool fold_layer_ok(int k, const samba_block_weights& w) {
  switch (k) {
    case SAMBA_LAYER_MAMBA: return all_aligned16({w.W_in, w.W_out, w.norm_g[0]});
    case SAMBA_LAYER_SWA: return all_aligned16({w.Wq, w.Wk, w.Wv, w.Wo, w.norm_g[2]});
    default: return all_aligned16({w.mlp1_W1, w.mlp1_W2, w.mlp1_W3, w.norm_g[1]});
  }
}

// The gain of a sub-layer's input norm.
static const float* layer_input_gain(int k, const samba_block_weights& w) {
  return k == SAMBA_LAYER_MAMBA ? w.norm_g[0] : k == SAMBA_LAYER_SWA ? w.norm_g[2] : w.norm_g[1];
}

// samba_step: norms 1..3 (out_proj and both MLP down projections produce,
// both MLP up projections and the QKV projection consume).
static bool step_norm_fold_ok(const samba_block_config& c, const samba_block_weights* w, int B) {
  return fold_dims_ok(c, B) && all_aligned16({w->W_out, w->mlp1_W1, w->mlp1_W2, w->mlp1_W3, w->mlp2_W1, w->mlp2_W2,
                                              w->mlp2_W3, w->Wq, w->Wk, w->Wv, w->Wo, w->norm_g[1], w->norm_g[2],
                                              w->norm_g[3]});
}

// samba_model_step: every norm after the first sub-layer's, the final norm
// included (the LM head consumes it).
static bool model_norm_fold_ok(const samba_model* m, int B, const void* logits) {
  if (m->n_layers < 1 || !fold_dims_ok(m->cfg, B)) return false;
  if (m->vocab % 8 || !all_aligned16({m->lm_head, m->final_norm, logits})) return false;
  for (int i = 0; i < m->n_layers; ++i)
    if (!fold_layer_ok(m->kinds[i], m->layers[i])) return false;
  return true;
}

}  // namespace samba

extern "C" {

size_t samba_model_step_workspace_size(const samba_model* m, int B) {
  if (!m || validate_cfg(&m->cfg) != SAMBA_OK || B < 1) return 0;
  return plan_model_step(m->cfg, B).total;
}

samba_status samba_model_step(const samba_model* m, const int32_t* ids_t, void* logits, samba_layer_state* states,
                              int64_t* pos, int B, void* workspace, size_t workspace_bytes, samba_stream stream) {
  NvtxRange nvtx_("samba_model_step");
  if (!m) return SAMBA_ERR_INVALID_ARG;
  TRY(validate_cfg(&m->cfg));
  if (!ids_t || !logits || !pos || B < 1 || m->n_layers < 0 || m->vocab < 1) return SAMBA_ERR_INVALID_ARG;
  if (B > kMaxGridYZ) return SAMBA_ERR_UNSUPPORTED;
  if (m->n_layers > 0 && (!m->kinds || !m->layers || !states)) return SAMBA_ERR_INVALID_ARG;
  if (!m->embedding || !m->final_norm || !m->lm_head) return SAMBA_ERR_INVALID_ARG;
  for (int i = 0; i < m->n_layers; ++i) {
    TRY(validate_layer(m->kinds[i], m->layers[i]));
    const samba_layer_state& sl = states[i];
    if (m->kinds[i] == SAMBA_LAYER_MAMBA && (!sl.ssm || !sl.conv)) return SAMBA_ERR_INVALID_ARG;
    if (m->kinds[i] == SAMBA_LAYER_MAMBA && !aligned16(sl.ssm)) return SAMBA_ERR_UNSUPPORTED;
    if (m->kinds[i] == SAMBA_LAYER_SWA && (!sl.k_ring || !sl.v_ring)) return SAMBA_ERR_INVALID_ARG;
  }
  const samba_block_config& c = m->cfg;
  const ModelStepPlan MP = plan_model_step(c, B);
  if (!workspace || workspace_bytes < MP.total) return SAMBA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const samba_dtype dt = c.dtype;
  char* base = (char*)(((uintptr_t)workspace + 255) & ~uintptr_t(255));
  const int Dm = c.d_model;
  char* cur = base + MP.xa;
  char* nxt = base + MP.xb;
  TRY(guards_arm(base, MP.cv, st));
  TRY(launch_embedding(ids_t, m->embedding, cur, B, Dm, m->vocab, dt, st));
  const LayerCtx X{c, MP.P, base, B, 1, (int64_t)B, st};
  // norm fold: every norm after the first sub-layer's rides on the projections
  // around it, through two alternating areas of B x d_model/8 partial sums of
  // squares (ss_in: the previous producer's, ss_out: this layer's)
  const bool fold = model_norm_fold_ok(m, B, logits);
  float* ss_in = nullptr;
  float* ss_out = fold ? (float*)(base + MP.P.ss) : nullptr;
  float* ss_spare = fold ? ss_out + (int64_t)B * (Dm / 8) : nullptr;
  for (int i = 0; i < m->n_layers; ++i) {
    const samba_block_weights& w = m->layers[i];
    const samba_layer_state& sl = states[i];
    const float* g_next = !fold ? nullptr
                          : i + 1 < m->n_layers ? layer_input_gain(m->kinds[i + 1], m->layers[i + 1])
                                                : m->final_norm;
    switch (m->kinds[i]) {
      case SAMBA_LAYER_MAMBA: TRY(mamba_step_layer(X, &w, cur, nxt, sl.ssm, sl.conv, ss_in, ss_out, g_next)); break;
      case SAMBA_LAYER_SWA:
        TRY(swa_step_layer(X, &w, cur, nxt, sl.k_ring, sl.v_ring, pos, base + MP.attn, MP.attn_bytes, ss_in, ss_out,
                           g_next));
        break;
      default:
        TRY(mlp_sublayer(c, w.norm_g[1], w.mlp1_W1, w.mlp1_W2, w.mlp1_W3, cur, nxt, base + MP.P.xn,
                         base + MP.P.hmlp, nullptr, B, st, true, nullptr, nullptr, ss_in, ss_out, g_next));
        break;
    }
    std::swap(cur, nxt);
    if (fold) {
      ss_in = ss_out;
      std::swap(ss_out, ss_spare);
    }
  }
  // the LM head: RMSNorm(x) from the last producer's x (.) g and sums (fold), else a norm launch
  if (!fold) TRY(launch_rmsnorm(cur, Dm, m->final_norm, base + MP.xl, Dm, B, Dm, c.norm_eps, dt, st, true));
  GemmArgs g = gemm1(base + (fold ? MP.P.xn : MP.xl), Dm, m->lm_head, B, m->vocab, Dm, logits, m->vocab, dt);
  g.pdl = true;
  g.ss_in = ss_in;
  g.norm_dim = Dm;
  g.norm_eps = c.norm_eps;
  TRY(launch_gemm(g, st));
  TRY(guards_check(base, MP.cv, st));
  return launch_pos_update(pos, B, 1, false, st, true);
}

// ------------------------------------------------------------------ decode step

// The step's workspace: one block's activations for B tokens, then (rings
// above 2048 slots) the split decode attention's partials.
static size_t step_attn_offset(const samba_block_config& c, int B) {
  return plan_block(c, B).cv.off;  // 256-byte aligned end of the block's carve
}

size_t samba_step_workspace_size(const samba_block_config* cfg, int B) {
  if (validate_cfg(cfg) != SAMBA_OK || B < 1) return 0;
  // + 256: slack for aligning the caller's base pointer
  return step_attn_offset(*cfg, B) + attn_decode_workspace_bytes(B, cfg->n_kv, cfg->window) + 256;
}

samba_status samba_step(const samba_block_config* cfg, const samba_block_weights* w, const void* x_t, void* y_t,
                        samba_decode_state* stt, int B, void* workspace, size_t workspace_bytes,
                        samba_stream stream) {
  NvtxRange nvtx_("samba_step");
  TRY(validate_cfg(cfg));
  TRY(validate_weights(w));
  if (!x_t || !y_t || !stt || B < 1 || x_t == y_t) return SAMBA_ERR_INVALID_ARG;
  if (B > kMaxGridYZ) return SAMBA_ERR_UNSUPPORTED;
  if (!stt->ssm || !stt->conv || !stt->k_ring || !stt->v_ring || !stt->pos) return SAMBA_ERR_INVALID_ARG;
  if (!aligned16(stt->ssm)) return SAMBA_ERR_UNSUPPORTED;  // the state is moved in 16-byte pieces
  const samba_block_config& c = *cfg;
  const BlockPlan P = plan_block(c, B);
  if (!workspace || workspace_bytes < samba_step_workspace_size(cfg, B)) return SAMBA_ERR_INVALID_ARG;
  if (!aligned16(x_t) || !aligned16(y_t)) return SAMBA_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  char* base = (char*)(((uintptr_t)workspace + 255) & ~uintptr_t(255));
  const LayerCtx X{c, P, base, B, 1, (int64_t)B, st};
  void *x1 = base + P.x1, *x2 = base + P.x2, *x3 = base + P.x3;
  TRY(guards_arm(base, P.cv, st));
  // norm fold: norms 1..3 are completed by the projections around them, through
  // three areas of B x d_model/8 partial sums of squares
  float* ssf = step_norm_fold_ok(c, w, B) ? (float*)(base + P.ss) : nullptr;
  const int64_t nss = (int64_t)B * (c.d_model / 8);
  TRY(mamba_step_layer(X, w, x_t, x1, stt->ssm, stt->conv, nullptr, ssf, w->norm_g[1]));
  TRY(mlp_sublayer(c, w->norm_g[1], w->mlp1_W1, w->mlp1_W2, w->mlp1_W3, x1, x2, base + P.xn, base + P.hmlp, nullptr,
                   B, st, true, nullptr, nullptr, ssf, ssf ? ssf + nss : nullptr, w->norm_g[2]));
  const size_t attn_bytes = attn_decode_workspace_bytes(B, c.n_kv, c.window);
  TRY(swa_step_layer(X, w, x2, x3, stt->k_ring, stt->v_ring, stt->pos,
                     attn_bytes ? base + step_attn_offset(c, B) : nullptr, attn_bytes, ssf ? ssf + nss : nullptr,
                     ssf ? ssf + 2 * nss : nullptr, w->norm_g[3]));
  bool pos_done = false;
  TRY(mlp_sublayer(c, w->norm_g[3], w->mlp2_W1, w->mlp2_W2, w->mlp2_W3, x3, y_t, base + P.xn, base + P.hmlp, nullptr,
                   B, st, true, stt->pos, &pos_done, ssf ? ssf + 2 * nss : nullptr));
  TRY(guards_check(base, P.cv, st));
  return pos_done ? SAMBA_OK : launch_pos_update(stt->pos, B, 1, false, st, true);
}

}  // extern "C"
