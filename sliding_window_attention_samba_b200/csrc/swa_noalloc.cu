// samba_swa_fwd_noalloc: the sliding-window attention entry point for callers
// that cannot allocate device memory.
//
// Who needs it: code that cannot call cudaMalloc -- e.g. a plugin loaded into a
// host application that owns all device memory and gives the plugin no
// allocator, so the plugin has no way to obtain a scratch buffer.
// samba_swa_fwd needs caller-provided scratch when RoPE is on (the fp64-built
// rotation table and the rotated copies of q and k); this variant keeps that
// scratch in a fixed array compiled into the library instead.
//
// Properties:
//   * The scratch is a file-scope static __device__ array of kNoallocScratchBytes
//     (16 MiB).  Every GPU that loads the library holds it until the process exits.
//   * Host code never passes the array's name to a kernel (on the host it is only
//     a stand-in symbol); the device address is looked up with
//     cudaGetSymbolAddress, with that device current, on the first call made on
//     that device (and again if the device's context was replaced, e.g. by
//     cudaDeviceReset).  Make that first call before any stream capture.
//   * Calls reject sizes whose scratch would not fit (SAMBA_ERR_UNSUPPORTED) and
//     never call cudaMalloc/cudaFree or any allocating routine.
//   * All calls share the one array and it keeps the last call's contents; the
//     table and the rotated copies are fully rewritten by each call, so nothing
//     needs clearing.  Calls that overlap on the GPU (different streams, or
//     different host threads on the same device) race on the array.
#include <mutex>

#define SAMBA_TU_ID 8  // site id of this file in debug-check reports
#include "common.cuh"
#include "kernels.h"

namespace samba {

namespace {

constexpr size_t kNoallocScratchBytes = size_t(16) << 20;  // 16 MiB

static __device__ __align__(256) unsigned char g_swa_noalloc_scratch[kNoallocScratchBytes];

// Device address of the scratch array on the current device (set-up on first
// use, and again whenever the device's context changed, e.g. after
// cudaDeviceReset: the array lives in the context that loaded the module).
unsigned char* noalloc_scratch_ptr() {
  static unsigned char* ptr[64] = {nullptr};
  static uintptr_t ctx[64] = {0};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  const uintptr_t c = current_context_id();
  std::lock_guard<std::mutex> lk(mu);
  if (!ptr[dev] || ctx[dev] != c) {
    unsigned char* p = nullptr;
    if (cudaGetSymbolAddress((void**)&p, g_swa_noalloc_scratch) != cudaSuccess) return nullptr;
    ptr[dev] = p;
    ctx[dev] = c;
  }
  return ptr[dev];
}

size_t carve256(size_t& off, size_t bytes) {
  const size_t o = off;
  off = (off + bytes + 255) & ~size_t(255);
  return o;
}

}  // namespace

}  // namespace samba

using namespace samba;

extern "C" samba_status samba_swa_fwd_noalloc(const void* q, const void* k, const void* v, void* o, int B, int L,
                                              int Hq, int Hkv, int head_dim, int window, float rope_base,
                                              int64_t pos0, float softmax_scale, samba_dtype dtype,
                                              samba_stream stream) {
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype != SAMBA_F32 && dtype != SAMBA_BF16) return SAMBA_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || B < 1 || L < 0 || Hq < 1 || Hkv < 1 || window < 1 || pos0 < 0 || rope_base < 0.f)
    return SAMBA_ERR_INVALID_ARG;
  if (Hq % Hkv) return SAMBA_ERR_INVALID_ARG;
  if (head_dim != 16 && head_dim != 32 && head_dim != 64 && !(head_dim == 256 && dtype == SAMBA_BF16))
    return SAMBA_ERR_UNSUPPORTED;
  if (pos0 + (int64_t)L > (int64_t(1) << 30)) return SAMBA_ERR_UNSUPPORTED;
  if (B > kMaxGridYZ || Hq > kMaxGridYZ) return SAMBA_ERR_UNSUPPORTED;  // before any launch
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
    const size_t es = dtype_size(dtype);
    size_t off = 0;
    const size_t o_tab = carve256(off, rope_table_bytes(head_dim));
    const size_t o_q = carve256(off, (size_t)B * L * Hq * head_dim * es);
    const size_t o_k = carve256(off, (size_t)B * L * Hkv * head_dim * es);
    if (off > kNoallocScratchBytes) return SAMBA_ERR_UNSUPPORTED;  // does not fit the fixed scratch
    unsigned char* base = noalloc_scratch_ptr();
    if (!base) return SAMBA_ERR_CUDA;
    float2* tab = (float2*)(base + o_tab);
    void* qr = base + o_q;
    void* kr = base + o_k;
    samba_status s = launch_build_rope_table(tab, head_dim, rope_base, st);
    if (s == SAMBA_OK) s = launch_rope_apply(q, qr, B, L, Hq, head_dim, pos0, tab, dtype, st);
    if (s == SAMBA_OK) s = launch_rope_apply(k, kr, B, L, Hkv, head_dim, pos0, tab, dtype, st);
    if (s != SAMBA_OK) return s;
    a.q = qr;
    a.k = kr;
  }
  return launch_swa(a, st);
}
