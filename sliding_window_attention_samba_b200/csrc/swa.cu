// Causal sliding-window attention with grouped-query heads
// [Samba 3.4 "Window Specification", "Implementation"; GQA per the model-size
// table]: query t of head h attends to keys s in [max(0, t-w+1), t] of kv head
// h / (Hq/Hkv), softmax over scaled dot products, fp32 accumulation.
//
// This file holds the CUDA-core kernel (fp32 path, small head dims, and the
// reference-precision path).  Only key blocks that intersect the band of the
// CTA's 128 queries are visited, so work is O(L * w), never O(L^2).
#define SAMBA_TU_ID 7  // site id of this file in debug-check reports
#include "common.cuh"
#include "kernels.h"

namespace samba {

namespace {

constexpr int SW_Q = 128;  // queries per CTA (one per thread)
constexpr int SW_K = 32;   // keys per shared-memory block

template <typename T, int D>
__global__ void __launch_bounds__(SW_Q) swa_simt_kernel(const SwaArgs a) {
  __shared__ float Ks[SW_K][D];
  __shared__ float Vs[SW_K][D];
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * SW_Q;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int g = h / (a.Hq / a.Hkv);
  const int t = t0 + tid;
  const bool active = t < a.L;
  const int Lk = a.L + a.qoff;  // key rows per batch row
  const int tk = t + a.qoff;    // this query's own key row
  const float sl2 = a.scale * 1.4426950408889634f;  // scores in log2 units

  float q[D], o[D];
  const T* qp = (const T*)a.q + ((size_t)b * a.L + (active ? t : 0)) * a.ld_q + (size_t)h * D;
#pragma unroll
  for (int i = 0; i < D; ++i) {
    q[i] = active ? Elt<T>::to_f(qp[i]) * sl2 : 0.f;
    o[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  const int kmin = max(0, t0 + a.qoff - a.window + 1);
  const int kmax = min(Lk - 1, t0 + a.qoff + SW_Q - 1);
  const T* kbase = (const T*)a.k + (size_t)b * Lk * a.ld_k + (size_t)g * D;
  const T* vbase = (const T*)a.v + (size_t)b * Lk * a.ld_v + (size_t)g * D;
  for (int kb = kmin; kb <= kmax; kb += SW_K) {
    for (int e = tid; e < SW_K * D; e += SW_Q) {
      const int j = e / D, i = e % D;
      const int s = kb + j;
      Ks[j][i] = s <= kmax ? Elt<T>::to_f(kbase[(size_t)s * a.ld_k + i]) : 0.f;
      Vs[j][i] = s <= kmax ? Elt<T>::to_f(vbase[(size_t)s * a.ld_v + i]) : 0.f;
    }
    __syncthreads();
    if (active) {
      float sc[SW_K];
      float bmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < SW_K; ++j) {
        const int s = kb + j;
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < D; ++i) acc = fmaf(q[i], Ks[j][i], acc);
        const bool in_band = s <= tk && s > tk - a.window;
        sc[j] = in_band ? acc : -INFINITY;
        bmax = fmaxf(bmax, sc[j]);
      }
      if (bmax > -INFINITY) {
        const float mnew = fmaxf(m, bmax);
        const float corr = exp2f(m - mnew);
        l *= corr;
#pragma unroll
        for (int i = 0; i < D; ++i) o[i] *= corr;
#pragma unroll
        for (int j = 0; j < SW_K; ++j) {
          const float p = exp2f(sc[j] - mnew);
          l += p;
#pragma unroll
          for (int i = 0; i < D; ++i) o[i] = fmaf(p, Vs[j][i], o[i]);
        }
        m = mnew;
      }
    }
    __syncthreads();
  }
  if (active) {
    const float inv = 1.f / l;
    T* op = (T*)a.o + ((size_t)b * a.L + t) * a.ld_o + (size_t)h * D;
#pragma unroll
    for (int i = 0; i < D; ++i) op[i] = Elt<T>::from_f(o[i] * inv);
  }
}

template <typename T, int D>
samba_status simt_launch(const SwaArgs& a, cudaStream_t st) {
  dim3 grid((a.L + SW_Q - 1) / SW_Q, a.Hq, a.B);
  swa_simt_kernel<T, D><<<grid, SW_Q, 0, st>>>(a);
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

template <typename T>
samba_status simt_dispatch(const SwaArgs& a, cudaStream_t st) {
  switch (a.d) {
    case 16: return simt_launch<T, 16>(a, st);
    case 32: return simt_launch<T, 32>(a, st);
    case 64: return simt_launch<T, 64>(a, st);
  }
  return SAMBA_ERR_UNSUPPORTED;
}

}  // namespace

samba_status launch_swa_simt(const SwaArgs& a, cudaStream_t st) {
  return a.dtype == SAMBA_BF16 ? simt_dispatch<bf16>(a, st) : simt_dispatch<float>(a, st);
}

samba_status launch_swa(const SwaArgs& a, cudaStream_t st) {
  if (!a.q || !a.k || !a.v || !a.o || a.B < 1 || a.L < 0 || a.Hq < 1 || a.Hkv < 1 || a.window < 1 || a.qoff < 0)
    return SAMBA_ERR_INVALID_ARG;
  if (a.Hq % a.Hkv) return SAMBA_ERR_INVALID_ARG;
  if (a.B > kMaxGridYZ || a.Hq > kMaxGridYZ) return SAMBA_ERR_UNSUPPORTED;
  if (a.L == 0) return SAMBA_OK;
  if (swa_tc_supported(a)) return launch_swa_tc(a, st);
  return launch_swa_simt(a, st);
}

}  // namespace samba
