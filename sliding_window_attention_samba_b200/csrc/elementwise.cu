// HBM-bound helper kernels: RMSNorm, causal depthwise conv + SiLU, RoPE tables
// and the standalone RoPE rotation.
#define SAMBA_TU_ID 3  // site id of this file in debug-check reports
#include "common.cuh"
#include "kernels.h"

namespace samba {

// ===========================================================================
// RMSNorm [Samba 3.2: every layer is preceded by an RMSNorm]
//   out = x / sqrt(mean(x^2) + eps) * g
// One warp per row; 8-element vector accesses; fp32 sum of squares.
// ===========================================================================
template <typename T>
__global__ void rmsnorm_kernel(const T* __restrict__ x, int64_t ld_x, const float* __restrict__ g,
                               T* __restrict__ out, int64_t ld_out, int64_t rows, int dim, float eps) {
  pdl_wait();
  pdl_trigger();
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const T* xr = x + row * ld_x;
  T* orow = out + row * ld_out;
  float ss = 0.f;
  for (int c = lane * 8; c < dim; c += 256) {
    float f[8];
    load8(xr + c, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss / (float)dim + eps);
  for (int c = lane * 8; c < dim; c += 256) {
    float f[8], gg[8];
    load8(xr + c, f);
    load8(g + c, gg);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = f[i] * r * gg[i];
    store8(orow + c, f);
  }
}

// Few rows (decode: one row per sequence): one CTA per row, each thread one
// 8-element piece held in registers, the sum of squares reduced across the CTA
// (one global load per element instead of two dependent passes of a warp).
template <typename T>
__global__ void rmsnorm_row_kernel(const T* __restrict__ x, int64_t ld_x, const float* __restrict__ g,
                                   T* __restrict__ out, int64_t ld_out, int dim, float eps) {
  pdl_wait();
  pdl_trigger();
  __shared__ float part[32];
  const int64_t row = blockIdx.x;
  const int c = threadIdx.x * 8;
  const bool in = c < dim;
  float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, gg[8];
  if (in) {
    load8(x + row * ld_x + c, f);
    load8(g + c, gg);
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) part[warp] = ss;
  __syncthreads();
  if (warp == 0) {
    float t = lane < (int)(blockDim.x >> 5) ? part[lane] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) part[0] = t;
  }
  __syncthreads();
  const float r = rsqrtf(part[0] / (float)dim + eps);
  if (in) {
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = f[i] * r * gg[i];
    store8(out + row * ld_out + c, f);
  }
}

samba_status launch_rmsnorm(const void* x, int64_t ld_x, const float* g, void* out, int64_t ld_out, int64_t rows,
                            int dim, float eps, samba_dtype dt, cudaStream_t st, bool pdl) {
  if (!x || !g || !out || rows < 0 || dim <= 0) return SAMBA_ERR_INVALID_ARG;
  if (dim % 8 || ld_x % 8 || ld_out % 8 || !aligned16(x) || !aligned16(out) || !aligned16(g))
    return SAMBA_ERR_UNSUPPORTED;
  if (rows == 0) return SAMBA_OK;
  if (rows <= num_sms() && dim <= 8 * 1024) {
    const int threads = ((dim / 8 + 31) / 32) * 32;
    const cudaError_t e =
        dt == SAMBA_BF16
            ? launch_k(rmsnorm_row_kernel<bf16>, dim3((unsigned)rows), dim3(threads), 0, st, pdl, (const bf16*)x,
                       ld_x, g, (bf16*)out, ld_out, dim, eps)
            : launch_k(rmsnorm_row_kernel<float>, dim3((unsigned)rows), dim3(threads), 0, st, pdl, (const float*)x,
                       ld_x, g, (float*)out, ld_out, dim, eps);
    return e == cudaSuccess ? SAMBA_OK : SAMBA_ERR_CUDA;
  }
  const int warps = 8;
  dim3 grid((unsigned)((rows + warps - 1) / warps));
  const cudaError_t e =
      dt == SAMBA_BF16
          ? launch_k(rmsnorm_kernel<bf16>, grid, dim3(warps * 32), 0, st, pdl, (const bf16*)x, ld_x, g, (bf16*)out,
                     ld_out, rows, dim, eps)
          : launch_k(rmsnorm_kernel<float>, grid, dim3(warps * 32), 0, st, pdl, (const float*)x, ld_x, g,
                     (float*)out, ld_out, rows, dim, eps);
  return e == cudaSuccess ? SAMBA_OK : SAMBA_ERR_CUDA;
}

// ===========================================================================
// Token embedding lookup [Samba 3.2: token embeddings enter the first layer]:
// one warp per token, 16-byte pieces of the row.
// ===========================================================================
__global__ void embedding_kernel(const int32_t* __restrict__ ids, const uint4* __restrict__ table,
                                 uint4* __restrict__ out, int64_t T, int vec, int vocab, int* err) {
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const int id = ids[t];
  const bool ok = id >= 0 && id < vocab;
  if (!ok && lane == 0) raise_error(err, kErrDevice);
  for (int i = lane; i < vec; i += 32) out[t * vec + i] = ok ? table[(int64_t)id * vec + i] : make_uint4(0, 0, 0, 0);
}

samba_status launch_embedding(const int32_t* ids, const void* table, void* out, int64_t T, int d_model, int vocab,
                              samba_dtype dt, cudaStream_t st) {
  if (!ids || !table || !out || T < 0 || d_model <= 0 || vocab < 1) return SAMBA_ERR_INVALID_ARG;
  const size_t row = (size_t)d_model * dtype_size(dt);
  if (row % 16 || !aligned16(table) || !aligned16(out)) return SAMBA_ERR_UNSUPPORTED;
  if (T == 0) return SAMBA_OK;
  const int warps = 8;
  embedding_kernel<<<(unsigned)((T + warps - 1) / warps), warps * 32, 0, st>>>(
      ids, (const uint4*)table, (uint4*)out, T, (int)(row / 16), vocab, device_error_word());
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

// ===========================================================================
// Short convolution [Samba 3.4 "Input Projection and Short Convolution"]
//   u[b,t,c] = SiLU(sum_j w[c,j] x[b,t-(k-1)+j,c] + bias[c])
// A thread owns 8 consecutive channels and a run of kRun tokens, keeping the
// last k-1 inputs in registers (each input is read once from HBM per run plus
// k-1 halo rows).  Also writes the conv state (last k-1 inputs) when asked.
// ===========================================================================
constexpr int kConvRun = kConvRunTokens;
constexpr int kMaxK = 8;

template <typename T, int K>
__global__ void conv_silu_kernel(const T* __restrict__ x, int64_t ld_x, const float* __restrict__ w,
                                 const float* __restrict__ bias, T* __restrict__ u, T* __restrict__ state,
                                 const T* __restrict__ hist_in, int L, int D) {
  const int cg = blockIdx.x * blockDim.x + threadIdx.x;  // channel group of 8
  const int c0 = cg * 8;
  const int t0 = blockIdx.y * kConvRun;
  const int b = blockIdx.z;
  if (c0 >= D) return;
  float wr[8][K], bb[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
#pragma unroll
    for (int j = 0; j < K; ++j) wr[i][j] = w[(size_t)(c0 + i) * K + j];
    bb[i] = bias ? bias[c0 + i] : 0.f;
  }
  const T* xb = x + (size_t)b * L * ld_x + c0;
  // input at token t < 0: the carried history (slot K-1+t of each channel), or zero
  auto before = [&](int t, float* f) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      f[i] = hist_in ? Elt<T>::to_f(hist_in[((size_t)b * D + c0 + i) * (K - 1) + (K - 1) + t]) : 0.f;
  };
  float hist[K][8];  // hist[j] = x[t-(K-1)+j]
#pragma unroll
  for (int j = 0; j < K - 1; ++j) {
    const int t = t0 - (K - 1) + j;
    if (t >= 0) load8(xb + (size_t)t * ld_x, hist[j]);
    else before(t, hist[j]);
  }
  const int tend = min(t0 + kConvRun, L);
  // kConvAhead tokens' loads in flight at a time, then their outputs
  constexpr int kConvAhead = 4;
  for (int tb = t0; tb < tend; tb += kConvAhead) {
    float xr[kConvAhead][8];
#pragma unroll
    for (int k = 0; k < kConvAhead; ++k)
      if (tb + k < tend) load8(xb + (size_t)(tb + k) * ld_x, xr[k]);
#pragma unroll
    for (int k = 0; k < kConvAhead; ++k) {
      if (tb + k >= tend) break;
#pragma unroll
      for (int i = 0; i < 8; ++i) hist[K - 1][i] = xr[k][i];
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float acc = bb[i];
#pragma unroll
        for (int j = 0; j < K; ++j) acc = fmaf(wr[i][j], hist[j][i], acc);
        if constexpr (sizeof(T) == 4) o[i] = acc * sigmoid_acc(acc);
        else o[i] = acc * sigmoid_fast(acc);
      }
      store8(u + ((size_t)b * L + tb + k) * D + c0, o);
#pragma unroll
      for (int j = 0; j < K - 1; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) hist[j][i] = hist[j + 1][i];
    }
  }
  // conv state: the last K-1 inputs of the sequence, oldest first, [B, D, K-1]
  if (state && t0 <= L - 1 && L - 1 < t0 + kConvRun) {
    for (int j = 0; j < K - 1; ++j) {
      const int t = L - (K - 1) + j;
      float f[8];
      if (t >= 0) load8(xb + (size_t)t * ld_x, f);
      else before(t, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) state[((size_t)b * D + c0 + i) * (K - 1) + j] = Elt<T>::from_f(f[i]);
    }
  }
}

template <typename T>
__global__ void conv_state_zero_kernel(T* state, size_t n) {
  size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (i < n) state[i] = Elt<T>::from_f(0.f);
}

template <typename T, int K>
samba_status launch_conv_k(const ConvArgs& a, cudaStream_t st) {
  const int groups = a.D / 8;
  if (a.B > kMaxGridYZ || a.L > kMaxConvTokens) return SAMBA_ERR_UNSUPPORTED;
  dim3 block(128);
  dim3 grid((groups + 127) / 128, (a.L + kConvRun - 1) / kConvRun, a.B);
  conv_silu_kernel<T, K><<<grid, block, 0, st>>>((const T*)a.x, a.ld_x, a.w, a.bias, (T*)a.u, (T*)a.state,
                                                 (const T*)a.hist, a.L, a.D);
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

template <typename T>
samba_status launch_conv_t(const ConvArgs& a, cudaStream_t st) {
  switch (a.k) {
    case 2: return launch_conv_k<T, 2>(a, st);
    case 3: return launch_conv_k<T, 3>(a, st);
    case 4: return launch_conv_k<T, 4>(a, st);
    case 5: return launch_conv_k<T, 5>(a, st);
    case 6: return launch_conv_k<T, 6>(a, st);
    case 7: return launch_conv_k<T, 7>(a, st);
    case 8: return launch_conv_k<T, 8>(a, st);
  }
  return SAMBA_ERR_UNSUPPORTED;
}

samba_status launch_causal_conv(const ConvArgs& a, cudaStream_t st) {
  if (!a.x || !a.w || !a.u || a.B < 1 || a.L < 0 || a.D < 1 || a.ld_x < a.D) return SAMBA_ERR_INVALID_ARG;
  if (a.k < 2 || a.k > kMaxK || a.D % 8 || a.ld_x % 8 || !aligned16(a.x) || !aligned16(a.u))
    return SAMBA_ERR_UNSUPPORTED;
  if (a.hist && a.hist == a.state) return SAMBA_ERR_INVALID_ARG;
  if (a.L == 0) {
    if (a.state && a.hist) {  // no new inputs: the history is the state
      const size_t bytes = (size_t)a.B * a.D * (a.k - 1) * dtype_size(a.dtype);
      if (cudaMemcpyAsync(a.state, a.hist, bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return SAMBA_ERR_CUDA;
    } else if (a.state) {
      const size_t n = (size_t)a.B * a.D * (a.k - 1);
      if (a.dtype == SAMBA_BF16) conv_state_zero_kernel<bf16><<<(unsigned)((n + 255) / 256), 256, 0, st>>>((bf16*)a.state, n);
      else conv_state_zero_kernel<float><<<(unsigned)((n + 255) / 256), 256, 0, st>>>((float*)a.state, n);
      SAMBA_CHECK_LAUNCH();
    }
    return SAMBA_OK;
  }
  return a.dtype == SAMBA_BF16 ? launch_conv_t<bf16>(a, st) : launch_conv_t<float>(a, st);
}

// ===========================================================================
// RoPE tables [Samba 3.4 "Positional Encoding": base 10000, standard RoPE]
//   tab[l][r][i] = (cos, sin)(r * 1024^l * theta_i),  theta_i = base^(-2i/d)
// built in fp64 so that a position p = a*2^20 + b*2^10 + c is rotated by the
// product of three table rotations with ~1e-7 rad error up to p < 2^30.
// ===========================================================================
size_t rope_table_bytes(int head_dim) {
  return (size_t)kRopeLevels * kRopeRadix * (head_dim / 2) * sizeof(float2);
}

__global__ void build_rope_table_kernel(float2* tab, int half, int head_dim, double base) {
  pdl_wait();
  pdl_trigger();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int total = kRopeLevels * kRopeRadix * half;
  if (idx >= total) return;
  const int i = idx % half;
  const int r = (idx / half) % kRopeRadix;
  const int l = idx / (half * kRopeRadix);
  const double theta = pow(base, -2.0 * (double)i / (double)head_dim);
  const double scale = l == 0 ? 1.0 : (l == 1 ? 1024.0 : 1048576.0);
  const double ang = (double)r * scale * theta;
  double s, c;
  sincos(ang, &s, &c);
  tab[idx] = make_float2((float)c, (float)s);
}

samba_status launch_build_rope_table(float2* tab, int head_dim, float base, cudaStream_t st, bool pdl) {
  const int half = head_dim / 2;
  const int total = kRopeLevels * kRopeRadix * half;
  return launch_k(build_rope_table_kernel, dim3((total + 255) / 256), dim3(256), 0, st, pdl, tab, half, head_dim,
                  (double)base) == cudaSuccess
             ? SAMBA_OK
             : SAMBA_ERR_CUDA;
}

template <typename T>
__global__ void rope_apply_kernel(const T* __restrict__ x, T* __restrict__ out, int64_t rows, int L, int H,
                                  int head_dim, int64_t pos0, const float2* __restrict__ tab) {
  // one thread per (row, head, i < half)
  const int half = head_dim / 2;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = rows * H * half;
  if (idx >= total) return;
  const int i = (int)(idx % half);
  const int64_t rh = idx / half;  // row * H + h
  const int64_t row = rh / H;
  const int64_t p = pos0 + row % L;
  const float2 c0 = tab[(0 * kRopeRadix + (p & 1023)) * half + i];
  const float2 c1 = tab[(1 * kRopeRadix + ((p >> 10) & 1023)) * half + i];
  const float2 c2 = tab[(2 * kRopeRadix + ((p >> 20) & 1023)) * half + i];
  float cr = c0.x * c1.x - c0.y * c1.y, sr = c0.x * c1.y + c0.y * c1.x;
  const float cs = cr * c2.x - sr * c2.y, sn = cr * c2.y + sr * c2.x;
  const T* xp = x + rh * head_dim;
  const float a = Elt<T>::to_f(xp[i]), bq = Elt<T>::to_f(xp[i + half]);
  T* op = out + rh * head_dim;
  op[i] = Elt<T>::from_f(a * cs - bq * sn);
  op[i + half] = Elt<T>::from_f(bq * cs + a * sn);
}

samba_status launch_rope_apply(const void* x, void* out, int B, int L, int H, int head_dim, int64_t pos0,
                               const float2* tab, samba_dtype dt, cudaStream_t st) {
  const int64_t rows = (int64_t)B * L;
  const int64_t total = rows * H * (head_dim / 2);
  if (total == 0) return SAMBA_OK;
  const unsigned grid = (unsigned)((total + 255) / 256);
  if (dt == SAMBA_BF16)
    rope_apply_kernel<bf16><<<grid, 256, 0, st>>>((const bf16*)x, (bf16*)out, rows, L, H, head_dim, pos0, tab);
  else
    rope_apply_kernel<float><<<grid, 256, 0, st>>>((const float*)x, (float*)out, rows, L, H, head_dim, pos0, tab);
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

// ===========================================================================
// Workspace guard bands of the debug-check build: a fixed 16-byte pattern,
// one thread per 16 bytes, one CTA row per band.
// ===========================================================================
__device__ __forceinline__ uint4 guard_pattern() { return make_uint4(0xA5C3E187u, 0x5A3C1E78u, 0xC0FFEE11u, 0x0DDBA115u); }

__global__ void guard_fill_kernel(char* base, GuardList g) {
  const int band = blockIdx.y;
  uint4* p = reinterpret_cast<uint4*>(base + g.off[band]);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < (int)(kGuardBytes / 16); i += gridDim.x * blockDim.x)
    p[i] = guard_pattern();
}

__global__ void guard_check_kernel(const char* base, GuardList g, int* err) {
  const int band = blockIdx.y;
  const uint4* p = reinterpret_cast<const uint4*>(base + g.off[band]);
  const uint4 e = guard_pattern();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < (int)(kGuardBytes / 16); i += gridDim.x * blockDim.x) {
    const uint4 v = p[i];
    if (v.x != e.x || v.y != e.y || v.z != e.z || v.w != e.w)
      raise_error(err, kErrBounds | (kGuardSiteTu << 4) | (band << 8));
  }
}

// The guarded store's index is masked into the array as well, so that the
// kernel stays in bounds even in a build whose checks are compiled out.
__global__ void dcheck_selftest_kernel(int* err, int idx, int n, int* sink) {
  __shared__ int buf[32];
  buf[threadIdx.x & 31] = 0;
  __syncthreads();
  if (SAMBA_DCHECK(err, idx >= 0 && idx < n)) buf[idx & 31] = 1;
  __syncthreads();
  if (threadIdx.x == 0 && sink) *sink = buf[0];
}

samba_status launch_dcheck_selftest(cudaStream_t st) {
  dcheck_selftest_kernel<<<1, 32, 0, st>>>(device_error_word(), 32, 32, nullptr);
  return cudaGetLastError() == cudaSuccess ? SAMBA_OK : SAMBA_ERR_CUDA;
}

samba_status launch_guard_fill(char* base, const GuardList& g, cudaStream_t st) {
  if (!kGuardBytes || g.n <= 0) return SAMBA_OK;
  guard_fill_kernel<<<dim3(1, g.n), 256, 0, st>>>(base, g);
  return cudaGetLastError() == cudaSuccess ? SAMBA_OK : SAMBA_ERR_CUDA;
}

samba_status launch_guard_check(const char* base, const GuardList& g, cudaStream_t st) {
  if (!kGuardBytes || g.n <= 0) return SAMBA_OK;
  guard_check_kernel<<<dim3(1, g.n), 256, 0, st>>>(base, g, device_error_word());
  return cudaGetLastError() == cudaSuccess ? SAMBA_OK : SAMBA_ERR_CUDA;
}

}  // namespace samba
