// Decode-step kernels: one new token per sequence with a fixed-size state
// [Samba 5: decoding cost stays constant per token because the SSM state is
// fixed-size and the SWA keeps only the last w keys; the blog page's
// ring-buffer KV cache of w slots].  Plus the prefill -> decode-state handoff
// (ring fill, position set).
#include "common.cuh"
#include "decode.h"

namespace samba {

namespace {

// conv state shift + one output:  window = [state (k-1, oldest first), x_new]
template <typename T>
__global__ void conv_step_kernel(const T* __restrict__ hz, int64_t ld_hz, const float* __restrict__ w,
                                 const float* __restrict__ bias, T* __restrict__ state, T* __restrict__ u, int B,
                                 int D, int k) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * D) return;
  const int b = idx / D, c = idx % D;
  T* sp = state + ((size_t)b * D + c) * (k - 1);
  float win[8];
  for (int j = 0; j < k - 1; ++j) win[j] = Elt<T>::to_f(sp[j]);
  const T xn = hz[(size_t)b * ld_hz + c];
  win[k - 1] = Elt<T>::to_f(xn);
  float acc = bias ? bias[c] : 0.f;
  for (int j = 0; j < k; ++j) acc = fmaf(w[(size_t)c * k + j], win[j], acc);
  for (int j = 0; j < k - 2; ++j) sp[j] = sp[j + 1];
  sp[k - 2] = xn;
  const float s = sizeof(T) == 4 ? sigmoid_acc(acc) : sigmoid_fast(acc);
  u[(size_t)b * D + c] = Elt<T>::from_f(acc * s);
}

// one recurrence step per (b, c), 16 fp32 states
template <typename T>
__global__ void scan_step_kernel(const T* __restrict__ u, const T* __restrict__ dlt, const T* __restrict__ z,
                                 int64_t ld_z, const T* __restrict__ xdbl, int64_t ld_x, int r_off,
                                 const float* __restrict__ A_log, const float* __restrict__ Dskip,
                                 float* __restrict__ ssm, T* __restrict__ y, int B, int D) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * D) return;
  const int b = idx / D, c = idx % D;
  const float delta = Elt<T>::to_f(dlt[(size_t)b * D + c]);
  const float uv = Elt<T>::to_f(u[(size_t)b * D + c]);
  const T* Bp = xdbl + (size_t)b * ld_x + r_off;
  const T* Cp = Bp + 16;
  float* hp = ssm + ((size_t)b * D + c) * 16;
  float yv = 0.f;
  const float du = delta * uv;
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    const float A = -expf(A_log[(size_t)c * 16 + n]);
    const float dA = expf(delta * A);
    const float hn = fmaf(dA, hp[n], du * Elt<T>::to_f(Bp[n]));
    hp[n] = hn;
    yv = fmaf(Elt<T>::to_f(Cp[n]), hn, yv);
  }
  yv = fmaf(Dskip ? Dskip[c] : 0.f, uv, yv);
  const float zv = Elt<T>::to_f(z[(size_t)b * ld_z + c]);
  const float s = sizeof(T) == 4 ? sigmoid_acc(zv) : sigmoid_fast(zv);
  y[(size_t)b * D + c] = Elt<T>::from_f(yv * zv * s);
}

// k, v (post-RoPE) of the new token into ring slot pos mod w
template <typename T>
__global__ void ring_write_kernel(const T* __restrict__ qkv, int64_t ld, int k_off, int v_off,
                                  const int64_t* __restrict__ pos, T* __restrict__ k_ring, T* __restrict__ v_ring,
                                  int window, int kvw) {
  const int b = blockIdx.x;
  const int64_t slot = pos[b] % window;
  const T* src = qkv + (size_t)b * ld;
  T* kd = k_ring + ((size_t)b * window + slot) * kvw;
  T* vd = v_ring + ((size_t)b * window + slot) * kvw;
  for (int i = threadIdx.x; i < kvw; i += blockDim.x) {
    kd[i] = src[k_off + i];
    vd[i] = src[v_off + i];
  }
}

// Attention of the new query over the min(pos+1, w) valid ring slots.  The set
// of valid slots is {0 .. min(pos+1, w) - 1} whatever the wrap state, and the
// softmax sum does not depend on their order.  CTA = (kv head, batch row),
// one warp per query head of the group; K/V blocks shared through smem.
constexpr int kDecKB = 64;

template <typename T>
__global__ void attn_decode_kernel(const T* __restrict__ qkv, int64_t ld, const int64_t* __restrict__ pos,
                                   const T* __restrict__ k_ring, const T* __restrict__ v_ring, T* __restrict__ o,
                                   int Hq, int Hkv, int hd, int window, float scale) {
  extern __shared__ float dsm[];
  const int g = blockIdx.x, b = blockIdx.y;
  const int grp = Hq / Hkv;
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int h = g * grp + warp;
  float* Ks = dsm;                       // [kDecKB][hd+1]
  float* Vs = dsm + kDecKB * (hd + 1);   // [kDecKB][hd+1]
  const int64_t P = pos[b];
  const int nvalid = (int)(P + 1 < window ? P + 1 : window);
  const T* qrow = qkv + (size_t)b * ld + (size_t)h * hd;
  float q[4], oacc[4];
  const int nd = (hd + 31) / 32;  // dims per lane (<= 4)
  for (int r = 0; r < 4; ++r) {
    const int i = lane + 32 * r;
    q[r] = (r < nd && i < hd) ? Elt<T>::to_f(qrow[i]) * scale : 0.f;
    oacc[r] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const size_t kvw = (size_t)Hkv * hd;
  for (int s0 = 0; s0 < nvalid; s0 += kDecKB) {
    const int nb = min(kDecKB, nvalid - s0);
    for (int e = threadIdx.x; e < nb * hd; e += blockDim.x) {
      const int j = e / hd, i = e % hd;
      const size_t off = ((size_t)b * window + s0 + j) * kvw + (size_t)g * hd + i;
      Ks[j * (hd + 1) + i] = Elt<T>::to_f(k_ring[off]);
      Vs[j * (hd + 1) + i] = Elt<T>::to_f(v_ring[off]);
    }
    __syncthreads();
    if (warp < grp) {
      // scores: lane handles keys lane and lane+32
      float sc[2];
      for (int r = 0; r < 2; ++r) {
        const int j = lane + 32 * r;
        float acc = 0.f;
        for (int i = 0; i < hd; ++i) {
          const float qi = __shfl_sync(0xffffffffu, q[i / 32], i % 32);
          acc = fmaf(qi, j < nb ? Ks[j * (hd + 1) + i] : 0.f, acc);
        }
        sc[r] = j < nb ? acc : -INFINITY;
      }
      float bm = fmaxf(sc[0], sc[1]);
      for (int off = 16; off; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
      const float mnew = fmaxf(m, bm);
      const float corr = expf(m - mnew);
      float p[2];
      float ps = 0.f;
      for (int r = 0; r < 2; ++r) {
        p[r] = sc[r] == -INFINITY ? 0.f : expf(sc[r] - mnew);
        ps += p[r];
      }
      for (int off = 16; off; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l = l * corr + ps;
      for (int r = 0; r < 4; ++r) oacc[r] *= corr;
      for (int j = 0; j < nb; ++j) {
        const float pj = __shfl_sync(0xffffffffu, p[j / 32], j % 32);
        for (int r = 0; r < nd; ++r) {
          const int i = lane + 32 * r;
          if (i < hd) oacc[r] = fmaf(pj, Vs[j * (hd + 1) + i], oacc[r]);
        }
      }
      m = mnew;
    }
    __syncthreads();
  }
  if (warp < grp) {
    const float inv = 1.f / l;
    T* orow = o + (size_t)b * Hq * hd + (size_t)h * hd;
    for (int r = 0; r < nd; ++r) {
      const int i = lane + 32 * r;
      if (i < hd) orow[i] = Elt<T>::from_f(oacc[r] * inv);
    }
  }
}

__global__ void pos_add_kernel(int64_t* pos, int B, int64_t inc, int set) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < B) pos[i] = set ? inc : pos[i] + inc;
}

// prefill -> ring: positions max(0, L-w) .. L-1 into slot p mod w
template <typename T>
__global__ void ring_fill_kernel(const T* __restrict__ qkv, int64_t ld, int k_off, int v_off, T* __restrict__ k_ring,
                                 T* __restrict__ v_ring, int L, int window, int kvw) {
  const int j = blockIdx.x;  // 0 .. min(L, w)-1
  const int b = blockIdx.y;
  const int n = min(L, window);
  if (j >= n) return;
  const int p = L - n + j;
  const int slot = p % window;
  const T* src = qkv + ((size_t)b * L + p) * ld;
  T* kd = k_ring + ((size_t)b * window + slot) * kvw;
  T* vd = v_ring + ((size_t)b * window + slot) * kvw;
  for (int i = threadIdx.x; i < kvw; i += blockDim.x) {
    kd[i] = src[k_off + i];
    vd[i] = src[v_off + i];
  }
}

}  // namespace

#define SAMBA_DT_DISPATCH(dt, KERNEL_CALL_BF16, KERNEL_CALL_F32) \
  do {                                                           \
    if ((dt) == SAMBA_BF16) {                                    \
      KERNEL_CALL_BF16;                                          \
    } else {                                                     \
      KERNEL_CALL_F32;                                           \
    }                                                            \
  } while (0)

samba_status launch_conv_step(const void* hz, int64_t ld_hz, const float* w, const float* bias, void* state, void* u,
                              int B, int D, int k, samba_dtype dt, cudaStream_t st) {
  if (k < 2 || k > 8) return SAMBA_ERR_UNSUPPORTED;
  const int n = B * D;
  SAMBA_DT_DISPATCH(dt,
                    (conv_step_kernel<bf16><<<(n + 255) / 256, 256, 0, st>>>((const bf16*)hz, ld_hz, w, bias,
                                                                             (bf16*)state, (bf16*)u, B, D, k)),
                    (conv_step_kernel<float><<<(n + 255) / 256, 256, 0, st>>>((const float*)hz, ld_hz, w, bias,
                                                                              (float*)state, (float*)u, B, D, k)));
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

samba_status launch_scan_step(const void* u, const void* dlt, const void* z, int64_t ld_z, const void* xdbl,
                              int64_t ld_x, int r_off, const float* A_log, const float* Dskip, float* ssm, void* y,
                              int B, int D, samba_dtype dt, cudaStream_t st) {
  const int n = B * D;
  SAMBA_DT_DISPATCH(dt,
                    (scan_step_kernel<bf16><<<(n + 127) / 128, 128, 0, st>>>(
                        (const bf16*)u, (const bf16*)dlt, (const bf16*)z, ld_z, (const bf16*)xdbl, ld_x, r_off, A_log,
                        Dskip, ssm, (bf16*)y, B, D)),
                    (scan_step_kernel<float><<<(n + 127) / 128, 128, 0, st>>>(
                        (const float*)u, (const float*)dlt, (const float*)z, ld_z, (const float*)xdbl, ld_x, r_off,
                        A_log, Dskip, ssm, (float*)y, B, D)));
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

samba_status launch_ring_write(const void* qkv, int64_t ld, int k_off, int v_off, const int64_t* pos, void* k_ring,
                               void* v_ring, int B, int window, int kvw, samba_dtype dt, cudaStream_t st) {
  SAMBA_DT_DISPATCH(dt,
                    (ring_write_kernel<bf16><<<B, 128, 0, st>>>((const bf16*)qkv, ld, k_off, v_off, pos,
                                                                (bf16*)k_ring, (bf16*)v_ring, window, kvw)),
                    (ring_write_kernel<float><<<B, 128, 0, st>>>((const float*)qkv, ld, k_off, v_off, pos,
                                                                 (float*)k_ring, (float*)v_ring, window, kvw)));
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

samba_status launch_attn_decode(const void* qkv, int64_t ld, const int64_t* pos, const void* k_ring,
                                const void* v_ring, void* o, int B, int Hq, int Hkv, int hd, int window, float scale,
                                samba_dtype dt, cudaStream_t st) {
  if (hd > 128) return SAMBA_ERR_UNSUPPORTED;
  const int grp = Hq / Hkv;
  const int threads = ((grp * 32) < 128 ? 128 : grp * 32);
  if (threads > 1024) return SAMBA_ERR_UNSUPPORTED;
  const size_t smem = 2 * kDecKB * (hd + 1) * sizeof(float);
  dim3 grid(Hkv, B);
  SAMBA_DT_DISPATCH(dt,
                    (attn_decode_kernel<bf16><<<grid, threads, smem, st>>>(
                        (const bf16*)qkv, ld, pos, (const bf16*)k_ring, (const bf16*)v_ring, (bf16*)o, Hq, Hkv, hd,
                        window, scale)),
                    (attn_decode_kernel<float><<<grid, threads, smem, st>>>(
                        (const float*)qkv, ld, pos, (const float*)k_ring, (const float*)v_ring, (float*)o, Hq, Hkv,
                        hd, window, scale)));
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

samba_status launch_pos_update(int64_t* pos, int B, int64_t value, bool set, cudaStream_t st) {
  pos_add_kernel<<<(B + 127) / 128, 128, 0, st>>>(pos, B, value, set ? 1 : 0);
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

samba_status launch_ring_fill(const void* qkv, int64_t ld, int k_off, int v_off, void* k_ring, void* v_ring, int B,
                              int L, int window, int kvw, samba_dtype dt, cudaStream_t st) {
  const int n = L < window ? L : window;
  if (n == 0) return SAMBA_OK;
  dim3 grid(n, B);
  SAMBA_DT_DISPATCH(dt,
                    (ring_fill_kernel<bf16><<<grid, 128, 0, st>>>((const bf16*)qkv, ld, k_off, v_off, (bf16*)k_ring,
                                                                  (bf16*)v_ring, L, window, kvw)),
                    (ring_fill_kernel<float><<<grid, 128, 0, st>>>((const float*)qkv, ld, k_off, v_off,
                                                                   (float*)k_ring, (float*)v_ring, L, window, kvw)));
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

}  // namespace samba
