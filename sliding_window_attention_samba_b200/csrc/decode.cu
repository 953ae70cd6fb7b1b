// Decode-step kernels: one new token per sequence with a fixed-size state
// [Samba 5: decoding cost stays constant per token because the SSM state is
// fixed-size and the SWA keeps only the last w keys; the blog page's
// ring-buffer KV cache of w slots].  Plus the prefill -> decode-state handoff
// (ring fill, position set).
#include <string.h>

#define SAMBA_TU_ID 2  // site id of this file in debug-check reports
#include "common.cuh"
#include "decode.h"

namespace samba {

namespace {

__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t* r, const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row_addr)));
}
__device__ __forceinline__ void ldmatrix_x2(uint32_t* r, const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(smem_u32(row_addr)));
}

// conv state shift + one output:  window = [state (k-1, oldest first), x_new]
template <typename T>
__global__ void conv_step_kernel(const T* __restrict__ hz, int64_t ld_hz, const float* __restrict__ w,
                                 const float* __restrict__ bias, T* __restrict__ state, T* __restrict__ u, int B,
                                 int D, int k) {
  pdl_wait();
  pdl_trigger();
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

// One recurrence step per (b, c), 16 fp32 states: four lanes per channel, each
// holding four states, so that the state, A_log, B and C are read and the
// state written in contiguous runs of the warp (16-byte pieces per lane); the
// read-out sum is completed across the four lanes with two shuffles.
template <typename T>
__global__ void scan_step_kernel(const T* __restrict__ u, const T* __restrict__ dlt, const T* __restrict__ z,
                                 int64_t ld_z, const T* __restrict__ xdbl, int64_t ld_x, int r_off,
                                 const float* __restrict__ A_log, const float* __restrict__ Dskip,
                                 float* __restrict__ ssm, T* __restrict__ y, int B, int D) {
  pdl_wait();
  pdl_trigger();
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int q = (int)(gid & 3);  // states 4q .. 4q+3
  const int64_t idx = gid >> 2;  // (b, c)
  const bool live = idx < (int64_t)B * D;
  const int b = live ? (int)(idx / D) : 0, c = live ? (int)(idx % D) : 0;
  float yv = 0.f, uv = 0.f;
  if (live) {
    const float delta = Elt<T>::to_f(dlt[(size_t)b * D + c]);
    uv = Elt<T>::to_f(u[(size_t)b * D + c]);
    const T* Bp = xdbl + (size_t)b * ld_x + r_off + 4 * q;
    const T* Cp = Bp + 16;
    float4* hp = reinterpret_cast<float4*>(ssm + ((size_t)b * D + c) * 16 + 4 * q);
    const float4 av = *reinterpret_cast<const float4*>(A_log + (size_t)c * 16 + 4 * q);
    const float4 hv = *hp;
    float Bv[4], Cv[4];
    load4(Bp, Bv);
    load4(Cp, Cv);
    const float al[4] = {av.x, av.y, av.z, av.w};
    float h[4] = {hv.x, hv.y, hv.z, hv.w};
    const float du = delta * uv;
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      const float A = -expf(al[n]);
      const float dA = sizeof(T) == 4 ? expf(delta * A) : ex2_approx(delta * A * 1.4426950408889634f);
      h[n] = fmaf(dA, h[n], du * Bv[n]);
      yv = fmaf(Cv[n], h[n], yv);
    }
    *hp = make_float4(h[0], h[1], h[2], h[3]);
  }
  // the four lanes of a channel are consecutive lanes of one warp
  yv += __shfl_xor_sync(0xffffffffu, yv, 1);
  yv += __shfl_xor_sync(0xffffffffu, yv, 2);
  if (live && q == 0) {
    yv = fmaf(Dskip ? Dskip[c] : 0.f, uv, yv);
    const float zv = Elt<T>::to_f(z[(size_t)b * ld_z + c]);
    const float s = sizeof(T) == 4 ? sigmoid_acc(zv) : sigmoid_fast(zv);
    y[(size_t)b * D + c] = Elt<T>::from_f(yv * zv * s);
  }
}

// Recurrence step with the dt projection folded in [Samba 3.4 "Input-Dependent
// Selective Gating": Delta = softplus(dt_low W_dt^T + b)]: a CTA takes 16
// channels for 32 batch rows with 16 warps, warp w the rows w and w + 16
// (lane = 8 * q + i, lane q holding states 4q .. 4q+3 of channels i and i + 8).
// 512 threads at up to 64 registers put two CTAs on an SM, so that batch 32 at
// d_inner 4096 (256 CTAs) runs in one wave.  Everything that does not come from
// the kernels before it (the state, A, the 16 rows of W_dt into shared memory)
// is fetched before waiting for them; then the 32 rows of dt_low
// are staged and Delta is formed (tensor-core tiles for bf16 with R % 16 == 0,
// else each lane a quarter of the dot product and two shuffles), so Delta never
// goes through memory.  The state update and the read-out are those of the
// kernel above.
constexpr int kSdCh = 16;    // channels per CTA
constexpr int kSdRows = 32;  // batch rows per CTA
constexpr int kSdWarps = 16;  // two rows per warp
constexpr int kSdMaxR = 512;

template <typename T>
__global__ void __launch_bounds__(kSdWarps * 32, 2)
    scan_step_dt_kernel(const T* __restrict__ u, const T* __restrict__ z, int64_t ld_z, const T* __restrict__ xdbl,
                        int64_t ld_x, int R, const T* __restrict__ W_dt, const float* __restrict__ dt_bias,
                        const float* __restrict__ A_log, const float* __restrict__ Dskip, float* __restrict__ ssm,
                        T* __restrict__ y, int B, int D) {
  extern __shared__ __align__(16) unsigned char sd_smem[];
  constexpr int kVec = 16 / sizeof(T);  // elements per 16-byte piece
  const int pitch = R + kVec;            // padded rows (W rows of 8 channels land in distinct banks)
  T* Ws = reinterpret_cast<T*>(sd_smem);
  T* Xs = Ws + kSdCh * pitch;
  const int c0 = blockIdx.x * kSdCh, b0 = blockIdx.y * kSdRows;
  const int nv = R / kVec;  // 16-byte pieces per row
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ci = lane & 7, q = lane >> 3;
  // ---- before the wait: weights, A and the state (written only by this kernel's previous step)
  for (int e = threadIdx.x; e < kSdCh * nv; e += blockDim.x) {
    const int r = e / nv, k = e % nv;
    *reinterpret_cast<uint4*>(Ws + r * pitch + k * kVec) =
        *reinterpret_cast<const uint4*>(W_dt + (size_t)(c0 + r) * R + k * kVec);
  }
  float4 hv[2][2], av[2];  // [row][channel half], [channel half]: A (x log2 e for bf16)
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int c = c0 + ci + 8 * hh;
    const float4 al = *reinterpret_cast<const float4*>(A_log + (size_t)c * 16 + 4 * q);
    const float sc = sizeof(T) == 4 ? -1.f : -1.4426950408889634f;
    av[hh] = make_float4(sc * expf(al.x), sc * expf(al.y), sc * expf(al.z), sc * expf(al.w));
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int b = b0 + warp + kSdWarps * rr;
      hv[rr][hh] = b < B ? *reinterpret_cast<const float4*>(ssm + ((size_t)b * D + c) * 16 + 4 * q)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  pdl_wait();
  pdl_trigger();
  // ---- after it: dt_low rows (shared), B, C, u, z of this warp's rows
  for (int e = threadIdx.x; e < kSdRows * nv; e += blockDim.x) {
    const int r = e / nv, k = e % nv;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (b0 + r < B) v = *reinterpret_cast<const uint4*>(xdbl + (size_t)(b0 + r) * ld_x + k * kVec);
    *reinterpret_cast<uint4*>(Xs + r * pitch + k * kVec) = v;
  }
  float Bv[2][4], Cv[2][4], uv[2][2], zv[2][2];
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int b = b0 + warp + kSdWarps * rr;
#pragma unroll
    for (int n = 0; n < 4; ++n) Bv[rr][n] = Cv[rr][n] = 0.f;
    uv[rr][0] = uv[rr][1] = zv[rr][0] = zv[rr][1] = 0.f;
    if (b < B) {
      const T* Bp = xdbl + (size_t)b * ld_x + R + 4 * q;
      load4(Bp, Bv[rr]);
      load4(Bp + 16, Cv[rr]);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int c = c0 + ci + 8 * hh;
        uv[rr][hh] = Elt<T>::to_f(u[(size_t)b * D + c]);
        zv[rr][hh] = Elt<T>::to_f(z[(size_t)b * ld_z + c]);
      }
    }
  }
  __syncthreads();
  // bf16 with R % 16 == 0: the CTA's [32 rows x 16 channels] of dt_low W_dt^T as
  // four m16n8k16 tensor-core tiles (one warp each) through shared memory
  __shared__ float Dpre[kSdRows][kSdCh + 1];
  const bool tc_dot = sizeof(T) == 2 && R % 16 == 0;
  if (tc_dot) {
    if constexpr (sizeof(T) == 2) {
      if (warp < 4) {
        const int mt = warp >> 1, ntl = warp & 1;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        for (int ks = 0; ks < R / 16; ++ks) {
          uint32_t af[4], bfr[2];
          ldmatrix_x4(af, Xs + (mt * 16 + (lane & 15)) * pitch + ks * 16 + (lane >> 4) * 8);
          ldmatrix_x2(bfr, Ws + (ntl * 8 + (lane & 7)) * pitch + ks * 16 + ((lane >> 3) & 1) * 8);
          mma_bf16_16816(d, af, bfr[0], bfr[1]);
        }
        const int r0 = mt * 16 + (lane >> 2), cc = ntl * 8 + 2 * (lane & 3);
        Dpre[r0][cc] = d[0];
        Dpre[r0][cc + 1] = d[1];
        Dpre[r0 + 8][cc] = d[2];
        Dpre[r0 + 8][cc + 1] = d[3];
      }
    }
    __syncthreads();
  }
  const int n8 = R / 8;
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int row = warp + kSdWarps * rr;  // row within the CTA
    const int b = b0 + row;
    const bool live = b < B;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int c = c0 + ci + 8 * hh;
      float acc = 0.f;
      if (tc_dot) {
        acc = Dpre[row][ci + 8 * hh];
      } else {
        // Delta: lane q takes the 8-element pieces q, q + 4, q + 8, ... of the dot product
        for (int k = q; k < n8; k += 4) {
          float wv[8], xv[8];
          load8(Ws + (ci + 8 * hh) * pitch + k * 8, wv);
          load8(Xs + row * pitch + k * 8, xv);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc = fmaf(wv[j], xv[j], acc);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 8);
        acc += __shfl_xor_sync(0xffffffffu, acc, 16);
      }
      float delta = acc + (dt_bias ? dt_bias[c] : 0.f);
      if constexpr (sizeof(T) == 4) delta = softplus_acc(delta);
      else delta = softplus_1x(delta);
      const float A[4] = {av[hh].x, av[hh].y, av[hh].z, av[hh].w};
      float h[4] = {hv[rr][hh].x, hv[rr][hh].y, hv[rr][hh].z, hv[rr][hh].w};
      const float du = delta * uv[rr][hh];
      float yv = 0.f;
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        const float dA = sizeof(T) == 4 ? expf(delta * A[n]) : ex2_approx(delta * A[n]);
        h[n] = fmaf(dA, h[n], du * Bv[rr][n]);
        yv = fmaf(Cv[rr][n], h[n], yv);
      }
      if (live)
        *reinterpret_cast<float4*>(ssm + ((size_t)b * D + c) * 16 + 4 * q) = make_float4(h[0], h[1], h[2], h[3]);
      yv += __shfl_xor_sync(0xffffffffu, yv, 8);
      yv += __shfl_xor_sync(0xffffffffu, yv, 16);
      if (live && q == 0) {
        yv = fmaf(Dskip ? Dskip[c] : 0.f, uv[rr][hh], yv);
        const float sg = sizeof(T) == 4 ? sigmoid_acc(zv[rr][hh]) : sigmoid_fast(zv[rr][hh]);
        y[(size_t)b * D + c] = Elt<T>::from_f(yv * zv[rr][hh] * sg);
      }
    }
  }
}

// k, v (post-RoPE) of the new token into ring slot pos mod w.  A negative
// position (a corrupted state) latches SAMBA_ERR_DEVICE and writes nothing.
template <typename T>
__global__ void ring_write_kernel(const T* __restrict__ qkv, int64_t ld, int k_off, int v_off,
                                  const int64_t* __restrict__ pos, T* __restrict__ k_ring, T* __restrict__ v_ring,
                                  int window, int kvw, int* err) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x;
  if (pos[b] < 0) {
    if (threadIdx.x == 0) raise_error(err, kErrDevice);
    return;
  }
  const int64_t slot = pos[b] % window;
  if (!SAMBA_DCHECK(err, slot >= 0 && slot < window && k_off + kvw <= ld && v_off + kvw <= ld)) return;
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
constexpr int kDecMaxDpl = 8;  // head dims per lane: head_dim <= 256

template <typename T>
__global__ void attn_decode_kernel(const T* __restrict__ qkv, int64_t ld, const int64_t* __restrict__ pos,
                                   const T* __restrict__ k_ring, const T* __restrict__ v_ring, T* __restrict__ o,
                                   int Hq, int Hkv, int hd, int window, float scale) {
  pdl_wait();
  pdl_trigger();
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
  float q[kDecMaxDpl], oacc[kDecMaxDpl];
  const int nd = (hd + 31) / 32;  // dims per lane (<= 8: head_dim <= 256)
  for (int r = 0; r < kDecMaxDpl; ++r) {
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
      for (int r = 0; r < kDecMaxDpl; ++r) oacc[r] *= corr;
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

// Split-ring decode attention for bf16, head_dim 64, up to 8 query heads per kv
// head: a cluster of kSplit CTAs per (kv head, batch row), each CTA attending to
// a slice of the valid ring slots (flash-decoding), partial (max, sum, o) merged
// across the cluster through distributed shared memory.
constexpr int kSplit = 8;
constexpr int kSliceMax = 256;  // slots per CTA (window <= kSplit * kSliceMax)
constexpr int kHd = 64;
constexpr int kKvPad = kHd + 8;  // bf16 row pitch in smem (144 B: conflict-free 16-B reads)

struct DecPart {
  float m[8], l[8];
  float o[8][kHd];
};

__device__ __forceinline__ uint32_t dec_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Returns 0; peer loads add it to their address so that they depend on the
// barrier and cannot be scheduled above it.
__device__ __forceinline__ uint32_t dec_cluster_sync() {
  uint32_t tok;
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;\n\tmov.u32 %0, 0;"
               : "=r"(tok)::"memory");
  return tok;
}
__device__ __forceinline__ float dec_ld_remote(const float* p, uint32_t rank, uint32_t tok) {
  uint32_t ra;
  asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(p) + tok), "r"(rank));
  float v;
  asm("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra));
  return v;
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t* r, const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row_addr)));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Each warp owns 32 keys of the CTA's slice; the up to 8 query heads of the
// group are the rows of warp-level m16n8k16 tensor-core products (rows 8..15
// are zero padding): S = Q K^T, then O = P V with P taken straight from the S
// accumulators.  Max/sum/O are combined across the 8 warps in shared memory,
// then across the cluster's CTAs through distributed shared memory.
// Partial attention of the grp <= 8 query heads of kv head g (batch row b) over
// the ring slots [s0, s0 + n), n <= kSliceMax (the first `slice` rows of the
// shared K/V tiles are written, rows past n as zeros).  Leaves the per-head
// max, sum and unnormalised O in `part`.  All 256 threads take part.
__device__ __forceinline__ void dec_slice_partial(const bf16* __restrict__ qkv, int64_t ld,
                                                  const bf16* __restrict__ k_ring, const bf16* __restrict__ v_ring,
                                                  int Hkv, int grp, int window, int g, int b, int s0, int n,
                                                  int slice, float scale_log2, bf16* Ks, bf16* Vs, DecPart& part,
                                                  float (&wm)[8][8], float (&wl)[8][8], float (&wo)[8][8][kHd]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t kvw = (size_t)Hkv * kHd;
  // ---- K/V slice -> smem (16-byte vectors, all loads in flight before the stores);
  // rows past n are zero-filled so that the tensor-core tiles read finite values
  constexpr int kVecPerThread = kSliceMax * (kHd / 8) / 256;  // 8
  uint4 kreg[kVecPerThread], vreg[kVecPerThread];
#pragma unroll
  for (int it = 0; it < kVecPerThread; ++it) {
    const int e = threadIdx.x + 256 * it;
    const int j = e / (kHd / 8), c = e % (kHd / 8);
    kreg[it] = vreg[it] = make_uint4(0u, 0u, 0u, 0u);
    if (j < n) {
      const size_t off = ((size_t)b * window + s0 + j) * kvw + (size_t)g * kHd + c * 8;
      kreg[it] = *reinterpret_cast<const uint4*>(k_ring + off);
      vreg[it] = *reinterpret_cast<const uint4*>(v_ring + off);
    }
  }
#pragma unroll
  for (int it = 0; it < kVecPerThread; ++it) {
    const int e = threadIdx.x + 256 * it;
    const int j = e / (kHd / 8), c = e % (kHd / 8);
    if (j < slice) {
      *reinterpret_cast<uint4*>(&Ks[j * kKvPad + c * 8]) = kreg[it];
      *reinterpret_cast<uint4*>(&Vs[j * kKvPad + c * 8]) = vreg[it];
    }
  }
  // Q fragments (A operand, rows = heads): a0/a2 hold head lane/4, a1/a3 padding
  const int qr = lane >> 2, qc = 2 * (lane & 3);
  uint32_t qa[kHd / 16][4];
#pragma unroll
  for (int ks = 0; ks < kHd / 16; ++ks) {
    qa[ks][1] = qa[ks][3] = 0u;
    if (qr < grp) {
      const bf16* qrow = qkv + (size_t)b * ld + (size_t)(g * grp + qr) * kHd + ks * 16 + qc;
      qa[ks][0] = *reinterpret_cast<const uint32_t*>(qrow);
      qa[ks][2] = *reinterpret_cast<const uint32_t*>(qrow + 8);
    } else {
      qa[ks][0] = qa[ks][2] = 0u;
    }
  }
  __syncthreads();

  const int kb = warp * 32;  // this warp's keys within the slice
  const bool active = kb < n;
  // ---- S = Q K^T over this warp's 32 keys (4 n-tiles of 8 keys)
  float sacc[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
    for (int i = 0; i < 4; ++i) sacc[nt][i] = 0.f;
    if (active) {
#pragma unroll
      for (int ks = 0; ks < kHd / 16; ++ks) {
        const bf16* kp = &Ks[(kb + nt * 8 + qr) * kKvPad + ks * 16 + qc];
        mma_bf16_16816(sacc[nt], qa[ks], *reinterpret_cast<const uint32_t*>(kp),
                       *reinterpret_cast<const uint32_t*>(kp + 8));
      }
    }
  }
  // scale into the log2 domain, mask keys past n, warp max per head (row qr)
  float mx = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int key = kb + nt * 8 + qc + c;
      const float v = key < n ? sacc[nt][c] * scale_log2 : -INFINITY;
      sacc[nt][c] = v;
      mx = fmaxf(mx, v);
    }
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  if ((lane & 3) == 0) wm[warp][qr] = mx;
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < 8; ++w) M = fmaxf(M, wm[w][qr]);
  const float msub = M == -INFINITY ? 0.f : M;
  // P = exp2(s - M) (bf16 for the product), row sums
  float ls = 0.f;
  uint32_t pa[2][4];  // A fragments of P for the two 16-key steps
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    const float p0 = ex2_approx(sacc[nt][0] - msub), p1 = ex2_approx(sacc[nt][1] - msub);
    ls += p0 + p1;
    pa[nt >> 1][(nt & 1) ? 2 : 0] = pack_bf16x2(p0, p1);
    pa[nt >> 1][(nt & 1) ? 3 : 1] = 0u;
  }
  ls += __shfl_xor_sync(0xffffffffu, ls, 1);
  ls += __shfl_xor_sync(0xffffffffu, ls, 2);
  if ((lane & 3) == 0) wl[warp][qr] = ls;
  // ---- O_w = P V over this warp's 32 keys (2 k-steps x 8 n-tiles of dims)
  float oacc[kHd / 8][4];
#pragma unroll
  for (int nt = 0; nt < kHd / 8; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) oacc[nt][i] = 0.f;
  if (active) {
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
      for (int np = 0; np < kHd / 16; ++np) {
        uint32_t vb[4];
        const int key = kb + ks * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int dim = np * 16 + 8 * (lane >> 4);
        ldmatrix_x4_trans(vb, &Vs[key * kKvPad + dim]);
        mma_bf16_16816(oacc[2 * np], pa[ks], vb[0], vb[1]);
        mma_bf16_16816(oacc[2 * np + 1], pa[ks], vb[2], vb[3]);
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < kHd / 8; ++nt) {
    wo[warp][qr][nt * 8 + qc] = oacc[nt][0];
    wo[warp][qr][nt * 8 + qc + 1] = oacc[nt][1];
  }
  __syncthreads();
  // ---- CTA partial per head: m = M, l = sum_w, o = sum_w
  for (int e = threadIdx.x; e < grp * kHd; e += 256) {
    const int h = e / kHd, d = e % kHd;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) acc += wo[w][h][d];
    part.o[h][d] = acc;
    if (d == 0) {
      float mm = -INFINITY, ll = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        mm = fmaxf(mm, wm[w][h]);
        ll += wl[w][h];
      }
      part.m[h] = mm;
      part.l[h] = ll;
    }
  }
}

__global__ void __launch_bounds__(256, 1)
    attn_decode_split_kernel(const bf16* __restrict__ qkv, int64_t ld, const int64_t* __restrict__ pos,
                             const bf16* __restrict__ k_ring, const bf16* __restrict__ v_ring, bf16* __restrict__ o,
                             int Hq, int Hkv, int window, float scale_log2, int* err) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) unsigned char dec_dyn[];  // K slice | V slice (bf16, padded rows)
  bf16* Ks = reinterpret_cast<bf16*>(dec_dyn);
  bf16* Vs = Ks + kSliceMax * kKvPad;
  __shared__ DecPart part;
  __shared__ float wm[8][8], wl[8][8];  // [warp][head] partial max / sum
  __shared__ float wo[8][8][kHd];       // [warp][head][dim] partial O
  const uint32_t rank = dec_cluster_rank();
  const int g = blockIdx.y, b = blockIdx.z;
  const int grp = Hq / Hkv;
  const int64_t P = pos[b];
  const int nvalid = (int)(P + 1 < window ? P + 1 : window);
  const int slice = ((nvalid + kSplit - 1) / kSplit + 31) & ~31;
  const int s0 = (int)rank * slice;
  int n = max(0, min(nvalid, s0 + slice) - s0);
  // the slice's rows must fit the shared-memory slice and stay inside the ring
  if (!SAMBA_DCHECK(err, slice <= kSliceMax && (n == 0 || s0 + n <= window))) n = 0;
  dec_slice_partial(qkv, ld, k_ring, v_ring, Hkv, grp, window, g, b, s0, n, slice, scale_log2, Ks, Vs, part, wm, wl,
                    wo);
  __syncthreads();
  const uint32_t tok = dec_cluster_sync();
  // ---- merge: rank r finalises query head r of the group
  if ((int)rank < grp && threadIdx.x < kHd) {
    const int hw = (int)rank;
    float ms[kSplit], ls[kSplit], os[kSplit], M = -INFINITY;
#pragma unroll
    for (int s = 0; s < kSplit; ++s) {
      ms[s] = dec_ld_remote(&part.m[hw], s, tok);
      ls[s] = dec_ld_remote(&part.l[hw], s, tok);
      os[s] = dec_ld_remote(&part.o[hw][threadIdx.x], s, tok);
    }
#pragma unroll
    for (int s = 0; s < kSplit; ++s) M = fmaxf(M, ms[s]);
    float Lsum = 0.f, O = 0.f;
#pragma unroll
    for (int s = 0; s < kSplit; ++s) {
      const float wgt = ms[s] == -INFINITY ? 0.f : ex2_approx(ms[s] - M);
      Lsum += wgt * ls[s];
      O += wgt * os[s];
    }
    const int h = g * grp + hw;
    o[(size_t)b * Hq * kHd + (size_t)h * kHd + threadIdx.x] = __float2bfloat16_rn(O / Lsum);
  }
  (void)dec_cluster_sync();  // peers' shared memory stays valid until every merge is done
}

// Streaming decode attention for bf16, head_dim 64, up to 8 query heads per kv
// head, when there are enough (kv head, batch row) pairs to give every SM one:
// one CTA per pair walks all min(pos + 1, w) valid ring slots in 64-slot tiles
// that a producer warp streams through a TMA ring (no split, no merge across
// CTAs).  Four consumer warps each take 16 slots of every tile and keep their
// own online-softmax state (running max, sum, O) for the group's heads as rows
// of m16n8k16 products (rows 8..15 padding): S = Q K^T, P = exp2(S - m), O +=
// P V; the four partial states are merged in shared memory at the end.  K and
// V tiles land 128-byte swizzled (16-byte piece j of row r at piece j ^ (r % 8)).
constexpr int kStTile = 64;
constexpr int kStStages = 6;
constexpr int kStWarps = 4;
constexpr int kStThreads = (kStWarps + 1) * 32;

struct StSmem {
  bf16 K[kStStages][kStTile * kHd];
  bf16 V[kStStages][kStTile * kHd];
  uint64_t full[kStStages], empty[kStStages];
  float wm[kStWarps][8], wl[kStWarps][8];
  float wo[kStWarps][8][kHd];
};

__device__ __forceinline__ uint32_t st_swz(int row, int col) {  // byte offset of element (row, col) of a tile
  return (uint32_t)(row * 128 + ((((col >> 3) ^ row) & 7) << 4) + ((col & 7) << 1));
}

__global__ void __launch_bounds__(kStThreads, 1)
    attn_decode_stream_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                              const bf16* __restrict__ qkv, int64_t ld, const int64_t* __restrict__ pos,
                              bf16* __restrict__ o, int Hq, int Hkv, int window, float scale_log2, int* err) {
  extern __shared__ __align__(1024) unsigned char st_raw[];
  StSmem& S = *reinterpret_cast<StSmem*>(st_raw + smem_align_pad(st_raw, 1024));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, b = blockIdx.y;
  const int grp = Hq / Hkv;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStStages; ++i) {
      mbar_init(&S.full[i], 1);
      mbar_init(&S.empty[i], kStWarps);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  __syncthreads();
  pdl_wait();  // the position, the query and this step's ring entry come from earlier kernels
  pdl_trigger();
  const int64_t P = pos[b];
  const int nvalid = (int)(P + 1 < window ? P + 1 : window);
  const int ntile = nvalid > 0 ? (nvalid + kStTile - 1) / kStTile : 0;
  const int qr = lane >> 2, qc = 2 * (lane & 3);
  float m_run = -INFINITY, l_run = 0.f;
  float oacc[kHd / 8][4];
#pragma unroll
  for (int nt = 0; nt < kHd / 8; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) oacc[nt][i] = 0.f;

  if (warp == kStWarps) {
    // ---- producer: K and V tiles of slots [64t, 64t + 64) of ring row b
    if (lane == 0) {
      const int z0 = b * window;
      int issued = 0;
      for (int t = 0; t < ntile; ++t) {
        const int s = t % kStStages;
        if (t >= kStStages && !mbar_wait(&S.empty[s], ((t / kStStages) & 1) ^ 1, err)) break;
        mbar_arrive_expect_tx(&S.full[s], 2u * kStTile * kHd * 2u);
        tma_load_3d(S.K[s], &tmK, &S.full[s], 0, g, z0 + t * kStTile);
        tma_load_3d(S.V[s], &tmV, &S.full[s], 0, g, z0 + t * kStTile);
        issued = t + 1;
      }
      // the CTA leaves only once its own copies have landed (after a timeout too)
      for (int t = issued > kStStages ? issued - kStStages : 0; t < issued; ++t)
        (void)mbar_wait(&S.full[t % kStStages], (t / kStStages) & 1, err);
    }
  } else {
    // ---- consumers: Q fragments (A operand, rows = heads), then the tiles
    uint32_t qa[kHd / 16][4];
#pragma unroll
    for (int ks = 0; ks < kHd / 16; ++ks) {
      qa[ks][1] = qa[ks][3] = 0u;
      qa[ks][0] = qa[ks][2] = 0u;
      if (qr < grp) {
        const bf16* qrow = qkv + (size_t)b * ld + (size_t)(g * grp + qr) * kHd + ks * 16 + qc;
        qa[ks][0] = *reinterpret_cast<const uint32_t*>(qrow);
        qa[ks][2] = *reinterpret_cast<const uint32_t*>(qrow + 8);
      }
    }
    const int kb = warp * 16;  // this warp's slots within a tile
    for (int t = 0; t < ntile; ++t) {
      const int s = t % kStStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&S.full[s], (t / kStStages) & 1, err))) break;
      const unsigned char* Kt = reinterpret_cast<const unsigned char*>(S.K[s]);
      const unsigned char* Vt = reinterpret_cast<const unsigned char*>(S.V[s]);
      float sacc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int i = 0; i < 4; ++i) sacc[nt][i] = 0.f;
        const int key = kb + nt * 8 + qr;
#pragma unroll
        for (int ks = 0; ks < kHd / 16; ++ks) {
          const uint32_t b0 = *reinterpret_cast<const uint32_t*>(Kt + st_swz(key, ks * 16 + qc));
          const uint32_t b1 = *reinterpret_cast<const uint32_t*>(Kt + st_swz(key, ks * 16 + 8 + qc));
          mma_bf16_16816(sacc[nt], qa[ks], b0, b1);
        }
      }
      // scale into the log2 domain, mask slots past the valid ones, online softmax per head (row qr)
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int slot = t * kStTile + kb + nt * 8 + qc + c;
          const float v = slot < nvalid ? sacc[nt][c] * scale_log2 : -INFINITY;
          sacc[nt][c] = v;
          mx = fmaxf(mx, v);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mnew = fmaxf(m_run, mx);
      const float msub = mnew == -INFINITY ? 0.f : mnew;
      const float corr = ex2_approx(m_run - msub);
      m_run = mnew;
      uint32_t pa[4];
      float ps = 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const float p0 = ex2_approx(sacc[nt][0] - msub), p1 = ex2_approx(sacc[nt][1] - msub);
        ps += p0 + p1;
        pa[nt ? 2 : 0] = pack_bf16x2(p0, p1);
        pa[nt ? 3 : 1] = 0u;
      }
      l_run = l_run * corr + ps;
#pragma unroll
      for (int nt = 0; nt < kHd / 8; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) oacc[nt][i] *= corr;
      // O += P V over the warp's 16 slots (V rows through ldmatrix.trans)
#pragma unroll
      for (int np = 0; np < kHd / 16; ++np) {
        uint32_t vb[4];
        const int key = kb + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int dim = np * 16 + 8 * (lane >> 4);
        ldmatrix_x4_trans(vb, Vt + st_swz(key, dim));
        mma_bf16_16816(oacc[2 * np], pa, vb[0], vb[1]);
        mma_bf16_16816(oacc[2 * np + 1], pa, vb[2], vb[3]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[s]);
    }
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    if ((lane & 3) == 0) {
      S.wm[warp][qr] = m_run;
      S.wl[warp][qr] = l_run;
    }
#pragma unroll
    for (int nt = 0; nt < kHd / 8; ++nt) {
      S.wo[warp][qr][nt * 8 + qc] = oacc[nt][0];
      S.wo[warp][qr][nt * 8 + qc + 1] = oacc[nt][1];
    }
  }
  __syncthreads();
  // ---- merge the four warps' states per head
  for (int e = threadIdx.x; e < grp * kHd; e += kStThreads) {
    const int h = e / kHd, d = e % kHd;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kStWarps; ++w) M = fmaxf(M, S.wm[w][h]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kStWarps; ++w) {
      const float mw = S.wm[w][h];
      const float wgt = mw == -INFINITY ? 0.f : ex2_approx(mw - M);
      L += wgt * S.wl[w][h];
      O += wgt * S.wo[w][h][d];
    }
    o[(size_t)b * Hq * kHd + (size_t)(g * grp + h) * kHd + d] = __float2bfloat16_rn(O / L);
  }
}

// Long caches (more than kSplit * kSliceMax slots, e.g. a full-attention KV
// cache): one CTA per 256-slot slice, grid (cache / 256, Hkv, B); CTAs past the
// valid slots publish an empty partial.  Partials go to `ws`, and
// attn_decode_merge_kernel combines them (flash-decoding).
__global__ void __launch_bounds__(256, 1)
    attn_decode_long_kernel(const bf16* __restrict__ qkv, int64_t ld, const int64_t* __restrict__ pos,
                            const bf16* __restrict__ k_ring, const bf16* __restrict__ v_ring,
                            DecPart* __restrict__ ws, int Hq, int Hkv, int window, float scale_log2, int* err) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) unsigned char dec_dyn[];
  bf16* Ks = reinterpret_cast<bf16*>(dec_dyn);
  bf16* Vs = Ks + kSliceMax * kKvPad;
  __shared__ DecPart part;
  __shared__ float wm[8][8], wl[8][8];
  __shared__ float wo[8][8][kHd];
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int grp = Hq / Hkv;
  const int64_t P = pos[b];
  const int nvalid = (int)(P + 1 < window ? P + 1 : window);
  const int s0 = split * kSliceMax;
  int n = max(0, min(nvalid, s0 + kSliceMax) - s0);
  if (!SAMBA_DCHECK(err, n == 0 || s0 + n <= window)) n = 0;
  DecPart* dst = ws + ((size_t)b * Hkv + g) * gridDim.x + split;
  if (n == 0) {  // block-uniform: past the valid slots
    if (threadIdx.x < 8) {
      dst->m[threadIdx.x] = -INFINITY;
      dst->l[threadIdx.x] = 0.f;
    }
    return;
  }
  dec_slice_partial(qkv, ld, k_ring, v_ring, Hkv, grp, window, g, b, s0, n, (n + 31) & ~31, scale_log2, Ks, Vs,
                    part, wm, wl, wo);
  __syncthreads();
  for (int e = threadIdx.x; e < grp * kHd; e += 256) dst->o[e / kHd][e % kHd] = part.o[e / kHd][e % kHd];
  if (threadIdx.x < grp) {
    dst->m[threadIdx.x] = part.m[threadIdx.x];
    dst->l[threadIdx.x] = part.l[threadIdx.x];
  }
}

// o[b, h] = merge over the splits of (m, l, O) of query head h: one CTA of 64
// threads (head dims) per (query head, batch row).
__global__ void attn_decode_merge_kernel(const DecPart* __restrict__ ws, bf16* __restrict__ o, int Hq, int Hkv,
                                         int nsplit) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int grp = Hq / Hkv, g = h / grp, hw = h % grp;
  const DecPart* src = ws + ((size_t)b * Hkv + g) * nsplit;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, src[s].m[hw]);
  float Lsum = 0.f, O = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float ms = src[s].m[hw];
    if (ms == -INFINITY) continue;
    const float wgt = ex2_approx(ms - M);
    Lsum += wgt * src[s].l[hw];
    O += wgt * src[s].o[hw][d];
  }
  o[(size_t)b * Hq * kHd + (size_t)h * kHd + d] = __float2bfloat16_rn(O / Lsum);
}

__global__ void pos_add_kernel(int64_t* pos, int B, int64_t inc, int set) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < B) pos[i] = set ? inc : pos[i] + inc;
}

__global__ void pos_check_set_kernel(int64_t* pos, int B, int64_t expect, int64_t value, int* err) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < B) {
    if (pos[i] != expect) raise_error(err, kErrDevice);
    pos[i] = value;
  }
}

// prefill -> ring: chunk tokens max(0, L-w) .. L-1 (absolute position pos0 + t) into slot (pos0 + t) mod w
template <typename T>
__global__ void ring_fill_kernel(const T* __restrict__ qkv, int64_t ld, int k_off, int v_off, T* __restrict__ k_ring,
                                 T* __restrict__ v_ring, int L, int64_t pos0, int window, int kvw, int* err) {
  const int j = blockIdx.x;  // 0 .. min(L, w)-1
  const int b = blockIdx.y;
  const int n = min(L, window);
  if (j >= n) return;
  const int p = L - n + j;
  const int slot = (int)((pos0 + p) % window);
  if (!SAMBA_DCHECK(err, p >= 0 && p < L && slot >= 0 && slot < window)) return;
  const T* src = qkv + ((size_t)b * L + p) * ld;
  T* kd = k_ring + ((size_t)b * window + slot) * kvw;
  T* vd = v_ring + ((size_t)b * window + slot) * kvw;
  for (int i = threadIdx.x; i < kvw; i += blockDim.x) {
    kd[i] = src[k_off + i];
    vd[i] = src[v_off + i];
  }
}

// Row j of kx/vx: j < h is the ring entry of position pos0 - h + j, else chunk token j - h.
// Rows are copied as 16-byte pieces (`vec` per row); dtype-agnostic.
__global__ void kv_window_gather_kernel(const char* __restrict__ qkv, int64_t ld_b, int64_t k_off_b,
                                        int64_t v_off_b, const char* __restrict__ k_ring,
                                        const char* __restrict__ v_ring, char* __restrict__ kx,
                                        char* __restrict__ vx, int L, int64_t pos0, int h, int window, int vec,
                                        int* err) {
  const int j = blockIdx.x;
  const int b = blockIdx.y;
  const int64_t row_b = (int64_t)vec * 16;
  const char *ks, *vs;
  if (j < h) {
    const int slot = (int)((pos0 - h + j) % window);
    if (!SAMBA_DCHECK(err, pos0 - h + j >= 0 && slot < window)) return;
    ks = k_ring + ((int64_t)b * window + slot) * row_b;
    vs = v_ring + ((int64_t)b * window + slot) * row_b;
  } else {
    const char* src = qkv + ((int64_t)b * L + (j - h)) * ld_b;
    ks = src + k_off_b;
    vs = src + v_off_b;
  }
  char* kd = kx + ((int64_t)b * (h + L) + j) * row_b;
  char* vd = vx + ((int64_t)b * (h + L) + j) * row_b;
  for (int i = threadIdx.x; i < vec; i += blockDim.x) {
    reinterpret_cast<uint4*>(kd)[i] = reinterpret_cast<const uint4*>(ks)[i];
    reinterpret_cast<uint4*>(vd)[i] = reinterpret_cast<const uint4*>(vs)[i];
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
  if (B > kMaxGridYZ || (int64_t)B * D > INT32_MAX) return SAMBA_ERR_UNSUPPORTED;
  if (k < 2 || k > 8) return SAMBA_ERR_UNSUPPORTED;
  const int n = B * D;
  cudaError_t e;
  SAMBA_DT_DISPATCH(dt,
                    (e = launch_k(conv_step_kernel<bf16>, dim3((n + 255) / 256), dim3(256), 0, st, true,
                                  (const bf16*)hz, ld_hz, w, bias, (bf16*)state, (bf16*)u, B, D, k)),
                    (e = launch_k(conv_step_kernel<float>, dim3((n + 255) / 256), dim3(256), 0, st, true,
                                  (const float*)hz, ld_hz, w, bias, (float*)state, (float*)u, B, D, k)));
  if (e != cudaSuccess) return note_cuda_failure("decode kernel launch", e);
  return SAMBA_OK;
}

samba_status launch_scan_step(const void* u, const void* dlt, const void* z, int64_t ld_z, const void* xdbl,
                              int64_t ld_x, int r_off, const float* A_log, const float* Dskip, float* ssm, void* y,
                              int B, int D, samba_dtype dt, cudaStream_t st) {
  if (B > kMaxGridYZ || (int64_t)B * D > INT32_MAX) return SAMBA_ERR_UNSUPPORTED;
  if (!aligned16(A_log) || !aligned16(ssm)) return SAMBA_ERR_UNSUPPORTED;  // 16-byte pieces of A and the state
  const int n = B * D;
  cudaError_t e;
  SAMBA_DT_DISPATCH(dt,
                    (e = launch_k(scan_step_kernel<bf16>, dim3((unsigned)((4 * (int64_t)n + 127) / 128)), dim3(128), 0, st, true,
                                  (const bf16*)u, (const bf16*)dlt, (const bf16*)z, ld_z, (const bf16*)xdbl, ld_x,
                                  r_off, A_log, Dskip, ssm, (bf16*)y, B, D)),
                    (e = launch_k(scan_step_kernel<float>, dim3((unsigned)((4 * (int64_t)n + 127) / 128)), dim3(128), 0, st, true,
                                  (const float*)u, (const float*)dlt, (const float*)z, ld_z, (const float*)xdbl, ld_x,
                                  r_off, A_log, Dskip, ssm, (float*)y, B, D)));
  if (e != cudaSuccess) return note_cuda_failure("decode kernel launch", e);
  return SAMBA_OK;
}

bool scan_step_dt_supported(int R, int D, int64_t ld_x, samba_dtype dt) {
  const int vec = dt == SAMBA_BF16 ? 8 : 4;
  return R >= 8 && R <= kSdMaxR && R % 8 == 0 && D % kSdCh == 0 && ld_x % vec == 0;
}

samba_status launch_scan_step_dt(const void* u, const void* z, int64_t ld_z, const void* xdbl, int64_t ld_x, int R,
                                 const void* W_dt, const float* dt_bias, const float* A_log, const float* Dskip,
                                 float* ssm, void* y, int B, int D, samba_dtype dt, cudaStream_t st) {
  if (!scan_step_dt_supported(R, D, ld_x, dt)) return SAMBA_ERR_UNSUPPORTED;
  if (!aligned16(xdbl) || !aligned16(W_dt) || !aligned16(ssm) || !aligned16(A_log)) return SAMBA_ERR_UNSUPPORTED;
  const int es = dt == SAMBA_BF16 ? 2 : 4;
  const size_t smem = (size_t)(kSdCh + kSdRows) * (R + 16 / es) * es;
  const dim3 grid(D / kSdCh, (B + kSdRows - 1) / kSdRows);
  if (grid.y > (unsigned)kMaxGridYZ) return SAMBA_ERR_UNSUPPORTED;
  constexpr size_t kMaxSmem = (size_t)(kSdCh + kSdRows) * (kSdMaxR + 4) * 4;
  if (!ensure_smem_attr(scan_step_dt_kernel<bf16>, kMaxSmem) || !ensure_smem_attr(scan_step_dt_kernel<float>, kMaxSmem))
    return SAMBA_ERR_CUDA;
  cudaError_t e;
  SAMBA_DT_DISPATCH(dt,
                    (e = launch_k(scan_step_dt_kernel<bf16>, grid, dim3(kSdWarps * 32), smem, st, true, (const bf16*)u,
                                  (const bf16*)z, ld_z, (const bf16*)xdbl, ld_x, R, (const bf16*)W_dt, dt_bias, A_log,
                                  Dskip, ssm, (bf16*)y, B, D)),
                    (e = launch_k(scan_step_dt_kernel<float>, grid, dim3(kSdWarps * 32), smem, st, true, (const float*)u,
                                  (const float*)z, ld_z, (const float*)xdbl, ld_x, R, (const float*)W_dt, dt_bias,
                                  A_log, Dskip, ssm, (float*)y, B, D)));
  if (e != cudaSuccess) return note_cuda_failure("decode kernel launch", e);
  return SAMBA_OK;
}

samba_status launch_ring_write(const void* qkv, int64_t ld, int k_off, int v_off, const int64_t* pos, void* k_ring,
                               void* v_ring, int B, int window, int kvw, samba_dtype dt, cudaStream_t st) {
  cudaError_t e;
  SAMBA_DT_DISPATCH(dt,
                    (e = launch_k(ring_write_kernel<bf16>, dim3(B), dim3(128), 0, st, true, (const bf16*)qkv, ld,
                                  k_off, v_off, pos, (bf16*)k_ring, (bf16*)v_ring, window, kvw,
                                  device_error_word())),
                    (e = launch_k(ring_write_kernel<float>, dim3(B), dim3(128), 0, st, true, (const float*)qkv, ld,
                                  k_off, v_off, pos, (float*)k_ring, (float*)v_ring, window, kvw,
                                  device_error_word())));
  if (e != cudaSuccess) return note_cuda_failure("decode kernel launch", e);
  return SAMBA_OK;
}

size_t attn_decode_workspace_bytes(int B, int Hkv, int window) {
  if (window <= kSplit * kSliceMax) return 0;
  return (size_t)B * Hkv * ((window + kSliceMax - 1) / kSliceMax) * sizeof(DecPart);
}

samba_status launch_attn_decode(const void* qkv, int64_t ld, const int64_t* pos, const void* k_ring,
                                const void* v_ring, void* o, int B, int Hq, int Hkv, int hd, int window, float scale,
                                samba_dtype dt, cudaStream_t st, void* ws, size_t ws_bytes) {
  if (B > kMaxGridYZ) return SAMBA_ERR_UNSUPPORTED;
  if (hd > 32 * kDecMaxDpl) return SAMBA_ERR_UNSUPPORTED;
  if (dt == SAMBA_BF16 && hd == kHd && Hq / Hkv <= 8 && window <= 4096 && ld % 8 == 0 &&
      (int64_t)B * Hkv >= (int64_t)num_sms() * 3 / 4 && aligned16(k_ring) && aligned16(v_ring)) {
    // enough (kv head, row) pairs for every SM: one streaming CTA per pair
    CUtensorMap tmK, tmV;
    const uint64_t dims[3] = {(uint64_t)kHd, (uint64_t)Hkv, (uint64_t)B * (uint64_t)window};
    const uint64_t strides[2] = {(uint64_t)kHd, (uint64_t)Hkv * kHd};
    const uint32_t box[3] = {(uint32_t)kHd, 1u, (uint32_t)kStTile};
    if (!make_tmap(&tmK, k_ring, SAMBA_BF16, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap(&tmV, v_ring, SAMBA_BF16, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return SAMBA_ERR_CUDA;
    const size_t smem = sizeof(StSmem) + 1024;
    if (!ensure_smem_attr(attn_decode_stream_kernel, smem)) return SAMBA_ERR_CUDA;
    const cudaError_t e = launch_k(attn_decode_stream_kernel, dim3(Hkv, B), dim3(kStThreads), smem, st, true, tmK,
                                   tmV, (const bf16*)qkv, ld, pos, (bf16*)o, Hq, Hkv, window,
                                   scale * 1.4426950408889634f, device_error_word());
    if (e != cudaSuccess) return note_cuda_failure("decode attention launch", e);
    return SAMBA_OK;
  }
  if (dt == SAMBA_BF16 && hd == kHd && Hq / Hkv <= 8 && window > kSplit * kSliceMax && ld % 8 == 0) {
    const int nsplit = (window + kSliceMax - 1) / kSliceMax;
    if (!ws || ws_bytes < attn_decode_workspace_bytes(B, Hkv, window) || !aligned16(ws))
      return SAMBA_ERR_INVALID_ARG;
    const size_t smem = 2 * kSliceMax * kKvPad * sizeof(bf16);
    if (!ensure_smem_attr(attn_decode_long_kernel, smem)) return SAMBA_ERR_CUDA;
    if (launch_k(attn_decode_long_kernel, dim3(nsplit, Hkv, B), dim3(256), smem, st, true, (const bf16*)qkv, ld,
                 pos, (const bf16*)k_ring, (const bf16*)v_ring, (DecPart*)ws, Hq, Hkv, window,
                 scale * 1.4426950408889634f, device_error_word()) != cudaSuccess)
      return SAMBA_ERR_CUDA;
    if (launch_k(attn_decode_merge_kernel, dim3(Hq, B), dim3(kHd), 0, st, true, (const DecPart*)ws, (bf16*)o, Hq,
                 Hkv, nsplit) != cudaSuccess)
      return SAMBA_ERR_CUDA;
    return SAMBA_OK;
  }
  if (dt == SAMBA_BF16 && hd == kHd && Hq / Hkv <= 8 && window <= kSplit * kSliceMax && ld % 8 == 0) {
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(kSplit, Hkv, B);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = 2 * kSliceMax * kKvPad * sizeof(bf16);
    cfg.stream = st;
    if (!ensure_smem_attr(attn_decode_split_kernel, cfg.dynamicSmemBytes)) return SAMBA_ERR_CUDA;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kSplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, attn_decode_split_kernel, (const bf16*)qkv, ld, pos,
                                             (const bf16*)k_ring, (const bf16*)v_ring, (bf16*)o, Hq, Hkv, window,
                                             scale * 1.4426950408889634f, device_error_word());
    if (e != cudaSuccess) return note_cuda_failure("cudaLaunchKernelEx (decode attention cluster)", e);
    SAMBA_CHECK_LAUNCH();
    return SAMBA_OK;
  }
  const int grp = Hq / Hkv;
  const int threads = ((grp * 32) < 128 ? 128 : grp * 32);
  if (threads > 1024) return SAMBA_ERR_UNSUPPORTED;
  const size_t smem = 2 * kDecKB * (hd + 1) * sizeof(float);
  // the limit is raised once to the largest head_dim's need (131.6 KB at 256),
  // so that a smaller head_dim first does not leave it too low for a larger one
  constexpr size_t kMaxSmem = 2 * kDecKB * (32 * kDecMaxDpl + 1) * sizeof(float);
  if (!ensure_smem_attr(attn_decode_kernel<bf16>, kMaxSmem) || !ensure_smem_attr(attn_decode_kernel<float>, kMaxSmem))
    return SAMBA_ERR_CUDA;
  dim3 grid(Hkv, B);
  cudaError_t e;
  SAMBA_DT_DISPATCH(dt,
                    (e = launch_k(attn_decode_kernel<bf16>, grid, dim3(threads), smem, st, true, (const bf16*)qkv, ld,
                                  pos, (const bf16*)k_ring, (const bf16*)v_ring, (bf16*)o, Hq, Hkv, hd, window,
                                  scale)),
                    (e = launch_k(attn_decode_kernel<float>, grid, dim3(threads), smem, st, true, (const float*)qkv,
                                  ld, pos, (const float*)k_ring, (const float*)v_ring, (float*)o, Hq, Hkv, hd, window,
                                  scale)));
  if (e != cudaSuccess) return note_cuda_failure("decode kernel launch", e);
  return SAMBA_OK;
}

samba_status launch_pos_update(int64_t* pos, int B, int64_t value, bool set, cudaStream_t st, bool pdl) {
  if (launch_k(pos_add_kernel, dim3((B + 127) / 128), dim3(128), 0, st, pdl, pos, B, value, set ? 1 : 0) !=
      cudaSuccess)
    return SAMBA_ERR_CUDA;
  return SAMBA_OK;
}

samba_status launch_ring_fill(const void* qkv, int64_t ld, int k_off, int v_off, void* k_ring, void* v_ring, int B,
                              int L, int64_t pos0, int window, int kvw, samba_dtype dt, cudaStream_t st) {
  if (B > kMaxGridYZ) return SAMBA_ERR_UNSUPPORTED;
  const int n = L < window ? L : window;
  if (n == 0) return SAMBA_OK;
  dim3 grid(n, B);
  SAMBA_DT_DISPATCH(dt,
                    (ring_fill_kernel<bf16><<<grid, 128, 0, st>>>((const bf16*)qkv, ld, k_off, v_off, (bf16*)k_ring,
                                                                  (bf16*)v_ring, L, pos0, window, kvw,
                                                                  device_error_word())),
                    (ring_fill_kernel<float><<<grid, 128, 0, st>>>((const float*)qkv, ld, k_off, v_off,
                                                                   (float*)k_ring, (float*)v_ring, L, pos0, window,
                                                                   kvw, device_error_word())));
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

samba_status launch_kv_window_gather(const void* qkv, int64_t ld, int k_off, int v_off, const void* k_ring,
                                     const void* v_ring, void* kx, void* vx, int B, int L, int64_t pos0, int h,
                                     int window, int kvw, samba_dtype dt, cudaStream_t st) {
  if (B > kMaxGridYZ) return SAMBA_ERR_UNSUPPORTED;
  const size_t es = dtype_size(dt);
  const int vec = (int)(kvw * es / 16);  // 16-byte pieces per row
  if ((kvw * es) % 16 || (ld * es) % 16 || (k_off * es) % 16 || (v_off * es) % 16 || h < 0 || h > pos0 ||
      h >= window + 1)
    return SAMBA_ERR_UNSUPPORTED;
  if (h + L == 0) return SAMBA_OK;
  dim3 grid(h + L, B);
  kv_window_gather_kernel<<<grid, 64, 0, st>>>((const char*)qkv, ld * es, k_off * es, v_off * es,
                                               (const char*)k_ring, (const char*)v_ring, (char*)kx, (char*)vx, L,
                                               pos0, h, window, vec, device_error_word());
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

samba_status launch_pos_check_set(int64_t* pos, int B, int64_t expect, int64_t value, cudaStream_t st) {
  pos_check_set_kernel<<<(B + 127) / 128, 128, 0, st>>>(pos, B, expect, value, device_error_word());
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

}  // namespace samba
