// Dense projections out = epilogue(A W^T) of the Samba block: Mamba in/x/dt/out
// projections, the SwiGLU MLP and the attention Q/K/V/O projections
// [Samba 3.4: eqs. H = X W_in, Delta = Softplus(U W_r W_q + b), B = U W_b,
// C = U W_c, O = (Y (.) SiLU(X W_g)) W_out, "SwiGLU Formulation"].
//
// Two kernels:
//  * gemm_tc: bf16 operands, fp32 accumulation on the 5th-generation tensor
//    cores.  Persistent, warp specialised (warp 0: TMA producer, warp 1: MMA
//    issuer + TMEM owner, warps 2..: epilogue, two per TMEM lane quadrant, four
//    for the softplus instance).  A 4-stage ring of 128x64 A and
//    up to 256x64 B tiles in 128-byte-swizzled shared memory feeds
//    tcgen05.mma (M=128, N<=256, K=16) issued by one thread into a double
//    buffered 2x256-column TMEM accumulator, so the epilogue of one tile
//    overlaps the main loop of the next.  Epilogues (residual add, SwiGLU,
//    softplus+bias, RoPE) are fused on the TMEM read-out; each epilogue warp
//    writes its 32 rows x 32 columns through a shared-memory staging buffer
//    and a TMA store (RoPE tiles store directly).
//  * gemm_simt: CUDA-core fp32 FMA tiles, used for fp32 data (no TF32: its
//    ~1e-3 error would break the fp32 tolerance) and for shapes the tensor-core
//    kernel does not take.
#include <stdlib.h>

#include <atomic>
#include <mutex>
#include <vector>

#define SAMBA_TU_ID 4  // site id of this file in debug-check reports
#include "common.cuh"
#include "kernels.h"

namespace samba {

namespace {

// ---------------------------------------------------------------------------
// Shared epilogue pieces
// ---------------------------------------------------------------------------
__device__ __forceinline__ int64_t rope_position(const GemmArgs& a, int64_t row) {
  return a.pos_dev ? a.pos_dev[row] : a.pos0 + row % a.seq_len;
}
// (cos, sin) of p * theta_i from the three-level fp64-built table
__device__ __forceinline__ float2 rope_cs(const float2* __restrict__ tab, int half, int64_t p, int i) {
  const float2 c0 = tab[(0 * kRopeRadix + (p & 1023)) * half + i];
  const float2 c1 = tab[(1 * kRopeRadix + ((p >> 10) & 1023)) * half + i];
  const float2 c2 = tab[(2 * kRopeRadix + ((p >> 20) & 1023)) * half + i];
  const float cr = c0.x * c1.x - c0.y * c1.y, sr = c0.x * c1.y + c0.y * c1.x;
  return make_float2(cr * c2.x - sr * c2.y, cr * c2.y + sr * c2.x);
}

// (cos, sin) of pairs i0 .. i0+15 at position p: the three table rows read as
// 16-byte pieces (i0 a multiple of 16)
__device__ __forceinline__ void rope_cs16(const float2* __restrict__ tab, int half, int64_t p, int i0, float2 (&cs)[16]) {
  const float4* t0 = reinterpret_cast<const float4*>(tab + (0 * kRopeRadix + (p & 1023)) * half + i0);
  const float4* t1 = reinterpret_cast<const float4*>(tab + (1 * kRopeRadix + ((p >> 10) & 1023)) * half + i0);
  const float4* t2 = reinterpret_cast<const float4*>(tab + (2 * kRopeRadix + ((p >> 20) & 1023)) * half + i0);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float4 a = t0[k], b = t1[k], c = t2[k];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float ax = e ? a.z : a.x, ay = e ? a.w : a.y;
      const float bx = e ? b.z : b.x, by = e ? b.w : b.y;
      const float cx = e ? c.z : c.x, cy = e ? c.w : c.y;
      const float cr = ax * bx - ay * by, sr = ax * by + ay * bx;
      cs[2 * k + e] = make_float2(cr * cx - sr * cy, cr * cy + sr * cx);
    }
  }
}

template <typename T>
__device__ __forceinline__ float silu_t(float g) {
  if constexpr (sizeof(T) == 4) return g * sigmoid_acc(g);
  else return g * sigmoid_fast(g);
}
template <typename T>
__device__ __forceinline__ float softplus_t(float x) {
  if constexpr (sizeof(T) == 4) return softplus_acc(x);
  else return softplus_1x(x);
}

__device__ __forceinline__ void seg_lookup(const GemmArgs& a, int n, int& s, int& row) {
  int base = 0;
  s = 0;
  while (s < a.nseg - 1 && n >= base + a.seg[s].n) {
    base += a.seg[s].n;
    ++s;
  }
  row = n - base;
}

// ===========================================================================
// CUDA-core kernel: 64x64 tile, 256 threads x (4x4) outputs, BK = 16
// ===========================================================================
constexpr int SB_M = 64, SB_N = 64, SB_K = 16;

template <typename T, int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const GemmArgs a) {
  __shared__ float As[SB_K][SB_M + 4];
  __shared__ float Bs[SB_K][SB_N + 4];
  __shared__ float B2s[EPI == kEpiSwiglu ? SB_K : 1][SB_N + 4];
  __shared__ float Cs[SB_M][SB_N + 1];
  const int tid = threadIdx.x;
  const int64_t m0 = (int64_t)blockIdx.y * SB_M;
  const int n0 = blockIdx.x * SB_N;
  const T* A = (const T*)a.A;
  const int ty = tid / 16, tx = tid % 16;
  float acc[4][4] = {}, acc2[4][4] = {};

  // loader coordinates: row lr (0..63), k offset lk (0,4,8,12)
  const int lr = tid / 4, lk = (tid % 4) * 4;
  const int64_t arow = m0 + lr;
  const int bn = n0 + lr;
  int bseg = 0, brow = 0;
  if (bn < a.N) seg_lookup(a, bn, bseg, brow);
  const T* Wrow = bn < a.N ? (const T*)a.seg[bseg].W + (size_t)brow * a.K : nullptr;
  const T* W2row = (EPI == kEpiSwiglu && bn < a.N) ? (const T*)a.seg[bseg].W2 + (size_t)brow * a.K : nullptr;

  for (int k0 = 0; k0 < a.K; k0 += SB_K) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int k = k0 + lk + j;
      As[lk + j][lr] = (arow < a.M && k < a.K) ? Elt<T>::to_f(A[arow * a.lda + k]) : 0.f;
      Bs[lk + j][lr] = (Wrow && k < a.K) ? Elt<T>::to_f(Wrow[k]) : 0.f;
      if (EPI == kEpiSwiglu) B2s[lk + j][lr] = (W2row && k < a.K) ? Elt<T>::to_f(W2row[k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SB_K; ++kk) {
      float av[4], bv[4], b2v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = As[kk][ty * 4 + i];
        bv[i] = Bs[kk][tx * 4 + i];
        if (EPI == kEpiSwiglu) b2v[i] = B2s[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
          if (EPI == kEpiSwiglu) acc2[i][j] = fmaf(av[i], b2v[j], acc2[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
      Cs[ty * 4 + i][tx * 4 + j] = EPI == kEpiSwiglu ? acc[i][j] * silu_t<T>(acc2[i][j]) : acc[i][j];
  __syncthreads();

  T* out = (T*)a.out;
  for (int e = tid; e < SB_M * SB_N; e += 256) {
    const int r = e / SB_N, c = e % SB_N;
    const int64_t row = m0 + r;
    const int col = n0 + c;
    if (row >= a.M || col >= a.N) continue;
    float v = Cs[r][c];
    if (EPI == kEpiResid) {
      if (a.tap) ((T*)a.tap)[row * a.ldt + col] = Elt<T>::from_f(v);
      v += Elt<T>::to_f(((const T*)a.resid)[row * a.ldr + col]);
    } else if (EPI == kEpiSoftplus) {
      v = softplus_t<T>(v + a.bias[col]);
    } else if (EPI == kEpiRope) {
      if (col < a.rope_cols) {
        const int hd = a.head_dim, half = hd / 2;
        const int j = col % hd;
        const int cb = c - j;  // head start within the tile
        const int i = j % half;
        const float x1 = Cs[r][cb + i], x2 = Cs[r][cb + i + half];
        const float2 cs = rope_cs(a.rope_tab, half, rope_position(a, row), i);
        v = j < half ? x1 * cs.x - x2 * cs.y : x2 * cs.x + x1 * cs.y;
      }
    }
    out[row * a.ldo + col] = Elt<T>::from_f(v);
  }
}

template <typename T>
samba_status simt_dispatch(const GemmArgs& a, cudaStream_t st) {
  if ((a.M + SB_M - 1) / SB_M > kMaxGridYZ) return SAMBA_ERR_UNSUPPORTED;
  dim3 grid((a.N + SB_N - 1) / SB_N, (unsigned)((a.M + SB_M - 1) / SB_M));
  switch (a.epi) {
    case kEpiNone: gemm_simt_kernel<T, kEpiNone><<<grid, 256, 0, st>>>(a); break;
    case kEpiResid: gemm_simt_kernel<T, kEpiResid><<<grid, 256, 0, st>>>(a); break;
    case kEpiSwiglu: gemm_simt_kernel<T, kEpiSwiglu><<<grid, 256, 0, st>>>(a); break;
    case kEpiSoftplus: gemm_simt_kernel<T, kEpiSoftplus><<<grid, 256, 0, st>>>(a); break;
    case kEpiRope: gemm_simt_kernel<T, kEpiRope><<<grid, 256, 0, st>>>(a); break;
    default: return SAMBA_ERR_INVALID_ARG;
  }
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

// ===========================================================================
// tcgen05 kernel
// ===========================================================================
constexpr int TC_BM = 128, TC_BK = 64, TC_STAGES = 4, TC_MAXN = 256;
// Epilogue warps per TMEM lane quadrant (column parts).  Two keep up with the
// mainloop of every projection with K >= 2048; the dt projection (K = 128,
// softplus) has almost no mainloop, so its epilogue sets the pace and gets four.
template <int EPI>
struct TcEpi {
  static constexpr int parts = EPI == kEpiSoftplus ? 4 : 2;
  static constexpr int warps = 4 * parts;
  static constexpr int threads = 64 + 32 * warps;
};
constexpr uint32_t TC_A_BYTES = TC_BM * TC_BK * 2;

// Output staging of the epilogue warps: each warp's 32 rows x 32 columns of
// bf16 (64-byte rows, 16-byte pieces swizzled as the tensor map's 64B swizzle
// expects: piece j of row r at j ^ ((r >> 1) & 3)), written back by a TMA
// store so that the global writes are whole row segments rather than 16 bytes
// in each of 32 rows per warp store.
constexpr int TC_MAX_EPI_WARPS = 16;
constexpr int TC_OST_BYTES = 32 * 64;

struct TcSmem {
  bf16 A[TC_STAGES][TC_BM * TC_BK];
  bf16 B[TC_STAGES][TC_MAXN * TC_BK];
  alignas(1024) unsigned char ost[TC_MAX_EPI_WARPS][TC_OST_BYTES];
  uint64_t full[TC_STAGES], empty[TC_STAGES], tfull[2], tempty[2];
  uint32_t tmem_base;
};

struct TcParams {
  CUtensorMap tmA;
  CUtensorMap tmB[3];
  CUtensorMap tmB2;
  CUtensorMap tmO;  // output, boxes of 32 rows x 32 columns, 64B swizzle (when tma_out)
  int tma_out;      // the epilogue writes through the staging buffers and TMA stores
  GemmArgs a;
  int bn;          // output columns per tile
  int umma_n;      // accumulator columns per tile (2*bn for SwiGLU)
  int n_tiles, m_tiles, k_blocks;
  int group_n;  // n-tiles per raster group (divides n_tiles)
  int a_evict_first;  // activations streamed with an evict-first L2 policy
  int seg_start[3];
};

// Tile order: groups of group_n n-tiles; within a group every m-tile in turn,
// the group's n-tiles consecutive.  The CTAs in flight then share one group's
// weight panel (kept in L2 for the whole sweep) and each A row block is read
// once per group, instead of every wave streaming the whole weight matrix.
__device__ __forceinline__ void tc_tile_coords(const TcParams& p, int tile, int& mt, int& nt) {
  const int per_group = p.group_n * p.m_tiles;
  const int g = tile / per_group, w = tile % per_group;
  mt = w / p.group_n;
  nt = g * p.group_n + w % p.group_n;
}

// Units [lo, hi) of part `part` when n units (32-column chunks; 64-column
// RoPE units) are split over `parts` warps of one lane quadrant.
__device__ __forceinline__ void part_range(int n, int part, int parts, int& lo, int& hi) {
  lo = (n * part) / parts;
  hi = (n * (part + 1)) / parts;
}

// A warp writes its 32 rows x 32 columns (row = lane) at columns
// [col, col + 32) in four 8-column pieces: through the warp's staging buffer
// and one TMA store (p.tma_out; rows past M and columns past N are clipped by
// the tensor map), or directly (rows past M skipped, only valid pieces).
__device__ __forceinline__ void tc_emit_begin(const TcParams& p) {
  if (!p.tma_out) return;
  if ((threadIdx.x & 31) == 0) tma_store_wait_read<0>();  // the previous store has read the buffer
  __syncwarp();
}
__device__ __forceinline__ void tc_emit_piece(const TcParams& p, unsigned char* ost, int64_t row, int col, int j,
                                              bool valid, const float* f8) {
  const int lane = threadIdx.x & 31;
  if (p.tma_out) {
    uint4 v;
    uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 h = __floats2bfloat162_rn(f8[2 * e], f8[2 * e + 1]);
      w[e] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(ost + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) = v;
    return;
  }
  if (valid && row < p.a.M) store8((bf16*)p.a.out + row * p.a.ldo + col + 8 * j, f8);
}
__device__ __forceinline__ void tc_emit_end(const TcParams& p, unsigned char* ost, int64_t row, int col) {
  if (!p.tma_out) return;
  const int lane = threadIdx.x & 31;
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(&p.tmO, ost, col, (int)(row - lane));
    tma_store_commit();
  }
}
__device__ __forceinline__ void tc_emit32(const TcParams& p, unsigned char* ost, int64_t row, int col, int nv,
                                          const float* f) {
  tc_emit_begin(p);
#pragma unroll
  for (int j = 0; j < 4; ++j) tc_emit_piece(p, ost, row, col, j, j < nv, f + 8 * j);
  tc_emit_end(p, ost, row, col);
}

// One epilogue warp's share of a tile: TMEM lane quadrant = 32 rows, and part
// `part` of the tile's column units (32-column chunks; 64-column RoPE units).
template <int EPI>
__device__ __forceinline__ void tc_epilogue_tile(const TcParams& p, uint32_t tbase, int64_t row, int nt, int part,
                                                 unsigned char* ost) {
  const GemmArgs& a = p.a;
  const bool in_range = row < a.M;
  const int col0 = nt * p.bn;
  bf16* out = (bf16*)a.out;
  uint32_t r[32], r2[32];
  int u_lo, u_hi;
  if (EPI == kEpiSwiglu) {
    part_range(p.bn / 32, part, TcEpi<EPI>::parts, u_lo, u_hi);
    for (int cc = u_lo * 32; cc < u_hi * 32; cc += 32) {
      tmem_ld32(tbase + cc, r);
      tmem_ld32(tbase + p.bn + cc, r2);
      tmem_wait_ld();
      float f[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float g = __uint_as_float(r2[i]);
        f[i] = __uint_as_float(r[i]) * (g * sigmoid_fast(g));
      }
      tc_emit32(p, ost, row, col0 + cc, 4, f);
    }
    return;
  }
  if (EPI == kEpiRope && col0 < a.rope_cols) {
    // heads of head_dim columns (a multiple of 64): rotate (i, i + hd/2) pairs,
    // 32 pairs per step; the warp's share is half of the tile's heads (or, for
    // one head per tile, half of its pair chunks)
    const int hd = a.head_dim, hd2 = hd / 2;
    const int64_t pos = in_range ? rope_position(a, row) : 0;
    const int nunits = p.bn / 64;  // (head, 32-pair chunk) units
    part_range(nunits, part, TcEpi<EPI>::parts, u_lo, u_hi);
    if (hd == 64) {
      // every unit is a whole head with pairs 0..31: the (cos, sin) of each
      // 16-pair run is formed once and applied to all of this part's heads
      for (int j0 = 0; j0 < 32; j0 += 16) {
        float2 cs[16];
        rope_cs16(a.rope_tab, 32, pos, j0, cs);
        for (int u = u_lo; u < u_hi; ++u) {
          const int hc = u * 64;
          tmem_ld16(tbase + hc + j0, r);
          tmem_ld16(tbase + hc + 32 + j0, r2);
          tmem_wait_ld();
          if (in_range) {
            float lo[16], hi[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float x1 = __uint_as_float(r[i]), x2 = __uint_as_float(r2[i]);
              lo[i] = x1 * cs[i].x - x2 * cs[i].y;
              hi[i] = x2 * cs[i].x + x1 * cs[i].y;
            }
            bf16* o = out + row * a.ldo + col0 + hc + j0;
            store8(o, lo);
            store8(o + 8, lo + 8);
            store8(o + 32, hi);
            store8(o + 40, hi + 8);
          }
        }
      }
      return;
    }
    for (int u = u_lo; u < u_hi; ++u) {
      const int hh = (u * 64) / hd;         // head within the tile
      const int j0 = (u * 32) % hd2;        // first pair index of this unit
      const int hc = hh * hd;
      tmem_ld32(tbase + hc + j0, r);
      tmem_ld32(tbase + hc + hd2 + j0, r2);
      tmem_wait_ld();
      if (in_range) {
        float lo[32], hi[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 cs = rope_cs(a.rope_tab, hd2, pos, j0 + i);
          const float x1 = __uint_as_float(r[i]), x2 = __uint_as_float(r2[i]);
          lo[i] = x1 * cs.x - x2 * cs.y;
          hi[i] = x2 * cs.x + x1 * cs.y;
        }
        bf16* o = out + row * a.ldo + col0 + hc + j0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          store8(o + 8 * i, lo + 8 * i);
          store8(o + hd2 + 8 * i, hi + 8 * i);
        }
      }
    }
    return;
  }
  if (EPI == kEpiSoftplus) {
    // Delta = softplus(acc + bias): the next chunk's TMEM load is in flight while
    // this one is evaluated (the K = 128 main loop is short, so this read-out
    // sets the kernel's pace); one MUFU operation per element
    part_range((p.bn + 31) / 32, part, TcEpi<EPI>::parts, u_lo, u_hi);
    auto chunk = [&](const uint32_t (&rc)[32], int u) {
      const int cc = u * 32;
      const int nv = min(4, (p.bn - cc) / 8);
      const int col = col0 + cc;
      const float4* bp = reinterpret_cast<const float4*>(a.bias + col);  // 16-byte aligned (checked at launch)
      tc_emit_begin(p);
#pragma unroll
      for (int i = 0; i < 4; ++i) {  // 8 columns at a time
        const bool valid = i < nv;
        const float4 b0 = valid ? bp[2 * i] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 b1 = valid ? bp[2 * i + 1] : make_float4(0.f, 0.f, 0.f, 0.f);
        float f[8];
        f[0] = softplus_1x(__uint_as_float(rc[8 * i + 0]) + b0.x);
        f[1] = softplus_1x(__uint_as_float(rc[8 * i + 1]) + b0.y);
        f[2] = softplus_1x(__uint_as_float(rc[8 * i + 2]) + b0.z);
        f[3] = softplus_1x(__uint_as_float(rc[8 * i + 3]) + b0.w);
        f[4] = softplus_1x(__uint_as_float(rc[8 * i + 4]) + b1.x);
        f[5] = softplus_1x(__uint_as_float(rc[8 * i + 5]) + b1.y);
        f[6] = softplus_1x(__uint_as_float(rc[8 * i + 6]) + b1.z);
        f[7] = softplus_1x(__uint_as_float(rc[8 * i + 7]) + b1.w);
        tc_emit_piece(p, ost, row, col, i, valid, f);
      }
      tc_emit_end(p, ost, row, col);
    };
    uint32_t ra[32], rb[32];
    if (u_lo < u_hi) tmem_ld32(tbase + u_lo * 32, ra);
    for (int u = u_lo; u < u_hi; u += 2) {  // two buffers, named statically
      tmem_wait_ld();
      if (u + 1 < u_hi) tmem_ld32(tbase + (u + 1) * 32, rb);
      chunk(ra, u);
      if (u + 1 < u_hi) {
        tmem_wait_ld();
        if (u + 2 < u_hi) tmem_ld32(tbase + (u + 2) * 32, ra);
        chunk(rb, u + 1);
      }
    }
    return;
  }
  // 32-column chunks; a tile width of 16 mod 32 ends in a 16-column chunk (the
  // TMEM columns past it are read but not stored)
  part_range((p.bn + 31) / 32, part, TcEpi<EPI>::parts, u_lo, u_hi);
  for (int cc = u_lo * 32; cc < u_hi * 32; cc += 32) {
    tmem_ld32(tbase + cc, r);
    tmem_wait_ld();
    const int nv = min(4, (p.bn - cc) / 8);  // valid 8-column groups: 4, or 2 in a 16-column tail
    float f[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(r[i]);
    const int col = col0 + cc;
    if (EPI == kEpiResid && in_range) {
      if (a.tap) {
        bf16* t = (bf16*)a.tap + row * a.ldt + col;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (i < nv) store8(t + 8 * i, f + 8 * i);
      }
      const bf16* rs = (const bf16*)a.resid + row * a.ldr + col;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (i >= nv) continue;
        float g[8];
        load8(rs + 8 * i, g);
#pragma unroll
        for (int j = 0; j < 8; ++j) f[8 * i + j] += g[j];
      }
    }
    tc_emit32(p, ost, row, col, nv, f);
  }
}

template <int EPI>
__global__ void __launch_bounds__(TcEpi<EPI>::threads, 1) gemm_tc_kernel(const __grid_constant__ TcParams p, int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  TcSmem& S = *reinterpret_cast<TcSmem*>(smem_raw + smem_align_pad(smem_raw, 1024));
  const int warp = warp_id_sync();
  const int lane = threadIdx.x & 31;
  const int ntiles = p.m_tiles * p.n_tiles;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.tfull[i], 1);
      mbar_init(&S.tempty[i], TcEpi<EPI>::warps);
    }
    fence_mbar_init();
    tma_prefetch_desc(&p.tmA);
    for (int i = 0; i < p.a.nseg; ++i) tma_prefetch_desc(&p.tmB[i]);
    if (EPI == kEpiSwiglu) tma_prefetch_desc(&p.tmB2);
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer
    if (elect_one()) {
      const uint32_t bytes = TC_A_BYTES + (uint32_t)p.umma_n * TC_BK * 2;
      // The group's weight panel is reused by every m-tile: kept in L2 ahead of
      // the activations.  When K is long, a 128-row activation block (>= 1 MB)
      // is the bulk of the traffic and is streamed evict-first; shorter blocks
      // are left at normal priority, since the group's n-tiles read each one
      // several times while it is in flight.
      const uint64_t pol_a = p.a_evict_first ? l2_policy_evict_first() : l2_policy_evict_normal();
      const uint64_t pol_b = l2_policy_evict_last();
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        int mt, nt;
        tc_tile_coords(p, tile, mt, nt);
        int seg = 0;
        while (seg < p.a.nseg - 1 && nt * p.bn >= p.seg_start[seg + 1]) ++seg;
        const int brow = nt * p.bn - p.seg_start[seg];
        // loads are clipped by the tensor maps; a bad tile is reported, not skipped (the pipeline stays in step)
        (void)SAMBA_DCHECK(err, mt >= 0 && mt < p.m_tiles && nt >= 0 && nt < p.n_tiles && brow >= 0 &&
                                    brow < p.a.seg[seg].n);
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int s = it % TC_STAGES;
          const uint32_t j = it / TC_STAGES;
          if (!mbar_wait(&S.empty[s], (j & 1) ^ 1, err)) { ok = false; break; }
          mbar_arrive_expect_tx(&S.full[s], bytes);
          tma_load_2d_hint(S.A[s], &p.tmA, &S.full[s], kb * TC_BK, mt * TC_BM, pol_a);
          if (EPI == kEpiSwiglu) {
            tma_load_2d_hint(S.B[s], &p.tmB[0], &S.full[s], kb * TC_BK, brow, pol_b);
            tma_load_2d_hint(S.B[s] + p.bn * TC_BK, &p.tmB2, &S.full[s], kb * TC_BK, brow, pol_b);
          } else {
            tma_load_2d_hint(S.B[s], &p.tmB[seg], &S.full[s], kb * TC_BK, brow, pol_b);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    const uint32_t idesc = idesc_bf16_f32(TC_BM, p.umma_n);
    if (elect_one()) {
      int it = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++tc) {
        const int acc = tc & 1;
        const uint32_t use = tc >> 1;
        if (!mbar_wait(&S.tempty[acc], (use & 1) ^ 1, err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * TC_MAXN;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int s = it % TC_STAGES;
          const uint32_t j = it / TC_STAGES;
          if (!mbar_wait(&S.full[s], j & 1, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(S.A[s]);
          const uint32_t b_base = smem_u32(S.B[s]);
#pragma unroll
          for (int k = 0; k < TC_BK / 16; ++k) {
            const uint64_t ad = smem_desc(a_base + k * 32, 16, 1024, kLayoutSw128);
            const uint64_t bd = smem_desc(b_base + k * 32, 16, 1024, kLayoutSw128);
            umma_f16_ss(d_tmem, ad, bd, idesc, (kb | k) != 0);
          }
          umma_commit(&S.empty[s]);
        }
        if (ok) umma_commit(&S.tfull[acc]);
      }
    }
  } else {
    // ---------------- epilogue warps 2.. -> TMEM lane quadrant warp % 4, column part (warp - 2) / 4
    const int q = warp & 3;
    const int part = (warp - 2) >> 2;
    int tc = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tc) {
      int mt, nt;
      tc_tile_coords(p, tile, mt, nt);
      const int acc = tc & 1;
      const uint32_t use = tc >> 1;
      // tcgen05.ld in the epilogue is warp-collective: keep the wait warp-uniform
      const bool got = mbar_wait(&S.tfull[acc], use & 1, err);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + acc * TC_MAXN + ((uint32_t)(q * 32) << 16);
      const int64_t row = (int64_t)mt * TC_BM + q * 32 + lane;
      if (SAMBA_DCHECK(err, mt < p.m_tiles && (nt + 1) * p.bn <= p.a.N))
        tc_epilogue_tile<EPI>(p, tbase, row, nt, part, S.ost[warp - 2]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.tempty[acc]);
    }
    if (lane == 0) tma_store_wait_all<0>();  // this warp's output stores complete before the CTA exits
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

bool tc_bn_for(const GemmArgs& a, int& bn) {
  if (a.epi == kEpiSwiglu) {
    bn = 128;
    return a.nseg == 1 && a.N % 128 == 0;
  }
  if (a.nseg == 1 && a.N <= TC_MAXN && a.N % 16 == 0) {
    bn = a.N;
    return true;
  }
  for (int cand : {256, 128, 64, 32}) {
    bool okc = true;
    for (int s = 0; s < a.nseg; ++s) okc = okc && (a.seg[s].n % cand == 0);
    if (okc) {
      bn = cand;
      return true;
    }
  }
  return false;
}

static_assert(sizeof(TcSmem) + 1024 <= 232448, "tcgen05 GEMM shared memory above the 227 KB per-block limit");

template <int EPI>
samba_status tc_launch(TcParams& p, cudaStream_t st) {
  const size_t smem = sizeof(TcSmem) + 1024;
  auto kern = gemm_tc_kernel<EPI>;
  if (!ensure_smem_attr(kern, smem))
    return SAMBA_ERR_CUDA;
  const int ntiles = p.m_tiles * p.n_tiles;
  const int grid = ntiles < num_sms() ? ntiles : num_sms();
  kern<<<grid, TcEpi<EPI>::threads, smem, st>>>(p, device_error_word());
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

}  // namespace

bool gemm_tc_supported(const GemmArgs& a) {
  // K need not be a multiple of 64: the tensor maps end at K and fill the last
  // k-block with zeros
  if (a.dtype != SAMBA_BF16 || a.K % 8 != 0 || a.lda % 8 || a.ldo % 8 || a.M < 1) return false;
  if (!aligned16(a.A) || !aligned16(a.out)) return false;
  int bn;
  if (!tc_bn_for(a, bn)) return false;
  if (a.epi == kEpiRope && (a.head_dim % 64 != 0 || a.rope_cols % a.head_dim != 0)) return false;
  if (a.epi == kEpiRope && bn % a.head_dim != 0) return false;  // whole heads per tile
  if (a.epi == kEpiResid && (a.ldr % 8 || (a.tap && a.ldt % 8))) return false;
  if (a.epi == kEpiSoftplus && !aligned16(a.bias)) return false;
  for (int s = 0; s < a.nseg; ++s)
    if (!aligned16(a.seg[s].W) || (a.seg[s].W2 && !aligned16(a.seg[s].W2))) return false;
  return true;
}

samba_status launch_gemm_tc(const GemmArgs& a, cudaStream_t st) {
  if (!gemm_tc_supported(a)) return SAMBA_ERR_UNSUPPORTED;
  TcParams p;
  memset(&p, 0, sizeof(p));
  p.a = a;
  tc_bn_for(a, p.bn);
  p.umma_n = a.epi == kEpiSwiglu ? 2 * p.bn : p.bn;
  p.n_tiles = a.N / p.bn;
  p.m_tiles = (int)((a.M + TC_BM - 1) / TC_BM);
  {
    // largest divisor of n_tiles whose weight panel stays within 32 MB of L2
    const size_t panel = (size_t)p.umma_n * a.K * 2;  // bytes of B per n-tile
    p.group_n = 1;
    for (int g = 1; g <= p.n_tiles; ++g)
      if (p.n_tiles % g == 0 && (size_t)g * panel <= (size_t(32) << 20)) p.group_n = g;
  }
  p.k_blocks = (a.K + TC_BK - 1) / TC_BK;
  p.a_evict_first = a.K >= 4096 ? 1 : 0;
  {
    // output through staging buffers and TMA stores (64B swizzle, 32 x 32 boxes)
    uint64_t dims[2] = {(uint64_t)a.N, (uint64_t)a.M};
    uint64_t strides[1] = {(uint64_t)a.ldo};
    uint32_t box[2] = {32, 32};
    if (!make_tmap(&p.tmO, a.out, SAMBA_BF16, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B)) return SAMBA_ERR_CUDA;
    p.tma_out = 1;
  }
  {
    uint64_t dims[2] = {(uint64_t)a.K, (uint64_t)a.M};
    uint64_t strides[1] = {(uint64_t)a.lda};
    uint32_t box[2] = {TC_BK, TC_BM};
    if (!make_tmap(&p.tmA, a.A, SAMBA_BF16, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return SAMBA_ERR_CUDA;
  }
  int start = 0;
  const uint32_t brows = (uint32_t)(a.epi == kEpiSwiglu ? p.bn : p.bn);
  for (int s = 0; s < a.nseg; ++s) {
    p.seg_start[s] = start;
    uint64_t dims[2] = {(uint64_t)a.K, (uint64_t)a.seg[s].n};
    uint64_t strides[1] = {(uint64_t)a.K};
    uint32_t box[2] = {TC_BK, brows};
    if (!make_tmap(&p.tmB[s], a.seg[s].W, SAMBA_BF16, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return SAMBA_ERR_CUDA;
    if (a.epi == kEpiSwiglu &&
        !make_tmap(&p.tmB2, a.seg[s].W2, SAMBA_BF16, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return SAMBA_ERR_CUDA;
    start += a.seg[s].n;
  }
  switch (a.epi) {
    case kEpiNone: return tc_launch<kEpiNone>(p, st);
    case kEpiResid: return tc_launch<kEpiResid>(p, st);
    case kEpiSwiglu: return tc_launch<kEpiSwiglu>(p, st);
    case kEpiSoftplus: return tc_launch<kEpiSoftplus>(p, st);
    case kEpiRope: return tc_launch<kEpiRope>(p, st);
  }
  return SAMBA_ERR_INVALID_ARG;
}

samba_status launch_gemm_simt(const GemmArgs& a, cudaStream_t st) {
  if (a.M == 0) return SAMBA_OK;
  return a.dtype == SAMBA_BF16 ? simt_dispatch<bf16>(a, st) : simt_dispatch<float>(a, st);
}

static bool force_simt() {
  const char* e = getenv("SAMBA_GEMM_KERNEL");
  return e && e[0] == 's';
}

// ---- measurement hook: CUDA events around the launches of one epilogue kind
// (no effect, beyond one relaxed atomic load per launch, unless installed)
namespace {
std::mutex g_tm_mu;
std::atomic<int> g_tm_epi{-1};
std::vector<cudaEvent_t> g_tm_start, g_tm_stop;
int g_tm_count = 0;

// Records the next start event on `st` and returns its stop event, or nullptr.
cudaEvent_t timing_begin(int epi, cudaStream_t st) {
  if (g_tm_epi.load(std::memory_order_relaxed) != epi) return nullptr;
  cudaEvent_t s0 = nullptr, s1 = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_tm_mu);
    if (g_tm_epi.load(std::memory_order_relaxed) != epi || g_tm_count >= (int)g_tm_start.size()) return nullptr;
    s0 = g_tm_start[g_tm_count];
    s1 = g_tm_stop[g_tm_count];
    ++g_tm_count;
  }
  if (cudaEventRecord(s0, st) != cudaSuccess) {
    (void)cudaGetLastError();  // a bad event handle must not fail the launch that follows
    return nullptr;
  }
  return s1;
}

void timing_end(cudaEvent_t s1, cudaStream_t st) {
  if (s1 && cudaEventRecord(s1, st) != cudaSuccess) (void)cudaGetLastError();
}
}  // namespace

samba_status gemm_timing_set(int epi, void* const* start, void* const* stop, int capacity) {
  std::lock_guard<std::mutex> lk(g_tm_mu);
  g_tm_epi.store(-1);
  g_tm_start.clear();
  g_tm_stop.clear();
  g_tm_count = 0;
  if (epi < 0) return SAMBA_OK;
  if (epi > kEpiRope || !start || !stop || capacity < 1) return SAMBA_ERR_INVALID_ARG;
  for (int i = 0; i < capacity; ++i)
    if (!start[i] || !stop[i]) return SAMBA_ERR_INVALID_ARG;
  for (int i = 0; i < capacity; ++i) {
    g_tm_start.push_back((cudaEvent_t)start[i]);
    g_tm_stop.push_back((cudaEvent_t)stop[i]);
  }
  g_tm_epi.store(epi);
  return SAMBA_OK;
}

int gemm_timing_count() {
  std::lock_guard<std::mutex> lk(g_tm_mu);
  return g_tm_count;
}

bool gemm_takes_skinny(const GemmArgs& a) { return !force_simt() && a.M <= 64 && gemm_skinny_supported(a); }

static samba_status gemm_dispatch(const GemmArgs& a, cudaStream_t st) {
  if (gemm_takes_skinny(a)) return launch_gemm_skinny(a, st);
  if (!force_simt() && gemm_tc_supported(a)) return launch_gemm_tc(a, st);
  if (a.epi == kEpiRope && 64 % a.head_dim != 0) return SAMBA_ERR_UNSUPPORTED;
  return launch_gemm_simt(a, st);
}

samba_status launch_gemm(const GemmArgs& a, cudaStream_t st) {
  if (!a.A || !a.out || a.M < 0 || a.N <= 0 || a.K <= 0 || a.nseg < 1 || a.nseg > 3) return SAMBA_ERR_INVALID_ARG;
  int nsum = 0;
  for (int s = 0; s < a.nseg; ++s) {
    if (!a.seg[s].W || a.seg[s].n <= 0) return SAMBA_ERR_INVALID_ARG;
    if (a.epi == kEpiSwiglu && !a.seg[s].W2) return SAMBA_ERR_INVALID_ARG;
    nsum += a.seg[s].n;
  }
  if (nsum != a.N) return SAMBA_ERR_INVALID_ARG;
  if (a.epi == kEpiResid && !a.resid) return SAMBA_ERR_INVALID_ARG;
  if (a.epi == kEpiSoftplus && !a.bias) return SAMBA_ERR_INVALID_ARG;
  if (a.epi == kEpiRope && ((!a.rope_tab && !(a.rope_base > 0.f && gemm_takes_skinny(a))) || a.head_dim <= 0 ||
                            a.rope_cols % a.head_dim))
    return SAMBA_ERR_INVALID_ARG;
  if (a.M == 0) return SAMBA_OK;
  // the norm fold is implemented by the skinny kernel only
  if ((a.ss_in || a.ss_out) && !gemm_takes_skinny(a)) return SAMBA_ERR_UNSUPPORTED;
  const cudaEvent_t tstop = timing_begin(a.epi, st);
  const samba_status r = gemm_dispatch(a, st);
  timing_end(tstop, st);
  return r;
}

}  // namespace samba
