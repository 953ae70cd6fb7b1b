// Banded sliding-window GQA attention on the 5th-generation tensor cores
// [Samba 3.4 "Window Specification", "Implementation": query t attends keys
// t-w+1 .. t; GQA kv head = h / (Hq/Hkv)].
//
// One CTA = one 128-query tile of one query head.  It visits only the 128-key
// tiles that intersect the band of its queries (17 tiles for w = 2048), masks
// just the two edge tiles, and keeps all matrix products on tcgen05:
//   warp 0      TMA producer: Q once, then K_j and V_j per key tile (3 stages,
//               128-byte swizzle, no multicast); the K/V rows are shared by the
//               8 query heads of a group through L2.
//   warp 1      owns TMEM (S0 | S1 | O) and issues, from one thread,
//               S_j = Q K_j^T (M128 N128 K16 x4) into S[j%2] and
//               O += P_j V_j  (M128 N64 K16 x8, V read MN-major).
//   warps 2..5  softmax, one query row per thread (TMEM lane): S_j -> registers,
//               band mask on edge tiles, online max/sum in the log2 domain,
//               P_j = exp2(s - m) as bf16 into 128B-swizzled smem.  O is
//               rescaled in TMEM only when the running max grows by more than
//               2^8 (P then stays below 256), so the rescale is rare.
//   epilogue    O / l -> bf16 -> global, by the softmax threads.
// All waits are bounded (error word + early exit on timeout).
#include <stdlib.h>
#include <string.h>

#define SAMBA_TU_ID 9  // site id of this file in debug-check reports
#include "common.cuh"
#include "kernels.h"

namespace samba {

namespace {

constexpr int AT_BM = 128;       // queries per CTA
constexpr int AT_BN = 128;       // keys per tile
constexpr int AT_D = 64;         // head dim handled here
constexpr int AT_STAGES = 3;     // K/V stages
constexpr int AT_THREADS = 192;  // 6 warps
constexpr float kRescaleThresh = 8.0f;  // log2 units

constexpr uint32_t kTileBytes = AT_BM * AT_D * 2;  // 16 KB (Q, K or V tile)

struct AtSmem {
  bf16 Q[AT_BM * AT_D];
  bf16 K[AT_STAGES][AT_BN * AT_D];
  bf16 V[AT_STAGES][AT_BN * AT_D];
  bf16 P[2][2][AT_BM * 64];  // [buffer][key half][row][64 keys], 128B-swizzled
  uint64_t q_full;
  uint64_t kv_full[AT_STAGES], kv_empty[AT_STAGES];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
  uint32_t tmem_base;
};

struct AtParams {
  CUtensorMap tmQ, tmK, tmV;
  bf16* o;
  int64_t ld_o;
  int L, window, Hq, Hkv;
  int qoff, Lk;  // query row t is key row t + qoff; Lk = L + qoff key rows
  float scale_log2;
};

// three-input maximum (one instruction on sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x for a pair of x <= 0 on the FMA pipe, to take part of the exponentials off
// the MUFU unit.  Range reduction: x is clamped to >= -126 (so the exponent
// field below cannot wrap) and n = round(x) is
// taken with the 1.5*2^23 shift (the sum's low mantissa bits hold n, the
// difference is exact); f = x - n lies in [-1/2, 1/2]; 2^f is a degree-3
// polynomial fitted here by relative-error-weighted least squares on Chebyshev
// nodes of [-1/2, 1/2] (max relative error 7.5e-5, far below the bf16 rounding
// of P); 2^n is added to the exponent field, i.e. bits(p) + bits(shifted sum)
// * 2^23 modulo 2^32 (the shift constant's bits vanish under that product).
// Results for x <= -126 (masked keys: x = -inf) are exact zeros.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x = make_float2(fmaxf(x.x, -126.f), fmaxf(x.y, -126.f));
  const float2 r = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
  const float2 n = __fadd2_rn(r, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
  float2 q = __ffma2_rn(make_float2(0.05517137f, 0.05517137f), f, make_float2(0.24261110f, 0.24261110f));
  q = __ffma2_rn(q, f, make_float2(0.69326103f, 0.69326103f));
  q = __ffma2_rn(q, f, make_float2(0.99992806f, 0.99992806f));
  const float2 y = make_float2(__uint_as_float(__float_as_uint(q.x) + __float_as_uint(r.x) * 8388608u),
                               __uint_as_float(__float_as_uint(q.y) + __float_as_uint(r.y) * 8388608u));
  return make_float2(x.x > -126.f ? y.x : 0.f, x.y > -126.f ? y.y : 0.f);  // masked keys give exact zeros
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__global__ void __launch_bounds__(AT_THREADS, 1) swa_tc_kernel(const __grid_constant__ AtParams p, int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  AtSmem& S = *reinterpret_cast<AtSmem*>(smem_raw + smem_align_pad(smem_raw, 1024));
  const int warp = warp_id_sync();
  const int lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * AT_BM;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int g = h / (p.Hq / p.Hkv);

  // key tiles intersecting the band of rows t0 .. t0+127 (key rows tk0 .. tk0+127)
  const int tk0 = t0 + p.qoff;
  const int lo = tk0 - p.window + 1;
  const int kb0 = lo <= 0 ? 0 : (lo / AT_BN) * AT_BN;
  const int ntile = (min(tk0 + AT_BM - 1, p.Lk - 1) - kb0) / AT_BN + 1;
  // the visited key tiles start inside the key rows (loads past Lk are clipped by the tensor map)
  (void)SAMBA_DCHECK(err, t0 < p.L && kb0 >= 0 && ntile >= 1 && kb0 + (ntile - 1) * AT_BN < p.Lk);

  if (warp == 0 && lane == 0) {
    mbar_init(&S.q_full, 1);
    for (int s = 0; s < AT_STAGES; ++s) {
      mbar_init(&S.kv_full[s], 1);
      mbar_init(&S.kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_free[i], 4);
      mbar_init(&S.p_full[i], 4);
      mbar_init(&S.pv_done[i], 1);
    }
    fence_mbar_init();
    tma_prefetch_desc(&p.tmQ);
    tma_prefetch_desc(&p.tmK);
    tma_prefetch_desc(&p.tmV);
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const uint32_t tO = tmem + 256;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      mbar_arrive_expect_tx(&S.q_full, kTileBytes);
      tma_load_3d(S.Q, &p.tmQ, &S.q_full, h * AT_D, t0, b);
      for (int j = 0; j < ntile; ++j) {
        const int s = j % AT_STAGES;
        const uint32_t use = j / AT_STAGES;
        if (!mbar_wait(&S.kv_empty[s], (use & 1) ^ 1, err)) break;
        mbar_arrive_expect_tx(&S.kv_full[s], 2 * kTileBytes);
        const int kb = kb0 + j * AT_BN;
        tma_load_3d(S.K[s], &p.tmK, &S.kv_full[s], g * AT_D, kb, b);
        tma_load_3d(S.V[s], &p.tmV, &S.kv_full[s], g * AT_D, kb, b);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc_s = idesc_bf16_f32(AT_BM, AT_BN, false);
    const uint32_t idesc_o = idesc_bf16_f32(AT_BM, AT_D, true);  // V is N-contiguous (MN-major B)
    if (elect_one()) {
      bool ok = mbar_wait(&S.q_full, 0, err);
      const uint32_t q_base = smem_u32(S.Q);
      auto issue_s = [&](int j) -> bool {
        const int s = j % AT_STAGES;
        if (!mbar_wait(&S.kv_full[s], (j / AT_STAGES) & 1, err)) return false;
        if (j >= 2 && !mbar_wait(&S.s_free[j & 1], ((j - 2) >> 1) & 1, err)) return false;
        tc_fence_after();
        const uint32_t k_base = smem_u32(S.K[s]);
#pragma unroll
        for (int k = 0; k < AT_D / 16; ++k)
          umma_f16_ss((tmem + ((j & 1) ? 128u : 0u)), smem_desc(q_base + k * 32, 16, 1024, kLayoutSw128),
                      smem_desc(k_base + k * 32, 16, 1024, kLayoutSw128), idesc_s, k != 0);
        umma_commit(&S.s_full[j & 1]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int s = j % AT_STAGES;
        if (!mbar_wait(&S.p_full[j & 1], (j >> 1) & 1, err)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(S.V[s]);
#pragma unroll
        for (int k = 0; k < AT_BN / 16; ++k) {
          const uint32_t a_addr = smem_u32(S.P[j & 1][k >> 2]) + (k & 3) * 32;
          const uint32_t b_addr = v_base + k * 16 * AT_D * 2;  // 16 keys x 128 B
          umma_f16_ss(tO, smem_desc(a_addr, 16, 1024, kLayoutSw128), smem_desc(b_addr, 16, 1024, kLayoutSw128),
                      idesc_o, (j | k) != 0);
        }
        umma_commit(&S.kv_empty[s]);
        umma_commit(&S.pv_done[j & 1]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < ntile; ++j) {
        if (j + 1 < ntile) ok = issue_s(j + 1);
        if (ok) ok = issue_pv(j);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    // Every tcgen05.ld/st below is warp-collective (.sync.aligned): the waits in
    // front of them and the rescale decision are made warp-uniform.
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // query row within the tile == TMEM lane
    const int tq = t0 + r;         // query row
    const int t = tk0 + r;         // its key row
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
      const bool w = mbar_wait(bar, par, err);
      return __all_sync(0xffffffffu, w);
    };
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < ntile; ++j) {
      const int kb = kb0 + j * AT_BN;
      const uint32_t tSj = tmem + ((j & 1) ? 128u : 0u);
      if (!wait_all(&S.s_full[j & 1], (j >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tSj + lane_off + c * 32, sr + c * 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.s_free[j & 1]);

      // Row max on the raw scores (the softmax scale is positive and folded into
      // the exponent below).  Only the two edge tiles need the band mask; there the
      // valid key offsets of row t are (t - w - kb, t - kb], empty for t >= L.
      const bool edge = (kb + AT_BN - 1 > tk0) || (kb < tk0 + AT_BM - p.window);
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
      if (edge) {
        const int hi = tq < p.L ? t - kb : -1;
        const int lo = t - p.window - kb;
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i > hi || i <= lo) sr[i] = __float_as_uint(-INFINITY);
      }
#pragma unroll
      for (int i = 0; i < 128; i += 2)
        m8[(i >> 1) & 7] = fmax3(m8[(i >> 1) & 7], __uint_as_float(sr[i]), __uint_as_float(sr[i + 1]));
      const float mraw = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      const float mt = mraw * p.scale_log2;  // -inf stays -inf
      // Online max with conditional rescale: a row moves its reference max only
      // when the tile max exceeds it by more than 2^8; O is then rescaled in TMEM.
      const bool need = mt > m_run + kRescaleThresh;
      float alpha = 1.f;
      if (need) {
        if (m_run != -INFINITY) alpha = exp2f(m_run - mt);
        l_run *= alpha;
        m_run = mt;
      }
      if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!wait_all(&S.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        uint32_t orr[64];
        tmem_ld32(tO + lane_off, orr);
        tmem_ld32(tO + lane_off + 32, orr + 32);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 64; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
        tmem_st16(tO + lane_off, orr);
        tmem_st16(tO + lane_off + 16, orr + 16);
        tmem_st16(tO + lane_off + 32, orr + 32);
        tmem_st16(tO + lane_off + 48, orr + 48);
        tmem_wait_st();
      }
      const float msub = m_run == -INFINITY ? 0.f : m_run;
      // P buffer j%2 was last read by PV_{j-2}
      if (j >= 2 && !wait_all(&S.pv_done[j & 1], ((j - 2) >> 1) & 1)) { ok = false; break; }
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(-msub, -msub);
      float2 ls2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        unsigned char* prow = reinterpret_cast<unsigned char*>(S.P[j & 1][half]) + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float e[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i = half * 64 + c * 8 + 2 * q;
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), sc2, nm2);
            e[2 * q] = ex2_approx(x.x);
            e[2 * q + 1] = ex2_approx(x.y);
            ls2[q] = __fadd2_rn(ls2[q], make_float2(e[2 * q], e[2 * q + 1]));
          }
          uint4 v4 = make_uint4(pack_bf16(e[0], e[1]), pack_bf16(e[2], e[3]), pack_bf16(e[4], e[5]),
                                pack_bf16(e[6], e[7]));
          *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) = v4;
        }
      }
      l_run += ((ls2[0].x + ls2[0].y) + (ls2[1].x + ls2[1].y)) + ((ls2[2].x + ls2[2].y) + (ls2[3].x + ls2[3].y));
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.p_full[j & 1]);
    }
    // epilogue: wait for the last P.V, then O / l
    if (ok && wait_all(&S.pv_done[(ntile - 1) & 1], ((ntile - 1) >> 1) & 1)) {
      tc_fence_after();
      uint32_t orr[64];
      tmem_ld32(tO + lane_off, orr);
      tmem_ld32(tO + lane_off + 32, orr + 32);
      tmem_wait_ld();
      if (tq < p.L && l_run > 0.f && SAMBA_DCHECK(err, h < p.Hq)) {
        const float inv = 1.f / l_run;
        bf16* op = p.o + ((int64_t)b * p.L + tq) * p.ld_o + (int64_t)h * AT_D;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float f[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) f[q] = __uint_as_float(orr[c * 8 + q]) * inv;
          store8(op + c * 8, f);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Head dim 256 (the 3.8B shapes: 11 query heads over one kv head), one query
// head per CTA.  Q (128 x 256) and each K/V tile (64 keys x 256) are four
// 64-column 128B-swizzled sub-tiles; S = Q K^T is 16 K16 steps into a
// double-buffered 64-column S; O = P V is M128 x N256 (V MN-major across four
// 64-wide atoms, 8 KB apart) accumulated over four K16 key steps.  TMEM:
// S0 | S1 | O = 64 + 64 + 256 columns.  Shared memory: Q 64 KB, two K/V stages
// 128 KB, two P tiles 32 KB.  Roles as in swa_tc_kernel.
constexpr int H_BN = 64;      // keys per tile
constexpr int H_D = 256;      // head dim
constexpr int H_STAGES = 2;
constexpr uint32_t kHQBytes = AT_BM * H_D * 2;    // 64 KB
constexpr uint32_t kHKVBytes = H_BN * H_D * 2;    // 32 KB (K or V tile)

struct AtHSmem {
  bf16 Q[4][AT_BM * 64];             // [d atom][row][64]
  bf16 K[H_STAGES][4][H_BN * 64];    // [stage][d atom][key][64]
  bf16 V[H_STAGES][4][H_BN * 64];
  bf16 P[2][AT_BM * 64];             // [buffer][row][64 keys]
  uint64_t q_full;
  uint64_t kv_full[H_STAGES], kv_empty[H_STAGES];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
  uint32_t tmem_base;
};

__global__ void __launch_bounds__(AT_THREADS, 1) swa_tc256_kernel(const __grid_constant__ AtParams p, int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  AtHSmem& S = *reinterpret_cast<AtHSmem*>(smem_raw + smem_align_pad(smem_raw, 1024));
  const int warp = warp_id_sync();
  const int lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * AT_BM;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int g = h / (p.Hq / p.Hkv);
  const int tk0 = t0 + p.qoff;
  const int lo = tk0 - p.window + 1;
  const int kb0 = lo <= 0 ? 0 : (lo / H_BN) * H_BN;
  const int ntile = (min(tk0 + AT_BM - 1, p.Lk - 1) - kb0) / H_BN + 1;
  // the visited key tiles start inside the key rows (loads past Lk are clipped by the tensor map)
  (void)SAMBA_DCHECK(err, t0 < p.L && kb0 >= 0 && ntile >= 1 && kb0 + (ntile - 1) * H_BN < p.Lk);

  if (warp == 0 && lane == 0) {
    mbar_init(&S.q_full, 1);
    for (int s = 0; s < H_STAGES; ++s) {
      mbar_init(&S.kv_full[s], 1);
      mbar_init(&S.kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_free[i], 4);
      mbar_init(&S.p_full[i], 4);
      mbar_init(&S.pv_done[i], 1);
    }
    fence_mbar_init();
    tma_prefetch_desc(&p.tmQ);
    tma_prefetch_desc(&p.tmK);
    tma_prefetch_desc(&p.tmV);
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const uint32_t tO = tmem + 256;

  if (warp == 0) {
    if (elect_one()) {
      mbar_arrive_expect_tx(&S.q_full, kHQBytes);
#pragma unroll
      for (int a = 0; a < 4; ++a) tma_load_3d(S.Q[a], &p.tmQ, &S.q_full, h * H_D + a * 64, t0, b);
      for (int j = 0; j < ntile; ++j) {
        const int s = j % H_STAGES;
        if (!mbar_wait(&S.kv_empty[s], ((j / H_STAGES) & 1) ^ 1, err)) break;
        mbar_arrive_expect_tx(&S.kv_full[s], 2 * kHKVBytes);
        const int kb = kb0 + j * H_BN;
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          tma_load_3d(S.K[s][a], &p.tmK, &S.kv_full[s], g * H_D + a * 64, kb, b);
          tma_load_3d(S.V[s][a], &p.tmV, &S.kv_full[s], g * H_D + a * 64, kb, b);
        }
      }
    }
  } else if (warp == 1) {
    const uint32_t idesc_s = idesc_bf16_f32(AT_BM, H_BN, false);
    const uint32_t idesc_o = idesc_bf16_f32(AT_BM, H_D, true);  // V MN-major
    if (elect_one()) {
      bool ok = mbar_wait(&S.q_full, 0, err);
      auto issue_s = [&](int j) -> bool {
        const int s = j % H_STAGES;
        if (!mbar_wait(&S.kv_full[s], (j / H_STAGES) & 1, err)) return false;
        if (j >= 2 && !mbar_wait(&S.s_free[j & 1], ((j - 2) >> 1) & 1, err)) return false;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < H_D / 16; ++k) {
          const uint32_t qa = smem_u32(S.Q[k >> 2]) + (k & 3) * 32;
          const uint32_t ka = smem_u32(S.K[s][k >> 2]) + (k & 3) * 32;
          umma_f16_ss(tmem + ((j & 1) ? 64u : 0u), smem_desc(qa, 16, 1024, kLayoutSw128),
                      smem_desc(ka, 16, 1024, kLayoutSw128), idesc_s, k != 0);
        }
        umma_commit(&S.s_full[j & 1]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int s = j % H_STAGES;
        if (!mbar_wait(&S.p_full[j & 1], (j >> 1) & 1, err)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(S.V[s][0]);
        const uint32_t atom = (uint32_t)(H_BN * 64 * 2);  // bytes between 64-wide atoms along N
#pragma unroll
        for (int k = 0; k < H_BN / 16; ++k) {
          const uint32_t a_addr = smem_u32(S.P[j & 1]) + k * 32;
          const uint32_t b_addr = v_base + k * 16 * 128;  // 16 keys x 128 B
          umma_f16_ss(tO, smem_desc(a_addr, 16, 1024, kLayoutSw128), smem_desc(b_addr, atom, 1024, kLayoutSw128),
                      idesc_o, (j | k) != 0);
        }
        umma_commit(&S.kv_empty[s]);
        umma_commit(&S.pv_done[j & 1]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < ntile; ++j) {
        if (j + 1 < ntile) ok = issue_s(j + 1);
        if (ok) ok = issue_pv(j);
      }
    }
  } else {
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int tq = t0 + r;
    const int t = tk0 + r;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
      const bool w = mbar_wait(bar, par, err);
      return __all_sync(0xffffffffu, w);
    };
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < ntile; ++j) {
      const int kb = kb0 + j * H_BN;
      const uint32_t tSj = tmem + ((j & 1) ? 64u : 0u);
      if (!wait_all(&S.s_full[j & 1], (j >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(tSj + lane_off, sr);
      tmem_ld32(tSj + lane_off + 32, sr + 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.s_free[j & 1]);
      const bool edge = (kb + H_BN - 1 > tk0) || (kb < tk0 + AT_BM - p.window);
      if (edge) {
        const int hi = tq < p.L ? t - kb : -1;
        const int lo_i = t - p.window - kb;
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i > hi || i <= lo_i) sr[i] = __float_as_uint(-INFINITY);
      }
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; i += 2)
        m8[(i >> 1) & 7] = fmax3(m8[(i >> 1) & 7], __uint_as_float(sr[i]), __uint_as_float(sr[i + 1]));
      const float mraw = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      const float mt = mraw * p.scale_log2;
      const bool need = mt > m_run + kRescaleThresh;
      float alpha = 1.f;
      if (need) {
        if (m_run != -INFINITY) alpha = exp2f(m_run - mt);
        l_run *= alpha;
        m_run = mt;
      }
      if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!wait_all(&S.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < H_D / 32; ++c) {
          uint32_t orr[32];
          tmem_ld32(tO + lane_off + c * 32, orr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
          tmem_st16(tO + lane_off + c * 32, orr);
          tmem_st16(tO + lane_off + c * 32 + 16, orr + 16);
        }
        tmem_wait_st();
      }
      const float msub = m_run == -INFINITY ? 0.f : m_run;
      if (j >= 2 && !wait_all(&S.pv_done[j & 1], ((j - 2) >> 1) & 1)) { ok = false; break; }
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(-msub, -msub);
      float2 ls2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      unsigned char* prow = reinterpret_cast<unsigned char*>(S.P[j & 1]) + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float e[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = c * 8 + 2 * q;
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), sc2, nm2);
          if (q == 0) {
            const float2 y = exp2_poly2(x);
            e[0] = y.x;
            e[1] = y.y;
          } else {
            e[2 * q] = ex2_approx(x.x);
            e[2 * q + 1] = ex2_approx(x.y);
          }
          ls2[q] = __fadd2_rn(ls2[q], make_float2(e[2 * q], e[2 * q + 1]));
        }
        uint4 v4 = make_uint4(pack_bf16(e[0], e[1]), pack_bf16(e[2], e[3]), pack_bf16(e[4], e[5]),
                              pack_bf16(e[6], e[7]));
        *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) = v4;
      }
      l_run += ((ls2[0].x + ls2[0].y) + (ls2[1].x + ls2[1].y)) + ((ls2[2].x + ls2[2].y) + (ls2[3].x + ls2[3].y));
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.p_full[j & 1]);
    }
    if (ok && wait_all(&S.pv_done[(ntile - 1) & 1], ((ntile - 1) >> 1) & 1)) {
      tc_fence_after();
      const bool store = tq < p.L && l_run > 0.f && SAMBA_DCHECK(err, h < p.Hq);
      const float inv = store ? 1.f / l_run : 0.f;
      bf16* op = p.o + ((int64_t)b * p.L + tq) * p.ld_o + (int64_t)h * H_D;
#pragma unroll
      for (int c = 0; c < H_D / 32; ++c) {
        uint32_t orr[32];
        tmem_ld32(tO + lane_off + c * 32, orr);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            float f[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) f[q] = __uint_as_float(orr[q8 * 8 + q]) * inv;
            store8(op + c * 32 + q8 * 8, f);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Two query heads per CTA (same kv head): two softmax warpgroups ping-pong on
// the exp/FMA pipes while sharing every K/V tile.
//   warp 0      TMA: Q of both heads, then K_j/V_j (3 stages)
//   warp 1      TMEM owner + MMA issuer: S_A, S_B (M128 N128) and O_A, O_B (M128 N64)
//   warps 2..5  softmax of head A, warps 6..9 softmax of head B (TMEM lane
//               quadrant = warp % 4 in both groups)
// The scores are read from TMEM twice (row max, then exponentials), which keeps
// the softmax threads at ~100 registers so that 10 warps fit the register file.
constexpr int A2_THREADS = 320;

struct At2Smem {
  bf16 Q[2][AT_BM * AT_D];
  bf16 K[AT_STAGES][AT_BN * AT_D];
  bf16 V[AT_STAGES][AT_BN * AT_D];
  bf16 P[2][2][AT_BM * 64];  // [warpgroup][key half][row][64 keys], 128B-swizzled
  uint64_t q_full;
  uint64_t kv_full[AT_STAGES], kv_empty[AT_STAGES];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
  uint32_t tmem_base;
};

// kPolyPairs: pairs (of the four per 8-key group) whose exponentials run on the
// FMA pipe (exp2_poly2) instead of the MUFU unit.
template <int kPolyPairs>
__global__ void __launch_bounds__(A2_THREADS, 1) swa_tc2_kernel(const __grid_constant__ AtParams p, int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  At2Smem& S = *reinterpret_cast<At2Smem*>(smem_raw + smem_align_pad(smem_raw, 1024));
  const int warp = warp_id_sync();
  const int lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * AT_BM;
  const int h0 = blockIdx.y * 2;
  const int b = blockIdx.z;
  const int g = h0 / (p.Hq / p.Hkv);
  const int tk0 = t0 + p.qoff;  // key row of query row t0
  const int lo = tk0 - p.window + 1;
  const int kb0 = lo <= 0 ? 0 : (lo / AT_BN) * AT_BN;
  const int ntile = (min(tk0 + AT_BM - 1, p.Lk - 1) - kb0) / AT_BN + 1;
  // the visited key tiles start inside the key rows (loads past Lk are clipped by the tensor map)
  (void)SAMBA_DCHECK(err, t0 < p.L && kb0 >= 0 && ntile >= 1 && kb0 + (ntile - 1) * AT_BN < p.Lk);

  if (warp == 0 && lane == 0) {
    mbar_init(&S.q_full, 1);
    for (int s = 0; s < AT_STAGES; ++s) {
      mbar_init(&S.kv_full[s], 1);
      mbar_init(&S.kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_free[i], 4);
      mbar_init(&S.p_full[i], 4);
      mbar_init(&S.pv_done[i], 1);
    }
    fence_mbar_init();
    tma_prefetch_desc(&p.tmQ);
    tma_prefetch_desc(&p.tmK);
    tma_prefetch_desc(&p.tmV);
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  // TMEM: S_A [0,128) S_B [128,256) O_A [256,320) O_B [320,384)

  if (warp == 0) {
    if (elect_one()) {
      mbar_arrive_expect_tx(&S.q_full, 2 * kTileBytes);
      tma_load_3d(S.Q[0], &p.tmQ, &S.q_full, h0 * AT_D, t0, b);
      tma_load_3d(S.Q[1], &p.tmQ, &S.q_full, (h0 + 1) * AT_D, t0, b);
      for (int j = 0; j < ntile; ++j) {
        const int s = j % AT_STAGES;
        if (!mbar_wait(&S.kv_empty[s], ((j / AT_STAGES) & 1) ^ 1, err)) break;
        mbar_arrive_expect_tx(&S.kv_full[s], 2 * kTileBytes);
        const int kb = kb0 + j * AT_BN;
        tma_load_3d(S.K[s], &p.tmK, &S.kv_full[s], g * AT_D, kb, b);
        tma_load_3d(S.V[s], &p.tmV, &S.kv_full[s], g * AT_D, kb, b);
      }
    }
  } else if (warp == 1) {
    const uint32_t idesc_s = idesc_bf16_f32(AT_BM, AT_BN, false);
    const uint32_t idesc_o = idesc_bf16_f32(AT_BM, AT_D, true);
    if (elect_one()) {
      bool ok = mbar_wait(&S.q_full, 0, err);
      auto issue_s = [&](int wg, int j) -> bool {
        const int s = j % AT_STAGES;
        if (wg == 0 && !mbar_wait(&S.kv_full[s], (j / AT_STAGES) & 1, err)) return false;
        if (j >= 1 && !mbar_wait(&S.s_free[wg], (j - 1) & 1, err)) return false;
        tc_fence_after();
        const uint32_t q_base = smem_u32(S.Q[wg]);
        const uint32_t k_base = smem_u32(S.K[s]);
#pragma unroll
        for (int k = 0; k < AT_D / 16; ++k)
          umma_f16_ss(tmem + wg * 128u, smem_desc(q_base + k * 32, 16, 1024, kLayoutSw128),
                      smem_desc(k_base + k * 32, 16, 1024, kLayoutSw128), idesc_s, k != 0);
        umma_commit(&S.s_full[wg]);
        return true;
      };
      auto issue_pv = [&](int wg, int j) -> bool {
        const int s = j % AT_STAGES;
        if (!mbar_wait(&S.p_full[wg], j & 1, err)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(S.V[s]);
#pragma unroll
        for (int k = 0; k < AT_BN / 16; ++k) {
          const uint32_t a_addr = smem_u32(S.P[wg][k >> 2]) + (k & 3) * 32;
          const uint32_t b_addr = v_base + k * 16 * AT_D * 2;
          umma_f16_ss(tmem + 256u + wg * 64u, smem_desc(a_addr, 16, 1024, kLayoutSw128),
                      smem_desc(b_addr, 16, 1024, kLayoutSw128), idesc_o, (j | k) != 0);
        }
        if (wg == 1) umma_commit(&S.kv_empty[s]);  // both heads are done with K_j, V_j
        umma_commit(&S.pv_done[wg]);
        return true;
      };
      // S_{j+1} of a head is issued as soon as its softmax has read S_j (before
      // it has finished P_j), then PV_j once P_j is in shared memory.
      if (ok) ok = issue_s(0, 0);
      if (ok) ok = issue_s(1, 0);
      for (int j = 0; ok && j < ntile; ++j) {
        if (j + 1 < ntile) ok = issue_s(0, j + 1);
        if (ok) ok = issue_pv(0, j);
        if (ok && j + 1 < ntile) ok = issue_s(1, j + 1);
        if (ok) ok = issue_pv(1, j);
      }
    }
  } else {
    const int wg = (warp - 2) >> 2;  // 0: head h0, 1: head h0 + 1
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int tq = t0 + r;  // query row
    const int t = tk0 + r;  // its key row
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tmem + wg * 128u + lane_off;
    const uint32_t tO = tmem + 256u + wg * 64u + lane_off;
    auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
      const bool w = mbar_wait(bar, par, err);
      return __all_sync(0xffffffffu, w);
    };
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < ntile; ++j) {
      const int kb = kb0 + j * AT_BN;
      if (!wait_all(&S.s_full[wg], j & 1)) { ok = false; break; }
      tc_fence_after();
      const bool edge = (kb + AT_BN - 1 > tk0) || (kb < tk0 + AT_BM - p.window);
      const int hi = tq < p.L ? t - kb : -1;  // valid key offsets of row t: (lo_i, hi]
      const int lo_i = t - p.window - kb;
      // pass 1: row max of the raw scores, two 32-column loads per TMEM round trip
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
      auto max_chunk = [&](uint32_t (&sr)[32], int c) {
        if (edge) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int kk = c * 32 + i;
            if (kk > hi || kk <= lo_i) sr[i] = __float_as_uint(-INFINITY);
          }
        }
#pragma unroll
        for (int i = 0; i < 32; i += 2)
          m8[(i >> 1) & 7] = fmax3(m8[(i >> 1) & 7], __uint_as_float(sr[i]), __uint_as_float(sr[i + 1]));
      };
#pragma unroll
      for (int c = 0; c < 4; c += 2) {
        uint32_t sa[32], sb[32];
        tmem_ld32(tS + c * 32, sa);
        tmem_ld32(tS + (c + 1) * 32, sb);
        tmem_wait_ld();
        max_chunk(sa, c);
        max_chunk(sb, c + 1);
      }
      const float mraw = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      const float mt = mraw * p.scale_log2;
      const bool need = mt > m_run + kRescaleThresh;
      float alpha = 1.f;
      if (need) {
        if (m_run != -INFINITY) alpha = exp2f(m_run - mt);
        l_run *= alpha;
        m_run = mt;
      }
      // PV_{j-1} must be complete before O is rescaled and before P is overwritten
      if (j >= 1 && !wait_all(&S.pv_done[wg], (j - 1) & 1)) { ok = false; break; }
      tc_fence_after();
      if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t orr[16];
          tmem_ld16(tO + c * 16, orr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
          tmem_st16(tO + c * 16, orr);
        }
        tmem_wait_st();
      }
      const float msub = m_run == -INFINITY ? 0.f : m_run;
      // pass 2: P = exp2(s * scale - m) as bf16 into the swizzled P tile.  The band
      // mask is applied in a separate (tile-uniform) branch so that the 15 of 17
      // interior tiles of a band pay nothing for it; scale-subtract and row sums
      // run as packed fp32x2 operations.
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(-msub, -msub);
      float2 ls2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      // software pipeline: the load of chunk c+1 is in flight while chunk c is exponentiated
      uint32_t sbuf[2][32];
      tmem_ld32(tS, sbuf[0]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c + 1 < 4) tmem_ld32(tS + (c + 1) * 32, sbuf[(c + 1) & 1]);
        uint32_t (&sr)[32] = sbuf[c & 1];
        if (edge) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int kk = c * 32 + i;
            if (kk > hi || kk <= lo_i) sr[i] = __float_as_uint(-INFINITY);
          }
        }
        unsigned char* prow = reinterpret_cast<unsigned char*>(S.P[wg][c >> 1]) + r * 128;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int chunk = (c & 1) * 4 + cc;  // 16-byte chunk (8 keys) within the 64-key half
          float e[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i = cc * 8 + 2 * q;
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), sc2, nm2);
            if (q < kPolyPairs) {
              const float2 y = exp2_poly2(x);
              e[2 * q] = y.x;
              e[2 * q + 1] = y.y;
            } else {
              e[2 * q] = ex2_approx(x.x);
              e[2 * q + 1] = ex2_approx(x.y);
            }
            ls2[q] = __fadd2_rn(ls2[q], make_float2(e[2 * q], e[2 * q + 1]));
          }
          uint4 v4 = make_uint4(pack_bf16(e[0], e[1]), pack_bf16(e[2], e[3]), pack_bf16(e[4], e[5]),
                                pack_bf16(e[6], e[7]));
          *reinterpret_cast<uint4*>(prow + ((chunk ^ (r & 7)) << 4)) = v4;
        }
        if (c + 1 < 4) {
          tmem_wait_ld();
          if (c + 1 == 3) {  // every score of this tile is in registers: S may be overwritten
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.s_free[wg]);
          }
        }
      }
      l_run += ((ls2[0].x + ls2[0].y) + (ls2[1].x + ls2[1].y)) + ((ls2[2].x + ls2[2].y) + (ls2[3].x + ls2[3].y));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.p_full[wg]);
    }
    if (ok && wait_all(&S.pv_done[wg], (ntile - 1) & 1)) {
      tc_fence_after();
      uint32_t orr[64];
      tmem_ld32(tO, orr);
      tmem_ld32(tO + 32, orr + 32);
      tmem_wait_ld();
      if (tq < p.L && l_run > 0.f && SAMBA_DCHECK(err, h0 + wg < p.Hq)) {
        const float inv = 1.f / l_run;
        bf16* op = p.o + ((int64_t)b * p.L + tq) * p.ld_o + (int64_t)(h0 + wg) * AT_D;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float f[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) f[q] = __uint_as_float(orr[c * 8 + q]) * inv;
          store8(op + c * 8, f);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Four query heads per CTA (four heads of one kv group at the same 128 query
// rows), 64-key tiles.  Sixteen softmax warps (four per head, one per TMEM lane
// quadrant) keep the exponential unit fed while any one head waits on its
// matrix products; every K/V tile is read once for four heads.
//   warp 0      TMA: Q of the four heads, then K_j / V_j (64 keys, 4 stages)
//   warp 1      TMEM owner + MMA issuer.  It issues, per head and as soon as
//               its inputs are ready (polled, no fixed head order),
//               S_h(j) = Q_h K_j^T (M128 N64 K16 x4) and O_h += P_h(j) V_j
//               (M128 N64 K16 x4); a K/V stage is released once all four
//               heads' products of its tile completed.
//   warps 2..17 softmax of head (warp - 2) / 4, query row = TMEM lane: the 64
//               scores of a tile in registers, band mask on edge tiles, online
//               max with lazy O rescale (> 2^8), P as bf16 into 128B-swizzled
//               shared memory, one pair in four of the exponentials on the FMA
//               pipe.
// TMEM: S_h at columns 64h, O_h at 256 + 64h.
constexpr int A4_HEADS = 4;
constexpr int A4_BN = 64;
constexpr int A4_STAGES = 4;
constexpr int A4_THREADS = (2 + 4 * A4_HEADS) * 32;
constexpr uint32_t kKV64Bytes = A4_BN * AT_D * 2;  // 8 KB

struct At4Smem {
  bf16 Q[A4_HEADS][AT_BM * AT_D];
  bf16 K[A4_STAGES][A4_BN * AT_D];
  bf16 V[A4_STAGES][A4_BN * AT_D];
  bf16 P[A4_HEADS][AT_BM * A4_BN];  // [row][64 keys], 128B-swizzled
  uint64_t q_full;
  uint64_t kv_full[A4_STAGES], kv_empty[A4_STAGES];
  uint64_t s_full[A4_HEADS], s_free[A4_HEADS], p_full[A4_HEADS], pv_done[A4_HEADS];
  uint32_t tmem_base;
};

template <int kPolyPairs>
__global__ void __launch_bounds__(A4_THREADS, 1) swa_tc4_kernel(const __grid_constant__ AtParams p, int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  At4Smem& S = *reinterpret_cast<At4Smem*>(smem_raw + smem_align_pad(smem_raw, 1024));
  const int warp = warp_id_sync();
  const int lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * AT_BM;
  const int h0 = blockIdx.y * A4_HEADS;
  const int b = blockIdx.z;
  const int g = h0 / (p.Hq / p.Hkv);
  const int tk0 = t0 + p.qoff;  // key row of query row t0
  const int lo = tk0 - p.window + 1;
  const int kb0 = lo <= 0 ? 0 : (lo / A4_BN) * A4_BN;
  const int ntile = (min(tk0 + AT_BM - 1, p.Lk - 1) - kb0) / A4_BN + 1;
  // the visited key tiles start inside the key rows (loads past Lk are clipped by the tensor map)
  (void)SAMBA_DCHECK(err, t0 < p.L && kb0 >= 0 && ntile >= 1 && kb0 + (ntile - 1) * A4_BN < p.Lk);

  if (warp == 0 && lane == 0) {
    mbar_init(&S.q_full, 1);
    for (int s = 0; s < A4_STAGES; ++s) {
      mbar_init(&S.kv_full[s], 1);
      mbar_init(&S.kv_empty[s], 1);
    }
    for (int i = 0; i < A4_HEADS; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_free[i], 4);
      mbar_init(&S.p_full[i], 4);
      mbar_init(&S.pv_done[i], 1);
    }
    fence_mbar_init();
    tma_prefetch_desc(&p.tmQ);
    tma_prefetch_desc(&p.tmK);
    tma_prefetch_desc(&p.tmV);
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
    if (elect_one()) {
      mbar_arrive_expect_tx(&S.q_full, A4_HEADS * kTileBytes);
      for (int hh = 0; hh < A4_HEADS; ++hh)
        tma_load_3d(S.Q[hh], &p.tmQ, &S.q_full, (h0 + hh) * AT_D, t0, b);
      for (int j = 0; j < ntile; ++j) {
        const int s = j % A4_STAGES;
        if (!mbar_wait(&S.kv_empty[s], ((j / A4_STAGES) & 1) ^ 1, err)) break;
        mbar_arrive_expect_tx(&S.kv_full[s], 2 * kKV64Bytes);
        const int kb = kb0 + j * A4_BN;
        tma_load_3d(S.K[s], &p.tmK, &S.kv_full[s], g * AT_D, kb, b);
        tma_load_3d(S.V[s], &p.tmV, &S.kv_full[s], g * AT_D, kb, b);
      }
    }
  } else if (warp == 1) {
    const uint32_t idesc_s = idesc_bf16_f32(AT_BM, A4_BN, false);
    const uint32_t idesc_o = idesc_bf16_f32(AT_BM, AT_D, true);  // V is N-contiguous (MN-major B)
    if (elect_one()) {
      bool ok = mbar_wait(&S.q_full, 0, err);
      int ns[A4_HEADS], npv[A4_HEADS], cnt[A4_STAGES];
      for (int i = 0; i < A4_HEADS; ++i) ns[i] = npv[i] = 0;
      for (int i = 0; i < A4_STAGES; ++i) cnt[i] = 0;
      uint64_t t_last = globaltimer_ns();
      while (ok) {
        bool done = true, progress = false;
#pragma unroll
        for (int hh = 0; hh < A4_HEADS; ++hh) {
          const int j = ns[hh];
          if (j < ntile) {
            done = false;
            const int s = j % A4_STAGES;
            if (mbar_test(&S.kv_full[s], (j / A4_STAGES) & 1) &&
                (j == 0 || mbar_test(&S.s_free[hh], (j - 1) & 1))) {
              tc_fence_after();
              const uint32_t q_base = smem_u32(S.Q[hh]);
              const uint32_t k_base = smem_u32(S.K[s]);
#pragma unroll
              for (int k = 0; k < AT_D / 16; ++k)
                umma_f16_ss(tmem + hh * 64u, smem_desc(q_base + k * 32, 16, 1024, kLayoutSw128),
                            smem_desc(k_base + k * 32, 16, 1024, kLayoutSw128), idesc_s, k != 0);
              umma_commit(&S.s_full[hh]);
              ns[hh] = j + 1;
              progress = true;
            }
          }
          const int jp = npv[hh];
          if (jp < ntile) {
            done = false;
            if (jp < ns[hh] && mbar_test(&S.p_full[hh], jp & 1)) {
              tc_fence_after();
              const int s = jp % A4_STAGES;
              const uint32_t a_base = smem_u32(S.P[hh]);
              const uint32_t v_base = smem_u32(S.V[s]);
#pragma unroll
              for (int k = 0; k < A4_BN / 16; ++k)
                umma_f16_ss(tmem + 256u + hh * 64u, smem_desc(a_base + k * 32, 16, 1024, kLayoutSw128),
                            smem_desc(v_base + k * 16 * AT_D * 2, 16, 1024, kLayoutSw128), idesc_o,
                            (jp | k) != 0);
              umma_commit(&S.pv_done[hh]);
              // the K/V stage of tile jp is released once all four heads' products
              // of that tile are issued (they complete in issue order)
              int c4 = 0;
#pragma unroll
              for (int i = 0; i < A4_STAGES; ++i)
                if (i == s) c4 = ++cnt[i];
              if (c4 == A4_HEADS) {
#pragma unroll
                for (int i = 0; i < A4_STAGES; ++i)
                  if (i == s) cnt[i] = 0;
                umma_commit(&S.kv_empty[s]);
              }
              npv[hh] = jp + 1;
              progress = true;
            }
          }
        }
        if (done) break;
        const uint64_t now = globaltimer_ns();
        if (progress) {
          t_last = now;
        } else if (now - t_last > kWaitLimitNs) {
          raise_error(err, kErrTimeout);
          ok = false;
        } else {
          __nanosleep(32);
        }
      }
    }
  } else {
    const int hh = (warp - 2) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // query row within the tile == TMEM lane
    const int tq = t0 + r;
    const int t = tk0 + r;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tmem + hh * 64u + lane_off;
    const uint32_t tO = tmem + 256u + hh * 64u + lane_off;
    auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
      const bool w = mbar_wait(bar, par, err);
      return __all_sync(0xffffffffu, w);
    };
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    for (int j = 0; j < ntile; ++j) {
      const int kb = kb0 + j * A4_BN;
      if (!wait_all(&S.s_full[hh], j & 1)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(tS, sr);
      tmem_ld32(tS + 32, sr + 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.s_free[hh]);
      // band mask on the edge tiles: valid key offsets of row t are (t - w - kb, t - kb]
      const bool edge = (kb + A4_BN - 1 > tk0) || (kb < tk0 + AT_BM - p.window);
      if (edge) {
        const int hi = tq < p.L ? t - kb : -1;
        const int lo_i = t - p.window - kb;
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i > hi || i <= lo_i) sr[i] = __float_as_uint(-INFINITY);
      }
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; i += 2)
        m8[(i >> 1) & 7] = fmax3(m8[(i >> 1) & 7], __uint_as_float(sr[i]), __uint_as_float(sr[i + 1]));
      const float mraw = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      const float mt = mraw * p.scale_log2;
      const bool need = mt > m_run + kRescaleThresh;
      float alpha = 1.f;
      if (need) {
        if (m_run != -INFINITY) alpha = exp2f(m_run - mt);
        l_run *= alpha;
        m_run = mt;
      }
      // O_h += P_h(j-1) V_{j-1} must be complete before O is rescaled and P rewritten
      if (j >= 1 && !wait_all(&S.pv_done[hh], (j - 1) & 1)) { ok = false; break; }
      tc_fence_after();
      if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t orr[16];
          tmem_ld16(tO + c * 16, orr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
          tmem_st16(tO + c * 16, orr);
        }
        tmem_wait_st();
      }
      const float msub = m_run == -INFINITY ? 0.f : m_run;
      const float2 nm2 = make_float2(-msub, -msub);
      float2 ls2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      unsigned char* prow = reinterpret_cast<unsigned char*>(S.P[hh]) + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {  // 16-byte chunk c holds keys 8c .. 8c + 7
        float e[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = c * 8 + 2 * q;
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), sc2, nm2);
          if (q < kPolyPairs) {
            const float2 y = exp2_poly2(x);
            e[2 * q] = y.x;
            e[2 * q + 1] = y.y;
          } else {
            e[2 * q] = ex2_approx(x.x);
            e[2 * q + 1] = ex2_approx(x.y);
          }
          ls2[q] = __fadd2_rn(ls2[q], make_float2(e[2 * q], e[2 * q + 1]));
        }
        *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) =
            make_uint4(pack_bf16(e[0], e[1]), pack_bf16(e[2], e[3]), pack_bf16(e[4], e[5]), pack_bf16(e[6], e[7]));
      }
      l_run += ((ls2[0].x + ls2[0].y) + (ls2[1].x + ls2[1].y)) + ((ls2[2].x + ls2[2].y) + (ls2[3].x + ls2[3].y));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.p_full[hh]);
    }
    if (ok && wait_all(&S.pv_done[hh], (ntile - 1) & 1)) {
      tc_fence_after();
      uint32_t orr[64];
      tmem_ld32(tO, orr);
      tmem_ld32(tO + 32, orr + 32);
      tmem_wait_ld();
      if (tq < p.L && l_run > 0.f && SAMBA_DCHECK(err, h0 + hh < p.Hq)) {
        const float inv = 1.f / l_run;
        bf16* op = p.o + ((int64_t)b * p.L + tq) * p.ld_o + (int64_t)(h0 + hh) * AT_D;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float f[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) f[q] = __uint_as_float(orr[c * 8 + q]) * inv;
          store8(op + c * 8, f);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// [B, L, H * d] rows of stride ld; boxes of 64 columns x `rows` rows (128B swizzle)
bool make_head_map(CUtensorMap* m, const void* base, int64_t ld, int H, int d, int L, int B, int rows) {
  uint64_t dims[3] = {(uint64_t)H * d, (uint64_t)L, (uint64_t)B};
  uint64_t strides[2] = {(uint64_t)ld, (uint64_t)ld * (uint64_t)L};
  uint32_t box[3] = {64, (uint32_t)rows, 1};
  return make_tmap(m, base, SAMBA_BF16, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

bool swa_tc_supported(const SwaArgs& a) {
  if (a.dtype != SAMBA_BF16 || (a.d != AT_D && a.d != H_D)) return false;
  if (a.ld_q % 8 || a.ld_k % 8 || a.ld_v % 8 || a.ld_o % 8) return false;
  if (!aligned16(a.q) || !aligned16(a.k) || !aligned16(a.v) || !aligned16(a.o)) return false;
  if (getenv("SAMBA_SWA_KERNEL") && getenv("SAMBA_SWA_KERNEL")[0] == 's') return false;
  return true;
}

samba_status launch_swa_tc(const SwaArgs& a, cudaStream_t st) {
  AtParams p;
  memset(&p, 0, sizeof(p));
  const int Lk = a.L + a.qoff;
  const int kv_rows = a.d == H_D ? H_BN : AT_BN;
  if (!make_head_map(&p.tmQ, a.q, a.ld_q, a.Hq, a.d, a.L, a.B, AT_BM) ||
      !make_head_map(&p.tmK, a.k, a.ld_k, a.Hkv, a.d, Lk, a.B, kv_rows) ||
      !make_head_map(&p.tmV, a.v, a.ld_v, a.Hkv, a.d, Lk, a.B, kv_rows))
    return SAMBA_ERR_CUDA;
  p.o = (bf16*)a.o;
  p.ld_o = a.ld_o;
  p.L = a.L;
  p.qoff = a.qoff;
  p.Lk = Lk;
  p.window = a.window;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  const int grp = a.Hq / a.Hkv;
  if (a.d == H_D) {
    const size_t smem = sizeof(AtHSmem) + 1024;
    if (!ensure_smem_attr(swa_tc256_kernel, smem)) return SAMBA_ERR_CUDA;
    dim3 grid((a.L + AT_BM - 1) / AT_BM, a.Hq, a.B);
    swa_tc256_kernel<<<grid, AT_THREADS, smem, st>>>(p, device_error_word());
    SAMBA_CHECK_LAUNCH();
    return SAMBA_OK;
  }
  const char* kenv = getenv("SAMBA_SWA_KERNEL");
  if (grp % A4_HEADS == 0 && !(kenv && (kenv[0] == '1' || kenv[0] == '2'))) {
    CUtensorMap tk, tv;
    if (!make_head_map(&tk, a.k, a.ld_k, a.Hkv, a.d, Lk, a.B, A4_BN) ||
        !make_head_map(&tv, a.v, a.ld_v, a.Hkv, a.d, Lk, a.B, A4_BN))
      return SAMBA_ERR_CUDA;
    p.tmK = tk;
    p.tmV = tv;
    const char* pe = getenv("SAMBA_SWA_POLY");
    const int poly = (pe && pe[0] >= '0' && pe[0] <= '3') ? pe[0] - '0' : 1;
    auto kern = poly == 0 ? swa_tc4_kernel<0> : poly == 2 ? swa_tc4_kernel<2> : poly == 3 ? swa_tc4_kernel<3>
                                                                                            : swa_tc4_kernel<1>;
    const size_t smem = sizeof(At4Smem) + 1024;
    if (!ensure_smem_attr(kern, smem)) return SAMBA_ERR_CUDA;
    dim3 grid((a.L + AT_BM - 1) / AT_BM, a.Hq / A4_HEADS, a.B);
    kern<<<grid, A4_THREADS, smem, st>>>(p, device_error_word());
    SAMBA_CHECK_LAUNCH();
    return SAMBA_OK;
  }
  if (grp % 2 == 0 && !(kenv && kenv[0] == '1')) {
    // share of the exponentials on the FMA pipe: SAMBA_SWA_POLY = 0..3 pairs of 4 (default 1)
    const char* pe = getenv("SAMBA_SWA_POLY");
    const int poly = (pe && pe[0] >= '0' && pe[0] <= '3') ? pe[0] - '0' : 1;
    auto kern = poly == 0 ? swa_tc2_kernel<0> : poly == 2 ? swa_tc2_kernel<2> : poly == 3 ? swa_tc2_kernel<3>
                                                                                            : swa_tc2_kernel<1>;
    const size_t smem = sizeof(At2Smem) + 1024;
    if (!ensure_smem_attr(kern, smem)) return SAMBA_ERR_CUDA;
    dim3 grid((a.L + AT_BM - 1) / AT_BM, a.Hq / 2, a.B);
    kern<<<grid, A2_THREADS, smem, st>>>(p, device_error_word());
    SAMBA_CHECK_LAUNCH();
    return SAMBA_OK;
  }
  const size_t smem = sizeof(AtSmem) + 1024;
  if (!ensure_smem_attr(swa_tc_kernel, smem)) return SAMBA_ERR_CUDA;
  dim3 grid((a.L + AT_BM - 1) / AT_BM, a.Hq, a.B);
  swa_tc_kernel<<<grid, AT_THREADS, smem, st>>>(p, device_error_word());
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

}  // namespace samba
