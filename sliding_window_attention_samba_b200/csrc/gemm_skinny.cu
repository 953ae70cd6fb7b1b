// Skinny projections for decode (M = batch <= 64 tokens): out = epi(X W^T).
//
// At batch 32 a decode step is bound by streaming the weights once, and the
// down/out projections have only N/128 = 16 tiles of 128 output features, far
// too few CTAs to pull HBM bandwidth.  Design:
//   * swap-AB on the tensor cores: the 128 weight rows of a tile are the UMMA M
//     side (TMEM lanes), the zero-padded batch is the UMMA N side (16..64);
//   * split-K across a thread-block cluster of S <= 8 CTAs (one n-tile per
//     cluster), each CTA streaming a K range of the weight tile through a
//     4-stage TMA ring into tcgen05.mma;
//   * the S fp32 partial tiles are pushed into their owner CTA's shared memory
//     (st.shared::cluster, feature-innermost) and each owner finalises 8
//     consecutive features of a batch row per thread with 16-byte accesses;
//     the epilogue (residual, SwiGLU, softplus+bias, RoPE at per-row
//     positions from a table or evaluated from the position) is applied in
//     the same kernel, so no partial sums ever reach HBM;
//   * decode-step folds: the short-conv step on in_proj's x columns, the new
//     token's k, v into the ring slot by the QKV projection, the position
//     advance by the step's last projection.
// No cluster multicast is used (each CTA loads its own tiles).
#include <stdlib.h>
#include <string.h>

#define SAMBA_TU_ID 5  // site id of this file in debug-check reports
#include "common.cuh"
#include "kernels.h"

namespace samba {

namespace {

constexpr int SK_BM = 128;     // weight rows (output features) per tile
constexpr int SK_BK = 64;
constexpr int SK_STAGES = 8;  // upper bound; the stage count is ring bytes / stage bytes
constexpr int SK_MAXB = 64;    // max padded batch
constexpr int SK_THREADS = 192;

// Shared memory: a ring of stages (W tile | W2 tile (SwiGLU) | X tile) that is
// reused, once every MMA has completed, for the fp32 partial tile(s) of the
// cluster reduction; barriers and the TMEM address live after it.
// 96 KB for single-weight projections: two CTAs fit an SM, so that (with
// programmatic dependent launch) the next projection's CTAs become resident and
// fetch their first weight stages while the previous projection's CTAs reduce
// and write their outputs.  200 KB for the SwiGLU pair: its stages carry two
// weight tiles, and bytes in flight matter more there than the overlap.
constexpr int SK_RING_BYTES = 96 * 1024;
constexpr int SK_RING_BYTES_DUAL = 200 * 1024;
// Receive buffers of the cluster reduction: recv[acc][src][batch][slot] with
// the slot (the owner's output features) innermost, padded by 4 floats, so that
// the reduction reads 8 consecutive features of one batch row as two 16-byte
// loads per source and writes them as one 16-byte store.
constexpr int SK_RED_PAD = 4;
// largest receive area: 2 accumulators x S sources x 64 rows x (128/S + 4) floats, S <= 8;
// one accumulator with S = 16 (the narrow projections' non-portable clusters)
static_assert(2 * SK_MAXB * (SK_BM + 8 * SK_RED_PAD) * 4 <= SK_RING_BYTES, "reduction tiles must fit in the ring");
static_assert(SK_MAXB * (SK_BM + 16 * SK_RED_PAD) * 4 <= SK_RING_BYTES, "reduction tiles must fit in the ring");

template <int kRing>
struct SkSmem {
  unsigned char ring[kRing];
  uint64_t full[SK_STAGES], empty[SK_STAGES], done;
  uint32_t tmem_base;
  float rn[SK_MAXB];  // norm fold: each batch row's RMS scale
};
template <int EPI> constexpr int sk_ring_bytes() { return EPI == kEpiSwiglu ? SK_RING_BYTES_DUAL : SK_RING_BYTES; }

struct SkParams {
  CUtensorMap tmW[3];
  CUtensorMap tmW2;
  CUtensorMap tmX;
  GemmArgs a;
  int MB;          // padded batch (UMMA N)
  int stages;      // ring stages in use
  int stage_bytes; // bytes per stage (multiple of 1024)
  int S;           // cluster size = K splits
  int kb_total, kps;
  int seg_start[3];
  double theta[64];  // RoPE without a table: base^(-2i/head_dim), i < head_dim / 2 (fp64)
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// All threads of all CTAs of the cluster (non-.aligned form: callers may arrive
// from diverged role branches).
// Returns 0; peer loads add it to their address so that they depend on the
// barrier and cannot be scheduled above it.
__device__ __forceinline__ uint32_t cluster_sync_all() {
  uint32_t tok;
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;\n\tmov.u32 %0, 0;"
               : "=r"(tok)::"memory");
  return tok;
}
// Peer shared-memory load.  Not volatile and no memory clobber: the loads are
// ordered by the cluster barrier before them, and this lets the compiler issue
// the loads of all peers back to back instead of one round trip at a time.
__device__ __forceinline__ float ld_dsmem_f32(const float* local_ptr, uint32_t rank, uint32_t tok) {
  uint32_t raddr;
  asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(raddr) : "r"(smem_u32(local_ptr) + tok), "r"(rank));
  float v;
  asm("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(raddr));
  return v;
}

// Fire-and-forget store of 4 floats into a peer CTA's shared memory.
__device__ __forceinline__ void st_dsmem_v4(const float* local_ptr, uint32_t rank, float4 v, uint32_t tok) {
  uint32_t raddr;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(raddr) : "r"(smem_u32(local_ptr) + tok), "r"(rank));
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(raddr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

__device__ __forceinline__ void st_dsmem_f32(const float* local_ptr, uint32_t rank, float v, uint32_t tok) {
  uint32_t raddr;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(raddr) : "r"(smem_u32(local_ptr) + tok), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(raddr), "f"(v) : "memory");
}

// (cos, sin) of pos * theta without a table: the angle is formed and reduced
// modulo 2*pi in fp64 (exact product up to 2^-53 relative, Cody-Waite
// two-term 2*pi), then evaluated in fp32 on [-pi, pi].
__device__ __forceinline__ float2 rope_cs_direct(double theta, int64_t p) {
  const double ang = (double)p * theta;
  const double k = rint(ang * 0.15915494309189535);  // 1 / (2 pi)
  double r = fma(-k, 6.283185307179586, ang);
  r = fma(-k, 2.4492935982947064e-16, r);
  float s, c;
  sincosf((float)r, &s, &c);
  return make_float2(c, s);
}

__device__ __forceinline__ float2 rope_cs_sk(const float2* __restrict__ tab, int half, int64_t p, int i) {
  const float2 c0 = tab[(0 * kRopeRadix + (p & 1023)) * half + i];
  const float2 c1 = tab[(1 * kRopeRadix + ((p >> 10) & 1023)) * half + i];
  const float2 c2 = tab[(2 * kRopeRadix + ((p >> 20) & 1023)) * half + i];
  const float cr = c0.x * c1.x - c0.y * c1.y, sr = c0.x * c1.y + c0.y * c1.x;
  return make_float2(cr * c2.x - sr * c2.y, cr * c2.y + sr * c2.x);
}

template <int EPI>
__global__ void __launch_bounds__(SK_THREADS, 2) gemm_skinny_kernel(const __grid_constant__ SkParams p, int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  SkSmem<sk_ring_bytes<EPI>()>& S =
      *reinterpret_cast<SkSmem<sk_ring_bytes<EPI>()>*>(smem_raw + smem_align_pad(smem_raw, 1024));
  const GemmArgs& a = p.a;
  const int warp = warp_id_sync();
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int ntile = blockIdx.x / p.S;
  const int n0 = ntile * SK_BM;  // first output feature of this tile
  const int kb_begin = (int)rank * p.kps;
  const int kb_end = min(p.kb_total, kb_begin + p.kps);
  const int nkb = max(0, kb_end - kb_begin);
  constexpr bool kDual = EPI == kEpiSwiglu;

  constexpr uint32_t kWBytes = SK_BM * SK_BK * 2;
  auto stW = [&](int s) { return S.ring + (size_t)s * p.stage_bytes; };
  auto stW2 = [&](int s) { return S.ring + (size_t)s * p.stage_bytes + kWBytes; };
  auto stX = [&](int s) { return S.ring + (size_t)s * p.stage_bytes + (kDual ? 2 : 1) * kWBytes; };
  float* red = reinterpret_cast<float*>(S.ring);  // [acc][row][SK_RED_PITCH], valid after `done`
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < SK_STAGES; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    mbar_init(&S.done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == 0) {
    if (elect_one()) {
      int seg = 0;
      while (seg < a.nseg - 1 && n0 >= p.seg_start[seg + 1]) ++seg;
      const int wrow = n0 - p.seg_start[seg];
      const uint32_t bytes = (uint32_t)(SK_BM * SK_BK * 2) * (kDual ? 2 : 1) + (uint32_t)p.MB * SK_BK * 2;
      // The weights are never written by a kernel: the first ring stages are
      // fetched before waiting for the previous kernel (programmatic dependent
      // launch), the activations only after it.
      const int npre = min(nkb, p.stages);
      for (int i = 0; i < npre; ++i) {
        mbar_arrive_expect_tx(&S.full[i], bytes);
        const int kx = (kb_begin + i) * SK_BK;
        tma_load_2d(stW(i), &p.tmW[seg], &S.full[i], kx, wrow);
        if (kDual) tma_load_2d(stW2(i), &p.tmW2, &S.full[i], kx, wrow);
      }
      pdl_wait();
      pdl_trigger();
      for (int i = 0; i < npre; ++i) tma_load_2d(stX(i), &p.tmX, &S.full[i], (kb_begin + i) * SK_BK, 0);
      for (int i = npre; i < nkb; ++i) {
        const int s = i % p.stages;
        if (!mbar_wait(&S.empty[s], ((i / p.stages) & 1) ^ 1, err)) break;
        mbar_arrive_expect_tx(&S.full[s], bytes);
        const int kx = (kb_begin + i) * SK_BK;
        tma_load_2d(stW(s), &p.tmW[seg], &S.full[s], kx, wrow);
        if (kDual) tma_load_2d(stW2(s), &p.tmW2, &S.full[s], kx, wrow);
        tma_load_2d(stX(s), &p.tmX, &S.full[s], kx, 0);
      }
    }
  } else {
    pdl_wait();  // the epilogue reads and writes activations
    pdl_trigger();
    // every kernel before this one has completed: the step's position may advance
    if (a.pos_inc && blockIdx.x == 0 && warp == 2)
      for (int i = lane; i < (int)a.M; i += 32) a.pos_inc[i] += 1;
  }
  if (warp == 1) {
    const uint32_t idesc = idesc_bf16_f32(SK_BM, p.MB);
    if (elect_one()) {
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % p.stages;
        if (!mbar_wait(&S.full[s], (i / p.stages) & 1, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t wb = smem_u32(stW(s)), w2b = smem_u32(stW2(s)), xb = smem_u32(stX(s));
#pragma unroll
        for (int k = 0; k < SK_BK / 16; ++k) {
          const uint64_t bd = smem_desc(xb + k * 32, 16, 1024, kLayoutSw128);
          umma_f16_ss(tmem, smem_desc(wb + k * 32, 16, 1024, kLayoutSw128), bd, idesc, (i | k) != 0);
          if (kDual)
            umma_f16_ss(tmem + SK_MAXB, smem_desc(w2b + k * 32, 16, 1024, kLayoutSw128), bd, idesc, (i | k) != 0);
        }
        umma_commit(&S.empty[s]);
      }
      if (ok) umma_commit(&S.done);
    }
  }
  // Every row of the tile has one owner rank that finalises it: contiguous
  // slices of 128/S rows, or, for RoPE tiles, the two rows (i, i + hd/2) of
  // each rotated pair together (slots [0, P) the first rows of the owner's P
  // pairs, [P, 2P) the second).  Receive buffers in the now idle ring.
  const bool rope_tile = EPI == kEpiRope && n0 < a.rope_cols;
  const int rows_per = SK_BM / p.S;
  const int pitch = rows_per + SK_RED_PAD;
  const int MB = p.MB;
  const int per_pairs = (SK_BM / 2) / p.S;
  auto owner_of = [&](int r, int& slot) -> int {
    if (rope_tile) {
      const int hd = a.head_dim, half = hd / 2;
      const int pair = (r / hd) * half + (r % half);
      slot = pair % per_pairs + ((r % hd) >= half ? per_pairs : 0);
      return pair / per_pairs;
    }
    slot = r % rows_per;
    return r / rows_per;
  };
  auto recv = [&](int acc, int src, int b) -> float* {
    return red + ((size_t)(acc * p.S + src) * MB + b) * pitch;
  };
  // the receive area (every source, batch row and slot) must fit the ring
  const bool area_ok = SAMBA_DCHECK(err, (size_t)(kDual ? 2 : 1) * p.S * MB * pitch * 4 <= sizeof(S.ring));
  uint32_t tok = 0;
  if (warp >= 2) {
    // TMEM -> registers (zeros if this CTA had no K range)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    if (a.ss_in) {
      // norm fold, while the MMAs run: row b's RMS scale from its norm_dim/8
      // partial sums of squares, in one fixed order (lane-strided, then a
      // butterfly), so that every CTA and every run gets the same value
      const int np = a.norm_dim / 8;
      for (int b = q; b < (int)a.M; b += 4) {
        const float* sp = a.ss_in + (int64_t)b * np;
        float s = 0.f;
        for (int j = lane; j < np; j += 32) s += sp[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) S.rn[b] = rsqrtf(s / (float)a.norm_dim + a.norm_eps);
      }
    }
    bool got = true;
    if (nkb > 0) got = __all_sync(0xffffffffu, mbar_wait(&S.done, 0, err));
    if (got) tc_fence_after();
    uint32_t v[2][SK_MAXB];
#pragma unroll
    for (int acc = 0; acc < (kDual ? 2 : 1); ++acc)
#pragma unroll
      for (int c = 0; c < SK_MAXB; c += 16)
        if (c < MB) {
          if (nkb > 0 && got) {
            tmem_ld16(tmem + acc * SK_MAXB + lane_off + c, &v[acc][c]);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[acc][c + i] = 0u;
          }
        }
    if (nkb > 0 && got) tmem_wait_ld();
    tc_fence_before();
    // all MMAs of all CTAs are complete once everyone passes this barrier, so
    // every ring may be overwritten by the pushes below
    tok = cluster_sync_all();
    int slot;
    const int own = owner_of(row, slot);
    const bool fits = area_ok && SAMBA_DCHECK(err, own >= 0 && own < p.S && slot >= 0 && slot < rows_per);
    // the 32 lanes of a warp hold consecutive rows, i.e. consecutive slots of
    // one or two owners: each store below writes a contiguous run of the peer
#pragma unroll
    for (int acc = 0; acc < (kDual ? 2 : 1) && fits; ++acc)
#pragma unroll
      for (int c = 0; c < SK_MAXB; ++c)
        if (c < MB) st_dsmem_f32(recv(acc, (int)rank, c) + slot, own, __uint_as_float(v[acc][c]), tok);
  } else {
    tc_fence_before();
    tok = cluster_sync_all();
  }
  tok = cluster_sync_all();  // every push has landed; nothing remote is touched after this

  // ---- reduction of the S received partials of this rank's rows + epilogue:
  // one item = 8 consecutive output features of one batch row (RoPE: 8 pairs)
  const int M = (int)a.M;
  bf16* out = (bf16*)a.out;
  const int G = (rope_tile ? per_pairs : rows_per) / 8;  // feature groups per batch row
  for (int e = threadIdx.x; e < G * M && area_ok; e += SK_THREADS) {
    const int g = e % G, b = e / G;  // consecutive threads -> consecutive groups of one row
    if (rope_tile) {
      const int hd = a.head_dim, half = hd / 2;
      const int pair0 = (int)rank * per_pairs + 8 * g;
      const int hh = pair0 / half, i0 = pair0 % half;  // 8 pairs inside one head (8 | half)
      const int r1 = hh * hd + i0, r2 = r1 + half;
      if (!SAMBA_DCHECK(err, i0 + 8 <= half && r2 + 8 <= SK_BM)) continue;
      const int64_t pos = a.pos_dev ? a.pos_dev[b] : a.pos0 + b % a.seq_len;
      float x1[8], x2[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) x1[j] = x2[j] = 0.f;
      const float rn = a.ss_in ? S.rn[b] : 1.f;
      for (int sidx = 0; sidx < p.S; ++sidx) {
        const float* q = recv(0, sidx, b);
        const float4 a0 = *reinterpret_cast<const float4*>(q + 8 * g);
        const float4 a1 = *reinterpret_cast<const float4*>(q + 8 * g + 4);
        const float4 c0 = *reinterpret_cast<const float4*>(q + per_pairs + 8 * g);
        const float4 c1 = *reinterpret_cast<const float4*>(q + per_pairs + 8 * g + 4);
        x1[0] += a0.x; x1[1] += a0.y; x1[2] += a0.z; x1[3] += a0.w;
        x1[4] += a1.x; x1[5] += a1.y; x1[6] += a1.z; x1[7] += a1.w;
        x2[0] += c0.x; x2[1] += c0.y; x2[2] += c0.z; x2[3] += c0.w;
        x2[4] += c1.x; x2[5] += c1.y; x2[6] += c1.z; x2[7] += c1.w;
      }
      float o1[8], o2[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        x1[j] *= rn;
        x2[j] *= rn;
        const float2 cs = a.rope_tab ? rope_cs_sk(a.rope_tab, half, pos, i0 + j) : rope_cs_direct(p.theta[i0 + j], pos);
        o1[j] = x1[j] * cs.x - x2[j] * cs.y;
        o2[j] = x2[j] * cs.x + x1[j] * cs.y;
      }
      bf16* o = out + (int64_t)b * a.ldo + n0;
      if (n0 + r1 < a.N) store8(o + r1, o1);
      if (n0 + r2 < a.N) store8(o + r2, o2);
      const int kc = n0 + r1 - a.ring_k_col;  // rotated key columns also go to the ring
      if (a.k_ring && kc >= 0 && kc < a.ring_kvw) {
        if (pos < 0) {
          raise_error(err, kErrDevice);  // a corrupted position: nothing is written outside the ring
        } else if (SAMBA_DCHECK(err, kc + half + 8 <= a.ring_kvw)) {
          bf16* kr = (bf16*)a.k_ring + ((int64_t)b * a.ring_window + pos % a.ring_window) * a.ring_kvw;
          store8(kr + kc, o1);
          store8(kr + kc + half, o2);
        }
      }
    } else {
      const int n = n0 + (int)rank * rows_per + 8 * g;
      if (n >= a.N) continue;  // N % 8 == 0: a group is wholly inside or outside
      if (!SAMBA_DCHECK(err, n + 8 <= a.N && b < M)) continue;
      float extra[8];
      const float rn = a.ss_in ? S.rn[b] : 1.f;
      if (EPI == kEpiResid) load8((const bf16*)a.resid + (int64_t)b * a.ldr + n, extra);
      if (EPI == kEpiSoftplus) load8(a.bias + n, extra);
      // norm fold: the next norm's gain, fetched together with the residual
      float4 gn0 = make_float4(0.f, 0.f, 0.f, 0.f), gn1 = gn0;
      if (EPI == kEpiResid && a.ss_out) {
        gn0 = reinterpret_cast<const float4*>(a.g_next + n)[0];
        gn1 = reinterpret_cast<const float4*>(a.g_next + n)[1];
      }
      float v[8], v2[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = v2[j] = 0.f;
      for (int sidx = 0; sidx < p.S; ++sidx) {
        const float* q = recv(0, sidx, b) + 8 * g;
        const float4 a0 = *reinterpret_cast<const float4*>(q);
        const float4 a1 = *reinterpret_cast<const float4*>(q + 4);
        v[0] += a0.x; v[1] += a0.y; v[2] += a0.z; v[3] += a0.w;
        v[4] += a1.x; v[5] += a1.y; v[6] += a1.z; v[7] += a1.w;
        if (kDual) {
          const float* q2 = recv(1, sidx, b) + 8 * g;
          const float4 c0 = *reinterpret_cast<const float4*>(q2);
          const float4 c1 = *reinterpret_cast<const float4*>(q2 + 4);
          v2[0] += c0.x; v2[1] += c0.y; v2[2] += c0.z; v2[3] += c0.w;
          v2[4] += c1.x; v2[5] += c1.y; v2[6] += c1.z; v2[7] += c1.w;
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        v[j] *= rn;
        v2[j] *= rn;
        if (EPI == kEpiSwiglu) v[j] = v[j] * (v2[j] * sigmoid_fast(v2[j]));
        if (EPI == kEpiSoftplus) v[j] = softplus_1x(v[j] + extra[j]);
      }
      if (EPI == kEpiResid) {
        if (a.tap) store8((bf16*)a.tap + (int64_t)b * a.ldt + n, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] += extra[j];
        if (a.ss_out) {  // the next norm's input: the stored row times its gain, and the row's sum of squares
          float xg[8], sq = 0.f;
          const float gg[8] = {gn0.x, gn0.y, gn0.z, gn0.w, gn1.x, gn1.y, gn1.z, gn1.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float vb = __bfloat162float(__float2bfloat16_rn(v[j]));
            sq = fmaf(vb, vb, sq);
            xg[j] = vb * gg[j];
          }
          store8((bf16*)a.xg_out + (int64_t)b * a.ldo + n, xg);
          a.ss_out[(int64_t)b * (a.N / 8) + n / 8] = sq;
        }
      }
      if (EPI == kEpiNone && a.conv_u && n < a.conv_cols) {
        // short convolution step of channels n .. n+7 (the state keeps inputs as stored, in bf16)
        if (!SAMBA_DCHECK(err, n + 8 <= a.conv_cols)) continue;
        bf16* sp = (bf16*)a.conv_state + ((int64_t)b * a.conv_cols + n) * 3;
        uint4 raw[3];
#pragma unroll
        for (int j = 0; j < 3; ++j) raw[j] = reinterpret_cast<const uint4*>(sp)[j];
        const bf16* sv = reinterpret_cast<const bf16*>(raw);  // [channel][3], oldest first
        bf16 xs[8];
        float wv[32], uo[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) xs[j] = __float2bfloat16_rn(v[j]);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 w4 = reinterpret_cast<const float4*>(a.conv_w + (int64_t)(n + j) * 4)[0];
          wv[4 * j] = w4.x;
          wv[4 * j + 1] = w4.y;
          wv[4 * j + 2] = w4.z;
          wv[4 * j + 3] = w4.w;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float acc = a.conv_b ? a.conv_b[n + j] : 0.f;
          acc = fmaf(wv[4 * j], __bfloat162float(sv[3 * j]), acc);
          acc = fmaf(wv[4 * j + 1], __bfloat162float(sv[3 * j + 1]), acc);
          acc = fmaf(wv[4 * j + 2], __bfloat162float(sv[3 * j + 2]), acc);
          acc = fmaf(wv[4 * j + 3], __bfloat162float(xs[j]), acc);
          uo[j] = acc * sigmoid_fast(acc);
        }
        bf16 ns[24];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          ns[3 * j] = sv[3 * j + 1];
          ns[3 * j + 1] = sv[3 * j + 2];
          ns[3 * j + 2] = xs[j];
        }
#pragma unroll
        for (int j = 0; j < 3; ++j) reinterpret_cast<uint4*>(sp)[j] = reinterpret_cast<const uint4*>(ns)[j];
        store8((bf16*)a.conv_u + (int64_t)b * a.conv_cols + n, uo);
        continue;
      }
      store8(out + (int64_t)b * a.ldo + n, v);
      if (EPI == kEpiRope && a.v_ring) {  // value columns also go to the ring
        const int vc = n - a.ring_v_col;
        const int64_t pos = a.pos_dev[b];
        if (vc >= 0 && vc < a.ring_kvw) {
          if (pos < 0)
            raise_error(err, kErrDevice);
          else if (SAMBA_DCHECK(err, vc + 8 <= a.ring_kvw))
            store8((bf16*)a.v_ring + ((int64_t)b * a.ring_window + pos % a.ring_window) * a.ring_kvw + vc, v);
        }
      }
    }
  }
  (void)tok;
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace

bool gemm_skinny_supported(const GemmArgs& a) {
  if (a.dtype != SAMBA_BF16 || a.M < 1 || a.M > SK_MAXB || a.K % SK_BK) return false;
  if (a.lda % 8 || a.ldo % 8 || !aligned16(a.A) || !aligned16(a.out)) return false;
  // the epilogue moves 8 consecutive features at a time (16-byte accesses)
  if (a.N % 8) return false;
  if (a.epi == kEpiResid && (a.ldr % 8 || !aligned16(a.resid) || (a.tap && (a.ldt % 8 || !aligned16(a.tap)))))
    return false;
  if (a.epi == kEpiSoftplus && !aligned16(a.bias)) return false;
  if (a.epi == kEpiRope && (a.head_dim < 16 || SK_BM % a.head_dim || a.rope_cols % SK_BM)) return false;
  if (a.epi == kEpiRope && !a.rope_tab && !(a.rope_base > 0.f && a.head_dim / 2 <= 64)) return false;
  int start = 0;
  for (int s = 0; s < a.nseg; ++s) {
    if (!aligned16(a.seg[s].W) || (a.seg[s].W2 && !aligned16(a.seg[s].W2))) return false;
    if (s + 1 < a.nseg && (start + a.seg[s].n) % SK_BM) return false;  // tiles never straddle segments
    start += a.seg[s].n;
  }
  if (a.epi == kEpiSwiglu && a.nseg != 1) return false;
  if (a.ss_in && (a.norm_dim <= 0 || a.norm_dim % 8)) return false;
  if (a.ss_out && (a.epi != kEpiResid || !a.g_next || !a.xg_out || !aligned16(a.g_next) || !aligned16(a.xg_out)))
    return false;
  if (a.conv_u) {  // the short convolution step on columns [0, conv_cols)
    if (a.epi != kEpiNone || a.conv_k != 4 || a.conv_cols % 8 || a.conv_cols > a.N || !a.conv_w || !a.conv_state ||
        !aligned16(a.conv_w) || !aligned16(a.conv_state) || !aligned16(a.conv_u))
      return false;
  }
  if (a.k_ring || a.v_ring) {  // ring columns: whole 8-column groups, rotated keys inside the RoPE columns
    if (a.epi != kEpiRope || !a.pos_dev || a.ring_window < 1 || a.ring_kvw % 8 || a.ring_k_col % 8 ||
        a.ring_v_col % 8 || !aligned16(a.k_ring) || !aligned16(a.v_ring) ||
        a.ring_k_col + a.ring_kvw > a.rope_cols || a.ring_v_col < a.rope_cols)
      return false;
  }
  const char* e = getenv("SAMBA_GEMM_KERNEL");
  return !(e && e[0] == 's');
}

template <int EPI>
static samba_status skinny_launch(const SkParams& p, int ntiles, cudaStream_t st) {
  const size_t smem = sizeof(SkSmem<sk_ring_bytes<EPI>()>) + 1024;
  auto kern = gemm_skinny_kernel<EPI>;
  if (!ensure_smem_attr(kern, smem)) return SAMBA_ERR_CUDA;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(ntiles * p.S, 1, 1);
  cfg.blockDim = dim3(SK_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.a.pdl ? 2 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p, device_error_word());
  if (e != cudaSuccess) return note_cuda_failure("cudaLaunchKernelEx (skinny projection cluster)", e);
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

// Clusters of 16 CTAs (non-portable) for the narrow projections: whether this
// device launches them for the kernel of epilogue EPI, asked once per device
// and never under stream capture (a capture-time call could invalidate it).
template <int EPI>
static bool cluster16_ok(cudaStream_t st) {
  static int state[64];  // per device: 0 not asked yet, 1 yes, -1 no
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (state[dev]) return state[dev] > 0;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return false;
  const size_t smem = sizeof(SkSmem<sk_ring_bytes<EPI>()>) + 1024;
  auto kern = gemm_skinny_kernel<EPI>;
  bool ok = ensure_smem_attr(kern, smem) &&
            cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
  if (ok) {
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(16, 1, 1);
    cfg.blockDim = dim3(SK_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 16;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    ok = cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n >= 1;
  }
  if (!ok) (void)cudaGetLastError();  // a refusal here only means portable clusters
  state[dev] = ok ? 1 : -1;
  return ok;
}

static bool cluster16_ok_epi(int epi, cudaStream_t st) {
  switch (epi) {
    case kEpiNone: return cluster16_ok<kEpiNone>(st);
    case kEpiResid: return cluster16_ok<kEpiResid>(st);
    case kEpiSoftplus: return cluster16_ok<kEpiSoftplus>(st);
  }
  return false;  // SwiGLU (two accumulators) and RoPE (8-pair items) keep S <= 8
}

samba_status launch_gemm_skinny(const GemmArgs& a, cudaStream_t st) {
  if (!gemm_skinny_supported(a)) return SAMBA_ERR_UNSUPPORTED;
  SkParams p;
  memset(&p, 0, sizeof(p));
  p.a = a;
  p.MB = (int)((a.M + 15) / 16) * 16;
  if (a.epi == kEpiRope && !a.rope_tab)
    for (int i = 0; i < a.head_dim / 2; ++i) p.theta[i] = pow((double)a.rope_base, -2.0 * i / (double)a.head_dim);
  {
    const int xb = ((p.MB * SK_BK * 2) + 1023) / 1024 * 1024;
    p.stage_bytes = (a.epi == kEpiSwiglu ? 2 : 1) * SK_BM * SK_BK * 2 + xb;
    p.stages = (a.epi == kEpiSwiglu ? SK_RING_BYTES_DUAL : SK_RING_BYTES) / p.stage_bytes;
    if (p.stages > SK_STAGES) p.stages = SK_STAGES;
  }
  const int ntiles = (a.N + SK_BM - 1) / SK_BM;
  p.kb_total = a.K / SK_BK;
  // splits: about one CTA per SM (one wave; the SM's second CTA slot is left to
  // the neighbouring projection), at most 8 (portable cluster size; 16 below)
  // and at least one k-block each
  const int want = num_sms() / ntiles;
  int S = 1;
  while (S * 2 <= want && S * 2 <= 8 && S * 2 <= p.kb_total) S *= 2;
  // a projection too narrow to fill the SMs with 8-CTA clusters (x_proj: two
  // tiles) splits K 16 ways where the device launches 16-CTA clusters
  if (S == 8 && want >= 16 && p.kb_total >= 16 && cluster16_ok_epi(a.epi, st)) S = 16;
  p.S = S;
  p.kps = (p.kb_total + S - 1) / S;
  {
    uint64_t dims[2] = {(uint64_t)a.K, (uint64_t)a.M};
    uint64_t strides[1] = {(uint64_t)a.lda};
    uint32_t box[2] = {SK_BK, (uint32_t)p.MB};
    if (!make_tmap(&p.tmX, a.A, SAMBA_BF16, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return SAMBA_ERR_CUDA;
  }
  int start = 0;
  for (int s = 0; s < a.nseg; ++s) {
    p.seg_start[s] = start;
    uint64_t dims[2] = {(uint64_t)a.K, (uint64_t)a.seg[s].n};
    uint64_t strides[1] = {(uint64_t)a.K};
    uint32_t box[2] = {SK_BK, SK_BM};
    if (!make_tmap(&p.tmW[s], a.seg[s].W, SAMBA_BF16, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return SAMBA_ERR_CUDA;
    if (a.epi == kEpiSwiglu &&
        !make_tmap(&p.tmW2, a.seg[s].W2, SAMBA_BF16, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return SAMBA_ERR_CUDA;
    start += a.seg[s].n;
  }
  switch (a.epi) {
    case kEpiNone: return skinny_launch<kEpiNone>(p, ntiles, st);
    case kEpiResid: return skinny_launch<kEpiResid>(p, ntiles, st);
    case kEpiSwiglu: return skinny_launch<kEpiSwiglu>(p, ntiles, st);
    case kEpiSoftplus: return skinny_launch<kEpiSoftplus>(p, ntiles, st);
    case kEpiRope: return skinny_launch<kEpiRope>(p, ntiles, st);
  }
  return SAMBA_ERR_INVALID_ARG;
}

}  // namespace samba
