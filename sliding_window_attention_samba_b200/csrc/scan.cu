// Chunked selective scan (S6) for sm_100a.
//
// Computes, per batch row b and channel d [Samba 3.4 "The State Space Model
// Update (S6)", "Input-Dependent Selective Gating", "Gated Output"]:
//   Delta_t = softplus(dt_t + bias)            (or dt_t + bias)
//   h_t     = exp(Delta_t A) (.) h_{t-1} + Delta_t u_t B_t
//   y_t     = <C_t, h_t> + D u_t,   y_t *= SiLU(z_t)
//
// Design (one CTA = 16 channels of one batch row for the whole sequence, two
// CTAs per SM):
//   * 64-token chunks of u, dt, z (16 channels wide) and B, C (16 wide) are
//     staged through shared memory by TMA, kStages deep.
//   * Lane l of every warp owns channel l & 15 and half of its 16 fp32 states
//     (l >> 4 selects states 0-7 or 8-15).  Warp w owns tokens [8w, 8w + 8) of
//     every chunk.
//   * Each warp converts its own 8 rows once (B, C to fp32; Delta, Delta u,
//     the SiLU(z) gate and D u gate per token and channel), so the walks never
//     repeat per-token work between the two lanes of a channel.
//   * Walk 1: each lane runs its 8 tokens from a zero state, keeping the 8x8
//     decays exp(Delta A) in registers (one exp per element), and forms the
//     slice aggregate (product of decays P, end state H).
//   * Carry chain: warp w waits for its entry state E_w (an mbarrier per warp
//     slot), passes E_{w+1} = P (.) E_w + H to warp w + 1 through shared memory,
//     warp 7 hands the next chunk's entry state to warp 0.  There is no
//     CTA-wide barrier in the steady state: warps drift one hop apart, so the
//     exp-heavy walk 1 of one warp overlaps the FMA-heavy walk 2 of another.
//   * Walk 2: each lane re-runs its tokens from E_w with the cached decays,
//     the two lanes of a channel add their partial read-outs with one shuffle
//     per token pair, and y goes to a shared tile written back by a TMA store.
//   * Warp 7's lane 0 recycles input stages (once every warp converted the
//     chunk) and stores y tiles (once every warp wrote its rows).
// Every wait is bounded (error word on timeout); a timed-out CTA drains its
// own copies in flight before it returns.
//
// With the dt projection folded in (kDt, bf16, dt_rank R <= 128, R % 16 == 0)
// [Samba 3.4 "Input-Dependent Selective Gating": Delta = softplus(dt_low
// W_dt^T + b)], the stages carry the chunk's rows of dt_low (128B-swizzled
// boxes of 64 columns) instead of Delta, the CTA keeps its 16 rows of W_dt in
// shared memory, and each warp forms Delta for its 8 tokens x 16 channels with
// m16n8k16 tensor-core products (its 8 token rows repeated as the upper 8 rows
// of the A tile) before the conversion, so Delta never goes through memory.
#define SAMBA_TU_ID 6  // site id of this file in debug-check reports
#include "common.cuh"
#include "kernels.h"

namespace samba {

namespace {

constexpr int kCh = 16;               // channels per CTA
constexpr int kWarps = 8;             // token slices per chunk
constexpr int kTs = 8;                // tokens per warp slice
constexpr int kChunk = kWarps * kTs;  // 64 tokens
constexpr int kN = 16;                // state size
constexpr int kHalf = 8;              // states per lane
constexpr int kThreads = kWarps * 32;
constexpr int kYBuf = 3;              // y tiles in flight
constexpr int kBCPitch = 2 * kN + 4;  // 36 floats: rows 16 bytes apart in the bank space

template <typename T> struct ScanCfg { static constexpr int kStages = sizeof(T) == 2 ? 4 : 2; };

constexpr int kDtBox = 64;      // dt_low columns per TMA box (128 bytes of bf16)
constexpr int kDtMaxBoxes = 2;  // dt_rank <= 128 on the folded path
constexpr int kDtMaxR = kDtBox * kDtMaxBoxes;

template <typename T, bool kDt>
struct ScanSmem {
  static constexpr int S = kDt ? 2 : ScanCfg<T>::kStages;
  bf16 dtl[kDt ? S : 1][kDtMaxBoxes][kDt ? kChunk * kDtBox : 64];  // dt_low rows, 128B-swizzled (kDt)
  bf16 Wd[kDt ? kCh : 1][kDt ? kDtMaxR + 8 : 64];                 // the CTA's rows of W_dt (kDt)
  alignas(128) T u[S][kChunk * kCh];  // [token][channel]
  T dt[kDt ? 1 : S][kChunk * kCh];
  T z[S][kChunk * kCh];
  T Bm[S][kChunk * kN];  // [token][state]
  T Cm[S][kChunk * kN];
  T y[kYBuf][kChunk * kCh];
  float BC[kWarps][kTs][kBCPitch];  // each warp's rows: B | C in fp32 (row padded: conflict-free stores)
  float2 dd[kWarps][kTs][kCh];     // (Delta, Delta u)
  float2 gg[kWarps][kTs][kCh];     // (gate, D u gate)
  float4 E[2][kWarps][2][32];      // entry states [chunk parity][warp slot][state quad][lane]
  uint64_t full[S];                // stage landed (TMA transaction count)
  uint64_t sfree[S];               // every warp converted the stage's chunk (8 arrivals)
  uint64_t ydone[kYBuf];           // every warp wrote its y rows (8 arrivals)
  uint64_t eready[kWarps];         // entry state of slot w published (32 arrivals)
  int abort;
};

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

__device__ __forceinline__ void ldsm_x4(uint32_t* r, const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row_addr)));
}
__device__ __forceinline__ void mma_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <typename T, bool kSoftplus, bool kHasZ, bool kDt>
__global__ void __launch_bounds__(kThreads, 2)
    scan_chunked_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_dt,
                        const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_B,
                        const __grid_constant__ CUtensorMap tm_C, const __grid_constant__ CUtensorMap tm_y,
                        const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                        const float* __restrict__ Dskip, const float* __restrict__ h0, float* __restrict__ hT,
                        int L, int D, int* err, int stop_chunk, uint64_t wait_limit_ns,
                        const bf16* __restrict__ W_dt, int R) {
  using Smem = ScanSmem<T, kDt>;
  constexpr int S = Smem::S;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem& Sm = *reinterpret_cast<Smem*>(smem_raw + smem_align_pad(smem_raw, 1024));

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int ch = lane & 15;   // channel within the CTA
  const int hf = lane >> 4;   // state half
  const int d0 = blockIdx.x * kCh;
  const int b = blockIdx.y;
  const int d = d0 + ch;
  const int nchunk = (L + kChunk - 1) / kChunk;
  const bool producer = warp == kWarps - 1 && lane == 0;

  constexpr uint32_t kStageBytes = (3 * kChunk * kCh + 2 * kChunk * kN) * sizeof(T);
  const int nbox = kDt ? (R + kDtBox - 1) / kDtBox : 0;
  const uint32_t stage_bytes = (kHasZ ? kStageBytes : kStageBytes - kChunk * kCh * sizeof(T)) -
                               (kDt ? kChunk * kCh * sizeof(T) - (uint32_t)nbox * kChunk * kDtBox * 2u : 0u);
  if constexpr (kDt) {  // the CTA's 16 rows of W_dt (16-byte pieces; R % 16 == 0)
    const int nv = R / 8;
    for (int e = tid; e < kCh * nv; e += kThreads) {
      const int r = e / nv, k = e % nv;
      *reinterpret_cast<uint4*>(&Sm.Wd[r][k * 8]) =
          *reinterpret_cast<const uint4*>(W_dt + (size_t)(d0 + r) * R + k * 8);
    }
  }

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&Sm.full[s], 1);
      mbar_init(&Sm.sfree[s], kWarps);
    }
    for (int i = 0; i < kYBuf; ++i) mbar_init(&Sm.ydone[i], kWarps);
    for (int w = 0; w < kWarps; ++w) mbar_init(&Sm.eready[w], 32);
    Sm.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // Bounded wait that also gives up once another warp of the CTA gave up.
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
      if (mbar_try_wait(bar, parity)) return true;
      if ((it & 15u) == 15u) {
        if (*reinterpret_cast<volatile int*>(&Sm.abort)) return false;
        if (globaltimer_ns() - t0 > wait_limit_ns) {
          raise_error(err, kErrTimeout);
          *reinterpret_cast<volatile int*>(&Sm.abort) = 1;
          return false;
        }
      }
    }
  };

  // The carry hand-off is on the critical path of every chunk: poll it without
  // suspending (a suspended waiter resumes later than a polling one), bounded.
  auto wait_spin = [&](uint64_t* bar, uint32_t parity) -> bool {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
      if (mbar_test(bar, parity)) return true;
      if ((it & 255u) == 255u) {
        if (*reinterpret_cast<volatile int*>(&Sm.abort)) return false;
        if (globaltimer_ns() - t0 > wait_limit_ns) {
          raise_error(err, kErrTimeout);
          *reinterpret_cast<volatile int*>(&Sm.abort) = 1;
          return false;
        }
      }
    }
  };

  int issued = 0;  // chunks whose loads the producer issued
  auto issue = [&](int c) {
    if (c >= stop_chunk || c >= nchunk) return;  // failure-detection test hook: nothing issued past stop
    const int s = c % S;
    const int t0 = c * kChunk;
    mbar_arrive_expect_tx(&Sm.full[s], stage_bytes);
    tma_load_3d(Sm.u[s], &tm_u, &Sm.full[s], d0, t0, b);
    if constexpr (kDt) {
      for (int k = 0; k < nbox; ++k) tma_load_3d(Sm.dtl[s][k], &tm_dt, &Sm.full[s], k * kDtBox, t0, b);
    } else {
      tma_load_3d(Sm.dt[s], &tm_dt, &Sm.full[s], d0, t0, b);
    }
    if (kHasZ) tma_load_3d(Sm.z[s], &tm_z, &Sm.full[s], d0, t0, b);
    tma_load_3d(Sm.Bm[s], &tm_B, &Sm.full[s], 0, t0, b);
    tma_load_3d(Sm.Cm[s], &tm_C, &Sm.full[s], 0, t0, b);
    issued = c + 1;
  };
  if (producer) {
    tma_prefetch_desc(&tm_u);
    tma_prefetch_desc(&tm_dt);
    tma_prefetch_desc(&tm_B);
    tma_prefetch_desc(&tm_C);
    tma_prefetch_desc(&tm_y);
    if (kHasZ) tma_prefetch_desc(&tm_z);
    for (int c = 0; c < S; ++c) issue(c);
  }

  // Walk constants: A * log2(e) for this lane's 8 states, as pairs.
  float2 A2[kHalf / 2];
#pragma unroll
  for (int k = 0; k < kHalf / 2; ++k) {
    const float* a = A_log + (size_t)d * kN + hf * kHalf + 2 * k;
    A2[k] = make_float2(-expf(a[0]) * 1.4426950408889634f, -expf(a[1]) * 1.4426950408889634f);
  }
  // Conversion-role constants: this lane's channel; row pr of the B | C runs.
  const int pr = lane >> 2;
  const float bias1 = dt_bias ? dt_bias[d] : 0.f;
  const float D1 = Dskip ? Dskip[d] : 0.f;
  // folded dt projection: this lane's (token, channel) entries are the
  // accumulator places of the m16n8k16 products: token lane / 4 of the warp's
  // 8, channels 2q, 2q+1 (n-tile 0) and 8+2q, 9+2q (n-tile 1), q = lane % 4
  float biasq[4] = {0.f, 0.f, 0.f, 0.f}, Dq[4] = {0.f, 0.f, 0.f, 0.f};
  if (kDt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = d0 + (e >> 1) * 8 + 2 * (lane & 3) + (e & 1);
      biasq[e] = dt_bias ? dt_bias[c] : 0.f;
      Dq[e] = Dskip ? Dskip[c] : 0.f;
    }
  }

  bool ok = true;
  int consumed = 0;  // chunks whose stage this warp saw land
  for (int c = 0; c < nchunk && ok; ++c) {
    const int s = c % S;
    // ---- this warp's rows of chunk c: wait for the stage, convert once
    // (every decision to stop is taken by the whole warp, so that no lane
    // leaves the loop while the others still meet at a warp barrier)
    if (!__all_sync(0xffffffffu, wait(&Sm.full[s], (c / S) & 1))) { ok = false; break; }
    consumed = c + 1;
    if constexpr (kDt) {
      // Delta_pre[8 tokens x 16 channels] = dt_low rows x W_dt^T on the tensor cores
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      const int arow = warp * kTs + (lane & 7);  // rows 8..15 of the A tile repeat rows 0..7
      for (int ks = 0; ks < R / 16; ++ks) {
        const int box = ks >> 2;
        const int acol = (ks & 3) * 16 + ((lane >> 4) & 1) * 8;  // column within the 64-column box
        const unsigned char* abase = reinterpret_cast<const unsigned char*>(Sm.dtl[s][box]);
        uint32_t af[4], bfr[4];
        ldsm_x4(af, abase + arow * 128 + ((((acol >> 3) ^ arow) & 7) << 4));
        ldsm_x4(bfr, &Sm.Wd[((lane >> 4) & 1) * 8 + (lane & 7)][ks * 16 + ((lane >> 3) & 1) * 8]);
        mma_16816(acc[0], af, bfr[0], bfr[1]);
        mma_16816(acc[1], af, bfr[2], bfr[3]);
      }
      const int i = lane >> 2;  // token within the warp's slice
      const int row = warp * kTs + i;
      const int tg = c * kChunk + row;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int chq = (e >> 1) * 8 + 2 * (lane & 3) + (e & 1);
        float delta = acc[e >> 1][e & 1] + biasq[e];
        delta = softplus_1x(delta);
        float uv = Elt<T>::to_f(Sm.u[s][row * kCh + chq]);
        if (tg >= L) { delta = 0.f; uv = 0.f; }  // padding past the sequence: state unchanged
        float g = 1.f;
        if (kHasZ) {
          const float zv = Elt<T>::to_f(Sm.z[s][row * kCh + chq]);
          g = zv * sigmoid_fast(zv);
        }
        Sm.dd[warp][i][chq] = make_float2(delta, delta * uv);
        Sm.gg[warp][i][chq] = make_float2(g, Dq[e] * uv * g);
      }
    }
    {
      // per (token, channel): lane = (channel ch, token half hf), tokens hf*4 .. hf*4+3
      // of the warp's slice, so each store writes whole 128-byte rows
#pragma unroll
      for (int k = 0; k < 4 && !kDt; ++k) {
        const int i = hf * 4 + k;
        const int row = warp * kTs + i;
        const int tg = c * kChunk + row;
        float delta = Elt<T>::to_f(Sm.dt[s][row * kCh + ch]) + bias1;
        if (kSoftplus) {
          if constexpr (sizeof(T) == 4) delta = softplus_acc(delta);
          else delta = softplus_1x(delta);
        }
        float uv = Elt<T>::to_f(Sm.u[s][row * kCh + ch]);
        if (tg >= L) { delta = 0.f; uv = 0.f; }  // padding past the sequence: state unchanged
        float g = 1.f;
        if (kHasZ) {
          const float zv = Elt<T>::to_f(Sm.z[s][row * kCh + ch]);
          if constexpr (sizeof(T) == 4) g = zv * sigmoid_acc(zv);
          else g = zv * sigmoid_fast(zv);
        }
        Sm.dd[warp][i][ch] = make_float2(delta, delta * uv);
        Sm.gg[warp][i][ch] = make_float2(g, D1 * uv * g);
      }
      // B | C of the 8 rows: 4 runs of 8 values per row, one run per lane
      const int part = lane & 3;
      const int row = warp * kTs + pr;
      const T* src = (part < 2 ? Sm.Bm[s] : Sm.Cm[s]) + row * kN + (part & 1) * 8;
      float f[8];
      load8(src, f);
      float4* dst = reinterpret_cast<float4*>(&Sm.BC[warp][pr][part * 8]);
      dst[0] = make_float4(f[0], f[1], f[2], f[3]);
      dst[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&Sm.sfree[s]);
    if (warp == kWarps - 1) {
      bool pok = true;
      if (producer && c + S < nchunk) {  // recycle the stage once every warp converted it
        pok = wait(&Sm.sfree[s], (c / S) & 1);
        if (pok) issue(c + S);
      }
      if (!__shfl_sync(0xffffffffu, pok, 0)) { ok = false; break; }
    }

    // ---- walk 1: local scan from zero, decays cached
    float2 dA[kTs][kHalf / 2];
    float2 h[kHalf / 2];
#pragma unroll
    for (int k = 0; k < kHalf / 2; ++k) h[k] = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kTs; ++i) {
      const float2 dl = Sm.dd[warp][i][ch];
      const float2 dlt = f2(dl.x), du = f2(dl.y);
      const float4* Bp = reinterpret_cast<const float4*>(&Sm.BC[warp][i][hf * kHalf]);
      const float4 b0 = Bp[0], b1 = Bp[1];
      const float2 bq[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w), make_float2(b1.x, b1.y),
                            make_float2(b1.z, b1.w)};
#pragma unroll
      for (int k = 0; k < kHalf / 2; ++k) {
        const float2 x = __fmul2_rn(dlt, A2[k]);
        dA[i][k] = make_float2(ex2_approx(x.x), ex2_approx(x.y));
        h[k] = __ffma2_rn(dA[i][k], h[k], __fmul2_rn(du, bq[k]));
      }
    }
    float2 P[kHalf / 2];
#pragma unroll
    for (int k = 0; k < kHalf / 2; ++k) {
      P[k] = dA[0][k];
#pragma unroll
      for (int i = 1; i < kTs; ++i) P[k] = __fmul2_rn(P[k], dA[i][k]);
    }

    // ---- carry chain: entry state of this slice, hand the next one on
    float2 e[kHalf / 2];
    if (c == 0 && warp == 0) {
#pragma unroll
      for (int k = 0; k < kHalf / 2; ++k) {
        if (h0) {
          const float* hp = h0 + ((size_t)b * D + d) * kN + hf * kHalf + 2 * k;
          e[k] = make_float2(hp[0], hp[1]);
        } else {
          e[k] = make_float2(0.f, 0.f);
        }
      }
    } else {
      const uint32_t par = warp == 0 ? ((c - 1) & 1) : (c & 1);
      if (!__all_sync(0xffffffffu, wait_spin(&Sm.eready[warp], par))) { ok = false; break; }
      const float4 q0 = Sm.E[c & 1][warp][0][lane], q1 = Sm.E[c & 1][warp][1][lane];
      e[0] = make_float2(q0.x, q0.y);
      e[1] = make_float2(q0.z, q0.w);
      e[2] = make_float2(q1.x, q1.y);
      e[3] = make_float2(q1.z, q1.w);
    }
    {
      float2 en[kHalf / 2];
#pragma unroll
      for (int k = 0; k < kHalf / 2; ++k) en[k] = __ffma2_rn(P[k], e[k], h[k]);
      if (warp < kWarps - 1 || c + 1 < nchunk) {
        const int nw = warp < kWarps - 1 ? warp + 1 : 0;
        const int np = warp < kWarps - 1 ? (c & 1) : ((c + 1) & 1);
        Sm.E[np][nw][0][lane] = make_float4(en[0].x, en[0].y, en[1].x, en[1].y);
        Sm.E[np][nw][1][lane] = make_float4(en[2].x, en[2].y, en[3].x, en[3].y);
        mbar_arrive(&Sm.eready[nw]);
      } else if (hT && SAMBA_DCHECK(err, d < D && b < (int)gridDim.y)) {  // the state after the last token
        float* hp = hT + ((size_t)b * D + d) * kN + hf * kHalf;
#pragma unroll
        for (int k = 0; k < kHalf / 2; ++k) {
          hp[2 * k] = en[k].x;
          hp[2 * k + 1] = en[k].y;
        }
      }
    }

    // ---- walk 2: exact states from the entry state, read-out, gate
    T* ytile = Sm.y[c % kYBuf];
    float yp[kTs];
#pragma unroll
    for (int k = 0; k < kHalf / 2; ++k) h[k] = e[k];
#pragma unroll
    for (int i = 0; i < kTs; ++i) {
      const float2 du = f2(Sm.dd[warp][i][ch].y);
      const float4* Bp = reinterpret_cast<const float4*>(&Sm.BC[warp][i][hf * kHalf]);
      const float4* Cp = reinterpret_cast<const float4*>(&Sm.BC[warp][i][kN + hf * kHalf]);
      const float4 b0 = Bp[0], b1 = Bp[1], c0 = Cp[0], c1 = Cp[1];
      const float2 bq[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w), make_float2(b1.x, b1.y),
                            make_float2(b1.z, b1.w)};
      const float2 cq[4] = {make_float2(c0.x, c0.y), make_float2(c0.z, c0.w), make_float2(c1.x, c1.y),
                            make_float2(c1.z, c1.w)};
#pragma unroll
      for (int k = 0; k < kHalf / 2; ++k) h[k] = __ffma2_rn(dA[i][k], h[k], __fmul2_rn(du, bq[k]));
      const float2 ya = __ffma2_rn(cq[1], h[1], __fmul2_rn(cq[0], h[0]));
      const float2 yb = __ffma2_rn(cq[3], h[3], __fmul2_rn(cq[2], h[2]));
      const float2 ys = __fadd2_rn(ya, yb);
      yp[i] = ys.x + ys.y;
    }
    // the two lanes of a channel: lane half 0 finishes the even token of each
    // pair, half 1 the odd one (one shuffle per pair)
#pragma unroll
    for (int i = 0; i < kTs; i += 2) {
      const float send = hf ? yp[i] : yp[i + 1];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
      const int ti = i + hf;
      const float ysum = (hf ? yp[i + 1] : yp[i]) + recv;
      const float2 g = Sm.gg[warp][ti][ch];
      ytile[(warp * kTs + ti) * kCh + ch] = Elt<T>::from_f(fmaf(ysum, g.x, g.y));
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&Sm.ydone[c % kYBuf]);
    if (warp == kWarps - 1) {
      bool pok = true;
      if (producer) {  // every warp wrote its rows: store the tile
        pok = wait(&Sm.ydone[c % kYBuf], (c / kYBuf) & 1);
        if (pok) {
          // the tensor map clips rows >= L and channels >= D; the tile's origin must lie inside
          if (SAMBA_DCHECK(err, d0 < D && c * kChunk < L)) tma_store_3d(&tm_y, ytile, d0, c * kChunk, b);
          tma_store_commit();
          tma_store_wait_read<1>();  // the tile of chunk c - 1 has been read: reusable at chunk c + 2
        }
      }
      if (!__shfl_sync(0xffffffffu, pok, 0)) { ok = false; break; }
    }
    __syncwarp();
  }
  if (producer) {
    tma_store_wait_all<0>();
    // after a timeout, loads still in flight must land before the CTA leaves
    for (int c = consumed; c < issued; ++c) {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&Sm.full[c % S], (c / S) & 1))
        if (globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
  }
}

__global__ void copy_state_kernel(const float* __restrict__ h0, float* __restrict__ hT, size_t n) {
  size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (i < n) hT[i] = h0 ? h0[i] : 0.f;
}

template <typename T>
bool make_rows_map(CUtensorMap* m, const void* base, int64_t ld, int width, int box_w, int L, int B) {
  const samba_dtype dt = Elt<T>::id;
  uint64_t dims[3] = {(uint64_t)width, (uint64_t)L, (uint64_t)B};
  uint64_t strides[2] = {(uint64_t)ld, (uint64_t)ld * (uint64_t)L};
  uint32_t box[3] = {(uint32_t)box_w, (uint32_t)kChunk, 1};
  return make_tmap(m, base, dt, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <typename T, bool kSoftplus, bool kHasZ, bool kDt>
samba_status launch_typed(const ScanArgs& a, cudaStream_t st) {
  CUtensorMap mu, mdt, mz, mB, mC, my;
  bool ok = make_rows_map<T>(&mu, a.u, a.ld_u, a.D, kCh, a.L, a.B);
  if (kDt) {  // dt_low rows: 64-column boxes, 128B-swizzled, columns past R read as zeros
    uint64_t dims[3] = {(uint64_t)a.R, (uint64_t)a.L, (uint64_t)a.B};
    uint64_t strides[2] = {(uint64_t)a.ld_dtl, (uint64_t)a.ld_dtl * (uint64_t)a.L};
    uint32_t box[3] = {(uint32_t)kDtBox, (uint32_t)kChunk, 1};
    ok = ok && make_tmap(&mdt, a.dt_low, SAMBA_BF16, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    ok = ok && make_rows_map<T>(&mdt, a.dt, a.ld_dt, a.D, kCh, a.L, a.B);
  }
  ok = ok && make_rows_map<T>(&mB, a.Bm, a.ld_bc, kN, kN, a.L, a.B) &&
            make_rows_map<T>(&mC, a.Cm, a.ld_bc, kN, kN, a.L, a.B) &&
            make_rows_map<T>(&my, a.y, a.ld_y, a.D, kCh, a.L, a.B);
  if (kHasZ) ok = ok && make_rows_map<T>(&mz, a.z, a.ld_z, a.D, kCh, a.L, a.B);
  else mz = mu;
  if (!ok) return SAMBA_ERR_CUDA;
  const size_t smem = sizeof(ScanSmem<T, kDt>) + 1024;
  auto kern = scan_chunked_kernel<T, kSoftplus, kHasZ, kDt>;
  if (!ensure_smem_attr(kern, smem))
    return SAMBA_ERR_CUDA;
  dim3 grid(a.D / kCh, a.B);
  const StallHook hk = scan_stall_hook();
  kern<<<grid, kThreads, smem, st>>>(mu, mdt, mz, mB, mC, my, a.A_log, a.dt_bias, a.Dskip, a.h0, a.hT, a.L, a.D,
                                     device_error_word(), hk.stop_chunk < 0 ? INT32_MAX : hk.stop_chunk,
                                     hk.stop_chunk < 0 ? kWaitLimitNs : hk.wait_limit_ns,
                                     (const bf16*)a.W_dt, a.R);
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

template <typename T>
samba_status launch_dispatch(const ScanArgs& a, cudaStream_t st) {
  if (a.softplus) {
    return a.z ? launch_typed<T, true, true, false>(a, st) : launch_typed<T, true, false, false>(a, st);
  }
  return a.z ? launch_typed<T, false, true, false>(a, st) : launch_typed<T, false, false, false>(a, st);
}

}  // namespace

bool scan_dt_fold_supported(const ScanArgs& a) {
  return a.dtype == SAMBA_BF16 && a.dt_low && a.W_dt && a.R >= 16 && a.R <= kDtMaxR && a.R % 16 == 0 &&
         aligned16(a.dt_low) && aligned16(a.W_dt) && (a.ld_dtl * 2) % 16 == 0 && a.ld_dtl >= a.R;
}

samba_status validate_scan(const ScanArgs& a) {
  if (!a.u || !(a.dt || a.dt_low) || !a.A_log || !a.Bm || !a.Cm || !a.y) return SAMBA_ERR_INVALID_ARG;
  if (!a.dt && !scan_dt_fold_supported(a)) return SAMBA_ERR_UNSUPPORTED;
  if (a.B < 1 || a.L < 0 || a.D < 1 || a.N < 1) return SAMBA_ERR_INVALID_ARG;
  if (a.N != kN || a.D % kCh != 0 || a.B > kMaxGridYZ) return SAMBA_ERR_UNSUPPORTED;
  const size_t es = dtype_size(a.dtype);
  const void* ptrs[] = {a.u, a.dt, a.Bm, a.Cm, a.y, a.z};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return SAMBA_ERR_UNSUPPORTED;
  const int64_t lds[] = {a.ld_u, a.dt ? a.ld_dt : a.ld_u, a.ld_bc, a.ld_y, a.z ? a.ld_z : a.ld_u};
  for (int64_t ld : lds)
    if ((ld * (int64_t)es) % 16 != 0) return SAMBA_ERR_UNSUPPORTED;
  if (a.ld_u < a.D || (a.dt && a.ld_dt < a.D) || a.ld_y < a.D || a.ld_bc < a.N || (a.z && a.ld_z < a.D))
    return SAMBA_ERR_INVALID_ARG;
  return SAMBA_OK;
}

samba_status launch_selective_scan(const ScanArgs& a, cudaStream_t st) {
  samba_status v = validate_scan(a);
  if (v != SAMBA_OK) return v;
  if (a.L == 0) {
    if (a.hT) {
      const size_t n = (size_t)a.B * a.D * a.N;
      copy_state_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a.h0, a.hT, n);
      SAMBA_CHECK_LAUNCH();
    }
    return SAMBA_OK;
  }
  if (!a.dt) {  // the dt projection folded in (bf16; softplus always applied)
    return a.z ? launch_typed<bf16, true, true, true>(a, st) : launch_typed<bf16, true, false, true>(a, st);
  }
  return a.dtype == SAMBA_BF16 ? launch_dispatch<bf16>(a, st) : launch_dispatch<float>(a, st);
}

}  // namespace samba
