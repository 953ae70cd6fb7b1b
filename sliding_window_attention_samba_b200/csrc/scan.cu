// Chunked selective scan (S6) for sm_100a.
//
// Computes, per batch row b and channel d [Samba 3.4 "The State Space Model
// Update (S6)", "Input-Dependent Selective Gating", "Gated Output"]:
//   Delta_t = softplus(dt_t + bias)            (or dt_t + bias)
//   h_t     = exp(Delta_t A) (.) h_{t-1} + Delta_t u_t B_t
//   y_t     = <C_t, h_t> + D u_t,   y_t *= SiLU(z_t)
//
// Design (one CTA = 32 channels of one batch row, the whole sequence):
//   * 64-token chunks of u, dt, z (32 channels wide) and B, C (16 wide) are
//     staged through shared memory by TMA, NSTAGE deep.
//   * 8 warps split each chunk in time: warp w owns tokens [8w, 8w+8), lane l
//     owns channel l and its 16 fp32 states in registers.
//   * B and C of a chunk are converted to fp32 once into a shared tile (all 32
//     lanes of a warp read the same values, so per-lane conversion would repeat
//     it 32 times).
//   * Walk 1: each lane runs its 8 tokens from a zero state, keeping the 8x16
//     decays exp(Delta A) in registers, and publishes (prod of decays, end state).
//     States are processed in pairs with packed fp32x2 FMA/MUL.
//   * Combine: 256 threads each own two (channel, state) pairs and chain the
//     8 warp aggregates sequentially from the carry of the previous chunk
//     (kept in registers across chunks); this yields every warp's entry state.
//   * Walk 2: each lane re-runs its tokens from the right entry state with the
//     cached decays (one exp per element in total), emits y into a shared tile
//     written back by a TMA store.
// No inter-CTA communication, no workspace, no spin waits except the TMA
// mbarrier waits (bounded, error word on timeout).
#include "common.cuh"
#include "kernels.h"

namespace samba {

namespace {

constexpr int kCh = 32;       // channels per CTA
constexpr int kWarps = 8;     // time sub-chunks per chunk
constexpr int kTs = 8;        // tokens per warp sub-chunk
constexpr int kChunk = kWarps * kTs;  // 64 tokens
constexpr int kN = 16;        // state size
constexpr int kStages = 3;
constexpr int kThreads = kWarps * 32;

template <typename T>
struct ScanSmem {
  T u[kStages][kChunk * kCh];
  T dt[kStages][kChunk * kCh];
  T z[kStages][kChunk * kCh];
  T Bm[kStages][kChunk * kN];
  T Cm[kStages][kChunk * kN];
  T y[2][kChunk * kCh];
  float BC[2][kChunk][2 * kN];  // fp32 copy of B | C per token, converted once per chunk
  float aggP[kWarps][kN][kCh];
  float aggH[kWarps][kN][kCh];
  uint64_t full[kStages];
};

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

template <typename T, bool kSoftplus, bool kHasZ>
__global__ void __launch_bounds__(kThreads, 1)
    scan_chunked_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_dt,
                        const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_B,
                        const __grid_constant__ CUtensorMap tm_C, const __grid_constant__ CUtensorMap tm_y,
                        const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                        const float* __restrict__ Dskip, const float* __restrict__ h0, float* __restrict__ hT,
                        int L, int D, int* err, int stop_chunk, uint64_t wait_limit_ns) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  ScanSmem<T>& S = *reinterpret_cast<ScanSmem<T>*>(smem_raw + smem_align_pad(smem_raw, 128));

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int d0 = blockIdx.x * kCh;
  const int b = blockIdx.y;
  const int d = d0 + lane;
  const int nchunk = (L + kChunk - 1) / kChunk;

  constexpr uint32_t kStageBytes = (3 * kChunk * kCh + 2 * kChunk * kN) * sizeof(T);
  const uint32_t stage_bytes = kHasZ ? kStageBytes : kStageBytes - kChunk * kCh * sizeof(T);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&S.full[s], 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_u);
    tma_prefetch_desc(&tm_dt);
    tma_prefetch_desc(&tm_B);
    tma_prefetch_desc(&tm_C);
    tma_prefetch_desc(&tm_y);
    if (kHasZ) tma_prefetch_desc(&tm_z);
  }
  __syncthreads();

  auto issue = [&](int c) {
    if (c >= stop_chunk) return;  // failure-detection test hook: nothing issued past here
    const int s = c % kStages;
    const int t0 = c * kChunk;
    mbar_arrive_expect_tx(&S.full[s], stage_bytes);
    tma_load_3d(S.u[s], &tm_u, &S.full[s], d0, t0, b);
    tma_load_3d(S.dt[s], &tm_dt, &S.full[s], d0, t0, b);
    if (kHasZ) tma_load_3d(S.z[s], &tm_z, &S.full[s], d0, t0, b);
    tma_load_3d(S.Bm[s], &tm_B, &S.full[s], 0, t0, b);
    tma_load_3d(S.Cm[s], &tm_C, &S.full[s], 0, t0, b);
  };
  // wait for chunk c's stage, then convert its B and C to fp32 (one element per thread pass)
  auto arrive_chunk = [&](int c) -> bool {
    const int s = c % kStages;
    const bool ok = mbar_wait(&S.full[s], (c / kStages) & 1, err, wait_limit_ns);
    if (ok) {
      // 64 rows x (16 B | 16 C) = 256 runs of 8 values: one per thread
      static_assert(kChunk * 4 == kThreads, "one 8-value run of B or C per thread");
      const int row = tid >> 2, part = tid & 3;
      const T* src = (part < 2 ? S.Bm[s] : S.Cm[s]) + row * kN + (part & 1) * 8;
      float f[8];
      load8(src, f);
      float4* dst = reinterpret_cast<float4*>(&S.BC[c & 1][row][part * 8]);
      dst[0] = make_float4(f[0], f[1], f[2], f[3]);
      dst[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
    return ok;
  };
  if (tid == 0)
    for (int c = 0; c < kStages - 1 && c < nchunk; ++c) issue(c);

  // Per-lane constants: A * log2(e), as pairs of states.
  float2 A2[kN / 2];
#pragma unroll
  for (int n = 0; n < kN / 2; ++n)
    A2[n] = make_float2(-expf(A_log[(size_t)d * kN + 2 * n]) * 1.4426950408889634f,
                        -expf(A_log[(size_t)d * kN + 2 * n + 1]) * 1.4426950408889634f);
  const float bias = dt_bias ? dt_bias[d] : 0.f;
  const float Dd = Dskip ? Dskip[d] : 0.f;

  // Combine-role ownership: channel cl, states cn and cn+1; their carries.
  const int cl = tid & 31;
  const int cn = (tid >> 5) * 2;
  float carry[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) carry[j] = h0 ? h0[((size_t)b * D + d0 + cl) * kN + cn + j] : 0.f;

  bool ok = nchunk > 0 ? __syncthreads_and(arrive_chunk(0)) : true;
  for (int c = 0; c < nchunk && ok; ++c) {
    const int s = c % kStages;
    if (tid == 0 && c + kStages - 1 < nchunk) issue(c + kStages - 1);
    const float* BC = &S.BC[c & 1][0][0];

    const int tb = warp * kTs;       // first token of this warp within the chunk
    const int tg = c * kChunk + tb;  // global index of that token
    float2 dA[kTs][kN / 2];
    float du[kTs];
    float2 h[kN / 2];
#pragma unroll
    for (int n = 0; n < kN / 2; ++n) h[n] = make_float2(0.f, 0.f);

    // ---- walk 1: local scan from zero, decays cached (pairs of states per FMA2)
#pragma unroll
    for (int i = 0; i < kTs; ++i) {
      const int row = tb + i;
      const float dtv = Elt<T>::to_f(S.dt[s][row * kCh + lane]) + bias;
      float delta;
      if (kSoftplus) {
        if constexpr (sizeof(T) == 4) delta = softplus_acc(dtv);
        else delta = softplus_fast(dtv);
      } else {
        delta = dtv;
      }
      float uv = Elt<T>::to_f(S.u[s][row * kCh + lane]);
      if (tg + i >= L) { delta = 0.f; uv = 0.f; }
      du[i] = delta * uv;
      const float2 dl = f2(delta), dd = f2(du[i]);
      const float4* Bp = reinterpret_cast<const float4*>(BC + row * 2 * kN);
#pragma unroll
      for (int q = 0; q < kN / 4; ++q) {
        const float4 Bq = Bp[q];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int n = 2 * q + hh;
          const float2 x = __fmul2_rn(dl, A2[n]);
          dA[i][n] = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          const float2 bu = __fmul2_rn(dd, hh ? make_float2(Bq.z, Bq.w) : make_float2(Bq.x, Bq.y));
          h[n] = __ffma2_rn(dA[i][n], h[n], bu);
        }
      }
    }
#pragma unroll
    for (int n = 0; n < kN / 2; ++n) {
      float2 p = dA[0][n];
#pragma unroll
      for (int i = 1; i < kTs; ++i) p = __fmul2_rn(p, dA[i][n]);
      S.aggP[warp][2 * n][lane] = p.x;
      S.aggP[warp][2 * n + 1][lane] = p.y;
      S.aggH[warp][2 * n][lane] = h[n].x;
      S.aggH[warp][2 * n + 1][lane] = h[n].y;
    }
    __syncthreads();

    // ---- combine across the 8 warps, chained from the previous chunk's carry
    // (all aggregates are loaded before the first entry state is stored: the
    // dependent chain is then 8 FMAs, not 8 shared-memory round trips)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float P[kWarps], hl[kWarps];
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        P[w] = S.aggP[w][cn + j][cl];
        hl[w] = S.aggH[w][cn + j][cl];
      }
      float H = carry[j];
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        S.aggH[w][cn + j][cl] = H;
        H = fmaf(P[w], H, hl[w]);
      }
      carry[j] = H;
    }
    if (tid == 0) tma_store_wait_read<1>();  // y tile (c & 1) free again
    __syncthreads();

    // ---- walk 2: exact states from the entry state, outputs
#pragma unroll
    for (int n = 0; n < kN / 2; ++n) h[n] = make_float2(S.aggH[warp][2 * n][lane], S.aggH[warp][2 * n + 1][lane]);
    T* ytile = S.y[c & 1];
#pragma unroll
    for (int i = 0; i < kTs; ++i) {
      const int row = tb + i;
      const float4* Bp = reinterpret_cast<const float4*>(BC + row * 2 * kN);
      const float4* Cp = Bp + kN / 4;
      const float2 dd = f2(du[i]);
      float2 y2[4];  // four partial sums: the readout is not one serial chain of 8 FMAs
#pragma unroll
      for (int q = 0; q < kN / 4; ++q) {
        const float4 Bq = Bp[q];
        const float4 Cq = Cp[q];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int n = 2 * q + hh;
          const float2 bu = __fmul2_rn(dd, hh ? make_float2(Bq.z, Bq.w) : make_float2(Bq.x, Bq.y));
          h[n] = __ffma2_rn(dA[i][n], h[n], bu);
          const float2 cq = hh ? make_float2(Cq.z, Cq.w) : make_float2(Cq.x, Cq.y);
          y2[q] = hh ? __ffma2_rn(cq, h[n], y2[q]) : __fmul2_rn(cq, h[n]);
        }
      }
      const float2 ya = __fadd2_rn(__fadd2_rn(y2[0], y2[1]), __fadd2_rn(y2[2], y2[3]));
      float y = ya.x + ya.y;
      const float uv = Elt<T>::to_f(S.u[s][row * kCh + lane]);
      y = fmaf(Dd, uv, y);
      if (kHasZ) {
        const float zv = Elt<T>::to_f(S.z[s][row * kCh + lane]);
        if constexpr (sizeof(T) == 4) y *= zv * sigmoid_acc(zv);
        else y *= zv * sigmoid_fast(zv);
      }
      ytile[row * kCh + lane] = Elt<T>::from_f(y);
    }
    fence_proxy_async_smem();
    // next chunk's stage has (usually) landed: convert its B and C while we are here
    bool nxt = true;
    if (c + 1 < nchunk) nxt = arrive_chunk(c + 1);
    ok = __syncthreads_and(nxt);
    if (tid == 0) {
      tma_store_3d(&tm_y, ytile, d0, c * kChunk, b);
      tma_store_commit();
    }
  }
  if (tid == 0) tma_store_wait_all<0>();
  if (ok && hT) {
#pragma unroll
    for (int j = 0; j < 2; ++j) hT[((size_t)b * D + d0 + cl) * kN + cn + j] = carry[j];
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

template <typename T, bool kSoftplus, bool kHasZ>
samba_status launch_typed(const ScanArgs& a, cudaStream_t st) {
  CUtensorMap mu, mdt, mz, mB, mC, my;
  bool ok = make_rows_map<T>(&mu, a.u, a.ld_u, a.D, kCh, a.L, a.B) &&
            make_rows_map<T>(&mdt, a.dt, a.ld_dt, a.D, kCh, a.L, a.B) &&
            make_rows_map<T>(&mB, a.Bm, a.ld_bc, kN, kN, a.L, a.B) &&
            make_rows_map<T>(&mC, a.Cm, a.ld_bc, kN, kN, a.L, a.B) &&
            make_rows_map<T>(&my, a.y, a.ld_y, a.D, kCh, a.L, a.B);
  if (kHasZ) ok = ok && make_rows_map<T>(&mz, a.z, a.ld_z, a.D, kCh, a.L, a.B);
  else mz = mu;
  if (!ok) return SAMBA_ERR_CUDA;
  const size_t smem = sizeof(ScanSmem<T>) + 128;
  auto kern = scan_chunked_kernel<T, kSoftplus, kHasZ>;
  if (!ensure_smem_attr(kern, smem))
    return SAMBA_ERR_CUDA;
  dim3 grid(a.D / kCh, a.B);
  const StallHook hk = scan_stall_hook();
  kern<<<grid, kThreads, smem, st>>>(mu, mdt, mz, mB, mC, my, a.A_log, a.dt_bias, a.Dskip, a.h0, a.hT, a.L, a.D,
                                     device_error_word(), hk.stop_chunk < 0 ? INT32_MAX : hk.stop_chunk,
                                     hk.stop_chunk < 0 ? kWaitLimitNs : hk.wait_limit_ns);
  SAMBA_CHECK_LAUNCH();
  return SAMBA_OK;
}

template <typename T>
samba_status launch_dispatch(const ScanArgs& a, cudaStream_t st) {
  if (a.softplus) {
    return a.z ? launch_typed<T, true, true>(a, st) : launch_typed<T, true, false>(a, st);
  }
  return a.z ? launch_typed<T, false, true>(a, st) : launch_typed<T, false, false>(a, st);
}

}  // namespace

samba_status validate_scan(const ScanArgs& a) {
  if (!a.u || !a.dt || !a.A_log || !a.Bm || !a.Cm || !a.y) return SAMBA_ERR_INVALID_ARG;
  if (a.B < 1 || a.L < 0 || a.D < 1 || a.N < 1) return SAMBA_ERR_INVALID_ARG;
  if (a.N != kN || a.D % kCh != 0 || a.B > kMaxGridYZ) return SAMBA_ERR_UNSUPPORTED;
  const size_t es = dtype_size(a.dtype);
  const void* ptrs[] = {a.u, a.dt, a.Bm, a.Cm, a.y, a.z};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return SAMBA_ERR_UNSUPPORTED;
  const int64_t lds[] = {a.ld_u, a.ld_dt, a.ld_bc, a.ld_y, a.z ? a.ld_z : a.ld_u};
  for (int64_t ld : lds)
    if ((ld * (int64_t)es) % 16 != 0) return SAMBA_ERR_UNSUPPORTED;
  if (a.ld_u < a.D || a.ld_dt < a.D || a.ld_y < a.D || a.ld_bc < a.N || (a.z && a.ld_z < a.D))
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
  return a.dtype == SAMBA_BF16 ? launch_dispatch<bf16>(a, st) : launch_dispatch<float>(a, st);
}

}  // namespace samba
