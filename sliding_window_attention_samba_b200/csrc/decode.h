// Internal launchers of the decode-step kernels (not part of the C ABI).  The
// single-token kernels (conv_step, scan_step, ring_write, attn_decode) are
// launched as programmatic dependents of the previous kernel (see pdl_wait).
#pragma once

#include "kernels.h"

namespace samba {

samba_status launch_conv_step(const void* hz, int64_t ld_hz, const float* w, const float* bias, void* state, void* u,
                              int B, int D, int k, samba_dtype dt, cudaStream_t st);
samba_status launch_scan_step(const void* u, const void* dlt, const void* z, int64_t ld_z, const void* xdbl,
                              int64_t ld_x, int r_off, const float* A_log, const float* Dskip, float* ssm, void* y,
                              int B, int D, samba_dtype dt, cudaStream_t st);
// The recurrence step with Delta = softplus(xdbl[:, :R] W_dt^T + dt_bias) formed
// in the kernel (B, C at columns R, R + 16 of xdbl); supported for dt_rank R
// <= 512, R % 8 == 0.
bool scan_step_dt_supported(int R, int D, int64_t ld_x, samba_dtype dt);
samba_status launch_scan_step_dt(const void* u, const void* z, int64_t ld_z, const void* xdbl, int64_t ld_x, int R,
                                 const void* W_dt, const float* dt_bias, const float* A_log, const float* Dskip,
                                 float* ssm, void* y, int B, int D, samba_dtype dt, cudaStream_t st);
samba_status launch_ring_write(const void* qkv, int64_t ld, int k_off, int v_off, const int64_t* pos, void* k_ring,
                               void* v_ring, int B, int window, int kvw, samba_dtype dt, cudaStream_t st);
// Decode attention over the ring (bf16, head_dim 64, up to 8 query heads per kv
// head): with at least 3/4 of an SM's worth of (kv head, row) pairs per SM and
// rings up to 4096 slots, one streaming CTA per pair; otherwise an 8-CTA
// cluster per pair (rings up to 2048 slots) or, above 2048 slots, one CTA per
// 256-slot slice whose partials need attn_decode_workspace_bytes() of
// workspace (0 when not needed).  Other dtypes and head dims: a CUDA-core kernel.
size_t attn_decode_workspace_bytes(int B, int Hkv, int window);
samba_status launch_attn_decode(const void* qkv, int64_t ld, const int64_t* pos, const void* k_ring,
                                const void* v_ring, void* o, int B, int Hq, int Hkv, int hd, int window, float scale,
                                samba_dtype dt, cudaStream_t st, void* ws = nullptr, size_t ws_bytes = 0);
samba_status launch_pos_update(int64_t* pos, int B, int64_t value, bool set, cudaStream_t st, bool pdl = false);
// prefill -> ring: the last min(L, w) tokens of a prefill whose token 0 is at absolute position pos0
samba_status launch_ring_fill(const void* qkv, int64_t ld, int k_off, int v_off, void* k_ring, void* v_ring, int B,
                              int L, int64_t pos0, int window, int kvw, samba_dtype dt, cudaStream_t st);
// K/V rows of a prefill chunk preceded by the h ring entries of positions pos0-h .. pos0-1:
// kx, vx [B, h + L, kvw] (contiguous)
samba_status launch_kv_window_gather(const void* qkv, int64_t ld, int k_off, int v_off, const void* k_ring,
                                     const void* v_ring, void* kx, void* vx, int B, int L, int64_t pos0, int h,
                                     int window, int kvw, samba_dtype dt, cudaStream_t st);
// pos[b] must equal `expect` (else the device error word is set); then pos[b] = value
samba_status launch_pos_check_set(int64_t* pos, int B, int64_t expect, int64_t value, cudaStream_t st);

}  // namespace samba
