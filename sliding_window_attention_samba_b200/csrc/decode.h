// Internal launchers of the decode-step kernels (not part of the C ABI).
#pragma once

#include "kernels.h"

namespace samba {

samba_status launch_conv_step(const void* hz, int64_t ld_hz, const float* w, const float* bias, void* state, void* u,
                              int B, int D, int k, samba_dtype dt, cudaStream_t st);
samba_status launch_scan_step(const void* u, const void* dlt, const void* z, int64_t ld_z, const void* xdbl,
                              int64_t ld_x, int r_off, const float* A_log, const float* Dskip, float* ssm, void* y,
                              int B, int D, samba_dtype dt, cudaStream_t st);
samba_status launch_ring_write(const void* qkv, int64_t ld, int k_off, int v_off, const int64_t* pos, void* k_ring,
                               void* v_ring, int B, int window, int kvw, samba_dtype dt, cudaStream_t st);
samba_status launch_attn_decode(const void* qkv, int64_t ld, const int64_t* pos, const void* k_ring,
                                const void* v_ring, void* o, int B, int Hq, int Hkv, int hd, int window, float scale,
                                samba_dtype dt, cudaStream_t st);
samba_status launch_pos_update(int64_t* pos, int B, int64_t value, bool set, cudaStream_t st);
samba_status launch_ring_fill(const void* qkv, int64_t ld, int k_off, int v_off, void* k_ring, void* v_ring, int B,
                              int L, int window, int kvw, samba_dtype dt, cudaStream_t st);

}  // namespace samba
