// Tensor-core (tcgen05) sliding-window attention: placeholder until the
// banded tcgen05 kernel lands; the CUDA-core kernel serves every case.
#include "common.cuh"
#include "kernels.h"

namespace samba {

bool swa_tc_supported(const SwaArgs&) { return false; }
samba_status launch_swa_tc(const SwaArgs&, cudaStream_t) { return SAMBA_ERR_UNSUPPORTED; }

}  // namespace samba
