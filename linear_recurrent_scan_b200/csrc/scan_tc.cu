// Tensor-core (tcgen05 + TMA) chunked prefill -- not built yet.
#include "common.cuh"
#include "internal.h"

namespace m3 {
int tc_scan_supported(const ScanArgs&) { return MAMBA3_ERR_UNSUPPORTED; }
int launch_scan_tc(const ScanArgs&, cudaStream_t) { return MAMBA3_ERR_UNSUPPORTED; }
}  // namespace m3
