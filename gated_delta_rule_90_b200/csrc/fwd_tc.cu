// Tensor-core (tcgen05/TMEM + TMA) chunkwise prefill -- placeholder until the
// kernels land: the path reports that it does not apply.
#include "common.cuh"

namespace gdr_host {
bool tc_applies(int, int, int, gdr_dtype) { return false; }
size_t tc_workspace_bytes(int, int, int, int, int, gdr_gate) { return 0; }
cudaError_t fwd_tc_dispatch(const void *, const void *, const void *, const float *, const float *,
                            const float *, void *, float *, int, int, int, const int32_t *, int,
                            gdr_gate, void *, size_t, unsigned int *, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace gdr_host
