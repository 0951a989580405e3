// chunk_tc.cu -- tensor-core (tcgen05) chunkwise EFLA forward for sm_100a.
#include "common.cuh"
#include "launchers.h"

namespace efla {

static __device__ unsigned int g_tc_error = 0;

bool tc_supported(int, int, int, int, int, int, bool) { return false; }
size_t tc_workspace_bytes(int, int, int, int, int, int) { return 0; }
cudaError_t launch_chunk_tc(const void *, const void *, const void *, const void *, const float *,
                            void *, float *, int, int, int, int, int, int, bool, void *,
                            cudaStream_t) {
    return cudaErrorNotSupported;
}

cudaError_t tc_read_and_clear_error(unsigned int *out, cudaStream_t s) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(out, g_tc_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(unsigned int));
}

}  // namespace efla
