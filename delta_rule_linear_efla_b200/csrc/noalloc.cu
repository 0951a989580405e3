// noalloc.cu -- efla_chunk_fwd_noalloc: the chunk forward for callers that cannot
// allocate device memory (they are handed only their input and output buffers,
// or must not call cudaMalloc on their hot path).  The tensor-core path's
// scratch lives in a fixed file-scope device array instead of a caller
// workspace.  The method itself has no counterpart of this entry point.
#include <mutex>

#include "../../include/efla.h"
#include "launchers.h"

namespace {

// Fixed scratch: the per-chunk T*diag(alpha) tiles of the tensor-core path.
// Loaded with the library's device code on each GPU that uses it; every call
// shares it.  Nothing here needs to start at zero.
static __device__ __align__(256) unsigned char g_noalloc_scratch[EFLA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};  // device address of g_noalloc_scratch, per device

// Device address of the scratch array on the current device (looked up once per
// device; host code may not use the symbol itself as an address).
efla_status scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return EFLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return EFLA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return EFLA_OK;
}

}  // namespace

extern "C" efla_status efla_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                              const void *beta, const float *S0, void *o,
                                              float *S_final, int B, int H, int L, int dk, int dv,
                                              int chunk, efla_dtype dt, efla_dtype o_dt,
                                              void *stream) {
    // Scratch the call needs: with sequence segments where the sizes would take them, else in
    // the one-pass form, which needs less (no segment states).  Sizes that fit neither way are
    // refused before anything else happens.
    size_t need = efla_chunk_fwd_workspace_size(B, H, L, dk, dv, chunk, dt, o_dt);
    bool allow_segments = true;
    if (need > EFLA_NOALLOC_SCRATCH_BYTES && dt == EFLA_BF16 &&
        efla::tc_supported(B, H, L, dk, dv, chunk, true)) {
        need = efla::tc_workspace_bytes(B, H, L, dk, dv, chunk, false);
        allow_segments = false;
    }
    if (need > EFLA_NOALLOC_SCRATCH_BYTES) return EFLA_ERR_TOO_LARGE;
    void *scratch = nullptr;
    if (need > 0) {
        const efla_status st = scratch_address(&scratch);
        if (st != EFLA_OK) return st;
    }
    return (efla_status)efla::chunk_fwd_entry(q, k, v, beta, S0, o, S_final, B, H, L, dk, dv, chunk, dt,
                                              o_dt, EFLA_RULE_EXACT, scratch,
                                              need > 0 ? (size_t)EFLA_NOALLOC_SCRATCH_BYTES : 0, stream,
                                              allow_segments, nullptr);
}
