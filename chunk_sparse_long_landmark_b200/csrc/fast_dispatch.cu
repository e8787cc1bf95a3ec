// fast_dispatch.cu -- chooses between the fast kernels for a problem.
#include "hils_fast.cuh"

namespace hils {

bool fast_path_supported(const Problem &p) {
    (void)p;
    return false;
}

size_t fast_workspace_bytes(const Problem &p) {
    (void)p;
    return 0;
}

cudaError_t launch_fast(Problem &p, void *ws, size_t ws_bytes, cudaStream_t st) {
    (void)p; (void)ws; (void)ws_bytes; (void)st;
    return cudaErrorNotSupported;
}

}  // namespace hils
