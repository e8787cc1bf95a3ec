// fast_dispatch.cu -- chooses between the fast kernels for a problem.
#include <atomic>

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

cudaError_t launch_fast_select(Problem &p, void *ws, size_t ws_bytes,
                               cudaStream_t st) {
    (void)p; (void)ws; (void)ws_bytes; (void)st;
    return cudaErrorNotSupported;
}

cudaError_t launch_fast_attend(Problem &p, void *ws, size_t ws_bytes,
                               cudaStream_t st) {
    (void)p; (void)ws; (void)ws_bytes; (void)st;
    return cudaErrorNotSupported;
}

namespace {
std::atomic<uint64_t> g_launches{0};
}

void count_launches(int n) { g_launches.fetch_add((uint64_t)n); }
uint64_t launch_total() { return g_launches.load(); }

}  // namespace hils
