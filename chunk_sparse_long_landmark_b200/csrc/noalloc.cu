// noalloc.cu -- hils_fwd_decode_noalloc: the decode step without a caller
// workspace. The scratch lives in a fixed file-scope device array instead.
//
// Some callers cannot allocate device memory at call time: a serving loop
// whose memory is reserved up front (nothing left for an allocator to hand
// out), code whose latency budget rules out cudaMalloc's implicit device
// synchronisation, or a host that has no way to size and own a workspace
// buffer. This entry point serves them: it takes the same argument record as
// hils_fwd_decode, ignores its workspace fields, and runs the CUDA-core decode
// kernels (scoring + top-K, then attention) on the static scratch below.
//
// The array is a file-scope __device__ symbol. In host code its name is only
// a host-side stand-in, not a device address, so the address is obtained
// once per device with cudaGetSymbolAddress (with that device current) and
// passed to the kernels as a plain pointer.
#include <mutex>

#include "hils_internal.cuh"

namespace hils {
namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;   // 8 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call per device). Returns nullptr if the runtime refuses.
void *scratch_for_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess)
            return nullptr;
        g_scratch_ptr[dev] = ptr;
    }
    return g_scratch_ptr[dev];
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

// Defined in hils_host.cu: argument checks of the decode record.
hils_status decode_problem_checked(const hils_decode_args *a, Problem *p);

}  // namespace hils

extern "C" hils_status hils_fwd_decode_noalloc(const hils_decode_args *args,
                                               void *stream) {
    using namespace hils;
    Problem p;
    hils_status s = decode_problem_checked(args, &p);
    if (s != HILS_OK) return s;
    if (p.S > simt_max_chunk()) return HILS_ERR_UNSUPPORTED;

    // scratch plan: [selected scores, when the caller gave no sel_score]
    //               [scoring slab: one (G+1) x nc_max block per CTA]
    size_t sel_bytes = 0;
    if (!p.sel) sel_bytes = round256(sizeof(float) * (size_t)p.B * p.Hq * p.K);
    int64_t w0, ncm;
    window_bounds((int64_t)p.kv_rows - 1, p.S, p.W, &w0, &ncm);
    const size_t per_cta = sizeof(float) * simt_score_scratch_floats(p, (int)ncm);
    if (sel_bytes + per_cta > kNoAllocScratchBytes)
        return HILS_ERR_WORKSPACE_TOO_SMALL;     // shape beyond the fixed scratch
    const int64_t fit = (int64_t)((kNoAllocScratchBytes - sel_bytes) / per_cta);
    int grid = simt_score_grid(p);
    if (grid > fit) grid = (int)fit;

    char *base = (char *)scratch_for_current_device();
    if (!base) return HILS_ERR_CUDA;
    if (!p.sel) p.sel = (float *)base;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = launch_simt_score(p, (float *)(base + sel_bytes), grid, st);
    count_launches(1);
    if (e == cudaSuccess) {
        e = launch_simt_attend(p, st);
        count_launches(1);
    }
    return e == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
}
