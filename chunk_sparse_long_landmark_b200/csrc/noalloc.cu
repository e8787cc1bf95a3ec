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
// with cudaGetSymbolAddress (with the device current) on the first call in a
// device's context and passed to the kernels as a plain pointer. The cached
// address is keyed on the context's process-unique ID (cuCtxGetId): after a
// cudaDeviceReset the library's module is loaded again in a new context,
// where the array may sit elsewhere, and the address is looked up again.
#include <mutex>

#include <cuda.h>

#include "hils_internal.cuh"

namespace hils {
namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;   // 8 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

struct CachedScratch {
    unsigned long long ctx_id;      // context the address belongs to
    void *ptr;
};

std::mutex g_mu;
CachedScratch g_scratch[kMaxDevices] = {};

// Unique ID of the calling thread's current context (false: none current,
// or the driver entry points are unavailable).
bool current_context_id(unsigned long long *id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault,
                                    &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = (CtxGetCurrentFn)f;
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault,
                                    &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = (CtxGetIdFn)f;
    });
    CUcontext ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx)
        return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array in the current device's context,
// looked up on the first call in that context. nullptr if the runtime
// refuses.
void *scratch_for_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    unsigned long long id = 0;
    if (g_scratch[dev].ptr && current_context_id(&id) &&
        id == g_scratch[dev].ctx_id)
        return g_scratch[dev].ptr;
    void *ptr = nullptr;           // (creates the primary context if needed)
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess)
        return nullptr;
    if (!current_context_id(&id)) return nullptr;
    g_scratch[dev].ctx_id = id;
    g_scratch[dev].ptr = ptr;
    return ptr;
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
