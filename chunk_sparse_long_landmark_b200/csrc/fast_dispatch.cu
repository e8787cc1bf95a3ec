// fast_dispatch.cu -- host side of the tensor-core path: decides whether a
// problem fits the sm_100a kernels, builds their TMA tensor maps and
// launches them. Problems outside the tile set run on the SIMT kernels.
#include <atomic>
#include <mutex>

#include <cuda.h>

#include "hils_fast.cuh"
#include "tc_kernels.cuh"

namespace hils {

namespace {

std::atomic<uint64_t> g_launches{0};

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t,
                                  void *, const cuuint64_t *, const cuuint64_t *,
                                  const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p,
                                    cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    });
    return fn;
}

// 4-D bf16 tensor [d3][d2][rows][d] (d innermost) with a {64, box_rows}
// tile, 128-byte swizzle, out-of-range elements read as zero.
bool make_map(CUtensorMap *m, const void *base, int d, int64_t rows, int d2,
              int d3, int box_rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)d2,
                          (cuuint64_t)d3};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)d * 2 * rows,
                             (cuuint64_t)d * 2 * rows * d2};
    cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base),
             dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

TcParams tc_params(const Problem &p) {
    TcParams t;
    t.Q = p.Q; t.Klm = p.Klm; t.bias = p.bias; t.O = p.O; t.idx = p.idx; t.sel = p.sel;
    t.status = p.status;
    t.B = p.B; t.Hq = p.Hq; t.Hkv = p.Hkv; t.G = p.G; t.N = p.n_query;
    t.d = p.d; t.S = p.S; t.W = p.W; t.K = p.K; t.nC = p.nC;
    t.M = 128 / p.G;
    const int64_t uc = (int64_t)t.M * p.K;
    t.ucap = (int)(uc < p.nC ? uc : (p.nC > 0 ? p.nC : 1));
    t.inv_sqrt_d = p.inv_sqrt_d;
    for (int k = 0; k < kMaxHeads; ++k) t.group_heads[k] = p.group_heads[k];
    return t;
}

bool attend_supported(const Problem &p) {
    if (p.decode || p.dtype != HILS_BF16) return false;
    if (!(p.d == 64 || p.d == 128) || !(p.S == 64 || p.S == 128)) return false;
    if (128 % p.G != 0) return false;
    if (p.nC > 65536) return false;
    if (!encode_fn()) return false;
    TcParams tp = tc_params(p);
    return tc_attend_smem_bytes(tp, p.S, p.d) <= 227 * 1024;
}

}  // namespace

void count_launches(int n) { g_launches.fetch_add((uint64_t)n); }

bool tc_make_map(CUtensorMap *m, const void *base, int d, int64_t rows, int d2,
                 int d3, int box_rows) {
    return make_map(m, base, d, rows, d2, d3, box_rows);
}

bool tc_maps_available() { return encode_fn() != nullptr; }
uint64_t launch_total() { return g_launches.load(); }

bool fast_path_supported(const Problem &p) {
    if (p.decode) return p.dtype == HILS_BF16 && encode_fn() && dec_fast_supported(p);
    return attend_supported(p);
}

bool fast_select_supported(const Problem &p) {
    if (p.decode) return p.dtype == HILS_BF16 && encode_fn() && dec_fast_supported(p);
    if (p.dtype != HILS_BF16) return false;
    if (!(p.d == 64 || p.d == 128)) return false;
    if (128 % p.G != 0 || p.nC < 1) return false;
    if (!encode_fn()) return false;
    TcParams tp = tc_params(p);
    return tc_score_smem_bytes(tp, p.d) <= 227 * 1024;
}

size_t fast_workspace_bytes(const Problem &p) {
    return p.decode ? dec_workspace_bytes(p) : 0;
}

cudaError_t launch_fast_select(Problem &p, void *ws, size_t ws_bytes,
                               cudaStream_t st) {
    (void)ws_bytes;
    if (p.decode) return launch_dec_select(p, ws, st);
    TcParams tp = tc_params(p);
    const void *qhat = p.Qs ? p.Qs : p.Q;
    cudaError_t e;
    if (tc_select_supported(tp)) {
        // one thread per query, all heads of the group in its TMEM lane
        CUtensorMap lm32, q128;
        if (!make_map(&lm32, p.Klm, p.d, p.nC, p.Hkv, p.B, 32) ||
            !make_map(&q128, qhat, p.d, p.n_query, p.Hq, p.B, 128))
            return cudaErrorInvalidValue;
        e = launch_tc_select(tp, lm32, q128, st);
    } else {
        // wider groups (G > 4) or K > 32: per-row heaps
        TcMaps maps;
        if (!make_map(&maps.lm, p.Klm, p.d, p.nC, p.Hkv, p.B, 128))
            return cudaErrorInvalidValue;
        e = launch_tc_score(tp, maps, qhat, st);
    }
    count_launches(1);
    return e;
}

cudaError_t launch_fast_attend(Problem &p, void *ws, size_t ws_bytes,
                               cudaStream_t st) {
    (void)ws_bytes;
    if (p.decode) return launch_dec_attend(p, ws, st);
    TcParams tp = tc_params(p);
    TcMaps maps;
    if (!make_map(&maps.k, p.Kc, p.d, p.kv_rows, p.Hkv, p.B, p.S) ||
        !make_map(&maps.v, p.V, p.d, p.kv_rows, p.Hkv, p.B, p.S))
        return cudaErrorInvalidValue;
    cudaError_t e = launch_tc_attend(tp, maps, st);
    count_launches(1);
    return e;
}

}  // namespace hils
