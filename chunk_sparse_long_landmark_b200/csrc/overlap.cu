// overlap.cu -- chunk-overlap diagnostics of a selection.
//
// "Hierarchical Sparse Attention Done Right", Sec. 7.2: adjacent queries
// retrieve overlapping chunks, Overlap = (M K - |union of I_m|) / ((M-1) K).
// For every block of M consecutive query rows this counts the selected
// entries, the distinct chunks, and the distinct chunks the previous block
// already had.
//
// One warp walks a run of kSeg consecutive blocks of one (batch, kv head)
// (plus the block before the run, for its reuse count). A block's chunks are
// marked in a bitset in shared memory (one bit per chunk, atomicOr), two
// bitsets alternating so the previous block's set is at hand; counts are
// popcounts reduced over the warp. idx is read once (and one block per run
// twice).
#include <stdint.h>

#include "hils_fast.cuh"

namespace hils {
namespace {

constexpr int kOvWarps = 4;
constexpr int kSeg = 16;                         // blocks per warp

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void __launch_bounds__(kOvWarps * 32)
overlap_kernel(const int32_t *__restrict__ idx, int Hkv, int N, int K, int nC,
               int M, int nb, int64_t nruns, int32_t *__restrict__ n_sel,
               int32_t *__restrict__ n_union, int32_t *__restrict__ n_reuse) {
    extern __shared__ uint32_t ov_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwords = (nC + 31) >> 5;
    const int runs_per_bg = (nb + kSeg - 1) / kSeg;
    for (int64_t run = (int64_t)blockIdx.x * kOvWarps + warp; run < nruns;
         run += (int64_t)gridDim.x * kOvWarps) {
        const int64_t bg = run / runs_per_bg;
        const int k0 = (int)(run - bg * runs_per_bg) * kSeg;
        const int k1 = min(k0 + kSeg, nb);
        const int32_t *rows = idx + bg * (int64_t)N * K;
        int cur = 0;
        for (int k = (k0 > 0 ? k0 - 1 : 0); k < k1; ++k) {
            uint32_t *bs = ov_smem + (2 * warp + cur) * nwords;
            for (int w = lane; w < nwords; w += 32) bs[w] = 0u;
            __syncwarp();
            const int r0 = k * M, r1 = min(r0 + M, N);
            const int ne = (r1 - r0) * K;
            int mine = 0;
            for (int e = lane; e < ne; e += 32) {
                const int c = rows[(int64_t)r0 * K + e];
                if (c >= 0 && c < nC) {
                    atomicOr(&bs[c >> 5], 1u << (c & 31));
                    ++mine;
                }
            }
            __syncwarp();
            if (k >= k0) {
                const uint32_t *pv = ov_smem + (2 * warp + (cur ^ 1)) * nwords;
                int u = 0, rr = 0;
                for (int w = lane; w < nwords; w += 32) {
                    u += __popc(bs[w]);
                    if (k > 0) rr += __popc(bs[w] & pv[w]);
                }
                u = warp_sum(u);
                rr = warp_sum(rr);
                mine = warp_sum(mine);
                if (lane == 0) {
                    const int64_t o = bg * nb + k;
                    n_sel[o] = mine;
                    n_union[o] = u;
                    n_reuse[o] = rr;
                }
            }
            __syncwarp();                        // reads of both sets done
            cur ^= 1;
        }
    }
}

}  // namespace
}  // namespace hils

extern "C" hils_status hils_chunk_overlap(const int32_t *idx, int32_t B, int32_t Hkv,
                                          int32_t N, int32_t K, int32_t nC, int32_t M,
                                          int32_t *n_sel, int32_t *n_union,
                                          int32_t *n_reuse, void *stream) {
    using namespace hils;
    if (B < 1 || Hkv < 1 || N < 1 || K < 1 || K > 64 || nC < 1 || M < 2 || M > 128)
        return HILS_ERR_INVALID_ARG;
    if (!idx || !n_sel || !n_union || !n_reuse) return HILS_ERR_INVALID_ARG;
    const int nwords = (nC + 31) >> 5;
    const size_t smem = (size_t)kOvWarps * 2 * nwords * 4;
    if (smem > 200 * 1024) return HILS_ERR_UNSUPPORTED;     // nC > ~200K chunks
    const int nb = (N + M - 1) / M;
    const int64_t nruns = (int64_t)B * Hkv * ((nb + kSeg - 1) / kSeg);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return HILS_ERR_CUDA;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaFuncSetAttribute(overlap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return HILS_ERR_CUDA;
    const int64_t want = (nruns + kOvWarps - 1) / kOvWarps;
    const int grid = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
    overlap_kernel<<<grid, kOvWarps * 32, smem, static_cast<cudaStream_t>(stream)>>>(
        idx, Hkv, N, K, nC, M, nb, nruns, n_sel, n_union, n_reuse);
    count_launches(1);
    return cudaGetLastError() == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
}
