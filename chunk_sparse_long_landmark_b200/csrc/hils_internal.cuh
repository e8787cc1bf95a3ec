// hils_internal.cuh -- definitions shared by the kernels and the host side of
// libhils. Not part of the public ABI (that is include/hils.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hils.h"

namespace hils {

constexpr int kMaxHeads = 256;   // Hq limit of the kernel parameter tables

// One problem, as every kernel sees it. Prefill and decode share the shape
// of this record: a decode step is the prefill computation at the single
// position i = cache_len[b]-1 (n_query = 1, q_rows = 1, kv_rows = Lmax).
struct Problem {
    const void *Q, *Qs, *Kc, *V, *Klm;
    const float *bias;
    void *O;
    int32_t *idx;
    float *sel;                  // s^ of the selected chunks [B,Hq,n_query,K]
    const int32_t *cache_len;    // decode only
    const int32_t *block_table;  // decode over a paged cache: [B, kv_rows/S]
    int n_pages;                 // pages of S tokens in the pool (paged only)
    int32_t *status;             // nullable
    int B, Hq, Hkv, G, d, S, W, K;
    int n_query;                 // query rows per (b, h): N, or T (decode)
    int T;                       // decode: query tokens per sequence (1: plain)
    int kv_rows;                 // token rows per (b, g): N or Lmax
    int nC;                      // landmark rows per (b, g)
    int decode;                  // 1: position from cache_len
    int dtype;                   // hils_dtype of Q, Qs, Kc, V, Klm, O
    float inv_sqrt_d;
    int16_t group_heads[kMaxHeads];  // group g's heads at [g*G .. g*G+G)
    int16_t head_map[kMaxHeads];
};

__host__ __device__ inline int64_t floordiv64(int64_t a, int64_t b) {
    int64_t q = a / b;
    if ((a % b != 0) && ((a < 0) != (b < 0))) q -= 1;
    return q;
}

// Window start w0 = max(l(i), 0) and candidate count nc = max(l(i)/S, 0),
// l(i) = floor((i - W + 1)/S) * S.
__host__ __device__ inline void window_bounds(int64_t i, int S, int W,
                                              int64_t *w0, int64_t *nc) {
    int64_t lq = floordiv64(i - W + 1, S);
    *nc = lq > 0 ? lq : 0;
    *w0 = lq > 0 ? lq * S : 0;
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ void report(int32_t *status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// Process-wide count of kernel launches enqueued by the library.
void count_launches(int n);
uint64_t launch_total();

// Kernel launchers (defined in the .cu files).
cudaError_t launch_simt_score(const Problem &p, float *scratch, int grid,
                              cudaStream_t st);
cudaError_t launch_simt_attend(const Problem &p, cudaStream_t st);
int simt_score_grid(const Problem &p);
int simt_max_chunk();
size_t simt_score_scratch_floats(const Problem &p, int nc_max);

}  // namespace hils
