// landmarks.cu -- landmark summaries (k', b') of every chunk, HBM-bound.
//
// "Hierarchical Sparse Attention Done Right", Sec. 3 (answering RQ1, the
// surrogate of Eq. 7): (k'_c, b'_c) = Attn(q'_c, K_c, K_c), i.e. with
// p = softmax_j(q'_c . k_j / sqrt(d)) over the chunk's S keys, k'_c the
// p-weighted key sum and b'_c the entropy of p; Sec. 4.1 for the shared
// per-kv-head query variant.
//
// One warp per chunk, chunks spread over a grid-stride loop. Lane j scores
// tokens j, j+32, ... (each key row read as 16-byte units, q' broadcast from
// shared memory), the softmax statistics are warp reductions, and the
// weighted key sum runs over the tokens with lane l owning dims
// [l*d/32, (l+1)*d/32) (the second pass over the chunk hits L1). The keys are
// read from HBM once: the kernel streams K.
#include <math.h>
#include <stdint.h>

#include "hils_fast.cuh"

namespace hils {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// one 16-byte unit of a key row: its element count and its dot product
// with the matching q' values
template <typename T>
struct Unit;

template <>
struct Unit<__nv_bfloat16> {
    static constexpr int E = 8;                 // elements per 16 bytes
    __device__ static float dot(const uint4 &u, const float *q) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        float a = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            a = fmaf(__uint_as_float(w[k] << 16), q[2 * k], a);
            a = fmaf(__uint_as_float(w[k] & 0xffff0000u), q[2 * k + 1], a);
        }
        return a;
    }
};

template <>
struct Unit<float> {
    static constexpr int E = 4;
    __device__ static float dot(const uint4 &u, const float *q) {
        float a = __uint_as_float(u.x) * q[0];
        a = fmaf(__uint_as_float(u.y), q[1], a);
        a = fmaf(__uint_as_float(u.z), q[2], a);
        return fmaf(__uint_as_float(u.w), q[3], a);
    }
};

__device__ __forceinline__ void store_out(float *dst, const float *v, int n) {
    for (int e = 0; e < n; ++e) dst[e] = v[e];
}
__device__ __forceinline__ void store_out(__nv_bfloat16 *dst, const float *v, int n) {
    for (int e = 0; e < n; ++e) dst[e] = __float2bfloat16_rn(v[e]);
}

template <typename T, int D, int TPL>
__global__ void __launch_bounds__(kWarps * 32)
landmark_kernel(const T *__restrict__ Kc, const T *__restrict__ Qlm, int shared_q,
                T *__restrict__ Klm, float *__restrict__ bias, int Hkv, int N,
                int nC, int64_t total, float inv_sqrt_d) {
    constexpr int S = TPL * 32;
    constexpr int E = Unit<T>::E;
    constexpr int UNITS = D / E;                // 16-byte units per key row
    constexpr int DPL = D / 32;                 // dims per lane, weighted sum
    __shared__ float qs[kWarps][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float l2e = 1.4426950408889634f;

    for (int64_t w = (int64_t)blockIdx.x * kWarps + warp; w < total;
         w += (int64_t)gridDim.x * kWarps) {
        const int64_t bg = w / nC;
        const int c = (int)(w - bg * nC);
        const int g = (int)(bg % Hkv);
        const T *k0 = Kc + (bg * N + (int64_t)c * S) * D;
        const T *q = shared_q ? Qlm + (int64_t)g * D : Qlm + w * D;
        for (int e = lane; e < D; e += 32) qs[warp][e] = to_f(q[e]);
        __syncwarp();

        // scores of this lane's tokens lane + 32 s
        float sc[TPL];
        float mx = -INFINITY;
#pragma unroll
        for (int s = 0; s < TPL; ++s) {
            const uint4 *kr = reinterpret_cast<const uint4 *>(k0 + (int64_t)(lane + 32 * s) * D);
            uint4 u[UNITS];
#pragma unroll
            for (int x = 0; x < UNITS; ++x) u[x] = __ldg(kr + x);
            float a = 0.f;
#pragma unroll
            for (int x = 0; x < UNITS; ++x) a += Unit<T>::dot(u[x], &qs[warp][x * E]);
            sc[s] = a * inv_sqrt_d;
            mx = fmaxf(mx, sc[s]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float p[TPL], z = 0.f;
#pragma unroll
        for (int s = 0; s < TPL; ++s) { p[s] = exp2f((sc[s] - mx) * l2e); z += p[s]; }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        const float iz = 1.f / z;
        float ps = 0.f;
#pragma unroll
        for (int s = 0; s < TPL; ++s) { p[s] *= iz; ps = fmaf(p[s], sc[s], ps); }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);

        // k' = sum_j p_j k_j over this lane's dims
        float acc[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
#pragma unroll
        for (int s = 0; s < TPL; ++s) {
#pragma unroll 8
            for (int src = 0; src < 32; ++src) {
                const float pj = __shfl_sync(0xffffffffu, p[s], src);
                const T *kr = k0 + (int64_t)(src + 32 * s) * D + lane * DPL;
                T kv[DPL];
                if (sizeof(T) * DPL == 8)
                    *reinterpret_cast<uint2 *>(kv) = __ldg(reinterpret_cast<const uint2 *>(kr));
                else if (sizeof(T) * DPL == 16)
                    *reinterpret_cast<uint4 *>(kv) = __ldg(reinterpret_cast<const uint4 *>(kr));
                else
                    for (int e = 0; e < DPL; ++e) kv[e] = kr[e];
#pragma unroll
                for (int e = 0; e < DPL; ++e) acc[e] = fmaf(pj, to_f(kv[e]), acc[e]);
            }
        }
        store_out(Klm + w * D + lane * DPL, acc, DPL);
        // entropy = LSE - sum_j p_j s_j
        if (lane == 0) bias[w] = (mx + logf(z)) - ps;
        __syncwarp();                            // qs is rewritten next chunk
    }
}

template <typename T, int D>
cudaError_t launch_d(const hils_landmark_args &a, int nC, int64_t total, int grid,
                     cudaStream_t st) {
    const T *K = static_cast<const T *>(a.Kc);
    const T *Q = static_cast<const T *>(a.Qlm);
    T *O = static_cast<T *>(a.Klm);
    const float isd = 1.f / sqrtf((float)a.d);
    switch (a.S) {
    case 32:
        landmark_kernel<T, D, 1><<<grid, kWarps * 32, 0, st>>>(K, Q, a.shared_query, O, a.bias, a.Hkv, a.N, nC, total, isd);
        break;
    case 64:
        landmark_kernel<T, D, 2><<<grid, kWarps * 32, 0, st>>>(K, Q, a.shared_query, O, a.bias, a.Hkv, a.N, nC, total, isd);
        break;
    case 128:
        landmark_kernel<T, D, 4><<<grid, kWarps * 32, 0, st>>>(K, Q, a.shared_query, O, a.bias, a.Hkv, a.N, nC, total, isd);
        break;
    default:
        landmark_kernel<T, D, 8><<<grid, kWarps * 32, 0, st>>>(K, Q, a.shared_query, O, a.bias, a.Hkv, a.N, nC, total, isd);
        break;
    }
    return cudaGetLastError();
}

bool al16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace
}  // namespace hils

extern "C" hils_status hils_build_landmarks(const hils_landmark_args *a, void *stream) {
    using namespace hils;
    if (!a) return HILS_ERR_INVALID_ARG;
    if (a->B < 1 || a->Hkv < 1 || a->N < 1 || a->d < 1 || a->S < 1)
        return HILS_ERR_INVALID_ARG;
    if (a->dtype != HILS_F32 && a->dtype != HILS_BF16) return HILS_ERR_INVALID_ARG;
    if (a->shared_query != 0 && a->shared_query != 1) return HILS_ERR_INVALID_ARG;
    if (!(a->d == 64 || a->d == 128)) return HILS_ERR_UNSUPPORTED;
    if (!(a->S == 32 || a->S == 64 || a->S == 128 || a->S == 256)) return HILS_ERR_UNSUPPORTED;
    if (a->N < a->S) return HILS_ERR_INVALID_ARG;
    if (!a->Kc || !a->Qlm || !a->Klm || !a->bias) return HILS_ERR_INVALID_ARG;
    if (!al16(a->Kc) || !al16(a->Qlm) || !al16(a->Klm) || !al16(a->bias))
        return HILS_ERR_MISALIGNED;
    const int nC = a->N / a->S;
    const int64_t total = (int64_t)a->B * a->Hkv * nC;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return HILS_ERR_CUDA;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // up to 4 resident 8-warp CTAs per SM, one wave, chunks grid-strided
    const int64_t want = (total + kWarps - 1) / kWarps;
    const int grid = (int)(want < (int64_t)sms * 4 ? want : (int64_t)sms * 4);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (a->dtype == HILS_BF16)
        e = a->d == 128 ? launch_d<__nv_bfloat16, 128>(*a, nC, total, grid, st)
                        : launch_d<__nv_bfloat16, 64>(*a, nC, total, grid, st);
    else
        e = a->d == 128 ? launch_d<float, 128>(*a, nC, total, grid, st)
                        : launch_d<float, 64>(*a, nC, total, grid, st);
    count_launches(1);
    return e == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
}
