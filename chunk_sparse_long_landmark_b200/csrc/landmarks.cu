// landmarks.cu -- landmark summaries (k', b') of every chunk, HBM-bound.
//
// "Hierarchical Sparse Attention Done Right", Sec. 3 (answering RQ1, the
// surrogate of Eq. 7): (k'_c, b'_c) = Attn(q'_c, K_c, K_c), i.e. with
// p = softmax_j(q'_c . k_j / sqrt(d)) over the chunk's S keys, k'_c the
// p-weighted key sum and b'_c the entropy of p; Sec. 4.1 for the shared
// per-kv-head query variant.
//
// One warp per chunk, chunks spread over a grid-stride loop. A chunk's keys
// are one contiguous S x d block: the warp copies it (and q'_c) into its own
// shared-memory buffer with cp.async, 16-byte units XOR-swizzled by row, two
// buffers deep so the next chunk is in flight while this one is computed.
// Then lane j scores tokens j, j+32, ...; the softmax statistics are warp
// reductions; and the weighted key sum runs over the tokens with lane l
// owning dims [l*d/32, (l+1)*d/32). Both passes read shared memory without
// bank conflicts; HBM sees every key once.
#include <math.h>
#include <stdint.h>

#include "hils_fast.cuh"

namespace hils {
namespace {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// one 16-byte unit of a key row: its element count and its dot product
// with the matching 16 bytes of q' (same element type)
template <typename T>
struct Unit;

template <>
struct Unit<__nv_bfloat16> {
    static constexpr int E = 8;                 // elements per 16 bytes
    __device__ static float dot(const uint4 &u, const float *q) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        const float4 q0 = *reinterpret_cast<const float4 *>(q);
        const float4 q1 = *reinterpret_cast<const float4 *>(q + 4);
        const float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        float a = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            a = fmaf(__uint_as_float(w[k] << 16), qv[2 * k], a);
            a = fmaf(__uint_as_float(w[k] & 0xffff0000u), qv[2 * k + 1], a);
        }
        return a;
    }
};

template <>
struct Unit<float> {
    static constexpr int E = 4;
    __device__ static float dot(const uint4 &u, const float *q) {
        const float4 qv = *reinterpret_cast<const float4 *>(q);
        float a = __uint_as_float(u.x) * qv.x;
        a = fmaf(__uint_as_float(u.y), qv.y, a);
        a = fmaf(__uint_as_float(u.z), qv.z, a);
        return fmaf(__uint_as_float(u.w), qv.w, a);
    }
};

__device__ __forceinline__ void store_out(float *dst, const float *v, int n) {
    for (int e = 0; e < n; ++e) dst[e] = v[e];
}
__device__ __forceinline__ void store_out(__nv_bfloat16 *dst, const float *v, int n) {
    for (int e = 0; e < n; ++e) dst[e] = __float2bfloat16_rn(v[e]);
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                 :: "r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory");
}

template <typename T, int D, int TPL>
struct LmCfg {
    static constexpr int S = TPL * 32;
    static constexpr int ROWB = D * (int)sizeof(T);          // bytes per key row
    static constexpr int UNITS = ROWB / 16;                  // 16-byte units per row
    static constexpr int CB = S * ROWB;                      // one chunk
    static constexpr int BUF = CB + ROWB;                    // chunk + q'
    static constexpr int BUDGET = 200 * 1024;
    static constexpr int NBUF = (2 * BUF <= BUDGET) ? 2 : 1;
    static constexpr int W0 = BUDGET / (NBUF * BUF);
    static constexpr int WARPS = W0 < 1 ? 1 : (W0 > 8 ? 8 : W0);
    static constexpr int SMEM = WARPS * (NBUF * BUF + D * 4);  // + q' in f32
    static_assert((UNITS & (UNITS - 1)) == 0, "swizzle needs a power of two");
};

template <typename T, int D, int TPL>
__global__ void __launch_bounds__(LmCfg<T, D, TPL>::WARPS * 32)
landmark_kernel(const T *__restrict__ Kc, const T *__restrict__ Qlm, int shared_q,
                T *__restrict__ Klm, float *__restrict__ bias, int Hkv, int N,
                int nC, int64_t total, float inv_sqrt_d) {
    using C = LmCfg<T, D, TPL>;
    constexpr int S = C::S, UNITS = C::UNITS, ROWB = C::ROWB;
    constexpr int DPL = D / 32;                 // dims per lane, weighted sum
    extern __shared__ __align__(16) uint8_t lm_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *wb = lm_smem + warp * (C::NBUF * C::BUF + D * 4);
    float *qf = reinterpret_cast<float *>(wb + C::NBUF * C::BUF);   // q' in f32
    const float l2e = 1.4426950408889634f;
    const int64_t stride = (int64_t)gridDim.x * C::WARPS;

    // chunk w -> buffer bi: key rows with unit u of row r at (u ^ r%UNITS),
    // then q' unswizzled after them
    auto fetch = [&](int64_t w, int bi) {
        const int64_t bg = w / nC;
        const int c = (int)(w - bg * nC);
        const uint8_t *src = reinterpret_cast<const uint8_t *>(
            Kc + (bg * N + (int64_t)c * S) * D);
        uint8_t *dst = wb + bi * C::BUF;
        for (int e = lane; e < S * UNITS; e += 32) {
            const int r = e / UNITS, u = e % UNITS;
            cp_async16(dst + r * ROWB + ((u ^ (r & (UNITS - 1))) << 4), src + (int64_t)e * 16);
        }
        const uint8_t *qs = reinterpret_cast<const uint8_t *>(
            shared_q ? Qlm + (int64_t)(bg % Hkv) * D : Qlm + w * D);
        if (lane < UNITS) cp_async16(dst + C::CB + lane * 16, qs + lane * 16);
        cp_async_commit();
    };

    int64_t w = (int64_t)blockIdx.x * C::WARPS + warp;
    if (w < total) fetch(w, 0);
    for (int it = 0; w < total; w += stride, ++it) {
        const int64_t wn = w + stride;
        if (C::NBUF == 2) {
            if (wn < total) fetch(wn, (it + 1) & 1);
            else cp_async_commit();              // keeps the group count
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncwarp();
        const uint8_t *buf = wb + (C::NBUF == 2 ? (it & 1) : 0) * C::BUF;
        {
            const T *qt = reinterpret_cast<const T *>(buf + C::CB);
            for (int e = lane; e < D; e += 32) qf[e] = to_f(qt[e]);
        }
        __syncwarp();

        // scores of this lane's tokens lane + 32 s
        float sc[TPL];
        float mx = -INFINITY;
#pragma unroll
        for (int s = 0; s < TPL; ++s) {
            const int r = lane + 32 * s;
            const uint8_t *row = buf + r * ROWB;
            float a = 0.f;
#pragma unroll
            for (int x = 0; x < UNITS; ++x)
                a += Unit<T>::dot(*reinterpret_cast<const uint4 *>(
                                      row + ((x ^ (r & (UNITS - 1))) << 4)),
                                  qf + x * Unit<T>::E);
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

        // k' = sum_j p_j k_j over this lane's dims [lane*DPL, +DPL)
        constexpr int LB = DPL * (int)sizeof(T);             // bytes per lane
        const int u0 = (lane * LB) >> 4, o0 = (lane * LB) & 15;
        float acc[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
#pragma unroll
        for (int s = 0; s < TPL; ++s) {
#pragma unroll 8
            for (int src = 0; src < 32; ++src) {
                const int j = src + 32 * s;
                const float pj = __shfl_sync(0xffffffffu, p[s], src);
                const T *kv = reinterpret_cast<const T *>(
                    buf + j * ROWB + ((u0 ^ (j & (UNITS - 1))) << 4) + o0);
#pragma unroll
                for (int e = 0; e < DPL; ++e) acc[e] = fmaf(pj, to_f(kv[e]), acc[e]);
            }
        }
        store_out(Klm + w * D + lane * DPL, acc, DPL);
        // entropy = LSE - sum_j p_j s_j
        if (lane == 0) bias[w] = (mx + logf(z)) - ps;
        __syncwarp();                            // buffer reads done before refill
        if (C::NBUF == 1 && wn < total) fetch(wn, 0);
    }
    cp_async_wait<0>();
}

template <typename T, int D, int TPL>
cudaError_t launch_t(const hils_landmark_args &a, int nC, int64_t total, int sms,
                     cudaStream_t st) {
    using C = LmCfg<T, D, TPL>;
    cudaError_t e = cudaFuncSetAttribute(landmark_kernel<T, D, TPL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM);
    if (e != cudaSuccess) return e;
    const int64_t want = (total + C::WARPS - 1) / C::WARPS;
    const int grid = (int)(want < sms ? want : sms);         // one CTA per SM
    landmark_kernel<T, D, TPL><<<grid, C::WARPS * 32, C::SMEM, st>>>(
        static_cast<const T *>(a.Kc), static_cast<const T *>(a.Qlm), a.shared_query,
        static_cast<T *>(a.Klm), a.bias, a.Hkv, a.N, nC, total,
        1.f / sqrtf((float)a.d));
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_d(const hils_landmark_args &a, int nC, int64_t total, int sms,
                     cudaStream_t st) {
    switch (a.S) {
    case 32: return launch_t<T, D, 1>(a, nC, total, sms, st);
    case 64: return launch_t<T, D, 2>(a, nC, total, sms, st);
    case 128: return launch_t<T, D, 4>(a, nC, total, sms, st);
    default: return launch_t<T, D, 8>(a, nC, total, sms, st);
    }
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
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (a->dtype == HILS_BF16)
        e = a->d == 128 ? launch_d<__nv_bfloat16, 128>(*a, nC, total, sms, st)
                        : launch_d<__nv_bfloat16, 64>(*a, nC, total, sms, st);
    else
        e = a->d == 128 ? launch_d<float, 128>(*a, nC, total, sms, st)
                        : launch_d<float, 64>(*a, nC, total, sms, st);
    count_launches(1);
    return e == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
}
