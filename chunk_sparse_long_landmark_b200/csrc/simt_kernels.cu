// simt_kernels.cu -- general-shape HiLS kernels on the CUDA cores (FFMA).
//
// These serve every shape and both element types; they are the float32 path
// (no TF32 anywhere, so float32 results stay within 1e-5 of fp64) and the
// fallback for bf16 shapes outside the tensor-core kernels' tile set.
//
// Paper: "Hierarchical Sparse Attention Done Right", Sec. 2.1 (window and
// candidates), Sec. 3 (surrogate score, top-K, hierarchical softmax),
// Sec. 4.1 (Q-Cal scoring query; GQA group selection).
#include <math.h>

#include "hils_internal.cuh"

namespace hils {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kAttnWarps = 4;
constexpr int kMaxS = 256;      // chunk length limit of the SIMT attention

template <typename T>
__device__ __forceinline__ float ldf(const void *base, int64_t e) {
    return to_f(reinterpret_cast<const T *>(base)[e]);
}

struct ArgMax { float v; int c; };

// a "beats" b: larger value, ties to the lower chunk index.
__device__ __forceinline__ bool beats(float av, int ac, float bv, int bc) {
    return av > bv || (av == bv && ac < bc && ac >= 0);
}

__device__ ArgMax block_argmax(ArgMax x, ArgMax *red) {
    for (int o = 16; o > 0; o >>= 1) {
        float v = __shfl_xor_sync(0xffffffffu, x.v, o);
        int c = __shfl_xor_sync(0xffffffffu, x.c, o);
        if (beats(v, c, x.v, x.c) || x.c < 0) { if (c >= 0) { x.v = v; x.c = c; } }
    }
    int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) red[w] = x;
    __syncthreads();
    ArgMax r = red[0];
    for (int k = 1; k < (int)(blockDim.x >> 5); ++k) {
        ArgMax y = red[k];
        if (y.c >= 0 && (r.c < 0 || beats(y.v, y.c, r.v, r.c))) r = y;
    }
    __syncthreads();
    return r;
}

__device__ float block_reduce(float x, float *red, bool is_max) {
    for (int o = 16; o > 0; o >>= 1) {
        float y = __shfl_xor_sync(0xffffffffu, x, o);
        x = is_max ? fmaxf(x, y) : x + y;
    }
    int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) red[w] = x;
    __syncthreads();
    float r = red[0];
    for (int k = 1; k < (int)(blockDim.x >> 5); ++k)
        r = is_max ? fmaxf(r, red[k]) : r + red[k];
    __syncthreads();
    return r;
}

// Scoring + group top-K, one (b, g, query row) at a time per CTA.
//   scratch: per CTA (G + 1) * nc_stride floats: s^ per head, then a_c.
template <typename T>
__global__ void __launch_bounds__(kScoreThreads)
simt_score_kernel(const Problem p, float *scratch, int64_t nc_stride) {
    extern __shared__ float qs[];                 // [G][d] scoring query
    __shared__ ArgMax red[kScoreThreads / 32];
    __shared__ float redf[kScoreThreads / 32];
    __shared__ float lse[HILS_MAX_GROUP];
    __shared__ int sel[HILS_MAX_TOPK];

    const int G = p.G, d = p.d, K = p.K;
    float *sc = scratch + (int64_t)blockIdx.x * (G + 1) * nc_stride;
    float *av = sc + (int64_t)G * nc_stride;
    const int64_t total = (int64_t)p.B * p.Hkv * p.n_query;
    const void *qb = p.Qs ? p.Qs : p.Q;

    for (int64_t rg = blockIdx.x; rg < total; rg += gridDim.x) {
        const int r = (int)(rg % p.n_query);
        const int g = (int)((rg / p.n_query) % p.Hkv);
        const int b = (int)(rg / ((int64_t)p.n_query * p.Hkv));
        int64_t i = r;
        if (p.decode) {
            int L = p.cache_len[b];
            if (L < 1 || L > p.kv_rows) {
                if (threadIdx.x == 0) report(p.status, HILS_ERR_DEVICE_BAD_LENGTH);
                continue;
            }
            i = L - 1;
        }
        int64_t w0, nc;
        window_bounds(i, p.S, p.W, &w0, &nc);
        if (nc > nc_stride) nc = nc_stride;      // host sizes nc_stride >= max nc

        for (int e = threadIdx.x; e < G * d; e += blockDim.x) {
            int hh = e / d, k = e % d;
            int h = p.group_heads[g * G + hh];
            qs[e] = ldf<T>(qb, (((int64_t)b * p.Hq + h) * p.n_query + r) * d + k);
        }
        __syncthreads();

        // s^_c = q^ . k'_c / sqrt(d) + b'_c for every head of the group
        const int64_t lmo = ((int64_t)b * p.Hkv + g) * p.nC;
        for (int64_t c = threadIdx.x; c < nc; c += blockDim.x) {
            float acc[HILS_MAX_GROUP];
#pragma unroll
            for (int hh = 0; hh < HILS_MAX_GROUP; ++hh) acc[hh] = 0.f;
            for (int k = 0; k < d; ++k) {
                float kv = ldf<T>(p.Klm, (lmo + c) * d + k);
#pragma unroll
                for (int hh = 0; hh < HILS_MAX_GROUP; ++hh)
                    if (hh < G) acc[hh] = fmaf(qs[hh * d + k], kv, acc[hh]);
            }
            float bc = p.bias[lmo + c];
            for (int hh = 0; hh < G; ++hh)
                sc[hh * nc_stride + c] = fmaf(acc[hh], p.inv_sqrt_d, bc);
        }
        __syncthreads();

        // per-head normaliser over C_i (Sec. 4.1)
        for (int hh = 0; hh < G; ++hh) {
            float m = -INFINITY;
            for (int64_t c = threadIdx.x; c < nc; c += blockDim.x)
                m = fmaxf(m, sc[hh * nc_stride + c]);
            m = block_reduce(m, redf, true);
            float s = 0.f;
            for (int64_t c = threadIdx.x; c < nc; c += blockDim.x)
                s += expf(sc[hh * nc_stride + c] - m);
            s = block_reduce(s, redf, false);
            if (threadIdx.x == 0) lse[hh] = m + logf(s);
        }
        __syncthreads();
        for (int64_t c = threadIdx.x; c < nc; c += blockDim.x) {
            float a = -INFINITY;
            for (int hh = 0; hh < G; ++hh)
                a = fmaxf(a, sc[hh * nc_stride + c] - lse[hh]);
            av[c] = a;
        }
        __syncthreads();

        // top-K by a_c, ties to the lower index (K rounds of block argmax)
        const int nsel = (int)(nc < K ? nc : K);
        for (int k = 0; k < nsel; ++k) {
            ArgMax x{-INFINITY, -1};
            for (int64_t c = threadIdx.x; c < nc; c += blockDim.x) {
                float v = av[c];
                if (v != -INFINITY || x.c < 0) {
                    if (x.c < 0 || beats(v, (int)c, x.v, x.c)) { x.v = v; x.c = (int)c; }
                }
            }
            // every a_c of a candidate is finite, so a taken chunk (set to
            // -inf) loses to every untaken one; nsel <= nc keeps one untaken
            ArgMax best = block_argmax(x, red);
            if (threadIdx.x == 0) { sel[k] = best.c; av[best.c] = -INFINITY; }
            __syncthreads();
        }
        if (threadIdx.x == 0) {                  // ascending order
            for (int a = 1; a < nsel; ++a) {
                int v = sel[a], j = a - 1;
                while (j >= 0 && sel[j] > v) { sel[j + 1] = sel[j]; --j; }
                sel[j + 1] = v;
            }
        }
        __syncthreads();
        int32_t *io = p.idx + (((int64_t)b * p.Hkv + g) * p.n_query + r) * K;
        for (int k = threadIdx.x; k < K; k += blockDim.x) io[k] = k < nsel ? sel[k] : -1;
        for (int e = threadIdx.x; e < G * K; e += blockDim.x) {
            int hh = e / K, k = e % K;
            int h = p.group_heads[g * G + hh];
            p.sel[(((int64_t)b * p.Hq + h) * p.n_query + r) * K + k] =
                k < nsel ? sc[hh * nc_stride + sel[k]] : __int_as_float(0x7fc00000);
        }
        __syncthreads();
    }
}

// Attention + hierarchical fusion: one warp per (b, h, query row).
template <typename T>
__global__ void __launch_bounds__(kAttnWarps * 32)
simt_attend_kernel(const Problem p) {
    extern __shared__ float sm[];
    const int d = p.d, S = p.S, K = p.K;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *qv = sm + warp * (d + kMaxS);          // [d] query
    float *pj = qv + d;                           // [S] chunk logits / weights
    const int64_t row = (int64_t)blockIdx.x * kAttnWarps + warp;
    const int64_t total = (int64_t)p.B * p.Hq * p.n_query;
    if (row >= total) return;
    const int r = (int)(row % p.n_query);
    const int h = (int)((row / p.n_query) % p.Hq);
    const int b = (int)(row / ((int64_t)p.n_query * p.Hq));
    const int g = p.head_map[h];
    int64_t i = r;
    if (p.decode) {
        int L = p.cache_len[b];
        if (L < 1 || L > p.kv_rows) return;     // reported by the scoring kernel
        i = L - 1;
    }
    int64_t w0, nc;
    window_bounds(i, S, p.W, &w0, &nc);

    const int64_t qo = (((int64_t)b * p.Hq + h) * p.n_query + r) * d;
    for (int k = lane; k < d; k += 32) qv[k] = ldf<T>(p.Q, qo + k);
    __syncwarp();
    const int64_t kvo = ((int64_t)b * p.Hkv + g) * p.kv_rows;
    const int32_t *io = p.idx + (((int64_t)b * p.Hkv + g) * p.n_query + r) * K;
    const float *so = p.sel + (((int64_t)b * p.Hq + h) * p.n_query + r) * K;

    constexpr int kMaxDPerLane = HILS_MAX_HEAD_DIM / 32;
    float o[kMaxDPerLane];
#pragma unroll
    for (int u = 0; u < kMaxDPerLane; ++u) o[u] = 0.f;

    // reference point: the largest selected chunk score (every fused chunk
    // weight exp(s - m_c)/z_c * exp(s^_c - M) is then <= 1)
    // idx entries outside C_i (caller-supplied selections) are ignored
    float M = -INFINITY;
    for (int k = 0; k < K; ++k)
        if (io[k] >= 0 && io[k] < nc) M = fmaxf(M, so[k]);
    float l = 0.f;

    auto logit = [&](int64_t j) {
        const int64_t ko = (kvo + j) * d;
        float acc = 0.f;
        for (int k = 0; k < d; ++k) acc = fmaf(qv[k], ldf<T>(p.Kc, ko + k), acc);
        return acc * p.inv_sqrt_d;
    };

    // selected chunks: intra-chunk softmax, weighted by Z^_c (Sec. 3)
    for (int k = 0; k < K; ++k) {
        const int c = io[k];
        if (c < 0 || c >= nc) continue;
        float mc = -INFINITY;
        for (int t = lane; t < S; t += 32) {
            float s = logit((int64_t)c * S + t);
            pj[t] = s;
            mc = fmaxf(mc, s);
        }
        for (int o2 = 16; o2 > 0; o2 >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o2));
        float z = 0.f;
        for (int t = lane; t < S; t += 32) { float e = expf(pj[t] - mc); pj[t] = e; z += e; }
        for (int o2 = 16; o2 > 0; o2 >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o2);
        const float zc = expf(so[k] - M);       // Z^_c / exp(M)
        const float f = zc / z;
        l += zc;
        __syncwarp();
        for (int t = 0; t < S; ++t) {
            const float w = pj[t] * f;
            const int64_t vo = (kvo + (int64_t)c * S + t) * d;
#pragma unroll
            for (int u = 0; u < kMaxDPerLane; ++u) {
                int k2 = lane + 32 * u;
                if (k2 < d) o[u] = fmaf(w, ldf<T>(p.V, vo + k2), o[u]);
            }
        }
        __syncwarp();
    }

    // aligned window [w0, i]: plain softmax mass, online max (Sec. 2.1)
    for (int64_t j0 = w0; j0 <= i; j0 += 32) {
        const int64_t j = j0 + lane;
        float s = (j <= i) ? logit(j) : -INFINITY;
        float mx = s;
        for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
        const float Mn = fmaxf(M, mx);
        const float scale = (M == -INFINITY) ? 0.f : expf(M - Mn);
        l *= scale;
#pragma unroll
        for (int u = 0; u < kMaxDPerLane; ++u) o[u] *= scale;
        M = Mn;
        float e = (j <= i) ? expf(s - M) : 0.f;
        pj[lane] = e;
        float es = e;
        for (int o2 = 16; o2 > 0; o2 >>= 1) es += __shfl_xor_sync(0xffffffffu, es, o2);
        l += es;
        __syncwarp();
        const int nt = (int)((i - j0 + 1) < 32 ? (i - j0 + 1) : 32);
        for (int t = 0; t < nt; ++t) {
            const float w = pj[t];
            const int64_t vo = (kvo + j0 + t) * d;
#pragma unroll
            for (int u = 0; u < kMaxDPerLane; ++u) {
                int k2 = lane + 32 * u;
                if (k2 < d) o[u] = fmaf(w, ldf<T>(p.V, vo + k2), o[u]);
            }
        }
        __syncwarp();
    }

    T *out = reinterpret_cast<T *>(p.O) + qo;
    const float inv = 1.f / l;
#pragma unroll
    for (int u = 0; u < kMaxDPerLane; ++u) {
        int k2 = lane + 32 * u;
        if (k2 < d) out[k2] = from_f<T>(o[u] * inv);
    }
}

}  // namespace

int simt_score_grid(const Problem &p) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t total = (int64_t)p.B * p.Hkv * p.n_query;
    int64_t g = (int64_t)sms * 8;
    return (int)(total < g ? total : g);
}

size_t simt_score_scratch_floats(const Problem &p, int nc_max) {
    return (size_t)(p.G + 1) * (size_t)(nc_max > 0 ? nc_max : 1);
}

cudaError_t launch_simt_score(const Problem &p, float *scratch, int grid,
                              cudaStream_t st) {
    int64_t w0, ncm;
    window_bounds((int64_t)p.kv_rows - 1, p.S, p.W, &w0, &ncm);
    const int64_t stride = ncm > 0 ? ncm : 1;
    const size_t smem = sizeof(float) * p.G * p.d;
    if (grid <= 0) return cudaSuccess;
    if (p.dtype == HILS_BF16)
        simt_score_kernel<__nv_bfloat16><<<grid, kScoreThreads, smem, st>>>(p, scratch, stride);
    else
        simt_score_kernel<float><<<grid, kScoreThreads, smem, st>>>(p, scratch, stride);
    return cudaGetLastError();
}

cudaError_t launch_simt_attend(const Problem &p, cudaStream_t st) {
    const int64_t total = (int64_t)p.B * p.Hq * p.n_query;
    const int64_t grid = (total + kAttnWarps - 1) / kAttnWarps;
    const size_t smem = sizeof(float) * kAttnWarps * (p.d + kMaxS);
    if (grid <= 0) return cudaSuccess;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (p.dtype == HILS_BF16)
        simt_attend_kernel<__nv_bfloat16><<<(unsigned)grid, kAttnWarps * 32, smem, st>>>(p);
    else
        simt_attend_kernel<float><<<(unsigned)grid, kAttnWarps * 32, smem, st>>>(p);
    return cudaGetLastError();
}

int simt_max_chunk() { return kMaxS; }

}  // namespace hils
