// tc_score.cu -- HiLS prefill chunk scoring + group top-K on the sm_100a
// tensor cores.
//
// "Hierarchical Sparse Attention Done Right": Sec. 3 (surrogate score
// s^_ic = q^_i.k'_c/sqrt(d) + b'_c, top-K), Sec. 4.1 (Q-Cal scoring query;
// GQA: per-head normalised chunk weights, max over the group's heads, one
// top-K set per group).
//
// One CTA owns the G heads of one kv group x M = 128/G adjacent queries, as
// 128 query-major rows (row r = query_slot * G + head_slot, so a query's
// heads sit in adjacent lanes of one warp). The scoring query tile Q^ stays
// in shared memory; landmark-key tiles of 128 chunks stream in by TMA and
//   S = Q^ K'^T   tcgen05.mma, 128 x 128, f32 in TMEM
// is computed twice per tile:
//   pass 1  per row: x = S/sqrt(d) + b' (log2 units), masked to C_i, online
//           log-sum-exp  -> LSE of the row's head over C_i;
//   pass 2  a = x - LSE, max over the G lanes of the query (shuffles) = the
//           group score; every lane of the query keeps an identical min-heap
//           of the K best (a, c) (ties: lower c ranks higher) whose payload
//           is its own head's s^_c, so no score is recomputed afterwards.
// Output: idx [B,Hkv,N,K] ascending, -1 padded; s^ of the selected chunks
// [B,Hq,N,K] in idx order, NaN on padding.
#include <math.h>

#include "hils_fast.cuh"
#include "sm100.cuh"
#include "tc_kernels.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kRows = 128;
constexpr int kTileC = 128;            // chunks per MMA tile
constexpr int kStages = 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kGrp = 16;               // columns per candidate group (pass 2)

template <int D>
struct ScoreLayout {
    static constexpr uint32_t Q_BYTES = kRows * D * 2;
    static constexpr uint32_t KT_BYTES = kTileC * D * 2;
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = Q_BYTES;
    static constexpr uint32_t OFF_BIAS = OFF_K + kStages * KT_BYTES;  // 4 warps x 128 f32
    static constexpr uint32_t OFF_SMALL = OFF_BIAS + 4 * kTileC * 4;
};

struct ScoreState {
    uint64_t kv_full[kStages];
    uint64_t kv_empty[kStages];
    uint64_t s_full[2];
    uint64_t s_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort;
};

// Heap entry order: x ranks below y iff x.a < y.a, or equal a and x.c > y.c.
__device__ __forceinline__ bool below(float a1, int c1, float a2, int c2) {
    return a1 < a2 || (a1 == a2 && c1 > c2);
}

// Min-heap over the K best candidates of a row (arrays [K][kRows], column r
// of the row): the root is the lowest-ranked entry, i.e. the K-th best.
// Sift (a, c, s) down from `pos` into a heap of `n` entries.
__device__ __forceinline__ void heap_sift_down(float *h_a, int *h_c, float *h_s,
                                               int r, int n, int pos, float a,
                                               int c, float s) {
    for (;;) {
        const int l1 = 2 * pos + 1;
        if (l1 >= n) break;
        int ch = l1;
        float ca = h_a[l1 * kRows + r];
        int cc = h_c[l1 * kRows + r];
        if (l1 + 1 < n) {
            const float ra = h_a[(l1 + 1) * kRows + r];
            const int rc = h_c[(l1 + 1) * kRows + r];
            if (below(ra, rc, ca, cc)) { ch = l1 + 1; ca = ra; cc = rc; }
        }
        if (!below(ca, cc, a, c)) break;
        h_a[pos * kRows + r] = ca;
        h_c[pos * kRows + r] = cc;
        h_s[pos * kRows + r] = h_s[ch * kRows + r];
        pos = ch;
    }
    h_a[pos * kRows + r] = a;
    h_c[pos * kRows + r] = c;
    h_s[pos * kRows + r] = s;
}

// Offer candidate (a, c, s) to the row's top-K. The first K offers are
// appended as they come and heapified once (Floyd) when the K-th arrives;
// after that an offer replaces the root if it ranks above it. Chunks arrive
// in ascending order, so an offer equal to the root in score ranks below it.
// Returns the new count.
__device__ __forceinline__ int topk_offer(float *h_a, int *h_c, float *h_s,
                                          int r, int K, int cnt, float a,
                                          int c, float s) {
    if (cnt < K) {
        h_a[cnt * kRows + r] = a;
        h_c[cnt * kRows + r] = c;
        h_s[cnt * kRows + r] = s;
        ++cnt;
        if (cnt == K)
            for (int pos = K / 2 - 1; pos >= 0; --pos)
                heap_sift_down(h_a, h_c, h_s, r, K, pos, h_a[pos * kRows + r],
                               h_c[pos * kRows + r], h_s[pos * kRows + r]);
        return cnt;
    }
    if (below(h_a[r], h_c[r], a, c))
        heap_sift_down(h_a, h_c, h_s, r, K, 0, a, c, s);
    return cnt;
}

template <int D, int KMAX>
__global__ void __launch_bounds__(kThreads, 1)
tc_score_kernel(const __grid_constant__ CUtensorMap tmL, const void *qhat,
                const TcParams p) {
    using L = ScoreLayout<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    ScoreState &st = *reinterpret_cast<ScoreState *>(smem + L::OFF_SMALL);
    // per-row heaps, column r of [K][128]: group score, chunk, own s^
    float *h_a = reinterpret_cast<float *>(smem + L::OFF_SMALL + 128);
    int *h_c = reinterpret_cast<int *>(h_a + p.K * kRows);
    float *h_s = reinterpret_cast<float *>(h_c + p.K * kRows);
    float *slot_a = h_s + p.K * kRows;           // [kGrp][128] spill of one group
    float *slot_x = slot_a + kGrp * kRows;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.G, M = p.M;
    const int nqb = (p.N + M - 1) / M;
    const int qb = blockIdx.x % nqb;
    const int g = (blockIdx.x / nqb) % p.Hkv;
    const int b = blockIdx.x / (nqb * p.Hkv);
    const int i0 = qb * M;
    const int i_last = min(i0 + M, p.N) - 1;
    int64_t w0x, nc_max;
    window_bounds(i_last, p.S, p.W, &w0x, &nc_max);
    const int nT = (int)((nc_max + kTileC - 1) / kTileC);
    volatile int *abort = &st.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&st.kv_full[s], 1);
            mbar_init(&st.kv_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&st.s_full[s], 1);
            mbar_init(&st.s_empty[s], 128);
        }
        mbar_init(&st.mma_done, 1);
        st.abort = (p.status && *(volatile int32_t *)p.status ==
                                    HILS_ERR_DEVICE_TIMEOUT) ? 1 : 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(&st.tmem_base, 256);
    if (warp == 0 && lane == 0) prefetch_tmap(&tmL);

    // scoring-query tile, query-major rows, K-major 128B-swizzled halves;
    // every load is issued before the first store so they overlap
    {
        constexpr int kUnits = kRows * (D / 8);           // 16-byte units
        constexpr int kPer = (kUnits + kThreads - 1) / kThreads;
        uint4 v[kPer];
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int e = threadIdx.x + q * kThreads;
            v[q] = make_uint4(0, 0, 0, 0);
            if (e < kUnits) {
                const int r = e / (D / 8), u = e % (D / 8);
                const int i = i0 + r / G;
                if (i < p.N) {
                    const int h = p.group_heads[g * G + r % G];
                    v[q] = __ldg(reinterpret_cast<const uint4 *>(
                        reinterpret_cast<const __nv_bfloat16 *>(qhat) +
                        (((int64_t)b * p.Hq + h) * p.N + i) * D + u * 8));
                }
            }
        }
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int e = threadIdx.x + q * kThreads;
            if (e < kUnits) {
                const int r = e / (D / 8), u = e % (D / 8);
                const int half = u >> 3, uu = u & 7;
                *reinterpret_cast<uint4 *>(smem + L::OFF_Q + half * (kRows * 128) +
                                           r * 128 + ((uu ^ (r & 7)) << 4)) = v[q];
            }
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = st.tmem_base;
    const int T = st.abort ? 0 : 2 * nT;        // two passes over the tiles

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0 && T > 0) {
            int issued = 0;
            for (int t = 0; t < T; ++t) {
                const int s = t % kStages;
                if (t >= kStages &&
                    !mbar_wait(&st.kv_empty[s], ((t / kStages) - 1) & 1, abort))
                    break;
                const int tt = t % nT;
                mbar_expect_tx(&st.kv_full[s], L::KT_BYTES);
                for (int dh = 0; dh < D / 64; ++dh)
                    tma_load_4d(smem + L::OFF_K + s * L::KT_BYTES + dh * (kTileC * 128),
                                &tmL, &st.kv_full[s], dh * 64, tt * kTileC, g, b);
                issued = t + 1;
            }
            if (*abort)
                for (int t = (issued > kStages ? issued - kStages : 0); t < issued; ++t)
                    mbar_drain(&st.kv_full[t % kStages], (t / kStages) & 1);
        }
    } else if (warp == 1) {
        // ----------------------------------------------------- MMA issuer
        if (lane == 0 && T > 0) {
            constexpr uint32_t id = idesc_bf16(kRows, kTileC, false);
            const uint32_t sQ = smem_u32(smem + L::OFF_Q);
            const uint32_t sK = smem_u32(smem + L::OFF_K);
            for (int t = 0; t < T; ++t) {
                const int s = t % kStages, sb = t & 1;
                if (!mbar_wait(&st.kv_full[s], (t / kStages) & 1, abort)) break;
                if (t >= 2 && !mbar_wait(&st.s_empty[sb], ((t >> 1) - 1) & 1, abort)) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint64_t ad = desc_sw128(sQ + (k / 4) * (kRows * 128) + (k % 4) * 32, 16, 1024);
                    const uint64_t bd = desc_sw128(sK + s * L::KT_BYTES + (k / 4) * (kTileC * 128) + (k % 4) * 32, 16, 1024);
                    mma_ss(tmem + sb * kTileC, ad, bd, id, k > 0 ? 1u : 0u);
                }
                mma_commit(&st.s_full[sb]);
                mma_commit(&st.kv_empty[s]);
            }
            mma_commit(&st.mma_done);
            mbar_drain(&st.mma_done, 0);
        }
    } else {
        // ------------------------------------------- scoring epilogue warps
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int m = r / G, hh = r % G;
        const int i = i0 + m;
        const bool valid = i < p.N;
        const int h = p.group_heads[g * G + (valid ? hh : 0)];
        int64_t w0, nc = 0;
        if (valid) window_bounds(i, p.S, p.W, &w0, &nc);
        float *bias_w = reinterpret_cast<float *>(smem + L::OFF_BIAS) + quad * kTileC;
        const float *bias_g = p.bias + ((int64_t)b * p.Hkv + g) * p.nC;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        const float sl2 = p.inv_sqrt_d * kLog2e;
        const int K = p.K;

        float m_run = -INFINITY, s_run = 0.f, lse2 = 0.f;
        int cnt = 0;
        float thr = -INFINITY;
        bool ok = true;

        // bias of a tile's 128 chunks: 4 per lane, loaded one tile ahead
        // (scalar loads: a kv head's bias row need not be 16-byte aligned)
        auto load_bias = [&](int t) {
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (t < T) {
                const int c = (t % nT) * kTileC + lane * 4;
                if (c + 0 < p.nC) v.x = bias_g[c + 0];
                if (c + 1 < p.nC) v.y = bias_g[c + 1];
                if (c + 2 < p.nC) v.z = bias_g[c + 2];
                if (c + 3 < p.nC) v.w = bias_g[c + 3];
            }
            return v;
        };
        float4 bnext = load_bias(0);
        for (int t = 0; t < T; ++t) {
            const int sb = t & 1;
            const bool pass2 = t >= nT;
            const int c0 = (t % nT) * kTileC;
            {
                float4 bv = bnext;
                bv.x *= kLog2e; bv.y *= kLog2e; bv.z *= kLog2e; bv.w *= kLog2e;
                __syncwarp();                       // previous tile's reads done
                *reinterpret_cast<float4 *>(bias_w + lane * 4) = bv;
                __syncwarp();
                bnext = load_bias(t + 1);
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&st.s_full[sb], (t >> 1) & 1, abort))) { ok = false; break; }
            tc_fence_after();
            float x[kTileC];
#pragma unroll
            for (int q0 = 0; q0 < kTileC; q0 += 32) {
                uint32_t rr[32];
                tmem_ld32(trow + sb * kTileC + q0, rr);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    x[q0 + j] = fmaf(__uint_as_float(rr[j]), sl2, bias_w[q0 + j]);
            }
            tc_fence_before();
            mbar_arrive(&st.s_empty[sb]);
            const int lim = (int)(nc - c0);            // valid columns of this row

            if (!pass2) {
                float mt = -INFINITY;
#pragma unroll
                for (int j = 0; j < kTileC; ++j) if (j < lim) mt = fmaxf(mt, x[j]);
                if (mt > -INFINITY) {
                    const float mn = fmaxf(m_run, mt);
                    float acc = 0.f;
#pragma unroll
                    for (int j = 0; j < kTileC; ++j)
                        if (j < lim) acc += fast_exp2(x[j] - mn);
                    s_run = s_run * fast_exp2(m_run - mn) + acc;
                    m_run = mn;
                }
                if (t == nT - 1) lse2 = (s_run > 0.f) ? m_run + __log2f(s_run) : 0.f;
            } else {
                // group score of 16 columns at a time; the rare columns that
                // beat the current K-th best go through a per-thread slot in
                // shared memory to the heap (runtime-indexed)
#pragma unroll
                for (int q0 = 0; q0 < kTileC; q0 += kGrp) {
                    float a[kGrp];
                    uint32_t bits = 0;
#pragma unroll
                    for (int j = 0; j < kGrp; ++j)
                        a[j] = (q0 + j < lim) ? x[q0 + j] - lse2 : -INFINITY;
                    for (int o = 1; o < G; o <<= 1) {     // 16 independent chains
#pragma unroll
                        for (int j = 0; j < kGrp; ++j)
                            a[j] = fmaxf(a[j], __shfl_xor_sync(0xffffffffu, a[j], o));
                    }
#pragma unroll
                    for (int j = 0; j < kGrp; ++j)
                        bits |= (a[j] > thr ? 1u : 0u) << j;
                    if (bits) {
#pragma unroll
                        for (int j = 0; j < kGrp; ++j) {
                            slot_a[j * kRows + r] = a[j];
                            slot_x[j * kRows + r] = x[q0 + j];
                        }
                        while (bits) {
                            const int j = __ffs(bits) - 1;
                            bits &= bits - 1;
                            const float aj = slot_a[j * kRows + r];
                            if (!(aj > thr)) continue;
                            cnt = topk_offer(h_a, h_c, h_s, r, K, cnt, aj,
                                             c0 + q0 + j, slot_x[j * kRows + r] * kLn2);
                            if (cnt == K) thr = h_a[r];   // root = K-th best
                        }
                    }
                }
            }
        }

        // heap -> ascending chunk order -> outputs: rank of every entry among
        // the row's (distinct) chunks, computed from registers
        if (ok && valid) {
            int cr[KMAX];
            float sr[KMAX];
#pragma unroll
            for (int k = 0; k < KMAX; ++k) {
                cr[k] = k < cnt ? h_c[k * kRows + r] : 0x7fffffff;
                sr[k] = k < cnt ? h_s[k * kRows + r] : 0.f;
            }
            float *so = p.sel + (((int64_t)b * p.Hq + h) * p.N + i) * K;
            int32_t *io = p.idx + (((int64_t)b * p.Hkv + g) * p.N + i) * K;
#pragma unroll
            for (int k = 0; k < KMAX; ++k) {
                if (k < cnt) {
                    int rank = 0;
#pragma unroll
                    for (int k2 = 0; k2 < KMAX; ++k2) rank += (cr[k2] < cr[k]) ? 1 : 0;
                    so[rank] = sr[k];
                    if (hh == 0) io[rank] = cr[k];
                }
            }
            for (int k = cnt; k < K; ++k) {
                so[k] = __int_as_float(0x7fc00000);
                if (hh == 0) io[k] = -1;
            }
        }
    }

    if (*abort && (threadIdx.x & 31) == 0) report(p.status, HILS_ERR_DEVICE_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace

size_t tc_score_smem_bytes(const TcParams &tp, int d) {
    return 1024 + (size_t)kRows * d * 2 + (size_t)kStages * kTileC * d * 2 +
           4 * kTileC * 4 + 128 + (size_t)3 * tp.K * kRows * 4 +
           (size_t)2 * kGrp * kRows * 4;
}

template <int D, int KMAX>
cudaError_t launch_score_t(const TcParams &tp, const TcMaps &maps,
                           const void *qhat, size_t smem, unsigned grid,
                           cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(tc_score_kernel<D, KMAX>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    tc_score_kernel<D, KMAX><<<grid, kThreads, smem, st>>>(maps.lm, qhat, tp);
    return cudaGetLastError();
}

cudaError_t launch_tc_score(const TcParams &tp, const TcMaps &maps,
                            const void *qhat, cudaStream_t st) {
    const size_t smem = tc_score_smem_bytes(tp, tp.d);
    const int nqb = (tp.N + tp.M - 1) / tp.M;
    const int64_t grid = (int64_t)tp.B * tp.Hkv * nqb;
    if (grid <= 0) return cudaSuccess;
    const unsigned gr = (unsigned)grid;
    if (tp.d == 128) {
        if (tp.K <= 16) return launch_score_t<128, 16>(tp, maps, qhat, smem, gr, st);
        if (tp.K <= 32) return launch_score_t<128, 32>(tp, maps, qhat, smem, gr, st);
        return launch_score_t<128, 64>(tp, maps, qhat, smem, gr, st);
    }
    if (tp.d == 64) {
        if (tp.K <= 16) return launch_score_t<64, 16>(tp, maps, qhat, smem, gr, st);
        if (tp.K <= 32) return launch_score_t<64, 32>(tp, maps, qhat, smem, gr, st);
        return launch_score_t<64, 64>(tp, maps, qhat, smem, gr, st);
    }
    return cudaErrorNotSupported;
}

}  // namespace hils
