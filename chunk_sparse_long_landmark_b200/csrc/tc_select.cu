// tc_select.cu -- HiLS prefill chunk scoring + group top-K on the sm_100a
// tensor cores, one thread per query.
//
// "Hierarchical Sparse Attention Done Right": Sec. 3 (surrogate score
// s^_ic = q^_i.k'_c/sqrt(d) + b'_c, top-K chunks per query), Sec. 4.1
// (Q-Cal scoring query; GQA: chunk weights normalised per head over the
// candidates, maximum over the group's heads, one selected set per group).
//
// One CTA owns 128 adjacent queries of one kv group. Thread r of the four
// epilogue warps owns query i0 + r and sees the scores of all G heads of
// that query in its own TMEM lane: the scoring queries of the G heads sit in
// TMEM as the A operand (one 128 x d block per head) and every landmark-key
// tile of 32 chunks is multiplied once per head,
//   S_h = Q^_h K'^T    tcgen05.mma, A from TMEM, 128 x 32, f32 in TMEM,
// so no value ever crosses lanes. Every tile is computed twice:
//   pass 1  x_hc = S_hc/sqrt(d) + b'_c (log2 units), masked to C_i; online
//           log-sum-exp per head -> L_h; and, for y_c = max_h x_hc, the two
//           largest y of each of NB chunk classes (c mod NB).
//   After pass 1 the NB-th largest of those 2 NB values, t, belongs to NB
//   distinct chunks, each with group score a_c = max_h (x_hc - L_h) >=
//   y_c - max_h L_h; so tau = t - max_h L_h is a lower bound on the K-th
//   best group score (K <= NB). Rounding keeps the bound: pass 2 forms
//   x_hc with the same instructions, and fl(x - L_h) >= fl(x - max L) for
//   the head that attains y_c.
//   pass 2  a_c = max_h (x_hc - L_h); only chunks with a_c >= tau are
//           appended (score, chunk, x of every head) to the query's
//           candidate list in shared memory, which therefore stays in
//           ascending chunk order. Should it fill, it is cut to its K best
//           and tau rises to just above the K-th of them.
// The exact top-K (ties: lower chunk ranks higher) is then taken from the
// list by dropping its lowest entries; the survivors are already in
// ascending chunk order. Output: idx [B,Hkv,N,K] (-1 padded) and s^ of the
// selected chunks [B,Hq,N,K] (NaN on padding), written through shared
// memory by coalesced stores.
#include <math.h>

#include "hils_fast.cuh"
#include "sm100.cuh"
#include "tc_kernels.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kQ = 128;                // queries per CTA = TMEM lanes
constexpr int kTc = 32;                // chunks per tile
constexpr int kLd = kQ + 1;            // padded row of the candidate arrays
constexpr int kMaxStages = 4;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr uint32_t align1k(uint32_t x) { return (x + 1023u) & ~1023u; }
constexpr uint32_t pow2ceil(uint32_t x) {
    uint32_t p = 32;
    while (p < x) p <<= 1;
    return p;
}

template <int D, int G, int NB>
struct SelLayout {
    // list capacity: after a cut to K <= NB entries there is room for the
    // 16 appends of a half tile plus 16 more, so cuts stay rare
    static constexpr int CAP = NB + 32;
    static_assert(CAP <= 64, "list cuts track at most 64 entries");
    static constexpr uint32_t KT_BYTES = kTc * D * 2;          // one k' tile
    static constexpr uint32_t QST_BYTES = G * kQ * D * 2;      // Q^ staging
    static constexpr uint32_t LIST_BYTES = CAP * kLd * 4 * (2 + G);
    static constexpr uint32_t REGION =
        align1k(QST_BYTES > LIST_BYTES ? QST_BYTES : LIST_BYTES);
    static constexpr uint32_t BIAS_BYTES = 4 * 2 * kTc * 4;    // per warp, 2 tiles
    static constexpr uint32_t STATE_BYTES = 256;
    static constexpr uint32_t TMEM_S = 2 * G * kTc;            // S double buffer
    static constexpr uint32_t TMEM_COLS = pow2ceil(TMEM_S + G * D / 2);
    static size_t smem(int nst) {
        return 1024 + (size_t)nst * KT_BYTES + REGION + BIAS_BYTES + STATE_BYTES;
    }
};

struct SelState {
    uint64_t kv_full[kMaxStages];
    uint64_t kv_empty[kMaxStages];
    uint64_t s_full[2];
    uint64_t s_empty[2];
    uint64_t q_full;
    uint64_t q_ready;
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ void epi_bar() {
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

// Sort N registers into descending order (bitonic network, fully unrolled).
template <int N>
__device__ __forceinline__ void sort_desc(float (&v)[N]) {
#pragma unroll
    for (int k = 2; k <= N; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const float hi = fmaxf(v[i], v[l]), lo = fminf(v[i], v[l]);
                    if ((i & k) == 0) { v[i] = hi; v[l] = lo; }
                    else { v[i] = lo; v[l] = hi; }
                }
            }
        }
    }
}

// Candidate list of query column r: ca[e*kLd + r] group score, cc[..] chunk,
// cx[(h*CAP + e)*kLd + r] x of head h. Drops the lowest-ranked entries
// (lowest score; among equal scores the later, i.e. higher, chunk) until
// `keep` remain, and closes the gaps in order. Returns the smallest score
// kept (NaN scores rank lowest of all).
template <int G, int CAP>
__device__ __noinline__ float list_cut(float *ca, int *cc, float *cx, int r,
                                       int cnt, int keep) {
    uint64_t live = cnt >= 64 ? ~0ull : ((1ull << cnt) - 1ull);
    for (int d = cnt - keep; d > 0; --d) {
        float best = INFINITY;
        int be = 0;
        for (int e = 0; e < cnt; ++e) {
            if (!((live >> e) & 1ull)) continue;
            const float v = ca[e * kLd + r];
            if (!(v > best)) { best = v; be = e; }
        }
        live &= ~(1ull << be);
    }
    int w = 0;
    float mn = INFINITY;
    for (int e = 0; e < cnt; ++e) {
        if (!((live >> e) & 1ull)) continue;
        const float v = ca[e * kLd + r];
        if (w != e) {
            ca[w * kLd + r] = v;
            cc[w * kLd + r] = cc[e * kLd + r];
#pragma unroll
            for (int h = 0; h < G; ++h)
                cx[(h * CAP + w) * kLd + r] = cx[(h * CAP + e) * kLd + r];
        }
        mn = fminf(mn, v);
        ++w;
    }
    return mn;
}

// list_cut for lists of at most RN entries, with the scores held in
// registers: drops the lowest-ranked entries (lowest score, then the later
// chunk) until `keep` remain and closes the gaps in order.
template <int G, int CAP, int RN>
__device__ __forceinline__ void list_cut_regs(float *ca, int *cc, float *cx, int r,
                                              int cnt, int keep) {
    float av[RN];
#pragma unroll
    for (int e = 0; e < RN; ++e) av[e] = e < cnt ? ca[e * kLd + r] : INFINITY;
    uint64_t drop = 0;
    for (int d = cnt - keep; d > 0; --d) {
        float mv[RN / 2];                       // min tree
#pragma unroll
        for (int e = 0; e < RN / 2; ++e) mv[e] = fminf(av[e], av[e + RN / 2]);
#pragma unroll
        for (int w = RN / 4; w >= 1; w >>= 1)
#pragma unroll
            for (int e = 0; e < w; ++e) mv[e] = fminf(mv[e], mv[e + w]);
        int be = -1;
#pragma unroll
        for (int e = 0; e < RN; ++e) be = (e < cnt && av[e] == mv[0]) ? e : be;
        if (be < 0) break;                      // only NaN scores left
#pragma unroll
        for (int e = 0; e < RN; ++e) av[e] = (e == be) ? INFINITY : av[e];
        drop |= 1ull << be;
    }
    int w = 0;
#pragma unroll
    for (int e = 0; e < RN; ++e) {
        if (e < cnt && !((drop >> e) & 1ull)) {
            if (w != e) {
                ca[w * kLd + r] = ca[e * kLd + r];
                cc[w * kLd + r] = cc[e * kLd + r];
#pragma unroll
                for (int h = 0; h < G; ++h)
                    cx[(h * CAP + w) * kLd + r] = cx[(h * CAP + e) * kLd + r];
            }
            ++w;
        }
    }
}

template <int D, int G, int NB>
__global__ void __launch_bounds__(kThreads, 1)
tc_select_kernel(const __grid_constant__ CUtensorMap tmL,
                 const __grid_constant__ CUtensorMap tmQ, const TcParams p,
                 const int nst) {
    using L = SelLayout<D, G, NB>;
    constexpr int CAP = L::CAP;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *region = smem + nst * L::KT_BYTES;
    float *bias_s = reinterpret_cast<float *>(region + L::REGION);
    SelState &st = *reinterpret_cast<SelState *>(region + L::REGION + L::BIAS_BYTES);
    float *ca = reinterpret_cast<float *>(region);       // [CAP][kLd]
    int *cc = reinterpret_cast<int *>(ca + CAP * kLd);   // [CAP][kLd]
    float *cx = reinterpret_cast<float *>(cc + CAP * kLd);  // [G][CAP][kLd]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nqb = (p.N + kQ - 1) / kQ;
    const int qb = blockIdx.x % nqb;
    const int g = (blockIdx.x / nqb) % p.Hkv;
    const int b = blockIdx.x / (nqb * p.Hkv);
    const int i0 = qb * kQ;
    const int nq = min(kQ, p.N - i0);
    int64_t w0x, nc_max;
    window_bounds(i0 + nq - 1, p.S, p.W, &w0x, &nc_max);
    const int nT = (int)((nc_max + kTc - 1) / kTc);
    volatile int *abort = &st.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(&st.kv_full[s], 1);
            mbar_init(&st.kv_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&st.s_full[s], 1);
            mbar_init(&st.s_empty[s], kQ);
        }
        mbar_init(&st.q_full, 1);
        mbar_init(&st.q_ready, kQ);
        mbar_init(&st.mma_done, 1);
        st.abort = (p.status && *(volatile int32_t *)p.status ==
                                    HILS_ERR_DEVICE_TIMEOUT) ? 1 : 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(&st.tmem_base, L::TMEM_COLS);
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmL);
        prefetch_tmap(&tmQ);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = st.tmem_base;
    const int T = st.abort ? 0 : 2 * nT;       // two passes over the tiles

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0 && T > 0) {
            mbar_expect_tx(&st.q_full, L::QST_BYTES);
            for (int hh = 0; hh < G; ++hh) {
                const int h = p.group_heads[g * G + hh];
                for (int dh = 0; dh < D / 64; ++dh)
                    tma_load_4d(region + (hh * (D / 64) + dh) * (kQ * 128), &tmQ,
                                &st.q_full, dh * 64, i0, h, b);
            }
            int issued = 0;
            for (int t = 0; t < T; ++t) {
                const int s = t % nst;
                if (t >= nst &&
                    !mbar_wait(&st.kv_empty[s], ((t / nst) - 1) & 1, abort))
                    break;
                const int c0 = (t % nT) * kTc;
                mbar_expect_tx(&st.kv_full[s], L::KT_BYTES);
                for (int dh = 0; dh < D / 64; ++dh)
                    tma_load_4d(smem + s * L::KT_BYTES + dh * (kTc * 128), &tmL,
                                &st.kv_full[s], dh * 64, c0, g, b);
                issued = t + 1;
            }
            if (*abort) {
                mbar_drain(&st.q_full, 0);
                for (int t = (issued > nst ? issued - nst : 0); t < issued; ++t)
                    mbar_drain(&st.kv_full[t % nst], (t / nst) & 1);
            }
        }
    } else if (warp == 1) {
        // ----------------------------------------------------- MMA issuer
        if (lane == 0 && T > 0) {
            constexpr uint32_t id = idesc_bf16(kQ, kTc, false);
            const uint32_t sK = smem_u32(smem);
            if (mbar_wait(&st.q_ready, 0, abort)) {
                tc_fence_after();
                for (int t = 0; t < T; ++t) {
                    const int s = t % nst, sb = t & 1;
                    if (!mbar_wait(&st.kv_full[s], (t / nst) & 1, abort)) break;
                    if (t >= 2 && !mbar_wait(&st.s_empty[sb], ((t >> 1) - 1) & 1, abort))
                        break;
                    tc_fence_after();
                    // k-steps outer, heads inner: consecutive MMAs write
                    // different accumulators, so none waits on the previous
                    const uint64_t bd0 = desc_sw128(sK + s * L::KT_BYTES, 16, 1024);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        // descriptor start address is in 16-byte units
                        const uint64_t bd = bd0 + (uint64_t)(((k / 4) * (kTc * 128) + (k % 4) * 32) >> 4);
#pragma unroll
                        for (int hh = 0; hh < G; ++hh)
                            mma_ts(tmem + sb * (G * kTc) + hh * kTc,
                                   tmem + L::TMEM_S + hh * (D / 2) + k * 8, bd, id,
                                   k > 0 ? 1u : 0u);
                    }
                    mma_commit(&st.s_full[sb]);
                    mma_commit(&st.kv_empty[s]);
                }
            }
            mma_commit(&st.mma_done);
            mbar_drain(&st.mma_done, 0);
        }
    } else {
        // ------------------------------------------------ epilogue warps
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int i = i0 + r;
        int64_t w0, nc64 = 0;
        if (r < nq) window_bounds(i, p.S, p.W, &w0, &nc64);
        const int nc = (int)nc64;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        const int K = p.K;

        // scoring queries: staging (TMA, 128B-swizzled rows) -> own TMEM lane
        if (T > 0) {
            if (__all_sync(0xffffffffu, mbar_wait(&st.q_full, 0, abort))) {
#pragma unroll
                for (int hh = 0; hh < G; ++hh) {
#pragma unroll
                    for (int dh = 0; dh < D / 64; ++dh) {
                        const uint8_t *row = region + (hh * (D / 64) + dh) * (kQ * 128) + r * 128;
                        uint32_t w[32];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(
                                row + ((u ^ (r & 7)) << 4));
                            w[4 * u + 0] = v.x; w[4 * u + 1] = v.y;
                            w[4 * u + 2] = v.z; w[4 * u + 3] = v.w;
                        }
                        tmem_st32(trow + L::TMEM_S + hh * (D / 2) + dh * 32, w);
                    }
                }
                tmem_wait_st();
            }
        }
        tc_fence_before();
        mbar_arrive(&st.q_ready);
        epi_bar();                  // staging is read before the lists overwrite it

        const float sl2 = p.inv_sqrt_d * kLog2e;
        const float2 sl2v = make_float2(sl2, sl2);
        float *bias_w = bias_s + quad * (2 * kTc);
        const float *bias_g = p.bias + ((int64_t)b * p.Hkv + g) * p.nC;
        float bnext = 0.f;
        if (T > 0 && lane < p.nC) bnext = bias_g[lane];
        // b' of tile t's 32 chunks (log2 units) into this warp's slot t & 1,
        // the next tile's loaded ahead
        auto stage_bias = [&](int t) -> const float * {
            float *bw = bias_w + (t & 1) * kTc;
            bw[lane] = bnext * kLog2e;
            __syncwarp();
            if (t + 1 < T) {
                const int cn = ((t + 1) % nT) * kTc + lane;
                bnext = cn < p.nC ? bias_g[cn] : 0.f;
            }
            return bw;
        };
        bool ok = true;

        // ---------------------------------------------------------- pass 1
        float mrun[G], srun[G], lse2[G];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
            mrun[hh] = -1e30f;          // finite: the rescale needs no branch
            srun[hh] = 0.f;
            lse2[hh] = 0.f;
        }
        float m1[NB], m2[NB];
#pragma unroll
        for (int k = 0; k < NB; ++k) { m1[k] = -INFINITY; m2[k] = -INFINITY; }
        for (int t = 0; t < nT; ++t) {
            const float *bw = stage_bias(t);
            if (!__all_sync(0xffffffffu, mbar_wait(&st.s_full[t & 1], (t >> 1) & 1, abort))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int lim = nc - t * kTc;              // valid columns of this row
            const bool edge = __any_sync(0xffffffffu, lim < kTc);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int j0 = half * 16;
                uint32_t raw[G][16];
#pragma unroll
                for (int hh = 0; hh < G; ++hh)
                    tmem_ld16(trow + (t & 1) * (G * kTc) + hh * kTc + j0, raw[hh]);
                tmem_wait_ld();
                if (half == 1) {
                    tc_fence_before();
                    mbar_arrive(&st.s_empty[t & 1]);
                }
                // x = S/sqrt(d) + b' for column pairs (f32x2: each element
                // rounded as the scalar fma, so pass 2 forms the same x)
                float x[G][16];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float2 b2 = *reinterpret_cast<const float2 *>(bw + j0 + 2 * k);
#pragma unroll
                    for (int hh = 0; hh < G; ++hh) {
                        const float2 v = f2_fma(make_float2(__uint_as_float(raw[hh][2 * k]),
                                                            __uint_as_float(raw[hh][2 * k + 1])),
                                                sl2v, b2);
                        x[hh][2 * k] = v.x;
                        x[hh][2 * k + 1] = v.y;
                    }
                }
                if (edge) {
#pragma unroll
                    for (int hh = 0; hh < G; ++hh)
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            x[hh][j] = (j0 + j < lim) ? x[hh][j] : -INFINITY;
                }
#pragma unroll
                for (int hh = 0; hh < G; ++hh) {
                    // short dependency chains: a max tree, four partial sums
                    float t8[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) t8[j] = fmaxf(x[hh][j], x[hh][j + 8]);
#pragma unroll
                    for (int j = 0; j < 4; ++j) t8[j] = fmaxf(t8[j], t8[j + 4]);
                    const float mt = fmaxf(fmaxf(t8[0], t8[2]), fmaxf(t8[1], t8[3]));
                    const float mn = fmaxf(mrun[hh], mt);
                    const float2 nm2 = make_float2(-mn, -mn);
                    float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        float2 e = f2_add(make_float2(x[hh][2 * k], x[hh][2 * k + 1]), nm2);
                        e.x = fast_exp2(e.x);
                        e.y = fast_exp2(e.y);
                        acc[k & 1] = f2_add(acc[k & 1], e);
                    }
                    srun[hh] = fmaf(srun[hh], fast_exp2(mrun[hh] - mn),
                                    (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y));
                    mrun[hh] = mn;
                }
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    float y = x[0][j];
#pragma unroll
                    for (int hh = 1; hh < G; ++hh) y = fmaxf(y, x[hh][j]);
                    const int k = (j0 + j) % NB;
                    m2[k] = fmaxf(m2[k], fminf(m1[k], y));
                    m1[k] = fmaxf(m1[k], y);
                }
            }
        }

        // per-head normalisers; lower bound tau on the K-th best group score
        float tau = -INFINITY;
        if (ok && nc > 0) {
            float lmax = -INFINITY;
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
                lse2[hh] = mrun[hh] + log2f(srun[hh]);
                lmax = fmaxf(lmax, lse2[hh]);
            }
            sort_desc<NB>(m1);
            sort_desc<NB>(m2);
            float tk = INFINITY;
#pragma unroll
            for (int k = 0; k < NB; ++k) tk = fminf(tk, fmaxf(m1[k], m2[NB - 1 - k]));
            tau = tk - lmax;
        }

        // ---------------------------------------------------------- pass 2
        float2 nl2[G];                          // -L_h, twice
#pragma unroll
        for (int hh = 0; hh < G; ++hh) nl2[hh] = make_float2(-lse2[hh], -lse2[hh]);
        int cnt = 0;
        for (int t = nT; ok && t < T; ++t) {
            const float *bw = stage_bias(t);
            if (!__all_sync(0xffffffffu, mbar_wait(&st.s_full[t & 1], (t >> 1) & 1, abort))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int c0 = (t - nT) * kTc;
            const int lim = nc - c0;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int j0 = half * 16;
                uint32_t raw[G][16];
#pragma unroll
                for (int hh = 0; hh < G; ++hh)
                    tmem_ld16(trow + (t & 1) * (G * kTc) + hh * kTc + j0, raw[hh]);
                tmem_wait_ld();
                if (half == 1) {
                    tc_fence_before();
                    mbar_arrive(&st.s_empty[t & 1]);
                }
                if (cnt > CAP - 16) {                  // room for 16 more, rarely needed
                    const float mn = list_cut<G, CAP>(ca, cc, cx, r, cnt, K);
                    cnt = K;
                    tau = nextafterf(mn, INFINITY);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    // x and a = max_h (x_h - L_h) for the column pair 2k, 2k+1
                    const float2 b2 = *reinterpret_cast<const float2 *>(bw + j0 + 2 * k);
                    float2 x2[G];
#pragma unroll
                    for (int hh = 0; hh < G; ++hh)
                        x2[hh] = f2_fma(make_float2(__uint_as_float(raw[hh][2 * k]),
                                                    __uint_as_float(raw[hh][2 * k + 1])),
                                        sl2v, b2);
                    float2 a2 = f2_add(x2[0], nl2[0]);
#pragma unroll
                    for (int hh = 1; hh < G; ++hh) {
                        const float2 v = f2_add(x2[hh], nl2[hh]);
                        a2.x = fmaxf(a2.x, v.x);
                        a2.y = fmaxf(a2.y, v.y);
                    }
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int j = 2 * k + e;
                        const float a = e ? a2.y : a2.x;
                        const bool take = (j0 + j < lim) && (a >= tau);
                        if (take) {
                            ca[cnt * kLd + r] = a;
                            cc[cnt * kLd + r] = c0 + j0 + j;
#pragma unroll
                            for (int hh = 0; hh < G; ++hh)
                                cx[(hh * CAP + cnt) * kLd + r] = e ? x2[hh].y : x2[hh].x;
                        }
                        cnt += take ? 1 : 0;
                    }
                }
            }
        }

        // exact top-K of the list, kept in ascending chunk order; padding
        if (ok && r < nq) {
            if (cnt > K) {
                if (cnt <= 32) list_cut_regs<G, CAP, 32>(ca, cc, cx, r, cnt, K);
                else list_cut_regs<G, CAP, 64>(ca, cc, cx, r, cnt, K);
                cnt = K;
            }
            for (int k = cnt; k < K; ++k) {
                cc[k * kLd + r] = -1;
#pragma unroll
                for (int hh = 0; hh < G; ++hh)
                    cx[(hh * CAP + k) * kLd + r] = __int_as_float(0x7fc00000);
            }
        }
        epi_bar();
        if (!*abort) {
            // coalesced copy-out of the CTA's nq x K block of every output
            const int tid = threadIdx.x - 64;
            if ((K & 3) == 0) {
                const int K4 = K >> 2, tot = nq * K4, dq = kQ / K4, dk = kQ % K4;
                {
                    int4 *io = reinterpret_cast<int4 *>(
                        p.idx + (((int64_t)b * p.Hkv + g) * p.N + i0) * K);
                    int q = tid / K4, k = tid % K4;
                    for (int u = tid; u < tot; u += kQ) {
                        const int *src = cc + 4 * k * kLd + q;
                        io[u] = make_int4(src[0], src[kLd], src[2 * kLd], src[3 * kLd]);
                        q += dq; k += dk;
                        if (k >= K4) { k -= K4; ++q; }
                    }
                }
#pragma unroll
                for (int hh = 0; hh < G; ++hh) {
                    const int h = p.group_heads[g * G + hh];
                    float4 *so = reinterpret_cast<float4 *>(
                        p.sel + (((int64_t)b * p.Hq + h) * p.N + i0) * K);
                    int q = tid / K4, k = tid % K4;
                    for (int u = tid; u < tot; u += kQ) {
                        const float *src = cx + (hh * CAP + 4 * k) * kLd + q;
                        so[u] = make_float4(src[0] * kLn2, src[kLd] * kLn2,
                                            src[2 * kLd] * kLn2, src[3 * kLd] * kLn2);
                        q += dq; k += dk;
                        if (k >= K4) { k -= K4; ++q; }
                    }
                }
            } else {
                const int tot = nq * K, dq = kQ / K, dk = kQ % K;
                {
                    int32_t *io = p.idx + (((int64_t)b * p.Hkv + g) * p.N + i0) * K;
                    int q = tid / K, k = tid % K;
                    for (int e = tid; e < tot; e += kQ) {
                        io[e] = cc[k * kLd + q];
                        q += dq; k += dk;
                        if (k >= K) { k -= K; ++q; }
                    }
                }
#pragma unroll
                for (int hh = 0; hh < G; ++hh) {
                    const int h = p.group_heads[g * G + hh];
                    float *so = p.sel + (((int64_t)b * p.Hq + h) * p.N + i0) * K;
                    const float *src = cx + hh * CAP * kLd;
                    int q = tid / K, k = tid % K;
                    for (int e = tid; e < tot; e += kQ) {
                        so[e] = src[k * kLd + q] * kLn2;
                        q += dq; k += dk;
                        if (k >= K) { k -= K; ++q; }
                    }
                }
            }
        }
    }

    if (*abort && (threadIdx.x & 31) == 0) report(p.status, HILS_ERR_DEVICE_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

template <int D, int G, int NB>
int stages_for() {
    for (int n = kMaxStages; n >= 2; --n)
        if (SelLayout<D, G, NB>::smem(n) <= 227 * 1024) return n;
    return 0;
}

template <int D, int G>
int stages_for_k(int K) {
    return K <= 16 ? stages_for<D, G, 16>() : stages_for<D, G, 32>();
}

int select_stages(const TcParams &tp) {
    if (tp.K < 1 || tp.K > 32) return 0;
    if (tp.d == 128) {
        if (tp.G == 1) return stages_for_k<128, 1>(tp.K);
        if (tp.G == 2) return stages_for_k<128, 2>(tp.K);
        if (tp.G == 4) return stages_for_k<128, 4>(tp.K);
    } else if (tp.d == 64) {
        if (tp.G == 1) return stages_for_k<64, 1>(tp.K);
        if (tp.G == 2) return stages_for_k<64, 2>(tp.K);
        if (tp.G == 4) return stages_for_k<64, 4>(tp.K);
    }
    return 0;
}

template <int D, int G, int NB>
cudaError_t launch_sel_t(const TcParams &tp, const CUtensorMap &lm32,
                         const CUtensorMap &q128, unsigned grid, cudaStream_t st) {
    const int nst = stages_for<D, G, NB>();
    const size_t smem = SelLayout<D, G, NB>::smem(nst);
    cudaError_t e = cudaFuncSetAttribute(tc_select_kernel<D, G, NB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    tc_select_kernel<D, G, NB><<<grid, kThreads, smem, st>>>(lm32, q128, tp, nst);
    return cudaGetLastError();
}

template <int D, int G>
cudaError_t launch_sel_k(const TcParams &tp, const CUtensorMap &lm32,
                         const CUtensorMap &q128, unsigned grid, cudaStream_t st) {
    return tp.K <= 16 ? launch_sel_t<D, G, 16>(tp, lm32, q128, grid, st)
                      : launch_sel_t<D, G, 32>(tp, lm32, q128, grid, st);
}

}  // namespace

bool tc_select_supported(const TcParams &tp) { return select_stages(tp) > 0; }

cudaError_t launch_tc_select(const TcParams &tp, const CUtensorMap &lm32,
                             const CUtensorMap &q128, cudaStream_t st) {
    if (!tc_select_supported(tp)) return cudaErrorNotSupported;
    const int64_t grid = (int64_t)tp.B * tp.Hkv * ((tp.N + kQ - 1) / kQ);
    if (grid <= 0) return cudaSuccess;
    const unsigned gr = (unsigned)grid;
    if (tp.d == 128) {
        if (tp.G == 1) return launch_sel_k<128, 1>(tp, lm32, q128, gr, st);
        if (tp.G == 2) return launch_sel_k<128, 2>(tp, lm32, q128, gr, st);
        return launch_sel_k<128, 4>(tp, lm32, q128, gr, st);
    }
    if (tp.G == 1) return launch_sel_k<64, 1>(tp, lm32, q128, gr, st);
    if (tp.G == 2) return launch_sel_k<64, 2>(tp, lm32, q128, gr, st);
    return launch_sel_k<64, 4>(tp, lm32, q128, gr, st);
}

}  // namespace hils
