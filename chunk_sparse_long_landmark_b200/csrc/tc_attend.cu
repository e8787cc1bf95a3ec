// tc_attend.cu -- HiLS prefill gather-attention on the sm_100a tensor cores.
//
// "Hierarchical Sparse Attention Done Right", Sec. 3 (hierarchical softmax,
// RQ2 display) and Sec. 4.2 (M adjacent queries x G heads share one tile).
//
// One CTA owns 128 rows = the G query heads of one kv group x M = 128/G
// adjacent queries (row r = query_slot * G + head_slot). It loads the union
// of the M queries' selected chunks once and then every tile of the aligned
// window the block touches, each tile S tokens of K and V brought in by TMA:
//   S   = Q K^T      tcgen05.mma, 128 x S_TOK, f32 accumulator in TMEM
//   P   = softmax    per row, in registers (chunk tiles: intra-chunk softmax
//                    scaled by exp(s^_c - M0)/z_c, zero for rows that did not
//                    select the chunk -- a warp whose queries all skipped it
//                    stores zeros without reading S; window tiles: causal +
//                    window mask, running reference max), stored as bf16 over
//                    the S columns
//   O  += P V        tcgen05.mma, 128 x d, A = P from TMEM, f32 in TMEM
// Shared memory holds only Q and a K/V ring (two stages at S = 64, one at
// S = 128; at most ~105 KB) and TMEM 256 columns, so two CTAs share an SM
// and hide each other's latencies. A K stage is handed back when its QK
// product completes and a V stage when its PV product does, so the copy of
// K runs ahead of the PV chain.
// Warp roles: warp 0 TMA producer (K, V), warp 1 MMA issuer (and TMEM
// owner), warps 2-5 Q loader, softmax and epilogue (warp w reads TMEM lanes
// 32*(w%4)..+31). Elementwise softmax arithmetic uses packed f32x2 ops.
// All waits are bounded (sm100::mbar_wait): a lost arrival ends the kernel
// with HILS_ERR_DEVICE_TIMEOUT in the status word.
#include <math.h>

#include "hils_fast.cuh"
#include "sm100.cuh"
#include "tc_kernels.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kRows = 128;
constexpr int kMaxStages = 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;      // lazy O rescale threshold (log2)

// max over n >= 8 scores (n a multiple of 4), four independent chains
__device__ __forceinline__ float row_max(const uint32_t *rr, int n) {
    float m[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) m[k] = __uint_as_float(rr[k]);
#pragma unroll
    for (int j = 4; j < n; j += 4)
#pragma unroll
        for (int k = 0; k < 4; ++k) m[k] = fmaxf(m[k], __uint_as_float(rr[j + k]));
    return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// a += the two bf16 halves of a packed pair (mixed-precision adds: no
// unpacking instructions; each sum rounds as the f32 add of the widened value)
__device__ __forceinline__ void acc_bf16x2(float2 &a, uint32_t v) {
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
        : "+f"(a.x), "+f"(a.y) : "r"(v));
}

// Two CTAs share an SM in every configuration: TMEM holds O (D columns) and
// NSB buffers of S / P (S_TOK columns each) within 256 columns, shared
// memory Q and NST stages each of K and V. With S_TOK = 64 both are double
// buffered; with S_TOK = 128 one S buffer and one K / V stage fit, and the
// other CTA on the SM covers the latencies the single buffers expose.
template <int S_TOK, int D>
struct AttnLayout {
    static constexpr int NSB = (D + 2 * S_TOK) <= 256 ? 2 : 1;   // S buffers
    static constexpr int NST = NSB;                              // K/V stages
    static constexpr uint32_t Q_BYTES = kRows * D * 2;
    static constexpr uint32_t KV_BYTES = S_TOK * D * 2;        // one of K or V
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + NST * KV_BYTES;
    static constexpr uint32_t OFF_SMALL = OFF_V + NST * KV_BYTES;
    static constexpr int TMEM_O = 0;                 // columns [0, D)
    static constexpr int TMEM_S = D;                 // NSB buffers of S_TOK (S, then P)
    static constexpr uint32_t TMEM_COLS = 256u;
    static constexpr int MIN_BLOCKS = 2;
    static_assert(D + NSB * S_TOK <= 256, "TMEM budget of two CTAs per SM");
};

struct SmallState {
    uint64_t q_full;
    uint64_t k_full[kMaxStages];
    uint64_t v_full[kMaxStages];
    uint64_t k_empty[kMaxStages];                    // QK of that stage done
    uint64_t v_empty[kMaxStages];                    // PV of that stage done
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t p_empty[2];                             // PV of that buffer done
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort;
    int n_union;
    int n_win_tiles;
    int win_start;
};

template <int S_TOK, int D>
__global__ void __launch_bounds__(kThreads, AttnLayout<S_TOK, D>::MIN_BLOCKS)
tc_attend_kernel(const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV,
                 const TcParams p) {
    using L = AttnLayout<S_TOK, D>;
    constexpr int NSB = L::NSB, NST = L::NST;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    SmallState &st = *reinterpret_cast<SmallState *>(smem + L::OFF_SMALL);
    // selected chunks of the block's queries, [K][M]; the chunk union; its bitmap
    int *s_idx = reinterpret_cast<int *>(smem + L::OFF_SMALL + sizeof(SmallState));
    int *s_union = s_idx + p.M * p.K;
    uint32_t *s_bits = reinterpret_cast<uint32_t *>(s_union + p.ucap);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nqb = (p.N + p.M - 1) / p.M;
    const int qb = blockIdx.x % nqb;
    const int g = (blockIdx.x / nqb) % p.Hkv;
    const int b = blockIdx.x / (nqb * p.Hkv);
    const int i0 = qb * p.M;
    const int i_last = min(i0 + p.M, p.N) - 1;
    volatile int *abort = &st.abort;

    // ---------------------------------------------------------- prologue
    if (threadIdx.x == 0) {
        mbar_init(&st.q_full, 128);             // the softmax threads load Q
        for (int s = 0; s < NST; ++s) {
            mbar_init(&st.k_full[s], 1);
            mbar_init(&st.v_full[s], 1);
            mbar_init(&st.k_empty[s], 1);
            mbar_init(&st.v_empty[s], 1);
        }
        for (int s = 0; s < NSB; ++s) {
            mbar_init(&st.s_full[s], 1);
            mbar_init(&st.p_full[s], 128);
            mbar_init(&st.p_empty[s], 1);
        }
        mbar_init(&st.mma_done, 1);
        // a CTA that timed out already: the rest of the grid skips its work
        st.abort = (p.status && *(volatile int32_t *)p.status ==
                                    HILS_ERR_DEVICE_TIMEOUT) ? 1 : 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(&st.tmem_base, L::TMEM_COLS);
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    // selected chunks of the block's queries -> smem; union bitmap
    const int nwords = (p.nC + 31) >> 5;
    for (int w = threadIdx.x; w < nwords; w += kThreads) s_bits[w] = 0u;
    __syncthreads();
    // The block's idx rows are one contiguous [M][K] range, its scores G
    // contiguous [M][K] ranges: loads are issued in batches of 8 per thread
    // before their stores so their latencies overlap.
    {
        const int nidx = p.M * p.K;
        const int32_t *gidx = p.idx + (((int64_t)b * p.Hkv + g) * p.N + i0) * p.K;
        const int nvalid = (min(i0 + p.M, p.N) - i0) * p.K;
        for (int e0 = 0; e0 < nidx; e0 += 8 * kThreads) {
            int c8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int e = e0 + q * kThreads + threadIdx.x;
                c8[q] = (e < nvalid) ? __ldg(gidx + e) : -1;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int e = e0 + q * kThreads + threadIdx.x;
                if (e < nidx) {
                    const int m = e / p.K, k = e % p.K;
                    int c = c8[q];
                    if (c >= 0) {
                        int64_t w0, nc;
                        window_bounds(i0 + m, p.S, p.W, &w0, &nc);
                        if (c >= nc) c = -1;
                    }
                    s_idx[k * p.M + m] = c;
                    if (c >= 0) atomicOr(&s_bits[c >> 5], 1u << (c & 31));
                }
            }
        }
    }
    __syncthreads();
    if (warp == 0) {                       // ascending compaction of the union
        int base = 0;
        for (int w0i = 0; w0i < nwords; w0i += 32) {
            const int w = w0i + lane;
            uint32_t bits = w < nwords ? s_bits[w] : 0u;
            const int cnt = __popc(bits);
            int incl = cnt;
            for (int o = 1; o < 32; o <<= 1) {
                int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            int pos = base + incl - cnt;
            while (bits) {
                const int bit = __ffs(bits) - 1;
                bits &= bits - 1;
                if (pos < p.ucap) s_union[pos] = w * 32 + bit;
                ++pos;
            }
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            st.n_union = min(base, p.ucap);
            int64_t w0, nc;
            window_bounds(i0, p.S, p.W, &w0, &nc);
            st.win_start = (int)w0;
            st.n_win_tiles = (i_last - (int)w0) / S_TOK + 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = st.tmem_base;
    const int U = st.n_union;
    const int T = st.abort ? 0 : U + st.n_win_tiles;
    const int wstart = st.win_start;

    if (T == 0) {
        // skipped (see above): straight to teardown
    } else if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            // K of a stage is free once the QK product of its tile is done,
            // V once the PV product is: K copies run ahead of V copies, and
            // two V copies stay in flight behind the PV chain.
            auto load = [&](int t, bool is_v) {
                const int s = t % NST;
                const int row = (t < U) ? s_union[t] * p.S
                                        : wstart + (t - U) * S_TOK;
                uint64_t *bar = is_v ? &st.v_full[s] : &st.k_full[s];
                mbar_expect_tx(bar, L::KV_BYTES);
                for (int dh = 0; dh < D / 64; ++dh)
                    tma_load_4d(smem + (is_v ? L::OFF_V : L::OFF_K) + s * L::KV_BYTES +
                                    dh * (S_TOK * 128),
                                is_v ? &tmV : &tmK, bar, dh * 64, row, g, b);
            };
            int nk = 0, nv = 0;                          // copies issued
            while (nv < T) {
                // next K copy whose stage is already free, else the next V copy
                if (nk < T && nk < nv + NST &&
                    (nk < NST ||
                     mbar_test(smem_u32(&st.k_empty[nk % NST]), ((nk / NST) - 1) & 1))) {
                    load(nk++, false);
                    continue;
                }
                if (nv < nk) {
                    if (nv >= NST &&
                        !mbar_wait(&st.v_empty[nv % NST], ((nv / NST) - 1) & 1, abort))
                        break;
                    load(nv++, true);
                    continue;
                }
                // nv == nk: the K copy must go first
                if (!mbar_wait(&st.k_empty[nk % NST], ((nk / NST) - 1) & 1, abort))
                    break;
                load(nk++, false);
            }
            // on abort: let the copies already issued land before exiting
            if (*abort) {
                for (int t = (nk > NST ? nk - NST : 0); t < nk; ++t)
                    mbar_drain(&st.k_full[t % NST], (t / NST) & 1);
                for (int t = (nv > NST ? nv - NST : 0); t < nv; ++t)
                    mbar_drain(&st.v_full[t % NST], (t / NST) & 1);
            }
        }
    } else if (warp == 1) {
        // ----------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(kRows, S_TOK, false);
            constexpr uint32_t id_o = idesc_bf16(kRows, D, true);
            const uint32_t sQ = smem_u32(smem + L::OFF_Q);
            const uint32_t sK = smem_u32(smem + L::OFF_K);
            const uint32_t sV = smem_u32(smem + L::OFF_V);
            bool ok = mbar_wait(&st.q_full, 0, abort);
            tc_fence_after();
            auto do_pv = [&](int u) -> bool {
                const int pb = u % NSB;
                if (!mbar_wait(&st.p_full[pb], (u / NSB) & 1, abort)) return false;
                const int s = u % NST;
                if (!mbar_wait(&st.v_full[s], (u / NST) & 1, abort)) return false;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < S_TOK / 16; ++k) {
                    // A = P of this tile, bf16 in the S buffer: 8 columns per 16 tokens
                    const uint32_t at = tmem + L::TMEM_S + pb * S_TOK + k * 8;
                    const uint64_t bd = desc_sw128(
                        sV + s * L::KV_BYTES + k * 16 * 128, S_TOK * 128, 1024);
                    mma_ts(tmem + L::TMEM_O, at, bd, id_o, (u > 0 || k > 0) ? 1u : 0u);
                }
                mma_commit(&st.v_empty[s]);
                mma_commit(&st.p_empty[pb]);
                return true;
            };
            for (int t = 0; ok && t < T; ++t) {
                const int s = t % NST;
                const int sb = t % NSB;
                // one S buffer: PV(t-1) reads its P, so it goes first
                if (NSB == 1 && t >= 1 && !do_pv(t - 1)) { ok = false; break; }
                if (!mbar_wait(&st.k_full[s], (t / NST) & 1, abort)) { ok = false; break; }
                // S buffer sb is free once PV(t-NSB), which read its P, is done
                if (t >= NSB && !mbar_wait(&st.p_empty[sb], ((t / NSB) - 1) & 1, abort)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint64_t ad = desc_sw128(
                        sQ + (k / 4) * (kRows * 128) + (k % 4) * 32, 16, 1024);
                    const uint64_t bd = desc_sw128(
                        sK + s * L::KV_BYTES + (k / 4) * (S_TOK * 128) + (k % 4) * 32,
                        16, 1024);
                    mma_ss(tmem + L::TMEM_S + sb * S_TOK, ad, bd, id_s, k > 0 ? 1u : 0u);
                }
                mma_commit(&st.s_full[sb]);
                mma_commit(&st.k_empty[s]);
                if (NSB > 1 && t >= 1 && !do_pv(t - 1)) { ok = false; break; }
            }
            if (ok && T > 0) do_pv(T - 1);
            // every MMA of this CTA has completed before TMEM is released
            mma_commit(&st.mma_done);
            mbar_drain(&st.mma_done, 0);
        }
    } else {
        // -------------------------------------------- softmax / epilogue
        // Query-major rows: row r = query_slot * G + head_slot, so a warp
        // holds 32 / G whole queries and can skip, as a unit, every union
        // chunk none of them selected.
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int m = r / p.G, hh = r % p.G;
        const int i = i0 + m;
        const bool valid = i < p.N;
        const int h = p.group_heads[g * p.G + hh];
        int64_t w0 = 0, nc = 0;
        if (valid) window_bounds(i, p.S, p.W, &w0, &nc);

        // the block's Q rows -> shared memory (A operand: K-major, 128-byte
        // swizzle), 16-byte units, all loads issued before the stores
        {
            constexpr int UPR = D / 8;
            constexpr int NU = kRows * UPR / 128 / 2;     // two batches
            const int tid = threadIdx.x - 64;
#pragma unroll 1
            for (int bt = 0; bt < 2; ++bt) {
            uint4 v[NU];
#pragma unroll
            for (int q = 0; q < NU; ++q) {
                const int e = tid + (bt * NU + q) * 128;
                const int rr = e / UPR, u = e % UPR;
                const int mi = i0 + rr / p.G;
                v[q] = make_uint4(0u, 0u, 0u, 0u);
                if (mi < p.N) {
                    const int hq = p.group_heads[g * p.G + rr % p.G];
                    v[q] = __ldg(reinterpret_cast<const uint4 *>(
                               reinterpret_cast<const __nv_bfloat16 *>(p.Q) +
                               (((int64_t)b * p.Hq + hq) * p.N + mi) * D) + u);
                }
            }
#pragma unroll
            for (int q = 0; q < NU; ++q) {
                const int e = tid + (bt * NU + q) * 128;
                const int rr = e / UPR, u = e % UPR;
                *reinterpret_cast<uint4 *>(smem + L::OFF_Q + (u >> 3) * (kRows * 128) +
                                           rr * 128 + (((u & 7) ^ (rr & 7)) << 4)) = v[q];
            }
            }
            fence_async_smem();
            mbar_arrive(&st.q_full);
        }

        const int *myidx = s_idx + m;                    // stride M
        const int M_ = p.M;
        const float *mysel = p.sel + (((int64_t)b * p.Hq + h) * p.N + i) * p.K;
        float M0 = -INFINITY;                            // natural-log units
        if (valid)
            for (int k = 0; k < p.K; ++k)
                if (myidx[k * M_] >= 0) M0 = fmaxf(M0, __ldg(mysel + k));
        const float M0l2 = M0 * kLog2e;
        float mref = M0l2;                               // log2 units
        float l = 0.f;
        int kp = 0;
        // s^ of the next selected chunk, loaded ahead of its tile
        float sh_next = (valid && p.K > 0) ? __ldg(mysel) : 0.f;
        const float sl2 = p.inv_sqrt_d * kLog2e;
        const float2 sl2v = make_float2(sl2, sl2);
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        bool ok = true;

        for (int t = 0; t < T; ++t) {
            const int sb = t % NSB;
            const uint32_t tS = trow + L::TMEM_S + sb * S_TOK;
            // every lane takes the same branch around warp-collective
            // tcgen05.ld / st, so wait outcomes are agreed across the warp
            if (!__all_sync(0xffffffffu, mbar_wait(&st.s_full[sb], (t / NSB) & 1, abort))) { ok = false; break; }
            tc_fence_after();
            float2 ps[4];                                // sum of the rounded P
#pragma unroll
            for (int k = 0; k < 4; ++k) ps[k] = make_float2(0.f, 0.f);
            // chunk tiles: does this row's query select the chunk, and s^_c
            bool sel = false;
            float sh = 0.f;
            if (t < U) {
                const int c = s_union[t];
                int ck = kp < p.K ? myidx[kp * M_] : 0x7fffffff;
                while (kp < p.K && ck < c) {
                    ++kp;
                    ck = kp < p.K ? myidx[kp * M_] : 0x7fffffff;
                    sh_next = (valid && kp < p.K) ? __ldg(mysel + kp) : 0.f;
                }
                sel = valid && kp < p.K && ck == c;
                if (sel) {
                    sh = sh_next * kLog2e;
                    ++kp;
                    sh_next = (kp < p.K) ? __ldg(mysel + kp) : 0.f;
                }
            }
            const int j0 = wstart + (t - U) * S_TOK;     // window tiles
            // masks only where a row's window starts or ends in the tile
            const bool edge = t >= U && (!valid || j0 < w0 || j0 + S_TOK - 1 > i);
            const bool any_edge = __any_sync(0xffffffffu, edge);
            // raise the reference max of the rows whose window scores exceed
            // it by more than 2^8 and rescale their O once PV(t-1) is done
            // (warp-wide: the TMEM load / store are collective; other rows
            // use a factor of 1). Returns false if the wait gave up.
            auto window_rescale = [&](float mx) -> bool {
                const bool mine = mx > mref + kRescaleLog2;
                if (__any_sync(0xffffffffu, mine)) {
                    const float fac = !mine ? 1.f
                                    : (mref == -INFINITY) ? 0.f : fast_exp2(mref - mx);
                    if (t >= 1) {
                        const int u = t - 1;
                        if (!__all_sync(0xffffffffu, mbar_wait(&st.p_empty[u % NSB], (u / NSB) & 1, abort)))
                            return false;
                        tc_fence_after();
#pragma unroll
                        for (int c0 = 0; c0 < D; c0 += 16) {
                            uint32_t ro[16];
                            tmem_ld16(trow + L::TMEM_O + c0, ro);
                            tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                ro[j] = __float_as_uint(__uint_as_float(ro[j]) * fac);
                            tmem_st16(trow + L::TMEM_O + c0, ro);
                        }
                        tmem_wait_st();
                    }
                    if (mine) { l *= fac; mref = mx; }
                }
                return true;
            };

            if constexpr (S_TOK <= 64) {
            uint32_t pk[S_TOK / 2];                      // P, bf16 pairs
            if (t < U) {
                if (__any_sync(0xffffffffu, sel)) {
                    uint32_t rr[S_TOK];
#pragma unroll
                    for (int c0 = 0; c0 < S_TOK; c0 += 32) tmem_ld32(tS + c0, rr + c0);
                    tmem_wait_ld();
                    if (sel) {
                        // intra-chunk softmax scaled by exp(s^_c - M0) / z_c
                        const float mx = row_max(rr, S_TOK);
                        const float2 nb = make_float2(-mx * sl2, -mx * sl2);
                        float2 e[S_TOK / 2];
                        float2 z2[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) z2[k] = make_float2(0.f, 0.f);
#pragma unroll
                        for (int j = 0; j < S_TOK / 2; ++j) {
                            e[j] = f2_fma(make_float2(__uint_as_float(rr[2 * j]),
                                                      __uint_as_float(rr[2 * j + 1])), sl2v, nb);
                            e[j].x = fast_exp2(e[j].x);
                            e[j].y = fast_exp2(e[j].y);
                            z2[j & 3] = f2_add(z2[j & 3], e[j]);
                        }
                        const float2 zz = f2_add(f2_add(z2[0], z2[1]), f2_add(z2[2], z2[3]));
                        const float f = __fdividef(fast_exp2(sh - M0l2), zz.x + zz.y);
                        const float2 fv = make_float2(f, f);
#pragma unroll
                        for (int j = 0; j < S_TOK / 2; ++j) {
                            const float2 pv = f2_mul(e[j], fv);
                            pk[j] = pack_bf16(pv.x, pv.y);
                            acc_bf16x2(ps[j & 3], pk[j]);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < S_TOK / 2; ++j) pk[j] = 0u;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < S_TOK / 2; ++j) pk[j] = 0u;
                }
            } else {
                uint32_t rr[S_TOK];
#pragma unroll
                for (int c0 = 0; c0 < S_TOK; c0 += 32) tmem_ld32(tS + c0, rr + c0);
                tmem_wait_ld();
                if (any_edge) {
#pragma unroll
                    for (int j = 0; j < S_TOK; ++j) {
                        const int pos = j0 + j;
                        const bool in = valid && pos >= w0 && pos <= i;
                        rr[j] = in ? rr[j] : __float_as_uint(-INFINITY);
                    }
                }
                if (!window_rescale(row_max(rr, S_TOK) * sl2)) { ok = false; break; }
                // rows with nothing in the window yet keep mref = -inf:
                // their masked scores still give exp2(-inf) = 0
                const float nm = (mref == -INFINITY) ? 0.f : -mref;
                const float2 nmv = make_float2(nm, nm);
#pragma unroll
                for (int j = 0; j < S_TOK / 2; ++j) {
                    float2 e = f2_fma(make_float2(__uint_as_float(rr[2 * j]),
                                                  __uint_as_float(rr[2 * j + 1])), sl2v, nmv);
                    e.x = fast_exp2(e.x);
                    e.y = fast_exp2(e.y);
                    pk[j] = pack_bf16(e.x, e.y);
                    acc_bf16x2(ps[j & 3], pk[j]);
                }
            }
            // P -> TMEM over this tile's S columns (bf16 pairs), then the MMA.
#pragma unroll
            for (int c0 = 0; c0 < S_TOK / 2; c0 += 32) tmem_st32(tS + c0, pk + c0);
            } else {
            // S_TOK = 128: the scores are handled in 64-column halves (two
            // CTAs per SM leave no room for 128 scores next to their
            // exponentials). P of tokens [0, 64) goes to columns [0, 32),
            // of tokens [64, 128) to [32, 64); each store lands on columns
            // whose f32 scores were already read.
            uint32_t rr[64];
            if (t < U) {
                if (__any_sync(0xffffffffu, sel)) {
                    tmem_ld32(tS + 0, rr);
                    tmem_ld32(tS + 32, rr + 32);
                    tmem_wait_ld();
                    float mx = row_max(rr, 64);
                    tmem_ld32(tS + 64, rr);
                    tmem_ld32(tS + 96, rr + 32);
                    tmem_wait_ld();
                    mx = fmaxf(mx, row_max(rr, 64));
                    const float2 nb = make_float2(-mx * sl2, -mx * sl2);
                    float2 z2[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) z2[k] = make_float2(0.f, 0.f);
                    // exponentials of tokens [64, 128): kept in rr (f32 bits)
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        float2 e = f2_fma(make_float2(__uint_as_float(rr[2 * j]),
                                                      __uint_as_float(rr[2 * j + 1])), sl2v, nb);
                        e.x = fast_exp2(e.x);
                        e.y = fast_exp2(e.y);
                        z2[j & 3] = f2_add(z2[j & 3], e);
                        rr[2 * j] = __float_as_uint(e.x);
                        rr[2 * j + 1] = __float_as_uint(e.y);
                    }
                    // exponentials of tokens [0, 64): back into their columns
#pragma unroll
                    for (int c0 = 0; c0 < 64; c0 += 32) {
                        uint32_t r0[32];
                        tmem_ld32(tS + c0, r0);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            float2 e = f2_fma(make_float2(__uint_as_float(r0[2 * j]),
                                                          __uint_as_float(r0[2 * j + 1])), sl2v, nb);
                            e.x = fast_exp2(e.x);
                            e.y = fast_exp2(e.y);
                            z2[j & 3] = f2_add(z2[j & 3], e);
                            r0[2 * j] = __float_as_uint(e.x);
                            r0[2 * j + 1] = __float_as_uint(e.y);
                        }
                        tmem_st32(tS + c0, r0);
                    }
                    tmem_wait_st();
                    // intra-chunk softmax scaled by exp(s^_c - M0) / z_c;
                    // rows that did not select the chunk get zero weights
                    const float2 zz = f2_add(f2_add(z2[0], z2[1]), f2_add(z2[2], z2[3]));
                    const float f = sel ? __fdividef(fast_exp2(sh - M0l2), zz.x + zz.y) : 0.f;
                    const float2 fv = make_float2(f, f);
#pragma unroll
                    for (int c0 = 0; c0 < 64; c0 += 32) {
                        uint32_t r0[32], pk[16];
                        tmem_ld32(tS + c0, r0);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float2 pv = f2_mul(make_float2(__uint_as_float(r0[2 * j]),
                                                                 __uint_as_float(r0[2 * j + 1])), fv);
                            pk[j] = pack_bf16(pv.x, pv.y);
                            acc_bf16x2(ps[j & 3], pk[j]);
                        }
                        tmem_st16(tS + c0 / 2, pk);
                    }
                    {
                        uint32_t pk[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float2 pv = f2_mul(make_float2(__uint_as_float(rr[2 * j]),
                                                                 __uint_as_float(rr[2 * j + 1])), fv);
                            pk[j] = pack_bf16(pv.x, pv.y);
                            acc_bf16x2(ps[j & 3], pk[j]);
                        }
                        tmem_st32(tS + 32, pk);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 64; ++j) rr[j] = 0u;
                    tmem_st32(tS + 0, rr);
                    tmem_st32(tS + 32, rr + 32);
                }
            } else {
                // masked row max over both halves
                float mx = -INFINITY;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    tmem_ld32(tS + 64 * hf, rr);
                    tmem_ld32(tS + 64 * hf + 32, rr + 32);
                    tmem_wait_ld();
                    if (any_edge) {
#pragma unroll
                        for (int j = 0; j < 64; ++j) {
                            const int pos = j0 + 64 * hf + j;
                            const bool in = valid && pos >= w0 && pos <= i;
                            rr[j] = in ? rr[j] : __float_as_uint(-INFINITY);
                        }
                    }
                    mx = fmaxf(mx, row_max(rr, 64));
                }
                if (!window_rescale(mx * sl2)) { ok = false; break; }
                const float nm = (mref == -INFINITY) ? 0.f : -mref;
                const float2 nmv = make_float2(nm, nm);
                // half 1 is still in rr: its P goes to columns [32, 64) only
                // after half 0 (columns [0, 64)) has been read back
                uint32_t pk[32];
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t r0[64];
                    const uint32_t *src = rr;
                    if (hf == 0) {
                        tmem_ld32(tS + 0, r0);
                        tmem_ld32(tS + 32, r0 + 32);
                        tmem_wait_ld();
                        if (any_edge) {
#pragma unroll
                            for (int j = 0; j < 64; ++j) {
                                const int pos = j0 + j;
                                const bool in = valid && pos >= w0 && pos <= i;
                                r0[j] = in ? r0[j] : __float_as_uint(-INFINITY);
                            }
                        }
                        src = r0;
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        float2 e = f2_fma(make_float2(__uint_as_float(src[2 * j]),
                                                      __uint_as_float(src[2 * j + 1])), sl2v, nmv);
                        e.x = fast_exp2(e.x);
                        e.y = fast_exp2(e.y);
                        pk[j] = pack_bf16(e.x, e.y);
                        acc_bf16x2(ps[j & 3], pk[j]);
                    }
                    tmem_st32(tS + 32 * hf, pk);
                }
            }
            }
            // The normaliser l sums the rounded weights the MMA consumes, so
            // the weights applied to V add up to one: in a peaked row the
            // rounding of P then moves O by ~2^-9 w(1-w)|v| instead of
            // ~2^-9 w|v|.
            {
                const float2 pt = f2_add(f2_add(ps[0], ps[1]), f2_add(ps[2], ps[3]));
                l += pt.x + pt.y;
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&st.p_full[sb]);
        }

        // final: O / l once the last PV is done
        if (ok && T > 0) {
            const int u = T - 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&st.p_empty[u % NSB], (u / NSB) & 1, abort));
        }
        if (ok) {
            tc_fence_after();
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.O) +
                                  (((int64_t)b * p.Hq + h) * p.N + i) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t ro[32];
                tmem_ld32(trow + L::TMEM_O + c0, ro);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint4 v;
                        v.x = pack_bf16(__uint_as_float(ro[j + 0]) * inv, __uint_as_float(ro[j + 1]) * inv);
                        v.y = pack_bf16(__uint_as_float(ro[j + 2]) * inv, __uint_as_float(ro[j + 3]) * inv);
                        v.z = pack_bf16(__uint_as_float(ro[j + 4]) * inv, __uint_as_float(ro[j + 5]) * inv);
                        v.w = pack_bf16(__uint_as_float(ro[j + 6]) * inv, __uint_as_float(ro[j + 7]) * inv);
                        *reinterpret_cast<uint4 *>(orow + c0 + j) = v;
                    }
                }
            }
        }
    }

    // ------------------------------------------------------------ teardown
    if (*abort && (threadIdx.x & 31) == 0) report(p.status, HILS_ERR_DEVICE_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
    if (threadIdx.x == 0 && st.abort) report(p.status, HILS_ERR_DEVICE_TIMEOUT);
}

template <int S_TOK, int D>
cudaError_t launch_attend_t(const TcParams &tp, const TcMaps &maps,
                            cudaStream_t st) {
    using L = AttnLayout<S_TOK, D>;
    const size_t smem = tc_attend_smem_bytes(tp, S_TOK, D);
    auto kern = tc_attend_kernel<S_TOK, D>;
    cudaError_t e = cudaFuncSetAttribute(
        kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const int nqb = (tp.N + tp.M - 1) / tp.M;
    const int64_t grid = (int64_t)tp.B * tp.Hkv * nqb;
    if (grid <= 0) return cudaSuccess;
    kern<<<(unsigned)grid, kThreads, smem, st>>>(maps.k, maps.v, tp);
    (void)sizeof(L);
    return cudaGetLastError();
}

}  // namespace

size_t tc_attend_smem_bytes(const TcParams &tp, int s_tok, int d) {
    const size_t nst = (d + 2 * s_tok) <= 256 ? 2 : 1;     // AttnLayout::NST
    size_t big = (size_t)kRows * d * 2 + 2ull * nst * s_tok * d * 2;
    size_t small = sizeof(SmallState) + sizeof(int) * ((size_t)tp.M * tp.K + tp.ucap) +
                   sizeof(uint32_t) * (((size_t)tp.nC + 31) / 32);
    return 1024 + big + ((small + 15) / 16) * 16;
}

cudaError_t launch_tc_attend(const TcParams &tp, const TcMaps &maps,
                             cudaStream_t st) {
    if (tp.S == 64 && tp.d == 128) return launch_attend_t<64, 128>(tp, maps, st);
    if (tp.S == 64 && tp.d == 64) return launch_attend_t<64, 64>(tp, maps, st);
    if (tp.S == 128 && tp.d == 128) return launch_attend_t<128, 128>(tp, maps, st);
    if (tp.S == 128 && tp.d == 64) return launch_attend_t<128, 64>(tp, maps, st);
    return cudaErrorNotSupported;
}

}  // namespace hils
