// bwd_rows_tc.cu -- query side of the prefill backward on the sm_100a tensor
// cores (bf16 inputs): dQ, and the per-(row, head) statistics the key side
// consumes.
//
// "Hierarchical Sparse Attention Done Right", Sec. 3 (RQ2: the fused
// chunk-level softmax) and Sec. 4 (native sparse training). For one row i,
// head h (kv group g), with s_j = q.k_j/sqrt(d), u_j = dO.v_j,
// s^_c = qs.k'_c/sqrt(d) + b'_c:
//   lz_c   = log sum_{j in c} e^{s_j},  Ubar_c = sum_{j in c} e^{s_j - lz_c} u_j
//   L      = log(sum_c e^{s^_c} + sum_win e^{s_j})
//   D      = sum_c e^{s^_c - L} Ubar_c + sum_win e^{s_j - L} u_j
//   ds_j   = e^{s_j - a_c} (u_j - Ubar_c), a_c = lz_c - s^_c + L  (chunk c)
//   ds_j   = e^{s_j - L} (u_j - D)                                 (window)
//   dq     = sum_j ds_j k_j / sqrt(d);  dsh_c = e^{s^_c - L} (Ubar_c - D)
//
// Three kernels:
//   bwd_sh     s^_c of every valid selection (warp per (b, g, i), lanes
//              split the dims), into slot 3 of the (row, head, slot) record.
//   bwd_rows   one CTA per (b, g, 128/G adjacent queries) x G heads = 128
//              rows (row = TMEM lane), like the forward's attention: the
//              union of the queries' selected chunks and the aligned window,
//              in 64-token tiles (a 128-token chunk is two), each brought in
//              by TMA. Two passes over the tiles:
//                A: S = Q K^T, U = dO V^T (tcgen05.mma, f32 in TMEM) give
//                   lz_c, Ubar_c of the selected chunks and the window sums;
//                   then L, D, a_c and dsh_c per row.
//                B: S, U again; dS (bf16) over the S columns; dQ += dS K
//                   (tcgen05.mma, A from TMEM, f32 accumulator in TMEM).
//              Writes dQ (the part through the tokens), L and D, and
//              (a_c, Ubar_c, dsh_c, s^_c) per selected slot.
//   bwd_dqs    dqs = sum_c dsh_c k'_c / sqrt(d) per (row, head): into dQs
//              under query calibration, else added to dQ.
// Warp roles of bwd_rows: warp 0 TMA producer (K, V), warp 1 MMA issuer and
// TMEM owner, warps 2-5 Q / dO loader and softmax (warp w reads TMEM lanes
// 32*(w%4)..+31); two CTAs per SM. L and D are summed online during pass A
// (each selected chunk's record is fetched one chunk ahead). Every wait is
// bounded; a lost arrival ends the kernel with HILS_ERR_DEVICE_TIMEOUT in the
// status word. No floating-point atomics: every sum has one fixed order.
#include <math.h>

#include "hils_fast.cuh"
#include "sm100.cuh"
#include "tc_kernels.cuh"

namespace hils {

namespace {

using namespace sm100;

constexpr int kRT = 192;          // threads of bwd_rows
constexpr int kRows = 128;
constexpr int kTile = 64;         // tokens per tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// DL consecutive bf16 values (DL = 2 or 4) in one load, as f32
template <int DL>
__device__ __forceinline__ void load_bf16s(const __nv_bfloat16 *src, float *f) {
    if constexpr (DL == 4) {
        const uint2 w = __ldg(reinterpret_cast<const uint2 *>(src));
        f[0] = __uint_as_float(w.x << 16); f[1] = __uint_as_float(w.x & 0xffff0000u);
        f[2] = __uint_as_float(w.y << 16); f[3] = __uint_as_float(w.y & 0xffff0000u);
    } else {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(src));
        f[0] = __uint_as_float(w << 16); f[1] = __uint_as_float(w & 0xffff0000u);
    }
}

// ------------------------------------------------------------------ s^_c
// Lanes over top-K slots: a lane takes one (row, slot) and forms the whole
// dot products of the slot's landmark key with the G scoring rows, which
// the warp first stages in shared memory as f32 (no cross-lane reductions).
// With K <= 16 a warp takes two rows (16 lanes each), with K > 32 a lane
// takes two slots.
constexpr int kShWarps = 4;

template <int D>
__global__ void __launch_bounds__(32 * kShWarps) bwd_sh_kernel(const BwdRowsParams p) {
    __shared__ __align__(16) float qsm[kShWarps][2][8][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rpw = p.K <= 16 ? 2 : 1;               // rows per warp
    const int lpr = 32 / rpw;                        // lanes per row
    const int64_t nrows = (int64_t)p.B * p.Hkv * p.N;
    const int64_t row0 = ((int64_t)blockIdx.x * kShWarps + warp) * rpw;
    if (row0 >= nrows) return;
    const __nv_bfloat16 *Qs = reinterpret_cast<const __nv_bfloat16 *>(p.Qs ? p.Qs : p.Q);
    const __nv_bfloat16 *Kl = reinterpret_cast<const __nv_bfloat16 *>(p.Klm);
    // stage the scoring rows of the warp's rows (f32), 8 values per lane step
    for (int e = lane; e < rpw * p.G * (D / 8); e += 32) {
        const int rs = e / (p.G * (D / 8)), h = (e / (D / 8)) % p.G, u = e % (D / 8);
        const int64_t row = row0 + rs;
        float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (row < nrows) {
            const int i = (int)(row % p.N), g = (int)((row / p.N) % p.Hkv);
            const int b = (int)(row / ((int64_t)p.N * p.Hkv));
            const uint4 w = __ldg(reinterpret_cast<const uint4 *>(
                Qs + (((int64_t)b * p.Hq + p.group_heads[g * p.G + h]) * p.N + i) * D) + u);
            const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                f[2 * k] = __uint_as_float(x[k] << 16);
                f[2 * k + 1] = __uint_as_float(x[k] & 0xffff0000u);
            }
        }
        float4 *dst = reinterpret_cast<float4 *>(&qsm[warp][rs][h][u * 8]);
        dst[0] = make_float4(f[0], f[1], f[2], f[3]);
        dst[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
    __syncwarp();
    const int rs = lane / lpr;
    const int64_t row = row0 + rs;
    if (row >= nrows) return;
    const int i = (int)(row % p.N), g = (int)((row / p.N) % p.Hkv);
    const int b = (int)(row / ((int64_t)p.N * p.Hkv));
    const int64_t bg = (int64_t)b * p.Hkv + g;
    int64_t w0, nc;
    window_bounds(i, p.S, p.W, &w0, &nc);
    for (int k = lane % lpr; k < p.K; k += lpr) {
        const int c = __ldg(p.idx + (bg * p.N + i) * p.K + k);
        if (c < 0 || c >= nc) continue;
        const uint4 *kr = reinterpret_cast<const uint4 *>(Kl + (bg * p.nC + c) * D);
        float acc[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) acc[h] = 0.f;
#pragma unroll 4
        for (int u = 0; u < D / 8; ++u) {
            const uint4 w = __ldg(kr + u);
            const uint32_t x[4] = {w.x, w.y, w.z, w.w};
            float kv[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                kv[2 * q] = __uint_as_float(x[q] << 16);
                kv[2 * q + 1] = __uint_as_float(x[q] & 0xffff0000u);
            }
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                if (h >= p.G) break;
                const float4 qa = *reinterpret_cast<const float4 *>(&qsm[warp][rs][h][u * 8]);
                const float4 qb = *reinterpret_cast<const float4 *>(&qsm[warp][rs][h][u * 8 + 4]);
                acc[h] = fmaf(qa.x, kv[0], acc[h]); acc[h] = fmaf(qa.y, kv[1], acc[h]);
                acc[h] = fmaf(qa.z, kv[2], acc[h]); acc[h] = fmaf(qa.w, kv[3], acc[h]);
                acc[h] = fmaf(qb.x, kv[4], acc[h]); acc[h] = fmaf(qb.y, kv[5], acc[h]);
                acc[h] = fmaf(qb.z, kv[6], acc[h]); acc[h] = fmaf(qb.w, kv[7], acc[h]);
            }
        }
        const float bc = __ldg(p.bias + bg * p.nC + c);
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            if (h >= p.G) break;
            const int64_t rq = ((int64_t)b * p.Hq + p.group_heads[g * p.G + h]) * p.N + i;
            p.chunkstat[(rq * p.K + k) * 4 + 3] = acc[h] * p.inv_sqrt_d + bc;
        }
    }
}

// --------------------------------------------------------------- dqs
// Same layout: slots 32 at a time, each head's dsh of the slot read by the
// slot's lane and broadcast, four landmark rows in flight.
template <int D>
__global__ void __launch_bounds__(128) bwd_dqs_kernel(const BwdRowsParams p) {
    constexpr int DL = D / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 4 + warp;      // (b, g, i)
    if (row >= (int64_t)p.B * p.Hkv * p.N) return;
    const int i = (int)(row % p.N);
    const int g = (int)((row / p.N) % p.Hkv);
    const int b = (int)(row / ((int64_t)p.N * p.Hkv));
    const int64_t bg = (int64_t)b * p.Hkv + g;
    const __nv_bfloat16 *Kl = reinterpret_cast<const __nv_bfloat16 *>(p.Klm);
    int64_t w0, nc;
    window_bounds(i, p.S, p.W, &w0, &nc);
    float acc[8][DL];
#pragma unroll
    for (int h = 0; h < 8; ++h)
#pragma unroll
        for (int r = 0; r < DL; ++r) acc[h][r] = 0.f;
    const int32_t *ir = p.idx + (bg * p.N + i) * p.K;
    for (int k0 = 0; k0 < p.K; k0 += 32) {
        int cl = k0 + lane < p.K ? __ldg(ir + k0 + lane) : -1;
        if (cl >= nc) cl = -1;
        float dl[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            dl[h] = 0.f;
            if (h >= p.G || cl < 0) continue;
            const int64_t rq = ((int64_t)b * p.Hq + p.group_heads[g * p.G + h]) * p.N + i;
            dl[h] = p.chunkstat[(rq * p.K + k0 + lane) * 4 + 2];
        }
        const int kn = min(32, p.K - k0);
        for (int k1 = 0; k1 < kn; k1 += 4) {
            float kv[4][DL];
            int cc[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                cc[u] = __shfl_sync(0xffffffffu, cl, (k1 + u) & 31);
                if (k1 + u >= kn) cc[u] = -1;
                load_bf16s<DL>(Kl + (bg * p.nC + (cc[u] < 0 ? 0 : cc[u])) * D + lane * DL, kv[u]);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
#pragma unroll
                for (int h = 0; h < 8; ++h) {
                    if (h >= p.G) break;
                    const float dsh = __shfl_sync(0xffffffffu, dl[h], (k1 + u) & 31);
                    if (cc[u] < 0) continue;
#pragma unroll
                    for (int r = 0; r < DL; ++r) acc[h][r] = fmaf(dsh, kv[u][r], acc[h][r]);
                }
            }
        }
    }
#pragma unroll
    for (int h = 0; h < 8; ++h) {
        if (h >= p.G) break;
        const int64_t rq = ((int64_t)b * p.Hq + p.group_heads[g * p.G + h]) * p.N + i;
        if (p.dQs) {
            float *o = p.dQs + rq * D + lane * DL;
#pragma unroll
            for (int r = 0; r < DL; ++r) o[r] = acc[h][r] * p.inv_sqrt_d;
        } else {
            float *o = p.dQ + rq * D + lane * DL;
#pragma unroll
            for (int r = 0; r < DL; ++r) o[r] += acc[h][r] * p.inv_sqrt_d;
        }
    }
}

// ---------------------------------------------------------------- rows
// Two CTAs share an SM: TMEM holds dQ (D columns) and S, U of one tile (64
// columns each) within 256 columns, shared memory Q, dO and one stage each of
// K and V; each CTA's softmax covers the other's MMA and copy latencies. K of
// a pass-A tile is handed back when its S product is done, of a pass-B tile
// when its dQ product is; V when its U product is.
template <int D>
struct RowLayout {
    static constexpr uint32_t Q_BYTES = kRows * D * 2;        // Q or dO rows
    static constexpr uint32_t KV_BYTES = kTile * D * 2;       // K or V tile
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_O = Q_BYTES;                // dO
    static constexpr uint32_t OFF_K = 2 * Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + KV_BYTES;
    static constexpr uint32_t OFF_SMALL = OFF_V + KV_BYTES;
    static constexpr int TM_DQ = 0, TM_S = D, TM_U = D + kTile;
    static constexpr uint32_t TMEM_COLS = 256u;
    static_assert(D + 2 * kTile <= 256, "TMEM budget of two CTAs per SM");
};

struct RowSmall {
    uint64_t q_full;
    uint64_t k_full, v_full, k_empty, v_empty;
    uint64_t s_full, p_full;
    uint64_t acc_done;
    uint32_t tmem_base;
    int abort;
    int n_union;
    int n_win;
    int win_start;
};

__device__ __forceinline__ float row_max32(const uint32_t *r) {
    float m[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) m[k] = __uint_as_float(r[k]);
#pragma unroll
    for (int j = 4; j < 32; j += 4)
#pragma unroll
        for (int k = 0; k < 4; ++k) m[k] = fmaxf(m[k], __uint_as_float(r[j + k]));
    return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

template <int D>
__global__ void __launch_bounds__(kRT, 2)
bwd_rows_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV,
                   const BwdRowsParams p) {
    using L = RowLayout<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    RowSmall &st = *reinterpret_cast<RowSmall *>(smem + L::OFF_SMALL);
    int *s_idx = reinterpret_cast<int *>(smem + L::OFF_SMALL + sizeof(RowSmall));
    int *s_union = s_idx + p.M * p.K;
    uint32_t *s_bits = reinterpret_cast<uint32_t *>(s_union + p.ucap);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nqb = (p.N + p.M - 1) / p.M;
    const int qb = blockIdx.x % nqb;
    const int g = (blockIdx.x / nqb) % p.Hkv;
    const int b = blockIdx.x / (nqb * p.Hkv);
    const int i0 = qb * p.M;
    const int i_last = min(i0 + p.M, p.N) - 1;
    const int HT = p.S / kTile;                      // tiles per chunk
    volatile int *abort = &st.abort;

    if (threadIdx.x == 0) {
        mbar_init(&st.q_full, 128);
        mbar_init(&st.k_full, 1);
        mbar_init(&st.v_full, 1);
        mbar_init(&st.k_empty, 1);
        mbar_init(&st.v_empty, 1);
        mbar_init(&st.s_full, 1);
        mbar_init(&st.p_full, 4);                   // one arrival per softmax warp
        mbar_init(&st.acc_done, 1);
        st.abort = (p.status && *(volatile int32_t *)p.status ==
                                    HILS_ERR_DEVICE_TIMEOUT) ? 1 : 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(&st.tmem_base, L::TMEM_COLS);
    // selected chunks of the block's queries -> smem [K][M]; union bitmap
    const int nwords = (p.nC + 31) >> 5;
    for (int w = threadIdx.x; w < nwords; w += kRT) s_bits[w] = 0u;
    __syncthreads();
    {
        const int32_t *gidx = p.idx + (((int64_t)b * p.Hkv + g) * p.N + i0) * p.K;
        const int nvalid = (i_last - i0 + 1) * p.K;
        for (int e = threadIdx.x; e < p.M * p.K; e += kRT) {
            const int m = e / p.K, k = e % p.K;
            int c = e < nvalid ? __ldg(gidx + e) : -1;
            if (c >= 0) {
                int64_t w0, nc;
                window_bounds(i0 + m, p.S, p.W, &w0, &nc);
                if (c >= nc) c = -1;
            }
            s_idx[k * p.M + m] = c;
            if (c >= 0) atomicOr(&s_bits[c >> 5], 1u << (c & 31));
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
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
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
            st.n_win = (i_last - (int)w0) / kTile + 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = st.tmem_base;
    const int U = st.n_union;
    const int NT = U * HT + st.n_win;                // tiles of one pass
    const int NS = st.abort ? 0 : 2 * NT;            // steps: pass A, pass B
    const int wstart = st.win_start;
    auto tile_row = [&](int t) -> int {              // first token of tile t
        return t < U * HT ? s_union[t / HT] * p.S + (t % HT) * kTile
                          : wstart + (t - U * HT) * kTile;
    };

    if (NS == 0) {
        // skipped: straight to teardown
    } else if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            auto load = [&](int n, bool is_v) {
                uint64_t *bar = is_v ? &st.v_full : &st.k_full;
                const int row = tile_row(n % NT);
                mbar_expect_tx(bar, L::KV_BYTES);
                for (int dh = 0; dh < D / 64; ++dh)
                    tma_load_4d(smem + (is_v ? L::OFF_V : L::OFF_K) + dh * (kTile * 128),
                                is_v ? &tmV : &tmK, bar, dh * 64, row, g, b);
            };
            // each copy goes as soon as its stage has been handed back
            int nk = 0, nv = 0;
            uint64_t t_last = globaltimer();
            for (uint32_t it = 0; nk < NS || nv < NS; ++it) {
                if (nk < NS && (nk == 0 || mbar_test(smem_u32(&st.k_empty), (nk - 1) & 1))) {
                    load(nk++, false);
                    t_last = globaltimer();
                    continue;
                }
                if (nv < NS && (nv == 0 || mbar_test(smem_u32(&st.v_empty), (nv - 1) & 1))) {
                    load(nv++, true);
                    t_last = globaltimer();
                    continue;
                }
                if ((it & 255u) == 0) {
                    if (*abort) break;
                    if (globaltimer() - t_last > kWaitLimitNs) { *abort = 1; break; }
                }
            }
            // on abort: let the copies already issued land before exiting
            if (*abort) {
                if (nk > 0) mbar_drain(&st.k_full, (nk - 1) & 1);
                if (nv > 0) mbar_drain(&st.v_full, (nv - 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ----------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(kRows, kTile, false);
            constexpr uint32_t id_q = idesc_bf16(kRows, D, true);
            const uint32_t sQ = smem_u32(smem + L::OFF_Q);
            const uint32_t sO = smem_u32(smem + L::OFF_O);
            const uint32_t sK = smem_u32(smem + L::OFF_K);
            const uint32_t sV = smem_u32(smem + L::OFF_V);
            bool ok = mbar_wait(&st.q_full, 0, abort);
            int ndq = 0;                             // dQ products issued
            // dQ += dS K for pass-B step u (dS in the S columns); hands K back
            auto dq = [&](int u) {
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    const uint64_t bk = desc_sw128(sK + kk * 16 * 128, kTile * 128, 1024);
                    mma_ts(tmem + L::TM_DQ, tmem + L::TM_S + kk * 8, bk, id_q,
                           (ndq > 0 || kk > 0) ? 1u : 0u);
                }
                ++ndq;
                mma_commit(&st.k_empty);
                (void)u;
            };
            for (int n = 0; ok && n < NS; ++n) {
                // the softmax warps are done with step n-1's S / U (and, in
                // pass B, have left dS for its dQ product)
                if (n >= 1) {
                    if (!mbar_wait(&st.p_full, (n - 1) & 1, abort)) { ok = false; break; }
                    tc_fence_after();
                    if (n - 1 >= NT) dq(n - 1);
                }
                if (!mbar_wait(&st.k_full, n & 1, abort)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t aq = desc_sw128(sQ + (kk / 4) * (kRows * 128) + (kk % 4) * 32, 16, 1024);
                    const uint64_t bk = desc_sw128(sK + (kk / 4) * (kTile * 128) + (kk % 4) * 32, 16, 1024);
                    mma_ss(tmem + L::TM_S, aq, bk, id_s, kk > 0 ? 1u : 0u);
                }
                if (n < NT) mma_commit(&st.k_empty);
                if (!mbar_wait(&st.v_full, n & 1, abort)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ao = desc_sw128(sO + (kk / 4) * (kRows * 128) + (kk % 4) * 32, 16, 1024);
                    const uint64_t bv = desc_sw128(sV + (kk / 4) * (kTile * 128) + (kk % 4) * 32, 16, 1024);
                    mma_ss(tmem + L::TM_U, ao, bv, id_s, kk > 0 ? 1u : 0u);
                }
                mma_commit(&st.v_empty);
                mma_commit(&st.s_full);
            }
            if (ok && mbar_wait(&st.p_full, (NS - 1) & 1, abort)) {
                tc_fence_after();
                dq(NS - 1);
            }
            mma_commit(&st.acc_done);
            mbar_drain(&st.acc_done, 0);
        }
    } else {
        // -------------------------------------------- softmax / epilogue
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int m = r / p.G, hh = r % p.G;
        const int i = i0 + m;
        const bool valid = i < p.N;
        const int h = p.group_heads[g * p.G + hh];
        const int64_t rq = ((int64_t)b * p.Hq + h) * p.N + (valid ? i : 0);
        float *cs = p.chunkstat + rq * p.K * 4;      // this row's slot records
        int64_t w0 = 0, nc = 0;
        if (valid) window_bounds(i, p.S, p.W, &w0, &nc);

        // Q and dO rows -> shared memory (A operands: K-major, 128-byte
        // swizzle), 16-byte units
        {
            constexpr int UPR = D / 8;
            const int tid = threadIdx.x - 64;
            const __nv_bfloat16 *Qp = reinterpret_cast<const __nv_bfloat16 *>(p.Q);
            const __nv_bfloat16 *Op = reinterpret_cast<const __nv_bfloat16 *>(p.dO);
#pragma unroll 1
            for (int arr = 0; arr < 2; ++arr) {
                const __nv_bfloat16 *src = arr == 0 ? Qp : Op;
                uint8_t *dstb = smem + (arr == 0 ? L::OFF_Q : L::OFF_O);
#pragma unroll 1
                for (int e0 = 0; e0 < kRows * UPR; e0 += 8 * 128) {
                    uint4 v[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int e = e0 + q * 128 + tid;
                        const int rr = e / UPR, u = e % UPR;
                        const int mi = i0 + rr / p.G;
                        v[q] = make_uint4(0u, 0u, 0u, 0u);
                        if (e < kRows * UPR && mi < p.N) {
                            const int hq = p.group_heads[g * p.G + rr % p.G];
                            v[q] = __ldg(reinterpret_cast<const uint4 *>(
                                       src + (((int64_t)b * p.Hq + hq) * p.N + mi) * D) + u);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int e = e0 + q * 128 + tid;
                        if (e >= kRows * UPR) continue;
                        const int rr = e / UPR, u = e % UPR;
                        *reinterpret_cast<uint4 *>(dstb + (u >> 3) * (kRows * 128) + rr * 128 +
                                                   (((u & 7) ^ (rr & 7)) << 4)) = v[q];
                    }
                }
            }
            fence_async_smem();
            mbar_arrive(&st.q_full);
        }

        const int *myidx = s_idx + m;                // stride M; valid slots form a prefix
        const int M_ = p.M;
        const float sl2 = p.inv_sqrt_d * kLog2e;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        // The row's next selected slot kp, its chunk ck, and that slot's
        // record prefetched (lz, Ubar, -, s^).
        int kp = 0, ck = 0x7fffffff;
        float4 rec = make_float4(0.f, 0.f, 0.f, 0.f);
        // move to the first selected slot at or after k and fetch its record
        auto seek = [&](int k) {
            while (valid && k < p.K && myidx[k * M_] < 0) ++k;
            kp = k;
            ck = (valid && k < p.K) ? myidx[k * M_] : 0x7fffffff;
            if (ck != 0x7fffffff) rec = *reinterpret_cast<const float4 *>(cs + k * 4);
        };
        seek(0);
        // pass A: the current chunk's (max, sum, sum * u) and the selected
        // chunks' running (max, sum of e^s^, sum of e^s^ Ubar), log2 units;
        // the window's (max, sum, sum * u)
        float cm = -INFINITY, cz = 0.f, czu = 0.f;
        float rm = -INFINITY, rz = 0.f, rd = 0.f;
        float wm = -INFINITY, wz = 0.f, wzu = 0.f;
        float L2 = 0.f, Dr = 0.f;
        float a2 = 0.f, ub = 0.f;                    // pass B: current chunk's a (log2), Ubar
        bool ok = true;

        for (int n = 0; n < NS; ++n) {
            const bool passB = n >= NT;
            const int t = passB ? n - NT : n;
            if (n == NT) {
                // ---- between the passes: L, D of the row
                if (valid) {
                    const float top = fmaxf(rm, wm);           // the window holds token i
                    const float tot = (rm == -INFINITY ? 0.f : rz * fast_exp2(rm - top)) +
                                      wz * fast_exp2(wm - top);
                    L2 = top + __log2f(tot);
                    Dr = (rm == -INFINITY ? 0.f : rd * fast_exp2(rm - L2)) + wzu * fast_exp2(wm - L2);
                    p.rowstat[rq * 2] = L2 * kLn2;
                    p.rowstat[rq * 2 + 1] = Dr;
                }
                seek(0);
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&st.s_full, n & 1, abort))) { ok = false; break; }
            tc_fence_after();
            const uint32_t tS = trow + L::TM_S, tU = trow + L::TM_U;
            // does this row's query select the tile's chunk (chunk tiles)
            bool sel = false, first = false, last = false;
            if (t < U * HT) {
                const int c = s_union[t / HT];
                first = (t % HT) == 0;
                last = (t % HT) == HT - 1;
                if (first)
                    while (ck < c) seek(kp + 1);         // not ascending: skip
                sel = ck == c;
            }
            const bool win = t >= U * HT;
            const int j0 = win ? wstart + (t - U * HT) * kTile : 0;
            const bool edge = win && (!valid || j0 < w0 || j0 + kTile - 1 > i);
            const bool any_edge = __any_sync(0xffffffffu, edge);
            const bool need = win || __any_sync(0xffffffffu, sel);
            if (!passB) {
                // ------------------------------------------------ pass A
                // TMEM loads are warp-collective: every lane of a warp that
                // needs the tile loads S and U in one round trip; lanes whose
                // row does not take part discard the sums.
                if (need) {
                    uint32_t sr[64], ur[64];
                    tmem_ld32(tS, sr);
                    tmem_ld32(tS + 32, sr + 32);
                    tmem_ld32(tU, ur);
                    tmem_ld32(tU + 32, ur + 32);
                    tmem_wait_ld();
                    if (any_edge) {
#pragma unroll
                        for (int j = 0; j < 64; ++j) {
                            const int pos = j0 + j;
                            const bool in = valid && pos >= w0 && pos <= i;
                            sr[j] = in ? sr[j] : __float_as_uint(-INFINITY);
                        }
                    }
                    const float mx = fmaxf(row_max32(sr), row_max32(sr + 32)) * sl2;
                    const bool act = win || sel;
                    if (act && !win && first) { cm = -INFINITY; cz = 0.f; czu = 0.f; }
                    float &Mv = win ? wm : cm;
                    float &Zv = win ? wz : cz;
                    float &ZUv = win ? wzu : czu;
                    const float mn = fmaxf(Mv, mx);
                    const bool go = act && mn != -INFINITY;
                    const float mref = go ? mn : 0.f;
                    float2 z2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                    float2 zu2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                    const float2 nmn = make_float2(-mref, -mref), sl2v = make_float2(sl2, sl2);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        // masked scores are -inf: their weights are exp2(-inf) = 0
                        float2 e = f2_fma(make_float2(__uint_as_float(sr[2 * j]),
                                                      __uint_as_float(sr[2 * j + 1])), sl2v, nmn);
                        e.x = fast_exp2(e.x);
                        e.y = fast_exp2(e.y);
                        z2[j & 1] = f2_add(z2[j & 1], e);
                        zu2[j & 1] = f2_fma(e, make_float2(__uint_as_float(ur[2 * j]),
                                                           __uint_as_float(ur[2 * j + 1])),
                                            zu2[j & 1]);
                    }
                    if (go) {
                        const float f = fast_exp2(Mv - mn);
                        Zv = Zv * f + ((z2[0].x + z2[0].y) + (z2[1].x + z2[1].y));
                        ZUv = ZUv * f + ((zu2[0].x + zu2[0].y) + (zu2[1].x + zu2[1].y));
                        Mv = mn;
                    }
                    if (sel && last) {
                        // lz_c (natural log), Ubar_c; fold e^s^_c into the
                        // running sums; move to the next slot
                        const float ubc = czu / cz;
                        cs[kp * 4] = (cm + __log2f(cz)) * kLn2;
                        cs[kp * 4 + 1] = ubc;
                        const float sh2 = rec.w * kLog2e;
                        const float nr = fmaxf(rm, sh2);
                        const float f = rm == -INFINITY ? 0.f : fast_exp2(rm - nr);
                        const float e = fast_exp2(sh2 - nr);
                        rz = rz * f + e;
                        rd = rd * f + e * ubc;
                        rm = nr;
                        seek(kp + 1);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&st.p_full);
            } else {
                // ------------------------------------------------ pass B
                if (sel && first) {
                    // a_c = lz_c - s^_c + L; dsh_c = e^{s^_c - L} (Ubar_c - D)
                    a2 = (rec.x - rec.w) * kLog2e + L2;
                    ub = rec.y;
                    cs[kp * 4] = a2 * kLn2;
                    cs[kp * 4 + 2] = fast_exp2(rec.w * kLog2e - L2) * (rec.y - Dr);
                }
                const float sub = win ? L2 : a2;
                const float del = win ? Dr : ub;
                const bool act = win ? valid : sel;
                const float2 nsub = make_float2(-sub, -sub), ndel = make_float2(-del, -del);
                const float2 sl2v = make_float2(sl2, sl2);
                uint32_t pk[32];
                if (need) {
                    uint32_t sr[64], ur[64];
                    tmem_ld32(tS, sr);
                    tmem_ld32(tS + 32, sr + 32);
                    tmem_ld32(tU, ur);
                    tmem_ld32(tU + 32, ur + 32);
                    tmem_wait_ld();
                    if (any_edge) {
#pragma unroll
                        for (int j = 0; j < 64; ++j) {
                            const int pos = j0 + j;
                            const bool in = valid && pos >= w0 && pos <= i;
                            sr[j] = in ? sr[j] : __float_as_uint(-INFINITY);
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        float2 e = f2_fma(make_float2(__uint_as_float(sr[2 * j]),
                                                      __uint_as_float(sr[2 * j + 1])), sl2v, nsub);
                        e.x = fast_exp2(e.x);
                        e.y = fast_exp2(e.y);
                        const float2 du = f2_add(make_float2(__uint_as_float(ur[2 * j]),
                                                             __uint_as_float(ur[2 * j + 1])), ndel);
                        const float2 ds = f2_mul(e, du);
                        pk[j] = act ? pack_bf16(ds.x, ds.y) : 0u;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) pk[j] = 0u;
                }
                // dS over S columns [0, 32), already read
                tmem_st32(tS, pk);
                if (sel && last) seek(kp + 1);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&st.p_full);
            }
        }
        // dQ (through the tokens) once the last product is done
        if (ok && NS > 0) ok = __all_sync(0xffffffffu, mbar_wait(&st.acc_done, 0, abort));
        if (ok) {
            tc_fence_after();
            float *dqr = p.dQ + rq * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t rv[32];
                tmem_ld32(trow + L::TM_DQ + c0, rv);     // collective: every lane
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int q = 0; q < 32; q += 4)
                        *reinterpret_cast<float4 *>(dqr + c0 + q) = make_float4(
                            __uint_as_float(rv[q]) * p.inv_sqrt_d, __uint_as_float(rv[q + 1]) * p.inv_sqrt_d,
                            __uint_as_float(rv[q + 2]) * p.inv_sqrt_d, __uint_as_float(rv[q + 3]) * p.inv_sqrt_d);
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
}

template <int D>
size_t rows_smem(const BwdRowsParams &p) {
    size_t small = sizeof(RowSmall) + sizeof(int) * ((size_t)p.M * p.K + p.ucap) +
                   sizeof(uint32_t) * (((size_t)p.nC + 31) / 32);
    return 1024 + RowLayout<D>::OFF_SMALL + ((small + 15) / 16) * 16;
}

template <int D>
cudaError_t launch_rows_tc_t(const BwdRowsParams &p, cudaStream_t st) {
    CUtensorMap mk, mv;
    if (!tc_make_map(&mk, p.Kc, D, p.N, p.Hkv, p.B, kTile) ||
        !tc_make_map(&mv, p.V, D, p.N, p.Hkv, p.B, kTile))
        return cudaErrorInvalidValue;
    const int64_t rows = (int64_t)p.B * p.Hkv * p.N;
    const unsigned wgrid = (unsigned)((rows + 3) / 4);
    const int64_t sh_rows = (int64_t)kShWarps * (p.K <= 16 ? 2 : 1);
    if (p.nC > 0) bwd_sh_kernel<D><<<(unsigned)((rows + sh_rows - 1) / sh_rows), 32 * kShWarps, 0, st>>>(p);
    const size_t smem = rows_smem<D>(p);
    auto kern = bwd_rows_tc_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int nqb = (p.N + p.M - 1) / p.M;
    kern<<<(unsigned)((int64_t)p.B * p.Hkv * nqb), kRT, smem, st>>>(mk, mv, p);
    if (p.nC > 0 || p.dQs) bwd_dqs_kernel<D><<<wgrid, 128, 0, st>>>(p);
    count_launches(1 + (p.nC > 0 ? 1 : 0) + ((p.nC > 0 || p.dQs) ? 1 : 0));
    return cudaGetLastError();
}

}  // namespace

size_t bwd_rows_tc_smem(const BwdRowsParams &p) {
    return p.d == 128 ? rows_smem<128>(p) : rows_smem<64>(p);
}

cudaError_t launch_bwd_rows_tc(const BwdRowsParams &p, cudaStream_t st) {
    return p.d == 128 ? launch_rows_tc_t<128>(p, st) : launch_rows_tc_t<64>(p, st);
}

}  // namespace hils
