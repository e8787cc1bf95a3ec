// decode_fast.cu -- HiLS decode step, HBM-bound kernels for sm_100a.
//
// "Hierarchical Sparse Attention Done Right", Sec. 3 (surrogate score, top-K,
// hierarchical softmax) and Sec. 4.1 (GQA group selection), for one query
// per sequence at i = cache_len-1 (the pages' decode setting, Sec. 7.1).
//
// The step reads every candidate landmark key once (the O(N/S) routing
// scan) and the selected chunks + window of the caches once:
//   dec_score   an equal run of the (b, kv head, 64-chunk tile) space per
//               CTA, three CTAs per SM: landmark tiles (and their b') by
//               TMA, s^ for the G heads of the group (mma.sync m16n8k16 used
//               as a dot-product engine: 16 chunks x 8 head slots x 16
//               dims), raw s^ -> workspace, per-segment (max, sum-exp) per
//               head.
//   dec_select  one CTA per (b, kv head): merge the log-sum-exp partials,
//               group score a_c = max_h (s^_hc - LSE_h); a provable lower
//               bound on the K-th best score (from each warp's two best)
//               keeps K + a few candidates, ordered by a warp bitonic sort
//               (ties to the lower chunk); longer lists get exact ranks
//               counted in shared memory, and lists of more than 1024
//               entries (mass ties) a radix select. idx ascending, s^ of
//               the selected chunks.
//   dec_attend  one CTA per (b, kv head, group of selected-chunk / window
//               tiles), one wave in all: K/V tiles triple-buffered by TMA,
//               QK^T and PV with mma.sync, intra-chunk softmax scaled by
//               exp(s^_c) (chunk tiles) or plain masked softmax (window
//               tiles), merged online -> partial (m, l, o) per group; the
//               CTA that arrives last for its (b, kv head) combines the
//               partials in group order (deterministic) and writes O.
//
// Multi-token (speculative) decode, Sec. 4.2 / Sec. 7.1: T query tokens per
// sequence at positions cache_len-T .. cache_len-1, token-major ([B, T, H,
// ...] = [B*T, H, ...]). dec_score scans each landmark tile once for all T x
// G queries of a (b, kv head) (the T tokens are extra columns of the same
// MMA); dec_select and dec_attend then run per (token, kv head) -- a
// "virtual sequence" v = b*T + t -- reading the physical cache of b. T = 1
// is plain decode.
#include <math.h>

#include "hils_fast.cuh"
#include "sm100.cuh"
#include "tc_kernels.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr int kScoreWarps = 4;
constexpr int kTileChunks = 64;                 // chunks per landmark tile
constexpr int kMaxScanStages = 16;              // landmark tiles in flight per CTA
// Scan CTAs per SM: three share the SM's landmark stages (the
// per-tile work of one CTA is latency-bound; measured: one CTA per SM with
// ten stages 118.8 us per decode step, two 86.0, three 75.8, four 75.8)
constexpr int kScanCtasPerSm = 3;
constexpr int kSelThreads = 1024;
constexpr int kAttThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;

struct DecParams {
    const void *Q, *Qs;
    const float *bias;
    const int32_t *cache_len;
    const int32_t *block_table;  // paged cache: [B, Lmax/S] page of each chunk
    int n_pages;
    void *O;
    int32_t *idx;
    float *sel;
    int32_t *status;
    float *ws_s;        // [B, Hkv, T, G, ncs] raw s^
    float *ws_p;        // [B, Hkv, T, nsplit, G, 2] (max, sum exp(s^ - max))
    float *ws_o;        // [B*T, Hkv, ntile, G, d] partial outputs
    float *ws_ml;       // [B*T, Hkv, ntile, G, 2] partial (m, l)
    int32_t *ws_cnt;    // [B*T, Hkv] arrival tickets
    int B, Hq, Hkv, G, d, S, W, K, Lmax, nC;
    int T;              // query tokens per sequence (1: plain decode)
    int ncs;            // chunk stride of ws_s (max candidates of any row)
    int nsplit;         // scan segments per (b, g), at most
    int scan_tpu;       // landmark tiles per (b, g)
    int scan_per;       // landmark tiles per scan CTA
    int scan_stages;    // tiles in flight per scan CTA
    int ntile;          // attention tiles per (b, g): K + window tiles
    int att_per;        // attention tiles per CTA
    float inv_sqrt_d;
    int16_t group_heads[kMaxHeads];
};

__device__ __forceinline__ void mma_bf16(float *c, const uint32_t *a,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t *r) {
    asm volatile("ldmatrix.sync.aligned.x4.m8n8.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t *r) {
    asm volatile("ldmatrix.sync.aligned.x4.trans.m8n8.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map,
                                            uint64_t *bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile"
        ".mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        :: "r"(smem_u32(dst)), "l"((uint64_t)map), "r"(c0), "r"(c1),
           "r"(smem_u32(bar))
        : "memory");
}

// Contiguous global -> shared copy of `bytes` (a multiple of 16, both
// addresses 16-byte aligned), completing on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(smem_u32(dst)), "l"((uint64_t)src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Byte offset of 16-byte unit u of row r in a TMA 128B-swizzled tile whose
// rows are 128 bytes (one 64-column half of a d=128 row).
__device__ __forceinline__ uint32_t swz(int r, int u) {
    return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4));
}

// Position of token `tok` (0..T-1) of sequence b: cache_len[b] - T + tok.
// False when cache_len[b] is outside [T, Lmax].
__device__ __forceinline__ bool tok_ok(const DecParams &p, int b, int tok,
                                       int64_t *i, int64_t *w0, int64_t *nc) {
    const int L = p.cache_len[b];
    if (L < p.T || L > p.Lmax) return false;
    *i = (int64_t)L - p.T + tok;
    window_bounds(*i, p.S, p.W, w0, nc);
    return true;
}

// --------------------------------------------------------------- dec_score
// The landmark scan, balanced over the SMs: a fixed number of CTAs per SM,
// each streaming an equal run of the flattened (unit, tile) space, unit u =
// (b, kv head),
// tile = kTileChunks landmark rows of that unit. A run crosses unit
// boundaries; each stretch of one unit inside a run is a segment, which
// emits its own (max, sum-exp) partials: segment s of unit u is the one of
// CTA firstcta(u) + s. NG column groups of 8: column n = token * G + head
// slot (n < T*G <= 8*NG).
template <int D, int NG>
__global__ void __launch_bounds__(kScoreWarps * 32)
dec_score_kernel(const __grid_constant__ CUtensorMap tmL, const DecParams p) {
    constexpr int HALVES = D / 64;
    constexpr uint32_t STAGE = kTileChunks * D * 2;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t full[kMaxScanStages];
    __shared__ float red_m[kScoreWarps][8 * NG], red_s[kScoreWarps][8 * NG];
    __shared__ __align__(16) float bias_st[kMaxScanStages][kTileChunks];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gi = lane >> 2, t = lane & 3;
    const int G = p.G, T = p.T, ncol = T * G;
    const int ns = p.scan_stages;
    // b' comes with its tile (one bulk copy into the stage) when every row
    // of it starts on a 16-byte boundary; otherwise lanes load it a tile
    // ahead
    const bool bias_bulk = (p.nC % 4 == 0) && (((uintptr_t)p.bias & 15u) == 0);
    const int64_t total = (int64_t)p.B * p.Hkv * p.scan_tpu;
    const int64_t gt0 = (int64_t)blockIdx.x * p.scan_per;
    const int64_t gt1 = min(gt0 + p.scan_per, total);
    const int ntiles = gt1 > gt0 ? (int)(gt1 - gt0) : 0;
    const void *qb = p.Qs ? p.Qs : p.Q;
    const float sl2 = p.inv_sqrt_d * kLog2e;
    volatile int dummy_abort = 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ns; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    __syncthreads();
    // TMA row of tile k of this run: landmark row u * nC + tile * kTileChunks
    // of the flattened [B*Hkv*nC, d] map (rows past the unit's candidates
    // are read and masked). Thread 0 issues the tiles in order; its cursor
    // (iu, itl) walks the (unit, tile) space without divisions.
    int iu = (int)(gt0 / p.scan_tpu), itl = (int)(gt0 % p.scan_tpu);
    auto issue = [&](int k) {
        const int64_t u = iu, tl = itl;
        if (++itl == p.scan_tpu) { itl = 0; ++iu; }
        const int s = k % ns;
        // b' of the tile's chunks inside [0, nC): a multiple of 4 floats
        const int nb = bias_bulk ? (int)min((int64_t)kTileChunks, p.nC - tl * kTileChunks) : 0;
        mbar_expect_tx(&full[s], STAGE + (nb > 0 ? 4u * nb : 0u));
        for (int hf = 0; hf < HALVES; ++hf)
            tma_load_2d(smem + s * STAGE + hf * (kTileChunks * 128), &tmL, &full[s],
                        hf * 64, (int)(u * p.nC + tl * kTileChunks));
        if (nb > 0)
            bulk_load(&bias_st[s][0], p.bias + u * p.nC + tl * kTileChunks, 4u * nb, &full[s]);
    };
    if (threadIdx.x == 0)
        for (int k = 0; k < min(ntiles, ns); ++k) issue(k);

    // state of the current unit
    int cur = -1, b = 0, g = 0, nc_last = 0;
    uint32_t bq[NG][D / 16][2];
    int nc_col[NG][2];
    float mx[NG][2], sm[NG][2];
    // the partials of the unit's segment held by this CTA
    auto finalize = [&](int u) {
#pragma unroll
        for (int ng = 0; ng < NG; ++ng)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                for (int o = 4; o < 32; o <<= 1) {
                    const float om = __shfl_xor_sync(0xffffffffu, mx[ng][k], o);
                    const float os = __shfl_xor_sync(0xffffffffu, sm[ng][k], o);
                    const float mn = fmaxf(mx[ng][k], om);
                    sm[ng][k] = (mn == -INFINITY) ? 0.f
                                : sm[ng][k] * fast_exp2(mx[ng][k] - mn) + os * fast_exp2(om - mn);
                    mx[ng][k] = mn;
                }
                if (gi == 0) {
                    red_m[warp][ng * 8 + 2 * t + k] = mx[ng][k];
                    red_s[warp][ng * 8 + 2 * t + k] = sm[ng][k];
                }
            }
        __syncthreads();
        if (threadIdx.x < ncol) {
            const int n = threadIdx.x;
            float m = -INFINITY, s2 = 0.f;
            for (int w = 0; w < kScoreWarps; ++w) {
                const float om = red_m[w][n], os = red_s[w][n];
                const float mn = fmaxf(m, om);
                s2 = (mn == -INFINITY) ? 0.f : s2 * fast_exp2(m - mn) + os * fast_exp2(om - mn);
                m = mn;
            }
            const int seg = (int)blockIdx.x - (int)(((int64_t)u * p.scan_tpu) / p.scan_per);
            // partials of (b, g, token) at ((u * T + token) * nsplit + seg) * G + slot
            float *pp = p.ws_p + ((((int64_t)u * T + n / G) * p.nsplit + seg) * G + n % G) * 2;
            pp[0] = m;          // log2 units
            pp[1] = s2;
        }
        __syncthreads();                         // red_m / red_s free again
    };
    auto setup = [&](int u, bool first_tile) {
        b = u / p.Hkv;
        g = u - b * p.Hkv;
        if (first_tile && threadIdx.x < T)       // tickets of dec_attend
            p.ws_cnt[((int64_t)b * T + threadIdx.x) * p.Hkv + g] = 0;
        int64_t i, w0, nc = 0;
        if (!tok_ok(p, b, T - 1, &i, &w0, &nc)) {
            nc = 0;                              // reported once, scanned as empty
            if (first_tile && threadIdx.x == 0) report(p.status, HILS_ERR_DEVICE_BAD_LENGTH);
        }
        nc_last = (int)nc;                       // the last token's nc is the largest
        // scoring queries as the B operand: column n = (token, head slot), rows = dims
#pragma unroll
        for (int ng = 0; ng < NG; ++ng) {
            const int n = ng * 8 + gi;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                bq[ng][ks][0] = bq[ng][ks][1] = 0u;
                if (n < ncol) {
                    const int h = p.group_heads[g * G + n % G];
                    const uint32_t *q = reinterpret_cast<const uint32_t *>(
                        reinterpret_cast<const __nv_bfloat16 *>(qb) +
                        (((int64_t)b * T + n / G) * p.Hq + h) * D);
                    bq[ng][ks][0] = q[(ks * 16 + 2 * t) >> 1];
                    bq[ng][ks][1] = q[(ks * 16 + 8 + 2 * t) >> 1];
                }
            }
        }
        // candidates of this lane's output columns 8 ng + 2t + k (token of
        // the column): a token before the last may have fewer
#pragma unroll
        for (int ng = 0; ng < NG; ++ng)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int n = ng * 8 + 2 * t + k;
                int64_t ii, ww, nn = 0;
                if (n < ncol && nc_last > 0) tok_ok(p, b, n / G, &ii, &ww, &nn);
                nc_col[ng][k] = (int)nn;
                mx[ng][k] = -INFINITY;
                sm[ng][k] = 0.f;
            }
    };
    // bias of the lane's 2 chunks of tile k, loaded a tile ahead
    auto load_bias = [&](int k, int u, int tl, float *bv) {
        bv[0] = bv[1] = 0.f;
        if (bias_bulk || k >= ntiles) return;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int c = (int)tl * kTileChunks + warp * 16 + gi + q * 8;
            if (c < p.nC) bv[q] = __ldg(p.bias + u * p.nC + c);
        }
    };
    // consumer cursor over (unit, tile), and the next tile's
    int u = (int)(gt0 / p.scan_tpu), tl = (int)(gt0 % p.scan_tpu);
    int un = u, tn = tl + 1;
    if (tn == p.scan_tpu) { tn = 0; ++un; }
    float bnext[2];
    load_bias(0, u, tl, bnext);
    for (int k = 0; k < ntiles; ++k) {
        if (k > 0) {
            u = un; tl = tn;
            if (++tn == p.scan_tpu) { tn = 0; ++un; }
        }
        if (u != cur) {                          // uniform over the CTA
            if (cur >= 0) finalize(cur);
            setup(u, tl == 0);
            cur = u;
        }
        const int s = k % ns;
        float bcur[2] = {bnext[0], bnext[1]};
        load_bias(k + 1, un, tn, bnext);
        mbar_wait(&full[s], (k / ns) & 1, &dummy_abort);
        if (bias_bulk) {
            bcur[0] = bias_st[s][warp * 16 + gi];
            bcur[1] = bias_st[s][warp * 16 + gi + 8];
        }
        // two independent accumulator chains (even / odd k-steps) halve the
        // dependent MMA latency of a tile
        float acc[NG][4], acc2[NG][4];
#pragma unroll
        for (int ng = 0; ng < NG; ++ng)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[ng][q] = acc2[ng][q] = 0.f;
        const uint32_t base = smem_u32(smem + s * STAGE);
        const int r = warp * 16 + (lane & 15);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const int hf = ks / 4, uu = (ks % 4) * 2 + (lane >> 4);
            uint32_t a[4];
            ldsm_x4(base + hf * (kTileChunks * 128) + swz(r, uu), a);
#pragma unroll
            for (int ng = 0; ng < NG; ++ng)
                if (ng * 8 < ncol) mma_bf16((ks & 1) ? acc2[ng] : acc[ng], a, bq[ng][ks][0], bq[ng][ks][1]);
        }
#pragma unroll
        for (int ng = 0; ng < NG; ++ng)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[ng][q] += acc2[ng][q];
        __syncthreads();                         // stage s fully read
        if (threadIdx.x == 0 && k + ns < ntiles) issue(k + ns);
        // s^ of column n = (token, head slot) at ((u * T + token) * G + slot) * ncs
        float *outs = p.ws_s + (int64_t)u * T * G * p.ncs;
        // acc[ng]: chunks (gi, gi+8) of this warp's 16, columns 8 ng + (2t, 2t+1);
        // each column's running (max, sum) takes both of its chunks at once
        const int c_lo = tl * kTileChunks + warp * 16 + gi;
#pragma unroll
        for (int ng = 0; ng < NG; ++ng)
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const int n = ng * 8 + 2 * t + kk;
                if (n >= ncol) continue;
                float x[2];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int c = c_lo + 8 * h2;
                    const float shat = fmaf(acc[ng][kk + 2 * h2], p.inv_sqrt_d, bcur[h2]);
                    if (c < nc_last) outs[(int64_t)n * p.ncs + c] = shat;
                    x[h2] = (c < nc_col[ng][kk]) ? shat * kLog2e : -INFINITY;
                }
                const float mn = fmaxf(mx[ng][kk], fmaxf(x[0], x[1]));
                if (mn != -INFINITY) {
                    sm[ng][kk] = sm[ng][kk] * fast_exp2(mx[ng][kk] - mn) +
                                 fast_exp2(x[0] - mn) + fast_exp2(x[1] - mn);
                    mx[ng][kk] = mn;
                }
            }
    }
    (void)sl2;
    grid_dep_launch();                           // dec_select may start now
    if (dummy_abort) {                           // a tile never arrived
        if (threadIdx.x == 0) {
            report(p.status, HILS_ERR_DEVICE_TIMEOUT);
            for (int k = max(0, ntiles - ns); k < ntiles; ++k)
                mbar_drain(&full[k % ns], (k / ns) & 1);
        }
        __syncthreads();
        return;
    }
    if (cur >= 0) finalize(cur);
}

// -------------------------------------------------------------- dec_select
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// exclusive prefix over the block (kSelThreads threads) of v; returns it and
// writes the block total to *total.
__device__ int block_excl_scan(int v, int *scratch, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = scratch[lane];
        int xi = w;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, xi, o);
            if (lane >= o) xi += y;
        }
        scratch[lane] = xi - w;                  // exclusive warp offsets
        if (lane == 31) scratch[32] = xi;
    }
    __syncthreads();
    const int r = scratch[warp] + x - v;
    *total = scratch[32];
    __syncthreads();
    return r;
}

constexpr int kSelPer = 16;                      // chunks per thread (<= 16384)

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
    return ((uint64_t)hi << 32) | lo;
}

// Sorts the warp's 64 values, element e = 2*lane + j in v[j], into
// descending order (bitonic network: 21 compare-exchange rounds, partners
// at distance 1 in the same lane, the others one shuffle away).
__device__ __forceinline__ void warp_sort64_desc(uint64_t v[2]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
        for (int s = k >> 1; s >= 1; s >>= 1) {
            uint64_t o[2];
            if (s == 1) {
                o[0] = v[1];
                o[1] = v[0];
            } else {
                o[0] = shfl_xor_u64(v[0], s >> 1);
                o[1] = shfl_xor_u64(v[1], s >> 1);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int e = 2 * lane + j;
                // the lower element of a pair keeps the larger value in a
                // descending block ((e & k) == 0), the smaller otherwise
                const bool keep_max = ((e & s) == 0) == ((e & k) == 0);
                v[j] = keep_max ? (v[j] > o[j] ? v[j] : o[j])
                                : (v[j] < o[j] ? v[j] : o[j]);
            }
        }
    }
}
constexpr int kCandCap = 1024;                   // threshold-path candidate list
constexpr int kMaxSplits = 64;                   // staged landmark-split partials

// s^ of head slot hh for this thread's chunks cbeg .. cbeg+per-1 (16-byte
// loads; rows are padded to a multiple of 4, values past nc are read but
// never turned into keys)
template <int PER>
__device__ __forceinline__ void sel_load_row(const float *ss, int ncs, int hh,
                                             int cbeg, int per, int nc,
                                             float (&v)[PER]) {
    const float *row = ss + (int64_t)hh * ncs;
#pragma unroll
    for (int q4 = 0; q4 < PER / 4; ++q4) {
        float4 f = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        if (4 * q4 < per && cbeg + 4 * q4 < nc)
            f = __ldcg(reinterpret_cast<const float4 *>(row + cbeg + 4 * q4));
        v[4 * q4 + 0] = f.x; v[4 * q4 + 1] = f.y;
        v[4 * q4 + 2] = f.z; v[4 * q4 + 3] = f.w;
    }
}

template <int PER>
__global__ void __launch_bounds__(kSelThreads)
dec_select_kernel(const DecParams p) {
    __shared__ float lse[HILS_MAX_GROUP];
    __shared__ int hist[256];
    __shared__ int scan_scr[33];
    __shared__ int sh_digit, sh_need;
    __shared__ float part[kMaxSplits * 8][2];
    __shared__ uint32_t wtop[2 * (kSelThreads / 32)];
    __shared__ uint32_t sh_tau;
    __shared__ int ncand;
    __shared__ uint32_t cand_k[kCandCap];
    __shared__ int cand_c[kCandCap];
    // one CTA per (token v = b*T + tok, kv head g)
    const int g = blockIdx.x, v = blockIdx.y;
    const int b = v / p.T, tok = v - b * p.T;
    const int bgt = (b * p.Hkv + g) * p.T + tok;     // score workspace row
    const int bgv = v * p.Hkv + g;                   // idx row
    const int G = p.G, K = p.K;
    int64_t i, w0, nc64;
    if (!tok_ok(p, b, tok, &i, &w0, &nc64)) return;
    const int nc = (int)nc64;
    const float *ss = p.ws_s + (int64_t)bgt * G * p.ncs;
    grid_dep_wait();                             // dec_score's s^ and partials
    grid_dep_launch();                           // dec_attend may start now

    // chunks of this thread: c = tid * per + q, per a multiple of 4 (16-byte
    // loads), at most PER. The s^ of the first two heads are loaded before
    // the log-sum-exp merge so both round trips overlap.
    const int per = ((nc + kSelThreads - 1) / kSelThreads + 3) & ~3;
    const int cbeg = threadIdx.x * per;
    float v0[PER], v1[PER];
    sel_load_row<PER>(ss, p.ncs, 0, cbeg, per, nc, v0);
    if (G > 1) sel_load_row<PER>(ss, p.ncs, 1, cbeg, per, nc, v1);

    // merge the split partials: all loaded at once into shared memory, then
    // folded in split order by one thread per head
    // the scan segments of this (b, g): CTAs firstcta .. lastcta
    const int64_t u0 = (int64_t)(b * p.Hkv + g) * p.scan_tpu;
    const int nsp = (int)((u0 + p.scan_tpu - 1) / p.scan_per - u0 / p.scan_per) + 1;
    const bool staged = nsp * G <= kSelThreads && nsp <= kMaxSplits;
    if (staged && threadIdx.x < nsp * G) {
        const float *pp = p.ws_p + ((int64_t)bgt * p.nsplit * G + threadIdx.x) * 2;
        part[threadIdx.x][0] = pp[0];
        part[threadIdx.x][1] = pp[1];
    }
    __syncthreads();
    if (threadIdx.x < G) {
        const int hh = threadIdx.x;
        float m = -INFINITY, s2 = 0.f;
        for (int sp = 0; sp < nsp; ++sp) {
            const float *pp = staged ? part[sp * G + hh]
                                     : p.ws_p + (((int64_t)bgt * p.nsplit + sp) * G + hh) * 2;
            const float om = pp[0], os = pp[1];
            const float mn = fmaxf(m, om);
            s2 = (mn == -INFINITY) ? 0.f : s2 * exp2f(m - mn) + os * exp2f(om - mn);
            m = mn;
        }
        lse[hh] = (m == -INFINITY) ? 0.f : (m + log2f(s2)) / kLog2e;   // natural
    }
    __syncthreads();

    // group scores a_c = max_h (s^_hc - LSE_h), heads two at a time
    float amax[PER];
#pragma unroll
    for (int q = 0; q < PER; ++q) amax[q] = v0[q] - lse[0];
    if (G > 1) {
#pragma unroll
        for (int q = 0; q < PER; ++q) amax[q] = fmaxf(amax[q], v1[q] - lse[1]);
    }
    for (int hh = 2; hh < G; hh += 2) {
        sel_load_row<PER>(ss, p.ncs, hh, cbeg, per, nc, v0);
        if (hh + 1 < G) sel_load_row<PER>(ss, p.ncs, hh + 1, cbeg, per, nc, v1);
        const float l0 = lse[hh], l1 = hh + 1 < G ? lse[hh + 1] : 0.f;
#pragma unroll
        for (int q = 0; q < PER; ++q) amax[q] = fmaxf(amax[q], v0[q] - l0);
        if (hh + 1 < G) {
#pragma unroll
            for (int q = 0; q < PER; ++q) amax[q] = fmaxf(amax[q], v1[q] - l1);
        }
    }
    uint32_t key[PER];
#pragma unroll
    for (int q = 0; q < PER; ++q)                    // 0: below every real key
        key[q] = (q < per && cbeg + q < nc) ? order_key(amax[q]) : 0u;
    const int nsel = min(nc, K);

    // Threshold path. Each warp's two largest keys belong to distinct
    // chunks, so the K-th largest of those 2 x 32 values is a lower bound on
    // the K-th largest key (K <= 64). Only keys at or above it become
    // candidates. Up to 64 candidates are ordered by one warp (sort by key,
    // ties to the lower chunk, then the first K by chunk); a longer list
    // gets exact ranks counted over it; one longer than kCandCap (exact or
    // near ties over many chunks) falls through to the radix select below.
    if (nc > K && K <= 2 * (kSelThreads / 32)) {
        uint32_t t1 = 0u, t2 = 0u;               // this thread's two largest
#pragma unroll
        for (int q = 0; q < PER; ++q) {
            const uint32_t k = key[q];
            t2 = max(t2, min(t1, k));
            t1 = max(t1, k);
        }
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        for (int o = 1; o < 32; o <<= 1) {       // warp top-2 (merge of pairs)
            const uint32_t o1 = __shfl_xor_sync(0xffffffffu, t1, o);
            const uint32_t o2 = __shfl_xor_sync(0xffffffffu, t2, o);
            const uint32_t n1 = max(t1, o1);
            t2 = max(min(t1, o1), max(t2, o2));
            t1 = n1;
        }
        if (lane == 0) { wtop[2 * warp] = t1; wtop[2 * warp + 1] = t2; }
        if (threadIdx.x == 0) ncand = 0;
        __syncthreads();
        if (warp == 0) {
            // the K-th largest of the 64 warp maxima
            uint64_t w[2] = {(uint64_t)wtop[2 * lane] << 32,
                             (uint64_t)wtop[2 * lane + 1] << 32};
            warp_sort64_desc(w);
            const uint64_t wk = __shfl_sync(0xffffffffu, (uint32_t)(w[(K - 1) & 1] >> 32),
                                            (K - 1) >> 1);
            if (lane == 0) sh_tau = (uint32_t)wk;
        }
        __syncthreads();
        const uint32_t tau = sh_tau;
#pragma unroll
        for (int q = 0; q < PER; ++q) {
            const int c = cbeg + q;
            if (q < per && c < nc && key[q] >= tau) {
                const int at = atomicAdd(&ncand, 1);
                if (at < kCandCap) { cand_k[at] = key[q]; cand_c[at] = c; }
            }
        }
        __syncthreads();
        const int m = ncand;
        if (m <= 64) {
            if (warp == 0) {
                // by key descending, ties to the lower chunk: (key, ~chunk)
                uint64_t w[2];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int e = 2 * lane + j;
                    w[j] = e < m ? ((uint64_t)cand_k[e] << 32) | (0xffffffffu - (uint32_t)cand_c[e])
                                 : 0ull;
                }
                warp_sort64_desc(w);
                // the first K, by chunk ascending: (1, ~chunk) descending
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int e = 2 * lane + j;
                    w[j] = e < K ? ((1ull << 32) | (uint32_t)w[j]) : 0ull;
                }
                warp_sort64_desc(w);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int pos = 2 * lane + j;
                    if (pos < K) {
                        const int c = (int)(0xffffffffu - (uint32_t)w[j]);
                        p.idx[(int64_t)bgv * K + pos] = c;
                        for (int hh = 0; hh < G; ++hh) {
                            const int h = p.group_heads[g * G + hh];
                            p.sel[((int64_t)v * p.Hq + h) * K + pos] = ss[(int64_t)hh * p.ncs + c];
                        }
                    }
                }
            }
            return;                              // nc > K: no padding
        }
        if (m <= kCandCap) {
            bool mine = false;
            uint32_t mk = 0u;
            int mc = 0;
            if (threadIdx.x < m) {
                mk = cand_k[threadIdx.x];
                mc = cand_c[threadIdx.x];
                int rank = 0;
                for (int f = 0; f < m; ++f) {
                    const uint32_t fk = cand_k[f];
                    rank += (fk > mk || (fk == mk && cand_c[f] < mc)) ? 1 : 0;
                }
                mine = rank < K;
            }
            __syncthreads();                     // ranks read the list first
            if (threadIdx.x < m) cand_k[threadIdx.x] = mine ? 1u : 0u;
            __syncthreads();
            if (mine) {                          // ascending chunk order
                int pos = 0;
                for (int f = 0; f < m; ++f) pos += (cand_k[f] && cand_c[f] < mc) ? 1 : 0;
                p.idx[(int64_t)bgv * K + pos] = mc;
                for (int hh = 0; hh < G; ++hh) {
                    const int h = p.group_heads[g * G + hh];
                    p.sel[((int64_t)v * p.Hq + h) * K + pos] = ss[(int64_t)hh * p.ncs + mc];
                }
            }
            return;                              // nc > K: no padding
        }
    }

    uint32_t thr = 0u;                           // selected: key > thr, or == thr and early
    int need_eq = 0;
    if (nc > K) {
        // radix select of the K-th largest key, 8 bits per round
        uint32_t prefix = 0u, pmask = 0u;
        int need = K;                            // still to take among matching keys
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int x = threadIdx.x; x < 256; x += kSelThreads) hist[x] = 0;
            __syncthreads();
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                const int c = cbeg + q;
                if (q < per && c < nc && (key[q] & pmask) == prefix)
                    atomicAdd(&hist[(key[q] >> shift) & 255], 1);
            }
            __syncthreads();
            if (threadIdx.x < 32) {              // digit holding the need-th largest
                const int lane = threadIdx.x;
                int cnt[8], sum = 0;
#pragma unroll
                for (int k = 0; k < 8; ++k) { cnt[k] = hist[255 - (lane * 8 + k)]; sum += cnt[k]; }
                int incl = sum;                  // inclusive count from the top
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                int above = incl - sum;          // keys in higher digits of lower lanes
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (above < need && above + cnt[k] >= need) {
                        sh_digit = 255 - (lane * 8 + k);
                        sh_need = need - above;
                    }
                    above += cnt[k];
                }
            }
            __syncthreads();
            const int dg = sh_digit;
            need = sh_need;
            prefix |= (uint32_t)dg << shift;
            pmask |= 255u << shift;
            __syncthreads();
        }
        thr = prefix;                            // exact K-th largest key
        need_eq = need;                          // how many keys equal to thr to take
    }

    // selected: key > thr, or key == thr among the first need_eq such chunks
    // (chunk order = thread order, then q); positions in ascending chunk order
    int n_eq = 0;
#pragma unroll
    for (int q = 0; q < PER; ++q)
        if (q < per && cbeg + q < nc && nc > K && key[q] == thr) ++n_eq;
    int tot;
    int rank_eq = block_excl_scan(n_eq, scan_scr, &tot);
    uint32_t selbits = 0u;
    int n_sel = 0;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
        const int c = cbeg + q;
        bool sc = false;
        if (q < per && c < nc) {
            if (nc <= K) sc = true;
            else if (key[q] > thr) sc = true;
            else if (key[q] == thr) { sc = rank_eq < need_eq; ++rank_eq; }
        }
        if (sc) { selbits |= 1u << q; ++n_sel; }
    }
    int pos = block_excl_scan(n_sel, scan_scr, &tot);
    while (selbits) {
        const int q = __ffs(selbits) - 1;
        selbits &= selbits - 1;
        const int c = cbeg + q;
        if (pos < K) {
            p.idx[(int64_t)bgv * K + pos] = c;
            for (int hh = 0; hh < G; ++hh) {
                const int h = p.group_heads[g * G + hh];
                p.sel[((int64_t)v * p.Hq + h) * K + pos] = ss[(int64_t)hh * p.ncs + c];
            }
        }
        ++pos;
    }
    for (int k = nsel + threadIdx.x; k < K; k += kSelThreads) {
        p.idx[(int64_t)bgv * K + k] = -1;
        for (int hh = 0; hh < G; ++hh) {
            const int h = p.group_heads[g * G + hh];
            p.sel[((int64_t)v * p.Hq + h) * K + k] = __int_as_float(0x7fc00000);
        }
    }
}

// -------------------------------------------------------------- dec_attend
// One CTA = (b, kv head, group of kAttPer consecutive tiles of that (b, g)'s
// tile list: the selected chunks in idx order, then the window tiles). The
// CTA streams its tiles through a triple-buffered TMA pipeline and merges
// them online per head: running reference max M, O accumulated in the MMA
// registers (rescaled when M rises), l in registers.
constexpr int kAttPerMin = 4;                    // tiles per CTA, at least
constexpr int kAttBuf = 3;                       // K/V tile buffers per CTA

template <int S_TOK, int D>
__global__ void __launch_bounds__(kAttThreads)
dec_attend_kernel(const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const DecParams p) {
    constexpr int HALVES = D / 64;
    constexpr uint32_t TB = S_TOK * D * 2;       // one of K or V
    constexpr int TOK_W = S_TOK / 4;             // tokens per warp (16 or 32)
    constexpr int NT = TOK_W / 8;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t bar[kAttBuf];
    __shared__ float red[4][8];
    __shared__ float rmx[2][4][8], rsm[2][4][8];
    __shared__ int last;
    __shared__ int s_idx[HILS_MAX_TOPK];
    __shared__ float s_sel[8 * HILS_MAX_TOPK];   // G <= 8 on this path
    // [4][8][D] partial O of the 4 warps: used only after the tile loop, when
    // every copy has landed and been read, so it shares the stage buffers
    float *ored = reinterpret_cast<float *>(smem);

    // (token v = b*T + tok, kv head g): cache rows of sequence b, everything
    // else (Q, idx, s^, O, partials, tickets) of the token
    const int grp = blockIdx.x, g = blockIdx.y, v = blockIdx.z;
    const int b = v / p.T, tok = v - b * p.T;
    const int bgc = b * p.Hkv + g;                   // cache rows
    const int bg = v * p.Hkv + g;                    // the token's rows
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gi = lane >> 2, t = lane & 3;
    const int G = p.G;
    int64_t i = 0, w0 = 0, nc = 0;
    const bool ok = tok_ok(p, b, tok, &i, &w0, &nc);
    // the selection always holds min(|C_i|, K) chunks, so the tile list is
    // known before the selection itself is read
    const int nsel = ok ? (int)min(nc, (int64_t)p.K) : 0;
    const int nwin = ok ? (int)((i - w0 + 1 + S_TOK - 1) / S_TOK) : 0;
    const int ntot = nsel + nwin;
    const int tb = grp * p.att_per;
    const int te = min(tb + p.att_per, ntot);
    const int nmine = te > tb ? te - tb : 0;
    auto tile_j0 = [&](int tau) -> int64_t {
        return tau < nsel ? (int64_t)s_idx[tau] * p.S
                          : w0 + (int64_t)(tau - nsel) * S_TOK;
    };
    volatile int dummy_abort = 0;
    bool arrived_all = true;

    if (threadIdx.x == 0 && nmine > 0) {
        for (int k = 0; k < kAttBuf; ++k) mbar_init(&bar[k], 1);
        fence_barrier_init();
    }
    __syncthreads();
    // TMA row of a tile: contiguous cache [B,Hkv,Lmax,d], or the page pool
    // [n_pages,Hkv,S,d] (a tile is one chunk, i.e. one page)
    auto tile_row = [&](int tau) -> int64_t {
        const int64_t j0 = tile_j0(tau);
        if (!p.block_table) return (int64_t)bgc * p.Lmax + j0;
        const int pg = p.block_table[(int64_t)b * (p.Lmax / p.S) + j0 / p.S];
        if (pg < 0 || pg >= p.n_pages) {         // a box wholly before row 0:
            report(p.status, HILS_ERR_DEVICE_BAD_LENGTH);   // TMA reads zeros
            return -(int64_t)p.S;
        }
        return ((int64_t)pg * p.Hkv + g) * p.S;
    };
    auto issue = [&](int k) {                    // tile tb + k into buffer k % kAttBuf
        const int64_t row = tile_row(tb + k);
        const int bi = k % kAttBuf;
        uint8_t *dst = smem + bi * 2 * TB;
        mbar_expect_tx(&bar[bi], 2 * TB);
        for (int hf = 0; hf < HALVES; ++hf) {
            tma_load_2d(dst + hf * (S_TOK * 128), &tmK, &bar[bi], hf * 64, (int)row);
            tma_load_2d(dst + TB + hf * (S_TOK * 128), &tmV, &bar[bi], hf * 64, (int)row);
        }
    };
    // window tiles need nothing from the selection: their copies start
    // before the wait for the selection kernel
    if (threadIdx.x == 0)
        for (int k = 0; k < min(nmine, kAttBuf); ++k)
            if (tb + k >= nsel) issue(k);
    grid_dep_wait();                             // dec_select's idx and s^
    // this (b, g)'s selection -- chunk indices and the heads' s^ -- staged
    // once, so no tile waits on a global load for them
    for (int e = threadIdx.x; e < p.K; e += kAttThreads)
        s_idx[e] = ok ? p.idx[(int64_t)bg * p.K + e] : -1;
    for (int e = threadIdx.x; e < G * p.K; e += kAttThreads) {
        const int hh = e / p.K, kk = e % p.K;
        const int h = p.group_heads[g * G + hh];
        s_sel[e] = ok ? p.sel[((int64_t)v * p.Hq + h) * p.K + kk] : 0.f;
    }
    __syncthreads();
    if (threadIdx.x == 0)
        for (int k = 0; k < min(nmine, kAttBuf); ++k)
            if (tb + k < nsel) issue(k);

    if (nmine > 0) {
        // Q as the A operand: row = head slot gi (< G), cols = dims
        uint32_t aq[D / 16][4];
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            aq[ks][0] = aq[ks][1] = aq[ks][2] = aq[ks][3] = 0u;
            if (gi < G) {
                const int h = p.group_heads[g * G + gi];
                const uint32_t *q = reinterpret_cast<const uint32_t *>(
                    reinterpret_cast<const __nv_bfloat16 *>(p.Q) + ((int64_t)v * p.Hq + h) * D);
                aq[ks][0] = q[(ks * 16 + 2 * t) >> 1];
                aq[ks][2] = q[(ks * 16 + 8 + 2 * t) >> 1];
            }
        }
        const float sl2 = p.inv_sqrt_d * kLog2e;
        float Mrun = -INFINITY, lrun = 0.f;      // natural-log units, per head gi
        float oacc[D / 8][4];
#pragma unroll
        for (int n = 0; n < D / 8; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;

        for (int k = 0; k < nmine; ++k) {
            const int tau = tb + k;
            const bool is_chunk = tau < nsel;
            const int64_t j0 = tile_j0(tau);
            if (!__syncthreads_and(mbar_wait(&bar[k % kAttBuf], (k / kAttBuf) & 1, &dummy_abort) ? 1 : 0)) {
                arrived_all = false;
                break;
            }
            const uint32_t sK = smem_u32(smem + (k % kAttBuf) * 2 * TB);
            const uint32_t sV = sK + TB;
            float sacc[NT][4];
#pragma unroll
            for (int n = 0; n < NT; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
#pragma unroll
            for (int np2 = 0; np2 < NT; np2 += 2) {
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const int hf = ks / 4;
                    const int tok = warp * TOK_W + np2 * 8 + (lane & 7) + ((lane >> 4) << 3);
                    const int u = (ks % 4) * 2 + ((lane >> 3) & 1);
                    uint32_t bm[4];
                    ldsm_x4(sK + hf * (S_TOK * 128) + swz(tok, u), bm);
                    mma_bf16(sacc[np2], aq[ks], bm[0], bm[1]);
                    mma_bf16(sacc[np2 + 1], aq[ks], bm[2], bm[3]);
                }
            }
            // row max and sum: each warp over its tokens (relative to its
            // own max), then one exchange; the arrays alternate with the
            // tile parity, so the next tile's writes never meet this tile's
            // reads (all threads pass the next top barrier first)
            float mloc = -INFINITY;
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int64_t j = j0 + warp * TOK_W + n * 8 + 2 * t + q;
                    float x = sacc[n][q] * sl2;
                    if (!is_chunk && (j < w0 || j > i)) x = -INFINITY;
                    sacc[n][q] = x;
                    mloc = fmaxf(mloc, x);
                }
            mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
            mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
            float sloc = 0.f;
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const float e = (sacc[n][q] == -INFINITY) ? 0.f : fast_exp2(sacc[n][q] - mloc);
                    sacc[n][q] = e;
                    sloc += e;
                }
            sloc += __shfl_xor_sync(0xffffffffu, sloc, 1);
            sloc += __shfl_xor_sync(0xffffffffu, sloc, 2);
            if (t == 0) { rmx[k & 1][warp][gi] = mloc; rsm[k & 1][warp][gi] = sloc; }
            __syncthreads();
            float m = -INFINITY;
#pragma unroll
            for (int w = 0; w < 4; ++w) m = fmaxf(m, rmx[k & 1][w][gi]);
            float z = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float mw = rmx[k & 1][w][gi];
                z += (mw == -INFINITY) ? 0.f : rsm[k & 1][w][gi] * fast_exp2(mw - m);
            }
            // this warp's values are relative to mloc: bring them to m
            const float fw = (mloc == -INFINITY) ? 0.f : fast_exp2(mloc - m);
            // this tile's weights relative to its own reference m_t:
            // chunk tile: m_t = s^_c, weights e/z; window: m_t = max, weights e
            float m_t, scale_t;
            if (is_chunk) {
                m_t = (gi < G) ? s_sel[gi * p.K + tau] : 0.f;
                scale_t = 1.f / z;
            } else {
                m_t = m / kLog2e;
                scale_t = 1.f;
            }
            // online merge with the running reference
            const float Mn = fmaxf(Mrun, m_t);
            const float fo = (Mrun == -INFINITY) ? 0.f : fast_exp2((Mrun - Mn) * kLog2e);
            const float fn = fast_exp2((m_t - Mn) * kLog2e);
            // lrun: this lane's share of the normaliser, summed from the
            // rounded weights the MMA consumes (reduced over lanes / warps
            // at the end), so the weights applied to V add up to one
            lrun *= fo;
            Mrun = Mn;
#pragma unroll
            for (int n = 0; n < D / 8; ++n) { oacc[n][0] *= fo; oacc[n][1] *= fo; }
            const float ws = scale_t * fn * fw;
#pragma unroll
            for (int kk = 0; kk < TOK_W / 16; ++kk) {
                uint32_t ap[4];
                ap[0] = pack_bf16(sacc[2 * kk][0] * ws, sacc[2 * kk][1] * ws);
                ap[1] = 0u;
                ap[2] = pack_bf16(sacc[2 * kk + 1][0] * ws, sacc[2 * kk + 1][1] * ws);
                ap[3] = 0u;
                if (gi >= G) ap[0] = ap[2] = 0u;
                lrun += (__uint_as_float(ap[0] << 16) + __uint_as_float(ap[0] & 0xffff0000u)) +
                        (__uint_as_float(ap[2] << 16) + __uint_as_float(ap[2] & 0xffff0000u));
                const int tok = warp * TOK_W + kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
                for (int n = 0; n < D / 8; n += 2) {
                    const int hf = n / 8;
                    const int u = (n % 8) + (lane >> 4);
                    uint32_t bm[4];
                    ldsm_x4_t(sV + hf * (S_TOK * 128) + swz(tok, u), bm);
                    mma_bf16(oacc[n], ap, bm[0], bm[1]);
                    mma_bf16(oacc[n + 1], ap, bm[2], bm[3]);
                }
            }
            __syncthreads();                     // buffer k % kAttBuf fully read
            if (threadIdx.x == 0 && k + kAttBuf < nmine) issue(k + kAttBuf);
        }
        if (!arrived_all) {
            if (threadIdx.x == 0) {
                report(p.status, HILS_ERR_DEVICE_TIMEOUT);
                for (int k = 0; k < kAttBuf; ++k) mbar_drain(&bar[k], 0);
            }
            __syncthreads();
            return;                              // no ticket: O stays unwritten
        }
        // reduce the 4 warps' O (rows gi < G; cols 8n + 2t, +1) and l
        lrun += __shfl_xor_sync(0xffffffffu, lrun, 1);
        lrun += __shfl_xor_sync(0xffffffffu, lrun, 2);
        if (t == 0) red[warp][gi] = lrun;
        if (gi < G) {
#pragma unroll
            for (int n = 0; n < D / 8; ++n) {
                ored[(warp * 8 + gi) * D + 8 * n + 2 * t] = oacc[n][0];
                ored[(warp * 8 + gi) * D + 8 * n + 2 * t + 1] = oacc[n][1];
            }
        }
        __syncthreads();
        for (int e = threadIdx.x; e < G * D; e += kAttThreads) {
            const int hh = e / D, c = e % D;
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) v += ored[(w * 8 + hh) * D + c];
            p.ws_o[(((int64_t)bg * p.ntile + grp) * G + hh) * D + c] = v;
        }
        if (t == 0 && warp == 0 && gi < G) {
            float *ml = p.ws_ml + (((int64_t)bg * p.ntile + grp) * G + gi) * 2;
            ml[0] = Mrun;
            ml[1] = red[0][gi] + red[1][gi] + red[2][gi] + red[3][gi];
        }
    }

    // arrival ticket; the last CTA of this (b, g) combines the groups in order
    __threadfence();                             // this thread's partials, device-wide
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const int prev = atomicAdd(&p.ws_cnt[bg], 1);
        last = (prev == (int)gridDim.x - 1) ? 1 : 0;
    }
    __syncthreads();
    if (!last || !ok) return;
    __threadfence();
    const int ngrp = (ntot + p.att_per - 1) / p.att_per;
    // per group and head: w_gg / sum_gg' w_gg' l_gg' with w = exp(m - max m).
    // All (m, l) partials of this (b, g) come in with one round trip (the
    // stage buffers are free now), then O = sum of weighted partial O in
    // group order, the partial loads of 8 groups issued together.
    float *cml = reinterpret_cast<float *>(smem);            // [ngrp][G][2]
    float *cw = cml + 2 * ngrp * G;                          // [ngrp][G]
    {
        const float *src = p.ws_ml + (int64_t)bg * p.ntile * G * 2;
        for (int e = threadIdx.x; e < 2 * ngrp * G; e += kAttThreads) cml[e] = __ldcg(src + e);
    }
    __syncthreads();
    if (threadIdx.x < G) {
        const int hh = threadIdx.x;
        float M = -INFINITY;
        for (int gg = 0; gg < ngrp; ++gg) M = fmaxf(M, cml[(gg * G + hh) * 2]);
        float den = 0.f;
        for (int gg = 0; gg < ngrp; ++gg) {
            const float w = exp2f((cml[(gg * G + hh) * 2] - M) * kLog2e);
            cw[gg * G + hh] = w;
            den += w * cml[(gg * G + hh) * 2 + 1];
        }
        const float inv = 1.f / den;
        for (int gg = 0; gg < ngrp; ++gg) cw[gg * G + hh] *= inv;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < G * D; e += kAttThreads) {
        const int hh = e / D, c = e % D;
        const float *ob = p.ws_o + ((int64_t)bg * p.ntile * G + hh) * D + c;
        float num = 0.f;
        for (int g0 = 0; g0 < ngrp; g0 += 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = (g0 + u < ngrp) ? __ldcg(ob + (int64_t)(g0 + u) * G * D) : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (g0 + u < ngrp) num += cw[(g0 + u) * G + hh] * v[u];
        }
        const int h = p.group_heads[g * G + hh];
        reinterpret_cast<__nv_bfloat16 *>(p.O)[((int64_t)v * p.Hq + h) * D + c] =
            __float2bfloat16_rn(num);
    }
    if (threadIdx.x == 0) p.ws_cnt[bg] = 0;      // ready for the next call
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t,
                                  void *, const cuuint64_t *, const cuuint64_t *,
                                  const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

bool map_2d(CUtensorMap *m, const void *base, int d, int64_t rows, int box_rows) {
    void *fp = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fp, cudaEnableDefault,
                                &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return false;
    EncodeTiledFn f = (EncodeTiledFn)fp;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
             strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DecPlan {
    int ncs, nsplit, scan_tpu, scan_per, scan_stages, scan_ctas, ntile, att_per;
    size_t off_s, off_p, off_o, off_ml, off_cnt, total;
};

DecPlan dec_plan(const Problem &p) {
    DecPlan pl;
    int64_t w0, ncm;
    window_bounds((int64_t)p.kv_rows - 1, p.S, p.W, &w0, &ncm);
    // s^ rows padded to a multiple of 4 floats: 16-byte loads in dec_select
    pl.ncs = (int)(((ncm > 0 ? ncm : 1) + 3) & ~(int64_t)3);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // the scan: kScanCtasPerSm CTAs per SM, each streaming an equal run of
    // the (unit, tile) space, 192 KB of landmark tiles in flight per SM; the
    // T tokens of a sequence share its scan
    pl.scan_tpu = (int)((pl.ncs + kTileChunks - 1) / kTileChunks);
    const int64_t total = (int64_t)p.B * p.Hkv * pl.scan_tpu;
    const int64_t slots = (int64_t)sms * kScanCtasPerSm;
    int64_t ctas = total < slots ? total : slots;
    const int64_t per = (total + ctas - 1) / ctas;
    pl.scan_per = (int)per;
    pl.scan_ctas = (int)((total + per - 1) / per);
    // a unit's tiles lie in at most this many CTA runs
    pl.nsplit = (pl.scan_tpu + pl.scan_per - 1) / pl.scan_per + 1;
    {
        const int stage = kTileChunks * p.d * 2;
        int ns = (192 * 1024) / kScanCtasPerSm / stage;
        pl.scan_stages = ns < kMaxScanStages ? ns : kMaxScanStages;
    }
    pl.ntile = p.K + (p.W + 2 * p.S - 2) / p.S + 1;
    // attention: one wave of CTAs, 2 per SM at S = 64 (measured faster than
    // 3 shorter ones), 1 at S = 128
    {
        const int64_t slots = (int64_t)sms * (p.S == 64 ? 2 : 1);
        int64_t groups = slots / ((int64_t)p.B * p.T * p.Hkv);
        if (groups < 1) groups = 1;
        int per = (int)((pl.ntile + groups - 1) / groups);
        if (per < kAttPerMin) per = kAttPerMin;
        pl.att_per = per;
    }
    auto al = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t bg = (size_t)p.B * p.T * p.Hkv;
    pl.off_s = 0;
    pl.off_p = al(pl.off_s + sizeof(float) * bg * p.G * pl.ncs);
    pl.off_o = al(pl.off_p + sizeof(float) * bg * pl.nsplit * p.G * 2);
    pl.off_ml = al(pl.off_o + sizeof(float) * bg * pl.ntile * p.G * p.d);
    pl.off_cnt = al(pl.off_ml + sizeof(float) * bg * pl.ntile * p.G * 2);
    pl.total = al(pl.off_cnt + sizeof(int32_t) * bg);
    return pl;
}

DecParams dec_params(const Problem &p, void *ws) {
    DecPlan pl = dec_plan(p);
    DecParams d;
    char *base = (char *)ws;
    d.Q = p.Q; d.Qs = p.Qs; d.bias = p.bias; d.cache_len = p.cache_len;
    d.block_table = p.block_table; d.n_pages = p.n_pages;
    d.O = p.O; d.idx = p.idx; d.sel = p.sel; d.status = p.status;
    d.ws_s = (float *)(base + pl.off_s);
    d.ws_p = (float *)(base + pl.off_p);
    d.ws_o = (float *)(base + pl.off_o);
    d.ws_ml = (float *)(base + pl.off_ml);
    d.ws_cnt = (int32_t *)(base + pl.off_cnt);
    d.B = p.B; d.Hq = p.Hq; d.Hkv = p.Hkv; d.G = p.G; d.d = p.d; d.S = p.S;
    d.W = p.W; d.K = p.K; d.Lmax = p.kv_rows; d.nC = p.nC; d.T = p.T;
    d.ncs = pl.ncs; d.nsplit = pl.nsplit; d.ntile = pl.ntile;
    d.scan_tpu = pl.scan_tpu; d.scan_per = pl.scan_per; d.scan_stages = pl.scan_stages;
    d.att_per = pl.att_per;
    d.inv_sqrt_d = p.inv_sqrt_d;
    for (int k = 0; k < kMaxHeads; ++k) d.group_heads[k] = p.group_heads[k];
    return d;
}

}  // namespace

// Launch with programmatic stream serialisation: the kernel may start while
// its predecessor finishes, and waits for it (grid_dep_wait) before reading
// what it wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block,
                             size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

bool dec_fast_supported(const Problem &p) {
    if (!p.decode || p.dtype != HILS_BF16) return false;
    if (!(p.d == 64 || p.d == 128) || !(p.S == 64 || p.S == 128)) return false;
    if (p.G > 8 || p.nC < 1) return false;
    if (p.T < 1 || p.T * p.G > 32) return false;
    int64_t w0, ncm;
    window_bounds((int64_t)p.kv_rows - 1, p.S, p.W, &w0, &ncm);
    if (ncm > (int64_t)kSelPer * kSelThreads) return false;
    if ((int64_t)p.B * p.Hkv * p.kv_rows >= (1ll << 31)) return false;
    return true;
}

size_t dec_workspace_bytes(const Problem &p) { return dec_plan(p).total; }

template <int D, int NG>
cudaError_t launch_score_t(dim3 grid, size_t smem, cudaStream_t st,
                           const CUtensorMap &tl, const DecParams &d) {
    cudaError_t e = cudaFuncSetAttribute(dec_score_kernel<D, NG>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dec_score_kernel<D, NG><<<grid, kScoreWarps * 32, smem, st>>>(tl, d);
    return cudaGetLastError();
}

cudaError_t launch_dec_select(Problem &p, void *ws, cudaStream_t st) {
    DecParams d = dec_params(p, ws);
    CUtensorMap tl;
    if (!map_2d(&tl, p.Klm, p.d, (int64_t)p.B * p.Hkv * p.nC, kTileChunks))
        return cudaErrorInvalidValue;
    const size_t smem = 1024 + (size_t)d.scan_stages * kTileChunks * p.d * 2;
    dim3 grid((unsigned)dec_plan(p).scan_ctas);
    const int ncol = p.T * p.G;
    cudaError_t e;
    if (p.d == 128) {
        if (ncol <= 8) e = launch_score_t<128, 1>(grid, smem, st, tl, d);
        else if (ncol <= 16) e = launch_score_t<128, 2>(grid, smem, st, tl, d);
        else e = launch_score_t<128, 4>(grid, smem, st, tl, d);
    } else {
        if (ncol <= 8) e = launch_score_t<64, 1>(grid, smem, st, tl, d);
        else if (ncol <= 16) e = launch_score_t<64, 2>(grid, smem, st, tl, d);
        else e = launch_score_t<64, 4>(grid, smem, st, tl, d);
    }
    if (e != cudaSuccess) return e;
    // chunks per selection thread: the largest candidate count over 1024
    // threads, in {4, 8, 16}
    const int per = ((d.ncs + kSelThreads - 1) / kSelThreads + 3) & ~3;
    const dim3 sg(p.Hkv, p.B * p.T);
    if (per <= 4) e = launch_dependent(dec_select_kernel<4>, sg, dim3(kSelThreads), 0, st, d);
    else if (per <= 8) e = launch_dependent(dec_select_kernel<8>, sg, dim3(kSelThreads), 0, st, d);
    else e = launch_dependent(dec_select_kernel<16>, sg, dim3(kSelThreads), 0, st, d);
    count_launches(2);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int S_TOK, int D>
cudaError_t launch_att_t(const DecParams &d, const CUtensorMap &tk,
                         const CUtensorMap &tv, cudaStream_t st) {
    static_assert(4 * 8 * D * 4 <= 2 * kAttBuf * S_TOK * D * 2, "partial O fits the stages");
    const size_t smem = 1024 + 2ull * kAttBuf * S_TOK * D * 2;
    cudaError_t e = cudaFuncSetAttribute(dec_attend_kernel<S_TOK, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int ngrp = (d.ntile + d.att_per - 1) / d.att_per;
    e = launch_dependent(dec_attend_kernel<S_TOK, D>, dim3(ngrp, d.Hkv, d.B * d.T),
                         dim3(kAttThreads), smem, st, tk, tv, d);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_dec_attend(Problem &p, void *ws, cudaStream_t st) {
    DecParams d = dec_params(p, ws);
    CUtensorMap tk, tv;
    const int64_t rows = p.block_table ? (int64_t)p.n_pages * p.Hkv * p.S
                                       : (int64_t)p.B * p.Hkv * p.kv_rows;
    if (!map_2d(&tk, p.Kc, p.d, rows, p.S) || !map_2d(&tv, p.V, p.d, rows, p.S))
        return cudaErrorInvalidValue;
    cudaError_t e;
    if (p.S == 64 && p.d == 128) e = launch_att_t<64, 128>(d, tk, tv, st);
    else if (p.S == 64 && p.d == 64) e = launch_att_t<64, 64>(d, tk, tv, st);
    else if (p.S == 128 && p.d == 128) e = launch_att_t<128, 128>(d, tk, tv, st);
    else e = launch_att_t<128, 64>(d, tk, tv, st);
    count_launches(1);
    return e;
}

}  // namespace hils
