// backward.cu -- gradients of the HiLS prefill output, selection held fixed.
//
// "Hierarchical Sparse Attention Done Right", Sec. 3 (RQ2: the chunk-level
// softmax fused with the intra-chunk softmax is what lets the language-model
// loss reach the landmark scores) and Sec. 4 (native sparse training). The
// top-K choice is discrete; every continuous quantity of the fused output
// gets its gradient. For one row i, head h (kv group g):
//   s_j = q.k_j/sqrt(d); sh_c = qs.k'_c/sqrt(d) + b'_c; lz_c = log sum_c e^s
//   e_j = s_j - lz_c + sh_c (selected chunks), s_j (window); p = softmax(e)
//   u_j = dO.v_j; D = sum p_j u_j; L = log(sum_c e^{sh_c} + sum_win e^{s_j})
//   chunk c: P_c = e^{sh_c - L}, Ubar_c = sum_{j in c} e^{s_j - lz_c} u_j,
//            ds_j = p_j (u_j - Ubar_c), dsh_c = P_c (Ubar_c - D)
//   window:  p_j = e^{s_j - L}, ds_j = p_j (u_j - D)
//   dV_j += p_j dO; dK_j += ds_j q/sqrt(d); dq += ds_j k_j/sqrt(d)
//   dqs += dsh_c k'_c/sqrt(d); dk'_c += dsh_c qs/sqrt(d); db'_c += dsh_c
//
// Two kernels, no floating-point atomics (every output element is summed by
// one thread in a fixed order, so results are bitwise reproducible):
//   bwd_rows  one warp per (b, g, i) with the group's G heads: two passes
//             over the row's tokens (lane per token) give lz_c, L, D, then
//             p and ds; dq accumulates with lane l owning d/32 dims. Writes
//             dQ (dQs) and per (row, head) L, D and per (row, head, chunk)
//             a = lz_c - s^_c + L, Ubar_c and dsh_c for the key side.
//   bwd_keys  one CTA per (b, g, chunk of S tokens): the query rows that
//             selected the chunk (found by scanning idx, ascending) and the
//             rows whose window covers it, in ascending order; thread
//             (token, eighth of dims) keeps its K/V slice and its dK/dV
//             accumulators in registers. Also dk'_c and db'_c.
// Inputs f32 or bf16, arithmetic and outputs f32.
#include <math.h>
#include <stdint.h>

#include "hils_fast.cuh"
#include "tc_kernels.cuh"

namespace hils {
namespace {

__device__ __forceinline__ float ld_f(const float *p) { return *p; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

struct BwdParams {
    const void *Q, *Qs, *Kc, *Vc, *Klm, *dO;
    const float *bias;
    const int32_t *idx;
    float *dQ, *dQs, *dK, *dV, *dKlm, *dbias;
    float *rowstat;     // [B, Hq, N, 2]: L, D
    // [B, Hq, N, K, 4] for valid selected entries: a = lz_c - s^_c + L (the
    // chunk's tokens get p_j = exp(s_j - a)), Ubar_c, dsh_c = P_c (Ubar_c - D)
    float *chunkstat;
    int *csr_off;       // inverse index (tensor-core key side)
    int32_t *csr_ent;
    int2 *units;        // work units of the tensor-core key side
    int *nunits_blk, *tickets, *n_units;
    float *partial;
    int64_t max_units;
    int32_t *status;
    bool tc_keys;
    int B, Hq, Hkv, G, N, S, W, K, nC;
    float inv_sqrt_d;
    int16_t group_heads[kMaxHeads];
};

__device__ __forceinline__ void bwd_bounds(int64_t i, int S, int W, int64_t *w0,
                                           int64_t *nc) {
    window_bounds(i, S, W, w0, nc);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

constexpr int kRowWarps = 4;

// Shared memory of one warp in bwd_rows: the G heads' q, qs and dO rows
// (f32), the row's valid selected chunks with their idx position, s^, lz and
// Ubar.
template <int D, int GM>
struct RowSmem {
    float q[GM][D], qs[GM][D], go[GM][D];
    int chunk[HILS_MAX_TOPK], kpos[HILS_MAX_TOPK];
    float sh[GM][HILS_MAX_TOPK], lz[GM][HILS_MAX_TOPK], ub[GM][HILS_MAX_TOPK];
};

// 16 bytes of a row as f32: 8 bf16 or 4 f32 values
__device__ __forceinline__ void unpack16(const uint4 &w, const __nv_bfloat16 *, float *f) {
    const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        f[2 * k] = __uint_as_float(x[k] << 16);
        f[2 * k + 1] = __uint_as_float(x[k] & 0xffff0000u);
    }
}
__device__ __forceinline__ void unpack16(const uint4 &w, const float *, float *f) {
    f[0] = __uint_as_float(w.x); f[1] = __uint_as_float(w.y);
    f[2] = __uint_as_float(w.z); f[3] = __uint_as_float(w.w);
}

// s = q_h . k_j and u = dO_h . v_j for the G heads, one token per lane:
// the token's rows in 16-byte loads, q and dO as float4 broadcasts from
// shared memory.
template <typename T, int D, int GM>
__device__ __forceinline__ void token_dots(const RowSmem<D, GM> &sm, int G,
                                           const T *krow, const T *vrow,
                                           float *s, float *u) {
    constexpr int E = 16 / (int)sizeof(T);
#pragma unroll
    for (int h = 0; h < GM; ++h) s[h] = u[h] = 0.f;
#pragma unroll 2
    for (int k0 = 0; k0 < D; k0 += E) {
        float kf[E], vf[E];
        unpack16(__ldg(reinterpret_cast<const uint4 *>(krow + k0)), krow, kf);
        unpack16(__ldg(reinterpret_cast<const uint4 *>(vrow + k0)), vrow, vf);
#pragma unroll
        for (int h = 0; h < GM; ++h) {
            if (h >= G) break;
#pragma unroll
            for (int e4 = 0; e4 < E; e4 += 4) {
                const float4 q4 = *reinterpret_cast<const float4 *>(&sm.q[h][k0 + e4]);
                const float4 g4 = *reinterpret_cast<const float4 *>(&sm.go[h][k0 + e4]);
                s[h] = fmaf(q4.x, kf[e4], s[h]);
                s[h] = fmaf(q4.y, kf[e4 + 1], s[h]);
                s[h] = fmaf(q4.z, kf[e4 + 2], s[h]);
                s[h] = fmaf(q4.w, kf[e4 + 3], s[h]);
                u[h] = fmaf(g4.x, vf[e4], u[h]);
                u[h] = fmaf(g4.y, vf[e4 + 1], u[h]);
                u[h] = fmaf(g4.z, vf[e4 + 2], u[h]);
                u[h] = fmaf(g4.w, vf[e4 + 3], u[h]);
            }
        }
    }
}

template <typename T, int D, int GM>
__global__ void __launch_bounds__(kRowWarps * 32)
bwd_rows_kernel(const BwdParams p) {
    constexpr int DL = D / 32;                   // dims per lane
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    RowSmem<D, GM> &sm = reinterpret_cast<RowSmem<D, GM> *>(smem_raw)[warp];
    const int64_t row = (int64_t)blockIdx.x * kRowWarps + warp;     // (b, g, i)
    if (row >= (int64_t)p.B * p.Hkv * p.N) return;
    const int i = (int)(row % p.N);
    const int g = (int)((row / p.N) % p.Hkv);
    const int b = (int)(row / ((int64_t)p.N * p.Hkv));
    const int G = p.G;
    const float isd = p.inv_sqrt_d;
    const T *Kg = reinterpret_cast<const T *>(p.Kc) + ((int64_t)b * p.Hkv + g) * p.N * D;
    const T *Vg = reinterpret_cast<const T *>(p.Vc) + ((int64_t)b * p.Hkv + g) * p.N * D;
    const T *Lg = reinterpret_cast<const T *>(p.Klm) + ((int64_t)b * p.Hkv + g) * p.nC * D;
    const T *Qs = reinterpret_cast<const T *>(p.Qs ? p.Qs : p.Q);

    // the G heads' rows -> shared memory (f32)
    for (int h = 0; h < G; ++h) {
        const int hq = p.group_heads[g * G + h];
        const int64_t off = (((int64_t)b * p.Hq + hq) * p.N + i) * D;
        for (int k = lane; k < D; k += 32) {
            sm.q[h][k] = ld_f(reinterpret_cast<const T *>(p.Q) + off + k);
            sm.qs[h][k] = ld_f(Qs + off + k);
            sm.go[h][k] = ld_f(reinterpret_cast<const T *>(p.dO) + off + k);
        }
    }
    int64_t w0, nc;
    bwd_bounds(i, p.S, p.W, &w0, &nc);
    // valid selected chunks (ascending, entries outside C_i ignored)
    const int32_t *ir = p.idx + (((int64_t)b * p.Hkv + g) * p.N + i) * p.K;
    int nsel = 0;
    for (int k = 0; k < p.K; ++k) {              // uniform over the warp
        const int c = ir[k];
        if (c >= 0 && c < nc) {
            if (lane == 0) { sm.chunk[nsel] = c; sm.kpos[nsel] = k; }
            ++nsel;
        }
    }
    __syncwarp();
    // s^ of the selected chunks (warp dot products)
    for (int n = 0; n < nsel; ++n) {
        const T *kl = Lg + (int64_t)sm.chunk[n] * D;
        const float bn = p.bias[((int64_t)b * p.Hkv + g) * p.nC + sm.chunk[n]];
        for (int h = 0; h < G; ++h) {
            float a = 0.f;
#pragma unroll
            for (int r = 0; r < DL; ++r) a = fmaf(sm.qs[h][lane * DL + r], ld_f(kl + lane * DL + r), a);
            a = warp_sum(a);
            if (lane == 0) sm.sh[h][n] = a * isd + bn;
        }
    }
    __syncwarp();

    // ---- pass 1: lz_c and Ubar_c per chunk; window sums; then L and D
    float s[GM], u[GM];
    for (int n = 0; n < nsel; ++n) {
        const int64_t j0 = (int64_t)sm.chunk[n] * p.S;
        float m[GM], z[GM], zu[GM];
#pragma unroll
        for (int h = 0; h < GM; ++h) { m[h] = -INFINITY; z[h] = zu[h] = 0.f; }
        for (int t = lane; t < p.S; t += 32) {   // online per lane
            token_dots<T, D, GM>(sm, G, Kg + (j0 + t) * D, Vg + (j0 + t) * D, s, u);
#pragma unroll
            for (int h = 0; h < GM; ++h) {
                const float x = s[h] * isd;
                const float mn = fmaxf(m[h], x);
                const float f = expf(m[h] - mn), e = expf(x - mn);
                z[h] = z[h] * f + e;
                zu[h] = zu[h] * f + e * u[h];
                m[h] = mn;
            }
        }
#pragma unroll
        for (int h = 0; h < GM; ++h) {
            if (h >= G) break;
            const float M = warp_max(m[h]);
            const float f = (m[h] == -INFINITY) ? 0.f : expf(m[h] - M);
            const float Z = warp_sum(z[h] * f), ZU = warp_sum(zu[h] * f);
            if (lane == 0) {
                sm.lz[h][n] = M + logf(Z);
                sm.ub[h][n] = ZU / Z;
            }
        }
    }
    const int64_t nw = (int64_t)i - w0 + 1;      // window tokens
    float wm[GM], wz[GM], wzu[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) { wm[h] = -INFINITY; wz[h] = wzu[h] = 0.f; }
    for (int64_t t = lane; t < nw; t += 32) {
        const int64_t j = w0 + t;
        token_dots<T, D, GM>(sm, G, Kg + j * D, Vg + j * D, s, u);
#pragma unroll
        for (int h = 0; h < GM; ++h) {
            const float x = s[h] * isd;
            const float mn = fmaxf(wm[h], x);
            const float f = expf(wm[h] - mn), e = expf(x - mn);
            wz[h] = wz[h] * f + e;
            wzu[h] = wzu[h] * f + e * u[h];
            wm[h] = mn;
        }
    }
    __syncwarp();
    float Lr[GM], Dr[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        Lr[h] = Dr[h] = 0.f;
        if (h >= G) continue;
        const float M = warp_max(wm[h]);
        const float f = (wm[h] == -INFINITY) ? 0.f : expf(wm[h] - M);
        const float Zw = warp_sum(wz[h] * f), ZUw = warp_sum(wzu[h] * f);
        float top = M;                           // window holds token i: M finite
        for (int n = 0; n < nsel; ++n) top = fmaxf(top, sm.sh[h][n]);
        float tot = Zw * expf(M - top);
        for (int n = 0; n < nsel; ++n) tot += expf(sm.sh[h][n] - top);
        const float L = top + logf(tot);
        float Dv = ZUw * expf(M - L);
        for (int n = 0; n < nsel; ++n) Dv += expf(sm.sh[h][n] - L) * sm.ub[h][n];
        Lr[h] = L;
        Dr[h] = Dv;
    }

    // ---- pass 2: p, ds; dq with lane l owning dims l*DL .. l*DL+DL-1
    float dq[GM][DL], dqs[GM][DL];
#pragma unroll
    for (int h = 0; h < GM; ++h)
#pragma unroll
        for (int r = 0; r < DL; ++r) dq[h][r] = dqs[h][r] = 0.f;
    // contributions of tokens j0 + t (t < cnt, lane = token) with ds[h]
    auto accumulate = [&](int64_t j0, int cnt, const float *ds) {
        for (int tt = 0; tt < cnt; ++tt) {
            const T *kr = Kg + (j0 + tt) * D + lane * DL;
            float kv[DL];
#pragma unroll
            for (int r = 0; r < DL; ++r) kv[r] = ld_f(kr + r);
#pragma unroll
            for (int h = 0; h < GM; ++h) {
                if (h >= G) break;
                const float dsv = __shfl_sync(0xffffffffu, ds[h], tt);
#pragma unroll
                for (int r = 0; r < DL; ++r) dq[h][r] = fmaf(dsv, kv[r], dq[h][r]);
            }
        }
    };
    float ds[GM];
    for (int n = 0; n < nsel; ++n) {
        const int64_t j0 = (int64_t)sm.chunk[n] * p.S;
        for (int t0 = 0; t0 < p.S; t0 += 32) {
            const int t = t0 + lane;
            const int cnt = min(32, p.S - t0);
#pragma unroll
            for (int h = 0; h < GM; ++h) ds[h] = 0.f;
            if (t < p.S) {
                token_dots<T, D, GM>(sm, G, Kg + (j0 + t) * D, Vg + (j0 + t) * D, s, u);
#pragma unroll
                for (int h = 0; h < GM; ++h) {
                    if (h >= G) break;
                    const float P = expf(sm.sh[h][n] - Lr[h]);
                    const float pj = P * expf(s[h] * isd - sm.lz[h][n]);
                    ds[h] = pj * (u[h] - sm.ub[h][n]);
                }
            }
            accumulate(j0 + t0, cnt, ds);
        }
        // s^ gradient: dsh = P (Ubar - D) -> dqs += dsh k'_c
        const T *kl = Lg + (int64_t)sm.chunk[n] * D + lane * DL;
#pragma unroll
        for (int h = 0; h < GM; ++h) {
            if (h >= G) break;
            const float P = expf(sm.sh[h][n] - Lr[h]);
            const float dsh = P * (sm.ub[h][n] - Dr[h]);
#pragma unroll
            for (int r = 0; r < DL; ++r) dqs[h][r] = fmaf(dsh, ld_f(kl + r), dqs[h][r]);
        }
    }
    for (int64_t t0 = 0; t0 < nw; t0 += 32) {
        const int64_t t = t0 + lane;
        const int cnt = (int)min((int64_t)32, nw - t0);
#pragma unroll
        for (int h = 0; h < GM; ++h) ds[h] = 0.f;
        if (t < nw) {
            const int64_t j = w0 + t;
            token_dots<T, D, GM>(sm, G, Kg + j * D, Vg + j * D, s, u);
#pragma unroll
            for (int h = 0; h < GM; ++h) {
                if (h >= G) break;
                const float pj = expf(s[h] * isd - Lr[h]);
                ds[h] = pj * (u[h] - Dr[h]);
            }
        }
        accumulate(w0 + t0, cnt, ds);
    }

    // ---- outputs
    for (int h = 0; h < G; ++h) {
        const int hq = p.group_heads[g * G + h];
        const int64_t rq = ((int64_t)b * p.Hq + hq) * p.N + i;
        float *dq_out = p.dQ + rq * D + lane * DL;
#pragma unroll
        for (int r = 0; r < DL; ++r) {
            float v = dq[h][r] * isd;
            if (!p.dQs) v += dqs[h][r] * isd;
            dq_out[r] = v;
        }
        if (p.dQs) {
            float *o = p.dQs + rq * D + lane * DL;
#pragma unroll
            for (int r = 0; r < DL; ++r) o[r] = dqs[h][r] * isd;
        }
        if (lane == 0) {
            p.rowstat[rq * 2] = Lr[h];
            p.rowstat[rq * 2 + 1] = Dr[h];
        }
        for (int n = lane; n < nsel; n += 32) {
            // chunk tokens: p_j = exp(s_j - a), a = lz_c - s^_c + L
            float *cs = p.chunkstat + (rq * p.K + sm.kpos[n]) * 4;
            const float P = expf(sm.sh[h][n] - Lr[h]);
            cs[0] = sm.lz[h][n] - sm.sh[h][n] + Lr[h];
            cs[1] = sm.ub[h][n];
            cs[2] = P * (sm.ub[h][n] - Dr[h]);
        }
    }
}

// ------------------------------------------------------------------ keys
constexpr int kKeyBatch = 16;                    // (row, head) pairs per round
constexpr int kKeySplit = 8;                     // threads per token

// A pair's q / dO / qs row is stored as kKeySplit slices of D/kKeySplit
// floats, each padded by 4: the 8 threads of a token read their slices as
// float4 from 8 disjoint bank groups (slice stride 80 or 48 bytes).
template <int D>
constexpr int kSlice = D / kKeySplit + 4;

template <int D, int GM>
struct KeySmem {
    float q[kKeyBatch][kKeySplit][kSlice<D>], go[kKeyBatch][kKeySplit][kSlice<D>],
          qs[kKeyBatch][kKeySplit][kSlice<D>];
    // per pair: chunk role (a, Ubar), window role (L, D); the row's token
    // range inside the chunk; dsh = P (Ubar - D) (chunk role)
    float a0[kKeyBatch], a1[kKeyBatch], dsh[kKeyBatch];
    int lo[kKeyBatch], hi[kKeyBatch];
    float dklm[D];
    float dbias;
    int list_i[1024], list_k[1024];              // rows of this round
    int nlist;
    int scan[33];
};

template <typename T, int D, int S_TOK, int GM>
__global__ void __launch_bounds__(S_TOK * kKeySplit)
bwd_keys_kernel(const BwdParams p) {
    constexpr int DQ = D / kKeySplit;            // dims per thread
    constexpr int NT = S_TOK * kKeySplit;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    KeySmem<D, GM> &sm = *reinterpret_cast<KeySmem<D, GM> *>(smem_raw);
    // one CTA per block of S_TOK tokens; a chunk of p.S = m * S_TOK tokens
    // spans m blocks, and only its first block sums dk' and db'
    const int nblocks = (p.N + S_TOK - 1) / S_TOK;
    const int blk = blockIdx.x % nblocks;
    const int g = (blockIdx.x / nblocks) % p.Hkv;
    const int b = blockIdx.x / (nblocks * p.Hkv);
    const int c = blk / (p.S / S_TOK);           // the chunk holding the block
    const bool first_blk = blk % (p.S / S_TOK) == 0;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int jl = tid / kKeySplit, qd = tid % kKeySplit;
    const int64_t j = (int64_t)blk * S_TOK + jl; // this thread's token
    const bool jok = j < p.N;
    const int G = p.G;
    const float isd = p.inv_sqrt_d;
    const int64_t bg = (int64_t)b * p.Hkv + g;
    float kreg[DQ], vreg[DQ], adk[DQ], adv[DQ];
    {
        const T *kr = reinterpret_cast<const T *>(p.Kc) + (bg * p.N + (jok ? j : 0)) * D + qd * DQ;
        const T *vr = reinterpret_cast<const T *>(p.Vc) + (bg * p.N + (jok ? j : 0)) * D + qd * DQ;
#pragma unroll
        for (int r = 0; r < DQ; ++r) {
            kreg[r] = jok ? ld_f(kr + r) : 0.f;
            vreg[r] = jok ? ld_f(vr + r) : 0.f;
            adk[r] = adv[r] = 0.f;
        }
    }
    for (int k = tid; k < D; k += NT) sm.dklm[k] = 0.f;
    if (tid == 0) sm.dbias = 0.f;
    const T *Qp = reinterpret_cast<const T *>(p.Q);
    const T *Qsp = reinterpret_cast<const T *>(p.Qs ? p.Qs : p.Q);
    const T *dOp = reinterpret_cast<const T *>(p.dO);
    const bool is_lm = c < p.nC;                 // a complete chunk: selectable
    const bool own_lm = is_lm && first_blk;      // this CTA writes dk'_c, db'_c

    // process the (row, head) pairs of rows list_i[0..nlist) in batches
    auto run_rows = [&](int role) {
        const int npairs = sm.nlist * G;
        for (int e0 = 0; e0 < npairs; e0 += kKeyBatch) {
            const int ne = min(kKeyBatch, npairs - e0);
            __syncthreads();                     // previous batch consumed
            for (int e = warp; e < ne; e += NT / 32) {
                const int pr = e0 + e;
                const int ri = sm.list_i[pr / G], h = pr % G;
                const int hq = p.group_heads[g * G + h];
                const int64_t rq = ((int64_t)b * p.Hq + hq) * p.N + ri;
                for (int k = lane; k < D; k += 32) {
                    sm.q[e][k / DQ][k % DQ] = ld_f(Qp + rq * D + k);
                    sm.go[e][k / DQ][k % DQ] = ld_f(dOp + rq * D + k);
                    if (role == 0) sm.qs[e][k / DQ][k % DQ] = ld_f(Qsp + rq * D + k);
                }
                if (lane == 0) {
                    if (role == 0) {             // a, Ubar and dsh of the row
                        const float *cs = p.chunkstat + (rq * p.K + sm.list_k[pr / G]) * 4;
                        sm.a0[e] = cs[0];
                        sm.a1[e] = cs[1];
                        sm.dsh[e] = cs[2];
                        sm.lo[e] = 0;
                        sm.hi[e] = S_TOK - 1;
                    } else {                     // L, D and the window's span
                        sm.a0[e] = p.rowstat[rq * 2];
                        sm.a1[e] = p.rowstat[rq * 2 + 1];
                        int64_t w0, nc;
                        bwd_bounds(ri, p.S, p.W, &w0, &nc);
                        const int64_t base = (int64_t)blk * S_TOK;
                        sm.lo[e] = (int)max((int64_t)0, w0 - base);
                        sm.hi[e] = (int)min((int64_t)S_TOK - 1, (int64_t)ri - base);
                    }
                }
            }
            __syncthreads();
            for (int e = 0; e < ne; ++e) {       // fixed order: deterministic
                const float4 *q4p = reinterpret_cast<const float4 *>(&sm.q[e][qd][0]);
                const float4 *g4p = reinterpret_cast<const float4 *>(&sm.go[e][qd][0]);
                float4 q4[DQ / 4], g4[DQ / 4];
#pragma unroll
                for (int r = 0; r < DQ / 4; ++r) { q4[r] = q4p[r]; g4[r] = g4p[r]; }
                float sp = 0.f, up = 0.f;
#pragma unroll
                for (int r = 0; r < DQ / 4; ++r) {
                    const float4 a = q4[r], c4 = g4[r];
                    sp = fmaf(a.x, kreg[4 * r], sp);
                    sp = fmaf(a.y, kreg[4 * r + 1], sp);
                    sp = fmaf(a.z, kreg[4 * r + 2], sp);
                    sp = fmaf(a.w, kreg[4 * r + 3], sp);
                    up = fmaf(c4.x, vreg[4 * r], up);
                    up = fmaf(c4.y, vreg[4 * r + 1], up);
                    up = fmaf(c4.z, vreg[4 * r + 2], up);
                    up = fmaf(c4.w, vreg[4 * r + 3], up);
                }
#pragma unroll
                for (int o = 1; o < kKeySplit; o <<= 1) {   // the token's threads
                    sp += __shfl_xor_sync(0xffffffffu, sp, o);
                    up += __shfl_xor_sync(0xffffffffu, up, o);
                }
                const float x = sp * isd;
                float pj = 0.f, dsj = 0.f;
                if (jok && jl >= sm.lo[e] && jl <= sm.hi[e]) {
                    if (role == 0) {
                        pj = expf(x - sm.a0[e]);
                        dsj = pj * (up - sm.a1[e]);
                    } else {
                        pj = expf(x - sm.a0[e]);
                        dsj = pj * (up - sm.a1[e]);
                    }
                }
#pragma unroll
                for (int r = 0; r < DQ / 4; ++r) {
                    const float4 a = q4[r], c4 = g4[r];
                    adv[4 * r] = fmaf(pj, c4.x, adv[4 * r]);
                    adv[4 * r + 1] = fmaf(pj, c4.y, adv[4 * r + 1]);
                    adv[4 * r + 2] = fmaf(pj, c4.z, adv[4 * r + 2]);
                    adv[4 * r + 3] = fmaf(pj, c4.w, adv[4 * r + 3]);
                    adk[4 * r] = fmaf(dsj, a.x, adk[4 * r]);
                    adk[4 * r + 1] = fmaf(dsj, a.y, adk[4 * r + 1]);
                    adk[4 * r + 2] = fmaf(dsj, a.z, adk[4 * r + 2]);
                    adk[4 * r + 3] = fmaf(dsj, a.w, adk[4 * r + 3]);
                }
            }
            if (role == 0 && own_lm) {           // k' and b' of the chunk
                for (int k = tid; k < D; k += NT) {
                    float a = sm.dklm[k];
                    for (int e = 0; e < ne; ++e) a = fmaf(sm.dsh[e], sm.qs[e][k / DQ][k % DQ], a);
                    sm.dklm[k] = a;
                }
                if (tid == NT - 1) {
                    float a = sm.dbias;
                    for (int e = 0; e < ne; ++e) a += sm.dsh[e];
                    sm.dbias = a;
                }
            }
        }
        __syncthreads();
    };

    // rows that selected chunk c: i >= (c+1) S + W - 1, scanned in rounds of
    // NT rows; each round's hits are compacted in ascending order
    if (is_lm) {
        const int64_t i_min = (int64_t)(c + 1) * p.S + p.W - 1;
        for (int64_t r0 = i_min; r0 < p.N; r0 += NT) {
            const int64_t ri = r0 + tid;
            int hitk = -1;
            if (ri < p.N) {
                const int32_t *ir = p.idx + (bg * p.N + ri) * p.K;
                for (int k = 0; k < p.K; ++k) {
                    const int v = ir[k];
                    if (v < 0 || v > c) break;
                    if (v == c) { hitk = k; break; }
                }
            }
            const unsigned m = __ballot_sync(0xffffffffu, hitk >= 0);
            __syncthreads();
            if (lane == 0) sm.scan[warp] = __popc(m);
            __syncthreads();
            if (tid == 0) {
                int acc = 0;
                for (int w = 0; w < NT / 32; ++w) { const int v = sm.scan[w]; sm.scan[w] = acc; acc += v; }
                sm.nlist = acc;
            }
            __syncthreads();
            if (hitk >= 0) {
                const int pos = sm.scan[warp] + __popc(m & ((1u << lane) - 1u));
                sm.list_i[pos] = (int)ri;
                sm.list_k[pos] = hitk;
            }
            __syncthreads();
            if (sm.nlist > 0) run_rows(0);
        }
    }
    // rows whose window covers part of the block: i in [base, ...] with
    // w0 <= base + S_TOK - 1
    {
        const int64_t base = (int64_t)blk * S_TOK;
        for (int64_t r0 = base; r0 < p.N; r0 += 1024) {
            __syncthreads();
            if (tid == 0) {
                int n = 0;
                for (int64_t ri = r0; ri < min((int64_t)p.N, r0 + 1024); ++ri) {
                    int64_t w0, nc;
                    bwd_bounds(ri, p.S, p.W, &w0, &nc);
                    if (w0 > base + S_TOK - 1) break;
                    sm.list_i[n] = (int)ri;
                    sm.list_k[n] = 0;
                    ++n;
                }
                sm.nlist = n;
            }
            __syncthreads();
            const int n = sm.nlist;
            if (n > 0) run_rows(1);
            if (n < 1024) break;
        }
    }

    if (jok) {
        float *dk = p.dK + (bg * p.N + j) * D + qd * DQ;
        float *dv = p.dV + (bg * p.N + j) * D + qd * DQ;
#pragma unroll
        for (int r = 0; r < DQ; ++r) {
            dk[r] = adk[r] * isd;
            dv[r] = adv[r];
        }
    }
    __syncthreads();
    if (own_lm) {
        for (int k = tid; k < D; k += NT) p.dKlm[(bg * p.nC + c) * D + k] = sm.dklm[k] * isd;
        if (tid == 0) p.dbias[bg * p.nC + c] = sm.dbias;
    }
}

template <typename T, int D, int GM>
cudaError_t launch_rows_t(const BwdParams &p, cudaStream_t st) {
    const size_t smem = sizeof(RowSmem<D, GM>) * kRowWarps;
    cudaError_t e = cudaFuncSetAttribute(bwd_rows_kernel<T, D, GM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)p.B * p.Hkv * p.N;
    bwd_rows_kernel<T, D, GM><<<(unsigned)((rows + kRowWarps - 1) / kRowWarps),
                                kRowWarps * 32, smem, st>>>(p);
    return cudaGetLastError();
}

template <typename T, int D, int GM>
cudaError_t launch_keys_t(const BwdParams &p, cudaStream_t st) {
    constexpr int S_TOK = 64;
    const size_t smem = sizeof(KeySmem<D, GM>);
    cudaError_t e = cudaFuncSetAttribute(bwd_keys_kernel<T, D, S_TOK, GM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)p.B * p.Hkv * ((p.N + S_TOK - 1) / S_TOK);
    bwd_keys_kernel<T, D, S_TOK, GM><<<(unsigned)grid, S_TOK * kKeySplit, smem, st>>>(p);
    return cudaGetLastError();
}

template <typename T, int D, int GM>
cudaError_t launch_bwd_t(const BwdParams &p, cudaStream_t st) {
    cudaError_t e = launch_rows_t<T, D, GM>(p, st);
    if (e != cudaSuccess) return e;
    return launch_keys_t<T, D, GM>(p, st);
}

template <typename T, int D>
cudaError_t launch_rows_d(const BwdParams &p, cudaStream_t st) {
    if (p.G == 1) return launch_rows_t<T, D, 1>(p, st);
    if (p.G == 2) return launch_rows_t<T, D, 2>(p, st);
    if (p.G <= 4) return launch_rows_t<T, D, 4>(p, st);
    return launch_rows_t<T, D, 8>(p, st);
}

template <typename T, int D>
cudaError_t launch_bwd_d(const BwdParams &p, cudaStream_t st) {
    if (p.G == 1) return launch_bwd_t<T, D, 1>(p, st);
    if (p.G == 2) return launch_bwd_t<T, D, 2>(p, st);
    if (p.G <= 4) return launch_bwd_t<T, D, 4>(p, st);
    return launch_bwd_t<T, D, 8>(p, st);
}

bool al16b(const void *q) { return ((uintptr_t)q & 15u) == 0; }

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

// bf16 problems whose key side runs on the tensor cores
bool keys_tc_ok(const hils_backward_args *a, int G, int nC) {
    if (a->dtype != HILS_BF16 || !(a->d == 64 || a->d == 128)) return false;
    if (!(a->S == 64 || a->S == 128) || G > 8 || a->K > 64) return false;
    if (a->N >= (1 << 25) || (size_t)nC * sizeof(int) > 200 * 1024) return false;
    if ((int64_t)a->B * a->Hq * a->N >= (1ll << 31)) return false;
    // the key side's grid is an upper bound on its work units
    if (bwd_keys_max_units(a->B, a->Hkv, a->N, a->S, a->W, a->K, G) >= (1ll << 31))
        return false;
    if (bwd_keys_tc_smem(a->d, a->Qs != nullptr) > 227 * 1024) return false;
    return tc_maps_available();
}

// Shape checks of a backward record; fills p (pointers only when need_ptrs).
hils_status bwd_problem(const hils_backward_args *a, BwdParams *p, bool need_ptrs,
                        size_t *ws_bytes) {
    if (!a) return HILS_ERR_INVALID_ARG;
    if (a->dtype != HILS_F32 && a->dtype != HILS_BF16) return HILS_ERR_INVALID_ARG;
    if (a->B < 1 || a->Hq < 1 || a->Hkv < 1 || a->N < 1 || a->d < 1 || a->S < 1 ||
        a->W < 1 || a->K < 1 || !a->head_map)
        return HILS_ERR_INVALID_ARG;
    if (a->Hq % a->Hkv) return HILS_ERR_INVALID_ARG;
    if (a->K > HILS_MAX_TOPK || a->Hq > kMaxHeads) return HILS_ERR_UNSUPPORTED;
    const int G = a->Hq / a->Hkv;
    if (G > 8 || !(a->d == 64 || a->d == 128) || !(a->S == 64 || a->S == 128))
        return HILS_ERR_UNSUPPORTED;
    if ((int64_t)a->B * a->Hq * a->N * a->d >= (1ll << 40)) return HILS_ERR_UNSUPPORTED;
    int count[kMaxHeads];
    for (int g = 0; g < a->Hkv; ++g) count[g] = 0;
    for (int h = 0; h < a->Hq; ++h) {
        const int g = a->head_map[h];
        if (g < 0 || g >= a->Hkv || count[g] >= G) return HILS_ERR_INVALID_ARG;
        p->group_heads[g * G + count[g]] = (int16_t)h;
        count[g]++;
    }
    p->B = a->B; p->Hq = a->Hq; p->Hkv = a->Hkv; p->G = G; p->N = a->N;
    p->S = a->S; p->W = a->W; p->K = a->K; p->nC = a->N / a->S;
    p->inv_sqrt_d = (float)(1.0 / sqrt((double)a->d));
    const size_t rows = (size_t)a->B * a->Hq * a->N;
    // rowstat, chunkstat, then (tensor-core key side) the inverse index
    size_t need = round256(rows * 2 * sizeof(float)) +
                  round256(rows * (size_t)a->K * 4 * sizeof(float));
    const bool tc = keys_tc_ok(a, G, a->N / a->S);
    BwdIndexParams ip{};
    int64_t max_units = 0, nbt = 0;
    if (tc) {
        bwd_index_shape(a->N, a->N / a->S, &ip);
        max_units = bwd_keys_max_units(a->B, a->Hkv, a->N, a->S, a->W, a->K, G);
        nbt = (int64_t)a->B * a->Hkv * ((a->N + 127) / 128);
        need += round256((size_t)a->B * a->Hkv * ip.off_stride * sizeof(int)) +
                round256((size_t)a->B * a->Hkv * a->N * a->K * sizeof(int32_t)) +
                round256((size_t)max_units * sizeof(int2)) +
                round256((size_t)nbt * 2 * sizeof(int) + sizeof(int)) +
                round256((size_t)max_units * bwd_keys_partial_floats(a->d) * sizeof(float));
    }
    if (ws_bytes) *ws_bytes = need;
    if (!need_ptrs) return HILS_OK;
    if (!a->Q || !a->Kc || !a->V || !a->dO || !a->idx || !a->dQ || !a->dK || !a->dV)
        return HILS_ERR_INVALID_ARG;
    if (p->nC > 0 && (!a->Klm || !a->bias || !a->dKlm || !a->dbias))
        return HILS_ERR_INVALID_ARG;
    if ((a->Qs != nullptr) != (a->dQs != nullptr)) return HILS_ERR_INVALID_ARG;
    if (!a->workspace) return HILS_ERR_INVALID_ARG;
    if (a->workspace_bytes < need) return HILS_ERR_WORKSPACE_TOO_SMALL;
    const void *ptrs[] = {a->Q, a->Qs, a->Kc, a->V, a->Klm, a->bias, a->dO, a->idx,
                          a->dQ, a->dQs, a->dK, a->dV, a->dKlm, a->dbias, a->workspace};
    for (const void *q : ptrs)
        if (q && !al16b(q)) return HILS_ERR_MISALIGNED;
    p->Q = a->Q; p->Qs = a->Qs; p->Kc = a->Kc; p->Vc = a->V; p->Klm = a->Klm;
    p->dO = a->dO; p->bias = a->bias; p->idx = a->idx;
    p->dQ = a->dQ; p->dQs = a->dQs; p->dK = a->dK; p->dV = a->dV;
    p->dKlm = a->dKlm; p->dbias = a->dbias;
    uint8_t *w = (uint8_t *)a->workspace;
    p->rowstat = (float *)w;
    w += round256(rows * 2 * sizeof(float));
    p->chunkstat = (float *)w;
    w += round256(rows * (size_t)a->K * 4 * sizeof(float));
    p->tc_keys = tc;
    if (tc) {
        p->csr_off = (int *)w;
        w += round256((size_t)a->B * a->Hkv * ip.off_stride * sizeof(int));
        p->csr_ent = (int32_t *)w;
        w += round256((size_t)a->B * a->Hkv * a->N * a->K * sizeof(int32_t));
        p->units = (int2 *)w;
        w += round256((size_t)max_units * sizeof(int2));
        p->nunits_blk = (int *)w;
        p->tickets = p->nunits_blk + nbt;
        p->n_units = p->tickets + nbt;
        w += round256((size_t)nbt * 2 * sizeof(int) + sizeof(int));
        p->partial = (float *)w;
        p->max_units = max_units;
    }
    p->status = a->status;
    return HILS_OK;
}

}  // namespace
}  // namespace hils

extern "C" hils_status hils_bwd_prefill_workspace_size(const hils_backward_args *a,
                                                       size_t *bytes) {
    using namespace hils;
    if (!bytes) return HILS_ERR_INVALID_ARG;
    BwdParams p;
    size_t n = 0;
    hils_status s = bwd_problem(a, &p, false, &n);
    if (s != HILS_OK) return s;
    *bytes = n;
    return HILS_OK;
}

extern "C" hils_status hils_bwd_prefill(const hils_backward_args *a, void *stream) {
    using namespace hils;
    BwdParams p;
    hils_status s = bwd_problem(a, &p, true, nullptr);
    if (s != HILS_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (p.tc_keys) {
        BwdRowsParams rp{};
        rp.Q = p.Q; rp.Qs = p.Qs; rp.Kc = p.Kc; rp.V = p.Vc; rp.dO = p.dO; rp.Klm = p.Klm;
        rp.bias = p.bias; rp.idx = p.idx; rp.rowstat = p.rowstat; rp.chunkstat = p.chunkstat;
        rp.dQ = p.dQ; rp.dQs = p.dQs; rp.status = p.status;
        rp.B = p.B; rp.Hq = p.Hq; rp.Hkv = p.Hkv; rp.G = p.G; rp.N = p.N; rp.d = a->d;
        rp.S = p.S; rp.W = p.W; rp.K = p.K; rp.nC = p.nC > 0 ? p.nC : 0;
        rp.M = 128 / p.G;
        const int64_t uc = (int64_t)rp.M * p.K;
        rp.ucap = (int)(uc < rp.nC ? uc : (rp.nC > 0 ? rp.nC : 1));
        rp.inv_sqrt_d = p.inv_sqrt_d;
        for (int k = 0; k < kMaxHeads; ++k) rp.group_heads[k] = p.group_heads[k];
        if (128 % p.G == 0 && bwd_rows_tc_smem(rp) <= 227 * 1024) {
            e = launch_bwd_rows_tc(rp, st);
        } else {
            e = a->d == 128 ? launch_rows_d<__nv_bfloat16, 128>(p, st)
                            : launch_rows_d<__nv_bfloat16, 64>(p, st);
            count_launches(1);
        }
        if (e != cudaSuccess) return HILS_ERR_CUDA;
        BwdIndexParams ip{};
        bwd_index_shape(p.N, p.nC, &ip);
        ip.idx = p.idx; ip.off = p.csr_off; ip.ent = p.csr_ent;
        ip.ent_stride = (int64_t)p.N * p.K;
        ip.BH = p.B * p.Hkv; ip.N = p.N; ip.S = p.S; ip.W = p.W; ip.K = p.K;
        if (p.nC > 0) {
            e = launch_bwd_index(ip, st);
            if (e != cudaSuccess) return HILS_ERR_CUDA;
        }
        BwdTcParams tp{};
        tp.Q = p.Q; tp.Qs = p.Qs; tp.Kc = p.Kc; tp.V = p.Vc; tp.dO = p.dO;
        tp.rowstat = p.rowstat; tp.chunkstat = p.chunkstat;
        tp.off = p.csr_off; tp.ent = p.csr_ent;
        tp.dK = p.dK; tp.dV = p.dV; tp.dKlm = p.dKlm; tp.dbias = p.dbias;
        tp.status = p.status;
        tp.units = p.units; tp.nunits_blk = p.nunits_blk; tp.tickets = p.tickets;
        tp.n_units = p.n_units; tp.partial = p.partial; tp.max_units = p.max_units;
        tp.unit_batches = bwd_keys_unit_batches(p.B, p.Hkv, p.N, p.S, p.W, p.K, p.G);
        tp.off_stride = ip.off_stride; tp.ent_stride = ip.ent_stride;
        tp.B = p.B; tp.Hq = p.Hq; tp.Hkv = p.Hkv; tp.G = p.G; tp.N = p.N;
        tp.d = a->d; tp.S = p.S; tp.W = p.W; tp.K = p.K;
        tp.nC = p.nC > 0 ? p.nC : 0; tp.nseg = ip.nseg;
        tp.inv_sqrt_d = p.inv_sqrt_d;
        for (int k = 0; k < kMaxHeads; ++k) tp.group_heads[k] = p.group_heads[k];
        e = launch_bwd_keys_tc(tp, st);
        return e == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
    }
    if (a->dtype == HILS_BF16)
        e = a->d == 128 ? launch_bwd_d<__nv_bfloat16, 128>(p, st)
                        : launch_bwd_d<__nv_bfloat16, 64>(p, st);
    else
        e = a->d == 128 ? launch_bwd_d<float, 128>(p, st)
                        : launch_bwd_d<float, 64>(p, st);
    count_launches(2);
    return e == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
}
