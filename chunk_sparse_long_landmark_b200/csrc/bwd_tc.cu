// bwd_tc.cu -- key side of the prefill backward on the sm_100a tensor cores
// (bf16 inputs), and the inverse index (chunk -> rows that selected it) it
// walks.
//
// "Hierarchical Sparse Attention Done Right", Sec. 3 (RQ2: the fused
// chunk-level softmax carries the loss to the landmark scores) and Sec. 4
// (native sparse training). With the per-(row, head) statistics of the row
// side -- L, D, and for each selected chunk a = lz_c - s^_c + L, Ubar_c and
// dsh_c = P_c (Ubar_c - D) -- every (row, head) pair that reads a token j
// contributes
//   p_j = exp(s_j - a),  ds_j = p_j (u_j - delta),  s_j = q.k_j/sqrt(d),
//   u_j = dO.v_j         (chunk role: a, delta = Ubar_c; window role:
//                         a = L, delta = D)
//   dV_j += p_j dO,  dK_j += ds_j q / sqrt(d),
//   dk'_c += dsh_c qs / sqrt(d),  db'_c += dsh_c   (chunk role only).
//
// One CTA owns 128 consecutive tokens of one kv group (TMEM lane = token):
// one 128-token chunk, or two 64-token chunks. Its pairs are the rows that
// selected one of its chunks (from the inverse index, one column per (row,
// chunk)) and the rows whose window reaches into the block, times the G
// heads, taken 64 pairs per batch. Per batch:
//   S^T = K_blk Q_g^T, U^T = V_blk dO_g^T   tcgen05.mma 128 x 64, K = d
//   P^T, dS^T (bf16, in place over S^T / U^T)  by the softmax warps
//   dV += P^T dO_g, dK += dS^T Q_g          tcgen05.mma 128 x d, A from TMEM
// dV and dK stay in TMEM for the whole CTA; S^T / U^T are double buffered.
// Q_g, dO_g (and Qs_g under query calibration) are gathered row by row with
// cp.async into 128-byte-swizzled stages (the same layout TMA writes), the
// pairs' statistics with them. dk' and db' are summed by the softmax warps
// from the gathered rows, in a fixed order.
// A block whose pairs fill more than unit_batches batches (a chunk that most
// rows select) is cut into work units of that many batches, one CTA each:
// they write partial sums, and the last unit to finish (an integer ticket)
// adds them in unit order.
// Warp roles: warps 0-1 gather producers (32 pairs of each batch apiece;
// thread 0 also issues the one-time TMA of the K / V block), warps 2-5
// softmax and epilogue, warp 6 MMA issuer and TMEM owner.
// Every wait is bounded; a lost arrival ends the kernel with
// HILS_ERR_DEVICE_TIMEOUT in the status word. No floating-point atomics:
// each output element is summed in one fixed order.
//
// Inverse index: entries (row << 6 | topk slot) of every valid selection,
// grouped by chunk. Rows are cut into segments; a histogram per (segment,
// chunk), an exclusive scan over [chunk][segment], and a fill in which one
// warp per segment walks its rows in order give every entry a position that
// depends only on the input.
#include <math.h>

#include "hils_fast.cuh"
#include "sm100.cuh"
#include "tc_kernels.cuh"

namespace hils {

namespace {

using namespace sm100;

constexpr int kProd = 2;          // gather producer warps of the key kernel
constexpr int kKT = 32 * (kProd + 4 + 1);   // + 4 softmax warps + the MMA warp
constexpr int kBlk = 128;         // tokens per CTA
constexpr int kNP = 64;           // pairs per batch
constexpr int kUnitMin = 8, kUnitMax = 256;   // batches per work unit
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------ inverse index
__global__ void bwd_hist_kernel(const BwdIndexParams p) {
    extern __shared__ int hist[];
    const int seg = blockIdx.x % p.nseg;
    const int bg = blockIdx.x / p.nseg;
    for (int c = threadIdx.x; c < p.nC; c += blockDim.x) hist[c] = 0;
    __syncthreads();
    const int64_t r0 = (int64_t)seg * p.R;
    const int64_t r1 = min((int64_t)p.N, r0 + p.R);
    for (int64_t i = r0 + threadIdx.x; i < r1; i += blockDim.x) {
        int64_t w0, nc;
        window_bounds(i, p.S, p.W, &w0, &nc);
        const int32_t *ir = p.idx + ((int64_t)bg * p.N + i) * p.K;
        for (int k = 0; k < p.K; ++k) {
            const int c = __ldg(ir + k);
            if (c >= 0 && c < nc) atomicAdd(&hist[c], 1);
        }
    }
    __syncthreads();
    int *out = p.off + (int64_t)bg * p.off_stride;
    for (int c = threadIdx.x; c < p.nC; c += blockDim.x)
        out[(int64_t)c * p.nseg + seg] = hist[c];
}

// Exclusive scan of one (b, g)'s [nC][nseg] counts, in place; the total goes
// to position nC * nseg. Tiles of 4 * 1024 values, a running carry.
__global__ void __launch_bounds__(1024) bwd_scan_kernel(const BwdIndexParams p) {
    __shared__ int wsum[32];
    __shared__ int carry_s;
    int *a = p.off + (int64_t)blockIdx.x * p.off_stride;
    const int64_t n = (int64_t)p.nC * p.nseg;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry_s = 0;
    __syncthreads();
    for (int64_t t0 = 0; t0 < n; t0 += 4 * 1024) {
        const int64_t e = t0 + 4 * threadIdx.x;
        int v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] = (e + q < n) ? a[e + q] : 0;
        const int tot = v[0] + v[1] + v[2] + v[3];
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int x = wsum[lane];
            int wi = x;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += y;
            }
            wsum[lane] = wi - x;                 // exclusive over warps
        }
        __syncthreads();
        int run = carry_s + wsum[warp] + incl - tot;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (e + q < n) a[e + q] = run;
            run += v[q];
        }
        __syncthreads();
        if (threadIdx.x == 1023) carry_s = run;  // the last thread ends the tile
        __syncthreads();
    }
    if (threadIdx.x == 0) a[n] = carry_s;
}

// One warp per (b, g, segment): rows in ascending order, 32 at a time, the
// top-K slots in order; lanes that hit the same chunk in the same slot take
// consecutive positions in lane order.
__global__ void __launch_bounds__(32) bwd_fill_kernel(const BwdIndexParams p) {
    extern __shared__ int cur[];
    const int seg = blockIdx.x % p.nseg;
    const int bg = blockIdx.x / p.nseg;
    const int lane = threadIdx.x;
    const int *off = p.off + (int64_t)bg * p.off_stride;
    for (int c = lane; c < p.nC; c += 32) cur[c] = off[(int64_t)c * p.nseg + seg];
    __syncwarp();
    int32_t *ent = p.ent + (int64_t)bg * p.ent_stride;
    const int64_t r0 = (int64_t)seg * p.R;
    const int64_t r1 = min((int64_t)p.N, r0 + p.R);
    const unsigned lt = (1u << lane) - 1u;
    for (int64_t i0 = r0; i0 < r1; i0 += 32) {
        const int64_t i = i0 + lane;
        int64_t nc = 0;
        if (i < r1) {
            int64_t w0;
            window_bounds(i, p.S, p.W, &w0, &nc);
        }
        const int32_t *ir = p.idx + ((int64_t)bg * p.N + (i < r1 ? i : r0)) * p.K;
        for (int k = 0; k < p.K; ++k) {
            const int c = (i < r1) ? __ldg(ir + k) : -1;
            const bool ok = c >= 0 && c < nc;
            const unsigned peers = __match_any_sync(0xffffffffu, ok ? c : -1 - lane);
            int base = 0;
            if (ok) base = cur[c];
            __syncwarp();
            if (ok) {
                ent[base + __popc(peers & lt)] = (int32_t)((i << 6) | k);
                if ((peers & lt) == 0) cur[c] = base + __popc(peers);
            }
            __syncwarp();
        }
    }
}

// ------------------------------------------------------------- key kernel
// Pairs of one key block: the index entries of its chunks, then its window
// rows (rows i >= base whose window start is at most base + 127), G heads
// each, in that order.
struct BlockWork {
    int cstart[2], ccount[2];
    int nlist, nwin;
    int npairs;
};

__device__ __forceinline__ BlockWork block_work(const int *off, int64_t off_stride,
                                                int nseg, int nC, int S, int W,
                                                int N, int G, int bg, int blk) {
    BlockWork w;
    const int cpb = kBlk / S;
    const int *o = off + (int64_t)bg * off_stride;
    w.cstart[0] = w.cstart[1] = w.ccount[0] = w.ccount[1] = 0;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const int c = blk * cpb + q;
        if (q < cpb && c < nC) {
            w.cstart[q] = __ldg(o + (int64_t)c * nseg);
            w.ccount[q] = __ldg(o + (int64_t)(c + 1) * nseg) - w.cstart[q];
        }
    }
    const int base = blk * kBlk;
    w.nlist = w.ccount[0] + w.ccount[1];
    w.nwin = min(N - 1, base + kBlk + W - 2) - base + 1;
    w.npairs = (w.nlist + w.nwin) * G;
    return w;
}

// Work units: a key block whose pairs fill more than unit_batches batches is
// cut into units of unit_batches; units of one block are consecutive. One
// CTA, blocks in order.
__global__ void __launch_bounds__(1024) bwd_plan_kernel(const BwdTcParams p) {
    __shared__ int wsum[32];
    __shared__ int carry_s;
    const int nblk = (p.N + kBlk - 1) / kBlk;
    const int nbt = p.B * p.Hkv * nblk;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry_s = 0;
    __syncthreads();
    for (int t0 = 0; t0 < nbt; t0 += 1024) {
        const int gb = t0 + threadIdx.x;
        int n = 0;
        if (gb < nbt) {
            const BlockWork w = block_work(p.off, p.off_stride, p.nseg, p.nC, p.S, p.W,
                                           p.N, p.G, gb / nblk, gb % nblk);
            const int T = (w.npairs + kNP - 1) / kNP;
            n = max(1, (T + p.unit_batches - 1) / p.unit_batches);
            p.nunits_blk[gb] = n;
            p.tickets[gb] = 0;
        }
        int incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int x = wsum[lane];
            int wi = x;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += y;
            }
            wsum[lane] = wi - x;
        }
        __syncthreads();
        const int start = carry_s + wsum[warp] + incl - n;
        for (int k = 0; k < n && start + k < p.max_units; ++k)
            p.units[start + k] = make_int2(gb, k);
        __syncthreads();
        if (threadIdx.x == 1023) carry_s = start + n;
        __syncthreads();
    }
    if (threadIdx.x == 0) *p.n_units = (int)min((int64_t)carry_s, p.max_units);
}

template <int D, bool QCAL>
struct KeyLayout {
    static constexpr int NSTG = (QCAL && D == 128) ? 3 : 4;   // gather stages
    static constexpr uint32_t KV_BYTES = kBlk * D * 2;       // K or V block
    static constexpr uint32_t ROWS_BYTES = kNP * D * 2;      // one gathered array
    static constexpr int NARR = QCAL ? 3 : 2;                // Q, dO (, Qs)
    static constexpr uint32_t STG_BYTES = NARR * ROWS_BYTES;
    static constexpr uint32_t OFF_K = 0;
    static constexpr uint32_t OFF_V = KV_BYTES;
    static constexpr uint32_t OFF_STG = 2 * KV_BYTES;
    static constexpr uint32_t OFF_SMALL = OFF_STG + NSTG * STG_BYTES;
    // TMEM: dV [0, D), dK [D, 2D), S^T / U^T buffer sb at BUF + 128 sb
    static constexpr int TM_DV = 0, TM_DK = D, TM_BUF = 2 * D;
    static constexpr uint32_t TMEM_COLS = 512u;
    static constexpr int TPD = D / 2;                        // threads per pair range
    static constexpr int NPH = 128 / TPD;                    // pair ranges
    static_assert(2 * D + 256 <= 512, "TMEM budget");
};

template <int D, int NSTG>
struct KeySmall {
    uint64_t kv_full;
    uint64_t full[NSTG];
    uint64_t empty[NSTG];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t buf_free[2];
    uint64_t acc_done;
    uint32_t tmem_base;
    int abort;
    int last;
    // per stage and pair: {a, delta, dsh, -} (cp.async), lo | len << 8
    float4 st4[NSTG][kNP];
    int meta[NSTG][kNP];
    float dkl[2][128 / (D / 2)][D];             // partial dk' per chunk and range
    float dbl[2][128 / (D / 2)];                // partial db' per chunk and range
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t n) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 :: "r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;"
                 :: "r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_wait1() {
    asm volatile("cp.async.wait_group 1;" ::: "memory");
}
__device__ __forceinline__ void cp_wait0() {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// floats of one unit's partial sums: dV, dK of the block, dk' and db' of its
// (up to) two chunks, padded to 16 bytes
template <int D>
constexpr int64_t kPartFloats = 2 * kBlk * D + 2 * D + 4;

template <int D, bool QCAL>
__global__ void __launch_bounds__(kKT, 1)
bwd_keys_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV,
                   const BwdTcParams p) {
    using L = KeyLayout<D, QCAL>;
    constexpr int NSTG = L::NSTG;
    // A batch is handed over once the next one is issued (LAG = 1): handing
    // it over later ties its start to the release of an older stage.
    constexpr int LAG = 1;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    KeySmall<D, NSTG> &st = *reinterpret_cast<KeySmall<D, NSTG> *>(smem + L::OFF_SMALL);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = blockIdx.x;
    if (unit >= __ldg(p.n_units)) return;            // the grid is an upper bound
    const int2 un = __ldg(&p.units[unit]);
    const int nblk = (p.N + kBlk - 1) / kBlk;
    const int gb = un.x, sub = un.y;
    const int blk = gb % nblk;
    const int g = (gb / nblk) % p.Hkv;
    const int b = gb / (nblk * p.Hkv);
    const int bg = b * p.Hkv + g;
    const int base = blk * kBlk;
    const int G = p.G;
    const int nun = __ldg(p.nunits_blk + gb);
    const int cpb = kBlk / p.S;                      // chunks per block: 1 or 2
    const BlockWork w = block_work(p.off, p.off_stride, p.nseg, p.nC, p.S, p.W, p.N, G, bg, blk);
    const int Tall = (w.npairs + kNP - 1) / kNP;
    const int t0 = sub * p.unit_batches;             // this unit's batches
    const int T = min(Tall - t0, p.unit_batches);
    volatile int *abort = &st.abort;

    if (threadIdx.x == 0) {
        mbar_init(&st.kv_full, 1);
        for (int s = 0; s < NSTG; ++s) {
            mbar_init(&st.full[s], 32 * kProd);
            mbar_init(&st.empty[s], 1 + 4);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&st.s_full[s], 1);
            mbar_init(&st.p_full[s], 4);            // one arrival per softmax warp
            mbar_init(&st.buf_free[s], 1);
        }
        mbar_init(&st.acc_done, 1);
        st.abort = (p.status && *(volatile int32_t *)p.status ==
                                    HILS_ERR_DEVICE_TIMEOUT) ? 1 : 0;
        st.last = 0;
        fence_barrier_init();
    }
    if (warp == kProd + 4) tmem_alloc(&st.tmem_base, L::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = st.tmem_base;
    const bool run = !st.abort && T > 0;

    if (warp < kProd) {
        // ----------------------------------------------------- producers
        // warp pw gathers pairs [32 pw, 32 pw + 32) of every batch; lane l
        // resolves pair 32 pw + l
        const int pw = warp;
        if (run && threadIdx.x == 0) {
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            mbar_expect_tx(&st.kv_full, 2 * L::KV_BYTES);
            for (int dh = 0; dh < D / 64; ++dh) {
                tma_load_4d(smem + L::OFF_K + dh * (kBlk * 128), &tmK, &st.kv_full,
                            dh * 64, base, g, b);
                tma_load_4d(smem + L::OFF_V + dh * (kBlk * 128), &tmV, &st.kv_full,
                            dh * 64, base, g, b);
            }
        }
        const __nv_bfloat16 *Qp = reinterpret_cast<const __nv_bfloat16 *>(p.Q);
        const __nv_bfloat16 *Op = reinterpret_cast<const __nv_bfloat16 *>(p.dO);
        const __nv_bfloat16 *Sp = reinterpret_cast<const __nv_bfloat16 *>(p.Qs);
        const int pr = pw * 32 + lane;
        const int32_t *ent = p.ent + (int64_t)bg * p.ent_stride;
        auto entry_of = [&](int t) -> int {          // index entry of pair pr of batch t
            const int e = (t0 + t) * kNP + pr;
            if (t >= T || e >= w.npairs) return -1;
            const int item = e / G;
            if (item >= w.nlist) return -1;
            return __ldg(ent + (item < w.ccount[0] ? w.cstart[0] + item
                                                   : w.cstart[1] + item - w.ccount[0]));
        };
        int ecur = run ? entry_of(0) : -1, enx = run ? entry_of(1) : -1;
        constexpr int UPR = D / 8;                   // 16-byte units per row
        constexpr int PPI = 32 / UPR;                // pairs per gather instruction
        int t = 0;
        for (; run && t < T; ++t) {
            const int s = t % NSTG;
            if (t >= NSTG &&
                !__all_sync(0xffffffffu, mbar_wait(&st.empty[s], ((t / NSTG) - 1) & 1, abort)))
                break;
            const int efar = entry_of(t + 2);
            int roff = -1;
            {
                const int e = (t0 + t) * kNP + pr;
                const uint32_t dst4 = smem_u32(&st.st4[s][pr]);
                int meta = 0;                        // len = 0: no token
                if (e < w.npairs) {
                    const int item = e / G;
                    const int hq = p.group_heads[g * G + (e - item * G)];
                    if (item < w.nlist) {
                        const int q = item < w.ccount[0] ? 0 : 1;
                        const int i = ecur >> 6, k = ecur & 63;
                        roff = (b * p.Hq + hq) * p.N + i;
                        cp_async16(dst4, p.chunkstat + ((int64_t)roff * p.K + k) * 4, 16);
                        meta = (cpb == 2 ? 64 * q : 0) | (p.S << 8);
                    } else {
                        const int i = base + item - w.nlist;
                        roff = (b * p.Hq + hq) * p.N + i;
                        cp_async8(dst4, p.rowstat + (int64_t)roff * 2);
                        st.st4[s][pr].z = 0.f;
                        // window start: max(floor((i - W + 1) / S) * S, 0)
                        const int x = i - p.W + 1;
                        const int w0 = x > 0 ? (x / p.S) * p.S : 0;
                        const int lo = max(w0 - base, 0);
                        const int hi = min(i - base, kBlk - 1);
                        meta = lo | ((hi - lo + 1) << 8);
                    }
                } else {
                    st.st4[s][pr] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                st.meta[s][pr] = meta;
            }
            uint8_t *stg = smem + L::OFF_STG + s * L::STG_BYTES;
#pragma unroll
            for (int arr = 0; arr < L::NARR; ++arr) {
                const __nv_bfloat16 *src = arr == 0 ? Qp : (arr == 1 ? Op : Sp);
#pragma unroll
                for (int j = 0; j < 32 / PPI; ++j) {
                    const int pl = j * PPI + lane / UPR;     // pair within the warp's 32
                    const int u = lane % UPR;
                    const int ro = __shfl_sync(0xffffffffu, roff, pl);
                    const int pp = pw * 32 + pl;
                    const uint32_t dst = smem_u32(stg + arr * L::ROWS_BYTES + (u >> 3) * (kNP * 128) +
                                                  pp * 128 + (((u & 7) ^ (pp & 7)) << 4));
                    cp_async16(dst, ro >= 0 ? (const void *)(src + (int64_t)ro * D + u * 8)
                                            : (const void *)src,
                               ro >= 0 ? 16u : 0u);
                }
            }
            cp_commit();
            // batch t - LAG's copies have landed: hand it to the MMA warp
            if (t >= LAG) {
                cp_wait1();
                fence_async_smem();
                mbar_arrive(&st.full[(t - LAG) % NSTG]);
            }
            ecur = enx;
            enx = efar;
        }
        cp_wait0();
        fence_async_smem();
        if (run && t == T)
            for (int u = max(T - LAG, 0); u < T; ++u) mbar_arrive(&st.full[u % NSTG]);
    } else if (warp == kProd + 4) {
        // ----------------------------------------------------- MMA issuer
        if (run && lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(kBlk, kNP, false);
            constexpr uint32_t id_g = idesc_bf16(kBlk, D, true);
            const uint32_t sK = smem_u32(smem + L::OFF_K);
            const uint32_t sV = smem_u32(smem + L::OFF_V);
            bool ok = mbar_wait(&st.kv_full, 0, abort);
            auto grad = [&](int u) -> bool {
                const int sb = u & 1, s = u % NSTG;
                if (!mbar_wait(&st.p_full[sb], (u >> 1) & 1, abort)) return false;
                tc_fence_after();
                const uint32_t stg = smem_u32(smem + L::OFF_STG + s * L::STG_BYTES);
#pragma unroll
                for (int kk = 0; kk < kNP / 16; ++kk) {
                    const uint32_t acc = (u > 0 || kk > 0) ? 1u : 0u;
                    const uint64_t bo = desc_sw128(stg + L::ROWS_BYTES + kk * 16 * 128,
                                                   kNP * 128, 1024);
                    mma_ts(tmem + L::TM_DV, tmem + L::TM_BUF + sb * 128 + kk * 8, bo, id_g, acc);
                    const uint64_t bq = desc_sw128(stg + kk * 16 * 128, kNP * 128, 1024);
                    mma_ts(tmem + L::TM_DK, tmem + L::TM_BUF + sb * 128 + 64 + kk * 8, bq, id_g, acc);
                }
                mma_commit(&st.buf_free[sb]);
                mma_commit(&st.empty[s]);
                return true;
            };
            for (int t = 0; ok && t < T; ++t) {
                const int s = t % NSTG, sb = t & 1;
                if (!mbar_wait(&st.full[s], (t / NSTG) & 1, abort)) { ok = false; break; }
                if (t >= 2 && !mbar_wait(&st.buf_free[sb], ((t >> 1) - 1) & 1, abort)) { ok = false; break; }
                tc_fence_after();
                const uint32_t stg = smem_u32(smem + L::OFF_STG + s * L::STG_BYTES);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ak = desc_sw128(sK + (kk / 4) * (kBlk * 128) + (kk % 4) * 32, 16, 1024);
                    const uint64_t bq = desc_sw128(stg + (kk / 4) * (kNP * 128) + (kk % 4) * 32, 16, 1024);
                    mma_ss(tmem + L::TM_BUF + sb * 128, ak, bq, id_s, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t av = desc_sw128(sV + (kk / 4) * (kBlk * 128) + (kk % 4) * 32, 16, 1024);
                    const uint64_t bo = desc_sw128(stg + L::ROWS_BYTES + (kk / 4) * (kNP * 128) + (kk % 4) * 32,
                                                   16, 1024);
                    mma_ss(tmem + L::TM_BUF + sb * 128 + 64, av, bo, id_s, kk > 0 ? 1u : 0u);
                }
                mma_commit(&st.s_full[sb]);
                if (t >= 1 && !grad(t - 1)) { ok = false; break; }
            }
            if (ok && T > 0) grad(T - 1);
            mma_commit(&st.acc_done);
            mbar_drain(&st.acc_done, 0);
        }
    } else {
        // -------------------------------------------- softmax / epilogue
        const int quad = warp & 3;
        const int tok = quad * 32 + lane;            // TMEM lane = token of the block
        const int et = threadIdx.x - 32 * kProd;     // 0..127
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        const float sl2 = p.inv_sqrt_d * kLog2e;
        // dk' ranges: thread et owns dims 2*(et % TPD) +{0,1} of pairs
        // [range * kNP/NPH, +kNP/NPH)
        const int dm = 2 * (et % L::TPD);
        const int rng = et / L::TPD;
        constexpr int PPR = kNP / L::NPH;
        float2 dk0 = make_float2(0.f, 0.f), dk1 = make_float2(0.f, 0.f);
        float db0 = 0.f, db1 = 0.f;
        bool ok = run;
        for (int t = 0; ok && t < T; ++t) {
            const int s = t % NSTG, sb = t & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&st.s_full[sb], (t >> 1) & 1, abort) &&
                                             mbar_wait(&st.full[s], (t / NSTG) & 1, abort))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tb = trow + L::TM_BUF + sb * 128;
            {
                // S^T and U^T of the 64 pairs in one TMEM round trip
                uint32_t sr[64], ur[64], pk[32], dk[32];
                tmem_ld32(tb, sr);
                tmem_ld32(tb + 32, sr + 32);
                tmem_ld32(tb + 64, ur);
                tmem_ld32(tb + 96, ur + 32);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int e0 = 2 * j;
                    const float4 A = st.st4[s][e0], B = st.st4[s][e0 + 1];
                    const int ma = st.meta[s][e0], mb = st.meta[s][e0 + 1];
                    const float2 x = f2_fma(make_float2(__uint_as_float(sr[2 * j]),
                                                        __uint_as_float(sr[2 * j + 1])),
                                            make_float2(sl2, sl2),
                                            make_float2(-A.x * kLog2e, -B.x * kLog2e));
                    const bool ina = (unsigned)(tok - (ma & 255)) < (unsigned)((ma >> 8) & 511);
                    const bool inb = (unsigned)(tok - (mb & 255)) < (unsigned)((mb >> 8) & 511);
                    const float2 pv = make_float2(ina ? fast_exp2(x.x) : 0.f,
                                                  inb ? fast_exp2(x.y) : 0.f);
                    const float2 du = f2_add(make_float2(__uint_as_float(ur[2 * j]),
                                                         __uint_as_float(ur[2 * j + 1])),
                                             make_float2(-A.y, -B.y));
                    const float2 ds = f2_mul(pv, du);
                    pk[j] = pack_bf16(pv.x, pv.y);
                    dk[j] = pack_bf16(ds.x, ds.y);
                }
                // P^T over S^T columns [0, 32), dS^T over U^T columns [0, 32)
                tmem_st32(tb, pk);
                tmem_st32(tb + 64, dk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&st.p_full[sb]);
            // dk' and db' of the chunk-role pairs of this thread's range, from
            // the gathered scoring rows. A batch holds, in order, pairs of the
            // block's first chunk, of its second chunk, then window pairs: the
            // two boundaries follow from the batch's first pair index.
            {
                const int eb = (t0 + t) * kNP;
                const int b0 = min(max(w.ccount[0] * G - eb, 0), kNP);
                const int b1 = min(max(w.nlist * G - eb, 0), kNP);
                const int lo = rng * PPR, hi = lo + PPR;
                const uint8_t *qs = smem + L::OFF_STG + s * L::STG_BYTES + (QCAL ? 2 : 0) * L::ROWS_BYTES +
                                    (dm >> 6) * (kNP * 128);
                const int byte = (dm & 63) * 2;
                auto acc = [&](int e, float2 &dk, float &db) {
                    const float dsh = st.st4[s][e].z;
                    const uint32_t wq = *reinterpret_cast<const uint32_t *>(
                        qs + e * 128 + ((((byte >> 4) ^ (e & 7)) << 4) | (byte & 15)));
                    dk.x = fmaf(dsh, __uint_as_float(wq << 16), dk.x);
                    dk.y = fmaf(dsh, __uint_as_float(wq & 0xffff0000u), dk.y);
                    db += dsh;
                };
#pragma unroll 4
                for (int e = lo; e < min(hi, b0); ++e) acc(e, dk0, db0);
#pragma unroll 4
                for (int e = max(lo, b0); e < min(hi, b1); ++e) acc(e, dk1, db1);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&st.empty[s]);
        }
        // dV, dK of the block's tokens once the last gradient MMA is done:
        // the final rows (dK scaled by 1/sqrt(d)), or this unit's partial sums
        if (ok && T > 0)
            ok = __all_sync(0xffffffffu, mbar_wait(&st.acc_done, 0, abort));
        if (ok) {
            tc_fence_after();
            const int j = base + tok;
            float *dv, *dkp;
            float ks = p.inv_sqrt_d;
            if (nun == 1) {
                dv = p.dV + ((int64_t)bg * p.N + (j < p.N ? j : 0)) * D;
                dkp = p.dK + ((int64_t)bg * p.N + (j < p.N ? j : 0)) * D;
            } else {
                float *part = p.partial + (int64_t)unit * kPartFloats<D>;
                dv = part + tok * D;
                dkp = part + kBlk * D + tok * D;
                ks = 1.f;
            }
            const bool wr = nun > 1 || j < p.N;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t rv[32], rk[32];
                tmem_ld32(trow + L::TM_DV + c0, rv);
                tmem_ld32(trow + L::TM_DK + c0, rk);
                tmem_wait_ld();
                if (wr) {
#pragma unroll
                    for (int q = 0; q < 32; q += 4) {
                        *reinterpret_cast<float4 *>(dv + c0 + q) = make_float4(
                            __uint_as_float(rv[q]), __uint_as_float(rv[q + 1]),
                            __uint_as_float(rv[q + 2]), __uint_as_float(rv[q + 3]));
                        *reinterpret_cast<float4 *>(dkp + c0 + q) = make_float4(
                            __uint_as_float(rk[q]) * ks, __uint_as_float(rk[q + 1]) * ks,
                            __uint_as_float(rk[q + 2]) * ks, __uint_as_float(rk[q + 3]) * ks);
                    }
                }
            }
        }
        st.dkl[0][rng][dm] = dk0.x;
        st.dkl[0][rng][dm + 1] = dk0.y;
        st.dkl[1][rng][dm] = dk1.x;
        st.dkl[1][rng][dm + 1] = dk1.y;
        if (dm == 0) { st.dbl[0][rng] = db0; st.dbl[1][rng] = db1; }
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kProd + 4) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
    if (*abort) {
        if (threadIdx.x == 0) report(p.status, HILS_ERR_DEVICE_TIMEOUT);
        return;
    }
    if (nun == 1) {
        // dk', db' of the block's complete chunks, ranges summed in order
        for (int x = threadIdx.x; x < cpb * D; x += kKT) {
            const int q = x / D, k = x % D;
            const int c = blk * cpb + q;
            if (c >= p.nC) continue;
            float a = 0.f, db = 0.f;
            for (int r = 0; r < L::NPH; ++r) { a += st.dkl[q][r][k]; db += st.dbl[q][r]; }
            p.dKlm[((int64_t)bg * p.nC + c) * D + k] = a * p.inv_sqrt_d;
            if (k == 0) p.dbias[(int64_t)bg * p.nC + c] = db;
        }
        return;
    }
    // a block cut into units: this unit's dk', db' partials, then the last
    // unit to finish sums every unit's partials in unit order
    {
        float *part = p.partial + (int64_t)unit * kPartFloats<D> + 2 * kBlk * D;
        for (int x = threadIdx.x; x < 2 * D; x += kKT) {
            const int q = x / D, k = x % D;
            float a = 0.f;
            for (int r = 0; r < L::NPH; ++r) a += st.dkl[q][r][k];
            part[x] = a;
        }
        if (threadIdx.x < 2) {
            float db = 0.f;
            for (int r = 0; r < L::NPH; ++r) db += st.dbl[threadIdx.x][r];
            part[2 * D + threadIdx.x] = db;
        }
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) st.last = atomicAdd(p.tickets + gb, 1) == nun - 1;
    __syncthreads();
    if (!st.last) return;
    __threadfence();
    const float *p0 = p.partial + (int64_t)(unit - sub) * kPartFloats<D>;
    for (int x = threadIdx.x; x < (2 * kBlk * D) / 4; x += kKT) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k = 0; k < nun; ++k) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(p0 + (int64_t)k * kPartFloats<D>) + x);
            a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
        }
        const int e = 4 * x;
        const bool is_k = e >= kBlk * D;
        const int r = (e % (kBlk * D)) / D, c = e % D;
        const int j = base + r;
        if (j >= p.N) continue;
        float *dst = (is_k ? p.dK : p.dV) + ((int64_t)bg * p.N + j) * D + c;
        const float s = is_k ? p.inv_sqrt_d : 1.f;
        *reinterpret_cast<float4 *>(dst) = make_float4(a.x * s, a.y * s, a.z * s, a.w * s);
    }
    for (int x = threadIdx.x; x < 2 * D + 2; x += kKT) {
        float a = 0.f;
        for (int k = 0; k < nun; ++k) a += __ldcg(p0 + (int64_t)k * kPartFloats<D> + 2 * kBlk * D + x);
        const int q = x < 2 * D ? x / D : x - 2 * D;
        const int c = blk * cpb + q;
        if (q >= cpb || c >= p.nC) continue;
        if (x < 2 * D) p.dKlm[((int64_t)bg * p.nC + c) * D + x % D] = a * p.inv_sqrt_d;
        else p.dbias[(int64_t)bg * p.nC + c] = a;
    }
}

// Shared memory of one CTA, at least 116 KB: two CTAs on one SM would
// contend for its 512 TMEM columns.
template <int D, bool QCAL>
constexpr size_t keys_smem() {
    return 1024 + KeyLayout<D, QCAL>::OFF_SMALL + sizeof(KeySmall<D, KeyLayout<D, QCAL>::NSTG>) <
                   116 * 1024
               ? 116 * 1024
               : 1024 + KeyLayout<D, QCAL>::OFF_SMALL + sizeof(KeySmall<D, KeyLayout<D, QCAL>::NSTG>);
}

template <int D, bool QCAL>
cudaError_t launch_keys_tc_t(const BwdTcParams &p, const CUtensorMap &mk,
                             const CUtensorMap &mv, cudaStream_t stream) {
    const size_t smem = keys_smem<D, QCAL>();
    auto kern = bwd_keys_tc_kernel<D, QCAL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)p.max_units, kKT, smem, stream>>>(mk, mv, p);
    return cudaGetLastError();
}


}  // namespace

void bwd_index_shape(int N, int nC, BwdIndexParams *ip) {
    int64_t r = (N + 127) / 128;
    r = ((r + 31) / 32) * 32;
    ip->R = (int)(r < 256 ? 256 : r);
    ip->nseg = (N + ip->R - 1) / ip->R;
    ip->nC = nC;
    ip->off_stride = (int64_t)nC * ip->nseg + 1;
}

size_t bwd_keys_tc_smem(int d, bool qcal) {
    if (d == 128) return qcal ? keys_smem<128, true>() : keys_smem<128, false>();
    return qcal ? keys_smem<64, true>() : keys_smem<64, false>();
}

// Batches per work unit: about four units per SM of a 148-SM part for the
// problem's upper bound of batches, within [kUnitMin, kUnitMax].
int bwd_keys_unit_batches(int B, int Hkv, int N, int S, int W, int K, int G) {
    (void)S;
    const int64_t nbt = (int64_t)B * Hkv * ((N + kBlk - 1) / kBlk);
    const int64_t pairs = (int64_t)G * ((int64_t)B * Hkv * N * K + nbt * (kBlk + W - 1));
    const int64_t ub = (pairs / kNP) / (4 * 148);
    return (int)(ub < kUnitMin ? kUnitMin : (ub > kUnitMax ? kUnitMax : ub));
}

int64_t bwd_keys_max_units(int B, int Hkv, int N, int S, int W, int K, int G) {
    const int64_t nbt = (int64_t)B * Hkv * ((N + kBlk - 1) / kBlk);
    // pairs: every valid selection plus each block's window rows, G heads
    const int64_t pairs = (int64_t)G * ((int64_t)B * Hkv * N * K + nbt * (kBlk + W - 1));
    const int64_t batches = pairs / kNP + nbt;
    return nbt + batches / bwd_keys_unit_batches(B, Hkv, N, S, W, K, G) + 1;
}

int64_t bwd_keys_partial_floats(int d) {
    return d == 128 ? kPartFloats<128> : kPartFloats<64>;
}

cudaError_t launch_bwd_index(const BwdIndexParams &ip, cudaStream_t st) {
    const int grid = ip.BH * ip.nseg;
    const size_t sm = (size_t)ip.nC * sizeof(int);
    cudaError_t e;
    if (sm > 48 * 1024) {
        e = cudaFuncSetAttribute(bwd_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(bwd_fill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
    }
    bwd_hist_kernel<<<grid, 256, sm, st>>>(ip);
    bwd_scan_kernel<<<ip.BH, 1024, 0, st>>>(ip);
    bwd_fill_kernel<<<grid, 32, sm, st>>>(ip);
    count_launches(3);
    return cudaGetLastError();
}

cudaError_t launch_bwd_keys_tc(const BwdTcParams &p, cudaStream_t st) {
    CUtensorMap mk, mv;
    if (!tc_make_map(&mk, p.Kc, p.d, p.N, p.Hkv, p.B, kBlk) ||
        !tc_make_map(&mv, p.V, p.d, p.N, p.Hkv, p.B, kBlk))
        return cudaErrorInvalidValue;
    bwd_plan_kernel<<<1, 1024, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const bool qcal = p.Qs != nullptr;
    if (p.d == 128)
        e = qcal ? launch_keys_tc_t<128, true>(p, mk, mv, st) : launch_keys_tc_t<128, false>(p, mk, mv, st);
    else
        e = qcal ? launch_keys_tc_t<64, true>(p, mk, mv, st) : launch_keys_tc_t<64, false>(p, mk, mv, st);
    count_launches(2);
    return e;
}

}  // namespace hils
