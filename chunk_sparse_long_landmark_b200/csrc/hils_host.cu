// hils_host.cu -- host side of libhils: the C ABI of include/hils.h.
//
// Validates arguments before anything is enqueued, lays out the caller's
// workspace, fills the kernel parameter record and launches the kernels on
// the caller's stream. Allocates nothing; never synchronises.
#include <math.h>
#include <string.h>

#include <cuda_runtime.h>

#include "hils_internal.cuh"
#include "hils_fast.cuh"

using namespace hils;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Checks shared by prefill and decode. `rows` is N (prefill) or Lmax.
hils_status check_common(int32_t dtype, int B, int Hq, int Hkv, int rows,
                         int d, int S, int W, int K, const int32_t *head_map,
                         Problem *p) {
    if (dtype != HILS_F32 && dtype != HILS_BF16) return HILS_ERR_INVALID_ARG;
    if (B < 1 || Hq < 1 || Hkv < 1 || rows < 1 || d < 1 || S < 1 || W < 1 ||
        K < 1)
        return HILS_ERR_INVALID_ARG;
    if (!head_map) return HILS_ERR_INVALID_ARG;
    if (Hq % Hkv) return HILS_ERR_INVALID_ARG;
    if (K > HILS_MAX_TOPK) return HILS_ERR_UNSUPPORTED;
    if (Hq > kMaxHeads) return HILS_ERR_UNSUPPORTED;
    const int G = Hq / Hkv;
    if (G > HILS_MAX_GROUP) return HILS_ERR_UNSUPPORTED;
    if (d > HILS_MAX_HEAD_DIM) return HILS_ERR_UNSUPPORTED;
    const int esz = dtype == HILS_BF16 ? 2 : 4;
    if ((d * esz) % 16) return HILS_ERR_UNSUPPORTED;   // 16-byte rows
    if (S > simt_max_chunk()) return HILS_ERR_UNSUPPORTED;
    // head_map: every kv head used by exactly G query heads
    int count[kMaxHeads];
    for (int g = 0; g < Hkv; ++g) count[g] = 0;
    for (int h = 0; h < Hq; ++h) {
        int g = head_map[h];
        if (g < 0 || g >= Hkv) return HILS_ERR_INVALID_ARG;
        if (count[g] >= G) return HILS_ERR_INVALID_ARG;
        p->group_heads[g * G + count[g]] = (int16_t)h;
        p->head_map[h] = (int16_t)g;
        count[g]++;
    }
    for (int g = 0; g < Hkv; ++g)
        if (count[g] != G) return HILS_ERR_INVALID_ARG;
    p->dtype = dtype;
    p->B = B; p->Hq = Hq; p->Hkv = Hkv; p->G = G; p->d = d; p->S = S;
    p->W = W; p->K = K;
    p->inv_sqrt_d = (float)(1.0 / sqrt((double)d));
    return HILS_OK;
}

// Workspace plan: where each scratch array lives inside the caller's buffer.
struct Plan {
    size_t sel_off = 0, sel_bytes = 0;      // s^ of selected chunks (if user gave none)
    size_t scr_off = 0, scr_bytes = 0;      // SIMT scoring scratch
    size_t fast_off = 0, fast_bytes = 0;    // fast-path scratch
    int score_grid = 0;
    bool fast_select = false;               // tensor-core selection kernels
    bool fast_attend = false;               // tensor-core attention kernels
    size_t total = 0;
};

void plan_simt_scratch(const Problem &p, Plan *pl) {
    int64_t w0, ncm;
    window_bounds((int64_t)p.kv_rows - 1, p.S, p.W, &w0, &ncm);
    pl->score_grid = simt_score_grid(p);
    pl->scr_bytes = sizeof(float) * simt_score_scratch_floats(p, (int)ncm) *
                    (size_t)(pl->score_grid > 0 ? pl->score_grid : 1);
}

hils_status prefill_problem(const hils_prefill_args *a, Problem *p,
                            bool need_ptrs) {
    if (!a) return HILS_ERR_INVALID_ARG;
    memset(p, 0, sizeof(*p));
    hils_status s = check_common(a->dtype, a->B, a->Hq, a->Hkv, a->N, a->d,
                                 a->S, a->W, a->K, a->head_map, p);
    if (s != HILS_OK) return s;
    p->n_query = a->N;
    p->T = 1;
    p->kv_rows = a->N;
    p->nC = a->N / a->S;
    p->decode = 0;
    if (need_ptrs) {
        if (!a->Q || !a->Kc || !a->V || !a->O || !a->idx)
            return HILS_ERR_INVALID_ARG;
        if (p->nC > 0 && (!a->Klm || !a->bias)) return HILS_ERR_INVALID_ARG;
        const void *ptrs[] = {a->Q, a->Qs, a->Kc, a->V, a->Klm, a->bias,
                              a->O, a->idx, a->sel_score, a->workspace};
        for (const void *q : ptrs)
            if (q && !aligned16(q)) return HILS_ERR_MISALIGNED;
        p->Q = a->Q; p->Qs = a->Qs; p->Kc = a->Kc; p->V = a->V;
        p->Klm = a->Klm; p->bias = a->bias; p->O = a->O; p->idx = a->idx;
        p->sel = a->sel_score; p->status = a->status;
    }
    return HILS_OK;
}

hils_status decode_problem(const hils_decode_args *a, Problem *p,
                           bool need_ptrs) {
    if (!a) return HILS_ERR_INVALID_ARG;
    memset(p, 0, sizeof(*p));
    hils_status s = check_common(a->dtype, a->B, a->Hq, a->Hkv, a->Lmax, a->d,
                                 a->S, a->W, a->K, a->head_map, p);
    if (s != HILS_OK) return s;
    p->n_query = 1;
    p->T = 1;
    p->kv_rows = a->Lmax;
    p->nC = a->Lmax / a->S;
    p->decode = 1;
    if (need_ptrs) {
        if (!a->Q || !a->Kc || !a->V || !a->O || !a->idx || !a->cache_len)
            return HILS_ERR_INVALID_ARG;
        if (p->nC > 0 && (!a->Klm || !a->bias)) return HILS_ERR_INVALID_ARG;
        const void *ptrs[] = {a->Q, a->Qs, a->Kc, a->V, a->Klm, a->bias,
                              a->O, a->idx, a->sel_score, a->workspace};
        for (const void *q : ptrs)
            if (q && !aligned16(q)) return HILS_ERR_MISALIGNED;
        p->Q = a->Q; p->Qs = a->Qs; p->Kc = a->Kc; p->V = a->V;
        p->Klm = a->Klm; p->bias = a->bias; p->O = a->O; p->idx = a->idx;
        p->sel = a->sel_score; p->cache_len = a->cache_len;
        p->status = a->status;
    }
    return HILS_OK;
}

void plan_workspace(const Problem &p, bool user_sel, Plan *pl) {
    size_t off = 0;
    if (!user_sel) {
        pl->sel_off = off;
        pl->sel_bytes = sizeof(float) * (size_t)p.B * p.Hq * p.n_query * p.K;
        off = align_up(off + pl->sel_bytes);
    }
    pl->fast_attend = fast_path_supported(p);
    pl->fast_select = pl->fast_attend && fast_select_supported(p);
    if (pl->fast_attend || pl->fast_select) {
        pl->fast_off = off;
        pl->fast_bytes = fast_workspace_bytes(p);
        off = align_up(off + pl->fast_bytes);
    }
    if (!pl->fast_select) {
        plan_simt_scratch(p, pl);
        pl->scr_off = off;
        off = align_up(off + pl->scr_bytes);
    }
    pl->total = off > 0 ? off : kAlign;
}

enum Stage { kSelect = 1, kAttend = 2, kBoth = 3 };

hils_status run(Problem &p, const Plan &pl, void *ws, size_t ws_bytes,
                cudaStream_t st, int stages) {
    if (ws_bytes < pl.total) return HILS_ERR_WORKSPACE_TOO_SMALL;
    if (!ws) return HILS_ERR_INVALID_ARG;
    char *base = (char *)ws;
    if (!p.sel) p.sel = (float *)(base + pl.sel_off);
    cudaError_t e = cudaSuccess;
    if (stages & kSelect) {
        if (pl.fast_select) {
            e = launch_fast_select(p, base + pl.fast_off, pl.fast_bytes, st);
        } else {
            e = launch_simt_score(p, (float *)(base + pl.scr_off),
                                  pl.score_grid, st);
            count_launches(1);
        }
    }
    if (e == cudaSuccess && (stages & kAttend)) {
        if (pl.fast_attend) {
            e = launch_fast_attend(p, base + pl.fast_off, pl.fast_bytes, st);
        } else {
            e = launch_simt_attend(p, st);
            count_launches(1);
        }
    }
    return e == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
}

hils_status prefill_entry(const hils_prefill_args *args, void *stream,
                          int stages) {
    Problem p;
    hils_status s = prefill_problem(args, &p, true);
    if (s != HILS_OK) return s;
    Plan pl;
    plan_workspace(p, args->sel_score != nullptr, &pl);
    return run(p, pl, args->workspace, args->workspace_bytes,
               (cudaStream_t)stream, stages);
}

// The paged record: the decode record's checks, plus the page table, and
// only the shapes the HBM decode kernels run.
hils_status paged_problem(const hils_decode_paged_args *a, Problem *p,
                          bool need_ptrs) {
    if (!a) return HILS_ERR_INVALID_ARG;
    hils_status s = decode_problem(&a->base, p, need_ptrs);
    if (s != HILS_OK) return s;
    if (a->base.Lmax % a->base.S != 0 || a->n_pages < 1) return HILS_ERR_INVALID_ARG;
    if ((int64_t)a->n_pages * a->base.Hkv * a->base.S >= (1ll << 31))
        return HILS_ERR_UNSUPPORTED;                 // TMA row coordinates are int32
    if (need_ptrs && !a->block_table) return HILS_ERR_INVALID_ARG;
    p->block_table = a->block_table;
    p->n_pages = a->n_pages;
    if (!fast_path_supported(*p) || !fast_select_supported(*p))
        return HILS_ERR_UNSUPPORTED;
    return HILS_OK;
}

// The multi-token record: T query tokens per sequence (token-major Q, O,
// idx, sel_score), optionally over a paged cache; HBM decode kernels only.
hils_status multi_problem(const hils_decode_multi_args *a, Problem *p,
                          bool need_ptrs) {
    if (!a) return HILS_ERR_INVALID_ARG;
    hils_status s = decode_problem(&a->base, p, need_ptrs);
    if (s != HILS_OK) return s;
    if (a->T < 1 || a->T > a->base.Lmax) return HILS_ERR_INVALID_ARG;
    if (a->T * p->G > 32) return HILS_ERR_UNSUPPORTED;
    p->T = a->T;
    p->n_query = a->T;
    if (a->block_table) {
        if (a->base.Lmax % a->base.S != 0 || a->n_pages < 1) return HILS_ERR_INVALID_ARG;
        if ((int64_t)a->n_pages * a->base.Hkv * a->base.S >= (1ll << 31))
            return HILS_ERR_UNSUPPORTED;
        p->block_table = a->block_table;
        p->n_pages = a->n_pages;
    }
    if (!fast_path_supported(*p) || !fast_select_supported(*p))
        return HILS_ERR_UNSUPPORTED;
    return HILS_OK;
}

hils_status decode_entry(const hils_decode_args *args, void *stream,
                         int stages) {
    Problem p;
    hils_status s = decode_problem(args, &p, true);
    if (s != HILS_OK) return s;
    Plan pl;
    plan_workspace(p, args->sel_score != nullptr, &pl);
    return run(p, pl, args->workspace, args->workspace_bytes,
               (cudaStream_t)stream, stages);
}

}  // namespace

namespace hils {
// Full argument check of a decode record (shapes and pointers), shared with
// the allocation-free entry point.
hils_status decode_problem_checked(const hils_decode_args *a, Problem *p) {
    return decode_problem(a, p, true);
}
}  // namespace hils

extern "C" {

const char *hils_status_string(hils_status s) {
    switch (s) {
        case HILS_OK: return "HILS_OK";
        case HILS_ERR_INVALID_ARG: return "HILS_ERR_INVALID_ARG";
        case HILS_ERR_UNSUPPORTED: return "HILS_ERR_UNSUPPORTED";
        case HILS_ERR_MISALIGNED: return "HILS_ERR_MISALIGNED";
        case HILS_ERR_WORKSPACE_TOO_SMALL: return "HILS_ERR_WORKSPACE_TOO_SMALL";
        case HILS_ERR_CUDA: return "HILS_ERR_CUDA";
        case HILS_ERR_DEVICE_TIMEOUT: return "HILS_ERR_DEVICE_TIMEOUT";
        case HILS_ERR_DEVICE_BAD_LENGTH: return "HILS_ERR_DEVICE_BAD_LENGTH";
    }
    return "HILS_ERR_UNKNOWN";
}

int32_t hils_version(void) { return 100; }

hils_status hils_prefill_workspace_size(const hils_prefill_args *args,
                                        size_t *bytes) {
    if (!bytes) return HILS_ERR_INVALID_ARG;
    Problem p;
    hils_status s = prefill_problem(args, &p, false);
    if (s != HILS_OK) return s;
    Plan pl;
    plan_workspace(p, args->sel_score != nullptr, &pl);
    *bytes = pl.total;
    return HILS_OK;
}

hils_status hils_decode_workspace_size(const hils_decode_args *args,
                                       size_t *bytes) {
    if (!bytes) return HILS_ERR_INVALID_ARG;
    Problem p;
    hils_status s = decode_problem(args, &p, false);
    if (s != HILS_OK) return s;
    Plan pl;
    plan_workspace(p, args->sel_score != nullptr, &pl);
    *bytes = pl.total;
    return HILS_OK;
}

hils_status hils_fwd_prefill(const hils_prefill_args *args, void *stream) {
    return prefill_entry(args, stream, kBoth);
}

hils_status hils_prefill_select(const hils_prefill_args *args, void *stream) {
    return prefill_entry(args, stream, kSelect);
}

hils_status hils_prefill_attend(const hils_prefill_args *args, void *stream) {
    return prefill_entry(args, stream, kAttend);
}

hils_status hils_fwd_decode(const hils_decode_args *args, void *stream) {
    return decode_entry(args, stream, kBoth);
}

hils_status hils_decode_select(const hils_decode_args *args, void *stream) {
    return decode_entry(args, stream, kSelect);
}

hils_status hils_decode_attend(const hils_decode_args *args, void *stream) {
    return decode_entry(args, stream, kAttend);
}

hils_status hils_decode_paged_workspace_size(const hils_decode_paged_args *args,
                                             size_t *bytes) {
    if (!bytes) return HILS_ERR_INVALID_ARG;
    Problem p;
    hils_status s = paged_problem(args, &p, false);
    if (s != HILS_OK) return s;
    Plan pl;
    plan_workspace(p, args->base.sel_score != nullptr, &pl);
    *bytes = pl.total;
    return HILS_OK;
}

hils_status hils_fwd_decode_paged(const hils_decode_paged_args *args, void *stream) {
    Problem p;
    hils_status s = paged_problem(args, &p, true);
    if (s != HILS_OK) return s;
    Plan pl;
    plan_workspace(p, args->base.sel_score != nullptr, &pl);
    return run(p, pl, args->base.workspace, args->base.workspace_bytes,
               (cudaStream_t)stream, kBoth);
}

hils_status hils_decode_multi_workspace_size(const hils_decode_multi_args *args,
                                             size_t *bytes) {
    if (!bytes) return HILS_ERR_INVALID_ARG;
    Problem p;
    hils_status s = multi_problem(args, &p, false);
    if (s != HILS_OK) return s;
    Plan pl;
    plan_workspace(p, args->base.sel_score != nullptr, &pl);
    *bytes = pl.total;
    return HILS_OK;
}

hils_status hils_fwd_decode_multi(const hils_decode_multi_args *args, void *stream) {
    Problem p;
    hils_status s = multi_problem(args, &p, true);
    if (s != HILS_OK) return s;
    Plan pl;
    plan_workspace(p, args->base.sel_score != nullptr, &pl);
    return run(p, pl, args->base.workspace, args->base.workspace_bytes,
               (cudaStream_t)stream, kBoth);
}

uint64_t hils_launch_count(void) { return launch_total(); }

}  // extern "C"
