/*
 * hils.h -- C ABI of the HiLS (Hierarchical Landmark Sparse) attention
 * forward library, libhils.so (CUDA, sm_100a).
 *
 * The operation is the one of "Hierarchical Sparse Attention Done Right:
 * Toward Infinite Context Modeling" (Hu et al.):
 *   Sec. 2.1   chunks of S tokens, c(j) = floor(j/S); aligned window start
 *              l(i) = floor((i-W+1)/S)*S; candidates C_i = {0..l(i)/S-1};
 *              token logit s_ij = q_i.k_j/sqrt(d).
 *   Sec. 3     surrogate score s^_ic = q^_i.k'_c/sqrt(d) + b'_c (display
 *              after Eq. (7)); top-K chunks I_i; Z^_ic = exp s^_ic;
 *              Z^_i = sum_{c in I_i} Z^_ic + Z_swa.
 *   Sec. 3     hierarchical softmax (RQ2 display): for a token j of a
 *              selected chunk, w_ij = exp(s_ij)/Z_{i,c(j)} * Z^_{i,c(j)}/Z^_i;
 *              for a window token (l(i) <= j <= i) the chunk-level mass is
 *              the exact window mass, so w_ij = exp(s_ij)/Z^_i.
 *   Sec. 4.1   Q-Cal: the optional scoring query q^ enters only s^.
 *   Sec. 4.1   GQA: per query head, chunk weights normalised over C_i;
 *              maximum over the heads of a kv group; one top-K set per group.
 * Output o_i = sum_j w_ij v_j over the selected chunks and the window.
 *
 * Conventions fixed by this library where the paper is silent:
 *   positions are 0-based; the window starts at max(l(i), 0); C_i is empty
 *   when l(i) <= 0 (the row is then exact causal attention); b'_c is not
 *   scaled by 1/sqrt(d); per-head normalisation is a softmax over C_i only;
 *   top-K ties go to the lower chunk index; when |C_i| <= K all of C_i is
 *   selected; idx lists the selected chunks in ascending order, padded -1.
 *
 * Layouts: every tensor is dense, row-major, with the innermost dimension
 * contiguous, in the order given below. Q, Qs, K, V, landmark keys and O
 * share one element type (hils_dtype); bias and sel_score are float32; idx
 * and cache_len are int32. All tensor pointers are DEVICE pointers except
 * head_map, which is a HOST array read during the call.
 *
 * Ownership: the caller owns every buffer, including the workspace; the
 * library allocates no memory and keeps no state between calls other than
 * a per-device cache of kernel attributes.
 *
 * Streams and errors: calls enqueue work on `stream` (a cudaStream_t, NULL
 * = legacy default stream) and return without synchronising. Argument
 * errors are detected on the host before any launch and returned as a
 * hils_status; nothing is enqueued in that case. A failed launch returns
 * HILS_ERR_CUDA. Errors found on the device (a cache_len out of range, a
 * bounded wait that gave up) are written to *status (a device int32 the
 * caller zeroes and reads after synchronising; NULL disables reporting);
 * the affected outputs are then unspecified.
 *
 * Determinism: no floating-point atomics; repeated calls with the same
 * inputs give bitwise identical outputs.
 */
#ifndef HILS_H
#define HILS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HILS_OK = 0,
    HILS_ERR_INVALID_ARG = 1,       /* null pointer, bad size, bad head_map */
    HILS_ERR_UNSUPPORTED = 2,       /* valid but outside the supported set */
    HILS_ERR_MISALIGNED = 3,        /* a tensor pointer not 16-byte aligned */
    HILS_ERR_WORKSPACE_TOO_SMALL = 4,
    HILS_ERR_CUDA = 5,              /* a CUDA runtime call or launch failed */
    HILS_ERR_DEVICE_TIMEOUT = 6,    /* device-side bounded wait gave up */
    HILS_ERR_DEVICE_BAD_LENGTH = 7  /* device-side: cache_len outside [1, Lmax] */
} hils_status;

typedef enum { HILS_F32 = 0, HILS_BF16 = 1 } hils_dtype;

/* Limits of this build (checked on the host). */
#define HILS_MAX_HEAD_DIM 128       /* d in {64, 128} for bf16; d <= 128, d % 4 == 0 for f32 */
#define HILS_MAX_TOPK 64            /* 1 <= K <= 64 */
#define HILS_MAX_GROUP 16           /* G = Hq/Hkv <= 16 */

/*
 * Prefill: every position i in [0, N) of B sequences is a query.
 *   Q, Qs  [B, Hq, N, d]   query; Qs = scoring query q^ (NULL: use Q)
 *   Kc, V  [B, Hkv, N, d]  keys, values
 *   Klm    [B, Hkv, nC, d] landmark keys k'_c, nC = floor(N/S)
 *   bias   [B, Hkv, nC]    chunk bias b'_c (float32)
 *   O      [B, Hq, N, d]   output (written)
 *   idx    [B, Hkv, N, K]  selected chunks per (row, kv group) (written)
 *   sel_score [B, Hq, N, K] float32: s^ of each selected chunk for every
 *          query head, in idx order, NaN on padding (written; may be NULL,
 *          then the workspace holds it)
 *   head_map [Hq] HOST: kv head of each query head; every kv head must be
 *          used by exactly G = Hq/Hkv query heads.
 * Sizes: B, Hq, Hkv, N >= 1; S >= 1; W >= 1; 1 <= K <= HILS_MAX_TOPK.
 */
typedef struct {
    int32_t dtype;                  /* hils_dtype */
    int32_t B, Hq, Hkv, N, d, S, W, K;
    const int32_t *head_map;        /* host [Hq] */
    const void *Q, *Qs, *Kc, *V, *Klm;
    const float *bias;
    void *O;
    int32_t *idx;
    float *sel_score;               /* nullable */
    void *workspace;                /* device, >= hils_prefill_workspace_size */
    size_t workspace_bytes;
    int32_t *status;                /* device, nullable */
} hils_prefill_args;

/*
 * Decode: one query per sequence, the last cached token i = cache_len[b]-1,
 * whose own key and value are already in the cache.
 *   Q, Qs  [B, Hq, d]          query; Qs = scoring query (NULL: use Q)
 *   Kc, V  [B, Hkv, Lmax, d]   caches
 *   Klm    [B, Hkv, Lmax/S, d] landmark keys of the complete chunks
 *   bias   [B, Hkv, Lmax/S]    float32
 *   cache_len [B] DEVICE int32, each in [1, Lmax]
 *   O      [B, Hq, d]          output (written)
 *   idx    [B, Hkv, K]         selected chunks (written)
 *   sel_score [B, Hq, K]       float32, nullable
 */
typedef struct {
    int32_t dtype;
    int32_t B, Hq, Hkv, Lmax, d, S, W, K;
    const int32_t *head_map;        /* host [Hq] */
    const void *Q, *Qs, *Kc, *V, *Klm;
    const float *bias;
    const int32_t *cache_len;       /* device [B] */
    void *O;
    int32_t *idx;
    float *sel_score;               /* nullable */
    void *workspace;
    size_t workspace_bytes;
    int32_t *status;                /* device, nullable */
} hils_decode_args;

/* Human-readable name of a status code (static string). */
const char *hils_status_string(hils_status s);

/* Library version, as 10000*major + 100*minor + patch. */
int32_t hils_version(void);

/*
 * Workspace bytes a call with these arguments needs (only the shape fields,
 * dtype, head_map and the nullness of sel_score are read). Writes *bytes and
 * returns HILS_OK, or an argument error without writing.
 */
hils_status hils_prefill_workspace_size(const hils_prefill_args *args,
                                        size_t *bytes);
hils_status hils_decode_workspace_size(const hils_decode_args *args,
                                       size_t *bytes);

/*
 * HiLS prefill forward (Sec. 2.1, Sec. 3, Sec. 4.1): landmark scoring with
 * the causal candidate mask, per-group top-K, intra-chunk and window softmax
 * attention, chunk-level softmax fusion. Enqueued on `stream`.
 */
hils_status hils_fwd_prefill(const hils_prefill_args *args, void *stream);

/*
 * HiLS decode forward: the same computation for the last query of each
 * sequence, reading the caches. Enqueued on `stream`; graph-capturable (no
 * host synchronisation, cache_len read on the device).
 */
hils_status hils_fwd_decode(const hils_decode_args *args, void *stream);

/*
 * The two stages of hils_fwd_prefill / hils_fwd_decode, callable alone (same
 * argument record, same stream rules). hils_fwd_* is exactly select followed
 * by attend.
 *
 * *_select: chunk scoring, per-head normaliser, group top-K (Sec. 3, Sec. 4.1).
 *   Writes idx and the selected chunks' scores (sel_score, or the workspace
 *   when sel_score is NULL). Reads Q / Qs, Klm, bias; O is not touched.
 * *_attend: intra-chunk softmax attention over the chunks listed in idx and
 *   the aligned window, fused with the chunk-level softmax (Sec. 3, RQ2).
 *   Reads Q, Kc, V, idx and the selected scores; writes O. With sel_score
 *   NULL it must be given the same workspace as the select call. idx entries
 *   that are negative or not in C_i are ignored; each listed chunk must
 *   appear once, in ascending order.
 */
hils_status hils_prefill_select(const hils_prefill_args *args, void *stream);
hils_status hils_prefill_attend(const hils_prefill_args *args, void *stream);
hils_status hils_decode_select(const hils_decode_args *args, void *stream);
hils_status hils_decode_attend(const hils_decode_args *args, void *stream);

/*
 * hils_fwd_decode without a caller workspace (the paper has no counterpart:
 * this is a deployment variant). For callers that cannot allocate device
 * memory when they call: a serving loop whose memory is reserved up front, a
 * latency-critical path that cannot afford cudaMalloc's implicit device
 * synchronisation, or a host with no way to size and own a workspace.
 *
 * Same record and semantics as hils_fwd_decode; `workspace` and
 * `workspace_bytes` are ignored. Scratch comes from one fixed 8 MiB device
 * array inside the library (every GPU that loads the library holds it until
 * exit). It runs the CUDA-core decode kernels. The library allocates
 * nothing on this path.
 *   - The first call in a device's context, with that device current, looks
 *     up the array's device address (cudaGetSymbolAddress); make that first
 *     call before any stream capture. The address is cached per device and
 *     keyed on the context's process-unique ID, so after cudaDeviceReset (a
 *     new context, where the array may sit elsewhere) the next call looks it
 *     up again; make that call before any capture too.
 *   - Every call shares the one array and the next call overwrites it; calls
 *     whose executions overlap on the GPU (different streams, concurrent
 *     graphs) race on it. Nothing in it needs to start at zero.
 *   - A shape whose scratch exceeds the array (sel_score NULL adds B*Hq*K
 *     floats; scoring needs (Hq/Hkv + 1) * floor((Lmax-W)/S) floats per
 *     block) returns HILS_ERR_WORKSPACE_TOO_SMALL without enqueuing work.
 */
hils_status hils_fwd_decode_noalloc(const hils_decode_args *args, void *stream);

/*
 * Decode over a paged KV cache with page = chunk ("Hierarchical Sparse
 * Attention Done Right", Sec. 7.1: the serving setup keeps the cache in
 * pages of one chunk). Same computation and outputs as hils_fwd_decode;
 * only where K and V live changes:
 *   base.Kc, base.V   the page pool [n_pages, Hkv, S, d] (dtype): page p
 *                     holds S consecutive tokens of every kv head
 *   block_table       device int32 [B, base.Lmax / S]: the page holding
 *                     logical chunk c (tokens cS .. cS+S-1) of sequence b;
 *                     only the chunks a step reads (the selected ones and
 *                     the window's) need valid entries
 *   n_pages           pages in the pool
 * base.Lmax is the logical capacity per sequence (a multiple of S); the
 * landmark tensors Klm [B,Hkv,Lmax/S,d] and bias stay per sequence, as in
 * hils_fwd_decode. Supported: bf16, d in {64,128}, S in {64,128}, G <= 8
 * (the HBM decode kernels); other shapes return HILS_ERR_UNSUPPORTED. A page
 * index outside [0, n_pages) reads zeros and raises
 * HILS_ERR_DEVICE_BAD_LENGTH in the status word.
 */
typedef struct {
    hils_decode_args base;
    const int32_t *block_table;
    int32_t n_pages;
} hils_decode_paged_args;

hils_status hils_decode_paged_workspace_size(const hils_decode_paged_args *args,
                                             size_t *bytes);
hils_status hils_fwd_decode_paged(const hils_decode_paged_args *args, void *stream);

/*
 * Multi-token (speculative) decode: T query tokens per sequence, at
 * positions cache_len[b]-T .. cache_len[b]-1, whose keys and values are
 * already in the cache ("Hierarchical Sparse Attention Done Right", Sec. 4.2:
 * adjacent queries share one scan and their chunk unions; Sec. 7.1 for the
 * serving setting). Token t of sequence b gets exactly the decode result of
 * a query at position cache_len[b]-T+t (its own window, candidates and
 * top-K). The landmark keys of a (sequence, kv head) are read once for all
 * T x G scoring queries.
 *   base              as in hils_decode_args, except the token-major
 *                     query/output layouts:
 *     Q, Qs   [B, T, Hq, d]      O [B, T, Hq, d]
 *     idx     [B, T, Hkv, K]     sel_score [B, T, Hq, K] (nullable)
 *   T                 tokens per sequence, 1 <= T, T * (Hq/Hkv) <= 32
 *   block_table       nullable: when given, base.Kc / base.V are the page
 *                     pool of hils_decode_paged_args and n_pages its size
 * cache_len[b] must lie in [T, Lmax] (else HILS_ERR_DEVICE_BAD_LENGTH in
 * the status word). Supported: bf16, d in {64,128}, S in {64,128}, G <= 8;
 * other shapes return HILS_ERR_UNSUPPORTED. T = 1 is hils_fwd_decode
 * (or hils_fwd_decode_paged).
 */
typedef struct {
    hils_decode_args base;
    int32_t T;
    const int32_t *block_table;     /* device, nullable */
    int32_t n_pages;
} hils_decode_multi_args;

hils_status hils_decode_multi_workspace_size(const hils_decode_multi_args *args,
                                             size_t *bytes);
hils_status hils_fwd_decode_multi(const hils_decode_multi_args *args, void *stream);

/*
 * Backward of the prefill forward, for a fixed selection ("Hierarchical
 * Sparse Attention Done Right", Sec. 3, RQ2: the fused chunk-level softmax
 * lets the loss reach the landmark scores; Sec. 4, native sparse training).
 * The top-K choice is discrete and held fixed; gradients of sum(O * dO) flow
 * to Q, the scoring query, K, V, the landmark keys and the biases through
 * the intra-chunk softmax, the chunk scores s^ and the window softmax.
 *   Q, Qs, dO [B,Hq,N,d]; Kc, V [B,Hkv,N,d]; Klm [B,Hkv,nC,d]; bias
 *   [B,Hkv,nC] f32; idx [B,Hkv,N,K] int32 (the forward's selection:
 *   ascending, -1 padded; entries outside C_i are ignored, as the forward
 *   ignores them); dtype of Q, Qs, dO, Kc, V, Klm: f32 or bf16.
 *   Outputs, f32, overwritten (not accumulated): dQ [B,Hq,N,d], dQs (must be
 *   given exactly when Qs is; without Qs the scoring gradient is in dQ), dK,
 *   dV [B,Hkv,N,d], dKlm [B,Hkv,nC,d], dbias [B,Hkv,nC].
 *   workspace >= hils_bwd_prefill_workspace_size (per (row, head) and
 *   (row, head, selected chunk) softmax statistics; for bf16, also the
 *   chunk -> (row, slot) index of the selection and the key side's work
 *   units with room for their partial sums).
 *   status: device int32, nullable; a kernel whose bounded wait gave up
 *   writes HILS_ERR_DEVICE_TIMEOUT there (the gradients are then undefined).
 * bf16 runs on the tensor cores (products of bf16 operands -- the weights
 * p_j and ds_j are rounded to bf16 -- with f32 accumulation), f32 on the
 * CUDA cores in f32. Deterministic: no floating-point atomics; every output
 * element is summed in one fixed order, so repeated calls are bitwise equal.
 * Supported: d in {64,128}, S in {64,128}, G = Hq/Hkv <= 8; other shapes
 * return HILS_ERR_UNSUPPORTED. Kernel launches on `stream`: at most 8 for
 * bf16, 2 for f32.
 */
typedef struct {
    int32_t dtype;
    int32_t B, Hq, Hkv, N, d, S, W, K;
    const int32_t *head_map;        /* host [Hq] */
    const void *Q, *Qs, *Kc, *V, *Klm;
    const float *bias;
    const void *dO;
    const int32_t *idx;
    float *dQ, *dQs, *dK, *dV, *dKlm, *dbias;
    void *workspace;
    size_t workspace_bytes;
    int32_t *status;                /* device, nullable */
} hils_backward_args;

hils_status hils_bwd_prefill_workspace_size(const hils_backward_args *args,
                                            size_t *bytes);
hils_status hils_bwd_prefill(const hils_backward_args *args, void *stream);

/*
 * Landmark summaries of the chunks: the (k', b') inputs of the scoring step.
 * "Hierarchical Sparse Attention Done Right", Sec. 3 (answering RQ1, the
 * surrogate of Eq. 7): for every full chunk c (nC = floor(N/S) of them) of
 * every (batch, kv head), a landmark query q'_c induces
 *   p_j  = softmax_j(q'_c . k_j / sqrt(d)),   j = cS .. cS+S-1,
 *   k'_c = sum_j p_j k_j                      (the weighted key sum),
 *   b'_c = -sum_j p_j log p_j                 (its entropy, in [0, log S]),
 * i.e. Attn(q'_c, K_c, K_c). At q = q'_c the surrogate q.k'_c/sqrt(d) + b'_c
 * equals the exact chunk log-mass. shared_query = 1 is the pages'
 * landmark-token-free variant (Sec. 4.1): one query per kv head for every
 * chunk and batch.
 *
 * Layout (device pointers, 16-byte aligned, innermost dimension contiguous):
 *   Kc    [B,Hkv,N,d]              dtype
 *   Qlm   [B,Hkv,nC,d], or [Hkv,d] when shared_query = 1,   dtype
 *   Klm   out [B,Hkv,nC,d]         dtype (k' rounded to it)
 *   bias  out [B,Hkv,nC]           float32
 * Supported: d in {64, 128}; S in {32, 64, 128, 256}; N >= S.
 * The caller owns all buffers; nothing is allocated. Asynchronous on
 * `stream`; argument errors are returned before anything is enqueued
 * (HILS_ERR_INVALID_ARG, HILS_ERR_UNSUPPORTED, HILS_ERR_MISALIGNED), launch
 * failures as HILS_ERR_CUDA.
 */
typedef struct {
    int32_t dtype;                  /* hils_dtype of Kc, Qlm, Klm */
    int32_t B, Hkv, N, d, S;
    const void *Kc;
    const void *Qlm;
    int32_t shared_query;
    void *Klm;
    float *bias;
} hils_landmark_args;

hils_status hils_build_landmarks(const hils_landmark_args *args, void *stream);

/*
 * Chunk-overlap diagnostics of a selection ("Hierarchical Sparse Attention
 * Done Right", Sec. 7.2: Overlap = (M K - |I_1 u ... u I_M|) / ((M-1) K) for
 * M adjacent queries). For every block of M consecutive query rows (the last
 * block may be shorter) of every (batch, kv head):
 *   n_sel   = entries >= 0 of the block's idx rows,
 *   n_union = distinct chunks among them,
 *   n_reuse = distinct chunks also in the previous block's union (0 for the
 *             first block).
 * Overlap of a full block whose rows hold K chunks each is
 * (M*K - n_union) / ((M-1)*K).
 *   idx      [B,Hkv,N,K] int32, device (as the select stage writes it);
 *            entries outside [0, nC) other than -1 are an argument error the
 *            kernel cannot see: they are skipped
 *   n_sel, n_union, n_reuse   out [B,Hkv,ceil(N/M)] int32, device
 *   nC       bound on the chunk indices; 2 <= M <= 128; 1 <= K <= 64.
 * Asynchronous on `stream`; nothing allocated; argument errors returned
 * before anything is enqueued.
 */
hils_status hils_chunk_overlap(const int32_t *idx, int32_t B, int32_t Hkv,
                               int32_t N, int32_t K, int32_t nC, int32_t M,
                               int32_t *n_sel, int32_t *n_union,
                               int32_t *n_reuse, void *stream);

/*
 * Number of kernel launches this library has enqueued in this process so far
 * (all devices, all threads). A diagnostic for counting launches per call.
 */
uint64_t hils_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* HILS_H */
