// tc_kernels.cuh -- parameters shared by the host dispatch and the sm_100a
// tensor-core kernels (TMA tensor maps are passed as __grid_constant__).
#pragma once

#include <cuda.h>

#include "hils_internal.cuh"

namespace hils {

struct TcParams {
    const void *Q;  // [B,Hq,N,d] (the attention kernel loads its rows itself)
    const void *Klm;
    const float *bias;
    void *O;
    int32_t *idx;
    float *sel;
    int32_t *status;
    int B, Hq, Hkv, G, N, d, S, W, K, nC;
    int M;          // queries per CTA tile: 128 / G
    int ucap;       // capacity of the chunk-union list: min(M*K, nC)
    float inv_sqrt_d;
    int16_t group_heads[kMaxHeads];
};

struct TcMaps {
    CUtensorMap k;  // K [B,Hkv,N,d]: box {64, S, 1, 1}
    CUtensorMap v;  // V [B,Hkv,N,d]: box {64, S, 1, 1}
    CUtensorMap lm; // Klm [B,Hkv,nC,d]: box {64, 128, 1, 1}
};

// Inverse index of a selection (chunk -> its (row, top-K slot) entries) for
// the backward's key side.
struct BwdIndexParams {
    const int32_t *idx;   // [B*Hkv][N][K]
    int *off;             // [B*Hkv][off_stride]: exclusive scan over [chunk][segment]
    int32_t *ent;         // [B*Hkv][ent_stride]: row << 6 | slot, grouped by chunk
    int64_t off_stride, ent_stride;
    int BH, N, S, W, K, nC;
    int R, nseg;          // rows per segment, segments
};

// Key side of the backward on the tensor cores (bf16).
struct BwdTcParams {
    const void *Q, *Qs, *Kc, *V, *dO;
    const float *rowstat;     // [B,Hq,N,2]: L, D
    const float *chunkstat;   // [B,Hq,N,K,4]: a, Ubar, dsh, -
    const int *off;
    const int32_t *ent;
    float *dK, *dV, *dKlm, *dbias;
    int32_t *status;
    // work units (a key block with many pairs is cut into several)
    int2 *units;              // [max_units]: (global block, unit of the block)
    int *nunits_blk;          // [B*Hkv*nblk]
    int *tickets;             // [B*Hkv*nblk]: units finished
    int *n_units;             // [1]
    float *partial;           // [max_units][bwd_keys_partial_floats(d)]
    int64_t max_units;
    int unit_batches;         // batches per work unit
    int64_t off_stride, ent_stride;
    int B, Hq, Hkv, G, N, d, S, W, K, nC, nseg;
    float inv_sqrt_d;
    int16_t group_heads[kMaxHeads];
};

// Query side of the backward on the tensor cores (bf16, 128 % G == 0).
struct BwdRowsParams {
    const void *Q, *Qs, *Kc, *V, *dO, *Klm;
    const float *bias;
    const int32_t *idx;
    float *rowstat;           // [B,Hq,N,2]: L, D
    float *chunkstat;         // [B,Hq,N,K,4]: a, Ubar, dsh, s^
    float *dQ, *dQs;
    int32_t *status;
    int B, Hq, Hkv, G, N, d, S, W, K, nC;
    int M;                    // queries per CTA: 128 / G
    int ucap;                 // capacity of the chunk-union list: min(M*K, nC)
    float inv_sqrt_d;
    int16_t group_heads[kMaxHeads];
};

size_t bwd_rows_tc_smem(const BwdRowsParams &p);
cudaError_t launch_bwd_rows_tc(const BwdRowsParams &p, cudaStream_t st);
void bwd_index_shape(int N, int nC, BwdIndexParams *ip);
size_t bwd_keys_tc_smem(int d, bool qcal);
int64_t bwd_keys_max_units(int B, int Hkv, int N, int S, int W, int K, int G);
int bwd_keys_unit_batches(int B, int Hkv, int N, int S, int W, int K, int G);
int64_t bwd_keys_partial_floats(int d);
cudaError_t launch_bwd_index(const BwdIndexParams &ip, cudaStream_t st);
cudaError_t launch_bwd_keys_tc(const BwdTcParams &p, cudaStream_t st);
// bf16 tensor map over [d3][d2][rows][d] with a {64, box_rows} tile,
// 128-byte swizzle (false when the driver entry point is missing)
bool tc_make_map(CUtensorMap *m, const void *base, int d, int64_t rows, int d2,
                 int d3, int box_rows);
bool tc_maps_available();

bool dec_fast_supported(const Problem &p);
size_t dec_workspace_bytes(const Problem &p);
cudaError_t launch_dec_select(Problem &p, void *ws, cudaStream_t st);
cudaError_t launch_dec_attend(Problem &p, void *ws, cudaStream_t st);
bool tc_select_supported(const TcParams &tp);
cudaError_t launch_tc_select(const TcParams &tp, const CUtensorMap &lm32,
                             const CUtensorMap &q128, cudaStream_t st);
size_t tc_score_smem_bytes(const TcParams &tp, int d);
cudaError_t launch_tc_score(const TcParams &tp, const TcMaps &maps,
                            const void *qhat, cudaStream_t st);
size_t tc_attend_smem_bytes(const TcParams &tp, int s_tok, int d);
cudaError_t launch_tc_attend(const TcParams &tp, const TcMaps &maps,
                             cudaStream_t st);

}  // namespace hils
