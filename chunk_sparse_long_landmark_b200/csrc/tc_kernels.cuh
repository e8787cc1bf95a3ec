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
