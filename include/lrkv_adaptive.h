/*
 * lrkv_adaptive.h - attention-aware partial decompression on the low-rank KV cache of
 * lrkv.h ("AttentionPack", Metodologia 2.B: not every token matters equally at every
 * step; tokens with high accumulated attention are decompressed at the original rank,
 * the others at a reduced rank, which cuts the decompression FLOPs).
 *
 * Per (batch row, KV head, token) the caller keeps an importance value, a moving
 * average of the token's attention mass. One call attends exactly like
 * lrkv_decode_attn except that a token t with importance[b][g][t] < tau is rebuilt
 * from the leading r_low rank components of its latents only (K_t = sum_{j < r_low}
 * Z_K[t][j] B_K[j], likewise V_t; the factor rows are ordered by singular value, so
 * the prefix is the best rank-r_low part). It then updates, for every attended
 * position t < seqlens[b],
 *     mass[b][g][t]       = sum over the G query heads h of group g of
 *                           exp(score[b][h][t] - lse[b][h])   (the softmax weight)
 *     importance[b][g][t] = beta * importance[b][g][t] + (1 - beta) * mass[b][g][t]
 * and leaves the other positions untouched. The comparison importance >= tau is made
 * on the stored fp32 values. The append does not touch importance: initialise a new
 * token's slot yourself (a value >= tau rebuilds it at full rank).
 *
 * Runs on the CUDA-core kernel (the per-token rank is a loop bound there); with
 * dims->algo == LRKV_ALGO_TCGEN05 it returns LRKV_ERR_UNSUPPORTED.
 *   importance [B][Hkv][max_seq] fp32, device, in/out
 *   tau        threshold; r_low in [1, rank]; beta in [0, 1]
 *   scores     [B][Hq][max_seq] fp32, device scratch (the scores in log2 units)
 *   lse_out    [B][Hq] fp32, device, required (the merge's LSE, used for the mass)
 *   workspace  at least lrkv_workspace_bytes(dims with algo = LRKV_ALGO_SIMT) bytes
 *   other arguments as lrkv_decode_attn (modality-separated factors included).
 * Errors: those of lrkv_decode_attn; LRKV_ERR_ARG (NULL importance, scores or lse_out;
 * r_low outside [1, rank]; beta outside [0, 1]); LRKV_ERR_UNSUPPORTED (tcgen05 asked).
 * Launches the split kernel, the merge kernel and the moving-average kernel on stream.
 */
#ifndef LRKV_ADAPTIVE_H
#define LRKV_ADAPTIVE_H

#include "lrkv.h"

#ifdef __cplusplus
extern "C" {
#endif

int lrkv_decode_attn_adaptive(const lrkv_dims* dims, const void* q, const void* ZK,
                              const void* ZV, const float* ZK_scale, const float* ZV_scale,
                              const void* BK, const void* BV, const int32_t* seqlens,
                              float* importance, float tau, int32_t r_low, float beta,
                              float* scores, void* out, float* lse_out, void* workspace,
                              size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LRKV_ADAPTIVE_H */
