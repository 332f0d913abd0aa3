/*
 * lrkv_shared.h - decode attention over a cross-head shared latent ("AttentionPack",
 * Metodologia 2.A, multi-head compression: the key (value) rows of all KV heads are
 * concatenated along the head axis and factored once, so the cache holds one latent
 * row of rank R per token for every head, plus one decompression matrix of
 * R x (n_kv_heads * d_head) instead of per-head factors).
 *
 * KV head g's keys are K_g = Z_K D_K[:, g d : (g+1) d] and its values V_g likewise
 * (head-major concatenation); otherwise the call is lrkv_decode_attn: query head h
 * reads KV head h / G, split-KV partials and the log-sum-exp merge, status word,
 * lse_out optional.
 *   dims->rank     R, the shared latent width (the lrkv_dims rules for rank apply)
 *   ZK, ZV         [B][max_seq][R]       latent_dtype
 *   ZK_scale/ZV_scale [B][max_seq]        fp32 (I8/E4M3 only)
 *   DK, DV         [R][n_kv_heads * d]   io_dtype
 *   workspace      at least lrkv_workspace_bytes(dims with algo = LRKV_ALGO_SIMT)
 * Runs on the CUDA-core kernel (each KV head's CTAs read the shared rows; a kernel that
 * reads a tile once for all heads is not built). LRKV_ERR_UNSUPPORTED when
 * dims->algo == LRKV_ALGO_TCGEN05 or one head's decompression block (R x d) does not
 * fit the kernel's shared memory; LRKV_ERR_DIMS when dims->n_visual != 0; the other
 * errors as lrkv_decode_attn.
 */
#ifndef LRKV_SHARED_H
#define LRKV_SHARED_H

#include "lrkv.h"

#ifdef __cplusplus
extern "C" {
#endif

int lrkv_decode_attn_shared(const lrkv_dims* dims, const void* q, const void* ZK,
                            const void* ZV, const float* ZK_scale, const float* ZV_scale,
                            const void* DK, const void* DV, const int32_t* seqlens, void* out,
                            float* lse_out, void* workspace, size_t workspace_bytes,
                            void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LRKV_SHARED_H */
