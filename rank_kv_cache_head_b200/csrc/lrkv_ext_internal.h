// Internal declarations of the CUDA-core decode variants beyond the per-head cache:
// the attention-aware partial decompression (a per-token rank, and the attention-mass
// moving average) and the cross-head shared latent (one latent per token for every KV
// head, one decompression matrix).
#pragma once

#include "lrkv_internal.h"

namespace lrkv {

// What the adaptive split kernel reads besides SplitArgs.
struct AdaptArgs {
  const float* imp;  // [B][Hkv][Lcap] importance (read here, updated by the mass kernel)
  float tau;         // importance >= tau: full rank
  int r_low;         // rank of the other tokens
  float* scores;     // [B][Hq][Lcap] scores in log2 units (written for attended tokens)
};

// The moving average of the attention mass, run after the merge.
struct MassArgs {
  const float* scores;   // [B][Hq][Lcap], log2 units
  const float* lse;      // [B][Hq], natural log
  float* imp;            // [B][Hkv][Lcap], updated in place
  const int32_t* seqlens;
  uint32_t* header;
  int B, Hq, Hkv, Lcap, max_seqlen;
  float beta;
};

cudaError_t launch_split_simt_adaptive(const SplitArgs& a, const AdaptArgs& ad, const Plan& p,
                                       cudaStream_t st);
cudaError_t launch_mass_ema(const MassArgs& m, cudaStream_t st);
// Shared latent: ZK/ZV [B][Lcap][r] and scales [B][Lcap]; BK/BV hold the decompression
// matrices [r][Hkv * d] (KV head g owns columns g d .. g d + d - 1).
cudaError_t launch_split_simt_shared(const SplitArgs& a, const Plan& p, cudaStream_t st);

}  // namespace lrkv
