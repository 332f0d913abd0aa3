// CUDA-core kernels of liblrkv:
//  * lrkv_split_simt: split-KV decode attention over a per-head low-rank cache in
//    fp32 arithmetic, for every dtype combination (the fp32-I/O path, and the
//    fallback for shapes the tcgen05 kernel does not take);
//  * lrkv_merge: the log-sum-exp merge of the split partials (Flash Decoding);
//  * lrkv_append: one new latent row per (batch row, KV head), with the per-token
//    int8 / e4m3 absmax quantiser.
// The method: per-head factors W_K,g = A_K,g B_K,g, keys/values rebuilt from the
// latent as K = Z_K B_K, V = Z_V B_V inside the attention kernel and never written
// to HBM ("WSVD: Weighted Low-Rank Approximation for Fast and Efficient Execution of
// Low-Precision Vision-Language Models", sections 2.A and 2.C).
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <math_constants.h>

#include "lrkv_ext_internal.h"
#include "lrkv_internal.h"
#include "lrkv_sm100.cuh"

namespace lrkv {
namespace {

using namespace sm100;

constexpr int kSimtThreads = 256;
constexpr int kSimtTile = 32;  // tokens per inner tile of the CUDA-core kernel

__device__ __forceinline__ float load_io(const void* p, size_t i, int io_dtype) {
  if (io_dtype == LRKV_F32) return static_cast<const float*>(p)[i];
  return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}

__device__ __forceinline__ float load_lat(const void* p, size_t i, int lat) {
  switch (lat) {
    case LRKV_F32: return static_cast<const float*>(p)[i];
    case LRKV_BF16: return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
    case LRKV_I8: return static_cast<float>(static_cast<const int8_t*>(p)[i]);
    default: {
      __nv_fp8_e4m3 v;
      v.__x = static_cast<const __nv_fp8_storage_t*>(p)[i];
      return static_cast<float>(v);
    }
  }
}

// Valid length of batch row b under the call's contract; flags violations and
// treats such a row as empty. Split and merge kernels apply the same rule.
__device__ __forceinline__ int checked_len(const int32_t* seqlens, int b, int Lcap,
                                           int max_seqlen, uint32_t* header, bool flag) {
  int L = seqlens[b];
  uint32_t bad = 0;
  if (L < 0 || L > Lcap) bad = LRKV_STATUS_SEQLEN_RANGE;
  else if (L > max_seqlen) bad = LRKV_STATUS_SEQLEN_HINT;
  if (bad) {
    if (flag) atomicOr(header + kStatusWord, bad);
    return 0;
  }
  return L;
}

// grid (S, Hkv, B); one CTA = one split of one (batch row, KV head), all G query
// heads of the group. Tiles of 32 tokens: latents -> smem (dequantised), rebuild the
// K tile = Z_K B_K, scores for the G heads, rebuild the V tile = Z_V B_V, online
// softmax, accumulate P V. fp32 throughout.
// ADAPT: attention-aware partial decompression. A token whose importance is below
// ad.tau is rebuilt from its first ad.r_low latent components (the loop bound of the
// reconstruction), and the scores of the attended tokens are kept for the moving
// average of the attention mass.
// SHARED: cross-head shared latent. The latents are [B][Lcap][r] (one row per token
// for every KV head) and BK/BV the decompression matrices [r][Hkv * d], of which KV
// head g uses columns g d .. g d + d - 1.
template <bool ADAPT, bool SHARED>
__device__ __forceinline__ void split_simt_body(const SplitArgs& a, const AdaptArgs& ad) {
  extern __shared__ float sm[];
  griddep_wait();
  griddep_launch_dependents();
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = a.d, r = a.r, G = a.G, T = kSimtTile;

  const int L = checked_len(a.seqlens, b, a.Lcap, a.max_seqlen, a.header, false);
  int t_begin, t_end;
  const int fset = split_range(s, L, a.n_visual, a.max_seqlen, a.chunk, &t_begin, &t_end);
  if (t_begin >= t_end) return;  // empty split: the merge skips it

  float* bk = sm;                 // [r][d]
  float* bv = bk + r * d;         // [r][d]
  float* qs = bv + r * d;         // [G][d]
  float* zk = qs + G * d;         // [T][r]
  float* zv = zk + T * r;         // [T][r]
  float* kv = zv + T * r;         // [T][d+1]
  float* sc = kv + T * (d + 1);   // [G][T] scores, then probabilities
  float* acc = sc + G * T;        // [G][d]
  float* ms = acc + G * d;        // [G] running max (log2 units)
  float* ls = ms + G;             // [G] running sum
  float* al = ls + G;             // [G] rescale factor of the current tile
  int* rk = reinterpret_cast<int*>(al + G);   // [T] rank of each token of the tile

  const size_t fac_base = ((size_t)fset * a.Hkv + g) * r * d;   // factor set, then head
  for (int i = tid; i < r * d; i += kSimtThreads) {
    size_t src = fac_base + i;
    if (SHARED) {   // row k of the decompression matrix, this head's column block
      const int k = i / d, c = i - k * d;
      src = (size_t)k * a.Hkv * d + (size_t)g * d + c;
    }
    bk[i] = load_io(a.BK, src, a.io_dtype);
    bv[i] = load_io(a.BV, src, a.io_dtype);
  }
  const size_t q_base = ((size_t)b * a.Hq + (size_t)g * G) * d;
  for (int i = tid; i < G * d; i += kSimtThreads) {
    qs[i] = load_io(a.q, q_base + i, a.io_dtype);
    acc[i] = 0.f;
  }
  if (tid < G) {
    ms[tid] = -CUDART_INF_F;
    ls[tid] = 0.f;
  }
  // token index base: the (batch row, KV head) block, or the batch row's shared rows
  const size_t row_base = SHARED ? (size_t)b * a.Lcap : ((size_t)b * a.Hkv + g) * (size_t)a.Lcap;
  const bool quant = a.latent_dtype == LRKV_I8 || a.latent_dtype == LRKV_E4M3;

  for (int t0 = t_begin; t0 < t_end; t0 += T) {
    const int n = min(T, t_end - t0);
    __syncthreads();
    for (int i = tid; i < T * r; i += kSimtThreads) {
      const int t = i / r;
      float vk = 0.f, vv = 0.f;
      if (t < n) {
        const size_t tok = row_base + t0 + t;
        const size_t e = tok * r + (i - t * r);
        vk = load_lat(a.ZK, e, a.latent_dtype);
        vv = load_lat(a.ZV, e, a.latent_dtype);
        if (quant) {
          vk *= a.SK[tok];
          vv *= a.SV[tok];
        }
      }
      zk[i] = vk;
      zv[i] = vv;
    }
    if (ADAPT) {
      for (int t = tid; t < T; t += kSimtThreads)
        rk[t] = (t < n && ad.imp[row_base + t0 + t] >= ad.tau) ? r : ad.r_low;
    }
    __syncthreads();
    // rebuilt key tile K = Z_K B_K (a warp shares one token, so the rank is uniform)
    for (int i = tid; i < T * d; i += kSimtThreads) {
      const int t = i / d, c = i - t * d;
      const int kr = ADAPT ? rk[t] : r;
      float sum = 0.f;
      for (int k = 0; k < kr; ++k) sum = fmaf(zk[t * r + k], bk[k * d + c], sum);
      kv[t * (d + 1) + c] = sum;
    }
    __syncthreads();
    // scores s[g][t] = q_g . K_t / sqrt(d), in log2 units; masked past the row end
    for (int pair = warp; pair < G * T; pair += kSimtThreads / 32) {
      const int gi = pair / T, t = pair - gi * T;
      float dot = 0.f;
      for (int c = lane; c < d; c += 32) dot = fmaf(qs[gi * d + c], kv[t * (d + 1) + c], dot);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (lane == 0) sc[gi * T + t] = (t < n) ? dot * a.scale_log2 : -CUDART_INF_F;
      if (ADAPT && lane == 0 && t < n)
        ad.scores[((size_t)b * a.Hq + (size_t)g * G + gi) * a.Lcap + t0 + t] = dot * a.scale_log2;
    }
    __syncthreads();
    // rebuilt value tile V = Z_V B_V (overwrites the key tile)
    for (int i = tid; i < T * d; i += kSimtThreads) {
      const int t = i / d, c = i - t * d;
      const int kr = ADAPT ? rk[t] : r;
      float sum = 0.f;
      for (int k = 0; k < kr; ++k) sum = fmaf(zv[t * r + k], bv[k * d + c], sum);
      kv[t * (d + 1) + c] = sum;
    }
    // online softmax, one thread per query head
    if (tid < G) {
      const int gi = tid;
      float mt = -CUDART_INF_F;
      for (int t = 0; t < n; ++t) mt = fmaxf(mt, sc[gi * T + t]);
      const float m_old = ms[gi];
      const float m_new = fmaxf(m_old, mt);
      const float alpha = exp2f(m_old - m_new);  // 0 on the first tile (m_old = -inf)
      float sum = 0.f;
      for (int t = 0; t < T; ++t) {
        const float p = (t < n) ? exp2f(sc[gi * T + t] - m_new) : 0.f;
        sc[gi * T + t] = p;
        sum += p;
      }
      ms[gi] = m_new;
      ls[gi] = ls[gi] * alpha + sum;
      al[gi] = alpha;
    }
    __syncthreads();
    for (int i = tid; i < G * d; i += kSimtThreads) {
      const int gi = i / d, c = i - gi * d;
      float v = acc[i] * al[gi];
      for (int t = 0; t < n; ++t) v = fmaf(sc[gi * T + t], kv[t * (d + 1) + c], v);
      acc[i] = v;
    }
  }
  __syncthreads();
  for (int i = tid; i < G * d; i += kSimtThreads) {
    const int gi = i / d, c = i - gi * d;
    const size_t h = (size_t)g * G + gi;
    a.o_part[(((size_t)b * a.Hq + h) * a.S + s) * d + c] = acc[i] / ls[gi];
  }
  if (tid < G) {
    const size_t h = (size_t)g * G + tid;
    a.lse_part[((size_t)b * a.Hq + h) * a.S + s] = (ms[tid] + log2f(ls[tid])) * CUDART_LN2_F;
  }
}

__global__ void __launch_bounds__(kSimtThreads) lrkv_split_simt(SplitArgs a) {
  split_simt_body<false, false>(a, AdaptArgs{});
}

__global__ void __launch_bounds__(kSimtThreads) lrkv_split_simt_adaptive(SplitArgs a, AdaptArgs ad) {
  split_simt_body<true, false>(a, ad);
}

__global__ void __launch_bounds__(kSimtThreads) lrkv_split_simt_shared(SplitArgs a) {
  split_simt_body<false, true>(a, AdaptArgs{});
}

// grid (ceil(max_seqlen / 256), Hkv, B), 256 threads: for every attended token of row
// b and KV head g, the attention mass (the softmax weights of the group's G query
// heads, from the kept log2 scores and the merged natural-log LSE) and the moving
// average importance = beta * importance + (1 - beta) * mass. Launched after the
// merge as a programmatic dependent: it waits for the merge (and so the split) first.
__global__ void __launch_bounds__(256) lrkv_mass_ema(MassArgs m) {
  griddep_wait();
  griddep_launch_dependents();
  const int g = blockIdx.y, b = blockIdx.z;
  const int t = blockIdx.x * 256 + threadIdx.x;
  const int L = checked_len(m.seqlens, b, m.Lcap, m.max_seqlen, m.header, false);
  if (t >= L) return;
  const int G = m.Hq / m.Hkv;
  float mass = 0.f;
  for (int gi = 0; gi < G; ++gi) {
    const size_t h = (size_t)b * m.Hq + (size_t)g * G + gi;
    mass += exp2f(m.scores[h * m.Lcap + t] - m.lse[h] * CUDART_L2E_F);
  }
  float* p = m.imp + ((size_t)b * m.Hkv + g) * m.Lcap + t;
  *p = m.beta * *p + (1.f - m.beta) * mass;
}

// grid (B * Hq), 128 threads (one per output dimension, d <= 128), S floats of dynamic
// shared memory. out[b][h] = sum_s exp(lse_s - LSE) o_s over the non-empty splits of
// row b, with LSE = log sum_s exp(lse_s) (the log-sum-exp merge of Flash Decoding); an
// empty row gives 0 and -inf. The loads that do not depend on the row's length (the
// first split LSEs and partials) are issued before it is read; warp 0 turns the split
// LSEs into weights once; every thread sums its dimension with four partial sums.
// Launched as a programmatic dependent of the split kernel: it waits for the split
// grid's results before reading them.
__global__ void __launch_bounds__(128) lrkv_merge(MergeArgs a) {
  extern __shared__ float wsm[];   // [S] split weights
  griddep_wait();
  griddep_launch_dependents();
  const int bh = blockIdx.x;
  const int b = bh / a.Hq;
  const int tid = threadIdx.x, lane = tid & 31;
  const float* lse = a.lse_part + (size_t)bh * a.S;
  const float* o = a.o_part + (size_t)bh * a.S * a.d;
  constexpr int kPre = 4;
  const bool active = tid < a.d;
  float lse0 = -CUDART_INF_F;
  if (tid < 32 && lane < a.S) lse0 = lse[lane];
  float opre[kPre];
#pragma unroll
  for (int k = 0; k < kPre; ++k) opre[k] = (active && k < a.S) ? o[(size_t)k * a.d + tid] : 0.f;
  const int L = checked_len(a.seqlens, b, a.Lcap, a.max_seqlen, a.header,
                            (bh % a.Hq) == 0 && tid == 0);
  // the split size: the plan's, or the one the tensor-core split kernel chose
  const int chunk = a.device_chunk ? (int)*reinterpret_cast<volatile uint32_t*>(a.header + kChunkWord)
                                   : a.chunk;
  // the row's non-empty splits, in order: the first n1 are physical splits 0..n1-1
  // (the visual segment, or the whole row), the rest start at physical split sv
  // (the text segment of modality-separated factors)
  int ns, n1, sv = 0;
  if (a.n_visual > 0) {
    sv = visual_splits(a.n_visual, a.max_seqlen, chunk);
    n1 = (min(L, a.n_visual) + chunk - 1) / chunk;
    ns = min(a.S, n1 + (max(0, L - a.n_visual) + chunk - 1) / chunk);
  } else {
    ns = min(a.S, (L + chunk - 1) / chunk);
    n1 = ns;
  }
  auto phys = [&](int j) { return j < n1 ? j : sv + (j - n1); };
  // the prefetched values are physical splits 0..: reload the ones past n1
  if (tid < 32 && lane >= n1 && lane < ns) lse0 = lse[phys(lane)];
#pragma unroll
  for (int k = 0; k < kPre; ++k)
    if (active && k >= n1 && k < ns) opre[k] = o[(size_t)phys(k) * a.d + tid];
  if (tid < 32) {
    float mx = lane < ns ? lse0 : -CUDART_INF_F;
    for (int s = lane + 32; s < ns; s += 32) mx = fmaxf(mx, lse[phys(s)]);
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, k));
    float tot = lane < ns ? expf(lse0 - mx) : 0.f;
    for (int s = lane + 32; s < ns; s += 32) tot += expf(lse[phys(s)] - mx);
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, k);
    const float LSE = (ns > 0) ? mx + logf(tot) : -CUDART_INF_F;
    if (lane < ns) wsm[lane] = expf(lse0 - LSE);
    for (int s = lane + 32; s < ns; s += 32) wsm[s] = expf(lse[phys(s)] - LSE);
    if (a.lse_out && lane == 0) a.lse_out[bh] = LSE;
  }
  __syncthreads();
  if (!active) return;
  float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int k = 0; k < kPre; ++k)
    if (k < ns) v[k] = wsm[k] * opre[k];
  int s = kPre;
  for (; s + 4 <= ns; s += 4) {
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = fmaf(wsm[s + k], o[(size_t)phys(s + k) * a.d + tid], v[k]);
  }
  for (; s < ns; ++s) v[0] = fmaf(wsm[s], o[(size_t)phys(s) * a.d + tid], v[0]);
  const float r = (v[0] + v[1]) + (v[2] + v[3]);
  const size_t oi = (size_t)bh * a.d + tid;
  if (a.io_dtype == LRKV_F32) static_cast<float*>(a.out)[oi] = r;
  else static_cast<__nv_bfloat16*>(a.out)[oi] = __float2bfloat16_rn(r);
}

// grid (B), 1024 threads: one warp per (KV head, K|V) row of batch row b, two rows
// per pass with both rows' loads issued before any store (the kernel is latency-bound).
// Rows are written at slot seqlens[b]; int8 / e4m3 rows get a per-row absmax scale.
template <int LAT>
__device__ __forceinline__ void append_row(const AppendArgs& a, int b, int row, int slot, int lane,
                                           const float (&z)[8]) {
  const int r = a.r;
  const int g = row >> 1;
  const bool is_v = row & 1;
  void* dst = is_v ? a.ZV : a.ZK;
  float* sdst = is_v ? a.SV : a.SK;
  const size_t tok = ((size_t)b * a.Hkv + g) * (size_t)a.Lcap + slot;
  const size_t out_base = tok * r;
  if (LAT == LRKV_F32 || LAT == LRKV_BF16) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = lane + 32 * k;
      if (i < r) {
        if (LAT == LRKV_F32) static_cast<float*>(dst)[out_base + i] = z[k];
        else static_cast<__nv_bfloat16*>(dst)[out_base + i] = __float2bfloat16_rn(z[k]);
      }
    }
    return;
  }
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (lane + 32 * k < r) amax = fmaxf(amax, fabsf(z[k]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const bool i8 = LAT == LRKV_I8;
  const float scale = (amax == 0.f) ? 1.f : __fdiv_rn(amax, i8 ? 127.f : 448.f);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int i = lane + 32 * k;
    if (i < r) {
      const float v = __fdiv_rn(z[k], scale);
      if (i8) {
        const int c = min(127, max(-127, __float2int_rn(v)));
        static_cast<int8_t*>(dst)[out_base + i] = static_cast<int8_t>(c);
      } else {
        static_cast<__nv_fp8_storage_t*>(dst)[out_base + i] =
            __nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
      }
    }
  }
  if (lane == 0) sdst[tok] = scale;
}

template <int LAT>
__global__ void __launch_bounds__(1024) lrkv_append_kernel(AppendArgs a) {
  griddep_wait();
  griddep_launch_dependents();
  const int b = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int slot = a.seqlens[b];
  if (slot < 0 || slot >= a.Lcap) {
    if (threadIdx.x == 0) atomicOr(a.header + kStatusWord, LRKV_STATUS_APPEND_FULL);
    return;
  }
  const int r = a.r;   // <= 256: at most eight elements a lane
  const int nrows = 2 * a.Hkv;
  for (int row0 = warp; row0 < nrows; row0 += 2 * nwarps) {
    const int row1 = row0 + nwarps;
    float z0[8], z1[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = lane + 32 * k;
      z0[k] = 0.f;
      z1[k] = 0.f;
      if (i < r) {
        const void* s0 = (row0 & 1) ? a.zv_new : a.zk_new;
        z0[k] = load_io(s0, ((size_t)b * a.Hkv + (row0 >> 1)) * r + i, a.io_dtype);
        if (row1 < nrows) {
          const void* s1 = (row1 & 1) ? a.zv_new : a.zk_new;
          z1[k] = load_io(s1, ((size_t)b * a.Hkv + (row1 >> 1)) * r + i, a.io_dtype);
        }
      }
    }
    append_row<LAT>(a, b, row0, slot, lane, z0);
    if (row1 < nrows) append_row<LAT>(a, b, row1, slot, lane, z1);
  }
  __syncthreads();
  if (threadIdx.x == 0) a.seqlens[b] = slot + 1;
}


// Fused latent projection + append (the step before decode attention): for every
// batch row b and KV head g, the new token's latents z_K = x_b A_K,g and
// z_V = x_b A_V,g ("WSVD: Weighted Low-Rank Approximation for Fast and Efficient
// Execution of Low-Precision Vision-Language Models", section 2.A: the cached latent
// is the token's hidden state times the down factor), accumulated in fp32 and
// written at slot seqlens[b] exactly as lrkv_append writes a row (bf16 RNE, or int8 /
// e4m3 codes with a per-row absmax scale). The last CTA to finish advances seqlens.
// grid (2 Hkv, nsplit): CTA = (KV head, K | V, slice of the hidden size), 256
// threads. One thread issues a bulk copy of the CTA's factor rows into shared memory
// (they are contiguous in A) while the others stage a block of rows of x as fp32
// (16-byte loads where x allows), so the factor crosses HBM once and every pass over
// the batch reads both operands from shared memory. A factor row (r columns) is read
// by tpr lanes, 8 columns each (tpr = r / 8 rounded up to a power of two); the other
// lanes of the warp and the 8 warps take other rows. Each thread keeps 8 batch rows x
// 8 columns of fp32 sums in packed pairs (fma.rn.f32x2). The sums are reduced over the
// lanes that share columns (a butterfly in which each step halves the values a lane
// holds), then over the warps in a fixed order. With nsplit > 1 every CTA writes its
// partial sums to the workspace and the last CTA of a KV head adds them in a fixed
// order and writes that head's rows (deterministic). A slice larger than the
// shared-memory budget is taken in chunks, copied again for every pass of 8 rows.
constexpr int kProjThreads = 256;
constexpr int kProjWarps = kProjThreads / 32;
constexpr int kProjRows = 8;              // batch rows per pass
constexpr int kProjMaxChunk = 1024;       // factor rows staged at a time, at most
constexpr int kProjABytes = 64 * 1024;    // shared-memory budget for factor rows
constexpr int kProjSmemTarget = 110 * 1024;  // two CTAs per SM
constexpr int kProjMinSpan = 64;          // fewest hidden-size rows a CTA takes when splitting
constexpr int kProjMaxCluster = 8;        // CTAs sharing one factor: one portable cluster
constexpr int kProjClusterBytes = 32 * 1024;  // a CTA's partial sums [B][r] must fit this

// batch rows per block of the grid's z dimension (a multiple of 8)
__host__ __device__ inline int proj_batch_rows(int B, int nbz) {
  return ((B + nbz - 1) / nbz + 7) / 8 * 8;
}

// hidden-size rows per CTA: a multiple of 8, so 16-byte loads of x stay aligned
__host__ __device__ inline int proj_dspan(int D, int ns) { return ((D + ns - 1) / ns + 7) / 8 * 8; }

// factor rows a CTA stages at a time (a multiple of 8), for row width r, element size e
__host__ __device__ inline int proj_chunk_rows(int r, int e, int dspan) {
  const int cap = min(kProjMaxChunk, kProjABytes / (r * e)) / 8 * 8;
  return max(8, min(cap, dspan));
}

// batch rows of x staged at once (a multiple of 8): as many as the budget holds when
// the slice is resident, 8 when it is taken in chunks
__host__ __device__ inline int proj_batch_block(int B, int r, int e, int cr, bool chunked, int ns) {
  const int b8 = (B + 7) / 8 * 8;
  if (chunked) return 8;
  const long long room = (long long)kProjSmemTarget - 16 - (long long)cr * r * e -
                         (long long)(kProjWarps + 1) * kProjRows * r * 4 -
                         (ns > 1 ? (long long)B * r * 4 : 0);
  const int rows = (int)(room > 0 ? room / (cr * 4) : 0) / 8 * 8;
  return max(8, min(rows, b8));
}

// dynamic shared memory: barrier, factor rows, x rows, the warps' partial sums, sums,
// and with a split hidden size this CTA's partial sums of every batch row
__host__ __device__ inline size_t proj_smem_bytes(int B, int r, int e, int cr, int bblk, int ns) {
  return 16 + (size_t)cr * r * e +
         sizeof(float) * ((size_t)bblk * cr + (size_t)(kProjWarps + 1) * kProjRows * r +
                          (ns > 1 ? (size_t)B * r : 0));
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// fp32 at a shared-memory address of another CTA of the cluster
__device__ __forceinline__ float ld_cluster_f32(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

template <int LAT>
__device__ __forceinline__ void proj_write_rows(const ProjArgs& pa, int row, int b0, int nb,
                                                const float* zs, int lane, int warp) {
  const AppendArgs& a = pa.app;
  for (int bb = warp; bb < nb; bb += kProjWarps) {
    const int b = b0 + bb;
    const int slot = a.seqlens[b];
    if (slot < 0 || slot >= a.Lcap) {
      if (lane == 0) atomicOr(a.header + kStatusWord, LRKV_STATUS_APPEND_FULL);
      continue;
    }
    float zz[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) zz[e] = (lane + 32 * e < a.r) ? zs[bb * a.r + lane + 32 * e] : 0.f;
    append_row<LAT>(a, b, row, slot, lane, zz);
  }
}

// 8 consecutive factor columns as 4 packed fp32 pairs, from shared memory
template <int IO>
__device__ __forceinline__ void proj_row8(const char* p, uint64_t (&a2)[4]) {
  if constexpr (IO == LRKV_F32) {
    const uint4 w0 = reinterpret_cast<const uint4*>(p)[0];
    const uint4 w1 = reinterpret_cast<const uint4*>(p)[1];
    a2[0] = pack2(__uint_as_float(w0.x), __uint_as_float(w0.y));
    a2[1] = pack2(__uint_as_float(w0.z), __uint_as_float(w0.w));
    a2[2] = pack2(__uint_as_float(w1.x), __uint_as_float(w1.y));
    a2[3] = pack2(__uint_as_float(w1.z), __uint_as_float(w1.w));
  } else {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j)   // bf16 -> fp32 is exact: the bits move up
      a2[j] = pack2(__uint_as_float(u[j] << 16), __uint_as_float(u[j] & 0xffff0000u));
  }
}

// xs[row][i] = x[b0 + row][d0 + i] as fp32 for row < srows, i < cr; zero past nrows
// rows or dn columns. vec: x rows and d0 are 16-byte aligned and dn, cr are multiples
// of 8, so every thread moves 16-byte words, eight in flight.
template <int IO>
__device__ __forceinline__ void proj_stage_x(float* xs, const void* x, int b0, int nrows,
                                             int srows, int D, int d0, int dn, int cr, int t,
                                             bool vec) {
  constexpr int E = IO == LRKV_F32 ? 4 : 2;
  constexpr int V = 16 / E;                          // elements a 16-byte word
  const char* xb = static_cast<const char*>(x);
  if (vec) {
    const int wpr = cr / V, total = srows * wpr;
    for (int w0 = t; w0 < total; w0 += 8 * kProjThreads) {
      uint4 buf[8];
      int row = w0 / wpr, iw = w0 - row * wpr;       // advanced by kProjThreads words
      const int drow = kProjThreads / wpr, diw = kProjThreads - drow * wpr;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int w = w0 + k * kProjThreads, i = iw * V;
        buf[k] = make_uint4(0u, 0u, 0u, 0u);
        if (w < total && row < nrows && i < dn)
          buf[k] = __ldg(reinterpret_cast<const uint4*>(xb + ((size_t)(b0 + row) * D + d0 + i) * E));
        row += drow;
        iw += diw;
        if (iw >= wpr) { iw -= wpr; ++row; }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int w = w0 + k * kProjThreads;
        if (w >= total) continue;
        // xs is [row][cr] and a row holds wpr words: word w starts at element w * V
        float4* o = reinterpret_cast<float4*>(xs + (size_t)w * V);
        if constexpr (IO == LRKV_F32) {
          o[0] = make_float4(__uint_as_float(buf[k].x), __uint_as_float(buf[k].y),
                             __uint_as_float(buf[k].z), __uint_as_float(buf[k].w));
        } else {
          o[0] = make_float4(__uint_as_float(buf[k].x << 16), __uint_as_float(buf[k].x & 0xffff0000u),
                             __uint_as_float(buf[k].y << 16), __uint_as_float(buf[k].y & 0xffff0000u));
          o[1] = make_float4(__uint_as_float(buf[k].z << 16), __uint_as_float(buf[k].z & 0xffff0000u),
                             __uint_as_float(buf[k].w << 16), __uint_as_float(buf[k].w & 0xffff0000u));
        }
      }
    }
  } else {
    const int total = srows * cr;
    for (int e0 = t; e0 < total; e0 += 8 * kProjThreads) {
      float v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int e = e0 + k * kProjThreads;
        const int row = e / cr, i = e - row * cr;
        v[k] = (e < total && row < nrows && i < dn) ? load_io(x, (size_t)(b0 + row) * D + d0 + i, IO) : 0.f;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (e0 + k * kProjThreads < total) xs[e0 + k * kProjThreads] = v[k];
    }
  }
}

template <int LAT, int IO>
__global__ void __launch_bounds__(kProjThreads, 2) lrkv_project_append_kernel(ProjArgs pa) {
  constexpr int E = IO == LRKV_F32 ? 4 : 2;          // bytes an element
  constexpr uint64_t kWaitNs = 1000000000ull;        // bounded waits: one second
  extern __shared__ __align__(16) unsigned char proj_smem[];
  __shared__ int abort_flag;
  const AppendArgs& a = pa.app;
  const int r = a.r;
  const int gk = blockIdx.x, g = gk >> 1, kv = gk & 1, sp = blockIdx.y, ns = pa.nsplit;
  // this CTA's block of batch rows [Blo, Blo + B) (blockIdx.z; may be empty)
  const int Bb = proj_batch_rows(a.B, gridDim.z);
  const int Blo = min(a.B, (int)blockIdx.z * Bb), B = min(a.B, Blo + Bb) - Blo;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int D = pa.d_model;
  const int dspan = proj_dspan(D, ns);
  const int dlo = min(D, sp * dspan), dhi = min(D, dlo + dspan);
  const int cr = proj_chunk_rows(r, E, dspan);
  const int nchunks = max(1, (dhi - dlo + cr - 1) / cr);
  const bool resident = nchunks == 1;
  // the launch's shared memory is sized for the longest slice, so the block of batch
  // rows depends on that slice, not on this CTA's (the last one may be shorter)
  const int bblk = proj_batch_block(Bb, r, E, cr, min(dspan, D) > cr, ns);
  const bool vec = (D % 8 == 0) && ((reinterpret_cast<uintptr_t>(pa.x) & 15) == 0);
  const uint32_t bar = smem_addr(proj_smem);
  char* As = reinterpret_cast<char*>(proj_smem + 16);              // [row][r] as in A
  float* xs = reinterpret_cast<float*>(As + (size_t)cr * r * E);   // [batch row][row]
  float* red = xs + (size_t)bblk * cr;                             // [warp][batch row][col]
  float* zs = red + kProjWarps * kProjRows * r;                    // [batch row][col]
  float* zc = zs + kProjRows * r;              // ns > 1: this CTA's partial sums [Bb][r]
  const char* A = static_cast<const char*>(kv ? pa.AV : pa.AK) + (size_t)g * D * r * E;
  const size_t row_bytes = (size_t)r * E;
  if (t == 0) {
    abort_flag = 0;
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();
  uint32_t copies = 0;     // bulk copies issued so far (the barrier's phase count)
  bool timed_out = false;
  auto issue = [&](int d0, int dn) {
    if (t == 0 && dn > 0) {
      mbar_arrive_expect_tx(bar, (uint32_t)(dn * row_bytes));
      bulk_load(smem_addr(As), A + (size_t)d0 * row_bytes, (uint32_t)(dn * row_bytes), bar);
    }
    if (dn > 0) ++copies;
  };
  if (resident) issue(dlo, dhi - dlo);

  int tpr = 1;
  while (tpr * 8 < r) tpr <<= 1;
  const int spw = 32 / tpr, c0 = (lane & (tpr - 1)) * 8;
  const int nslots = kProjWarps * spw, slot = warp * spw + lane / tpr;
  const bool active = c0 < r;

  for (int blk0 = Blo; blk0 < Blo + B; blk0 += bblk) {
    const int nblk = min(bblk, Blo + B - blk0);
    for (int g8 = 0; g8 < nblk; g8 += kProjRows) {
      const int b0 = blk0 + g8, nb = min(kProjRows, nblk - g8);
      uint64_t acc[kProjRows][4];
#pragma unroll
      for (int bb = 0; bb < kProjRows; ++bb)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[bb][j] = 0ull;
      for (int ch = 0; ch < nchunks; ++ch) {
        const int d0 = dlo + ch * cr, dn = min(cr, dhi - d0);
        if (!resident || g8 == 0) {
          // resident slice: the block's x rows once; chunked: this pass's rows per chunk
          __syncthreads();                       // earlier readers of xs / As are done
          if (!resident) issue(d0, dn);
          if (resident) proj_stage_x<IO>(xs, pa.x, blk0, nblk, bblk, D, d0, dn, cr, t, vec);
          else proj_stage_x<IO>(xs, pa.x, b0, nb, kProjRows, D, d0, dn, cr, t, vec);
          __syncthreads();
          if (dn > 0 && !mbar_wait(bar, (copies - 1) & 1, &abort_flag, kWaitNs)) timed_out = true;
        }
        const float* xg = xs + (size_t)(resident ? g8 : 0) * cr;
        if (active) {
          for (int i = slot; i < dn; i += nslots) {
            uint64_t a2[4];
            proj_row8<IO>(As + (size_t)i * row_bytes + (size_t)c0 * E, a2);
#pragma unroll
            for (int bb = 0; bb < kProjRows; ++bb) {
              const float xv = xg[bb * cr + i];
              const uint64_t x2 = pack2(xv, xv);
#pragma unroll
              for (int j = 0; j < 4; ++j) acc[bb][j] = ffma2p(x2, a2[j], acc[bb][j]);
            }
          }
        }
      }
      // lanes that share columns: each butterfly step sends half of the values a lane
      // holds to its partner and keeps the other half, so after s steps a lane holds
      // 64 / 2^s sums; which ones depends on the lane's bits (index base `off`)
      float v[64];
#pragma unroll
      for (int bb = 0; bb < kProjRows; ++bb)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack2(acc[bb][j]);
          v[bb * 8 + 2 * j] = f.x;
          v[bb * 8 + 2 * j + 1] = f.y;
        }
      int off = 0, held = 64;
#pragma unroll
      for (int s = 0; s < 5; ++s) {
        const int h = 32 >> s;                   // values sent (and kept) in this step
        const int o = tpr << s;
        if (o < 32) {
          const bool hi = lane & o;
#pragma unroll
          for (int j = 0; j < h; ++j) {
            const float send = hi ? v[j] : v[j + h];
            const float keep = hi ? v[j + h] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
          }
          if (hi) off += h;
          held = h;
        }
      }
      if (active) {
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          if (j < held) {
            const int idx = off + j, bb = idx >> 3, c = idx & 7;
            red[(warp * kProjRows + bb) * r + c0 + c] = v[j];
          }
        }
      }
      __syncthreads();
      for (int idx = t; idx < nb * r; idx += kProjThreads) {
        const int bb = idx / r, k = idx - bb * r;
        float z = 0.f;
#pragma unroll
        for (int w = 0; w < kProjWarps; ++w) z += red[(w * kProjRows + bb) * r + k];
        if (ns == 1) zs[idx] = z;
        else zc[(size_t)(b0 - Blo) * r + idx] = z;
      }
      __syncthreads();
      if (ns == 1) proj_write_rows<LAT>(pa, 2 * g + kv, b0, nb, zs, lane, warp);
    }
  }
  if (timed_out) {
    // results are invalid; make sure no copy still writes this CTA's shared memory
    if (t == 0) atomicOr(a.header + kStatusWord, LRKV_STATUS_TIMEOUT);
    abort_flag = 0;
    mbar_wait(bar, (copies - 1) & 1, &abort_flag, kWaitNs);
  }
  if (ns > 1) {
    // the ns CTAs of this factor form one cluster: once every partial is in shared
    // memory, CTA c adds the ns partials of its share of the batch rows (read from the
    // other CTAs' shared memory, always in rank order) and writes those rows
    cluster_sync_all();
    const uint32_t crank = cluster_rank();
    const int per = (B + ns - 1) / ns;
    const int blo = min(B, (int)crank * per), bhi = min(B, blo + per);   // within the block
    const uint32_t zc_addr = smem_addr(zc);
    for (int l0 = blo; l0 < bhi; l0 += kProjRows) {
      const int nb = min(kProjRows, bhi - l0), b0 = Blo + l0;
      __syncthreads();
      for (int idx = t; idx < nb * r; idx += kProjThreads) {
        const uint32_t off = (uint32_t)(((size_t)l0 * r + idx) * sizeof(float));
        float z = 0.f;
        for (int q = 0; q < ns; ++q) z += ld_cluster_f32(zc_addr + off, (uint32_t)q);
        zs[idx] = z;
      }
      __syncthreads();
      proj_write_rows<LAT>(pa, 2 * g + kv, b0, nb, zs, lane, warp);
    }
    cluster_sync_all();   // no CTA leaves while another still reads its partial sums
  }
  // the last writer advances every valid row's length (all writers have read it)
  __syncthreads();
  if (t == 0) {
    __threadfence();
    const unsigned writers = gridDim.x * gridDim.y * gridDim.z;
    const unsigned prev = atomicAdd(a.header + kProjCounter, 1u);
    if (prev == writers - 1) {
      __threadfence();
      for (int b = 0; b < a.B; ++b) {
        const int slot = a.seqlens[b];
        if (slot >= 0 && slot < a.Lcap) a.seqlens[b] = slot + 1;
      }
      atomicExch(a.header + kProjCounter, 0u);
      __threadfence();
    }
  }
}

}  // namespace

size_t simt_smem_bytes(int r, int d, int G) {
  const int T = kSimtTile;
  return sizeof(float) * ((size_t)2 * r * d + 2 * (size_t)G * d + 2 * (size_t)T * r +
                          (size_t)T * (d + 1) + (size_t)G * T + 3 * (size_t)G + (size_t)T);
}

cudaError_t launch_split_simt(const SplitArgs& a, const Plan& p, cudaStream_t st) {
  static int configured_smem = 0;
  if (p.smem > configured_smem) {
    cudaError_t e = cudaFuncSetAttribute(lrkv_split_simt,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem);
    if (e != cudaSuccess) return e;
    configured_smem = p.smem;
  }
  dim3 grid(a.S, a.Hkv, a.B);
  return launch_pdl(lrkv_split_simt, grid, dim3(kSimtThreads), (size_t)p.smem, st, a);
}

cudaError_t launch_split_simt_adaptive(const SplitArgs& a, const AdaptArgs& ad, const Plan& p,
                                       cudaStream_t st) {
  static int configured_smem = 0;
  if (p.smem > configured_smem) {
    cudaError_t e = cudaFuncSetAttribute(lrkv_split_simt_adaptive,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem);
    if (e != cudaSuccess) return e;
    configured_smem = p.smem;
  }
  dim3 grid(a.S, a.Hkv, a.B);
  return launch_pdl(lrkv_split_simt_adaptive, grid, dim3(kSimtThreads), (size_t)p.smem, st, a, ad);
}

cudaError_t launch_split_simt_shared(const SplitArgs& a, const Plan& p, cudaStream_t st) {
  static int configured_smem = 0;
  if (p.smem > configured_smem) {
    cudaError_t e = cudaFuncSetAttribute(lrkv_split_simt_shared,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem);
    if (e != cudaSuccess) return e;
    configured_smem = p.smem;
  }
  dim3 grid(a.S, a.Hkv, a.B);
  return launch_pdl(lrkv_split_simt_shared, grid, dim3(kSimtThreads), (size_t)p.smem, st, a);
}

cudaError_t launch_mass_ema(const MassArgs& m, cudaStream_t st) {
  const int tiles = std::max(1, (m.max_seqlen + 255) / 256);
  return launch_pdl(lrkv_mass_ema, dim3(tiles, m.Hkv, m.B), dim3(256), 0, st, m);
}

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)a.S * sizeof(float);
  static size_t configured = 48 * 1024;
  if (smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(lrkv_merge, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  return launch_pdl(lrkv_merge, dim3(a.B * a.Hq), dim3(128), smem, st, a);
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t st) {
  const int threads = 32 * std::min(32, std::max(1, 2 * a.Hkv));
  switch (a.latent_dtype) {
    case LRKV_F32: return launch_pdl(lrkv_append_kernel<LRKV_F32>, dim3(a.B), dim3(threads), 0, st, a);
    case LRKV_BF16: return launch_pdl(lrkv_append_kernel<LRKV_BF16>, dim3(a.B), dim3(threads), 0, st, a);
    case LRKV_I8: return launch_pdl(lrkv_append_kernel<LRKV_I8>, dim3(a.B), dim3(threads), 0, st, a);
    default: return launch_pdl(lrkv_append_kernel<LRKV_E4M3>, dim3(a.B), dim3(threads), 0, st, a);
  }
}

template <int LAT, int IO>
cudaError_t launch_project_typed(const ProjArgs& a, cudaStream_t st) {
  const int e = IO == LRKV_F32 ? 4 : 2;
  const int dspan = proj_dspan(a.d_model, a.nsplit);
  const int cr = proj_chunk_rows(a.app.r, e, dspan);
  // the largest slice decides (the last slice is shorter, never longer)
  const bool chunked = std::min(dspan, a.d_model) > cr;
  // batch blocks over the grid's z dimension while the (factor, slice) CTAs leave SMs
  // idle: about two CTAs per SM in all, each with at least 8 rows
  const int ctas = 2 * a.app.Hkv * a.nsplit;
  const int nbz = std::max(1, std::min((a.app.B + 7) / 8, 2 * num_sms() / ctas));
  const int Bb = proj_batch_rows(a.app.B, nbz);
  const size_t smem = proj_smem_bytes(Bb, a.app.r, e, cr,
                                      proj_batch_block(Bb, a.app.r, e, cr, chunked, a.nsplit),
                                      a.nsplit);
  static size_t configured = 48 * 1024;
  if (smem > configured) {
    cudaError_t err = cudaFuncSetAttribute(lrkv_project_append_kernel<LAT, IO>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    configured = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.app.Hkv, a.nsplit, nbz);
  cfg.blockDim = dim3(kProjThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;   // the CTAs of one factor
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = a.nsplit;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, lrkv_project_append_kernel<LAT, IO>, a);
}

template <int LAT>
cudaError_t launch_project_lat(const ProjArgs& a, cudaStream_t st) {
  return a.app.io_dtype == LRKV_F32 ? launch_project_typed<LAT, LRKV_F32>(a, st)
                                    : launch_project_typed<LAT, LRKV_BF16>(a, st);
}

cudaError_t launch_project_append(const ProjArgs& a, cudaStream_t st) {
  switch (a.app.latent_dtype) {
    case LRKV_F32: return launch_project_lat<LRKV_F32>(a, st);
    case LRKV_BF16: return launch_project_lat<LRKV_BF16>(a, st);
    case LRKV_I8: return launch_project_lat<LRKV_I8>(a, st);
    default: return launch_project_lat<LRKV_E4M3>(a, st);
  }
}

int project_nsplit(int Hkv, int B, int r, int d_model, int io_bytes, size_t workspace_bytes) {
  (void)workspace_bytes;   // the partial sums live in the cluster's shared memory
  // the CTAs of one factor form a cluster and keep every batch row's partial sums
  if ((size_t)B * r * sizeof(float) > (size_t)kProjClusterBytes) return 1;
  // one wave of two CTAs per SM, or more CTAs if a slice would not fit in shared
  // memory; at most one portable cluster, each CTA with at least kProjMinSpan rows
  const int cap = proj_chunk_rows(r, io_bytes, d_model);
  int ns = std::max(std::max(1, 2 * num_sms() / (2 * Hkv)), (d_model + cap - 1) / cap);
  ns = std::min(ns, kProjMaxCluster);
  ns = std::min(ns, std::max(1, d_model / kProjMinSpan));
  return std::max(1, ns);
}

}  // namespace lrkv
