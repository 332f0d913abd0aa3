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

#include "lrkv_internal.h"

namespace lrkv {
namespace {

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
__global__ void __launch_bounds__(kSimtThreads) lrkv_split_simt(SplitArgs a) {
  extern __shared__ float sm[];
  griddep_wait();
  griddep_launch_dependents();
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = a.d, r = a.r, G = a.G, T = kSimtTile;

  const int L = checked_len(a.seqlens, b, a.Lcap, a.max_seqlen, a.header, false);
  const int t_begin = s * a.chunk;
  const int t_end = min(L, t_begin + a.chunk);
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

  const size_t fac_base = (size_t)g * r * d;
  for (int i = tid; i < r * d; i += kSimtThreads) {
    bk[i] = load_io(a.BK, fac_base + i, a.io_dtype);
    bv[i] = load_io(a.BV, fac_base + i, a.io_dtype);
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
  const size_t row_base = ((size_t)b * a.Hkv + g) * (size_t)a.Lcap;  // token index base
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
    __syncthreads();
    // rebuilt key tile K = Z_K B_K
    for (int i = tid; i < T * d; i += kSimtThreads) {
      const int t = i / d, c = i - t * d;
      float sum = 0.f;
      for (int k = 0; k < r; ++k) sum = fmaf(zk[t * r + k], bk[k * d + c], sum);
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
    }
    __syncthreads();
    // rebuilt value tile V = Z_V B_V (overwrites the key tile)
    for (int i = tid; i < T * d; i += kSimtThreads) {
      const int t = i / d, c = i - t * d;
      float sum = 0.f;
      for (int k = 0; k < r; ++k) sum = fmaf(zv[t * r + k], bv[k * d + c], sum);
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
  const int ns = min(a.S, (L + a.chunk - 1) / a.chunk);
  if (tid < 32) {
    float mx = lane < ns ? lse0 : -CUDART_INF_F;
    for (int s = lane + 32; s < ns; s += 32) mx = fmaxf(mx, lse[s]);
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, k));
    float tot = lane < ns ? expf(lse0 - mx) : 0.f;
    for (int s = lane + 32; s < ns; s += 32) tot += expf(lse[s] - mx);
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, k);
    const float LSE = (ns > 0) ? mx + logf(tot) : -CUDART_INF_F;
    if (lane < ns) wsm[lane] = expf(lse0 - LSE);
    for (int s = lane + 32; s < ns; s += 32) wsm[s] = expf(lse[s] - LSE);
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
    for (int k = 0; k < 4; ++k) v[k] = fmaf(wsm[s + k], o[(size_t)(s + k) * a.d + tid], v[k]);
  }
  for (; s < ns; ++s) v[0] = fmaf(wsm[s], o[(size_t)s * a.d + tid], v[0]);
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
// grid (2 Hkv, nsplit): CTA = (KV head, K | V, slice of the hidden size); 256 threads
// = column k (t % r) x row group (t / r). Rows of x are staged in shared memory 256
// columns at a time, 16 batch rows per pass. With nsplit > 1 every CTA writes its
// partial sums to the workspace and the last CTA of a KV head adds them in a fixed
// order and writes that head's rows (deterministic).
constexpr int kProjThreads = 256;
constexpr int kProjRows = 16;     // batch rows per pass (accumulators a thread)
constexpr int kProjChunk = 256;   // columns of x staged per step
constexpr int kProjMaxHeads = 60; // per-head counters live in header words 4..63

template <int LAT>
__device__ __forceinline__ void proj_write_rows(const ProjArgs& pa, int row, int b0, int nb,
                                                const float* zs, int lane, int warp) {
  const AppendArgs& a = pa.app;
  for (int bb = warp; bb < nb; bb += kProjThreads / 32) {
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

template <int LAT>
__global__ void __launch_bounds__(kProjThreads) lrkv_project_append_kernel(ProjArgs pa) {
  __shared__ float xs[kProjRows * kProjChunk];
  __shared__ float red[kProjThreads * kProjRows];   // [row group][batch row][column]
  __shared__ float zs[kProjRows * 256];
  griddep_wait();
  griddep_launch_dependents();
  const AppendArgs& a = pa.app;
  const int gk = blockIdx.x, g = gk >> 1, kv = gk & 1, sp = blockIdx.y, ns = pa.nsplit;
  const int r = a.r, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int ngr = kProjThreads / r;                 // row groups
  const int k = t % r, rg = t / r;
  const bool active = rg < ngr;
  const int D = pa.d_model;
  const int dspan = ((D + ns - 1) / ns + kProjChunk - 1) / kProjChunk * kProjChunk;
  const int dlo = min(D, sp * dspan), dhi = min(D, dlo + dspan);
  const void* A = kv ? pa.AV : pa.AK;
  const size_t abase = (size_t)g * D * r;
  for (int b0 = 0; b0 < a.B; b0 += kProjRows) {
    const int nb = min(kProjRows, a.B - b0);
    float acc[kProjRows];
#pragma unroll
    for (int bb = 0; bb < kProjRows; ++bb) acc[bb] = 0.f;
    for (int d0 = dlo; d0 < dhi; d0 += kProjChunk) {
      __syncthreads();
      for (int idx = t; idx < kProjRows * kProjChunk; idx += kProjThreads) {
        const int bb = idx / kProjChunk, dd = idx - bb * kProjChunk;
        xs[idx] = (bb < nb && d0 + dd < dhi) ? load_io(pa.x, (size_t)(b0 + bb) * D + d0 + dd, a.io_dtype) : 0.f;
      }
      __syncthreads();
      if (active) {
        const int dn = min(kProjChunk, dhi - d0);
        int i = rg;
        // eight rows of the factor in flight a thread (the loop is load-latency-bound)
        for (; i + 7 * ngr < dn; i += 8 * ngr) {
          float av[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) av[u] = load_io(A, abase + (size_t)(d0 + i + u * ngr) * r + k, a.io_dtype);
#pragma unroll
          for (int u = 0; u < 8; ++u)
#pragma unroll
            for (int bb = 0; bb < kProjRows; ++bb)
              acc[bb] = fmaf(xs[bb * kProjChunk + i + u * ngr], av[u], acc[bb]);
        }
        for (; i < dn; i += ngr) {
          const float av = load_io(A, abase + (size_t)(d0 + i) * r + k, a.io_dtype);
#pragma unroll
          for (int bb = 0; bb < kProjRows; ++bb) acc[bb] = fmaf(xs[bb * kProjChunk + i], av, acc[bb]);
        }
      }
    }
    __syncthreads();
    if (active) {
#pragma unroll
      for (int bb = 0; bb < kProjRows; ++bb) red[(rg * kProjRows + bb) * r + k] = acc[bb];
    }
    __syncthreads();
    // the row groups' partial sums in a fixed order
    for (int idx = t; idx < nb * r; idx += kProjThreads) {
      const int bb = idx / r, kk = idx - bb * r;
      float z = 0.f;
      for (int q = 0; q < ngr; ++q) z += red[(q * kProjRows + bb) * r + kk];
      if (ns == 1) zs[bb * r + kk] = z;
      else pa.part[(((size_t)gk * ns + sp) * a.B + b0 + bb) * r + kk] = z;
    }
    __syncthreads();
    if (ns == 1) proj_write_rows<LAT>(pa, 2 * g + kv, b0, nb, zs, lane, warp);
  }
  if (ns > 1) {
    // the last of the head's 2 nsplit CTAs adds the slices (fixed order) and writes
    // the head's K and V rows
    __syncthreads();
    bool last = false;
    if (t == 0) {
      __threadfence();
      last = atomicAdd(a.header + 4 + g, 1u) == 2u * ns - 1u;
    }
    if (!__syncthreads_or(last)) return;
    __threadfence();
    for (int kvv = 0; kvv < 2; ++kvv) {
      for (int b0 = 0; b0 < a.B; b0 += kProjRows) {
        const int nb = min(kProjRows, a.B - b0);
        __syncthreads();
        for (int idx = t; idx < nb * r; idx += kProjThreads) {
          const int bb = idx / r, kk = idx - bb * r;
          float z = 0.f;
          for (int q = 0; q < ns; ++q)
            z += __ldcg(&pa.part[((((size_t)(2 * g + kvv)) * ns + q) * a.B + b0 + bb) * r + kk]);
          zs[bb * r + kk] = z;
        }
        __syncthreads();
        proj_write_rows<LAT>(pa, 2 * g + kvv, b0, nb, zs, lane, warp);
      }
    }
    if (t == 0) atomicExch(a.header + 4 + g, 0u);
  }
  // the last writer advances every valid row's length (all writers have read it)
  __syncthreads();
  if (t == 0) {
    __threadfence();
    const unsigned writers = ns > 1 ? (unsigned)a.Hkv : gridDim.x;
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
                          (size_t)T * (d + 1) + (size_t)G * T + 3 * (size_t)G);
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

cudaError_t launch_project_append(const ProjArgs& a, cudaStream_t st) {
  const dim3 grid(2 * a.app.Hkv, a.nsplit), block(kProjThreads);
  switch (a.app.latent_dtype) {
    case LRKV_F32: return launch_pdl(lrkv_project_append_kernel<LRKV_F32>, grid, block, 0, st, a);
    case LRKV_BF16: return launch_pdl(lrkv_project_append_kernel<LRKV_BF16>, grid, block, 0, st, a);
    case LRKV_I8: return launch_pdl(lrkv_project_append_kernel<LRKV_I8>, grid, block, 0, st, a);
    default: return launch_pdl(lrkv_project_append_kernel<LRKV_E4M3>, grid, block, 0, st, a);
  }
}

int project_nsplit(int Hkv, int B, int r, int d_model, size_t workspace_bytes) {
  if (Hkv > kProjMaxHeads) return 1;
  int ns = (2 * num_sms() + 2 * Hkv - 1) / (2 * Hkv);
  ns = std::min(ns, std::max(1, d_model / kProjChunk));
  const size_t per = (size_t)2 * Hkv * B * r * sizeof(float);
  const size_t room = workspace_bytes > kHeaderBytes ? workspace_bytes - kHeaderBytes : 0;
  ns = (int)std::min<size_t>((size_t)ns, room / per);
  return std::max(1, ns);
}

}  // namespace lrkv
