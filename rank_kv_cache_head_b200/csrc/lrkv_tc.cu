// Tensor-core split-KV decode attention over a per-head low-rank KV cache (sm_100a).
//
// What it computes: for each (batch row b, KV head g) and each 128-token tile of a
// split, the keys and values are rebuilt on chip from the cached latents,
//     K = Z_K B_K,   V = Z_V B_V
// (per-head factors W_K,g = A_K,g B_K,g: "WSVD: Weighted Low-Rank Approximation for
// Fast and Efficient Execution of Low-Precision Vision-Language Models", section
// 2.A) and consumed at once by the scores q K^T / sqrt(d), an online softmax and
// P V, with reconstruction, attention and Flash Decoding in one fused flow and no
// intermediate written to HBM (same page, section 2.C). Each split writes a
// normalised partial and its log-sum-exp; lrkv_merge combines the splits.
//
// B200 design. Two CTAs share each SM (persistent; 256 tensor-memory columns each),
// and every CTA is a short warp-specialised pipeline:
//   warp 0      producer: takes (split, b, g) units from an atomic counter, brings the
//               unit's factors B_K, B_V and its q rows in once (TMA, bulk copy), and
//               streams its latent tiles through a ring of shared-memory stages (TMA).
//   warp 1      MMA issuer and tensor-memory owner. The rank-r reconstruction,
//               4 r d flops per token, is the dense contraction of the path and runs
//               on the 5th-generation tensor cores, bf16 x bf16 -> fp32 in TMEM:
//                 MMA1  Khat   [128 tok x 128 d] = Z_K tile (K-major) x B_K (MN-major)
//                 MMA2  Vhat^T [128 d x 128 tok] = B_V^T (MN-major) x Z_V tile^T
//               One TMEM slot for each; the next tile's MMA1 starts as soon as the
//               consumers hold this tile's key rows in registers, and its MMA2 as soon
//               as they hold the value rows, so the rebuild of tile t+1 runs under the
//               softmax and P V of tile t.
//   warps 2-5   one consumer warpgroup. Per tile, each thread first owns a token (a
//               TMEM lane of Khat): its G scores against q (fp32, in shared memory)
//               with packed fp32 FMAs; the warpgroup exchanges warp maxima once
//               (named barrier), updates the running max, and writes P. Then each
//               thread owns an output dimension (a TMEM lane of Vhat^T) and
//               accumulates P Vhat over the tile's tokens; token columns past the
//               row's length are zeroed, so cache contents beyond seq_len never reach
//               the result. At the unit's end it writes the split partial and LSE.
//   warps 6-7   (int8 / e4m3 latents only) convert each tile's codes to bf16 (exact)
//               for MMA1/2; the per-token scales multiply the scores (K) and are
//               folded into P (V), which is exact algebra.
// The scores and P V are matrix-vector work (G <= 16 query rows per KV head) and stay
// on CUDA cores: as tcgen05 MMAs they would be N = 16 instructions that cost more
// tensor-pipe time per tile than the tile's HBM time.
// Every wait is bounded: a role that waits more than a second sets the CTA's abort
// flag and LRKV_STATUS_TIMEOUT; the consumer warps take the decision to unwind
// together at their named barriers; every role drains its in-flight copies and MMAs
// and TMEM is freed before the CTA exits.
//
// Restrictions: io bf16, latents bf16 / int8 / e4m3, d_head = 128, rank a multiple of
// 16 in [16, 128], G <= 16, max_seq a multiple of 4 for quantised latents.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <math_constants.h>
#include <string.h>

#include "lrkv_internal.h"
#include "lrkv_sm100.cuh"
#include "lrkv_tmap.h"

namespace lrkv {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kT = 128;          // tokens per tile
constexpr int kUR = 4;           // unit-descriptor ring depth
constexpr int kMaxStages = 8;
constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s
// dynamic shared memory of one CTA when two share an SM (228 KB per SM, 1 KB of it
// reserved per CTA), and of a lone CTA (227 KB opt-in)
constexpr int kSmemPair = 113 * 1024;
constexpr int kSmemSolo = 227 * 1024;
constexpr uint32_t kTmemCols = 256;

enum LatKind { kLatBF16 = 0, kLatI8 = 1, kLatE4M3 = 2 };

template <int LAT> struct Roles {
  static constexpr int kCons = 2;   // first consumer warp
  static constexpr int kDQ = 6;     // converter warps 6, 7 (quantised latents)
  static constexpr int kWarps = LAT == kLatBF16 ? 6 : 8;
  static constexpr int kThreads = 32 * kWarps;
};

// Consumer layouts. For G <= 4 each thread reads its slots with the 16x256b shape:
// four rows of the warp's 32 TMEM lanes (g, g+8, g+16, g+24 with g = lane / 4) and a
// quarter of the columns (8i + 2k, 8i + 2k + 1 with k = lane % 4). Every q (key phase)
// or P (value phase) pair a thread loads then serves four rows, and a four-lane
// reduction completes each row's sum; for G = 1 the thread's q pairs stay in registers
// for the whole unit. kN repetitions of 8 columns are read per tensor-memory wait.
// For larger G each thread owns one lane (32x32b shape) and reads kBC columns per wait
// together with the q or P values of the batch for every head (64 registers of them;
// 32 under the 128-register budget of the quantised kernel); kCh independent packed
// accumulators per head keep the FMA chains short.
template <int LAT, int GP> struct Shape {
  static constexpr bool kL16 = GP <= 4;
  static constexpr int kN = LAT == kLatBF16 ? (GP == 1 ? 8 : 4) : (GP == 1 ? 4 : 2);
  static constexpr int kQRegs = LAT == kLatBF16 ? 64 : 32;
  static constexpr int kBC = (kQRegs / GP) < 4 ? 4 : ((kQRegs / GP) > 64 ? 64 : (kQRegs / GP));
  static constexpr int kCh = GP <= 1 ? 4 : 2;
};

// Sum over the four lanes of a 16x256b row group (lanes 4g .. 4g+3) of four per-row
// partials a[t] (rows g + 8t); lane 4g + k returns the complete sum of row g + 8k.
__device__ __forceinline__ float reduce_rows4(float a0, float a1, float a2, float a3, int lane) {
  const bool b0 = lane & 1, b1 = lane & 2;
  float keep0 = b0 ? a1 : a0, keep1 = b0 ? a3 : a2;
  const float send0 = b0 ? a0 : a1, send1 = b0 ? a2 : a3;
  keep0 += __shfl_xor_sync(0xffffffffu, send0, 1);   // rows b0 and 2 + b0 over lanes k, k^1
  keep1 += __shfl_xor_sync(0xffffffffu, send1, 1);
  float keep = b1 ? keep1 : keep0;
  const float send = b1 ? keep0 : keep1;
  keep += __shfl_xor_sync(0xffffffffu, send, 2);     // row b0 + 2 b1 over all four lanes
  return keep;
}

// named barriers of the consumer warpgroup (id 0 is __syncthreads)
enum { NB_Q = 1, NB_MAX = 2, NB_P = 3, NB_END = 4, NB_RED = 5 };

// 16x256b consumers keep a reference max per head and weight a tile's tokens by
// 2^(s - reference) with no per-tile max exchange; only a tile with a score above the
// reference by more than kTau (log2 units) moves it (an exact rescale). Weights stay
// below 2^kTau, far from fp32 overflow.
constexpr float kTau = 8.f;

struct alignas(64) TcParams {
  CUtensorMap tm_zk, tm_zv, tm_bk, tm_bv, tm_sk, tm_sv;
  SplitArgs a;
  int total_units;
  int W;        // bytes per swizzled row block of a bf16 latent tile (32/64/128)
  int nkb;      // row blocks per tile (2r / W)
  int nstage;   // TMA ring depth
  int nbuf;     // factor (and q) buffers: 1 or 2
  uint32_t off_stage, stage_bytes;  // TMA ring
  uint32_t off_zop;                  // bf16 operand tiles [2][K,V] (quantised latents)
  uint32_t off_b;                    // factors: [nbuf] x {BK, BV}, r*256 bytes each
  uint32_t off_qraw;                 // q rows of the unit, bf16 [nbuf][G][128]
  uint32_t off_qs;                   // q of the unit, fp32 scaled [G][128]
  uint32_t off_p;                    // P of the tile, fp32 [2][G][128]
  uint32_t off_misc;
  uint32_t smem_bytes;
};

// small shared arrays
struct Misc {
  float red[2][16][4];      // per tile parity, head, warp: warp maximum of the scores
  float lsum[16][4];        // unit end: per head, warp: sum of the softmax weights
  float scl[2][2][kT];      // per tile slot, K/V: per-token scales (quantised latents)
  int unit[kUR][8];         // b, g, s, t0, t1, ntiles, terminate
  uint32_t tmem_base;
  int abort_flag;
  int status_reported;
  int pad;
  uint64_t bar[48];
};

enum BarIdx {
  BAR_FULL = 0,                       // [kMaxStages] TMA tile landed
  BAR_EMPTY = BAR_FULL + kMaxStages,  // [kMaxStages] stage free again (consumers)
  BAR_KFULL = BAR_EMPTY + kMaxStages, // key slot rebuilt (MMA1 done)
  BAR_KFREE,                          // key slot read into registers
  BAR_VFULL,                          // value slot rebuilt (MMA2 done)
  BAR_VFREE,                          // value slot read into registers
  BAR_UFULL,                          // [kUR] unit descriptor written
  BAR_UEMPTY = BAR_UFULL + kUR,       // [kUR] unit descriptor consumed
  BAR_BQFULL = BAR_UEMPTY + kUR,      // [2] factors and q rows landed
  BAR_BQEMPTY = BAR_BQFULL + 2,       // [2] factors and q rows no longer needed
  BAR_DQFULL = BAR_BQEMPTY + 2,       // [2] bf16 operand tile and scales ready
  BAR_DQEMPTY = BAR_DQFULL + 2,       // [2] bf16 operand tile consumed (consumers)
  BAR_SCFREE = BAR_DQEMPTY + 2,       // [2] scales of the tile read by the consumers
  BAR_FINAL = BAR_SCFREE + 2,
  BAR_COUNT = BAR_FINAL + 1
};
static_assert(BAR_COUNT <= 48, "barrier array too small");

__device__ __forceinline__ int checked_len_tc(const SplitArgs& a, int b) {
  const int L = a.seqlens[b];
  if (L < 0 || L > a.Lcap || L > a.max_seqlen) return 0;  // flagged by the merge kernel
  return L;
}

__device__ __forceinline__ float warp_max(float x) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// K-major, swizzled latent tile: rows of W bytes, nkb row blocks of 128 rows each.
__device__ __forceinline__ uint64_t desc_latent(uint32_t base, int ks, int W) {
  const int byte = ks * 32;
  const uint32_t addr = base + (uint32_t)((byte / W) * (kT * W) + (byte % W));
  const uint32_t layout = (W == 128) ? 2u : (W == 64 ? 4u : 6u);
  return smem_desc(addr, 16, 8 * W, layout);
}

// MN-major, 128-byte swizzled factor: [2 blocks of 64 columns][r rows][128 B].
__device__ __forceinline__ uint64_t desc_factor(uint32_t base, int ks, int r) {
  return smem_desc(base + (uint32_t)ks * 2048u, (uint32_t)r * 128u, 1024u, 2u);
}

__device__ __forceinline__ void raise_timeout(const SplitArgs& a, Misc* ms) {
  if (atomicExch(&ms->status_reported, 1) == 0) atomicOr(a.header + kStatusWord, LRKV_STATUS_TIMEOUT);
}

template <int LAT, int GP, bool EXACT>
__global__ void __launch_bounds__(Roles<LAT>::kThreads, 2)
    lrkv_split_tc(const __grid_constant__ TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles, by pointer arithmetic on the shared
  // array so the compiler keeps the shared address space (plain shared loads/stores,
  // not generic ones) for every pointer derived from it
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);
  Misc* ms = reinterpret_cast<Misc*>(smem + p.off_misc);
  const SplitArgs& a = p.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = a.r;
  const int G = EXACT ? GP : a.G;   // heads per KV head; a compile-time constant when exact
  constexpr bool kQuant = LAT != kLatBF16;
  volatile int* abort_flag = &ms->abort_flag;
  auto bar = [&](int i) -> uint32_t { return smem_addr(&ms->bar[i]); };

  // ---- set-up ------------------------------------------------------------------------
  if (threadIdx.x == 0) {
    ms->abort_flag = 0;
    ms->status_reported = 0;
    for (int i = 0; i < p.nstage; ++i) {
      mbar_init(bar(BAR_FULL + i), 1);
      mbar_init(bar(BAR_EMPTY + i), kQuant ? 2 : 1);   // converters, or a consumer
    }
    mbar_init(bar(BAR_KFULL), 1);
    mbar_init(bar(BAR_KFREE), 4);
    mbar_init(bar(BAR_VFULL), 1);
    mbar_init(bar(BAR_VFREE), 4);
    for (int u = 0; u < kUR; ++u) {
      mbar_init(bar(BAR_UFULL + u), 1);
      mbar_init(bar(BAR_UEMPTY + u), 1 + 4 + (kQuant ? 2 : 0));
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(BAR_BQFULL + x), 1);
      mbar_init(bar(BAR_BQEMPTY + x), 1);   // consumers, after the unit's last MMA2
      mbar_init(bar(BAR_DQFULL + x), 2);
      mbar_init(bar(BAR_DQEMPTY + x), 1);
      mbar_init(bar(BAR_SCFREE + x), 4);
    }
    mbar_init(bar(BAR_FINAL), 3);   // one commit from each MMA-issuing lane
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&ms->tmem_base), kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  griddep_launch_dependents();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  const uint32_t tK = tmem;          // Khat: 128 lanes (tokens) x 128 columns (d)
  const uint32_t tV = tmem + 128u;   // Vhat^T: 128 lanes (d) x 128 columns (tokens)

  const uint32_t s_b = sbase + p.off_b;
  const uint32_t fac_bytes = (uint32_t)r * 256u;      // one factor, bf16
  const uint32_t tile_bytes = (uint32_t)kT * 2u * r;  // one bf16 latent tile
  const uint32_t q_bytes = (uint32_t)G * kD * 2u;     // q rows of one unit, bf16

  if (warp == 0) {
    // ================================ producer ======================================
    // The whole warp runs the loop (waits are warp-wide); lane 0 issues the copies.
    const bool leader = lane == 0;
    if (leader) {
      prefetch_tmap(&p.tm_zk);
      prefetch_tmap(&p.tm_zv);
      prefetch_tmap(&p.tm_bk);
      prefetch_tmap(&p.tm_bv);
      if (kQuant) {
        prefetch_tmap(&p.tm_sk);
        prefetch_tmap(&p.tm_sv);
      }
    }
    // everything this kernel reads from earlier kernels (seqlens, latents, the work
    // counter) is read here or after units handed out from here
    griddep_wait();
    const int BH = a.B * a.Hkv;
    // split size: the plan's, or the full-length choice scaled by the share of
    // tiles the rows actually hold (every CTA computes the same), never finer
    // than the plan's chunk, which bounds the number of splits
    int chunk = a.chunk, total_units = p.total_units;
    if (a.device_chunk) {
      long long tiles = 0;
      for (int b = lane; b < a.B; b += 32) tiles += (checked_len_tc(a, b) + kT - 1) / kT;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) tiles += __shfl_xor_sync(0xffffffffu, tiles, o);
      const int tiles_max = max(1, (a.max_seqlen + kT - 1) / kT);
      const long long full = (long long)a.B * tiles_max;
      int ct = (int)((a.chunk_hint * tiles + full - 1) / full);
      ct = max(a.chunk / kT, min(ct, a.chunk_hint));
      chunk = ct * kT;
      total_units = total_splits(a.n_visual, a.max_seqlen, chunk) * BH;
      if (blockIdx.x == 0 && lane == 0) atomicExch(a.header + kChunkWord, (unsigned)chunk);
    }
    uint32_t tile_seq = 0;
    int unit_seq = 0;
    int last_bq_unit = -1;
    bool ok = true;
    while (ok) {
      int u = 0;
      if (leader) u = (int)atomicAdd(a.header + kWorkCounter, 1u);
      u = __shfl_sync(0xffffffffu, u, 0);
      const bool term = u >= total_units;
      int b = 0, g = 0, s = 0, t0 = 0, t1 = 0, fset = 0;
      if (!term) {
        s = u / BH;
        const int rem = u - s * BH;
        b = rem / a.Hkv;
        g = rem - b * a.Hkv;
        const int L = checked_len_tc(a, b);
        fset = split_range(s, L, a.n_visual, a.max_seqlen, chunk, &t0, &t1);
        if (t0 >= t1) continue;  // empty split: nothing to do, the merge skips it
      }
      const int us = unit_seq % kUR;
      if (unit_seq >= kUR &&
          !mbar_wait_warp(bar(BAR_UEMPTY + us), ((unit_seq / kUR) - 1) & 1, abort_flag, kWaitNs)) {
        ok = false;
        break;
      }
      const int ntiles = term ? 0 : (t1 - t0 + kT - 1) / kT;
      if (leader) {
        int* d = ms->unit[us];
        d[0] = b; d[1] = g; d[2] = s; d[3] = t0; d[4] = t1; d[5] = ntiles; d[6] = term ? 1 : 0;
        mbar_arrive(bar(BAR_UFULL + us));
      }
      __syncwarp();
      if (term) break;
      const int bx = unit_seq % p.nbuf;
      if (unit_seq >= p.nbuf &&
          !mbar_wait_warp(bar(BAR_BQEMPTY + bx), ((unit_seq / p.nbuf) - 1) & 1, abort_flag, kWaitNs)) {
        ok = false;
        break;
      }
      if (leader) {
        const uint32_t sbk = s_b + (uint32_t)bx * 2u * fac_bytes;
        const uint32_t sbv = sbk + fac_bytes;
        mbar_arrive_expect_tx(bar(BAR_BQFULL + bx), 2u * fac_bytes + q_bytes);
        for (int blk = 0; blk < 2; ++blk) {
          // factor rows of this head in the unit's set (visual / text when separated)
          const int frow = (fset * a.Hkv + g) * r;
          tma_load_2d(sbk + (uint32_t)blk * (uint32_t)r * 128u, &p.tm_bk, bar(BAR_BQFULL + bx), blk * 64, frow);
          tma_load_2d(sbv + (uint32_t)blk * (uint32_t)r * 128u, &p.tm_bv, bar(BAR_BQFULL + bx), blk * 64, frow);
        }
        const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q) +
                                  ((size_t)b * a.Hq + (size_t)g * G) * kD;
        bulk_load(sbase + p.off_qraw + (uint32_t)bx * q_bytes, qg, q_bytes, bar(BAR_BQFULL + bx));
      }
      last_bq_unit = unit_seq;
      const int row0 = (b * a.Hkv + g) * a.Lcap + t0;
      for (int i = 0; i < ntiles; ++i, ++tile_seq) {
        const int st = (int)(tile_seq % (uint32_t)p.nstage);
        if (tile_seq >= (uint32_t)p.nstage &&
            !mbar_wait_warp(bar(BAR_EMPTY + st), ((tile_seq / p.nstage) - 1) & 1, abort_flag, kWaitNs)) {
          ok = false;
          break;
        }
        // test hook: the CTA that took work unit 0 withholds that unit's first tile (copy
        // and arrival), so the waits on it run out and the bounded-wait error path runs
        const bool withhold = a.debug_stall && u == 0 && i == 0;
        if (leader && !withhold) {
          const uint32_t sst = sbase + p.off_stage + (uint32_t)st * p.stage_bytes;
          const int row = row0 + i * kT;
          if (!kQuant) {
            mbar_arrive_expect_tx(bar(BAR_FULL + st), 2u * tile_bytes);
            for (int kb = 0; kb < p.nkb; ++kb) {
              const uint32_t off = (uint32_t)kb * (uint32_t)(kT * p.W);
              tma_load_2d(sst + off, &p.tm_zk, bar(BAR_FULL + st), kb * (p.W / 2), row);
              tma_load_2d(sst + tile_bytes + off, &p.tm_zv, bar(BAR_FULL + st), kb * (p.W / 2), row);
            }
          } else {
            const uint32_t cb = (uint32_t)kT * (uint32_t)r;  // code bytes per tile
            mbar_arrive_expect_tx(bar(BAR_FULL + st), 2u * cb + 2u * kT * 4u);
            tma_load_2d(sst, &p.tm_zk, bar(BAR_FULL + st), 0, row);
            tma_load_2d(sst + cb, &p.tm_zv, bar(BAR_FULL + st), 0, row);
            tma_load_2d(sst + 2u * cb, &p.tm_sk, bar(BAR_FULL + st), 0, row / 4);
            tma_load_2d(sst + 2u * cb + kT * 4u, &p.tm_sv, bar(BAR_FULL + st), 0, row / 4);
          }
        }
        __syncwarp();
      }
      ++unit_seq;
    }
    if (!ok) {
      if (leader) raise_timeout(a, ms);
      // drain the copies this warp issued before the CTA goes away
      int dummy = 0;
      const uint32_t first = tile_seq > (uint32_t)p.nstage ? tile_seq - p.nstage : 0u;
      for (uint32_t k = first; k < tile_seq; ++k)
        mbar_wait_warp(bar(BAR_FULL + (int)(k % p.nstage)), (k / p.nstage) & 1, &dummy, kWaitNs);
      if (last_bq_unit >= 0)
        mbar_wait_warp(bar(BAR_BQFULL + last_bq_unit % p.nbuf), (last_bq_unit / p.nbuf) & 1, &dummy,
                       kWaitNs);
    }
  } else if (warp == 1) {
    // ================================ MMA issuer ====================================
    // The whole warp runs the loop (waits are warp-wide). A commit tracks the MMAs of
    // the thread that issues it, and one thread's commits complete one after another
    // (a few hundred cycles each), so the work is spread: lane 0 issues every MMA1 and
    // its commit; lanes 1 and 2 take the MMA2s of alternate tiles with their commits.
    const bool leader = lane == 0;
    const uint32_t id_k = idesc_f16(1, 0, 1, 128, 128);   // Z_K (K-major) x B_K (MN-major)
    const uint32_t id_v = idesc_f16(1, 1, 0, 128, 128);   // B_V^T (MN-major) x Z_V^T (K-major)
    const int ksteps = r / 16;
    // descriptor pieces fixed for the launch: per K-step byte offsets inside a latent
    // tile and the constant fields, so each MMA costs a few integer ops to describe
    uint32_t zoff[8];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int byte = ks * 32;
      zoff[ks] = (uint32_t)((byte / p.W) * (kT * p.W) + (byte % p.W));
    }
    const uint64_t zdesc0 = desc_latent(0u, 0, p.W);     // address field zero
    const uint64_t fdesc0 = desc_factor(0u, 0, r);
    auto zdesc = [&](uint32_t base, int ks) { return zdesc0 | (uint64_t)(((base + zoff[ks]) >> 4) & 0x3FFFu); };
    auto fdesc = [&](uint32_t base, int ks) { return fdesc0 | (uint64_t)(((base + 2048u * ks) >> 4) & 0x3FFFu); };
    uint32_t tile_seq = 0;
    int unit_seq = 0;
    bool ok = true;
    while (ok) {
      const int us = unit_seq % kUR;
      if (!mbar_wait_warp(bar(BAR_UFULL + us), (unit_seq / kUR) & 1, abort_flag, kWaitNs)) {
        ok = false;
        break;
      }
      const int* d = ms->unit[us];
      if (d[6]) break;
      const int ntiles = d[5];
      __syncwarp();
      if (leader) mbar_arrive(bar(BAR_UEMPTY + us));
      const int bx = unit_seq % p.nbuf;
      if (!mbar_wait_warp(bar(BAR_BQFULL + bx), (unit_seq / p.nbuf) & 1, abort_flag, kWaitNs)) {
        ok = false;
        break;
      }
      const uint32_t sbk = s_b + (uint32_t)bx * 2u * fac_bytes;
      const uint32_t sbv = sbk + fac_bytes;
      for (int i = 0; i < ntiles; ++i, ++tile_seq) {
        const int x = (int)(tile_seq & 1u);
        uint32_t szk;
        int st = 0;
        if (!kQuant) {
          st = (int)(tile_seq % (uint32_t)p.nstage);
          if (!mbar_wait_warp(bar(BAR_FULL + st), (tile_seq / p.nstage) & 1, abort_flag, kWaitNs)) { ok = false; break; }
          szk = sbase + p.off_stage + (uint32_t)st * p.stage_bytes;
        } else {
          if (!mbar_wait_warp(bar(BAR_DQFULL + x), (tile_seq >> 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
          szk = sbase + p.off_zop + (uint32_t)x * 2u * tile_bytes;
        }
        // the key slot is free once the consumers hold the previous tile's key rows
        if (tile_seq >= 1 && !mbar_wait_warp(bar(BAR_KFREE), (tile_seq - 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
        if (leader) {
          tc_fence_after();
#pragma unroll 1
          for (int ks = 0; ks < ksteps; ++ks)
            mma_ss(tK, zdesc(szk, ks), fdesc(sbk, ks), id_k, ks > 0);
          tc_commit(bar(BAR_KFULL));
        }
        __syncwarp();
        if (tile_seq >= 1 && !mbar_wait_warp(bar(BAR_VFREE), (tile_seq - 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
        if (lane == 1 + (int)(tile_seq & 1u)) {
          tc_fence_after();
#pragma unroll 1
          for (int ks = 0; ks < ksteps; ++ks)
            mma_ss(tV, fdesc(sbv, ks), zdesc(szk + tile_bytes, ks), id_v, ks > 0);
          tc_commit(bar(BAR_VFULL));
        }
        __syncwarp();
      }
      ++unit_seq;
    }
    if (!ok && leader) raise_timeout(a, ms);
    // every MMA issued by this warp completes before TMEM is released
    if (lane < 3) tc_commit(bar(BAR_FINAL));
    __syncwarp();
    int dummy = 0;
    mbar_wait_warp(bar(BAR_FINAL), 0, &dummy, kWaitNs);
  } else if (warp >= Roles<LAT>::kCons && warp < Roles<LAT>::kCons + 4) {
    // ================================ consumers =====================================
    constexpr bool kL16 = Shape<LAT, GP>::kL16;  // 16x256b layout (G <= 4)
    constexpr int kN = Shape<LAT, GP>::kN;       // 16x256b: 8-column repetitions per wait
    constexpr int kBC = Shape<LAT, GP>::kBC;     // 32x32b: TMEM columns per wait
    constexpr int kCh = Shape<LAT, GP>::kCh;     // 32x32b: packed accumulators per head
    const int q4 = warp & 3;                     // TMEM lane quarter of this warp
    const int g4 = lane >> 2, k4 = lane & 3;     // 16x256b row group and column quarter
    // the token whose softmax this thread runs (key phase) and the output dimension it
    // writes (unit end): its own lane (32x32b), or row g + 8k of the quarter (16x256b)
    const int row = kL16 ? q4 * 32 + g4 + 8 * k4 : q4 * 32 + lane;
    const int c = row;
    const uint32_t lanebase = (uint32_t)(q4 * 32) << 16;
    const uint32_t lb1 = (uint32_t)(q4 * 32 + 16) << 16;   // 16x256b: second half of the quarter
    const uint32_t ctid = threadIdx.x - 32 * Roles<LAT>::kCons;
    float* qs = reinterpret_cast<float*>(smem + p.off_qs);            // [G][128]
    float* ps_all = reinterpret_cast<float*>(smem + p.off_p);         // [2][G][128]
    uint32_t tile_seq = 0;
    int unit_seq = 0;
    bool fail = false;
    for (;;) {
      const int us = unit_seq % kUR;
      fail = !mbar_wait_warp(bar(BAR_UFULL + us), (unit_seq / kUR) & 1, abort_flag, kWaitNs);
      const int* d = ms->unit[us];
      const bool term = fail ? true : d[6] != 0;
      const int bx = unit_seq % p.nbuf;
      if (!term)
        fail = !mbar_wait_warp(bar(BAR_BQFULL + bx), (unit_seq / p.nbuf) & 1, abort_flag, kWaitNs);
      if (!term && !fail) {
        // q of the G heads (bf16, brought in with the factors) -> fp32, pre-scaled by
        // log2(e) / sqrt(d) so the scores come out in log2 units
        const __nv_bfloat16* qr = reinterpret_cast<const __nv_bfloat16*>(
            smem + p.off_qraw + (size_t)bx * (size_t)G * kD * 2u);
        for (int j = 0; j < G; ++j) qs[j * kD + c] = __bfloat162float(qr[j * kD + c]) * a.scale_log2;
      }
      if (bar_any(NB_Q, 128, fail)) { fail = true; break; }
      if (term) break;
      const int b = d[0], g = d[1], s = d[2], t0 = d[3], t1 = d[4], ntiles = d[5];
      // G = 1, 16x256b: this thread's 16 q pairs (columns 8i + 2k, +1) for the unit
      uint64_t qreg[(kL16 && GP == 1) ? 16 : 1];
      if constexpr (kL16 && GP == 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) qreg[i] = *reinterpret_cast<const uint64_t*>(qs + 8 * i + 2 * k4);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_UEMPTY + us));

      float m_run[GP], l_run[GP];
      // packed partial sums of P Vhat: per head (32x32b), or per row and head (16x256b)
      constexpr int kAccA = kL16 ? 4 : GP, kAccB = kL16 ? GP : kCh;
      uint64_t acc[kAccA][kAccB];
#pragma unroll
      for (int j = 0; j < GP; ++j) {
        m_run[j] = -CUDART_INF_F;
        l_run[j] = 0.f;
      }
#pragma unroll
      for (int x = 0; x < kAccA; ++x)
#pragma unroll
        for (int y = 0; y < kAccB; ++y) acc[x][y] = 0ull;
      for (int i = 0; i < ntiles; ++i, ++tile_seq) {
        const uint32_t ph = tile_seq & 1u;           // KFULL / VFULL phase parity
        const int par = (int)(tile_seq & 1u);        // max / P buffer
        const int n_valid = min(kT, t1 - (t0 + i * kT));
        // ---- key phase: this thread's token, scores against the G heads ----
        fail = !mbar_wait_warp(bar(BAR_KFULL), ph, abort_flag, kWaitNs);
        float dsum[GP];   // this thread's token: q . Khat for each head
#pragma unroll
        for (int j = 0; j < GP; ++j) dsum[j] = 0.f;
        if constexpr (kL16) {
          uint64_t dot[4][GP];   // rows g, g+8, g+16, g+24 of the quarter
#pragma unroll
          for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int j = 0; j < GP; ++j) dot[t][j] = 0ull;
          if (!fail) {
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < kD; c0 += 8 * kN) {
              uint32_t v0[4 * kN], v1[4 * kN];
              tmem_ld16x256<kN>(tK + lanebase + (uint32_t)c0, v0);
              tmem_ld16x256<kN>(tK + lb1 + (uint32_t)c0, v1);
              uint64_t qp[GP][kN];
#pragma unroll
              for (int i = 0; i < kN; ++i) {
                if constexpr (GP == 1) {
                  qp[0][i] = qreg[c0 / 8 + i];
                } else {
#pragma unroll
                  for (int j = 0; j < GP; ++j)
                    if (j < G) qp[j][i] = *reinterpret_cast<const uint64_t*>(qs + j * kD + c0 + 8 * i + 2 * k4);
                }
              }
              tmem_wait_ld();
              if (c0 + 8 * kN == kD) {
                // every key column is in registers: the slot can be rebuilt again
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(BAR_KFREE));
              }
#pragma unroll
              for (int i = 0; i < kN; ++i) {
                const uint64_t kp[4] = {
                    pack2(__uint_as_float(v0[4 * i + 0]), __uint_as_float(v0[4 * i + 1])),
                    pack2(__uint_as_float(v0[4 * i + 2]), __uint_as_float(v0[4 * i + 3])),
                    pack2(__uint_as_float(v1[4 * i + 0]), __uint_as_float(v1[4 * i + 1])),
                    pack2(__uint_as_float(v1[4 * i + 2]), __uint_as_float(v1[4 * i + 3]))};
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                  for (int j = 0; j < GP; ++j)
                    if (j < G) dot[t][j] = ffma2p(kp[t], qp[j][i], dot[t][j]);
              }
            }
          }
#pragma unroll
          for (int j = 0; j < GP; ++j) {
            if (j < G) {
              float a4[4];
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const float2 d2 = unpack2(dot[t][j]);
                a4[t] = d2.x + d2.y;
              }
              dsum[j] = reduce_rows4(a4[0], a4[1], a4[2], a4[3], lane);
            }
          }
        } else {
          uint64_t dot[GP][kCh];
#pragma unroll
          for (int j = 0; j < GP; ++j)
#pragma unroll
            for (int u = 0; u < kCh; ++u) dot[j][u] = 0ull;
          if (!fail) {
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < kD; c0 += kBC) {
              uint32_t v[kBC];
              tmem_ld_cols<kBC>(tK + lanebase + (uint32_t)c0, v);
              ulonglong2 qv[GP][kBC / 4];
#pragma unroll
              for (int j = 0; j < GP; ++j)
                if (j < G)
#pragma unroll
                  for (int e = 0; e < kBC / 4; ++e)
                    qv[j][e] = *reinterpret_cast<const ulonglong2*>(qs + j * kD + c0 + 4 * e);
              tmem_wait_ld();
              if (c0 + kBC == kD) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(BAR_KFREE));
              }
#pragma unroll
              for (int e = 0; e < kBC / 4; ++e) {
                const uint64_t k01 = pack2(__uint_as_float(v[4 * e + 0]), __uint_as_float(v[4 * e + 1]));
                const uint64_t k23 = pack2(__uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
#pragma unroll
                for (int j = 0; j < GP; ++j) {
                  if (j < G) {
                    dot[j][(2 * e) % kCh] = ffma2p(k01, qv[j][e].x, dot[j][(2 * e) % kCh]);
                    dot[j][(2 * e + 1) % kCh] = ffma2p(k23, qv[j][e].y, dot[j][(2 * e + 1) % kCh]);
                  }
                }
              }
            }
          }
#pragma unroll
          for (int j = 0; j < GP; ++j) {
#pragma unroll
            for (int u = 0; u < kCh; ++u) {
              const float2 d2 = unpack2(dot[j][u]);
              dsum[j] += d2.x + d2.y;
            }
          }
        }
        const bool valid = row < n_valid;
        float sk = 1.f, sv = 1.f;
        if (kQuant) {
          const int x = (int)(tile_seq & 1u);
          if (!fail) fail = !mbar_wait_warp(bar(BAR_DQFULL + x), (tile_seq >> 1) & 1, abort_flag, kWaitNs);
          if (!fail) {
            sk = ms->scl[x][0][row];
            sv = ms->scl[x][1][row];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BAR_SCFREE + x));
          }
        }
        float sj[GP];
        float* P = ps_all + par * (G * kT);
        float alpha[GP];
        float pfin[GP];      // this thread's weight per head (added to the running sum)
        bool over = false;   // 16x256b: a score above the reference max + kTau
        if constexpr (kL16) {
#pragma unroll
          for (int j = 0; j < GP; ++j) {
            alpha[j] = 1.f;
            pfin[j] = 0.f;
            sj[j] = -CUDART_INF_F;
            if (j < G) {
              sj[j] = valid ? dsum[j] * sk : -CUDART_INF_F;
              over = over || (sj[j] > m_run[j] + kTau);
              const float pj = valid ? exp2f(sj[j] - m_run[j]) : 0.f;
              pfin[j] = pj;
              // masked tokens contribute an exact zero (their scale may be anything)
              P[j * kT + row] = valid ? pj * sv : 0.f;
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < GP; ++j) {
            if (j < G) {
              sj[j] = valid ? dsum[j] * sk : -CUDART_INF_F;
              const float wm = warp_max(sj[j]);
              if (lane == 0) ms->red[par][j][q4] = wm;
            }
          }
          if (bar_any(NB_MAX, 128, fail)) { fail = true; break; }
          // ---- online softmax over the tile: one running max per head ----
#pragma unroll
          for (int j = 0; j < GP; ++j) {
            alpha[j] = 1.f;
            if (j < G) {
              const float4 wm = *reinterpret_cast<const float4*>(&ms->red[par][j][0]);
              const float m_new = fmaxf(m_run[j], fmaxf(fmaxf(wm.x, wm.y), fmaxf(wm.z, wm.w)));
              alpha[j] = (m_new == -CUDART_INF_F) ? 1.f : exp2f(m_run[j] - m_new);
              const float pj = valid ? exp2f(sj[j] - m_new) : 0.f;
              l_run[j] = l_run[j] * alpha[j] + pj;
              m_run[j] = m_new;
              // masked tokens contribute an exact zero (their scale may be anything)
              P[j * kT + row] = valid ? pj * sv : 0.f;
            }
          }
        }
        // ---- value phase: this thread's output dimension ----
        fail = !mbar_wait_warp(bar(BAR_VFULL), ph, abort_flag, kWaitNs);
        if (!fail && ctid == 0) {
          // MMA1 (KFULL seen) and MMA2 of this tile are complete: their shared-memory
          // operands are free (a commit would only track its own thread's MMAs)
          if (!kQuant) mbar_arrive(bar(BAR_EMPTY + (int)(tile_seq % (uint32_t)p.nstage)));
          else mbar_arrive(bar(BAR_DQEMPTY + (int)(tile_seq & 1u)));
          if (i == ntiles - 1) mbar_arrive(bar(BAR_BQEMPTY + bx));   // factors and q rows
        }
        if constexpr (kL16) {
          uint32_t v0[4 * kN], v1[4 * kN];
          if (!fail) {
            tc_fence_after();
            tmem_ld16x256<kN>(tV + lanebase, v0);   // in flight across the barrier
            tmem_ld16x256<kN>(tV + lb1, v1);
          }
          // P of the tile complete; the barrier also ORs in a failed wait or a score
          // above the reference max
          const bool rare = bar_any(NB_P, 128, fail || over);
          if (rare) {
            if (bar_any(NB_MAX, 128, fail)) {
              if (!fail) tmem_wait_ld();
              fail = true;
              break;
            }
            // move the reference to the tile's max, rescale, and rewrite the tile's P
#pragma unroll
            for (int j = 0; j < GP; ++j) {
              if (j < G) {
                const float wm = warp_max(sj[j]);
                if (lane == 0) ms->red[par][j][q4] = wm;
              }
            }
            bar_any(NB_RED, 128, false);
#pragma unroll
            for (int j = 0; j < GP; ++j) {
              if (j < G) {
                const float4 wm = *reinterpret_cast<const float4*>(&ms->red[par][j][0]);
                const float m_new = fmaxf(m_run[j], fmaxf(fmaxf(wm.x, wm.y), fmaxf(wm.z, wm.w)));
                alpha[j] = (m_new == -CUDART_INF_F) ? 1.f : exp2f(m_run[j] - m_new);
                pfin[j] = valid ? exp2f(sj[j] - m_new) : 0.f;
                m_run[j] = m_new;
                P[j * kT + row] = valid ? pfin[j] * sv : 0.f;
              }
            }
            bar_any(NB_RED, 128, false);
#pragma unroll
            for (int j = 0; j < GP; ++j) {
              if (j < G) {
                const uint64_t a2 = pack2(alpha[j], alpha[j]);
#pragma unroll
                for (int t = 0; t < 4; ++t) acc[t][j] = ffma2p(acc[t][j], a2, 0ull);
              }
            }
          }
#pragma unroll
          for (int j = 0; j < GP; ++j)
            if (j < G) l_run[j] = l_run[j] * alpha[j] + pfin[j];
#pragma unroll
          for (int c0 = 0; c0 < kD; c0 += 8 * kN) {
            if (c0 > 0) {
              tmem_ld16x256<kN>(tV + lanebase + (uint32_t)c0, v0);
              tmem_ld16x256<kN>(tV + lb1 + (uint32_t)c0, v1);
            }
            uint64_t pp[GP][kN];
#pragma unroll
            for (int j = 0; j < GP; ++j)
              if (j < G)
#pragma unroll
                for (int i = 0; i < kN; ++i)
                  pp[j][i] = *reinterpret_cast<const uint64_t*>(P + j * kT + c0 + 8 * i + 2 * k4);
            tmem_wait_ld();
            if (c0 + 8 * kN == kD) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(bar(BAR_VFREE));
            }
            if (n_valid < c0 + 8 * kN) {
              // token columns past the row's length: exact zeros, whatever the cache holds
#pragma unroll
              for (int i = 0; i < kN; ++i) {
                const int col = c0 + 8 * i + 2 * k4;
                if (col >= n_valid) {
                  v0[4 * i + 0] = 0u; v0[4 * i + 2] = 0u; v1[4 * i + 0] = 0u; v1[4 * i + 2] = 0u;
                }
                if (col + 1 >= n_valid) {
                  v0[4 * i + 1] = 0u; v0[4 * i + 3] = 0u; v1[4 * i + 1] = 0u; v1[4 * i + 3] = 0u;
                }
              }
            }
#pragma unroll
            for (int i = 0; i < kN; ++i) {
              const uint64_t vp[4] = {
                  pack2(__uint_as_float(v0[4 * i + 0]), __uint_as_float(v0[4 * i + 1])),
                  pack2(__uint_as_float(v0[4 * i + 2]), __uint_as_float(v0[4 * i + 3])),
                  pack2(__uint_as_float(v1[4 * i + 0]), __uint_as_float(v1[4 * i + 1])),
                  pack2(__uint_as_float(v1[4 * i + 2]), __uint_as_float(v1[4 * i + 3]))};
#pragma unroll
              for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int j = 0; j < GP; ++j)
                  if (j < G) acc[t][j] = ffma2p(pp[j][i], vp[t], acc[t][j]);
            }
          }
        } else {
          uint32_t v[kBC];
          if (!fail) {
            tc_fence_after();
            tmem_ld_cols<kBC>(tV + lanebase, v);   // in flight across the barrier
          }
          const bool stop = bar_any(NB_P, 128, fail);
          if (stop) {
            if (!fail) tmem_wait_ld();
            fail = true;
            break;
          }
#pragma unroll
          for (int j = 0; j < GP; ++j) {
            if (j < G) {
              const uint64_t a2 = pack2(alpha[j], alpha[j]);
#pragma unroll
              for (int u = 0; u < kCh; ++u) acc[j][u] = ffma2p(acc[j][u], a2, 0ull);
            }
          }
#pragma unroll
          for (int c0 = 0; c0 < kD; c0 += kBC) {
            if (c0 > 0) tmem_ld_cols<kBC>(tV + lanebase + (uint32_t)c0, v);
            ulonglong2 pv[GP][kBC / 4];
#pragma unroll
            for (int j = 0; j < GP; ++j)
              if (j < G)
#pragma unroll
                for (int e = 0; e < kBC / 4; ++e)
                  pv[j][e] = *reinterpret_cast<const ulonglong2*>(P + j * kT + c0 + 4 * e);
            tmem_wait_ld();
            if (c0 + kBC == kD) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(bar(BAR_VFREE));
            }
            if (n_valid < c0 + kBC) {
              // token columns past the row's length: exact zeros, whatever the cache holds
#pragma unroll
              for (int e = 0; e < kBC; ++e)
                if (c0 + e >= n_valid) v[e] = 0u;
            }
#pragma unroll
            for (int e = 0; e < kBC / 4; ++e) {
              const uint64_t v01 = pack2(__uint_as_float(v[4 * e + 0]), __uint_as_float(v[4 * e + 1]));
              const uint64_t v23 = pack2(__uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
#pragma unroll
              for (int j = 0; j < GP; ++j) {
                if (j < G) {
                  acc[j][(2 * e) % kCh] = ffma2p(pv[j][e].x, v01, acc[j][(2 * e) % kCh]);
                  acc[j][(2 * e + 1) % kCh] = ffma2p(pv[j][e].y, v23, acc[j][(2 * e + 1) % kCh]);
                }
              }
            }
          }
        }
      }
      if (fail) break;
      // ---- unit end: the softmax sum over the warpgroup, the partial and its LSE ----
#pragma unroll
      for (int j = 0; j < GP; ++j) {
        if (j < G) {
          const float lw = warp_sum(l_run[j]);
          if (lane == 0) ms->lsum[j][q4] = lw;
        }
      }
      bar_any(NB_END, 128, false);
      const size_t hb = (size_t)b * a.Hq + (size_t)g * G;
#pragma unroll
      for (int j = 0; j < GP; ++j) {
        if (j < G) {
          const float4 l4 = *reinterpret_cast<const float4*>(&ms->lsum[j][0]);
          const float L = (l4.x + l4.y) + (l4.z + l4.w);
          float num = 0.f;
          if constexpr (kL16) {
            float a4[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const float2 a2 = unpack2(acc[t][j]);
              a4[t] = a2.x + a2.y;
            }
            num = reduce_rows4(a4[0], a4[1], a4[2], a4[3], lane);   // output dimension c
          } else {
#pragma unroll
            for (int u = 0; u < kCh; ++u) {
              const float2 a2 = unpack2(acc[j][u]);
              num += a2.x + a2.y;
            }
          }
          a.o_part[((hb + j) * a.S + s) * kD + c] = num / L;
          if (c == j) a.lse_part[(hb + j) * a.S + s] = (m_run[j] + log2f(L)) * CUDART_LN2_F;
        }
      }
      ++unit_seq;
    }
    if (fail) raise_timeout(a, ms);
  } else if (kQuant && warp >= Roles<LAT>::kDQ) {
    // ============================ code -> bf16 converter ============================
    // two warps; each thread converts two token rows (rbase, rbase + 64) of the tile.
    // int8 codes become floats without the int-to-float unit: the biased code byte
    // is placed in the low mantissa bits of 2^23 and 2^23 + 128 is subtracted (exact);
    // e4m3 codes convert two at a time through f16 (exact).
    const int W = p.W;
    const int rbase = (warp - Roles<LAT>::kDQ) * 32 + lane;
    uint32_t tile_seq = 0;
    int unit_seq = 0;
    bool ok = true;
    const uint32_t cb = (uint32_t)kT * (uint32_t)r;
    while (ok) {
      const int us = unit_seq % kUR;
      if (!mbar_wait_warp(bar(BAR_UFULL + us), (unit_seq / kUR) & 1, abort_flag, kWaitNs)) { ok = false; break; }
      const int* d = ms->unit[us];
      if (d[6]) break;
      const int ntiles = d[5];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_UEMPTY + us));
      for (int i = 0; i < ntiles && ok; ++i, ++tile_seq) {
        const int st = (int)(tile_seq % (uint32_t)p.nstage);
        const int x = (int)(tile_seq & 1u);
        if (!mbar_wait_warp(bar(BAR_FULL + st), (tile_seq / p.nstage) & 1, abort_flag, kWaitNs)) { ok = false; break; }
        if (tile_seq >= 2) {
          // operand slot x free (MMA2 of the tile two back done) and its scales read
          if (!mbar_wait_warp(bar(BAR_DQEMPTY + x), ((tile_seq >> 1) - 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
          if (!mbar_wait_warp(bar(BAR_SCFREE + x), ((tile_seq >> 1) - 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
        }
        const uint8_t* stage = smem + p.off_stage + (size_t)st * p.stage_bytes;
        uint8_t* zop = smem + p.off_zop + (size_t)x * 2u * tile_bytes;
        const float* scs = reinterpret_cast<const float*>(stage + 2 * cb);
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int row = rbase + 64 * rr;
#pragma unroll
          for (int kv = 0; kv < 2; ++kv) {
            const uint8_t* src = stage + kv * cb + (size_t)row * r;
            uint8_t* dst = zop + kv * tile_bytes;
            for (int k0 = 0; k0 < r; k0 += 16) {
              const uint4 raw = *reinterpret_cast<const uint4*>(src + k0);
              const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
              uint32_t w[8];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float f[4];
                if (LAT == kLatI8) {
                  const uint32_t xb = rw[e] ^ 0x80808080u;   // code + 128, per byte
                  f[0] = __int_as_float((int)__byte_perm(xb, 0x4B000000u, 0x7540u)) - 8388736.f;
                  f[1] = __int_as_float((int)__byte_perm(xb, 0x4B000000u, 0x7541u)) - 8388736.f;
                  f[2] = __int_as_float((int)__byte_perm(xb, 0x4B000000u, 0x7542u)) - 8388736.f;
                  f[3] = __int_as_float((int)__byte_perm(xb, 0x4B000000u, 0x7543u)) - 8388736.f;
                } else {
                  const __half2_raw h01 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(rw[e] & 0xFFFFu), __NV_E4M3);
                  const __half2_raw h23 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(rw[e] >> 16), __NV_E4M3);
                  const float2 a01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
                  const float2 a23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
                  f[0] = a01.x; f[1] = a01.y; f[2] = a23.x; f[3] = a23.y;
                }
                const __nv_bfloat162 b01 = __floats2bfloat162_rn(f[0], f[1]);
                const __nv_bfloat162 b23 = __floats2bfloat162_rn(f[2], f[3]);
                w[2 * e] = *reinterpret_cast<const uint32_t*>(&b01);
                w[2 * e + 1] = *reinterpret_cast<const uint32_t*>(&b23);
              }
              // bf16 bytes [2*k0, 2*k0 + 32) of this row: two 16-byte chunks, swizzled
#pragma unroll
              for (int half = 0; half < 2; ++half) {
                const int byte = 2 * k0 + 16 * half;
                const int kb = byte / W, inrow = byte % W;
                const int chunk = inrow >> 4;
                int sw;
                if (W == 128) sw = chunk ^ (row & 7);
                else if (W == 64) sw = chunk ^ ((row >> 1) & 3);
                else sw = chunk ^ ((row >> 2) & 1);
                uint4 o;
                o.x = w[4 * half + 0];
                o.y = w[4 * half + 1];
                o.z = w[4 * half + 2];
                o.w = w[4 * half + 3];
                *reinterpret_cast<uint4*>(dst + (size_t)kb * (kT * W) + (size_t)row * W + sw * 16) = o;
              }
            }
          }
          ms->scl[x][0][row] = scs[row];
          ms->scl[x][1][row] = scs[kT + row];
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(BAR_DQFULL + x));
          mbar_arrive(bar(BAR_EMPTY + st));
        }
      }
      if (!ok) break;
      ++unit_seq;
    }
    if (!ok) raise_timeout(a, ms);
  }

  // ---- tear-down -----------------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0) {
    // the last CTA to finish resets the work counter for the next launch
    __threadfence();
    const unsigned prev = atomicAdd(a.header + kDoneCounter, 1u);
    if (prev == gridDim.x - 1) {
      atomicExch(a.header + kWorkCounter, 0u);
      atomicExch(a.header + kDoneCounter, 0u);
      __threadfence();
    }
  }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------

struct Layout {
  int W, nkb, nstage, nbuf, ctas_per_sm;
  uint32_t off_stage, stage_bytes, off_zop, off_b, off_qraw, off_qs, off_p, off_misc, smem;
};

uint32_t round_up(uint32_t x, uint32_t m) { return (x + m - 1) / m * m; }

// Shared-memory layout for `nbuf` factor buffers within `limit` bytes; false when
// fewer than `min_stages` latent stages fit.
bool layout_for(int r, int G, bool quant, int nbuf, int limit, int min_stages, Layout* L) {
  const int rowb = 2 * r;
  L->W = (rowb % 128 == 0) ? 128 : (rowb % 64 == 0 ? 64 : 32);
  L->nkb = rowb / L->W;
  L->nbuf = nbuf;
  const uint32_t tile = 128u * rowb;           // one bf16 latent tile
  const uint32_t fac = (uint32_t)r * 256u;     // one bf16 factor
  uint32_t off = 0;
  L->off_b = off;                              // 1024-aligned (128-byte swizzle)
  off += (uint32_t)nbuf * 2u * fac;
  L->off_zop = off;
  if (quant) off += 2u * 2u * tile;
  L->off_qraw = off;
  off += round_up((uint32_t)nbuf * (uint32_t)G * 256u, 128u);
  L->off_qs = off;
  off += round_up((uint32_t)G * 512u, 128u);
  L->off_p = off;
  off += round_up(2u * (uint32_t)G * 512u, 128u);
  L->off_misc = off;
  off = round_up(off + (uint32_t)sizeof(Misc), 1024u);   // swizzled tiles: 1024-aligned
  L->off_stage = off;
  L->stage_bytes = quant ? round_up(2u * 128u * (uint32_t)r + 2u * 512u, 1024u) : 2u * tile;
  const int avail = limit - 1024 - (int)off;   // 1024: alignment of the dynamic array
  int ns = avail / (int)L->stage_bytes;
  if (ns > kMaxStages) ns = kMaxStages;
  if (ns < min_stages) return false;
  L->nstage = ns;
  L->smem = 1024u + off + (uint32_t)ns * L->stage_bytes;
  return true;
}

// Two CTAs per SM when the tiles fit (double-buffered factors when that still leaves
// three stages), else one CTA with the whole shared memory.
bool plan_layout(int r, int G, bool quant, Layout* L) {
  if (r < 16 || r > 128 || r % 16) return false;
  if (G < 1 || G > 16) return false;
  L->ctas_per_sm = 2;
  if (layout_for(r, G, quant, 2, kSmemPair, 3, L)) return true;
  if (layout_for(r, G, quant, 1, kSmemPair, 2, L)) return true;
  L->ctas_per_sm = 1;
  if (layout_for(r, G, quant, 2, kSmemSolo, 3, L)) return true;
  return layout_for(r, G, quant, 1, kSmemSolo, 2, L);
}

template <int LAT, int GP, bool EXACT>
cudaError_t launch_typed(const TcParams& prm, int grid, cudaStream_t st) {
  auto kern = lrkv_split_tc<LAT, GP, EXACT>;
  static int configured = 0;
  if ((int)prm.smem_bytes > configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)prm.smem_bytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    configured = (int)prm.smem_bytes;
  }
  return launch_pdl(kern, dim3(grid), dim3(Roles<LAT>::kThreads), (size_t)prm.smem_bytes, st, prm);
}

template <int LAT>
cudaError_t launch_g(const TcParams& prm, int grid, cudaStream_t st) {
  switch (prm.a.G) {
    case 1: return launch_typed<LAT, 1, true>(prm, grid, st);
    case 2: return launch_typed<LAT, 2, true>(prm, grid, st);
    case 4: return launch_typed<LAT, 4, true>(prm, grid, st);
    case 8: return launch_typed<LAT, 8, true>(prm, grid, st);
    case 16: return launch_typed<LAT, 16, true>(prm, grid, st);
    default: break;
  }
  const int G = prm.a.G;
  if (G <= 4) return launch_typed<LAT, 4, false>(prm, grid, st);
  if (G <= 8) return launch_typed<LAT, 8, false>(prm, grid, st);
  return launch_typed<LAT, 16, false>(prm, grid, st);
}

}  // namespace

bool tc_supported(const lrkv_dims& d, int* smem_bytes, int* ctas_per_sm) {
  *smem_bytes = 0;
  *ctas_per_sm = 0;
  if (d.io_dtype != LRKV_BF16 || d.d_head != 128) return false;
  if (d.latent_dtype != LRKV_BF16 && d.latent_dtype != LRKV_I8 && d.latent_dtype != LRKV_E4M3)
    return false;
  const int G = d.n_q_heads / d.n_kv_heads;
  if (G < 1 || G > 16) return false;
  const bool quant = d.latent_dtype != LRKV_BF16;
  if (quant && d.max_seq % 4 != 0) return false;
  if ((double)d.batch * d.n_kv_heads * d.max_seq >= 2147483647.0) return false;
  Layout L;
  if (!plan_layout(d.rank, G, quant, &L)) return false;
  *smem_bytes = (int)L.smem;
  *ctas_per_sm = L.ctas_per_sm;
  return true;
}

cudaError_t launch_split_tc(const SplitArgs& a, const Plan& plan, cudaStream_t st) {
  const bool quant = a.latent_dtype != LRKV_BF16;
  Layout L;
  if (!plan_layout(a.r, a.G, quant, &L)) return cudaErrorInvalidValue;
  TcParams prm;
  memset(&prm, 0, sizeof(prm));
  const uint64_t rows = (uint64_t)a.B * a.Hkv * a.Lcap;
  bool ok = true;
  if (!quant) {
    ok &= make_tmap_2d(&prm.tm_zk, a.ZK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.r, rows, L.W / 2,
                       kT, L.W);
    ok &= make_tmap_2d(&prm.tm_zv, a.ZV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.r, rows, L.W / 2,
                       kT, L.W);
  } else {
    ok &= make_tmap_2d(&prm.tm_zk, a.ZK, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.r, rows, a.r, kT, 0);
    ok &= make_tmap_2d(&prm.tm_zv, a.ZV, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.r, rows, a.r, kT, 0);
    ok &= make_tmap_vec_f32(&prm.tm_sk, a.SK, rows);
    ok &= make_tmap_vec_f32(&prm.tm_sv, a.SV, rows);
  }
  const uint64_t fac_rows = (uint64_t)(a.n_visual > 0 ? 2 : 1) * a.Hkv * a.r;
  ok &= make_tmap_2d(&prm.tm_bk, a.BK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, fac_rows, 64, a.r, 128);
  ok &= make_tmap_2d(&prm.tm_bv, a.BV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, fac_rows, 64, a.r, 128);
  if (!ok) return cudaErrorInvalidValue;
  prm.a = a;
  prm.total_units = a.S * a.B * a.Hkv;
  prm.W = L.W;
  prm.nkb = L.nkb;
  prm.nstage = L.nstage;
  prm.nbuf = L.nbuf;
  prm.off_stage = L.off_stage;
  prm.stage_bytes = L.stage_bytes;
  prm.off_zop = L.off_zop;
  prm.off_b = L.off_b;
  prm.off_qraw = L.off_qraw;
  prm.off_qs = L.off_qs;
  prm.off_p = L.off_p;
  prm.off_misc = L.off_misc;
  prm.smem_bytes = L.smem;
  switch (a.latent_dtype) {
    case LRKV_BF16: return launch_g<kLatBF16>(prm, plan.grid, st);
    case LRKV_I8: return launch_g<kLatI8>(prm, plan.grid, st);
    default: return launch_g<kLatE4M3>(prm, plan.grid, st);
  }
}

}  // namespace lrkv
