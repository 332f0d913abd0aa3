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
// B200 design (one persistent CTA per SM, warp-specialised, mbarrier pipelines):
//   warp 0      producer: takes (split, b, g) units from an atomic counter, TMA-loads
//               the unit's factors B_K, B_V once and its latent tiles through a ring
//               of shared-memory stages;
//   warp 1      MMA issuer (one thread) and TMEM owner. The rank-r reconstruction,
//               4 r d flops per token, is the dense contraction of the path and runs
//               on the 5th-generation tensor cores, bf16 x bf16 -> fp32 in TMEM:
//                 MMA1  Khat   [128 tok x 128 d] = Z_K tile (K-major) x B_K (MN-major)
//                 MMA2  Vhat^T [128 d x 128 tok] = B_V^T (MN-major) x Z_V tile^T
//               Keys and values each have a two-slot TMEM ring (128 columns a slot);
//               MMA2 trails MMA1 by one tile so a key slot is recycled as soon as its
//               rows have been read.
//   warps 4-7   key side, one thread per token (TMEM lane): reads its rebuilt key row
//               (fp32), forms its G scores against q (held in shared memory), and
//               runs an online softmax. Each of the four warps owns the same 32-token
//               slice of every tile and keeps its own running max and sum (its own
//               "stream"), so no cross-warp exchange sits on the per-tile path;
//               writes P (fp32) and the per-stream rescale factors.
//   warps 8-11  value side, one thread per output dimension (TMEM lane of Vhat^T):
//               keeps one accumulator per (head, stream) -- token chunk w of Vhat^T
//               belongs to stream w -- skips token columns past the row's length
//               (cache contents beyond seq_len never reach the result), and at the
//               unit's end merges the four streams by their log-sum-exp and writes
//               the split partial.
//   warps 12-15 (int8 / e4m3 latents only) convert each tile's codes to bf16 (exact)
//               for MMA1/2; the per-token scales multiply the scores (K) and are
//               folded into P (V), which is exact algebra.
// Every wait is bounded: a role that waits more than a second sets the CTA's abort
// flag and LRKV_STATUS_TIMEOUT, and all roles unwind, drain their in-flight copies
// and MMAs, and free TMEM before the CTA exits.
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
constexpr int kMaxStages = 16;
constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s
constexpr int kSmemLimit = 232448;           // 227 KB opt-in per block

enum LatKind { kLatBF16 = 0, kLatI8 = 1, kLatE4M3 = 2 };

// warpgroups per side: two key-side and two value-side warpgroups alternate tiles for
// bf16 latents (more independent warps to hide latency); quantised latents keep one
// of each plus the converter warpgroup (register budget)
template <int LAT> struct Roles {
  static constexpr int kNwg = LAT == kLatBF16 ? 2 : 1;
  static constexpr int kKFirst = 2;                  // warps 0, 1: producer, MMA
  static constexpr int kVFirst = kKFirst + 4 * kNwg;
  static constexpr int kDQFirst = kVFirst + 4 * kNwg;
  static constexpr int kWarps = kDQFirst + (LAT == kLatBF16 ? 0 : 4);
  static constexpr int kThreads = 32 * kWarps;
};

struct alignas(64) TcParams {
  CUtensorMap tm_zk, tm_zv, tm_bk, tm_bv, tm_sk, tm_sv;
  SplitArgs a;
  int total_units;
  int W;        // bytes per swizzled row block of a bf16 latent tile (32/64/128)
  int nkb;      // row blocks per tile (2r / W)
  int nstage;   // TMA ring depth
  int nbuf;     // factor buffers (1 or 2)
  uint32_t off_stage, stage_bytes;  // TMA ring
  uint32_t off_zop;                  // bf16 operand ring (quantised latents)
  uint32_t off_b;                    // factors: [nbuf] x {BK, BV}, r*256 bytes each
  uint32_t off_q;                    // q of the unit, fp32 [2][16][128]
  uint32_t off_p;                    // P of the tile, fp32 [2][16][128]
  uint32_t off_x;                    // second value-side warpgroup's output, fp32 [2][16][128]
  uint32_t off_misc;
  uint32_t smem_bytes;
};

// small shared arrays after the tiles
struct Misc {
  float alpha[2][4][16];       // per tile slot, key-side warp (softmax stream), head
  float stat_m[2][2][4][16];   // unit end, per unit parity and warpgroup: each stream's max
  float stat_l[2][2][4][16];   // ... and running sum
  float xm[2][16], xl[2][16];  // second value-side warpgroup's merged max and sum
  float scl[2][2][kT];      // per-token scales of the tile (quantised latents)
  int unit[kUR][8];         // b, g, s, t0, t1, ntiles, terminate
  uint32_t tmem_base;
  int abort_flag;
  int status_reported;
  int pad;
  uint64_t bar[96];
};

enum BarIdx {
  BAR_FULL = 0,                       // [kMaxStages] TMA tile landed
  BAR_EMPTY = BAR_FULL + kMaxStages,  // [kMaxStages] stage free again
  BAR_KFULL = BAR_EMPTY + kMaxStages, // [2] key slot rebuilt (MMA1 done)
  BAR_KFREE = BAR_KFULL + 2,          // [2] key slot read by the key side
  BAR_VFULL = BAR_KFREE + 2,          // [2] value slot rebuilt (MMA2 done)
  BAR_VFREE = BAR_VFULL + 2,          // [2] value slot read by the value side
  BAR_PFULL = BAR_VFREE + 2,          // [2] P and alpha of the tile written
  BAR_PFREE = BAR_PFULL + 2,          // [2] P and alpha of the tile consumed
  BAR_QREADY = BAR_PFREE + 2,         // [2] q of the unit in shared memory
  BAR_UFULL = BAR_QREADY + 2,         // [kUR] unit descriptor written
  BAR_UEMPTY = BAR_UFULL + kUR,       // [kUR] unit descriptor consumed
  BAR_BQFULL = BAR_UEMPTY + kUR,      // [2] factors landed
  BAR_BQEMPTY = BAR_BQFULL + 2,       // [2] factors no longer needed
  BAR_STFULL = BAR_BQEMPTY + 2,       // [2 x 2] unit statistics written (parity, warpgroup)
  BAR_STEMPTY = BAR_STFULL + 4,       // [2 x 2] unit statistics read
  BAR_XFULL = BAR_STEMPTY + 4,        // [2] second value-side warpgroup's result written
  BAR_XEMPTY = BAR_XFULL + 2,         // [2] ... and read
  BAR_DQFULL = BAR_XEMPTY + 2,        // [2] bf16 operand tile converted
  BAR_DQEMPTY = BAR_DQFULL + 2,       // [2] bf16 operand tile consumed by MMA2
  BAR_FINAL = BAR_DQEMPTY + 2,
  BAR_COUNT = BAR_FINAL + 1
};
static_assert(BAR_COUNT <= 96, "barrier array too small");

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
__global__ void __launch_bounds__(Roles<LAT>::kThreads, 1)
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
      mbar_init(bar(BAR_EMPTY + i), kQuant ? 4 : 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(BAR_KFULL + x), 1);
      mbar_init(bar(BAR_KFREE + x), 4);
      mbar_init(bar(BAR_VFULL + x), 1);
      mbar_init(bar(BAR_VFREE + x), 4);
      mbar_init(bar(BAR_PFULL + x), 4);
      mbar_init(bar(BAR_PFREE + x), 4);
      mbar_init(bar(BAR_QREADY + x), 4 * Roles<LAT>::kNwg);
      mbar_init(bar(BAR_BQFULL + x), 1);
      mbar_init(bar(BAR_BQEMPTY + x), 1);
      mbar_init(bar(BAR_STFULL + 2 * x), 4);
      mbar_init(bar(BAR_STFULL + 2 * x + 1), 4);
      mbar_init(bar(BAR_STEMPTY + 2 * x), 4);
      mbar_init(bar(BAR_STEMPTY + 2 * x + 1), 4);
      mbar_init(bar(BAR_XFULL + x), 4);
      mbar_init(bar(BAR_XEMPTY + x), 4);
      mbar_init(bar(BAR_DQFULL + x), 4);
      mbar_init(bar(BAR_DQEMPTY + x), 1);
    }
    for (int u = 0; u < kUR; ++u) {
      mbar_init(bar(BAR_UFULL + u), 1);
      mbar_init(bar(BAR_UEMPTY + u), 1 + 8 * Roles<LAT>::kNwg + (kQuant ? 4 : 0));
    }
    mbar_init(bar(BAR_FINAL), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&ms->tmem_base), 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;

  const uint32_t s_b = sbase + p.off_b;
  const uint32_t fac_bytes = (uint32_t)r * 256u;      // one factor, bf16
  const uint32_t tile_bytes = (uint32_t)kT * 2u * r;  // one bf16 latent tile
  // TMEM: key slots at columns [0,128) and [128,256), value slots at [256,384), [384,512)
  auto tK = [&](int x) { return tmem + 128u * x; };
  auto tV = [&](int x) { return tmem + 256u + 128u * x; };

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
    const int BH = a.B * a.Hkv;
    uint32_t tile_seq = 0;
    int unit_seq = 0;
    int last_bq_unit = -1;
    bool ok = true;
    while (ok) {
      int u = 0;
      if (leader) u = (int)atomicAdd(a.header + kWorkCounter, 1u);
      u = __shfl_sync(0xffffffffu, u, 0);
      const bool term = u >= p.total_units;
      int b = 0, g = 0, s = 0, t0 = 0, t1 = 0;
      if (!term) {
        s = u / BH;
        const int rem = u - s * BH;
        b = rem / a.Hkv;
        g = rem - b * a.Hkv;
        const int L = checked_len_tc(a, b);
        t0 = s * a.chunk;
        t1 = min(L, t0 + a.chunk);
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
        mbar_arrive_expect_tx(bar(BAR_BQFULL + bx), 2u * fac_bytes);
        for (int blk = 0; blk < 2; ++blk) {
          tma_load_2d(sbk + (uint32_t)blk * (uint32_t)r * 128u, &p.tm_bk, bar(BAR_BQFULL + bx), blk * 64, g * r);
          tma_load_2d(sbv + (uint32_t)blk * (uint32_t)r * 128u, &p.tm_bv, bar(BAR_BQFULL + bx), blk * 64, g * r);
        }
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
        if (leader) {
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
    // The whole warp runs the loop (waits are warp-wide); lane 0 issues the MMAs and
    // the commits that track them.
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
    // the tile whose MMA2 is still to be issued (MMA2 trails MMA1 by one tile)
    bool pend = false;
    uint32_t pend_seq = 0, pend_zv = 0, pend_bv = 0;
    int pend_st = 0, pend_bx = 0;
    bool pend_last = false;

    auto issue_v = [&]() -> bool {
      const int x = (int)(pend_seq & 1u);
      if (pend_seq >= 2 &&
          !mbar_wait_warp(bar(BAR_VFREE + x), ((pend_seq >> 1) - 1) & 1, abort_flag, kWaitNs))
        return false;
      if (leader) {
        tc_fence_after();
#pragma unroll 1
        for (int ks = 0; ks < ksteps; ++ks)
          mma_ss(tV(x), fdesc(pend_bv, ks), zdesc(pend_zv, ks), id_v, ks > 0);
        tc_commit(bar(BAR_VFULL + x));
        if (!kQuant) tc_commit(bar(BAR_EMPTY + pend_st));
        else tc_commit(bar(BAR_DQEMPTY + x));
        if (pend_last) tc_commit(bar(BAR_BQEMPTY + pend_bx));
      }
      __syncwarp();
      pend = false;
      return true;
    };

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
      if (p.nbuf == 1 && pend && !issue_v()) { ok = false; break; }
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
        if (tile_seq >= 2 && !mbar_wait_warp(bar(BAR_KFREE + x), ((tile_seq >> 1) - 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
        if (leader) {
          tc_fence_after();
#pragma unroll 1
          for (int ks = 0; ks < ksteps; ++ks)
            mma_ss(tK(x), zdesc(szk, ks), fdesc(sbk, ks), id_k, ks > 0);
          tc_commit(bar(BAR_KFULL + x));
        }
        __syncwarp();
        if (pend && !issue_v()) { ok = false; break; }
        pend = true;
        pend_seq = tile_seq;
        pend_zv = szk + tile_bytes;
        pend_bv = sbv;
        pend_st = st;
        pend_bx = bx;
        pend_last = (i == ntiles - 1);
      }
      ++unit_seq;
    }
    if (ok && pend) ok = issue_v();
    if (!ok && leader) raise_timeout(a, ms);
    // every MMA issued by this warp completes before TMEM is released
    if (leader) tc_commit(bar(BAR_FINAL));
    __syncwarp();
    int dummy = 0;
    mbar_wait_warp(bar(BAR_FINAL), 0, &dummy, kWaitNs);
  } else if (warp >= Roles<LAT>::kKFirst && warp < Roles<LAT>::kVFirst) {
    // ================================ key side ======================================
    constexpr int kNwg = Roles<LAT>::kNwg;
    const int wg = (warp - Roles<LAT>::kKFirst) >> 2;   // warpgroup: tiles of this parity
    const int q4 = warp & 3;                 // TMEM lane quarter = softmax stream
    const int row = q4 * 32 + lane;          // token within the tile
    const uint32_t lanebase = (uint32_t)(q4 * 32) << 16;
    const int tid = threadIdx.x - 32 * Roles<LAT>::kKFirst;  // across every key-side warp
    float* qs_all = reinterpret_cast<float*>(smem + p.off_q);   // [2][16][128]
    float* ps_all = reinterpret_cast<float*>(smem + p.off_p);   // [2][16][128]
    // chunks of 32 columns loaded per TMEM wait (register budget) and independent
    // partial sums per head (to break the FMA dependency chain)
    constexpr int kLd = GP >= 4 ? 1 : 2;   // 32-column chunks per TMEM wait (register budget)
    constexpr int kNpk = GP >= 4 ? 1 : 2;   // packed partial sums per head
    uint32_t tile_seq = 0;
    int unit_seq = 0;
    bool ok = true;
    while (ok) {
      const int us = unit_seq % kUR;
      if (!mbar_wait_warp(bar(BAR_UFULL + us), (unit_seq / kUR) & 1, abort_flag, kWaitNs)) { ok = false; break; }
      const int* d = ms->unit[us];
      if (d[6]) break;
      const int b = d[0], g = d[1], t0 = d[3], t1 = d[4], ntiles = d[5];
      // q of the G heads (bf16 in HBM) -> fp32 in shared memory, pre-scaled by
      // log2(e) / sqrt(d) so the scores come out in log2 units
      const int qx = unit_seq & 1;
      const float* qs = qs_all + qx * (16 * kD);
      {
        float* qw = qs_all + qx * (16 * kD);
        const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q) +
                                  ((size_t)b * a.Hq + (size_t)g * G) * kD;
        for (int idx = tid; idx < G * (kD / 8); idx += 128 * kNwg) {
          const int j = idx / (kD / 8), kc = idx % (kD / 8);
          const uint4 raw = *reinterpret_cast<const uint4*>(qg + (size_t)j * kD + kc * 8);
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
          float4 lo, hi;
          float2 f;
          f = __bfloat1622float2(h2[0]); lo.x = f.x * a.scale_log2; lo.y = f.y * a.scale_log2;
          f = __bfloat1622float2(h2[1]); lo.z = f.x * a.scale_log2; lo.w = f.y * a.scale_log2;
          f = __bfloat1622float2(h2[2]); hi.x = f.x * a.scale_log2; hi.y = f.y * a.scale_log2;
          f = __bfloat1622float2(h2[3]); hi.z = f.x * a.scale_log2; hi.w = f.y * a.scale_log2;
          *reinterpret_cast<float4*>(qw + j * kD + kc * 8) = lo;
          *reinterpret_cast<float4*>(qw + j * kD + kc * 8 + 4) = hi;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_QREADY + qx));
        if (!mbar_wait_warp(bar(BAR_QREADY + qx), (unit_seq >> 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
      }
      float m_run[GP], l_run[GP];
#pragma unroll
      for (int j = 0; j < GP; ++j) {
        m_run[j] = -CUDART_INF_F;
        l_run[j] = 0.f;
      }
      for (int i = 0; i < ntiles && ok; ++i) {
        const uint32_t ts = tile_seq + (uint32_t)i;     // tile index in this CTA's stream
        if (kNwg == 2 && (int)(ts & 1u) != wg) continue;
        const int x = (int)(ts & 1u);
        const uint32_t ph = (ts >> 1) & 1u;
        const int n_valid = min(kT, t1 - (t0 + i * kT));
        if (!mbar_wait_warp(bar(BAR_KFULL + x), ph, abort_flag, kWaitNs)) { ok = false; break; }
        tc_fence_after();
        // scores of this token against the G heads, straight from its fp32 key row;
        // packed fp32 FMAs, with two partial sums per head when G is small
        float2 dot[GP][kNpk];
#pragma unroll
        for (int j = 0; j < GP; ++j)
#pragma unroll
          for (int u = 0; u < kNpk; ++u) dot[j][u] = make_float2(0.f, 0.f);
#pragma unroll
        for (int c0 = 0; c0 < kD / 32; c0 += kLd) {
          uint32_t v[kLd][32];
#pragma unroll
          for (int cl = 0; cl < kLd; ++cl) tmem_ld32(tK(x) + lanebase + 32u * (c0 + cl), v[cl]);
          tmem_wait_ld();
          if (c0 + kLd == kD / 32) {
            // every column of the key slot has been read: it can be rebuilt again
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BAR_KFREE + x));
          }
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
#pragma unroll
            for (int cl = 0; cl < kLd; ++cl) {
              const float2 k01 = make_float2(__uint_as_float(v[cl][4 * e4 + 0]), __uint_as_float(v[cl][4 * e4 + 1]));
              const float2 k23 = make_float2(__uint_as_float(v[cl][4 * e4 + 2]), __uint_as_float(v[cl][4 * e4 + 3]));
#pragma unroll
              for (int j = 0; j < GP; ++j) {
                if (j < G) {
                  const float4 qq = *reinterpret_cast<const float4*>(qs + j * kD + 32 * (c0 + cl) + 4 * e4);
                  dot[j][0] = ffma2(k01, make_float2(qq.x, qq.y), dot[j][0]);
                  dot[j][kNpk - 1] = ffma2(k23, make_float2(qq.z, qq.w), dot[j][kNpk - 1]);
                }
              }
            }
          }
        }
        const bool valid = row < n_valid;
        float sk = 1.f, sv = 1.f;
        if (kQuant) {
          if (!mbar_wait_warp(bar(BAR_DQFULL + x), ph, abort_flag, kWaitNs)) { ok = false; break; }
          sk = ms->scl[x][0][row];
          sv = ms->scl[x][1][row];
        }
        // P(x) and alpha(x) are free once the value side has consumed the tile two back
        if (ts >= 2 &&
            !mbar_wait_warp(bar(BAR_PFREE + x), ((ts >> 1) - 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
        float* P = ps_all + x * (16 * kT);
#pragma unroll
        for (int j = 0; j < GP; ++j) {
          if (j < G) {
            float dj = 0.f;
#pragma unroll
            for (int u = 0; u < kNpk; ++u) dj += dot[j][u].x + dot[j][u].y;
            const float sj = valid ? dj * sk : -CUDART_INF_F;
            const float m_new = fmaxf(m_run[j], warp_max(sj));   // this stream's running max
            // a stream with no valid token yet keeps max -inf: nothing to rescale
            const float alpha = (m_new == -CUDART_INF_F) ? 1.f : exp2f(m_run[j] - m_new);
            const float pj = valid ? exp2f(sj - m_new) : 0.f;
            l_run[j] = l_run[j] * alpha + pj;
            m_run[j] = m_new;
            // masked tokens contribute an exact zero (their scale may be anything)
            P[j * kT + row] = valid ? pj * sv : 0.f;
            if (lane == 0) ms->alpha[x][q4][j] = alpha;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_PFULL + x));
      }
      if (!ok) break;
      tile_seq += (uint32_t)ntiles;
      // unit statistics of this warpgroup's streams for the value side
      const int sx = unit_seq & 1;
      if (unit_seq >= 2 && !mbar_wait_warp(bar(BAR_STEMPTY + 2 * sx + wg), ((unit_seq >> 1) - 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
#pragma unroll
      for (int j = 0; j < GP; ++j) {
        const float lw = warp_sum(l_run[j]);
        if (lane == 0) {
          ms->stat_l[sx][wg][q4][j] = lw;
          ms->stat_m[sx][wg][q4][j] = m_run[j];
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(BAR_STFULL + 2 * sx + wg));
        mbar_arrive(bar(BAR_UEMPTY + us));
      }
      ++unit_seq;
    }
    if (!ok) raise_timeout(a, ms);
  } else if (warp >= Roles<LAT>::kVFirst && warp < Roles<LAT>::kDQFirst) {
    // ================================ value side ====================================
    constexpr int kNwg = Roles<LAT>::kNwg;
    const int wg = (warp - Roles<LAT>::kVFirst) >> 2;   // warpgroup: tiles of this parity
    const int q4 = warp & 3;
    const int c = q4 * 32 + lane;            // output dimension
    const uint32_t lanebase = (uint32_t)(q4 * 32) << 16;
    const float* ps_all = reinterpret_cast<const float*>(smem + p.off_p);
    constexpr int kLd = GP >= 4 ? 1 : 2;   // 32-token chunks per TMEM wait (register budget)
    constexpr int kNpv = GP >= 4 ? 1 : 2;               // partial sums per (head, stream)
    uint32_t tile_seq = 0;
    int unit_seq = 0;
    bool ok = true;
    while (ok) {
      const int us = unit_seq % kUR;
      if (!mbar_wait_warp(bar(BAR_UFULL + us), (unit_seq / kUR) & 1, abort_flag, kWaitNs)) { ok = false; break; }
      const int* d = ms->unit[us];
      if (d[6]) break;
      const int b = d[0], g = d[1], s = d[2], t0 = d[3], t1 = d[4], ntiles = d[5];
      // per head and softmax stream (token chunk): packed partial sums
      float2 acc[GP][4][kNpv];
#pragma unroll
      for (int j = 0; j < GP; ++j)
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
          for (int u = 0; u < kNpv; ++u) acc[j][w][u] = make_float2(0.f, 0.f);
      for (int i = 0; i < ntiles && ok; ++i) {
        const uint32_t ts = tile_seq + (uint32_t)i;
        if (kNwg == 2 && (int)(ts & 1u) != wg) continue;
        const int x = (int)(ts & 1u);
        const uint32_t ph = (ts >> 1) & 1u;
        const int n_valid = min(kT, t1 - (t0 + i * kT));
        if (!mbar_wait_warp(bar(BAR_VFULL + x), ph, abort_flag, kWaitNs)) { ok = false; break; }
        tc_fence_after();
        const float* P = ps_all + x * (16 * kT);
#pragma unroll
        for (int w0 = 0; w0 < 4; w0 += kLd) {
          uint32_t v[kLd][32];
#pragma unroll
          for (int wl = 0; wl < kLd; ++wl) tmem_ld32(tV(x) + lanebase + 32u * (w0 + wl), v[wl]);
          // the value loads are in flight while P of this tile is awaited
          if (w0 == 0) {
            if (!mbar_wait_warp(bar(BAR_PFULL + x), ph, abort_flag, kWaitNs)) ok = false;
            if (ok) {
#pragma unroll
              for (int j = 0; j < GP; ++j)
                if (j < G)
#pragma unroll
                  for (int w = 0; w < 4; ++w) {
                    const float al = ms->alpha[x][w][j];
#pragma unroll
                    for (int u = 0; u < kNpv; ++u) {
                      acc[j][w][u].x *= al;
                      acc[j][w][u].y *= al;
                    }
                  }
            }
          }
          tmem_wait_ld();
          if (w0 + kLd == 4) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BAR_VFREE + x));
          }
          if (!ok) break;
#pragma unroll
          for (int wl = 0; wl < kLd; ++wl) {
            const int w = w0 + wl;
            if (32 * w + 32 > n_valid) {
              // token columns past the row's length: exact zeros, whatever the cache holds
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (32 * w + e >= n_valid) v[wl][e] = 0u;
            }
          }
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
#pragma unroll
            for (int wl = 0; wl < kLd; ++wl) {
#pragma unroll
              for (int j = 0; j < GP; ++j) {
                if (j < G) {
                  const int w = w0 + wl;
                  const float4 pp = *reinterpret_cast<const float4*>(P + j * kT + 32 * w + 4 * e4);
                  acc[j][w][0] = ffma2(make_float2(pp.x, pp.y),
                                       make_float2(__uint_as_float(v[wl][4 * e4 + 0]), __uint_as_float(v[wl][4 * e4 + 1])),
                                       acc[j][w][0]);
                  acc[j][w][kNpv - 1] = ffma2(make_float2(pp.z, pp.w),
                                              make_float2(__uint_as_float(v[wl][4 * e4 + 2]), __uint_as_float(v[wl][4 * e4 + 3])),
                                              acc[j][w][kNpv - 1]);
                }
              }
            }
          }
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_PFREE + x));
      }
      if (!ok) break;
      tile_seq += (uint32_t)ntiles;
      const int sx = unit_seq & 1;
      if (!mbar_wait_warp(bar(BAR_STFULL + 2 * sx + wg), (unit_seq >> 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
      // merge this warpgroup's four softmax streams of each head by their log-sum-exp:
      // numerator num / sum L relative to max M (log2 units)
      float num[GP], Ms[GP], Ls[GP];
#pragma unroll
      for (int j = 0; j < GP; ++j) {
        num[j] = 0.f;
        Ms[j] = -CUDART_INF_F;
        Ls[j] = 0.f;
        if (j < G) {
          const float m0 = ms->stat_m[sx][wg][0][j], m1 = ms->stat_m[sx][wg][1][j];
          const float m2 = ms->stat_m[sx][wg][2][j], m3 = ms->stat_m[sx][wg][3][j];
          const float M = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
          // a stream that never saw a valid token (max -inf) contributes nothing
          auto wgt = [&](float m) { return m == -CUDART_INF_F ? 0.f : exp2f(m - M); };
          const float f0 = wgt(m0), f1 = wgt(m1), f2 = wgt(m2), f3 = wgt(m3);
          Ls[j] = ms->stat_l[sx][wg][0][j] * f0 + ms->stat_l[sx][wg][1][j] * f1 +
                  ms->stat_l[sx][wg][2][j] * f2 + ms->stat_l[sx][wg][3][j] * f3;
          float aw[4];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            aw[w] = 0.f;
#pragma unroll
            for (int u = 0; u < kNpv; ++u) aw[w] += acc[j][w][u].x + acc[j][w][u].y;
          }
          num[j] = aw[0] * f0 + aw[1] * f1 + aw[2] * f2 + aw[3] * f3;
          Ms[j] = M;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_STEMPTY + 2 * sx + wg));
      if (kNwg == 2 && wg == 1) {
        // hand the second warpgroup's merged result to the first
        float* xo = reinterpret_cast<float*>(smem + p.off_x) + sx * (16 * kD);
        if (unit_seq >= 2 && !mbar_wait_warp(bar(BAR_XEMPTY + sx), ((unit_seq >> 1) - 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
#pragma unroll
        for (int j = 0; j < GP; ++j)
          if (j < G) {
            xo[j * kD + c] = num[j];
            if (c == 0) {
              ms->xm[sx][j] = Ms[j];
              ms->xl[sx][j] = Ls[j];
            }
          }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(BAR_XFULL + sx));
          mbar_arrive(bar(BAR_UEMPTY + us));
        }
        ++unit_seq;
        continue;
      }
      if (kNwg == 2) {
        const float* xo = reinterpret_cast<const float*>(smem + p.off_x) + sx * (16 * kD);
        if (!mbar_wait_warp(bar(BAR_XFULL + sx), (unit_seq >> 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
#pragma unroll
        for (int j = 0; j < GP; ++j)
          if (j < G) {
            const float M1 = ms->xm[sx][j], L1 = ms->xl[sx][j], n1 = xo[j * kD + c];
            const float M = fmaxf(Ms[j], M1);
            const float f0 = Ms[j] == -CUDART_INF_F ? 0.f : exp2f(Ms[j] - M);
            const float f1 = M1 == -CUDART_INF_F ? 0.f : exp2f(M1 - M);
            num[j] = num[j] * f0 + n1 * f1;
            Ls[j] = Ls[j] * f0 + L1 * f1;
            Ms[j] = M;
          }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_XEMPTY + sx));
      }
      const size_t hb = (size_t)b * a.Hq + (size_t)g * G;
#pragma unroll
      for (int j = 0; j < GP; ++j) {
        if (j < G) a.o_part[((hb + j) * a.S + s) * kD + c] = num[j] / Ls[j];
      }
      if (c < G) {
        float lc = 0.f;
#pragma unroll
        for (int j = 0; j < GP; ++j)
          if (j == c) lc = Ms[j] + log2f(Ls[j]);
        a.lse_part[(hb + c) * a.S + s] = lc * CUDART_LN2_F;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_UEMPTY + us));
      ++unit_seq;
    }
    if (!ok) raise_timeout(a, ms);
  } else if (kQuant && warp >= Roles<LAT>::kDQFirst) {
    // ============================ code -> bf16 converter ============================
    const int row = (warp - Roles<LAT>::kDQFirst) * 32 + lane;   // token within the tile
    const int W = p.W;
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
      for (int i = 0; i < ntiles && ok; ++i, ++tile_seq) {
        const int st = (int)(tile_seq % (uint32_t)p.nstage);
        const int x = (int)(tile_seq & 1u);
        if (!mbar_wait_warp(bar(BAR_FULL + st), (tile_seq / p.nstage) & 1, abort_flag, kWaitNs)) { ok = false; break; }
        if (tile_seq >= 2) {
          // operand slot x free (MMA2 of the tile two back done) and its scales read
          if (!mbar_wait_warp(bar(BAR_DQEMPTY + x), ((tile_seq >> 1) - 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
          if (!mbar_wait_warp(bar(BAR_PFULL + x), ((tile_seq >> 1) - 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
        }
        const uint8_t* stage = smem + p.off_stage + (size_t)st * p.stage_bytes;
        uint8_t* zop = smem + p.off_zop + (size_t)x * 2u * tile_bytes;
#pragma unroll
        for (int kv = 0; kv < 2; ++kv) {
          const uint8_t* src = stage + kv * cb + (size_t)row * r;
          uint8_t* dst = zop + kv * tile_bytes;
          for (int k0 = 0; k0 < r; k0 += 16) {
            const uint4 raw = *reinterpret_cast<const uint4*>(src + k0);
            const uint8_t* cbytes = reinterpret_cast<const uint8_t*>(&raw);
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float f0, f1;
              if (LAT == kLatI8) {
                f0 = (float)(int8_t)cbytes[2 * e];
                f1 = (float)(int8_t)cbytes[2 * e + 1];
              } else {
                __nv_fp8_e4m3 c0, c1;
                c0.__x = cbytes[2 * e];
                c1.__x = cbytes[2 * e + 1];
                f0 = (float)c0;
                f1 = (float)c1;
              }
              const __nv_bfloat162 bb = __floats2bfloat162_rn(f0, f1);
              w[e] = *reinterpret_cast<const uint32_t*>(&bb);
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
        const float* scs = reinterpret_cast<const float*>(stage + 2 * cb);
        ms->scl[x][0][row] = scs[row];
        ms->scl[x][1][row] = scs[kT + row];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(BAR_DQFULL + x));
          mbar_arrive(bar(BAR_EMPTY + st));
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_UEMPTY + us));
      ++unit_seq;
    }
    if (!ok) raise_timeout(a, ms);
  }

  // ---- tear-down -----------------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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
  int W, nkb, nstage, nbuf;
  uint32_t off_stage, stage_bytes, off_zop, off_b, off_q, off_p, off_x, off_misc, smem;
};

bool plan_layout(int r, bool quant, Layout* L) {
  if (r < 16 || r > 128 || r % 16) return false;
  const int rowb = 2 * r;
  L->W = (rowb % 128 == 0) ? 128 : (rowb % 64 == 0 ? 64 : 32);
  L->nkb = rowb / L->W;
  L->nbuf = (r <= 64) ? 2 : 1;
  const uint32_t tile = 128u * rowb;
  const uint32_t fac = (uint32_t)r * 256u;
  uint32_t off = 0;
  L->off_b = off;
  off += L->nbuf * 2u * fac;
  L->off_q = off;
  off += 2u * 16u * 128u * 4u;
  L->off_p = off;
  off += 2u * 16u * 128u * 4u;
  L->off_x = off;
  if (!quant) off += 2u * 16u * 128u * 4u;
  L->off_zop = off;
  if (quant) off += 2u * 2u * tile;
  L->off_misc = off;
  off += (uint32_t)((sizeof(Misc) + 1023) / 1024 * 1024);
  L->off_stage = off;
  L->stage_bytes = quant ? (uint32_t)(((2u * 128u * r + 2u * 512u) + 1023u) / 1024u * 1024u) : 2u * tile;
  const int avail = kSmemLimit - 1024 - (int)off;
  int ns = avail / (int)L->stage_bytes;
  if (ns > kMaxStages) ns = kMaxStages;
  if (ns < 2) return false;
  L->nstage = ns;
  L->smem = 1024u + off + (uint32_t)ns * L->stage_bytes;
  return true;
}

template <int LAT, int GP, bool EXACT>
cudaError_t launch_typed(const TcParams& prm, int grid, cudaStream_t st) {
  auto kern = lrkv_split_tc<LAT, GP, EXACT>;
  static int configured = 0;
  if ((int)prm.smem_bytes > configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)prm.smem_bytes);
    if (e != cudaSuccess) return e;
    configured = (int)prm.smem_bytes;
  }
  kern<<<grid, Roles<LAT>::kThreads, prm.smem_bytes, st>>>(prm);
  return cudaGetLastError();
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

bool tc_supported(const lrkv_dims& d, int* smem_bytes) {
  *smem_bytes = 0;
  if (d.io_dtype != LRKV_BF16 || d.d_head != 128) return false;
  if (d.latent_dtype != LRKV_BF16 && d.latent_dtype != LRKV_I8 && d.latent_dtype != LRKV_E4M3)
    return false;
  const int G = d.n_q_heads / d.n_kv_heads;
  if (G < 1 || G > 16) return false;
  const bool quant = d.latent_dtype != LRKV_BF16;
  if (quant && d.max_seq % 4 != 0) return false;
  if ((double)d.batch * d.n_kv_heads * d.max_seq >= 2147483647.0) return false;
  Layout L;
  if (!plan_layout(d.rank, quant, &L)) return false;
  *smem_bytes = (int)L.smem;
  return true;
}

cudaError_t launch_split_tc(const SplitArgs& a, const Plan& plan, cudaStream_t st) {
  const bool quant = a.latent_dtype != LRKV_BF16;
  Layout L;
  if (!plan_layout(a.r, quant, &L)) return cudaErrorInvalidValue;
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
  ok &= make_tmap_2d(&prm.tm_bk, a.BK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD,
                     (uint64_t)a.Hkv * a.r, 64, a.r, 128);
  ok &= make_tmap_2d(&prm.tm_bv, a.BV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD,
                     (uint64_t)a.Hkv * a.r, 64, a.r, 128);
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
  prm.off_q = L.off_q;
  prm.off_p = L.off_p;
  prm.off_x = L.off_x;
  prm.off_misc = L.off_misc;
  prm.smem_bytes = L.smem;
  switch (a.latent_dtype) {
    case LRKV_BF16: return launch_g<kLatBF16>(prm, plan.grid, st);
    case LRKV_I8: return launch_g<kLatI8>(prm, plan.grid, st);
    default: return launch_g<kLatE4M3>(prm, plan.grid, st);
  }
}

}  // namespace lrkv
