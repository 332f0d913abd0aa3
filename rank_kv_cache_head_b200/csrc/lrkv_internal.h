// Internal declarations shared by the kernels and the C-ABI layer of liblrkv.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "lrkv.h"

namespace lrkv {

constexpr int kTile = 128;            // tokens per pipeline tile / split granule
constexpr size_t kHeaderBytes = 256;  // workspace header: status word + counters

// Workspace header words.
enum HeaderWord {
  kStatusWord = 0, kWorkCounter = 1, kDoneCounter = 2, kProjCounter = 3,
  kChunkWord = 4,      // split size chosen on the device (tokens), read by the merge
  kProjHeadWord = 8,   // words 8..63: per-KV-head counters of the projection
};

// Split layout. A row is two segments when the factors are modality-separated:
// [0, n_visual) rebuilt with the visual set and [n_visual, L) with the text set
// (one segment [0, L) otherwise, n_visual = 0). Each segment is cut into splits of
// `chunk` tokens; the visual splits come first. No split straddles the boundary.
__host__ __device__ inline int visual_splits(int n_visual, int max_seqlen, int chunk) {
  const int P = n_visual < max_seqlen ? n_visual : max_seqlen;
  return (P + chunk - 1) / chunk;
}
__host__ __device__ inline int total_splits(int n_visual, int max_seqlen, int chunk) {
  const int rest = max_seqlen > n_visual ? max_seqlen - n_visual : 0;
  const int S = visual_splits(n_visual, max_seqlen, chunk) + (rest + chunk - 1) / chunk;
  return S > 0 ? S : 1;
}
// Token range [t0, t1) of split s in a row of length L (empty when t0 >= t1), and
// the factor set it uses (0 visual / single set, 1 text).
__host__ __device__ inline int split_range(int s, int L, int n_visual, int max_seqlen, int chunk,
                                           int* t0, int* t1) {
  const int sv = visual_splits(n_visual, max_seqlen, chunk);
  if (s < sv) {
    *t0 = s * chunk;
    const int end = L < n_visual ? L : n_visual;
    *t1 = end < *t0 + chunk ? end : *t0 + chunk;
    return 0;
  }
  *t0 = n_visual + (s - sv) * chunk;
  *t1 = L < *t0 + chunk ? L : *t0 + chunk;
  return n_visual > 0 ? 1 : 0;
}

// Launch plan for one call (depends only on dims and the device).
struct Plan {
  int algo;         // LRKV_ALGO_SIMT or LRKV_ALGO_TCGEN05
  int S;            // splits per (b, KV head) at max_seqlen
  int chunk;        // tokens per split, multiple of kTile (device_chunk: the finest)
  int device_chunk; // the tensor-core kernel picks the split size from the actual lengths
  int chunk_hint;   // device_chunk: tiles per split for rows at full length
  int grid;         // CTAs of the split kernel
  int smem;         // dynamic shared memory of the split kernel
  size_t lse_off;   // byte offset of lse partials in the workspace
  size_t o_off;     // byte offset of o partials
  size_t ws_bytes;  // total workspace bytes
};

// Everything the split kernels read (device pointers and sizes).
struct SplitArgs {
  const void* q;
  const void* ZK;
  const void* ZV;
  const float* SK;
  const float* SV;
  const void* BK;
  const void* BV;
  const int32_t* seqlens;
  float* o_part;    // [B][Hq][S][d]
  float* lse_part;  // [B][Hq][S]
  uint32_t* header;
  int B, Hq, Hkv, G, d, r, Lcap, max_seqlen, S, chunk;
  int io_dtype, latent_dtype;
  float scale_log2;  // log2(e) / sqrt(d)
  int debug_stall;   // test hook: work unit 0's first tile is withheld (see lrkv.h)
  int device_chunk;  // choose the split size on the device (chunk = the finest, S its bound)
  int chunk_hint;    // device_chunk: the split size, in tiles, for rows at full length
  int n_visual;      // > 0: modality-separated factors, BK/BV [2][Hkv][r][d]
};

struct MergeArgs {
  const float* o_part;
  const float* lse_part;
  const int32_t* seqlens;
  void* out;
  float* lse_out;
  uint32_t* header;
  int B, Hq, d, S, chunk, Lcap, max_seqlen;
  int io_dtype;
  int n_visual;      // split layout (see split_range)
  int device_chunk;  // read the split size the split kernel chose from the header
};

struct AppendArgs {
  const void* zk_new;
  const void* zv_new;
  void* ZK;
  void* ZV;
  float* SK;
  float* SV;
  int32_t* seqlens;
  uint32_t* header;
  int B, Hkv, r, Lcap;
  int io_dtype, latent_dtype;
};

// The fused latent projection + append: the new token's latents z = x A_g are
// computed here instead of being passed in.
struct ProjArgs {
  AppendArgs app;   // zk_new / zv_new unused
  const void* x;    // [B][d_model], io dtype
  const void* AK;   // [Hkv][d_model][r], io dtype
  const void* AV;
  int d_model;
  int nsplit;       // CTAs sharing one (KV head, K|V) over the hidden size
  float* part;      // nsplit > 1: [2 Hkv][nsplit][B][r] partial sums (workspace)
};

// Programmatic dependent launch: every kernel of the library is launched so that it
// may start while the previous kernel of the stream finishes, and waits for that
// kernel (and so, transitively, every earlier one) before it touches memory they
// produce; each kernel lets its dependent launch as soon as it has started.
#ifdef __CUDACC__
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
#endif

// cudaLaunchKernelEx with the programmatic-stream-serialization attribute.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Launchers (return a cudaError_t from the launch).
cudaError_t launch_split_simt(const SplitArgs& a, const Plan& p, cudaStream_t st);
cudaError_t launch_merge(const MergeArgs& a, cudaStream_t st);
cudaError_t launch_append(const AppendArgs& a, cudaStream_t st);
cudaError_t launch_project_append(const ProjArgs& a, cudaStream_t st);
// hidden-size split of the projection for this workspace size (1: none)
int project_nsplit(int Hkv, int B, int r, int d_model, int io_bytes, size_t workspace_bytes);

// tcgen05 path: whether it supports these dims, its shared memory per CTA and CTAs
// per SM, and the launcher.
bool tc_supported(const lrkv_dims& d, int* smem_bytes, int* ctas_per_sm);
cudaError_t launch_split_tc(const SplitArgs& a, const Plan& p, cudaStream_t st);

int num_sms();

}  // namespace lrkv
