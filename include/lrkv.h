/*
 * lrkv.h - C ABI of liblrkv.so: single-token decode attention over a per-head
 * low-rank (SVD-factored) KV cache, for NVIDIA B200 (sm_100a).
 *
 * The operation. Each KV head g keeps only latents Z_K,g and Z_V,g (L x r) and
 * small up-projection factors B_K,g and B_V,g (r x d_head), from the per-head
 * factorisation W_K,g = A_K,g B_K,g of "WSVD: Weighted Low-Rank Approximation for
 * Fast and Efficient Execution of Low-Precision Vision-Language Models" (section 2.A,
 * per-head SVD). One decode step rebuilds K_g = Z_K,g B_K,g and V_g = Z_V,g B_V,g
 * tile by tile in on-chip memory (never in HBM) and consumes them at once:
 *     out[b][h] = softmax(q[b][h] . K_g^T / sqrt(d_head)) . V_g,   g = h / G,
 * with reconstruction, attention and Flash Decoding fused into one flow (same page,
 * section 2.C). The sequence is split across CTAs (split-KV / Flash Decoding); each
 * split writes a normalised partial and its log-sum-exp, and a second kernel merges
 * them: out = sum_s exp(lse_s - LSE) o_s, LSE = log sum_s exp(lse_s).
 * Query head h reads KV head h / G with G = n_q_heads / n_kv_heads (contiguous
 * groups).
 *
 * Conventions for every entry point:
 *  - All tensor arguments are DEVICE pointers unless stated otherwise; all are
 *    contiguous, row-major, in the layouts given below. The caller owns and
 *    allocates every buffer; the library allocates no device memory, launches only
 *    on the given stream (a cudaStream_t passed as void*, NULL = legacy default
 *    stream) and never synchronises, except lrkv_read_status and
 *    lrkv_decode_step_host's documented copies.
 *  - Return value: 0 on success, a negative LRKV_ERR_* code otherwise; on a
 *    negative return nothing was launched. lrkv_strerror() names each code.
 *  - Errors that only the device can see (a sequence length outside [0, max_seq]
 *    or above the max_seqlen planning hint, an append into a full cache, a pipeline
 *    wait that ran out of time) are OR-ed into the status word at the start of the
 *    workspace; the affected batch row's output is written as zeros with
 *    lse = -inf. Read it with lrkv_read_status.
 *
 * Layouts (B = batch, Hq = n_q_heads, Hkv = n_kv_heads, d = d_head, r = rank,
 * Lc = max_seq, the cache capacity):
 *   q, out          [B][Hq][d]          io_dtype
 *   ZK, ZV          [B][Hkv][Lc][r]     latent_dtype (int8 codes, or e4m3 bytes)
 *   ZK_scale/ZV_scale [B][Hkv][Lc]      fp32, one per token (I8/E4M3 only)
 *   BK, BV          [Hkv][r][d]         io_dtype
 *                   [2][Hkv][r][d] when n_visual > 0 (visual set, then text set)
 *   seqlens         [B]                 int32, valid positions per row
 *   lse_out         [B][Hq]             fp32, natural log (optional)
 */
#ifndef LRKV_H
#define LRKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LRKV_VERSION 2

/* element types */
typedef enum {
  LRKV_F32 = 0,  /* IEEE binary32 */
  LRKV_BF16 = 1, /* bfloat16 */
  LRKV_I8 = 2,   /* int8 codes in [-127, 127], value = code * per-token scale */
  LRKV_E4M3 = 3  /* OCP FP8 E4M3FN byte, value = decode(code) * per-token scale */
} lrkv_dtype;

/* kernel selection */
typedef enum {
  LRKV_ALGO_AUTO = 0,    /* tensor-core kernel when the shape allows, else CUDA-core */
  LRKV_ALGO_SIMT = 1,    /* CUDA-core fp32 kernel (every dtype and shape) */
  LRKV_ALGO_TCGEN05 = 2  /* tcgen05/TMEM/TMA kernel: io BF16, latent BF16/I8/E4M3,
                            d_head 128, rank a multiple of 16 up to 128, G <= 16 */
} lrkv_algo;

/* return codes */
#define LRKV_OK 0
#define LRKV_ERR_DIMS (-1)        /* invalid dimensions */
#define LRKV_ERR_DTYPE (-2)       /* unsupported dtype combination */
#define LRKV_ERR_ALIGN (-3)       /* a pointer is not 16-byte aligned */
#define LRKV_ERR_WORKSPACE (-4)   /* workspace missing or too small */
#define LRKV_ERR_LAUNCH (-5)      /* a CUDA launch or copy failed */
#define LRKV_ERR_UNSUPPORTED (-6) /* the requested algo cannot run this shape */
#define LRKV_ERR_ARG (-7)         /* a required pointer is NULL */

/* device status bits (OR-ed into the workspace status word) */
#define LRKV_STATUS_SEQLEN_RANGE 1u  /* seqlens[b] < 0 or > max_seq */
#define LRKV_STATUS_SEQLEN_HINT 2u   /* seqlens[b] > max_seqlen planning hint */
#define LRKV_STATUS_APPEND_FULL 4u   /* append with seqlens[b] >= max_seq: row skipped */
#define LRKV_STATUS_TIMEOUT 8u       /* a pipeline wait gave up; results invalid */

/*
 * Problem description, passed by pointer to every call.
 *  batch, n_q_heads, n_kv_heads >= 1, n_q_heads % n_kv_heads == 0;
 *  d_head in {64, 128}; rank in [8, 256], a multiple of 8;
 *  max_seq (Lc) >= 1: capacity, i.e. the row stride of ZK/ZV in tokens;
 *  max_seqlen in [0, max_seq]: host-side planning hint, an upper bound on every
 *      seqlens[b] seen by lrkv_decode_attn (a row above it is flagged and zeroed);
 *  io_dtype: LRKV_F32 or LRKV_BF16 (q, out, BK, BV, and the append inputs);
 *  latent_dtype: any lrkv_dtype (F32 latents require F32 io);
 *  num_splits: 0 = choose automatically, else the split count to use (clamped to
 *      the number of 128-token tiles of max_seqlen);
 *  algo: an lrkv_algo;
 *  n_visual: 0 = one factor set. Otherwise modality-separated factors
 *      ("AttentionPack", Metodologia 2.A: visual and text tokens are compressed
 *      separately, their distributions differ): positions [0, n_visual) of every
 *      row are rebuilt with the first (visual) factor set and positions >= n_visual
 *      with the second (text) set, BK/BV [2][Hkv][r][d]. A multiple of 16 in
 *      [0, max_seq]. The split size is chosen as without it; splits are then laid
 *      out over the two segments separately, so none straddles the boundary.
 */
typedef struct {
  int32_t batch;
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t d_head;
  int32_t rank;
  int32_t max_seq;
  int32_t max_seqlen;
  int32_t io_dtype;
  int32_t latent_dtype;
  int32_t num_splits;
  int32_t algo;
  int32_t n_visual;
} lrkv_dims;

/* What lrkv_decode_attn will do for these dims (for tests and benchmarks). */
typedef struct {
  int32_t algo;         /* LRKV_ALGO_SIMT or LRKV_ALGO_TCGEN05 */
  int32_t num_splits;   /* S: the most splits per (batch row, KV head), at max_seqlen */
  int32_t chunk;        /* tokens per split (a multiple of 128); with device_chunk the
                           finest the kernel may pick */
  int32_t grid;         /* CTAs of the split kernel */
  int32_t smem_bytes;   /* dynamic shared memory of the split kernel */
  int32_t full_chunk;   /* tokens per split when every row is at max_seqlen */
  int32_t device_chunk; /* 1: the kernel scales full_chunk by the share of 128-token
                           tiles the rows hold (clamped to [chunk, full_chunk]) */
  int32_t reserved;
} lrkv_plan_info;

/* Fill *plan for dims. Returns 0 or a negative code. */
int lrkv_plan(const lrkv_dims* dims, lrkv_plan_info* plan);

/*
 * Bytes of device workspace lrkv_decode_attn / lrkv_append need for dims: a 256-byte
 * header (status word, scheduler counters) followed by the split partials
 * (fp32 lse [B][Hq][S] and fp32 o [B][Hq][S][d]). Returns 0 for invalid dims.
 * The workspace must be zero-filled once before its first use (lrkv_workspace_init
 * or any memset); afterwards the library keeps its header consistent itself.
 */
size_t lrkv_workspace_bytes(const lrkv_dims* dims);

/* Zero the workspace header on the stream (asynchronous). */
int lrkv_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode attention for one new token per batch row (one layer).
 * Inputs q, ZK, ZV, (ZK_scale, ZV_scale), BK, BV, seqlens; output out [B][Hq][d]
 * in io_dtype and, when lse_out is not NULL, the fp32 natural-log LSE per (b, h).
 * ZK_scale/ZV_scale must be non-NULL exactly for I8/E4M3 latents.
 * Positions t >= seqlens[b] of ZK/ZV/scales are never used (they may hold NaN).
 * A row with seqlens[b] == 0 gets out = 0 and lse = -inf.
 * q, ZK, ZV, BK, BV, out and the workspace must be 16-byte aligned, and
 * r * sizeof(latent) must be a multiple of 16 bytes (LRKV_ERR_ALIGN otherwise).
 * Launches the split kernel and the merge kernel on stream.
 */
int lrkv_decode_attn(const lrkv_dims* dims, const void* q, const void* ZK, const void* ZV,
                     const float* ZK_scale, const float* ZV_scale, const void* BK,
                     const void* BV, const int32_t* seqlens, void* out, float* lse_out,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * Same as lrkv_decode_attn, and additionally records ev_split_begin / ev_split_end
 * (cudaEvent_t handles created by the caller, either may be NULL) on stream
 * immediately before and after the split kernel, so that kernel's duration can be
 * read with cudaEventElapsedTime. While the stream is being captured into a CUDA
 * graph the events are recorded as external event nodes.
 */
int lrkv_decode_attn_timed(const lrkv_dims* dims, const void* q, const void* ZK,
                           const void* ZV, const float* ZK_scale, const float* ZV_scale,
                           const void* BK, const void* BV, const int32_t* seqlens, void* out,
                           float* lse_out, void* workspace, size_t workspace_bytes,
                           void* stream, void* ev_split_begin, void* ev_split_end);

/*
 * Append one new latent row per (batch row, KV head): writes zk_new/zv_new
 * ([B][Hkv][r], io_dtype) into slot seqlens[b] of ZK/ZV and then sets
 * seqlens[b] += 1 (device-side, in place). For I8 latents the row is quantised
 * with scale = absmax / 127 (fp32 IEEE division; an all-zero row gets scale 1) and
 * code = round-half-even(z / scale) clamped to [-127, 127]; for E4M3 with
 * scale = absmax / 448 and code = round-to-nearest-even, saturating. The scale is
 * written to ZK_scale/ZV_scale at the same slot. A row whose slot is >= max_seq is
 * left unchanged and LRKV_STATUS_APPEND_FULL is raised. This is the cache-side
 * step that precedes attention in a decode step; the latent itself (x A_K,g, the
 * token's projection onto the per-head down factor, WSVD section 2.A) is computed
 * upstream.
 */
int lrkv_append(const lrkv_dims* dims, const void* zk_new, const void* zv_new, void* ZK,
                void* ZV, float* ZK_scale, float* ZV_scale, int32_t* seqlens,
                void* workspace, size_t workspace_bytes, void* stream);

/*
 * One full decode step with HOST inputs and output: copies q_host and the new
 * latent rows (pinned host memory recommended) to the device staging buffers
 * q_dev / zk_new_dev / zv_new_dev, runs lrkv_append and lrkv_decode_attn, and
 * copies out_dev back to out_host, all on stream (asynchronous: synchronise the
 * stream before reading out_host). The cache (ZK, ZV, scales, BK, BV, seqlens) stays
 * resident on the device.
 */
int lrkv_decode_step_host(const lrkv_dims* dims, const void* q_host, const void* zk_new_host,
                          const void* zv_new_host, void* out_host, void* q_dev,
                          void* zk_new_dev, void* zv_new_dev, void* out_dev, void* ZK,
                          void* ZV, float* ZK_scale, float* ZV_scale, const void* BK,
                          const void* BV, int32_t* seqlens, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * Fused latent projection + append, the step that produces the row lrkv_append
 * writes ("WSVD: Weighted Low-Rank Approximation for Fast and Efficient Execution of
 * Low-Precision Vision-Language Models", section 2.A: the cached latent of a head is
 * the token's hidden state times that head's down factor A, W = A B). For every batch
 * row b and KV head g:
 *     z_K = x[b] . AK[g],   z_V = x[b] . AV[g]     (fp32 accumulation)
 * written at slot seqlens[b] exactly as lrkv_append writes a row (fp32, bf16 RNE, or
 * int8 / e4m3 codes with a per-row fp32 absmax scale), then seqlens[b] += 1.
 *   x      [B][d_model], io dtype, device
 *   AK, AV [H_kv][d_model][rank], io dtype, device, 16-byte aligned
 *   other arguments as lrkv_append. Only the workspace's 256-byte header is used.
 *   The hidden size is split over up to 8 CTAs per factor (one thread-block
 *   cluster) that add their partial sums through distributed shared memory in a
 *   fixed order, so a call is deterministic.
 * Errors: LRKV_ERR_DIMS (dims, d_model outside [1, 2^20]), LRKV_ERR_ARG (NULL pointer,
 * scales present iff quantised latents), LRKV_ERR_ALIGN, LRKV_ERR_WORKSPACE,
 * LRKV_ERR_LAUNCH. A row whose slot is past the capacity is left untouched, keeps its
 * length and sets LRKV_STATUS_APPEND_FULL. LRKV_STATUS_TIMEOUT: the wait for a factor
 * copy into shared memory ran out after one second (the appended rows are invalid).
 */
int lrkv_project_append(const lrkv_dims* dims, int32_t d_model, const void* x, const void* AK,
                        const void* AV, void* ZK, void* ZV, float* ZK_scale, float* ZV_scale,
                        int32_t* seqlens, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode attention for callers that cannot allocate device memory (a host program
 * without a device memory manager, or a runtime whose memory budget forbids new
 * allocations while it serves). The paper has no counterpart: this is a deployment
 * convenience. Same inputs, outputs and semantics as lrkv_decode_attn, but no
 * workspace argument: the scratch (split partials, status word, scheduler counters)
 * is a fixed LRKV_NOALLOC_MAX_WORKSPACE_BYTES area inside the library's own device
 * memory, which every GPU that loads the library holds until the process exits.
 *  - Allocates nothing. Returns LRKV_ERR_WORKSPACE when lrkv_workspace_bytes(dims)
 *    exceeds LRKV_NOALLOC_MAX_WORKSPACE_BYTES.
 *  - The first call on a device looks up the area's device address
 *    (cudaGetSymbolAddress, once per device, with that device current); make that
 *    first call before any stream capture.
 *  - Every call clears the area's header and reuses the rest, which keeps the
 *    previous call's partials. All calls share one area per device, so calls that can
 *    overlap on the GPU (different streams without ordering) race: serialise them.
 *  - status_out (optional, DEVICE pointer): receives this call's device status word
 *    (LRKV_STATUS_* bits), written on stream after the kernels.
 */
#define LRKV_NOALLOC_MAX_WORKSPACE_BYTES (16u << 20)
int lrkv_decode_attn_noalloc(const lrkv_dims* dims, const void* q, const void* ZK,
                             const void* ZV, const float* ZK_scale, const float* ZV_scale,
                             const void* BK, const void* BV, const int32_t* seqlens, void* out,
                             float* lse_out, uint32_t* status_out, void* stream);

/*
 * Test hook for the bounded-wait error path (the paper has no counterpart). With on
 * != 0, the next tensor-core split launch (and only that one) runs with the producer
 * of the CTA that takes work unit 0 withholding the copy and the arrival of that
 * unit's first latent tile: the mbarrier waits on that tile run out after their
 * one-second bound, that CTA unwinds
 * (it drains its own copies and MMAs and frees its tensor memory) and the launch
 * sets LRKV_STATUS_TIMEOUT in the workspace status word; the other CTAs finish
 * normally and the context stays usable. Outputs of such a launch are not valid.
 * Returns 0.
 */
int lrkv_debug_stall_next_launch(int32_t on);

/*
 * Synchronise stream, copy the workspace status word to *status and clear it.
 * Returns 0, or LRKV_ERR_LAUNCH if the copy failed.
 */
int lrkv_read_status(void* workspace, void* stream, uint32_t* status);

/* Static description of a return code. */
const char* lrkv_strerror(int code);

/* LRKV_VERSION of the loaded library. */
int lrkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LRKV_H */
