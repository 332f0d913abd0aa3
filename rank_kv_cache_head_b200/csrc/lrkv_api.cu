// C ABI of liblrkv (declared in include/lrkv.h): argument checks, the split plan,
// the workspace layout and the kernel launches. No device memory is allocated here.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <functional>
#include <map>
#include <mutex>
#include <queue>
#include <tuple>
#include <vector>

#include "lrkv_ext_internal.h"
#include "lrkv_internal.h"
#include "lrkv_adaptive.h"
#include "lrkv_shared.h"

namespace lrkv {

size_t simt_smem_bytes(int r, int d, int G);

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

namespace {

// set by lrkv_debug_stall_next_launch, consumed by the next tensor-core launch
std::atomic<int> g_debug_stall{0};

size_t dtype_bytes(int t) { return t == LRKV_F32 ? 4 : (t == LRKV_BF16 ? 2 : 1); }

int check_dims(const lrkv_dims* d) {
  if (!d) return LRKV_ERR_ARG;
  if (d->batch < 1 || d->n_q_heads < 1 || d->n_kv_heads < 1) return LRKV_ERR_DIMS;
  if (d->n_q_heads % d->n_kv_heads != 0) return LRKV_ERR_DIMS;
  if (d->d_head != 64 && d->d_head != 128) return LRKV_ERR_DIMS;
  if (d->rank < 8 || d->rank > 256 || d->rank % 8 != 0) return LRKV_ERR_DIMS;
  if (d->max_seq < 1 || d->max_seqlen < 0 || d->max_seqlen > d->max_seq) return LRKV_ERR_DIMS;
  if (d->num_splits < 0) return LRKV_ERR_DIMS;
  if (d->n_visual < 0 || d->n_visual > d->max_seq || d->n_visual % 16 != 0) return LRKV_ERR_DIMS;
  if (d->io_dtype != LRKV_F32 && d->io_dtype != LRKV_BF16) return LRKV_ERR_DTYPE;
  if (d->latent_dtype < LRKV_F32 || d->latent_dtype > LRKV_E4M3) return LRKV_ERR_DTYPE;
  if (d->latent_dtype == LRKV_F32 && d->io_dtype != LRKV_F32) return LRKV_ERR_DTYPE;
  if (d->algo < LRKV_ALGO_AUTO || d->algo > LRKV_ALGO_TCGEN05) return LRKV_ERR_DIMS;
  if ((size_t)d->rank * dtype_bytes(d->latent_dtype) % 16 != 0) return LRKV_ERR_ALIGN;
  // element counts must stay well inside int64 and the partial index space
  const double cache = (double)d->batch * d->n_kv_heads * d->max_seq * d->rank;
  if (cache > 9.0e15) return LRKV_ERR_DIMS;
  return LRKV_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Makespan of greedy list scheduling of the split units on P persistent CTAs, in
// tile units, when every row has max_seqlen tokens. Units are taken in the order
// the kernels use (split index outermost), each by the CTA that frees up first.
double simulate_makespan(int rows, int tiles_max, int chunk_tiles, int P, double overhead) {
  const int S = (tiles_max + chunk_tiles - 1) / chunk_tiles;
  std::priority_queue<double, std::vector<double>, std::greater<double>> free_at;
  for (int i = 0; i < P; ++i) free_at.push(0.0);
  double makespan = 0.0;
  for (int s = 0; s < S; ++s) {
    const int ntiles = std::min(chunk_tiles, tiles_max - s * chunk_tiles);
    const double cost = ntiles + overhead;
    for (int u = 0; u < rows; ++u) {
      double t = free_at.top();
      free_at.pop();
      t += cost;
      makespan = std::max(makespan, t);
      free_at.push(t);
    }
  }
  return makespan;
}

int choose_chunk_tiles(int rows, int tiles_max, int P) {
  // a unit costs its tiles plus a fixed overhead (factor load, pipeline drain,
  // partial write); among plans within 0.5% of the best, take the longest chunk
  // (fewer partials to write and merge)
  static const int cands[] = {1, 2, 3, 4, 5, 6, 8, 10, 12, 16, 20, 24, 32, 48, 64, 96, 128};
  double t[sizeof(cands) / sizeof(cands[0])];
  double best_t = 1e300;
  int n = 0;
  for (int c : cands) {
    if (c > tiles_max && c != 1) break;
    t[n] = simulate_makespan(rows, tiles_max, c, P, 0.6);
    best_t = std::min(best_t, t[n]);
    ++n;
  }
  int best = 1;
  for (int i = 0; i < n; ++i)
    if (t[i] <= best_t * 1.005) best = cands[i];
  return best;
}

int make_plan(const lrkv_dims* d, Plan* p) {
  int rc = check_dims(d);
  if (rc) return rc;
  const int G = d->n_q_heads / d->n_kv_heads;
  int tc_smem = 0, tc_ctas = 0;
  const bool tc_ok = tc_supported(*d, &tc_smem, &tc_ctas);
  if (d->algo == LRKV_ALGO_TCGEN05 && !tc_ok) return LRKV_ERR_UNSUPPORTED;
  p->algo = (d->algo == LRKV_ALGO_SIMT || !tc_ok) ? LRKV_ALGO_SIMT : LRKV_ALGO_TCGEN05;

  const int tiles_max = std::max(1, (d->max_seqlen + kTile - 1) / kTile);
  const int rows = d->batch * d->n_kv_heads;
  // persistent CTAs of the split kernel (the tensor-core kernel runs two per SM when
  // its tiles fit); the SIMT kernel's plan is sized against the SM count
  const int P = num_sms() * (p->algo == LRKV_ALGO_TCGEN05 ? tc_ctas : 1);
  int chunk_tiles;
  if (d->num_splits > 0) {
    const int S = std::min(d->num_splits, tiles_max);
    chunk_tiles = (tiles_max + S - 1) / S;
  } else {
    static std::mutex mu;
    static std::map<std::tuple<int, int, int>, int> memo;
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_tuple(rows, tiles_max, P);
    auto it = memo.find(key);
    if (it != memo.end()) {
      chunk_tiles = it->second;
    } else {
      chunk_tiles = choose_chunk_tiles(rows, tiles_max, P);
      memo[key] = chunk_tiles;
    }
  }
  p->device_chunk = 0;
  p->chunk_hint = chunk_tiles;
  if (p->algo == LRKV_ALGO_TCGEN05 && d->num_splits == 0 && chunk_tiles > 1) {
    // the kernel scales the split size down to the tiles the rows actually hold;
    // the plan (workspace, merge bound) is for the finest it may pick
    p->device_chunk = 1;
    chunk_tiles = (chunk_tiles + 3) / 4;
  }
  p->chunk = chunk_tiles * kTile;
  p->S = total_splits(d->n_visual, d->max_seqlen, p->chunk);
  if (p->algo == LRKV_ALGO_TCGEN05) {
    p->smem = tc_smem;
    p->grid = std::min(P, rows * p->S);
  } else {
    const size_t sm = simt_smem_bytes(d->rank, d->d_head, G);
    if (sm > 227 * 1024) return LRKV_ERR_UNSUPPORTED;
    p->smem = (int)sm;
    p->grid = rows * p->S;
  }
  const size_t parts = (size_t)d->batch * d->n_q_heads * p->S;
  p->lse_off = kHeaderBytes;
  p->o_off = kHeaderBytes + ((parts * sizeof(float) + 255) / 256) * 256;
  p->ws_bytes = p->o_off + parts * d->d_head * sizeof(float);
  return LRKV_OK;
}

}  // namespace
}  // namespace lrkv

using namespace lrkv;

extern "C" {

int lrkv_version(void) { return LRKV_VERSION; }

const char* lrkv_strerror(int code) {
  switch (code) {
    case LRKV_OK: return "success";
    case LRKV_ERR_DIMS: return "invalid dimensions";
    case LRKV_ERR_DTYPE: return "unsupported dtype combination";
    case LRKV_ERR_ALIGN: return "pointer or row not 16-byte aligned";
    case LRKV_ERR_WORKSPACE: return "workspace missing or too small";
    case LRKV_ERR_LAUNCH: return "CUDA launch or copy failed";
    case LRKV_ERR_UNSUPPORTED: return "requested kernel cannot run this shape";
    case LRKV_ERR_ARG: return "required pointer is NULL";
    default: return "unknown error";
  }
}

int lrkv_plan(const lrkv_dims* dims, lrkv_plan_info* info) {
  if (!info) return LRKV_ERR_ARG;
  Plan p;
  int rc = make_plan(dims, &p);
  if (rc) return rc;
  memset(info, 0, sizeof(*info));
  info->algo = p.algo;
  info->num_splits = p.S;
  info->chunk = p.chunk;
  info->grid = p.grid;
  info->smem_bytes = p.smem;
  info->full_chunk = p.chunk_hint * kTile;
  info->device_chunk = p.device_chunk;
  return LRKV_OK;
}

size_t lrkv_workspace_bytes(const lrkv_dims* dims) {
  Plan p;
  if (make_plan(dims, &p)) return 0;
  return p.ws_bytes;
}

int lrkv_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace) return LRKV_ERR_ARG;
  if (workspace_bytes < kHeaderBytes) return LRKV_ERR_WORKSPACE;
  if (cudaMemsetAsync(workspace, 0, kHeaderBytes, (cudaStream_t)stream) != cudaSuccess)
    return LRKV_ERR_LAUNCH;
  return LRKV_OK;
}

static void record_event(void* ev, cudaStream_t st) {
  if (!ev) return;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags((cudaEvent_t)ev, st, cudaEventRecordExternal);
  else
    cudaEventRecord((cudaEvent_t)ev, st);
}

int lrkv_decode_attn(const lrkv_dims* dims, const void* q, const void* ZK, const void* ZV,
                     const float* ZK_scale, const float* ZV_scale, const void* BK,
                     const void* BV, const int32_t* seqlens, void* out, float* lse_out,
                     void* workspace, size_t workspace_bytes, void* stream) {
  return lrkv_decode_attn_timed(dims, q, ZK, ZV, ZK_scale, ZV_scale, BK, BV, seqlens, out,
                                lse_out, workspace, workspace_bytes, stream, nullptr, nullptr);
}

// The decode attention call behind every entry point. ad != nullptr: the attention-
// aware partial decompression (CUDA-core kernel with a per-token rank, then the
// moving average of the attention mass after the merge).
static int decode_impl(const lrkv_dims* dims, const void* q, const void* ZK, const void* ZV,
                       const float* ZK_scale, const float* ZV_scale, const void* BK,
                       const void* BV, const int32_t* seqlens, void* out, float* lse_out,
                       void* workspace, size_t workspace_bytes, void* stream,
                       void* ev_split_begin, void* ev_split_end, const AdaptArgs* ad,
                       float beta, bool shared = false) {
  Plan p;
  int rc = make_plan(dims, &p);
  if (rc) return rc;
  if ((ad || shared) && p.algo != LRKV_ALGO_SIMT) return LRKV_ERR_UNSUPPORTED;
  const bool quant = dims->latent_dtype == LRKV_I8 || dims->latent_dtype == LRKV_E4M3;
  if (!q || !ZK || !ZV || !BK || !BV || !seqlens || !out || !workspace) return LRKV_ERR_ARG;
  if (quant != (ZK_scale != nullptr) || quant != (ZV_scale != nullptr)) return LRKV_ERR_ARG;
  if (!aligned16(q) || !aligned16(ZK) || !aligned16(ZV) || !aligned16(BK) || !aligned16(BV) ||
      !aligned16(out) || !aligned16(workspace))
    return LRKV_ERR_ALIGN;
  if (quant && ((reinterpret_cast<uintptr_t>(ZK_scale) | reinterpret_cast<uintptr_t>(ZV_scale)) & 3u))
    return LRKV_ERR_ALIGN;
  if (workspace_bytes < p.ws_bytes) return LRKV_ERR_WORKSPACE;

  cudaStream_t st = (cudaStream_t)stream;
  uint32_t* header = static_cast<uint32_t*>(workspace);
  char* ws = static_cast<char*>(workspace);
  SplitArgs a;
  a.q = q;
  a.ZK = ZK;
  a.ZV = ZV;
  a.SK = ZK_scale;
  a.SV = ZV_scale;
  a.BK = BK;
  a.BV = BV;
  a.seqlens = seqlens;
  a.o_part = reinterpret_cast<float*>(ws + p.o_off);
  a.lse_part = reinterpret_cast<float*>(ws + p.lse_off);
  a.header = header;
  a.B = dims->batch;
  a.Hq = dims->n_q_heads;
  a.Hkv = dims->n_kv_heads;
  a.G = dims->n_q_heads / dims->n_kv_heads;
  a.d = dims->d_head;
  a.r = dims->rank;
  a.Lcap = dims->max_seq;
  a.max_seqlen = dims->max_seqlen;
  a.S = p.S;
  a.chunk = p.chunk;
  a.n_visual = dims->n_visual;
  a.io_dtype = dims->io_dtype;
  a.latent_dtype = dims->latent_dtype;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)dims->d_head));
  a.debug_stall = 0;
  a.device_chunk = 0;
  a.chunk_hint = p.chunk_hint;

  if (p.algo == LRKV_ALGO_TCGEN05 && quant &&
      ((reinterpret_cast<uintptr_t>(ZK_scale) | reinterpret_cast<uintptr_t>(ZV_scale)) & 15u)) {
    if (dims->algo == LRKV_ALGO_TCGEN05) return LRKV_ERR_ALIGN;
    p.algo = LRKV_ALGO_SIMT;
    p.smem = (int)simt_smem_bytes(dims->rank, dims->d_head, dims->n_q_heads / dims->n_kv_heads);
    if (p.smem > 227 * 1024) return LRKV_ERR_UNSUPPORTED;
  }
  if (p.algo == LRKV_ALGO_TCGEN05) {
    a.debug_stall = g_debug_stall.exchange(0);
    a.device_chunk = p.device_chunk;
  }
  record_event(ev_split_begin, st);
  cudaError_t e = ad       ? launch_split_simt_adaptive(a, *ad, p, st)
                  : shared ? launch_split_simt_shared(a, p, st)
                  : (p.algo == LRKV_ALGO_TCGEN05) ? launch_split_tc(a, p, st)
                                                  : launch_split_simt(a, p, st);
  if (e != cudaSuccess) return LRKV_ERR_LAUNCH;
  record_event(ev_split_end, st);

  MergeArgs m;
  m.o_part = a.o_part;
  m.lse_part = a.lse_part;
  m.seqlens = seqlens;
  m.out = out;
  m.lse_out = lse_out;
  m.header = header;
  m.B = a.B;
  m.Hq = a.Hq;
  m.d = a.d;
  m.S = p.S;
  m.chunk = p.chunk;
  m.n_visual = a.n_visual;
  m.Lcap = a.Lcap;
  m.max_seqlen = a.max_seqlen;
  m.io_dtype = a.io_dtype;
  m.device_chunk = a.device_chunk;
  if (launch_merge(m, st) != cudaSuccess) return LRKV_ERR_LAUNCH;
  if (ad) {
    MassArgs ma;
    ma.scores = ad->scores;
    ma.lse = lse_out;
    ma.imp = const_cast<float*>(ad->imp);
    ma.seqlens = seqlens;
    ma.header = header;
    ma.B = a.B;
    ma.Hq = a.Hq;
    ma.Hkv = a.Hkv;
    ma.Lcap = a.Lcap;
    ma.max_seqlen = a.max_seqlen;
    ma.beta = beta;
    if (launch_mass_ema(ma, st) != cudaSuccess) return LRKV_ERR_LAUNCH;
  }
  return LRKV_OK;
}

int lrkv_decode_attn_timed(const lrkv_dims* dims, const void* q, const void* ZK,
                           const void* ZV, const float* ZK_scale, const float* ZV_scale,
                           const void* BK, const void* BV, const int32_t* seqlens, void* out,
                           float* lse_out, void* workspace, size_t workspace_bytes,
                           void* stream, void* ev_split_begin, void* ev_split_end) {
  return decode_impl(dims, q, ZK, ZV, ZK_scale, ZV_scale, BK, BV, seqlens, out, lse_out,
                     workspace, workspace_bytes, stream, ev_split_begin, ev_split_end, nullptr,
                     0.f);
}

int lrkv_decode_attn_shared(const lrkv_dims* dims, const void* q, const void* ZK,
                            const void* ZV, const float* ZK_scale, const float* ZV_scale,
                            const void* DK, const void* DV, const int32_t* seqlens, void* out,
                            float* lse_out, void* workspace, size_t workspace_bytes,
                            void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->algo == LRKV_ALGO_TCGEN05) return LRKV_ERR_UNSUPPORTED;
  if (dims->n_visual != 0) return LRKV_ERR_DIMS;
  lrkv_dims d = *dims;
  d.algo = LRKV_ALGO_SIMT;
  return decode_impl(&d, q, ZK, ZV, ZK_scale, ZV_scale, DK, DV, seqlens, out, lse_out,
                     workspace, workspace_bytes, stream, nullptr, nullptr, nullptr, 0.f, true);
}

int lrkv_decode_attn_adaptive(const lrkv_dims* dims, const void* q, const void* ZK,
                              const void* ZV, const float* ZK_scale, const float* ZV_scale,
                              const void* BK, const void* BV, const int32_t* seqlens,
                              float* importance, float tau, int32_t r_low, float beta,
                              float* scores, void* out, float* lse_out, void* workspace,
                              size_t workspace_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->algo == LRKV_ALGO_TCGEN05) return LRKV_ERR_UNSUPPORTED;
  if (!importance || !scores || !lse_out) return LRKV_ERR_ARG;
  if (r_low < 1 || r_low > dims->rank || !(beta >= 0.f && beta <= 1.f)) return LRKV_ERR_ARG;
  lrkv_dims d = *dims;
  d.algo = LRKV_ALGO_SIMT;   // the per-token rank is a loop bound of the CUDA-core kernel
  AdaptArgs ad;
  ad.imp = importance;
  ad.tau = tau;
  ad.r_low = r_low;
  ad.scores = scores;
  return decode_impl(&d, q, ZK, ZV, ZK_scale, ZV_scale, BK, BV, seqlens, out, lse_out,
                     workspace, workspace_bytes, stream, nullptr, nullptr, &ad, beta);
}

int lrkv_append(const lrkv_dims* dims, const void* zk_new, const void* zv_new, void* ZK,
                void* ZV, float* ZK_scale, float* ZV_scale, int32_t* seqlens, void* workspace,
                size_t workspace_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  const bool quant = dims->latent_dtype == LRKV_I8 || dims->latent_dtype == LRKV_E4M3;
  if (!zk_new || !zv_new || !ZK || !ZV || !seqlens || !workspace) return LRKV_ERR_ARG;
  if (quant != (ZK_scale != nullptr) || quant != (ZV_scale != nullptr)) return LRKV_ERR_ARG;
  if (workspace_bytes < kHeaderBytes) return LRKV_ERR_WORKSPACE;
  if (!aligned16(ZK) || !aligned16(ZV) || !aligned16(workspace)) return LRKV_ERR_ALIGN;
  AppendArgs a;
  a.zk_new = zk_new;
  a.zv_new = zv_new;
  a.ZK = ZK;
  a.ZV = ZV;
  a.SK = ZK_scale;
  a.SV = ZV_scale;
  a.seqlens = seqlens;
  a.header = static_cast<uint32_t*>(workspace);
  a.B = dims->batch;
  a.Hkv = dims->n_kv_heads;
  a.r = dims->rank;
  a.Lcap = dims->max_seq;
  a.io_dtype = dims->io_dtype;
  a.latent_dtype = dims->latent_dtype;
  if (launch_append(a, (cudaStream_t)stream) != cudaSuccess) return LRKV_ERR_LAUNCH;
  return LRKV_OK;
}

int lrkv_project_append(const lrkv_dims* dims, int32_t d_model, const void* x, const void* AK,
                        const void* AV, void* ZK, void* ZV, float* ZK_scale, float* ZV_scale,
                        int32_t* seqlens, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (d_model < 1 || d_model > (1 << 20)) return LRKV_ERR_DIMS;
  const bool quant = dims->latent_dtype == LRKV_I8 || dims->latent_dtype == LRKV_E4M3;
  if (!x || !AK || !AV || !ZK || !ZV || !seqlens || !workspace) return LRKV_ERR_ARG;
  if (quant != (ZK_scale != nullptr) || quant != (ZV_scale != nullptr)) return LRKV_ERR_ARG;
  if (workspace_bytes < kHeaderBytes) return LRKV_ERR_WORKSPACE;
  if (!aligned16(ZK) || !aligned16(ZV) || !aligned16(workspace) || !aligned16(AK) ||
      !aligned16(AV))
    return LRKV_ERR_ALIGN;
  ProjArgs a;
  a.app.zk_new = nullptr;
  a.app.zv_new = nullptr;
  a.app.ZK = ZK;
  a.app.ZV = ZV;
  a.app.SK = ZK_scale;
  a.app.SV = ZV_scale;
  a.app.seqlens = seqlens;
  a.app.header = static_cast<uint32_t*>(workspace);
  a.app.B = dims->batch;
  a.app.Hkv = dims->n_kv_heads;
  a.app.r = dims->rank;
  a.app.Lcap = dims->max_seq;
  a.app.io_dtype = dims->io_dtype;
  a.app.latent_dtype = dims->latent_dtype;
  a.x = x;
  a.AK = AK;
  a.AV = AV;
  a.d_model = d_model;
  a.nsplit = project_nsplit(a.app.Hkv, a.app.B, a.app.r, d_model,
                            (int)dtype_bytes(dims->io_dtype), workspace_bytes);
  a.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + kHeaderBytes);
  if (launch_project_append(a, (cudaStream_t)stream) != cudaSuccess) return LRKV_ERR_LAUNCH;
  return LRKV_OK;
}

int lrkv_decode_step_host(const lrkv_dims* dims, const void* q_host, const void* zk_new_host,
                          const void* zv_new_host, void* out_host, void* q_dev,
                          void* zk_new_dev, void* zv_new_dev, void* out_dev, void* ZK, void* ZV,
                          float* ZK_scale, float* ZV_scale, const void* BK, const void* BV,
                          int32_t* seqlens, void* workspace, size_t workspace_bytes,
                          void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!q_host || !zk_new_host || !zv_new_host || !out_host || !q_dev || !zk_new_dev ||
      !zv_new_dev || !out_dev)
    return LRKV_ERR_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t io = dtype_bytes(dims->io_dtype);
  const size_t qbytes = (size_t)dims->batch * dims->n_q_heads * dims->d_head * io;
  const size_t zbytes = (size_t)dims->batch * dims->n_kv_heads * dims->rank * io;
  if (cudaMemcpyAsync(q_dev, q_host, qbytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(zk_new_dev, zk_new_host, zbytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(zv_new_dev, zv_new_host, zbytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return LRKV_ERR_LAUNCH;
  rc = lrkv_append(dims, zk_new_dev, zv_new_dev, ZK, ZV, ZK_scale, ZV_scale, seqlens, workspace,
                   workspace_bytes, stream);
  if (rc) return rc;
  rc = lrkv_decode_attn(dims, q_dev, ZK, ZV, ZK_scale, ZV_scale, BK, BV, seqlens, out_dev,
                        nullptr, workspace, workspace_bytes, stream);
  if (rc) return rc;
  if (cudaMemcpyAsync(out_host, out_dev, qbytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return LRKV_ERR_LAUNCH;
  return LRKV_OK;
}

int lrkv_debug_stall_next_launch(int32_t on) {
  g_debug_stall.store(on ? 1 : 0);
  return LRKV_OK;
}

int lrkv_read_status(void* workspace, void* stream, uint32_t* status) {
  if (!workspace || !status) return LRKV_ERR_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return LRKV_ERR_LAUNCH;
  if (cudaStreamSynchronize(st) != cudaSuccess) return LRKV_ERR_LAUNCH;
  *status = v;
  if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), st) != cudaSuccess) return LRKV_ERR_LAUNCH;
  if (cudaStreamSynchronize(st) != cudaSuccess) return LRKV_ERR_LAUNCH;
  return LRKV_OK;
}

}  // extern "C"
