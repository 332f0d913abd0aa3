// lrkv_decode_attn_noalloc: decode attention for callers that cannot allocate device
// memory. Some callers have no way to obtain a device buffer for the workspace: a
// plain C host program without a device memory manager of its own, or a runtime
// with a fixed memory budget that forbids new allocations once it is serving. This
// entry point takes the same inputs and outputs as lrkv_decode_attn but uses a
// fixed scratch area that lives in this library's own device memory instead of a
// caller-provided workspace. It allocates nothing (no cudaMalloc, cudaFree or
// allocating library call), and runs the same kernels through lrkv_decode_attn.
#include <mutex>

#include "lrkv_internal.h"

namespace {

// The scratch area: split partials, the status word and the scheduler counters of
// one call. Every GPU that loads the library holds it until the process exits.
constexpr size_t kStaticScratchBytes = LRKV_NOALLOC_MAX_WORKSPACE_BYTES;  // 16 MiB
static __device__ __align__(256) unsigned char g_lrkv_static_scratch[kStaticScratchBytes];

// Device address of the scratch area per device, looked up once per device. On the
// host the array's name is only a stand-in for the symbol, never a device address.
void* scratch_address(int* rc) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *rc = LRKV_ERR_LAUNCH;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_lrkv_static_scratch) != cudaSuccess || !p) {
      *rc = LRKV_ERR_LAUNCH;
      return nullptr;
    }
    addr[dev] = p;
  }
  *rc = LRKV_OK;
  return addr[dev];
}

}  // namespace

extern "C" {

int lrkv_decode_attn_noalloc(const lrkv_dims* dims, const void* q, const void* ZK,
                             const void* ZV, const float* ZK_scale, const float* ZV_scale,
                             const void* BK, const void* BV, const int32_t* seqlens, void* out,
                             float* lse_out, uint32_t* status_out, void* stream) {
  const size_t need = lrkv_workspace_bytes(dims);
  if (need == 0) {
    // invalid dims: let the regular entry point report the precise code
    return lrkv_decode_attn(dims, q, ZK, ZV, ZK_scale, ZV_scale, BK, BV, seqlens, out, lse_out,
                            nullptr, 0, stream);
  }
  if (need > kStaticScratchBytes) return LRKV_ERR_WORKSPACE;  // above the fixed maximum
  int rc = LRKV_OK;
  void* ws = scratch_address(&rc);
  if (!ws) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  // the header (status word, work counter) starts every call at zero; the rest of the
  // area keeps the previous call's partials, which this call overwrites before use
  if (cudaMemsetAsync(ws, 0, lrkv::kHeaderBytes, st) != cudaSuccess) return LRKV_ERR_LAUNCH;
  rc = lrkv_decode_attn(dims, q, ZK, ZV, ZK_scale, ZV_scale, BK, BV, seqlens, out, lse_out, ws,
                        kStaticScratchBytes, stream);
  if (rc) return rc;
  if (status_out &&
      cudaMemcpyAsync(status_out, ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return LRKV_ERR_LAUNCH;
  return LRKV_OK;
}

}  // extern "C"
