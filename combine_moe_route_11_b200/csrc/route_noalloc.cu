// moe_route_topk_noalloc: the routing call for callers that cannot allocate
// device memory.  Its scratch is a fixed array compiled into this library
// instead of a caller-provided workspace.
#include "moe_internal.cuh"

#include <mutex>

namespace {

// Scratch of moe_route_topk_noalloc: the control words, the per-block count
// and base tables and the per-token ranks of one call.  Every GPU that loads
// this library holds these bytes until the process exits.
static __device__ __align__(256) unsigned char g_route_scratch[MOE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_route_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address must come from
// the runtime, once per device, with that device current.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    if (p == nullptr) return cudaErrorInvalidSymbol;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

namespace {

// Byte offsets inside the scratch array for a call with n tokens.
struct NoallocLayout {
  size_t totals, blk, bases, rank, end;
};

NoallocLayout noalloc_layout(const moe_plan& p, int32_t n) {
  const size_t table = moe::align256(size_t(moe::route_blocks(n)) * p.d.n_experts * 4);
  NoallocLayout L;
  L.totals = sizeof(moe::Ctrl);
  L.blk = L.totals + moe::align256(size_t(2) * p.d.n_experts * 4);
  L.bases = L.blk + table;
  L.rank = L.bases + table;
  L.end = L.rank + moe::align256(size_t(n) * p.d.top_k);
  return L;
}

}  // namespace

extern "C" MOE_API size_t moe_route_topk_noalloc_bytes(const moe_plan* p, int32_t n) {
  if (!p || n < 0) return 0;
  return noalloc_layout(*p, n).end;
}

extern "C" MOE_API moe_status moe_route_topk_noalloc(const moe_plan* p, int32_t n,
                                                     const float* logits, int32_t* topk_idx,
                                                     float* topk_w, int32_t* counts,
                                                     int32_t* expert_off, moe_stream_t stream) {
  if (!p || n < 0 || n > p->d.n_max) return MOE_ERR_INVALID_ARG;
  if (!counts || !expert_off || (n > 0 && (!logits || !topk_idx || !topk_w)))
    return MOE_ERR_INVALID_ARG;
  if (n > 0 && (reinterpret_cast<uintptr_t>(logits) & 15u)) return MOE_ERR_INVALID_ARG;
  const NoallocLayout L = noalloc_layout(*p, n);
  if (L.end > MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
  void* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* b = static_cast<char*>(base);
  // The array keeps whatever the previous call left: the control words
  // (status, the route kernel's counter and generation) and the expert
  // totals must start at zero.  The tables are fully rewritten.
  if (cudaMemsetAsync(b, 0, L.blk, st) != cudaSuccess) return MOE_ERR_CUDA;
  const cudaError_t e = moe::launch_route_on(
      *p, n, logits, topk_idx, topk_w, counts, expert_off, b,
      reinterpret_cast<int32_t*>(b + L.totals), reinterpret_cast<int32_t*>(b + L.blk), reinterpret_cast<int32_t*>(b + L.bases),
      reinterpret_cast<uint8_t*>(b + L.rank), st);
  if (e == cudaSuccess) return MOE_OK;
  return e == cudaErrorNotSupported ? MOE_ERR_UNSUPPORTED : MOE_ERR_CUDA;
}

extern "C" MOE_API moe_status moe_route_topk_noalloc_status(moe_stream_t stream) {
  void* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, &static_cast<moe::Ctrl*>(base)->status, sizeof(int),
                      cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  return static_cast<moe_status>(v);
}
