// Dispatch: copy every token row to its k slots of the rank-major receive
// buffer (the dispatch_local / dispatch_scatter_remote data movement of "MLX
// expert parallelism all_to_all PR 3158", Facts; the push into rank-major
// buffers of "One-Sided Expert-Parallel All-to-All for Mixture-of-Experts
// Inference over NVLink", abstract).  With R virtual ranks on one GPU, a
// "remote" region is a byte range of the same HBM, so the push is a store.
//
// Work item = (token, 1 KB column chunk of its row), one warp each; 1 KB
// divides both the 7168-byte FP8 rows and the 14336-byte bf16 rows of the
// workloads, and 32 registers per thread let 8 blocks share an SM.  Every
// lane loads 2 sixteen-byte vectors of the chunk first (they do not depend on
// routing), while lanes j < k resolve the slot of choice j -- the route
// call's per-block base plus the in-block rank, no metadata round trip --
// then the warp stores the chunk k times.  Scales and the index maps go with
// the first chunk of the row.  High occupancy keeps enough loads and stores
// in flight: on B200 this beats staging the chunks through shared memory
// with bulk (TMA) copies for these scattered row copies (measured about
// 5.6 vs 5.0 TB/s on the prefill shape, 2.6 vs 1.4 TB/s on the decode shape).
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kVec = 2;                 // 16-byte vectors per lane per chunk
constexpr int kChunkVec = 32 * kVec;    // vectors per chunk (1 KB)

struct DispatchArgs {
  const uint8_t* x;
  const float* x_scale;
  const int32_t* topk_idx;
  const int32_t* bases;  // [route blocks, E] absolute base slot of each block's run of an expert
  const uint8_t* rank;   // [n, k] rank of each pick among its block's tokens picking the expert
  uint8_t* recv;
  float* recv_scale;
  int32_t* slot_of;
  int32_t* src_of;
  void* ws;
  int32_t n, E, K, S;
  int64_t row_bytes;
  int32_t total;   // T
  int32_t chunks;  // chunks per row
};

__global__ void __launch_bounds__(kThreads, 8) dispatch_kernel(DispatchArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t nvec = a.row_bytes >> 4;
  const int64_t n_items = int64_t(a.n) * a.chunks;
  const int64_t stride = int64_t(gridDim.x) * kWarps;
  grid_dependency_wait();
  // Every CTA that runs this line has started, so once all have, the next
  // kernel in the stream may be scheduled into the SM room this grid leaves
  // (it waits for this grid to finish before it reads anything).
  grid_dependents_launch();
  for (int64_t item = int64_t(blockIdx.x) * kWarps + (threadIdx.x >> 5); item < n_items;
       item += stride) {
    const int64_t t = item / a.chunks;
    const int c = int(item % a.chunks);
    const uint8_t* src = a.x + t * a.row_bytes;
    uint4 v[kVec];
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      const int64_t g = int64_t(c) * kChunkVec + u * 32 + lane;
      if (g < nvec) v[u] = ld_nc_v4(src + (g << 4));
    }
    int slot = -1;
    if (lane < a.K) {
      const int64_t tk = t * a.K + lane;
      const int e = __ldg(a.topk_idx + tk);
      if (e >= 0 && e < a.E) {
        slot = __ldg(a.bases + (t / kRouteTokens) * a.E + e) + a.rank[tk];
        if (slot < 0 || slot >= a.total) slot = -1;
      }
      if (slot < 0) set_status(a.ws, MOE_ERR_DEVICE_INDEX);
      if (c == 0) {
        a.slot_of[tk] = slot;
        if (slot >= 0) a.src_of[slot] = int32_t(tk);
      }
    }
    for (int j = 0; j < a.K; ++j) {
      const int s = __shfl_sync(0xFFFFFFFFu, slot, j);
      if (s < 0) continue;  // uniform across the warp
      uint8_t* dst = a.recv + int64_t(s) * a.row_bytes;
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const int64_t g = int64_t(c) * kChunkVec + u * 32 + lane;
        if (g < nvec) st_cs_v4(dst + (g << 4), v[u]);
      }
    }
    if (c == 0 && a.S > 0) {
      if ((a.S & 3) == 0 && a.S <= 128) {
        // the row's scales as 16-byte vectors, one per lane (a single store
        // instruction per copy for the 56 scales of a 7168-column row)
        const int nv = a.S >> 2;
        float4 sv = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lane < nv) sv = __ldcs(reinterpret_cast<const float4*>(a.x_scale + t * a.S) + lane);
        for (int j = 0; j < a.K; ++j) {
          const int s = __shfl_sync(0xFFFFFFFFu, slot, j);
          if (s >= 0 && lane < nv)
            __stcs(reinterpret_cast<float4*>(a.recv_scale + int64_t(s) * a.S) + lane, sv);
        }
      } else {
        for (int i0 = 0; i0 < a.S; i0 += 32) {
          const int i = i0 + lane;
          const float sv = i < a.S ? __ldcs(a.x_scale + t * a.S + i) : 0.f;
          for (int j = 0; j < a.K; ++j) {
            const int s = __shfl_sync(0xFFFFFFFFu, slot, j);
            if (s >= 0 && i < a.S) __stcs(a.recv_scale + int64_t(s) * a.S + i, sv);
          }
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_dispatch(const moe_plan& p, int32_t n, const void* x, const float* x_scale,
                            const int32_t* topk_idx, void* recv, float* recv_scale,
                            int32_t* slot_of, int32_t* src_of, void* ws, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  DispatchArgs a;
  a.x = static_cast<const uint8_t*>(x);
  a.x_scale = x_scale;
  a.topk_idx = topk_idx;
  a.bases = reinterpret_cast<const int32_t*>(static_cast<const char*>(ws) + p.lay.bases);
  a.rank = reinterpret_cast<const uint8_t*>(static_cast<const char*>(ws) + p.lay.rank);
  a.recv = static_cast<uint8_t*>(recv);
  a.recv_scale = recv_scale;
  a.slot_of = slot_of;
  a.src_of = src_of;
  a.ws = ws;
  a.n = n;
  a.E = p.d.n_experts;
  a.K = p.d.top_k;
  a.S = p.scale_cols;
  a.row_bytes = int64_t(p.d.hidden) * elem_bytes(p.d.x_dtype);
  a.total = int32_t(total_rows(p, n));
  a.chunks = int32_t((a.row_bytes / 16 + kChunkVec - 1) / kChunkVec);
  const int sms = num_sms();
  int64_t grid = (int64_t(n) * a.chunks + kWarps - 1) / kWarps;
  const int64_t cap = int64_t(sms) * 16;
  if (grid > cap) grid = cap;
  return launch_pdl(dispatch_kernel, dim3(unsigned(grid)), dim3(kThreads), 0, st, a);
}

}  // namespace moe
