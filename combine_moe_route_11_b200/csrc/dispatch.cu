// Dispatch: copy every token row to its k slots of the rank-major receive
// buffer (the dispatch_local / dispatch_scatter_remote data movement of "MLX
// expert parallelism all_to_all PR 3158", Facts; the push into rank-major
// buffers of "One-Sided Expert-Parallel All-to-All for Mixture-of-Experts
// Inference over NVLink", abstract).  With R virtual ranks on one GPU, a
// "remote" region is a byte range of the same HBM, so the push is a store.
//
// Work item = (token, column chunk), one warp each.  The warp derives the k
// slots of its token from the route call's per-block bases plus the in-block
// ranks (no metadata round trip), loads its chunk of the source row once as
// 16-byte vectors and stores it k times.  Chunking keeps every SM busy when N
// is small (decode) without splitting rows into partial cache lines.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 8;  // 16-byte vectors per lane held in registers

struct DispatchArgs {
  const uint8_t* x;
  const float* x_scale;
  const int32_t* topk_idx;
  const int32_t* blk;    // per-(route block, expert) base slot
  const uint8_t* rank;   // [n, k] in-block rank
  uint8_t* recv;
  float* recv_scale;
  int32_t* slot_of;
  int32_t* src_of;
  void* ws;
  int32_t n, E, K, S;
  int64_t row_bytes;
  int32_t total;         // T
  int32_t chunks;        // column chunks per row
  int32_t chunk_vec;     // 16-byte vectors per chunk
};

__global__ void __launch_bounds__(kThreads) dispatch_kernel(DispatchArgs a) {
  __shared__ int32_t s_slot[kWarps][kMaxTopK];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t nvec = a.row_bytes >> 4;
  const int64_t n_items = int64_t(a.n) * a.chunks;
  const int64_t stride = int64_t(gridDim.x) * kWarps;
  for (int64_t item = int64_t(blockIdx.x) * kWarps + wib; item < n_items; item += stride) {
    const int t = int(item / a.chunks), c = int(item % a.chunks);
    int slot = -1;
    if (lane < a.K) {
      const int64_t tk = int64_t(t) * a.K + lane;
      const int e = a.topk_idx[tk];
      if (e >= 0 && e < a.E) {
        slot = a.blk[int64_t(t / kRouteTokens) * a.E + e] + a.rank[tk];
        if (slot < 0 || slot >= a.total) slot = -1;
      }
      if (slot < 0) set_status(a.ws, MOE_ERR_DEVICE_INDEX);
      if (c == 0) {
        a.slot_of[tk] = slot;
        if (slot >= 0) a.src_of[slot] = int32_t(tk);
      }
      s_slot[wib][lane] = slot;
    }
    __syncwarp();

    const int64_t v0 = int64_t(c) * a.chunk_vec;
    const int64_t v1 = min(v0 + a.chunk_vec, nvec);
    const uint8_t* src = a.x + int64_t(t) * a.row_bytes;
    for (int64_t vb = v0; vb < v1; vb += 32 * kBatch) {
      uint4 buf[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int64_t v = vb + u * 32 + lane;
        if (v < v1) buf[u] = ld_nc_v4(src + (v << 4));
      }
      for (int j = 0; j < a.K; ++j) {
        const int s = s_slot[wib][j];
        if (s < 0) continue;
        uint8_t* dst = a.recv + int64_t(s) * a.row_bytes;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int64_t v = vb + u * 32 + lane;
          if (v < v1) st_cs_v4(dst + (v << 4), buf[u]);
        }
      }
    }
    if (c == 0 && a.S > 0) {
      for (int i = lane; i < a.S; i += 32) {
        const float sv = __ldcs(a.x_scale + int64_t(t) * a.S + i);
        for (int j = 0; j < a.K; ++j) {
          const int s = s_slot[wib][j];
          if (s >= 0) __stcs(a.recv_scale + int64_t(s) * a.S + i, sv);
        }
      }
    }
    __syncwarp();
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
  a.blk = reinterpret_cast<const int32_t*>(static_cast<const char*>(ws) + p.lay.blk);
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
  // Enough (token, chunk) items to give every SM several warps; chunks are
  // whole multiples of 32 vectors so every lane moves the same bytes.
  const int sms = num_sms();
  const int64_t nvec = a.row_bytes / 16;
  const int64_t target = int64_t(sms) * 32;
  int64_t chunks = (target + n - 1) / n;
  const int64_t max_chunks = (nvec + 31) / 32;
  chunks = chunks < 1 ? 1 : (chunks > max_chunks ? max_chunks : chunks);
  int64_t cv = (nvec + chunks - 1) / chunks;
  cv = (cv + 31) / 32 * 32;
  a.chunk_vec = int32_t(cv);
  a.chunks = int32_t((nvec + cv - 1) / cv);
  const int64_t items = int64_t(n) * a.chunks;
  int64_t grid = (items + kWarps - 1) / kWarps;
  const int64_t cap = int64_t(sms) * 8;
  if (grid > cap) grid = cap;
  dispatch_kernel<<<dim3(unsigned(grid)), dim3(kThreads), 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
