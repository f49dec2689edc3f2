// Fused route + dispatch for small batches: top-k gating, counts, rank-major
// offsets and the row scatter in ONE cooperative launch.
//
// At decode sizes the work of each step is a few megabytes, so the fixed cost
// of separate launches and of the route kernel's second phase dominates
// ("One-Sided Expert-Parallel All-to-All for Mixture-of-Experts Inference over
// NVLink", abstract: fixed costs dominate at small batch; "backends/mlx:
// runtime MoE expert-sort for decode", Summary: decode skips the sort because
// of its overhead).  Here:
//  1. every warp issues the load of its first 512-byte chunk of x (it does
//     not depend on routing), then the blocks that own a route block of 32
//     tokens route it exactly as the route kernel does (same per-token code):
//     top-k, softmax, in-block ranks and the block's per-expert counts;
//  2. one bounded grid barrier;
//  3. every block rebuilds the whole [blocks, E] base table in shared memory
//     from the block counts (at most 32 route blocks, so a column is a few
//     loads): expert totals, their exclusive prefix, the rank-major offsets
//     and each block's base -- no second barrier;
//  4. each warp stores its chunk to the token's k slots (base + rank), and
//     the first chunk of a row carries the scales and the index maps.
// Results are identical to moe_route_topk followed by moe_dispatch.
#include "route_common.cuh"

namespace moe {
namespace {

struct FusedArgs {
  RouteArgs r;
  const uint8_t* x;
  const float* x_scale;
  uint8_t* recv;
  float* recv_scale;
  int32_t* slot_of;
  int32_t* src_of;
  int32_t S;        // scale columns per row (0 without scales)
  int32_t vecs;     // 16-byte vectors per row
  int32_t chunks;   // 512-byte chunks per row
  int32_t total;    // T
};

template <int VPL, int VEC>
__global__ void __launch_bounds__(kRouteThreads, 1) route_dispatch_kernel(FusedArgs f) {
  extern __shared__ int32_t s_base[];                 // [blocks, E] absolute bases
  __shared__ int32_t s_sel[kRouteTokens * kMaxTopK];  // picks of the block's tokens
  __shared__ uint32_t s_mask[kMaxExperts];            // token mask per expert
  __shared__ int32_t s_pre[kMaxExperts];              // exclusive prefix of expert totals
  __shared__ int32_t s_wsum[kWarps];
  __shared__ unsigned s_parity;
  const RouteArgs& a = f.r;
  const int E = a.E, K = a.K, B = a.blocks;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t row_bytes = int64_t(f.vecs) << 4;
  const int64_t n_items = int64_t(a.n) * f.chunks;
  const int64_t first = int64_t(blockIdx.x) * kWarps + warp;
  const int64_t stride = int64_t(gridDim.x) * kWarps;
  grid_dependency_wait();

  // ---- the first chunk of x, in flight while routing runs
  uint4 v0 = make_uint4(0u, 0u, 0u, 0u);
  if (first < n_items) {
    const int64_t t = first / f.chunks;
    const int64_t g = int64_t(first % f.chunks) * 32 + lane;
    if (g < f.vecs) v0 = ld_nc_v4(f.x + t * row_bytes + (g << 4));
  }
  if (blockIdx.x == 0 && tid == 0) s_parity = ld_acquire_gpu(&reinterpret_cast<Ctrl*>(a.ws)->gen) & 1u;

  // ---- phase 1: route blocks b = blockIdx.x, blockIdx.x + grid, ...
  for (int b = blockIdx.x; b < B; b += gridDim.x) {
    const int t_base = b * kRouteTokens;
    const int valid = max(0, min(kRouteTokens, a.n - t_base));
    for (int i = tid; i < E; i += kRouteThreads) s_mask[i] = 0;
    if (warp < valid) {
      const int e = route_token<VPL, VEC>(a, int64_t(t_base) + warp, lane);
      if (lane < K) s_sel[warp * K + lane] = e;
    }
    __syncthreads();
    for (int p = tid; p < valid * K; p += kRouteThreads)
      atomicOr(&s_mask[s_sel[p]], 1u << (p / K));
    __syncthreads();
    for (int p = tid; p < valid * K; p += kRouteThreads) {
      const int tl = p / K;
      a.rank[int64_t(t_base) * K + p] = uint8_t(__popc(s_mask[s_sel[p]] & ((1u << tl) - 1u)));
    }
    for (int e = tid; e < E; e += kRouteThreads) a.blk[int64_t(b) * E + e] = __popc(s_mask[e]);
    __syncthreads();
  }

  if (!grid_barrier(a.ws, gridDim.x)) return;

  // ---- phase 2, in every block: expert totals, offsets and the base table
  int tot = 0;
  if (tid < E)
    for (int b = 0; b < B; ++b) tot += __ldcg(a.blk + int64_t(b) * E + tid);
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = s_wsum[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, wi, o);
      if (lane >= o) wi += y;
    }
    s_wsum[lane] = wi - w;
  }
  __syncthreads();
  const int pre = incl - tot + s_wsum[warp];  // sum of the totals of experts below tid
  if (tid < E) s_pre[tid] = pre;
  __syncthreads();
  if (tid < E) {
    const int per_rank = E / a.R;
    const int r = tid / per_rank;
    const int off = r * a.region_rows + pre - s_pre[r * per_rank];
    int run = off;
    for (int b = 0; b < B; ++b) {
      s_base[b * E + tid] = run;
      run += __ldcg(a.blk + int64_t(b) * E + tid);
    }
    if (blockIdx.x == 0) {
      a.counts[tid] = tot;
      a.expert_off[tid] = off;
      // the route kernel's expert totals: the half the next call uses starts at zero
      a.totals[size_t(s_parity ^ 1u) * E + tid] = 0;
    }
  }
  if (blockIdx.x == 0 && tid == 0) a.expert_off[E] = a.R * a.region_rows;
  __syncthreads();

  // ---- phase 3: each warp's chunks to the k slots of their token
  for (int64_t item = first; item < n_items; item += stride) {
    const int64_t t = item / f.chunks;
    const int c = int(item % f.chunks);
    const int64_t g = int64_t(c) * 32 + lane;
    uint4 v = v0;
    if (item != first && g < f.vecs) v = ld_nc_v4(f.x + t * row_bytes + (g << 4));
    int slot = -1;
    if (lane < K) {
      const int64_t tk = t * K + lane;
      const int e = __ldcg(a.topk_idx + tk);
      if (e >= 0 && e < E) {
        slot = s_base[int(t / kRouteTokens) * E + e] + __ldcg(a.rank + tk);
        if (slot < 0 || slot >= f.total) slot = -1;
      }
      if (slot < 0) set_status(a.ws, MOE_ERR_DEVICE_INDEX);
      if (c == 0) {
        f.slot_of[tk] = slot;
        if (slot >= 0) f.src_of[slot] = int32_t(tk);
      }
    }
    for (int j = 0; j < K; ++j) {
      const int s = __shfl_sync(kFull, slot, j);
      if (s < 0) continue;  // uniform across the warp
      if (g < f.vecs) st_cs_v4(f.recv + int64_t(s) * row_bytes + (g << 4), v);
    }
    if (c == 0 && f.S > 0) {
      for (int i0 = 0; i0 < f.S; i0 += 32) {
        const int i = i0 + lane;
        const float sv = i < f.S ? __ldcs(f.x_scale + t * f.S + i) : 0.f;
        for (int j = 0; j < K; ++j) {
          const int s = __shfl_sync(kFull, slot, j);
          if (s >= 0 && i < f.S) __stcs(f.recv_scale + int64_t(s) * f.S + i, sv);
        }
      }
    }
  }
  grid_dependents_launch();
}

template <int VPL, int VEC>
cudaError_t launch_fused(const FusedArgs& f, int sms, cudaStream_t st) {
  static int per_sm[64] = {0};  // resident blocks per SM, per device
  constexpr int kMaxDyn = kFusedMaxBlocks * kMaxExperts * 4;
  auto kernel = route_dispatch_kernel<VPL, VEC>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  e = set_smem_limit(reinterpret_cast<const void*>(kernel), kMaxDyn);
  if (e != cudaSuccess) return e;
  if (per_sm[dev] == 0) {
    int nb = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, kRouteThreads, kMaxDyn);
    if (e != cudaSuccess) return e;
    if (nb < 1) return cudaErrorInvalidConfiguration;
    per_sm[dev] = nb;
  }
  const int64_t items = int64_t(f.r.n) * f.chunks;
  int64_t grid = (items + kWarps - 1) / kWarps;
  if (grid < f.r.blocks) grid = f.r.blocks;
  if (grid > int64_t(per_sm[dev]) * sms) grid = int64_t(per_sm[dev]) * sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.blockDim = dim3(kRouteThreads);
  cfg.dynamicSmemBytes = size_t(f.r.blocks) * f.r.E * 4;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, f);
}

}  // namespace

cudaError_t launch_route_dispatch(const moe_plan& p, int32_t n, const float* logits,
                                  const void* x, const float* x_scale, int32_t* topk_idx,
                                  float* topk_w, int32_t* counts, int32_t* expert_off, void* recv,
                                  float* recv_scale, int32_t* slot_of, int32_t* src_of, void* ws,
                                  cudaStream_t st) {
  char* w = static_cast<char*>(ws);
  FusedArgs f;
  RouteArgs& a = f.r;
  a.logits = logits;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.counts = counts;
  a.expert_off = expert_off;
  a.blk = reinterpret_cast<int32_t*>(w + p.lay.blk);
  a.bases = reinterpret_cast<int32_t*>(w + p.lay.bases);
  a.totals = reinterpret_cast<int32_t*>(w + p.lay.totals);
  a.rank = reinterpret_cast<uint8_t*>(w + p.lay.rank);
  a.ws = ws;
  a.n = n;
  a.E = p.d.n_experts;
  a.K = p.d.top_k;
  a.R = p.d.n_ranks;
  a.blocks = route_blocks(n);
  a.region_rows = int32_t(region_rows(p, n));
  f.x = static_cast<const uint8_t*>(x);
  f.x_scale = x_scale;
  f.recv = static_cast<uint8_t*>(recv);
  f.recv_scale = recv_scale;
  f.slot_of = slot_of;
  f.src_of = src_of;
  f.S = p.scale_cols;
  f.vecs = int32_t(int64_t(p.d.hidden) * elem_bytes(p.d.x_dtype) / 16);
  f.chunks = (f.vecs + 31) / 32;
  f.total = int32_t(total_rows(p, n));
  if (a.blocks > kFusedMaxBlocks) return cudaErrorInvalidValue;
  const int sms = num_sms();
  return with_route_shape(a.E, [&](auto vpl, auto vec) {
    return launch_fused<decltype(vpl)::value, decltype(vec)::value>(f, sms, st);
  });
}

}  // namespace moe
