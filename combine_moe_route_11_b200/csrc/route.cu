// Route: top-k gating, per-expert counts, rank-major expert offsets and the
// per-block bases from which moe_dispatch derives every slot.
//
// Slots follow the rank-major layout of the one-sided expert-parallel
// all-to-all ("One-Sided Expert-Parallel All-to-All for Mixture-of-Experts
// Inference over NVLink", abstract): every virtual rank owns a region at a
// fixed base, so destinations are computed locally with no metadata exchange.
// Inside a region the order is (expert, source token), i.e. the stable sort of
// the flattened [N, top_k] expert indices that the sorted gather path uses
// ("backends/mlx: runtime MoE expert-sort for decode", author update on the
// sorted branch) -- computed here as a counting sort, without any sort.
//
// One cooperative launch (all blocks resident), two phases split by a
// bounded grid barrier:
//  1. per route block of 32 tokens, one warp per token: the k largest logits
//     by k rounds of a warp argmax on order-preserving integer keys (two
//     single-instruction warp reductions per round; the lower expert id wins
//     a tie) and a softmax over the k winners; then, per expert, the bitmask
//     of the block's tokens that picked it gives each (token, expert) pair
//     its rank among the block's tokens (popcount of the lower lanes) and the
//     block's count of the expert;
//     Each block also adds its counts into the expert totals (integer
//     atomics: the sum does not depend on their order);
//  2. per column of (up to) 4 experts: the totals of the experts of its rank
//     below its own give the rank-major offsets, and an exclusive scan of its
//     own count columns over the route blocks gives each block's absolute
//     base slot.
// A slot is then base[block][e] + rank.  All integer results are
// deterministic: no atomic decides an order.
#include "route_common.cuh"

#include <atomic>

#include <float.h>
#include <limits.h>

#include <type_traits>

namespace moe {
namespace {

static_assert(kWarps == 32, "phase 2 scans one sum per warp with one warp");

// Phase 2 for column unit u (experts [u*W, u*W + W)): rank-major offsets
// from the expert totals, then the exclusive scan of the unit's count columns
// over the route blocks into absolute bases.
template <int W>
__device__ __forceinline__ void scan_column(const RouteArgs& a, int u, const int32_t* tot,
                                            void* s_warp_raw, int32_t* s_off) {
  using V = typename std::conditional<W == 4, int4, int>::type;
  V* s_warp = static_cast<V*>(s_warp_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int B = a.blocks, E = a.E;
  const int per_rank = E / a.R;
  const int e0 = u * W;
  const int64_t row = E / W;  // row stride in column units
  V zero;
  if constexpr (W == 4) zero = make_int4(0, 0, 0, 0);
  else zero = 0;
  auto add = [](V& x, const V& y) {
    if constexpr (W == 4) { x.x += y.x; x.y += y.y; x.z += y.z; x.w += y.w; }
    else x += y;
  };
  const V* cnt = reinterpret_cast<const V*>(a.blk);
  // ---- this thread's blocks of the unit's count columns, loaded first: they
  // do not depend on the offsets below
  V* base = reinterpret_cast<V*>(a.bases) + u;
  const V* own = cnt + u;
  const int per = (B + kRouteThreads - 1) / kRouteThreads;
  const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
  V sum = zero;
  for (int b = b0; b < b1; ++b) add(sum, __ldcg(own + int64_t(b) * row));
  // ---- offsets of this unit's experts from the phase-1 totals: one warp each
  if (warp < W) {
    const int e = e0 + warp;
    const int r = e / per_rank;
    int tsum = 0;
    for (int e2 = r * per_rank + lane; e2 < e; e2 += 32) tsum += __ldcg(tot + e2);
    tsum = __reduce_add_sync(kFull, tsum);
    if (lane == 0) {
      const int off = r * a.region_rows + tsum;
      s_off[warp] = off;
      a.expert_off[e] = off;
      a.counts[e] = __ldcg(tot + e);
    }
  }
  // ---- exclusive scan of the columns over the route blocks: within each
  // warp, then of the warp sums by warp 0
  V incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    V y;
    if constexpr (W == 4) {
      y.x = __shfl_up_sync(kFull, incl.x, o); y.y = __shfl_up_sync(kFull, incl.y, o);
      y.z = __shfl_up_sync(kFull, incl.z, o); y.w = __shfl_up_sync(kFull, incl.w, o);
    } else {
      y = __shfl_up_sync(kFull, incl, o);
    }
    if (lane >= o) add(incl, y);
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const V w = s_warp[lane];  // kWarps == 32 warp sums
    V wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      V y;
      if constexpr (W == 4) {
        y.x = __shfl_up_sync(kFull, wi.x, o); y.y = __shfl_up_sync(kFull, wi.y, o);
        y.z = __shfl_up_sync(kFull, wi.z, o); y.w = __shfl_up_sync(kFull, wi.w, o);
      } else {
        y = __shfl_up_sync(kFull, wi, o);
      }
      if (lane >= o) add(wi, y);
    }
    if constexpr (W == 4) { wi.x -= w.x; wi.y -= w.y; wi.z -= w.z; wi.w -= w.w; }
    else wi -= w;
    s_warp[lane] = wi;  // exclusive prefix of the warp sums
  }
  __syncthreads();
  V run;
  if constexpr (W == 4) run = make_int4(s_off[0], s_off[1], s_off[2], s_off[3]);
  else run = s_off[0];
  add(run, s_warp[warp]);
  // run + (incl - sum) = absolute base of this thread's first block
  V ex = incl;
  if constexpr (W == 4) { ex.x -= sum.x; ex.y -= sum.y; ex.z -= sum.z; ex.w -= sum.w; }
  else ex -= sum;
  add(run, ex);
  for (int b = b0; b < b1; ++b) {
    base[int64_t(b) * row] = run;
    if (b + 1 < b1) add(run, __ldcg(own + int64_t(b) * row));
  }
  __syncthreads();  // shared scratch is reused by the next unit
}

template <int VPL, int VEC>
__global__ void __launch_bounds__(kRouteThreads, 1) route_kernel(RouteArgs a) {
  __shared__ int32_t s_sel[kRouteTokens * kMaxTopK];  // picks of the block's tokens
  __shared__ uint32_t s_mask[kMaxExperts];            // token mask per expert
  __shared__ int4 s_warp[kWarps];
  __shared__ int32_t s_off[4];
  __shared__ unsigned s_parity;
  const int E = a.E, K = a.K;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  grid_dependency_wait();
  // This call's half of the totals: the barrier generation's parity, read
  // before any block can reach the barrier that bumps it.
  if (tid == 0) s_parity = ld_acquire_gpu(&reinterpret_cast<Ctrl*>(a.ws)->gen) & 1u;
  __syncthreads();
  int32_t* tot = a.totals + size_t(s_parity) * E;

  // ---- phase 1: route blocks b = blockIdx.x, blockIdx.x + grid, ...
  for (int b = blockIdx.x; b < a.blocks; b += gridDim.x) {
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
    for (int e = tid; e < E; e += kRouteThreads) {
      const int c = __popc(s_mask[e]);
      a.blk[int64_t(b) * E + e] = c;
      if (c) atomicAdd(tot + e, c);  // integer sums: the order does not matter
    }
    __syncthreads();
  }

  if (!grid_barrier(a.ws, gridDim.x)) return;

  // ---- phase 2: column units u = blockIdx.x, blockIdx.x + grid, ...
  if ((E & 3) == 0) {
    for (int u = blockIdx.x; u < E / 4; u += gridDim.x) scan_column<4>(a, u, tot, s_warp, s_off);
  } else {
    for (int u = blockIdx.x; u < E; u += gridDim.x) scan_column<1>(a, u, tot, s_warp, s_off);
  }
  if (blockIdx.x == 0) {
    // the other halves start the next call (of either route kernel) at zero
    int32_t* next = a.totals + size_t(s_parity ^ 1u) * E;
    for (int e = tid; e < E; e += kRouteThreads) next[e] = 0;
    if (a.masks) {
      uint32_t* m = a.masks + size_t(s_parity ^ 1u) * a.mask_rows * E;
      for (int i = tid; i < a.mask_rows * E; i += kRouteThreads) m[i] = 0u;
    }
    if (tid == 0) a.expert_off[E] = a.R * a.region_rows;
  }
  grid_dependents_launch();
}

// Cooperative launch: every block resident, as the grid barrier requires.
template <int VPL, int VEC>
cudaError_t launch_coop(const RouteArgs& a, int sms, cudaStream_t st) {
  static std::atomic<int> per_sm[64];  // resident blocks per SM, per device (0 = unknown)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  int nb_known = per_sm[dev].load(std::memory_order_relaxed);
  if (nb_known == 0) {
    int nb = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, route_kernel<VPL, VEC>, kRouteThreads, 0);
    if (e != cudaSuccess) return e;
    if (nb < 1) return cudaErrorInvalidConfiguration;
    per_sm[dev].store(nb, std::memory_order_relaxed);
    nb_known = nb;
  }
  const int cols = (a.E & 3) == 0 ? a.E / 4 : a.E;
  int grid = a.blocks > cols ? a.blocks : cols;
  if (grid > nb_known * sms) grid = nb_known * sms;
  return launch_cooperative(route_kernel<VPL, VEC>, dim3(unsigned(grid)), dim3(kRouteThreads), 0,
                            st, a);
}

}  // namespace

cudaError_t launch_route(const moe_plan& p, int32_t n, const float* logits, int32_t* topk_idx,
                         float* topk_w, int32_t* counts, int32_t* expert_off, void* ws,
                         cudaStream_t st) {
  char* w = static_cast<char*>(ws);
  RouteArgs a;
  a.logits = logits;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.counts = counts;
  a.expert_off = expert_off;
  a.blk = reinterpret_cast<int32_t*>(w + p.lay.blk);
  a.bases = reinterpret_cast<int32_t*>(w + p.lay.bases);
  a.totals = reinterpret_cast<int32_t*>(w + p.lay.totals);
  a.masks = reinterpret_cast<uint32_t*>(w + p.lay.masks);
  a.mask_rows = mask_rows(p);
  a.rank = reinterpret_cast<uint8_t*>(w + p.lay.rank);
  a.ws = ws;
  a.n = n;
  a.E = p.d.n_experts;
  a.K = p.d.top_k;
  a.R = p.d.n_ranks;
  a.blocks = route_blocks(n);
  a.region_rows = int32_t(region_rows(p, n));
  const int sms = num_sms();
  return with_route_shape(a.E, [&](auto vpl, auto vec) {
    return launch_coop<decltype(vpl)::value, decltype(vec)::value>(a, sms, st);
  });
}

}  // namespace moe

namespace moe {

// The route kernels on caller-chosen scratch: ctrl (control words), blk and
// bases ([route blocks, E] int32 each), totals ([2, E] int32, zero before the
// first call) and rank ([n, k] bytes).
cudaError_t launch_route_on(const moe_plan& p, int32_t n, const float* logits, int32_t* topk_idx,
                            float* topk_w, int32_t* counts, int32_t* expert_off, void* ctrl,
                            int32_t* blk, int32_t* bases, int32_t* totals, uint32_t* masks,
                            uint8_t* rank, cudaStream_t st) {
  RouteArgs a;
  a.logits = logits;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.counts = counts;
  a.expert_off = expert_off;
  a.blk = blk;
  a.bases = bases;
  a.totals = totals;
  a.masks = masks;
  a.mask_rows = mask_rows(p);
  a.rank = rank;
  a.ws = ctrl;
  a.n = n;
  a.E = p.d.n_experts;
  a.K = p.d.top_k;
  a.R = p.d.n_ranks;
  a.blocks = route_blocks(n);
  a.region_rows = int32_t(region_rows(p, n));
  const int sms = num_sms();
  return with_route_shape(a.E, [&](auto vpl, auto vec) {
    return launch_coop<decltype(vpl)::value, decltype(vec)::value>(a, sms, st);
  });
}

}  // namespace moe
