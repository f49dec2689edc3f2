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
#include "moe_internal.cuh"

#include <float.h>
#include <limits.h>

#include <type_traits>

namespace moe {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kWarps = kRouteThreads / 32;

struct RouteArgs {
  const float* logits;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* counts;
  int32_t* expert_off;
  int32_t* blk;    // [blocks, E] per-block counts
  int32_t* bases;  // [blocks, E] per-block absolute base slots
  int32_t* totals; // [2, E] expert totals, the half of this call chosen by barrier parity
  uint8_t* rank;   // [n, k]: rank of (t, j) among the block's tokens picking e
  void* ws;
  int32_t n, E, K, R;
  int32_t blocks;       // route blocks B = ceil(n / 32), at least 1
  int32_t region_rows;  // C_r
};

// Order-preserving unsigned key of a finite float (larger float -> larger
// key; -0 and +0 share a key so they tie; finite keys are >= 0x00800000).
// Non-finite logits get key 1, below every finite one, so they are picked
// only when fewer than k finite logits remain (lowest id first) and flag the
// row.  Key 0 marks padding and experts already picked.
__device__ __forceinline__ uint32_t order_key(float f) {
  if (!isfinite(f)) return 1u;
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Expert held in value slot q of `lane`.  VEC = 4: lane l holds experts
// 128*(q/4) + 4l + q%4 (loaded as float4; E % 128 == 0).  VEC = 1: expert
// 32q + l.  Either way the expert id grows with q for a fixed lane.
template <int VEC>
__device__ __forceinline__ int expert_of(int q, int lane) {
  if constexpr (VEC == 4) return (q >> 2) * 128 + lane * 4 + (q & 3);
  else return q * 32 + lane;
}

// Top-k and softmax of token t by the calling warp; returns lane j's pick.
template <int VPL, int VEC>
__device__ __forceinline__ int route_token(const RouteArgs& a, int64_t t, int lane) {
  const int E = a.E, K = a.K;
  const float* row = a.logits + t * E;
  uint32_t key[VPL];
  if constexpr (VEC == 4) {
#pragma unroll
    for (int q4 = 0; q4 < VPL / 4; ++q4) {
      const float4 v = __ldcs(reinterpret_cast<const float4*>(row + q4 * 128) + lane);
      key[4 * q4 + 0] = order_key(v.x);
      key[4 * q4 + 1] = order_key(v.y);
      key[4 * q4 + 2] = order_key(v.z);
      key[4 * q4 + 3] = order_key(v.w);
    }
  } else {
#pragma unroll
    for (int q = 0; q < VPL; ++q) {
      const int e = expert_of<VEC>(q, lane);
      key[q] = e < E ? order_key(__ldcs(row + e)) : 0u;
    }
  }
  // This lane's best two untaken values (strict compares keep the lower id
  // first among equal keys).  Each round the warp takes the largest head;
  // the owning lane moves its second value up, and rescans only when both
  // were taken -- rare, since the k winners spread over 32 lanes.
  uint32_t k1 = 0u, k2 = 0u, taken = 0u;
  int q1 = 0, q2 = 0;
#pragma unroll
  for (int q = 0; q < VPL; ++q) {
    const uint32_t v = key[q];
    if (v > k1) {
      k2 = k1; q2 = q1; k1 = v; q1 = q;
    } else if (v > k2) {
      k2 = v; q2 = q;
    }
  }
  bool have2 = true;
  uint32_t my_key = 0u;
  int my_i = 0;
  for (int j = 0; j < K; ++j) {
    const uint32_t m = __reduce_max_sync(kFull, k1);
    const int e1 = expert_of<VEC>(q1, lane);
    const int e = int(__reduce_min_sync(kFull, k1 == m ? uint32_t(e1) : 0xFFFFFFFFu));
    if (lane == j) {
      my_key = m;
      my_i = e;
    }
    if (k1 == m && e1 == e) {
      taken |= 1u << q1;
      if (have2) {
        k1 = k2; q1 = q2; have2 = false;
      } else {
        k1 = k2 = 0u; q1 = q2 = 0;
#pragma unroll
        for (int q = 0; q < VPL; ++q) {
          const uint32_t v = ((taken >> q) & 1u) ? 0u : key[q];
          if (v > k1) {
            k2 = k1; q2 = q1; k1 = v; q1 = q;
          } else if (v > k2) {
            k2 = v; q2 = q;
          }
        }
        have2 = true;
      }
    }
  }
  // softmax over the k winners, shifted by the largest (lane 0's)
  const float v = key_value(my_key);
  const float top = __shfl_sync(kFull, v, 0);
  const float ex = lane < K ? expf(v - top) : 0.f;
  float s = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(kFull, s, off);
  if (lane < K) {
    a.topk_idx[t * K + lane] = my_i;
    a.topk_w[t * K + lane] = ex / s;
  }
  if (__any_sync(kFull, lane < K && my_key == 1u) && lane == 0) set_status(a.ws, MOE_ERR_NONFINITE);
  return my_i;
}

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
  // ---- offsets of this unit's experts from the phase-1 totals: one warp each
  if (warp < W) {
    const int e = e0 + warp;
    const int r = e / per_rank;
    int sum = 0;
    for (int e2 = r * per_rank + lane; e2 < e; e2 += 32) sum += __ldcg(tot + e2);
    sum = __reduce_add_sync(kFull, sum);
    if (lane == 0) {
      const int off = r * a.region_rows + sum;
      s_off[warp] = off;
      a.expert_off[e] = off;
      a.counts[e] = __ldcg(tot + e);
    }
  }
  __syncthreads();
  // ---- exclusive scan of this unit's own columns over the route blocks
  V* base = reinterpret_cast<V*>(a.bases) + u;
  const V* own = cnt + u;
  const int per = (B + kRouteThreads - 1) / kRouteThreads;
  const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
  V sum = zero;
  for (int b = b0; b < b1; ++b) add(sum, __ldcg(own + int64_t(b) * row));
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
  V run;
  if constexpr (W == 4) run = make_int4(s_off[0], s_off[1], s_off[2], s_off[3]);
  else run = s_off[0];
  for (int w = 0; w < warp; ++w) add(run, s_warp[w]);
  // run + (incl - sum) = absolute base of this thread's first block
  V ex = incl;
  if constexpr (W == 4) { ex.x -= sum.x; ex.y -= sum.y; ex.z -= sum.z; ex.w -= sum.w; }
  else ex -= sum;
  add(run, ex);
  for (int b = b0; b < b1; ++b) {
    base[int64_t(b) * row] = run;
    add(run, __ldcg(own + int64_t(b) * row));
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
    // the other half starts the next call at zero
    int32_t* next = a.totals + size_t(s_parity ^ 1u) * E;
    for (int e = tid; e < E; e += kRouteThreads) next[e] = 0;
    if (tid == 0) a.expert_off[E] = a.R * a.region_rows;
  }
  grid_dependents_launch();
}

// Cooperative launch: every block resident, as the grid barrier requires.
template <int VPL, int VEC>
cudaError_t launch_coop(const RouteArgs& a, int sms, cudaStream_t st) {
  static int per_sm[64] = {0};  // resident blocks per SM, per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  if (per_sm[dev] == 0) {
    int nb = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, route_kernel<VPL, VEC>, kRouteThreads, 0);
    if (e != cudaSuccess) return e;
    if (nb < 1) return cudaErrorInvalidConfiguration;
    per_sm[dev] = nb;
  }
  const int cols = (a.E & 3) == 0 ? a.E / 4 : a.E;
  int grid = a.blocks > cols ? a.blocks : cols;
  if (grid > per_sm[dev] * sms) grid = per_sm[dev] * sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.blockDim = dim3(kRouteThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, route_kernel<VPL, VEC>, a);
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
  a.rank = reinterpret_cast<uint8_t*>(w + p.lay.rank);
  a.ws = ws;
  a.n = n;
  a.E = p.d.n_experts;
  a.K = p.d.top_k;
  a.R = p.d.n_ranks;
  a.blocks = route_blocks(n);
  a.region_rows = int32_t(region_rows(p, n));
  const int sms = num_sms();
  const int E = a.E;
  if (E % 128 == 0) {
    // float4 layout: E / 32 values per lane, a multiple of 4
    if (E == 128) return launch_coop<4, 4>(a, sms, st);
    if (E == 256) return launch_coop<8, 4>(a, sms, st);
    if (E == 384) return launch_coop<12, 4>(a, sms, st);
    return launch_coop<16, 4>(a, sms, st);
  }
  const int vpl = (E + 31) / 32;
  if (vpl <= 1) return launch_coop<1, 1>(a, sms, st);
  if (vpl <= 2) return launch_coop<2, 1>(a, sms, st);
  if (vpl <= 4) return launch_coop<4, 1>(a, sms, st);
  if (vpl <= 8) return launch_coop<8, 1>(a, sms, st);
  return launch_coop<16, 1>(a, sms, st);
}

}  // namespace moe

namespace moe {

// The route kernels on caller-chosen scratch: ctrl (control words), blk and
// bases ([route blocks, E] int32 each), totals ([2, E] int32, zero before the
// first call) and rank ([n, k] bytes).
cudaError_t launch_route_on(const moe_plan& p, int32_t n, const float* logits, int32_t* topk_idx,
                            float* topk_w, int32_t* counts, int32_t* expert_off, void* ctrl,
                            int32_t* blk, int32_t* bases, int32_t* totals, uint8_t* rank,
                            cudaStream_t st) {
  RouteArgs a;
  a.logits = logits;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.counts = counts;
  a.expert_off = expert_off;
  a.blk = blk;
  a.bases = bases;
  a.totals = totals;
  a.rank = rank;
  a.ws = ctrl;
  a.n = n;
  a.E = p.d.n_experts;
  a.K = p.d.top_k;
  a.R = p.d.n_ranks;
  a.blocks = route_blocks(n);
  a.region_rows = int32_t(region_rows(p, n));
  const int sms = num_sms();
  const int E = a.E;
  if (E % 128 == 0) {
    if (E == 128) return launch_coop<4, 4>(a, sms, st);
    if (E == 256) return launch_coop<8, 4>(a, sms, st);
    if (E == 384) return launch_coop<12, 4>(a, sms, st);
    return launch_coop<16, 4>(a, sms, st);
  }
  const int vpl = (E + 31) / 32;
  if (vpl <= 1) return launch_coop<1, 1>(a, sms, st);
  if (vpl <= 2) return launch_coop<2, 1>(a, sms, st);
  if (vpl <= 4) return launch_coop<4, 1>(a, sms, st);
  if (vpl <= 8) return launch_coop<8, 1>(a, sms, st);
  return launch_coop<16, 1>(a, sms, st);
}

}  // namespace moe
