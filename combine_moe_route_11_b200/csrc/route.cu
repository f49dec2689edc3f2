// Route: top-k gating, per-expert counts, rank-major expert offsets and the
// per-block base slots from which moe_dispatch derives every slot.
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
// One ordinary launch; no block ever waits for another:
//  1. per route block of 32 tokens (one CTA, one warp per token): the k
//     largest logits by k rounds of a warp argmax on order-preserving integer
//     keys (two single-instruction warp reductions per round; the lower
//     expert id wins a tie) and a softmax over the k winners; then, per
//     expert, the bitmask of the block's tokens that picked it gives each
//     (token, expert) pair its rank among the block's tokens (popcount of the
//     lower lanes) and the block's count of the expert, written to a
//     [blocks, E] table;
//  2. each CTA then counts itself done on a workspace counter; the CTA that
//     finishes last reads the whole count table at once (every load in
//     flight together), scans each expert's column over the route blocks,
//     turns the expert totals into the rank-major offsets and writes each
//     route block's absolute base slot per expert.
// A slot is then base[block][e] + rank.  All integer results are
// deterministic: no atomic decides an order.  The counter is reset by the
// CTA that read it last, so the next call finds it at zero.
#include "route_common.cuh"

#include <type_traits>

namespace moe {
namespace {

static_assert(kWarps == 32, "one warp per token of a 32-token route block");
constexpr int kScanCache = 32;  // count-table rows a scanning thread keeps in registers

// The last CTA: column sums of the [B, E] count table, the rank-major
// offsets, and the absolute base of every (route block, expert).  Thread
// (e, q) with e = tid % E, q = tid / E (Q = kRouteThreads / E threads per
// column) owns rows [q * rows_q, (q + 1) * rows_q) of column e.
__device__ __forceinline__ void scan_counts(const RouteArgs& a, int32_t* s_part, int32_t* s_pre,
                                            int32_t* s_wsum) {
  const int E = a.E, B = a.blocks;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Q = kRouteThreads / E;  // E <= 512, so Q >= 2
  const int rows_q = (B + Q - 1) / Q;
  const bool active = tid < Q * E;
  const int e = active ? tid % E : 0, q = active ? tid / E : 0;
  const int r0 = min(B, q * rows_q), r1 = min(B, r0 + rows_q);
  const int32_t* col = a.blk + e;
  int32_t* bcol = a.bases + e;
  // ---- pass 1: this thread's sum of its rows (kept when there are few)
  int32_t c[kScanCache];
  int sum = 0;
  const bool cached = rows_q <= kScanCache;
  if (active) {
    if (cached) {
#pragma unroll
      for (int i = 0; i < kScanCache; ++i)
        c[i] = r0 + i < r1 ? __ldcg(col + int64_t(r0 + i) * E) : 0;
#pragma unroll
      for (int i = 0; i < kScanCache; ++i) sum += c[i];
    } else {
      for (int r = r0; r < r1; r += 16) {
        int32_t v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = r + i < r1 ? __ldcg(col + int64_t(r + i) * E) : 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) sum += v[i];
      }
    }
    s_part[q * E + e] = sum;
  }
  __syncthreads();
  // ---- expert totals and their exclusive prefix over all experts
  int tot = 0;
  if (tid < E)
    for (int q2 = 0; q2 < Q; ++q2) tot += s_part[q2 * E + tid];
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
  const int pre = incl - tot + s_wsum[warp];
  if (tid < E) s_pre[tid] = pre;
  __syncthreads();
  const int per_rank = E / a.R;
  if (tid < E) {
    const int r = tid / per_rank;
    const int off = r * a.region_rows + pre - s_pre[r * per_rank];
    a.counts[tid] = tot;
    a.expert_off[tid] = off;
  }
  if (tid == 0) a.expert_off[E] = a.R * a.region_rows;
  // ---- pass 2: absolute bases of this thread's rows
  if (active) {
    const int rk = e / per_rank;
    int run = rk * a.region_rows + s_pre[e] - s_pre[rk * per_rank];
    for (int q2 = 0; q2 < q; ++q2) run += s_part[q2 * E + e];
    if (cached) {
#pragma unroll
      for (int i = 0; i < kScanCache; ++i)
        if (r0 + i < r1) {
          bcol[int64_t(r0 + i) * E] = run;
          run += c[i];
        }
    } else {
      for (int r = r0; r < r1; r += 16) {
        int32_t v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = r + i < r1 ? __ldcg(col + int64_t(r + i) * E) : 0;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (r + i < r1) {
            bcol[int64_t(r + i) * E] = run;
            run += v[i];
          }
      }
    }
  }
}

// kFromIdx: the picks are already in topk_idx (the router GEMM wrote them);
// the counts, offsets and bases are built from them and topk_idx / topk_w
// are left as they are.
template <int VPL, int VEC, bool kFromIdx>
__global__ void __launch_bounds__(kRouteThreads, 1) route_kernel(RouteArgs a) {
  __shared__ int32_t s_sel[kRouteTokens * kMaxTopK];  // picks of the block's tokens
  __shared__ uint32_t s_mask[kMaxExperts];            // token mask per expert
  __shared__ int32_t s_part[kRouteThreads];           // last CTA: partial column sums
  __shared__ int32_t s_pre[kMaxExperts];
  __shared__ int32_t s_wsum[kWarps];
  __shared__ int s_last;
  const int E = a.E, K = a.K, B = a.blocks;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x;
  const int t_base = b * kRouteTokens;
  const int valid = max(0, min(kRouteTokens, a.n - t_base));
  grid_dependency_wait();
  for (int i = tid; i < E; i += kRouteThreads) s_mask[i] = 0u;

  // ---- 1. top-k and softmax (one warp per token), or the given picks
  if constexpr (kFromIdx) {
    __syncthreads();
    for (int p = tid; p < valid * K; p += kRouteThreads) {
      int e = __ldg(a.topk_idx + int64_t(t_base) * K + p);
      if (e < 0 || e >= E) {
        set_status(a.ws, MOE_ERR_DEVICE_INDEX);
        e = -1;
      }
      s_sel[p] = e;
    }
  } else {
    if (warp < valid) {
      float w;
      bool nonfinite;
      const int64_t t = int64_t(t_base) + warp;
      const int e = route_row<VPL, VEC, true>(a.logits + t * E, E, K, lane, &w, &nonfinite);
      if (lane < K) {
        a.topk_idx[t * K + lane] = e;
        a.topk_w[t * K + lane] = w;
        s_sel[warp * K + lane] = e;
      }
      if (nonfinite && lane == 0) set_status(a.ws, MOE_ERR_NONFINITE);
    }
  }
  __syncthreads();
  // ---- per-expert token masks, in-block ranks, block counts
  for (int p = tid; p < valid * K; p += kRouteThreads)
    if (!kFromIdx || s_sel[p] >= 0) atomicOr(&s_mask[s_sel[p]], 1u << (p / K));
  __syncthreads();
  for (int p = tid; p < valid * K; p += kRouteThreads) {
    const int e = s_sel[p];
    a.rank[int64_t(t_base) * K + p] =
        kFromIdx && e < 0 ? uint8_t(0) : uint8_t(__popc(s_mask[e] & ((1u << (p / K)) - 1u)));
  }
  for (int e = tid; e < E; e += kRouteThreads) a.blk[int64_t(b) * E + e] = __popc(s_mask[e]);

  // ---- 2. the CTA that finishes last scans the count table
  __syncthreads();
  if (tid == 0) {
    Ctrl* ctrl = reinterpret_cast<Ctrl*>(a.ws);
    fence_acq_rel_gpu();  // this CTA's counts before its arrival
    s_last = atomicAdd(&ctrl->ticket, 1u) == unsigned(B - 1);
    if (s_last) {
      fence_acq_rel_gpu();  // every other CTA's counts before the reads below
      ctrl->ticket = 0u;    // every CTA has arrived: the next call starts at zero
    }
  }
  __syncthreads();
  if (s_last) scan_counts(a, s_part, s_pre, s_wsum);
  grid_dependents_launch();
}

template <int VPL, int VEC, bool kFromIdx>
cudaError_t launch_rk(const RouteArgs& a, cudaStream_t st) {
  return launch_pdl(route_kernel<VPL, VEC, kFromIdx>, dim3(unsigned(a.blocks)),
                    dim3(kRouteThreads), 0, st, a);
}

cudaError_t launch_with(RouteArgs& a, const moe_plan& p, int32_t n, cudaStream_t st,
                        bool from_idx = false) {
  a.n = n;
  a.E = p.d.n_experts;
  a.K = p.d.top_k;
  a.R = p.d.n_ranks;
  a.blocks = route_blocks(n);
  a.region_rows = int32_t(region_rows(p, n));
  a.masks = nullptr;
  a.mask_rows = 0;
  if (from_idx) return launch_rk<1, 1, true>(a, st);
  return with_route_shape(a.E, [&](auto vpl, auto vec) {
    return launch_rk<decltype(vpl)::value, decltype(vec)::value, false>(a, st);
  });
}

RouteArgs ws_args(const moe_plan& p, void* ws) {
  char* w = static_cast<char*>(ws);
  RouteArgs a;
  a.blk = reinterpret_cast<int32_t*>(w + p.lay.blk);
  a.bases = reinterpret_cast<int32_t*>(w + p.lay.bases);
  a.rank = reinterpret_cast<uint8_t*>(w + p.lay.rank);
  a.ws = ws;
  return a;
}

}  // namespace

cudaError_t launch_route(const moe_plan& p, int32_t n, const float* logits, int32_t* topk_idx,
                         float* topk_w, int32_t* counts, int32_t* expert_off, void* ws,
                         cudaStream_t st) {
  RouteArgs a = ws_args(p, ws);
  a.logits = logits;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.counts = counts;
  a.expert_off = expert_off;
  return launch_with(a, p, n, st);
}

// Counts, offsets and bases of picks already in topk_idx (launch_route
// without its top-k step).
cudaError_t launch_route_counts(const moe_plan& p, int32_t n, int32_t* topk_idx, int32_t* counts,
                                int32_t* expert_off, void* ws, cudaStream_t st) {
  RouteArgs a = ws_args(p, ws);
  a.logits = nullptr;
  a.topk_idx = topk_idx;
  a.topk_w = nullptr;
  a.counts = counts;
  a.expert_off = expert_off;
  return launch_with(a, p, n, st, true);
}

cudaError_t launch_route_on(const moe_plan& p, int32_t n, const float* logits, int32_t* topk_idx,
                            float* topk_w, int32_t* counts, int32_t* expert_off, void* ctrl,
                            int32_t* blk, int32_t* bases, uint8_t* rank, cudaStream_t st) {
  RouteArgs a;
  a.logits = logits;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.counts = counts;
  a.expert_off = expert_off;
  a.blk = blk;
  a.bases = bases;
  a.rank = rank;
  a.ws = ctrl;
  return launch_with(a, p, n, st);
}

}  // namespace moe
