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
// One ordinary launch of min(blocks, SMs) CTAs, each taking every G-th route
// block:
//  1. per route block of 32 tokens (one warp per token): the k
//     largest logits by k rounds of a warp argmax on order-preserving integer
//     keys (two single-instruction warp reductions per round; the lower
//     expert id wins a tie) and a softmax over the k winners; then, per
//     expert, the bitmask of the block's tokens that picked it gives each
//     (token, expert) pair its rank among the block's tokens (popcount of the
//     lower lanes) and the block's count of the expert, written to a
//     [blocks, E] table;
//  2. each CTA adds its counts into per-expert totals (integer atomics: the
//     sums do not depend on their order) and, after its last route block,
//     counts itself arrived on a workspace counter.  The last P = min(CTAs,
//     8) to arrive share the base table: each waits (bounded) until the very
//     last one has arrived, computes the rank-major offsets from the totals,
//     and scans 1/P of the expert columns over the route blocks into
//     absolute base slots, with all of its column loads in flight together.
//     Only CTAs that have finished their own blocks wait, at most P - 1 of
//     them, so the others always have SMs to run on.
// A slot is then base[block][e] + rank.  All integer results are
// deterministic: no atomic decides an order.  A generation word, bumped by
// each call's last arrival, selects which of two arrival counters and which
// half of the double-buffered totals a call uses; CTA 0 clears the other
// counter and half for the next call.
#include "route_common.cuh"

#include <type_traits>

namespace moe {
namespace {

static_assert(kWarps == 32, "one warp per token of a 32-token route block");
constexpr int kScanCache = 8;   // count-table rows a scanning thread keeps in registers
constexpr int kScanBatch = 8;  // count-table rows per batch when they are not all cached
constexpr int kScanners = 8;   // CTAs that share the base table: the last ones to arrive

// Rows [r, min(r + kScanBatch, r1)) of a count column (zero past r1); the
// column holds at most blocks * E < 2^31 elements past `col`.
__device__ __forceinline__ void load_rows(const int32_t* col, int r, int r1, int E,
                                          int32_t (&v)[kScanBatch]) {
#pragma unroll
  for (int i = 0; i < kScanBatch; ++i) v[i] = r + i < r1 ? __ldcg(col + (r + i) * E) : 0;
}

// One scanning CTA, once every CTA has arrived: the rank-major offsets of all
// experts from their totals (every scanner computes them; `writer` stores
// counts and expert_off), then the absolute base of every (route block,
// expert) for the experts [c0, c1).  Thread (e, q), e in [c0, c1), owns rows
// [q * rows_q, (q + 1) * rows_q) of column e.
__device__ __forceinline__ void scan_columns(const RouteArgs& a, const int32_t* tot, int c0,
                                             int c1, bool writer, int32_t* s_part,
                                             int32_t* s_pre, int32_t* s_wsum) {
  const int E = a.E, B = a.blocks;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the totals and this thread's count rows are loaded together: neither
  // waits for the other
  const int t_e = tid < E ? __ldcg(tot + tid) : 0;
  // ---- this scanner's columns: thread (e, q) and its rows
  const int ncol = max(0, c1 - c0);
  const int Q = ncol > 0 ? kRouteThreads / ncol : 0;  // threads per column (Q >= 2)
  const int rows_q = ncol > 0 ? (B + Q - 1) / Q : 0;
  const bool active = tid < Q * ncol;
  const int e = c0 + (active ? tid % ncol : 0), q = active ? tid / ncol : 0;
  const int r0 = min(B, q * rows_q), r1 = min(B, r0 + rows_q);
  const int32_t* col = a.blk + int64_t(r0) * E + e;
  int32_t* bcol = a.bases + int64_t(r0) * E + e;
  const int nr = r1 - r0;
  // pass 1: this thread's sum of its rows (kept when there are few)
  int32_t c[kScanCache];
  int sum = 0;
  const bool cached = rows_q <= kScanCache;
  if (active) {
    if (cached) {
#pragma unroll
      for (int i = 0; i < kScanCache; ++i) c[i] = i < nr ? __ldcg(col + i * E) : 0;
#pragma unroll
      for (int i = 0; i < kScanCache; ++i) sum += c[i];
    } else {
      int32_t v[kScanBatch];
      load_rows(col, 0, nr, E, v);
      for (int r = 0; r < nr; r += kScanBatch) {
        int32_t w[kScanBatch];
        load_rows(col, r + kScanBatch, nr, E, w);
#pragma unroll
        for (int i = 0; i < kScanBatch; ++i) sum += v[i];
#pragma unroll
        for (int i = 0; i < kScanBatch; ++i) v[i] = w[i];
      }
    }
    s_part[q * ncol + (e - c0)] = sum;
  }
  // ---- offsets of all experts: exclusive prefix of the totals
  int incl = t_e;
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
  const int pre = incl - t_e + s_wsum[warp];
  if (tid < E) s_pre[tid] = pre;
  __syncthreads();  // also publishes s_part
  const int per_rank = E / a.R;
  if (writer && tid < E) {
    const int r = tid / per_rank;
    a.counts[tid] = t_e;
    a.expert_off[tid] = r * a.region_rows + pre - s_pre[r * per_rank];
  }
  if (writer && tid == 0) a.expert_off[E] = a.R * a.region_rows;
  // pass 2: absolute bases of this thread's rows
  if (active) {
    const int rk = e / per_rank;
    int run = rk * a.region_rows + s_pre[e] - s_pre[rk * per_rank];
    for (int q2 = 0; q2 < q; ++q2) run += s_part[q2 * ncol + (e - c0)];
    if (cached) {
#pragma unroll
      for (int i = 0; i < kScanCache; ++i)
        if (i < nr) {
          bcol[i * E] = run;
          run += c[i];
        }
    } else {
      int32_t v[kScanBatch];
      load_rows(col, 0, nr, E, v);
      for (int r = 0; r < nr; r += kScanBatch) {
        int32_t w[kScanBatch];
        load_rows(col, r + kScanBatch, nr, E, w);
#pragma unroll
        for (int i = 0; i < kScanBatch; ++i)
          if (r + i < nr) {
            bcol[(r + i) * E] = run;
            run += v[i];
          }
#pragma unroll
        for (int i = 0; i < kScanBatch; ++i) v[i] = w[i];
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
  __shared__ int32_t s_part[kRouteThreads];           // scanners: partial column sums
  __shared__ int32_t s_pre[kMaxExperts];
  __shared__ int32_t s_wsum[kWarps];
  __shared__ int s_arrival;
  __shared__ unsigned s_gen;
  __shared__ int s_ok;
  const int E = a.E, K = a.K;
  const int G = gridDim.x;  // CTAs; each takes route blocks blockIdx.x, + G, + 2G, ...
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(a.ws);
  grid_dependency_wait();
  // the generation of this call: it selects the arrival counter and the half
  // of the totals, and the last arrival bumps it once every CTA has read it
  if (tid == 0) s_gen = ld_acquire_gpu(&ctrl->rgen);
  __syncthreads();
  const unsigned gen = s_gen;
  int32_t* tot = a.totals + size_t(gen & 1u) * E;
  // this call's arrival counter; the other one starts the next call at zero
  unsigned* ticket = (gen & 1u) ? &ctrl->ticket_b : &ctrl->ticket;
  if (blockIdx.x == 0) {
    for (int i = tid; i < E; i += kRouteThreads) a.totals[size_t((gen & 1u) ^ 1u) * E + i] = 0;
    if (tid == 0) st_relaxed_gpu((gen & 1u) ? &ctrl->ticket : &ctrl->ticket_b, 0u);
  }

  for (int b = blockIdx.x; b < a.blocks; b += G) {
    const int t_base = b * kRouteTokens;
    const int valid = max(0, min(kRouteTokens, a.n - t_base));
    for (int i = tid; i < E; i += kRouteThreads) s_mask[i] = 0u;
    // ---- 1. top-k and softmax (one warp per token), or the given picks
    if constexpr (kFromIdx) {
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
    // ---- per-expert token masks, in-block ranks, block counts, expert totals
    for (int p = tid; p < valid * K; p += kRouteThreads)
      if (!kFromIdx || s_sel[p] >= 0) atomicOr(&s_mask[s_sel[p]], 1u << (p / K));
    __syncthreads();
    for (int p = tid; p < valid * K; p += kRouteThreads) {
      const int e = s_sel[p];
      a.rank[int64_t(t_base) * K + p] =
          kFromIdx && e < 0 ? uint8_t(0) : uint8_t(__popc(s_mask[e] & ((1u << (p / K)) - 1u)));
    }
    for (int e = tid; e < E; e += kRouteThreads) {
      const int cnt = __popc(s_mask[e]);
      a.blk[int64_t(b) * E + e] = cnt;
      if (cnt) atomicAdd(tot + e, cnt);  // integer sums: the order does not matter
    }
    __syncthreads();  // s_sel and s_mask are reused by the next route block
  }

  // ---- 2. arrival; the last P CTAs to arrive build the base table together
  const int P = min(G, kScanners);
  if (tid == 0) {
    // release: this CTA's counts and totals (ordered before by the block
    // barrier) before its arrival
    fence_acq_rel_gpu();
    const int arrival = int(atomicAdd(ticket, 1u));
    int ok = 1;
    if (arrival == G - 1) {
      // every CTA has arrived: the fence acquires every CTA's counts (this
      // CTA scans too); the next call uses the other counter and half
      fence_acq_rel_gpu();
      atomicAdd(&ctrl->rgen, 1u);
    } else if (arrival >= G - P) {
      // a scanner: wait (bounded) until the counter shows every arrival; the
      // acquiring load that sees it orders the reads below
      const long long t0 = clock64();
      while (ld_acquire_gpu(ticket) != unsigned(G)) {
        if (clock64() - t0 > (1ll << 31)) {
          set_status(a.ws, MOE_ERR_TIMEOUT);
          ok = 0;
          break;
        }
      }
    }
    // the other CTAs read nothing after their arrival
    s_arrival = arrival;
    s_ok = ok;
  }
  __syncthreads();
  // Every CTA has started by now, so the next kernel in the stream may be
  // scheduled behind the scanners; it still waits for this grid to finish
  // before it reads anything.
  grid_dependents_launch();
  const int arrival = s_arrival;
  if (arrival >= G - P && s_ok) {
    const int s_idx = arrival - (G - P);
    const int per = (E + P - 1) / P;
    scan_columns(a, tot, min(E, s_idx * per), min(E, (s_idx + 1) * per), s_idx == P - 1, s_part,
                 s_pre, s_wsum);
  }
}

// One CTA per SM at most (a CTA of 1024 threads fills an SM): with more route
// blocks than SMs each CTA takes several, so no block waits for a second
// wave of CTAs to start.
template <int VPL, int VEC, bool kFromIdx>
cudaError_t launch_rk(const RouteArgs& a, cudaStream_t st) {
  const int grid = a.blocks < num_sms() ? a.blocks : num_sms();
  return launch_pdl(route_kernel<VPL, VEC, kFromIdx>, dim3(unsigned(grid)), dim3(kRouteThreads),
                    0, st, a);
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
  a.totals = reinterpret_cast<int32_t*>(w + p.lay.totals);
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
                            int32_t* totals, int32_t* blk, int32_t* bases, uint8_t* rank,
                            cudaStream_t st) {
  RouteArgs a;
  a.logits = logits;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.counts = counts;
  a.expert_off = expert_off;
  a.blk = blk;
  a.bases = bases;
  a.rank = rank;
  a.totals = totals;
  a.ws = ctrl;
  return launch_with(a, p, n, st);
}

}  // namespace moe
