// Route: top-k gating, per-expert counts, rank-major expert offsets and the
// in-expert position of every pick, from which moe_dispatch derives slots.
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
// One ordinary launch, one pass, no grid-wide barrier.  A block takes a
// ticket from a counter in the workspace: ticket b is route block b, tokens
// [32b, 32b + 32).  Tickets are handed out in the order blocks start, so a
// block only ever waits on blocks that are already running.
//  1. One warp per token (several tokens per warp): the k largest logits by
//     k rounds of a warp argmax on order-preserving integer keys (the lower
//     expert id wins a tie) and a softmax over the k winners.
//  2. Per expert, the bitmask of the block's tokens that picked it gives each
//     pick its rank among the block's tokens (popcount of the lower bits) and
//     the block's count c[b][e].
//  3. Decoupled look-back, one thread per expert column: block b publishes
//     c[b][e] as an aggregate, then sums the published words of blocks
//     b-1, b-2, ... (a window of loads at a time) until it meets an inclusive
//     prefix; it then publishes its own inclusive prefix.  Block 0 publishes
//     an inclusive prefix at once.  Each word is one 32-bit store: a ready
//     bit, an inclusive bit and the count, so no fence orders value and flag.
//  4. The position of every pick inside its expert's segment is the block's
//     exclusive prefix plus the in-block rank.
//  5. The block holding the last ticket has every expert's total as its
//     inclusive prefix: it turns them into the rank-major offsets.
// All integer results are deterministic: no atomic decides an order.
//
// The look-back words alternate between two halves of a table in the
// workspace: a call uses one half, clears the rows of the other half that
// the previous call wrote, and the last block flips the half for the next
// call.  Every wait is bounded; a wait that gives up records MOE_ERR_TIMEOUT
// and the workspace must be re-initialised.
#include "route_common.cuh"

#include <atomic>

namespace moe {
namespace {

constexpr int kLbWarps = 8;                    // warps per route block
constexpr int kLbThreads = kLbWarps * 32;
constexpr int kTokPerWarp = kRouteTokens / kLbWarps;
constexpr int kWindow = 16;                    // look-back words per window
constexpr int kExpPerThread = (kMaxExperts + kLbThreads - 1) / kLbThreads;

constexpr uint32_t kReady = 0x40000000u;
constexpr uint32_t kIncl = 0x80000000u;
constexpr uint32_t kValue = 0x3FFFFFFFu;

__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// A published look-back word; waits (bounded) until it is ready.  A wait
// that gives up records MOE_ERR_TIMEOUT and reads as an inclusive zero, so
// the look-back ends.
__device__ __forceinline__ uint32_t wait_ready(const uint32_t* p, uint32_t v, void* ws) {
  if (v & kReady) return v;
  const long long t0 = clock64();
  while (!((v = ld_relaxed_gpu(p)) & kReady)) {
    if (clock64() - t0 > (1ll << 31)) {
      set_status(ws, MOE_ERR_TIMEOUT);
      return kReady | kIncl;
    }
  }
  return v;
}

// Exclusive prefix of column `col` over the route blocks below b: windows of
// kWindow words, the next window's loads in flight while the current one is
// summed, until an inclusive prefix turns up.
__device__ __forceinline__ void load_window(const uint32_t* col, int p, int stride,
                                            uint32_t (&w)[kWindow]) {
#pragma unroll
  for (int i = 0; i < kWindow; ++i)
    w[i] = p - i >= 0 ? ld_relaxed_gpu(col + int64_t(p - i) * stride) : (kReady | kIncl);
}

__device__ __forceinline__ int look_back(const uint32_t* col, int b, int stride, void* ws) {
  int excl = 0;
  uint32_t cur[kWindow], nxt[kWindow];
  load_window(col, b - 1, stride, cur);
  for (int p = b - 1; p >= 0; p -= kWindow) {
    if (p - kWindow >= 0) load_window(col, p - kWindow, stride, nxt);
#pragma unroll
    for (int i = 0; i < kWindow; ++i) {
      const uint32_t v = wait_ready(col + int64_t(max(p - i, 0)) * stride, cur[i], ws);
      excl += int(v & kValue);
      if (v & kIncl) return excl;
    }
#pragma unroll
    for (int i = 0; i < kWindow; ++i) cur[i] = nxt[i];
  }
  return excl;  // not reached: block 0 publishes an inclusive prefix
}

// kFromIdx: the picks are already in topk_idx (the router GEMM wrote them);
// steps 2-5 run on them and topk_idx / topk_w are left as they are.
template <int VPL, int VEC, bool kFromIdx>
__global__ void __launch_bounds__(kLbThreads, 2) route_kernel(RouteArgs a) {
  __shared__ int32_t s_sel[kRouteTokens * kMaxTopK];  // picks of the block's tokens
  __shared__ uint32_t s_mask[kMaxExperts];            // token mask per expert
  __shared__ int32_t s_excl[kMaxExperts];             // exclusive prefix per expert
  __shared__ int32_t s_wsum[kLbWarps];
  __shared__ unsigned s_b, s_half, s_dirty;
  const int E = a.E, K = a.K, B = a.blocks;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(a.ws);
  grid_dependency_wait();
  if (tid == 0) {
    // the half and the rows to clear are read before the ticket is taken;
    // the last block changes them only after every ticket is out
    const unsigned half = a.flag_halves == 2 ? (ld_acquire_gpu(&ctrl->parity) & 1u) : 0u;
    s_half = half;
    s_dirty = a.flag_halves == 2 ? ld_relaxed_gpu(&ctrl->dirty[half ^ 1u]) : 0u;
    s_b = atomicAdd(&ctrl->ticket, 1u);
  }
  for (int e = tid; e < E; e += kLbThreads) s_mask[e] = 0u;
  __syncthreads();
  const int b = int(s_b);
  if (b >= B) {  // the counter was not reset: the workspace needs moe_workspace_init
    if (tid == 0) set_status(a.ws, MOE_ERR_TIMEOUT);
    return;
  }
  uint32_t* flags = a.flags + size_t(s_half) * a.flag_rows * E;
  const int t0 = b * kRouteTokens;
  const int valid = max(0, min(kRouteTokens, a.n - t0));

  // ---- 1. top-k and softmax: warp w routes tokens w, w + kLbWarps, ...
  if constexpr (kFromIdx) {
    for (int p = tid; p < valid * K; p += kLbThreads) {
      int e = __ldg(a.topk_idx + int64_t(t0) * K + p);
      if (e < 0 || e >= E) {
        set_status(a.ws, MOE_ERR_DEVICE_INDEX);
        e = -1;
      }
      s_sel[p] = e;
    }
  } else {
    uint32_t key[kTokPerWarp][VPL];
#pragma unroll
    for (int i = 0; i < kTokPerWarp; ++i) {
      const int tl = warp + i * kLbWarps;
      if (tl < valid) load_keys<VPL, VEC, true>(a.logits + int64_t(t0 + tl) * E, E, lane, key[i]);
    }
#pragma unroll
    for (int i = 0; i < kTokPerWarp; ++i) {
      const int tl = warp + i * kLbWarps;
      if (tl < valid) {
        float w;
        bool nonfinite;
        const int e = select_topk<VPL, VEC>(key[i], K, lane, &w, &nonfinite);
        if (lane < K) {
          const int64_t tk = int64_t(t0 + tl) * K + lane;
          a.topk_idx[tk] = e;
          a.topk_w[tk] = w;
          s_sel[tl * K + lane] = e;
        }
        if (nonfinite && lane == 0) set_status(a.ws, MOE_ERR_NONFINITE);
      }
    }
  }
  __syncthreads();
  // ---- 2. per-expert token masks of the block
  for (int p = tid; p < valid * K; p += kLbThreads)
    if (!kFromIdx || s_sel[p] >= 0) atomicOr(&s_mask[s_sel[p]], 1u << (p / K));
  __syncthreads();
  // ---- 3. publish, look back, publish the inclusive prefix
  // (every column's aggregate goes out before any of this thread's waits)
  for (int e = tid; e < E; e += kLbThreads)
    st_relaxed_u32(flags + int64_t(b) * E + e,
                   (b == 0 ? kReady | kIncl : kReady) | uint32_t(__popc(s_mask[e])));
  for (int e = tid; e < E; e += kLbThreads) {
    int excl = 0;
    if (b > 0) {
      excl = look_back(flags + e, b, E, a.ws);
      st_relaxed_u32(flags + int64_t(b) * E + e,
                     kReady | kIncl | uint32_t(excl + __popc(s_mask[e])));
    }
    s_excl[e] = excl;
  }
  // the rows of the other half that the previous call wrote start the next
  // call at zero; route blocks share them out
  if (a.flag_halves == 2) {
    uint32_t* other = a.flags + size_t(s_half ^ 1u) * a.flag_rows * E;
    for (int r = b; r < int(s_dirty); r += B)
      for (int e = tid; e < E; e += kLbThreads) other[int64_t(r) * E + e] = 0u;
  }
  __syncthreads();
  // ---- 4. in-expert positions of the block's picks
  for (int p = tid; p < valid * K; p += kLbThreads) {
    const int e = s_sel[p];
    a.pos[int64_t(t0) * K + p] =
        kFromIdx && e < 0 ? -1 : s_excl[e] + __popc(s_mask[e] & ((1u << (p / K)) - 1u));
  }
  // ---- 5. the last block: totals -> rank-major offsets
  if (b == B - 1) {
    // exclusive scan of the totals over the experts (kExpPerThread per thread)
    int tot[kExpPerThread];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < kExpPerThread; ++i) {
      const int e = tid * kExpPerThread + i;
      tot[i] = e < E ? s_excl[e] + __popc(s_mask[e]) : 0;
      sum += tot[i];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w2 = 0; w2 < warp; ++w2) before += s_wsum[w2];
    int pre = before + incl - sum;  // totals of the experts below this thread's first
    __syncthreads();                // s_excl is rewritten below
#pragma unroll
    for (int i = 0; i < kExpPerThread; ++i) {
      const int e = tid * kExpPerThread + i;
      if (e < E) s_excl[e] = pre;  // now: prefix of totals over all experts below e
      pre += tot[i];
    }
    __syncthreads();
    const int per_rank = E / a.R;
#pragma unroll
    for (int i = 0; i < kExpPerThread; ++i) {
      const int e = tid * kExpPerThread + i;
      if (e < E) {
        const int r = e / per_rank;
        const int off = r * a.region_rows + s_excl[e] - s_excl[r * per_rank];
        a.counts[e] = tot[i];
        a.expert_off[e] = off;
        a.off[e] = off;
      }
    }
    if (tid == 0) {
      a.expert_off[E] = a.R * a.region_rows;
      a.off[E] = a.R * a.region_rows;
      if (a.flag_halves == 2) {
        ctrl->dirty[s_half] = unsigned(B);
        ctrl->parity = s_half ^ 1u;
      }
      ctrl->ticket = 0u;
    }
  }
  grid_dependents_launch();
}

template <int VPL, int VEC, bool kFromIdx>
cudaError_t launch_lb(const RouteArgs& a, cudaStream_t st) {
  return launch_pdl(route_kernel<VPL, VEC, kFromIdx>, dim3(unsigned(a.blocks)), dim3(kLbThreads), 0,
                    st, a);
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
  if (from_idx) return launch_lb<1, 1, true>(a, st);
  return with_route_shape(a.E, [&](auto vpl, auto vec) {
    return launch_lb<decltype(vpl)::value, decltype(vec)::value, false>(a, st);
  });
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
  a.flags = reinterpret_cast<uint32_t*>(w + p.lay.flags);
  a.flag_halves = 2;
  a.flag_rows = p.blocks_max;
  a.pos = reinterpret_cast<int32_t*>(w + p.lay.pos);
  a.off = reinterpret_cast<int32_t*>(w + p.lay.off);
  a.ws = ws;
  return launch_with(a, p, n, st);
}

// Counts, offsets and positions of picks already in topk_idx (the workspace
// path of launch_route without its top-k step).
cudaError_t launch_route_counts(const moe_plan& p, int32_t n, int32_t* topk_idx, int32_t* counts,
                                int32_t* expert_off, void* ws, cudaStream_t st) {
  char* w = static_cast<char*>(ws);
  RouteArgs a;
  a.logits = nullptr;
  a.topk_idx = topk_idx;
  a.topk_w = nullptr;
  a.counts = counts;
  a.expert_off = expert_off;
  a.flags = reinterpret_cast<uint32_t*>(w + p.lay.flags);
  a.flag_halves = 2;
  a.flag_rows = p.blocks_max;
  a.pos = reinterpret_cast<int32_t*>(w + p.lay.pos);
  a.off = reinterpret_cast<int32_t*>(w + p.lay.off);
  a.ws = ws;
  return launch_with(a, p, n, st, true);
}

cudaError_t launch_route_on(const moe_plan& p, int32_t n, const float* logits, int32_t* topk_idx,
                            float* topk_w, int32_t* counts, int32_t* expert_off, void* ctrl,
                            uint32_t* flags, int32_t* pos, int32_t* off, cudaStream_t st) {
  RouteArgs a;
  a.logits = logits;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.counts = counts;
  a.expert_off = expert_off;
  a.flags = flags;
  a.flag_halves = 1;
  a.flag_rows = route_blocks(n);
  a.pos = pos;
  a.off = off;
  a.ws = ctrl;
  return launch_with(a, p, n, st);
}

}  // namespace moe
