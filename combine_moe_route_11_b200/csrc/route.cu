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
// One launch, three phases:
//  1. each warp routes tokens: the k largest logits by k rounds of a warp
//     argmax (lower expert id wins a tie), then a softmax over the k winners;
//  2. each block (64 tokens = two 32-token groups) builds, per expert, a
//     bitmask of the tokens of each group that picked it; the rank of token t
//     among the block's tokens picking e is a popcount of the lower lanes, and
//     the block's count of e is the popcount of the whole mask;
//  3. the last block to finish (ticket counter) scans the [blocks, E] count
//     table: expert totals, the rank-major expert offsets, and in place the
//     base slot of every (block, expert).
// All integer results are deterministic: no atomics decide an order.
#include "moe_internal.cuh"

#include <float.h>
#include <limits.h>

namespace moe {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kWarps = kRouteThreads / 32;
constexpr int kTokPerWarp = kRouteTokens / kWarps;

struct RouteArgs {
  const float* logits;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* counts;
  int32_t* expert_off;
  int32_t* blk;    // [blocks, E]: block counts, rewritten as block bases
  uint8_t* rank;   // [n, k]: rank of (t, j) among the block's tokens picking e
  void* ws;
  int32_t n, E, K, R;
  int32_t region_rows;  // C_r
};

template <int VPL>
__device__ __forceinline__ void route_token(const RouteArgs& a, const float (&v)[VPL], int t,
                                            int tl, int lane, int32_t* s_sel) {
  const int E = a.E, K = a.K;
  uint32_t picked = 0;
  float my_v = -INFINITY;
  int my_i = 0;
  bool nonfinite = false;
  for (int j = 0; j < K; ++j) {
    // best remaining (value, id) of this lane; ids ascend with q, so a strict
    // compare keeps the lowest id among equal values
    float bv = -INFINITY;
    int bi = INT_MAX;
#pragma unroll
    for (int q = 0; q < VPL; ++q) {
      const int e = q * 32 + lane;
      if (e < E && !((picked >> q) & 1u) && v[q] > bv) {
        bv = v[q];
        bi = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(kFull, bv, off);
      const int oi = __shfl_xor_sync(kFull, bi, off);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (bi == INT_MAX) {
      // fewer than k finite logits: take the lowest unpicked id, flag it
      int cand = INT_MAX;
#pragma unroll
      for (int q = VPL - 1; q >= 0; --q) {
        const int e = q * 32 + lane;
        if (e < E && !((picked >> q) & 1u)) cand = e;
      }
      bi = __reduce_min_sync(kFull, cand);
      bv = -INFINITY;
      nonfinite = true;
    }
    if ((bi & 31) == lane) picked |= 1u << (bi >> 5);
    if (lane == j) {
      my_v = bv;
      my_i = bi;
    }
  }
  // softmax over the k winners, shifted by the largest (lane 0's)
  const float m = __shfl_sync(kFull, my_v, 0);
  const float ex = lane < K ? expf(my_v - m) : 0.f;
  float s = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(kFull, s, off);
  if (lane < K) {
    a.topk_idx[int64_t(t) * K + lane] = my_i;
    a.topk_w[int64_t(t) * K + lane] = ex / s;
    s_sel[tl * K + lane] = my_i;
  }
  if (nonfinite && lane == 0) set_status(a.ws, MOE_ERR_NONFINITE);
}

template <int VPL>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(RouteArgs a) {
  __shared__ int32_t s_sel[kRouteTokens * kMaxTopK];  // picks of the block's tokens; scan scratch later
  __shared__ uint32_t s_mask[2 * kMaxExperts];        // [group][expert] token masks; scan scratch later
  __shared__ int s_last;

  const int E = a.E, K = a.K;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t_base = blockIdx.x * kRouteTokens;
  const int valid = max(0, min(kRouteTokens, a.n - t_base));
  for (int i = tid; i < 2 * E; i += kRouteThreads) s_mask[i] = 0;

  // ---- phase 1: route this warp's tokens, G at a time with their logits prefetched
  constexpr int G = (32 / VPL) < kTokPerWarp ? (32 / VPL < 1 ? 1 : 32 / VPL) : kTokPerWarp;
  for (int i0 = 0; i0 < kTokPerWarp; i0 += G) {
    float v[G][VPL];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int tl = warp * kTokPerWarp + i0 + g;
      const float* row = a.logits + int64_t(t_base + tl) * E;
#pragma unroll
      for (int q = 0; q < VPL; ++q) {
        const int e = q * 32 + lane;
        v[g][q] = (tl < valid && e < E) ? __ldcs(row + e) : -INFINITY;
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int tl = warp * kTokPerWarp + i0 + g;
      if (tl < valid) route_token<VPL>(a, v[g], t_base + tl, tl, lane, s_sel);
    }
  }
  __syncthreads();

  // ---- phase 2: group masks -> in-block ranks and block counts
  for (int p = tid; p < valid * K; p += kRouteThreads) {
    const int tl = p / K;
    atomicOr(&s_mask[(tl >> 5) * E + s_sel[p]], 1u << (tl & 31));
  }
  __syncthreads();
  for (int p = tid; p < valid * K; p += kRouteThreads) {
    const int tl = p / K, e = s_sel[p];
    int r = __popc(s_mask[(tl >> 5) * E + e] & ((1u << (tl & 31)) - 1u));
    if (tl >= 32) r += __popc(s_mask[e]);
    a.rank[int64_t(t_base) * K + p] = uint8_t(r);
  }
  for (int e = tid; e < E; e += kRouteThreads)
    a.blk[int64_t(blockIdx.x) * E + e] = __popc(s_mask[e]) + __popc(s_mask[E + e]);

  // ---- phase 3: the last block scans the count table
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    Ctrl* c = reinterpret_cast<Ctrl*>(a.ws);
    const unsigned prev = atomicAdd(&c->ticket, 1u);
    s_last = (prev == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  const int B = gridDim.x;
  // Column units are 4 experts read as one int4 when E % 4 == 0, else one
  // expert.  tpc threads split each column unit into tpc chunks of blocks.
  const bool quad = (E & 3) == 0;
  const int cols = quad ? E / 4 : E;
  int tpc = kRouteThreads / cols;
  tpc = tpc < 1 ? 1 : (tpc > B ? B : tpc);
  int32_t* s_part = s_sel;                              // [tpc][E] chunk sums -> chunk bases
  int32_t* s_cnt = reinterpret_cast<int32_t*>(s_mask);  // [E] totals
  int32_t* s_off = s_cnt + E;                           // [E] expert offsets
  for (int task = tid; task < cols * tpc; task += kRouteThreads) {
    const int col = task % cols, c = task / cols;
    const int b0 = int(int64_t(B) * c / tpc), b1 = int(int64_t(B) * (c + 1) / tpc);
    if (quad) {
      int4 sum = make_int4(0, 0, 0, 0);
#pragma unroll 16
      for (int b = b0; b < b1; ++b) {
        const int4 x = __ldcg(reinterpret_cast<const int4*>(a.blk + int64_t(b) * E) + col);
        sum.x += x.x; sum.y += x.y; sum.z += x.z; sum.w += x.w;
      }
      int32_t* dst = s_part + c * E + col * 4;
      dst[0] = sum.x; dst[1] = sum.y; dst[2] = sum.z; dst[3] = sum.w;
    } else {
      int sum = 0;
#pragma unroll 16
      for (int b = b0; b < b1; ++b) sum += __ldcg(a.blk + int64_t(b) * E + col);
      s_part[c * E + col] = sum;
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += kRouteThreads) {
    int run = 0;
    for (int c = 0; c < tpc; ++c) {
      const int x = s_part[c * E + e];
      s_part[c * E + e] = run;
      run += x;
    }
    s_cnt[e] = run;
    a.counts[e] = run;
  }
  __syncthreads();
  const int per_rank = E / a.R;
  for (int e = tid; e < E; e += kRouteThreads) {
    const int r = e / per_rank;
    int off = r * a.region_rows;
    for (int e2 = r * per_rank; e2 < e; ++e2) off += s_cnt[e2];
    s_off[e] = off;
    a.expert_off[e] = off;
  }
  if (tid == 0) a.expert_off[E] = a.R * a.region_rows;
  __syncthreads();
  for (int task = tid; task < cols * tpc; task += kRouteThreads) {
    const int col = task % cols, c = task / cols;
    const int b0 = int(int64_t(B) * c / tpc), b1 = int(int64_t(B) * (c + 1) / tpc);
    if (quad) {
      const int e = col * 4;
      int4 run = make_int4(s_off[e] + s_part[c * E + e], s_off[e + 1] + s_part[c * E + e + 1],
                           s_off[e + 2] + s_part[c * E + e + 2], s_off[e + 3] + s_part[c * E + e + 3]);
#pragma unroll 8
      for (int b = b0; b < b1; ++b) {
        int4* p = reinterpret_cast<int4*>(a.blk + int64_t(b) * E) + col;
        const int4 x = __ldcg(p);
        *p = run;
        run.x += x.x; run.y += x.y; run.z += x.z; run.w += x.w;
      }
    } else {
      int run = s_off[col] + s_part[c * E + col];
#pragma unroll 8
      for (int b = b0; b < b1; ++b) {
        int32_t* p = a.blk + int64_t(b) * E + col;
        const int x = __ldcg(p);
        *p = run;
        run += x;
      }
    }
  }
  if (tid == 0) reinterpret_cast<Ctrl*>(a.ws)->ticket = 0u;
}

}  // namespace

cudaError_t launch_route(const moe_plan& p, int32_t n, const float* logits, int32_t* topk_idx,
                         float* topk_w, int32_t* counts, int32_t* expert_off, void* ws,
                         cudaStream_t st) {
  RouteArgs a;
  a.logits = logits;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.counts = counts;
  a.expert_off = expert_off;
  a.blk = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + p.lay.blk);
  a.rank = reinterpret_cast<uint8_t*>(static_cast<char*>(ws) + p.lay.rank);
  a.ws = ws;
  a.n = n;
  a.E = p.d.n_experts;
  a.K = p.d.top_k;
  a.R = p.d.n_ranks;
  a.region_rows = int32_t(region_rows(p, n));
  const dim3 grid(route_blocks(n)), block(kRouteThreads);
  const int vpl = (a.E + 31) / 32;
  if (vpl <= 1) route_kernel<1><<<grid, block, 0, st>>>(a);
  else if (vpl <= 2) route_kernel<2><<<grid, block, 0, st>>>(a);
  else if (vpl <= 4) route_kernel<4><<<grid, block, 0, st>>>(a);
  else if (vpl <= 8) route_kernel<8><<<grid, block, 0, st>>>(a);
  else route_kernel<16><<<grid, block, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
