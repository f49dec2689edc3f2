// Fused route + dispatch for small batches: top-k gating, counts, rank-major
// offsets and the row scatter in ONE cooperative launch.
//
// At decode sizes the work of each step is a few megabytes, so the fixed cost
// of separate launches and of long serial phases dominates ("One-Sided
// Expert-Parallel All-to-All for Mixture-of-Experts Inference over NVLink",
// abstract: fixed costs dominate at small batch; "backends/mlx: runtime MoE
// expert-sort for decode", Summary: decode skips the sort because of its
// overhead).  Block c owns tokens c, c + G, c + 2G, ... (G blocks), so the
// routing of a batch is spread over as many SMs as it has tokens:
//  1. every warp issues the load of its first 512-byte chunk of x (it does
//     not depend on routing); then one warp per owned token routes it (the
//     same per-row code as the route kernel), keeps the picks in shared
//     memory, writes topk_idx / topk_w, and sets the token's bit in the
//     global mask of each picked expert for its 32-token route block
//     (integer atomics: the resulting masks do not depend on their order);
//  2. one bounded grid barrier;
//  3. every block reads the [blocks, E] masks, and from their popcounts
//     builds the expert totals, the exclusive prefix, the rank-major offsets
//     and each route block's base slot, all in shared memory;
//  4. the block's warps store the chunks of its tokens to their k slots:
//     base + popcount of the lower tokens' bits in the mask, the same
//     (expert, source token) order as the two-kernel path.
// The mask table is double-buffered by the barrier generation: the half a
// call uses was zeroed by the previous call, and each call zeroes the other
// half for the next one.
// Results are identical to moe_route_topk followed by moe_dispatch.
#include "route_common.cuh"

#include <atomic>

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
  int32_t owned;    // most tokens any block owns: ceil(n / grid)
};

template <int VPL, int VEC>
__global__ void __launch_bounds__(kRouteThreads, 1) route_dispatch_kernel(FusedArgs f) {
  extern __shared__ int32_t s_dyn[];  // masks [blocks, E], bases [blocks, E], picks [owned, K]
  __shared__ int32_t s_pre[kMaxExperts];
  __shared__ int32_t s_wsum[kWarps];
  __shared__ unsigned s_gen;
  const RouteArgs& a = f.r;
  const int E = a.E, K = a.K, B = a.blocks, n = a.n;
  const int G = gridDim.x;
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(s_dyn);
  int32_t* s_base = s_dyn + B * E;
  int32_t* s_pick = s_dyn + 2 * B * E;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t row_bytes = int64_t(f.vecs) << 4;
  // tokens of this block: blockIdx.x + i * G for i < mine
  const int mine = int(blockIdx.x) < n ? (n - 1 - int(blockIdx.x)) / G + 1 : 0;
  const int items = mine * f.chunks;  // (owned token i, chunk c) -> i * chunks + c
  grid_dependency_wait();
  unsigned gen = 0u;  // thread 0's copy of the barrier generation
  if (tid == 0) {
    gen = ld_acquire_gpu(&reinterpret_cast<Ctrl*>(a.ws)->gen);
    s_gen = gen;
  }

  // ---- the first chunk of x, in flight while routing runs
  uint4 v0 = make_uint4(0u, 0u, 0u, 0u);
  if (warp < items) {
    const int64_t t = blockIdx.x + int64_t(warp / f.chunks) * G;
    const int64_t g = int64_t(warp % f.chunks) * 32 + lane;
    if (g < f.vecs) v0 = ld_nc_v4(f.x + t * row_bytes + (g << 4));
  }
  __syncthreads();
  const unsigned parity = s_gen & 1u;
  uint32_t* gmask = a.masks + size_t(parity) * a.mask_rows * E;

  // ---- phase 1: one warp per owned token
  for (int i = warp; i < mine; i += kWarps) {
    const int t = int(blockIdx.x) + i * G;
    float w;
    bool nonfinite;
    const int e = route_row<VPL, VEC, true>(a.logits + int64_t(t) * E, E, K, lane, &w, &nonfinite);
    if (lane < K) {
      s_pick[i * K + lane] = e;
      a.topk_idx[int64_t(t) * K + lane] = e;
      a.topk_w[int64_t(t) * K + lane] = w;
      atomicOr(&gmask[(t / kRouteTokens) * E + e], 1u << (t % kRouteTokens));
    }
    if (nonfinite && lane == 0) set_status(a.ws, MOE_ERR_NONFINITE);
  }

  if (!grid_barrier(a.ws, G, gen)) return;

  // ---- phase 2, in every block: masks, totals, offsets and the base table
  int tot = 0;
  if (tid < E) {
    // eight rows' loads in flight at a time
    for (int b0 = 0; b0 < B; b0 += 8) {
      uint32_t m[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m[i] = b0 + i < B ? __ldcg(gmask + (b0 + i) * E + tid) : 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (b0 + i < B) {
          s_mask[(b0 + i) * E + tid] = m[i];
          tot += __popc(m[i]);
        }
    }
  }
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
      run += __popc(s_mask[b * E + tid]);
    }
    if (blockIdx.x == 0) {
      a.counts[tid] = tot;
      a.expert_off[tid] = off;
    }
  }
  if (blockIdx.x == 0) {
    uint32_t* next = a.masks + size_t(parity ^ 1u) * a.mask_rows * E;
    for (int i = tid; i < a.mask_rows * E; i += kRouteThreads) next[i] = 0u;
    if (tid == 0) a.expert_off[E] = a.R * a.region_rows;
  }
  __syncthreads();

  // ---- phase 3: the chunks of this block's tokens to their k slots
  for (int it = warp; it < items; it += kWarps) {
    const int i = it / f.chunks, c = it % f.chunks;
    const int t = int(blockIdx.x) + i * G;
    const int64_t g = int64_t(c) * 32 + lane;
    uint4 v = v0;
    if (it != warp && g < f.vecs) v = ld_nc_v4(f.x + int64_t(t) * row_bytes + (g << 4));
    int slot = -1;
    if (lane < K) {
      const int e = s_pick[i * K + lane];
      if (e >= 0 && e < E) {
        const int b = t / kRouteTokens, tl = t % kRouteTokens;
        slot = s_base[b * E + e] + __popc(s_mask[b * E + e] & ((1u << tl) - 1u));
        if (slot < 0 || slot >= f.total) slot = -1;
      }
      if (slot < 0) set_status(a.ws, MOE_ERR_DEVICE_INDEX);
      if (c == 0) {
        const int64_t tk = int64_t(t) * K + lane;
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
        const int si = i0 + lane;
        const float sv = si < f.S ? __ldcs(f.x_scale + int64_t(t) * f.S + si) : 0.f;
        for (int j = 0; j < K; ++j) {
          const int s = __shfl_sync(kFull, slot, j);
          if (s >= 0 && si < f.S) __stcs(f.recv_scale + int64_t(s) * f.S + si, sv);
        }
      }
    }
  }
  grid_dependents_launch();
}

// Dynamic shared memory of a launch: masks and bases [blocks, E] and the
// owned tokens' picks [owned, K].
size_t fused_smem(int blocks, int E, int owned, int K) {
  return (2 * size_t(blocks) * E + size_t(owned) * K) * 4;
}

template <int VPL, int VEC>
cudaError_t launch_fused(FusedArgs f, int sms, cudaStream_t st) {
  static std::atomic<int> per_sm[64];  // resident blocks per SM, per device (0 = unknown)
  // largest use: 32 route blocks of 512 experts, and the picks of up to 64
  // owned tokens of top-k 32 (1024 tokens need a grid of at least 16 blocks)
  constexpr int kMaxOwned = 64;
  const int kMaxDyn = int(fused_smem(kFusedMaxBlocks, kMaxExperts, kMaxOwned, kMaxTopK));
  auto kernel = route_dispatch_kernel<VPL, VEC>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  e = set_smem_limit(reinterpret_cast<const void*>(kernel), kMaxDyn);
  if (e != cudaSuccess) return e;
  int nb_known = per_sm[dev].load(std::memory_order_relaxed);
  if (nb_known == 0) {
    int nb = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, kRouteThreads, kMaxDyn);
    if (e != cudaSuccess) return e;
    if (nb < 1) return cudaErrorInvalidConfiguration;
    per_sm[dev].store(nb, std::memory_order_relaxed);
    nb_known = nb;
  }
  // one block per token up to the resident limit
  int64_t grid = f.r.n > 1 ? f.r.n : 1;
  if (grid > int64_t(nb_known) * sms) grid = int64_t(nb_known) * sms;
  f.owned = int32_t((int64_t(f.r.n) + grid - 1) / grid);
  if (f.owned > kMaxOwned) return cudaErrorNotSupported;
  return launch_cooperative(kernel, dim3(unsigned(grid)), dim3(kRouteThreads),
                            fused_smem(f.r.blocks, f.r.E, f.owned, f.r.K), st, f);
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
  a.blk = nullptr;
  a.bases = nullptr;
  a.rank = nullptr;
  a.totals = nullptr;
  a.masks = reinterpret_cast<uint32_t*>(w + p.lay.masks);
  a.mask_rows = mask_rows(p);
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
  f.owned = 0;
  if (a.blocks > a.mask_rows) return cudaErrorInvalidValue;
  const int sms = num_sms();
  return with_route_shape(a.E, [&](auto vpl, auto vec) {
    return launch_fused<decltype(vpl)::value, decltype(vec)::value>(f, sms, st);
  });
}

}  // namespace moe
