// Per-token routing shared by the route kernel and the fused small-batch
// route + dispatch kernel: top-k on order-preserving integer keys and the
// softmax over the k winners, one warp per token.
#pragma once

#include "moe_internal.cuh"

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
  uint8_t* rank;   // [n, k]: rank of (t, j) among the block's tokens picking e
  int32_t* totals; // [2, E] per-expert totals, alternate halves per call (route kernel)
  uint32_t* masks; // [2, mask_rows, E] token masks of the fused kernel (null: none)
  int32_t mask_rows;
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

// The logits of one row as order-preserving keys, in the lane layout of
// expert_of.  kStream loads the row as read-once data; otherwise it stays
// cached for other blocks reading it too.
template <int VPL, int VEC, bool kStream>
__device__ __forceinline__ void load_keys(const float* row, int E, int lane,
                                          uint32_t (&key)[VPL]) {
  if constexpr (VEC == 4) {
#pragma unroll
    for (int q4 = 0; q4 < VPL / 4; ++q4) {
      const float4* p = reinterpret_cast<const float4*>(row + q4 * 128) + lane;
      const float4 v = kStream ? __ldcs(p) : __ldg(p);
      key[4 * q4 + 0] = order_key(v.x);
      key[4 * q4 + 1] = order_key(v.y);
      key[4 * q4 + 2] = order_key(v.z);
      key[4 * q4 + 3] = order_key(v.w);
    }
  } else {
#pragma unroll
    for (int q = 0; q < VPL; ++q) {
      const int e = expert_of<VEC>(q, lane);
      key[q] = e < E ? order_key(kStream ? __ldcs(row + e) : __ldg(row + e)) : 0u;
    }
  }
}

// Top-k and softmax of one row's keys by the calling warp: lane j < K gets
// pick j and its weight; *nonfinite tells whether a pick had a non-finite
// logit (fewer than K finite values in the row).
template <int VPL, int VEC>
__device__ __forceinline__ int select_topk(const uint32_t (&key)[VPL], int K, int lane, float* w,
                                           bool* nonfinite) {
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
  *w = ex / s;
  *nonfinite = __any_sync(kFull, lane < K && my_key == 1u);
  return my_i;
}

// Top-k and softmax of one logit row by the calling warp (load_keys, then
// select_topk).
template <int VPL, int VEC, bool kStream>
__device__ __forceinline__ int route_row(const float* row, int E, int K, int lane, float* w,
                                         bool* nonfinite) {
  uint32_t key[VPL];
  load_keys<VPL, VEC, kStream>(row, E, lane, key);
  return select_topk<VPL, VEC>(key, K, lane, w, nonfinite);
}

// Calls f(VPL, VEC) -- as std::integral_constant values -- with the logits
// per lane and load width that fit E experts: float4 loads when E is a
// multiple of 128, scalar loads otherwise.
template <typename F>
cudaError_t with_route_shape(int E, F&& f) {
  using std::integral_constant;
  if (E % 128 == 0) {
    if (E == 128) return f(integral_constant<int, 4>{}, integral_constant<int, 4>{});
    if (E == 256) return f(integral_constant<int, 8>{}, integral_constant<int, 4>{});
    if (E == 384) return f(integral_constant<int, 12>{}, integral_constant<int, 4>{});
    return f(integral_constant<int, 16>{}, integral_constant<int, 4>{});
  }
  const int vpl = (E + 31) / 32;
  if (vpl <= 1) return f(integral_constant<int, 1>{}, integral_constant<int, 1>{});
  if (vpl <= 2) return f(integral_constant<int, 2>{}, integral_constant<int, 1>{});
  if (vpl <= 4) return f(integral_constant<int, 4>{}, integral_constant<int, 1>{});
  if (vpl <= 8) return f(integral_constant<int, 8>{}, integral_constant<int, 1>{});
  return f(integral_constant<int, 16>{}, integral_constant<int, 1>{});
}

}  // namespace
}  // namespace moe
