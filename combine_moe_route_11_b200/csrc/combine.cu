// Combine and the FP8 identity expert.
//
// Combine is the weighted gather-sum of the k expert outputs of every token
// back into token order (combine_gather_remote + combine_weighted_sum in "MLX
// expert parallelism all_to_all PR 3158", Facts):
//     out[t, c] = sum_{j<k} w[t, j] * Y[slot_of[t, j], c],
// accumulated in fp32 with fused multiply-adds in increasing j and rounded to
// nearest even once.  The k row reads are independent 16-byte loads that the
// load/store units keep in flight together; high occupancy, not a shared-
// memory staging ring, is what saturates HBM on this read-dominated gather
// (a bulk-copy staged version measured about two thirds of this one's rate).
//
// The identity expert on FP8 rows turns every filled slot of recv into
// Y = bf16(code * block scale), rounded to nearest even from the exact product.
#include "moe_internal.cuh"

#include <cuda_fp16.h>
#include <cuda_fp8.h>

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// combine: warp per (token, 512-byte column chunk of Y), 4 CTAs of 8 warps per SM
constexpr int kCThreads = 256;
constexpr int kCWarps = kCThreads / 32;
constexpr int kJB = 8;  // expert rows whose loads are in flight together

struct CombineArgs {
  const uint8_t* y;
  const float* w;
  const int32_t* slot_of;
  uint8_t* out;
  void* ws;
  int32_t n, K;
  int32_t total;        // T
  int64_t y_row_bytes;  // D * sizeof(TY)
  int64_t o_row_bytes;  // D * sizeof(TO)
  int32_t groups;       // 16-byte groups of a Y row
  int32_t chunks;       // ceil(groups / 32)
};

// Widen a 16-byte group of Y to fp32.
template <typename TY> struct Group;
template <> struct Group<float> {
  static constexpr int kElems = 4;
  __device__ static void widen(const uint4& v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
};
template <> struct Group<__nv_bfloat16> {
  static constexpr int kElems = 8;
  __device__ static void widen(const uint4& v, float (&f)[8]) {
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
  }
};

template <typename TO, int NE>
__device__ __forceinline__ void store_out(uint8_t* dst, const float (&acc)[NE]) {
  if constexpr (sizeof(TO) == 4) {
#pragma unroll
    for (int i = 0; i < NE; i += 4)
      *reinterpret_cast<uint4*>(dst + i * 4) =
          make_uint4(__float_as_uint(acc[i]), __float_as_uint(acc[i + 1]),
                     __float_as_uint(acc[i + 2]), __float_as_uint(acc[i + 3]));
  } else if constexpr (NE == 8) {
    *reinterpret_cast<uint4*>(dst) =
        make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                   pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  } else {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
  }
}

// Work item = (token, chunk of 32 sixteen-byte groups).  Lane j < k holds the
// slot and weight of choice j; every lane owns one group of the chunk, issues
// the loads of up to kJB expert rows together (read-once, not kept in L1) and
// accumulates them in increasing j with fused multiply-adds.  The kernel is
// limited to 64 registers so 32 warps per SM keep ~128 KB of loads in flight.
template <typename TY, typename TO>
__global__ void __launch_bounds__(kCThreads, 4) combine_kernel(CombineArgs a) {
  constexpr int NE = Group<TY>::kElems;
  const int lane = threadIdx.x & 31;
  const int64_t n_items = int64_t(a.n) * a.chunks;
  const int64_t stride = int64_t(gridDim.x) * kCWarps;
  grid_dependency_wait();
  // Every CTA that runs this line has started, so once all have, the next
  // kernel in the stream may be scheduled into the SM room this grid leaves
  // (it waits for this grid to finish before it reads anything).
  grid_dependents_launch();
  for (int64_t item = int64_t(blockIdx.x) * kCWarps + (threadIdx.x >> 5); item < n_items;
       item += stride) {
    const int64_t t = item / a.chunks;
    const int g = int(item % a.chunks) * 32 + lane;
    int slot = 0;
    float wt = 0.f;
    bool ok = true;
    if (lane < a.K) {
      slot = __ldg(a.slot_of + t * a.K + lane);
      wt = __ldg(a.w + t * a.K + lane);
      ok = slot >= 0 && slot < a.total;
    }
    if (!__all_sync(0xFFFFFFFFu, ok)) {
      if (lane == 0) set_status(a.ws, MOE_ERR_DEVICE_INDEX);
      continue;
    }
    const bool mine = g < a.groups;
    float acc[NE];
#pragma unroll
    for (int i = 0; i < NE; ++i) acc[i] = 0.f;
    for (int jb = 0; jb < a.K; jb += kJB) {
      uint4 v[kJB];
#pragma unroll
      for (int u = 0; u < kJB; ++u) {
        const int s = __shfl_sync(0xFFFFFFFFu, slot, (jb + u) & 31);
        if (jb + u < a.K && mine) v[u] = ld_nc_v4(a.y + int64_t(s) * a.y_row_bytes + int64_t(g) * 16);
      }
#pragma unroll
      for (int u = 0; u < kJB; ++u) {
        const float wj = __shfl_sync(0xFFFFFFFFu, wt, (jb + u) & 31);
        if (jb + u < a.K) {
          float f[NE];
          Group<TY>::widen(v[u], f);
#pragma unroll
          for (int i = 0; i < NE; ++i) acc[i] = __fmaf_rn(wj, f[i], acc[i]);
        }
      }
    }
    if (mine) store_out<TO, NE>(a.out + t * a.o_row_bytes + int64_t(g) * NE * sizeof(TO), acc);
  }
}

template <typename TY, typename TO>
cudaError_t launch_combine_k(const CombineArgs& a, dim3 grid, cudaStream_t st) {
  return launch_pdl(combine_kernel<TY, TO>, grid, dim3(kCThreads), 0, st, a);
}

// ------------------------------------------------------------------ FP8 identity expert

struct DequantArgs {
  const uint8_t* q;       // recv, e4m3 [T, D]
  const float* scale;     // recv_scale [T, S] or null
  const int32_t* slot_of;
  uint8_t* y;             // bf16 [T, D]
  void* ws;
  int32_t n, K, D, S, block;
  int32_t total;
  int32_t chunks, chunk_groups;  // groups of 16 codes
};

// bf16 bits of code * scale rounded to nearest even from the exact product.
// p = fl32(q*s) can land exactly on a bf16 rounding midpoint while the exact
// product lies just off it; the fma residual tells which side, and moving p
// one fp32 ulp toward it lets the final rounding see the true side (p never
// crosses the midpoint itself, which is an fp32 number).
__device__ __forceinline__ uint32_t mul_to_bf16_exact(float q, float s) {
  const float p = __fmul_rn(q, s);
  const float r = __fmaf_rn(q, s, -p);
  uint32_t b = __float_as_uint(p);
  if ((b & 0xFFFFu) == 0x8000u && r != 0.f) b = ((r > 0.f) == (p > 0.f)) ? b + 1u : b - 1u;
  __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(b));
  return *reinterpret_cast<uint16_t*>(&h);
}

__global__ void __launch_bounds__(kThreads) dequant_kernel(DequantArgs a) {
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int groups = a.D / 16;
  const int64_t n_items = int64_t(a.n) * a.K * a.chunks;
  grid_dependency_wait();
  const int64_t stride = int64_t(gridDim.x) * kWarps;
  for (int64_t item = int64_t(blockIdx.x) * kWarps + wib; item < n_items; item += stride) {
    const int64_t tk = item / a.chunks;
    const int c = int(item % a.chunks);
    const int s = a.slot_of[tk];
    if (s < 0 || s >= a.total) {
      if (lane == 0) set_status(a.ws, MOE_ERR_DEVICE_INDEX);
      continue;
    }
    const uint8_t* qrow = a.q + int64_t(s) * a.D;
    uint8_t* yrow = a.y + int64_t(s) * a.D * 2;
    const int g1 = min((c + 1) * a.chunk_groups, groups);
    for (int g = c * a.chunk_groups + lane; g < g1; g += 32) {
      const uint4 v = ld_nc_v4(qrow + int64_t(g) * 16);
      const float sc = a.scale ? __ldg(a.scale + int64_t(s) * a.S + (g * 16) / a.block) : 1.f;
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      float f[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const __nv_fp8x2_storage_t pair = __nv_fp8x2_storage_t((w4[i] >> (16 * h)) & 0xFFFFu);
          const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
          const float2 ff = __half22float2(*reinterpret_cast<const __half2*>(&hr));
          f[i * 4 + h * 2] = ff.x;
          f[i * 4 + h * 2 + 1] = ff.y;
        }
      }
      uint32_t o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        o[i] = mul_to_bf16_exact(f[2 * i], sc) | (mul_to_bf16_exact(f[2 * i + 1], sc) << 16);
      uint4* dst = reinterpret_cast<uint4*>(yrow + int64_t(g) * 32);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
  }
}

// (token, chunk) items so that small N still fills the GPU.
void pick_chunks(int64_t rows, int64_t groups, int sms, int32_t* chunks, int32_t* chunk_groups) {
  const int64_t target = int64_t(sms) * 32;
  int64_t ch = rows > 0 ? (target + rows - 1) / rows : 1;
  const int64_t max_ch = (groups + 31) / 32;
  ch = ch < 1 ? 1 : (ch > max_ch ? max_ch : ch);
  int64_t cg = (groups + ch - 1) / ch;
  cg = (cg + 31) / 32 * 32;
  *chunk_groups = int32_t(cg);
  *chunks = int32_t((groups + cg - 1) / cg);
}

dim3 item_grid(int64_t items, int sms) {
  int64_t g = (items + kWarps - 1) / kWarps;
  const int64_t cap = int64_t(sms) * 8;
  return dim3(unsigned(g < 1 ? 1 : (g > cap ? cap : g)));
}

}  // namespace

cudaError_t launch_combine(const moe_plan& p, int32_t n, const void* y, const float* topk_w,
                           const int32_t* slot_of, void* out, void* ws, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  CombineArgs a;
  a.y = static_cast<const uint8_t*>(y);
  a.w = topk_w;
  a.slot_of = slot_of;
  a.out = static_cast<uint8_t*>(out);
  a.ws = ws;
  a.n = n;
  a.K = p.d.top_k;
  a.total = int32_t(total_rows(p, n));
  a.y_row_bytes = int64_t(p.d.hidden) * elem_bytes(p.d.y_dtype);
  a.o_row_bytes = int64_t(p.d.hidden) * elem_bytes(p.d.out_dtype);
  a.groups = int32_t(a.y_row_bytes / 16);
  a.chunks = (a.groups + 31) / 32;
  const int sms = num_sms();
  int64_t grid = (int64_t(n) * a.chunks + kCWarps - 1) / kCWarps;
  const int64_t cap = int64_t(sms) * 4;
  if (grid > cap) grid = cap;
  const dim3 g(unsigned(grid < 1 ? 1 : grid));
  const bool yb = p.d.y_dtype == MOE_BF16, ob = p.d.out_dtype == MOE_BF16;
  if (yb && ob) return launch_combine_k<__nv_bfloat16, __nv_bfloat16>(a, g, st);
  if (yb) return launch_combine_k<__nv_bfloat16, float>(a, g, st);
  if (ob) return launch_combine_k<float, __nv_bfloat16>(a, g, st);
  return launch_combine_k<float, float>(a, g, st);
}

cudaError_t launch_dequant(const moe_plan& p, int32_t n, const void* recv, const float* recv_scale,
                           const int32_t* slot_of, void* y, void* ws, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  DequantArgs a;
  a.q = static_cast<const uint8_t*>(recv);
  a.scale = recv_scale;
  a.slot_of = slot_of;
  a.y = static_cast<uint8_t*>(y);
  a.ws = ws;
  a.n = n;
  a.K = p.d.top_k;
  a.D = p.d.hidden;
  a.S = p.scale_cols;
  a.block = p.d.scale_block > 0 ? p.d.scale_block : p.d.hidden;
  a.total = int32_t(total_rows(p, n));
  const int sms = num_sms();
  pick_chunks(int64_t(n) * a.K, a.D / 16, sms, &a.chunks, &a.chunk_groups);
  const dim3 grid = item_grid(int64_t(n) * a.K * a.chunks, sms);
  return launch_pdl(dequant_kernel, grid, dim3(kThreads), 0, st, a);
}

}  // namespace moe
