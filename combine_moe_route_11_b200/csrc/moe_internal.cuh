// Internal declarations shared by the CUDA translation units of libmoeroute.
// Nothing here is part of the C ABI (include/moeroute.h is).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "moeroute.h"

namespace moe {

// Tokens per route block.  One block's tokens form two 32-token groups whose
// membership masks give each (token, expert) pair its rank inside the block.
constexpr int kRouteTokens = 64;
constexpr int kRouteThreads = 256;
constexpr int kMaxExperts = 512;
constexpr int kMaxTopK = 32;

// Control words at the start of every workspace.
struct Ctrl {
  unsigned int ticket;  // route blocks finished so far (reset by the last one)
  int status;           // first device-detected error, 0 = none
  unsigned int pad[62];
};
static_assert(sizeof(Ctrl) == 256, "control block is 256 bytes");

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline int elem_bytes(int dtype) {
  return dtype == MOE_F32 ? 4 : dtype == MOE_BF16 ? 2 : 1;
}

// Byte offsets of every buffer inside a workspace, fixed by n_max.
struct Layout {
  size_t ctrl, blk, rank, route_end;
  size_t topk_idx, topk_w, counts, expert_off, slot_of, src_of, recv, recv_scale, y, h, end;
};

}  // namespace moe

struct moe_plan {
  moe_desc d;
  int32_t scale_cols;   // D / scale_block, 0 without scales
  int32_t blocks_max;   // route blocks for n_max
  int64_t total_max;    // T(n_max)
  moe::Layout lay;
};

namespace moe {

inline int64_t region_rows(const moe_plan& p, int32_t n) {
  int per_rank = p.d.n_experts / p.d.n_ranks;
  return int64_t(n) * (p.d.top_k < per_rank ? p.d.top_k : per_rank);
}
inline int64_t total_rows(const moe_plan& p, int32_t n) { return region_rows(p, n) * p.d.n_ranks; }
inline int route_blocks(int32_t n) { return n <= 0 ? 1 : (n + kRouteTokens - 1) / kRouteTokens; }

int num_sms();  // of the current device (cached per device)

// Launchers (return cudaGetLastError()).
cudaError_t launch_route(const moe_plan& p, int32_t n, const float* logits, int32_t* topk_idx,
                         float* topk_w, int32_t* counts, int32_t* expert_off, void* ws,
                         cudaStream_t st);
cudaError_t launch_dispatch(const moe_plan& p, int32_t n, const void* x, const float* x_scale,
                            const int32_t* topk_idx, void* recv, float* recv_scale,
                            int32_t* slot_of, int32_t* src_of, void* ws, cudaStream_t st);
cudaError_t launch_dequant(const moe_plan& p, int32_t n, const void* recv, const float* recv_scale,
                           const int32_t* slot_of, void* y, void* ws, cudaStream_t st);
cudaError_t launch_combine(const moe_plan& p, int32_t n, const void* y, const float* topk_w,
                           const int32_t* slot_of, void* out, void* ws, cudaStream_t st);
cudaError_t launch_swiglu(const moe_plan& p, int32_t n, const void* recv, const int32_t* counts,
                          const int32_t* expert_off, const void* w_gate_up, const void* w_down,
                          void* h, void* y, void* ws, cudaStream_t st);

// ------------------------------------------------------------------ device helpers
#ifdef __CUDACC__

__device__ __forceinline__ void set_status(void* ws, int code) {
  Ctrl* c = reinterpret_cast<Ctrl*>(ws);
  atomicCAS(&c->status, 0, code);
}

// 16-byte global load through the non-coherent path, not kept in L1.
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

// 16-byte global store marked evict-first (streaming).
__device__ __forceinline__ void st_cs_v4(void* p, const uint4& v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

#endif  // __CUDACC__

}  // namespace moe
