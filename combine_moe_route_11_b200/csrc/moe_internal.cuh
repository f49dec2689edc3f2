// Internal declarations shared by the CUDA translation units of libmoeroute.
// Nothing here is part of the C ABI (include/moeroute.h is).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "moeroute.h"

namespace moe {

// Tokens per route block: one warp per token, and the block's 32 tokens form
// the membership masks that give each (token, expert) pair its in-block rank.
constexpr int kRouteTokens = 32;
constexpr int kRouteThreads = 1024;
constexpr int kMaxExperts = 512;
constexpr int kMaxTopK = 32;
// Largest batch, in route blocks, that the fused route + dispatch launch
// takes (n <= 1024 tokens); larger batches run the two kernels.
constexpr int kFusedMaxBlocks = 32;

// Control words at the start of every workspace.
struct Ctrl {
  unsigned int arrive;    // fused kernel's grid barrier: blocks arrived (reset by the last one)
  int status;             // first device-detected error, 0 = none
  unsigned int gen;       // fused kernel's grid barrier: generation, bumped when all arrived
  unsigned int ticket;    // route kernel: CTAs arrived, calls of even generation
  unsigned int rgen;      // route kernel: calls completed; selects counter and totals half
  unsigned int tile_next; // grouped GEMMs: next tile to hand out (reset by the last CTA)
  unsigned int tile_done; // grouped GEMMs: CTAs finished (reset by the last one)
  unsigned int ticket_b;  // route kernel: CTAs arrived, calls of odd generation
  unsigned int pad[56];
};
static_assert(sizeof(Ctrl) == 256, "control block is 256 bytes");

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline int elem_bytes(int dtype) {
  return dtype == MOE_F32 ? 4 : dtype == MOE_BF16 ? 2 : 1;
}

// Byte offsets of every buffer inside a workspace, fixed by n_max.
struct Layout {
  size_t ctrl, masks, totals, blk, bases, rank, route_end;  // [ctrl, blk) is cleared by moe_workspace_init
  size_t topk_idx, topk_w, counts, expert_off, slot_of, src_of, recv, recv_scale, y, h;
  size_t hq, h_scale;  // FP8 SwiGLU experts: H in e4m3 and its per-128-column scales
  size_t end;
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
// Rows of each half of the fused kernel's [2, rows, E] token-mask table.
inline int mask_rows(const moe_plan& p) {
  return p.blocks_max < kFusedMaxBlocks ? p.blocks_max : kFusedMaxBlocks;
}

int num_sms();  // of the current device (cached per device)
// Raise a kernel's dynamic shared-memory limit once per device.
cudaError_t set_smem_limit(const void* kernel, int bytes);

// Launchers (return cudaGetLastError()).
cudaError_t launch_route(const moe_plan& p, int32_t n, const float* logits, int32_t* topk_idx,
                         float* topk_w, int32_t* counts, int32_t* expert_off, void* ws,
                         cudaStream_t st);
// The route kernel on caller-chosen scratch: ctrl (control words, the
// counter at zero), blk and bases ([route blocks, E] int32 each) and rank
// ([n, k] bytes).
cudaError_t launch_route_on(const moe_plan& p, int32_t n, const float* logits, int32_t* topk_idx,
                            float* topk_w, int32_t* counts, int32_t* expert_off, void* ctrl,
                            int32_t* totals, int32_t* blk, int32_t* bases, uint8_t* rank,
                            cudaStream_t st);
cudaError_t launch_route_counts(const moe_plan& p, int32_t n, int32_t* topk_idx, int32_t* counts,
                                int32_t* expert_off, void* ws, cudaStream_t st);
cudaError_t launch_router(const moe_plan& p, int32_t n, const void* x, const void* w_router,
                          float* logits, int32_t* topk_idx, float* topk_w, void* ws,
                          cudaStream_t st);
cudaError_t launch_dispatch(const moe_plan& p, int32_t n, const void* x, const float* x_scale,
                            const int32_t* topk_idx, void* recv, float* recv_scale,
                            int32_t* slot_of, int32_t* src_of, void* ws, cudaStream_t st);
cudaError_t launch_route_dispatch(const moe_plan& p, int32_t n, const float* logits,
                                  const void* x, const float* x_scale, int32_t* topk_idx,
                                  float* topk_w, int32_t* counts, int32_t* expert_off, void* recv,
                                  float* recv_scale, int32_t* slot_of, int32_t* src_of, void* ws,
                                  cudaStream_t st);
cudaError_t launch_dequant(const moe_plan& p, int32_t n, const void* recv, const float* recv_scale,
                           const int32_t* slot_of, void* y, void* ws, cudaStream_t st);
cudaError_t launch_combine(const moe_plan& p, int32_t n, const void* y, const float* topk_w,
                           const int32_t* slot_of, void* out, void* ws, cudaStream_t st);
cudaError_t launch_swiglu(const moe_plan& p, int32_t n, const void* recv, const int32_t* counts,
                          const int32_t* expert_off, const void* w_gate_up, const void* w_down,
                          void* h, void* y, void* ws, cudaStream_t st);
cudaError_t launch_swiglu_fp8(const moe_plan& p, int32_t n, const void* recv,
                              const float* recv_scale, const int32_t* counts,
                              const int32_t* expert_off, const int32_t* slot_of,
                              const void* w_gate_up, const float* w_gate_up_scale,
                              const void* w_down, const float* w_down_scale, void* h, void* hq,
                              float* h_scale, void* y, void* ws, cudaStream_t st);
// The driver's cuTensorMapEncodeTiled (null if unavailable), looked up once.
void* tensor_map_encoder();

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel of the stream finishes, and must call
// grid_dependency_wait() before its first global-memory access.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Cooperative launch: every block resident, as a grid barrier requires.
// (Adding programmatic stream serialization to it was measured: no gain in
// a CUDA graph, slower eager decode steps.)
template <typename... KArgs, typename... Args>
cudaError_t launch_cooperative(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                               cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ------------------------------------------------------------------ device helpers
#ifdef __CUDACC__

// Wait until the grids this one depends on have completed and their memory
// is visible (a no-op without a programmatic dependency).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Allow the next kernel of the stream to be scheduled (it still waits for
// this grid's completion before touching memory).
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void set_status(void* ws, int code) {
  Ctrl* c = reinterpret_cast<Ctrl*>(ws);
  atomicCAS(&c->status, 0, code);
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed_gpu(unsigned* p, unsigned v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Barrier across all `blocks` blocks of a grid whose blocks are all resident
// (cooperative launch).  `gen` is the generation word as thread 0 read it
// after the grid's dependency wait (no block of this grid can have bumped it
// before this block arrives).  The block barrier orders the block's writes
// before thread 0's release fence and arrival; the last arrival bumps the
// generation, which the others poll with acquire loads.  The wait is bounded
// (~2^31 cycles); on timeout it records MOE_ERR_TIMEOUT and returns false,
// and the workspace must be re-initialised before its next use.
__device__ __forceinline__ bool grid_barrier(void* ws, unsigned blocks, unsigned gen) {
  __shared__ int s_ok;
  Ctrl* c = reinterpret_cast<Ctrl*>(ws);
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = true;
    fence_acq_rel_gpu();
    if (atomicAdd(&c->arrive, 1u) + 1u == blocks) {
      st_relaxed_gpu(&c->arrive, 0u);
      fence_acq_rel_gpu();
      atomicAdd(&c->gen, 1u);
    } else {
      const long long t0 = clock64();
      while (ld_acquire_gpu(&c->gen) == gen) {
        if (clock64() - t0 > (1ll << 31)) {
          ok = false;
          set_status(ws, MOE_ERR_TIMEOUT);
          break;
        }
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
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

// ---- mbarriers (for the tensor-memory-accelerator copies of the grouped GEMM)
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Make mbarrier initialisation visible to the async proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for an mbarrier phase: gives up after ~2^31 SM cycles
// (about a second) and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > (1ll << 31)) return false;
  return true;
}

// ---- dynamic tile scheduling for the persistent grouped GEMMs
// Thread 0 of a CTA (the copy producer) takes tiles one at a time from a
// counter in the workspace's control block, so a CTA that finishes early
// takes more; it hands each index, in order, to the CTA's consumer warps
// through a ring of kTileQ slots in shared memory (one mbarrier pair per
// slot: `full` completes when the slot is written, `empty` when every
// consumer warp has read it).  An index >= the tile count ends the loops.
constexpr int kTileQ = 4;

struct TileQueue {
  int* slot;        // [kTileQ]
  uint64_t* full;   // [kTileQ], one arrival (the producer)
  uint64_t* empty;  // [kTileQ], one arrival per consumer warp
  int i;
  uint32_t phase;
};

__device__ __forceinline__ void tq_init(const TileQueue& q, uint32_t consumer_warps) {
  for (int s = 0; s < kTileQ; ++s) {
    mbar_init(&q.full[s], 1);
    mbar_init(&q.empty[s], consumer_warps);
  }
}

// Producer: publish tile t in the next slot; false if the wait gave up.
__device__ __forceinline__ bool tq_push(TileQueue& q, int t) {
  if (!mbar_wait(&q.empty[q.i], q.phase ^ 1u)) return false;
  q.slot[q.i] = t;
  mbar_arrive(&q.full[q.i]);
  if (++q.i == kTileQ) q.i = 0, q.phase ^= 1u;
  return true;
}

// One lane of a consumer warp: the next tile index, or false if the wait
// gave up.  The slot is released as soon as it has been read.
__device__ __forceinline__ bool tq_pop(TileQueue& q, int* t) {
  if (!mbar_wait(&q.full[q.i], q.phase)) return false;
  *t = q.slot[q.i];
  mbar_arrive(&q.empty[q.i]);
  if (++q.i == kTileQ) q.i = 0, q.phase ^= 1u;
  return true;
}

// The next tile for this CTA (thread 0 only); `total` once all are taken.
__device__ __forceinline__ int tq_take(void* ws, int total) {
  const unsigned t = atomicAdd(&reinterpret_cast<Ctrl*>(ws)->tile_next, 1u);
  return t < unsigned(total) ? int(t) : total;
}

// Thread 0 of every CTA, after its last access to the tile counter: the last
// CTA of the grid to finish resets both counters for the next launch.
__device__ __forceinline__ void tq_finish(void* ws) {
  Ctrl* c = reinterpret_cast<Ctrl*>(ws);
  fence_acq_rel_gpu();
  if (atomicAdd(&c->tile_done, 1u) == gridDim.x - 1) {
    atomicExch(&c->tile_next, 0u);
    atomicExch(&c->tile_done, 0u);
  }
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

#endif  // __CUDACC__

}  // namespace moe
