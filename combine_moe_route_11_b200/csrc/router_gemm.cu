// Router GEMM fused ahead of top-k: logits = x . W_r^T on the tensor cores
// (tcgen05, bf16 operands, fp32 accumulation), then the top-k selection and
// the softmax over the k winners of every row in the same kernel.  The gate
// produces the [N, top_k] expert indices that the sorted gather consumes
// ("backends/mlx: runtime MoE expert-sort for decode", author updates on the
// sorted path); the pages do not spell the gate out, and the reading taken
// is the plain linear map of the token's hidden row.
//
// One 128-token tile of x against all E (<= 256) router rows is a single
// M = 128, N = E MMA chain over K = D.  A tile alone would keep one SM busy
// for the whole reduction, so the reduction is split over the S CTAs of a
// thread-block cluster (S = 1, 2, 4 or 8: as many as keep all clusters of
// the grid resident at once):
// CTA r of the cluster accumulates k-blocks [r*D/S, (r+1)*D/S) in tensor
// memory.  Then
//   1. every CTA copies its 128 x E partial sums from tensor memory into its
//      own shared memory (the drained copy ring);
//   2. cluster barrier;
//   3. CTA r reduces rows [r*128/S, (r+1)*128/S), each of its 12 warps a
//      share of the rows: the warp loads a row's S partials through
//      distributed shared memory together and sums them in cluster-rank
//      order (a fixed order: the logits do not depend on timing), writes the
//      fp32 logits if asked, and runs the route kernel's warp top-k and
//      softmax on them (ties to the lower expert id);
//   4. cluster barrier, so no CTA leaves while a peer still reads its sums.
// Per CTA: warp 0 issues the TMA copies (x box 128 x 64, W_r box E x 64,
// 128-byte swizzle, 4-stage ring), warp 1 owns the tensor memory and issues
// tcgen05.mma (M = 128, N = E rounded up to 16, K = 16), warps 2..5 move the
// accumulators out, and all twelve reduce.  Every wait is bounded; a CTA whose wait
// gave up records MOE_ERR_TIMEOUT, drains its own copies and MMAs and still meets
// its cluster's barriers.
#include "route_common.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <type_traits>

namespace moe {
namespace {

constexpr int kRBM = 128;                 // tokens per tile (UMMA M)
constexpr int kRBK = 64;                  // reduction step: one 128-byte swizzle row of bf16
constexpr int kRUmmaK = 16;
constexpr int kRStages = 4;
constexpr int kRThreads = 384;          // 12 warps
constexpr int kRWarps = kRThreads / 32;
constexpr int kRMaxN = 256;               // experts per MMA (UMMA N)
constexpr int kRMaxSplit = 8;             // portable cluster size
constexpr uint32_t kRABytes = kRBM * kRBK * 2;
constexpr uint32_t kRStageBytes = kRABytes + kRMaxN * kRBK * 2;
constexpr int kPitch = kRMaxN + 4;        // floats per row of the partial sums in shared memory
constexpr size_t kRSmem = size_t(kRStages) * kRStageBytes + 1024 /*align*/ + 256 /*meta*/;
static_assert(size_t(kRBM) * kPitch * 4 <= size_t(kRStages) * kRStageBytes,
              "the partial sums fit in the drained copy ring");

struct RouterArgs {
  float* logits;      // [n, E] fp32, or null
  int32_t* topk_idx;  // [n, K]
  float* topk_w;      // [n, K]
  void* ws;
  int32_t n, E, K;
  int32_t n_mma;      // E rounded up to 16
  int32_t tmem_cols;  // power of two >= max(32, n_mma)
  int32_t k_steps;    // k-blocks per CTA of a cluster (D / 64 / split)
  int32_t split;      // CTAs per cluster
};

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  // K-major operand, 128-byte swizzle, 8-row groups 1024 bytes apart
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// kind::f16 instruction descriptor: bf16 A and B (K-major), fp32 D, M = 128, N = n.
__device__ __forceinline__ uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(kRBM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tcgen_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tcgen_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tma_2d(void* dst, const CUtensorMap* map, int x, int y,
                                       uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// 16 consecutive fp32 accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Every thread of every CTA of the cluster: release this CTA's shared-memory
// writes, then wait for the others.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}

// The shared::cluster address of `saddr` (a shared::cta address) in CTA `rank`.
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

__device__ __forceinline__ float ld_dsmem(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ float4 ld_dsmem4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

template <int VPL, int VEC>
__global__ void __launch_bounds__(kRThreads, 1)
    router_gemm_kernel(const __grid_constant__ CUtensorMap tma_x,
                       const __grid_constant__ CUtensorMap tma_w, RouterArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* meta = smem + size_t(kRStages) * kRStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(meta);
  uint64_t* empty = full + kRStages;
  uint64_t* acc_full = empty + kRStages;
  uint64_t* drained = acc_full + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drained + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  float* part = reinterpret_cast<float*>(smem);  // [128][kPitch] partial sums, after the loop

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int S = g.split;
  const int m_tile = int(blockIdx.x) / S;
  const int kb0 = int(rank) * g.k_steps;
  const uint32_t b_bytes = uint32_t(g.n_mma) * kRBK * 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drained, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  grid_dependency_wait();
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(s_tmem)),
                 "r"(g.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tcgen_fence_before();
  __syncthreads();
  tcgen_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int kb = 0; kb < g.k_steps; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u)) {
          set_status(g.ws, MOE_ERR_TIMEOUT);
          *s_abort = 1;
          break;
        }
        uint8_t* a_dst = smem + size_t(stage) * kRStageBytes;
        mbar_arrive_expect_tx(&full[stage], kRABytes + b_bytes);
        tma_2d(a_dst, &tma_x, (kb0 + kb) * kRBK, m_tile * kRBM, &full[stage]);
        tma_2d(a_dst + kRABytes, &tma_w, (kb0 + kb) * kRBK, 0, &full[stage]);
        ++issued;
        if (++stage == kRStages) stage = 0, phase ^= 1u;
      }
      // never leave a copy in flight into this CTA's shared memory: the last
      // min(issued, stages) copies are the only ones nobody may have waited for
      for (int i = issued - kRStages; i < issued; ++i) {
        if (i < 0) continue;
        if (!mbar_wait(&full[i % kRStages], uint32_t(i / kRStages) & 1u))
          set_status(g.ws, MOE_ERR_TIMEOUT);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t idesc = idesc_bf16(g.n_mma);
      for (int kb = 0; kb < g.k_steps && !*s_abort; ++kb) {
        if (!mbar_wait(&full[stage], phase)) {
          set_status(g.ws, MOE_ERR_TIMEOUT);
          *s_abort = 1;
          break;
        }
        tcgen_fence_after();
        const uint32_t a_addr = smem_addr(smem + size_t(stage) * kRStageBytes);
        const uint32_t b_addr = a_addr + kRABytes;
#pragma unroll
        for (int k = 0; k < kRBK / kRUmmaK; ++k)
          mma_bf16(tmem_base, desc_sw128(a_addr + k * kRUmmaK * 2),
                   desc_sw128(b_addr + k * kRUmmaK * 2), idesc, (kb | k) != 0 ? 1u : 0u);
        mma_commit(&empty[stage]);
        if (++stage == kRStages) stage = 0, phase ^= 1u;
      }
      mma_commit(acc_full);  // all MMAs issued above are complete when this arrives
      if (!mbar_wait(acc_full, 0)) set_status(g.ws, MOE_ERR_TIMEOUT);
      mma_commit(drained);
      if (!mbar_wait(drained, 0)) set_status(g.ws, MOE_ERR_TIMEOUT);
    }
  }
  // every copy has landed and every MMA has completed (or the CTA aborted)
  tcgen_fence_before();
  __syncthreads();
  tcgen_fence_after();
  // ---- 1. partial sums: tensor memory -> own shared memory
  if (warp >= 2) {
    const int quarter = warp & 3;  // TMEM lanes this warp may read
    const int row = quarter * 32 + lane;
    const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16);
    for (int c = 0; c < g.n_mma; c += 16) {
      float v[16];
      tmem_ld16(taddr + uint32_t(c), v);
      float4* dst = reinterpret_cast<float4*>(part + row * kPitch + c);
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
  }
  tcgen_fence_before();
  // ---- 2. every CTA's partial sums are in place
  cluster_sync();
  // ---- 3. rows [rank * 128/S, (rank + 1) * 128/S): one warp per row
  if (!*s_abort) {
    const int rows = kRBM / S;
    const uint32_t part_addr = smem_addr(part);
    for (int rl = warp; rl < rows; rl += kRWarps) {
      const int r = int(rank) * rows + rl;
      const int64_t t = int64_t(m_tile) * kRBM + r;
      if (t >= g.n) break;
      // the S partials of this row, loaded together, summed in rank order
      float v[VPL];
#pragma unroll
      for (int q = 0; q < VPL; ++q) v[q] = 0.f;
      if constexpr (VEC == 4) {
        float4 f[kRMaxSplit][VPL / 4];
#pragma unroll
        for (int p = 0; p < kRMaxSplit; ++p) {
          if (p < S) {
            const uint32_t base = map_rank(part_addr, uint32_t(p)) + uint32_t(r * kPitch) * 4u;
#pragma unroll
            for (int q4 = 0; q4 < VPL / 4; ++q4)
              f[p][q4] = ld_dsmem4(base + uint32_t(q4 * 128 + lane * 4) * 4u);
          }
        }
#pragma unroll
        for (int p = 0; p < kRMaxSplit; ++p) {
          if (p < S) {
#pragma unroll
            for (int q4 = 0; q4 < VPL / 4; ++q4) {
              v[4 * q4 + 0] += f[p][q4].x;
              v[4 * q4 + 1] += f[p][q4].y;
              v[4 * q4 + 2] += f[p][q4].z;
              v[4 * q4 + 3] += f[p][q4].w;
            }
          }
        }
      } else {
        float f[kRMaxSplit][VPL];
#pragma unroll
        for (int p = 0; p < kRMaxSplit; ++p) {
          if (p < S) {
            const uint32_t base = map_rank(part_addr, uint32_t(p)) + uint32_t(r * kPitch) * 4u;
#pragma unroll
            for (int q = 0; q < VPL; ++q) {
              const int e = expert_of<VEC>(q, lane);
              f[p][q] = e < g.E ? ld_dsmem(base + uint32_t(e) * 4u) : 0.f;
            }
          }
        }
#pragma unroll
        for (int p = 0; p < kRMaxSplit; ++p)
          if (p < S)
#pragma unroll
            for (int q = 0; q < VPL; ++q) v[q] += f[p][q];
      }
      uint32_t key[VPL];
#pragma unroll
      for (int q = 0; q < VPL; ++q) {
        const int e = expert_of<VEC>(q, lane);
        key[q] = e < g.E ? order_key(v[q]) : 0u;
        if (g.logits && e < g.E) g.logits[t * g.E + e] = v[q];
      }
      float w;
      bool nonfinite;
      const int e = select_topk<VPL, VEC>(key, g.K, lane, &w, &nonfinite);
      if (lane < g.K) {
        g.topk_idx[t * g.K + lane] = e;
        g.topk_w[t * g.K + lane] = w;
      }
      if (nonfinite && lane == 0) set_status(g.ws, MOE_ERR_NONFINITE);
    }
  }
  // ---- 4. peers may read this CTA's partial sums until here
  cluster_sync();
  tcgen_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(g.tmem_cols)
                 : "memory");
  grid_dependents_launch();
}

// 2D bf16 tensor map over a row-major [rows, cols] matrix; box = 64 columns
// (the 128-byte swizzle width) x box_rows rows, zero fill outside.
bool router_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                uint32_t box_rows) {
  auto fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {uint32_t(kRBK), box_rows};
  const cuuint32_t elem[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Clusters of `split` CTAs of this kernel that can be resident at once.
int max_active_clusters(const void* kernel, int split) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(split));
  cfg.blockDim = dim3(kRThreads);
  cfg.dynamicSmemBytes = kRSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = unsigned(split);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) return 0;
  return n;
}

template <int VPL, int VEC>
cudaError_t launch_router_k(const CUtensorMap& mx, const CUtensorMap& mw, RouterArgs g,
                            int m_tiles, int k_total, int sms, cudaStream_t st) {
  auto kernel = router_gemm_kernel<VPL, VEC>;
  cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(kernel), int(kRSmem));
  if (e != cudaSuccess) return e;
  // Split the reduction over as many CTAs per cluster as keep every cluster
  // of the grid resident at once (a second wave of clusters would double the
  // time), up to 8.
  static std::atomic<int> fits[64][4];  // per device and split 1,2,4,8: resident clusters (0 = unknown)
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  int split = 1;
  for (int lg = 1; lg < 4; ++lg) {
    const int s = 1 << lg;
    if (m_tiles * s > sms || k_total % s != 0) break;
    int c = fits[dev][lg].load(std::memory_order_relaxed);
    if (c == 0) {
      c = max_active_clusters(reinterpret_cast<const void*>(kernel), s);
      if (c <= 0) break;
      fits[dev][lg].store(c, std::memory_order_relaxed);
    }
    if (c < m_tiles) break;
    split = s;
  }
  g.split = split;
  g.k_steps = k_total / split;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(m_tiles * g.split));
  cfg.blockDim = dim3(kRThreads);
  cfg.dynamicSmemBytes = kRSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = unsigned(g.split);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, mx, mw, g);
}

// with_route_shape restricted to the E <= 256 experts of one MMA.
template <typename F>
cudaError_t with_router_shape(int E, F&& f) {
  using std::integral_constant;
  if (E == 128) return f(integral_constant<int, 4>{}, integral_constant<int, 4>{});
  if (E == 256) return f(integral_constant<int, 8>{}, integral_constant<int, 4>{});
  const int vpl = (E + 31) / 32;
  if (vpl <= 1) return f(integral_constant<int, 1>{}, integral_constant<int, 1>{});
  if (vpl <= 2) return f(integral_constant<int, 2>{}, integral_constant<int, 1>{});
  if (vpl <= 4) return f(integral_constant<int, 4>{}, integral_constant<int, 1>{});
  return f(integral_constant<int, 8>{}, integral_constant<int, 1>{});
}

}  // namespace

// Router logits and top-k for n tokens (n >= 1): x bf16 [n, D], w_router bf16
// [E, D]; writes topk_idx / topk_w and, when logits is not null, the fp32
// logits [n, E].  Requires D % 64 == 0 and E <= 256 (checked by the caller).
cudaError_t launch_router(const moe_plan& p, int32_t n, const void* x, const void* w_router,
                          float* logits, int32_t* topk_idx, float* topk_w, void* ws,
                          cudaStream_t st) {
  const int D = p.d.hidden, E = p.d.n_experts;
  if (n <= 0) return cudaSuccess;
  if (D % kRBK != 0 || E > kRMaxN) return cudaErrorNotSupported;
  RouterArgs g;
  g.logits = logits;
  g.topk_idx = topk_idx;
  g.topk_w = topk_w;
  g.ws = ws;
  g.n = n;
  g.E = E;
  g.K = p.d.top_k;
  g.n_mma = (E + 15) & ~15;
  g.tmem_cols = 32;
  while (g.tmem_cols < g.n_mma) g.tmem_cols *= 2;
  const int m_tiles = (n + kRBM - 1) / kRBM;
  const int k_total = D / kRBK;
  const int sms = num_sms();
  CUtensorMap mx, mw;
  if (!router_map(&mx, x, uint64_t(n), uint64_t(D), kRBM) ||
      !router_map(&mw, w_router, uint64_t(E), uint64_t(D), uint32_t(g.n_mma)))
    return cudaErrorInvalidValue;
  return with_router_shape(E, [&](auto vpl, auto vec) {
    return launch_router_k<decltype(vpl)::value, decltype(vec)::value>(mx, mw, g, m_tiles, k_total,
                                                                        sms, st);
  });
}

}  // namespace moe
