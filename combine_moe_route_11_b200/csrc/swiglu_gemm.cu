// Grouped SwiGLU expert GEMMs on the fifth-generation tensor cores (tcgen05),
// reading the rank-major receive buffer in place: the grouped GEMMs read the
// buffer where the dispatch left it instead of a per-expert copy ("One-Sided
// Expert-Parallel All-to-All for Mixture-of-Experts Inference over NVLink",
// abstract), and each expert's rows are one contiguous segment, the promise a
// sorted-index grouped GEMM relies on ("backends/mlx: runtime MoE expert-sort
// for decode", author update on the gather_mm contract).
//
//   GEMM1 (per expert e, rows [off_e, off_e + cnt_e) of recv):
//     h = bf16( silu(x Wg[e]^T) * (x Wu[e]^T) )   -> H[T, I]
//   GEMM2:  y = bf16( h Wd[e]^T )                  -> Y[T, D]
//
// One persistent kernel per GEMM, 192 threads per CTA, one CTA per SM:
//   warp 0      TMA producer: A tile 128x64 (16 KB) and B tile 256x64 (32 KB)
//               per stage, 128-byte swizzle, into a 4-stage ring;
//   warp 1      owns the tensor memory (512 columns: two 128x256 fp32
//               accumulators) and one lane issues tcgen05.mma (M=128, N=256,
//               K=16, bf16 in, fp32 accumulate), releasing stages and
//               publishing finished accumulators through tcgen05.commit;
//   warps 2..5  epilogue: tcgen05.ld of their 32-row quarter, SwiGLU (GEMM1)
//               or conversion (GEMM2), bf16 stores of the valid rows.
// Tiles (expert, n-tile, m-tile) are enumerated on the device from the
// routing counts, m-tile innermost; the producer thread takes them one at a
// time from a counter in the workspace and hands each to the CTA's other
// warps, so a CTA that finishes early takes more, and the CTAs sharing a
// weight tile start it at about the same time.  An expert's last m-tile usually holds only a few rows;
// when it holds at most 96, the tile swaps the operand roles -- the weight
// rows become the MMA's M side (two M=128 halves) and the token rows its N
// side, rounded up to 16 -- so the tensor cores do work in proportion to
// the rows present instead of a full 128.  Its accumulators are transposed
// (TMEM lane = weight row, column = token) and the epilogue stores them
// transposed.  Rows of a normal tile past the expert's segment are computed
// and not stored.  Every wait is bounded; on timeout the CTA records
// MOE_ERR_TIMEOUT, drains its own copies and MMAs, frees its tensor memory
// and returns.
#include "moe_internal.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace moe {
namespace {

constexpr int kBM = 128;             // rows per tile (UMMA M)
constexpr int kBN = 256;             // accumulator columns per tile (UMMA N)
constexpr int kBK = 64;              // reduction step: 64 bf16 = one 128-byte swizzle row
constexpr int kUmmaK = 16;
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;
constexpr int kTmemCols = 512;
constexpr uint32_t kABytes = kBM * kBK * 2;
constexpr uint32_t kBBytes = kBN * kBK * 2;
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr int kMaxE = kMaxExperts;
constexpr int kSwapMaxRows = 96;     // last m-tiles with at most this many rows swap roles
constexpr size_t kSmemBytes = size_t(kStages) * kStageBytes + 1024 /*align*/ + 1024 /*meta*/;

struct GemmArgs {
  const int32_t* counts;
  const int32_t* expert_off;
  __nv_bfloat16* out;  // H [T, I] (GEMM1) or Y [T, D] (GEMM2)
  int64_t out_ld;      // elements per output row
  int32_t E;
  int32_t k_steps;     // reduction size / kBK
  int32_t n_tiles;     // per expert
  int32_t b_rows;      // rows of B per expert in its 2D view (2I or D)
  int32_t inter;       // I (GEMM1: row offset of the up half inside an expert's B)
  int32_t total;       // T: rows of the receive buffer and of the outputs
  void* ws;
};

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  // K-major operand, 128-byte swizzle: 8-row groups 1024 bytes apart (SBO),
  // leading offset unused (1), descriptor version 1, layout type 2.
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// kind::f16 instruction descriptor: bf16 A and B (K-major), fp32 D, M=128,
// N = n (a multiple of 16, at most 256).
__host__ __device__ constexpr uint32_t idesc_m128(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// 32 consecutive fp32 accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

struct Tile {
  int e, n, m;
};

// Rows of tile tl that belong to its expert (1..128), from the clamped counts.
__device__ __forceinline__ int tile_rows(const Tile& tl, const int* s_cnt) {
  return min(s_cnt[tl.e] - tl.m * kBM, kBM);
}
__device__ __forceinline__ bool swapped_tile(int rows) { return rows <= kSwapMaxRows; }

// Tile t of the (expert, n-tile, m-tile) order with m innermost; s_pref[e] is
// the number of m-tiles of the experts below e.
__device__ __forceinline__ Tile tile_of(int t, const int* s_pref, int E, int n_tiles) {
  int lo = 0, hi = E;  // largest e with s_pref[e] * n_tiles <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_pref[mid] * n_tiles <= t) lo = mid;
    else hi = mid;
  }
  // skip experts without tiles (equal prefixes)
  while (lo + 1 < E && s_pref[lo + 1] * n_tiles <= t) ++lo;
  const int mt = s_pref[lo + 1] - s_pref[lo];
  const int r = t - s_pref[lo] * n_tiles;
  Tile x;
  x.e = lo;
  x.n = r / mt;
  x.m = r % mt;
  return x;
}

template <bool kSwiGLU>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tma_a,
                        const __grid_constant__ CUtensorMap tma_b, GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* meta = smem + size_t(kStages) * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(meta);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drained = acc_empty + 2;
  uint64_t* tq_full = drained + 1;
  uint64_t* tq_empty = tq_full + kTileQ;
  int* tq_slot = reinterpret_cast<int*>(tq_empty + kTileQ);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(tq_slot + kTileQ);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  __shared__ int s_pref[kMaxE + 1];
  __shared__ int s_cnt[kMaxE];  // counts clamped to [0, T]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = g.E;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    mbar_init(drained, 1);
    tq_init(TileQueue{tq_slot, tq_full, tq_empty, 0, 0u}, 1 + kEpiWarps);
    *s_abort = 0;
    fence_barrier_init();
  }
  grid_dependency_wait();
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(s_tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // m-tiles per expert -> prefix, from the routing counts
  if (warp == 2) {
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int c = e < E ? min(max(g.counts[e], 0), g.total) : 0;
      if (e < E) s_cnt[e] = c;
      const int mt = (c + kBM - 1) / kBM;
      int incl = mt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      if (e < E) s_pref[e] = carry + incl - mt;
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) s_pref[E] = carry;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total = s_pref[E] * g.n_tiles;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;  // copies issued, in ring order
      TileQueue q{tq_slot, tq_full, tq_empty, 0, 0u};
      for (;;) {
        // the next tile, published before its copies; `total` ends every loop
        const int t = *s_abort ? total : tq_take(g.ws, total);
        if (!tq_push(q, t)) {
          set_status(g.ws, MOE_ERR_TIMEOUT);
          *s_abort = 1;
          break;
        }
        if (t >= total) break;
        const Tile tl = tile_of(t, s_pref, E, g.n_tiles);
        const int a_row = g.expert_off[tl.e] + tl.m * kBM;
        const int b_row = tl.e * g.b_rows + tl.n * (kSwiGLU ? kBN / 2 : kBN);
        for (int kb = 0; kb < g.k_steps; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u)) {
            set_status(g.ws, MOE_ERR_TIMEOUT);
            *s_abort = 1;
            break;
          }
          uint8_t* a_dst = smem + size_t(stage) * kStageBytes;
          uint8_t* b_dst = a_dst + kABytes;
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          tma_load_2d(a_dst, &tma_a, kb * kBK, a_row, &full[stage]);
          if (kSwiGLU) {
            tma_load_2d(b_dst, &tma_b, kb * kBK, b_row, &full[stage]);
            tma_load_2d(b_dst + kBBytes / 2, &tma_b, kb * kBK, b_row + g.inter, &full[stage]);
          } else {
            tma_load_2d(b_dst, &tma_b, kb * kBK, b_row, &full[stage]);
          }
          ++issued;
          if (++stage == kStages) stage = 0, phase ^= 1u;
        }
      }
      // never leave a copy in flight into this CTA's shared memory: a copy
      // was only issued into a stage once the MMAs had consumed the copy
      // before it, so only the last kStages copies can still be unwaited
      for (int i = issued > kStages ? issued - kStages : 0; i < issued; ++i)
        if (!mbar_wait(&full[i % kStages], uint32_t(i / kStages) & 1u))
          set_status(g.ws, MOE_ERR_TIMEOUT);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      TileQueue q{tq_slot, tq_full, tq_empty, 0, 0u};
      for (;;) {
        int t = total;
        if (*s_abort || !tq_pop(q, &t)) {
          if (!*s_abort) set_status(g.ws, MOE_ERR_TIMEOUT);
          *s_abort = 1;
          break;
        }
        if (t >= total) break;
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u)) {
          set_status(g.ws, MOE_ERR_TIMEOUT);
          *s_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * kBN);
        const Tile tl = tile_of(t, s_pref, E, g.n_tiles);
        const int rows = tile_rows(tl, s_cnt);
        const bool swap = swapped_tile(rows);
        // swapped: M = 128 weight rows per half, N = the tile's rows rounded up to 16
        const uint32_t idesc = swap ? idesc_m128((rows + 15) & ~15) : idesc_m128(kBN);
        bool ok = true;
        for (int kb = 0; kb < g.k_steps; ++kb) {
          if (!mbar_wait(&full[stage], phase)) {
            set_status(g.ws, MOE_ERR_TIMEOUT);
            *s_abort = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(smem + size_t(stage) * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
          if (swap) {
#pragma unroll
            for (int k = 0; k < kBK / kUmmaK; ++k)
#pragma unroll
              for (int half = 0; half < 2; ++half)
                umma_bf16(d_tmem + uint32_t(half * (kBN / 2)),
                          smem_desc_sw128(b_addr + half * (kBBytes / 2) + k * kUmmaK * 2),
                          smem_desc_sw128(a_addr + k * kUmmaK * 2), idesc,
                          (kb | k) != 0 ? 1u : 0u);
          } else {
#pragma unroll
            for (int k = 0; k < kBK / kUmmaK; ++k)
              umma_bf16(d_tmem, smem_desc_sw128(a_addr + k * kUmmaK * 2),
                        smem_desc_sw128(b_addr + k * kUmmaK * 2), idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);  // stage free once these MMAs have read it
          if (++stage == kStages) stage = 0, phase ^= 1u;
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);  // accumulator ready for the epilogue
        if (++acc == 2) acc = 0, acc_phase ^= 1u;
      }
      // every MMA this thread issued has completed before the memory is freed
      umma_commit(drained);
      if (!mbar_wait(drained, 0)) set_status(g.ws, MOE_ERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may read
    const int r_local = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    TileQueue q{tq_slot, tq_full, tq_empty, 0, 0u};
    for (;;) {
      int t = total;
      bool got = true;
      if (lane == 0) got = !*s_abort && tq_pop(q, &t);
      got = __shfl_sync(0xFFFFFFFFu, got ? 1 : 0, 0) != 0;
      t = __shfl_sync(0xFFFFFFFFu, t, 0);
      if (!got) {
        if (lane == 0 && !*s_abort) set_status(g.ws, MOE_ERR_TIMEOUT);
        *s_abort = 1;
        break;
      }
      if (t >= total) break;
      const Tile tl = tile_of(t, s_pref, E, g.n_tiles);
      bool ready = true;
      if (lane == 0) ready = mbar_wait(&acc_full[acc], acc_phase);
      ready = __shfl_sync(0xFFFFFFFFu, ready ? 1 : 0, 0) != 0;
      if (!ready) {
        if (lane == 0) set_status(g.ws, MOE_ERR_TIMEOUT);
        *s_abort = 1;
        break;
      }
      tc_fence_after();
      const int rows = tile_rows(tl, s_cnt);
      const int64_t row0 = int64_t(g.expert_off[tl.e]) + tl.m * kBM;
      const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(acc * kBN);
      if (swapped_tile(rows)) {
        // transposed accumulators: this thread's TMEM lane is weight row
        // r_local of each half, column c is the tile's row c
#pragma unroll 1
        for (int c0 = 0; c0 < rows; c0 += 32) {
          if (kSwiGLU) {
            float gate[32], up[32];
            tmem_ld32(taddr + uint32_t(c0), gate);
            tmem_ld32(taddr + uint32_t(kBN / 2 + c0), up);
            const int64_t f = int64_t(tl.n) * (kBN / 2) + r_local;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int64_t row = row0 + c0 + i;
              if (c0 + i >= rows) break;
              if (row < 0 || row >= g.total) {
                set_status(g.ws, MOE_ERR_DEVICE_INDEX);
                continue;
              }
              const float h = gate[i] / (1.f + expf(-gate[i])) * up[i];
              g.out[row * g.out_ld + f] = __float2bfloat16_rn(h);
            }
          } else {
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
              float v[32];
              tmem_ld32(taddr + uint32_t(half * (kBN / 2) + c0), v);
              const int64_t f = int64_t(tl.n) * kBN + half * (kBN / 2) + r_local;
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int64_t row = row0 + c0 + i;
                if (c0 + i >= rows) break;
                if (row < 0 || row >= g.total) {
                  set_status(g.ws, MOE_ERR_DEVICE_INDEX);
                  continue;
                }
                g.out[row * g.out_ld + f] = __float2bfloat16_rn(v[i]);
              }
            }
          }
        }
      } else {
      const int64_t row = row0 + r_local;
      // a segment outside [0, T) (caller-supplied counts or offsets) is skipped
      const bool in_range = row >= 0 && row < g.total;
      const bool valid = r_local < rows && in_range;
      if (r_local < rows && !in_range) set_status(g.ws, MOE_ERR_DEVICE_INDEX);
      if (kSwiGLU) {
        __nv_bfloat16* dst = g.out + row * g.out_ld + int64_t(tl.n) * (kBN / 2);
#pragma unroll 1
        for (int c = 0; c < kBN / 2; c += 32) {
          float gate[32], up[32];
          tmem_ld32(taddr + uint32_t(c), gate);
          tmem_ld32(taddr + uint32_t(kBN / 2 + c), up);
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float h0 = gate[2 * i] / (1.f + expf(-gate[2 * i])) * up[2 * i];
            const float h1 = gate[2 * i + 1] / (1.f + expf(-gate[2 * i + 1])) * up[2 * i + 1];
            packed[i] = pack_bf16x2(h0, h1);
          }
          if (valid) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              d4[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
        }
      } else {
        __nv_bfloat16* dst = g.out + row * g.out_ld + int64_t(tl.n) * kBN;
#pragma unroll 1
        for (int c = 0; c < kBN; c += 32) {
          float v[32];
          tmem_ld32(taddr + uint32_t(c), v);
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) packed[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
          if (valid) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              d4[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
        }
      }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == 2) acc = 0, acc_phase ^= 1u;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols)
                 : "memory");
  if (threadIdx.x == 0) tq_finish(g.ws);
  grid_dependents_launch();
}

// ---------------------------------------------------------------- host side
}  // namespace

void* tensor_map_encoder() {
  // looked up once (thread-safe static initialisation); null if unavailable
  static void* const fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return p;
  }();
  return fn;
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
}

// 2D bf16 tensor map over a row-major [rows, cols] matrix; box = 64 columns
// (128 bytes, the swizzle width) x box_rows rows.
bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {uint32_t(kBK), box_rows};
  const cuuint32_t elem[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kSwiGLU>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& g, int sms,
                        cudaStream_t st) {
  cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(grouped_gemm_kernel<kSwiGLU>),
                                 int(kSmemBytes));
  if (e != cudaSuccess) return e;
  return launch_pdl(grouped_gemm_kernel<kSwiGLU>, dim3(unsigned(sms)), dim3(kThreads), kSmemBytes,
                    st, a, b, g);
}

}  // namespace

cudaError_t launch_swiglu(const moe_plan& p, int32_t n, const void* recv, const int32_t* counts,
                          const int32_t* expert_off, const void* w_gate_up, const void* w_down,
                          void* h, void* y, void* ws, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const int64_t T = total_rows(p, n);
  const int D = p.d.hidden, I = p.d.inter, E = p.d.n_experts;
  if (D % kBN != 0 || I % (kBN / 2) != 0 || E > kMaxE) return cudaErrorNotSupported;
  CUtensorMap a1, b1, a2, b2;
  if (!make_map(&a1, recv, uint64_t(T), uint64_t(D), kBM) ||
      !make_map(&b1, w_gate_up, uint64_t(E) * 2 * I, uint64_t(D), kBN / 2) ||
      !make_map(&a2, h, uint64_t(T), uint64_t(I), kBM) ||
      !make_map(&b2, w_down, uint64_t(E) * D, uint64_t(I), kBN))
    return cudaErrorInvalidValue;
  const int sms = num_sms();
  GemmArgs g1;
  g1.counts = counts;
  g1.expert_off = expert_off;
  g1.out = static_cast<__nv_bfloat16*>(h);
  g1.out_ld = I;
  g1.E = E;
  g1.k_steps = D / kBK;
  g1.n_tiles = I / (kBN / 2);
  g1.b_rows = 2 * I;
  g1.inter = I;
  g1.total = int32_t(T);
  g1.ws = ws;
  cudaError_t e = launch_gemm<true>(a1, b1, g1, sms, st);
  if (e != cudaSuccess) return e;
  GemmArgs g2 = g1;
  g2.out = static_cast<__nv_bfloat16*>(y);
  g2.out_ld = D;
  g2.k_steps = I / kBK;
  g2.n_tiles = D / kBN;
  g2.b_rows = D;
  g2.inter = 0;
  return launch_gemm<false>(a2, b2, g2, sms, st);
}

}  // namespace moe
