// FP8 block-scaled grouped SwiGLU expert GEMMs on the fifth-generation tensor
// cores (tcgen05.mma kind::f8f6f4), reading the FP8 rank-major receive buffer
// and its per-128-column scales where the dispatch left them: the grouped
// GEMMs read the buffer in place, and the interface does not depend on the
// activation quantisation format ("One-Sided Expert-Parallel All-to-All for
// Mixture-of-Experts Inference over NVLink", abstract).  The pages fix no
// format for an FP8 expert GEMM; the readings taken here, every scale fp32:
//   recv  e4m3 [T, D]      recv_scale [T, D/128]         per row and 128 columns
//   Wgu   e4m3 [E, 2I, D]  Wgu_scale  [E, 2I/128, D/128] per 128x128 tile
//   Wd    e4m3 [E, D, I]   Wd_scale   [E, D/128, I/128]
// Three launches:
//   GEMM1  h = bf16(silu(g) * u) with g[r, c] = sum_kb sa[r, kb] * sw[c/128, kb] * P_kb[r, c],
//          P_kb the tensor cores' fp32 sum of code products over k-block kb
//          (128 columns), u likewise from the up rows          -> H bf16 [T, I]
//   quant  Hq = e4m3(H / s) with s = amax of 128 columns / 448
//          (1 for an all-zero block), both quotients in fp32  -> Hq [T, I], Hs [T, I/128]
//   GEMM2  y = bf16(sum_kb hs[r, kb] * sw[c/128, kb] * P_kb[r, c])   -> Y bf16 [T, D]
//
// The scales change every 128 columns of the reduction, so each k-block's
// MMAs start a fresh partial sum in tensor memory, and the epilogue warps
// fold it, scaled, into fp32 registers.  One persistent kernel per GEMM, 320
// threads per CTA, one CTA per SM:
//   warp 0      TMA producer: A 128 rows x 128 B (16 KB) and B 256 rows x
//               128 B (32 KB) per stage, 128-byte swizzle, a 4-stage ring;
//   warp 1      owns the tensor memory (512 columns: two 128x256 fp32 partial
//               buffers); one lane issues 4 x tcgen05.mma (M=128, N=256,
//               K=32, e4m3 x e4m3 -> fp32) per k-block into the next free
//               partial buffer and publishes it with one tcgen05.commit (the
//               promotion warps free the stage when they see it);
//   warps 2..9  two warps per 32-lane quarter of tensor memory, each keeping
//               128 accumulator columns of its 32 rows in registers: wait for
//               a partial buffer, tcgen05.ld, multiply by the row scale times
//               the weight-tile scale and add, release the buffer; after the
//               last k-block of a tile, SwiGLU (GEMM1) or conversion (GEMM2)
//               and bf16 stores of the rows inside the expert's segment.
// Tiles (expert, n-tile, m-tile) come from the routing counts with the m-tile
// innermost; the producer thread takes them one at a time from a counter in
// the workspace and hands each to the CTA's other warps, so a CTA that
// finishes early takes more, and the CTAs that share a weight tile start it
// at about the same time.
// Every wait is bounded; on timeout the CTA records MOE_ERR_TIMEOUT, drains
// its copies and MMAs, frees its tensor memory and returns.
#include "moe_internal.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp8.h>

namespace moe {
namespace {

constexpr int kBM = 128;             // rows per tile (UMMA M)
constexpr int kBN = 256;             // accumulator columns per tile (UMMA N)
constexpr int kBK = 128;             // k-block: 128 e4m3 = one 128-byte swizzle row = one scale block
constexpr int kUmmaK = 32;           // e4m3 reduction per MMA
constexpr int kStages = 4;
constexpr int kPromoWarps = 8;
constexpr int kThreads = 64 + 32 * kPromoWarps;
constexpr int kTmemCols = 512;
constexpr int kCols = kBN / 2;       // accumulator columns per promotion thread
constexpr uint32_t kABytes = kBM * kBK;
constexpr uint32_t kBBytes = kBN * kBK;
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr size_t kSmemBytes = size_t(kStages) * kStageBytes + 1024 /*align*/ + 1024 /*meta*/;
constexpr int kQuantThreads = 256;

struct Fp8GemmArgs {
  const int32_t* counts;
  const int32_t* expert_off;
  const float* a_scale;  // [T, k_steps]: per row and k-block
  const float* b_scale;  // [E, b_rows / 128, k_steps]: per 128x128 weight tile
  __nv_bfloat16* out;    // H [T, I] (GEMM1) or Y [T, D] (GEMM2)
  int64_t out_ld;        // elements per output row
  int32_t E;
  int32_t k_steps;       // reduction size / kBK
  int32_t n_tiles;       // per expert
  int32_t b_rows;        // rows of B per expert (2I or D)
  int32_t inter;         // I (GEMM1: row offset of the up half inside an expert's B)
  int32_t total;         // T: rows of the receive buffer and of the outputs
  void* ws;
};

struct QuantArgs {
  const __nv_bfloat16* h;  // [T, I]
  const int32_t* slot_of;  // [n, k]
  uint8_t* hq;             // [T, I]
  float* h_scale;          // [T, I / 128]
  void* ws;
  int32_t n, K, inter, blocks, total;
};

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  // K-major operand, 128-byte swizzle: 8-row groups 1024 bytes apart (SBO),
  // leading offset unused (1), descriptor version 1, layout type 2.
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// kind::f8f6f4 instruction descriptor: e4m3 A and B (format 0, K-major),
// fp32 D, M = 128, N = n (a multiple of 16, at most 256).
__host__ __device__ constexpr uint32_t idesc_e4m3(int n) {
  return (1u << 4) | (uint32_t(n >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
}

__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
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

// 16 consecutive fp32 columns of this thread's TMEM lane.  Each load waits
// for its round trip to tensor memory, so wider loads mean fewer waits per
// k-block; but the 128 accumulators of a promotion thread and the
// temporaries of one load must fit in 168 registers (320 threads put three
// warps on one of the SM's four register-file partitions of 16 K registers,
// so no thread may have more), and 32 temporaries do not.  GEMM2 fits 16;
// GEMM1, whose SwiGLU epilogue needs a few more, loads 8 at a time.
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

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// Folds 32 partial-sum columns, scaled by sc, into acc[0..32).
template <bool kSwiGLU>
__device__ __forceinline__ void promote32(uint32_t taddr, float sc, float* acc) {
  constexpr int W = kSwiGLU ? 8 : 16;
#pragma unroll
  for (int h = 0; h < 32 / W; ++h) {
    float v[W];
    if constexpr (W == 8) tmem_ld8(taddr + uint32_t(h * W), v);
    else tmem_ld16(taddr + uint32_t(h * W), v);
#pragma unroll
    for (int i = 0; i < W; ++i) acc[h * W + i] = fmaf(v[i], sc, acc[h * W + i]);
  }
}

// The per-k-block waits of this kernel run about 50 times as often as the
// bf16 kernel's per-tile waits.  Poll by count first (mbarrier.try_wait
// already suspends the thread for a while when the phase is not complete)
// and read the clock only for a wait that lasts; still bounded, by
// kHotPolls polls plus mbar_wait's clock limit.
constexpr int kHotPolls = 1024;

__device__ __forceinline__ bool mbar_wait_hot(uint64_t* bar, uint32_t parity) {
  for (int i = 0; i < kHotPolls; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait(bar, parity);
}

struct Tile {
  int e, n, m;
};

// Tile t of the (expert, n-tile, m-tile) order with m innermost; s_pref[e] is
// the number of m-tiles of the experts below e.
__device__ __forceinline__ Tile tile_of(int t, const int* s_pref, int E, int n_tiles) {
  int lo = 0, hi = E;  // largest e with s_pref[e] * n_tiles <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_pref[mid] * n_tiles <= t) lo = mid;
    else hi = mid;
  }
  while (lo + 1 < E && s_pref[lo + 1] * n_tiles <= t) ++lo;  // experts without tiles
  const int mt = s_pref[lo + 1] - s_pref[lo];
  const int r = t - s_pref[lo] * n_tiles;
  Tile x;
  x.e = lo;
  x.n = r / mt;
  x.m = r % mt;
  return x;
}

// Column of tensor memory where this thread's accumulator chunk j (32
// columns) lives.  GEMM1: gate columns [0, 128) and up columns [128, 256) of
// the tile; the thread of half h owns gate [64h, 64h + 64) and the matching
// up columns, so it forms 64 outputs of H by itself.  GEMM2: [128h, 128h + 128).
template <bool kSwiGLU>
__device__ __forceinline__ int chunk_col(int half, int j) {
  if (kSwiGLU) return j < 2 ? half * 64 + j * 32 : kBN / 2 + half * 64 + (j - 2) * 32;
  return half * kCols + j * 32;
}

template <bool kSwiGLU>
__global__ void __launch_bounds__(kThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tma_a,
                    const __grid_constant__ CUtensorMap tma_b, Fp8GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* meta = smem + size_t(kStages) * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(meta);
  uint64_t* empty = full + kStages;
  uint64_t* pfull = empty + kStages;  // partial buffer b written by the MMAs
  uint64_t* pempty = pfull + 2;       // partial buffer b read by every promotion warp
  uint64_t* drained = pempty + 2;
  uint64_t* tq_full = drained + 1;
  uint64_t* tq_empty = tq_full + kTileQ;
  int* tq_slot = reinterpret_cast<int*>(tq_empty + kTileQ);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(tq_slot + kTileQ);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  __shared__ int s_pref[kMaxExperts + 1];
  __shared__ int s_cnt[kMaxExperts];  // counts clamped to [0, T]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = g.E;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&pfull[b], 1);
      mbar_init(&pempty[b], kPromoWarps);
    }
    mbar_init(drained, 1);
    tq_init(TileQueue{tq_slot, tq_full, tq_empty, 0, 0u}, 1 + kPromoWarps);
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
          if (!mbar_wait_hot(&empty[stage], phase ^ 1u)) {
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
    // The whole warp runs the loop and waits; one lane issues.
    int stage = 0, buf = 0;
    uint32_t phase = 0, buf_phase = 0;
    const uint32_t idesc = idesc_e4m3(kBN);
    // descriptor of stage 0's A tile; a stage, the B tile and a K step are
    // offsets in its 16-byte address field (shared addresses < 2^18)
    const uint64_t desc0 = smem_desc_sw128(smem_addr(smem));
    bool ok = true;
    TileQueue q{tq_slot, tq_full, tq_empty, 0, 0u};
    while (ok) {
      int t = total;
      bool got = true;
      if (lane == 0) got = !*s_abort && tq_pop(q, &t);
      got = __shfl_sync(0xFFFFFFFFu, got ? 1 : 0, 0) != 0;
      t = __shfl_sync(0xFFFFFFFFu, t, 0);
      if (!got) {
        if (lane == 0 && !*s_abort) set_status(g.ws, MOE_ERR_TIMEOUT);
        __syncwarp();
        *s_abort = 1;
        break;
      }
      if (t >= total) break;
      for (int kb = 0; kb < g.k_steps; ++kb) {
        bool w = !*s_abort;
        if (w) w = mbar_wait_hot(&full[stage], phase);
        if (w) w = mbar_wait_hot(&pempty[buf], buf_phase ^ 1u);
        w = __all_sync(0xFFFFFFFFu, w);
        if (!w) {
          if (lane == 0 && !*s_abort) set_status(g.ws, MOE_ERR_TIMEOUT);
          __syncwarp();
          *s_abort = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t d_tmem = tmem_base + uint32_t(buf * kBN);
          const uint64_t ad = desc0 + uint64_t((uint32_t(stage) * kStageBytes) >> 4);
          const uint64_t bd = ad + uint64_t(kABytes >> 4);
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k)
            umma_e4m3(d_tmem, ad + uint64_t(k * (kUmmaK >> 4)), bd + uint64_t(k * (kUmmaK >> 4)),
                      idesc, k != 0 ? 1u : 0u);
          // partial sum of this k-block ready; the promotion warps also free
          // the stage when they see it (the MMAs have read it by then)
          umma_commit(&pfull[buf]);
        }
        __syncwarp();
        if (++stage == kStages) stage = 0, phase ^= 1u;
        if (++buf == 2) buf = 0, buf_phase ^= 1u;
      }
    }
    // every MMA this warp issued has completed before the memory is freed
    if (lane == 0) {
      umma_commit(drained);
      if (!mbar_wait(drained, 0)) set_status(g.ws, MOE_ERR_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ promotion + epilogue
    const int quarter = warp & 3;           // TMEM lanes this warp may read
    const int half = (warp - 2) >> 2;       // which 128 of the tile's 256 columns
    const int r_local = quarter * 32 + lane;
    const int b_blocks = g.b_rows / 128;    // weight-tile scale rows per expert
    int buf = 0, stage = 0;
    uint32_t buf_phase = 0;
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
      const int rows = min(s_cnt[tl.e] - tl.m * kBM, kBM);
      const int64_t row = int64_t(g.expert_off[tl.e]) + tl.m * kBM + r_local;
      // a segment outside [0, T) (caller-supplied counts or offsets) is skipped
      const bool in_range = row >= 0 && row < g.total;
      // scale offsets as 32-bit element indices (T * k_steps and
      // E * b_rows / 128 * k_steps stay far below 2^31): fewer live registers
      // next to the 128 accumulators
      const int sa_off = int(in_range ? row : 0) * g.k_steps;
      // scale rows of the weight tiles under chunks 0-1 and 2-3
      int brow0, brow1;
      if (kSwiGLU) {
        brow0 = tl.e * b_blocks + tl.n;
        brow1 = tl.e * b_blocks + g.inter / 128 + tl.n;
      } else {
        brow0 = brow1 = tl.e * b_blocks + 2 * tl.n + half;
      }
      const int sb0_off = brow0 * g.k_steps;
      const int sb1_off = brow1 * g.k_steps;
      float acc[kCols];
#pragma unroll
      for (int i = 0; i < kCols; ++i) acc[i] = 0.f;
      bool ok = true;
      for (int kb = 0; kb < g.k_steps; ++kb) {
        const float sa = in_range ? __ldg(g.a_scale + (sa_off + kb)) : 0.f;
        const float s0 = sa * __ldg(g.b_scale + (sb0_off + kb));
        const float s1 = sa * __ldg(g.b_scale + (sb1_off + kb));
        bool ready = true;
        if (lane == 0) ready = !*s_abort && mbar_wait_hot(&pfull[buf], buf_phase);
        ready = __shfl_sync(0xFFFFFFFFu, ready ? 1 : 0, 0) != 0;
        if (!ready) {
          if (lane == 0 && !*s_abort) set_status(g.ws, MOE_ERR_TIMEOUT);
          *s_abort = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        if (warp == 2 && lane == 0) mbar_arrive(&empty[stage]);  // the stage's MMAs are done
        if (++stage == kStages) stage = 0;
        const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(buf * kBN);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float sc = (kSwiGLU && j >= 2) ? s1 : s0;
          promote32<kSwiGLU>(taddr + uint32_t(chunk_col<kSwiGLU>(half, j)), sc, acc + j * 32);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty[buf]);
        if (++buf == 2) buf = 0, buf_phase ^= 1u;
      }
      if (!ok) break;
      if (r_local < rows && !in_range) set_status(g.ws, MOE_ERR_DEVICE_INDEX);
      if (r_local < rows && in_range) {
        if (kSwiGLU) {
          uint4* dst = reinterpret_cast<uint4*>(g.out + row * g.out_ld +
                                                int64_t(tl.n) * (kBN / 2) + half * 64);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            uint32_t p[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const int i = q * 8 + w * 2;
              const float h0 = acc[i] / (1.f + expf(-acc[i])) * acc[64 + i];
              const float h1 = acc[i + 1] / (1.f + expf(-acc[i + 1])) * acc[64 + i + 1];
              p[w] = pack_bf16x2(h0, h1);
            }
            dst[q] = make_uint4(p[0], p[1], p[2], p[3]);
          }
        } else {
          uint4* dst = reinterpret_cast<uint4*>(g.out + row * g.out_ld + int64_t(tl.n) * kBN +
                                                half * kCols);
#pragma unroll
          for (int q = 0; q < 16; ++q)
            dst[q] = make_uint4(pack_bf16x2(acc[q * 8], acc[q * 8 + 1]),
                                pack_bf16x2(acc[q * 8 + 2], acc[q * 8 + 3]),
                                pack_bf16x2(acc[q * 8 + 4], acc[q * 8 + 5]),
                                pack_bf16x2(acc[q * 8 + 6], acc[q * 8 + 7]));
        }
      }
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

// H rows of every filled slot to e4m3 with one fp32 scale per 128 columns:
// one warp per (token pick, 128-column block), 4 columns per lane.  The
// scale amax / 448 and the quotients h / s are correctly rounded fp32
// divisions; the conversion rounds to nearest even and saturates at 448.
__global__ void __launch_bounds__(kQuantThreads) quant_h_kernel(QuantArgs q) {
  const int lane = threadIdx.x & 31;
  const int warps = kQuantThreads / 32;
  const int64_t items = int64_t(q.n) * q.K * q.blocks;
  grid_dependency_wait();
  for (int64_t it = int64_t(blockIdx.x) * warps + (threadIdx.x >> 5); it < items;
       it += int64_t(gridDim.x) * warps) {
    const int64_t tk = it / q.blocks;
    const int b = int(it % q.blocks);
    const int s = q.slot_of[tk];
    if (s < 0 || s >= q.total) {
      if (lane == 0) set_status(q.ws, MOE_ERR_DEVICE_INDEX);
      continue;
    }
    const int64_t at = int64_t(s) * q.inter + b * 128 + lane * 4;
    const uint2 raw = *reinterpret_cast<const uint2*>(q.h + at);
    const float v0 = bf16_lo(raw.x), v1 = bf16_hi(raw.x), v2 = bf16_lo(raw.y), v3 = bf16_hi(raw.y);
    float amax = fmaxf(fmaxf(fabsf(v0), fabsf(v1)), fmaxf(fabsf(v2), fabsf(v3)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    const uint32_t c01 = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(v0, sc), __fdiv_rn(v1, sc)), __NV_SATFINITE, __NV_E4M3);
    const uint32_t c23 = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(v2, sc), __fdiv_rn(v3, sc)), __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<uint32_t*>(q.hq + at) = (c01 & 0xFFFFu) | ((c23 & 0xFFFFu) << 16);
    if (lane == 0) q.h_scale[int64_t(s) * q.blocks + b] = sc;
  }
  grid_dependents_launch();
}

// ---------------------------------------------------------------- host side
// 2D e4m3 tensor map over a row-major [rows, cols] byte matrix; box = 128
// columns (128 bytes, the swizzle width) x box_rows rows.
bool make_map_e4m3(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {uint32_t(kBK), box_rows};
  const cuuint32_t elem[2] = {1, 1};
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn)(
             map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <bool kSwiGLU>
cudaError_t launch_fp8_gemm(const CUtensorMap& a, const CUtensorMap& b, const Fp8GemmArgs& g,
                            int sms, cudaStream_t st) {
  cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(fp8_gemm_kernel<kSwiGLU>),
                                 int(kSmemBytes));
  if (e != cudaSuccess) return e;
  return launch_pdl(fp8_gemm_kernel<kSwiGLU>, dim3(unsigned(sms)), dim3(kThreads), kSmemBytes,
                    st, a, b, g);
}

}  // namespace

cudaError_t launch_swiglu_fp8(const moe_plan& p, int32_t n, const void* recv,
                              const float* recv_scale, const int32_t* counts,
                              const int32_t* expert_off, const int32_t* slot_of,
                              const void* w_gate_up, const float* w_gate_up_scale,
                              const void* w_down, const float* w_down_scale, void* h, void* hq,
                              float* h_scale, void* y, void* ws, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const int64_t T = total_rows(p, n);
  const int D = p.d.hidden, I = p.d.inter, E = p.d.n_experts;
  if (D % kBN != 0 || I % kBK != 0 || E > kMaxExperts || p.d.scale_block != kBK)
    return cudaErrorNotSupported;
  CUtensorMap a1, b1, a2, b2;
  if (!make_map_e4m3(&a1, recv, uint64_t(T), uint64_t(D), kBM) ||
      !make_map_e4m3(&b1, w_gate_up, uint64_t(E) * 2 * I, uint64_t(D), kBN / 2) ||
      !make_map_e4m3(&a2, hq, uint64_t(T), uint64_t(I), kBM) ||
      !make_map_e4m3(&b2, w_down, uint64_t(E) * D, uint64_t(I), kBN))
    return cudaErrorInvalidValue;
  const int sms = num_sms();
  Fp8GemmArgs g1;
  g1.counts = counts;
  g1.expert_off = expert_off;
  g1.a_scale = recv_scale;
  g1.b_scale = w_gate_up_scale;
  g1.out = static_cast<__nv_bfloat16*>(h);
  g1.out_ld = I;
  g1.E = E;
  g1.k_steps = D / kBK;
  g1.n_tiles = I / (kBN / 2);
  g1.b_rows = 2 * I;
  g1.inter = I;
  g1.total = int32_t(T);
  g1.ws = ws;
  cudaError_t e = launch_fp8_gemm<true>(a1, b1, g1, sms, st);
  if (e != cudaSuccess) return e;

  QuantArgs q;
  q.h = static_cast<const __nv_bfloat16*>(h);
  q.slot_of = slot_of;
  q.hq = static_cast<uint8_t*>(hq);
  q.h_scale = h_scale;
  q.ws = ws;
  q.n = n;
  q.K = p.d.top_k;
  q.inter = I;
  q.blocks = I / 128;
  q.total = int32_t(T);
  const int64_t items = int64_t(n) * q.K * q.blocks;
  const int64_t per_block = kQuantThreads / 32;
  int64_t grid = (items + per_block - 1) / per_block;
  if (grid > int64_t(sms) * 16) grid = int64_t(sms) * 16;
  e = launch_pdl(quant_h_kernel, dim3(unsigned(grid)), dim3(kQuantThreads), 0, st, q);
  if (e != cudaSuccess) return e;

  Fp8GemmArgs g2 = g1;
  g2.a_scale = h_scale;
  g2.b_scale = w_down_scale;
  g2.out = static_cast<__nv_bfloat16*>(y);
  g2.out_ld = D;
  g2.k_steps = I / kBK;
  g2.n_tiles = D / kBN;
  g2.b_rows = D;
  g2.inter = 0;
  return launch_fp8_gemm<false>(a2, b2, g2, sms, st);
}

}  // namespace moe
