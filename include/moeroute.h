/*
 * moeroute -- Mixture-of-Experts token dispatch and combine on one B200.
 *
 * C ABI of libmoeroute.so.  Plain pointers and sizes only.
 *
 * The path (and the passages that define each step):
 *   moe_route_topk   top-k experts per token, gate weights, per-expert counts
 *                    and the rank-major expert offsets.  Rank-major buffers
 *                    with fixed per-rank regions let every source compute its
 *                    destinations locally, without exchanging metadata first
 *                    ("One-Sided Expert-Parallel All-to-All for Mixture-of-
 *                    Experts Inference over NVLink", abstract).  The selection
 *                    has the [N, top_k] shape of the expert indices that the
 *                    sorted/unsorted gather consumes ("backends/mlx: runtime
 *                    MoE expert-sort for decode", Summary and author updates).
 *   moe_router_topk  the router GEMM (logits = x W_r^T) on the tensor cores
 *                    with the top-k and softmax fused into its epilogue,
 *                    then the counts and offsets of moe_route_topk.
 *   moe_dispatch     copies every token row to its k expert slots
 *                    ("MLX expert parallelism all_to_all PR 3158", Facts:
 *                    dispatch_local / dispatch_scatter_remote).
 *   moe_route_dispatch  the two calls above as one launch for small batches.
 *   moe_expert_*     the expert step reading the dispatched buffer in place
 *                    (bf16, or FP8 with its scales, the interface being
 *                    agnostic to the activation quantisation format):
 *                    grouped GEMMs read the rank-major buffer instead of a
 *                    per-expert copy (arXiv 2611.13188 abstract); segments are
 *                    contiguous, which is the promise a sorted-index grouped
 *                    GEMM relies on ("backends/mlx: runtime MoE expert-sort
 *                    for decode", author update on the gather_mm contract).
 *   moe_combine      weighted sum of the k expert outputs back in token order
 *                    (PR 3158 Facts: combine_gather_remote, combine_weighted_sum).
 *   moe_layer        all of the above in order on one stream.
 *
 * Terms.  N = tokens of the call (n <= desc.n_max), D = hidden, E = experts,
 * k = top_k, R = virtual ranks.  Virtual rank r owns experts
 * [r*E/R, (r+1)*E/R) and the region of C_r = N*min(k, E/R) rows starting at
 * row r*C_r of the receive buffer, which has T = R*C_r rows.  Inside a region
 * experts ascend by id, inside an expert rows ascend by source token:
 *     slot(t, j) = expert_off[e] + #{t' < t : t' picked e},  e = topk_idx[t, j].
 * Rows of a region past its filled count are never written.
 *
 * Conventions for every entry point below.
 *  - Memory: the caller allocates and owns every buffer; the library never
 *    allocates or frees device memory.  "device" pointers must be device
 *    memory of the current device, 16-byte aligned, rows dense (row stride =
 *    D * element size).  Pointers named *_host are host memory.
 *  - Asynchrony: compute calls only enqueue work on `stream` and return; none
 *    synchronises except moe_get_status.  Results are visible after the usual
 *    stream ordering.
 *  - Errors: argument errors are detected on the host before anything is
 *    enqueued and returned as MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED; a
 *    failed launch returns MOE_ERR_CUDA.  Errors only the device can see (an
 *    expert id outside [0, E) or a slot outside [0, T) in caller-supplied
 *    arrays, a non-finite logit row) are recorded in the workspace status word
 *    (first error wins), the offending item is skipped, and the outputs of
 *    that call are unspecified.  moe_get_status returns and clears it.
 *  - Workspace: `ws` is caller memory of moe_workspace_bytes() (or
 *    moe_layer_workspace_bytes() for moe_layer), zero-filled before its first
 *    use; the library keeps its control words consistent afterwards.  Calls
 *    that share one workspace must be ordered on one stream.
 */
#ifndef MOEROUTE_H
#define MOEROUTE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (same underlying type); NULL is the legacy default stream. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,   /* bad pointer, size, alignment or n > n_max */
  MOE_ERR_UNSUPPORTED = -2,   /* valid but outside what this library implements */
  MOE_ERR_CUDA = -3,          /* a CUDA runtime call or launch failed */
  MOE_ERR_WORKSPACE = -4,     /* workspace too small or misaligned */
  MOE_ERR_DEVICE_INDEX = -5,  /* device saw an expert id or slot out of range */
  MOE_ERR_TIMEOUT = -6,       /* a bounded device-side wait gave up */
  MOE_ERR_NONFINITE = -7      /* device saw a logit row with fewer than k finite values */
} moe_status;

typedef enum {
  MOE_F32 = 0,       /* IEEE binary32 */
  MOE_BF16 = 1,      /* bfloat16 */
  MOE_FP8_E4M3 = 2   /* OCP FP8 E4M3 (finite, NaN = S.1111.111) */
} moe_dtype;

/* Static description of one MoE configuration. */
typedef struct {
  int32_t n_max;        /* largest N any call will pass (>= 1) */
  int32_t hidden;       /* D */
  int32_t n_experts;    /* E, 1..512 */
  int32_t top_k;        /* k, 1..min(E, 32) */
  int32_t n_ranks;      /* R >= 1, E % R == 0 */
  int32_t x_dtype;      /* moe_dtype of token rows x (and of recv) */
  int32_t y_dtype;      /* moe_dtype of expert outputs Y read by combine (F32|BF16) */
  int32_t out_dtype;    /* moe_dtype of combine output (F32|BF16) */
  int32_t scale_block;  /* FP8 rows: columns per fp32 scale (e.g. 128), 0 = no scales */
  int32_t inter;        /* SwiGLU intermediate size I for moe_layer, 0 = identity experts */
} moe_desc;

typedef struct moe_plan moe_plan;

/* Validate `desc` and build a plan (host only, no CUDA call).
 * Requires: every row (x, Y, out) a multiple of 16 bytes; scale_block > 0
 * only with FP8 rows and dividing D; T(n_max) < 2^31 and
 * ceil(n_max / 32) * E < 2^31; for inter > 0 also
 * y = BF16, D % 256 == 0, I % 128 == 0 and either x = BF16 (bf16 experts) or
 * x = FP8 with scale_block = 128 (FP8 experts).  *out is set only on MOE_OK. */
MOE_API moe_status moe_plan_create(const moe_desc* desc, moe_plan** out);
MOE_API void moe_plan_destroy(moe_plan* plan);

/* Bytes of scratch for the route/dispatch/combine/expert calls (n <= n_max). */
MOE_API size_t moe_workspace_bytes(const moe_plan* plan);
/* Bytes of scratch for moe_layer: the above plus every intermediate buffer. */
MOE_API size_t moe_layer_workspace_bytes(const moe_plan* plan);
/* C_r and T for a call with n tokens (rows per region, rows of recv). */
MOE_API int64_t moe_region_rows(const moe_plan* plan, int32_t n);
MOE_API int64_t moe_recv_rows(const moe_plan* plan, int32_t n);

/* Route: for each token t < n,
 *   topk_idx[t, 0..k)  experts by descending logit, ties to the lower id;
 *   topk_w[t, j]       = exp(L[t,idx_j] - L[t,idx_0]) / sum_i exp(L[t,idx_i] - L[t,idx_0]);
 *   counts[e]          = #{(t, j) : topk_idx[t, j] == e};
 *   expert_off[e]      = (e / (E/R)) * C_r + sum of counts of lower experts
 *                        of the same rank;  expert_off[E] = T.
 * logits: device fp32 [n, E] row-major.  topk_idx: device int32 [n, k];
 * topk_w: device fp32 [n, k]; counts: device int32 [E]; expert_off: device
 * int32 [E + 1].  Also leaves in `ws` the per-block bases that moe_dispatch
 * uses for the slots of this routing.  n = 0 writes zero counts and offsets.
 * One launch of at most one CTA per SM: a CTA routes route blocks of 32
 * tokens, writes each block's per-expert counts and adds them into
 * per-expert totals in `ws`; the last min(CTAs, 8) CTAs to finish share the
 * scan of all blocks' counts into the offsets and per-block bases (each
 * waits, bounded, only for the others to finish; MOE_ERR_TIMEOUT in the
 * status word if that wait ever ran out). */
MOE_API moe_status moe_route_topk(const moe_plan* plan, int32_t n, const float* logits,
                          int32_t* topk_idx, float* topk_w, int32_t* counts,
                          int32_t* expert_off, void* ws, moe_stream_t stream);

/* Router GEMM fused ahead of top-k: logits[t, e] = x[t] . w_router[e], bf16
 * operands summed in fp32 on the tensor cores, then the top-k selection and
 * the softmax over the k winners of every row in the same kernel, then the
 * counts, offsets and positions of moe_route_topk.  The gate that produces
 * the [N, top_k] expert indices ("backends/mlx: runtime MoE expert-sort for
 * decode", author updates on the sorted path) is not spelt out on the pages;
 * this is its plain reading as a linear map of the token's hidden row.
 * x: device bf16 [n, D] hidden rows (with FP8 dispatch rows, the bf16 rows
 * they were quantised from); w_router: device bf16 [E, D]; logits: device
 * fp32 [n, E] or NULL (not written); topk_idx, topk_w, counts, expert_off as
 * in moe_route_topk, and the call leaves the same per-block bases in ws for
 * moe_dispatch.  The selection is exact on the logits this call computes
 * (the same rule as moe_route_topk on them).  Requires D % 64 == 0 and
 * E <= 256 (MOE_ERR_UNSUPPORTED otherwise).  n = 0 writes zero counts and
 * offsets. */
MOE_API moe_status moe_router_topk(const moe_plan* plan, int32_t n, const void* x,
                                   const void* w_router, float* logits, int32_t* topk_idx,
                                   float* topk_w, int32_t* counts, int32_t* expert_off, void* ws,
                                   moe_stream_t stream);

/* Dispatch: recv[slot(t, j)] = x[t] (D elements of x_dtype, copied as bytes),
 * recv_scale[slot(t, j)] = x_scale[t] (D / scale_block fp32, when scale_block
 * > 0), slot_of[t, j] = slot(t, j), src_of[slot(t, j)] = t*k + j.
 * Must follow moe_route_topk on the same stream with the same n, topk_idx and
 * ws (the slots come from that call's per-block bases).  x: device [n, D];
 * x_scale: device fp32 [n, D/scale_block] or NULL when scale_block == 0;
 * recv: device [T, D]; recv_scale: device fp32 [T, D/scale_block] or NULL;
 * slot_of: device int32 [n, k]; src_of: device int32 [T] (only filled slots
 * are written). */
MOE_API moe_status moe_dispatch(const moe_plan* plan, int32_t n, const void* x, const float* x_scale,
                        const int32_t* topk_idx, void* recv, float* recv_scale,
                        int32_t* slot_of, int32_t* src_of, void* ws, moe_stream_t stream);

/* Route and dispatch in one call: the results of moe_route_topk followed by
 * moe_dispatch with the same arguments, bit for bit (same buffers, same
 * layouts, same errors).  For n <= 1024 tokens both run in ONE launch: the
 * decode-size step where fixed per-launch costs outweigh the bytes moved (the
 * small-batch regime of "One-Sided Expert-Parallel All-to-All for Mixture-of-
 * Experts Inference over NVLink", abstract): a cooperative launch in which
 * each block routes and scatters its own tokens, with a single grid barrier
 * between routing and scattering.  Larger n runs the two kernels.  Unlike
 * moe_route_topk, the one-launch form leaves no per-block bases in ws for a
 * later moe_dispatch.  n = 0 writes zero counts and offsets only.  No
 * counterpart call on the pages: it fuses two of their steps. */
MOE_API moe_status moe_route_dispatch(const moe_plan* plan, int32_t n, const float* logits,
                                      const void* x, const float* x_scale, int32_t* topk_idx,
                                      float* topk_w, int32_t* counts, int32_t* expert_off,
                                      void* recv, float* recv_scale, int32_t* slot_of,
                                      int32_t* src_of, void* ws, moe_stream_t stream);

/* Identity expert for FP8 rows: Y[s, c] = round_y(code[s, c] * recv_scale[s,
 * c / scale_block]) for every filled slot s = slot_of[t, j], correctly rounded
 * (to nearest even) from the exact product.  recv: device e4m3 [T, D];
 * recv_scale: device fp32 [T, D/scale_block] (NULL = scale 1); y: device
 * bf16 [T, D].  Plans whose x_dtype is not FP8 or whose y_dtype is not BF16
 * get MOE_ERR_UNSUPPORTED. */
MOE_API moe_status moe_expert_dequant(const moe_plan* plan, int32_t n, const void* recv,
                              const float* recv_scale, const int32_t* slot_of, void* y,
                              void* ws, moe_stream_t stream);

/* SwiGLU experts read in place from the rank-major buffer: for every expert e
 * and row s in [expert_off[e], expert_off[e] + counts[e]):
 *   h[s, :] = bf16( silu(recv[s] . Wg[e]^T) * (recv[s] . Wu[e]^T) ),
 *   y[s, :] = bf16( h[s] . Wd[e]^T ),   silu(z) = z / (1 + exp(-z)),
 * fp32 accumulation on the tensor cores.  w_gate_up: device bf16 [E, 2I, D]
 * (rows [0, I) are Wg[e], rows [I, 2I) are Wu[e]); w_down: device bf16
 * [E, D, I]; recv: device bf16 [T, D]; h: device bf16 [T, I]; y: device bf16
 * [T, D].  counts and expert_off as written by moe_route_topk.  Plans with
 * bf16 rows only (FP8 rows: moe_expert_swiglu_fp8). */
MOE_API moe_status moe_expert_swiglu(const moe_plan* plan, int32_t n, const void* recv,
                             const int32_t* counts, const int32_t* expert_off,
                             const void* w_gate_up, const void* w_down, void* h, void* y,
                             void* ws, moe_stream_t stream);

/* FP8 SwiGLU experts read in place from the FP8 rank-major buffer and its
 * scales (plans with x = FP8, scale_block = 128, inter > 0).  The pages fix
 * no FP8 GEMM format; this one takes e4m3 weights with one fp32 scale per
 * 128x128 tile, the 128-column granularity of the dispatched rows.  For every
 * expert e and row s in [expert_off[e], expert_off[e] + counts[e]), with
 * X[s, d] = recv[s, d] * recv_scale[s, d/128] and W = code * tile scale:
 *   h[s, c]  = bf16( silu(X[s] . Wg[e][c]) * (X[s] . Wu[e][c]) )
 *   hs[s, b] = amax(h[s, 128b .. 128b+127]) / 448 (fp32 quotient; 1 if zero)
 *   hq[s, c] = e4m3(h[s, c] / hs[s, c/128]), nearest even, saturating at 448
 *   y[s, c]  = bf16( sum_d hq[s, d] hs[s, d/128] * Wd[e][c, d] )
 * fp32 accumulation: the tensor cores sum each 128-column block of codes and
 * the block's scales are applied in fp32.  recv: device e4m3 [T, D];
 * recv_scale: device fp32 [T, D/128]; w_gate_up: device e4m3 [E, 2I, D] (rows
 * [0, I) Wg, [I, 2I) Wu) with w_gate_up_scale fp32 [E, 2I/128, D/128];
 * w_down: device e4m3 [E, D, I] with w_down_scale fp32 [E, D/128, I/128];
 * h: device bf16 [T, I]; hq: device e4m3 [T, I]; h_scale: device fp32
 * [T, I/128]; y: device bf16 [T, D].  counts, expert_off and slot_of as
 * written by moe_route_topk + moe_dispatch (or moe_route_dispatch). */
MOE_API moe_status moe_expert_swiglu_fp8(const moe_plan* plan, int32_t n, const void* recv,
                                         const float* recv_scale, const int32_t* counts,
                                         const int32_t* expert_off, const int32_t* slot_of,
                                         const void* w_gate_up, const float* w_gate_up_scale,
                                         const void* w_down, const float* w_down_scale, void* h,
                                         void* hq, float* h_scale, void* y, void* ws,
                                         moe_stream_t stream);

/* Combine: out[t, c] = sum_{j=0}^{k-1} topk_w[t, j] * Y[slot_of[t, j], c],
 * accumulated in fp32 with fused multiply-adds in increasing j, then rounded
 * to nearest even into out_dtype.  y: device y_dtype [T, D]; topk_w: device
 * fp32 [n, k]; slot_of: device int32 [n, k]; out: device out_dtype [n, D]. */
MOE_API moe_status moe_combine(const moe_plan* plan, int32_t n, const void* y, const float* topk_w,
                       const int32_t* slot_of, void* out, void* ws, moe_stream_t stream);

/* The whole layer on one stream: route -> dispatch -> expert -> combine,
 * route and dispatch through moe_route_dispatch (one launch up to 1024
 * tokens).  Experts are SwiGLU when desc.inter > 0 (w_gate_up, w_down as in
 * moe_expert_swiglu), else identity (FP8 rows dequantised to bf16, so then
 * y_dtype must be BF16; other rows read as Y directly, so then y_dtype must
 * equal x_dtype; MOE_ERR_UNSUPPORTED otherwise).  logits: device fp32
 * [n, E]; x, x_scale as in moe_dispatch; out: device out_dtype [n, D];
 * ws: moe_layer_workspace_bytes() of zero-filled device memory, which holds
 * every intermediate (see moe_layer_buffer).  Every argument error is
 * returned before the first stage is enqueued. */
MOE_API moe_status moe_layer(const moe_plan* plan, int32_t n, const float* logits, const void* x,
                     const float* x_scale, const void* w_gate_up, const void* w_down,
                     void* out, void* ws, moe_stream_t stream);

/* moe_layer for plans with FP8 experts (x = FP8, inter > 0), which need the
 * weight scales of moe_expert_swiglu_fp8; moe_layer returns
 * MOE_ERR_UNSUPPORTED for such plans and this call for any other plan. */
MOE_API moe_status moe_layer_fp8(const moe_plan* plan, int32_t n, const float* logits,
                                 const void* x, const float* x_scale, const void* w_gate_up,
                                 const float* w_gate_up_scale, const void* w_down,
                                 const float* w_down_scale, void* out, void* ws,
                                 moe_stream_t stream);

/* Where moe_layer keeps an intermediate inside its workspace, so a caller
 * can read it after the call: returns ws + byte offset, or NULL for an
 * unknown name.  Names: "topk_idx", "topk_w", "counts", "expert_off",
 * "slot_of", "src_of", "recv", "recv_scale", "y", "h", and with FP8 experts
 * "hq", "h_scale". */
MOE_API void* moe_layer_buffer(const moe_plan* plan, void* ws, const char* name);

/* Read and clear the device status word of `ws`: synchronises `stream`,
 * returns MOE_OK or the first device-detected error since the last call
 * (MOE_ERR_CUDA if the copy itself fails). */
MOE_API moe_status moe_get_status(const moe_plan* plan, void* ws, moe_stream_t stream);

/* Zero the control words, the route kernel's expert totals and the fused
 * kernel's token masks of a workspace (an alternative to zero-filling it),
 * enqueued on `stream`.  Required again after a call reported
 * MOE_ERR_TIMEOUT or a launch in the workspace's stream failed. */
MOE_API moe_status moe_workspace_init(const moe_plan* plan, void* ws, moe_stream_t stream);

/* Bytes of the fixed scratch array that moe_route_topk_noalloc uses. */
#define MOE_NOALLOC_SCRATCH_BYTES (1u << 20)

/* No counterpart in the method's description: a convenience of this library.
 * The same routing as moe_route_topk (same outputs, same layout) for callers
 * that cannot allocate device memory for a workspace -- for instance a plugin
 * whose host framework owns every device allocation and hands out none, or
 * code that must not allocate once it is running.  Its scratch (control
 * words, per-block tables, ranks) is one array of MOE_NOALLOC_SCRATCH_BYTES
 * compiled into this library, which every GPU that loads the library keeps
 * until the process exits; the call allocates and frees nothing.
 * moe_route_topk_noalloc_bytes(plan, n) is the scratch a call with n tokens
 * needs; larger calls return MOE_ERR_WORKSPACE before enqueueing anything.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  All calls on a device share the one array, so calls that overlap
 * on the GPU (other streams, other host threads) race and corrupt each
 * other: order them.  Each call clears the words that must start at zero.
 * Device-detected errors are recorded in the array, where moe_get_status
 * cannot see them: moe_route_topk_noalloc_status reads them (for the most
 * recent call on the current device; each call starts from MOE_OK).  The
 * per-block tables stay inside the array, so this call's routing cannot feed
 * moe_dispatch.  The array's device address is looked up once per device and
 * kept for the life of the process: after a cudaDeviceReset (or anything
 * else that destroys the device's primary context) it is stale, so do not
 * call these two entry points on that device again in the same process. */
MOE_API size_t moe_route_topk_noalloc_bytes(const moe_plan* plan, int32_t n);
MOE_API moe_status moe_route_topk_noalloc(const moe_plan* plan, int32_t n, const float* logits,
                                          int32_t* topk_idx, float* topk_w, int32_t* counts,
                                          int32_t* expert_off, moe_stream_t stream);
/* The device-detected status of the most recent moe_route_topk_noalloc call
 * on the current device: synchronises `stream` (which must be ordered after
 * that call) and returns MOE_OK or the first error that call recorded. */
MOE_API moe_status moe_route_topk_noalloc_status(moe_stream_t stream);

/* Human-readable name of a status code (static string). */
MOE_API const char* moe_strerror(moe_status status);

#ifdef __cplusplus
}
#endif
#endif /* MOEROUTE_H */
