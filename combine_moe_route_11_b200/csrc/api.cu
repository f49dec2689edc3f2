// C ABI of libmoeroute: plan validation, workspace layout and the entry
// points declared in include/moeroute.h.  Host code only; every step of the
// path runs in the kernels of route.cu, router_gemm.cu, route_dispatch.cu,
// dispatch.cu, combine.cu, swiglu_gemm.cu, fp8_gemm.cu and route_noalloc.cu.  The per-device caches
// here and in the launchers may be reached from several host threads.
#include "moe_internal.cuh"

#include <atomic>
#include <mutex>

#include <string.h>
#include <new>

namespace moe {

int num_sms() {
  // per device; a race only computes the same value twice
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < 64) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
    v = 148;
  if (dev < 64) cached[dev].store(v, std::memory_order_relaxed);
  return v;
}

cudaError_t set_smem_limit(const void* kernel, int bytes) {
  // (kernel, device) pairs already raised; a handful of kernels, few devices
  static std::mutex mu;
  static const void* done_k[64];
  static int done_d[64];
  static int done_n = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < done_n; ++i)
    if (done_k[i] == kernel && done_d[i] == dev) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && done_n < 64) {
    done_k[done_n] = kernel;
    done_d[done_n] = dev;
    ++done_n;
  }
  return e;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

Layout make_layout(const moe_plan& p) {
  const moe_desc& d = p.d;
  Layout L;
  size_t at = 0;
  auto take = [&](size_t bytes) {
    const size_t here = at;
    at = align256(at + bytes);
    return here;
  };
  L.ctrl = take(sizeof(Ctrl));
  // right after ctrl, cleared with it by moe_workspace_init: the fused
  // kernel's token masks [2, mask rows, E] (alternate halves by its
  // grid-barrier generation)
  L.masks = take(size_t(2) * mask_rows(p) * d.n_experts * 4);
  // the route kernel's per-expert totals [2, E], also cleared there: a call
  // adds into one half and clears the other for the next call
  L.totals = take(size_t(2) * d.n_experts * 4);
  L.blk = take(size_t(p.blocks_max) * d.n_experts * 4);
  L.bases = take(size_t(p.blocks_max) * d.n_experts * 4);
  L.rank = take(size_t(d.n_max) * d.top_k);
  L.route_end = at;
  const size_t nk = size_t(d.n_max) * d.top_k;
  const size_t T = size_t(p.total_max);
  L.topk_idx = take(nk * 4);
  L.topk_w = take(nk * 4);
  L.counts = take(size_t(d.n_experts) * 4);
  L.expert_off = take(size_t(d.n_experts + 1) * 4);
  L.slot_of = take(nk * 4);
  L.src_of = take(T * 4);
  L.recv = take(T * d.hidden * elem_bytes(d.x_dtype));
  L.recv_scale = take(T * p.scale_cols * 4);
  const bool needs_y = d.inter > 0 || d.x_dtype == MOE_FP8_E4M3;
  const bool fp8_experts = d.inter > 0 && d.x_dtype == MOE_FP8_E4M3;
  L.y = take(needs_y ? T * d.hidden * elem_bytes(d.y_dtype) : 0);
  L.h = take(d.inter > 0 ? T * size_t(d.inter) * 2 : 0);
  L.hq = take(fp8_experts ? T * size_t(d.inter) : 0);
  L.h_scale = take(fp8_experts ? T * size_t(d.inter / 128) * 4 : 0);
  L.end = at;
  return L;
}

moe_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  if (e == cudaErrorNotSupported) return MOE_ERR_UNSUPPORTED;
  return MOE_ERR_CUDA;
}

moe_status check_call(const moe_plan* p, int32_t n, const void* ws) {
  if (!p || n < 0 || n > p->d.n_max) return MOE_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_plan_create(const moe_desc* desc, moe_plan** out) {
  if (!desc || !out) return MOE_ERR_INVALID_ARG;
  const moe_desc d = *desc;
  if (d.n_max < 1 || d.hidden < 1 || d.n_experts < 1 || d.top_k < 1 || d.n_ranks < 1)
    return MOE_ERR_INVALID_ARG;
  if (d.n_experts > kMaxExperts || d.top_k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
  if (d.top_k > d.n_experts || d.n_experts % d.n_ranks != 0) return MOE_ERR_INVALID_ARG;
  auto dtype_ok = [](int t) { return t == MOE_F32 || t == MOE_BF16 || t == MOE_FP8_E4M3; };
  if (!dtype_ok(d.x_dtype) || !dtype_ok(d.y_dtype) || !dtype_ok(d.out_dtype))
    return MOE_ERR_INVALID_ARG;
  if (d.y_dtype == MOE_FP8_E4M3 || d.out_dtype == MOE_FP8_E4M3) return MOE_ERR_UNSUPPORTED;
  // every row is a whole number of 16-byte vectors
  if ((int64_t(d.hidden) * elem_bytes(d.x_dtype)) % 16 ||
      (int64_t(d.hidden) * elem_bytes(d.y_dtype)) % 16 ||
      (int64_t(d.hidden) * elem_bytes(d.out_dtype)) % 16)
    return MOE_ERR_INVALID_ARG;
  if (d.scale_block < 0) return MOE_ERR_INVALID_ARG;
  if (d.scale_block > 0) {
    if (d.x_dtype != MOE_FP8_E4M3) return MOE_ERR_INVALID_ARG;
    if (d.hidden % d.scale_block || d.scale_block % 16) return MOE_ERR_INVALID_ARG;
  }
  if (d.inter < 0) return MOE_ERR_INVALID_ARG;
  if (d.inter > 0) {
    // bf16 experts on bf16 rows, or FP8 experts on FP8 rows with 128-column scales
    const bool fp8 = d.x_dtype == MOE_FP8_E4M3;
    if ((d.x_dtype != MOE_BF16 && !fp8) || d.y_dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (fp8 && d.scale_block != 128) return MOE_ERR_UNSUPPORTED;
    if (d.hidden % 256 || d.inter % 128) return MOE_ERR_UNSUPPORTED;
  }
  moe_plan tmp;
  tmp.d = d;
  tmp.scale_cols = d.scale_block > 0 ? d.hidden / d.scale_block : 0;
  tmp.blocks_max = route_blocks(d.n_max);
  const int64_t T = total_rows(tmp, d.n_max);
  if (T >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  // the route kernel indexes its [blocks, E] tables with 32-bit offsets
  if (int64_t(tmp.blocks_max) * d.n_experts >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  tmp.total_max = T;
  tmp.lay = make_layout(tmp);
  moe_plan* p = new (std::nothrow) moe_plan(tmp);
  if (!p) return MOE_ERR_INVALID_ARG;
  *out = p;
  return MOE_OK;
}

void moe_plan_destroy(moe_plan* plan) { delete plan; }

size_t moe_workspace_bytes(const moe_plan* p) { return p ? p->lay.route_end : 0; }
size_t moe_layer_workspace_bytes(const moe_plan* p) { return p ? p->lay.end : 0; }

int64_t moe_region_rows(const moe_plan* p, int32_t n) {
  if (!p || n < 0 || n > p->d.n_max) return -1;
  return region_rows(*p, n);
}

int64_t moe_recv_rows(const moe_plan* p, int32_t n) {
  if (!p || n < 0 || n > p->d.n_max) return -1;
  return total_rows(*p, n);
}

moe_status moe_route_topk(const moe_plan* p, int32_t n, const float* logits, int32_t* topk_idx,
                          float* topk_w, int32_t* counts, int32_t* expert_off, void* ws,
                          moe_stream_t stream) {
  moe_status s = check_call(p, n, ws);
  if (s != MOE_OK) return s;
  if (!counts || !expert_off || (n > 0 && (!logits || !topk_idx || !topk_w)))
    return MOE_ERR_INVALID_ARG;
  if (n > 0 && !aligned16(logits)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_route(*p, n, logits, topk_idx, topk_w, counts, expert_off, ws,
                                  reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_router_topk(const moe_plan* p, int32_t n, const void* x, const void* w_router,
                           float* logits, int32_t* topk_idx, float* topk_w, int32_t* counts,
                           int32_t* expert_off, void* ws, moe_stream_t stream) {
  moe_status s = check_call(p, n, ws);
  if (s != MOE_OK) return s;
  if (p->d.hidden % 64 != 0 || p->d.n_experts > 256) return MOE_ERR_UNSUPPORTED;
  if (!counts || !expert_off || (n > 0 && (!x || !w_router || !topk_idx || !topk_w)))
    return MOE_ERR_INVALID_ARG;
  if (n > 0 && (!aligned16(x) || !aligned16(w_router))) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  s = cuda_status(launch_router(*p, n, x, w_router, logits, topk_idx, topk_w, ws, st));
  if (s != MOE_OK) return s;
  return cuda_status(launch_route_counts(*p, n, topk_idx, counts, expert_off, ws, st));
}

moe_status moe_dispatch(const moe_plan* p, int32_t n, const void* x, const float* x_scale,
                        const int32_t* topk_idx, void* recv, float* recv_scale, int32_t* slot_of,
                        int32_t* src_of, void* ws, moe_stream_t stream) {
  moe_status s = check_call(p, n, ws);
  if (s != MOE_OK) return s;
  if (n == 0) return MOE_OK;
  if (!x || !topk_idx || !recv || !slot_of || !src_of) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(recv)) return MOE_ERR_INVALID_ARG;
  if (p->scale_cols > 0 && (!x_scale || !recv_scale)) return MOE_ERR_INVALID_ARG;
  if (p->scale_cols > 0 && (!aligned16(x_scale) || !aligned16(recv_scale)))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_dispatch(*p, n, x, x_scale, topk_idx, recv, recv_scale, slot_of,
                                     src_of, ws, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_route_dispatch(const moe_plan* p, int32_t n, const float* logits, const void* x,
                              const float* x_scale, int32_t* topk_idx, float* topk_w,
                              int32_t* counts, int32_t* expert_off, void* recv, float* recv_scale,
                              int32_t* slot_of, int32_t* src_of, void* ws, moe_stream_t stream) {
  moe_status s = check_call(p, n, ws);
  if (s != MOE_OK) return s;
  if (!counts || !expert_off) return MOE_ERR_INVALID_ARG;
  if (n > 0) {
    if (!logits || !topk_idx || !topk_w || !x || !recv || !slot_of || !src_of)
      return MOE_ERR_INVALID_ARG;
    if (!aligned16(logits) || !aligned16(x) || !aligned16(recv)) return MOE_ERR_INVALID_ARG;
    if (p->scale_cols > 0 && (!x_scale || !recv_scale)) return MOE_ERR_INVALID_ARG;
    if (p->scale_cols > 0 && (!aligned16(x_scale) || !aligned16(recv_scale)))
      return MOE_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (route_blocks(n) <= kFusedMaxBlocks)
    return cuda_status(launch_route_dispatch(*p, n, logits, x, x_scale, topk_idx, topk_w, counts,
                                             expert_off, recv, recv_scale, slot_of, src_of, ws,
                                             st));
  s = cuda_status(launch_route(*p, n, logits, topk_idx, topk_w, counts, expert_off, ws, st));
  if (s != MOE_OK) return s;
  return cuda_status(launch_dispatch(*p, n, x, x_scale, topk_idx, recv, recv_scale, slot_of,
                                     src_of, ws, st));
}

moe_status moe_expert_dequant(const moe_plan* p, int32_t n, const void* recv,
                              const float* recv_scale, const int32_t* slot_of, void* y, void* ws,
                              moe_stream_t stream) {
  moe_status s = check_call(p, n, ws);
  if (s != MOE_OK) return s;
  if (p->d.x_dtype != MOE_FP8_E4M3 || p->d.y_dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (n == 0) return MOE_OK;
  if (!recv || !slot_of || !y || !aligned16(recv) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  if (p->scale_cols > 0 && !recv_scale) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_dequant(*p, n, recv, p->scale_cols > 0 ? recv_scale : nullptr,
                                    slot_of, y, ws, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_expert_swiglu(const moe_plan* p, int32_t n, const void* recv, const int32_t* counts,
                             const int32_t* expert_off, const void* w_gate_up, const void* w_down,
                             void* h, void* y, void* ws, moe_stream_t stream) {
  moe_status s = check_call(p, n, ws);
  if (s != MOE_OK) return s;
  if (p->d.inter <= 0 || p->d.x_dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (n == 0) return MOE_OK;
  if (!recv || !counts || !expert_off || !w_gate_up || !w_down || !h || !y)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(recv) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(h) ||
      !aligned16(y))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_swiglu(*p, n, recv, counts, expert_off, w_gate_up, w_down, h, y, ws,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_expert_swiglu_fp8(const moe_plan* p, int32_t n, const void* recv,
                                 const float* recv_scale, const int32_t* counts,
                                 const int32_t* expert_off, const int32_t* slot_of,
                                 const void* w_gate_up, const float* w_gate_up_scale,
                                 const void* w_down, const float* w_down_scale, void* h, void* hq,
                                 float* h_scale, void* y, void* ws, moe_stream_t stream) {
  moe_status s = check_call(p, n, ws);
  if (s != MOE_OK) return s;
  if (p->d.inter <= 0 || p->d.x_dtype != MOE_FP8_E4M3) return MOE_ERR_UNSUPPORTED;
  if (n == 0) return MOE_OK;
  if (!recv || !recv_scale || !counts || !expert_off || !slot_of || !w_gate_up ||
      !w_gate_up_scale || !w_down || !w_down_scale || !h || !hq || !h_scale || !y)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(recv) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(h) ||
      !aligned16(hq) || !aligned16(y))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_swiglu_fp8(*p, n, recv, recv_scale, counts, expert_off, slot_of,
                                       w_gate_up, w_gate_up_scale, w_down, w_down_scale, h, hq,
                                       h_scale, y, ws, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_combine(const moe_plan* p, int32_t n, const void* y, const float* topk_w,
                       const int32_t* slot_of, void* out, void* ws, moe_stream_t stream) {
  moe_status s = check_call(p, n, ws);
  if (s != MOE_OK) return s;
  if (n == 0) return MOE_OK;
  if (!y || !topk_w || !slot_of || !out || !aligned16(y) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_combine(*p, n, y, topk_w, slot_of, out, ws,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

void* moe_layer_buffer(const moe_plan* p, void* ws, const char* name) {
  if (!p || !ws || !name) return nullptr;
  const Layout& L = p->lay;
  char* b = static_cast<char*>(ws);
  struct { const char* n; size_t off; } tab[] = {
      {"topk_idx", L.topk_idx}, {"topk_w", L.topk_w},   {"counts", L.counts},
      {"expert_off", L.expert_off}, {"slot_of", L.slot_of}, {"src_of", L.src_of},
      {"recv", L.recv},         {"recv_scale", L.recv_scale}, {"y", L.y}, {"h", L.h},
      {"hq", L.hq},             {"h_scale", L.h_scale}};
  for (auto& e : tab)
    if (strcmp(e.n, name) == 0) return b + e.off;
  return nullptr;
}

}  // extern "C"

namespace {

// route -> dispatch -> expert -> combine on one stream; the weight scales are
// those of FP8 experts (null for bf16 or identity experts).
moe_status layer_impl(const moe_plan* p, int32_t n, const float* logits, const void* x,
                      const float* x_scale, const void* w_gate_up, const float* w_gate_up_scale,
                      const void* w_down, const float* w_down_scale, void* out, void* ws,
                      moe_stream_t stream) {
  moe_status s = check_call(p, n, ws);
  if (s != MOE_OK) return s;
  const moe_desc& d = p->d;
  const bool fp8_experts = d.inter > 0 && d.x_dtype == MOE_FP8_E4M3;
  if (fp8_experts && (!w_gate_up_scale || !w_down_scale)) return MOE_ERR_INVALID_ARG;
  // Every argument error is found here, before the first launch: the stages
  // below only receive pointers into ws (256-byte aligned by the layout) or
  // arguments checked here, so none of them can reject the call halfway.
  if (d.inter == 0 && d.x_dtype != MOE_FP8_E4M3 && d.y_dtype != d.x_dtype)
    return MOE_ERR_UNSUPPORTED;
  if (d.inter == 0 && d.x_dtype == MOE_FP8_E4M3 && d.y_dtype != MOE_BF16)
    return MOE_ERR_UNSUPPORTED;  // the FP8 identity expert writes bf16
  if (d.inter > 0 && (!w_gate_up || !w_down)) return MOE_ERR_INVALID_ARG;
  if (n > 0) {
    if (!logits || !x || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(logits) || !aligned16(x) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    if (p->scale_cols > 0 && (!x_scale || !aligned16(x_scale))) return MOE_ERR_INVALID_ARG;
    if (d.inter > 0 && (!aligned16(w_gate_up) || !aligned16(w_down))) return MOE_ERR_INVALID_ARG;
  }
  char* b = static_cast<char*>(ws);
  const Layout& L = p->lay;
  int32_t* topk_idx = reinterpret_cast<int32_t*>(b + L.topk_idx);
  float* topk_w = reinterpret_cast<float*>(b + L.topk_w);
  int32_t* counts = reinterpret_cast<int32_t*>(b + L.counts);
  int32_t* expert_off = reinterpret_cast<int32_t*>(b + L.expert_off);
  int32_t* slot_of = reinterpret_cast<int32_t*>(b + L.slot_of);
  int32_t* src_of = reinterpret_cast<int32_t*>(b + L.src_of);
  void* recv = b + L.recv;
  float* recv_scale = p->scale_cols > 0 ? reinterpret_cast<float*>(b + L.recv_scale) : nullptr;
  void* y = b + L.y;
  void* h = b + L.h;
  s = moe_route_dispatch(p, n, logits, x, x_scale, topk_idx, topk_w, counts, expert_off, recv,
                         recv_scale, slot_of, src_of, ws, stream);
  if (s != MOE_OK || n == 0) return s;
  const void* yin = recv;
  if (fp8_experts) {
    s = moe_expert_swiglu_fp8(p, n, recv, recv_scale, counts, expert_off, slot_of, w_gate_up,
                              w_gate_up_scale, w_down, w_down_scale, h, b + L.hq,
                              reinterpret_cast<float*>(b + L.h_scale), y, ws, stream);
    yin = y;
  } else if (d.inter > 0) {
    s = moe_expert_swiglu(p, n, recv, counts, expert_off, w_gate_up, w_down, h, y, ws, stream);
    yin = y;
  } else if (d.x_dtype == MOE_FP8_E4M3) {
    s = moe_expert_dequant(p, n, recv, recv_scale, slot_of, y, ws, stream);
    yin = y;
  }
  if (s != MOE_OK) return s;
  return moe_combine(p, n, yin, topk_w, slot_of, out, ws, stream);
}

}  // namespace

extern "C" {

moe_status moe_layer(const moe_plan* p, int32_t n, const float* logits, const void* x,
                     const float* x_scale, const void* w_gate_up, const void* w_down, void* out,
                     void* ws, moe_stream_t stream) {
  // FP8 experts need their weight scales: moe_layer_fp8
  if (p && p->d.inter > 0 && p->d.x_dtype == MOE_FP8_E4M3) return MOE_ERR_UNSUPPORTED;
  return layer_impl(p, n, logits, x, x_scale, w_gate_up, nullptr, w_down, nullptr, out, ws,
                    stream);
}

moe_status moe_layer_fp8(const moe_plan* p, int32_t n, const float* logits, const void* x,
                         const float* x_scale, const void* w_gate_up, const float* w_gate_up_scale,
                         const void* w_down, const float* w_down_scale, void* out, void* ws,
                         moe_stream_t stream) {
  if (p && !(p->d.inter > 0 && p->d.x_dtype == MOE_FP8_E4M3)) return MOE_ERR_UNSUPPORTED;
  return layer_impl(p, n, logits, x, x_scale, w_gate_up, w_gate_up_scale, w_down, w_down_scale,
                    out, ws, stream);
}

moe_status moe_get_status(const moe_plan* p, void* ws, moe_stream_t stream) {
  if (!p || !ws) return MOE_ERR_INVALID_ARG;
  Ctrl* c = reinterpret_cast<Ctrl*>(ws);
  int v = 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&v, &c->status, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  if (v != 0 && cudaMemsetAsync(&c->status, 0, sizeof(int), st) != cudaSuccess) return MOE_ERR_CUDA;
  return static_cast<moe_status>(v);
}

moe_status moe_workspace_init(const moe_plan* p, void* ws, moe_stream_t stream) {
  if (!p || !ws) return MOE_ERR_INVALID_ARG;
  // control words and token masks (which follow them)
  return cudaMemsetAsync(ws, 0, p->lay.blk, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

const char* moe_strerror(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_WORKSPACE: return "workspace too small or misaligned";
    case MOE_ERR_DEVICE_INDEX: return "device saw an expert id or slot out of range";
    case MOE_ERR_TIMEOUT: return "bounded device-side wait timed out";
    case MOE_ERR_NONFINITE: return "logit row with fewer than top_k finite values";
  }
  return "unknown status";
}

}  // extern "C"
