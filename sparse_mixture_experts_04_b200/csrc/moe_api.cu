// C ABI of libmoe_b200 (declared in include/moe_b200.h): argument checks,
// workspace layout and the launch sequence of each entry point.  Host code
// only; every step of the layer runs in the kernels of router.cu, dispatch.cu,
// expert_gemm.cu and combine.cu.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "../../include/moe_b200.h"
#include "common.cuh"
#include "internal.h"

namespace moe {

int num_sms() {
  static std::mutex mu;
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = getenv("MOE_B200_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

static size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

WsLayout make_layout(const Problem& p) {
  WsLayout L{};
  const size_t es = p.esize();
  const size_t TK = static_cast<size_t>(p.T) * p.K;
  const size_t R = static_cast<size_t>(p.max_rows);
  L.n_chunks = static_cast<int>((p.T + kDispatchChunk - 1) / kDispatchChunk);
  L.n_sel_blocks = static_cast<int>((p.T + kSelectTokens - 1) / kSelectTokens);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + (bytes ? bytes : 1));
    return o;
  };
  // status word, chunk histogram and chunk p sums first: one memset clears them
  const size_t ce = static_cast<size_t>(L.n_chunks) * p.E;
  L.status = 0;
  L.chunk_psum = 256;                              // 8-byte entries
  L.chunk_counts = align256(L.chunk_psum + ce * 8);
  L.zero_bytes = L.chunk_counts + ce * 4;
  off = align256(L.zero_bytes);
  L.logits = take(static_cast<size_t>(p.T) * p.E * 4);
  L.topk_idx = take(TK * 4);
  L.topk_w = take(TK * 4);
  L.counts = take(static_cast<size_t>(p.E) * 4);
  L.kept = take(static_cast<size_t>(p.E) * 4);
  L.seg_off = take(static_cast<size_t>(p.E + 1) * 4);
  L.slot_of = take(TK * 4);
  L.perm = take(R * 4);
  L.chunk_base = take(static_cast<size_t>(L.n_chunks) * p.E * 4);
  const int splits = (p.dtype == kBF16) ? router_k_splits(p) : 1;
  L.logit_parts = take(splits > 1 ? static_cast<size_t>(splits) * p.T * p.E * 4 : 0);
  // z-loss partials: one per selection block, or one per CTA of the fused router
  const size_t n_zp = std::max<size_t>(static_cast<size_t>(L.n_sel_blocks), static_cast<size_t>((p.T + 127) / 128) * 8);
  L.zpart = take(n_zp * 4);
  L.seg_map = take(static_cast<size_t>(2 * kMaxSegments + 1) * 4);
  L.x_perm = take(R * p.d * es);
  L.h_routed = take(R * p.F * es);
  L.y_perm = take(R * p.d * es);
  L.h_shared = take(static_cast<size_t>(p.T) * p.Ns * p.F * es);
  L.y_shared = take(p.Ns > 0 ? static_cast<size_t>(p.T) * p.d * es : 0);
  const bool save_gu = (p.flags & MOE_FLAG_SAVE_GU) && p.dtype == kBF16;
  L.gu_routed = take(save_gu ? R * 2 * p.F * es : 0);
  L.gu_shared = take(save_gu ? static_cast<size_t>(p.T) * p.Ns * 2 * p.F * es : 0);
  L.total = off;
  return L;
}

static bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// Validate the problem and derive cap / max_rows.  Returns MOE_OK or an error.
static int to_problem(const moe_problem_t* in, Problem* out) {
  if (!in) return MOE_ERR_INVALID_ARG;
  const moe_problem_t& q = *in;
  if (q.T < 1 || q.d_model < 8 || q.d_ff < 8 || (q.d_model % 8) || (q.d_ff % 8)) return MOE_ERR_INVALID_ARG;
  if (q.n_experts < 1 || q.top_k < 1 || q.top_k > q.n_experts || q.n_shared < 0) return MOE_ERR_INVALID_ARG;
  if (q.dtype != MOE_DTYPE_BF16 && q.dtype != MOE_DTYPE_F32) return MOE_ERR_INVALID_ARG;
  if (q.flags & ~(MOE_FLAG_LOGITS_GIVEN | MOE_FLAG_BIAS_LOGIT | MOE_FLAG_EXTENDED_STATS | MOE_FLAG_EXPERT_CAPACITY |
                  MOE_FLAG_SAVE_GU))
    return MOE_ERR_INVALID_ARG;
  if (!(q.alpha == q.alpha) || !(q.capacity_factor == q.capacity_factor)) return MOE_ERR_INVALID_ARG;
  if (q.n_experts > kMaxExperts || q.top_k > kMaxTopK || q.n_shared > 256) return MOE_ERR_UNSUPPORTED;
  const int64_t lim = static_cast<int64_t>(1) << 31;
  if (q.T >= lim / q.top_k || q.T >= lim / q.n_experts) return MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(q.d_ff) * (q.n_shared > 0 ? q.n_shared : 1) >= lim) return MOE_ERR_UNSUPPORTED;
  Problem p{};
  p.T = q.T;
  p.d = q.d_model;
  p.E = q.n_experts;
  p.K = q.top_k;
  p.Ns = q.n_shared;
  p.F = q.d_ff;
  p.dtype = q.dtype;
  p.flags = q.flags;
  p.alpha = q.alpha;
  // capacity: ceil(C * (T*K) / E) evaluated in float64; C <= 0 means no limit
  if (q.capacity_factor > 0.0f) {
    const double v = (static_cast<double>(q.capacity_factor) * static_cast<double>(q.T * q.top_k)) /
                     static_cast<double>(q.n_experts);
    const double c = ceil(v);
    p.cap_raw = c >= 4611686018427387904.0 ? (static_cast<int64_t>(1) << 62) : static_cast<int64_t>(c);
    // an expert serves at most T tokens (a token picks it at most once)
    p.cap = p.cap_raw >= q.T ? q.T : p.cap_raw;
  } else {
    p.cap = p.cap_raw = -1;
  }
  const int64_t TK = q.T * q.top_k;
  // per-expert capacities can give any expert up to T rows: only T*K bounds the total
  const bool uniform = !(q.flags & MOE_FLAG_EXPERT_CAPACITY);
  p.max_rows = (p.cap < 0 || !uniform) ? TK : (p.cap * q.n_experts < TK ? p.cap * q.n_experts : TK);
  *out = p;
  return MOE_OK;
}

int problem_from_abi(const moe_problem_t* in, Problem* out) { return to_problem(in, out); }

static int check_ws(const Problem& p, void* ws, size_t ws_bytes) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < make_layout(p).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

template <typename T>
static T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

unsigned long long test_stall_ns() {
  const char* e = getenv("MOE_B200_TEST_STALL_NS");
  if (!e || !e[0]) return 0;
  const unsigned long long v = strtoull(e, nullptr, 10);
  return v > kWaitLimitNs ? kWaitLimitNs : v;
}

// Router body shared by moe_route and moe_layer_forward.
// chunk_totals_cleared: the caller already zeroed the chunk totals;
// stats_in_route: finalise the statistics here (else the dispatch scan does).
// *n_zpart: number of z-loss partials written (for the statistics);
// *n_kernels (if given) += kernels enqueued.
static int route_impl(const Problem& p, const void* x, const void* w_gate, const float* offset,
                      const float* sel_bias, float* logits, int32_t* idx, float* w, float* stats, void* ws,
                      const WsLayout& L, cudaStream_t st, bool chunk_totals_cleared, bool stats_in_route,
                      int* n_zpart, int* n_kernels, unsigned long long* clk = nullptr) {
  unsigned* status = at<unsigned>(ws, L.status);
  // the chunk totals start at zero: the layer forward clears them with the
  // status word; a standalone call clears them here
  if (!chunk_totals_cleared) {
    if (cudaError_t e = cudaMemsetAsync(at<char>(ws, L.chunk_psum), 0, L.zero_bytes - L.chunk_psum, st))
      return cuda_rc(e);
  }
  int32_t* chunk_counts = at<int32_t>(ws, L.chunk_counts);
  unsigned long long* chunk_psum = at<unsigned long long>(ws, L.chunk_psum);
  float* zpart = (stats && (p.flags & MOE_FLAG_EXTENDED_STATS)) ? at<float>(ws, L.zpart) : nullptr;
  int kernels = 0;
  if (router_fused_ok(p)) {
    // the gate GEMM with its split reduction summed on chip; the tokens are
    // ranked in the same kernel, or by the selection kernel right after it
    const bool sel_here = router_selects(p);
    if (cudaError_t e = launch_router_fused(p, x, w_gate, offset, sel_bias, logits, idx, w, chunk_counts, chunk_psum,
                                            zpart, status, st, n_zpart, clk, sel_here))
      return cuda_rc(e);
    kernels += 1;
    if (!sel_here) {
      if (cudaError_t e = launch_route_select(p, logits, nullptr, 0, sel_bias, idx, w, chunk_counts, chunk_psum, zpart,
                                              st, clk))
        return cuda_rc(e);
      kernels += 1;
      *n_zpart = route_select_zparts(p);
    }
  } else {
    int n_parts = 0;
    float* parts = nullptr;
    if (!(p.flags & MOE_FLAG_LOGITS_GIVEN)) {
      if (p.dtype == kBF16) {
        const int splits = router_k_splits(p);
        if (splits > 1) {
          parts = at<float>(ws, L.logit_parts);
          n_parts = splits;
        }
        const int rc =
            launch_gate_logits_tc(p, x, w_gate, offset, splits > 1 ? parts : logits, splits, status, st, clk);
        if (rc) return MOE_ERR_CUDA;
      } else {
        if (cudaError_t e = launch_gate_logits_simt(p, x, w_gate, offset, logits, st)) return cuda_rc(e);
      }
      kernels += 1;
    }
    if (cudaError_t e = launch_route_select(p, logits, parts, n_parts, sel_bias, idx, w, chunk_counts, chunk_psum,
                                            zpart, st, clk))
      return cuda_rc(e);
    kernels += 1;
    *n_zpart = route_select_zparts(p);
  }
  if (stats && stats_in_route) {
    if (cudaError_t e = launch_route_stats(p, chunk_counts, chunk_psum, L.n_chunks, zpart, *n_zpart, stats, st))
      return cuda_rc(e);
    kernels += 1;
  }
  if (n_kernels) *n_kernels += kernels;
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

int moe_abi_version(void) { return MOE_ABI_VERSION; }

const char* moe_status_string(int code) {
  switch (code) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: problem outside this build's limits";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call failed";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK: a kernel reported bad data";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing, too small or not 256-byte aligned";
    default: return "unknown moe_status";
  }
}

int64_t moe_capacity(const moe_problem_t* q) {
  Problem p;
  if (to_problem(q, &p) != MOE_OK) return -2;
  return p.cap_raw;
}

int64_t moe_max_rows(const moe_problem_t* q) {
  Problem p;
  if (to_problem(q, &p) != MOE_OK) return -2;
  return p.max_rows;
}

int moe_workspace_size(const moe_problem_t* q, size_t* bytes) {
  Problem p;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  if (int rc = to_problem(q, &p)) return rc;
  *bytes = make_layout(p).total;
  return MOE_OK;
}

int moe_reset_device_status(void* ws, moe_stream_t stream) {
  if (!ws) return MOE_ERR_WORKSPACE;
  return cuda_rc(cudaMemsetAsync(ws, 0, sizeof(unsigned), reinterpret_cast<cudaStream_t>(stream)));
}

int moe_read_device_status(const void* ws, moe_stream_t stream, uint32_t* bits) {
  if (!ws || !bits) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(unsigned), cudaMemcpyDeviceToHost, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  *bits = v;
  return v ? MOE_ERR_DEVICE_CHECK : MOE_OK;
}

int moe_route(const moe_problem_t* q, const void* x, const void* w_gate, const float* logit_offset,
              const float* sel_bias, float* logits, int32_t* topk_idx, float* topk_w, float* stats, void* ws,
              size_t ws_bytes, moe_stream_t stream) {
  Problem p;
  if (int rc = to_problem(q, &p)) return rc;
  if (int rc = check_ws(p, ws, ws_bytes)) return rc;
  const bool given = p.flags & MOE_FLAG_LOGITS_GIVEN;
  if (!logits || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  // the drop figures of the extended statistics need the capacities the dispatch will use
  if ((p.flags & MOE_FLAG_EXTENDED_STATS) && (p.flags & MOE_FLAG_EXPERT_CAPACITY)) return MOE_ERR_INVALID_ARG;
  if (!given && (!x || !w_gate || !aligned16(x) || !aligned16(w_gate))) return MOE_ERR_INVALID_ARG;
  const WsLayout L = make_layout(p);
  int n_zpart = 0;
  return route_impl(p, x, w_gate, given ? nullptr : logit_offset, sel_bias, logits, topk_idx, topk_w, stats, ws,
                    L, reinterpret_cast<cudaStream_t>(stream), /*chunk_totals_cleared=*/false,
                    /*stats_in_route=*/true, &n_zpart, nullptr);
}

static int dispatch_entry(const moe_problem_t* q, const int32_t* topk_idx, const int32_t* expert_cap,
                          const void* x, int32_t* counts, int32_t* kept, int32_t* seg_off, int32_t* slot_of,
                          int32_t* perm, void* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  Problem p;
  if (int rc = to_problem(q, &p)) return rc;
  if (int rc = check_ws(p, ws, ws_bytes)) return rc;
  if (!topk_idx || !counts || !kept || !seg_off || !slot_of || !perm) return MOE_ERR_INVALID_ARG;
  if (x_perm && (!x || !aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  if (((p.flags & MOE_FLAG_EXPERT_CAPACITY) != 0) != (expert_cap != nullptr)) return MOE_ERR_INVALID_ARG;
  if (expert_cap && !aligned16(expert_cap)) return MOE_ERR_INVALID_ARG;
  const WsLayout L = make_layout(p);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaError_t e = launch_dispatch(p, topk_idx, counts, kept, seg_off, slot_of, perm,
                                      at<int32_t>(ws, L.chunk_counts), at<int32_t>(ws, L.chunk_base),
                                      at<unsigned>(ws, L.status), st, false, nullptr, nullptr, nullptr, 0,
                                      expert_cap))
    return cuda_rc(e);
  if (x_perm) {
    if (cudaError_t e = launch_gather(p, x, perm, seg_off, x_perm, st)) return cuda_rc(e);
  }
  return MOE_OK;
}

int moe_dispatch(const moe_problem_t* q, const int32_t* topk_idx, const void* x, int32_t* counts, int32_t* kept,
                 int32_t* seg_off, int32_t* slot_of, int32_t* perm, void* x_perm, void* ws, size_t ws_bytes,
                 moe_stream_t stream) {
  return dispatch_entry(q, topk_idx, nullptr, x, counts, kept, seg_off, slot_of, perm, x_perm, ws, ws_bytes, stream);
}

int moe_dispatch_capacity(const moe_problem_t* q, const int32_t* topk_idx, const int32_t* expert_capacity,
                          const void* x, int32_t* counts, int32_t* kept, int32_t* seg_off, int32_t* slot_of,
                          int32_t* perm, void* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!expert_capacity) return MOE_ERR_INVALID_ARG;
  return dispatch_entry(q, topk_idx, expert_capacity, x, counts, kept, seg_off, slot_of, perm, x_perm, ws, ws_bytes,
                        stream);
}

int moe_balance_update(const moe_problem_t* q, const int32_t* counts, float* sel_bias, float bias_rate,
                       int32_t bias_mode, int32_t* count_hist, int32_t hist_len, int64_t step, float c_base,
                       float gamma, int32_t* expert_capacity, moe_stream_t stream) {
  Problem p;
  if (int rc = to_problem(q, &p)) return rc;
  if (!counts || !aligned16(counts) || (!sel_bias && !expert_capacity)) return MOE_ERR_INVALID_ARG;
  if (sel_bias) {
    if (!aligned16(sel_bias) || !std::isfinite(bias_rate)) return MOE_ERR_INVALID_ARG;
    if (bias_mode != MOE_BIAS_UPDATE_SIGN && bias_mode != MOE_BIAS_UPDATE_PROPORTIONAL) return MOE_ERR_INVALID_ARG;
  }
  int slot = 0, rows = 0;
  if (expert_capacity) {
    if (!aligned16(expert_capacity) || !count_hist || !aligned16(count_hist)) return MOE_ERR_INVALID_ARG;
    if (hist_len < 1 || step < 0 || !std::isfinite(c_base) || !(c_base > 0.0f) || !std::isfinite(gamma))
      return MOE_ERR_INVALID_ARG;
    slot = static_cast<int>(step % hist_len);
    rows = step + 1 < hist_len ? static_cast<int>(step + 1) : hist_len;
  }
  return cuda_rc(launch_balance_update(p, counts, sel_bias, bias_rate, bias_mode, expert_capacity ? count_hist : nullptr,
                                       slot, rows, c_base, gamma, expert_capacity,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

int moe_expert_ffn(const moe_problem_t* q, int32_t mode, const void* x_rows, int64_t n_rows,
                   const int32_t* seg_off, const void* w13, const void* w2, void* y_rows, void* ws, size_t ws_bytes,
                   moe_stream_t stream) {
  Problem p;
  if (int rc = to_problem(q, &p)) return rc;
  if (int rc = check_ws(p, ws, ws_bytes)) return rc;
  if (mode != MOE_FFN_ROUTED && mode != MOE_FFN_SHARED) return MOE_ERR_INVALID_ARG;
  if (!x_rows || !w13 || !w2 || !y_rows || n_rows < 1) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_rows) || !aligned16(w13) || !aligned16(w2) || !aligned16(y_rows)) return MOE_ERR_INVALID_ARG;
  if (mode == MOE_FFN_ROUTED && (!seg_off || n_rows > p.max_rows)) return MOE_ERR_INVALID_ARG;
  if (mode == MOE_FFN_SHARED && (p.Ns < 1 || n_rows > p.T)) return MOE_ERR_INVALID_ARG;
  const WsLayout L = make_layout(p);
  void* h = at<void>(ws, mode == MOE_FFN_ROUTED ? L.h_routed : L.h_shared);
  const int rc = launch_expert_ffn(p, mode, x_rows, n_rows, seg_off, w13, w2, h, y_rows, at<unsigned>(ws, L.status),
                                   reinterpret_cast<cudaStream_t>(stream));
  return rc ? MOE_ERR_CUDA : MOE_OK;
}

int moe_expert_ffn_segments(const moe_problem_t* q, const void* x_rows, int64_t n_rows, const int32_t* seg_off,
                            int32_t n_segments, const void* w13, const void* w2, void* y_rows, void* ws,
                            size_t ws_bytes, moe_stream_t stream) {
  Problem p;
  if (int rc = to_problem(q, &p)) return rc;
  if (int rc = check_ws(p, ws, ws_bytes)) return rc;
  if (n_segments < 1 || !seg_off || !x_rows || !w13 || !w2 || !y_rows || n_rows < 1) return MOE_ERR_INVALID_ARG;
  if (n_segments > 256) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x_rows) || !aligned16(w13) || !aligned16(w2) || !aligned16(y_rows)) return MOE_ERR_INVALID_ARG;
  if (n_rows > p.max_rows) return MOE_ERR_INVALID_ARG;
  const WsLayout L = make_layout(p);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned* status = at<unsigned>(ws, L.status);
  if (n_segments <= p.E) {  // at most one segment per expert: run them as they lie
    const int rc = launch_expert_ffn(p, MOE_FFN_ROUTED, x_rows, n_rows, seg_off, w13, w2, at<void>(ws, L.h_routed),
                                     y_rows, status, st, nullptr, nullptr, nullptr, nullptr, nullptr, n_segments);
    return rc ? MOE_ERR_CUDA : MOE_OK;
  }
  // Several segments per expert (a few dozen rows each in the expert-parallel
  // receive buffer): each would end in a part tile that streams the expert's
  // weights again.  So the rows go into expert-major order in the workspace
  // (one group per expert, full tiles), and the outputs back to segment order.
  int32_t* dst_off = at<int32_t>(ws, L.seg_map);
  int32_t* expert_off = dst_off + kMaxSegments;
  const int row_bytes = static_cast<int>(p.d * p.esize());
  if (cudaError_t e = launch_segment_regroup_plan(seg_off, n_segments, p.E, dst_off, expert_off, st)) return cuda_rc(e);
  if (cudaError_t e = launch_segment_copy(x_rows, at<void>(ws, L.x_perm), seg_off, dst_off, n_segments, n_rows,
                                          row_bytes, true, st))
    return cuda_rc(e);
  if (launch_expert_ffn(p, MOE_FFN_ROUTED, at<void>(ws, L.x_perm), n_rows, expert_off, w13, w2,
                        at<void>(ws, L.h_routed), at<void>(ws, L.y_perm), status, st))
    return MOE_ERR_CUDA;
  return cuda_rc(launch_segment_copy(at<void>(ws, L.y_perm), y_rows, seg_off, dst_off, n_segments, n_rows, row_bytes,
                                     false, st));
}

int moe_combine(const moe_problem_t* q, const void* y_perm, const int32_t* slot_of, const float* topk_w,
                const void* y_shared, void* y, void* ws, size_t ws_bytes, moe_stream_t stream) {
  Problem p;
  if (int rc = to_problem(q, &p)) return rc;
  if (int rc = check_ws(p, ws, ws_bytes)) return rc;
  if (!slot_of || !topk_w || !y || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  if (p.max_rows > 0 && (!y_perm || !aligned16(y_perm))) return MOE_ERR_INVALID_ARG;
  if ((p.Ns > 0) != (y_shared != nullptr)) return MOE_ERR_INVALID_ARG;
  if (y_shared && !aligned16(y_shared)) return MOE_ERR_INVALID_ARG;
  return cuda_rc(launch_combine(p, y_perm, slot_of, topk_w, y_shared, y, reinterpret_cast<cudaStream_t>(stream)));
}

static int layer_forward_impl(const moe_problem_t* q, const void* x, const moe_weights_t* w, void* y,
                              const moe_routing_t* routing, float* stats, void* ws, size_t ws_bytes,
                              moe_stream_t stream, void* const* events, int32_t* n_kernels,
                              unsigned long long* clocks) {
  Problem p;
  if (int rc = to_problem(q, &p)) return rc;
  if (int rc = check_ws(p, ws, ws_bytes)) return rc;
  const bool given = p.flags & MOE_FLAG_LOGITS_GIVEN;
  if (!x || !w || !y || !aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  if (!w->w13 || !w->w2 || !aligned16(w->w13) || !aligned16(w->w2)) return MOE_ERR_INVALID_ARG;
  if (!given && (!w->w_gate || !aligned16(w->w_gate))) return MOE_ERR_INVALID_ARG;
  if (given && (!routing || !routing->logits)) return MOE_ERR_INVALID_ARG;
  if (p.Ns > 0 && (!w->w13_shared || !w->w2_shared || !aligned16(w->w13_shared) || !aligned16(w->w2_shared)))
    return MOE_ERR_INVALID_ARG;
  if (p.Ns == 0 && (w->w13_shared || w->w2_shared)) return MOE_ERR_INVALID_ARG;
  const int32_t* expert_cap = (p.flags & MOE_FLAG_EXPERT_CAPACITY) ? w->expert_capacity : nullptr;
  if ((p.flags & MOE_FLAG_EXPERT_CAPACITY) && (!expert_cap || !aligned16(expert_cap))) return MOE_ERR_INVALID_ARG;

  const WsLayout L = make_layout(p);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto mark = [&](int i) -> cudaError_t {
    if (!events || !events[i]) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st);
  };
  int kernels = 0;
  // the stage clock of stage s, or nullptr
  auto clk = [&](int s) -> unsigned long long* { return clocks ? clocks + 2 * s : nullptr; };
  moe_routing_t r{};
  if (routing) r = *routing;
  float* logits = r.logits ? r.logits : at<float>(ws, L.logits);
  int32_t* idx = r.topk_idx ? r.topk_idx : at<int32_t>(ws, L.topk_idx);
  float* gw = r.topk_w ? r.topk_w : at<float>(ws, L.topk_w);
  int32_t* counts = r.counts ? r.counts : at<int32_t>(ws, L.counts);
  int32_t* kept = r.kept ? r.kept : at<int32_t>(ws, L.kept);
  int32_t* seg_off = r.seg_off ? r.seg_off : at<int32_t>(ws, L.seg_off);
  int32_t* slot_of = r.slot_of ? r.slot_of : at<int32_t>(ws, L.slot_of);
  int32_t* perm = r.perm ? r.perm : at<int32_t>(ws, L.perm);
  unsigned* status = at<unsigned>(ws, L.status);
  void* x_perm = at<void>(ws, L.x_perm);
  void* y_perm = at<void>(ws, L.y_perm);
  void* y_sh = p.Ns > 0 ? at<void>(ws, L.y_shared) : nullptr;

  // status word, chunk histogram and chunk p sums (contiguous at offset 0) start at zero
  if (cudaError_t e = cudaMemsetAsync(ws, 0, L.zero_bytes, st)) return cuda_rc(e);
  if (cudaError_t e = mark(MOE_EV_START)) return cuda_rc(e);
  int n_zpart = 0;
  if (int rc = route_impl(p, x, w->w_gate, given ? nullptr : w->logit_offset, w->sel_bias, logits, idx, gw, stats,
                          ws, L, st, /*chunk_totals_cleared=*/true, /*stats_in_route=*/false, &n_zpart, &kernels,
                          clk(MOE_CLOCK_ROUTE)))
    return rc;
  if (cudaError_t e = mark(MOE_EV_ROUTED)) return cuda_rc(e);
  // scan+rank (the histogram came from the selection kernel); the scan also
  // finalises the balance statistics from the chunk totals
  if (cudaError_t e = launch_dispatch(p, idx, counts, kept, seg_off, slot_of, perm, at<int32_t>(ws, L.chunk_counts),
                                      at<int32_t>(ws, L.chunk_base), status, st, /*counts_ready=*/true,
                                      at<unsigned long long>(ws, L.chunk_psum), stats,
                                      (stats && (p.flags & MOE_FLAG_EXTENDED_STATS)) ? at<float>(ws, L.zpart) : nullptr,
                                      n_zpart, expert_cap, clk(MOE_CLOCK_DISPATCH)))
    return cuda_rc(e);
  kernels += dispatch_fused(p) ? 1 : 2;
  if (p.max_rows > 0) {
    if (cudaError_t e = launch_gather(p, x, perm, seg_off, x_perm, st, clk(MOE_CLOCK_GATHER))) return cuda_rc(e);
    kernels += 1;
  }
  if (cudaError_t e = mark(MOE_EV_DISPATCHED)) return cuda_rc(e);
  const bool save_gu = (p.flags & MOE_FLAG_SAVE_GU) && p.dtype == kBF16;
  cudaEvent_t up_ev = (events && events[MOE_EV_UP]) ? static_cast<cudaEvent_t>(events[MOE_EV_UP]) : nullptr;
  if (expert_ffn_mixed_ok(p)) {
    // routed and shared experts in the same two launches; the stage events
    // UP and DOWN then cover both, SHARED follows DOWN at once
    if (launch_expert_ffn_mixed(p, x_perm, seg_off, w->w13, w->w2, at<void>(ws, L.h_routed), y_perm,
                                save_gu ? at<void>(ws, L.gu_routed) : nullptr, x, w->w13_shared, w->w2_shared,
                                at<void>(ws, L.h_shared), y_sh, save_gu ? at<void>(ws, L.gu_shared) : nullptr,
                                status, st, up_ev, &kernels, clk(MOE_CLOCK_UP), clk(MOE_CLOCK_DOWN)))
      return MOE_ERR_CUDA;
    if (cudaError_t e = mark(MOE_EV_DOWN)) return cuda_rc(e);
  } else {
    if (p.max_rows > 0) {
      if (launch_expert_ffn(p, MOE_FFN_ROUTED, x_perm, p.max_rows, seg_off, w->w13, w->w2, at<void>(ws, L.h_routed),
                            y_perm, status, st, up_ev, &kernels, save_gu ? at<void>(ws, L.gu_routed) : nullptr,
                            clk(MOE_CLOCK_UP), clk(MOE_CLOCK_DOWN)))
        return MOE_ERR_CUDA;
    } else if (cudaError_t e = mark(MOE_EV_UP)) {
      return cuda_rc(e);
    }
    if (cudaError_t e = mark(MOE_EV_DOWN)) return cuda_rc(e);
    if (p.Ns > 0) {
      if (launch_expert_ffn(p, MOE_FFN_SHARED, x, p.T, nullptr, w->w13_shared, w->w2_shared,
                            at<void>(ws, L.h_shared), y_sh, status, st, nullptr, &kernels,
                            save_gu ? at<void>(ws, L.gu_shared) : nullptr, clk(MOE_CLOCK_SHARED),
                            clk(MOE_CLOCK_SHARED)))
        return MOE_ERR_CUDA;
    }
  }
  if (cudaError_t e = mark(MOE_EV_SHARED)) return cuda_rc(e);
  if (cudaError_t e = launch_combine(p, y_perm, slot_of, gw, y_sh, y, st, clk(MOE_CLOCK_COMBINE))) return cuda_rc(e);
  kernels += 1;
  if (cudaError_t e = mark(MOE_EV_END)) return cuda_rc(e);
  if (n_kernels) *n_kernels = kernels;
  return MOE_OK;
}

int moe_layer_forward(const moe_problem_t* q, const void* x, const moe_weights_t* w, void* y,
                      const moe_routing_t* routing, float* stats, void* ws, size_t ws_bytes, moe_stream_t stream) {
  return layer_forward_impl(q, x, w, y, routing, stats, ws, ws_bytes, stream, nullptr, nullptr, nullptr);
}

int moe_layer_forward_profiled(const moe_problem_t* q, const void* x, const moe_weights_t* w, void* y,
                               const moe_routing_t* routing, float* stats, void* ws, size_t ws_bytes,
                               moe_stream_t stream, void* const* events, int32_t* n_kernels) {
  return layer_forward_impl(q, x, w, y, routing, stats, ws, ws_bytes, stream, events, n_kernels, nullptr);
}

int moe_layer_forward_clocked(const moe_problem_t* q, const void* x, const moe_weights_t* w, void* y,
                              const moe_routing_t* routing, float* stats, void* ws, size_t ws_bytes,
                              moe_stream_t stream, uint64_t* clocks) {
  if (!clocks || (reinterpret_cast<uintptr_t>(clocks) & 7u)) return MOE_ERR_INVALID_ARG;
  static_assert(sizeof(unsigned long long) == sizeof(uint64_t), "64-bit clocks");
  return layer_forward_impl(q, x, w, y, routing, stats, ws, ws_bytes, stream, nullptr, nullptr,
                            reinterpret_cast<unsigned long long*>(clocks));
}

}  // extern "C"
