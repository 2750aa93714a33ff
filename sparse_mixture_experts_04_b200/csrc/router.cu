// Router: gate logits, softmax, top-K selection with optional selection bias,
// renormalised gate weights, and the Switch balance statistics.
//
//   Zen MoDE: Mixture of Distilled Experts Architecture, §3.1 Router
//     Architecture, eq. router_standard: TopK(softmax(W_r x), K).
//   Zen-Max, §2.3 Auxiliary-Loss-Free Load Balancing: s_ij = softmax(x_i W_g)_j + b_j
//     (the bias steers selection; gate weights use the unbiased softmax).
//   Scaling with experts, "The gating network": only the k best scores stay
//     non-zero, rescaled to add up to 1.  "A balance penalty":
//     alpha * N * sum f_i P_i.  Zen MoDE §5.2 eq. L_balance.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "router_select.cuh"

namespace moe {

// ----------------------------------------------------------------------------
// Gate logits on CUDA cores: logits[t, e] = sum_j x[t, j] * Wg[e, j] + off[e].
// One warp handles TPW tokens at a time; lanes stride over d in 16-byte
// vectors; each lane keeps TPW x EB partial sums (so every Wg vector it loads
// serves TPW tokens), then a butterfly reduction gives every lane the sums.
// Experts are processed in blocks of EB (several passes when E > EB).
// Used for FP32 problems and for BF16 problems with few experts.
// ----------------------------------------------------------------------------
template <typename Tin>
struct Vec16;
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static void load(const float* p, float (&v)[4]) {
    float4 q = *reinterpret_cast<const float4*>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
  }
};
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&v)[8]) {
    uint4 q = *reinterpret_cast<const uint4*>(p);
    v[0] = bf16_lo(q.x); v[1] = bf16_hi(q.x); v[2] = bf16_lo(q.y); v[3] = bf16_hi(q.y);
    v[4] = bf16_lo(q.z); v[5] = bf16_hi(q.z); v[6] = bf16_lo(q.w); v[7] = bf16_hi(q.w);
  }
};

template <typename Tin, int EB, int TPW>
__global__ void __launch_bounds__(256) gate_logits_simt_kernel(const Tin* __restrict__ x,
                                                               const Tin* __restrict__ wg,
                                                               const float* __restrict__ off,
                                                               float* __restrict__ logits, int64_t T, int d,
                                                               int E) {
  constexpr int V = Vec16<Tin>::N;
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t n_groups = (T + TPW - 1) / TPW;

  for (int64_t grp = warp_global; grp < n_groups; grp += n_warps) {
    const int64_t t0 = grp * TPW;
    for (int eb = 0; eb < E; eb += EB) {
      float acc[TPW][EB];
#pragma unroll
      for (int i = 0; i < TPW; ++i)
#pragma unroll
        for (int e = 0; e < EB; ++e) acc[i][e] = 0.f;

      for (int j = lane * V; j < d; j += 32 * V) {
        float xv[TPW][V];
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
          if (t0 + i < T) {
            Vec16<Tin>::load(x + (t0 + i) * d + j, xv[i]);
          } else {
#pragma unroll
            for (int v = 0; v < V; ++v) xv[i][v] = 0.f;
          }
        }
#pragma unroll
        for (int e = 0; e < EB; ++e) {
          if (eb + e < E) {
            float wv[V];
            Vec16<Tin>::load(wg + static_cast<int64_t>(eb + e) * d + j, wv);
#pragma unroll
            for (int i = 0; i < TPW; ++i)
#pragma unroll
              for (int v = 0; v < V; ++v) acc[i][e] = fmaf(xv[i][v], wv[v], acc[i][e]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < TPW; ++i)
#pragma unroll
        for (int e = 0; e < EB; ++e) acc[i][e] = warp_sum(acc[i][e]);
#pragma unroll
      for (int i = 0; i < TPW; ++i) {
#pragma unroll
        for (int e = 0; e < EB; ++e) {
          if (lane == e && t0 + i < T && eb + e < E)
            logits[(t0 + i) * E + eb + e] = acc[i][e] + (off ? off[eb + e] : 0.f);
        }
      }
    }
  }
}

template <typename Tin, int EB, int TPW>
static cudaError_t gate_simt(const Problem& p, const void* x, const void* wg, const float* off, float* logits,
                             cudaStream_t st) {
  const int64_t warps = (p.T + TPW - 1) / TPW;
  int64_t blocks = (warps + 7) / 8;
  const int64_t cap_blocks = static_cast<int64_t>(num_sms()) * 16;
  if (blocks > cap_blocks) blocks = cap_blocks;
  return launch_k(gate_logits_simt_kernel<Tin, EB, TPW>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st,
                  static_cast<const Tin*>(x), static_cast<const Tin*>(wg), off, logits, p.T, p.d, p.E);
}

cudaError_t launch_gate_logits_simt(const Problem& p, const void* x, const void* wg, const float* off,
                                    float* logits, cudaStream_t st) {
  if (p.dtype == kBF16) {
    if (p.E <= 8) return gate_simt<__nv_bfloat16, 8, 4>(p, x, wg, off, logits, st);
    if (p.E <= 16) return gate_simt<__nv_bfloat16, 16, 2>(p, x, wg, off, logits, st);
    return gate_simt<__nv_bfloat16, 32, 1>(p, x, wg, off, logits, st);
  }
  if (p.E <= 8) return gate_simt<float, 8, 4>(p, x, wg, off, logits, st);
  if (p.E <= 16) return gate_simt<float, 16, 2>(p, x, wg, off, logits, st);
  return gate_simt<float, 32, 1>(p, x, wg, off, logits, st);
}

// ----------------------------------------------------------------------------
// Selection.  One warp per token; lane l holds experts l, l+32, ... (EPL of
// them).  Per token:
//   m = max logit; ex_e = exp(l_e - m) (fp32); Z = sum ex; p_e = ex_e / Z
//   score_e (float64): l_e, or p64_e + b_e (bias on p), or l_e + b_e (bias on logit),
//     p64 = exp(l - m) / sum exp(l - m) evaluated in float64
//   K rounds of warp arg-max over (score desc, expert index asc), each three
//   redux.sync reductions over order-preserving 64-bit keys
//   w_k = ex_{idx_k} / sum_k ex_{idx_k}    (= renormalised softmax over the chosen)
// Per block: sum over its tokens of p_e (fp32, fixed order) and the number of
// times each expert was chosen (integer), for the balance statistics.
// ----------------------------------------------------------------------------
template <int EPL>
__global__ void __launch_bounds__(256) route_select_kernel(float* __restrict__ logits,
                                                           const float* __restrict__ parts, int n_parts,
                                                           const float* __restrict__ sel_bias, int bias_on_logit,
                                                           int32_t* __restrict__ topk_idx,
                                                           float* __restrict__ topk_w, int64_t T, int E, int K,
                                                           int32_t* __restrict__ chunk_counts,
                                                           unsigned long long* __restrict__ chunk_psum,
                                                           double pscale, float* __restrict__ zpart,
                                                           unsigned long long* clk) {
  __shared__ float s_psum[8][32 * EPL];
  __shared__ int s_count[32 * EPL];
  __shared__ float s_z[8];
  // the fixed-point block sums below cover at most kSelectTokens tokens
  static_assert(kDispatchChunk % kSelectTokens == 0, "a selection block must not straddle dispatch chunks");
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  pdl_wait();
  pdl_trigger();
  stage_clock_start(clk);
  for (int e = threadIdx.x; e < 32 * EPL; e += blockDim.x) s_count[e] = 0;
  __syncthreads();

  float pacc[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) pacc[i] = 0.f;
  float zacc = 0.f;  // sum over this warp's tokens of logsumexp^2 (router z-loss)

  const int64_t tok_begin = static_cast<int64_t>(blockIdx.x) * kSelectTokens;
  constexpr int kPerWarp = kSelectTokens / 8;
  for (int n = 0; n < kPerWarp; ++n) {
    const int64_t t = tok_begin + warp * kPerWarp + n;
    if (t >= T) break;
    float lg[EPL];
    float bias[EPL];
    // every load of the token first (the slices, the biases), then the adds
    // in slice order: the loads' latencies overlap instead of queueing
    if (n_parts > 0) {  // split-K gate GEMM: add the slices in order
      float pv[kMaxLogitParts][EPL];
#pragma unroll
      for (int sl = 0; sl < kMaxLogitParts; ++sl)
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const int e = lane + 32 * i;
          pv[sl][i] = (sl < n_parts && e < E) ? parts[static_cast<int64_t>(sl) * T * E + t * E + e] : 0.f;
        }
#pragma unroll
      for (int i = 0; i < EPL; ++i) bias[i] = (sel_bias && lane + 32 * i < E) ? sel_bias[lane + 32 * i] : 0.f;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        float v = 0.f;
#pragma unroll
        for (int sl = 0; sl < kMaxLogitParts; ++sl)
          if (sl < n_parts) v += pv[sl][i];
        if (e < E) logits[t * E + e] = v;
        lg[i] = e < E ? v : -INFINITY;
      }
    } else {
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        lg[i] = e < E ? logits[t * E + e] : -INFINITY;
        bias[i] = (sel_bias && e < E) ? sel_bias[e] : 0.f;
      }
    }
    select_token_group<EPL, 32>(lg, bias, sel_bias != nullptr, bias_on_logit, E, K, lane, pacc, zacc, topk_idx + t * K,
                           topk_w + t * K, s_count);
  }
#pragma unroll
  for (int i = 0; i < EPL; ++i) s_psum[warp][lane + 32 * i] = pacc[i];
  if (lane == 0) s_z[warp] = zacc;
  __syncthreads();
  // Per-dispatch-chunk totals (this block's tokens lie in one chunk, since
  // kDispatchChunk is a multiple of kSelectTokens): the expert histogram and
  // the sum of p as a fixed-point integer (scale p_fixed_scale(T)).  Integer adds commute, so the
  // totals do not depend on the order in which blocks arrive.
  const int64_t chunk = tok_begin / kDispatchChunk;
  if (zpart && threadIdx.x == 0) {
    float z = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) z += s_z[w];
    zpart[blockIdx.x] = z;
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += s_psum[w][e];
    if (s_count[e]) atomicAdd(&chunk_counts[chunk * E + e], s_count[e]);
    if (s > 0.f) atomicAdd(&chunk_psum[chunk * E + e], __double2ull_rn(static_cast<double>(s) * pscale));
  }
  if (clk) {
    __syncthreads();
    stage_clock_end(clk);
  }
}

int route_select_zparts(const Problem& p) { return static_cast<int>((p.T + kSelectTokens - 1) / kSelectTokens); }

cudaError_t launch_route_select(const Problem& p, float* logits, const float* parts, int n_parts,
                                const float* sel_bias, int32_t* topk_idx, float* topk_w, int32_t* chunk_counts,
                                unsigned long long* chunk_psum, float* zpart, cudaStream_t st,
                                unsigned long long* clk) {
  const unsigned blocks = static_cast<unsigned>((p.T + kSelectTokens - 1) / kSelectTokens);
  const int bias_on_logit = (p.flags & 0x2u) ? 1 : 0;
  if (p.E <= 32)
    return launch_k(route_select_kernel<1>, dim3(blocks), dim3(256), 0, st, logits, parts, n_parts, sel_bias,
                    bias_on_logit, topk_idx, topk_w, p.T, p.E, p.K, chunk_counts, chunk_psum, p_fixed_scale(p.T), zpart, clk);
  else if (p.E <= 64)
    return launch_k(route_select_kernel<2>, dim3(blocks), dim3(256), 0, st, logits, parts, n_parts, sel_bias,
                    bias_on_logit, topk_idx, topk_w, p.T, p.E, p.K, chunk_counts, chunk_psum, p_fixed_scale(p.T), zpart, clk);
  else if (p.E <= 128)
    return launch_k(route_select_kernel<4>, dim3(blocks), dim3(256), 0, st, logits, parts, n_parts, sel_bias,
                    bias_on_logit, topk_idx, topk_w, p.T, p.E, p.K, chunk_counts, chunk_psum, p_fixed_scale(p.T), zpart, clk);
  else
    return launch_k(route_select_kernel<8>, dim3(blocks), dim3(256), 0, st, logits, parts, n_parts, sel_bias,
                    bias_on_logit, topk_idx, topk_w, p.T, p.E, p.K, chunk_counts, chunk_psum, p_fixed_scale(p.T), zpart, clk);
}

// ----------------------------------------------------------------------------
// Balance statistics from the per-chunk totals the selection kernel adds:
//   f_e = count_e / (T K),  P_e = (1/T) sum_t p[t,e],  loss = alpha E sum_e f_e P_e
// stats layout: [f_0 .. f_{E-1}, P_0 .. P_{E-1}, loss].  Used by moe_route;
// the layer forward finalises the same statistics inside the dispatch scan.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) route_stats_kernel(const int32_t* __restrict__ chunk_counts,
                                                           const unsigned long long* __restrict__ chunk_psum,
                                                           int n_chunks, int64_t T, int E, int K, float alpha,
                                                           long long cap, const float* __restrict__ zpart,
                                                           int n_zpart, float* __restrict__ stats) {
  __shared__ double s_fp[kMaxExperts];
  __shared__ int s_c[kMaxExperts];
  __shared__ int s_k[kMaxExperts];
  __shared__ double s_zsum[1024];
  pdl_wait();
  pdl_trigger();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    long long c = 0;
    unsigned long long ps = 0;
    for (int ch = 0; ch < n_chunks; ++ch) {
      c += chunk_counts[static_cast<int64_t>(ch) * E + e];
      ps += chunk_psum[static_cast<int64_t>(ch) * E + e];
    }
    s_fp[e] = balance_stats_expert(c, ps, T, E, K, e, stats);
    s_c[e] = static_cast<int>(c);
    s_k[e] = (cap < 0 || c < cap) ? static_cast<int>(c) : static_cast<int>(cap);
  }
  if (zpart) {  // router z-loss partials: strided per thread, then a fixed-shape tree
    double z = 0.0;
    for (int b = threadIdx.x; b < n_zpart; b += blockDim.x) z += zpart[b];
    s_zsum[threadIdx.x] = z;
  }
  __syncthreads();
  if (zpart) {
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
      if (threadIdx.x < w) s_zsum[threadIdx.x] += s_zsum[threadIdx.x + w];
      __syncthreads();
    }
  }
  if (threadIdx.x == 0) {
    balance_loss(s_fp, E, alpha, stats);
    if (zpart) utilisation_stats(s_c, s_k, E, T, s_zsum[0], stats);
  }
}

cudaError_t launch_route_stats(const Problem& p, const int32_t* chunk_counts, const unsigned long long* chunk_psum,
                               int n_chunks, const float* zpart, int n_zpart, float* stats, cudaStream_t st) {
  return launch_k(route_stats_kernel, dim3(1), dim3(1024), 0, st, chunk_counts, chunk_psum, n_chunks, p.T, p.E,
                  p.K, p.alpha, static_cast<long long>(p.cap), zpart, n_zpart, stats);
}

}  // namespace moe
