// Backward of the whole layer, for training (BF16).
//
//   Scaling with experts, "The gating network": y_t = sum_k w_k E_k(x_t), the
//   w_k a softmax over the chosen logits; the loss reaches an expert only
//   through the tokens it processed, and the router through those gates.
//   "A balance penalty" / Zen MoDE §5.2: L = alpha E sum_e f_e P_e, with
//   P_e = mean_t p[t,e] (f_e counts chosen pairs: no gradient).
//   Zen-Max §3.2: the router z-loss (1/T) sum_t (logsumexp_t)^2.
//
// With the routing of the forward held fixed, for upstream gradients dy, d_loss
// (balance loss) and d_zloss (z-loss):
//   1. router kernel, one warp per token: dw_k = <dy_t, o_k> for each kept
//      pair (o_k the expert's output row the forward kept in its workspace),
//      do rows = w_k dy_t, and the logit gradient
//        dl_{i_k} += w_k (dw_k - sum_k' w_k' dw_k')             (gate softmax)
//        dl_e     += p_e (q_e - sum_j p_j q_j),  q_e = d_loss alpha E f_e / T
//        dl_e     += d_zloss (2 / T) lse_t p_e
//   2. routed experts: grad_gemm.cu (g, u recomputed; dGU; dX rows; dW13, dW2)
//   3. shared experts: the same with do = dy for every token
//   4. through the gate GEMM: dx_r = dl W_g, dW_g = dl^T x (tensor cores, dl in
//      BF16), d_offset = sum_t dl (FP32, fixed order)
//   5. dx_t = dx_r + dx_shared + sum_{kept k} dX_rows[slot(t,k)]  (FP32 sum, one rounding)
#include <math.h>
#include <string.h>

#include "../../include/moe_b200.h"
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kBwdEPL = kMaxExperts / 32;  // experts per lane in the router kernel

__global__ void __launch_bounds__(256) bwd_router_kernel(
    const __nv_bfloat16* __restrict__ dy, const __nv_bfloat16* __restrict__ y_rows,
    const int32_t* __restrict__ slot_of, const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w,
    const float* __restrict__ logits, const int32_t* __restrict__ counts, int64_t T, int E, int K, int d,
    int64_t max_rows, float alpha, float d_loss, float d_zloss, float* __restrict__ dl,
    __nv_bfloat16* __restrict__ dl16, int e_pad, __nv_bfloat16* __restrict__ dout) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int nv = d / 8;
  for (int64_t t = warp0; t < T; t += n_warps) {
    const uint4* dyv = reinterpret_cast<const uint4*>(dy + t * d);
    // gate-weight gradients; lane k keeps dw_k
    float my_dw = 0.f, my_w = 0.f;
    int my_e = -1;
    for (int k = 0; k < K; ++k) {
      const int slot = slot_of[t * K + k];
      const float w = topk_w[t * K + k];
      if (lane == k) {
        my_w = w;
        my_e = topk_idx[t * K + k];
      }
      if (slot < 0 || slot >= max_rows) continue;
      const uint4* ov = reinterpret_cast<const uint4*>(y_rows + static_cast<int64_t>(slot) * d);
      uint4* dov = reinterpret_cast<uint4*>(dout + static_cast<int64_t>(slot) * d);
      float acc = 0.f;
      for (int v = lane; v < nv; v += 32) {
        const uint4 a = dyv[v], b = ov[v];
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
        uint32_t pk[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc = fmaf(bf16_lo(aw[j]), bf16_lo(bw[j]), acc);
          acc = fmaf(bf16_hi(aw[j]), bf16_hi(bw[j]), acc);
          pk[j] = pack_bf16x2(w * bf16_lo(aw[j]), w * bf16_hi(aw[j]));
        }
        dov[v] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      acc = warp_sum(acc);
      if (lane == k) my_dw = acc;
    }
    const float wdw = warp_sum(lane < K ? my_w * my_dw : 0.f);

    // softmax over all experts
    float l[kBwdEPL], p[kBwdEPL], g[kBwdEPL];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kBwdEPL; ++i) {
      const int e = lane + 32 * i;
      l[i] = e < E ? logits[t * E + e] : -INFINITY;
      m = fmaxf(m, l[i]);
    }
    m = warp_max(m);
    float zl = 0.f;
#pragma unroll
    for (int i = 0; i < kBwdEPL; ++i) {
      p[i] = (lane + 32 * i) < E ? expf(l[i] - m) : 0.f;
      zl += p[i];
    }
    const float Z = warp_sum(zl);
    const float invZ = 1.0f / Z;
    const float lse = m + logf(Z);
    const float fscale = d_loss * alpha * static_cast<float>(E) / (static_cast<float>(T) * static_cast<float>(T) *
                                                                  static_cast<float>(K));
    float pq = 0.f;
#pragma unroll
    for (int i = 0; i < kBwdEPL; ++i) {
      const int e = lane + 32 * i;
      p[i] *= invZ;
      g[i] = e < E ? fscale * static_cast<float>(counts[e]) : 0.f;  // q_e
      pq += p[i] * g[i];
    }
    pq = warp_sum(pq);
    const float zc = d_zloss * 2.0f * lse / static_cast<float>(T);
#pragma unroll
    for (int i = 0; i < kBwdEPL; ++i) g[i] = p[i] * (g[i] - pq) + zc * p[i];
    // gate softmax over the chosen experts (each chosen once per token)
    for (int k = 0; k < K; ++k) {
      const int e = __shfl_sync(0xffffffffu, my_e, k);
      const float v = __shfl_sync(0xffffffffu, my_w * (my_dw - wdw), k);
      if (static_cast<unsigned>(e) < static_cast<unsigned>(E) && (e & 31) == lane) {
#pragma unroll
        for (int i = 0; i < kBwdEPL; ++i)
          if (i == (e >> 5)) g[i] += v;
      }
    }
#pragma unroll
    for (int i = 0; i < kBwdEPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) dl[t * E + e] = g[i];
      if (e < e_pad) dl16[t * e_pad + e] = __float2bfloat16_rn(e < E ? g[i] : 0.f);
    }
  }
}

// dx[t] = a[t] + b[t] + sum_{k: slot_of[t,k] >= 0} rows[slot_of[t,k]]  (a, b may be null)
__global__ void __launch_bounds__(256) bwd_combine_kernel(const __nv_bfloat16* __restrict__ rows,
                                                          const int32_t* __restrict__ slot_of, int64_t T, int K,
                                                          int d, int64_t max_rows,
                                                          const __nv_bfloat16* __restrict__ a,
                                                          const __nv_bfloat16* __restrict__ b,
                                                          __nv_bfloat16* __restrict__ dx) {
  pdl_wait();
  pdl_trigger();
  const int nv = d / 8;
  const int64_t total = T * nv;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / nv;
    const int v = static_cast<int>(i - t * nv);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    auto add = [&](const __nv_bfloat16* base, int64_t row) {
      const uint4 q = reinterpret_cast<const uint4*>(base + row * d)[v];
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc[2 * j] += bf16_lo(w[j]);
        acc[2 * j + 1] += bf16_hi(w[j]);
      }
    };
    if (a) add(a, t);
    if (b) add(b, t);
    for (int k = 0; k < K; ++k) {
      const int s = slot_of[t * K + k];
      if (s >= 0 && s < max_rows) add(rows, s);
    }
    reinterpret_cast<uint4*>(dx + t * d)[v] =
        make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                   pack_bf16x2(acc[6], acc[7]));
  }
}

// d_offset[e] = sum_t dl[t, e]: one block per expert, strided partial sums then
// a fixed-shape tree (float64 accumulation, deterministic).
__global__ void __launch_bounds__(256) bwd_colsum_kernel(const float* __restrict__ dl, int64_t T, int E,
                                                         float* __restrict__ out) {
  __shared__ double part[256];
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x;
  double s = 0.0;
  for (int64_t t = threadIdx.x; t < T; t += blockDim.x) s += static_cast<double>(dl[t * E + e]);
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) out[e] = static_cast<float>(part[0]);
}

}  // namespace moe

namespace moe {

// Backward scratch layout (bytes, 256-aligned): status, dl [T,E] f32,
// dl16 [T, e_pad] bf16, then per-row BF16 buffers.
struct BwdLayout {
  size_t status, dl, dl16, dout, gu, dgu, dx_rows, gu_sh, dgu_sh, dx_sh, dx_r, tail_a, tail_b, total;
  int e_pad;
};

static size_t a256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

static BwdLayout bwd_layout(const Problem& p) {
  BwdLayout B{};
  B.e_pad = (p.E + 7) & ~7;
  const size_t R = static_cast<size_t>(p.max_rows), T = static_cast<size_t>(p.T);
  size_t off = 256;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = a256(off + (bytes ? bytes : 1));
    return o;
  };
  B.status = 0;
  B.dl = take(T * p.E * 4);
  B.dl16 = take(T * B.e_pad * 2);
  B.dout = take(R * p.d * 2);
  const bool saved = p.flags & MOE_FLAG_SAVE_GU;  // the forward kept g, u in its workspace
  B.gu = take(saved ? 0 : R * 2 * p.F * 2);
  B.dgu = take(R * 2 * p.F * 2);
  B.dx_rows = take(R * p.d * 2);
  B.gu_sh = take(saved ? 0 : T * 2 * p.F * p.Ns * 2);
  B.dgu_sh = take(T * 2 * p.F * p.Ns * 2);
  B.dx_sh = take(p.Ns > 0 ? T * p.d * 2 : 0);
  B.dx_r = take(T * p.d * 2);
  B.tail_a = take(wgrad_tail_bytes(p, B.e_pad));
  B.tail_b = take(wgrad_tail_bytes(p, B.e_pad));
  B.total = off;
  return B;
}

}  // namespace moe

using namespace moe;

static bool al16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

template <typename T>
static T* wsat(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

extern "C" {

int moe_backward_workspace_size(const moe_problem_t* q, size_t* bytes) {
  Problem p;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  if (int rc = problem_from_abi(q, &p)) return rc;
  *bytes = bwd_layout(p).total;
  return MOE_OK;
}

int moe_layer_backward(const moe_problem_t* q, const void* x, const moe_weights_t* w, const moe_routing_t* routing,
                       const void* fwd_ws, size_t fwd_ws_bytes, const void* dy, float d_loss, float d_zloss,
                       const moe_grads_t* grads, void* ws, size_t ws_bytes, moe_stream_t stream) {
  Problem p;
  if (int rc = problem_from_abi(q, &p)) return rc;
  if (p.dtype != kBF16) return MOE_ERR_UNSUPPORTED;
  const bool given = p.flags & MOE_FLAG_LOGITS_GIVEN;
  if (!x || !w || !dy || !grads || !fwd_ws || !al16(x) || !al16(dy)) return MOE_ERR_INVALID_ARG;
  if (!(d_loss == d_loss) || !(d_zloss == d_zloss)) return MOE_ERR_INVALID_ARG;
  if (!w->w13 || !w->w2 || !al16(w->w13) || !al16(w->w2)) return MOE_ERR_INVALID_ARG;
  if (!grads->dw13 || !grads->dw2 || !al16(grads->dw13) || !al16(grads->dw2)) return MOE_ERR_INVALID_ARG;
  if (p.Ns > 0 && (!w->w13_shared || !w->w2_shared || !grads->dw13_shared || !grads->dw2_shared ||
                   !al16(w->w13_shared) || !al16(w->w2_shared) || !al16(grads->dw13_shared) ||
                   !al16(grads->dw2_shared)))
    return MOE_ERR_INVALID_ARG;
  if (p.Ns == 0 && (grads->dw13_shared || grads->dw2_shared)) return MOE_ERR_INVALID_ARG;
  if (grads->dw_gate && (given || !w->w_gate || !al16(grads->dw_gate) || !al16(w->w_gate))) return MOE_ERR_INVALID_ARG;
  if (grads->dx && !al16(grads->dx)) return MOE_ERR_INVALID_ARG;
  if (!given && grads->dx && (!w->w_gate || !al16(w->w_gate))) return MOE_ERR_INVALID_ARG;
  const WsLayout L = make_layout(p);
  if ((reinterpret_cast<uintptr_t>(fwd_ws) & 255u) || fwd_ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  const BwdLayout B = bwd_layout(p);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < B.total) return MOE_ERR_WORKSPACE;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void* fws = const_cast<void*>(fwd_ws);
  const bool saved = p.flags & MOE_FLAG_SAVE_GU;
  moe_routing_t r{};
  if (routing) r = *routing;
  const float* logits = r.logits ? r.logits : wsat<float>(fws, L.logits);
  const int32_t* idx = r.topk_idx ? r.topk_idx : wsat<int32_t>(fws, L.topk_idx);
  const float* gw = r.topk_w ? r.topk_w : wsat<float>(fws, L.topk_w);
  const int32_t* counts = r.counts ? r.counts : wsat<int32_t>(fws, L.counts);
  const int32_t* seg_off = r.seg_off ? r.seg_off : wsat<int32_t>(fws, L.seg_off);
  const int32_t* slot_of = r.slot_of ? r.slot_of : wsat<int32_t>(fws, L.slot_of);
  unsigned* status = wsat<unsigned>(ws, B.status);
  float* dl = grads->d_logits ? grads->d_logits : wsat<float>(ws, B.dl);
  __nv_bfloat16* dl16 = wsat<__nv_bfloat16>(ws, B.dl16);
  void* dout = wsat<void>(ws, B.dout);
  void* dx_rows = wsat<void>(ws, B.dx_rows);
  void* dx_sh = p.Ns > 0 ? wsat<void>(ws, B.dx_sh) : nullptr;
  void* dx_r = wsat<void>(ws, B.dx_r);

  if (cudaMemsetAsync(ws, 0, sizeof(unsigned), st) != cudaSuccess) return MOE_ERR_CUDA;
  // 1. router: dw, dl, do rows
  {
    int64_t blocks = (p.T * 32 + 255) / 256;
    const int64_t cap_blocks = static_cast<int64_t>(num_sms()) * 16;
    if (blocks > cap_blocks) blocks = cap_blocks;
    if (launch_k(bwd_router_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st,
                 static_cast<const __nv_bfloat16*>(dy), wsat<const __nv_bfloat16>(fws, L.y_perm), slot_of, idx, gw,
                 logits, counts, p.T, p.E, p.K, p.d, p.max_rows, p.alpha, d_loss, d_zloss, dl, dl16, B.e_pad,
                 static_cast<__nv_bfloat16*>(dout)) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  // 2. routed experts
  if (p.max_rows > 0) {
    if (launch_expert_ffn_backward(p, 0, wsat<void>(fws, L.x_perm), p.max_rows, seg_off, w->w13, w->w2, dout,
                                   wsat<void>(fws, L.h_routed), saved ? wsat<void>(fws, L.gu_routed) : wsat<void>(ws, B.gu),
                                   wsat<void>(ws, B.dgu), dx_rows, grads->dw13, grads->dw2, wsat<void>(ws, B.tail_a),
                                   wsat<void>(ws, B.tail_b), status, st, saved))
      return MOE_ERR_CUDA;
  }
  // 3. shared experts: do = dy for every token
  if (p.Ns > 0) {
    if (launch_expert_ffn_backward(p, 1, x, p.T, nullptr, w->w13_shared, w->w2_shared, dy,
                                   wsat<void>(fws, L.h_shared), saved ? wsat<void>(fws, L.gu_shared) : wsat<void>(ws, B.gu_sh),
                                   wsat<void>(ws, B.dgu_sh), dx_sh, grads->dw13_shared, grads->dw2_shared,
                                   wsat<void>(ws, B.tail_a), wsat<void>(ws, B.tail_b), status, st, saved))
      return MOE_ERR_CUDA;
  }
  // 4. through the gate GEMM
  const bool router_dx = grads->dx && !given;
  if (router_dx && launch_router_dgrad(p, dl16, B.e_pad, w->w_gate, dx_r, status, st)) return MOE_ERR_CUDA;
  if (grads->dw_gate && launch_router_wgrad(p, dl16, B.e_pad, x, grads->dw_gate, wsat<void>(ws, B.tail_a),
                                            wsat<void>(ws, B.tail_b), status, st))
    return MOE_ERR_CUDA;
  if (grads->d_offset) {
    if (launch_k(bwd_colsum_kernel, dim3(p.E), dim3(256), 0, st, static_cast<const float*>(dl), p.T, p.E,
                 grads->d_offset) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  // 5. dx
  if (grads->dx) {
    int64_t blocks = (p.T * (p.d / 8) + 255) / 256;
    const int64_t cap_blocks = static_cast<int64_t>(num_sms()) * 32;
    if (blocks > cap_blocks) blocks = cap_blocks;
    if (launch_k(bwd_combine_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st,
                 static_cast<const __nv_bfloat16*>(dx_rows), slot_of, p.T, p.K, p.d, p.max_rows,
                 router_dx ? static_cast<const __nv_bfloat16*>(dx_r) : nullptr,
                 static_cast<const __nv_bfloat16*>(dx_sh), static_cast<__nv_bfloat16*>(grads->dx)) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

}  // extern "C"
