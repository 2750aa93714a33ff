// Gate-weighted combine back to token order.
//
//   Scaling with experts, "The gating network": y = g1 * Expert1(x) + g2 * Expert2(x)
//   with g the renormalised gate weights; "A budget": a dropped pair adds
//   nothing; "A shared expert" / Zen-Max §2.2: shared experts are added unweighted.
//
//   y[t] = y_shared[t] + sum_{k : slot_of[t,k] >= 0} w[t,k] * y_perm[slot_of[t,k]]
// accumulated in fp32 in that order (shared first, then k ascending) and
// rounded once.  16-byte vectors along d.
#include "common.cuh"
#include "internal.h"

namespace moe {

template <typename T>
struct Pack16;
template <>
struct Pack16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const void* p, float (&v)[8]) {
    const uint4 q = *static_cast<const uint4*>(p);
    v[0] = bf16_lo(q.x); v[1] = bf16_hi(q.x); v[2] = bf16_lo(q.y); v[3] = bf16_hi(q.y);
    v[4] = bf16_lo(q.z); v[5] = bf16_hi(q.z); v[6] = bf16_lo(q.w); v[7] = bf16_hi(q.w);
  }
  __device__ static void store(void* p, const float (&v)[8]) {
    uint4 q;
    q.x = pack_bf16x2(v[0], v[1]); q.y = pack_bf16x2(v[2], v[3]);
    q.z = pack_bf16x2(v[4], v[5]); q.w = pack_bf16x2(v[6], v[7]);
    *static_cast<uint4*>(p) = q;
  }
};
template <>
struct Pack16<float> {
  static constexpr int N = 4;
  __device__ static void load(const void* p, float (&v)[4]) {
    const float4 q = *static_cast<const float4*>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
  }
  __device__ static void store(void* p, const float (&v)[4]) {
    *static_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

// 2-D grid: blockIdx.x selects a chunk of kCombineVPT * blockDim.x vectors of
// a row, blockIdx.y (grid-stride) the token.  A thread owns kCombineVPT
// vectors kCombineThreads apart and issues all their loads before the
// arithmetic, so many requests are in flight per thread; index math is 32-bit.
// The token's (slot, weight) pairs are the same for every thread of the block
// (broadcast loads).
constexpr int kCombineThreads = 128;
constexpr int kCombineVPT = 2;

template <typename T>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const T* __restrict__ y_perm,
                                                                  const int32_t* __restrict__ slot_of,
                                                                  const float* __restrict__ topk_w,
                                                                  const T* __restrict__ y_shared,
                                                                  T* __restrict__ y, int64_t Tn, int d, int K,
                                                                  int64_t n_perm_rows, unsigned long long* clk) {
  constexpr int V = Pack16<T>::N;
  pdl_wait();
  pdl_trigger();
  stage_clock_start(clk);
  const int nvec = d / V;
  const int v0 = blockIdx.x * (kCombineThreads * kCombineVPT) + threadIdx.x;
  for (int64_t t = blockIdx.y; t < Tn; t += gridDim.y) {
    float acc[kCombineVPT][V];
#pragma unroll
    for (int j = 0; j < kCombineVPT; ++j) {
      const int v = v0 + j * kCombineThreads;
#pragma unroll
      for (int i = 0; i < V; ++i) acc[j][i] = 0.f;
      if (y_shared && v < nvec) Pack16<T>::load(y_shared + t * d + v * V, acc[j]);
    }
    for (int k = 0; k < K; ++k) {
      const int slot = slot_of[t * K + k];
      if (slot < 0 || slot >= n_perm_rows) continue;
      const float w = topk_w[t * K + k];
      const T* row = y_perm + static_cast<int64_t>(slot) * d;
      float r[kCombineVPT][V];
#pragma unroll
      for (int j = 0; j < kCombineVPT; ++j) {
        const int v = v0 + j * kCombineThreads;
        if (v < nvec) Pack16<T>::load(row + v * V, r[j]);
      }
#pragma unroll
      for (int j = 0; j < kCombineVPT; ++j)
#pragma unroll
        for (int i = 0; i < V; ++i) acc[j][i] = fmaf(w, r[j][i], acc[j][i]);
    }
#pragma unroll
    for (int j = 0; j < kCombineVPT; ++j) {
      const int v = v0 + j * kCombineThreads;
      if (v < nvec) Pack16<T>::store(y + t * d + v * V, acc[j]);
    }
  }
  if (clk) {
    __syncthreads();
    stage_clock_end(clk);
  }
}

cudaError_t launch_combine(const Problem& p, const void* y_perm, const int32_t* slot_of, const float* topk_w,
                           const void* y_shared, void* y, cudaStream_t st, unsigned long long* clk) {
  const int V = p.dtype == kBF16 ? 8 : 4;
  const int nvec = p.d / V;
  const unsigned gx = static_cast<unsigned>((nvec + kCombineThreads * kCombineVPT - 1) / (kCombineThreads * kCombineVPT));
  int64_t gy = p.T;
  if (gy > 65535) gy = 65535;
  const dim3 grid(gx, static_cast<unsigned>(gy));
  if (p.dtype == kBF16)
    return launch_k(combine_kernel<__nv_bfloat16>, grid, dim3(kCombineThreads), 0, st,
                    static_cast<const __nv_bfloat16*>(y_perm), slot_of, topk_w,
                    static_cast<const __nv_bfloat16*>(y_shared), static_cast<__nv_bfloat16*>(y), p.T, p.d, p.K,
                    p.max_rows, clk);
  else
    return launch_k(combine_kernel<float>, grid, dim3(kCombineThreads), 0, st, static_cast<const float*>(y_perm),
                    slot_of, topk_w, static_cast<const float*>(y_shared), static_cast<float*>(y), p.T, p.d, p.K,
                    p.max_rows, clk);
  return cudaGetLastError();
}

}  // namespace moe
