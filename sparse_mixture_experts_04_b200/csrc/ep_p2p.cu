// Expert-parallel exchange over peer memory: the dispatch's row gather writes
// every kept row straight into the receive buffer of the rank that holds its
// expert, and the combine reads every expert output from the rank that
// computed it -- loads and stores to peer memory (NVLink) inside the kernels,
// no copy or collective on the data path.
//
//   "Scaling with experts" (jeff-ong.com), What you still pay for: with the
//   experts partitioned over devices, a token travels to the device holding
//   its assigned expert and the expert's output travels back.
//   Zen MoDE §7.2 Communication Overhead (Distributed Training): that routing
//   is an all-to-all exchange between the expert devices.
//
// Rank q of G holds the global experts [q E_l, (q+1) E_l), E_l = E / G.
// Every rank routes and ranks its own tokens as one device would (moe_route,
// moe_dispatch without the gather), so its kept rows of global expert e are
// its slots seg_off[e] .. seg_off[e+1].  A rank's receive buffer is
// expert-major: local expert el's rows from source 0, then from source 1, ...
// -- the order in which the grouped GEMM wants them (one group per expert, its
// tiles full, its weights streamed once per tile column).  So slot j of rank r
// for expert e (owner q = e / E_l) is row j + delta[e] of q's buffers, with
//   delta[e] = base(e) + sum_{s<r} rows(s, e) - seg_off_r[e],
//   base(e)  = sum over the owner's experts e' < e of sum_s rows(s, e'),
//   rows(s, e) = seg_off_s[e+1] - seg_off_s[e].
// The expert outputs lie at the same rows of the owner's output buffer.

#include <stdint.h>
#include <string.h>

#include "../../include/moe_b200.h"
#include "common.cuh"
#include "internal.h"

namespace moe {

// One block: thread e of E (E <= kMaxExperts = blockDim).
__global__ void __launch_bounds__(kMaxExperts) ep_peer_plan_kernel(const int32_t* __restrict__ seg_off_all, int G,
                                                                   int rank, int E, int64_t* __restrict__ delta,
                                                                   int32_t* __restrict__ local_seg_off) {
  __shared__ long long s_tot[kMaxExperts];
  pdl_wait();
  pdl_trigger();
  const int e = threadIdx.x;
  const int El = E / G;
  long long tot = 0, before = 0;
  if (e < E) {
    for (int s = 0; s < G; ++s) {
      const int32_t* so = seg_off_all + static_cast<int64_t>(s) * (E + 1);
      const long long r = static_cast<long long>(so[e + 1]) - so[e];
      tot += r;
      if (s < rank) before += r;
    }
    s_tot[e] = tot;
  }
  __syncthreads();
  if (e < E) {
    const int q = e / El;
    long long base = 0;
    for (int e2 = q * El; e2 < e; ++e2) base += s_tot[e2];
    const int32_t* mine = seg_off_all + static_cast<int64_t>(rank) * (E + 1);
    delta[e] = base + before - mine[e];
    if (q == rank) {
      local_seg_off[e - q * El] = static_cast<int32_t>(base);
      if (e == (q + 1) * El - 1) local_seg_off[El] = static_cast<int32_t>(base + tot);
    }
  }
}

// Warp per kept row j of this rank: its expert e is found in seg_off (binary
// search), its source token is perm[j] / K; 16-byte vectors, several loads in
// flight per lane before the stores (which may go to a peer).
constexpr int kScatterUnroll = 8;

__global__ void __launch_bounds__(256) ep_scatter_kernel(const uint4* __restrict__ x,
                                                         const int32_t* __restrict__ perm,
                                                         const int32_t* __restrict__ seg_off, int E, int K, int El,
                                                         int64_t T, int vec_per_row, int64_t max_rows,
                                                         uint4* const* __restrict__ recv_bufs,
                                                         const int64_t* __restrict__ delta) {
  __shared__ int32_t s_seg[kMaxExperts + 1];
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_seg[i] = seg_off[i];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t n_rows = s_seg[E];
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t j = warp0; j < n_rows && j < max_rows; j += n_warps) {
    // largest e with s_seg[e] <= j (empty experts share their offset with the next)
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_seg[mid] <= j) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int64_t tok = perm[j] / K;
    if (tok < 0 || tok >= T) continue;
    const uint4* src = x + tok * vec_per_row;
    uint4* dst = recv_bufs[e / El] + (j + delta[e]) * vec_per_row;
    for (int v0 = lane; v0 < vec_per_row; v0 += 32 * kScatterUnroll) {
      uint4 buf[kScatterUnroll];
#pragma unroll
      for (int u = 0; u < kScatterUnroll; ++u)
        if (v0 + 32 * u < vec_per_row) buf[u] = __ldg(src + v0 + 32 * u);
#pragma unroll
      for (int u = 0; u < kScatterUnroll; ++u)
        if (v0 + 32 * u < vec_per_row) dst[v0 + 32 * u] = buf[u];
    }
  }
}

template <typename T>
struct EpPack;
template <>
struct EpPack<__nv_bfloat16> {
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
struct EpPack<float> {
  static constexpr int N = 4;
  __device__ static void load(const void* p, float (&v)[4]) {
    const float4 q = *static_cast<const float4*>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
  }
  __device__ static void store(void* p, const float (&v)[4]) {
    *static_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

// The combine of the single-device layer (shared first, then k ascending,
// FP32 accumulation, one rounding), each kept pair's row read from the rank
// that computed it: out_bufs[e / El] + (slot + delta[e]) rows.  2-D grid:
// blockIdx.x a chunk of the row's vectors, blockIdx.y (grid-stride) the token.
constexpr int kEpCombineThreads = 128;
constexpr int kEpCombineVPT = 2;

template <typename T>
__global__ void __launch_bounds__(kEpCombineThreads) ep_combine_kernel(
    const T* const* __restrict__ out_bufs, const int64_t* __restrict__ delta, const int32_t* __restrict__ topk_idx,
    const int32_t* __restrict__ slot_of, const float* __restrict__ topk_w, const T* __restrict__ y_shared,
    T* __restrict__ y, int64_t Tn, int d, int K, int E, int El, int64_t max_slots) {
  constexpr int V = EpPack<T>::N;
  pdl_wait();
  pdl_trigger();
  const int nvec = d / V;
  const int v0 = blockIdx.x * (kEpCombineThreads * kEpCombineVPT) + threadIdx.x;
  for (int64_t t = blockIdx.y; t < Tn; t += gridDim.y) {
    float acc[kEpCombineVPT][V];
#pragma unroll
    for (int j = 0; j < kEpCombineVPT; ++j) {
      const int v = v0 + j * kEpCombineThreads;
#pragma unroll
      for (int i = 0; i < V; ++i) acc[j][i] = 0.f;
      if (y_shared && v < nvec) EpPack<T>::load(y_shared + t * d + v * V, acc[j]);
    }
    for (int k = 0; k < K; ++k) {
      const int slot = slot_of[t * K + k];
      const int e = topk_idx[t * K + k];
      if (slot < 0 || slot >= max_slots || e < 0 || e >= E) continue;
      const float w = topk_w[t * K + k];
      const T* row = out_bufs[e / El] + (static_cast<int64_t>(slot) + delta[e]) * d;
      float r[kEpCombineVPT][V];
#pragma unroll
      for (int j = 0; j < kEpCombineVPT; ++j) {
        const int v = v0 + j * kEpCombineThreads;
        if (v < nvec) EpPack<T>::load(row + v * V, r[j]);
      }
#pragma unroll
      for (int j = 0; j < kEpCombineVPT; ++j)
#pragma unroll
        for (int i = 0; i < V; ++i) acc[j][i] = fmaf(w, r[j][i], acc[j][i]);
    }
#pragma unroll
    for (int j = 0; j < kEpCombineVPT; ++j) {
      const int v = v0 + j * kEpCombineThreads;
      if (v < nvec) EpPack<T>::store(y + t * d + v * V, acc[j]);
    }
  }
}

}  // namespace moe

using namespace moe;

static bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

extern "C" int moe_ep_peer_plan(int32_t n_ranks, int32_t rank, int32_t n_experts, const int32_t* seg_off_all,
                                int64_t* delta, int32_t* local_seg_off, moe_stream_t stream) {
  if (n_ranks < 1 || rank < 0 || rank >= n_ranks || n_experts < 1 || n_experts > kMaxExperts ||
      n_experts % n_ranks != 0)
    return MOE_ERR_INVALID_ARG;
  if (!seg_off_all || !delta || !local_seg_off) return MOE_ERR_INVALID_ARG;
  return cuda_rc(launch_k(ep_peer_plan_kernel, dim3(1), dim3(kMaxExperts), 0, reinterpret_cast<cudaStream_t>(stream),
                          seg_off_all, static_cast<int>(n_ranks), static_cast<int>(rank),
                          static_cast<int>(n_experts), delta, local_seg_off));
}

extern "C" int moe_ep_scatter(const moe_problem_t* q, int32_t n_ranks, const void* x, const int32_t* perm,
                              const int32_t* seg_off, void* const* recv_bufs, const int64_t* delta,
                              moe_stream_t stream) {
  Problem p;
  if (int rc = problem_from_abi(q, &p)) return rc;
  if (n_ranks < 1 || p.E % n_ranks != 0) return MOE_ERR_INVALID_ARG;
  if (!x || !a16(x) || !perm || !seg_off || !recv_bufs || !delta) return MOE_ERR_INVALID_ARG;
  if (p.max_rows <= 0) return MOE_OK;
  const int vec_per_row = static_cast<int>(p.d * p.esize() / 16);
  int64_t blocks = (p.max_rows + 7) / 8;
  const int64_t cap_blocks = static_cast<int64_t>(num_sms()) * 16;
  if (blocks > cap_blocks) blocks = cap_blocks;
  return cuda_rc(launch_k(ep_scatter_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                          reinterpret_cast<cudaStream_t>(stream), static_cast<const uint4*>(x), perm, seg_off, p.E,
                          p.K, p.E / static_cast<int>(n_ranks), p.T, vec_per_row, p.max_rows,
                          reinterpret_cast<uint4* const*>(recv_bufs), delta));
}

extern "C" int moe_ep_combine(const moe_problem_t* q, int32_t n_ranks, const void* const* out_bufs,
                              const int64_t* delta, const int32_t* topk_idx, const int32_t* slot_of,
                              const float* topk_w, const void* y_shared, void* y, moe_stream_t stream) {
  Problem p;
  if (int rc = problem_from_abi(q, &p)) return rc;
  if (n_ranks < 1 || p.E % n_ranks != 0) return MOE_ERR_INVALID_ARG;
  if (!out_bufs || !delta || !topk_idx || !slot_of || !topk_w || !y || !a16(y)) return MOE_ERR_INVALID_ARG;
  if ((p.Ns > 0) != (y_shared != nullptr)) return MOE_ERR_INVALID_ARG;
  if (y_shared && !a16(y_shared)) return MOE_ERR_INVALID_ARG;
  const int V = p.dtype == kBF16 ? 8 : 4;
  const int nvec = p.d / V;
  const unsigned gx =
      static_cast<unsigned>((nvec + kEpCombineThreads * kEpCombineVPT - 1) / (kEpCombineThreads * kEpCombineVPT));
  int64_t gy = p.T;
  if (gy > 65535) gy = 65535;
  const dim3 grid(gx, static_cast<unsigned>(gy));
  const int El = p.E / static_cast<int>(n_ranks);
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (p.dtype == kBF16)
    return cuda_rc(launch_k(ep_combine_kernel<__nv_bfloat16>, grid, dim3(kEpCombineThreads), 0, st,
                            reinterpret_cast<const __nv_bfloat16* const*>(out_bufs), delta, topk_idx, slot_of,
                            topk_w, static_cast<const __nv_bfloat16*>(y_shared), static_cast<__nv_bfloat16*>(y), p.T,
                            p.d, p.K, p.E, El, p.max_rows));
  return cuda_rc(launch_k(ep_combine_kernel<float>, grid, dim3(kEpCombineThreads), 0, st,
                          reinterpret_cast<const float* const*>(out_bufs), delta, topk_idx, slot_of, topk_w,
                          static_cast<const float*>(y_shared), static_cast<float*>(y), p.T, p.d, p.K, p.E, El,
                          p.max_rows));
}

// Buffers other processes map (CUDA IPC): whole allocations, so that a peer
// that opens the handle gets the buffer's own base address.
extern "C" int moe_ipc_malloc(size_t bytes, void** ptr) {
  if (!ptr || bytes == 0) return MOE_ERR_INVALID_ARG;
  *ptr = nullptr;
  return cuda_rc(cudaMalloc(ptr, bytes));
}

extern "C" int moe_ipc_free(void* ptr) { return ptr ? cuda_rc(cudaFree(ptr)) : MOE_ERR_INVALID_ARG; }

extern "C" int moe_ipc_handle(const void* ptr, void* handle) {
  if (!ptr || !handle) return MOE_ERR_INVALID_ARG;
  static_assert(sizeof(cudaIpcMemHandle_t) == MOE_IPC_HANDLE_BYTES, "IPC handle size");
  cudaIpcMemHandle_t h;
  if (cudaError_t e = cudaIpcGetMemHandle(&h, const_cast<void*>(ptr))) return cuda_rc(e);
  memcpy(handle, &h, sizeof h);
  return MOE_OK;
}

extern "C" int moe_ipc_open(const void* handle, void** ptr) {
  if (!handle || !ptr) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof h);
  *ptr = nullptr;
  return cuda_rc(cudaIpcOpenMemHandle(ptr, h, cudaIpcMemLazyEnablePeerAccess));
}

extern "C" int moe_ipc_close(void* ptr) { return ptr ? cuda_rc(cudaIpcCloseMemHandle(ptr)) : MOE_ERR_INVALID_ARG; }
