// Capacity-limited dispatch: group the (token, k) assignments by expert.
//
//   Scaling with experts, "A budget": an expert accepts a bounded number of
//   tokens per batch; an assignment beyond the bound is dropped (the expert
//   does not process that token, which keeps only its residual path).
//   Zen MoDE, §5.3 Adaptive Capacity Factors: capacity_e = C * batch*seq / N_E
//   (scaled here by K for top-K routing).
//
// Order: earlier tokens are served first.  rank(t,k) = number of tokens
// t' < t that chose the same expert; (t,k) is kept iff rank < cap.  The result
// is independent of thread scheduling: ranks are counted, never claimed by
// racing atomics.
//
// Kernels (all multi-pass, no CTA waits on another):
//   1. hist      : per 256-token chunk, per-expert counts (fused into the
//                  selection kernel on the layer path)
//   2. scan+rank : per chunk, the expert totals and the earlier chunks' counts
//                  from the whole histogram, kept and seg_off; each warp builds
//                  a lane mask per expert (which of its 32 tokens chose it);
//                  rank = earlier chunks + earlier warps' counts + popcount of
//                  the lower lanes' bits.  Large problems run it as two
//                  kernels: scan (per expert, prefix over chunks, totals, kept,
//                  seg_off) then rank.
//   3. gather    : x_perm[slot] = x[perm[slot] / K]
#include "common.cuh"
#include "internal.h"

namespace moe {

__global__ void __launch_bounds__(256) dispatch_hist_kernel(const int32_t* __restrict__ idx, int64_t T, int K,
                                                            int E, int32_t* __restrict__ chunk_counts,
                                                            unsigned* status) {
  __shared__ int hist[kMaxExperts];
  pdl_wait();
  pdl_trigger();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t begin = static_cast<int64_t>(blockIdx.x) * kDispatchChunk * K;
  int64_t end = begin + static_cast<int64_t>(kDispatchChunk) * K;
  if (end > T * K) end = T * K;
  for (int64_t i = begin + threadIdx.x; i < end; i += blockDim.x) {
    const int e = idx[i];
    if (static_cast<unsigned>(e) < static_cast<unsigned>(E))
      atomicAdd(&hist[e], 1);
    else
      raise_status(status, kDevBadExpert);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    chunk_counts[static_cast<int64_t>(blockIdx.x) * E + e] = hist[e];
}

// Large problems: scan (one block) then rank (one block per chunk).
// One block of 1024 threads.  Thread (e, s) owns a contiguous run of chunks
// for expert e; runs are summed, scanned per expert, then re-walked to write
// each chunk's base.
// With stats != nullptr it also finalises the balance statistics from the
// chunk histogram and the chunk probability sums (fixed point) that the
// selection kernel added: f_e, P_e and the loss (see balance_stats_expert).
__global__ void __launch_bounds__(1024) dispatch_scan_kernel(const int32_t* __restrict__ chunk_counts,
                                                             int n_chunks, int E, long long cap,
                                                             int32_t* __restrict__ chunk_base,
                                                             int32_t* __restrict__ counts,
                                                             int32_t* __restrict__ kept,
                                                             int32_t* __restrict__ seg_off,
                                                             const unsigned long long* __restrict__ chunk_psum,
                                                             float* __restrict__ stats, int64_t T, int K,
                                                             float alpha, const float* __restrict__ zpart,
                                                             int n_zpart, const int32_t* __restrict__ expert_cap,
                                                             unsigned long long* clk) {
  __shared__ int part[1024];
  __shared__ unsigned long long ppart[1024];
  __shared__ int s_kept[kMaxExperts];
  __shared__ int s_count[kMaxExperts];
  __shared__ double s_fp[kMaxExperts];
  __shared__ double s_zsum[1024];
  pdl_wait();
  pdl_trigger();
  stage_clock_start(clk);
  int S = 1024 / E;
  if (S > n_chunks) S = n_chunks;
  if (S < 1) S = 1;
  const int per = (n_chunks + S - 1) / S;
  const int tid = threadIdx.x;
  const int e = tid / S;
  const int s = tid - e * S;
  const bool active = e < E;
  int c0 = s * per, c1 = c0 + per;
  if (c1 > n_chunks) c1 = n_chunks;
  int local = 0;
  unsigned long long plocal = 0;
  if (active) {
    for (int c = c0; c < c1; ++c) local += chunk_counts[static_cast<int64_t>(c) * E + e];
    if (stats)
      for (int c = c0; c < c1; ++c) plocal += chunk_psum[static_cast<int64_t>(c) * E + e];
  }
  part[tid] = local;
  ppart[tid] = plocal;
  __syncthreads();
  if (active && s == 0) {
    int run = 0;
    unsigned long long prun = 0;
    for (int i = 0; i < S; ++i) {
      const int v = part[tid + i];
      part[tid + i] = run;
      run += v;
      prun += ppart[tid + i];
    }
    counts[e] = run;
    long long ce = cap;
    if (expert_cap) ce = expert_cap[e];   // per-expert capacity (Zen MoDE §5.3 capacity_e)
    const int k = (ce < 0 || run < ce) ? run : static_cast<int>(ce);
    kept[e] = k;
    s_kept[e] = k;
    s_count[e] = run;
    if (stats) s_fp[e] = balance_stats_expert(run, prun, T, E, K, e, stats);
  }
  if (stats && zpart) {  // router z-loss partials: strided per thread, then a fixed-shape tree
    double z = 0.0;
    for (int b = tid; b < n_zpart; b += 1024) z += zpart[b];
    s_zsum[tid] = z;
  }
  __syncthreads();
  if (stats && zpart) {
    for (int w = 512; w > 0; w >>= 1) {
      if (tid < w) s_zsum[tid] += s_zsum[tid + w];
      __syncthreads();
    }
  }
  if (stats && tid == 32) {
    balance_loss(s_fp, E, alpha, stats);
    if (zpart) utilisation_stats(s_count, s_kept, E, T, s_zsum[0], stats);
  }
  if (active) {
    int run = part[tid];
    for (int c = c0; c < c1; ++c) {
      chunk_base[static_cast<int64_t>(c) * E + e] = run;
      run += chunk_counts[static_cast<int64_t>(c) * E + e];
    }
  }
  // seg_off = exclusive prefix of kept over experts (warp 0; 8 experts per lane)
  if (tid < 32) {
    constexpr int kPer = kMaxExperts / 32;
    int v[kPer];
    int loc = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int ee = tid * kPer + i;
      v[i] = ee < E ? s_kept[ee] : 0;
      loc += v[i];
    }
    int incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (tid >= o) incl += y;
    }
    int run = incl - loc;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int ee = tid * kPer + i;
      if (ee < E) seg_off[ee] = run;
      run += v[i];
    }
    if (tid == 31) seg_off[E] = incl;
  }
  if (clk) {
    __syncthreads();
    stage_clock_end(clk);
  }
}

__global__ void __launch_bounds__(256) dispatch_rank_kernel(const int32_t* __restrict__ idx, int64_t T, int K,
                                                            int E, const int32_t* __restrict__ chunk_base,
                                                            const int32_t* __restrict__ kept,
                                                            const int32_t* __restrict__ seg_off,
                                                            int32_t* __restrict__ slot_of,
                                                            int32_t* __restrict__ perm, unsigned long long* clk) {
  __shared__ uint32_t mask[8][kMaxExperts];
  __shared__ int wbase[8][kMaxExperts];
  pdl_wait();
  pdl_trigger();
  stage_clock_start(clk);
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 8 * E; i += blockDim.x) mask[i / E][i % E] = 0u;
  __syncthreads();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kDispatchChunk + warp * 32 + lane;
  const bool tok_ok = t < T;
  if (tok_ok) {
    for (int k = 0; k < K; ++k) {
      const int e = idx[t * K + k];
      if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) atomicOr(&mask[warp][e], 1u << lane);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = chunk_base[static_cast<int64_t>(blockIdx.x) * E + e];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      wbase[w][e] = run;
      run += __popc(mask[w][e]);
    }
  }
  __syncthreads();
  if (tok_ok) {
    const uint32_t lower = (1u << lane) - 1u;
    for (int k = 0; k < K; ++k) {
      const int64_t pair = t * K + k;
      const int e = idx[pair];
      int slot = -1;
      if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) {
        const int rank = wbase[warp][e] + __popc(mask[warp][e] & lower);
        if (rank < kept[e]) {
          slot = seg_off[e] + rank;
          perm[slot] = static_cast<int32_t>(pair);
        }
      }
      slot_of[pair] = slot;
    }
  }
  if (clk) {
    __syncthreads();
    stage_clock_end(clk);
  }
}

// Fused scan+rank reads n_chunks^2 * E histogram words from L2 in all (every
// block reads all of it); above this the separate scan is cheaper (measured
// even at 256 chunks x 256 experts, 2^24 words).
constexpr long long kFusedScanMaxReads = 1ll << 22;

// Scan and rank in one kernel, one block per 256-token chunk (no block waits
// on another): every block reads the whole [n_chunks, E] histogram (E x
// n_chunks int32, a few KB, from L2) to get each expert's total and the count
// in the chunks before its own, derives kept and seg_off itself, and ranks its
// 256 tokens.  Block 0 also writes counts / kept / seg_off.  With stats !=
// nullptr one more block (number n_chunks) finalises the balance statistics
// from the histogram and the chunk probability sums (fixed point) that the
// selection kernel added: f_e, P_e, the loss, and with zpart the z-loss and
// utilisation statistics.  It runs beside the ranking blocks: a ranking block
// that also did the statistics took 2.5x as long as the others (instrumented
// copy, fine-grained layer: 11.6 vs 4.7 us) and set the kernel's duration.
//   rank(t,k) = (tokens of earlier chunks for e) + (earlier warps of this
//   chunk, by popcount of their lane masks) + popcount of the lower lanes
__global__ void __launch_bounds__(256) dispatch_scan_rank_kernel(
    const int32_t* __restrict__ idx, int64_t T, int K, int E, const int32_t* __restrict__ chunk_counts,
    int n_chunks, long long cap, const int32_t* __restrict__ expert_cap, int32_t* __restrict__ counts,
    int32_t* __restrict__ kept_out, int32_t* __restrict__ seg_off_out, int32_t* __restrict__ slot_of,
    int32_t* __restrict__ perm, const unsigned long long* __restrict__ chunk_psum, float* __restrict__ stats,
    float alpha, const float* __restrict__ zpart, int n_zpart, unsigned long long* clk) {
  __shared__ int s_tot_part[256];
  __shared__ int s_pre_part[256];
  __shared__ int s_tot[kMaxExperts];
  __shared__ int s_pre[kMaxExperts];
  __shared__ int s_kept[kMaxExperts];
  __shared__ int s_seg[kMaxExperts + 1];
  __shared__ uint32_t mask[8][kMaxExperts];
  __shared__ int wbase[8][kMaxExperts];
  __shared__ double s_fp[kMaxExperts];
  __shared__ double s_red[256];
  __shared__ unsigned long long s_ps_part[256];
  pdl_wait();
  pdl_trigger();
  stage_clock_start(clk);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int b = blockIdx.x;
  if (b == n_chunks) {  // the statistics block (launched only with stats)
    // per expert: its count and fixed-point p sum over all chunks (integers,
    // so the sums do not depend on the order); thread (e, sl) takes the
    // chunks c = sl (mod S) with all its loads in flight
    int S = 256 / E;
    if (S > n_chunks) S = n_chunks;
    if (S < 1) S = 1;
    const int e = tid % E, sl = tid / E;
    int tot = 0;
    unsigned long long ps = 0;
    if (tid < E * S) {
#pragma unroll 16
      for (int c = sl; c < n_chunks; c += S) {
        tot += chunk_counts[static_cast<int64_t>(c) * E + e];
        ps += chunk_psum[static_cast<int64_t>(c) * E + e];
      }
    }
    double z = 0.0;
    if (zpart)
      for (int i = tid; i < n_zpart; i += blockDim.x) z += zpart[i];
    s_tot_part[tid] = tot;
    s_ps_part[tid] = ps;
    s_red[tid] = z;
    __syncthreads();
    for (int ee = tid; ee < E; ee += blockDim.x) {
      int tt = 0;
      unsigned long long pp = 0;
      for (int q = 0; q < S; ++q) {
        tt += s_tot_part[q * E + ee];
        pp += s_ps_part[q * E + ee];
      }
      const long long ce = expert_cap ? static_cast<long long>(expert_cap[ee]) : cap;  // Zen MoDE §5.3
      s_tot[ee] = tt;
      s_kept[ee] = (ce < 0 || tt < ce) ? tt : static_cast<int>(ce);
      s_fp[ee] = balance_stats_expert(tt, pp, T, E, K, ee, stats);
    }
    if (zpart) {
      for (int w = 128; w > 0; w >>= 1) {  // fixed-shape tree
        if (tid < w) s_red[tid] += s_red[tid + w];
        __syncthreads();
      }
    }
    __syncthreads();
    if (tid == 0) {
      balance_loss(s_fp, E, alpha, stats);
      if (zpart) utilisation_stats(s_tot, s_kept, E, T, s_red[0], stats);
    }
    if (clk) {
      __syncthreads();
      stage_clock_end(clk);
    }
    return;
  }
  // Every global load that does not depend on another is issued here, before
  // the first barrier, so that their latencies overlap (the kernel is a chain
  // of dependent steps, not bandwidth): this thread's token's experts, its
  // share of the chunk histogram.
  const int64_t t = static_cast<int64_t>(b) * kDispatchChunk + tid;
  const bool tok_ok = t < T;
  constexpr int kKReg = 8;  // the first experts of the token stay in registers
  int my_e[kKReg];
#pragma unroll
  for (int k = 0; k < kKReg; ++k) my_e[k] = (tok_ok && k < K) ? idx[t * K + k] : -1;
  // 1. per expert: total over all chunks and the count in chunks before b.
  //    Thread (e, sl) sums a strided set of chunks; E <= 256 experts, S slices.
  int S = 256 / E;
  if (S > n_chunks) S = n_chunks;
  if (S < 1) S = 1;
  {
    const int e = tid % E, sl = tid / E;
    int tot = 0, pre = 0;
    if (tid < E * S) {
#pragma unroll 16
      for (int c = sl; c < n_chunks; c += S) {
        const int v = chunk_counts[static_cast<int64_t>(c) * E + e];
        tot += v;
        pre += c < b ? v : 0;
      }
    }
    s_tot_part[tid] = tot;
    s_pre_part[tid] = pre;
  }
  for (int i = tid; i < 8 * E; i += blockDim.x) mask[i / E][i % E] = 0u;
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    int tot = 0, pre = 0;
    for (int sl = 0; sl < S; ++sl) {
      tot += s_tot_part[sl * E + e];
      pre += s_pre_part[sl * E + e];
    }
    long long ce = expert_cap ? static_cast<long long>(expert_cap[e]) : cap;  // Zen MoDE §5.3 capacity_e
    s_tot[e] = tot;
    s_pre[e] = pre;
    s_kept[e] = (ce < 0 || tot < ce) ? tot : static_cast<int>(ce);
  }
  __syncthreads();
  // 2. seg_off = exclusive prefix of kept over experts (warp 0; 8 experts per lane)
  if (warp == 0) {
    constexpr int kPer = kMaxExperts / 32;
    int v[kPer];
    int loc = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int ee = lane * kPer + i;
      v[i] = ee < E ? s_kept[ee] : 0;
      loc += v[i];
    }
    int incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - loc;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int ee = lane * kPer + i;
      if (ee < E) s_seg[ee] = run;
      run += v[i];
    }
    if (lane == 31) s_seg[E] = incl;
  }
  // 3. this chunk's lane masks
  if (tok_ok) {
#pragma unroll
    for (int k = 0; k < kKReg; ++k) {
      const int e = my_e[k];
      if (k < K && static_cast<unsigned>(e) < static_cast<unsigned>(E)) atomicOr(&mask[warp][e], 1u << lane);
    }
    for (int k = kKReg; k < K; ++k) {
      const int e = idx[t * K + k];
      if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) atomicOr(&mask[warp][e], 1u << lane);
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    int run = s_pre[e];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      wbase[w][e] = run;
      run += __popc(mask[w][e]);
    }
  }
  if (b == 0) {
    for (int e = tid; e < E; e += blockDim.x) {
      counts[e] = s_tot[e];
      kept_out[e] = s_kept[e];
    }
    for (int e = tid; e <= E; e += blockDim.x) seg_off_out[e] = s_seg[e];
  }
  __syncthreads();
  // 4. ranks and slots
  if (tok_ok) {
    const uint32_t lower = (1u << lane) - 1u;
    auto rank_pair = [&](int k, int e) {
      const int64_t pair = t * K + k;
      int slot = -1;
      if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) {
        const int rank = wbase[warp][e] + __popc(mask[warp][e] & lower);
        if (rank < s_kept[e]) {
          slot = s_seg[e] + rank;
          perm[slot] = static_cast<int32_t>(pair);
        }
      }
      slot_of[pair] = slot;
    };
#pragma unroll
    for (int k = 0; k < kKReg; ++k)
      if (k < K) rank_pair(k, my_e[k]);
    for (int k = kKReg; k < K; ++k) rank_pair(k, idx[t * K + k]);
  }
  if (clk) {
    __syncthreads();
    stage_clock_end(clk);
  }
}

bool dispatch_fused(const Problem& p) {
  const long long n_chunks = (p.T + kDispatchChunk - 1) / kDispatchChunk;
  return n_chunks * n_chunks * p.E <= kFusedScanMaxReads;
}

cudaError_t launch_dispatch(const Problem& p, const int32_t* idx, int32_t* counts, int32_t* kept,
                            int32_t* seg_off, int32_t* slot_of, int32_t* perm, int32_t* chunk_counts,
                            int32_t* chunk_base, unsigned* status, cudaStream_t st, bool counts_ready,
                            const unsigned long long* chunk_psum, float* stats, const float* zpart, int n_zpart,
                            const int32_t* expert_cap, unsigned long long* clk) {
  const int n_chunks = static_cast<int>((p.T + kDispatchChunk - 1) / kDispatchChunk);
  if (!counts_ready) {
    if (cudaError_t e = launch_k(dispatch_hist_kernel, dim3(n_chunks), dim3(256), 0, st, idx, p.T, p.K, p.E,
                                 chunk_counts, status))
      return e;
  }
  if (dispatch_fused(p))
    return launch_k(dispatch_scan_rank_kernel, dim3(n_chunks + (chunk_psum && stats ? 1 : 0)), dim3(256), 0, st,
                    idx, p.T, p.K, p.E,
                    static_cast<const int32_t*>(chunk_counts), n_chunks, static_cast<long long>(p.cap), expert_cap,
                    counts, kept, seg_off, slot_of, perm, chunk_psum, chunk_psum ? stats : nullptr, p.alpha, zpart,
                    n_zpart, clk);
  if (cudaError_t e = launch_k(dispatch_scan_kernel, dim3(1), dim3(1024), 0, st,
                               static_cast<const int32_t*>(chunk_counts), n_chunks, p.E, static_cast<long long>(p.cap),
                               chunk_base, counts, kept, seg_off, chunk_psum, chunk_psum ? stats : nullptr, p.T,
                               p.K, p.alpha, zpart, n_zpart, expert_cap, clk))
    return e;
  return launch_k(dispatch_rank_kernel, dim3(n_chunks), dim3(256), 0, st, idx, p.T, p.K, p.E,
                  static_cast<const int32_t*>(chunk_base), static_cast<const int32_t*>(kept),
                  static_cast<const int32_t*>(seg_off), slot_of, perm, clk);
}

constexpr int kGatherUnroll = 8;

// Row gather: one warp per destination row, 16-byte vectors.  Rows at or past
// seg_off[E] (the kept total) are left untouched.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x,
                                                          const int32_t* __restrict__ perm,
                                                          const int32_t* __restrict__ seg_off, int E, int K,
                                                          int64_t T, int vec_per_row, int64_t max_rows,
                                                          uint4* __restrict__ x_perm, unsigned long long* clk) {
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  stage_clock_start(clk);
  const int64_t n_rows = seg_off[E];
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = warp0; r < n_rows && r < max_rows; r += n_warps) {
    const int64_t tok = perm[r] / K;
    if (tok < 0 || tok >= T) continue;
    const uint4* src = x + tok * vec_per_row;
    uint4* dst = x_perm + r * vec_per_row;
    // up to kGatherUnroll 16-byte loads in flight per lane before any store
    for (int v0 = lane; v0 < vec_per_row; v0 += 32 * kGatherUnroll) {
      uint4 buf[kGatherUnroll];
#pragma unroll
      for (int j = 0; j < kGatherUnroll; ++j)
        if (v0 + 32 * j < vec_per_row) buf[j] = __ldg(src + v0 + 32 * j);
#pragma unroll
      for (int j = 0; j < kGatherUnroll; ++j)
        if (v0 + 32 * j < vec_per_row) dst[v0 + 32 * j] = buf[j];
    }
  }
  if (clk) {
    __syncthreads();
    stage_clock_end(clk);
  }
}

cudaError_t launch_gather(const Problem& p, const void* x, const int32_t* perm, const int32_t* seg_off,
                          void* x_perm, cudaStream_t st, unsigned long long* clk) {
  if (p.max_rows <= 0) return cudaSuccess;
  const int vec_per_row = static_cast<int>(p.d * p.esize() / 16);
  int64_t blocks = (p.max_rows + 7) / 8;
  const int64_t cap_blocks = static_cast<int64_t>(num_sms()) * 16;
  if (blocks > cap_blocks) blocks = cap_blocks;
  return launch_k(gather_rows_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st,
                  static_cast<const uint4*>(x), perm, seg_off, p.E, p.K, p.T, vec_per_row, p.max_rows,
                  static_cast<uint4*>(x_perm), clk);
}

// Segment regrouping (moe_expert_ffn_segments): segment s holds expert s % E
// (source s / E); expert-major order lists every source's rows of expert 0,
// then of expert 1, ... (sources ascending inside each expert).  One thread:
// n_seg <= kMaxSegments.
__global__ void segment_regroup_plan_kernel(const int32_t* __restrict__ seg_off, int n_seg, int E,
                                            int32_t* __restrict__ dst_off, int32_t* __restrict__ expert_off) {
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x != 0) return;
  const int n_src = (n_seg + E - 1) / E;
  int run = 0;
  for (int e = 0; e < E; ++e) {
    expert_off[e] = run;
    for (int s = 0; s < n_src; ++s) {
      const int seg = s * E + e;
      if (seg >= n_seg) continue;
      dst_off[seg] = run;
      run += seg_off[seg + 1] - seg_off[seg];
    }
  }
  expert_off[E] = run;
}

// Row r of segment s (segment order) <-> row dst_off[s] + (r - seg_off[s])
// (expert-major order); one warp per row, 16-byte vectors.
__global__ void __launch_bounds__(256) segment_copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                           const int32_t* __restrict__ seg_off,
                                                           const int32_t* __restrict__ dst_off, int n_seg,
                                                           int64_t n_rows, int vec_per_row, int to_expert) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t rows = min(n_rows, static_cast<int64_t>(seg_off[n_seg]));
  for (int64_t r = warp0; r < rows; r += n_warps) {
    int lo = 0, hi = n_seg - 1;  // the segment holding row r: largest s with seg_off[s] <= r
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (seg_off[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int64_t q = dst_off[lo] + (r - seg_off[lo]);
    if (q < 0 || q >= n_rows) continue;
    const uint4* from = src + (to_expert ? r : q) * vec_per_row;
    uint4* to = dst + (to_expert ? q : r) * vec_per_row;
    for (int v0 = lane; v0 < vec_per_row; v0 += 32 * kGatherUnroll) {
      uint4 buf[kGatherUnroll];
#pragma unroll
      for (int j = 0; j < kGatherUnroll; ++j)
        if (v0 + 32 * j < vec_per_row) buf[j] = from[v0 + 32 * j];
#pragma unroll
      for (int j = 0; j < kGatherUnroll; ++j)
        if (v0 + 32 * j < vec_per_row) to[v0 + 32 * j] = buf[j];
    }
  }
}

cudaError_t launch_segment_regroup_plan(const int32_t* seg_off, int n_seg, int E, int32_t* dst_off,
                                        int32_t* expert_off, cudaStream_t st) {
  return launch_k(segment_regroup_plan_kernel, dim3(1), dim3(32), 0, st, seg_off, n_seg, E, dst_off, expert_off);
}

cudaError_t launch_segment_copy(const void* src, void* dst, const int32_t* seg_off, const int32_t* dst_off, int n_seg,
                                int64_t n_rows, int row_bytes, bool to_expert, cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  int64_t blocks = (n_rows + 7) / 8;
  const int64_t cap_blocks = static_cast<int64_t>(num_sms()) * 16;
  if (blocks > cap_blocks) blocks = cap_blocks;
  return launch_k(segment_copy_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st,
                  static_cast<const uint4*>(src), static_cast<uint4*>(dst), seg_off, dst_off, n_seg, n_rows,
                  row_bytes / 16, to_expert ? 1 : 0);
}

}  // namespace moe
