// Fused router: the gate GEMM on the tensor cores, then softmax, top-K
// selection (optional selection bias), renormalised gate weights and the
// per-chunk balance statistics, in one launch.
//
//   Zen MoDE: Mixture of Distilled Experts Architecture, §3.1 Router
//     Architecture, eq. router_standard: TopK(softmax(W_r x), K).
//   Zen-Max, §2.3 Auxiliary-Loss-Free Load Balancing: s_ij = softmax(x_i W_g)_j + b_j
//     (the bias steers the choice; the gate weights use the unbiased softmax).
//   Scaling with experts, "The gating network": only the k best scores stay
//     non-zero, rescaled to add up to 1.  "A balance penalty": f_i and P_i.
//
// Work decomposition.  A tile is 128 tokens.  The reduction over d_model is
// split across a thread-block cluster of C CTAs (C = 1, 2, 4 or 8): CTA r of
// the cluster streams its contiguous share of the 64-wide k chunks of x (TMA,
// 128-byte swizzle) and of W_g, and accumulates a 128 x E_pad FP32 partial in
// TMEM with tcgen05.mma (M = 128 tokens, N = E_pad).  Each CTA owns 128 / C
// of the tile's tokens: after its MMAs every CTA writes its partial (128 rows)
// into its own shared memory (over its now idle TMA ring), a cluster barrier
// makes the partials visible, and the owner of a token reads that token's row
// from every CTA of the cluster (ld.shared::cluster, one coalesced 128-byte
// line per warp and instruction; no round trip through L2 or HBM) and adds the
// C partials in CTA order (deterministic) plus the logit offset.  A second
// cluster barrier keeps every CTA's shared memory alive until its peers have
// read it.  So x is read from HBM once, W_g from L2, and the logits are
// written once (moe_route returns them).
//
// Selection: kRtSelWarps warps per CTA, a group of G lanes per token (32 / G
// tokens per warp at a time; lane l of a group holds experts l, l + G, ...),
// the same per-token code as the selection kernel (router_select.cuh): softmax, K rounds of a warp arg-max over
// order-preserving keys, renormalised gate weights; a selection bias on p is
// screened in float32 and re-ranked in float64 where two of the best K+1
// scores are within rounding of each other.  Many warps per SM keep the
// per-token dependency chains (shuffles, reductions) overlapped.
//
// Warp roles (64 + 32 kRtSelWarps threads): warp 0 TMA producer, warp 1 TMEM
// owner and MMA issuer, warps 2.. TMEM drain, then selection.  Every wait is bounded
// (mbar_wait); on a timeout the kernel records MOE_DEV_WAIT_TIMEOUT, drains
// its own copies and MMAs, still joins both cluster barriers, frees TMEM and
// exits.
#include <cooperative_groups.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "router_select.cuh"

namespace moe {

constexpr int kRtSelWarps = 8;                    // TMEM drain warps (2 per lane quarter)
constexpr int kRtWarps = 2 + kRtSelWarps;          // every warp takes part in the selection
constexpr int kRtThreads = 32 * kRtWarps;
constexpr int kRtBM = 128;                     // tokens per tile (MMA M)
constexpr int kRtXBytes = kRtBM * 64 * 2;      // one 64-deep chunk of x: 16 KB

struct RouterArgs {
  int64_t T;
  int d, E, K;
  int n_kc;           // 64-wide chunks of d
  int csize;          // CTAs per cluster (split of the reduction)
  int stages;         // TMA ring depth
  int bias_mode;      // 0 none, 1 on p, 2 on the logit
  const float* offset;    // [E] or nullptr
  const float* sel_bias;  // [E] or nullptr
  float* logits;          // [T, E] out
  int32_t* topk_idx;      // [T, K] out
  float* topk_w;          // [T, K] out
  int32_t* chunk_counts;  // [chunks, E] += chosen counts
  unsigned long long* chunk_psum;  // [chunks, E] += sum of p, fixed point
  double pscale;
  float* zpart;           // [grid] sums of logsumexp^2, or nullptr
  unsigned* status;
  unsigned long long* clk;  // stage clock, or nullptr
  unsigned long long stall_ns;  // abort-path test hook (test_stall), 0 normally
  int select;  // 1: rank the tokens here; 0: only write the logits (a selection kernel follows)
};

// Shared-memory carve-up (bytes from the 1024-aligned base), the same on host
// and device.
struct RtLayout {
  int stage_bytes, main_bytes, part_stride;  // part_stride in floats
  int cnt_off, psum_off, z_off, bias_off, off_off, bar_off, total;
};

__host__ __device__ inline RtLayout rt_layout(int epad, int stages) {
  RtLayout L;
  L.stage_bytes = kRtXBytes + epad * 128;
  L.part_stride = epad + 4;  // rows 16 bytes apart in bank order: the row-per-thread stores do not conflict
  const int ring = stages * L.stage_bytes;
  const int part = kRtBM * L.part_stride * 4;
  L.main_bytes = ((ring > part ? ring : part) + 1023) & ~1023;
  L.cnt_off = L.main_bytes;                            // [epad] chosen counts
  L.psum_off = L.cnt_off + epad * 4;                   // [kRtWarps][epad] sums of p
  L.z_off = L.psum_off + kRtWarps * epad * 4;          // [kRtWarps] sums of logsumexp^2
  L.bias_off = L.z_off + kRtWarps * 4;                 // [epad]
  L.off_off = L.bias_off + epad * 4;                   // [epad]
  L.bar_off = (L.off_off + epad * 4 + 7) & ~7;         // full[stages], empty[stages], tfull, drain, tmem slot, abort
  L.total = L.bar_off + (2 * stages + 2) * 8 + 16;
  return L;
}


template <int EPAD, int G>
__global__ void __launch_bounds__(kRtThreads, 2)
    router_fused_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                        const __grid_constant__ RouterArgs a) {
  // selection: groups of G lanes per token (32 / G tokens per warp at once),
  // EPL experts per lane
  constexpr int EPL = EPAD <= G ? 1 : EPAD / G;
  constexpr int TPW = 32 / G;
  // tokens a group ranks at once (their reduction chains overlap): two for a
  // whole warp per token (up to 128 experts), else one
  constexpr int NT = (G == 32 && EPL <= 4) ? 2 : 1;
  constexpr uint32_t kTmemCols = EPAD < 32 ? 32 : EPAD;
  constexpr int kWBytes = EPAD * 128;
  constexpr int NS = kRtSelWarps;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int C = a.csize;
  const int TPC = kRtBM / C;  // tokens owned by this CTA
  const RtLayout L = rt_layout(EPAD, a.stages);
  float* part = reinterpret_cast<float*>(smem);  // [128][part_stride] this CTA's partial, over the ring
  int* s_count = reinterpret_cast<int*>(smem + L.cnt_off);
  float* s_psum = reinterpret_cast<float*>(smem + L.psum_off);
  float* s_z = reinterpret_cast<float*>(smem + L.z_off);
  float* s_bias = reinterpret_cast<float*>(smem + L.bias_off);
  float* s_off = reinterpret_cast<float*>(smem + L.off_off);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* empty = full + a.stages;
  uint64_t* tfull = empty + a.stages;
  uint64_t* drain = tfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int tile = static_cast<int>(blockIdx.x) / C;
  const int64_t row0 = static_cast<int64_t>(tile) * kRtBM;
  const int kc0 = static_cast<int>((static_cast<int64_t>(a.n_kc) * rank) / C);
  const int nk = static_cast<int>((static_cast<int64_t>(a.n_kc) * (rank + 1)) / C) - kc0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();  // from here on the predecessor's outputs (x, the bias) are read
  pdl_trigger();
  stage_clock_start(a.clk);
  for (int e = threadIdx.x; e < EPAD; e += blockDim.x) {
    s_count[e] = 0;
    s_bias[e] = (a.sel_bias && e < a.E) ? a.sel_bias[e] : 0.f;
    s_off[e] = (a.offset && e < a.E) ? a.offset[e] : 0.f;
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t stage_bytes = static_cast<uint32_t>(kRtXBytes + kWBytes);
      uint32_t issued = 0, last_par = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % a.stages;
        const uint32_t ph = static_cast<uint32_t>(kb / a.stages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) break;
        uint8_t* sx = smem + s * L.stage_bytes;
        mbar_arrive_expect_tx(&full[s], stage_bytes);
        tma_load_2d(sx, &tmX, &full[s], (kc0 + kb) * 64, static_cast<int>(row0));
        tma_load_2d(sx + kRtXBytes, &tmW, &full[s], (kc0 + kb) * 64, 0);
        issued |= 1u << s;
        last_par = (last_par & ~(1u << s)) | (ph << s);
      }
      if (*abort_flag) {  // let every copy this thread started land before the ring is reused or freed
        int never = 0;
        for (int s = 0; s < a.stages && s < 32; ++s)
          if ((issued >> s) & 1u) mbar_wait(&full[s], (last_par >> s) & 1u, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kRtBM, EPAD);
      bool ok = test_stall(drain, abort_flag, a.stall_ns);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % a.stages;
        const uint32_t ph = static_cast<uint32_t>(kb / a.stages) & 1u;
        if (!mbar_wait(&full[s], ph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint64_t adesc = smem_desc_k128(smem_addr(smem + s * L.stage_bytes));
        const uint64_t bdesc = smem_desc_k128(smem_addr(smem + s * L.stage_bytes + kRtXBytes));
#pragma unroll
        for (int k = 0; k < 4; ++k) umma_bf16(tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      if (ok) umma_commit(tfull);
      if (*abort_flag) {  // every MMA this thread issued completes before TMEM is freed
        umma_commit(drain);
        int never = 0;
        mbar_wait(drain, 0, &never);
      }
    }
  }
  if (warp >= 2) {
    // ------------------------------------------------- TMEM -> own smem
    // Warp w drains TMEM lanes [32 (w % 4), +32), the rows of those tokens;
    // the NS / 4 warps of a lane quarter take every (NS / 4)-th 32-column
    // block.  The ring is idle once the last MMA has completed.
    const int quarter = warp & 3;
    if (__all_sync(0xffffffffu, mbar_wait(tfull, 0, abort_flag))) {
      tc_fence_after_sync();
      float* row = part + (quarter * 32 + lane) * L.part_stride;
      for (int c = 32 * ((warp - 2) >> 2); c < EPAD; c += 32 * (NS / 4)) {
        uint32_t v[32];
        tmem_load_32x32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(c), v);
        tmem_load_wait();
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (c + 4 * u < EPAD)
            *reinterpret_cast<float4*>(row + c + 4 * u) =
                make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]), __uint_as_float(v[4 * u + 2]),
                            __uint_as_float(v[4 * u + 3]));
      }
    }
    tc_fence_before_sync();
  }
  // every CTA's partial is in its shared memory and visible cluster-wide
  cluster_sync();

  if (!a.select) {
    // --------------------------------------------- the logits only (warp per row)
    cooperative_groups::cluster_group cluster = cooperative_groups::this_cluster();
    const float* peer[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) peer[q] = q < C ? cluster.map_shared_rank(part, static_cast<unsigned>(q)) : part;
    for (int tl = warp; tl < TPC; tl += kRtWarps) {
      const int64_t t = row0 + static_cast<int64_t>(rank) * TPC + tl;
      if (t >= a.T) break;
      const int row = (static_cast<int>(rank) * TPC + tl) * L.part_stride;
      for (int e = lane; e < a.E; e += 32) {
        float pv[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) pv[q] = q < C ? peer[q][row + e] : 0.f;
        float v = pv[0];
#pragma unroll
        for (int q = 1; q < 8; ++q)
          if (q < C) v += pv[q];
        a.logits[t * a.E + e] = v + s_off[e];
      }
    }
  } else {
    // ------------------------------------------------------------ selection
    // every warp: the TMA and MMA warps are idle from here on
    constexpr int NW = kRtWarps;
    const int sw = warp;
    const int gl = lane & (G - 1);  // lane within the token's group
    const bool has_bias = a.bias_mode != 0;
    // the partials of every CTA of the cluster, read through generic
    // addresses of distributed shared memory (plain loads: the compiler keeps
    // a token's loads in flight together)
    cooperative_groups::cluster_group cluster = cooperative_groups::this_cluster();
    const float* peer[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) peer[q] = q < C ? cluster.map_shared_rank(part, static_cast<unsigned>(q)) : part;
    float pacc[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) pacc[i] = 0.f;
    float zacc = 0.f;
    // group slot g = (warp, group within the warp) takes the NT tokens
    // [g NT, g NT + NT) of each round of NW TPW NT tokens
    for (int base = (sw * TPW + lane / G) * NT; base < TPC; base += NW * TPW * NT) {
      float lg[NT][EPL], bias[EPL];
      bool live[NT];
      int32_t* irow[NT];
      float* wrow[NT];
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = gl + G * i;
        bias[i] = e < EPAD ? s_bias[e] : 0.f;
      }
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int tl = base + n;
        const int64_t t = row0 + static_cast<int64_t>(rank) * TPC + tl;
        live[n] = tl < TPC && t < a.T;  // the same for the whole group
        irow[n] = a.topk_idx + t * a.K;
        wrow[n] = a.topk_w + t * a.K;
        // the logits: the C partials in CTA order, then the offset
        const int row = (static_cast<int>(rank) * TPC + (live[n] ? tl : 0)) * L.part_stride;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const int e = gl + G * i;
          float v = 0.f;
          if (e < EPAD && live[n]) {
            float pv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) pv[q] = q < C ? peer[q][row + e] : 0.f;
            v = pv[0];
#pragma unroll
            for (int q = 1; q < 8; ++q)
              if (q < C) v += pv[q];
            v += s_off[e];
          }
          if (live[n] && e < a.E) a.logits[t * a.E + e] = v;
          lg[n][i] = e < a.E ? v : -INFINITY;
        }
      }
      if (live[0])
        select_tokens<EPL, G, NT>(lg, bias, has_bias, a.bias_mode == 2, a.E, a.K, lane, live, pacc, zacc, irow, wrow,
                                  s_count);
    }
    // this CTA's sums of p per expert and of logsumexp^2: over the warp's
    // groups, then over the warps in order
    __syncwarp();
#pragma unroll
    for (int i = 0; i < EPL; ++i)
#pragma unroll
      for (int o = G; o < 32; o <<= 1) pacc[i] += __shfl_xor_sync(0xffffffffu, pacc[i], o);
    float zw = gl == 0 ? zacc : 0.f;
#pragma unroll
    for (int o = G; o < 32; o <<= 1) zw += __shfl_xor_sync(0xffffffffu, zw, o);
    if (lane < G) {
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (lane + G * i < EPAD) s_psum[sw * EPAD + lane + G * i] = pacc[i];
    }
    if (lane == 0) s_z[sw] = zw;
    __syncthreads();
    const int64_t chunk = row0 / kDispatchChunk;
    for (int e = threadIdx.x; e < a.E; e += kRtThreads) {
      float ps = 0.f;
      for (int w = 0; w < NW; ++w) ps += s_psum[w * EPAD + e];
      if (ps > 0.f) atomicAdd(&a.chunk_psum[chunk * a.E + e], __double2ull_rn(static_cast<double>(ps) * a.pscale));
      if (s_count[e]) atomicAdd(&a.chunk_counts[chunk * a.E + e], s_count[e]);
    }
    if (a.zpart && threadIdx.x == 0) {
      float z = 0.f;
      for (int w = 0; w < NW; ++w) z += s_z[w];
      a.zpart[blockIdx.x] = z;
    }
  }

  // no CTA leaves while a peer may still read its partial
  cluster_sync();
  stage_clock_end(a.clk);
  if (threadIdx.x == 0 && *abort_flag) raise_status(a.status, kDevWaitTimeout);
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
static int rt_epad(int E) { return E <= 16 ? 16 : E <= 32 ? 32 : E <= 64 ? 64 : E <= 128 ? 128 : 256; }

struct RtPlan {
  int epad, csize, stages, smem, tiles;
};

// CTAs per SM the plan aims for: 2 (about half an SM's shared memory each)
// unless MOE_B200_ROUTER_OCC=1 (all of it).
static int rt_occupancy() {
  static const int v = [] {
    const char* e = getenv("MOE_B200_ROUTER_OCC");
    return (e && e[0] == '1') ? 1 : 2;
  }();
  return v;
}

// Split and ring depth: the largest split c (CTAs per cluster, at most 8 and
// at most the number of k chunks) whose tiles x c CTAs all fit on the SMs at
// once, and the deepest ring the shared-memory budget allows.  Two CTAs per SM
// when the receive buffer leaves room for a ring of two stages in half an SM.
// (The cluster occupancy query of the runtime is more pessimistic than what
// the device runs: 64 clusters of 4 CTAs at 105 KB started within 1.4 us.)
static RtPlan rt_plan(const Problem& p, int epad) {
  RtPlan pl{};
  pl.epad = epad;
  pl.tiles = static_cast<int>((p.T + kRtBM - 1) / kRtBM);
  const int n_kc = (p.d + 63) / 64;
  int occ = rt_occupancy();
  if (occ == 2 && rt_layout(epad, 2).total + 1024 > 110 * 1024) occ = 1;
  const int budget = (occ == 2 ? 110 : 220) * 1024;
  const int64_t slots = static_cast<int64_t>(num_sms()) * occ;
  int c = 8;
  while (c > 1 && (c > n_kc || static_cast<int64_t>(pl.tiles) * c > slots)) c >>= 1;
  pl.csize = c;
  const int nk_max = (n_kc + c - 1) / c;
  int stages = 1;
  while (stages < nk_max && stages < 16 && rt_layout(epad, stages + 1).total + 1024 <= budget) ++stages;
  pl.stages = stages;
  pl.smem = rt_layout(epad, stages).total + 1024;
  return pl;
}

template <int EPAD, int G>
static cudaError_t run_router(const Problem& p, const CUtensorMap& tx, const CUtensorMap& tw, RouterArgs a,
                              cudaStream_t st, int* n_zpart) {
  const RtPlan pl = rt_plan(p, EPAD);
  auto kern = router_fused_kernel<EPAD, G>;
  // the dynamic shared-memory opt-in is per device: set it once per device
  static std::mutex mu;
  static uint64_t configured = 0;
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev)) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!((configured >> dev) & 1u)) {
      if (cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024))
        return e;
      configured |= uint64_t(1) << dev;
    }
  }
  a.csize = pl.csize;
  a.stages = pl.stages;
  *n_zpart = pl.tiles * pl.csize;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.tiles * pl.csize));
  cfg.blockDim = dim3(kRtThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(pl.smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(pl.csize);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, tx, tw, a);
}

bool router_fused_ok(const Problem& p) {
  static const bool off = [] {
    const char* e = getenv("MOE_B200_ROUTER_FUSED");
    return e && e[0] == '0';
  }();
  return !off && p.dtype == kBF16 && !(p.flags & 0x1u /* MOE_FLAG_LOGITS_GIVEN */) && p.E <= kMaxExperts &&
         p.T <= (static_cast<int64_t>(1) << 31) - kRtBM;
}

// Where the tokens are ranked: in this kernel, unless MOE_B200_ROUTER_SPLIT=1
// (then it only writes the logits and the selection kernel ranks them, with
// more warps per SM).  In place on all four BF16 workloads the single launch
// was the faster (device-stamped spans, same box: 17.4 / 25.8 / 32.4 / 12.1 us
// against 23.5 / 32.3 / 38.3 / 17.0 us for mixtral / zen_fine / skewed /
// decode): the second launch and the logits' round trip through L2 cost more
// than the extra warps save.
bool router_selects(const Problem& p) {
  (void)p;
  const char* e = getenv("MOE_B200_ROUTER_SPLIT");
  return !(e && e[0] == '1');
}

int router_fused_zparts(const Problem& p) {
  // every CTA writes one partial; at most 8 CTAs per 128-token tile
  return static_cast<int>((p.T + kRtBM - 1) / kRtBM) * 8;
}

cudaError_t launch_router_fused(const Problem& p, const void* x, const void* w_gate, const float* offset,
                                const float* sel_bias, float* logits, int32_t* topk_idx, float* topk_w,
                                int32_t* chunk_counts, unsigned long long* chunk_psum, float* zpart,
                                unsigned* status, cudaStream_t st, int* n_zpart, unsigned long long* clk,
                                bool select) {
  const int epad = rt_epad(p.E);
  CUtensorMap tx, tw;
  const uint64_t dx[2] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(p.T)};
  const uint32_t bx[2] = {64, static_cast<uint32_t>(kRtBM)};
  const uint64_t dw[2] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(p.E)};
  const uint32_t bw[2] = {64, static_cast<uint32_t>(epad)};
  if (!make_map(&tx, x, 2, dx, bx) || !make_map(&tw, w_gate, 2, dw, bw)) return cudaErrorInvalidValue;
  RouterArgs a{};
  a.T = p.T;
  a.d = p.d;
  a.E = p.E;
  a.K = p.K;
  a.n_kc = (p.d + 63) / 64;
  a.bias_mode = sel_bias ? ((p.flags & 0x2u /* MOE_FLAG_BIAS_LOGIT */) ? 2 : 1) : 0;
  a.offset = offset;
  a.sel_bias = sel_bias;
  a.logits = logits;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.chunk_counts = chunk_counts;
  a.chunk_psum = chunk_psum;
  a.pscale = p_fixed_scale(p.T);
  a.zpart = zpart;
  a.status = status;
  a.clk = clk;
  a.stall_ns = test_stall_ns();
  a.select = select ? 1 : 0;
  switch (epad) {
    case 16:  // one expert per lane, a group of 8 or 16 lanes per token
      return p.E <= 8 ? run_router<16, 8>(p, tx, tw, a, st, n_zpart) : run_router<16, 16>(p, tx, tw, a, st, n_zpart);
    case 32: return run_router<32, 32>(p, tx, tw, a, st, n_zpart);
    case 64: return run_router<64, 32>(p, tx, tw, a, st, n_zpart);
    case 128: return run_router<128, 32>(p, tx, tw, a, st, n_zpart);
    default: return run_router<256, 32>(p, tx, tw, a, st, n_zpart);
  }
}

}  // namespace moe
