// Backward GEMMs of the expert FFNs on the tensor cores (tcgen05.mma, TMEM
// accumulators, TMA-staged operands), for training.
//
//   Zen-Max, §2.2 Fine-Grained Expert Architecture, eq. Expert_i:
//       o = W_down (SiLU(W_gate x) (.) W_up x)
//   With do the gradient at an expert's output (the token's dy times its gate
//   weight, or dy itself for a shared expert):
//       dh = W_down^T do;  dg = dh u silu'(g);  du = dh silu(g)
//       dx = W_gate^T dg + W_up^T du;  dW_down = do h^T;  dW_gate = dg x^T;  dW_up = du x^T
//
// Two shapes, one warp-specialised kernel (warp 0 TMA, warp 1 MMA, warps 2-5
// epilogue; 128 x 256 tiles, 64-deep k-blocks, double-buffered TMEM):
//   dgrad  M = a group's token rows, N = output columns, K fixed:
//          A = activations (token rows, K-major), B = the group's weights read
//          MN-major (the weights are stored [out, in] for the forward, so the
//          backward contracts over their row index).  Epilogues:
//            DSWIGLU  dh tile -> dg, du with g, u read from the recomputed
//                     gate/up projections; stores dGU [rows, 2F] (dg | du)
//            BF16     dX rows
//   wgrad  M, N = the weight's shape, K = the group's token rows: A and B are
//          activations read MN-major (rows = tokens); the k-block that runs
//          past the group's last row has those rows of A and B zeroed in shared
//          memory before its MMAs, so rows of the next group add nothing.
//          Stores the FP32 weight gradient (zeros for a group without rows).
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {

enum { GMODE_DGRAD = 0, GMODE_WGRAD = 1 };
enum { GEPI_DSWIGLU = 0, GEPI_BF16 = 1, GEPI_F32 = 2 };

constexpr int kGBM = 128;
constexpr int kGBN = 256;
constexpr int kGBK = 64;
constexpr int kGStages = 4;
constexpr int kGThreads = 192;
constexpr int kGMaxGroups = 256;
constexpr int kGABytes = kGBM * kGBK * 2;  // 16 KB
constexpr int kGBBytes = kGBN * kGBK * 2;  // 32 KB: four 64-column MN chunks of 64 K rows
constexpr int kGStageBytes = kGABytes + kGBBytes;
constexpr int kGChunk = 64 * kGBK * 2;  // one MN chunk (64 elements x 64 K rows) = 8 KB
// Room left after the ring, so that the operand descriptors of the last stage
// stay inside the allocation whatever they address.
constexpr int kGSlack = 32 * 1024;

constexpr int grad_smem_bytes() {
  return kGStages * kGStageBytes + kGSlack + 256 + 4 * (kGMaxGroups + 1) + 1024;
}
static_assert(grad_smem_bytes() <= 232448, "exceeds the per-block shared-memory limit");

struct GradArgs {
  int n_groups;
  const int32_t* seg_off;  // [n_groups + 1] token-row offsets, or nullptr: every group covers [0, n_rows)
  int n_rows;
  // dgrad: N output columns; reduction kdim per group matrix, k_groups matrices summed
  // wgrad: m_dim x n_dim output per group
  int n_dim, m_dim;
  int kdim, k_groups;
  int a_col_group;  // wgrad: group g's A block starts at column g * a_col_group
  int b_col_group;  // wgrad: group g's B block starts at column g * b_col_group
  void* out;
  int64_t ldo;               // output row stride (elements)
  int out_col_stride;        // dgrad: output column offset per group
  int64_t out_group_stride;  // wgrad: output element offset per group
  const __nv_bfloat16* gu;   // DSWIGLU: recomputed projections, g at column gu_col + f, u at gu_col + F + f
  int64_t ld_gu;
  int gu_group_cols;         // gu_col = group * gu_group_cols
  int F;
  unsigned* status;
  // 1: the MN-major operand's 64-column chunks of a k-block come in one box
  // (maps (64, K rows, columns/64[, matrices]), chunk stride 128 bytes)
  int merged_a, merged_b;
};

// Token rows [base, base + return) of group g, clamped to [0, n_rows).
__device__ __forceinline__ int grad_group_rows(const GradArgs& a, int g, int* base) {
  int b = 0, rows = a.n_rows;
  if (a.seg_off) {
    b = min(max(a.seg_off[g], 0), a.n_rows);
    rows = min(max(a.seg_off[g + 1], b), a.n_rows) - b;
  }
  *base = b;
  return rows;
}

struct GradTile {
  int g, m0, n0;
  int row_base, rows;  // the group's token rows
};

// Tiles per group: dgrad ceil(rows/128) x ceil(N/256); wgrad ceil(M/128) x ceil(N/256).
template <int MODE>
__device__ __forceinline__ int grad_tiles_of(const GradArgs& a, int g) {
  const int nt = (a.n_dim + kGBN - 1) / kGBN;
  if (MODE == GMODE_WGRAD) return ((a.m_dim + kGBM - 1) / kGBM) * nt;
  int base;
  return ((grad_group_rows(a, g, &base) + kGBM - 1) / kGBM) * nt;
}

template <int MODE>
__device__ __forceinline__ void grad_prefix_warp(const GradArgs& a, int* prefix, int lane) {
  const int per = (a.n_groups + 31) / 32;
  int local = 0;
  for (int i = 0; i < per; ++i) {
    const int g = lane * per + i;
    if (g < a.n_groups) local += grad_tiles_of<MODE>(a, g);
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int run = incl - local;
  for (int i = 0; i < per; ++i) {
    const int g = lane * per + i;
    if (g < a.n_groups) {
      prefix[g] = run;
      run += grad_tiles_of<MODE>(a, g);
    }
  }
  if (lane == 31) prefix[a.n_groups] = incl;
}

template <int MODE>
__device__ __forceinline__ GradTile grad_decode(int tile, const int* prefix, const GradArgs& a) {
  int lo = 0, hi = a.n_groups - 1;
  while (lo < hi) {  // largest g with prefix[g] <= tile (a group with tiles)
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  GradTile t;
  t.g = lo;
  t.rows = grad_group_rows(a, lo, &t.row_base);
  const int mt = MODE == GMODE_WGRAD ? (a.m_dim + kGBM - 1) / kGBM : (t.rows + kGBM - 1) / kGBM;
  const int local = tile - prefix[lo];
  const int n_idx = local / mt;
  const int m_idx = local - n_idx * mt;
  t.m0 = m_idx * kGBM;  // dgrad: row offset within the group; wgrad: output row
  t.n0 = n_idx * kGBN;
  return t;
}

// k-blocks of a tile: dgrad a fixed count, wgrad the group's rows in 64s.
template <int MODE>
__device__ __forceinline__ int grad_nkb(const GradArgs& a, const GradTile& t) {
  if (MODE == GMODE_WGRAD) return (t.rows + kGBK - 1) / kGBK;
  return ((a.kdim + kGBK - 1) / kGBK) * a.k_groups;
}

// Epilogue of one accumulator: this thread's TMEM lane r (0..127) holds row
// m0 + r of the tile, 256 columns from t_lane.  Every lane calls it (the TMEM
// loads are warp-collective); `zero` (wgrad, no rows in the group) stores
// zeros without reading TMEM.
template <int MODE, int EPI>
__device__ __forceinline__ void grad_epilogue(const GradArgs& a, const GradTile& t, int r, uint32_t t_lane,
                                              bool zero) {
  if (EPI == GEPI_F32) {
    const int m = t.m0 + r;
    float* orow = static_cast<float*>(a.out) + static_cast<int64_t>(t.g) * a.out_group_stride +
                  static_cast<int64_t>(m) * a.ldo;
    const bool row_ok = m < a.m_dim;
#pragma unroll 1
    for (int c = 0; c < kGBN; c += 32) {
      uint32_t v[32];
      if (!zero) {
        tmem_load_32x32(t_lane + static_cast<uint32_t>(c), v);
        tmem_load_wait();
      }
      if (row_ok) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int n = t.n0 + c + 4 * q;
          if (n < a.n_dim) {
            const float4 val = zero ? make_float4(0.f, 0.f, 0.f, 0.f)
                                    : make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                                  __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
            *reinterpret_cast<float4*>(orow + n) = val;
          }
        }
      }
    }
    return;
  }
  // dgrad: row = token
  const int tok = t.row_base + t.m0 + r;
  const bool row_ok = t.m0 + r < t.rows;
  __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) + static_cast<int64_t>(row_ok ? tok : 0) * a.ldo +
                        static_cast<int64_t>(t.g) * a.out_col_stride;
#pragma unroll 1
  for (int c = 0; c < kGBN; c += 32) {
    uint32_t v[32];
    tmem_load_32x32(t_lane + static_cast<uint32_t>(c), v);
    tmem_load_wait();
    if (!row_ok) continue;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int n = t.n0 + c + 8 * q;
      if (n >= a.n_dim) continue;
      if (EPI == GEPI_BF16) {
        uint32_t pk[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          pk[j] = pack_bf16x2(__uint_as_float(v[8 * q + 2 * j]), __uint_as_float(v[8 * q + 2 * j + 1]));
        *reinterpret_cast<uint4*>(orow + n) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      } else {
        // DSWIGLU: n is the hidden unit f; g, u from the recomputed projections
        const __nv_bfloat16* gurow = a.gu + static_cast<int64_t>(tok) * a.ld_gu +
                                     static_cast<int64_t>(t.g) * a.gu_group_cols;
        const uint4 gq = *reinterpret_cast<const uint4*>(gurow + n);
        const uint4 uq = *reinterpret_cast<const uint4*>(gurow + a.F + n);
        const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
        const uint32_t uw[4] = {uq.x, uq.y, uq.z, uq.w};
        uint32_t dg[4], du[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float gv[2] = {bf16_lo(gw[j]), bf16_hi(gw[j])};
          float uv[2] = {bf16_lo(uw[j]), bf16_hi(uw[j])};
          float og[2], ou[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float dh = __uint_as_float(v[8 * q + 2 * j + h]);
            const float s = 1.0f / (1.0f + __expf(-gv[h]));
            og[h] = dh * uv[h] * (s * (1.0f + gv[h] * (1.0f - s)));
            ou[h] = dh * gv[h] * s;
          }
          dg[j] = pack_bf16x2(og[0], og[1]);
          du[j] = pack_bf16x2(ou[0], ou[1]);
        }
        *reinterpret_cast<uint4*>(orow + n) = make_uint4(dg[0], dg[1], dg[2], dg[3]);
        *reinterpret_cast<uint4*>(orow + a.F + n) = make_uint4(du[0], du[1], du[2], du[3]);
      }
    }
  }
}

// tmA: dgrad 2-D (K total, rows) with 64 x 128 boxes (K-major);
//      wgrad 2-D (columns, rows) with 64 x 64 boxes (MN-major, two per k-block).
// tmB: dgrad 3-D (N total, K, matrices) with 64 x 64 x 1 boxes (MN-major, four per k-block);
//      wgrad 2-D (columns, rows) with 64 x 64 boxes (four per k-block).
template <int MODE, int EPI>
__global__ void __launch_bounds__(kGThreads, 1)
    grad_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const GradArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kGStages * kGABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGStages * kGStageBytes + kGSlack);
  uint64_t* empty = full + kGStages;
  uint64_t* tfull = empty + kGStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* prefix = reinterpret_cast<int*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  pdl_wait();
  pdl_trigger();
  if (warp == 2) grad_prefix_warp<MODE>(args, prefix, lane);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = prefix[args.n_groups];
  const int nkb_g = (args.kdim + kGBK - 1) / kGBK;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        const GradTile t = grad_decode<MODE>(tile, prefix, args);
        const int nkb = grad_nkb<MODE>(args, t);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = sA + stage * kGABytes;
          uint8_t* b_dst = sB + stage * kGBBytes;
          mbar_arrive_expect_tx(&full[stage], kGStageBytes);
          if (MODE == GMODE_DGRAD) {
            const int kg = kb / nkb_g;
            const int kk = (kb - kg * nkb_g) * kGBK;
            tma_load_2d(a_dst, &tmA, &full[stage], kg * args.kdim + kk, t.row_base + t.m0);
            if (args.merged_b) {  // the four 64-column chunks in one box; chunks past N read zeros
              tma_load_4d(b_dst, &tmB, &full[stage], 0, kk, t.n0 / 64, t.g * args.k_groups + kg);
            } else {
#pragma unroll
              for (int c = 0; c < kGBN / 64; ++c)
                tma_load_3d(b_dst + c * kGChunk, &tmB, &full[stage], t.n0 + 64 * c, kk, t.g * args.k_groups + kg);
            }
          } else {
            const int r0 = t.row_base + kb * kGBK;
            if (args.merged_a) {
              tma_load_3d(a_dst, &tmA, &full[stage], 0, r0, (t.g * args.a_col_group + t.m0) / 64);
            } else {
#pragma unroll
              for (int c = 0; c < kGBM / 64; ++c)
                tma_load_2d(a_dst + c * kGChunk, &tmA, &full[stage], t.g * args.a_col_group + t.m0 + 64 * c, r0);
            }
            if (args.merged_b) {
              tma_load_3d(b_dst, &tmB, &full[stage], 0, r0, (t.g * args.b_col_group + t.n0) / 64);
            } else {
#pragma unroll
              for (int c = 0; c < kGBN / 64; ++c)
                tma_load_2d(b_dst + c * kGChunk, &tmB, &full[stage], t.g * args.b_col_group + t.n0 + 64 * c, r0);
            }
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kGStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {  // let every copy this thread started land before exit
        int never = 0;
        for (int s = 0; s < kGStages; ++s)
          if ((issued >> s) & 1u) mbar_wait(&full[s], (last_par >> s) & 1u, &never);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (whole warp:
    // the lanes zero the rows past a group's end in a wgrad tile's last k-block)
    constexpr uint32_t idesc = idesc_bf16_f32_major(kGBM, kGBN, MODE == GMODE_WGRAD, true);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int it = 0;
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++it) {
      const GradTile t = grad_decode<MODE>(tile, prefix, args);
      const int nkb = grad_nkb<MODE>(args, t);
      const int acc = it & 1;
      const uint32_t acc_par = static_cast<uint32_t>(it >> 1) & 1u;
      ok = __all_sync(0xffffffffu, mbar_wait(&tempty[acc], acc_par ^ 1u, abort_flag));
      if (!ok) break;
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kGBN);
      for (int kb = 0; kb < nkb; ++kb) {
        ok = __all_sync(0xffffffffu, mbar_wait(&full[stage], phase, abort_flag));
        if (!ok) break;
        uint8_t* a_st = sA + stage * kGABytes;
        if (MODE == GMODE_WGRAD) {
          const int valid = t.rows - kb * kGBK;  // token rows of this k-block inside the group
          if (valid < kGBK) {
            // rows [valid, 64) of every 64-column chunk of A (2) and B (4): one
            // 128-byte row per K index, so the swizzle keeps each row in place.
            // Both operands, so that stale values past the last group (even
            // non-finite ones) cannot reach the sum.
            uint8_t* b_st = sB + stage * kGBBytes;
            const int n16 = (kGBK - valid) * 8;  // 16-byte pieces per chunk
            for (int i = lane; i < 6 * n16; i += 32) {
              const int c = i / n16, w = i - c * n16;
              const int row = valid + w / 8;
              uint8_t* base = c < 2 ? a_st + c * kGChunk : b_st + (c - 2) * kGChunk;
              *reinterpret_cast<uint4*>(base + row * 128 + (w & 7) * 16) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
          }
        }
        if (lane == 0) {
          tc_fence_after_sync();
          const uint32_t sa = smem_addr(a_st);
          const uint32_t sb = smem_addr(sB + stage * kGBBytes);
#pragma unroll
          for (int k = 0; k < kGBK / 16; ++k) {
            // 16 K per MMA: K-major A advances 32 bytes; an MN-major operand 16 rows of 128 bytes
            const uint64_t adesc = MODE == GMODE_WGRAD ? smem_desc_mn128(sa + k * 2048, kGChunk, 1024)
                                                       : smem_desc_k128(sa) + 2 * k;
            const uint64_t bdesc = smem_desc_mn128(sb + k * 2048, kGChunk, 1024);
            umma_bf16(d_tmem, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == kGStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&tfull[acc]);
      __syncwarp();
    }
    if (lane == 0 && *abort_flag) {  // wait for every MMA issued before TMEM is freed
      umma_commit(drain);
      int never = 0;
      mbar_wait(drain, 0, &never);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
      const GradTile t = grad_decode<MODE>(tile, prefix, args);
      const int acc = it & 1;
      const uint32_t acc_par = static_cast<uint32_t>(it >> 1) & 1u;
      const bool ready = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_par, abort_flag));
      if (!ready) break;
      tc_fence_after_sync();
      const uint32_t t_lane =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kGBN);
      grad_epilogue<MODE, EPI>(args, t, r, t_lane, grad_nkb<MODE>(args, t) == 0);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) raise_status(args.status, kDevWaitTimeout);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int MODE, int EPI>
static int run_grad(const CUtensorMap& ta, const CUtensorMap& tb, const GradArgs& a, int64_t tile_bound,
                    cudaStream_t st) {
  constexpr int smem = grad_smem_bytes();
  static std::mutex mu;
  static uint64_t done = 0;  // the dynamic shared-memory opt-in is per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -3;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!((done >> dev) & 1u)) {
      if (cudaFuncSetAttribute(grad_gemm_kernel<MODE, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess)
        return -3;
      done |= uint64_t(1) << dev;
    }
  }
  if (tile_bound <= 0) return 0;
  int64_t grid = num_sms();
  if (grid > tile_bound) grid = tile_bound;
  return launch_k(grad_gemm_kernel<MODE, EPI>, dim3(static_cast<unsigned>(grid)), dim3(kGThreads), smem, st, ta, tb,
                  a) == cudaSuccess
             ? 0
             : -3;
}

static int64_t gcdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// MN-major operand maps.  A matrix stack [mats, rows (the K index), cols]
// read in 64-column chunks of 64 rows: chunked, one box holds `chunks`
// consecutive chunks, (64, rows, cols/64, mats) with the chunk stride 128
// bytes; else (cols, rows, mats) with 64 x 64 boxes.  Chunked needs cols a
// multiple of 64 (MOE_B200_MERGED_K=0 turns it off).
static bool mn_chunked_ok(int64_t cols) {
  const char* e = getenv("MOE_B200_MERGED_K");
  if (e && !strcmp(e, "0")) return false;
  return cols % 64 == 0;
}

static bool make_mn_map(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t mats, int chunks,
                        bool chunked, bool with_mats) {
  const int rank = (chunked ? 3 : 2) + (with_mats ? 1 : 0);
  if (chunked) {
    const uint64_t d[4] = {64, static_cast<uint64_t>(rows), static_cast<uint64_t>(cols / 64),
                           static_cast<uint64_t>(mats)};
    const uint64_t st[3] = {static_cast<uint64_t>(cols) * 2, 128, static_cast<uint64_t>(cols * rows) * 2};
    const uint32_t b[4] = {64, kGBK, static_cast<uint32_t>(chunks), 1};
    return make_map_strided(m, base, rank, d, st, b);
  }
  const uint64_t d[3] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows), static_cast<uint64_t>(mats)};
  const uint32_t b[3] = {64, kGBK, 1};
  return make_map(m, base, rank, d, b);
}

// Backward of the expert FFNs, given do (the gradient at the experts' outputs,
// per row: a routed row's token dy times its gate weight; for the shared
// experts dy itself).  mode 0 routed (groups = experts over seg_off), 1 shared
// (every row through all N_s experts).  x_rows, h: the forward's expert inputs
// and hidden activations; gu, dgu: scratch [n_rows, G*2F] (routed G = 1 column
// block); dx_rows [n_rows, d] out (routed: per expert row; shared: summed over
// the experts); dw13 [G, 2F, d], dw2 [G, d, F] FP32 out.
int launch_expert_ffn_backward(const Problem& p, int mode, const void* x_rows, int64_t n_rows,
                               const int32_t* seg_off, const void* w13, const void* w2, const void* dout,
                               const void* h, void* gu, void* dgu, void* dx_rows, float* dw13, float* dw2,
                               unsigned* status, cudaStream_t st, bool gu_ready) {
  if (n_rows <= 0) return 0;
  const bool routed = mode == 0;
  const int G = routed ? p.E : p.Ns;
  const int64_t gu_cols = routed ? 2 * static_cast<int64_t>(p.F) : 2 * static_cast<int64_t>(p.F) * p.Ns;
  const int64_t h_cols = routed ? p.F : static_cast<int64_t>(p.F) * p.Ns;
  const int64_t row_tiles = routed ? gcdiv(n_rows, kGBM) + G : static_cast<int64_t>(G) * gcdiv(n_rows, kGBM);

  // 1. g, u: kept by the forward, or recomputed as GU = x W13^T (its up projection without SwiGLU)
  if (!gu_ready && launch_up_projections(p, mode, x_rows, n_rows, seg_off, w13, gu, status, st)) return -3;

  // 2. dGU: dh = do W2 (B = W2 read MN-major), epilogue -> (dg | du)
  {
    CUtensorMap ta, tb;
    const uint64_t da[2] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(n_rows)};
    const uint32_t ba[2] = {kGBK, kGBM};
    const bool mb = mn_chunked_ok(p.F);
    if (!make_map(&ta, dout, 2, da, ba) || !make_mn_map(&tb, w2, p.F, p.d, G, kGBN / 64, mb, true)) return -3;
    GradArgs a{};
    a.merged_b = mb;
    a.n_groups = G;
    a.seg_off = routed ? seg_off : nullptr;
    a.n_rows = static_cast<int>(n_rows);
    a.n_dim = p.F;
    a.kdim = p.d;
    a.k_groups = 1;
    a.out = dgu;
    a.ldo = gu_cols;
    a.out_col_stride = routed ? 0 : 2 * p.F;
    a.gu = static_cast<const __nv_bfloat16*>(gu);
    a.ld_gu = gu_cols;
    a.gu_group_cols = routed ? 0 : 2 * p.F;
    a.F = p.F;
    a.status = status;
    if (run_grad<GMODE_DGRAD, GEPI_DSWIGLU>(ta, tb, a, row_tiles * gcdiv(p.F, kGBN), st)) return -3;
  }
  // 3. dX = dGU W13 (B = W13 read MN-major); shared: the N_s experts summed along K
  {
    CUtensorMap ta, tb;
    const uint64_t da[2] = {static_cast<uint64_t>(gu_cols), static_cast<uint64_t>(n_rows)};
    const uint32_t ba[2] = {kGBK, kGBM};
    const bool mb = mn_chunked_ok(p.d);
    if (!make_map(&ta, dgu, 2, da, ba) || !make_mn_map(&tb, w13, p.d, 2 * p.F, G, kGBN / 64, mb, true)) return -3;
    GradArgs a{};
    a.merged_b = mb;
    a.n_groups = routed ? G : 1;
    a.seg_off = routed ? seg_off : nullptr;
    a.n_rows = static_cast<int>(n_rows);
    a.n_dim = p.d;
    a.kdim = 2 * p.F;
    a.k_groups = routed ? 1 : p.Ns;
    a.out = dx_rows;
    a.ldo = p.d;
    a.out_col_stride = 0;
    a.status = status;
    const int64_t rt = routed ? row_tiles : gcdiv(n_rows, kGBM);
    if (run_grad<GMODE_DGRAD, GEPI_BF16>(ta, tb, a, rt * gcdiv(p.d, kGBN), st)) return -3;
  }
  // 4. dW13[g] = dGU_g^T x (reduction over the group's rows)
  {
    CUtensorMap ta, tb;
    const bool ma = mn_chunked_ok(gu_cols) && (2 * p.F) % 64 == 0, mb = mn_chunked_ok(p.d);
    if (!make_mn_map(&ta, dgu, gu_cols, n_rows, 1, kGBM / 64, ma, false) ||
        !make_mn_map(&tb, x_rows, p.d, n_rows, 1, kGBN / 64, mb, false))
      return -3;
    GradArgs a{};
    a.merged_a = ma;
    a.merged_b = mb;
    a.n_groups = G;
    a.seg_off = routed ? seg_off : nullptr;
    a.n_rows = static_cast<int>(n_rows);
    a.m_dim = 2 * p.F;
    a.n_dim = p.d;
    a.a_col_group = routed ? 0 : 2 * p.F;
    a.b_col_group = 0;
    a.out = dw13;
    a.ldo = p.d;
    a.out_group_stride = 2 * static_cast<int64_t>(p.F) * p.d;
    a.status = status;
    if (run_grad<GMODE_WGRAD, GEPI_F32>(ta, tb, a, G * gcdiv(2 * p.F, kGBM) * gcdiv(p.d, kGBN), st)) return -3;
  }
  // 5. dW2[g] = do_g^T h_g
  {
    CUtensorMap ta, tb;
    const bool ma = mn_chunked_ok(p.d), mb = mn_chunked_ok(h_cols) && p.F % 64 == 0;
    if (!make_mn_map(&ta, dout, p.d, n_rows, 1, kGBM / 64, ma, false) ||
        !make_mn_map(&tb, h, h_cols, n_rows, 1, kGBN / 64, mb, false))
      return -3;
    GradArgs a{};
    a.merged_a = ma;
    a.merged_b = mb;
    a.n_groups = G;
    a.seg_off = routed ? seg_off : nullptr;
    a.n_rows = static_cast<int>(n_rows);
    a.m_dim = p.d;
    a.n_dim = p.F;
    a.a_col_group = 0;
    a.b_col_group = routed ? 0 : p.F;
    a.out = dw2;
    a.ldo = p.F;
    a.out_group_stride = static_cast<int64_t>(p.d) * p.F;
    a.status = status;
    if (run_grad<GMODE_WGRAD, GEPI_F32>(ta, tb, a, G * gcdiv(p.d, kGBM) * gcdiv(p.F, kGBN), st)) return -3;
  }
  return 0;
}

// Router backward through the gate GEMM, dl [T, e_pad] BF16 (columns >= E zero):
//   dx_r = dl W_g  (B = W_g [E, d] read MN-major, K = e_pad)
int launch_router_dgrad(const Problem& p, const void* dl16, int e_pad, const void* w_gate, void* dx_r,
                        unsigned* status, cudaStream_t st) {
  CUtensorMap ta, tb;
  const uint64_t da[2] = {static_cast<uint64_t>(e_pad), static_cast<uint64_t>(p.T)};
  const uint32_t ba[2] = {kGBK, kGBM};
  const bool mb = mn_chunked_ok(p.d);
  if (!make_map(&ta, dl16, 2, da, ba) || !make_mn_map(&tb, w_gate, p.d, p.E, 1, kGBN / 64, mb, true)) return -3;
  GradArgs a{};
  a.merged_b = mb;
  a.n_groups = 1;
  a.n_rows = static_cast<int>(p.T);
  a.n_dim = p.d;
  a.kdim = e_pad;
  a.k_groups = 1;
  a.out = dx_r;
  a.ldo = p.d;
  a.status = status;
  return run_grad<GMODE_DGRAD, GEPI_BF16>(ta, tb, a, gcdiv(p.T, kGBM) * gcdiv(p.d, kGBN), st);
}

//   dW_g = dl^T x  (reduction over all T tokens), FP32 [E, d]
int launch_router_wgrad(const Problem& p, const void* dl16, int e_pad, const void* x, float* dwg, unsigned* status,
                        cudaStream_t st) {
  CUtensorMap ta, tb;
  const bool ma = mn_chunked_ok(e_pad), mb = mn_chunked_ok(p.d);
  if (!make_mn_map(&ta, dl16, e_pad, p.T, 1, kGBM / 64, ma, false) ||
      !make_mn_map(&tb, x, p.d, p.T, 1, kGBN / 64, mb, false))
    return -3;
  GradArgs a{};
  a.merged_a = ma;
  a.merged_b = mb;
  a.n_groups = 1;
  a.n_rows = static_cast<int>(p.T);
  a.m_dim = p.E;
  a.n_dim = p.d;
  a.out = dwg;
  a.ldo = p.d;
  a.out_group_stride = 0;
  a.status = status;
  return run_grad<GMODE_WGRAD, GEPI_F32>(ta, tb, a, gcdiv(p.E, kGBM) * gcdiv(p.d, kGBN), st);
}

}  // namespace moe
