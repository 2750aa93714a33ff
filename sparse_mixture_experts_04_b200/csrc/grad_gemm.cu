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
// Two shapes, one warp-specialised kernel (warp 0 TMA, warp 1 MMA, then 4 or 8
// epilogue warps; 128 x 256 tiles, 64-deep k-blocks, double-buffered TMEM):
//   dgrad  M = a group's token rows, N = output columns, K fixed:
//          A = activations (token rows, K-major), B = the group's weights read
//          MN-major (the weights are stored [out, in] for the forward, so the
//          backward contracts over their row index).  Epilogues:
//            DSWIGLU  dh tile -> dg, du with g, u read from the recomputed
//                     gate/up projections; stores dGU [rows, 2F] (dg | du)
//            BF16     dX rows
//   wgrad  M, N = the weight's shape, K = the group's token rows: A and B are
//          activations read MN-major (rows = tokens); the k-block that runs
//          past the group's last row reads a copy of the group's last rows
//          padded with zero rows (gathered before the GEMM), so rows of the
//          next group add nothing and no shared memory is rewritten between
//          the copies and the MMAs.  Stores the FP32 weight gradient (zeros for
//          a group without rows).
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
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
// warp 0 TMA, warp 1 MMA, then the epilogue warps: 8 (two per TMEM lane
// quarter, each taking half of the 256 accumulator columns) for the dSwiGLU
// epilogue, whose loads and math set its pace; 4 for the others (8 measured
// 16% slower on the FP32 weight gradients, 4% faster on the dSwiGLU dgrad)
template <int EPI>
constexpr int grad_epi_warps() { return EPI == GEPI_DSWIGLU ? 8 : 4; }
template <int EPI>
constexpr int grad_threads() { return 32 * (2 + grad_epi_warps<EPI>()); }
constexpr int kGEpiWarpsMax = 8;
constexpr int kGMaxGroups = 256;
constexpr int kGABytes = kGBM * kGBK * 2;  // 16 KB
constexpr int kGBBytes = kGBN * kGBK * 2;  // 32 KB: four 64-column MN chunks of 64 K rows
constexpr int kGStageBytes = kGABytes + kGBBytes;
constexpr int kGChunk = 64 * kGBK * 2;  // one MN chunk (64 elements x 64 K rows) = 8 KB
// Room after the ring: the epilogue warps' 32 x 33 float staging buffers
// (17 KB), and a margin so that the operand descriptors of the last stage stay
// inside the allocation whatever they address.
constexpr int kGSlack = 32 * 1024;
static_assert(kGEpiWarpsMax * 32 * 32 * 4 <= kGSlack, "epilogue staging buffers do not fit");

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
  // wgrad: a k-block that runs past its group's last row reads the group's
  // zero-padded copy of those rows instead (tmAt / tmBt, built by
  // launch_wgrad_tails): k-block rows of group g start at row g * tail_stride
  // there (0: every group shares one copy)
  int tail_stride;
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

// Tiles per group: dgrad ceil(rows/BM) x ceil(N/256); wgrad ceil(M/BM) x ceil(N/256).
template <int MODE, int BM>
__device__ __forceinline__ int grad_tiles_of(const GradArgs& a, int g) {
  const int nt = (a.n_dim + kGBN - 1) / kGBN;
  if (MODE == GMODE_WGRAD) return ((a.m_dim + BM - 1) / BM) * nt;
  int base;
  return ((grad_group_rows(a, g, &base) + BM - 1) / BM) * nt;
}

template <int MODE, int BM>
__device__ __forceinline__ void grad_prefix_warp(const GradArgs& a, int* prefix, int lane) {
  const int per = (a.n_groups + 31) / 32;
  int local = 0;
  for (int i = 0; i < per; ++i) {
    const int g = lane * per + i;
    if (g < a.n_groups) local += grad_tiles_of<MODE, BM>(a, g);
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
      run += grad_tiles_of<MODE, BM>(a, g);
    }
  }
  if (lane == 31) prefix[a.n_groups] = incl;
}

template <int MODE, int BM>
__device__ __forceinline__ GradTile grad_decode(int tile, const int* prefix, const GradArgs& a) {
  int lo = 0, hi = a.n_groups - 1;
  while (lo < hi) {  // largest g with prefix[g] <= tile (a group with tiles)
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  GradTile t;
  t.g = lo;
  t.rows = grad_group_rows(a, lo, &t.row_base);
  const int mt = MODE == GMODE_WGRAD ? (a.m_dim + BM - 1) / BM : (t.rows + BM - 1) / BM;
  const int local = tile - prefix[lo];
  const int n_idx = local / mt;
  const int m_idx = local - n_idx * mt;
  t.m0 = m_idx * BM;  // dgrad: row offset within the group; wgrad: output row
  t.n0 = n_idx * kGBN;
  return t;
}

// k-blocks of a tile (BK deep): dgrad a fixed count, wgrad the group's rows in BKs.
template <int MODE, int BK>
__device__ __forceinline__ int grad_nkb(const GradArgs& a, const GradTile& t) {
  if (MODE == GMODE_WGRAD) return (t.rows + BK - 1) / BK;
  return ((a.kdim + BK - 1) / BK) * a.k_groups;
}

// Epilogue of one accumulator: this thread's TMEM lane r (0..127) holds row
// m0 + r of the tile, 256 columns from t_lane; this warp takes columns
// [c_lo, c_hi).  Every lane calls it (the TMEM loads are warp-collective);
// `zero` (wgrad, no rows in the group) stores zeros without reading TMEM.
// xw: this warp's 32 x 32 float staging buffer in shared memory, element
// (row, col) at row * 32 + (col ^ row) (conflict-free both ways); FP32 weight
// gradients are written row-coalesced through it.
template <int MODE, int EPI>
__device__ __forceinline__ void grad_epilogue(const GradArgs& a, const GradTile& t, int r, uint32_t t_lane,
                                              bool zero, float* xw, int c_lo, int c_hi) {
  const int lane = r & 31;
  if (EPI == GEPI_F32) {
    // each warp owns 32 rows; a 32 x 32 block goes lane-per-row into xw, then
    // out as 4 rows x 128 bytes per store instruction
    float* obase = static_cast<float*>(a.out) + static_cast<int64_t>(t.g) * a.out_group_stride;
    const int m_warp = t.m0 + (r & ~31);
    const int cq = (lane & 7) * 4;
#pragma unroll 1
    for (int c = c_lo; c < c_hi; c += 32) {
      uint32_t v[32];
      if (!zero) {
        tmem_load_32x32(t_lane + static_cast<uint32_t>(c), v);
        tmem_load_wait();
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) xw[lane * 32 + (j ^ lane)] = zero ? 0.f : __uint_as_float(v[j]);
      __syncwarp();
      const int n = t.n0 + c + cq;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rr = i * 4 + (lane >> 3);
        const int m = m_warp + rr;
        if (m < a.m_dim && n < a.n_dim) {
          const float* row = xw + rr * 32;
          *reinterpret_cast<float4*>(obase + static_cast<int64_t>(m) * a.ldo + n) =
              make_float4(row[cq ^ rr], row[(cq + 1) ^ rr], row[(cq + 2) ^ rr], row[(cq + 3) ^ rr]);
        }
      }
      __syncwarp();
    }
    return;
  }
  // dgrad: row = token
  const int tok = t.row_base + t.m0 + r;
  const bool row_ok = t.m0 + r < t.rows;
  __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) + static_cast<int64_t>(row_ok ? tok : 0) * a.ldo +
                        static_cast<int64_t>(t.g) * a.out_col_stride;
  const __nv_bfloat16* gurow = nullptr;
  if (EPI == GEPI_DSWIGLU)
    gurow = a.gu + static_cast<int64_t>(row_ok ? tok : 0) * a.ld_gu + static_cast<int64_t>(t.g) * a.gu_group_cols;
#pragma unroll 1
  for (int c = c_lo; c < c_hi; c += 32) {
    uint32_t v[32];
    uint4 gq[4], uq[4];
    if (EPI == GEPI_DSWIGLU) {
      // g, u of this row's 32 hidden units: all eight loads in flight before
      // the accumulator is read
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int n = t.n0 + c + 8 * q;
        if (row_ok && n < a.n_dim) {
          gq[q] = *reinterpret_cast<const uint4*>(gurow + n);
          uq[q] = *reinterpret_cast<const uint4*>(gurow + a.F + n);
        } else {
          gq[q] = uq[q] = make_uint4(0, 0, 0, 0);
        }
      }
    }
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
        // DSWIGLU: n is the hidden unit f
        const uint32_t gw[4] = {gq[q].x, gq[q].y, gq[q].z, gq[q].w};
        const uint32_t uw[4] = {uq[q].x, uq[q].y, uq[q].z, uq[q].w};
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
__global__ void __launch_bounds__(grad_threads<EPI>(), 1)
    grad_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmAt, const __grid_constant__ CUtensorMap tmBt,
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
      mbar_init(&tempty[a], grad_epi_warps<EPI>());
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (MODE == GMODE_WGRAD) {
      prefetch_tensormap(&tmAt);
      prefetch_tensormap(&tmBt);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  pdl_wait();
  pdl_trigger();
  if (warp == 2) grad_prefix_warp<MODE, kGBM>(args, prefix, lane);
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
        const GradTile t = grad_decode<MODE, kGBM>(tile, prefix, args);
        const int nkb = grad_nkb<MODE, kGBK>(args, t);
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
            const bool tail = t.rows - kb * kGBK < kGBK;  // runs past the group: its zero-padded copy
            const int r0 = tail ? t.g * args.tail_stride : t.row_base + kb * kGBK;
            const CUtensorMap* ma = tail ? &tmAt : &tmA;
            const CUtensorMap* mb = tail ? &tmBt : &tmB;
            if (args.merged_a) {
              tma_load_3d(a_dst, ma, &full[stage], 0, r0, (t.g * args.a_col_group + t.m0) / 64);
            } else {
#pragma unroll
              for (int c = 0; c < kGBM / 64; ++c)
                tma_load_2d(a_dst + c * kGChunk, ma, &full[stage], t.g * args.a_col_group + t.m0 + 64 * c, r0);
            }
            if (args.merged_b) {
              tma_load_3d(b_dst, mb, &full[stage], 0, r0, (t.g * args.b_col_group + t.n0) / 64);
            } else {
#pragma unroll
              for (int c = 0; c < kGBN / 64; ++c)
                tma_load_2d(b_dst + c * kGChunk, mb, &full[stage], t.g * args.b_col_group + t.n0 + 64 * c, r0);
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
    // ---------------------------------------------------------------- MMA issuer (lane 0; the
    // whole warp takes the waits)
    constexpr uint32_t idesc = idesc_bf16_f32_major(kGBM, kGBN, MODE == GMODE_WGRAD, true);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int it = 0;
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++it) {
      const GradTile t = grad_decode<MODE, kGBM>(tile, prefix, args);
      const int nkb = grad_nkb<MODE, kGBK>(args, t);
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
      const GradTile t = grad_decode<MODE, kGBM>(tile, prefix, args);
      const int acc = it & 1;
      const uint32_t acc_par = static_cast<uint32_t>(it >> 1) & 1u;
      const bool ready = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_par, abort_flag));
      if (!ready) break;
      tc_fence_after_sync();
      const uint32_t t_lane =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kGBN);
      constexpr int span = kGBN * 4 / grad_epi_warps<EPI>();  // columns per epilogue warp
      const int part = (warp - 2) >> 2;
      grad_epilogue<MODE, EPI>(args, t, r, t_lane, grad_nkb<MODE, kGBK>(args, t) == 0,
                               reinterpret_cast<float*>(smem + kGStages * kGStageBytes) + (warp - 2) * 32 * 32,
                               part * span, (part + 1) * span);
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

// ============================================================================
// CTA-pair version (cluster of 2, tcgen05.mma.cta_group::2): 256 x 256 tiles,
// CTA r holds rows [128 r, 128 r + 128) of A and columns [128 r, 128 r + 128)
// of B, 128-deep k-blocks in 3 stages of 64 KB per CTA, every operand in one
// chunk-merged box per stage.  Per CTA a stage moves 32 KB of A and 32 KB of
// B for 2 x 128 x 256 x 128 FLOPs, half the bytes per FLOP of the single-CTA
// 128 x 256 tile.  The leader (rank 0) issues the MMAs; both CTAs stage
// operands and run the epilogue on their own 128 accumulator rows.
//   dgrad  A K-major: map (64, rows, K_total/64), box (64, 128, 2);
//          B MN-major: map (64, K, N/64, matrices), box (64, 128, 2, 1)
//   wgrad  A, B MN-major: maps (64, rows, cols/64), box (64, 128, 2)
// A wgrad k-block past the group's last row reads the group's zero-padded
// copy of its last rows (tmAt / tmBt), as in the single-CTA kernel.
// ============================================================================
constexpr int kPGBM = 256;
constexpr int kPGBK = 128;
constexpr int kPGStages = 3;
constexpr int kPGHalf = 128 * kPGBK * 2;   // one CTA's A (or B) per stage: 32 KB
constexpr int kPGChunk = 128 * 64 * 2;     // a 64-wide chunk of 128 rows (K-major A) / 128 K rows (MN-major): 16 KB

constexpr int pgrad_smem_bytes() { return kPGStages * 2 * kPGHalf + kGSlack + 256 + 4 * (kGMaxGroups + 1) + 1024; }
static_assert(pgrad_smem_bytes() <= 232448, "exceeds the per-block shared-memory limit");

template <int MODE, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(grad_threads<EPI>(), 1)
    grad_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmAt, const __grid_constant__ CUtensorMap tmBt,
                          const GradArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kPGStages * kPGHalf;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPGStages * 2 * kPGHalf + kGSlack);
  uint64_t* empty = full + kPGStages;
  uint64_t* tfull = empty + kPGStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* prefix = reinterpret_cast<int*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPGStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * grad_epi_warps<EPI>());
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (MODE == GMODE_WGRAD) {
      prefetch_tensormap(&tmAt);
      prefetch_tensormap(&tmBt);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  pdl_wait();
  pdl_trigger();
  if (warp == 2) grad_prefix_warp<MODE, kPGBM>(args, prefix, lane);
  tc_fence_before_sync();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = prefix[args.n_groups];
  const int nkb_g = (args.kdim + kPGBK - 1) / kPGBK;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader = mapa_shared(smem_addr(&full[0]), 0);
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        const GradTile t = grad_decode<MODE, kPGBM>(tile, prefix, args);
        const int nkb = grad_nkb<MODE, kPGBK>(args, t);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 4 * kPGHalf);  // both CTAs' A and B
          const uint32_t bar = full_leader + static_cast<uint32_t>(stage * 8);
          uint8_t* a_dst = sA + stage * kPGHalf;
          uint8_t* b_dst = sB + stage * kPGHalf;
          const int half = 128 * static_cast<int>(rank);
          if (MODE == GMODE_DGRAD) {
            const int kg = kb / nkb_g;
            const int kk0 = (kb - kg * nkb_g) * kPGBK;  // past K: zeros (B's K rows are out of range)
            tma_load_3d_pair(a_dst, &tmA, bar, 0, t.row_base + t.m0 + half, (kg * args.kdim + kk0) / 64);
            tma_load_4d_pair(b_dst, &tmB, bar, 0, kk0, (t.n0 + half) / 64, t.g * args.k_groups + kg);
          } else {
            const bool tail = t.rows - kb * kPGBK < kPGBK;  // runs past the group: its zero-padded copy
            const int r0 = tail ? t.g * args.tail_stride : t.row_base + kb * kPGBK;
            tma_load_3d_pair(a_dst, tail ? &tmAt : &tmA, bar, 0, r0, (t.g * args.a_col_group + t.m0 + half) / 64);
            tma_load_3d_pair(b_dst, tail ? &tmBt : &tmB, bar, 0, r0, (t.g * args.b_col_group + t.n0 + half) / 64);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kPGStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        int never = 0;
        if (rank == 0) {  // the leader's full barriers count both CTAs' bytes
          for (int s = 0; s < kPGStages; ++s)
            if ((issued >> s) & 1u) mbar_wait(&full[s], (last_par >> s) & 1u, &never);
        } else {  // the peer cannot observe its copies: give them a bounded time to land
          const unsigned long long t0 = global_ns();
          while (global_ns() - t0 < 1000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32_major(kPGBM, kGBN, MODE == GMODE_WGRAD, true);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs, ++it) {
        const GradTile t = grad_decode<MODE, kPGBM>(tile, prefix, args);
        const int nkb = grad_nkb<MODE, kPGBK>(args, t);
        const int acc = it & 1;
        const uint32_t acc_par = static_cast<uint32_t>(it >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], acc_par ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kGBN);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sa = smem_addr(sA + stage * kPGHalf);
          const uint32_t sb = smem_addr(sB + stage * kPGHalf);
#pragma unroll
          for (int k = 0; k < kPGBK / 16; ++k) {
            // K-major A: two 64-deep chunks, 32 bytes per 16 K within one;
            // MN-major operands: 16 K rows of 128 bytes per 16 K, chunks kPGChunk apart
            const uint64_t adesc = MODE == GMODE_WGRAD ? smem_desc_mn128(sa + k * 2048, kPGChunk, 1024)
                                                       : smem_desc_k128(sa + (k >> 2) * kPGChunk) + 2 * (k & 3);
            const uint64_t bdesc = smem_desc_mn128(sb + k * 2048, kPGChunk, 1024);
            umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit_pair_multicast(&empty[stage], 0x3);
          if (++stage == kPGStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair_multicast(&tfull[acc], 0x3);
      }
      if (*abort_flag) {  // wait for every MMA issued before TMEM is freed
        umma_commit_pair_multicast(drain, 0x1);
        int never = 0;
        mbar_wait(drain, 0, &never);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t tempty_leader = mapa_shared(smem_addr(&tempty[0]), 0);
    int it = 0;
    for (int tile = pair; tile < total_tiles; tile += n_pairs, ++it) {
      GradTile t = grad_decode<MODE, kPGBM>(tile, prefix, args);
      const bool zero = grad_nkb<MODE, kPGBK>(args, t) == 0;
      const int acc = it & 1;
      const uint32_t acc_par = static_cast<uint32_t>(it >> 1) & 1u;
      const bool ready = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_par, abort_flag));
      if (!ready) break;
      tc_fence_after_sync();
      const uint32_t t_lane =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kGBN);
      t.m0 += 128 * static_cast<int>(rank);  // this CTA's accumulator rows
      constexpr int span = kGBN * 4 / grad_epi_warps<EPI>();  // columns per epilogue warp
      const int part = (warp - 2) >> 2;
      grad_epilogue<MODE, EPI>(args, t, r, t_lane, zero,
                               reinterpret_cast<float*>(smem + kPGStages * 2 * kPGHalf) + (warp - 2) * 32 * 32,
                               part * span, (part + 1) * span);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader + static_cast<uint32_t>(acc * 8));
    }
  }

  __syncwarp();
  tc_fence_before_sync();
  cluster_sync();  // no CTA leaves while its peer may still touch its shared memory or TMEM
  if (threadIdx.x == 0 && *abort_flag) raise_status(args.status, kDevWaitTimeout);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

template <int MODE, int EPI>
static int run_grad(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tat, const CUtensorMap& tbt,
                    const GradArgs& a, int64_t tile_bound,
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
  return launch_k(grad_gemm_kernel<MODE, EPI>, dim3(static_cast<unsigned>(grid)), dim3(grad_threads<EPI>()), smem, st,
                  ta, tb,
                  tat, tbt, a) == cudaSuccess
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
                        bool chunked, bool with_mats, uint32_t k_rows = kGBK) {
  const int rank = (chunked ? 3 : 2) + (with_mats ? 1 : 0);
  if (chunked) {
    const uint64_t d[4] = {64, static_cast<uint64_t>(rows), static_cast<uint64_t>(cols / 64),
                           static_cast<uint64_t>(mats)};
    const uint64_t st[3] = {static_cast<uint64_t>(cols) * 2, 128, static_cast<uint64_t>(cols * rows) * 2};
    const uint32_t b[4] = {64, k_rows, static_cast<uint32_t>(chunks), 1};
    return make_map_strided(m, base, rank, d, st, b);
  }
  const uint64_t d[3] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows), static_cast<uint64_t>(mats)};
  const uint32_t b[3] = {64, kGBK, 1};
  return make_map(m, base, rank, d, b);
}

template <int MODE, int EPI>
static int run_grad_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tat, const CUtensorMap& tbt,
                         const GradArgs& a, int64_t tile_bound,
                         cudaStream_t st) {
  constexpr int smem = pgrad_smem_bytes();
  static std::mutex mu;
  static int max_pairs[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -3;
  int pairs;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (max_pairs[dev] == 0) {
      if (cudaFuncSetAttribute(grad_gemm_pair_kernel<MODE, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               smem) != cudaSuccess)
        return -3;
      // a persistent grid must fit at once: ask how many 2-CTA clusters can be co-resident
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
      cfg.blockDim = dim3(grad_threads<EPI>(), 1, 1);
      cfg.dynamicSmemBytes = smem;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, grad_gemm_pair_kernel<MODE, EPI>, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = num_sms() / 2;
      }
      max_pairs[dev] = n;
    }
    pairs = max_pairs[dev];
  }
  if (tile_bound <= 0) return 0;
  if (pairs > tile_bound) pairs = static_cast<int>(tile_bound);
  return launch_k(grad_gemm_pair_kernel<MODE, EPI>, dim3(static_cast<unsigned>(2 * pairs)), dim3(grad_threads<EPI>()),
                  smem,
                  st, ta, tb, tat, tbt, a) == cudaSuccess
             ? 0
             : -3;
}

// The pair kernel needs every operand chunk-merged (column counts multiples
// of 64); dgrad also wants groups of at least 256 rows (else the 256-row tiles
// are mostly padding).  Measured on the Mixtral shape (8 groups of ~1024 rows,
// ncu per launch, single CTA -> pair): dW13 2.01 -> 1.74 ms, dW2 0.90 -> 0.80
// ms, dX rows 1.52 -> 1.40 ms; whole backward with the dSwiGLU dgrad on pairs
// too 2% faster (equal on the fine-grained and skewed workloads).
// MOE_B200_GRAD_PAIR=0 keeps every backward GEMM on single CTAs.
static bool grad_pair_ok() {
  const char* e = getenv("MOE_B200_GRAD_PAIR");
  if (e && !strcmp(e, "0")) return false;
  const char* m = getenv("MOE_B200_MERGED_K");
  return !(m && !strcmp(m, "0"));
}

// K-major activation map of the pair dgrad: (64, rows, cols/64), box (64, 128, 2).
static bool make_kmajor_pair_map(CUtensorMap* m, const void* base, int64_t cols, int64_t rows) {
  const uint64_t d[3] = {64, static_cast<uint64_t>(rows), static_cast<uint64_t>(cols / 64)};
  const uint64_t st[2] = {static_cast<uint64_t>(cols) * 2, 128};
  const uint32_t b[3] = {64, 128, 2};
  return make_map_strided(m, base, 3, d, st, b);
}

// The last k-block of each wgrad group, zero-padded: tail t (group t, or the
// one tail of groups that share their rows when seg_off is null) gets rows
// dst[t*bk + j] = src[start_t + j] for j < valid_t and zeros after, where the
// group's rows are cut into k-blocks of bk from its first row and start_t is
// the first row of its last k-block.  cols8: row length in 16-byte units.
__global__ void __launch_bounds__(256) wgrad_tail_kernel(const uint4* __restrict__ src, int64_t cols8,
                                                         const int32_t* __restrict__ seg_off, int n_rows, int bk,
                                                         uint4* __restrict__ dst) {
  // launched with programmatic dependent launch like every kernel here: wait
  // for the predecessor (which produced src, and may still read dst) first
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.y;
  int base = 0, rows = n_rows;
  if (seg_off) {
    base = min(max(seg_off[t], 0), n_rows);
    rows = min(max(seg_off[t + 1], base), n_rows) - base;
  }
  const int done = rows > 0 ? ((rows - 1) / bk) * bk : 0;  // rows before the last k-block
  const int start = base + done, valid = rows - done;
  const int64_t total = static_cast<int64_t>(bk) * cols8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(i / cols8);
    const int64_t q = i - static_cast<int64_t>(j) * cols8;
    const uint4 v = j < valid ? src[static_cast<int64_t>(start + j) * cols8 + q] : make_uint4(0, 0, 0, 0);
    dst[(static_cast<int64_t>(t) * bk + j) * cols8 + q] = v;
  }
}

struct WgradOperand {
  const void* base;  // [n_rows, cols] BF16, token rows
  int64_t cols;
  int col_group;     // group g's block starts at column g * col_group
};

// dW[g] (m_dim x n_dim, FP32, out + g * out_group_stride, row stride ldo) =
// A_g^T B_g over the group's token rows.  tail_a / tail_b: scratch for the
// groups' zero-padded last k-blocks (wgrad_tail_bytes each).
static int run_wgrad(const WgradOperand& A, const WgradOperand& B, int G, const int32_t* seg_off, int64_t n_rows,
                     int m_dim, int n_dim, float* out, int64_t ldo, int64_t out_group_stride, void* tail_a,
                     void* tail_b, unsigned* status, cudaStream_t st) {
  const bool ma = mn_chunked_ok(A.cols) && A.col_group % 64 == 0;
  const bool mb = mn_chunked_ok(B.cols) && B.col_group % 64 == 0;
  const bool pair = grad_pair_ok() && ma && mb && m_dim >= kPGBM && n_dim >= kGBN;
  const int bk = pair ? kPGBK : kGBK;
  const int n_tails = seg_off ? G : 1;
  const WgradOperand* ops[2] = {&A, &B};
  void* tails[2] = {tail_a, tail_b};
  for (int i = 0; i < 2; ++i) {
    const int64_t cols8 = ops[i]->cols / 8;
    int64_t blocks = gcdiv(bk * cols8, 256);
    if (blocks > 1024) blocks = 1024;
    if (launch_k(wgrad_tail_kernel, dim3(static_cast<unsigned>(blocks), static_cast<unsigned>(n_tails)), dim3(256), 0,
                 st, static_cast<const uint4*>(ops[i]->base), cols8, seg_off, static_cast<int>(n_rows), bk,
                 static_cast<uint4*>(tails[i])) != cudaSuccess)
      return -3;
  }
  CUtensorMap ta, tb, tat, tbt;
  const int ca = pair ? 2 : kGBM / 64, cb = pair ? 2 : kGBN / 64;
  if (!make_mn_map(&ta, A.base, A.cols, n_rows, 1, ca, ma, false, bk) ||
      !make_mn_map(&tb, B.base, B.cols, n_rows, 1, cb, mb, false, bk) ||
      !make_mn_map(&tat, tail_a, A.cols, static_cast<int64_t>(n_tails) * bk, 1, ca, ma, false, bk) ||
      !make_mn_map(&tbt, tail_b, B.cols, static_cast<int64_t>(n_tails) * bk, 1, cb, mb, false, bk))
    return -3;
  GradArgs a{};
  a.merged_a = ma;
  a.merged_b = mb;
  a.n_groups = G;
  a.seg_off = seg_off;
  a.n_rows = static_cast<int>(n_rows);
  a.m_dim = m_dim;
  a.n_dim = n_dim;
  a.a_col_group = A.col_group;
  a.b_col_group = B.col_group;
  a.out = out;
  a.ldo = ldo;
  a.out_group_stride = out_group_stride;
  a.status = status;
  a.tail_stride = seg_off ? bk : 0;
  return pair ? run_grad_pair<GMODE_WGRAD, GEPI_F32>(ta, tb, tat, tbt, a, G * gcdiv(m_dim, kPGBM) * gcdiv(n_dim, kGBN),
                                                     st)
              : run_grad<GMODE_WGRAD, GEPI_F32>(ta, tb, tat, tbt, a, G * gcdiv(m_dim, kGBM) * gcdiv(n_dim, kGBN), st);
}

// Bytes of one wgrad tail scratch buffer (A or B) for a problem: the widest
// operand row times 128 rows per tail, E tails (routed) or one.
size_t wgrad_tail_bytes(const Problem& p, int e_pad) {
  const int64_t routed = static_cast<int64_t>(p.E) * (2 * static_cast<int64_t>(p.F) > p.d ? 2 * p.F : p.d);
  int64_t one = p.d;
  if (p.Ns > 0) one = std::max<int64_t>(one, 2 * static_cast<int64_t>(p.F) * p.Ns);
  one = std::max<int64_t>(one, e_pad);
  return static_cast<size_t>(std::max(routed, one)) * kPGBK * 2;
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
                               void* tail_a, void* tail_b, unsigned* status, cudaStream_t st, bool gu_ready) {
  if (n_rows <= 0) return 0;
  const bool routed = mode == 0;
  const int G = routed ? p.E : p.Ns;
  const int64_t gu_cols = routed ? 2 * static_cast<int64_t>(p.F) : 2 * static_cast<int64_t>(p.F) * p.Ns;
  const int64_t h_cols = routed ? p.F : static_cast<int64_t>(p.F) * p.Ns;
  const int64_t row_tiles = routed ? gcdiv(n_rows, kGBM) + G : static_cast<int64_t>(G) * gcdiv(n_rows, kGBM);

  // 1. g, u: kept by the forward, or recomputed as GU = x W13^T (its up projection without SwiGLU)
  if (!gu_ready && launch_up_projections(p, mode, x_rows, n_rows, seg_off, w13, gu, status, st)) return -3;

  // expected rows per group (as in the forward): routed T*K/E capped by the capacity, shared all rows
  int64_t expected = routed ? (p.T * p.K) / p.E : n_rows;
  if (routed && p.cap >= 0 && p.cap < expected) expected = p.cap;
  const bool pair_rows = grad_pair_ok() && expected >= 256;
  const int64_t row_tiles2 = routed ? gcdiv(n_rows, kPGBM) + G : static_cast<int64_t>(G) * gcdiv(n_rows, kPGBM);

  // 2. dGU: dh = do W2 (B = W2 read MN-major), epilogue -> (dg | du)
  {
    CUtensorMap ta, tb;
    const bool pair = pair_rows && p.d % 64 == 0 && p.F % 64 == 0;
    const uint64_t da[2] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(n_rows)};
    const uint32_t ba[2] = {kGBK, kGBM};
    const bool mb = mn_chunked_ok(p.F);
    if (pair) {
      if (!make_kmajor_pair_map(&ta, dout, p.d, n_rows) || !make_mn_map(&tb, w2, p.F, p.d, G, 2, true, true, kPGBK))
        return -3;
    } else if (!make_map(&ta, dout, 2, da, ba) || !make_mn_map(&tb, w2, p.F, p.d, G, kGBN / 64, mb, true)) {
      return -3;
    }
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
    if (pair ? run_grad_pair<GMODE_DGRAD, GEPI_DSWIGLU>(ta, tb, ta, tb, a, row_tiles2 * gcdiv(p.F, kGBN), st)
             : run_grad<GMODE_DGRAD, GEPI_DSWIGLU>(ta, tb, ta, tb, a, row_tiles * gcdiv(p.F, kGBN), st))
      return -3;
  }
  // 3. dX = dGU W13 (B = W13 read MN-major); shared: the N_s experts summed along K
  {
    CUtensorMap ta, tb;
    const uint64_t da[2] = {static_cast<uint64_t>(gu_cols), static_cast<uint64_t>(n_rows)};
    const uint32_t ba[2] = {kGBK, kGBM};
    const bool mb = mn_chunked_ok(p.d);
    const bool pair = pair_rows && p.d % 64 == 0 && (2 * p.F) % 64 == 0;
    if (pair) {
      if (!make_kmajor_pair_map(&ta, dgu, gu_cols, n_rows) ||
          !make_mn_map(&tb, w13, p.d, 2 * p.F, G, 2, true, true, kPGBK))
        return -3;
    } else if (!make_map(&ta, dgu, 2, da, ba) || !make_mn_map(&tb, w13, p.d, 2 * p.F, G, kGBN / 64, mb, true)) {
      return -3;
    }
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
    const int64_t rt2 = routed ? row_tiles2 : gcdiv(n_rows, kPGBM);
    if (pair ? run_grad_pair<GMODE_DGRAD, GEPI_BF16>(ta, tb, ta, tb, a, rt2 * gcdiv(p.d, kGBN), st)
             : run_grad<GMODE_DGRAD, GEPI_BF16>(ta, tb, ta, tb, a, rt * gcdiv(p.d, kGBN), st))
      return -3;
  }
  // 4. dW13[g] = dGU_g^T x (reduction over the group's rows)
  if (run_wgrad({dgu, gu_cols, routed ? 0 : 2 * p.F}, {x_rows, p.d, 0}, G, routed ? seg_off : nullptr, n_rows,
                2 * p.F, p.d, dw13, p.d, 2 * static_cast<int64_t>(p.F) * p.d, tail_a, tail_b, status, st))
    return -3;
  // 5. dW2[g] = do_g^T h_g
  if (run_wgrad({dout, p.d, 0}, {h, h_cols, routed ? 0 : p.F}, G, routed ? seg_off : nullptr, n_rows, p.d, p.F, dw2,
                p.F, static_cast<int64_t>(p.d) * p.F, tail_a, tail_b, status, st))
    return -3;
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
  return run_grad<GMODE_DGRAD, GEPI_BF16>(ta, tb, ta, tb, a, gcdiv(p.T, kGBM) * gcdiv(p.d, kGBN), st);
}

//   dW_g = dl^T x  (reduction over all T tokens), FP32 [E, d]
int launch_router_wgrad(const Problem& p, const void* dl16, int e_pad, const void* x, float* dwg, void* tail_a,
                        void* tail_b, unsigned* status, cudaStream_t st) {
  return run_wgrad({dl16, e_pad, 0}, {x, p.d, 0}, 1, nullptr, p.T, p.E, p.d, dwg, p.d, 0, tail_a, tail_b, status, st);
}

}  // namespace moe
