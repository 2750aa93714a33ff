// Expert FFNs: grouped GEMMs on the 5th-generation tensor cores (tcgen05.mma,
// accumulators in TMEM, operands staged by TMA), with SwiGLU fused into the
// epilogue of the up/gate projection.
//
//   Zen-Max: Maximum Capability via Mixture-of-Experts Architecture, §2.2
//   Fine-Grained Expert Architecture, eq. Expert_i:
//       Expert_i(x) = (SiLU(x W_gate,i) (.) x W_up,i) W_down,i
//   Shared experts (always active) are added to the routed outputs
//   (same section; Scaling with experts, "A shared expert").
//
// One kernel template, three epilogues:
//   EPI_SWIGLU : H[r, n] = silu(A W_gate^T)[r, n] * (A W_up^T)[r, n]   (BF16 out)
//                the B tile stacks 128 gate rows over 128 up rows, so one
//                M=128 x N=256 MMA chain yields both halves for the same n.
//   EPI_BF16   : Y = A W_down^T                                          (BF16 out)
//   EPI_F32    : logits = A W_g^T + offset                               (FP32 out)
//
// Work decomposition: a "group" is a block of A rows that shares one B
// matrix (an expert).  Routed groups are the expert segments of the
// expert-grouped rows [seg_off[g], seg_off[g+1]) (read on the device, so no
// host sync); shared groups all cover rows [0, n_rows).  Tiles are 128 rows x
// (128 or 256) columns, enumerated group-major, then column tile, then row
// tile, so CTAs running at the same time share weight tiles through L2.
// Persistent CTAs (one per SM) walk the tile list with a stride of the grid.
// A launch may carry a second problem (its own tensor maps, arguments and
// tile prefix; the layer puts the shared experts there): the first problem's
// tiles are spread evenly through the combined tile list (decode_mixed_tile).
//
// Warp roles (192 threads): warp 0 issues TMA loads into a STAGES-deep ring of
// shared-memory stages; warp 1 allocates TMEM and issues the MMAs from one
// thread; warps 2-5 drain the TMEM accumulator (double-buffered, so the
// epilogue of tile i overlaps the main loop of tile i+1) and store.
// Every wait is bounded (see mbar_wait); on a timeout the kernel records
// MOE_DEV_WAIT_TIMEOUT, drains its own copies and MMAs, frees TMEM and exits.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {

enum { EPI_SWIGLU = 0, EPI_BF16 = 1, EPI_F32 = 2 };

constexpr int kBM = 128;
constexpr int kBK = 64;  // 64 BF16 = 128 bytes: one 128-byte swizzle row
constexpr int kGemmThreads = 192;
constexpr int kMaxGroups = 256;

struct GemmArgs {
  int n_groups;
  const int32_t* seg_off;  // [n_groups + 1] row offsets, or nullptr: every group covers [0, n_rows)
  int n_rows;
  int N;               // valid output columns of one group
  int K;               // valid reduction length of one B matrix
  int k_groups;        // B matrices summed along the reduction (A row holds k_groups * K)
  void* out;
  int64_t ldo;         // output row stride, elements
  int out_col_stride;  // output column offset per group
  const float* col_add;  // EPI_F32: per-column offset, or nullptr
  unsigned* status;
  // split-K (EPI_F32 only): group g reduces k in [g*k_split, (g+1)*k_split)
  // and writes its partial sums at out + g*out_group_stride (0: no split)
  int k_split;
  int64_t out_group_stride;
  // which rows of each group this launch covers: 0 all, 1 the head (rows
  // rounded down to a multiple of 256), 2 the tail (the rest)
  int row_mode;
  // pair kernel: a group's last row tile with at most swap_max rows (0: never)
  // is computed operand-swapped (see grouped_gemm_pair_kernel)
  int swap_max;
  // EPI_SWIGLU: when not null, the gate and up projections are also stored
  // (BF16): row r, group g: g at gu + r*ld_gu + g*gu_col_stride + col, u at
  // N columns further
  void* gu;
  int64_t ld_gu;
  int gu_col_stride;
  // pair kernel: 1 when the tensor maps address both 64-deep chunks of a
  // stage with one box (K a multiple of 64): A maps (64, rows, K/64), B maps
  // (64, rows, groups, K/64); 0: one 2-D / 3-D box per chunk
  int merged_k;
  // pair kernel, merged maps: swap tiles of at most 64 token rows take
  // 192-deep stages (tokens and weights of three chunks in one stage slot)
  int deep_swap;
  // stage clock of the launch (moe_layer_forward_clocked), or nullptr
  unsigned long long* clk;
  // single-CTA kernel: abort-path test hook (test_stall), 0 normally
  unsigned long long stall_ns;
  // > 0: group g is computed with the weights of expert g % weight_mod (row
  // segments that repeat the experts, e.g. one run of experts per source rank
  // in the expert-parallel receive buffer); 0: expert g
  int weight_mod;
};

// Reduction range of a tile of group g: first k, number of 64-wide k-blocks.
__device__ __forceinline__ void tile_k_range(const GemmArgs& a, int g, int* k0, int* nkb) {
  if (a.k_split > 0) {
    *k0 = g * a.k_split;
    const int len = min(a.K - *k0, a.k_split);
    *nkb = (len + 63) / 64;
  } else {
    *k0 = 0;
    *nkb = ((a.K + 63) / 64) * a.k_groups;
  }
}

template <int EPI, int BN>
struct TileCfg {
  static constexpr int kOutCols = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                   : (2 * BN <= 256) ? 256 : 512;
};

// FP32 epilogue staging: one 32 x 32 float block per epilogue warp
constexpr int kF32StageBytes = 4 * 32 * 32 * 4;

template <int EPI, int BN, int STAGES>
constexpr int gemm_smem_bytes() {
  return STAGES * TileCfg<EPI, BN>::kStageBytes + 256 /*barriers + flags*/ + 8 * (kMaxGroups + 1) +
         (EPI == EPI_F32 ? kF32StageBytes + 16 : 0) + 1024 /*alignment slack*/;
}

struct TileInfo {
  int g, row0, row_end, n0;
  int w;        // expert whose weights the tile uses (g, or g % weight_mod)
  bool swap;    // operand-swapped remainder tile (pair kernel only)
  bool second;  // tile of the pair kernel's second problem
};

// Rows [base, base + return) of group g (the part row_mode selects), clamped
// to the allocated rows [0, n_rows) whatever seg_off holds, so no tile reads
// or writes outside them.
__device__ __forceinline__ int group_rows(const GemmArgs& a, int g, int* base) {
  int b = 0, rows = a.n_rows;
  if (a.seg_off) {
    b = min(max(a.seg_off[g], 0), a.n_rows);
    rows = min(max(a.seg_off[g + 1], b), a.n_rows) - b;
  }
  const int head = rows & ~255;
  if (a.row_mode == 1) rows = head;
  if (a.row_mode == 2) {
    b += head;
    rows -= head;
  }
  *base = b;
  return rows;
}

template <int BM>
__device__ __forceinline__ TileInfo decode_tile(int tile, const int* prefix, const GemmArgs& a, int out_cols) {
  int lo = 0, hi = a.n_groups - 1;
  while (lo < hi) {  // largest g with prefix[g] <= tile (that group is never empty)
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  TileInfo ti;
  ti.g = lo;
  ti.w = a.weight_mod > 0 ? lo % a.weight_mod : lo;
  int base;
  const int rows = group_rows(a, lo, &base);
  const int mt = (rows + BM - 1) / BM;
  const int local = tile - prefix[lo];
  const int n_idx = local / mt;
  const int m_idx = local - n_idx * mt;
  ti.row0 = base + m_idx * BM;
  ti.row_end = base + rows;
  ti.n0 = n_idx * out_cols;
  ti.swap = m_idx == mt - 1 && rows - m_idx * BM <= a.swap_max;
  ti.second = false;
  return ti;
}

// Tile prefix over groups (one warp): lane l owns groups [l*per, (l+1)*per).
// prefix[g] = first tile of group g; prefix[n_groups] = total tiles.
template <int BM>
__device__ __forceinline__ void tile_prefix_warp(const GemmArgs& args, int n_tiles_n, int* prefix, int lane) {
  const int per = (args.n_groups + 31) / 32;
  int local = 0;
  for (int i = 0; i < per; ++i) {
    const int g = lane * per + i;
    if (g < args.n_groups) {
      int base;
      local += ((group_rows(args, g, &base) + BM - 1) / BM) * n_tiles_n;
    }
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
    if (g < args.n_groups) {
      prefix[g] = run;
      int base;
      run += ((group_rows(args, g, &base) + BM - 1) / BM) * n_tiles_n;
    }
  }
  if (lane == 31) prefix[args.n_groups] = incl;
}

// Tile `tile` of a launch over two problems with t1 and total - t1 tiles: the
// first problem's tiles are spread evenly through [0, total) (tile i is the
// first problem's number floor(i t1 / total) when that count steps at i), so
// every CTA's strided walk mixes both kinds in proportion.
template <int BM>
__device__ __forceinline__ TileInfo decode_mixed_tile(int tile, int t1, int total, const int* prefix,
                                                      const int* prefix2, const GemmArgs& a1, const GemmArgs& a2,
                                                      int out_cols) {
  const int lo = static_cast<int>(static_cast<long long>(tile) * t1 / total);
  const int hi = static_cast<int>(static_cast<long long>(tile + 1) * t1 / total);
  if (hi > lo) return decode_tile<BM>(lo, prefix, a1, out_cols);
  TileInfo ti = decode_tile<BM>(tile - lo, prefix2, a2, out_cols);
  ti.second = true;
  return ti;
}

// Drain one accumulator (this warp's 32 TMEM lanes, BN columns starting at
// t_row) and store the thread's row.  Every lane must call it (the TMEM loads
// are warp-collective); row_ok masks only the stores.
template <int EPI, int BN>
__device__ __forceinline__ void epilogue_rows(const GemmArgs& args, int g, int row, bool row_ok, int n0,
                                              uint32_t t_row) {
  if (EPI == EPI_SWIGLU) {
    __nv_bfloat16* out_row = static_cast<__nv_bfloat16*>(args.out) + static_cast<int64_t>(row) * args.ldo +
                             static_cast<int64_t>(g) * args.out_col_stride;
#pragma unroll 1
    for (int c = 0; c < BN / 2; c += 32) {
      uint32_t gr[32], ur[32];
      tmem_load_32x32(t_row + c, gr);
      tmem_load_32x32(t_row + BN / 2 + c, ur);
      tmem_load_wait();
      if (row_ok) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = n0 + c + q * 8;
          if (col < args.N) {
            uint32_t pk[4], gp[4], up[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float g0 = __uint_as_float(gr[q * 8 + 2 * j]), g1 = __uint_as_float(gr[q * 8 + 2 * j + 1]);
              const float u0 = __uint_as_float(ur[q * 8 + 2 * j]), u1 = __uint_as_float(ur[q * 8 + 2 * j + 1]);
              const float h0 = __fdividef(g0, 1.0f + __expf(-g0)) * u0;
              const float h1 = __fdividef(g1, 1.0f + __expf(-g1)) * u1;
              pk[j] = pack_bf16x2(h0, h1);
              gp[j] = pack_bf16x2(g0, g1);
              up[j] = pack_bf16x2(u0, u1);
            }
            *reinterpret_cast<uint4*>(out_row + col) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            if (args.gu) {
              __nv_bfloat16* gu_row = static_cast<__nv_bfloat16*>(args.gu) + static_cast<int64_t>(row) * args.ld_gu +
                                      static_cast<int64_t>(g) * args.gu_col_stride;
              *reinterpret_cast<uint4*>(gu_row + col) = make_uint4(gp[0], gp[1], gp[2], gp[3]);
              *reinterpret_cast<uint4*>(gu_row + args.N + col) = make_uint4(up[0], up[1], up[2], up[3]);
            }
          }
        }
      }
    }
  } else if (EPI == EPI_BF16) {
    __nv_bfloat16* out_row = static_cast<__nv_bfloat16*>(args.out) + static_cast<int64_t>(row) * args.ldo +
                             static_cast<int64_t>(g) * args.out_col_stride;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t vr[32];
      tmem_load_32x32(t_row + c, vr);
      tmem_load_wait();
      if (row_ok) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = n0 + c + q * 8;
          if (col < args.N) {
            uint32_t pk[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
              pk[j] = pack_bf16x2(__uint_as_float(vr[q * 8 + 2 * j]), __uint_as_float(vr[q * 8 + 2 * j + 1]));
            *reinterpret_cast<uint4*>(out_row + col) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
    }
  } else {
    float* out_row = static_cast<float*>(args.out) + static_cast<int64_t>(g) * args.out_group_stride +
                     static_cast<int64_t>(row) * args.ldo;
    const float* add = (g == 0) ? args.col_add : nullptr;  // a split-K offset goes into slice 0 only
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t vr[32];
      tmem_load_32x32(t_row + c, vr);
      tmem_load_wait();
      if (row_ok) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int col = c + j;
          if (col < args.N) out_row[col] = __uint_as_float(vr[j]) + (add ? add[col] : 0.f);
        }
      }
    }
  }
}

// FP32 epilogue through shared memory: each 32-column block of this warp's 32
// accumulator rows goes lane-per-row into xw (XOR-swizzled, no bank
// conflicts) and out lane-per-column, so every store instruction writes 32
// consecutive floats of one row instead of one float of 32 rows.
template <int BN>
__device__ __forceinline__ void epilogue_f32_staged(const GemmArgs& args, int g, int row_base, int row_end,
                                                    uint32_t t_row, int lane, float* xw) {
  float* obase = static_cast<float*>(args.out) + static_cast<int64_t>(g) * args.out_group_stride;
  const float* add = (g == 0) ? args.col_add : nullptr;  // a split-K offset goes into slice 0 only
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    uint32_t v[32];
    tmem_load_32x32(t_row + c, v);
    tmem_load_wait();
#pragma unroll
    for (int j = 0; j < 32; ++j) xw[lane * 32 + (j ^ lane)] = __uint_as_float(v[j]);
    __syncwarp();
    const int col = c + lane;
    const bool col_ok = col < args.N;
    const float ad = (add && col_ok) ? add[col] : 0.f;
#pragma unroll 4
    for (int rr = 0; rr < 32; ++rr) {
      const int row = row_base + rr;
      if (col_ok && row < row_end) obase[static_cast<int64_t>(row) * args.ldo + col] = xw[rr * 32 + (lane ^ rr)] + ad;
    }
    __syncwarp();
  }
}

template <int EPI, int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ GemmArgs args, const __grid_constant__ CUtensorMap tmA_2,
                           const __grid_constant__ CUtensorMap tmB_2, const __grid_constant__ GemmArgs args2) {
  using C = TileCfg<EPI, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * C::kBBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* prefix = reinterpret_cast<int*>(tmem_slot + 4);
  int* prefix2 = prefix + kMaxGroups + 1;
  float* xw_all = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(prefix2 + kMaxGroups + 1) + 15) & ~uintptr_t(15));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tiles_n = (args.N + C::kOutCols - 1) / C::kOutCols;
  const int n_tiles_n2 = (args2.N + C::kOutCols - 1) / C::kOutCols;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
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
    if (args2.n_groups > 0) {
      prefetch_tensormap(&tmA_2);
      prefetch_tensormap(&tmB_2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();  // everything above is local set-up; from here on the predecessor's outputs are read
  pdl_trigger();
  stage_clock_start(args.clk);
  if (warp == 2) tile_prefix_warp<kBM>(args, n_tiles_n, prefix, lane);
  if (warp == 3) {
    if (args2.n_groups > 0)
      tile_prefix_warp<kBM>(args2, n_tiles_n2, prefix2, lane);
    else if (lane == 0)
      prefix2[0] = 0;
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int tiles1 = prefix[args.n_groups];
  const int total_tiles = tiles1 + prefix2[max(args2.n_groups, 0)];

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        const TileInfo ti = decode_mixed_tile<kBM>(tile, tiles1, total_tiles, prefix, prefix2, args, args2,
                                                   C::kOutCols);
        const GemmArgs& A = ti.second ? args2 : args;
        const CUtensorMap* mA = ti.second ? &tmA_2 : &tmA;
        const CUtensorMap* mB = ti.second ? &tmB_2 : &tmB;
        const int nkb_g = (A.K + kBK - 1) / kBK;
        int k0, nkb;
        tile_k_range(A, ti.g, &k0, &nkb);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const int kg = kb / nkb_g;
          const int kk = k0 + (kb - kg * nkb_g) * kBK;
          uint8_t* a_dst = sA + stage * C::kABytes;
          uint8_t* b_dst = sB + stage * C::kBBytes;
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          tma_load_2d(a_dst, mA, &full[stage], kg * A.K + kk, ti.row0);
          if (EPI == EPI_SWIGLU) {
            tma_load_3d(b_dst, mB, &full[stage], kk, ti.n0, 2 * ti.w);
            tma_load_3d(b_dst + C::kBBytes / 2, mB, &full[stage], kk, ti.n0, 2 * ti.w + 1);
          } else if (EPI == EPI_BF16) {
            tma_load_3d(b_dst, mB, &full[stage], kk, ti.n0, ti.w * A.k_groups + kg);
          } else {
            tma_load_3d(b_dst, mB, &full[stage], kk, 0, 0);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {  // let every copy this thread started land before exit
        int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if ((issued >> s) & 1u) mbar_wait(&full[s], (last_par >> s) & 1u, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = test_stall(drain, abort_flag, args.stall_ns);
      int it = 0;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_par = static_cast<uint32_t>(it >> 1) & 1u;
        const TileInfo ti = decode_mixed_tile<kBM>(tile, tiles1, total_tiles, prefix, prefix2, args, args2,
                                                   C::kOutCols);
        int k0, nkb;
        tile_k_range(ti.second ? args2 : args, ti.g, &k0, &nkb);
        if (!mbar_wait(&tempty[acc], acc_par ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint64_t adesc = smem_desc_k128(smem_addr(sA + stage * C::kABytes));
          const uint64_t bdesc = smem_desc_k128(smem_addr(sB + stage * C::kBBytes));
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)  // advance 16 elements = 32 bytes = 2 descriptor units
            umma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
      }
      if (*abort_flag) {  // wait for every MMA this thread issued before TMEM is freed
        umma_commit(drain);
        int never = 0;
        mbar_wait(drain, 0, &never);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter+32) are this warp's
    const int r = quarter * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
      const TileInfo ti = decode_mixed_tile<kBM>(tile, tiles1, total_tiles, prefix, prefix2, args, args2,
                                                 C::kOutCols);
      const int acc = it & 1;
      const uint32_t acc_par = static_cast<uint32_t>(it >> 1) & 1u;
      // every lane waits; the result is made warp-uniform (and the warp
      // reconverged) before the .sync.aligned TMEM loads below
      const bool ready = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_par, abort_flag));
      if (!ready) break;
      tc_fence_after_sync();
      const int row = ti.row0 + r;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * BN);
      if (EPI == EPI_F32)
        epilogue_f32_staged<BN>(ti.second ? args2 : args, ti.g, ti.row0 + quarter * 32, ti.row_end, t_row, lane,
                                xw_all + quarter * 32 * 32);
      else
        epilogue_rows<EPI, BN>(ti.second ? args2 : args, ti.g, row, row < ti.row_end, ti.n0, t_row);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  __syncthreads();
  stage_clock_end(args.clk);
  if (threadIdx.x == 0 && *abort_flag) raise_status(args.status, kDevWaitTimeout);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ============================================================================
// Pair kernel: the same grouped GEMM on CTA pairs (clusters of 2) with M=256
// tiles.  Each CTA stages its own 128 A rows and HALF of the B tile (for
// SwiGLU: CTA 0 the 128 gate rows, CTA 1 the 128 up rows; otherwise B rows
// n0..n0+127 and n0+128..n0+255), so per FLOP each SM pulls 2/3 of the bytes
// a 128x256 one-CTA tile needs.  The leader (rank 0) issues the MMAs for both
// CTAs; every accumulator row lands in the TMEM of the CTA that owns it.
//   full[s]   (leader)  one arrive (leader, with both CTAs' bytes) + TMA bytes
//   empty[s]  (each)    one arrive from the leader's multicast commit
//   tfull[a]  (each)    one arrive from the leader's multicast commit
//   tempty[a] (leader)  8 arrives: 4 epilogue warps in each CTA
// Tiles are 256 rows; a group with r rows spans ceil(r/256) row tiles.  Stage
// s occupies [s * 64 KB, (s + 1) * 64 KB): the token / A rows first, then the
// weights (32 KB each; a deep swap stage: tokens, then 48 KB of weights).
// ============================================================================
constexpr int kPairBM = 256;
constexpr int kPairBN = 256;  // MMA N: both halves of B
// 128-deep stages (two 64-deep chunks, one TMA box per chunk and operand), 3
// of them: half the barrier round trips of 64-deep stages for the same bytes
// in flight; measured 6% faster on the up/gate GEMM than 6 stages of 64.
constexpr int kPairKC = 2;
constexpr int kPairStages = 3;
constexpr int kPairChunk = 128 * kBK * 2;  // one 128-row, 64-deep chunk: 16 KB
constexpr int kPairABytes = kPairKC * kPairChunk;
constexpr int kPairBBytes = kPairKC * kPairChunk;  // this CTA's half of B
constexpr int kPairStageBytes = kPairABytes + kPairBBytes;
// A deep swap stage (swap tiles of at most 64 token rows, merged maps): three
// 64-deep chunks in one 64 KB stage slot, the tokens (3 x at most 32 rows per
// CTA, 12 KB) at its start and the weights (3 x 16 KB) in its last 48 KB.
// Copy-bound swap tiles then keep 1.7x the bytes in flight per SM.
constexpr int kDeepKC = 3;
constexpr int kDeepWOffset = kPairStageBytes - kDeepKC * kPairChunk;
static_assert(kDeepKC * 32 * kBK * 2 <= kDeepWOffset, "deep swap tokens overlap the weights");

// 64-deep chunks per stage of a tile whose token box is a_box rows
__device__ __forceinline__ int pair_tile_kc(const GemmArgs& a, const TileInfo& ti, int a_box) {
  return (a.deep_swap && a.merged_k && ti.swap && a_box <= 32) ? kDeepKC : kPairKC;
}

// Swap-tile epilogues transpose through shared memory, 32 tokens at a time:
// xbuf[token][TMEM lane] (row stride 132 floats keeps 16-byte alignment).
constexpr int kSwapXStride = 132;
constexpr int kSwapXBytes = 32 * kSwapXStride * 4;
// A swap tile loads its tokens with the smallest box (16, 32, 64 or 128
// rows) that holds its N/2 tokens per CTA.
__device__ __forceinline__ int swap_box_rows(int half_n) {
  return half_n <= 16 ? 16 : half_n <= 32 ? 32 : half_n <= 64 ? 64 : 128;
}

constexpr int pair_smem_bytes() {
  return kPairStages * kPairStageBytes + 256 + 8 * (kMaxGroups + 1) + kSwapXBytes + 1024;
}

__device__ __forceinline__ TileInfo decode_pair_tile(int tile, int t1, int total, const int* prefix,
                                                     const int* prefix2, const GemmArgs& a1, const GemmArgs& a2,
                                                     int out_cols) {
  return decode_mixed_tile<kPairBM>(tile, t1, total, prefix, prefix2, a1, a2, out_cols);
}

// k-blocks (kc chunks of 64 deep) of one tile of a problem
__device__ __forceinline__ int pair_nkb(const GemmArgs& a, int kc) {
  return ((a.K + kBK * kc - 1) / (kBK * kc)) * a.k_groups;
}

// MMA N of a swap tile covering `rows` (1..256) token rows: a multiple of 16.
__device__ __forceinline__ int swap_n(int rows) { return (rows + 15) & ~15; }

// Epilogue of a swap tile (all four epilogue warps, uniform control flow):
// TMEM lane = weight row of this CTA, column = token of the tile.  Each
// 32-token chunk goes through xbuf so that every thread then stores 8
// consecutive outputs of one token (16 bytes).
//   SwiGLU: lanes 0..63 hold gate features n0 + 64*rank + (0..63), lanes
//   64..127 the same up features: h = silu(g) * u.
//   BF16: lane = output column n0 + 128*rank + lane.
template <int EPI>
__device__ __forceinline__ void epilogue_swap(const GemmArgs& args, const TileInfo& ti, uint32_t rank, int quarter,
                                              int lane, int et, uint32_t t_lane, float* xbuf) {
  const int rows = ti.row_end - ti.row0;
  const int n = swap_n(rows);
  const int my_lane = quarter * 32 + lane;
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out) + static_cast<int64_t>(ti.row0) * args.ldo +
                       static_cast<int64_t>(ti.g) * args.out_col_stride;
#pragma unroll 1
  for (int c = 0; c < n; c += 32) {
    uint32_t v[32];
    tmem_load_32x32(t_lane + c, v);
    tmem_load_wait();
#pragma unroll
    for (int j = 0; j < 32; ++j) xbuf[j * kSwapXStride + my_lane] = __uint_as_float(v[j]);
    named_bar_sync(1, 128);
    if (EPI == EPI_SWIGLU) {
      // 64 features = 8 groups of 8: 16 tokens per pass
      const int fg = et & 7;
      const int f = ti.n0 + 64 * static_cast<int>(rank) + 8 * fg;
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        const int j = pass * 16 + (et >> 3);
        if (c + j < rows && f < args.N) {
          const float4* gp = reinterpret_cast<const float4*>(xbuf + j * kSwapXStride + 8 * fg);
          const float4* up = reinterpret_cast<const float4*>(xbuf + j * kSwapXStride + 64 + 8 * fg);
          const float4 g0 = gp[0], g1 = gp[1], u0 = up[0], u1 = up[1];
          const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
          const float u[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
          uint32_t pk[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float h0 = __fdividef(g[2 * q], 1.0f + __expf(-g[2 * q])) * u[2 * q];
            const float h1 = __fdividef(g[2 * q + 1], 1.0f + __expf(-g[2 * q + 1])) * u[2 * q + 1];
            pk[q] = pack_bf16x2(h0, h1);
          }
          *reinterpret_cast<uint4*>(out + static_cast<int64_t>(c + j) * args.ldo + f) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
          if (args.gu) {
            __nv_bfloat16* gu_row = static_cast<__nv_bfloat16*>(args.gu) +
                                    static_cast<int64_t>(ti.row0 + c + j) * args.ld_gu +
                                    static_cast<int64_t>(ti.g) * args.gu_col_stride;
            *reinterpret_cast<uint4*>(gu_row + f) =
                make_uint4(pack_bf16x2(g[0], g[1]), pack_bf16x2(g[2], g[3]), pack_bf16x2(g[4], g[5]),
                           pack_bf16x2(g[6], g[7]));
            *reinterpret_cast<uint4*>(gu_row + args.N + f) =
                make_uint4(pack_bf16x2(u[0], u[1]), pack_bf16x2(u[2], u[3]), pack_bf16x2(u[4], u[5]),
                           pack_bf16x2(u[6], u[7]));
          }
        }
      }
    } else {
      // 128 columns = 16 groups of 8: 8 tokens per pass
      const int fg = et & 15;
      const int col = ti.n0 + 128 * static_cast<int>(rank) + 8 * fg;
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) {
        const int j = pass * 8 + (et >> 4);
        if (c + j < rows && col < args.N) {
          const float4* vp = reinterpret_cast<const float4*>(xbuf + j * kSwapXStride + 8 * fg);
          const float4 a = vp[0], b = vp[1];
          *reinterpret_cast<uint4*>(out + static_cast<int64_t>(c + j) * args.ldo + col) =
              make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
        }
      }
    }
    named_bar_sync(1, 128);
  }
}

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmA64, const __grid_constant__ CUtensorMap tmB64,
                             const __grid_constant__ CUtensorMap tmA32, const __grid_constant__ CUtensorMap tmA16,
                             const __grid_constant__ GemmArgs args,
                             const __grid_constant__ CUtensorMap tmA_2, const __grid_constant__ CUtensorMap tmB_2,
                             const __grid_constant__ CUtensorMap tmA64_2, const __grid_constant__ CUtensorMap tmB64_2,
                             const __grid_constant__ CUtensorMap tmA32_2, const __grid_constant__ CUtensorMap tmA16_2,
                             const __grid_constant__ GemmArgs args2,
                             const __grid_constant__ CUtensorMap tmA32d, const __grid_constant__ CUtensorMap tmA16d,
                             const __grid_constant__ CUtensorMap tmB64d, const __grid_constant__ CUtensorMap tmA32d_2,
                             const __grid_constant__ CUtensorMap tmA16d_2, const __grid_constant__ CUtensorMap tmB64d_2) {
  constexpr int kOutCols = (EPI == EPI_SWIGLU) ? kPairBN / 2 : kPairBN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // stage s: smem + s * kPairStageBytes (tokens / A rows first, then weights)
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPairStages * kPairStageBytes);
  uint64_t* empty = full + kPairStages;
  uint64_t* tfull = empty + kPairStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* prefix = reinterpret_cast<int*>(tmem_slot + 4);
  int* prefix2 = prefix + kMaxGroups + 1;
  float* xbuf = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(prefix2 + kMaxGroups + 1) + 15) & ~uintptr_t(15));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int n_tiles_n = (args.N + kOutCols - 1) / kOutCols;
  const int n_tiles_n2 = (args2.N + kOutCols - 1) / kOutCols;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmA64);
    prefetch_tensormap(&tmA32);
    prefetch_tensormap(&tmA16);
    prefetch_tensormap(&tmB64);
    if (args2.n_groups > 0) {
      prefetch_tensormap(&tmA_2);
      prefetch_tensormap(&tmB_2);
      prefetch_tensormap(&tmA64_2);
      prefetch_tensormap(&tmA32_2);
      prefetch_tensormap(&tmA16_2);
      prefetch_tensormap(&tmB64_2);
    }
    if (args.deep_swap) {
      prefetch_tensormap(&tmA32d);
      prefetch_tensormap(&tmA16d);
      prefetch_tensormap(&tmB64d);
      if (args2.n_groups > 0) {
        prefetch_tensormap(&tmA32d_2);
        prefetch_tensormap(&tmA16d_2);
        prefetch_tensormap(&tmB64d_2);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  pdl_wait();  // everything above is local set-up; from here on the predecessor's outputs are read
  pdl_trigger();
  stage_clock_start(args.clk);
  if (warp == 2) tile_prefix_warp<kPairBM>(args, n_tiles_n, prefix, lane);
  if (warp == 3) {
    if (args2.n_groups > 0)
      tile_prefix_warp<kPairBM>(args2, n_tiles_n2, prefix2, lane);
    else if (lane == 0)
      prefix2[0] = 0;
  }
  tc_fence_before_sync();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int tiles1 = prefix[args.n_groups];
  const int total_tiles = tiles1 + prefix2[max(args2.n_groups, 0)];
  // no split-K on the pair path

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader = mapa_shared(smem_addr(&full[0]), 0);
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        const TileInfo ti = decode_pair_tile(tile, tiles1, total_tiles, prefix, prefix2, args, args2, kOutCols);
        const GemmArgs& A = ti.second ? args2 : args;
        const CUtensorMap* mA = ti.second ? &tmA_2 : &tmA;
        const CUtensorMap* mB = ti.second ? &tmB_2 : &tmB;
        const CUtensorMap* mB64 = ti.second ? &tmB64_2 : &tmB64;
        // a swap tile's N token rows are split N/2 per CTA; the box (16, 32,
        // 64 or 128 rows) may load more, the MMA reads the first N/2
        const int half_n = ti.swap ? swap_n(ti.row_end - ti.row0) / 2 : 128;
        const int a_box = ti.swap ? swap_box_rows(half_n) : 128;
        const int kc = pair_tile_kc(A, ti, a_box);
        const bool deep = kc == kDeepKC;
        const int nkb_g = (A.K + kBK * kc - 1) / (kBK * kc);
        const int nkb = nkb_g * A.k_groups;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const int kg = kb / nkb_g;
          const int kk0 = (kb - kg * nkb_g) * kBK * kc;
          const uint32_t bar = full_leader + static_cast<uint32_t>(stage * 8);
          const CUtensorMap* a_map = a_box == 16   ? (deep ? (ti.second ? &tmA16d_2 : &tmA16d) : (ti.second ? &tmA16_2 : &tmA16))
                                     : a_box == 32 ? (deep ? (ti.second ? &tmA32d_2 : &tmA32d) : (ti.second ? &tmA32_2 : &tmA32))
                                     : a_box == 64 ? (ti.second ? &tmA64_2 : &tmA64)
                                                   : mA;
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * kc * (kPairChunk + a_box * kBK * 2));
          const int a_row = ti.row0 + static_cast<int>(rank) * half_n;
          uint8_t* a_dst = smem + stage * kPairStageBytes;
          uint8_t* b_dst = a_dst + (deep ? kDeepWOffset : kPairABytes);
          // Swap tiles are bound by the copies, not the MMAs: with merged maps
          // (args.merged_k) each of their operands comes in one box spanning
          // both 64-deep chunks (the tokens' chunk c at c * a_box rows, the
          // weights' at c * kPairChunk; chunks past K read zeros).  Full tiles
          // keep one box per chunk, which measured slightly faster for them.
          const bool merge = A.merged_k && ti.swap;
          if (merge && a_box <= 64) {
            tma_load_3d_pair(a_dst, a_map, bar, 0, a_row, (kg * A.K + kk0) / kBK);
          } else {
#pragma unroll
            for (int c = 0; c < kPairKC; ++c)  // past K: the box reads zeros
              tma_load_2d_pair(a_dst + c * a_box * kBK * 2, a_box == 128 ? mA : a_map, bar, kg * A.K + kk0 + c * kBK,
                               a_row);
          }
          if (merge) {
            const CUtensorMap* wmap = deep ? (ti.second ? &tmB64d_2 : &tmB64d) : mB64;
            if (EPI == EPI_SWIGLU)  // weights are the M operand: this CTA's 64 gate rows, then the same 64 up rows
              tma_load_4d_pair(b_dst, wmap, bar, 0, ti.n0 + 64 * static_cast<int>(rank), 2 * ti.w, kk0 / kBK);
            else
              tma_load_4d_pair(b_dst, wmap, bar, 0, ti.n0 + 128 * static_cast<int>(rank), ti.w * A.k_groups + kg,
                               kk0 / kBK);
          } else {
#pragma unroll
            for (int c = 0; c < kPairKC; ++c) {
              const int kk = kk0 + c * kBK;
              uint8_t* bc = b_dst + c * kPairChunk;
              if (EPI == EPI_SWIGLU && ti.swap) {
                const int f = ti.n0 + 64 * static_cast<int>(rank);
                tma_load_3d_pair(bc, mB64, bar, kk, f, 2 * ti.w);
                tma_load_3d_pair(bc + kPairChunk / 2, mB64, bar, kk, f, 2 * ti.w + 1);
              } else if (EPI == EPI_SWIGLU) {
                tma_load_3d_pair(bc, mB, bar, kk, ti.n0, 2 * ti.w + static_cast<int>(rank));
              } else {
                tma_load_3d_pair(bc, mB, bar, kk, ti.n0 + 128 * static_cast<int>(rank), ti.w * A.k_groups + kg);
              }
            }
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        int never = 0;
        if (rank == 0) {  // the leader's full barriers count both CTAs' bytes
          for (int s = 0; s < kPairStages; ++s)
            if ((issued >> s) & 1u) mbar_wait(&full[s], (last_par >> s) & 1u, &never);
        } else {  // the peer cannot observe its copies: give them a bounded time to land
          const unsigned long long t0 = global_ns();
          while (global_ns() - t0 < 1000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs, ++it) {
        const TileInfo ti = decode_pair_tile(tile, tiles1, total_tiles, prefix, prefix2, args, args2, kOutCols);
        const int a_box = ti.swap ? swap_box_rows(swap_n(ti.row_end - ti.row0) / 2) : 128;
        const int kc = pair_tile_kc(ti.second ? args2 : args, ti, a_box);
        const int nkb = pair_nkb(ti.second ? args2 : args, kc);
        const int w_off = kc == kDeepKC ? kDeepWOffset : kPairABytes;
        // normal tile: A = token rows (M = 256), B = weight rows (N = 256);
        // swap tile: A = weight rows (M = 256), B = the tile's N token rows
        const uint32_t idesc = idesc_bf16_f32(kPairBM, ti.swap ? swap_n(ti.row_end - ti.row0) : kPairBN);
        // the token operand's chunks sit a_box rows apart (see the producer)
        const int a_chunk = a_box * kBK * 2;
        const int acc = it & 1;
        const uint32_t acc_par = static_cast<uint32_t>(it >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], acc_par ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kPairBN);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          uint8_t* st_base = smem + stage * kPairStageBytes;
#pragma unroll
          for (int c = 0; c < kDeepKC; ++c) {
            if (c >= kc) break;
            const uint64_t tdesc = smem_desc_k128(smem_addr(st_base + c * a_chunk));
            const uint64_t wdesc = smem_desc_k128(smem_addr(st_base + w_off + c * kPairChunk));
            const uint64_t adesc = ti.swap ? wdesc : tdesc;
            const uint64_t bdesc = ti.swap ? tdesc : wdesc;
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
              umma_bf16_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | c | k) != 0 ? 1u : 0u);
          }
          umma_commit_pair_multicast(&empty[stage], 0x3);
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair_multicast(&tfull[acc], 0x3);
      }
      if (*abort_flag) {
        umma_commit_pair_multicast(drain, 0x1);
        int never = 0;
        mbar_wait(drain, 0, &never);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t tempty_leader = mapa_shared(smem_addr(&tempty[0]), 0);
    int it = 0;
    for (int tile = pair; tile < total_tiles; tile += n_pairs, ++it) {
      const TileInfo ti = decode_pair_tile(tile, tiles1, total_tiles, prefix, prefix2, args, args2, kOutCols);
      const GemmArgs& A = ti.second ? args2 : args;
      const int acc = it & 1;
      const uint32_t acc_par = static_cast<uint32_t>(it >> 1) & 1u;
      // all four epilogue warps take the same decision (a swap tile's
      // epilogue synchronises them), even when a wait gives up
      const bool ready = named_bar_and(2, 128, mbar_wait(&tfull[acc], acc_par, abort_flag));
      if (!ready) break;
      tc_fence_after_sync();
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kPairBN);
      if (ti.swap) {
        epilogue_swap<EPI>(A, ti, rank, quarter, lane, (warp - 2) * 32 + lane, t_row, xbuf);
      } else {
        const int row = ti.row0 + 128 * static_cast<int>(rank) + r;
        epilogue_rows<EPI, kPairBN>(A, ti.g, row, row < ti.row_end, ti.n0, t_row);
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader + static_cast<uint32_t>(acc * 8));
    }
  }

  __syncwarp();
  tc_fence_before_sync();
  cluster_sync();  // no CTA leaves while its peer may still touch its shared memory or TMEM
  stage_clock_end(args.clk);
  if (threadIdx.x == 0 && *abort_flag) raise_status(args.status, kDevWaitTimeout);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// ============================================================================
// Host side: tensor maps and launches.
// ============================================================================
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// BF16 tensor map: dims[0] innermost (contiguous), 128-byte swizzle, zero fill
// out of bounds.  Box inner extent is always 64 elements (128 bytes).
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[3], gstr[2];
  cuuint32_t bdim[3], estr[3] = {1, 1, 1};
  uint64_t stride = 2;
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    if (i > 0) gstr[i - 1] = stride;
    stride *= dims[i];
  }
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), gdim, gstr, bdim, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// BF16 tensor map with explicit byte strides for dims 1..rank-1 (dim 0
// contiguous), 128-byte swizzle, zero fill out of bounds.  Used for the
// chunk-merged views: (64, rows, K/64) with the chunk stride 128 bytes.
bool make_map_strided(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
                      const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rank < 2 || rank > 5) return false;
  cuuint64_t gdim[5], gstr[4];
  cuuint32_t bdim[5], estr[5] = {1, 1, 1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    if (i > 0) gstr[i - 1] = strides[i - 1];
  }
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), gdim, gstr, bdim, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Token maps of the pair kernel: a 2-D (cols, rows) map with 128-row boxes,
// and swap-tile maps with 64-, 32- and 16-row boxes: 2-D as well, or with
// merged chunks one box spanning both 64-deep chunks of a stage,
// (64, rows, cols/64) with the chunk stride 128 bytes.
static bool make_token_maps(CUtensorMap* t128, CUtensorMap* t64, CUtensorMap* t32, CUtensorMap* t16,
                            CUtensorMap* t32d, CUtensorMap* t16d, const void* base, int64_t cols, int64_t rows,
                            bool merged) {
  const uint64_t d2[2] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows)};
  const uint32_t b128[2] = {kBK, 128};
  if (!make_map(t128, base, 2, d2, b128)) return false;
  CUtensorMap* maps[3] = {t64, t32, t16};
  const uint32_t heights[3] = {64, 32, 16};
  for (int i = 0; i < 3; ++i) {
    if (merged) {
      const uint64_t d[3] = {static_cast<uint64_t>(kBK), static_cast<uint64_t>(rows), static_cast<uint64_t>(cols / kBK)};
      const uint64_t st[2] = {static_cast<uint64_t>(cols) * 2, static_cast<uint64_t>(kBK) * 2};
      const uint32_t b[3] = {kBK, heights[i], static_cast<uint32_t>(kPairKC)};
      if (!make_map_strided(maps[i], base, 3, d, st, b)) return false;
    } else {
      const uint32_t b[2] = {kBK, heights[i]};
      if (!make_map(maps[i], base, 2, d2, b)) return false;
    }
  }
  // deep swap stages: 32- and 16-row boxes spanning three chunks (merged only;
  // otherwise copies that no tile reads)
  if (!merged) {
    *t32d = *t32;
    *t16d = *t16;
    return true;
  }
  CUtensorMap* dmaps[2] = {t32d, t16d};
  const uint32_t dheights[2] = {32, 16};
  for (int i = 0; i < 2; ++i) {
    const uint64_t d[3] = {static_cast<uint64_t>(kBK), static_cast<uint64_t>(rows), static_cast<uint64_t>(cols / kBK)};
    const uint64_t st[2] = {static_cast<uint64_t>(cols) * 2, static_cast<uint64_t>(kBK) * 2};
    const uint32_t b[3] = {kBK, dheights[i], static_cast<uint32_t>(kDeepKC)};
    if (!make_map_strided(dmaps[i], base, 3, d, st, b)) return false;
  }
  return true;
}

// Weight map of the pair kernel over w [groups, rows, K] (row-major):
// merged (64, rows, groups, K/64) with box (64, box_rows, box_groups, 2);
// else (K, rows, groups) with box (64, box_rows, 1).
static bool make_weight_map(CUtensorMap* m, const void* base, int64_t K, int64_t rows, int64_t groups,
                            uint32_t box_rows, uint32_t box_groups, bool merged, int chunks = kPairKC) {
  if (merged) {
    const uint64_t d[4] = {static_cast<uint64_t>(kBK), static_cast<uint64_t>(rows), static_cast<uint64_t>(groups),
                           static_cast<uint64_t>(K / kBK)};
    const uint64_t st[3] = {static_cast<uint64_t>(K) * 2, static_cast<uint64_t>(K * rows) * 2,
                            static_cast<uint64_t>(kBK) * 2};
    const uint32_t b[4] = {kBK, box_rows, box_groups, static_cast<uint32_t>(chunks)};
    return make_map_strided(m, base, 4, d, st, b);
  }
  const uint64_t d[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(rows), static_cast<uint64_t>(groups)};
  const uint32_t b[3] = {kBK, box_rows, 1};
  return make_map(m, base, 3, d, b);
}

// Chunk-merged boxes need whole 64-wide chunks; MOE_B200_MERGED_K=0 turns them off.
static bool merged_k_ok(int64_t K) {
  const char* e = getenv("MOE_B200_MERGED_K");
  if (e && !strcmp(e, "0")) return false;
  return K % kBK == 0;
}

// (ta2, tb2, a2, tile_bound2): an optional second problem whose tiles the same
// launch interleaves with the first's (see decode_mixed_tile).
template <int EPI, int BN, int STAGES>
static int run_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& a, int64_t tile_bound,
                    cudaStream_t st, const CUtensorMap* ta2 = nullptr, const CUtensorMap* tb2 = nullptr,
                    const GemmArgs* a2 = nullptr, int64_t tile_bound2 = 0) {
  constexpr int smem = gemm_smem_bytes<EPI, BN, STAGES>();
  // the dynamic shared-memory opt-in is per device: set it once per device
  static std::mutex mu;
  static uint64_t done = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -3;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!((done >> dev) & 1u)) {
      if (cudaFuncSetAttribute(grouped_gemm_tc_kernel<EPI, BN, STAGES>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return -3;
      done |= uint64_t(1) << dev;
    }
  }
  const bool two = ta2 && tb2 && a2;
  if (two) tile_bound += tile_bound2;
  if (tile_bound <= 0) return 0;
  int64_t grid = num_sms();
  if (grid > tile_bound) grid = tile_bound;
  // without a second problem its maps are the first's (never read: no tiles)
  GemmArgs b = two ? *a2 : a;
  if (!two) b.n_groups = 0;
  return launch_k(grouped_gemm_tc_kernel<EPI, BN, STAGES>, dim3(static_cast<unsigned>(grid)), dim3(kGemmThreads),
                  smem, st, ta, tb, a, two ? *ta2 : ta, two ? *tb2 : tb, b) == cudaSuccess ? 0 : -3;
}

// One problem of a pair-kernel launch: its tensor maps (see the kernel's
// parameters), arguments and an upper bound on its tiles.
struct PairProblem {
  CUtensorMap ta, tb, ta64, tb64, ta32, ta16;
  CUtensorMap ta32d, ta16d, tb64d;  // deep swap stages (three chunks per box)
  GemmArgs a;
  int64_t tile_bound;
};

// p2 (or nullptr): a second problem whose tiles the same launch interleaves
// with p1's (same EPI and tile shape; see decode_pair_tile).
template <int EPI>
static int run_pair_gemm(const PairProblem& p1, const PairProblem* p2, cudaStream_t st) {
  constexpr int smem = pair_smem_bytes();
  static std::mutex mu;
  static int max_pairs[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -3;
  int pairs;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (max_pairs[dev] == 0) {
      if (cudaFuncSetAttribute(grouped_gemm_pair_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess)
        return -3;
      // a persistent grid must fit at once: ask how many 2-CTA clusters can be co-resident
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
      cfg.blockDim = dim3(kGemmThreads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, grouped_gemm_pair_kernel<EPI>, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = num_sms() / 2;
      }
      max_pairs[dev] = n;
    }
    pairs = max_pairs[dev];
  }
  const int64_t tile_bound = p1.tile_bound + (p2 ? p2->tile_bound : 0);
  if (tile_bound <= 0) return 0;
  if (pairs > tile_bound) pairs = static_cast<int>(tile_bound);
  // without a second problem its maps are p1's (never read: no tiles)
  const PairProblem& q = p2 ? *p2 : p1;
  GemmArgs a2 = q.a;
  if (!p2) a2.n_groups = 0;
  return launch_k(grouped_gemm_pair_kernel<EPI>, dim3(static_cast<unsigned>(2 * pairs)), dim3(kGemmThreads), smem,
                  st, p1.ta, p1.tb, p1.ta64, p1.tb64, p1.ta32, p1.ta16, p1.a, q.ta, q.tb, q.ta64, q.tb64, q.ta32,
                  q.ta16, a2, p1.ta32d, p1.ta16d, p1.tb64d, q.ta32d, q.ta16d, q.tb64d) == cudaSuccess ? 0 : -3;
}

static int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Tile shape of the expert GEMMs:
//   single     128-row tiles on single CTAs
//   pair+tail  each group's rows rounded down to a multiple of 256 as 256-row
//              tiles on CTA pairs, the rest (under 256 rows) as 128-row tiles
//              on single CTAs (second launch): padding as with 128-row tiles
//   pair       every group on 256-row pair tiles (padding up to 255 rows)
// Measured choice: the pair shape, with operand-swapped remainder tiles, for
// groups of at least 256 expected rows (routed: T*K/E capped by the capacity;
// shared: every row), single CTAs below (decode-sized groups, where the
// weights' HBM stream bounds both shapes).
// MOE_B200_GEMM_TILE=128|256|256all forces single, pair+tail or pair (all
// complete implementations; the tests run each).
enum TileMode { kTileSingle = 0, kTilePairTail = 1, kTilePair = 2 };

// Largest last row tile of a group that the pair kernel computes operand-
// swapped (weights as the 256-row M operand, the tile's tokens as N): its MMAs
// cost in proportion to the rows it has, not to 256.  MOE_B200_SWAP_MAX
// (0..255) overrides; 0 turns swap tiles off.  Measured: with at most 128
// rows a swap tile is clearly cheaper than a 256-row tile; near 256 rows it
// is not (the transposing epilogue costs more than the padding saves).
// Deep (192-deep) stages for swap tiles of at most 64 token rows
// (MOE_B200_DEEP_SWAP=0 turns them off).
static bool deep_swap_on() {
  const char* e = getenv("MOE_B200_DEEP_SWAP");
  return !(e && e[0] == '0');
}

static int swap_max_rows() {
  const char* e = getenv("MOE_B200_SWAP_MAX");
  if (e && *e) {
    const int v = atoi(e);
    return v < 0 ? 0 : v > 255 ? 255 : v;
  }
  return 128;
}

static int tile_mode(int64_t expected_rows_per_group) {
  const char* e = getenv("MOE_B200_GEMM_TILE");
  if (e && !strcmp(e, "128")) return kTileSingle;
  if (e && !strcmp(e, "256")) return kTilePairTail;
  if (e && !strcmp(e, "256all")) return kTilePair;
  return expected_rows_per_group >= 256 ? kTilePair : kTileSingle;
}

int router_k_splits(const Problem& p) {
  // as many slices as keep every (row tile, slice) in one wave of CTAs
  const int64_t tiles = cdiv(p.T, kBM);
  int64_t s = num_sms() / tiles;
  const int64_t max_by_k = p.d / 256;  // keep at least four 64-wide k-blocks per slice
  if (s > max_by_k) s = max_by_k;
  if (s > kMaxLogitParts) s = kMaxLogitParts;
  if (s < 1) s = 1;
  const int64_t len = cdiv(cdiv(p.d, s), kBK) * kBK;
  return static_cast<int>(cdiv(p.d, len));
}

// Gate logits on the tensor cores: A = x [T, d], B = w_gate [E, d] padded to
// BN rows.  With n_splits > 1 the reduction over d is split into slices; slice
// s writes its partial logits at out + s*T*E (the offset goes into slice 0) and
// the selection kernel adds the slices in order.
int launch_gate_logits_tc(const Problem& p, const void* x, const void* w_gate, const float* offset, float* out,
                          int n_splits, unsigned* status, cudaStream_t st, unsigned long long* clk) {
  CUtensorMap ta, tb;
  const uint64_t da[2] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(p.T)};
  const uint32_t ba[2] = {kBK, kBM};
  if (!make_map(&ta, x, 2, da, ba)) return -3;
  const int bn = p.E <= 32 ? 32 : p.E <= 64 ? 64 : p.E <= 128 ? 128 : 256;
  const uint64_t db[3] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(p.E), 1};
  const uint32_t bb[3] = {kBK, static_cast<uint32_t>(bn), 1};
  if (!make_map(&tb, w_gate, 3, db, bb)) return -3;
  GemmArgs a{};
  a.stall_ns = test_stall_ns();
  a.n_groups = n_splits;
  a.seg_off = nullptr;
  a.n_rows = static_cast<int>(p.T);
  a.N = p.E;
  a.K = p.d;
  a.k_groups = 1;
  a.out = out;
  a.ldo = p.E;
  a.out_col_stride = 0;
  a.col_add = offset;
  a.status = status;
  a.k_split = n_splits > 1 ? static_cast<int>(cdiv(cdiv(p.d, n_splits), kBK) * kBK) : 0;
  a.out_group_stride = p.T * p.E;
  a.clk = clk;
  const int64_t tiles = cdiv(p.T, kBM) * n_splits;
  switch (bn) {
    case 32: return run_gemm<EPI_F32, 32, 8>(ta, tb, a, tiles, st);
    case 64: return run_gemm<EPI_F32, 64, 8>(ta, tb, a, tiles, st);
    case 128: return run_gemm<EPI_F32, 128, 6>(ta, tb, a, tiles, st);
    default: return run_gemm<EPI_F32, 256, 4>(ta, tb, a, tiles, st);
  }
}

// ============================================================================
// FP32 path on CUDA cores (tensor-core TF32 would not meet an FP32 tolerance).
// C[r, n] = sum_k A[r, k] * B[n, k] over 32x32 output tiles; SWIGLU mode
// computes gate and up accumulators together and writes silu(g) * u.
// grid = (column tiles, row tiles of the largest group, groups).
// ============================================================================
template <bool SWIGLU>
__global__ void __launch_bounds__(256) ffn_simt_kernel(const float* __restrict__ A, int lda,
                                                       const float* __restrict__ B, const GemmArgs args,
                                                       int64_t b_group_stride, int64_t b_up_offset) {
  __shared__ float As[32][33];
  __shared__ float Bg[32][33];
  __shared__ float Bu[SWIGLU ? 32 : 1][33];
  pdl_wait();
  pdl_trigger();
  const int g = blockIdx.z;
  int base;
  const int rows = group_rows(args, g, &base);
  const int m0 = blockIdx.y * 32;
  if (m0 >= rows) return;
  const int n0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // ty: 8 row groups of 4 rows
  float accg[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
  for (int kg = 0; kg < args.k_groups; ++kg) {
    const int wg = args.weight_mod > 0 ? g % args.weight_mod : g;
    const float* Bm = B + static_cast<int64_t>(wg * args.k_groups + kg) * b_group_stride;
    for (int k0 = 0; k0 < args.K; k0 += 32) {
      for (int i = threadIdx.x; i < 32 * 32; i += 256) {
        const int rr = i / 32, kc = i % 32;
        const int arow = base + m0 + rr, acol = k0 + kc;
        As[rr][kc] = (m0 + rr < rows && acol < args.K) ? A[static_cast<int64_t>(arow) * lda + kg * args.K + acol] : 0.f;
        const int bn = n0 + rr;
        const bool bok = bn < args.N && acol < args.K;
        Bg[rr][kc] = bok ? Bm[static_cast<int64_t>(bn) * args.K + acol] : 0.f;
        if (SWIGLU) Bu[rr][kc] = bok ? Bm[b_up_offset + static_cast<int64_t>(bn) * args.K + acol] : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int kc = 0; kc < 32; ++kc) {
        const float bg = Bg[tx][kc];
        const float bu = SWIGLU ? Bu[tx][kc] : 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float av = As[ty * 4 + i][kc];
          accg[i] = fmaf(av, bg, accg[i]);
          if (SWIGLU) accu[i] = fmaf(av, bu, accu[i]);
        }
      }
      __syncthreads();
    }
  }
  const int n = n0 + tx;
  if (n >= args.N) return;
  float* out = static_cast<float*>(args.out);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = m0 + ty * 4 + i;
    if (rr < rows) {
      float v = accg[i];
      if (SWIGLU) v = v / (1.0f + expf(-v)) * accu[i];
      out[static_cast<int64_t>(base + rr) * args.ldo + static_cast<int64_t>(g) * args.out_col_stride + n] = v;
    }
  }
}

static int ffn_simt(const Problem& p, int mode, const void* x_rows, int64_t n_rows, const int32_t* seg_off,
                    const void* w13, const void* w2, void* h, void* y_rows, cudaStream_t st, cudaEvent_t after_up,
                    int n_seg) {
  const bool routed = mode == 0;
  const int G = routed ? (n_seg > 0 ? n_seg : p.E) : p.Ns;
  int64_t max_group_rows = routed ? (p.cap < 0 ? p.T : (p.cap < p.T ? p.cap : p.T)) : n_rows;
  if (n_seg > 0) max_group_rows = n_rows;  // a segment may hold any number of the rows
  if (max_group_rows > n_rows) max_group_rows = n_rows;
  if (max_group_rows <= 0) return 0;
  GemmArgs up{};
  up.n_groups = G;
  up.weight_mod = routed && n_seg > 0 ? p.E : 0;
  up.seg_off = routed ? seg_off : nullptr;
  up.n_rows = static_cast<int>(n_rows);
  up.N = p.F;
  up.K = p.d;
  up.k_groups = 1;
  up.out = h;
  up.ldo = routed ? p.F : static_cast<int64_t>(p.Ns) * p.F;
  up.out_col_stride = routed ? 0 : p.F;
  dim3 g1(static_cast<unsigned>(cdiv(p.F, 32)), static_cast<unsigned>(cdiv(max_group_rows, 32)), G);
  if (launch_k(ffn_simt_kernel<true>, g1, dim3(256), 0, st, static_cast<const float*>(x_rows), p.d,
               static_cast<const float*>(w13), up, 2LL * p.F * p.d, static_cast<int64_t>(p.F) * p.d) != cudaSuccess)
    return -3;
  if (after_up && cudaEventRecord(after_up, st) != cudaSuccess) return -3;
  GemmArgs dn{};
  dn.n_groups = routed ? G : 1;
  dn.weight_mod = up.weight_mod;
  dn.seg_off = routed ? seg_off : nullptr;
  dn.n_rows = static_cast<int>(n_rows);
  dn.N = p.d;
  dn.K = p.F;
  dn.k_groups = routed ? 1 : p.Ns;
  dn.out = y_rows;
  dn.ldo = p.d;
  dn.out_col_stride = 0;
  dim3 g2(static_cast<unsigned>(cdiv(p.d, 32)), static_cast<unsigned>(cdiv(max_group_rows, 32)), dn.n_groups);
  return launch_k(ffn_simt_kernel<false>, g2, dim3(256), 0, st, static_cast<const float*>(h),
                  static_cast<int>(up.ldo), static_cast<const float*>(w2), dn, static_cast<int64_t>(p.d) * p.F,
                  static_cast<int64_t>(0)) == cudaSuccess ? 0 : -3;
}

// The gate and up projections without SwiGLU, for the backward: gu = x W13^T
// as BF16 (routed: [n_rows, 2F] per expert row; shared: [n_rows, N_s * 2F],
// expert s in columns [2F s, 2F (s + 1))), columns 0..F-1 of a block the gate
// projection, F..2F-1 the up projection.
int launch_up_projections(const Problem& p, int mode, const void* x_rows, int64_t n_rows, const int32_t* seg_off,
                          const void* w13, void* gu, unsigned* status, cudaStream_t st) {
  if (n_rows <= 0) return 0;
  const bool routed = mode == 0;
  const int G = routed ? p.E : p.Ns;
  CUtensorMap ta, tb;
  const uint64_t da[2] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(n_rows)};
  const uint32_t ba[2] = {kBK, kBM};
  const uint64_t db[3] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(2 * p.F), static_cast<uint64_t>(G)};
  const uint32_t bb[3] = {kBK, 256, 1};
  if (!make_map(&ta, x_rows, 2, da, ba) || !make_map(&tb, w13, 3, db, bb)) return -3;
  GemmArgs a{};
  a.n_groups = G;
  a.seg_off = routed ? seg_off : nullptr;
  a.n_rows = static_cast<int>(n_rows);
  a.N = 2 * p.F;
  a.K = p.d;
  a.k_groups = 1;
  a.out = gu;
  a.ldo = routed ? 2 * static_cast<int64_t>(p.F) : 2 * static_cast<int64_t>(p.F) * p.Ns;
  a.out_col_stride = routed ? 0 : 2 * p.F;
  a.status = status;
  const int64_t mt = routed ? cdiv(n_rows, kBM) + G : G * cdiv(n_rows, kBM);
  return run_gemm<EPI_BF16, 256, 4>(ta, tb, a, mt * cdiv(2 * p.F, 256), st);
}

// Tile shape of one FFN (routed: expected rows per group T*K/E capped by the
// capacity; shared: every row).
static int ffn_tile_mode(const Problem& p, bool routed, int64_t n_rows) {
  int64_t expected = routed ? (p.T * p.K) / p.E : n_rows;
  if (routed && p.cap >= 0 && p.cap < expected) expected = p.cap;
  return tile_mode(expected);
}

// Pair-kernel problem of an up/gate projection + SwiGLU: A = x_rows [n_rows, d],
// B = w13 [G, 2F, d] viewed as (d, F, 2G): gate rows of group g at 2g, up rows
// at 2g+1; swap tiles take 64 gate and the same 64 up rows per CTA.
static bool up_pair_problem(const Problem& p, bool routed, const void* x_rows, int64_t n_rows,
                            const int32_t* seg_off, const void* w13, void* h, void* gu, unsigned* status, bool tail,
                            PairProblem* q, int n_seg = 0) {
  const int G = routed ? p.E : p.Ns;
  const bool merged = merged_k_ok(p.d);
  if (!make_token_maps(&q->ta, &q->ta64, &q->ta32, &q->ta16, &q->ta32d, &q->ta16d, x_rows, p.d, n_rows, merged) ||
      !make_weight_map(&q->tb, w13, p.d, p.F, 2 * G, 128, 1, false) ||
      !make_weight_map(&q->tb64, w13, p.d, p.F, 2 * G, 64, merged ? 2 : 1, merged))
    return false;
  if (merged) {
    if (!make_weight_map(&q->tb64d, w13, p.d, p.F, 2 * G, 64, 2, true, kDeepKC)) return false;
  } else {
    q->tb64d = q->tb64;
  }
  GemmArgs& a = q->a;
  a = GemmArgs{};
  a.n_groups = n_seg > 0 ? n_seg : G;  // routed row segments (n_seg: expert = segment % E)
  a.weight_mod = n_seg > 0 ? G : 0;
  a.seg_off = routed ? seg_off : nullptr;
  a.n_rows = static_cast<int>(n_rows);
  a.N = p.F;
  a.K = p.d;
  a.k_groups = 1;
  a.out = h;
  a.ldo = routed ? p.F : static_cast<int64_t>(p.Ns) * p.F;
  a.out_col_stride = routed ? 0 : p.F;
  a.status = status;
  a.swap_max = swap_max_rows();
  a.gu = gu;  // kept for the backward (routed [rows, 2F]; shared [rows, N_s 2F])
  a.ld_gu = 2 * static_cast<int64_t>(p.F) * (routed ? 1 : p.Ns);
  a.gu_col_stride = routed ? 0 : 2 * p.F;
  a.row_mode = tail ? 1 : 0;  // 1: full 256-row blocks only
  a.merged_k = merged ? 1 : 0;
  a.deep_swap = merged && deep_swap_on() ? 1 : 0;
  const int64_t mt = routed ? cdiv(n_rows, kBM) + a.n_groups : G * cdiv(n_rows, kBM);
  q->tile_bound = (mt / 2 + a.n_groups) * cdiv(p.F, 128);
  return true;
}

// Pair-kernel problem of a down projection: A = h [n_rows, k_groups * F],
// B = w2 [G, d, F] viewed as (F, d, G); a pair CTA stages half of the 256 B
// rows.  Shared: one group whose reduction runs over all N_s experts.
static bool down_pair_problem(const Problem& p, bool routed, const void* h, int64_t n_rows, const int32_t* seg_off,
                              const void* w2, void* y_rows, unsigned* status, bool tail, PairProblem* q,
                              int n_seg = 0) {
  const int G = routed ? p.E : p.Ns;
  const int64_t h_cols = routed ? p.F : static_cast<int64_t>(p.Ns) * p.F;
  const bool merged = merged_k_ok(p.F);
  if (!make_token_maps(&q->ta, &q->ta64, &q->ta32, &q->ta16, &q->ta32d, &q->ta16d, h, h_cols, n_rows, merged) ||
      !make_weight_map(&q->tb, w2, p.F, p.d, G, 128, 1, false) ||
      !make_weight_map(&q->tb64, w2, p.F, p.d, G, 128, 1, merged))
    return false;
  if (merged) {
    if (!make_weight_map(&q->tb64d, w2, p.F, p.d, G, 128, 1, true, kDeepKC)) return false;
  } else {
    q->tb64d = q->tb64;
  }
  GemmArgs& a = q->a;
  a = GemmArgs{};
  a.n_groups = routed ? (n_seg > 0 ? n_seg : G) : 1;
  a.weight_mod = routed && n_seg > 0 ? G : 0;
  a.seg_off = routed ? seg_off : nullptr;
  a.n_rows = static_cast<int>(n_rows);
  a.N = p.d;
  a.K = p.F;
  a.k_groups = routed ? 1 : p.Ns;
  a.out = y_rows;
  a.ldo = p.d;
  a.out_col_stride = 0;
  a.status = status;
  a.swap_max = swap_max_rows();
  a.row_mode = tail ? 1 : 0;
  a.merged_k = merged ? 1 : 0;
  a.deep_swap = merged && deep_swap_on() ? 1 : 0;
  const int64_t mt = routed ? cdiv(n_rows, kBM) + a.n_groups : cdiv(n_rows, kBM);
  q->tile_bound = (mt / 2 + a.n_groups) * cdiv(p.d, 256);
  return true;
}

// One problem of a single-CTA launch (128-row tiles).
struct SingleProblem {
  CUtensorMap ta, tb;
  GemmArgs a;
  int64_t tile_bound;
};

// Up/gate projection + SwiGLU on single CTAs: A = x_rows [n_rows, d], B = w13
// [G, 2F, d] viewed as (d, F, 2G) with 128-row boxes (gate rows of group g at
// 2g, up rows at 2g+1).
static bool up_single_problem(const Problem& p, bool routed, const void* x_rows, int64_t n_rows,
                              const int32_t* seg_off, const void* w13, void* h, void* gu, unsigned* status,
                              SingleProblem* q, int n_seg = 0) {
  const int G = routed ? p.E : p.Ns;
  const uint64_t da[2] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(n_rows)};
  const uint32_t ba[2] = {kBK, kBM};
  const uint64_t db[3] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(p.F), static_cast<uint64_t>(2 * G)};
  const uint32_t bb[3] = {kBK, 128, 1};
  if (!make_map(&q->ta, x_rows, 2, da, ba) || !make_map(&q->tb, w13, 3, db, bb)) return false;
  GemmArgs& a = q->a;
  a = GemmArgs{};
  a.stall_ns = test_stall_ns();
  a.n_groups = n_seg > 0 ? n_seg : G;
  a.weight_mod = n_seg > 0 ? G : 0;
  a.seg_off = routed ? seg_off : nullptr;
  a.n_rows = static_cast<int>(n_rows);
  a.N = p.F;
  a.K = p.d;
  a.k_groups = 1;
  a.out = h;
  a.ldo = routed ? p.F : static_cast<int64_t>(p.Ns) * p.F;
  a.out_col_stride = routed ? 0 : p.F;
  a.status = status;
  a.swap_max = swap_max_rows();
  a.gu = gu;
  a.ld_gu = 2 * static_cast<int64_t>(p.F) * (routed ? 1 : p.Ns);
  a.gu_col_stride = routed ? 0 : 2 * p.F;
  const int64_t mt = routed ? cdiv(n_rows, kBM) + a.n_groups : G * cdiv(n_rows, kBM);
  q->tile_bound = mt * cdiv(p.F, 128);
  return true;
}

// Down projection on single CTAs: A = h [n_rows, k_groups * F], B = w2 [G, d, F]
// viewed as (F, d, G) with 256-row boxes.
static bool down_single_problem(const Problem& p, bool routed, const void* h, int64_t n_rows,
                                const int32_t* seg_off, const void* w2, void* y_rows, unsigned* status,
                                SingleProblem* q, int n_seg = 0) {
  const int G = routed ? p.E : p.Ns;
  const int64_t h_cols = routed ? p.F : static_cast<int64_t>(p.Ns) * p.F;
  const uint64_t da[2] = {static_cast<uint64_t>(h_cols), static_cast<uint64_t>(n_rows)};
  const uint32_t ba[2] = {kBK, kBM};
  const uint64_t db[3] = {static_cast<uint64_t>(p.F), static_cast<uint64_t>(p.d), static_cast<uint64_t>(G)};
  const uint32_t bb[3] = {kBK, 256, 1};
  if (!make_map(&q->ta, h, 2, da, ba) || !make_map(&q->tb, w2, 3, db, bb)) return false;
  GemmArgs& a = q->a;
  a = GemmArgs{};
  a.stall_ns = test_stall_ns();
  a.n_groups = routed ? (n_seg > 0 ? n_seg : G) : 1;
  a.weight_mod = routed && n_seg > 0 ? G : 0;
  a.seg_off = routed ? seg_off : nullptr;
  a.n_rows = static_cast<int>(n_rows);
  a.N = p.d;
  a.K = p.F;
  a.k_groups = routed ? 1 : p.Ns;
  a.out = y_rows;
  a.ldo = p.d;
  a.out_col_stride = 0;
  a.status = status;
  a.swap_max = swap_max_rows();
  const int64_t mt = routed ? cdiv(n_rows, kBM) + a.n_groups : cdiv(n_rows, kBM);
  q->tile_bound = mt * cdiv(p.d, 256);
  return true;
}

// mode 0: routed (groups = experts over seg_off); mode 1: shared (every row
// through all N_s experts, summed).  h is scratch: [n_rows, F] (routed) or
// [n_rows, N_s * F] (shared).
int launch_expert_ffn(const Problem& p, int mode, const void* x_rows, int64_t n_rows, const int32_t* seg_off,
                      const void* w13, const void* w2, void* h, void* y_rows, unsigned* status, cudaStream_t st,
                      cudaEvent_t after_up, int* n_kernels, void* gu, unsigned long long* clk_up,
                      unsigned long long* clk_down, int n_seg) {
  if (n_rows <= 0) return 0;
  if (p.dtype == kF32) {
    if (n_kernels) *n_kernels += 2;
    return ffn_simt(p, mode, x_rows, n_rows, seg_off, w13, w2, h, y_rows, st, after_up, n_seg);
  }
  const bool routed = mode == 0;
  const int G = routed ? p.E : p.Ns;
  const int64_t h_cols = routed ? p.F : static_cast<int64_t>(p.Ns) * p.F;
  const int mode_t = ffn_tile_mode(p, routed, n_rows);
  const bool pair = mode_t != kTileSingle;
  const bool tail = mode_t == kTilePairTail;
  if (n_kernels) *n_kernels += tail ? 4 : 2;

  // up/gate projection + SwiGLU
  {
    const uint64_t da[2] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(n_rows)};
    const uint32_t ba[2] = {kBK, kBM};
    const uint64_t db[3] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(p.F), static_cast<uint64_t>(2 * G)};
    const uint32_t bb[3] = {kBK, 128, 1};
    CUtensorMap ta, tb;
    if (pair) {
      PairProblem q;
      if (!up_pair_problem(p, routed, x_rows, n_rows, seg_off, w13, h, gu, status, tail, &q, n_seg)) return -3;
      q.a.clk = clk_up;
      int rc = run_pair_gemm<EPI_SWIGLU>(q, nullptr, st);
      if (rc) return rc;
      if (tail) {
        GemmArgs a = q.a;
        a.row_mode = 2;  // the rest (under 256 rows per group) on single CTAs
        a.swap_max = 0;
        a.merged_k = 0;
        if (!make_map(&ta, x_rows, 2, da, ba) || !make_map(&tb, w13, 3, db, bb)) return -3;
        rc = run_gemm<EPI_SWIGLU, 256, 4>(ta, tb, a, 2 * a.n_groups * cdiv(p.F, 128), st);
        if (rc) return rc;
      }
    } else {
      SingleProblem q;
      if (!up_single_problem(p, routed, x_rows, n_rows, seg_off, w13, h, gu, status, &q, n_seg)) return -3;
      q.a.clk = clk_up;
      const int rc = run_gemm<EPI_SWIGLU, 256, 4>(q.ta, q.tb, q.a, q.tile_bound, st);
      if (rc) return rc;
    }
    if (after_up && cudaEventRecord(after_up, st) != cudaSuccess) return -3;
  }
  // down projection
  {
    const uint64_t da[2] = {static_cast<uint64_t>(h_cols), static_cast<uint64_t>(n_rows)};
    const uint32_t ba[2] = {kBK, kBM};
    const uint64_t db[3] = {static_cast<uint64_t>(p.F), static_cast<uint64_t>(p.d), static_cast<uint64_t>(G)};
    const uint32_t bb[3] = {kBK, 256, 1};
    CUtensorMap ta, tb;
    if (!make_map(&ta, h, 2, da, ba) || !make_map(&tb, w2, 3, db, bb)) return -3;
    if (pair) {
      PairProblem q;
      if (!down_pair_problem(p, routed, h, n_rows, seg_off, w2, y_rows, status, tail, &q, n_seg)) return -3;
      q.a.clk = clk_down;
      int rc = run_pair_gemm<EPI_BF16>(q, nullptr, st);
      if (rc) return rc;
      if (tail) {
        GemmArgs a = q.a;
        a.row_mode = 2;
        a.swap_max = 0;
        a.merged_k = 0;
        rc = run_gemm<EPI_BF16, 256, 4>(ta, tb, a, 2 * a.n_groups * cdiv(p.d, 256), st);
        if (rc) return rc;
      }
    } else {
      SingleProblem q;
      if (!down_single_problem(p, routed, h, n_rows, seg_off, w2, y_rows, status, &q, n_seg)) return -3;
      q.a.clk = clk_down;
      const int rc = run_gemm<EPI_BF16, 256, 4>(q.ta, q.tb, q.a, q.tile_bound, st);
      if (rc) return rc;
    }
  }
  return 0;
}

bool expert_ffn_mixed_ok(const Problem& p) {
  const char* e = getenv("MOE_B200_MIX_SHARED");
  if (e && e[0] == '0') return false;
  if (p.dtype != kBF16 || p.Ns <= 0 || p.max_rows <= 0) return false;
  const int mr = ffn_tile_mode(p, true, p.max_rows), ms = ffn_tile_mode(p, false, p.T);
  return mr == ms && mr != kTilePairTail;
}

// Routed and shared experts in the same two launches (up/gate + SwiGLU for
// both, then both down projections), on CTA pairs or on single CTAs: no
// launch of its own for the shared experts, whose few tiles (decode: one row
// tile) would otherwise run on a handful of SMs while the rest wait.
int launch_expert_ffn_mixed(const Problem& p, const void* x_perm, const int32_t* seg_off, const void* w13,
                            const void* w2, void* h, void* y_perm, void* gu, const void* x, const void* w13_shared,
                            const void* w2_shared, void* h_shared, void* y_shared, void* gu_shared, unsigned* status,
                            cudaStream_t st, cudaEvent_t after_up, int* n_kernels, unsigned long long* clk_up,
                            unsigned long long* clk_down) {
  if (!expert_ffn_mixed_ok(p)) return -3;
  if (n_kernels) *n_kernels += 2;
  if (ffn_tile_mode(p, true, p.max_rows) == kTileSingle) {
    SingleProblem r, s;
    if (!up_single_problem(p, true, x_perm, p.max_rows, seg_off, w13, h, gu, status, &r) ||
        !up_single_problem(p, false, x, p.T, nullptr, w13_shared, h_shared, gu_shared, status, &s))
      return -3;
    r.a.clk = clk_up;
    if (int rc = run_gemm<EPI_SWIGLU, 256, 4>(r.ta, r.tb, r.a, r.tile_bound, st, &s.ta, &s.tb, &s.a, s.tile_bound))
      return rc;
    if (after_up && cudaEventRecord(after_up, st) != cudaSuccess) return -3;
    if (!down_single_problem(p, true, h, p.max_rows, seg_off, w2, y_perm, status, &r) ||
        !down_single_problem(p, false, h_shared, p.T, nullptr, w2_shared, y_shared, status, &s))
      return -3;
    r.a.clk = clk_down;
    return run_gemm<EPI_BF16, 256, 4>(r.ta, r.tb, r.a, r.tile_bound, st, &s.ta, &s.tb, &s.a, s.tile_bound);
  }
  PairProblem r, s;
  if (!up_pair_problem(p, true, x_perm, p.max_rows, seg_off, w13, h, gu, status, false, &r) ||
      !up_pair_problem(p, false, x, p.T, nullptr, w13_shared, h_shared, gu_shared, status, false, &s))
    return -3;
  r.a.clk = clk_up;
  if (int rc = run_pair_gemm<EPI_SWIGLU>(r, &s, st)) return rc;
  if (after_up && cudaEventRecord(after_up, st) != cudaSuccess) return -3;
  if (!down_pair_problem(p, true, h, p.max_rows, seg_off, w2, y_perm, status, false, &r) ||
      !down_pair_problem(p, false, h_shared, p.T, nullptr, w2_shared, y_shared, status, false, &s))
    return -3;
  r.a.clk = clk_down;
  return run_pair_gemm<EPI_BF16>(r, &s, st);
}

}  // namespace moe
