// One token's softmax, top-K selection (optional selection bias) and
// renormalised gate weights on a group of G lanes (G = 8, 16 or 32: one warp
// ranks 32 / G tokens at once).  Shared by the selection kernel (router.cu,
// logits from global memory, G = 32) and the fused router (router_fused.cu,
// logits from shared memory), so both rank alike.
//
//   Zen MoDE: Mixture of Distilled Experts Architecture, §3.1 Router
//     Architecture, eq. router_standard: TopK(softmax(W_r x), K).
//   Zen-Max, §2.3 Auxiliary-Loss-Free Load Balancing: s_ij = softmax(x_i W_g)_j + b_j.
//   Scaling with experts, "The gating network": the chosen scores rescaled to add up to 1.
//
// Lane l of the group holds experts l, l + G, ... (EPL of them):
//   m = max logit; ex_e = exp(l_e - m) (fp32); Z = sum ex; p_e = ex_e / Z
//   score_e: l_e, or p_e + b_e (bias on p), or l_e + b_e (bias on the logit)
//   K rounds of a warp arg-max over (score descending, expert index ascending)
//   w_k = ex_{idx_k} / sum_k ex_{idx_k}   (= the softmax over the chosen)
// lg[i]: the logit of expert l + G i, -inf for e >= E; bias[i]: its
// selection bias (0 without one).  Adds p_e to pacc, logsumexp^2 to zacc,
// writes idx_row[k] and w_row[k] for k < K (lanes k of the group), and counts
// each chosen expert in s_count (shared memory).  Every lane of the group must
// call it, with K <= G or G = 32.  Cross-lane steps are shuffles within the
// group (width G); with G = 32 the arg-max rounds use redux.sync.
#pragma once

#include <math.h>

#include "common.cuh"

namespace moe {

// Lanes of the group of G lanes that `lane` belongs to.
template <int G>
__device__ __forceinline__ unsigned grp_mask(int lane) {
  return G == 32 ? 0xffffffffu : (((1u << G) - 1u) << (lane & ~(G - 1)));
}

template <int G>
__device__ __forceinline__ float grp_max(float v, unsigned gm) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(gm, v, o, G));
  return v;
}

template <int G, typename V>
__device__ __forceinline__ V grp_sum(V v, unsigned gm) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(gm, v, o, G);
  return v;
}

template <int G>
__device__ __forceinline__ unsigned grp_max_u32(unsigned v, unsigned gm) {
  if constexpr (G == 32) {
    return __reduce_max_sync(gm, v);
  } else {
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(gm, v, o, G));
    return v;
  }
}

template <int G>
__device__ __forceinline__ int grp_min_i32(int v, unsigned gm) {
  if constexpr (G == 32) {
    return __reduce_min_sync(gm, v);
  } else {
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(gm, v, o, G));
    return v;
  }
}

// Every cross-lane step names only the lanes of the calling group (gm), so the
// groups of a warp may take different branches (a float64 re-ranking in one,
// not in another) or skip the call altogether.

// Float64 ranking of one token (a bias on the logit, or a bias on p whose
// float32 screen found a near-tie): K rounds of a group arg-max over
// order-preserving 64-bit keys of the float64 scores; returns this lane's
// winner (lane k: the k-th) and its exp(l - m).
template <int EPL, int G>
__device__ __forceinline__ void rank_token_fp64(const float (&lg)[EPL], const float (&ex)[EPL],
                                                const float (&bias)[EPL], bool has_bias, int bias_on_logit, int E,
                                                int K, int lane, unsigned gm, float m, int& my_e, float& my_ex) {
  double score[EPL];
  if (!has_bias) {
#pragma unroll
    for (int i = 0; i < EPL; ++i) score[i] = static_cast<double>(lg[i]);
  } else if (bias_on_logit) {
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + G * i;
      score[i] = (e < E) ? static_cast<double>(lg[i]) + static_cast<double>(bias[i]) : -INFINITY;
    }
  } else {
    const double m64 = static_cast<double>(m);
    double ex64[EPL];
    double z64loc = 0.0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + G * i;
      ex64[i] = (e < E) ? exp(static_cast<double>(lg[i]) - m64) : 0.0;
      z64loc += ex64[i];
    }
    const double z64 = grp_sum<G>(z64loc, gm);
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + G * i;
      score[i] = (e < E) ? ex64[i] / z64 + static_cast<double>(bias[i]) : -INFINITY;
    }
  }
  // Order-preserving 64-bit keys: a larger key is a larger score (NaN ranks
  // as -inf, -0 as +0); padding lanes and chosen experts get key 0, below
  // every real score.  (key, index ascending) is a total order, so every
  // lane agrees on each round's winner, which is always a valid expert.
  unsigned long long key[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    double sc = score[i];
    if (sc != sc) sc = -INFINITY;
    sc += 0.0;
    const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(sc));
    key[i] = (lane + G * i) >= E ? 0ull : ((b >> 63) ? ~b : (b | 0x8000000000000000ull));
  }
  // this lane's best remaining entry (equal keys: the lower slot, i.e. expert)
  unsigned long long bk = 0;
  int bi = 0;
#pragma unroll
  for (int i = 0; i < EPL; ++i)
    if (key[i] > bk) {
      bk = key[i];
      bi = i;
    }
  for (int k = 0; k < K; ++k) {
    // group arg-max: high word, then low word among the maxima, then the
    // lowest expert index among equal keys
    const unsigned hi = static_cast<unsigned>(bk >> 32), lo = static_cast<unsigned>(bk);
    const unsigned hmax = grp_max_u32<G>(hi, gm);
    const unsigned lmax = grp_max_u32<G>(hi == hmax ? lo : 0u, gm);
    const bool cand = bk != 0ull && hi == hmax && lo == lmax;
    const int best_e = grp_min_i32<G>(cand ? lane + G * bi : 0x7fffffff, gm);
    const int wl = best_e & (G - 1);
    float ex_mine = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if (i == bi) ex_mine = ex[i];
    const float ex_sel = __shfl_sync(gm, ex_mine, wl, G);
    if (lane == wl) {  // the winner's lane drops it and finds its next best
      bk = 0;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        if (i == bi) key[i] = 0ull;
      }
      bi = 0;
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (key[i] > bk) {
          bk = key[i];
          bi = i;
        }
    }
    if (lane == k) {
      my_e = best_e;
      my_ex = ex_sel;
    }
  }
}

// NT tokens per call on the same group: every step runs for all NT tokens
// before the next, so their dependency chains (the cross-lane reductions of
// the softmax and of each ranking round) overlap.  Per token the arithmetic is
// exactly that of NT = 1.  live[nt] false: token nt does not exist (its lg
// are ignored; nothing is written or counted for it).
template <int EPL, int G, int NT>
__device__ __forceinline__ void select_tokens(const float (&lg_in)[NT][EPL], const float (&bias)[EPL], bool has_bias,
                                              int bias_on_logit, int E, int K, int lane, const bool (&live)[NT],
                                              float (&pacc)[EPL], float& zacc, int32_t* const (&idx_row)[NT],
                                              float* const (&w_row)[NT], int* s_count) {
  static_assert(G == 8 || G == 16 || G == 32, "group of 8, 16 or 32 lanes");
  const unsigned gm = grp_mask<G>(lane);
  lane &= G - 1;  // this lane's place in its group
  float lg[NT][EPL];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int i = 0; i < EPL; ++i) lg[n][i] = live[n] ? lg_in[n][i] : 0.f;
  float m[NT], ex[NT][EPL], invZ[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    float mloc = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) mloc = fmaxf(mloc, lg[n][i]);
    m[n] = grp_max<G>(mloc, gm);
  }
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    float zloc = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + G * i;
      ex[n][i] = (e < E) ? expf(lg[n][i] - m[n]) : 0.f;
      zloc += ex[n][i];
    }
    const float Z = grp_sum<G>(zloc, gm);
    invZ[n] = 1.0f / Z;
    if (live[n]) {
      const float lse = m[n] + logf(Z);
      zacc += lse * lse;
#pragma unroll
      for (int i = 0; i < EPL; ++i) pacc[i] += ex[n][i] * invZ[n];
    }
  }

  int my_e[NT];
  float my_ex[NT];
  bool done[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    my_e[n] = -1;
    my_ex[n] = 0.f;
    done[n] = false;
  }
  if (!has_bias || !bias_on_logit) {
    // Ranked on 32-bit keys of float32 scores.  Without a bias the score is
    // the float32 logit itself, so this ranking is the exact one (K rounds).
    // Bias on p: the float32 scores s = ex/Z + b (K+1 rounds).  Each is
    // within d = (E+8) eps p + eps (|s| + 1) of the exact p + b (eps =
    // 2^-23; terms: expf's 2 ulp, the sum Z, 1/Z, the product, the add, and
    // the rounding of l - m, whose effect on p is at most eps |l - m| p / 2
    // <= eps / (2e)); if every gap between consecutive ones of the best K+1
    // exceeds 2d, the exact ranking of the top K is the same, else the
    // token is ranked again in float64 (rank_token_fp64).
    const bool biased = has_bias;
    unsigned hk[NT][EPL];
    int hs[NT][EPL];
    float s32[NT][EPL];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + G * i;
        float sc = (e < E) ? (biased ? ex[n][i] * invZ[n] + bias[i] : lg[n][i]) : 0.f;
        if (sc != sc) sc = -INFINITY;
        sc += 0.0f;
        s32[n][i] = sc;
        const unsigned b = __float_as_uint(sc);
        hk[n][i] = e >= E ? 0u : ((b >> 31) ? ~b : (b | 0x80000000u));
        hs[n][i] = i;
      }
      // this lane's keys in descending order with their slots (equal keys:
      // the lower slot, i.e. expert, first): a round only pops the winner's head
#pragma unroll
      for (int pass = 0; pass < EPL; ++pass)
#pragma unroll
        for (int i = pass & 1; i + 1 < EPL; i += 2)
          if (hk[n][i + 1] > hk[n][i]) {  // slots start ascending and equal keys never swap
            const unsigned tk = hk[n][i];
            hk[n][i] = hk[n][i + 1];
            hk[n][i + 1] = tk;
            const int ts = hs[n][i];
            hs[n][i] = hs[n][i + 1];
            hs[n][i + 1] = ts;
          }
    }
    const int rounds = biased ? K + 1 : K;
    for (int r = 0; r < rounds && r < G; ++r) {
      bool any = false;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const unsigned kmax = grp_max_u32<G>(hk[n][0], gm);
        const int best_e = grp_min_i32<G>((hk[n][0] != 0u && hk[n][0] == kmax) ? lane + G * hs[n][0] : 0x7fffffff, gm);
        if (lane == (best_e & (G - 1))) {
#pragma unroll
          for (int i = 0; i + 1 < EPL; ++i) {
            hk[n][i] = hk[n][i + 1];
            hs[n][i] = hs[n][i + 1];
          }
          hk[n][EPL - 1] = 0u;
        }
        if (lane == r) my_e[n] = best_e;
        any |= best_e != 0x7fffffff;
      }
      if (!any) break;  // fewer than K+1 experts (K == E)
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      // the winners' ex and score: expert e sits in lane e % G, slot e / G
      float my_s = 0.f;
      {
        const int src = my_e[n] & (G - 1), slot = my_e[n] / G;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const float a = __shfl_sync(gm, ex[n][i], src, G);
          const float b = __shfl_sync(gm, s32[n][i], src, G);
          if (i == slot) {
            my_ex[n] = a;
            my_s = b;
          }
        }
      }
      const float my_p = my_ex[n] * invZ[n];
      const float s_next = __shfl_down_sync(gm, my_s, 1, G);
      const float p_next = __shfl_down_sync(gm, my_p, 1, G);
      const float eps = 1.1920928955078125e-7f;  // 2^-23
      const float d = (static_cast<float>(E) + 8.0f) * eps * fmaxf(my_p, p_next) +
                      eps * (fmaxf(fabsf(my_s), fabsf(s_next)) + 1.0f);
      // with K == E there is no (K+1)-th score: the last gap only orders the set
      const bool last_ok = lane == K - 1 && K == E;
      const bool gap_ok = !biased || lane >= K || last_ok || (my_s - s_next > 2.0f * d);
      done[n] = grp_min_i32<G>(gap_ok ? 1 : 0, gm) != 0;
      if (!done[n]) {
        my_e[n] = -1;
        my_ex[n] = 0.f;
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NT; ++n)
    if (!done[n]) rank_token_fp64<EPL, G>(lg[n], ex[n], bias, has_bias, bias_on_logit, E, K, lane, gm, m[n], my_e[n],
                                          my_ex[n]);
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const float wsum = grp_sum<G>(lane < K ? my_ex[n] : 0.f, gm);
    if (live[n] && lane < K) {
      idx_row[n][lane] = my_e[n];
      w_row[n][lane] = my_ex[n] / wsum;
      if (static_cast<unsigned>(my_e[n]) < static_cast<unsigned>(E)) atomicAdd(&s_count[my_e[n]], 1);
    }
  }
}

// One token (see select_tokens).
template <int EPL, int G>
__device__ __forceinline__ void select_token_group(const float (&lg)[EPL], const float (&bias)[EPL], bool has_bias,
                                                   int bias_on_logit, int E, int K, int lane, float (&pacc)[EPL],
                                                   float& zacc, int32_t* __restrict__ idx_row,
                                                   float* __restrict__ w_row, int* s_count) {
  const float (&lg1)[1][EPL] = *reinterpret_cast<const float(*)[1][EPL]>(&lg);
  const bool live[1] = {true};
  int32_t* const rows_i[1] = {idx_row};
  float* const rows_w[1] = {w_row};
  select_tokens<EPL, G, 1>(lg1, bias, has_bias, bias_on_logit, E, K, lane, live, pacc, zacc, rows_i, rows_w, s_count);
}

}  // namespace moe
