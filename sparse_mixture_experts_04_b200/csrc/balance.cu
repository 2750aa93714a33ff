// Load-balancing update between steps, from one step's pre-capacity counts.
//
//   Zen-Max, §2.3 Auxiliary-Loss-Free Load Balancing: the per-expert
//   selection bias b_e is adjusted after every step against the deviation of
//   the expert's load from its target (overloaded: lowered; underloaded:
//   raised).  Load = counts[e], target = T*K/E; step `rate` times the sign of
//   (target - load), or times the relative deviation (target - load)/target.
//
//   Zen MoDE, §5.3 Adaptive Capacity Factors: C_e = C_base + gamma *
//   (fbar_e - 1/N_E), fbar_e the load fraction counts[e]/(T*K) averaged over a
//   rolling window of steps; capacity_e = ceil(C_e * T*K / E) in [0, T].
//
// One block, one thread per expert.  All arithmetic is float64 with explicitly
// rounded operations (no contraction into fused multiply-adds), so the result
// is the correctly rounded value of each step of the formulas above, in the
// order written there.
#include "common.cuh"
#include "internal.h"

namespace moe {

__global__ void __launch_bounds__(kMaxExperts) balance_update_kernel(
    const int32_t* __restrict__ counts, int E, int64_t T, int K, float* __restrict__ bias, float rate, int mode,
    int32_t* __restrict__ hist, int hist_slot, int hist_rows, float c_base, float gamma,
    int32_t* __restrict__ caps) {
  pdl_wait();
  pdl_trigger();
  const int e = threadIdx.x;
  if (e >= E) return;
  const int c = counts[e];
  const int64_t TK = T * K;
  const double tk = static_cast<double>(TK);
  if (bias) {
    const int64_t dev = TK - static_cast<int64_t>(E) * c;   // E * (target - load), exact
    double step;
    if (mode == 0)
      step = __dmul_rn(static_cast<double>(rate), static_cast<double>((dev > 0) - (dev < 0)));
    else
      step = __dmul_rn(static_cast<double>(rate), __ddiv_rn(static_cast<double>(dev), tk));
    bias[e] = __double2float_rn(__dadd_rn(static_cast<double>(bias[e]), step));
  }
  if (caps) {
    // this thread owns column e of the ring: write this step's row, then sum
    // the rows written so far
    hist[static_cast<int64_t>(hist_slot) * E + e] = c;
    int64_t s = 0;
    for (int i = 0; i < hist_rows; ++i) s += hist[static_cast<int64_t>(i) * E + e];
    const double fbar = __ddiv_rn(static_cast<double>(s), __dmul_rn(static_cast<double>(hist_rows), tk));
    const double ce = __dadd_rn(static_cast<double>(c_base),
                                __dmul_rn(static_cast<double>(gamma),
                                          __dsub_rn(fbar, __ddiv_rn(1.0, static_cast<double>(E)))));
    const double v = ceil(__ddiv_rn(__dmul_rn(ce, tk), static_cast<double>(E)));
    caps[e] = v <= 0.0 ? 0 : (v >= static_cast<double>(T) ? static_cast<int32_t>(T) : static_cast<int32_t>(v));
  }
}

cudaError_t launch_balance_update(const Problem& p, const int32_t* counts, float* bias, float rate, int mode,
                                  int32_t* hist, int hist_slot, int hist_rows, float c_base, float gamma,
                                  int32_t* caps, cudaStream_t st) {
  return launch_k(balance_update_kernel, dim3(1), dim3(kMaxExperts), 0, st, counts, p.E, p.T, p.K, bias, rate, mode,
                  hist, hist_slot, hist_rows, c_base, gamma, caps);
}

}  // namespace moe
