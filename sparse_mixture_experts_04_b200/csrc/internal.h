// Internal declarations of libmoe_b200: the validated problem, the workspace
// layout and the kernel launchers each .cu file provides.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

struct moe_problem;  // include/moe_b200.h

namespace moe {

constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 32;
constexpr int kDispatchChunk = 256;  // tokens per block in the dispatch kernels
constexpr int kSelectTokens = 8;     // tokens per block in the selection kernel (one per warp)
constexpr int kMaxLogitParts = 8;    // most slices of the split-K gate GEMM
constexpr int kMaxSegments = 256;    // moe_expert_ffn_segments

enum Dtype { kBF16 = 0, kF32 = 1 };

struct Problem {
  int64_t T;
  int d, E, K, Ns, F;
  int64_t cap;       // effective per-expert capacity, min(cap_raw, T); -1: no limit
  int64_t cap_raw;   // ceil(C*T*K/E) as defined
  int64_t max_rows;  // upper bound on kept rows
  int dtype;
  uint32_t flags;
  float alpha;
  size_t esize() const { return dtype == kBF16 ? 2 : 4; }
};

// Byte offsets of every scratch array inside the caller's workspace.
struct WsLayout {
  size_t status, logits, topk_idx, topk_w, counts, kept, seg_off, slot_of, perm;
  size_t chunk_counts, chunk_psum, chunk_base, logit_parts, zpart;
  size_t seg_map;  // moe_expert_ffn_segments: [kMaxSegments] destinations + [kMaxSegments + 1] expert offsets
  size_t zero_bytes;  // status word + chunk histogram + chunk p sums: cleared together at offset 0
  size_t x_perm, h_routed, y_perm, h_shared, y_shared;
  size_t gu_routed, gu_shared;  // with MOE_FLAG_SAVE_GU: the gate/up projections for the backward
  size_t total;
  int n_chunks, n_sel_blocks;
};
WsLayout make_layout(const Problem& p);

// The ABI problem validated and converted (cap, max_rows derived); a moe_status.
int problem_from_abi(const ::moe_problem* in, Problem* out);

// router.cu
cudaError_t launch_gate_logits_simt(const Problem& p, const void* x, const void* w_gate,
                                    const float* offset, float* logits, cudaStream_t st);
// logits [T, E] are read, or (n_parts > 0) summed from n_parts slices at
// parts + s*T*E in slice order and written to logits.
// chunk_counts / chunk_psum: zeroed [n_chunks, E] arrays that receive, per
// dispatch chunk, the histogram of the chosen experts and the sum of p in
// fixed point (p_fixed_scale; integer atomics: exact and order-independent)
// zpart (or nullptr): [route_select_zparts(p)] partial sums of logsumexp^2
// (router z-loss), at most n_sel_blocks of them
int route_select_zparts(const Problem& p);
// clk (all launchers below; or nullptr): the stage clock the kernels stamp
// (moe_layer_forward_clocked)
cudaError_t launch_route_select(const Problem& p, float* logits, const float* parts, int n_parts,
                                const float* sel_bias, int32_t* topk_idx, float* topk_w, int32_t* chunk_counts,
                                unsigned long long* chunk_psum, float* zpart, cudaStream_t st,
                                unsigned long long* clk = nullptr);
// f, P and the loss from those chunk totals (moe_route's statistics); with
// zpart also the extended statistics (kept = min(counts, cap))
cudaError_t launch_route_stats(const Problem& p, const int32_t* chunk_counts, const unsigned long long* chunk_psum,
                               int n_chunks, const float* zpart, int n_zpart, float* stats, cudaStream_t st);

// dispatch.cu
// true when launch_dispatch ranks with one fused scan+rank kernel (else a
// scan kernel and a rank kernel)
bool dispatch_fused(const Problem& p);
// counts_ready: chunk_counts already hold the per-chunk expert histogram (the
// selection kernel adds it when given a zeroed chunk_counts)
// chunk_psum / stats: when both are given, the scan also finalises the
// balance statistics from the selection kernel's chunk totals.
// zpart / n_zpart: per-selection-block sums of logsumexp^2; given with stats,
// the extended statistics are written too.
// expert_cap (or nullptr): [E] per-expert capacities (negative: no limit)
// instead of p.cap.
cudaError_t launch_dispatch(const Problem& p, const int32_t* topk_idx, int32_t* counts, int32_t* kept,
                            int32_t* seg_off, int32_t* slot_of, int32_t* perm, int32_t* chunk_counts,
                            int32_t* chunk_base, unsigned* status, cudaStream_t st, bool counts_ready = false,
                            const unsigned long long* chunk_psum = nullptr, float* stats = nullptr,
                            const float* zpart = nullptr, int n_zpart = 0, const int32_t* expert_cap = nullptr,
                            unsigned long long* clk = nullptr);
cudaError_t launch_gather(const Problem& p, const void* x, const int32_t* perm, const int32_t* seg_off,
                          void* x_perm, cudaStream_t st, unsigned long long* clk = nullptr);

// dispatch.cu: rows of n_seg segments (segment s = source s / E, expert s % E)
// moved into expert-major order and back: segment_regroup_plan writes each
// segment's first row in expert-major order (dst_off [n_seg]) and the experts'
// offsets (expert_off [E + 1]); segment_copy copies rows src -> dst with
// to_expert (segment order -> expert-major) or back (expert-major -> segment order).
cudaError_t launch_segment_regroup_plan(const int32_t* seg_off, int n_seg, int E, int32_t* dst_off,
                                        int32_t* expert_off, cudaStream_t st);
cudaError_t launch_segment_copy(const void* src, void* dst, const int32_t* seg_off, const int32_t* dst_off, int n_seg,
                                int64_t n_rows, int row_bytes, bool to_expert, cudaStream_t st);

// balance.cu: selection-bias update and adaptive capacity from one step's
// counts (see moe_balance_update).  bias / caps may be nullptr.
cudaError_t launch_balance_update(const Problem& p, const int32_t* counts, float* bias, float rate, int mode,
                                  int32_t* hist, int hist_slot, int hist_rows, float c_base, float gamma,
                                  int32_t* caps, cudaStream_t st);

// router_fused.cu: gate GEMM (tcgen05, split-K over a thread-block cluster,
// partials summed through distributed shared memory); BF16, logits computed
// (router_fused_ok).  Writes the logits; with select (router_selects(p)) also
// ranks the tokens like route_select: topk_idx, topk_w, the chunk histogram
// and chunk p sums, and (zpart) *n_zpart z-loss partials, at most
// router_fused_zparts(p) <= ceil(T/128) * 8 of them.
bool router_fused_ok(const Problem& p);
bool router_selects(const Problem& p);
int router_fused_zparts(const Problem& p);
cudaError_t launch_router_fused(const Problem& p, const void* x, const void* w_gate, const float* offset,
                                const float* sel_bias, float* logits, int32_t* topk_idx, float* topk_w,
                                int32_t* chunk_counts, unsigned long long* chunk_psum, float* zpart,
                                unsigned* status, cudaStream_t st, int* n_zpart, unsigned long long* clk,
                                bool select);

// expert_gemm.cu -- returns a moe_status value
int router_k_splits(const Problem& p);  // slices of the tensor-core gate GEMM's reduction
int launch_gate_logits_tc(const Problem& p, const void* x, const void* w_gate, const float* offset, float* out,
                          int n_splits, unsigned* status, cudaStream_t st, unsigned long long* clk = nullptr);
int launch_expert_ffn(const Problem& p, int mode, const void* x_rows, int64_t n_rows, const int32_t* seg_off,
                      const void* w13, const void* w2, void* h, void* y_rows, unsigned* status,
                      cudaStream_t st, cudaEvent_t after_up = nullptr, int* n_kernels = nullptr,
                      void* gu = nullptr, unsigned long long* clk_up = nullptr,
                      unsigned long long* clk_down = nullptr, int n_seg = 0);
// (routed mode) n_seg > 0: seg_off has n_seg + 1 entries and row segment s is
// computed with expert s % p.E (moe_expert_ffn_segments).
// Routed (x_perm over seg_off, p.max_rows rows) and shared (x, T rows)
// experts in the same two launches, their tiles interleaved: requires
// expert_ffn_mixed_ok(p) (BF16, shared experts, both on the same tile shape:
// CTA pairs or single CTAs; MOE_B200_MIX_SHARED=0 turns it off).  gu / gu_shared: nullptr or the saved
// gate and up projections.
bool expert_ffn_mixed_ok(const Problem& p);
int launch_expert_ffn_mixed(const Problem& p, const void* x_perm, const int32_t* seg_off, const void* w13,
                            const void* w2, void* h, void* y_perm, void* gu, const void* x, const void* w13_shared,
                            const void* w2_shared, void* h_shared, void* y_shared, void* gu_shared, unsigned* status,
                            cudaStream_t st, cudaEvent_t after_up, int* n_kernels,
                            unsigned long long* clk_up = nullptr, unsigned long long* clk_down = nullptr);

// expert_gemm.cu: gu = x W13^T (gate | up projections, BF16) for the backward
int launch_up_projections(const Problem& p, int mode, const void* x_rows, int64_t n_rows, const int32_t* seg_off,
                          const void* w13, void* gu, unsigned* status, cudaStream_t st);
// grad_gemm.cu: backward of the expert FFNs (see there); returns a moe_status value
// gu_ready: gu already holds the forward's gate/up projections (no recompute)
// tail_a, tail_b: scratch of wgrad_tail_bytes each (the weight-gradient GEMMs'
// zero-padded last k-blocks)
int launch_expert_ffn_backward(const Problem& p, int mode, const void* x_rows, int64_t n_rows,
                               const int32_t* seg_off, const void* w13, const void* w2, const void* dout,
                               const void* h, void* gu, void* dgu, void* dx_rows, float* dw13, float* dw2,
                               void* tail_a, void* tail_b, unsigned* status, cudaStream_t st, bool gu_ready);
size_t wgrad_tail_bytes(const Problem& p, int e_pad);

// grad_gemm.cu: router gradients through the gate GEMM from dl [T, e_pad] BF16
int launch_router_dgrad(const Problem& p, const void* dl16, int e_pad, const void* w_gate, void* dx_r,
                        unsigned* status, cudaStream_t st);
int launch_router_wgrad(const Problem& p, const void* dl16, int e_pad, const void* x, float* dwg, void* tail_a,
                        void* tail_b, unsigned* status, cudaStream_t st);

// combine.cu
cudaError_t launch_combine(const Problem& p, const void* y_perm, const int32_t* slot_of, const float* topk_w,
                           const void* y_shared, void* y, cudaStream_t st, unsigned long long* clk = nullptr);

// device properties (cached per device)
int num_sms();

// moe_api.cu: the moe_status value reported for a CUDA error (MOE_OK for cudaSuccess)
int cuda_rc(cudaError_t e);

// moe_api.cu: test hook of the bounded-wait abort path.  MOE_B200_TEST_STALL_NS
// (read at every launch of the fused router and the single-CTA expert GEMM;
// unset or 0 normally) makes those kernels' MMA thread wait that long for a
// barrier phase that never completes, so the kernel records
// MOE_DEV_WAIT_TIMEOUT and returns through its abort path.
unsigned long long test_stall_ns();

}  // namespace moe
