// Device helpers shared by the kernels of libmoe_b200: status word, vector
// types, and thin inline-PTX wrappers for the sm_100a features the expert GEMM
// uses (mbarrier, TMA tensor copies, tcgen05 MMA / TMEM).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// BF16 TMA tensor map (host): dims[0] innermost, 128-byte swizzle, box inner
// extent 64 elements, zero fill out of bounds (expert_gemm.cu).
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint32_t* box);
// Same with explicit byte strides for dims 1..rank-1 (dim 0 contiguous).
bool make_map_strided(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
                      const uint32_t* box);

// Status bits written into the first word of the caller's workspace.
constexpr unsigned kDevBadExpert = 0x1u;
constexpr unsigned kDevWaitTimeout = 0x2u;

// A pipeline wait gives up after this long (then the kernel records
// kDevWaitTimeout, drains what it started and returns).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ void raise_status(unsigned* status, unsigned bit) {
  if (status) atomicOr(status, bit);
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase of `bar` with the given parity has completed.  Bounded:
// gives up when `abort` is raised by another role, or after limit_ns (then
// raises `abort` itself).  Returns false when it gave up.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, volatile int* abort,
                                              unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 31u) == 0) {
      if (*abort) return false;
      if (global_ns() - t0 > limit_ns) {
        *abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return mbar_wait_for(bar, parity, abort, kWaitLimitNs);
}

// Test hook of the bounded-wait abort path (stall_ns > 0, see
// test_stall_ns() in internal.h): the MMA-issuing thread first waits for a
// barrier phase that nothing completes (`bar`'s first phase, before anything
// arrives on it), gives up after stall_ns, raises `abort`, and the kernel then
// takes its abort path: every role drains what it started and returns.
__device__ __forceinline__ bool test_stall(uint64_t* bar, volatile int* abort, unsigned long long stall_ns) {
  return stall_ns == 0 || mbar_wait_for(bar, 0, abort, stall_ns);
}

// -------------------------------------------------------------- TMA copies
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------- tcgen05 / TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (BF16 inputs, FP32 accumulate).
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(bar))
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets row
// (lane base + i), columns [col, col+32).
__device__ __forceinline__ void tmem_load_32x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Barrier among `threads` threads (whole warps) of the CTA on hardware barrier
// `id` (1..15; 0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy reads of them (tcgen05.mma operands).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// named_bar_sync that also ANDs one predicate over the participating threads.
__device__ __forceinline__ bool named_bar_and(int id, int threads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void tmem_load_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor for a K-major BF16 tile whose rows are 128
// bytes (64 elements) written by TMA with 128-byte swizzling: 8-row groups
// 1024 bytes apart.  Tile base must be 1024-byte aligned.
__device__ __forceinline__ uint64_t smem_desc_k128(uint32_t saddr) {
  uint64_t desc = 0;
  desc |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);  // start address
  desc |= static_cast<uint64_t>(1) << 16;                  // leading byte offset (unused here)
  desc |= static_cast<uint64_t>(1024 >> 4) << 32;          // stride byte offset: 8 rows x 128 B
  desc |= static_cast<uint64_t>(1) << 46;                  // descriptor version (sm_100)
  desc |= static_cast<uint64_t>(2) << 61;                  // 128-byte swizzle
  return desc;
}

// Shared-memory matrix descriptor, MN-major operand with 128-byte swizzle: rows
// of 64 MN-elements (128 B) per K index, 8 K rows per 1024-byte atom.
//   lbo: bytes between consecutive 64-element MN chunks
//   sbo: bytes between consecutive groups of 8 K rows (1024 when the K rows
//        of a chunk are contiguous)
__device__ __forceinline__ uint64_t smem_desc_mn128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t desc = 0;
  desc |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  desc |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  desc |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  desc |= static_cast<uint64_t>(1) << 46;
  desc |= static_cast<uint64_t>(2) << 61;
  return desc;
}

// Instruction descriptor: BF16 x BF16 -> FP32, M x N; a_mn / b_mn select the
// MN-major ("transposed") layout for A / B (bits 15 / 16), else K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32_major(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn ? (1u << 15) : 0u) | (b_mn ? (1u << 16) : 0u) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor: BF16 x BF16 -> FP32, both operands K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                                   // D format FP32
         | (1u << 7)                                 // A format BF16
         | (1u << 10)                                // B format BF16
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// ------------------------------------------------- CTA pairs (cluster of 2)
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

// All threads of every CTA in the cluster (release / acquire).  Not the
// .aligned form: threads of one warp may reach it from different branches.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Arrive on an mbarrier given by its shared::cluster address (possibly in the peer CTA).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA loads of a CTA pair: the destination is this CTA's shared memory, the
// completion is signalled on the mbarrier at `bar_cluster` (the leader CTA's).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5, %6}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// M=256 MMA over the CTA pair: A rows 0-127 / 128-255 and B rows 0..N/2-1 /
// N/2..N-1 from the leader / peer CTA's shared memory (same offsets); D rows
// 0-127 / 128-255 land in the leader / peer CTA's TMEM.  Issued by the leader.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on the mbarrier at this shared-memory offset in every CTA of
// `cta_mask` once the pair MMAs issued so far by this thread completed.
__device__ __forceinline__ void umma_commit_pair_multicast(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_addr(bar)),
      "h"(cta_mask)
      : "memory");
}

// ------------------------------------------- balance statistics (shared)
// Per-expert probability sums travel as unsigned fixed-point integers (exact,
// order-independent integer adds).  Scale 2^s with s = min(40, 62 - ceil(log2 T))
// keeps T tokens' sum (each p <= 1) below 2^62; resolution 2^-s per token.
__host__ __device__ inline double p_fixed_scale(int64_t T) {
  int bits = 0;
  while ((static_cast<int64_t>(1) << bits) < T) ++bits;
  int s = 62 - bits;
  if (s > 40) s = 40;
  return static_cast<double>(static_cast<int64_t>(1) << s);
}

// Writes f_e and P_e of expert e into stats and returns f_e * P_e.
__device__ __forceinline__ double balance_stats_expert(long long count, unsigned long long psum_fixed, int64_t T,
                                                       int E, int K, int e, float* stats) {
  const double f = static_cast<double>(count) / (static_cast<double>(T) * K);
  const double P = static_cast<double>(psum_fixed) / p_fixed_scale(T) / static_cast<double>(T);
  stats[e] = static_cast<float>(f);
  stats[E + e] = static_cast<float>(P);
  return f * P;
}

// loss = alpha * E * sum_e f_e P_e, summed in expert order (one thread).
__device__ __forceinline__ void balance_loss(const double* fp, int E, float alpha, float* stats) {
  double acc = 0.0;
  for (int e = 0; e < E; ++e) acc += fp[e];
  stats[2 * E] = static_cast<float>(static_cast<double>(alpha) * E * acc);
}

// ----------------------------------------------------------- stage clocks
// moe_layer_forward_clocked: each kernel of a stage raises clk[0] to the
// bitwise complement of its start and clk[1] to its end (ns of the global
// timer), so a zero-filled pair ends up holding the stage's earliest start
// (complemented) and latest end whatever the order of the CTAs.  Thread 0 of
// every CTA stamps: the start once the predecessor's outputs may be read
// (after pdl_wait), the end after the CTA's last barrier.
__device__ __forceinline__ void stage_clock_start(unsigned long long* clk) {
  if (clk && threadIdx.x == 0) atomicMax(clk, ~global_ns());
}
__device__ __forceinline__ void stage_clock_end(unsigned long long* clk) {
  if (clk && threadIdx.x == 0) atomicMax(clk + 1, global_ns());
}

// ------------------------------------------- programmatic dependent launch
// Kernels of one forward are launched with programmatic stream serialisation:
// a kernel may be scheduled while its predecessor on the stream is finishing.
// Every kernel calls pdl_wait() before it reads anything the predecessor wrote
// (and every kernel calls it, so completion stays transitive along the
// stream), and pdl_trigger() once it no longer needs to hold back its
// successor's launch.  Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

bool pdl_enabled();  // MOE_B200_PDL=0 turns the attribute off (moe_api.cu)

template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                            Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Extended statistics (written after the 2E+1 balance entries when requested):
//   stats[2E+1] router z-loss  (1/T) sum_t (logsumexp_t)^2   (from zsum = sum of the squares)
//   stats[2E+2] entropy in bits of the load shares counts_e / sum(counts)
//   stats[2E+3] coefficient of variation of counts (population std / mean)
//   stats[2E+4] drop rate: sum(counts - kept) / sum(counts)
//   stats[2E+5] experts below 50% of the mean load; stats[2E+6] above 200%
// counts / kept are read from shared or global memory; one thread, expert order.
constexpr int kExtendedStats = 6;

__device__ __forceinline__ void utilisation_stats(const int* counts, const int* kept, int E, int64_t T,
                                                  double zsum, float* stats) {
  double n = 0.0, dropped = 0.0;
  for (int e = 0; e < E; ++e) {
    n += counts[e];
    dropped += static_cast<double>(counts[e] - kept[e]);
  }
  const double mean = n / E;
  double ent = 0.0, var = 0.0, below = 0.0, above = 0.0;
  for (int e = 0; e < E; ++e) {
    if (counts[e] > 0) {
      const double q = counts[e] / n;
      ent -= q * log2(q);
    }
    const double dv = counts[e] - mean;
    var += dv * dv;
    if (counts[e] < 0.5 * mean) below += 1.0;
    if (counts[e] > 2.0 * mean) above += 1.0;
  }
  var /= E;
  float* x = stats + 2 * E + 1;
  x[0] = static_cast<float>(zsum / static_cast<double>(T));
  x[1] = static_cast<float>(ent);
  x[2] = static_cast<float>(mean > 0.0 ? sqrt(var) / mean : 0.0);
  x[3] = static_cast<float>(n > 0.0 ? dropped / n : 0.0);
  x[4] = static_cast<float>(below);
  x[5] = static_cast<float>(above);
}

// ------------------------------------------------------------------ misc
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace moe
