// moe_dispatch_noalloc: moe_dispatch for callers that cannot hand the library
// device memory for scratch.
//
// Some callers cannot allocate: a program whose device-memory budget is fixed
// before it starts (every byte is already owned by its own pool or planner),
// or a host without a caching allocator, for which a cudaMalloc / cudaFree
// around every call would synchronise the device and fragment memory.  This
// entry point takes only the inputs and outputs of moe_dispatch; its scratch
// (the per-chunk expert histogram and the chunk bases) lives in a fixed array
// in device memory that the library itself declares.
//
// The array belongs to the library: every GPU that loads the library holds it
// (kNoAllocScratchWords 32-bit words = 1 MiB) until the process exits, and all
// calls on that GPU share it.  Two calls whose work overlaps on the GPU (for
// example on two streams) therefore race; serialise them.  A problem needs
// 2 * ceil(T / 256) * E words; larger problems are rejected with
// MOE_ERR_UNSUPPORTED before anything is enqueued.
//
// The first call on a device looks up the array's device address for that
// device (with the device current), and so does the first call after the
// device's context was reset; make that first call before any stream capture
// begins.  Expert indices outside [0, E) are skipped (their slot is
// -1) but, with no workspace, not reported.  The pages have no counterpart of
// this entry point: it only changes where scratch memory comes from.
#include <mutex>

#include "../../include/moe_b200.h"
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr size_t kNoAllocScratchWords = 262144;  // 1 MiB

static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocScratchWords];

// Device address of g_noalloc_scratch in the current context.  In host code
// the array's name is only a host-side handle, never a device pointer, so
// kernels get this address instead.  The address is looked up once per
// context, keyed by the context's unique ID: after cudaDeviceReset (or any
// other release of the primary context) the module is loaded again, possibly
// elsewhere, and the next call looks the address up afresh.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

static bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

static int32_t* noalloc_scratch(int* rc) {
  static std::mutex mu;
  static unsigned long long ctx_of[64] = {0};
  static int32_t* addr[64] = {nullptr};
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev)) {
    *rc = cuda_rc(e);
    return nullptr;
  }
  if (dev < 0 || dev >= 64) {
    *rc = MOE_ERR_UNSUPPORTED;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx);
  if (!addr[dev] || !have_ctx || ctx != ctx_of[dev]) {
    void* p = nullptr;
    // makes the device's primary context current if no context was yet
    if (cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch)) {
      *rc = cuda_rc(e);
      return nullptr;
    }
    if (!p || !current_context_id(&ctx)) {
      *rc = MOE_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = static_cast<int32_t*>(p);
    ctx_of[dev] = ctx;
  }
  *rc = MOE_OK;
  return addr[dev];
}

}  // namespace moe

using namespace moe;

extern "C" int moe_dispatch_noalloc(const moe_problem_t* q, const int32_t* topk_idx, const void* x, int32_t* counts,
                                    int32_t* kept, int32_t* seg_off, int32_t* slot_of, int32_t* perm,
                                    void* x_perm, moe_stream_t stream) {
  Problem p;
  if (int rc = problem_from_abi(q, &p)) return rc;
  if (p.flags & MOE_FLAG_EXPERT_CAPACITY) return MOE_ERR_INVALID_ARG;
  if (!topk_idx || !counts || !kept || !seg_off || !slot_of || !perm) return MOE_ERR_INVALID_ARG;
  if (x_perm && (!x || (reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(x_perm) & 15u)))
    return MOE_ERR_INVALID_ARG;
  const size_t n_chunks = static_cast<size_t>((p.T + kDispatchChunk - 1) / kDispatchChunk);
  const size_t words = 2 * n_chunks * static_cast<size_t>(p.E);
  if (words > kNoAllocScratchWords) return MOE_ERR_UNSUPPORTED;
  int rc = MOE_OK;
  int32_t* scratch = noalloc_scratch(&rc);
  if (rc) return rc;
  // chunk histogram and chunk bases; both are fully written by the kernels
  // before they are read, so the previous call's contents need no clearing
  int32_t* chunk_counts = scratch;
  int32_t* chunk_base = scratch + n_chunks * p.E;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaError_t e = launch_dispatch(p, topk_idx, counts, kept, seg_off, slot_of, perm, chunk_counts, chunk_base,
                                      /*status=*/nullptr, st))
    return cuda_rc(e);
  if (x_perm) {
    if (cudaError_t e = launch_gather(p, x, perm, seg_off, x_perm, st)) return cuda_rc(e);
  }
  return MOE_OK;
}
