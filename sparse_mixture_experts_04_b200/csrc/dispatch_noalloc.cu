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
// device (with the device current); make that first call before any stream
// capture begins.  Expert indices outside [0, E) are skipped (their slot is
// -1) but, with no workspace, not reported.  The pages have no counterpart of
// this entry point: it only changes where scratch memory comes from.
#include <mutex>

#include "../../include/moe_b200.h"
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr size_t kNoAllocScratchWords = 262144;  // 1 MiB

static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocScratchWords];

// Device address of g_noalloc_scratch on the current device (looked up once per
// device).  In host code the array's name is only a host-side handle, never a
// device pointer, so kernels get this address instead.
static int32_t* noalloc_scratch(int* rc) {
  static std::mutex mu;
  static int32_t* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *rc = MOE_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      *rc = MOE_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = static_cast<int32_t*>(p);
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
  if (launch_dispatch(p, topk_idx, counts, kept, seg_off, slot_of, perm, chunk_counts, chunk_base,
                      /*status=*/nullptr, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (x_perm && launch_gather(p, x, perm, seg_off, x_perm, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}
