// cp_usp_attention_static: the unified (Ulysses x Ring) attention for
// callers that cannot allocate device memory.
//
// cp_usp_attention needs a workspace for the head-sharded copies of q, k, v
// and of the output.  Some callers have no way to provide one: a plugin
// running inside another engine's enqueue/execute hook (where allocating
// would synchronise the device and is forbidden by the host engine), code
// whose device memory is owned entirely by a foreign pool it cannot draw
// from, or a plain-C host program that links this library but no CUDA
// allocator.  This entry point takes its workspace from a fixed array that
// lives in this file instead.
//
// The array is a file-scope __device__ object: every GPU that loads this
// module holds CP_USP_STATIC_SCRATCH_BYTES of it until the process exits.
// In host code its name is only a host-side handle, so its device address is
// looked up once per device with cudaGetSymbolAddress (with that device
// current) on the first call made on that device.  With CUDA's lazy module
// loading that first lookup is also what loads this module and reserves the
// array, and it may synchronise the device; so make the first call on each
// device outside any stream capture or latency-critical hook.  Any call that
// passes the argument and size checks does the set-up, including one with an
// empty problem (B = 0), which launches nothing.  No call here allocates or frees
// memory.  The workspace is written in full by the permutations before
// anything reads it, so nothing needs clearing between calls; but every call
// shares the one array, so calls whose GPU work overlaps (on different
// streams, or from different threads) race on it.

#include <atomic>

#include "internal.h"

namespace cpattn {
namespace {

static __device__ __align__(256) unsigned char g_usp_scratch[CP_USP_STATIC_SCRATCH_BYTES];

// Device address of g_usp_scratch on the current device (looked up once per
// device; concurrent first calls may each look it up and store the same
// value); NULL with *status set if the runtime refuses.
void* usp_scratch_address(int* status) {
  static std::atomic<void*> addr[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *status = CP_ERR_CUDA;
    return nullptr;
  }
  void* a = addr[dev].load(std::memory_order_acquire);
  if (!a) {
    if (cudaGetSymbolAddress(&a, g_usp_scratch) != cudaSuccess || a == nullptr) {
      *status = CP_ERR_CUDA;
      return nullptr;
    }
    addr[dev].store(a, std::memory_order_release);
  }
  return a;
}

}  // namespace
}  // namespace cpattn

extern "C" int cp_usp_attention_static(const cp_tensor* q_shards, const cp_tensor* k_shards,
                                       const cp_tensor* v_shards, int ring_degree,
                                       int ulysses_degree, float scale, cp_tensor* out_shards,
                                       cp_tensor* lse, void* stream) {
  int st = cpattn::usp_check_args(q_shards, k_shards, v_shards, ring_degree, ulysses_degree,
                                  out_shards, lse);
  if (st != CP_OK) return st;
  const int64_t G = q_shards->shape[0], B = q_shards->shape[1], Sg = q_shards->shape[2],
                H = q_shards->shape[3], D = q_shards->shape[4];
  const size_t need = cp_usp_workspace_bytes(B, Sg * G, H, D, q_shards->dtype,
                                             out_shards->dtype, ring_degree, ulysses_degree);
  if (need > (size_t)CP_USP_STATIC_SCRATCH_BYTES) return CP_ERR_WORKSPACE;
  void* ws = cpattn::usp_scratch_address(&st);
  if (!ws) return st;
  return cp_usp_attention(q_shards, k_shards, v_shards, ring_degree, ulysses_degree, scale, ws,
                          (size_t)CP_USP_STATIC_SCRATCH_BYTES, out_shards, lse, stream);
}
