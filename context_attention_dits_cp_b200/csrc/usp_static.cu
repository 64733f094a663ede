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
// current) on the first call made on that device; that first call should
// therefore happen before any stream capture.  No call here allocates or
// frees memory.  The workspace is written in full by the permutations
// before anything reads it, so nothing needs clearing between calls; but
// every call shares the one array, so calls whose GPU work overlaps (on
// different streams, or from different threads) race on it.

#include "internal.h"

namespace cpattn {
namespace {

static __device__ __align__(256) unsigned char g_usp_scratch[CP_USP_STATIC_SCRATCH_BYTES];

// Device address of g_usp_scratch on the current device (looked up once per
// device); NULL with *status set if the runtime refuses.
void* usp_scratch_address(int* status) {
  static void* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *status = CP_ERR_CUDA;
    return nullptr;
  }
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_usp_scratch) != cudaSuccess || p == nullptr) {
      *status = CP_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace
}  // namespace cpattn

extern "C" int cp_usp_attention_static(const cp_tensor* q_shards, const cp_tensor* k_shards,
                                       const cp_tensor* v_shards, int ring_degree,
                                       int ulysses_degree, float scale, cp_tensor* out_shards,
                                       cp_tensor* lse, void* stream) {
  if (!q_shards || !out_shards) return CP_ERR_NULL;
  if (q_shards->ndim != 5) return CP_ERR_SHAPE;
  const int64_t G = q_shards->shape[0], B = q_shards->shape[1], Sg = q_shards->shape[2],
                H = q_shards->shape[3], D = q_shards->shape[4];
  if (G < 0 || B < 0 || Sg < 0 || H < 0 || D < 0) return CP_ERR_SHAPE;
  const size_t need = cp_usp_workspace_bytes(B, Sg * G, H, D, q_shards->dtype,
                                             out_shards->dtype, ring_degree, ulysses_degree);
  if (need > (size_t)CP_USP_STATIC_SCRATCH_BYTES) return CP_ERR_WORKSPACE;
  int st = CP_OK;
  void* ws = cpattn::usp_scratch_address(&st);
  if (!ws) return st;
  return cp_usp_attention(q_shards, k_shards, v_shards, ring_degree, ulysses_degree, scale, ws,
                          (size_t)CP_USP_STATIC_SCRATCH_BYTES, out_shards, lse, stream);
}
