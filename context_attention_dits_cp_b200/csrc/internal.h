// Host-side glue shared by the C-ABI (api.cu) and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "cpattn.h"

namespace cpattn {

// A validated tensor: pointer, dtype and up to 6 sizes/strides in elements.
struct TensorView {
  void* data = nullptr;
  int dtype = CP_F32;
  int ndim = 0;
  int64_t shape[CP_MAX_DIMS] = {0, 0, 0, 0, 0, 0};
  int64_t stride[CP_MAX_DIMS] = {0, 0, 0, 0, 0, 0};
};

inline TensorView view_of(const cp_tensor* t) {
  TensorView v;
  if (!t) return v;
  v.data = t->data;
  v.dtype = t->dtype;
  v.ndim = t->ndim;
  for (int i = 0; i < CP_MAX_DIMS; ++i) {
    v.shape[i] = t->shape[i];
    v.stride[i] = t->stride[i];
  }
  return v;
}

inline int dtype_size(int dt) { return dt == CP_BF16 ? 2 : 4; }

// Elements from a view's first to its last element, plus one (0 when it is
// empty or has no data): every valid offset lies in [0, span).  The
// device-side bounds checks of debug builds test offsets against it.
inline long long span_elems(const TensorView& t) {
  if (!t.data) return 0;
  long long span = 1;
  for (int i = 0; i < t.ndim; ++i) {
    if (t.shape[i] == 0) return 0;
    span += (t.shape[i] - 1) * t.stride[i];
  }
  return span;
}

// Attention over a chunk list (one chunk = cp_attn_partial).
struct RingArgs {
  TensorView q, k, v;      // [B, S, H, D]; k, v may be [G, B, L, H, D] (token s = row s % L of slot s / L)
  TensorView out;          // [B, S_q, H, D] f32 or bf16
  TensorView lse;          // [B, H, S_q] f32; data may be null
  const int64_t* chunk_off = nullptr;   // host, n_chunks + 1: chunk starts (key tokens)
  const int64_t* chunk_end = nullptr;   // host, n_chunks chunk ends; null: chunk_off[c + 1]
  int n_chunks = 0;
  float scale = 0.f;
  bool merge = false;      // fold into (out, lse) with the fp32 LSE merge
  int* dev_err = nullptr;
};

int launch_attn_ring_tc(const RingArgs& a, cudaStream_t stream);    // bf16, tensor cores
int launch_attn_ring_f32(const RingArgs& a, cudaStream_t stream);   // f32, FFMA
int launch_fill_empty(const TensorView& out, const TensorView& lse, int* dev_err,
                      cudaStream_t stream);
int launch_lse_merge(const TensorView& out_acc, const TensorView& lse_acc,
                     const TensorView& out_i, const TensorView& lse_i, int* dev_err,
                     cudaStream_t stream);
int launch_ulysses_permute(const TensorView& x, const TensorView& y, int degree, int dir,
                           int* dev_err, cudaStream_t stream);
int launch_ulysses_anything_permute(const TensorView& x, const TensorView& y, int64_t B,
                                    int64_t H, int64_t D, int U, const int64_t* seq_off,
                                    const int64_t* head_off, int dir, int* dev_err,
                                    cudaStream_t stream);
int launch_wait_timeout_selftest(int spin_limit, int* dev_err, cudaStream_t stream);
int launch_bounds_selftest(int* dev_err, cudaStream_t stream);

// Argument checks of cp_usp_attention (everything but the workspace), shared
// with cp_usp_attention_static so both report the same error codes.
int usp_check_args(const cp_tensor* qs, const cp_tensor* ks, const cp_tensor* vs,
                   int ring_degree, int ulysses_degree, const cp_tensor* outs,
                   const cp_tensor* lse);

}  // namespace cpattn
