// The C-ABI of libcpattn: argument validation, dispatch and the composite
// (unified sequence parallelism) call.  Declarations and the contract of
// every entry point are in include/cpattn.h.

#include <cmath>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace cpattn {

// One error word per device (a __device__ variable exists once per device
// the library's module is loaded on); kernels get its address.
__device__ int g_device_error_word = 0;

namespace {

int* device_error_ptr() {
  static int* ptrs[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Byte range [lo, hi) a tensor's elements can touch.
void byte_range(const TensorView& t, uintptr_t* lo, uintptr_t* hi) {
  long long span = 0;
  bool empty = false;
  for (int i = 0; i < t.ndim; ++i) {
    if (t.shape[i] == 0) empty = true;
    span += (t.shape[i] - 1) * (t.stride[i] < 0 ? -t.stride[i] : t.stride[i]);
  }
  *lo = reinterpret_cast<uintptr_t>(t.data);
  *hi = empty ? *lo : *lo + (uintptr_t)((span + 1) * dtype_size(t.dtype));
}

bool overlaps(const TensorView& a, const TensorView& b) {
  uintptr_t a0, a1, b0, b1;
  byte_range(a, &a0, &a1);
  byte_range(b, &b0, &b1);
  if (a0 == a1 || b0 == b1) return false;
  return a0 < b1 && b0 < a1;
}

// A tensor with no elements may carry a NULL pointer; it is never read.
int check_basic(const cp_tensor* t, int ndim) {
  if (!t) return CP_ERR_NULL;
  if (t->ndim != ndim) return CP_ERR_SHAPE;
  if (t->dtype != CP_F32 && t->dtype != CP_BF16) return CP_ERR_DTYPE;
  bool empty = false;
  for (int i = 0; i < ndim; ++i) {
    if (t->shape[i] < 0 || t->shape[i] > 0x7fffffffLL) return CP_ERR_SHAPE;
    if (t->stride[i] < 0) return CP_ERR_ALIGN;
    if (t->shape[i] == 0) empty = true;
  }
  if (!t->data && !empty) return CP_ERR_NULL;
  return CP_OK;
}

// An output must not map two of its elements to one address (a zero stride,
// or dims that interleave): the kernels would race on it.  Sufficient test:
// with the dims of extent > 1 ordered by stride, each stride is at least the
// span of the dims below it.
bool self_overlapping(const cp_tensor* t) {
  int64_t st[CP_MAX_DIMS], sh[CP_MAX_DIMS];
  int n = 0;
  for (int i = 0; i < t->ndim; ++i) {
    if (t->shape[i] <= 1) continue;
    if (t->stride[i] == 0) return true;
    int j = n++;
    for (; j > 0 && st[j - 1] > t->stride[i]; --j) {
      st[j] = st[j - 1];
      sh[j] = sh[j - 1];
    }
    st[j] = t->stride[i];
    sh[j] = t->shape[i];
  }
  for (int k = 0; k + 1 < n; ++k)
    if (st[k + 1] < st[k] * sh[k]) return true;
  return false;
}

// Element-stride / base alignment to `bytes` for every dim but the last,
// which must be contiguous.
int check_vector_layout(const cp_tensor* t, int bytes) {
  const int es = dtype_size(t->dtype);
  if (t->stride[t->ndim - 1] != 1 && t->shape[t->ndim - 1] > 1) return CP_ERR_ALIGN;
  if (reinterpret_cast<uintptr_t>(t->data) % bytes) return CP_ERR_ALIGN;
  for (int i = 0; i < t->ndim - 1; ++i)
    if ((t->stride[i] * es) % bytes) return CP_ERR_ALIGN;
  return CP_OK;
}

float resolve_scale(float scale, int64_t D) {
  if (scale == 0.f || std::isnan(scale)) return 1.0f / std::sqrt((float)D);
  return scale;
}

// The unified composition folds its permutations into the attention
// kernel's tensor maps (one launch, no intermediates) for bf16 inputs when
// every 128-row tile lies inside one sequence shard.
bool usp_fusable_sizes(int in_dtype, int64_t D, int64_t G, int64_t Sg) {
  return in_dtype == CP_BF16 && (D == 64 || D == 128) && (G == 1 || Sg % 128 == 0);
}

// Workspace of the unfused composition: head-sharded q, k, v and output,
// each [U, B, S, H/U, D], 256-byte aligned.
size_t usp_unfused_bytes(int64_t B, int64_t S, int64_t H, int64_t D, int in_dtype,
                         int out_dtype) {
  const size_t n = (size_t)B * S * H * D;
  auto rnd = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return 3 * rnd(n * dtype_size(in_dtype)) + rnd(n * dtype_size(out_dtype));
}

// Shared validation of attention arguments.  On success fills `a` (without
// chunk offsets) and reports whether there is anything to compute.
// K/V are [B, S_kv, H, D], or with kv_ndim 5 the slots [G, B, L, H, D] of a
// padded all-gather (token s = row s % L of slot s / L).
int prepare_attention(const cp_tensor* q, const cp_tensor* k, const cp_tensor* v, float scale,
                      const cp_tensor* out, const cp_tensor* lse, bool lse_optional,
                      RingArgs* a, int kv_ndim = 4) {
  int st;
  if ((st = check_basic(q, 4)) || (st = check_basic(k, kv_ndim)) ||
      (st = check_basic(v, kv_ndim)) || (st = check_basic(out, 4)))
    return st;
  if (!lse_optional || lse) {
    if ((st = check_basic(lse, 3))) return st;
    if (lse->dtype != CP_F32) return CP_ERR_DTYPE;
  }
  if (q->dtype != k->dtype || q->dtype != v->dtype) return CP_ERR_DTYPE;
  if (self_overlapping(out) || (lse && self_overlapping(lse))) return CP_ERR_ALIAS;
  const int64_t B = q->shape[0], Sq = q->shape[1], H = q->shape[2], D = q->shape[3];
  if (D != 64 && D != 128) return CP_ERR_SHAPE;
  const int kb = kv_ndim - 4;   // index of the batch dim of k / v
  if (k->shape[kb] != B || k->shape[kb + 2] != H || k->shape[kb + 3] != D) return CP_ERR_SHAPE;
  for (int i = 0; i < kv_ndim; ++i)
    if (v->shape[i] != k->shape[i]) return CP_ERR_SHAPE;
  for (int i = 0; i < 4; ++i)
    if (out->shape[i] != q->shape[i]) return CP_ERR_SHAPE;
  if (lse && (lse->shape[0] != B || lse->shape[1] != H || lse->shape[2] != Sq))
    return CP_ERR_SHAPE;
  if (B * H * ((Sq + 255) / 256) > 0x7fffffffLL) return CP_ERR_SHAPE;
  // q/k/v: the tensor-core path reads through TMA (16-byte base and strides)
  if (q->dtype == CP_BF16) {
    if ((st = check_vector_layout(q, 16)) || (st = check_vector_layout(k, 16)) ||
        (st = check_vector_layout(v, 16)))
      return st;
  } else {
    if ((st = check_vector_layout(q, 4)) || (st = check_vector_layout(k, 4)) ||
        (st = check_vector_layout(v, 4)))
      return st;
  }
  // out rows are written with 16-byte vector stores
  if ((st = check_vector_layout(out, 16))) return st;
  a->q = view_of(q);
  a->k = view_of(k);
  a->v = view_of(v);
  a->out = view_of(out);
  a->lse = view_of(lse);
  if (overlaps(a->out, a->q) || overlaps(a->out, a->k) || overlaps(a->out, a->v))
    return CP_ERR_ALIAS;
  if (lse && (overlaps(a->lse, a->q) || overlaps(a->lse, a->k) || overlaps(a->lse, a->v) ||
              overlaps(a->lse, a->out)))
    return CP_ERR_ALIAS;
  a->scale = resolve_scale(scale, D);
  return CP_OK;
}

int run_attention(RingArgs& a, cudaStream_t stream) {
  if (a.q.shape[1] == 0 || a.q.shape[0] == 0 || a.q.shape[2] == 0) return CP_OK;
  a.dev_err = device_error_ptr();
  if (!a.dev_err) return CP_ERR_CUDA;
  int64_t total = 0;
  for (int c = 0; c < a.n_chunks; ++c) {
    const int64_t len = (a.chunk_end ? a.chunk_end[c] : a.chunk_off[c + 1]) - a.chunk_off[c];
    if (len > 0) total += len;
  }
  if (total == 0) return a.merge ? CP_OK : launch_fill_empty(a.out, a.lse, a.dev_err, stream);
  if (a.q.dtype == CP_BF16) return launch_attn_ring_tc(a, stream);
  return launch_attn_ring_f32(a, stream);
}

int ring_impl(const cp_tensor* q, const cp_tensor* k, const cp_tensor* v,
              const int64_t* chunk_offsets, int n_chunks, float scale, cp_tensor* out,
              cp_tensor* lse, void* stream) {
  RingArgs a;
  int st = prepare_attention(q, k, v, scale, out, lse, true, &a);
  if (st) return st;
  if (!chunk_offsets) return CP_ERR_NULL;
  if (n_chunks < 1 || n_chunks > CP_MAX_CHUNKS) return CP_ERR_OFFSETS;
  if (chunk_offsets[0] != 0 || chunk_offsets[n_chunks] != k->shape[1]) return CP_ERR_OFFSETS;
  for (int c = 0; c < n_chunks; ++c)
    if (chunk_offsets[c + 1] < chunk_offsets[c]) return CP_ERR_OFFSETS;
  a.chunk_off = chunk_offsets;
  a.n_chunks = n_chunks;
  return run_attention(a, as_stream(stream));
}

}  // namespace
}  // namespace cpattn

using namespace cpattn;

extern "C" {

int cp_attn_partial(const cp_tensor* q, const cp_tensor* k_chunk, const cp_tensor* v_chunk,
                    float scale, cp_tensor* out, cp_tensor* lse, void* stream) {
  RingArgs a;
  int st = prepare_attention(q, k_chunk, v_chunk, scale, out, lse, false, &a);
  if (st) return st;
  const int64_t offs[2] = {0, k_chunk->shape[1]};
  a.chunk_off = offs;
  a.n_chunks = 1;
  return run_attention(a, as_stream(stream));
}

int cp_attn_partial_merge(const cp_tensor* q, const cp_tensor* k_chunk,
                          const cp_tensor* v_chunk, float scale, cp_tensor* out_acc,
                          cp_tensor* lse_acc, void* stream) {
  RingArgs a;
  int st = prepare_attention(q, k_chunk, v_chunk, scale, out_acc, lse_acc, false, &a);
  if (st) return st;
  if (out_acc->dtype != CP_F32) return CP_ERR_DTYPE;   // the accumulator is fp32
  if (k_chunk->shape[1] == 0) return CP_OK;           // an empty chunk merges as identity
  const int64_t offs[2] = {0, k_chunk->shape[1]};
  a.chunk_off = offs;
  a.n_chunks = 1;
  a.merge = true;
  return run_attention(a, as_stream(stream));
}

int cp_ring_attention(const cp_tensor* q, const cp_tensor* k, const cp_tensor* v,
                      const int64_t* chunk_offsets, int n_chunks, float scale, cp_tensor* out,
                      cp_tensor* lse, void* stream) {
  return ring_impl(q, k, v, chunk_offsets, n_chunks, scale, out, lse, stream);
}

int cp_lse_merge(cp_tensor* out_acc, cp_tensor* lse_acc, const cp_tensor* out_i,
                 const cp_tensor* lse_i, void* stream) {
  int st;
  if ((st = check_basic(out_acc, 4)) || (st = check_basic(lse_acc, 3)) ||
      (st = check_basic(out_i, 4)) || (st = check_basic(lse_i, 3)))
    return st;
  if (out_acc->dtype != CP_F32 || lse_acc->dtype != CP_F32 || lse_i->dtype != CP_F32)
    return CP_ERR_DTYPE;
  const int64_t B = out_acc->shape[0], S = out_acc->shape[1], H = out_acc->shape[2],
                D = out_acc->shape[3];
  if (D != 64 && D != 128) return CP_ERR_SHAPE;
  for (int i = 0; i < 4; ++i)
    if (out_i->shape[i] != out_acc->shape[i]) return CP_ERR_SHAPE;
  const int64_t want[3] = {B, H, S};
  for (int i = 0; i < 3; ++i)
    if (lse_acc->shape[i] != want[i] || lse_i->shape[i] != want[i]) return CP_ERR_SHAPE;
  // one lane moves D/32 consecutive elements with a single vector access
  const int lane_bytes_acc = (int)(D / 32) * 4;
  const int lane_bytes_in = (int)(D / 32) * dtype_size(out_i->dtype);
  if ((st = check_vector_layout(out_acc, lane_bytes_acc)) ||
      (st = check_vector_layout(out_i, lane_bytes_in)))
    return st;
  if ((st = check_vector_layout(lse_acc, 4)) || (st = check_vector_layout(lse_i, 4))) {
    // lse may be strided in any dim; only natural alignment is needed
    if (reinterpret_cast<uintptr_t>(lse_acc->data) % 4 ||
        reinterpret_cast<uintptr_t>(lse_i->data) % 4)
      return CP_ERR_ALIGN;
  }
  if (self_overlapping(out_acc) || self_overlapping(lse_acc)) return CP_ERR_ALIAS;
  const TensorView va = view_of(out_acc), vla = view_of(lse_acc), vi = view_of(out_i),
                   vli = view_of(lse_i);
  if (overlaps(va, vi) || overlaps(va, vla) || overlaps(va, vli) || overlaps(vla, vi) ||
      overlaps(vla, vli))
    return CP_ERR_ALIAS;
  if (B == 0 || S == 0 || H == 0) return CP_OK;
  int* err = device_error_ptr();
  if (!err) return CP_ERR_CUDA;
  return launch_lse_merge(va, vla, vi, vli, err, as_stream(stream));
}

int cp_ring_attention_gathered(const cp_tensor* q, const cp_tensor* k_gathered,
                               const cp_tensor* v_gathered, const int64_t* chunk_lengths,
                               int n_chunks, int skip_chunk, float scale, int accumulate,
                               cp_tensor* out, cp_tensor* lse, void* stream) {
  RingArgs a;
  int st = prepare_attention(q, k_gathered, v_gathered, scale, out, lse, !accumulate, &a, 5);
  if (st) return st;
  if (accumulate && out->dtype != CP_F32) return CP_ERR_DTYPE;   // the accumulator is fp32
  if (!chunk_lengths) return CP_ERR_NULL;
  if (n_chunks < 1 || n_chunks > CP_MAX_CHUNKS || k_gathered->shape[0] != n_chunks)
    return CP_ERR_OFFSETS;
  if (skip_chunk < -1 || skip_chunk >= n_chunks) return CP_ERR_OFFSETS;
  const int64_t L = k_gathered->shape[2];
  if ((int64_t)n_chunks * L > 0x7fffffffLL) return CP_ERR_SHAPE;
  int64_t starts[CP_MAX_CHUNKS + 1], ends[CP_MAX_CHUNKS];
  for (int c = 0; c < n_chunks; ++c) {
    if (chunk_lengths[c] < 0 || chunk_lengths[c] > L) return CP_ERR_OFFSETS;
    starts[c] = c * L;
    ends[c] = starts[c] + (c == skip_chunk ? 0 : chunk_lengths[c]);
  }
  starts[n_chunks] = n_chunks * L;
  a.chunk_off = starts;
  a.chunk_end = ends;
  a.n_chunks = n_chunks;
  a.merge = accumulate != 0;
  return run_attention(a, as_stream(stream));
}

int cp_ulysses_permute(const cp_tensor* x, cp_tensor* y, int degree, int dir, void* stream) {
  int st;
  if ((st = check_basic(x, 5)) || (st = check_basic(y, 5))) return st;
  if (x->dtype != y->dtype) return CP_ERR_DTYPE;
  if (dir != 0 && dir != 1) return CP_ERR_SHAPE;
  if (degree < 1) return CP_ERR_DEGREE;
  const int64_t U = degree;
  if (x->shape[0] != U || y->shape[0] != U) return CP_ERR_SHAPE;
  const int64_t B = x->shape[1], D = x->shape[4];
  if (y->shape[1] != B || y->shape[4] != D) return CP_ERR_SHAPE;
  // seq-shard side [U, B, S/U, H, D] and head-shard side [U, B, S, H/U, D]
  const cp_tensor* seq = dir == 0 ? x : y;
  const cp_tensor* head = dir == 0 ? y : x;
  const int64_t H = seq->shape[3], S = head->shape[2];
  if (H % U || S % U) return CP_ERR_DEGREE;
  if (seq->shape[2] * U != S || head->shape[3] * U != H) return CP_ERR_SHAPE;
  // (heads, D) packed on both sides: every (rank, batch, token) run of H/U
  // heads is contiguous
  const cp_tensor* both[2] = {x, y};
  for (const cp_tensor* t : both) {
    if (t->shape[4] > 1 && t->stride[4] != 1) return CP_ERR_ALIGN;
    if (t->shape[3] > 1 && t->stride[3] != D) return CP_ERR_ALIGN;
  }
  const TensorView vx = view_of(x), vy = view_of(y);
  if (self_overlapping(y) || overlaps(vx, vy)) return CP_ERR_ALIAS;
  int* err = device_error_ptr();
  if (!err) return CP_ERR_CUDA;
  return launch_ulysses_permute(vx, vy, degree, dir, err, as_stream(stream));
}

size_t cp_usp_workspace_bytes(int64_t B, int64_t S, int64_t H, int64_t D, int in_dtype,
                              int out_dtype, int ring_degree, int ulysses_degree) {
  if (B < 0 || S < 0 || H < 0 || D < 0 || ring_degree < 1 || ulysses_degree < 1) return 0;
  if ((in_dtype != CP_F32 && in_dtype != CP_BF16) || (out_dtype != CP_F32 && out_dtype != CP_BF16))
    return 0;
  const int64_t G = (int64_t)ring_degree * ulysses_degree;
  if (usp_fusable_sizes(in_dtype, D, G, G > 0 ? S / G : 0)) return 0;   // no intermediates
  return usp_unfused_bytes(B, S, H, D, in_dtype, out_dtype);
}

}  // extern "C"

namespace cpattn {

int usp_check_args(const cp_tensor* qs, const cp_tensor* ks, const cp_tensor* vs,
                   int ring_degree, int ulysses_degree, const cp_tensor* outs,
                   const cp_tensor* lse) {
  int st;
  if ((st = check_basic(qs, 5)) || (st = check_basic(ks, 5)) || (st = check_basic(vs, 5)) ||
      (st = check_basic(outs, 5)))
    return st;
  if (qs->dtype != ks->dtype || qs->dtype != vs->dtype) return CP_ERR_DTYPE;
  const int64_t R = ring_degree, U = ulysses_degree;
  if (R < 1 || U < 1 || R * U > 4096) return CP_ERR_DEGREE;
  const int64_t G = qs->shape[0], B = qs->shape[1], Sg = qs->shape[2], H = qs->shape[3];
  const cp_tensor* others[3] = {ks, vs, outs};
  for (const cp_tensor* t : others)
    for (int i = 0; i < 5; ++i)
      if (t->shape[i] != qs->shape[i]) return CP_ERR_SHAPE;
  if (G != R * U) return CP_ERR_DEGREE;
  if (H % U) return CP_ERR_DEGREE;
  const int64_t S = Sg * G;
  if (lse) {
    if ((st = check_basic(lse, 3))) return st;
    if (lse->dtype != CP_F32) return CP_ERR_DTYPE;
    if (lse->shape[0] != B || lse->shape[1] != H || lse->shape[2] != S) return CP_ERR_SHAPE;
  }
  if (R > CP_MAX_CHUNKS) return CP_ERR_DEGREE;
  if (self_overlapping(outs) || (lse && self_overlapping(lse))) return CP_ERR_ALIAS;
  return CP_OK;
}

}  // namespace cpattn

extern "C" {

int cp_usp_attention(const cp_tensor* qs, const cp_tensor* ks, const cp_tensor* vs,
                     int ring_degree, int ulysses_degree, float scale, void* workspace,
                     size_t workspace_bytes, cp_tensor* outs, cp_tensor* lse, void* stream) {
  int st;
  if ((st = usp_check_args(qs, ks, vs, ring_degree, ulysses_degree, outs, lse))) return st;
  const int64_t R = ring_degree, U = ulysses_degree;
  const int64_t G = qs->shape[0], B = qs->shape[1], Sg = qs->shape[2], H = qs->shape[3],
                D = qs->shape[4];
  const int64_t S = Sg * G, SR = Sg * U, Hg = H / U;
  if (B == 0 || S == 0 || H == 0) return CP_OK;

  // Fused: attention reads q/k/v and writes out in the shard layout through
  // 5-D tensor maps; head group u of ring rank r is just heads u*H/U.. of
  // tokens r*S/R.., so one launch over all heads with R chunks is the whole
  // grid.
  if (usp_fusable_sizes(qs->dtype, D, G, Sg) && outs->stride[4] == 1 &&
      check_vector_layout(qs, 16) == CP_OK && check_vector_layout(ks, 16) == CP_OK &&
      check_vector_layout(vs, 16) == CP_OK && check_vector_layout(outs, 16) == CP_OK) {
    RingArgs a;
    a.q = view_of(qs);
    a.k = view_of(ks);
    a.v = view_of(vs);
    a.out = view_of(outs);
    a.lse = view_of(lse);
    if (overlaps(a.out, a.q) || overlaps(a.out, a.k) || overlaps(a.out, a.v)) return CP_ERR_ALIAS;
    if (lse && (overlaps(a.lse, a.q) || overlaps(a.lse, a.k) || overlaps(a.lse, a.v) ||
                overlaps(a.lse, a.out)))
      return CP_ERR_ALIAS;
    int64_t foffs[CP_MAX_CHUNKS + 1];
    for (int64_t c = 0; c <= R; ++c) foffs[c] = c * SR;
    a.chunk_off = foffs;
    a.n_chunks = (int)R;
    a.scale = resolve_scale(scale, D);
    a.dev_err = device_error_ptr();
    if (!a.dev_err) return CP_ERR_CUDA;
    return launch_attn_ring_tc(a, as_stream(stream));
  }

  // Unfused: Ulysses permute -> ring attention per head group -> inverse
  // permute, through the caller's workspace.
  if (!workspace) return CP_ERR_WORKSPACE;
  if (workspace_bytes < usp_unfused_bytes(B, S, H, D, qs->dtype, outs->dtype))
    return CP_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return CP_ERR_ALIGN;

  const size_t n = (size_t)B * S * H * D;
  auto rnd = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const int esi = dtype_size(qs->dtype), eso = dtype_size(outs->dtype);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* Y[3] = {ws, ws + rnd(n * esi), ws + 2 * rnd(n * esi)};
  uint8_t* Yo = ws + 3 * rnd(n * esi);
  // Head-sharded buffers, [U, B, S, H/U, D] contiguous: tokens of ring block
  // r sit at sequence offset r*S/R of every head group.
  auto head_view = [&](uint8_t* base, int dt, int64_t r, int64_t len) {
    cp_tensor t;
    memset(&t, 0, sizeof(t));
    t.dtype = dt;
    t.ndim = 5;
    const int64_t sh[5] = {U, B, len, Hg, D};
    const int64_t sd[5] = {B * S * Hg * D, S * Hg * D, Hg * D, D, 1};
    for (int i = 0; i < 5; ++i) {
      t.shape[i] = sh[i];
      t.stride[i] = sd[i];
    }
    t.data = base + (size_t)(r * SR * Hg * D) * dtype_size(dt);
    return t;
  };
  auto shard_slice = [&](const cp_tensor* t, int64_t r) {
    cp_tensor s = *t;
    s.shape[0] = U;
    s.data = static_cast<uint8_t*>(t->data) + (size_t)(r * U * t->stride[0]) * dtype_size(t->dtype);
    return s;
  };
  const cp_tensor* ins[3] = {qs, ks, vs};
  // 1. Ulysses all-to-all inside every ring group r
  for (int64_t r = 0; r < R; ++r)
    for (int i = 0; i < 3; ++i) {
      cp_tensor x = shard_slice(ins[i], r);
      cp_tensor y = head_view(Y[i], qs->dtype, r, SR);
      if ((st = cp_ulysses_permute(&x, &y, (int)U, 0, stream))) return st;
    }
  // 2. ring attention over the R blocks, per head group u
  int64_t offs[CP_MAX_CHUNKS + 1];
  for (int64_t c = 0; c <= R; ++c) offs[c] = c * SR;
  for (int64_t u = 0; u < U; ++u) {
    cp_tensor q4, k4, v4, o4, l3;
    cp_tensor* four[4] = {&q4, &k4, &v4, &o4};
    uint8_t* bases[4] = {Y[0], Y[1], Y[2], Yo};
    for (int i = 0; i < 4; ++i) {
      const int dt = i < 3 ? qs->dtype : outs->dtype;
      cp_tensor& t = *four[i];
      memset(&t, 0, sizeof(t));
      t.dtype = dt;
      t.ndim = 4;
      const int64_t sh[4] = {B, S, Hg, D};
      const int64_t sd[4] = {S * Hg * D, Hg * D, D, 1};
      for (int j = 0; j < 4; ++j) {
        t.shape[j] = sh[j];
        t.stride[j] = sd[j];
      }
      t.data = bases[i] + (size_t)(u * B * S * Hg * D) * dtype_size(dt);
    }
    cp_tensor* lp = nullptr;
    if (lse) {
      l3 = *lse;
      l3.shape[1] = Hg;
      l3.data = static_cast<float*>(lse->data) + u * Hg * lse->stride[1];
      lp = &l3;
    }
    if ((st = ring_impl(&q4, &k4, &v4, offs, (int)R, scale, &o4, lp, stream))) return st;
  }
  // 3. inverse all-to-all inside every ring group r
  for (int64_t r = 0; r < R; ++r) {
    cp_tensor x = head_view(Yo, outs->dtype, r, SR);
    cp_tensor y = shard_slice(outs, r);
    if ((st = cp_ulysses_permute(&x, &y, (int)U, 1, stream))) return st;
  }
  return CP_OK;
}

}  // extern "C"

namespace cpattn {
namespace {
// n+1 host offsets starting at 0, non-decreasing, ending at `total`.
int check_offsets(const int64_t* off, int n, int64_t total) {
  if (!off) return CP_ERR_NULL;
  if (off[0] != 0 || off[n] != total) return CP_ERR_OFFSETS;
  for (int i = 0; i < n; ++i)
    if (off[i + 1] < off[i]) return CP_ERR_OFFSETS;
  return CP_OK;
}

// Flat contiguous 1-D buffer of `n` elements.
int check_flat(const cp_tensor* t, int64_t n) {
  int st;
  if ((st = check_basic(t, 1))) return st;
  if (t->shape[0] != n) return CP_ERR_SHAPE;
  if (n > 1 && t->stride[0] != 1) return CP_ERR_ALIGN;
  return CP_OK;
}

cp_tensor flat_view(void* data, int dtype, int64_t n) {
  cp_tensor t;
  memset(&t, 0, sizeof(t));
  t.data = data;
  t.dtype = dtype;
  t.ndim = 1;
  t.shape[0] = n;
  t.stride[0] = 1;
  return t;
}
}  // namespace
}  // namespace cpattn

extern "C" {

int cp_ulysses_anything_permute(const cp_tensor* x, cp_tensor* y, int64_t B, int64_t H,
                                int64_t D, int degree, const int64_t* seq_offsets,
                                const int64_t* head_offsets, int dir, void* stream) {
  int st;
  if (degree < 1 || degree > CP_MAX_CHUNKS) return CP_ERR_DEGREE;
  if (dir != 0 && dir != 1) return CP_ERR_SHAPE;
  if (B < 0 || H < 0 || D < 1) return CP_ERR_SHAPE;
  if (!seq_offsets || !head_offsets) return CP_ERR_NULL;
  const int64_t S = seq_offsets[degree];
  if (S < 0 || S > 0x7fffffffLL || H > 0x7fffffffLL) return CP_ERR_SHAPE;
  if ((st = check_offsets(seq_offsets, degree, S)) || (st = check_offsets(head_offsets, degree, H)))
    return st;
  const int64_t n = B * S * H * D;
  if ((st = check_flat(x, n)) || (st = check_flat(y, n))) return st;
  if (x->dtype != y->dtype) return CP_ERR_DTYPE;
  const TensorView vx = view_of(x), vy = view_of(y);
  if (overlaps(vx, vy)) return CP_ERR_ALIAS;
  if (n == 0) return CP_OK;
  int* err = device_error_ptr();
  if (!err) return CP_ERR_CUDA;
  return launch_ulysses_anything_permute(vx, vy, B, H, D, degree, seq_offsets, head_offsets, dir,
                                         err, as_stream(stream));
}

size_t cp_ulysses_anything_workspace_bytes(int64_t B, int64_t S, int64_t H, int64_t D,
                                           int in_dtype, int out_dtype) {
  if (B < 0 || S < 0 || H < 0 || D < 0) return 0;
  if (B == 1) return 0;   // the rank buffers are read in place
  if ((in_dtype != CP_F32 && in_dtype != CP_BF16) || (out_dtype != CP_F32 && out_dtype != CP_BF16))
    return 0;
  return usp_unfused_bytes(B, S, H, D, in_dtype, out_dtype);
}

int cp_ulysses_anything_attention(const cp_tensor* q, const cp_tensor* k, const cp_tensor* v,
                                  int64_t B, int64_t H, int64_t D, int degree,
                                  const int64_t* seq_offsets, const int64_t* head_offsets,
                                  float scale, void* workspace, size_t workspace_bytes,
                                  cp_tensor* out, cp_tensor* lse, void* stream) {
  int st;
  if (degree < 1 || degree > CP_MAX_CHUNKS) return CP_ERR_DEGREE;
  if (B < 0 || H < 0 || (D != 64 && D != 128)) return CP_ERR_SHAPE;
  if (!seq_offsets || !head_offsets) return CP_ERR_NULL;
  const int64_t S = seq_offsets[degree];
  if (S < 0 || S > 0x7fffffffLL || H > 0x7fffffffLL) return CP_ERR_SHAPE;
  if ((st = check_offsets(seq_offsets, degree, S)) || (st = check_offsets(head_offsets, degree, H)))
    return st;
  const int64_t n = B * S * H * D;
  if ((st = check_flat(q, n)) || (st = check_flat(k, n)) || (st = check_flat(v, n)) ||
      (st = check_flat(out, n)))
    return st;
  if (q->dtype != k->dtype || q->dtype != v->dtype) return CP_ERR_DTYPE;
  if (lse) {
    if ((st = check_basic(lse, 3))) return st;
    if (lse->dtype != CP_F32) return CP_ERR_DTYPE;
    if (lse->shape[0] != B || lse->shape[1] != H || lse->shape[2] != S) return CP_ERR_SHAPE;
    if (self_overlapping(lse)) return CP_ERR_ALIAS;
  }
  const TensorView vo = view_of(out);
  if (overlaps(vo, view_of(q)) || overlaps(vo, view_of(k)) || overlaps(vo, view_of(v)))
    return CP_ERR_ALIAS;
  if (n == 0) return CP_OK;

  // On one GPU every head group sits on the same device, and attention of
  // each head group over the whole sequence is attention over all heads: so
  // the all-to-all is carried out only as far as the attention kernel needs.
  // Rank buffers [B, s_p, H, D] concatenated in rank order are, for B = 1,
  // already one contiguous [1, S, H, D] tensor, read in place; for B > 1 an
  // uneven all-to-all whose single head group holds all H heads gathers the
  // sequence into [B, S, H, D] (and its inverse scatters the output back).
  const int64_t one[2] = {0, S};
  auto bshd = [&](void* data, int dtype) {
    cp_tensor t;
    memset(&t, 0, sizeof(t));
    t.data = data;
    t.dtype = dtype;
    t.ndim = 4;
    const int64_t sh[4] = {B, S, H, D};
    const int64_t sd[4] = {S * H * D, H * D, D, 1};
    for (int j = 0; j < 4; ++j) {
      t.shape[j] = sh[j];
      t.stride[j] = sd[j];
    }
    return t;
  };
  if (B == 1) {
    cp_tensor t4[4] = {bshd(q->data, q->dtype), bshd(k->data, k->dtype), bshd(v->data, v->dtype),
                       bshd(out->data, out->dtype)};
    return ring_impl(&t4[0], &t4[1], &t4[2], one, 1, scale, &t4[3], lse, stream);
  }
  if (!workspace) return CP_ERR_WORKSPACE;
  if (workspace_bytes < usp_unfused_bytes(B, S, H, D, q->dtype, out->dtype))
    return CP_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return CP_ERR_ALIGN;
  auto rnd = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const int esi = dtype_size(q->dtype);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* Y[3] = {ws, ws + rnd(n * esi), ws + 2 * rnd(n * esi)};
  uint8_t* Yo = ws + 3 * rnd(n * esi);
  int64_t all_heads[CP_MAX_CHUNKS + 1];
  all_heads[0] = 0;
  for (int g = 1; g <= degree; ++g) all_heads[g] = H;
  const cp_tensor* ins[3] = {q, k, v};
  for (int i = 0; i < 3; ++i) {
    cp_tensor y = flat_view(Y[i], q->dtype, n);
    if ((st = cp_ulysses_anything_permute(ins[i], &y, B, H, D, degree, seq_offsets, all_heads, 0,
                                          stream)))
      return st;
  }
  cp_tensor t4[4] = {bshd(Y[0], q->dtype), bshd(Y[1], q->dtype), bshd(Y[2], q->dtype),
                     bshd(Yo, out->dtype)};
  if ((st = ring_impl(&t4[0], &t4[1], &t4[2], one, 1, scale, &t4[3], lse, stream))) return st;
  cp_tensor yo = flat_view(Yo, out->dtype, n);
  return cp_ulysses_anything_permute(&yo, out, B, H, D, degree, seq_offsets, all_heads, 1, stream);
}

int cp_ring_chunk_offsets(int64_t S, int R, int64_t* offsets) {
  if (!offsets) return CP_ERR_NULL;
  if (S < 0 || R < 1) return CP_ERR_SHAPE;
  const int64_t c = S > 0 ? (S + R - 1) / R : 0;
  offsets[0] = 0;
  for (int i = 0; i < R; ++i) {
    const int64_t nx = offsets[i] + c;
    offsets[i + 1] = nx < S ? nx : S;
  }
  return CP_OK;
}

const char* cp_status_string(int status) {
  switch (status) {
    case CP_OK: return "ok";
    case CP_ERR_NULL: return "null pointer or tensor";
    case CP_ERR_DTYPE: return "unsupported or mismatched dtype";
    case CP_ERR_SHAPE: return "bad or mismatched shape";
    case CP_ERR_ALIGN: return "misaligned pointer or stride, or non-contiguous last dim";
    case CP_ERR_OFFSETS: return "bad chunk offsets";
    case CP_ERR_DEGREE: return "degree does not divide sequence length or head count";
    case CP_ERR_CUDA: return "CUDA runtime or driver error";
    case CP_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    case CP_ERR_WORKSPACE: return "workspace missing or too small";
    case CP_ERR_ALIAS: return "output overlaps an input";
    case CP_ERR_BOUNDS: return "a device-side bounds check failed (debug build)";
    default: return "unknown status";
  }
}

int cp_last_device_error(void* stream) {
  int* p = device_error_ptr();
  if (!p) return CP_ERR_CUDA;
  int h = 0;
  cudaStream_t s = as_stream(stream);
  if (cudaMemcpyAsync(&h, p, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return CP_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return CP_ERR_CUDA;
  if (h != 0) {
    const int zero = 0;
    if (cudaMemcpyAsync(p, &zero, sizeof(int), cudaMemcpyHostToDevice, s) != cudaSuccess)
      return CP_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return CP_ERR_CUDA;
    return h == kDevErrBounds ? CP_ERR_BOUNDS : CP_ERR_TIMEOUT;
  }
  return CP_OK;
}

int cp_selftest_bounds_check(void* stream) {
  int* p = device_error_ptr();
  if (!p) return CP_ERR_CUDA;
  return launch_bounds_selftest(p, as_stream(stream));
}

int cp_selftest_wait_timeout(int spin_limit, void* stream) {
  if (spin_limit < 1 || spin_limit > (1 << 24)) return CP_ERR_SHAPE;
  int* p = device_error_ptr();
  if (!p) return CP_ERR_CUDA;
  return launch_wait_timeout_selftest(spin_limit, p, as_stream(stream));
}

}  // extern "C"

namespace cpattn {

namespace {
__global__ void wait_timeout_selftest_kernel(int spin_limit, int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the wait must give up after spin_limit
  // polls and record the timeout.
  if (threadIdx.x == 0) mbar_wait_polls(&bar, 0, (uint32_t)spin_limit, err);
}
}  // namespace

namespace {
// One deliberately failing bounds check: a debug build records it in the
// device error word, a release build compiles the check away.  The guarded
// store only touches this block's own shared memory in either build.
__global__ void bounds_selftest_kernel(int* err) {
  __shared__ volatile int cell;
  const int idx = 1 + (int)threadIdx.x;   // "one past the end" of a 1-element range
  if (CP_IN_BOUNDS(idx < 1, err)) cell = idx;
}
}  // namespace

int launch_bounds_selftest(int* dev_err, cudaStream_t stream) {
  bounds_selftest_kernel<<<1, 1, 0, stream>>>(dev_err);
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

int launch_wait_timeout_selftest(int spin_limit, int* dev_err, cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(spin_limit, dev_err);
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

}  // namespace cpattn
