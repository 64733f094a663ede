// The Ulysses all-to-all as an on-GPU layout permutation.
//
// diffusers context-parallelism guide, §Ulysses Attention: the first
// all-to-all regroups the data so that every GPU holds every token of a
// subset of the heads; the second regroups the result by token.  With the
// U ranks' shards held rank-major in one tensor:
//   dir 0:  x [U, B, S/U, H, D]  ->  y [U, B, S, H/U, D]
//           y[q, b, p*S/U + s, h', d] = x[p, b, s, q*H/U + h', d]
//   dir 1:  the inverse, x [U, B, S, H/U, D] -> y [U, B, S/U, H, D].
//
// For every (destination rank, batch, token) the H/U heads of one group are
// one contiguous run of (H/U)*D elements on both sides (1536 bytes for
// 6 heads of 128 bf16), so the permutation is a gather of contiguous runs:
// pure HBM traffic, one read and one write of every byte.  A warp owns one
// run at a time (index arithmetic once per run) and moves it with 16-byte
// vector loads, all issued before the stores; runs are walked in
// destination order so consecutive warps write consecutive memory.

#include "common.cuh"
#include "internal.h"

namespace cpattn {

namespace {

struct PermParams {
  const uint8_t* x;
  uint8_t* y;
  long long xs[4];   // byte strides of x dims 0..3
  long long ys[4];   // byte strides of y dims 0..3
  long long n_runs;
  int U, B, Sl, Hg;
  int run_words;     // run length in vector words
  int dir;
  int* err;
  long long span_x, span_y;   // bytes from the first to one past the last element
};

template <typename W>
__global__ void __launch_bounds__(256) ulysses_permute_kernel(const __grid_constant__ PermParams p) {
  constexpr int K = 4;   // words in flight per lane
  const int lane = threadIdx.x & 31;
  const long long warp0 = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long r = warp0; r < p.n_runs; r += n_warps) {
    const uint8_t* src;
    uint8_t* dst;
    if (p.dir == 0) {
      // r = ((q*B + b)*U + p)*Sl + s
      long long t = r;
      const int s = (int)(t % p.Sl); t /= p.Sl;
      const int pp = (int)(t % p.U); t /= p.U;
      const int b = (int)(t % p.B);
      const int q = (int)(t / p.B);
      src = p.x + pp * p.xs[0] + b * p.xs[1] + s * p.xs[2] + (long long)q * p.Hg * p.xs[3];
      dst = p.y + q * p.ys[0] + b * p.ys[1] + ((long long)pp * p.Sl + s) * p.ys[2];
    } else {
      // r = ((p*B + b)*Sl + s)*U + q
      long long t = r;
      const int q = (int)(t % p.U); t /= p.U;
      const int s = (int)(t % p.Sl); t /= p.Sl;
      const int b = (int)(t % p.B);
      const int pp = (int)(t / p.B);
      src = p.x + q * p.xs[0] + b * p.xs[1] + ((long long)pp * p.Sl + s) * p.xs[2];
      dst = p.y + pp * p.ys[0] + b * p.ys[1] + s * p.ys[2] + (long long)q * p.Hg * p.ys[3];
    }
    const long long run_b = (long long)p.run_words * (long long)sizeof(W);
    if (!CP_IN_BOUNDS(src >= p.x && src - p.x + run_b <= p.span_x && dst >= p.y &&
                          dst - p.y + run_b <= p.span_y,
                      p.err))
      continue;
    const W* sw = reinterpret_cast<const W*>(src);
    W* dw = reinterpret_cast<W*>(dst);
    for (int w0 = lane; w0 < p.run_words; w0 += 32 * K) {
      W buf[K];
#pragma unroll
      for (int k = 0; k < K; ++k)
        if (w0 + 32 * k < p.run_words) buf[k] = sw[w0 + 32 * k];
#pragma unroll
      for (int k = 0; k < K; ++k)
        if (w0 + 32 * k < p.run_words) dw[w0 + 32 * k] = buf[k];
    }
  }
}

bool aligned_to(uintptr_t v, int a) { return (v % (uintptr_t)a) == 0; }

// ---------------------------------------------------------------- uneven
// Ulysses Anything: rank p holds s_p tokens, rank q holds h_q heads (host
// offset tables).  Sequence side: the U rank buffers [B, s_p, H, D]
// concatenated; head side: the U rank buffers [B, S, h_q, D] concatenated.
// Every (b, token, head group) is again one contiguous run of h_q*D
// elements on both sides; runs are walked in destination order.
struct PermAnyParams {
  const uint8_t* x;
  uint8_t* y;
  long long B, S, H, D;
  long long n_runs;
  int U, dir, es, wbytes;
  int* err;
  long long n_elems;          // elements on either side (bounds checks)
  int seq_off[CP_MAX_CHUNKS + 1];
  int head_off[CP_MAX_CHUNKS + 1];
};

// The rank holding position v: the largest p with scale*off[p] <= v.  Since
// off is non-decreasing and v < scale*off[U], that rank is never empty.
__device__ __forceinline__ int find_rank(const int* off, int U, long long v, long long scale) {
  int lo = 0, hi = U - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (scale * off[mid] <= v) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <typename W>
__global__ void __launch_bounds__(256)
    ulysses_anything_kernel(const __grid_constant__ PermAnyParams p) {
  constexpr int K = 4;
  const int lane = threadIdx.x & 31;
  const long long warp0 = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = ((long long)gridDim.x * blockDim.x) >> 5;
  const long long HD = p.H * p.D;
  for (long long r = warp0; r < p.n_runs; r += n_warps) {
    long long src, dst, len;   // element offsets and run length
    if (p.dir == 0) {
      // destination rows: (q, b, t), group q has B*S rows of h_q*D
      const int q = (int)(r / (p.B * p.S));
      const long long rem = r - (long long)q * p.B * p.S;
      const long long b = rem / p.S, t = rem - b * p.S;
      const int pr = find_rank(p.seq_off, p.U, t, 1);
      const long long s0 = p.seq_off[pr], sp = p.seq_off[pr + 1] - s0;
      const long long h0 = p.head_off[q], hq = p.head_off[q + 1] - h0;
      len = hq * p.D;
      src = p.B * s0 * HD + (b * sp + (t - s0)) * HD + h0 * p.D;
      dst = p.B * p.S * h0 * p.D + (b * p.S + t) * len;
    } else {
      // destination rows: (p, b, s) of the sequence side, then q in order
      const long long row = r / p.U;
      const int q = (int)(r - row * p.U);
      const int pp = find_rank(p.seq_off, p.U, row, p.B);   // rank p owns rows [B*off_p, B*off_p+1)
      const long long s0 = p.seq_off[pp], sp = p.seq_off[pp + 1] - s0;
      const long long in_rank = row - p.B * s0;
      const long long b = in_rank / sp, s = in_rank - b * sp, t = s0 + s;
      const long long h0 = p.head_off[q], hq = p.head_off[q + 1] - h0;
      len = hq * p.D;
      src = p.B * p.S * h0 * p.D + (b * p.S + t) * len;
      dst = row * HD + h0 * p.D;
    }
    if (len == 0) continue;
    if (!CP_IN_BOUNDS(src >= 0 && src + len <= p.n_elems && dst >= 0 && dst + len <= p.n_elems,
                      p.err))
      continue;
    const W* sw = reinterpret_cast<const W*>(p.x + src * p.es);
    W* dw = reinterpret_cast<W*>(p.y + dst * p.es);
    const int words = (int)(len * p.es / p.wbytes);
    for (int w0 = lane; w0 < words; w0 += 32 * K) {
      W buf[K];
#pragma unroll
      for (int k = 0; k < K; ++k)
        if (w0 + 32 * k < words) buf[k] = sw[w0 + 32 * k];
#pragma unroll
      for (int k = 0; k < K; ++k)
        if (w0 + 32 * k < words) dw[w0 + 32 * k] = buf[k];
    }
  }
}

}  // namespace

int launch_ulysses_anything_permute(const TensorView& x, const TensorView& y, int64_t B,
                                    int64_t H, int64_t D, int U, const int64_t* seq_off,
                                    const int64_t* head_off, int dir, int* dev_err,
                                    cudaStream_t stream) {
  PermAnyParams p;
  p.err = dev_err;
  p.n_elems = B * seq_off[U] * H * D;
  p.x = static_cast<const uint8_t*>(x.data);
  p.y = static_cast<uint8_t*>(y.data);
  p.B = B;
  p.S = seq_off[U];
  p.H = H;
  p.D = D;
  p.U = U;
  p.dir = dir;
  p.es = dtype_size(x.dtype);
  for (int i = 0; i <= U; ++i) {
    p.seq_off[i] = (int)seq_off[i];
    p.head_off[i] = (int)head_off[i];
  }
  // every run is a multiple of D elements long and starts on a D boundary
  int wb = 16;
  const long long unit = D * p.es;
  while (wb > p.es && (unit % wb || !aligned_to((uintptr_t)x.data, wb) ||
                       !aligned_to((uintptr_t)y.data, wb)))
    wb >>= 1;
  p.wbytes = wb;
  p.n_runs = dir == 0 ? (long long)U * B * p.S : B * p.S * U;
  if (p.n_runs == 0) return CP_OK;
  long long blocks = (p.n_runs + 7) / 8;
  if (blocks > 148LL * 8) blocks = 148LL * 8;
  switch (wb) {
    case 16: ulysses_anything_kernel<uint4><<<(int)blocks, 256, 0, stream>>>(p); break;
    case 8: ulysses_anything_kernel<uint2><<<(int)blocks, 256, 0, stream>>>(p); break;
    case 4: ulysses_anything_kernel<uint32_t><<<(int)blocks, 256, 0, stream>>>(p); break;
    default: ulysses_anything_kernel<uint16_t><<<(int)blocks, 256, 0, stream>>>(p); break;
  }
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

// x, y as validated by the C-ABI: 5-D, same dtype, (heads, D) packed.
int launch_ulysses_permute(const TensorView& x, const TensorView& y, int U, int dir,
                           int* dev_err, cudaStream_t stream) {
  const int es = dtype_size(x.dtype);
  PermParams p;
  p.err = dev_err;
  p.span_x = span_elems(x) * es;
  p.span_y = span_elems(y) * es;
  p.x = static_cast<const uint8_t*>(x.data);
  p.y = static_cast<uint8_t*>(y.data);
  for (int i = 0; i < 4; ++i) {
    p.xs[i] = x.stride[i] * es;
    p.ys[i] = y.stride[i] * es;
  }
  p.U = U;
  p.dir = dir;
  p.B = (int)x.shape[1];
  const int64_t D = x.shape[4];
  if (dir == 0) {
    p.Sl = (int)x.shape[2];
    p.Hg = (int)(x.shape[3] / U);
  } else {
    p.Sl = (int)(x.shape[2] / U);
    p.Hg = (int)x.shape[3];
  }
  // the run's head offset is taken along dim 3 of whichever side holds all H
  // heads; its stride is D elements there.
  const long long run_bytes = (long long)p.Hg * D * es;
  p.n_runs = (long long)U * U * p.B * p.Sl;
  if (p.n_runs == 0 || run_bytes == 0) return CP_OK;

  int wb = 16;
  auto ok = [&](int a) {
    if (run_bytes % a) return false;
    if (!aligned_to((uintptr_t)x.data, a) || !aligned_to((uintptr_t)y.data, a)) return false;
    for (int i = 0; i < 4; ++i)
      if (p.xs[i] % a || p.ys[i] % a) return false;
    return true;
  };
  while (wb > es && !ok(wb)) wb >>= 1;
  if (!ok(wb)) return CP_ERR_ALIGN;
  p.run_words = (int)(run_bytes / wb);

  const long long warps_needed = p.n_runs;
  long long blocks = (warps_needed + 7) / 8;
  const long long cap = 148LL * 8;   // 8 blocks of 256 threads per SM
  if (blocks > cap) blocks = cap;
  switch (wb) {
    case 16: ulysses_permute_kernel<uint4><<<(int)blocks, 256, 0, stream>>>(p); break;
    case 8: ulysses_permute_kernel<uint2><<<(int)blocks, 256, 0, stream>>>(p); break;
    case 4: ulysses_permute_kernel<uint32_t><<<(int)blocks, 256, 0, stream>>>(p); break;
    default: ulysses_permute_kernel<uint16_t><<<(int)blocks, 256, 0, stream>>>(p); break;
  }
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

}  // namespace cpattn
