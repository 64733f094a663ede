// fp32 log-sum-exp merge of one ring partial into the accumulator, in place.
//
// diffusers parallelism API page, ContextParallelConfig.convert_to_fp32: the
// per-block output and LSE are converted to float32 and combined.  Per row,
// with a = lse_acc, b = lse_i (natural log):
//   lse' = max(a, b) + log1p(exp(-|a - b|))
//   out' = exp(a - lse') * out_acc + exp(b - lse') * out_i
// (0, -inf) is the identity; a = b = -inf leaves the accumulator alone.
//
// HBM-bound: per output row of D floats it reads out_acc and out_i and
// writes out_acc back (12 bytes per fp32 element, 10 with a bf16 out_i) plus
// 12 bytes of LSE.  One warp owns 8 consecutive tokens of one (batch, head):
// it loads their two LSEs and all 8 rows of both partials at once (one
// memory round trip), computes the two weights per token, and writes the 8
// merged rows, each lane moving D/32 consecutive elements per row with one
// vector access.

#include "common.cuh"
#include "internal.h"

namespace cpattn {

namespace {

struct MergeParams {
  float* acc;
  float* lse_acc;
  const void* oi;
  const float* lse_i;
  long long a_sb, a_ss, a_sh;      // out_acc strides
  long long i_sb, i_ss, i_sh;      // out_i strides
  long long la_sb, la_sh, la_ss;   // lse_acc strides
  long long li_sb, li_sh, li_ss;   // lse_i strides
  int B, S, H, n_sblocks;
  int* err;
  long long span_a, span_i, span_la, span_li;   // elements (bounds checks)
};

template <int V>
struct F32Vec;
template <>
struct F32Vec<4> {
  using T = float4;
};
template <>
struct F32Vec<2> {
  using T = float2;
};

template <int V, bool BF16_IN>
struct InVec {
  static __device__ __forceinline__ void load(const void* base, long long off, float* x) {
    if constexpr (BF16_IN) {
      const __nv_bfloat16* p = reinterpret_cast<const __nv_bfloat16*>(base) + off;
      if constexpr (V == 4) {
        const uint2 u = __ldcs(reinterpret_cast<const uint2*>(p));
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
        x[0] = __low2float(a);
        x[1] = __high2float(a);
        x[2] = __low2float(b);
        x[3] = __high2float(b);
      } else {
        const unsigned int w = __ldcs(reinterpret_cast<const unsigned int*>(p));
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&w);
        x[0] = __low2float(a);
        x[1] = __high2float(a);
      }
    } else {
      const float* p = reinterpret_cast<const float*>(base) + off;
      if constexpr (V == 4) {
        const float4 u = __ldcs(reinterpret_cast<const float4*>(p));
        x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
      } else {
        const float2 u = __ldcs(reinterpret_cast<const float2*>(p));
        x[0] = u.x; x[1] = u.y;
      }
    }
  }
};

// One warp owns kTok consecutive tokens of one (batch, head).  All of its
// row loads are issued together with the two LSE loads, so a warp needs a
// single memory round trip; loads and stores use the streaming (evict-first)
// cache policy since every byte is touched exactly once.
#ifndef CP_MERGE_TOKENS_PER_WARP
#define CP_MERGE_TOKENS_PER_WARP 8
#endif
constexpr int kTok = CP_MERGE_TOKENS_PER_WARP;
#ifndef CP_MERGE_BLOCKS
#define CP_MERGE_BLOCKS (148 * 8)
#endif
constexpr long long kMergeBlocks = CP_MERGE_BLOCKS;

template <int D, bool BF16_IN>
__global__ void __launch_bounds__(256) lse_merge_kernel(const __grid_constant__ MergeParams p) {
  constexpr int V = D / 32;   // elements per lane per row
  using FV = typename F32Vec<V>::T;
  const int lane = threadIdx.x & 31;
  const long long n_groups = (long long)p.n_sblocks * p.H * p.B;
  const long long n_warps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long gw = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; gw < n_groups;
       gw += n_warps) {
  // heads fastest: neighbouring warps merge neighbouring rows in memory
  const int h = (int)(gw % p.H);
  const long long sbb = gw / p.H;
  const int sb = (int)(sbb % p.n_sblocks);
  const int b = (int)(sbb / p.n_sblocks);
  const int s0 = sb * kTok;
  const int n_rows = min(kTok, p.S - s0);

  // lanes 0..kTok-1 read lse_acc, lanes 16..16+kTok-1 read lse_i
  float lv = -INFINITY;
  {
    const int tk = lane & 15;
    if (tk < n_rows) {
      const long long s = s0 + tk;
      const long long la = b * p.la_sb + h * p.la_sh + s * p.la_ss;
      const long long li = b * p.li_sb + h * p.li_sh + s * p.li_ss;
      if (lane < 16 ? CP_IN_BOUNDS(la >= 0 && la < p.span_la, p.err)
                    : CP_IN_BOUNDS(li >= 0 && li < p.span_li, p.err))
        lv = lane < 16 ? __ldcs(p.lse_acc + la) : __ldcs(p.lse_i + li);
    }
  }
  float x[kTok][V], y[kTok][V];
  // rows whose offsets fail a debug-build bounds check are neither read nor written
  bool row_ok[kTok];
#pragma unroll
  for (int t = 0; t < kTok; ++t) {
    const long long sr = s0 + t;
    const long long oa = b * p.a_sb + sr * p.a_ss + h * p.a_sh;
    const long long oi = b * p.i_sb + sr * p.i_ss + h * p.i_sh;
    row_ok[t] = t < n_rows && CP_IN_BOUNDS(oa >= 0 && oa + D <= p.span_a && oi >= 0 &&
                                               oi + D <= p.span_i,
                                           p.err);
  }
#pragma unroll
  for (int t = 0; t < kTok; ++t) {
    if (row_ok[t]) {
      const long long sr = s0 + t;
      const FV av = __ldcs(reinterpret_cast<const FV*>(p.acc + b * p.a_sb + sr * p.a_ss +
                                                        h * p.a_sh + lane * V));
      const float* af = reinterpret_cast<const float*>(&av);
#pragma unroll
      for (int i = 0; i < V; ++i) x[t][i] = af[i];
      InVec<V, BF16_IN>::load(p.oi, b * p.i_sb + sr * p.i_ss + h * p.i_sh + lane * V, y[t]);
    }
  }
  // weights of token `lane` (lanes 0..kTok-1)
  const float a = lv;
  const float bb = __shfl_sync(0xffffffffu, lv, (lane & 15) + 16);
  float wa = 1.f, wb = 0.f;
  if (lane < n_rows && !(a == -INFINITY && bb == -INFINITY)) {
    const float mx = fmaxf(a, bb);
    const float nl = mx + log1pf(expf(-fabsf(a - bb)));
    wa = expf(a - nl);
    wb = expf(bb - nl);
    const long long la = b * p.la_sb + h * p.la_sh + (long long)(s0 + lane) * p.la_ss;
    if (CP_IN_BOUNDS(la >= 0 && la < p.span_la, p.err)) __stcs(p.lse_acc + la, nl);
  }
#pragma unroll
  for (int t = 0; t < kTok; ++t) {
    const float ca = __shfl_sync(0xffffffffu, wa, t);
    const float cb = __shfl_sync(0xffffffffu, wb, t);
    if (row_ok[t]) {
      const long long sr = s0 + t;
      float r[V];
#pragma unroll
      for (int i = 0; i < V; ++i) r[i] = ca * x[t][i] + cb * y[t][i];
      __stcs(reinterpret_cast<FV*>(p.acc + b * p.a_sb + sr * p.a_ss + h * p.a_sh + lane * V),
             *reinterpret_cast<const FV*>(r));
    }
  }
  }
}

}  // namespace

int launch_lse_merge(const TensorView& acc, const TensorView& lse_acc, const TensorView& oi,
                     const TensorView& lse_i, int* dev_err, cudaStream_t stream) {
  MergeParams p;
  p.err = dev_err;
  p.span_a = span_elems(acc);
  p.span_i = span_elems(oi);
  p.span_la = span_elems(lse_acc);
  p.span_li = span_elems(lse_i);
  p.acc = static_cast<float*>(acc.data);
  p.lse_acc = static_cast<float*>(lse_acc.data);
  p.oi = oi.data;
  p.lse_i = static_cast<const float*>(lse_i.data);
  p.a_sb = acc.stride[0];
  p.a_ss = acc.stride[1];
  p.a_sh = acc.stride[2];
  p.i_sb = oi.stride[0];
  p.i_ss = oi.stride[1];
  p.i_sh = oi.stride[2];
  p.la_sb = lse_acc.stride[0];
  p.la_sh = lse_acc.stride[1];
  p.la_ss = lse_acc.stride[2];
  p.li_sb = lse_i.stride[0];
  p.li_sh = lse_i.stride[1];
  p.li_ss = lse_i.stride[2];
  p.B = (int)acc.shape[0];
  p.S = (int)acc.shape[1];
  p.H = (int)acc.shape[2];
  p.n_sblocks = (p.S + kTok - 1) / kTok;
  const int D = (int)acc.shape[3];
  const long long warps = (long long)p.n_sblocks * p.H * p.B;
  if (warps <= 0) return CP_OK;
  // persistent grid: 8 blocks of 8 warps per SM, grid-stride over the
  // token groups, so all warps start together and finish together
  long long blocks = (warps + 7) / 8;
  if (blocks > kMergeBlocks) blocks = kMergeBlocks;
  const bool bf = oi.dtype == CP_BF16;
  if (D == 128 && !bf) lse_merge_kernel<128, false><<<(int)blocks, 256, 0, stream>>>(p);
  else if (D == 128 && bf) lse_merge_kernel<128, true><<<(int)blocks, 256, 0, stream>>>(p);
  else if (D == 64 && !bf) lse_merge_kernel<64, false><<<(int)blocks, 256, 0, stream>>>(p);
  else if (D == 64 && bf) lse_merge_kernel<64, true><<<(int)blocks, 256, 0, stream>>>(p);
  else return CP_ERR_SHAPE;
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

}  // namespace cpattn
