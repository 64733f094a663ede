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
// 12 bytes of LSE.  One warp owns 32 consecutive tokens of one (batch,
// head): lane t reads both LSEs of token t with one coalesced 128-byte load,
// computes the two weights, and the warp then streams the 32 output rows,
// each lane moving D/32 consecutive elements with one vector access.

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
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
        x[0] = __low2float(a);
        x[1] = __high2float(a);
        x[2] = __low2float(b);
        x[3] = __high2float(b);
      } else {
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(p);
        x[0] = __low2float(a);
        x[1] = __high2float(a);
      }
    } else {
      const float* p = reinterpret_cast<const float*>(base) + off;
      if constexpr (V == 4) {
        const float4 u = *reinterpret_cast<const float4*>(p);
        x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
      } else {
        const float2 u = *reinterpret_cast<const float2*>(p);
        x[0] = u.x; x[1] = u.y;
      }
    }
  }
};

template <int D, bool BF16_IN>
__global__ void __launch_bounds__(256) lse_merge_kernel(const __grid_constant__ MergeParams p) {
  constexpr int V = D / 32;   // elements per lane per row
  constexpr int U = 4;        // rows in flight per lane
  const int lane = threadIdx.x & 31;
  const long long gw = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const int sb = (int)(gw % p.n_sblocks);
  const long long hb = gw / p.n_sblocks;
  const int h = (int)(hb % p.H);
  const int b = (int)(hb / p.H);
  if (b >= p.B) return;

  const int s0 = sb * 32;
  const int s = s0 + lane;
  float wa = 1.f, wb = 0.f;
  if (s < p.S) {
    float* la_p = p.lse_acc + b * p.la_sb + h * p.la_sh + (long long)s * p.la_ss;
    const float a = *la_p;
    const float bb = p.lse_i[b * p.li_sb + h * p.li_sh + (long long)s * p.li_ss];
    if (!(a == -INFINITY && bb == -INFINITY)) {
      const float mx = fmaxf(a, bb);
      const float nl = mx + log1pf(expf(-fabsf(a - bb)));
      wa = expf(a - nl);
      wb = expf(bb - nl);
      *la_p = nl;
    }
  }
  const int n_rows = min(32, p.S - s0);
  for (int t0 = 0; t0 < n_rows; t0 += U) {
    float x[U][V], y[U][V], ws[U][2];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = t0 + u;
      ws[u][0] = __shfl_sync(0xffffffffu, wa, t & 31);
      ws[u][1] = __shfl_sync(0xffffffffu, wb, t & 31);
      if (t < n_rows) {
        const long long sr = s0 + t;
        const float* ap = p.acc + b * p.a_sb + sr * p.a_ss + h * p.a_sh + lane * V;
        const typename F32Vec<V>::T av = *reinterpret_cast<const typename F32Vec<V>::T*>(ap);
        const float* af = reinterpret_cast<const float*>(&av);
#pragma unroll
        for (int i = 0; i < V; ++i) x[u][i] = af[i];
        InVec<V, BF16_IN>::load(p.oi, b * p.i_sb + sr * p.i_ss + h * p.i_sh + lane * V, y[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = t0 + u;
      if (t < n_rows) {
        const long long sr = s0 + t;
        float r[V];
#pragma unroll
        for (int i = 0; i < V; ++i) r[i] = ws[u][0] * x[u][i] + ws[u][1] * y[u][i];
        float* ap = p.acc + b * p.a_sb + sr * p.a_ss + h * p.a_sh + lane * V;
        *reinterpret_cast<typename F32Vec<V>::T*>(ap) =
            *reinterpret_cast<const typename F32Vec<V>::T*>(r);
      }
    }
  }
}

}  // namespace

int launch_lse_merge(const TensorView& acc, const TensorView& lse_acc, const TensorView& oi,
                     const TensorView& lse_i, cudaStream_t stream) {
  MergeParams p;
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
  p.n_sblocks = (p.S + 31) / 32;
  const int D = (int)acc.shape[3];
  const long long warps = (long long)p.n_sblocks * p.H * p.B;
  if (warps <= 0) return CP_OK;
  const long long blocks = (warps + 7) / 8;
  if (blocks > 0x7fffffffLL) return CP_ERR_SHAPE;
  const bool bf = oi.dtype == CP_BF16;
  if (D == 128 && !bf) lse_merge_kernel<128, false><<<(int)blocks, 256, 0, stream>>>(p);
  else if (D == 128 && bf) lse_merge_kernel<128, true><<<(int)blocks, 256, 0, stream>>>(p);
  else if (D == 64 && !bf) lse_merge_kernel<64, false><<<(int)blocks, 256, 0, stream>>>(p);
  else if (D == 64 && bf) lse_merge_kernel<64, true><<<(int)blocks, 256, 0, stream>>>(p);
  else return CP_ERR_SHAPE;
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

}  // namespace cpattn
