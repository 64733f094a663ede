// Ring attention in exact fp32 (CUDA cores, FFMA), for fp32 inputs.
//
// Same computation as the tensor-core kernel (diffusers context-parallelism
// guide, §Ring Attention / §Ring Anything; ContextParallelConfig
// .convert_to_fp32): walk the K/V chunks, keep one fp32 running max, sum and
// output accumulator per query row, never let a tile cross a chunk end.
// bf16 tensor-core MMAs would round the fp32 inputs to 8 mantissa bits, far
// outside a 1e-4 tolerance, so fp32 inputs take this path.
//
// Block = 4 warps, 16 query rows of one (batch, head); each warp owns 4
// rows.  Keys are staged 32 at a time in shared memory; lane j of a warp
// scores key j against the row, then the tile max and the tile sum are warp
// shuffle reductions, and lane i accumulates output dimensions i, i+32, ...

#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace cpattn {

namespace {

constexpr int kRowsPerBlock = 16;
constexpr int kRowsPerWarp = 4;
constexpr int kKeysPerTile = 32;

struct F32Params {
  const float* q;
  const float* k;
  const float* v;
  long long q_sb, q_ss, q_sh;
  // key token s is row s % seg_kv of slot s / seg_kv (one slot for [B, S, H, D])
  long long k_sb, k_ss, k_sh, k_sg;
  long long v_sb, v_ss, v_sh, v_sg;
  int seg_kv;
  void* out;
  int out_bf16;
  int merge;
  long long o_sb, o_ss, o_sh;
  float* lse;
  long long l_sb, l_sh, l_ss;
  int B, H, S_q, n_row_blocks, n_chunks;
  float scale;
  int* err;
  long long span_q, span_k, span_v, span_out, span_lse;   // elements (bounds checks)
  int chunk_off[CP_MAX_CHUNKS + 1];   // chunk c covers key tokens [chunk_off[c], chunk_end[c])
  int chunk_end[CP_MAX_CHUNKS];
};

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int D>
__global__ void __launch_bounds__(128) attn_ring_f32_kernel(const __grid_constant__ F32Params p) {
  constexpr int DP = D + 1;   // padded row: lane j reading row j hits bank (j + d) % 32
  constexpr int NV = D / 32;  // output dims per lane
  __shared__ float sQ[kRowsPerBlock][DP];
  __shared__ float sK[kKeysPerTile][DP];
  __shared__ float sV[kKeysPerTile][D];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rb = blockIdx.x % p.n_row_blocks;
  const int hb = blockIdx.x / p.n_row_blocks;
  const int h = hb % p.H, b = hb / p.H;
  const int r0 = rb * kRowsPerBlock;

  for (int i = threadIdx.x; i < kRowsPerBlock * D; i += blockDim.x) {
    const int r = i / D, d = i % D, s = r0 + r;
    const long long off = b * p.q_sb + (long long)s * p.q_ss + h * p.q_sh + d;
    sQ[r][d] = s < p.S_q && CP_IN_BOUNDS(off >= 0 && off < p.span_q, p.err) ? p.q[off] : 0.f;
  }

  float m[kRowsPerWarp], l[kRowsPerWarp], acc[kRowsPerWarp][NV];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) acc[r][i] = 0.f;
  }

  for (int c = 0; c < p.n_chunks; ++c) {
    const int lo = p.chunk_off[c], hi = p.chunk_end[c];
    for (int t0 = lo; t0 < hi; t0 += kKeysPerTile) {
      const int n = min(kKeysPerTile, hi - t0);
      __syncthreads();   // everyone is done with the previous tile
      for (int i = threadIdx.x; i < n * D; i += blockDim.x) {
        const int j = i / D, d = i % D;
        const int key = t0 + j;
        const long long row = key % p.seg_kv, slot = key / p.seg_kv;
        const long long ok_ = b * p.k_sb + row * p.k_ss + slot * p.k_sg + h * p.k_sh + d;
        const long long ov_ = b * p.v_sb + row * p.v_ss + slot * p.v_sg + h * p.v_sh + d;
        sK[j][d] = CP_IN_BOUNDS(ok_ >= 0 && ok_ < p.span_k, p.err) ? p.k[ok_] : 0.f;
        sV[j][d] = CP_IN_BOUNDS(ov_ >= 0 && ov_ < p.span_v, p.err) ? p.v[ov_] : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) {
        const int row = warp * kRowsPerWarp + r;
        float sc = -INFINITY;
        if (lane < n) {
          float dot = 0.f;
#pragma unroll 8
          for (int d = 0; d < D; ++d) dot = fmaf(sQ[row][d], sK[lane][d], dot);
          sc = dot * p.scale;
        }
        const float m_new = fmaxf(m[r], warp_max(sc));
        const float alpha = expf(m[r] - m_new);   // 0 on the first tile
        const float pj = lane < n ? expf(sc - m_new) : 0.f;
        l[r] = l[r] * alpha + warp_sum(pj);
#pragma unroll
        for (int i = 0; i < NV; ++i) acc[r][i] *= alpha;
        for (int j = 0; j < n; ++j) {
          const float pb = __shfl_sync(0xffffffffu, pj, j);
#pragma unroll
          for (int i = 0; i < NV; ++i) acc[r][i] = fmaf(pb, sV[j][lane + 32 * i], acc[r][i]);
        }
        m[r] = m_new;
      }
    }
  }

#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int s = r0 + warp * kRowsPerWarp + r;
    if (s >= p.S_q) continue;
    float o_w = 1.f / l[r];
    const float lse_c = m[r] + logf(l[r]);
    const long long base = b * p.o_sb + (long long)s * p.o_ss + h * p.o_sh;
    const long long l_off = b * p.l_sb + h * p.l_sh + (long long)s * p.l_ss;
    float* lse_p = p.lse != nullptr && CP_IN_BOUNDS(l_off >= 0 && l_off < p.span_lse, p.err)
                       ? p.lse + l_off
                       : nullptr;
    // every lane writes D/32 elements of the row, the last at base + D - 1
    if (!CP_IN_BOUNDS(base >= 0 && base + D <= p.span_out, p.err)) continue;
    if (p.merge) {
      // fp32 log-sum-exp merge with the accumulator already in (out, lse)
      if (lse_p == nullptr) continue;
      const float a = *lse_p;
      const float nl = a == -INFINITY ? lse_c
                                      : fmaxf(a, lse_c) + log1pf(expf(-fabsf(a - lse_c)));
      const float acc_w = a == -INFINITY ? 0.f : expf(a - nl);
      o_w *= expf(lse_c - nl);
      float* o = reinterpret_cast<float*>(p.out);
#pragma unroll
      for (int i = 0; i < NV; ++i)
        o[base + lane + 32 * i] = fmaf(acc_w, o[base + lane + 32 * i], acc[r][i] * o_w);
      __syncwarp();
      if (lane == 0) *lse_p = nl;
      continue;
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const float o = acc[r][i] * o_w;
      if (p.out_bf16)
        reinterpret_cast<__nv_bfloat16*>(p.out)[base + lane + 32 * i] = __float2bfloat16_rn(o);
      else
        reinterpret_cast<float*>(p.out)[base + lane + 32 * i] = o;
    }
    if (lane == 0 && lse_p != nullptr) *lse_p = lse_c;
  }
}

// out = 0, lse = -inf: the result of attending to no keys at all.
__global__ void fill_empty_kernel(void* out, int out_bf16, long long o_sb, long long o_ss,
                                  long long o_sh, float* lse, long long l_sb, long long l_sh,
                                  long long l_ss, int B, int S, int H, int D, int* err,
                                  long long span_o, long long span_l) {
  const long long n = (long long)B * S * H * D;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int d = (int)(i % D);
    long long r = i / D;
    const int h = (int)(r % H);
    r /= H;
    const int s = (int)(r % S);
    const int b = (int)(r / S);
    const long long o = b * o_sb + s * o_ss + h * o_sh + d;
    if (!CP_IN_BOUNDS(o >= 0 && o < span_o, err)) continue;
    if (out_bf16)
      reinterpret_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(0.f);
    else
      reinterpret_cast<float*>(out)[o] = 0.f;
    const long long lo = b * l_sb + h * l_sh + s * l_ss;
    if (d == 0 && lse != nullptr && CP_IN_BOUNDS(lo >= 0 && lo < span_l, err)) lse[lo] = -INFINITY;
  }
}

}  // namespace

int launch_attn_ring_f32(const RingArgs& a, cudaStream_t stream) {
  F32Params prm;
  memset(&prm, 0, sizeof(prm));
  prm.q = static_cast<const float*>(a.q.data);
  prm.k = static_cast<const float*>(a.k.data);
  prm.v = static_cast<const float*>(a.v.data);
  prm.q_sb = a.q.stride[0];
  prm.q_ss = a.q.stride[1];
  prm.q_sh = a.q.stride[2];
  if (a.k.ndim == 5) {   // [G, B, L, H, D] slots
    prm.k_sg = a.k.stride[0];
    prm.k_sb = a.k.stride[1];
    prm.k_ss = a.k.stride[2];
    prm.k_sh = a.k.stride[3];
    prm.v_sg = a.v.stride[0];
    prm.v_sb = a.v.stride[1];
    prm.v_ss = a.v.stride[2];
    prm.v_sh = a.v.stride[3];
    prm.seg_kv = (int)a.k.shape[2];
  } else {
    prm.k_sb = a.k.stride[0];
    prm.k_ss = a.k.stride[1];
    prm.k_sh = a.k.stride[2];
    prm.v_sb = a.v.stride[0];
    prm.v_ss = a.v.stride[1];
    prm.v_sh = a.v.stride[2];
    prm.k_sg = prm.v_sg = 0;
    prm.seg_kv = (int)a.k.shape[1];
  }
  if (prm.seg_kv <= 0) prm.seg_kv = 1;
  prm.out = a.out.data;
  prm.out_bf16 = a.out.dtype == CP_BF16;
  prm.merge = a.merge ? 1 : 0;
  prm.o_sb = a.out.stride[0];
  prm.o_ss = a.out.stride[1];
  prm.o_sh = a.out.stride[2];
  prm.lse = static_cast<float*>(a.lse.data);
  prm.l_sb = a.lse.stride[0];
  prm.l_sh = a.lse.stride[1];
  prm.l_ss = a.lse.stride[2];
  prm.B = (int)a.q.shape[0];
  prm.S_q = (int)a.q.shape[1];
  prm.H = (int)a.q.shape[2];
  prm.n_row_blocks = (prm.S_q + kRowsPerBlock - 1) / kRowsPerBlock;
  prm.n_chunks = a.n_chunks;
  for (int c = 0; c <= a.n_chunks; ++c) prm.chunk_off[c] = (int)a.chunk_off[c];
  for (int c = 0; c < a.n_chunks; ++c)
    prm.chunk_end[c] = (int)(a.chunk_end ? a.chunk_end[c] : a.chunk_off[c + 1]);
  prm.scale = a.scale;
  prm.err = a.dev_err;
  prm.span_q = span_elems(a.q);
  prm.span_k = span_elems(a.k);
  prm.span_v = span_elems(a.v);
  prm.span_out = span_elems(a.out);
  prm.span_lse = span_elems(a.lse);
  const long long grid = (long long)prm.n_row_blocks * prm.H * prm.B;
  if (grid <= 0) return CP_OK;
  if (grid > 0x7fffffffLL) return CP_ERR_SHAPE;
  const int D = (int)a.q.shape[3];
  if (D == 128)
    attn_ring_f32_kernel<128><<<(int)grid, 128, 0, stream>>>(prm);
  else if (D == 64)
    attn_ring_f32_kernel<64><<<(int)grid, 128, 0, stream>>>(prm);
  else
    return CP_ERR_SHAPE;
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

int launch_fill_empty(const TensorView& out, const TensorView& lse, int* dev_err,
                      cudaStream_t stream) {
  const long long n = out.shape[0] * out.shape[1] * out.shape[2] * out.shape[3];
  if (n <= 0) return CP_OK;
  const int grid = (int)((n + 255) / 256 < 148 * 16 ? (n + 255) / 256 : 148 * 16);
  fill_empty_kernel<<<grid, 256, 0, stream>>>(
      out.data, out.dtype == CP_BF16, out.stride[0], out.stride[1], out.stride[2],
      static_cast<float*>(lse.data), lse.stride[0], lse.stride[1], lse.stride[2],
      (int)out.shape[0], (int)out.shape[1], (int)out.shape[2], (int)out.shape[3], dev_err,
      span_elems(out), span_elems(lse));
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

}  // namespace cpattn
