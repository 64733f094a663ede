// Ring attention on the sm_100a tensor cores (bf16 in, fp32 accumulate).
//
// What it computes (diffusers context-parallelism guide, §Ring Attention and
// §Ring Anything; parallelism API page, ContextParallelConfig.convert_to_fp32):
// the local query block attends to every K/V chunk of the ring in turn; each
// chunk's softmax statistics are folded into one fp32 accumulator at the
// chunk boundary, which is the fp32 log-sum-exp merge of the per-chunk
// partials.  With O kept unnormalised in tensor memory, merging the chunk
// partial (O_c / l_c, m_c + ln l_c) into the running (O / l, m + ln l) is
// the same rescale-and-add the online softmax does inside a chunk, so one
// fp32 accumulator and one (m, l) pair per row carry the whole walk.  K/V
// tiles never straddle a chunk boundary; keys past a chunk's end inside its
// last tile are masked to -inf (that is the Ring Anything trim).
//
// CTA = one work unit: two 128-row query tiles of one (batch, head), so each
// K/V tile brought in by TMA feeds four MMAs.  Warp roles (384 threads):
//   warp 0      TMA producer: Q once, then K_j, V_j into a ring of NST slots
//   warp 1      MMA issuer (one thread): S_t = Q_t K^T, O_t += P_t V
//   warp 2      tensor-memory allocator
//   warps 4-7   softmax + epilogue of query tile 0 (one row per thread)
//   warps 8-11  softmax + epilogue of query tile 1
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   [0,128)   S_0 (fp32), overwritten in place by P_0 (bf16, 64 columns)
//   [128,256) S_1 / P_1
//   [256, 256+D)  O_0;  [256+D, 256+2D)  O_1   (fp32 accumulators)
// MMA order per key tile j (S of tile j+1 is issued as soon as P of tile j
// has been consumed, so one softmax overlaps the other tile's MMAs):
//   O_0 += P_0 V_j ; S_0 = Q_0 K_{j+1}^T ; O_1 += P_1 V_j ; S_1 = Q_1 K_{j+1}^T
// tcgen05 MMAs of one CTA execute in issue order, and a commit arrives only
// when all earlier MMAs are complete, so "S_t ready" also means the previous
// O_t update has landed: the softmax warps may rescale O_t in place then.
// Row statistics are per thread (one TMEM lane = one query row), so the row
// max and row sum need no shuffles at all.
// The softmax rescales lazily: the running max only moves when a tile's max
// exceeds it by more than 8 (log2 units), so P <= 2^8; the final division by
// l uses the same stale max, so the result is exact.

#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace cpattn {

constexpr int kTcThreads = 384;
constexpr int kBlockM = 128;    // query rows per tile
constexpr int kBlockN = 128;    // keys per tile
// Lazy rescaling: the running max m of a row only moves when a tile's max
// exceeds it by more than this many log2 units, so P <= 2^threshold.  P is
// rounded to bf16, whose relative precision does not depend on magnitude;
// the threshold only has to keep the fp32 accumulators finite:
// O <= S_kv * 2^threshold * max|V| and l <= S_kv * 2^threshold.
#ifndef CP_RESCALE_LOG2_THRESHOLD
#define CP_RESCALE_LOG2_THRESHOLD 8
#endif
constexpr float kRescaleThreshold = (float)CP_RESCALE_LOG2_THRESHOLD;
// K/V ring slots (one 128-key tile of K or V each).  Each K/V tile feeds
// two query tiles, so a slot stays busy for most of an iteration; the ring
// must be deep enough that the next K tile is already resident when the
// MMA warp reaches it.
#ifndef CP_TC_STAGES_D128
#define CP_TC_STAGES_D128 4
#endif
constexpr int kStagesD128 = CP_TC_STAGES_D128;   // 64 KB Q + NST x 32 KB
constexpr int kStagesD64 = 6;                    // 32 KB Q + NST x 16 KB
// Register split: the producer/MMA warpgroup gives registers to the two
// softmax warpgroups (80 + 2 * 208 <= 3 * 168 per thread, the launch budget).
constexpr int kRegsControl = 80;
constexpr int kRegsSoftmax = 208;

struct AttnTcParams {
  // 5-D maps {D, seg, H, G, B}: token s of the sequence is row s % seg of
  // segment s / seg.  Plain [B, S, H, D] tensors have one segment (G = 1);
  // Ulysses sequence shards [G, B, S/G, H, D] are read and written in place.
  CUtensorMap tmap_q;   // box {64, 128, 1, 1, 1}, 128B swizzle
  CUtensorMap tmap_k;
  CUtensorMap tmap_v;
  CUtensorMap tmap_out; // box {128 bytes of columns, 128, 1, 1, 1}, 128B swizzle
  void* out;
  float* lse;
  int* err;
  long long l_sb, l_sh, l_ss;    // lse strides (elements)
  int out_bf16;
  int merge;                     // fold this result into (out, lse) instead of overwriting
  int B, H, S_q, S_kv;
  int seg_q, seg_kv;             // tokens per segment (S itself for one segment)
  int n_q_blocks;                // ceil(S_q / 256)
  int n_tiles;                   // key tiles over all chunks
  int n_chunks;
  int G_q, G_kv;                 // segments of q and of k/v
  long long span_lse;            // elements the lse view spans (bounds checks)
  float scale_log2;              // scale * log2(e)
  int chunk_off[CP_MAX_CHUNKS + 1];   // chunk c covers key tokens [chunk_off[c], chunk_end[c])
  int chunk_end[CP_MAX_CHUNKS];
};

// Walks the key tiles chunk by chunk: [start, start+128) clipped to the
// chunk end; empty chunks are skipped.  Chunks need not be adjacent: in a
// padded all-gather buffer the rows between one chunk's end and the next
// chunk's start are padding, never attended.
struct TileWalk {
  int c, start, end;
  __device__ __forceinline__ void skip_empty(const AttnTcParams& p) {
    while (c < p.n_chunks && p.chunk_end[c] <= p.chunk_off[c]) ++c;
    if (c < p.n_chunks) {
      start = p.chunk_off[c];
      end = p.chunk_end[c];
    }
  }
  __device__ __forceinline__ void init(const AttnTcParams& p) {
    c = 0;
    start = end = 0;
    skip_empty(p);
  }
  __device__ __forceinline__ void next(const AttnTcParams& p) {
    start += kBlockN;
    if (start >= end) {
      ++c;
      skip_empty(p);
    }
  }
  __device__ __forceinline__ int valid() const { return min(kBlockN, end - start); }
};

template <int D>
struct TcSmem {
  static constexpr int kTileBytes = 128 * D * 2;   // 128 rows x D bf16
  static constexpr int kHalfBytes = 128 * 64 * 2;  // one 64-column TMA box
};

template <int D, int NST>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_ring_tc_kernel(const __grid_constant__ AttnTcParams p) {
  using L = TcSmem<D>;
  // tensor memory: S_0, S_1 (128 columns each), then O_0, O_1 (D each)
  static_assert(2 * kBlockN + 2 * D <= 512, "tensor memory holds 512 columns");
  static_assert(L::kTileBytes % (128 * 128) == 0, "staging rounds are whole 128x128-byte boxes");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                  // 2 tiles
  uint8_t* sKV = smem + 2 * L::kTileBytes;             // NST slots
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + NST * L::kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + NST;
  uint64_t* s_ready = kv_empty + NST;   // [2]
  uint64_t* p_ready = s_ready + 2;      // [2]
  uint64_t* o_done = p_ready + 2;       // [2]
  uint64_t* epi_full = o_done + 2;      // [2] a round of staged output is in smem
  uint64_t* epi_free = epi_full + 2;    // [2] TMA has read the staged round
  uint64_t* acc_full = epi_free + 2;    // [2] merge mode: the accumulator round is in smem
  uint64_t* drain = acc_full + 2;       // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int unit = blockIdx.x;
  const int qblk = unit % p.n_q_blocks;
  const int hb = unit / p.n_q_blocks;
  const int h = hb % p.H;
  const int b = hb / p.H;
  const int q0 = qblk * 2 * kBlockM;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_ready[t], 1);
      mbar_init(&p_ready[t], kBlockM / 32);   // one arrive per softmax warp
      mbar_init(&o_done[t], 1);
      mbar_init(&epi_full[t], kBlockM / 32);   // one arrive per softmax warp
      mbar_init(&epi_free[t], 1);
      mbar_init(&acc_full[t], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // let the next launch of the stream be scheduled, then wait until the
  // previous grid has finished and its writes are visible (programmatic
  // dependent launch; both are no-ops for an ordinary launch)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp < 4) {
   regs_dec<kRegsControl>();
   if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tmap_q);
      tma_prefetch_desc(&p.tmap_k);
      tma_prefetch_desc(&p.tmap_v);
      bool ok = CP_IN_BOUNDS(q0 < p.S_q && h < p.H && b < p.B, p.err);
      const bool q_issued = ok;
      if (ok) {
        mbar_arrive_expect_tx(q_full, 2 * L::kTileBytes);
        for (int t = 0; t < 2; ++t) {
          const int r0 = q0 + t * kBlockM;
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_5d(sQ + t * L::kTileBytes + hh * L::kHalfBytes, &p.tmap_q, q_full,
                        hh * 64, r0 % p.seg_q, h, r0 / p.seg_q, b);
        }
      } else {
        *abort_flag = 1;
      }
      TileWalk w;
      w.init(p);
      int n_issued = 0;
      for (int n = 0; ok && n < 2 * p.n_tiles; ++n) {
        const int slot = n % NST;
        const int use = n / NST;
        if (use > 0 && !mbar_wait(&kv_empty[slot], (use - 1) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        if (!CP_IN_BOUNDS(w.c < p.n_chunks && w.start >= p.chunk_off[w.c] &&
                              w.start < p.chunk_end[w.c] && w.start / p.seg_kv < p.G_kv,
                          p.err)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&kv_full[slot], L::kTileBytes);
        const CUtensorMap* m = (n & 1) ? &p.tmap_v : &p.tmap_k;
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_5d(sKV + slot * L::kTileBytes + hh * L::kHalfBytes, m, &kv_full[slot],
                      hh * 64, w.start % p.seg_kv, h, w.start / p.seg_kv, b);
        n_issued = n + 1;
        if (n & 1) w.next(p);
      }
      // Let every copy this CTA started land before its shared memory goes.
      if (q_issued) mbar_wait_drain(q_full, 0, p.err);
      if (!ok)
        for (int n = n_issued - NST < 0 ? 0 : n_issued - NST; n < n_issued; ++n)
          mbar_wait_drain(&kv_full[n % NST], (n / NST) & 1, p.err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, D, true);
      const uint32_t sQa = smem_u32(sQ);
      const uint32_t sKVa = smem_u32(sKV);
      // S_t / P_t at columns t*128, O_t at 256 + t*D

      auto issue_s = [&](int t, int slot) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * L::kHalfBytes + (k & 3) * 32;
          const uint64_t ad = smem_desc_sw128(sQa + t * L::kTileBytes + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sKVa + slot * L::kTileBytes + off, 16, 1024);
          mma_bf16_ss(tmem + t * 128, ad, bd, idesc_qk, k > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int slot, bool acc) {
#pragma unroll
        for (int k = 0; k < kBlockN / 16; ++k) {
          const uint64_t bd =
              smem_desc_sw128(sKVa + slot * L::kTileBytes + k * 2048, L::kHalfBytes, 1024);
          mma_bf16_ts(tmem + 256 + t * D, tmem + t * 128 + k * 8, bd, idesc_pv,
                      (acc || k > 0) ? 1u : 0u);
        }
      };
      auto wait_kv = [&](int n) -> bool {
        if (!mbar_wait(&kv_full[n % NST], (n / NST) & 1, abort_flag, p.err)) return false;
        tc_fence_after();
        return true;
      };

      bool ok = mbar_wait(q_full, 0, abort_flag, p.err) && wait_kv(0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        mma_commit(&s_ready[0]);
        issue_s(1, 0);
        mma_commit(&s_ready[1]);
        mma_commit(&kv_empty[0]);
      }
      for (int j = 0; ok && j < p.n_tiles; ++j) {
        const int nv = 2 * j + 1, nk = 2 * j + 2;
        const bool more = j + 1 < p.n_tiles;
        if (!(ok = wait_kv(nv))) break;
        if (!(ok = mbar_wait(&p_ready[0], j & 1, abort_flag, p.err))) break;
        tc_fence_after();
        issue_pv(0, nv % NST, j > 0);
        if (more) {
          if (!(ok = wait_kv(nk))) break;
          issue_s(0, nk % NST);
          mma_commit(&s_ready[0]);
        } else {
          mma_commit(&o_done[0]);
        }
        if (!(ok = mbar_wait(&p_ready[1], j & 1, abort_flag, p.err))) break;
        tc_fence_after();
        issue_pv(1, nv % NST, j > 0);
        mma_commit(&kv_empty[nv % NST]);
        if (more) {
          issue_s(1, nk % NST);
          mma_commit(&s_ready[1]);
          mma_commit(&kv_empty[nk % NST]);
        } else {
          mma_commit(&o_done[1]);
        }
      }
      // Every MMA issued so far must finish before tensor memory is freed.
      mma_commit(drain);
      mbar_wait_drain(drain, 0, p.err);
    }
   }
  } else {
    // ------------------------------------------------------------ softmax
    regs_inc<kRegsSoftmax>();
    const int t = (warp - 4) >> 2;                 // query tile 0 or 1
    const int quarter = warp & 3;                  // TMEM lane quarter
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * 128;
    const uint32_t tO = tmem + lane_base + 256 + t * D;
    const float sl2 = p.scale_log2;

    float m_run = -INFINITY;   // running max, log2 units (scaled)
    float l_run = 0.f;         // running sum of 2^(s*sl2 - m_run)
    bool ok = true;
    TileWalk w;
    w.init(p);
    for (int j = 0; j < p.n_tiles; ++j) {
      if (!(ok = mbar_wait(&s_ready[t], j & 1, abort_flag, p.err))) break;
      tc_fence_after();
      // S in four 32-column chunks: chunk c + 1 is in flight while the row
      // max of chunk c is taken (eight independent max chains)
      float s[kBlockN];
      float mx[8];
      tmem_ld32(tS, s);
      tmem_wait_ld_into(s);
      tmem_ld32(tS + 32, s + 32);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        mx[i] = max3f(s[4 * i], s[4 * i + 1], fmaxf(s[4 * i + 2], s[4 * i + 3]));
#pragma unroll
      for (int c = 1; c < kBlockN / 32; ++c) {
        tmem_wait_ld_into(s + 32 * c);
        if (c + 1 < kBlockN / 32) tmem_ld32(tS + 32 * (c + 1), s + 32 * (c + 1));
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          mx[i] = max3f(mx[i], s[32 * c + 4 * i], s[32 * c + 4 * i + 1]);
          mx[i] = max3f(mx[i], s[32 * c + 4 * i + 2], s[32 * c + 4 * i + 3]);
        }
      }
      const int valid = w.valid();
      if (valid < kBlockN) {
        // a chunk's last tile: columns past the chunk end are masked (rare,
        // so the max is simply taken again over the masked row)
#pragma unroll
        for (int c = 0; c < kBlockN; ++c)
          if (c >= valid) s[c] = -INFINITY;
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = s[i];
#pragma unroll
        for (int c = 8; c < kBlockN; ++c) mx[c & 7] = fmaxf(mx[c & 7], s[c]);
      }
      const float m_tile =
          max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) *
          sl2;
      {
        // Rescale the rows whose max moved beyond the threshold, then
        // exponentiate on the MUFU unit, which maps the masked -inf columns
        // of a tile cut by its chunk's end to exactly 0.
        const bool need = m_tile > m_run + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2_approx(m_run - m_tile) : 1.0f;
          if (need) {
            l_run *= alpha;
            m_run = m_tile;
          }
          if (j > 0) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              float o[32];
              tmem_ld32(tO + c * 32, o);
              tmem_wait_ld_into(o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] *= alpha;
              tmem_st32(tO + c * 32, o);
            }
          }
        }
        const float2 sl2x2 = make_float2(sl2, sl2), nmx2 = make_float2(-m_run, -m_run);
        float2 acc[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int e = c * 32 + 2 * i;
            const float2 x = fma2(make_float2(s[e], s[e + 1]), sl2x2, nmx2);
            const float2 pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            acc[i & 3] = add2(acc[i & 3], pp);
            pk[i] = pack_bf16x2(pp.x, pp.y);
          }
          tmem_st16(tS + c * 16, pk);
        }
        const float2 a01 = add2(acc[0], acc[1]), a23 = add2(acc[2], acc[3]);
        l_run += (a01.x + a01.y) + (a23.x + a23.y);
      }
      if (t == 0 && valid < kBlockN) {
        // Ring Anything trim, V side: a chunk's last tile was loaded whole,
        // and the rows past the chunk end may be padding of any value (a
        // padded all-gather slot).  Their P is exactly 0, but 0 * NaN is
        // NaN in the MMA, so the rows are zeroed in shared memory before
        // P V reads them.  Tile 0's P V is issued first and the slot is not
        // refilled before both tiles have consumed it.
        const int n = 2 * j + 1;
        if (!(ok = mbar_wait(&kv_full[n % NST], (n / NST) & 1, abort_flag, p.err))) break;
        if (row >= valid) {
          uint8_t* vrow = sKV + (n % NST) * L::kTileBytes + row * 128;
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh)
#pragma unroll
            for (int k = 0; k < 8; ++k)
              reinterpret_cast<uint4*>(vrow + hh * L::kHalfBytes)[k] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[t]);
      w.next(p);
    }
    int rounds = 0;   // epilogue rounds staged (phase of epi_full / epi_free)
    if (ok && mbar_wait(&o_done[t], 0, abort_flag, p.err)) {
      tc_fence_after();
      // Epilogue: O / l goes through this tile's Q buffer (idle once o_done
      // fired) in 128-byte swizzled boxes of 128 rows, and leaves with TMA
      // stores; rows past S_q are clipped by the tensor map.  The warps hand
      // the staging buffer to the storing thread and back through bounded
      // mbarrier waits, so a warp that gave up never blocks the others.
      const int s_row = q0 + t * kBlockM + row;
      const float lse_c = (m_run + log2f(l_run)) * 0.69314718055994530942f;
      float o_w = 1.0f / l_run;   // weight of the raw accumulator O
      float acc_w = 0.f;          // merge mode: weight of the (out, lse) already there
      const long long l_off = b * p.l_sb + h * p.l_sh + (long long)s_row * p.l_ss;
      float* lse_p = p.lse != nullptr && s_row < p.S_q &&
                             CP_IN_BOUNDS(l_off >= 0 && l_off < p.span_lse, p.err)
                         ? p.lse + l_off
                         : nullptr;
      if (p.merge) {
        // fp32 log-sum-exp merge with the accumulator (ContextParallelConfig
        // .convert_to_fp32): lse' = max + log1p(exp(-|a - b|))
        const float a = lse_p ? *lse_p : -INFINITY;
        const float mx = fmaxf(a, lse_c);
        const float nl = a == -INFINITY ? lse_c : mx + log1pf(expf(-fabsf(a - lse_c)));
        acc_w = a == -INFINITY ? 0.f : expf(a - nl);
        o_w *= expf(lse_c - nl);
        if (lse_p) *lse_p = nl;
      } else if (lse_p) {
        *lse_p = lse_c;
      }
      const float inv_l = o_w;
      uint8_t* stage = sQ + t * L::kTileBytes;
      const int esz = p.out_bf16 ? 2 : 4;
      const int cols_per_box = 128 / esz;               // 32 fp32 or 64 bf16
      const int boxes = D / cols_per_box;               // per 128-row tile
      const int boxes_per_round = L::kTileBytes / (128 * 128);
      const bool leader = (warp & 3) == 0 && lane == 0;
      for (int b0 = 0; ok && b0 < boxes; b0 += boxes_per_round, ++rounds) {
        // the previous round's TMA stores must have read the staging buffer
        if (rounds > 0 && !(ok = mbar_wait(&epi_free[t], (rounds - 1) & 1, abort_flag, p.err)))
          break;
        const int r0 = q0 + t * kBlockM;
        if (p.merge) {
          // bring this round's accumulator boxes into the staging buffer
          if (leader) {
            mbar_arrive_expect_tx(&acc_full[t], boxes_per_round * (128 * 128));
            for (int bx = b0; bx < b0 + boxes_per_round; ++bx)
              tma_load_5d(stage + (bx - b0) * (128 * 128), &p.tmap_out, &acc_full[t],
                          bx * cols_per_box, r0 % p.seg_q, h, r0 / p.seg_q, b);
          }
          if (!(ok = mbar_wait(&acc_full[t], rounds & 1, abort_flag, p.err))) break;
        }
        for (int bx = b0; bx < b0 + boxes_per_round; ++bx) {
          uint8_t* box = stage + (bx - b0) * (128 * 128) + row * 128;
          // this box holds O columns [bx * cols_per_box, (bx+1) * cols_per_box)
          if (p.merge) {          // fp32 accumulator: out' = acc_w * out + o_w * O
            float o[32];
            tmem_ld32(tO + bx * 32, o);
            tmem_wait_ld_into(o);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              float4* cell = reinterpret_cast<float4*>(box + ((k ^ (row & 7)) << 4));
              const float4 a4 = *cell;
              *cell = make_float4(fmaf(acc_w, a4.x, o[4 * k] * inv_l),
                                  fmaf(acc_w, a4.y, o[4 * k + 1] * inv_l),
                                  fmaf(acc_w, a4.z, o[4 * k + 2] * inv_l),
                                  fmaf(acc_w, a4.w, o[4 * k + 3] * inv_l));
            }
          } else if (p.out_bf16) {
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
              float o[32];
              tmem_ld32(tO + bx * 64 + hlf * 32, o);
              tmem_wait_ld_into(o);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                uint4 v;
                v.x = pack_bf16x2(o[8 * k + 0] * inv_l, o[8 * k + 1] * inv_l);
                v.y = pack_bf16x2(o[8 * k + 2] * inv_l, o[8 * k + 3] * inv_l);
                v.z = pack_bf16x2(o[8 * k + 4] * inv_l, o[8 * k + 5] * inv_l);
                v.w = pack_bf16x2(o[8 * k + 6] * inv_l, o[8 * k + 7] * inv_l);
                const int chunk = hlf * 4 + k;
                *reinterpret_cast<uint4*>(box + ((chunk ^ (row & 7)) << 4)) = v;
              }
            }
          } else {
            float o[32];
            tmem_ld32(tO + bx * 32, o);
            tmem_wait_ld_into(o);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              *reinterpret_cast<float4*>(box + ((k ^ (row & 7)) << 4)) =
                  make_float4(o[4 * k] * inv_l, o[4 * k + 1] * inv_l, o[4 * k + 2] * inv_l,
                              o[4 * k + 3] * inv_l);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&epi_full[t]);
        if (leader) {
          if (!(ok = mbar_wait(&epi_full[t], rounds & 1, abort_flag, p.err))) break;
          for (int bx = b0; bx < b0 + boxes_per_round; ++bx)
            tma_store_5d(&p.tmap_out, stage + (bx - b0) * (128 * 128), bx * cols_per_box,
                         r0 % p.seg_q, h, r0 / p.seg_q, b);
          bulk_commit();
          bulk_wait_read_all();
          mbar_arrive(&epi_free[t]);
        }
      }
    }
    // shared memory must not be released while TMA still reads it
    if (rounds > 0) mbar_wait_drain(&epi_free[t], (rounds - 1) & 1, p.err);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// The five extents/strides of a [B, S, H, D] view (one segment) or of a
// [G, B, S/G, H, D] shard view, as {D, seg, H, G, B}; strides in bytes of
// dims 1..4.
void seg_geometry(const TensorView& t, cuuint64_t dims[5], cuuint64_t strides[4]) {
  const cuuint64_t es = dtype_size(t.dtype);
  if (t.ndim == 4) {
    dims[0] = t.shape[3]; dims[1] = t.shape[1]; dims[2] = t.shape[2]; dims[3] = 1;
    dims[4] = t.shape[0];
    strides[0] = t.stride[1] * es; strides[1] = t.stride[2] * es;
    strides[2] = t.stride[1] * es * (t.shape[1] > 0 ? t.shape[1] : 1);
    strides[3] = t.stride[0] * es;
  } else {
    dims[0] = t.shape[4]; dims[1] = t.shape[2]; dims[2] = t.shape[3]; dims[3] = t.shape[0];
    dims[4] = t.shape[1];
    strides[0] = t.stride[2] * es; strides[1] = t.stride[3] * es; strides[2] = t.stride[0] * es;
    strides[3] = t.stride[1] * es;
  }
}

// bf16 q/k/v -> 5-D map, box {64, 128, 1, 1, 1}, 128B swizzle.
int encode_in(CUtensorMap* map, const TensorView& t) {
  auto fn = get_encode_fn();
  if (!fn) return CP_ERR_CUDA;
  cuuint64_t dims[5], strides[4];
  seg_geometry(t, dims, strides);
  const cuuint32_t box[5] = {64, 128, 1, 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, t.data, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CP_OK : CP_ERR_CUDA;
}

// Output (f32 or bf16) -> 5-D map with 128-byte, 128-row boxes.
int encode_out(CUtensorMap* map, const TensorView& t) {
  auto fn = get_encode_fn();
  if (!fn) return CP_ERR_CUDA;
  const int es = dtype_size(t.dtype);
  cuuint64_t dims[5], strides[4];
  seg_geometry(t, dims, strides);
  const cuuint32_t box[5] = {(cuuint32_t)(128 / es), 128, 1, 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, t.dtype == CP_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                          : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  5, t.data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CP_OK : CP_ERR_CUDA;
}

template <int D, int NST>
int launch_tc(const AttnTcParams& prm, int grid, cudaStream_t stream) {
  constexpr size_t smem = 1024 + (2 + NST) * (size_t)TcSmem<D>::kTileBytes + 256;
  auto kern = attn_ring_tc_kernel<D, NST>;
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CP_ERR_CUDA;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return CP_ERR_CUDA;
    configured[dev] = true;
  }
  // Programmatic dependent launch: the kernel may be scheduled while the
  // previous kernel of the stream drains; it waits for that grid (and its
  // memory) before touching global memory, so only its set-up overlaps.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, prm) != cudaSuccess) return CP_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

}  // namespace

int launch_attn_ring_tc(const RingArgs& a, cudaStream_t stream) {
  AttnTcParams prm;
  memset(&prm, 0, sizeof(prm));
  int st;
  if ((st = encode_in(&prm.tmap_q, a.q)) != CP_OK) return st;
  if ((st = encode_in(&prm.tmap_k, a.k)) != CP_OK) return st;
  if ((st = encode_in(&prm.tmap_v, a.v)) != CP_OK) return st;
  if ((st = encode_out(&prm.tmap_out, a.out)) != CP_OK) return st;
  prm.out = a.out.data;
  prm.out_bf16 = a.out.dtype == CP_BF16;
  prm.merge = a.merge ? 1 : 0;
  prm.lse = static_cast<float*>(a.lse.data);
  prm.l_sb = a.lse.stride[0];
  prm.l_sh = a.lse.stride[1];
  prm.l_ss = a.lse.stride[2];
  prm.err = a.dev_err;
  prm.G_q = a.q.ndim == 5 ? (int)a.q.shape[0] : 1;
  prm.G_kv = a.k.ndim == 5 ? (int)a.k.shape[0] : 1;
  prm.span_lse = span_elems(a.lse);
  if (a.q.ndim == 5) {   // [G, B, S/G, H, D] shards, read in place
    prm.B = (int)a.q.shape[1];
    prm.seg_q = (int)a.q.shape[2];
    prm.S_q = (int)(a.q.shape[0] * a.q.shape[2]);
    prm.H = (int)a.q.shape[3];
  } else {
    prm.B = (int)a.q.shape[0];
    prm.S_q = prm.seg_q = (int)a.q.shape[1];
    prm.H = (int)a.q.shape[2];
  }
  if (a.k.ndim == 5) {   // [G, B, L, H, D]: shards, or the slots of a padded all-gather
    prm.seg_kv = (int)a.k.shape[2];
    prm.S_kv = (int)(a.k.shape[0] * a.k.shape[2]);
  } else {
    prm.S_kv = prm.seg_kv = (int)a.k.shape[1];
  }
  if (prm.seg_q <= 0) prm.seg_q = 1;
  if (prm.seg_kv <= 0) prm.seg_kv = 1;
  prm.n_q_blocks = (prm.S_q + 2 * kBlockM - 1) / (2 * kBlockM);
  prm.n_chunks = a.n_chunks;
  int n_tiles = 0;
  for (int c = 0; c <= a.n_chunks; ++c) prm.chunk_off[c] = (int)a.chunk_off[c];
  for (int c = 0; c < a.n_chunks; ++c) {
    prm.chunk_end[c] = (int)(a.chunk_end ? a.chunk_end[c] : a.chunk_off[c + 1]);
    const int len = prm.chunk_end[c] - prm.chunk_off[c];
    if (len > 0) n_tiles += (len + kBlockN - 1) / kBlockN;
  }
  prm.n_tiles = n_tiles;
  prm.scale_log2 = a.scale * 1.4426950408889634f;
  const long long grid = (long long)prm.n_q_blocks * prm.H * prm.B;
  if (grid <= 0 || n_tiles <= 0) return CP_OK;
  if (grid > 0x7fffffffLL) return CP_ERR_SHAPE;
  const int D = (int)a.q.shape[a.q.ndim - 1];
  if (D == 128) return launch_tc<128, kStagesD128>(prm, (int)grid, stream);
  if (D == 64) return launch_tc<64, kStagesD64>(prm, (int)grid, stream);
  return CP_ERR_SHAPE;
}

}  // namespace cpattn
