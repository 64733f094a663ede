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
// Work unit = two 128-row query tiles of one (batch, head), so each K/V
// tile brought in by TMA feeds four MMAs.  The grid is persistent: one CTA
// per SM walks the units round-robin, and the K/V ring, the barriers and
// tensor memory carry on from one unit to the next, so the next unit's Q
// and K/V loads and its first S MMAs overlap the previous unit's last tiles
// and epilogue.  Warp roles (384 threads):
//   warp 0      TMA producer: per unit Q (once the previous unit's last S
//               MMAs have read the Q buffer), then K_j, V_j into a ring of
//               NST slots
//   warp 1      MMA issuer (lane 0): S_t = Q_t K^T, O_t += P_t V; the
//               first P V of a unit waits until the previous unit's epilogue
//               has read O_t out of tensor memory
//   warp 2      tensor-memory allocator, then the watchdog of the P barriers
//   warps 4-7   softmax + epilogue of query tile 0 (one row per thread)
//   warps 8-11  softmax + epilogue of query tile 1
// The softmax warps publish P_t on a hardware named barrier (arrive) that
// the MMA warp syncs on.  A shared-memory signal (an mbarrier or a flag)
// would be observed late: the MMA warp's polls queue behind the softmax
// warps' MUFU instructions on the same sub-partition (~150-250 clocks per
// poll, measured).  Every other hand-off uses mbarriers with bounded waits.
// Epilogue, per warp and its 32 rows: O in rounds of 128 bytes of columns
// from tensor memory, scaled (or, for the fp32 accumulator, merged with the
// box the same warp TMA-loads), staged in the warp's own 4 KB of shared
// memory in the 128-byte swizzled layout and written by one 32-row TMA
// store; the store's read of the staging area overlaps the next round.
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

#include <atomic>
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
// softmax warpgroups (72 + 2 * 216 = 3 * 168 per thread, the launch budget);
// at this split neither role spills.
constexpr int kRegsControl = 72;
constexpr int kRegsSoftmax = 216;
// Named barriers on which P_t is published: id 1 + t, the four softmax warps
// of query tile t (arrive) and the MMA warp (sync).
constexpr uint32_t kPBarBase = 1;
constexpr uint32_t kPBarThreads = (kBlockM / 32 + 1) * 32;

struct AttnTcParams {
  // 5-D maps {D, seg, H, G, B}: token s of the sequence is row s % seg of
  // segment s / seg.  Plain [B, S, H, D] tensors have one segment (G = 1);
  // Ulysses sequence shards [G, B, S/G, H, D] are read and written in place.
  CUtensorMap tmap_q;   // box {64, 128, 1, 1, 1}, 128B swizzle
  CUtensorMap tmap_k;
  CUtensorMap tmap_v;
  CUtensorMap tmap_out; // box {128 bytes of columns, 128, 1, 1, 1}, 128B swizzle
  CUtensorMap tmap_out32; // same, 32-row boxes: one warp's rows of one epilogue round
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
  int n_units;                   // work units (2 query tiles of one batch, head)
  unsigned int* unit_ctr;        // [2]: next unit to hand out, CTAs done (reset by the last)
  long long o_sg, o_sb, o_ss, o_sh;   // out strides (elements); token s is row s % seg_q
  long long span_out;            // elements the out view spans (bounds checks)
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

// tcgen05 MMAs whose shared-memory descriptors are formed inside the asm
// statement: the 32-bit low word (start address >> 4 | LBO >> 4 << 16) is a
// base register plus an immediate, the high word (SBO, version, 128-byte
// swizzle) an immediate.  The compiler cannot hoist 64-bit descriptors out of
// the loop, which keeps the issuing thread's register footprint small.
constexpr uint32_t kDescHi = (uint32_t)((1024u >> 4) | (1u << 14) | (2u << 29));   // bits 32..63
__device__ __forceinline__ uint32_t desc_lo(uint32_t saddr, uint32_t lbo_bytes) {
  return ((saddr >> 4) & 0x3FFFu) | ((lbo_bytes >> 4) << 16);
}
template <uint32_t AOFF, uint32_t BOFF>
__device__ __forceinline__ void mma_ss_lo(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b32 al, bl;\n\t.reg .b64 ad, bd;\n\t"
      "add.u32 al, %1, %5;\n\tadd.u32 bl, %2, %6;\n\t"
      "mov.b64 ad, {al, %7};\n\tmov.b64 bd, {bl, %7};\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "n"(AOFF), "n"(BOFF), "n"(kDescHi)
      : "memory");
}
template <uint32_t BOFF>
__device__ __forceinline__ void mma_ts_lo(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b32 bl;\n\t.reg .b64 bd;\n\t"
      "add.u32 bl, %2, %5;\n\tmov.b64 bd, {bl, %6};\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(idesc), "r"(accumulate), "n"(BOFF), "n"(kDescHi)
      : "memory");
}

// Pull a tensor box into L2 (no shared-memory destination, no completion).
__device__ __forceinline__ void tma_prefetch_l2_5d(const CUtensorMap* map, int c0, int c1,
                                                   int c2, int c3, int c4) {
  asm volatile("cp.async.bulk.prefetch.tensor.5d.L2.global [%0, {%1, %2, %3, %4, %5}];" ::"l"(map),
               "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
               : "memory");
}

template <int D, int NST>
struct PersistSmem {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kStageBytes = 32 * 128;              // per warp: 32 rows x 128 B
  static constexpr int kStageOff = (2 + NST) * kTileBytes;
  static constexpr int kBarOff = kStageOff + 8 * kStageBytes;
  static constexpr size_t kBytes = 1024 + (size_t)kBarOff + 512;
};

template <int D, int NST>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_ring_tc_kernel(const __grid_constant__ AttnTcParams p) {
  using L = TcSmem<D>;
  using PS = PersistSmem<D, NST>;
  static_assert(2 * kBlockN + 2 * D <= 512, "tensor memory holds 512 columns");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                  // 2 tiles
  uint8_t* sKV = smem + 2 * L::kTileBytes;             // NST slots
  uint8_t* sStage = smem + PS::kStageOff;              // 8 warps x 4 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PS::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* q_free = bars + 1;          // the unit's last S MMAs are done: Q may be replaced
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = kv_full + NST;
  uint64_t* s_ready = kv_empty + NST;   // [2]
  uint64_t* o_done = s_ready + 2;       // [2]
  uint64_t* o_free = o_done + 2;        // [2] the epilogue has read O_t out of tensor memory
  uint64_t* drain = o_free + 2;         // [1]
  uint64_t* acc_bar = drain + 1;        // [8] merge mode: a warp's accumulator box is in staging
  uint64_t* unit_full = acc_bar + 8;    // [2] the unit index of slot k & 1 is published
  uint64_t* unit_free = unit_full + 2;  // [2] every role has read it
  int* unit_ring_raw = reinterpret_cast<int*>(unit_free + 2);   // [2] published unit indices
  volatile int* unit_ring = unit_ring_raw;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(unit_ring_raw + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* mma_exited = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_free, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_ready[t], 1);
      mbar_init(&o_done[t], 1);
      mbar_init(&o_free[t], kBlockM / 32);    // one arrive per softmax warp
    }
    mbar_init(drain, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&unit_full[i], 1);
      mbar_init(&unit_free[i], 1 + 8);   // the MMA thread and the eight softmax warps
    }
    for (int i = 0; i < 8; ++i) mbar_init(&acc_bar[i], 1);
    *abort_flag = 0;
    *mma_exited = 0;
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
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // unit u -> (batch, head, first query row); units run round-robin over CTAs
  auto decode = [&](int u, int& b, int& h, int& q0) {
    const int qblk = u % p.n_q_blocks;
    const int hb = u / p.n_q_blocks;
    h = hb % p.H;
    b = hb / p.H;
    q0 = qblk * 2 * kBlockM;
  };
  const int tiles2 = 2 * p.n_tiles;   // K/V tile loads per unit

  if (warp < 4) {
   regs_dec<kRegsControl>();
   if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tmap_q);
      tma_prefetch_desc(&p.tmap_k);
      tma_prefetch_desc(&p.tmap_v);
      bool ok = true;
      int n = 0;          // K/V tile loads issued, over all units
      int q_loads = 0;
      for (int k = 0;; ++k) {
        // the next unit: handed out in index order to whichever CTA asks
        // first, once this CTA's previous unit no longer needs its Q buffer
        if (k > 0 && !(ok = mbar_wait(q_free, (k - 1) & 1, abort_flag, p.err))) break;
        int u = (int)atomicAdd(&p.unit_ctr[0], 1u);
        if (u >= p.n_units) u = -1;
        if (k >= 2 && !(ok = mbar_wait(&unit_free[k & 1], ((k >> 1) - 1) & 1, abort_flag, p.err)))
          break;
        unit_ring[k & 1] = u;
        mbar_arrive(&unit_full[k & 1]);
        if (u < 0) break;
        int b, h, q0;
        decode(u, b, h, q0);
        if (!(ok = CP_IN_BOUNDS(q0 < p.S_q && h < p.H && b < p.B, p.err))) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(q_full, 2 * L::kTileBytes);
        for (int t = 0; t < 2; ++t) {
          const int r0 = q0 + t * kBlockM;
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_5d(sQ + t * L::kTileBytes + hh * L::kHalfBytes, &p.tmap_q, q_full,
                        hh * 64, r0 % p.seg_q, h, r0 / p.seg_q, b);
        }
        ++q_loads;
        TileWalk w;
        w.init(p);
        for (int i = 0; i < tiles2; ++i) {
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
          const CUtensorMap* m = (i & 1) ? &p.tmap_v : &p.tmap_k;
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_5d(sKV + slot * L::kTileBytes + hh * L::kHalfBytes, m, &kv_full[slot],
                        hh * 64, w.start % p.seg_kv, h, w.start / p.seg_kv, b);
          ++n;
          if (i & 1) w.next(p);
        }
      }
      // Every fetch of this CTA is done: count it, and the last CTA resets
      // the counters for the next launch that uses them.
      if (atomicAdd(&p.unit_ctr[1], 1u) == gridDim.x - 1) {
        atomicExch(&p.unit_ctr[0], 0u);
        atomicExch(&p.unit_ctr[1], 0u);
      }
      // Let every copy this CTA started land before its shared memory goes.
      if (q_loads > 0) mbar_wait_drain(q_full, (q_loads - 1) & 1, p.err);
      for (int i = n - NST < 0 ? 0 : n - NST; i < n; ++i)
        mbar_wait_drain(&kv_full[i % NST], (i / NST) & 1, p.err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Lane 0 waits on the mbarriers and issues; the whole warp takes part in
    // the named barriers on which P is published, so every branch below is
    // taken by the whole warp with lane 0's outcome.
    constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN, false);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, D, true);
    const uint32_t sQa = smem_u32(sQ);
    const uint32_t sKVa = smem_u32(sKV);
    // descriptor low words: start address (16-byte units) | LBO << 16; the
    // k-steps of one MMA group add compile-time offsets to one base
    auto issue_s = [&](int t, int slot) {
      const uint32_t a0 = desc_lo(sQa + t * L::kTileBytes, 16);
      const uint32_t b0 = desc_lo(sKVa + slot * L::kTileBytes, 16);
      const uint32_t d = tmem + t * 128;
      mma_ss_lo<0, 0>(d, a0, b0, idesc_qk, 0u);
      mma_ss_lo<2, 2>(d, a0, b0, idesc_qk, 1u);
      mma_ss_lo<4, 4>(d, a0, b0, idesc_qk, 1u);
      mma_ss_lo<6, 6>(d, a0, b0, idesc_qk, 1u);
      if constexpr (D == 128) {
        constexpr uint32_t H = L::kHalfBytes >> 4;
        mma_ss_lo<H + 0, H + 0>(d, a0, b0, idesc_qk, 1u);
        mma_ss_lo<H + 2, H + 2>(d, a0, b0, idesc_qk, 1u);
        mma_ss_lo<H + 4, H + 4>(d, a0, b0, idesc_qk, 1u);
        mma_ss_lo<H + 6, H + 6>(d, a0, b0, idesc_qk, 1u);
      }
    };
    auto issue_pv = [&](int t, int slot, bool acc) {
      const uint32_t b0 = desc_lo(sKVa + slot * L::kTileBytes, L::kHalfBytes);
      const uint32_t d = tmem + 256 + t * D;
      const uint32_t a = tmem + t * 128;
      const uint32_t a1 = acc ? 1u : 0u;
      mma_ts_lo<0 * 128>(d, a + 0, b0, idesc_pv, a1);
      mma_ts_lo<1 * 128>(d, a + 8, b0, idesc_pv, 1u);
      mma_ts_lo<2 * 128>(d, a + 16, b0, idesc_pv, 1u);
      mma_ts_lo<3 * 128>(d, a + 24, b0, idesc_pv, 1u);
      mma_ts_lo<4 * 128>(d, a + 32, b0, idesc_pv, 1u);
      mma_ts_lo<5 * 128>(d, a + 40, b0, idesc_pv, 1u);
      mma_ts_lo<6 * 128>(d, a + 48, b0, idesc_pv, 1u);
      mma_ts_lo<7 * 128>(d, a + 56, b0, idesc_pv, 1u);
    };
    auto wait_kv = [&](int n) -> bool {
      if (!mbar_wait(&kv_full[n % NST], (n / NST) & 1, abort_flag, p.err)) return false;
      tc_fence_after();
      return true;
    };
    auto warp_ok = [&](bool v) { return __shfl_sync(0xffffffffu, v ? 1 : 0, 0) != 0; };
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int u = -1;
      if (lane == 0) {
        ok = mbar_wait(&unit_full[k & 1], (k >> 1) & 1, abort_flag, p.err);
        if (ok) {
          u = unit_ring[k & 1];
          mbar_arrive(&unit_free[k & 1]);
        }
      }
      ok = warp_ok(ok);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (!ok || u < 0) break;
      const int c0 = k * tiles2;   // this unit's first K/V load
      if (lane == 0) {
        ok = mbar_wait(q_full, k & 1, abort_flag, p.err) && wait_kv(c0);
        if (ok) {
          issue_s(0, c0 % NST);
          mma_commit(&s_ready[0]);
          issue_s(1, c0 % NST);
          mma_commit(&s_ready[1]);
          mma_commit(&kv_empty[c0 % NST]);
          if (p.n_tiles == 1) mma_commit(q_free);
        }
      }
      ok = warp_ok(ok);
      for (int j = 0; ok && j < p.n_tiles; ++j) {
        const int nv = c0 + 2 * j + 1, nk = c0 + 2 * j + 2;
        const bool more = j + 1 < p.n_tiles;
        if (lane == 0) ok = wait_kv(nv);
        if (!(ok = warp_ok(ok))) break;
        named_sync(kPBarBase + 0, kPBarThreads);   // the tile-0 softmax warps published P_0
        if (lane == 0) {
          // the previous unit's epilogue must have read O_0 before it is overwritten
          if (j == 0 && k > 0) ok = mbar_wait(&o_free[0], (k - 1) & 1, abort_flag, p.err);
          if (ok) {
            tc_fence_after();
            issue_pv(0, nv % NST, j > 0);
            if (more) {
              ok = wait_kv(nk);
              if (ok) {
                issue_s(0, nk % NST);
                mma_commit(&s_ready[0]);
              }
            } else {
              mma_commit(&o_done[0]);
            }
          }
        }
        if (!(ok = warp_ok(ok))) break;
        named_sync(kPBarBase + 1, kPBarThreads);   // P_1 published
        if (lane == 0) {
          if (j == 0 && k > 0) ok = mbar_wait(&o_free[1], (k - 1) & 1, abort_flag, p.err);
          if (ok) {
            tc_fence_after();
            issue_pv(1, nv % NST, j > 0);
            mma_commit(&kv_empty[nv % NST]);
            if (more) {
              issue_s(1, nk % NST);
              mma_commit(&s_ready[1]);
              mma_commit(&kv_empty[nk % NST]);
              if (j + 2 == p.n_tiles) mma_commit(q_free);   // the unit's last S MMAs
            } else {
              mma_commit(&o_done[1]);
            }
          }
        }
        ok = warp_ok(ok);
      }
    }
    if (lane == 0) {
      *mma_exited = 1;
      // Every MMA issued so far must finish before tensor memory is freed.
      mma_commit(drain);
      mbar_wait_drain(drain, 0, p.err);
    }
    __syncwarp();
   } else if (warp == 2) {
    // ------------------------------------------------------------ watchdog
    // The MMA warp's named-barrier syncs have no time limit.  A softmax warp
    // stops arriving only after a bounded wait has failed, which raises the
    // abort flag first; from then on this warp arrives on both P barriers
    // every microsecond, releasing any sync the softmax warps no longer
    // serve, until the MMA warp has left its loop (all its other waits are
    // bounded and return at once once the flag is up).
    const uint64_t t0 = globaltimer_ns();
    uint64_t t_abort = 0;
    for (;;) {
      int state = 0;
      if (lane == 0) state = (*mma_exited ? 1 : 0) | (*abort_flag ? 2 : 0);
      state = __shfl_sync(0xffffffffu, state, 0);
      if (state & 1) break;
      const uint64_t now = globaltimer_ns();
      if (state & 2) {
        if (t_abort == 0) t_abort = now;
        named_arrive(kPBarBase + 0, kPBarThreads);
        named_arrive(kPBarBase + 1, kPBarThreads);
        if (now - t_abort > 4 * kWaitTimeoutNs) break;
      }
      if (now - t0 > 64 * kWaitTimeoutNs) break;
      __nanosleep(1000);
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
    uint8_t* stage = sStage + (warp - 4) * PS::kStageBytes;   // this warp's 32 x 128 B
    bool ok = true;
    for (int k = 0; ok; ++k) {
      if (!(ok = mbar_wait(&unit_full[k & 1], (k >> 1) & 1, abort_flag, p.err))) break;
      const int u = unit_ring[k & 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(&unit_free[k & 1]);
      if (u < 0) break;
      float m_run = -INFINITY;   // running max, log2 units (scaled)
      float l_run = 0.f;         // running sum of 2^(s*sl2 - m_run)
      TileWalk w;
      w.init(p);
      for (int j = 0; j < p.n_tiles; ++j) {
        const int js = k * p.n_tiles + j;   // key-tile step over all units
        if (!(ok = mbar_wait(&s_ready[t], js & 1, abort_flag, p.err))) break;
        if (p.merge && j == 0 && lane == 0) {
          // the accumulator rows this warp merges into at the end of the unit
          int b, h, q0;
          decode(u, b, h, q0);
          const int r0w = q0 + t * kBlockM + quarter * 32;
          for (int c = 0; c < D / 32; ++c)
            tma_prefetch_l2_5d(&p.tmap_out32, c * 32, r0w % p.seg_q, h, r0w / p.seg_q, b);
        }
        tc_fence_after();
        // S in one round trip: four 32-column loads behind one wait (the
        // load latency, not the bandwidth, is what a per-chunk wait exposes),
        // then the row max in eight independent chains
        float s[kBlockN];
        float mx[8];
        tmem_ld32(tS, s);
        tmem_ld32(tS + 32, s + 32);
        tmem_ld32(tS + 64, s + 64);
        tmem_ld32(tS + 96, s + 96);
        tmem_wait_ld_into(s);
        tmem_tie32(s + 32);
        tmem_tie32(s + 64);
        tmem_tie32(s + 96);
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = s[i];
#pragma unroll
        for (int c = 8; c < kBlockN; ++c) mx[c & 7] = fmaxf(mx[c & 7], s[c]);
        const int valid = w.valid();
        if (valid < kBlockN) {
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
          const int n = k * tiles2 + 2 * j + 1;
          if (!(ok = mbar_wait(&kv_full[n % NST], (n / NST) & 1, abort_flag, p.err))) break;
          if (row >= valid) {
            uint8_t* vrow = sKV + (n % NST) * L::kTileBytes + row * 128;
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh)
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                reinterpret_cast<uint4*>(vrow + hh * L::kHalfBytes)[kk] = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        named_arrive(kPBarBase + t, kPBarThreads);   // P_t of this warp is in tensor memory
        w.next(p);
      }
      if (!ok) break;
      int b, h, q0;
      decode(u, b, h, q0);
      const int r0w = q0 + t * kBlockM + quarter * 32;     // first row of this warp
      if (!(ok = mbar_wait(&o_done[t], k & 1, abort_flag, p.err))) break;
      tc_fence_after();
      // ---- epilogue, per warp (its 32 rows), in rounds of 128 bytes of
      // columns: O from tensor memory, scaled (and merged) into the warp's
      // 4 KB staging area in the 128-byte swizzled layout, stored with one
      // 32-row TMA box.  The staging area is reused once the previous
      // round's store has read it.
      const int s_row = q0 + t * kBlockM + row;
      const float lse_c = (m_run + log2f(l_run)) * 0.69314718055994530942f;
      float o_w = 1.0f / l_run;
      float acc_w = 0.f;
      const long long l_off = b * p.l_sb + h * p.l_sh + (long long)s_row * p.l_ss;
      float* lse_p = p.lse != nullptr && s_row < p.S_q &&
                             CP_IN_BOUNDS(l_off >= 0 && l_off < p.span_lse, p.err)
                         ? p.lse + l_off
                         : nullptr;
      if (p.merge) {
        const float a = lse_p ? *lse_p : -INFINITY;
        const float mx = fmaxf(a, lse_c);
        const float nl = a == -INFINITY ? lse_c : mx + log1pf(expf(-fabsf(a - lse_c)));
        acc_w = a == -INFINITY ? 0.f : expf(a - nl);
        o_w *= expf(lse_c - nl);
        if (lse_p) *lse_p = nl;
      } else if (lse_p) {
        *lse_p = lse_c;
      }
      const int c1 = r0w % p.seg_q, c3 = r0w / p.seg_q;    // its TMA row / segment coordinates
      uint8_t* cell_row = stage + lane * 128;
      // the previous round's store must have read the staging area before it
      // is written again (the wait overlaps this round's TMEM load and math)
      auto staging_free = [&]() {
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
      };
      auto store_box = [&](int col0) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_5d(&p.tmap_out32, stage, col0, c1, h, c3, b);
          bulk_commit();
        }
      };
      if (p.merge) {
        // per round: the accumulator box (already pulled into L2 when the
        // unit started) into the staging area, merged with O in place, stored
        uint64_t* abar = &acc_bar[warp - 4];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          staging_free();
          if (lane == 0) {
            mbar_arrive_expect_tx(abar, 32 * 128);
            tma_load_5d(stage, &p.tmap_out32, abar, c * 32, c1, h, c3, b);
          }
          float o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld_into(o);
          if (c == D / 32 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_free[t]);
          }
          if (!(ok = mbar_wait(abar, (k * (D / 32) + c) & 1, abort_flag, p.err))) break;
#pragma unroll
          for (int kq = 0; kq < 8; ++kq) {
            float4* cell = reinterpret_cast<float4*>(cell_row + ((kq ^ (lane & 7)) << 4));
            const float4 a4 = *cell;
            *cell = make_float4(fmaf(acc_w, a4.x, o[4 * kq] * o_w),
                                fmaf(acc_w, a4.y, o[4 * kq + 1] * o_w),
                                fmaf(acc_w, a4.z, o[4 * kq + 2] * o_w),
                                fmaf(acc_w, a4.w, o[4 * kq + 3] * o_w));
          }
          store_box(c * 32);
        }
        if (!ok) break;
      } else if (p.out_bf16) {
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
#pragma unroll
          for (int hlf = 0; hlf < 2; ++hlf) {
            float o[32];
            tmem_ld32(tO + c * 64 + hlf * 32, o);
            tmem_wait_ld_into(o);
            if (c == D / 64 - 1 && hlf == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&o_free[t]);
            }
            if (hlf == 0) staging_free();
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
              uint4 v;
              v.x = pack_bf16x2(o[8 * kq + 0] * o_w, o[8 * kq + 1] * o_w);
              v.y = pack_bf16x2(o[8 * kq + 2] * o_w, o[8 * kq + 3] * o_w);
              v.z = pack_bf16x2(o[8 * kq + 4] * o_w, o[8 * kq + 5] * o_w);
              v.w = pack_bf16x2(o[8 * kq + 6] * o_w, o[8 * kq + 7] * o_w);
              const int chunk = hlf * 4 + kq;
              *reinterpret_cast<uint4*>(cell_row + ((chunk ^ (lane & 7)) << 4)) = v;
            }
          }
          store_box(c * 64);
        }
      } else {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld_into(o);
          if (c == D / 32 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_free[t]);
          }
          staging_free();
#pragma unroll
          for (int kq = 0; kq < 8; ++kq)
            *reinterpret_cast<float4*>(cell_row + ((kq ^ (lane & 7)) << 4)) =
                make_float4(o[4 * kq] * o_w, o[4 * kq + 1] * o_w, o[4 * kq + 2] * o_w,
                            o[4 * kq + 3] * o_w);
          store_box(c * 32);
        }
      }
    }
    // shared memory must not be released while TMA still reads it
    if (lane == 0) bulk_wait_read_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host side
// Work counters of the persistent grid: kUnitSlots pairs per device (next
// unit, CTAs done), zero between launches.  Launches take the pairs in turn,
// so launches in flight at the same time on different streams use different
// pairs unless more than kUnitSlots of them overlap.
constexpr int kUnitSlots = 64;
__device__ unsigned int g_unit_counters[2 * kUnitSlots];

namespace {

unsigned int* unit_counters(int dev) {
  static std::atomic<unsigned int*> addr[64];
  unsigned int* a = addr[dev].load(std::memory_order_acquire);
  if (!a) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_unit_counters) != cudaSuccess) return nullptr;
    a = static_cast<unsigned int*>(p);
    addr[dev].store(a, std::memory_order_release);
  }
  return a;
}


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
int encode_out(CUtensorMap* map, const TensorView& t, int box_rows = 128) {
  auto fn = get_encode_fn();
  if (!fn) return CP_ERR_CUDA;
  const int es = dtype_size(t.dtype);
  cuuint64_t dims[5], strides[4];
  seg_geometry(t, dims, strides);
  const cuuint32_t box[5] = {(cuuint32_t)(128 / es), (cuuint32_t)box_rows, 1, 1, 1};
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
  constexpr size_t smem = PersistSmem<D, NST>::kBytes;
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
  if ((st = encode_out(&prm.tmap_out32, a.out, 32)) != CP_OK) return st;
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
  prm.span_out = span_elems(a.out);
  if (a.out.ndim == 5) {
    prm.o_sg = a.out.stride[0];
    prm.o_sb = a.out.stride[1];
    prm.o_ss = a.out.stride[2];
    prm.o_sh = a.out.stride[3];
  } else {
    prm.o_sg = 0;
    prm.o_sb = a.out.stride[0];
    prm.o_ss = a.out.stride[1];
    prm.o_sh = a.out.stride[2];
  }
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
  const long long units = (long long)prm.n_q_blocks * prm.H * prm.B;
  if (units <= 0 || n_tiles <= 0) return CP_OK;
  if (units > 0x7fffffffLL) return CP_ERR_SHAPE;
  prm.n_units = (int)units;
  // persistent: one CTA per SM walks the units round-robin
  static int sm_count[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CP_ERR_CUDA;
  if (sm_count[dev] == 0 &&
      cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return CP_ERR_CUDA;
  const long long grid = units < sm_count[dev] ? units : sm_count[dev];
  // a counter pair for this launch, round-robin over kUnitSlots pairs; each
  // launch's last CTA leaves its pair at zero
  unsigned int* ctr = unit_counters(dev);
  if (!ctr) return CP_ERR_CUDA;
  static std::atomic<unsigned> seq[64];
  prm.unit_ctr = ctr + 2 * (seq[dev].fetch_add(1, std::memory_order_relaxed) % kUnitSlots);
  const int D = (int)a.q.shape[a.q.ndim - 1];
  if (D == 128) return launch_tc<128, kStagesD128>(prm, (int)grid, stream);
  if (D == 64) return launch_tc<64, kStagesD64>(prm, (int)grid, stream);
  return CP_ERR_SHAPE;
}

}  // namespace cpattn
