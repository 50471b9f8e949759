// mlra_decode_kernel.cuh -- K1: split-KV MLRA decode attention on sm_100a.
//
// Computes step 2 of the absorbed three-step decode ("Multi-Head Low-Rank Attention",
// yunpan.plus page, section 1.3) for the branch form of section 3.1: for every branch b,
// scores of the absorbed query block against latent block c_b plus the shared RoPE term,
// an online softmax of its own over positions, and the probability-weighted sum of c_b.
//
// One persistent CTA per (work range, branch, group of 64 heads).  A work range is a contiguous
// run of KV tiles (T positions each) of the batch (see mlra_plan.cuh).  A group's 64 heads are
// the M = 64 rows of every tcgen05 MMA (more than 64 heads: several groups read the same tiles,
// which mostly meet in L2), the tile's T positions the N of the score product:
//   score:  S[64 x T]     = Q~_b[64 x d] . C_b^T  +  Q^R[64 x 64] . K^R^T     (TMEM, fp32)
//   output: O[64 x d]    += P[64 x T] . C_b[T x d]                           (TMEM, fp32)
// The RoPE product is accumulated into the same score tile by the MMA chain.  An MMA costs at
// least ~57 cycles and N/2 cycles for N >= 128, so T = 128 keeps the score products efficient.
//
// TMEM.  An M = 64 accumulator occupies 16 of the 32 lanes of each sub-partition (rows 16k..16k+15
// in lanes 32k + [0,16) + 16h for lane half h).  The score buffers (one per stage, T columns
// each) fill lane half 0; O, cut into chunks of up to 128 columns, sits in lane half 1, followed
// there by one P slot per stage (T / 2 columns of bf16 pairs): the output product reads P from
// TMEM as its A operand (which must share the accumulator's lanes).  The landed tile implies the
// output product of the tile NS earlier, the slot's last reader, completed.  P is released in
// 64-position halves: the output product of the first half starts while the softmax still
// computes the second.  Keeping P out of shared memory leaves the tensor core's operand reads
// and the TMA writes the shared-memory bandwidth (both products were slowed by it).  Where O
// leaves no room (512-wide branches), P goes into shared memory over the tile's RoPE block,
// which only the score product reads ([64 heads x T positions], K-major, the 128-byte swizzled
// image of an MMA operand).
//
// Shared memory: the branch's queries (per segment), an NS-deep ring of cache tiles
// [latent blocks | RoPE block].
//
// Warp roles (224 threads): warps 0-3 softmax / rescale / epilogue, warp 4 TMA producer,
// warp 5 score-MMA issuer and TMEM owner, warp 6 output-MMA issuer.  The two issuers feed the
// tensor core independently, each blocking on its own barriers.  Softmax warp w owns heads
// 16w..16w+15; the thread pair (l, l ^ 16) shares head 16w + (l & 15) and splits every row's
// columns between them.
//
// Ordering facts the parity waits rely on (a parity wait is only safe when the barrier is at
// most one phase past the previous phase awaited):
//   * tile s is loaded only after the output product of tile s - NS completed (stage reuse), and
//     there are as many score buffers as stages (NSB = NS), so the score of tile s, issued after
//     tile s landed, never overwrites a score buffer the softmax still reads; neither issuer runs
//     more than NS tiles ahead of the other;
//   * once the score of tile s is done, every output product up to s - NS is done: the
//     output-completion ring bar_pv_done has NS entries.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <math_constants.h>

#include "mlra_internal.h"
#include "mlra_plan.cuh"
#include "sm100_ptx.cuh"

namespace mlra {

template <int DBLK, int T, int NS>
struct DecodeCfg {
  static constexpr int NCB = DBLK / 64;             // 64-column latent blocks
  static constexpr int TB = T / 64;                 // 64-row sub-boxes per tile
  static constexpr int BOX = 64 * 64 * 2;           // one [64 x 64] bf16 box, 8 KB
  static constexpr int CBLK = T * 128;              // one 64-column block of a tile (T rows)
  static constexpr int STAGE = (NCB + 1) * CBLK;    // latent blocks + RoPE block
  static constexpr int QBYTES = (NCB + 1) * BOX;    // query blocks + RoPE-query block
  static constexpr int OCW = DBLK < 128 ? DBLK : 128;   // O chunk width (columns)
  static constexpr int OCH = DBLK / OCW;                // O chunks
  static constexpr int O_COLS = OCH * OCW;              // TMEM columns of O (lane half 1)
  static constexpr int NSB = NS;                        // score buffers (lane half 0)
  static constexpr int NPV = NS;                    // ring of output-MMA completion barriers
  // P slots in lane half 1 after O (one per stage), when they fit
  static constexpr bool P_TMEM = O_COLS + NS * (T / 2) <= 512;
  static constexpr int P_COL = O_COLS;
  static constexpr int HALF1 = O_COLS + (P_TMEM ? NS * (T / 2) : 0);
  static constexpr int TMEM_USED = HALF1 > NSB * T ? HALF1 : NSB * T;
  static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 :
                                   TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_STAGE = QBYTES;
  static constexpr int OFF_BAR = OFF_STAGE + NS * STAGE;
  static constexpr int NBAR = 2 * NS + 2 + NSB + TB * NSB + NPV + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // TMEM address, abort flag, status bits
  static constexpr int OFF_PLAN = OFF_MISC + 16;       // in-kernel plan (self_plan)
  static constexpr int PLAN_BYTES = 16 * kSelfPlanMaxSeqs +     // segment list
                                    4 * kSelfPlanMaxSeqs + 16;    // lengths, count, stale, hook
  static constexpr int OFF_HOOK_BAR = OFF_PLAN + 20 * kSelfPlanMaxSeqs + 8;  // force_timeout
  // epilogue staging: one [16 rows x 32 fp32] box per softmax warp, 128-byte swizzled
  static constexpr int OFF_STG = (OFF_PLAN + PLAN_BYTES + 1023) / 1024 * 1024;
  static constexpr int STG_BYTES = 16 * 128;
  static constexpr int SMEM = OFF_STG + 4 * STG_BYTES;
  static constexpr int SMEM_ALLOC = SMEM + 1024;    // slack to align the base to 1024 B
  static_assert(DBLK % 64 == 0 && DBLK <= 512, "branch width must be a multiple of 64, <= 512");
  static_assert(T == 64 || T == 128, "tile of 64 or 128 positions");
  static_assert(NSB >= 2 && NSB == NS, "score buffers: one per stage, at least 2");
  static_assert(TB * BOX == CBLK, "P of a tile fills the RoPE block of its stage");
  static_assert(TMEM_USED <= 512, "TMEM budget");
  static_assert(OFF_HOOK_BAR % 8 == 0 && OFF_HOOK_BAR + 8 <= OFF_PLAN + PLAN_BYTES, "hook barrier");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

constexpr uint32_t kFull = 0xffffffffu;

// Three-input maximum / minimum (one instruction; a NaN input is ignored, as by fmaxf / fminf).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
constexpr int kFirstTiles = 2;  // tiles issued at once when a CTA starts (the rest after tile 0)

// Warp-collective bounded wait on an mbarrier phase.  Every lane polls; on time-out the
// status word gets kFlagTimeout, the CTA abort flag is raised and all lanes return false.
// With honor_abort == false the wait ignores the abort flag (used to drain in-flight copies and
// MMAs before the CTA exits) but still gives up after timeout_ns.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                          volatile int* abort_flag, uint32_t* status,
                                          bool honor_abort = true) {
  bool ok = mbar_try_wait(bar, parity);
  if (!ok) {
    const uint64_t t0 = global_timer_ns();
    uint32_t spins = 0;
    while (true) {
      if (mbar_try_wait(bar, parity)) { ok = true; break; }
      if ((++spins & 63u) == 0) {
        if (honor_abort && *abort_flag) break;
        if (global_timer_ns() - t0 > timeout_ns) {
          atomicOr(status, kFlagTimeout);
          *abort_flag = 1;
          break;
        }
      }
    }
  }
  return __all_sync(kFull, ok);
}

// Test hook (force_timeout): the producer waits, with a short limit, on an mbarrier that nothing
// arrives at, so that the time-out path runs for real: the status flag, the CTA abort seen by the
// other warps, the drain of the copies already issued and the release of TMEM.  Returns false.
__device__ __forceinline__ bool forced_timeout_wait(uint32_t bar, uint64_t timeout_ns,
                                                    volatile int* abort_flag, uint32_t* status,
                                                    int lane) {
  if (lane == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  const bool ok = wait_warp(bar, 0, timeout_ns, abort_flag, status);
  if (lane == 0) mbar_inval(bar);
  __syncwarp();
  return ok;
}

// First cache row of the 64-position block t (positions [64t, 64t+64)) of sequence s.  Shared by
// the decode kernel and the row-resolution test hook.  An invalid page id flags the status word
// and returns a row past the end of the cache, where TMA reads zeros.
__device__ __forceinline__ int tile_row(const int32_t* page_table, int max_pages, int page_size,
                                        int max_seq_len, int64_t n_pages, int oob_row, int s,
                                        int t, uint32_t* status) {
  if (page_table == nullptr) return s * max_seq_len + t * kTile;
  const int j = t * kTile;
  const int pid = __ldg(page_table + (int64_t)s * max_pages + j / page_size);
  if (pid < 0 || pid >= n_pages) {
    if (status) atomicOr(status, kFlagBadPage);
    return oob_row;
  }
  return pid * page_size + j % page_size;
}

constexpr int kDecodeThreads = 224;

// In-kernel plan for N <= kSelfPlanMaxSeqs = 64.  Warp 0's lane l holds the adjacent sequences
// 2 l and 2 l + 1, so one warp scan covers the batch.
//
// plan_read_lengths: the lengths (virtual lengths for several tokens per sequence), clamped to
// [0, limit]; bit 6 of `bits` reports a length outside that range.
//
// plan_segments: scans the real and virtual tile prefixes (mlra_plan.cuh) across the warp, finds
// the sequence holding each of the range's two virtual boundaries with one ballot, and lets every
// sequence that overlaps the range write its own segment at its rank (shared memory only).  Per
// lane it adds to `bits`: bit c (c = 0, 1) sequence 2 lane + c has its first tile in this range,
// bit 2 + c its last tile, bit 4 + c it is empty.  Returns the segment count.
//
// plan_commit: the plan's global records, written once the lengths are final: the CTAs of group 0
// record for the combine kernel the ranges holding each sequence's first and last tile, CTA 0
// the records of empty sequences, and the bad-length status bit.
//
// The decode kernel runs the first two before its dependency wait on the lengths as they are then
// (a speculative plan), reads the lengths again after the wait and keeps the plan when they are
// unchanged.
__device__ __forceinline__ void plan_read_lengths(const DecodeParams& p, int lane, int (&L)[2],
                                                  uint32_t& bits) {
  bits = 0;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int i = 2 * lane + c;
    int x = i < p.N ? (p.q_per_seq == 1 ? __ldcg(p.seq_lens + i)
                                        : __ldcg(p.seq_lens + i / p.q_per_seq) -
                                              (p.q_per_seq - 1 - i % p.q_per_seq) * p.unit_tokens)
                    : 0;
    if (i < p.N && (x - (p.unit_tokens - 1) < 0 || x > p.limit)) {  // (or the unit's first token)
      bits |= 64u;
      x = x < 0 ? 0 : (x > p.limit ? p.limit : x);
    }
    L[c] = x;
  }
}

// floor(a / b) for 0 <= a < 2^53, b >= 1.  Below 2^24 a single-precision quotient is within one
// of the result and one correction step each way makes it exact (the common case: a few thousand
// virtual tiles times the range index); above, a double division and the same correction.
__device__ __forceinline__ int64_t floor_div_i64(int64_t a, int64_t b) {
  int64_t q;
  if (a < (int64_t{1} << 24))
    q = static_cast<int64_t>(__fdiv_rz(static_cast<float>(a), static_cast<float>(b)));
  else
    q = static_cast<int64_t>(__ddiv_rz(static_cast<double>(a), static_cast<double>(b)));
  if (q * b > a) --q;
  if ((q + 1) * b <= a) ++q;
  return q;
}

__device__ __forceinline__ int plan_segments(const DecodeParams& p, int range, int L0, int L1,
                                             uint8_t* plan, uint32_t& bits) {
  int4* list = reinterpret_cast<int4*>(plan);                       // [kSelfPlanMaxSeqs]
  int32_t* lens = reinterpret_cast<int32_t*>(list + kSelfPlanMaxSeqs);
  const int lane = threadIdx.x & 31, N = p.N, cost = p.seg_cost;
  const int i0 = 2 * lane, i1 = i0 + 1;
  const int tile_shift = p.tile == 64 ? 6 : 7;  // tiles of 64 or 128 positions
  const int t0 = i0 < N ? (L0 + p.tile - 1) >> tile_shift : 0;
  const int t1 = i1 < N ? (L1 + p.tile - 1) >> tile_shift : 0;
  const int v0 = t0 > 0 ? t0 + cost : 0, v1 = t1 > 0 ? t1 + cost : 0;
  bits &= 64u;
  if (i0 < N && t0 == 0) bits |= 16u;
  if (i1 < N && t1 == 0) bits |= 32u;
  if (i0 < N) lens[i0] = L0;
  if (i1 < N) lens[i1] = L1;
  int x = t0 + t1, v = v0 + v1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {  // inclusive scans of the pairs' tiles and virtual tiles
    const int yx = __shfl_up_sync(kFull, x, o), yv = __shfl_up_sync(kFull, v, o);
    if (lane >= o) {
      x += yx;
      v += yv;
    }
  }
  const int total = __shfl_sync(kFull, x, 31), vtotal = __shfl_sync(kFull, v, 31);
  const int lo0 = x - t0 - t1, hi0 = lo0 + t0, lo1 = hi0, hi1 = lo1 + t1;
  const int vlo0 = v - v0 - v1, vhi0 = vlo0 + v0, vlo1 = vhi0, vhi1 = vlo1 + v1;
  const int64_t R = effective_ranges(p.num_ranges, total);
  if (range >= R || total == 0) return 0;
  // real tile of a virtual position: the sequence whose virtual interval holds it
  auto tile_of = [&](int64_t vp) -> int {
    const bool own0 = t0 > 0 && vlo0 <= vp && vp < vhi0;
    const bool own1 = t1 > 0 && vlo1 <= vp && vp < vhi1;
    const int64_t o = vp - (own0 ? vlo0 : vlo1) - cost;
    const int mine = (own0 ? lo0 : lo1) + static_cast<int>(o > 0 ? o : 0);
    const uint32_t m = __ballot_sync(kFull, own0 || own1);
    return __shfl_sync(kFull, mine, m ? __ffs(m) - 1 : 0);
  };
  // both boundaries' virtual positions first (independent divisions), then their tiles
  const bool has_next = range + 1 < R;
  const int64_t vp0 = floor_div_i64(range * (int64_t)vtotal, R);
  const int64_t vp1 = has_next ? floor_div_i64((range + 1) * (int64_t)vtotal, R) : 0;
  const int g0 = tile_of(vp0);
  const int g1 = has_next ? tile_of(vp1) : total;
  const bool ov0 = t0 > 0 && lo0 < g1 && hi0 > g0;
  const bool ov1 = t1 > 0 && lo1 < g1 && hi1 > g0;
  const uint32_t m0 = __ballot_sync(kFull, ov0), m1 = __ballot_sync(kFull, ov1);
  const uint32_t below = (1u << lane) - 1u;
  const int rank0 = __popc(m0 & below) + __popc(m1 & below);
  if (ov0) {
    const int a = g0 > lo0 ? g0 : lo0, e = g1 < hi0 ? g1 : hi0;
    list[rank0] = make_int4(i0, a - lo0, e - a,
                            L0 | ((a == lo0 && e == hi0) ? (int32_t)0x80000000u : 0));
    if (a == lo0) bits |= 1u;  // the sequence's first tile is in this range
    if (e == hi0) bits |= 4u;  // ... its last tile
  }
  if (ov1) {
    const int a = g0 > lo1 ? g0 : lo1, e = g1 < hi1 ? g1 : hi1;
    list[rank0 + (ov0 ? 1 : 0)] = make_int4(i1, a - lo1, e - a,
                                            L1 | ((a == lo1 && e == hi1) ? (int32_t)0x80000000u : 0));
    if (a == lo1) bits |= 2u;
    if (e == hi1) bits |= 8u;
  }
  return __popc(m0) + __popc(m1);
}

__device__ __forceinline__ void plan_commit(const DecodeParams& p, int range, int group,
                                            uint32_t bits, uint32_t* flags) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int i = 2 * lane + c;
    if (group == 0) {
      if (bits & (1u << c)) p.seqs[i].r0 = range;
      if (bits & (4u << c)) p.seqs[i].r1 = range;
    }
    if (blockIdx.x == 0 && (bits & (16u << c))) p.seqs[i] = SeqInfo{0, -1};
  }
  if (bits & 64u) atomicOr(flags, kFlagBadLength);
}

// Outputs of empty sequences (out = 0, lse = -inf), written by CTA 0's warps 1.. after the plan.
__device__ __forceinline__ void plan_empty_outputs(const DecodeParams& p, const uint8_t* plan) {
  const int32_t* lens =
      reinterpret_cast<const int32_t*>(reinterpret_cast<const int4*>(plan) + kSelfPlanMaxSeqs);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int sq = warp - 1; sq < p.N; sq += kDecodeThreads / 32 - 1) {
    if (lens[sq] != 0) continue;
    float* row = p.out + (int64_t)sq * p.H * p.out_width;
    for (int i = lane; i < p.H * p.out_width; i += 32) row[i] = 0.f;
    if (p.lse)
      for (int i = lane; i < p.H * p.B; i += 32) p.lse[(int64_t)sq * p.H * p.B + i] = -CUDART_INF_F;
  }
}

// The segments of one work range, read one ahead of use: from the prep kernel's descriptors in
// global memory, or from the CTA's own list in shared memory.
struct SegCursor {
  const int4* segs;
  bool global;
  int count, i;
  int4 nxt;
  __device__ __forceinline__ int4 load(int k) const {
    return global ? __ldcg(segs + k) : segs[k];
  }
  __device__ __forceinline__ SegCursor(const int4* list, bool in_global, int n)
      : segs(list), global(in_global), count(n), i(0) {
    if (count > 0) nxt = load(0);
  }
  __device__ __forceinline__ bool next(Segment& seg, int& len) {
    if (i >= count) return false;
    const int4 d = nxt;
    if (++i < count) nxt = load(i);
    seg.seq = d.x;
    seg.tile0 = d.y;
    seg.ntiles = d.z;
    seg.whole = d.w < 0;
    len = d.w & 0x7fffffff;
    return true;
  }
};

template <int DBLK, int T, int NS>
__global__ void __launch_bounds__(kDecodeThreads, 1)
mlra_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                   const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_kr,
                   const __grid_constant__ CUtensorMap tm_out, const __grid_constant__ CUtensorMap tm_part,
                   const __grid_constant__ DecodeParams p) {
  using C = DecodeCfg<DBLK, T, NS>;
  constexpr int NSB = C::NSB, NPV = C::NPV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sStage = sbase + C::OFF_STAGE;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  // barrier map
  const uint32_t bar_stage_full = bar0;                     // [NS]  TMA -> MMA
  const uint32_t bar_stage_empty = bar0 + 8 * NS;           // [NS]  MMA (PV done) -> TMA
  const uint32_t bar_q_full = bar0 + 16 * NS;               //       TMA -> MMA
  const uint32_t bar_q_empty = bar_q_full + 8;              //       MMA (last score) -> TMA
  const uint32_t bar_s_full = bar_q_full + 16;              // [NSB] MMA (score) -> softmax
  const uint32_t bar_p_full = bar_s_full + 8 * NSB;         // [TB][NSB] softmax (P half) -> MMA
  const uint32_t bar_pv_done = bar_p_full + 8 * C::TB * NSB; // [NPV] MMA (PV done) -> softmax
  const uint32_t bar_final_s = bar_pv_done + 8 * NPV;       // drains of the two issuers
  const uint32_t bar_final_pv = bar_final_s + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  uint32_t* spec_flags = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 8);  // see below
  uint32_t* flags = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 12);  // this CTA's status bits
  uint8_t* plan = smem + C::OFF_PLAN;
  volatile int32_t* plan_count = reinterpret_cast<volatile int32_t*>(plan + 20 * kSelfPlanMaxSeqs);
  volatile int32_t* plan_stale = plan_count + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int range = blockIdx.x / p.n_groups;
  const int group = blockIdx.x % p.n_groups;  // (64-head group, branch) of this CTA
  const int branch = group % p.B;
  const int h0 = 64 * (group / p.B);          // first head of this CTA's group
  const uint64_t tmo = p.timeout_ns;
  // The combine kernel may be scheduled now; it waits for this grid before reading anything.
  pdl_launch_dependents();

  auto init_barriers = [&]() {
    for (int k = 0; k < NS; ++k) {
      mbar_init(bar_stage_full + 8 * k, 1);
      mbar_init(bar_stage_empty + 8 * k, 1);
    }
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, 1);
    for (int k = 0; k < NSB; ++k) mbar_init(bar_s_full + 8 * k, 1);
    for (int k = 0; k < C::TB * NSB; ++k) mbar_init(bar_p_full + 8 * k, 128);
    for (int k = 0; k < NPV; ++k) mbar_init(bar_pv_done + 8 * k, 1);
    mbar_init(bar_final_s, 1);
    mbar_init(bar_final_pv, 1);
  };
  if (warp == 6 && lane == 0) {  // (warp 0 starts the plan meanwhile)
    init_barriers();
    *abort_flag = 0;
    *spec_flags = 0;
    *flags = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_qr);
    tma_prefetch_desc(&tm_c);
    tma_prefetch_desc(&tm_kr);
    tma_prefetch_desc(&tm_part);
    if (p.tma_out) tma_prefetch_desc(&tm_out);
  }
  // Speculative plan (N <= kSelfPlanMaxSeqs): made from the lengths as they are before the
  // dependency wait, while the previous kernel on the stream may still run.  It is used only if
  // the lengths read again after the wait are the same (below); nothing global is written here.
  int spec_len[2] = {0, 0};
  uint32_t plan_bits = 0;
  if (p.self_plan && warp == 0) {
    plan_read_lengths(p, lane, spec_len, plan_bits);
    const int n = plan_segments(p, range, spec_len[0], spec_len[1], plan, plan_bits);
    if (lane == 0) *plan_count = n;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int col0 = branch * DBLK;  // first latent column of this CTA's branch
  int4 first_seg = make_int4(0, 0, 0, 0);  // the producer's copy of the first speculative segment
  const bool speculate = p.self_plan && warp == 4 && *plan_count > 0;
  if (speculate) first_seg = reinterpret_cast<const int4*>(plan)[0];

  // Loads of one tile into stage st (lane 0 of the producer): the latent block's 64-row
  // sub-boxes and the RoPE block, counted on the stage's full barrier.
  const uint64_t once = l2_policy_evict_first();
  auto issue_tile = [&](int st, const int (&rows)[C::TB]) {
    const uint32_t full = bar_stage_full + 8 * st;
    const uint32_t dst = sStage + st * C::STAGE;
    mbar_arrive_expect_tx(full, C::STAGE);
    // the latent rows are read once per call (by this CTA alone): first out of L2, so the
    // queries, RoPE rows (shared by the branch CTAs) and partial results stay
#pragma unroll
    for (int l = 0; l < C::TB; ++l) {
#pragma unroll
      for (int k = 0; k < C::NCB; ++k)
        tma_load_2d_hint(dst + k * C::CBLK + l * C::BOX, &tm_c, full, col0 + 64 * k, rows[l], once);
      tma_load_2d(dst + C::NCB * C::CBLK + l * C::BOX, &tm_kr, full, 0, rows[l]);
    }
  };
  auto issue_queries = [&](int seq) {
    mbar_arrive_expect_tx(bar_q_full, C::QBYTES);
#pragma unroll
    for (int k = 0; k < C::NCB; ++k)
      tma_load_3d(sQ + k * C::BOX, &tm_q, bar_q_full, col0 + 64 * k, h0, seq);
    tma_load_3d(sQ + C::NCB * C::BOX, &tm_qr, bar_q_full, 0, h0, seq);
  };
  // cache rows of tile t of virtual sequence v's cache (length len; past the end: zeros)
  auto tile_rows = [&](int cache_seq, int t, int len, uint32_t* status, int (&rows)[C::TB]) {
#pragma unroll
    for (int l = 0; l < C::TB; ++l) {
      const int t64 = t * C::TB + l;
      rows[l] = (t64 * kTile < len)
                    ? tile_row(p.page_table, p.max_pages, p.page_size, p.max_seq_len, p.n_pages,
                               p.oob_row, cache_seq, t64, lane == 0 ? status : nullptr)
                    : p.oob_row;
    }
  };

  // Everything above overlapped the previous kernel on the stream (the prep kernel, or the
  // previous call's combine); the lengths, queries, cache and the prep kernel's plan are read
  // only after it.
  pdl_wait_prerequisites();
  int pre_tiles = 0;      // producer: tiles of the first segment already issued
  bool pre_q = false;     // ... and its queries
  if (p.self_plan) {
    if (speculate) {
      // The first segment's queries and tiles go out at once, on the speculative plan (bad-page
      // bits into spec_flags until the plan is confirmed).
      const int len = first_seg.w & 0x7fffffff;
      pre_tiles = first_seg.z < kFirstTiles ? first_seg.z : kFirstTiles;
      pre_q = true;
      const int cache_seq = first_seg.x / p.q_per_seq;
      if (lane == 0) issue_queries(first_seg.x);
      for (int i = 0; i < pre_tiles; ++i) {
        int rows[C::TB];
        tile_rows(cache_seq, first_seg.y + i, len, spec_flags, rows);
        if (lane == 0) issue_tile(i, rows);
      }
      __syncwarp();
    }
    if (warp == 0) {
      // the lengths now final: keep the speculative plan if they did not change
      int len_now[2];
      uint32_t bits_now;
      plan_read_lengths(p, lane, len_now, bits_now);
      const bool same = __all_sync(kFull, len_now[0] == spec_len[0] && len_now[1] == spec_len[1]);
      if (!same || p.force_replan) {
        plan_bits = bits_now;
        const int n = plan_segments(p, range, len_now[0], len_now[1], plan, plan_bits);
        if (lane == 0) *plan_count = n;
      }
      if (lane == 0) *plan_stale = (!same || p.force_replan) ? 1 : 0;
      plan_commit(p, range, group, plan_bits, flags);
    }
    __syncthreads();
    if (*plan_stale) {
      // The lengths changed under the speculative plan: let its loads land, reset the barriers
      // and start over with the new plan.
      if (speculate) {
        if (pre_q) wait_warp(bar_q_full, 0, tmo, abort_flag, flags, false);
        for (int i = 0; i < pre_tiles; ++i)
          wait_warp(bar_stage_full + 8 * i, 0, tmo, abort_flag, flags, false);
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        for (int k = 0; k < C::NBAR; ++k) mbar_inval(bar0 + 8 * k);
        init_barriers();
        fence_barrier_init();
      }
      __syncthreads();
      pre_tiles = 0;
      pre_q = false;
    } else if (speculate && lane == 0) {
      atomicOr(flags, *spec_flags);
    }
    if (blockIdx.x == 0 && warp >= 1) plan_empty_outputs(p, plan);
  }
  const int4* seg_list;
  int seg_count;
  if (p.self_plan) {
    seg_count = *plan_count;
    seg_list = reinterpret_cast<const int4*>(plan);
  } else {
    const int2 r2 = __ldcg(reinterpret_cast<const int2*>(p.ranges + range));
    seg_list = reinterpret_cast<const int4*>(p.segs + r2.x);
    seg_count = r2.y;
  }
  const bool list_global = !p.self_plan;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    SegCursor walk(seg_list, list_global, seg_count);
    Segment seg;
    int L = 0;
    int it = 0, nseg = 0;
    int q_loads = pre_q ? 1 : 0;  // query loads issued so far (for a drain)
    bool ok = true;
    while (ok && walk.next(seg, L)) {
      if (nseg > 0) ok = wait_warp(bar_q_empty, (nseg - 1) & 1, tmo, abort_flag, flags);
      if (!ok) break;
      if (!(nseg == 0 && pre_q)) {
        if (lane == 0) issue_queries(seg.seq);
        ++q_loads;
      }
      __syncwarp();
      const int cache_seq = seg.seq / p.q_per_seq;  // whose cache rows (once per segment)
      for (int i = 0; i < seg.ntiles; ++i, ++it) {
        if (nseg == 0 && i < pre_tiles) continue;  // issued before the plan was confirmed
        if (p.force_timeout) {
          ok = forced_timeout_wait(smem_u32(smem + C::OFF_HOOK_BAR), tmo >> 10, abort_flag, flags,
                                   lane);
          if (!ok) break;
        }
        if (it == kFirstTiles && pre_tiles == kFirstTiles) {
          // the remaining first stages once tile 0 has landed: every CTA's first tile arrives
          // sooner (fewer bytes ahead of it in the memory queues), so the tensor core starts and
          // frees stages while the first loads are still streaming
          ok = wait_warp(bar_stage_full, 0, tmo, abort_flag, flags);
          if (!ok) break;
        }
        int rows[C::TB];
        tile_rows(cache_seq, seg.tile0 + i, L, flags, rows);
        const int st = it % NS;
        if (it >= NS) {
          ok = wait_warp(bar_stage_empty + 8 * st, ((it / NS) - 1) & 1, tmo, abort_flag, flags);
          if (!ok) break;
        }
        if (lane == 0) issue_tile(st, rows);
        __syncwarp();
      }
      ++nseg;
    }
    if (!ok) {
      // Aborting: let the copies already issued land before the CTA can exit.
      if (q_loads > 0) wait_warp(bar_q_full, (q_loads - 1) & 1, tmo / 8, abort_flag, flags, false);
      for (int k = (it > NS ? it - NS : 0); k < it; ++k)
        wait_warp(bar_stage_full + 8 * (k % NS), (k / NS) & 1, tmo / 8, abort_flag, flags, false);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ score-MMA issuer
    constexpr uint32_t kIdScore = idesc_bf16_f32(64, T, false, false);
    SegCursor walk(seg_list, list_global, seg_count);
    Segment seg;
    int L = 0;
    int it = 0, nseg = 0;
    bool ok = true;
    while (ok && walk.next(seg, L)) {
      ok = wait_warp(bar_q_full, nseg & 1, tmo, abort_flag, flags);
      for (int i = 0; ok && i < seg.ntiles; ++i, ++it) {
        // the landed tile implies the output product of tile it - NS completed, so its softmax
        // has read score buffer it % NSB (NSB == NS)
        ok = wait_warp(bar_stage_full + 8 * (it % NS), (it / NS) & 1, tmo, abort_flag, flags);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t stg = sStage + (it % NS) * C::STAGE;
          const uint32_t d = tmem + (it % NSB) * T;  // lane half 0
#pragma unroll
          for (int kb = 0; kb < C::NCB; ++kb) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sw128_desc(sQ + kb * C::BOX + kk * 32, 16, 1024);
              const uint64_t bd = sw128_desc(stg + kb * C::CBLK + kk * 32, 16, 1024);
              umma_bf16(d, ad, bd, kIdScore, (kb | kk) ? 1u : 0u);
            }
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sw128_desc(sQ + C::NCB * C::BOX + kk * 32, 16, 1024);
            const uint64_t bd = sw128_desc(stg + C::NCB * C::CBLK + kk * 32, 16, 1024);
            umma_bf16(d, ad, bd, kIdScore, 1u);
          }
          umma_commit(bar_s_full + 8 * (it % NSB));
          if (i == seg.ntiles - 1) umma_commit(bar_q_empty);
        }
        __syncwarp();
      }
      ++nseg;
    }
    // Nothing of ours may still run on the tensor core when TMEM is released.
    if (lane == 0) umma_commit(bar_final_s);
    __syncwarp();
    wait_warp(bar_final_s, 0, tmo, abort_flag, flags, false);
  } else if (warp == 6) {
    // ------------------------------------------------------------------ output-MMA issuer
    constexpr uint32_t kIdPV = idesc_bf16_f32(64, C::OCW, false, true);
    SegCursor walk(seg_list, list_global, seg_count);
    Segment seg;
    int L = 0;
    int j = 0;
    bool ok = true;
    while (ok && walk.next(seg, L)) {
      for (int i = 0; ok && i < seg.ntiles; ++i, ++j) {
        const uint32_t stg = sStage + (j % NS) * C::STAGE;
        const uint32_t pa = stg + C::NCB * C::CBLK;  // P over the tile's RoPE block (!P_TMEM)
        const uint32_t pt = tmem + (16u << 16) + C::P_COL + (j % NS) * (T / 2);  // P slot (P_TMEM)
#pragma unroll 1
        for (int hb = 0; hb < C::TB; ++hb) {  // one 64-position half of P at a time
          ok = wait_warp(bar_p_full + 8 * (hb * NSB + j % NSB), (j / NSB) & 1, tmo, abort_flag,
                         flags);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            const bool first = (i == 0 && hb == 0);  // the segment's first product overwrites O
#pragma unroll
            for (int ch = 0; ch < C::OCH; ++ch) {
              const uint32_t d = tmem + (16u << 16) + ch * C::OCW;  // lane half 1
              const uint32_t b0 = stg + ch * (C::OCW / 64) * C::CBLK;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bd = sw128_desc(b0 + (4 * hb + kk) * 2048, C::CBLK, 1024);
                if constexpr (C::P_TMEM) {  // 16 positions: 8 TMEM columns of P
                  umma_bf16_ts(d, pt + 8 * (4 * hb + kk), bd, kIdPV, (kk > 0 || !first) ? 1u : 0u);
                } else {
                  const uint64_t ad = sw128_desc(pa + hb * C::BOX + kk * 32, 16, 1024);
                  umma_bf16(d, ad, bd, kIdPV, (kk > 0 || !first) ? 1u : 0u);
                }
              }
            }
            if (hb == C::TB - 1) {
              umma_commit(bar_stage_empty + 8 * (j % NS));
              umma_commit(bar_pv_done + 8 * (j % NPV));
            }
          }
          __syncwarp();
        }
      }
    }
    if (lane == 0) umma_commit(bar_final_pv);
    __syncwarp();
    wait_warp(bar_final_pv, 0, tmo, abort_flag, flags, false);
  } else {
    // ------------------------------------------------------------------ softmax warps 0-3
    const int q = lane >> 4;                   // which half of the row's columns
    const int h = h0 + 16 * warp + (lane & 15);  // head
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    uint8_t* stg = smem + C::OFF_STG + warp * C::STG_BYTES;  // this warp's store staging box
    const uint32_t stg_u = smem_u32(stg);
    bool stg_pending = false;  // a bulk store may still be reading stg
    SegCursor walk(seg_list, list_global, seg_count);
    Segment seg;
    int L = 0;
    int it = 0;
    bool ok = true;
    while (ok && walk.next(seg, L)) {
      float m_used = -CUDART_INF_F, l_sum = 0.f;
      for (int i = 0; i < seg.ntiles; ++i, ++it) {
        const int t = seg.tile0 + i;
        ok = wait_warp(bar_s_full + 8 * (it % NSB), (it / NSB) & 1, tmo, abort_flag, flags);
        if (!ok) break;
        tc_fence_after();
        // this thread's scores: positions 64 l + 32 q + [0, 32) of the tile, l < T / 64 (both
        // loads in flight, one wait)
        float v[C::TB][32];
#pragma unroll
        for (int l = 0; l < C::TB; ++l)
          tmem_ld16x2_32(tmem + lane_base + (it % NSB) * T + 64 * l,
                         reinterpret_cast<uint32_t(&)[32]>(v[l]));
        tmem_wait_ld();
        const int valid = min(T, L - T * t);
        // Row maximum of the scaled scores (log2 units).  A whole tile holds only finite scores:
        // the maximum of the raw dot products (the minimum for a negative scale) times the scale,
        // and the scale is folded into each exponent below (one FFMA per score).  The ragged last
        // tile scales first and masks the positions past the sequence end with -inf.
        const bool whole_tile = valid == T;
        const float sc = p.scale_log2;
        float mx;
        if (whole_tile) {
          float a[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) a[u] = v[0][u];
          if (sc >= 0.f) {
#pragma unroll
            for (int l = 0; l < C::TB; ++l)
#pragma unroll
              for (int k = 0; k < 32; k += 2) a[(k >> 1) & 3] = max3f(a[(k >> 1) & 3], v[l][k], v[l][k + 1]);
            mx = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])) * sc;
          } else {
#pragma unroll
            for (int l = 0; l < C::TB; ++l)
#pragma unroll
              for (int k = 0; k < 32; k += 2) a[(k >> 1) & 3] = min3f(a[(k >> 1) & 3], v[l][k], v[l][k + 1]);
            mx = fminf(fminf(a[0], a[1]), fminf(a[2], a[3])) * sc;
          }
        } else {
          mx = -CUDART_INF_F;
#pragma unroll
          for (int l = 0; l < C::TB; ++l) {
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const float x = (64 * l + 32 * q + k < valid) ? v[l][k] * sc : -CUDART_INF_F;
              v[l][k] = x;
              mx = fmaxf(mx, x);
            }
          }
        }
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
        bool rescale = false;
        float alpha = 1.f;
        if (i == 0) {
          m_used = mx;
        } else if (mx > m_used + 8.f) {  // lazy rescale: only when p could exceed 2^8
          alpha = ex2_approx(m_used - mx);
          m_used = mx;
          rescale = true;
        }
        l_sum *= alpha;
        if (__any_sync(kFull, rescale)) {
          // O holds the output products up to tile it-1: wait for them, then scale O
          ok = wait_warp(bar_pv_done + 8 * ((it - 1) % NPV), ((it - 1) / NPV) & 1, tmo, abort_flag,
                         flags);
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int ch = 0; ch < C::OCH; ++ch) {
#pragma unroll 1
            for (int c0 = 0; c0 < C::OCW; c0 += 64) {
              const uint32_t a = tmem + ((uint32_t)(32 * warp + 16) << 16) + ch * C::OCW + c0;
              uint32_t r[32];
              tmem_ld16x2_32(a, r);
              tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
              tmem_st16x2_32(a, r);
            }
          }
          tmem_wait_st();
        }
        uint8_t* stage_ptr = smem + C::OFF_STAGE + (it % NS) * C::STAGE;
        if (valid < T) {
          // Ragged last tile: zero the latent rows past the sequence end so that the zero
          // probabilities never multiply a non-finite value left in the cache (before the first
          // half of P is released: the output product reads these rows)
          for (int k = threadIdx.x; k < C::NCB * T * 8; k += 128) {
            const int row = (k >> 3) % T;
            if (row >= valid)
              *reinterpret_cast<uint4*>(stage_ptr + (k / (T * 8)) * C::CBLK + row * 128 + (k & 7) * 16) =
                  make_uint4(0u, 0u, 0u, 0u);
          }
        }
        // probabilities -> bf16 P, each 64-position block l released to the output product as
        // soon as it is written: into the tile's P slot in TMEM (position 64 l + 32 q + k in
        // column 32 l + 16 q + k / 2 of the head row's lane), or over the tile's RoPE block, the
        // K-major image of the output product's A operand (head row r, position 64 l + 32 q + k in
        // 64-position block l, row r, 16-byte chunk (4 q + k / 8) ^ (r & 7), 128-byte swizzle).
        // p = 2^(score - m): whole tiles hold the raw products (one FFMA applies the scale),
        // the ragged tile the scaled and masked scores
        const float mul = whole_tile ? sc : 1.f, neg_m = -m_used;
        const int prow = 16 * warp + (lane & 15);
        uint8_t* p_base = stage_ptr + C::NCB * C::CBLK + prow * 128;
        const uint32_t p_slot =
            tmem + ((uint32_t)(32 * warp + 16) << 16) + C::P_COL + (it % NS) * (T / 2);
        // (pairs of positions through the packed two-lane FMA and add)
        const float2 mul2 = make_float2(mul, mul), negm2 = make_float2(neg_m, neg_m);
        float2 sum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int l = 0; l < C::TB; ++l) {
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float2 x = __ffma2_rn(make_float2(v[l][k], v[l][k + 1]), mul2, negm2);
            const float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
            sum2[(k >> 1) & 1] = __fadd2_rn(sum2[(k >> 1) & 1], make_float2(p0, p1));
            pk[k / 2] = pack_bf16x2(p0, p1);
          }
          if constexpr (C::P_TMEM) {
            tmem_st16x2_16(p_slot + 32 * l, pk);
            tmem_wait_st();
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              *reinterpret_cast<uint4*>(p_base + l * C::BOX + (((4 * q + c) ^ (prow & 7)) << 4)) =
                  make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          }
          fence_proxy_async_smem();  // P (and the zeroed rows) are read by the MMA (async proxy)
          tc_fence_before();         // ... after this thread's TMEM accesses (and O rescale)
          mbar_arrive(bar_p_full + 8 * (l * NSB + it % NSB));
        }
        float sum = (sum2[0].x + sum2[0].y) + (sum2[1].x + sum2[1].y);
        sum += __shfl_xor_sync(kFull, sum, 16);
        l_sum += sum;
      }
      if (!ok) break;
      // ------------------------------------------------ epilogue of the segment
      ok = wait_warp(bar_pv_done + 8 * ((it - 1) % NPV), ((it - 1) / NPV) & 1, tmo, abort_flag,
                     flags);
      if (!ok) break;
      tc_fence_after();
      const bool to_final = seg.whole && p.write_final;
      const bool live = h < p.H;
      float scale;
      int ncols_out;
      if (to_final) {
        scale = p.gamma / l_sum;
        ncols_out = p.d_blk_out;
      } else {
        scale = 1.f;
        ncols_out = DBLK;
      }
      if (h0 + 16 * warp >= p.H) {
        // no head of this warp exists: nothing to store
      } else if (!to_final || p.tma_out) {
        // Through shared memory and the TMA: each [16 heads x 32 columns] box is staged in the
        // 128-byte swizzled layout and stored by one bulk copy (rows past H are clipped by the
        // tensor map).  Partials go to slot range + seq of part_o, finals to out.  In the
        // range's last segment the stage ring is idle (every load landed, every product that
        // read it completed), so each warp stages all its boxes there and issues them back to
        // back; otherwise the boxes take turns in the warp's own 2 KB buffer.
        const bool last_seg = walk.i == walk.count;
        uint8_t* ring = smem + C::OFF_STAGE + warp * (16 * DBLK * 4);
        const CUtensorMap* map = to_final ? &tm_out : &tm_part;
        const int x0 = to_final ? branch * p.d_blk_out : branch * DBLK;
        const int z = to_final ? seg.seq : range + seg.seq;
        const int row = lane & 15;
        if (last_seg) {
          // both halves of every 64-column chunk at once (distinct boxes), one fence, then the
          // whole warp's boxes are issued together
#pragma unroll 1
          for (int ch = 0; ch < C::OCH; ++ch) {
#pragma unroll 1
            for (int c0 = 0; c0 < C::OCW; c0 += 64) {
              uint32_t r[32];
              tmem_ld16x2_32(tmem + ((uint32_t)(32 * warp + 16) << 16) + ch * C::OCW + c0, r);
              tmem_wait_ld();
              const int col = ch * C::OCW + c0 + 32 * q;
              if (col < ncols_out) {
                uint8_t* buf = ring + (col / 32) * C::STG_BYTES;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                  *reinterpret_cast<float4*>(buf + row * 128 + ((k ^ (row & 7)) << 4)) =
                      make_float4(__uint_as_float(r[4 * k]) * scale, __uint_as_float(r[4 * k + 1]) * scale,
                                  __uint_as_float(r[4 * k + 2]) * scale, __uint_as_float(r[4 * k + 3]) * scale);
              }
            }
          }
          fence_proxy_async_smem();  // the staged boxes are read by the bulk copies (async proxy)
          __syncwarp();
          if (lane == 0) {
            for (int col = 0; col < ncols_out && col < DBLK; col += 32)
              tma_store_3d(map, smem_u32(ring + (col / 32) * C::STG_BYTES), x0 + col, h0 + 16 * warp, z);
            bulk_commit();
          }
        } else {
#pragma unroll 1
          for (int ch = 0; ch < C::OCH; ++ch) {
#pragma unroll 1
            for (int c0 = 0; c0 < C::OCW; c0 += 64) {
              uint32_t r[32];
              tmem_ld16x2_32(tmem + ((uint32_t)(32 * warp + 16) << 16) + ch * C::OCW + c0, r);
              tmem_wait_ld();
#pragma unroll
              for (int half = 0; half < 2; ++half) {
                const int col = ch * C::OCW + c0 + 32 * half;  // column inside the branch block
                if (col >= ncols_out) continue;
                if (lane == 0 && stg_pending) bulk_wait_read_all();
                __syncwarp();
                if (q == half) {
#pragma unroll
                  for (int k = 0; k < 8; ++k)
                    *reinterpret_cast<float4*>(stg + row * 128 + ((k ^ (row & 7)) << 4)) =
                        make_float4(__uint_as_float(r[4 * k]) * scale, __uint_as_float(r[4 * k + 1]) * scale,
                                    __uint_as_float(r[4 * k + 2]) * scale, __uint_as_float(r[4 * k + 3]) * scale);
                }
                fence_proxy_async_smem();  // the staged box is read by the bulk copy (async proxy)
                __syncwarp();
                if (lane == 0) {
                  tma_store_3d(map, stg_u, x0 + col, h0 + 16 * warp, z);
                  bulk_commit();
                }
                stg_pending = true;
              }
            }
          }
        }
      } else {
        float* dst = p.out + ((int64_t)seg.seq * p.H + h) * p.out_width + (int64_t)branch * p.d_blk_out;
#pragma unroll 1
        for (int ch = 0; ch < C::OCH; ++ch) {
#pragma unroll 1
          for (int c0 = 0; c0 < C::OCW; c0 += 64) {
            uint32_t r[32];
            tmem_ld16x2_32(tmem + ((uint32_t)(32 * warp + 16) << 16) + ch * C::OCW + c0, r);
            tmem_wait_ld();
            if (live) {
              const int cbase = ch * C::OCW + c0 + 32 * q;
              if (cbase + 32 <= ncols_out && ((reinterpret_cast<uintptr_t>(dst + cbase)) & 15) == 0) {
#pragma unroll
                for (int k = 0; k < 32; k += 4) {
                  float4 o4 = make_float4(__uint_as_float(r[k]) * scale, __uint_as_float(r[k + 1]) * scale,
                                          __uint_as_float(r[k + 2]) * scale, __uint_as_float(r[k + 3]) * scale);
                  *reinterpret_cast<float4*>(dst + cbase + k) = o4;
                }
              } else {
#pragma unroll
                for (int k = 0; k < 32; ++k)
                  if (cbase + k < ncols_out) dst[cbase + k] = __uint_as_float(r[k]) * scale;
              }
            }
          }
        }
      }
      if (live && q == 0) {
        if (to_final) {
          if (p.lse) p.lse[((int64_t)seg.seq * p.H + h) * p.B + branch] = (m_used + __log2f(l_sum)) * 0.69314718055994531f;
        } else {
          const int64_t slot = (int64_t)range + seg.seq;
          float* ml = p.part_ml + ((slot * p.H + h) * p.B + branch) * 2;
          ml[0] = m_used;
          ml[1] = l_sum;
        }
      }
    }
    // the staged boxes must stay in shared memory until the bulk stores have read them; their
    // global writes complete with the grid, before a dependent kernel's wait returns
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, C::TMEM_COLS);
  if (threadIdx.x == 0) p.cta_flags[blockIdx.x] = *flags;  // folded into the status word by K2
}

}  // namespace mlra
