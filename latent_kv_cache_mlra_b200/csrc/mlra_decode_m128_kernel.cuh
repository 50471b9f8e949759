// mlra_decode_m128_kernel.cuh -- K1M: the attention kernel with 128 query rows per CTA.
//
// The same computation as K1 (mlra_decode_kernel.cuh: step 2 of the absorbed decode, section 1.3
// of the "Multi-Head Low-Rank Attention" page, in the branch form of section 3.1), for calls that
// carry 128 query rows against the same cache rows: two consecutive query tokens of one sequence
// with 64 heads each (several new tokens per sequence, causal among them), or one token of 128
// heads (rows = heads, unit_tokens = 1).  Every tcgen05 product then has M = 128 rows, the tensor
// core's full rate, and each cache tile is read once for all 128 rows:
//   score:  S[128 x 128]  = Q[128 x d] . C_b^T  +  Q^R[128 x 64] . K^R^T     (TMEM, fp32)
//   output: O[128 x d]   += P[128 x 128] . C_b[128 x d]                     (TMEM, fp32)
// For two tokens, rows 0..63 are the unit's first token (heads 0..63), rows 64..127 its second;
// the first token sits one position earlier, so its row attends one position fewer.
//
// One persistent CTA per (work range, branch); a work range covers units (pairs of tokens of a
// sequence) exactly as K1's ranges cover sequences (mlra_plan.cuh).  Branch width 128, tiles of
// 128 positions.  The latent blocks of a tile (32 KB, read by both products) sit in a ring of
// NS = 4 stages; its RoPE block (16 KB, read by the score product only) in a ring of its own of
// NR = 2 slots, so that the 48 KB of queries leave room for four latent stages.
//
// TMEM (512 columns, all 128 lanes): O in columns [0, 128); one score buffer of 128 columns; four
// P slots of 64 columns (bf16 pairs), one per latent stage.  The softmax warps release the score
// buffer as soon as they have loaded it (the next tile's score product may start), and write a
// tile's P into its stage's P slot: the landed tile implies the output product that last read
// the slot (four tiles earlier) completed.  The output product reads P from TMEM (A operand).
//
// Warps (352 threads): 0-7 softmax, 8 TMA producer, 9 score-MMA issuer and TMEM owner, 10
// output-MMA issuer.  Softmax warp w reads the 16 TMEM lanes 32 (w % 4) + 16 (w / 4) .. + 15 (one
// row each) in the 16-lane load shape: lanes l and l + 16 of the warp share row l % 16, lane l
// taking the positions 64 k + 32 (l / 16) .. + 31 (k = 0, 1) of every tile, so a row's maximum and
// sum need one shuffle.  P is released in two halves (positions 64 k ..), each once all 256
// softmax threads wrote it.
//
// Ordering facts the parity waits rely on (a barrier at most one phase past the phase awaited):
//   * latent tile s loads after the output product of tile s - NS completed; RoPE block s loads
//     after the score product of tile s - NR completed;
//   * the score of tile s is issued after the softmax loaded the scores of tile s - 1 (one score
//     buffer), so the score issuer runs at most one tile ahead of the softmax;
//   * the softmax writes P of tile s into slot s % NS: tile s landed after the output product of
//     tile s - NS, the slot's last reader, completed.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <math_constants.h>

#include "mlra_decode_kernel.cuh"
#include "mlra_internal.h"
#include "mlra_plan.cuh"
#include "sm100_ptx.cuh"

namespace mlra {

template <int NS>
struct DecodeM128Cfg {
  static constexpr int DBLK = 128, T = 128, QR = 128;
  static constexpr int NCB = DBLK / 64;             // 64-column latent blocks
  static constexpr int TB = T / 64;                 // 64-row sub-boxes per tile
  static constexpr int BOX = 64 * 64 * 2;           // cache box [64 rows x 64 columns] bf16
  static constexpr int QBOX = QR * 64 * 2;          // query box [128 rows x 64 columns] bf16
  static constexpr int CBLK = T * 128;              // one 64-column block of a tile
  static constexpr int STAGE = NCB * CBLK;          // the latent blocks of a tile
  static constexpr int NR = 2;                      // RoPE slots
  static constexpr int QBYTES = (NCB + 1) * QBOX;   // query blocks + RoPE-query block
  static constexpr int O_COLS = DBLK;
  static constexpr int NSB = 1;                     // score buffers
  static constexpr int NP = NS;                     // P slots, one per latent stage
  static constexpr int S_COL = O_COLS;              // first score buffer
  static constexpr int P_COL = S_COL + NSB * T;     // first P slot (T / 2 columns each)
  static constexpr int NPV = NS;
  static constexpr int TMEM_COLS = 512;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_STAGE = QBYTES;
  static constexpr int OFF_ROPE = OFF_STAGE + NS * STAGE;
  static constexpr int OFF_BAR = OFF_ROPE + NR * CBLK;
  static constexpr int NBAR = 2 * NS + 2 * NR + 2 + 2 * NSB + TB * NP + NPV + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_PLAN = OFF_MISC + 16;
  static constexpr int PLAN_BYTES = 16 * kSelfPlanMaxSeqs + 4 * kSelfPlanMaxSeqs + 16;
  static constexpr int OFF_HOOK_BAR = OFF_PLAN + 20 * kSelfPlanMaxSeqs + 8;  // force_timeout
  static_assert(OFF_HOOK_BAR % 8 == 0 && OFF_HOOK_BAR + 8 <= OFF_PLAN + PLAN_BYTES, "hook barrier");
  static constexpr int SMEM = OFF_PLAN + PLAN_BYTES;
  static constexpr int SMEM_ALLOC = SMEM + 1024;
  static_assert(P_COL + NP * (T / 2) <= TMEM_COLS, "TMEM budget");
  static_assert(NSB == 1 && NP == NS, "one score buffer; a P slot per latent stage");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

constexpr int kDecodeM128Threads = 352;

template <int NS>
__global__ void __launch_bounds__(kDecodeM128Threads, 1)
mlra_decode_m128_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                        const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_kr,
                        const __grid_constant__ DecodeParams p) {
  using C = DecodeM128Cfg<NS>;
  constexpr int NSB = C::NSB, NPV = C::NPV, T = C::T;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sStage = sbase + C::OFF_STAGE;
  const uint32_t sRope = sbase + C::OFF_ROPE;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t bar_stage_full = bar0;                      // [NS]  TMA -> MMA
  const uint32_t bar_stage_empty = bar0 + 8 * NS;            // [NS]  MMA (PV done) -> TMA
  const uint32_t bar_rope_full = bar0 + 16 * NS;             // [NR]  TMA -> MMA
  const uint32_t bar_rope_empty = bar_rope_full + 8 * C::NR;  // [NR]  MMA (score done) -> TMA
  const uint32_t bar_q_full = bar_rope_empty + 8 * C::NR;    //       TMA -> MMA
  const uint32_t bar_q_empty = bar_q_full + 8;               //       MMA (last score) -> TMA
  const uint32_t bar_s_full = bar_q_full + 16;               // [NSB] MMA (score) -> softmax
  const uint32_t bar_s_free = bar_s_full + 8 * NSB;          // [NSB] softmax (scores loaded) -> MMA
  const uint32_t bar_p_full = bar_s_free + 8 * NSB;          // [TB][NP] softmax (P half) -> MMA
  const uint32_t bar_pv_done = bar_p_full + 8 * C::TB * C::NP;  // [NPV] MMA (PV done) -> softmax
  const uint32_t bar_final_s = bar_pv_done + 8 * NPV;
  const uint32_t bar_final_pv = bar_final_s + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  uint32_t* spec_flags = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 8);
  uint32_t* flags = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 12);
  uint8_t* plan = smem + C::OFF_PLAN;
  volatile int32_t* plan_count = reinterpret_cast<volatile int32_t*>(plan + 20 * kSelfPlanMaxSeqs);
  volatile int32_t* plan_stale = plan_count + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int range = blockIdx.x / p.n_groups;
  const int branch = blockIdx.x % p.n_groups;
  const uint64_t tmo = p.timeout_ns;
  pdl_launch_dependents();

  auto init_barriers = [&]() {
    for (int k = 0; k < NS; ++k) {
      mbar_init(bar_stage_full + 8 * k, 1);
      mbar_init(bar_stage_empty + 8 * k, 1);
    }
    for (int k = 0; k < C::NR; ++k) {
      mbar_init(bar_rope_full + 8 * k, 1);
      mbar_init(bar_rope_empty + 8 * k, 1);
    }
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, 1);
    for (int k = 0; k < NSB; ++k) {
      mbar_init(bar_s_full + 8 * k, 1);
      mbar_init(bar_s_free + 8 * k, 256);
    }
    for (int k = 0; k < C::TB * C::NP; ++k) mbar_init(bar_p_full + 8 * k, 256);
    for (int k = 0; k < NPV; ++k) mbar_init(bar_pv_done + 8 * k, 1);
    mbar_init(bar_final_s, 1);
    mbar_init(bar_final_pv, 1);
  };
  if (threadIdx.x == 0) {
    init_barriers();
    *abort_flag = 0;
    *spec_flags = 0;
    *flags = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_qr);
    tma_prefetch_desc(&tm_c);
    tma_prefetch_desc(&tm_kr);
  }
  // speculative plan over the units (see K1)
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
  const int col0 = branch * C::DBLK;
  int4 first_seg = make_int4(0, 0, 0, 0);
  const bool speculate = p.self_plan && warp == 8 && *plan_count > 0;
  if (speculate) first_seg = reinterpret_cast<const int4*>(plan)[0];

  const uint64_t once = l2_policy_evict_first();
  auto issue_latent = [&](int st, const int (&rows)[C::TB]) {
    const uint32_t full = bar_stage_full + 8 * st;
    const uint32_t dst = sStage + st * C::STAGE;
    mbar_arrive_expect_tx(full, C::STAGE);
#pragma unroll
    for (int l = 0; l < C::TB; ++l)
#pragma unroll
      for (int k = 0; k < C::NCB; ++k)
        tma_load_2d_hint(dst + k * C::CBLK + l * C::BOX, &tm_c, full, col0 + 64 * k, rows[l], once);
  };
  auto issue_rope = [&](int rs, const int (&rows)[C::TB]) {
    const uint32_t full = bar_rope_full + 8 * rs;
    mbar_arrive_expect_tx(full, C::CBLK);
#pragma unroll
    for (int l = 0; l < C::TB; ++l)
      tma_load_2d(sRope + rs * C::CBLK + l * C::BOX, &tm_kr, full, 0, rows[l]);
  };
  auto issue_queries = [&](int unit) {  // the unit's 128 query rows
    mbar_arrive_expect_tx(bar_q_full, C::QBYTES);
#pragma unroll
    for (int k = 0; k < C::NCB; ++k)
      tma_load_3d(sQ + k * C::QBOX, &tm_q, bar_q_full, col0 + 64 * k, 0, unit);
    tma_load_3d(sQ + C::NCB * C::QBOX, &tm_qr, bar_q_full, 0, 0, unit);
  };
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

  pdl_wait_prerequisites();
  int pre_tiles = 0;   // latent tiles of the first segment already issued
  int pre_rope = 0;    // ... and RoPE blocks
  bool pre_q = false;
  if (p.self_plan) {
    if (speculate) {
      const int len = first_seg.w & 0x7fffffff;
      pre_tiles = first_seg.z < NS ? first_seg.z : NS;
      pre_rope = pre_tiles < C::NR ? pre_tiles : C::NR;
      pre_q = true;
      const int cache_seq = first_seg.x / p.q_per_seq;
      if (lane == 0) issue_queries(first_seg.x);
      for (int i = 0; i < pre_tiles; ++i) {
        int rows[C::TB];
        tile_rows(cache_seq, first_seg.y + i, len, spec_flags, rows);
        if (lane == 0) {
          if (i < pre_rope) issue_rope(i, rows);
          issue_latent(i, rows);
        }
      }
      __syncwarp();
    }
    if (warp == 0) {
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
      plan_commit(p, range, branch, plan_bits, flags);
    }
    __syncthreads();
    if (*plan_stale) {
      if (speculate) {
        if (pre_q) wait_warp(bar_q_full, 0, tmo, abort_flag, flags, false);
        for (int i = 0; i < pre_tiles; ++i)
          wait_warp(bar_stage_full + 8 * i, 0, tmo, abort_flag, flags, false);
        for (int i = 0; i < pre_rope; ++i)
          wait_warp(bar_rope_full + 8 * i, 0, tmo, abort_flag, flags, false);
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        for (int k = 0; k < C::NBAR; ++k) mbar_inval(bar0 + 8 * k);
        init_barriers();
        fence_barrier_init();
      }
      __syncthreads();
      pre_tiles = 0;
      pre_rope = 0;
      pre_q = false;
    } else if (speculate && lane == 0) {
      atomicOr(flags, *spec_flags);
    }
    if (blockIdx.x == 0 && warp >= 1 && warp < 7) plan_empty_outputs(p, plan);
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

  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    SegCursor walk(seg_list, list_global, seg_count);
    Segment seg;
    int L = 0;
    int it = 0, nseg = 0;
    int lat_issued = pre_tiles, rope_issued = pre_rope;  // copies issued so far (for a drain)
    int q_loads = pre_q ? 1 : 0;
    bool ok = true;
    while (ok && walk.next(seg, L)) {
      if (nseg > 0) ok = wait_warp(bar_q_empty, (nseg - 1) & 1, tmo, abort_flag, flags);
      if (!ok) break;
      if (!(nseg == 0 && pre_q)) {
        if (lane == 0) issue_queries(seg.seq);
        ++q_loads;
      }
      __syncwarp();
      const int cache_seq = seg.seq / p.q_per_seq;
      for (int i = 0; i < seg.ntiles; ++i, ++it) {
        const bool latent_done = nseg == 0 && i < pre_tiles;  // issued before the plan was
        const bool rope_done = nseg == 0 && i < pre_rope;     // confirmed
        if (latent_done && rope_done) continue;
        if (p.force_timeout) {
          ok = forced_timeout_wait(smem_u32(smem + C::OFF_HOOK_BAR), tmo >> 10, abort_flag, flags,
                                   lane);
          if (!ok) break;
        }
        int rows[C::TB];
        tile_rows(cache_seq, seg.tile0 + i, L, flags, rows);
        if (!latent_done) {
          const int st = it % NS;
          if (it >= NS) {
            ok = wait_warp(bar_stage_empty + 8 * st, ((it / NS) - 1) & 1, tmo, abort_flag, flags);
            if (!ok) break;
          }
          if (lane == 0) issue_latent(st, rows);
          ++lat_issued;
        }
        if (!rope_done) {
          const int rs = it % C::NR;
          if (it >= C::NR) {
            ok = wait_warp(bar_rope_empty + 8 * rs, ((it / C::NR) - 1) & 1, tmo, abort_flag, flags);
            if (!ok) break;
          }
          if (lane == 0) issue_rope(rs, rows);
          ++rope_issued;
        }
        __syncwarp();
      }
      ++nseg;
    }
    if (!ok) {
      // let the copies already issued land before the CTA can exit
      if (q_loads > 0) wait_warp(bar_q_full, (q_loads - 1) & 1, tmo / 8, abort_flag, flags, false);
      for (int k = (lat_issued > NS ? lat_issued - NS : 0); k < lat_issued; ++k)
        wait_warp(bar_stage_full + 8 * (k % NS), (k / NS) & 1, tmo / 8, abort_flag, flags, false);
      for (int k = (rope_issued > C::NR ? rope_issued - C::NR : 0); k < rope_issued; ++k)
        wait_warp(bar_rope_full + 8 * (k % C::NR), (k / C::NR) & 1, tmo / 8, abort_flag, flags, false);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ score-MMA issuer
    constexpr uint32_t kIdScore = idesc_bf16_f32(128, T, false, false);
    SegCursor walk(seg_list, list_global, seg_count);
    Segment seg;
    int L = 0;
    int it = 0, nseg = 0;
    bool ok = true;
    while (ok && walk.next(seg, L)) {
      ok = wait_warp(bar_q_full, nseg & 1, tmo, abort_flag, flags);
      for (int i = 0; ok && i < seg.ntiles; ++i, ++it) {
        ok = wait_warp(bar_stage_full + 8 * (it % NS), (it / NS) & 1, tmo, abort_flag, flags);
        if (ok)
          ok = wait_warp(bar_rope_full + 8 * (it % C::NR), (it / C::NR) & 1, tmo, abort_flag, flags);
        if (ok && it >= NSB)  // score buffer free: the softmax loaded the scores of tile it - 1
          ok = wait_warp(bar_s_free + 8 * ((it - NSB) % NSB), ((it - NSB) / NSB) & 1, tmo,
                         abort_flag, flags);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t stg = sStage + (it % NS) * C::STAGE;
          const uint32_t rope = sRope + (it % C::NR) * C::CBLK;
          const uint32_t d = tmem + C::S_COL + (it % NSB) * T;
#pragma unroll
          for (int kb = 0; kb < C::NCB; ++kb) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sw128_desc(sQ + kb * C::QBOX + kk * 32, 16, 1024);
              const uint64_t bd = sw128_desc(stg + kb * C::CBLK + kk * 32, 16, 1024);
              umma_bf16(d, ad, bd, kIdScore, (kb | kk) ? 1u : 0u);
            }
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sw128_desc(sQ + C::NCB * C::QBOX + kk * 32, 16, 1024);
            const uint64_t bd = sw128_desc(rope + kk * 32, 16, 1024);
            umma_bf16(d, ad, bd, kIdScore, 1u);
          }
          umma_commit(bar_s_full + 8 * (it % NSB));
          umma_commit(bar_rope_empty + 8 * (it % C::NR));
          if (i == seg.ntiles - 1) umma_commit(bar_q_empty);
        }
        __syncwarp();
      }
      ++nseg;
    }
    if (lane == 0) umma_commit(bar_final_s);
    __syncwarp();
    wait_warp(bar_final_s, 0, tmo, abort_flag, flags, false);
  } else if (warp == 10) {
    // ------------------------------------------------------------------ output-MMA issuer
    constexpr uint32_t kIdPV = idesc_bf16_f32(128, C::DBLK, false, true);
    SegCursor walk(seg_list, list_global, seg_count);
    Segment seg;
    int L = 0;
    int j = 0;
    bool ok = true;
    while (ok && walk.next(seg, L)) {
      for (int i = 0; ok && i < seg.ntiles; ++i, ++j) {
        const uint32_t stg = sStage + (j % NS) * C::STAGE;
        const uint32_t pa = tmem + C::P_COL + (j % C::NP) * (T / 2);  // P slot of the tile
#pragma unroll 1
        for (int hb = 0; hb < C::TB; ++hb) {
          ok = wait_warp(bar_p_full + 8 * (hb * C::NP + j % C::NP), (j / C::NP) & 1, tmo,
                         abort_flag, flags);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            const bool first = (i == 0 && hb == 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const int k16 = 4 * hb + kk;  // 16 positions: 8 TMEM columns of P
              const uint64_t bd = sw128_desc(stg + k16 * 2048, C::CBLK, 1024);
              umma_bf16_ts(tmem, pa + 8 * k16, bd, kIdPV, (kk > 0 || !first) ? 1u : 0u);
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
    // ------------------------------------------------------------------ softmax warps 0-7
    const int q = lane >> 4;                               // which 32 of every 64 positions
    const int row = 32 * (warp & 3) + 16 * (warp >> 2) + (lane & 15);  // query row (TMEM lane)
    // token row / 64 of the unit, head row % 64
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3) + 16 * (warp >> 2)) << 16;
    SegCursor walk(seg_list, list_global, seg_count);
    Segment seg;
    int L = 0;
    int it = 0;
    bool ok = true;
    while (ok && walk.next(seg, L)) {
      // the unit's first token (rows 0..63) attends one position fewer than its second
      const int row_len = L - (row < 64 ? p.unit_tokens - 1 : 0);
      float m_used = -CUDART_INF_F, l_sum = 0.f;
      for (int i = 0; i < seg.ntiles; ++i, ++it) {
        const int t = seg.tile0 + i;
        ok = wait_warp(bar_s_full + 8 * (it % NSB), (it / NSB) & 1, tmo, abort_flag, flags);
        if (!ok) break;
        tc_fence_after();
        // v[32 k + j] = score of position 64 k + 32 q + j
        float v[64];
        const uint32_t sbuf = tmem + lane_base + C::S_COL + (it % NSB) * T;
        tmem_ld16x2_32(sbuf, reinterpret_cast<uint32_t(&)[32]>(v[0]));
        tmem_ld16x2_32(sbuf + 64, reinterpret_cast<uint32_t(&)[32]>(v[32]));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar_s_free + 8 * (it % NSB));  // the score buffer may take the next tile
        const int rvalid = min(T, row_len - T * t);  // positions of this row in the tile
        const int tile_valid = min(T, L - T * t);    // of the unit's longest row
        const float sc = p.scale_log2;
        const bool whole = rvalid >= T;
        float mx;
        if (whole) {
          float a[4] = {v[0], v[1], v[2], v[3]};
          if (sc >= 0.f) {
#pragma unroll
            for (int k = 4; k < 64; k += 2) a[(k >> 1) & 3] = max3f(a[(k >> 1) & 3], v[k], v[k + 1]);
            mx = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])) * sc;
          } else {
#pragma unroll
            for (int k = 4; k < 64; k += 2) a[(k >> 1) & 3] = min3f(a[(k >> 1) & 3], v[k], v[k + 1]);
            mx = fminf(fminf(a[0], a[1]), fminf(a[2], a[3])) * sc;
          }
        } else {
          mx = -CUDART_INF_F;
#pragma unroll
          for (int k = 0; k < 64; ++k) {
            const float x = 64 * (k >> 5) + 32 * q + (k & 31) < rvalid ? v[k] * sc : -CUDART_INF_F;
            v[k] = x;
            mx = fmaxf(mx, x);
          }
        }
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));  // the row's maximum over the tile
        bool rescale = false;
        float alpha = 1.f;
        if (mx == -CUDART_INF_F) {
          // no position of this row in the tile (its token ends earlier): nothing changes
        } else if (m_used == -CUDART_INF_F) {
          alpha = 0.f;
          m_used = mx;
        } else if (mx > m_used + 8.f) {  // lazy rescale: only when p could exceed 2^8
          alpha = ex2_approx(m_used - mx);
          m_used = mx;
          rescale = true;
        }
        l_sum *= (i == 0 ? 1.f : alpha);
        if (__any_sync(kFull, rescale)) {
          // O holds the output products up to tile it-1: wait for them, then scale this thread's
          // 64 columns of its row
          ok = wait_warp(bar_pv_done + 8 * ((it - 1) % NPV), ((it - 1) / NPV) & 1, tmo, abort_flag,
                         flags);
          if (!ok) break;
          tc_fence_after();
          const float f = rescale ? alpha : 1.f;
#pragma unroll 1
          for (int c0 = 0; c0 < C::DBLK; c0 += 64) {
            uint32_t r[32];
            tmem_ld16x2_32(tmem + lane_base + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * f);
            tmem_st16x2_32(tmem + lane_base + c0, r);
          }
          tmem_wait_st();
        }
        // Ragged last tile: the latent rows past the unit's end are zeroed before P is released
        // (a zero probability must never meet a non-finite value left in the cache).
        uint8_t* stage_ptr = smem + C::OFF_STAGE + (it % NS) * C::STAGE;
        if (tile_valid < T) {
          const int tid = threadIdx.x;  // the 256 softmax threads
          for (int k = tid; k < C::NCB * T * 8; k += 256) {
            const int r = (k >> 3) % T;
            if (r >= tile_valid)
              *reinterpret_cast<uint4*>(stage_ptr + (k / (T * 8)) * C::CBLK + r * 128 + (k & 7) * 16) =
                  make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
        // P: positions 64 k + 32 q + j -> bf16 pairs in columns 32 k + 16 q + j / 2 of the tile's
        // P slot, released half k by half k
        const float mul = whole ? sc : 1.f;
        const float neg_m = m_used == -CUDART_INF_F ? 0.f : -m_used;
        const float2 mul2 = make_float2(mul, mul), negm2 = make_float2(neg_m, neg_m);
        float2 sum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        const uint32_t pslot = tmem + lane_base + C::P_COL + (it % C::NP) * (T / 2);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 32; k += 2) {  // pairs through the packed two-lane FMA and add
            const float2 x = __ffma2_rn(make_float2(v[32 * kb + k], v[32 * kb + k + 1]), mul2, negm2);
            const float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
            sum2[(k >> 1) & 1] = __fadd2_rn(sum2[(k >> 1) & 1], make_float2(p0, p1));
            pk[k / 2] = pack_bf16x2(p0, p1);
          }
          tmem_st16x2_16(pslot + 32 * kb, pk);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar_p_full + 8 * (kb * C::NP + it % C::NP));
        }
        l_sum += (sum2[0].x + sum2[0].y) + (sum2[1].x + sum2[1].y);
      }
      if (!ok) break;
      // ------------------------------------------------ epilogue of the segment
      ok = wait_warp(bar_pv_done + 8 * ((it - 1) % NPV), ((it - 1) / NPV) & 1, tmo, abort_flag,
                     flags);
      if (!ok) break;
      tc_fence_after();
      const float l_row = l_sum + __shfl_xor_sync(kFull, l_sum, 16);
      const bool to_final = seg.whole && p.write_final;
      const float scale = to_final ? (l_row > 0.f ? p.gamma / l_row : 0.f) : 1.f;
      float* dst;
      if (to_final)
        dst = p.out + ((int64_t)seg.seq * C::QR + row) * p.out_width + (int64_t)branch * p.d_blk_out;
      else
        dst = p.part_o + (((int64_t)range + seg.seq) * C::QR + row) * p.dck + (int64_t)branch * C::DBLK;
#pragma unroll 1
      for (int c0 = 0; c0 < C::DBLK; c0 += 64) {
        uint32_t r[32];
        tmem_ld16x2_32(tmem + lane_base + c0, r);
        tmem_wait_ld();
        const int col = c0 + 32 * q;  // this thread's 32 columns
        if (!to_final || col + 32 <= p.d_blk_out) {
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            *reinterpret_cast<float4*>(dst + col + k) =
                make_float4(__uint_as_float(r[k]) * scale, __uint_as_float(r[k + 1]) * scale,
                            __uint_as_float(r[k + 2]) * scale, __uint_as_float(r[k + 3]) * scale);
        }
      }
      if (q == 0) {
        if (to_final) {
          if (p.lse)
            p.lse[((int64_t)seg.seq * C::QR + row) * p.B + branch] =
                l_row > 0.f ? (m_used + __log2f(l_row)) * 0.69314718055994531f : -CUDART_INF_F;
        } else {
          float* ml = p.part_ml + ((((int64_t)range + seg.seq) * C::QR + row) * p.B + branch) * 2;
          ml[0] = m_used;
          ml[1] = l_row;
        }
      }
      tc_fence_before();  // the O loads precede the next segment's first (overwriting) product
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, C::TMEM_COLS);
  if (threadIdx.x == 0) p.cta_flags[blockIdx.x] = *flags;
}

}  // namespace mlra
