// mlra_decode_kernel.cuh -- K1: split-KV MLRA decode attention on sm_100a.
//
// Computes step 2 of the absorbed three-step decode ("Multi-Head Low-Rank Attention",
// yunpan.plus page, section 1.3) for the branch form of section 3.1: for every branch b,
// scores of the absorbed query block against latent block c_b plus the shared RoPE term,
// an online softmax of its own over positions, and the probability-weighted sum of c_b.
//
// One persistent CTA per (work range, branch group).  A work range is a contiguous run of KV
// tiles (64 positions) of the batch (see mlra_plan.cuh); a branch group is G branches whose
// latent columns the CTA reads.  Heads are the M = 64 rows of every tcgen05 MMA:
//   score:  S_b[64 x T]  = Q~_b[64 x d_blk] . C_b^T  +  Q^R[64 x 64] . K^R^T   (TMEM, fp32)
//   output: O_b[64 x d]  += P_b[64 x T] . C_b[T x d]                             (TMEM, fp32)
// The RoPE product is accumulated into every branch's score tile by the same MMA chain.
//
// TMEM: an M = 64 accumulator occupies 16 of the 32 lanes of each sub-partition; two
// accumulators share columns in the lower (lanes 0-15) and upper (lanes 16-31) halves.
//   G = 2: half x holds branch x of the group: O_x in columns [0, d_blk), S_x in two
//          buffers of 64 columns after it.
//   G = 1: the single branch is split by half: half x holds output columns
//          [x d_blk/2, (x+1) d_blk/2) and the scores of tile positions [32x, 32x+32).
// Softmax thread (warp w < 4, lane l) owns TMEM lane 32w + l: head 16w + (l & 15), half l >> 4.
//
// Warp roles (192 threads): warps 0-3 softmax / rescale / epilogue, warp 4 TMA producer,
// warp 5 MMA issuer and TMEM owner.  Shared memory: the group's queries (resident per
// segment), an NS-deep ring of cache tiles, NP probability buffers, mbarriers.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <math_constants.h>

#include "mlra_internal.h"
#include "mlra_plan.cuh"
#include "sm100_ptx.cuh"

namespace mlra {

template <int DBLK, int G, int NS, int NP>
struct DecodeCfg {
  static constexpr int T = kTile;
  static constexpr int DG = DBLK * G;               // latent columns per CTA
  static constexpr int NCB = DG / 64;               // 64-column boxes of latent per tile
  static constexpr int BOX = 64 * 64 * 2;           // one [64 x 64] bf16 box, 8 KB
  static constexpr int STAGE = (NCB + 1) * BOX;     // latent boxes + RoPE box
  static constexpr int QBYTES = (NCB + 1) * BOX;    // query boxes + RoPE-query box
  static constexpr int PBYTES = G * BOX;            // P_g [64 heads x 64 positions] bf16
  static constexpr int O_COLS = (G == 2) ? DBLK : DBLK / 2;
  static constexpr int S_COLS = (G == 2) ? T : T / 2;
  static constexpr int N_SCORE = S_COLS;
  static constexpr int N_PV = O_COLS;
  static constexpr int TMEM_USED = O_COLS + 2 * S_COLS;
  static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 :
                                   TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_STAGE = QBYTES;
  static constexpr int OFF_P = OFF_STAGE + NS * STAGE;
  static constexpr int OFF_BAR = OFF_P + NP * PBYTES;
  static constexpr int NBAR = 2 * NS + 9;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM + 1024;    // slack to align the base to 1024 B
  static_assert(DBLK % 64 == 0 && (G == 1 || G == 2), "branch width must be a multiple of 64");
  static_assert(G == 2 || DBLK >= 128, "single-branch CTAs need d_blk >= 128");
  static_assert(N_PV % 8 == 0 && N_PV <= 256, "UMMA N must be a multiple of 8, at most 256");
  static_assert(TMEM_USED <= 512, "TMEM budget");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

constexpr uint32_t kFull = 0xffffffffu;

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

// First cache row of tile t (positions [64t, 64t+64)) of sequence s.  Shared by the decode
// kernel and the row-resolution test hook.  An invalid page id flags the status word and
// returns a row past the end of the cache, where TMA reads zeros.
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

template <int DBLK, int G, int NS, int NP>
__global__ void __launch_bounds__(192, 1)
mlra_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                   const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_kr,
                   const __grid_constant__ DecodeParams p) {
  using C = DecodeCfg<DBLK, G, NS, NP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sStage = sbase + C::OFF_STAGE;
  const uint32_t sP = sbase + C::OFF_P;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  // barrier map
  const uint32_t bar_stage_full = bar0;                 // [NS]
  const uint32_t bar_stage_empty = bar0 + 8 * NS;       // [NS]
  const uint32_t bar_q_full = bar0 + 16 * NS;
  const uint32_t bar_q_empty = bar_q_full + 8;
  const uint32_t bar_s_full = bar_q_full + 16;          // [2]
  const uint32_t bar_p_full = bar_q_full + 32;          // [2]
  // PV of tile j commits to bar_pv_done[j & 1].  Two barriers keep every waiter within one
  // phase of the phase it waits for (the commit before on the same barrier, PV of tile j-2, is
  // known to be complete), which a parity wait needs to be unambiguous.
  const uint32_t bar_pv_done = bar_q_full + 48;         // [2]
  const uint32_t bar_final = bar_q_full + 64;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int range = blockIdx.x / p.n_groups;
  const int group = blockIdx.x % p.n_groups;
  const int64_t total = p.prefix[p.N];
  const int64_t R = effective_ranges(p.num_ranges, total);
  const uint64_t tmo = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int k = 0; k < NS; ++k) {
      mbar_init(bar_stage_full + 8 * k, 1);
      mbar_init(bar_stage_empty + 8 * k, 1);
    }
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, 1);
    mbar_init(bar_s_full, 1);
    mbar_init(bar_s_full + 8, 1);
    mbar_init(bar_p_full, 128);
    mbar_init(bar_p_full + 8, 128);
    mbar_init(bar_pv_done, 1);
    mbar_init(bar_pv_done + 8, 1);
    mbar_init(bar_final, 1);
    *abort_flag = 0;
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
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    SegmentWalker walk(p.prefix, p.N, total, R, range);
    Segment seg;
    int it = 0, nseg = 0;
    bool ok = true;
    const int col0 = group * C::DG;
    while (ok && walk.next(seg)) {
      if (nseg > 0) ok = wait_warp(bar_q_empty, (nseg - 1) & 1, tmo, abort_flag, p.status);
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar_q_full, C::QBYTES);
#pragma unroll
        for (int k = 0; k < C::NCB; ++k)
          tma_load_3d(sQ + k * C::BOX, &tm_q, bar_q_full, col0 + 64 * k, 0, seg.seq);
        tma_load_3d(sQ + C::NCB * C::BOX, &tm_qr, bar_q_full, 0, 0, seg.seq);
      }
      __syncwarp();
      for (int i = 0; i < seg.ntiles; ++i, ++it) {
        const int row0 = tile_row(p.page_table, p.max_pages, p.page_size, p.max_seq_len,
                                  p.n_pages, p.oob_row, seg.seq, seg.tile0 + i,
                                  lane == 0 ? p.status : nullptr);
        const int st = it % NS;
        if (it >= NS) {
          ok = wait_warp(bar_stage_empty + 8 * st, ((it / NS) - 1) & 1, tmo, abort_flag, p.status);
          if (!ok) break;
        }
        if (lane == 0) {
          const uint32_t full = bar_stage_full + 8 * st;
          const uint32_t dst = sStage + st * C::STAGE;
          mbar_arrive_expect_tx(full, C::STAGE);
#pragma unroll
          for (int k = 0; k < C::NCB; ++k) tma_load_2d(dst + k * C::BOX, &tm_c, full, col0 + 64 * k, row0);
          tma_load_2d(dst + C::NCB * C::BOX, &tm_kr, full, 0, row0);
        }
        __syncwarp();
      }
      ++nseg;
    }
    if (!ok) {
      // Aborting: let the copies already issued land before the CTA can exit.
      if (nseg > 0) wait_warp(bar_q_full, (nseg - 1) & 1, tmo / 8, abort_flag, p.status, false);
      for (int k = (it > NS ? it - NS : 0); k < it; ++k)
        wait_warp(bar_stage_full + 8 * (k % NS), (k / NS) & 1, tmo / 8, abort_flag, p.status, false);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdScore = idesc_bf16_f32(64, C::N_SCORE, false, false);
    constexpr uint32_t kIdPV = idesc_bf16_f32(64, C::N_PV, false, true);
    SegmentWalker walk(p.prefix, p.N, total, R, range);
    Segment seg;
    int it = 0, nseg = 0, prev = -1;
    bool prev_first = false, ok = true;

    auto issue_pv = [&](int j, bool first) -> bool {
      if (!wait_warp(bar_p_full + 8 * (j & 1), (j >> 1) & 1, tmo, abort_flag, p.status)) return false;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t pbuf = sP + (j % NP) * C::PBYTES;
        const uint32_t stg = sStage + (j % NS) * C::STAGE;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const uint32_t d = tmem + ((uint32_t)(16 * x) << 16);
          const uint32_t a0 = pbuf + (G == 2 ? x * C::BOX : 0);
          const uint32_t b0 = stg + (G == 2 ? x * (DBLK / 64) : x * (DBLK / 128)) * C::BOX;
#pragma unroll
          for (int kk = 0; kk < C::T / 16; ++kk) {
            const uint64_t ad = sw128_desc(a0 + kk * 32, 16, 1024);
            const uint64_t bd = sw128_desc(b0 + kk * 2048, C::BOX, 1024);
            umma_bf16(d, ad, bd, kIdPV, (kk > 0 || !first) ? 1u : 0u);
          }
        }
        umma_commit(bar_stage_empty + 8 * (j % NS));
        umma_commit(bar_pv_done + 8 * (j & 1));
      }
      __syncwarp();
      return true;
    };

    while (ok && walk.next(seg)) {
      for (int i = 0; i < seg.ntiles; ++i, ++it) {
        if (i == 0) {
          // Finish the previous segment first so that its epilogue overlaps this query load.
          if (prev >= 0) {
            ok = issue_pv(prev, prev_first);
            if (!ok) break;
            prev = -1;
          }
          ok = wait_warp(bar_q_full, nseg & 1, tmo, abort_flag, p.status);
          if (!ok) break;
        }
        ok = wait_warp(bar_stage_full + 8 * (it % NS), (it / NS) & 1, tmo, abort_flag, p.status);
        if (!ok) break;
        if (it >= 2) {
          // score buffer (it & 1) is free once the softmax of tile it-2 has read it
          ok = wait_warp(bar_p_full + 8 * (it & 1), ((it - 2) >> 1) & 1, tmo, abort_flag, p.status);
          if (!ok) break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t stg = sStage + (it % NS) * C::STAGE;
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const uint32_t d = tmem + ((uint32_t)(16 * x) << 16) + C::O_COLS + (it & 1) * C::S_COLS;
            const int box0 = (G == 2) ? x * (DBLK / 64) : 0;
            const uint32_t brow = (G == 2) ? 0u : (uint32_t)x * 4096u;  // 32 rows of 128 B
#pragma unroll
            for (int kb = 0; kb < DBLK / 64; ++kb) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = sw128_desc(sQ + (box0 + kb) * C::BOX + kk * 32, 16, 1024);
                const uint64_t bd = sw128_desc(stg + (box0 + kb) * C::BOX + brow + kk * 32, 16, 1024);
                umma_bf16(d, ad, bd, kIdScore, (kb | kk) ? 1u : 0u);
              }
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sw128_desc(sQ + C::NCB * C::BOX + kk * 32, 16, 1024);
              const uint64_t bd = sw128_desc(stg + C::NCB * C::BOX + brow + kk * 32, 16, 1024);
              umma_bf16(d, ad, bd, kIdScore, 1u);
            }
          }
          umma_commit(bar_s_full + 8 * (it & 1));
          if (i == seg.ntiles - 1) umma_commit(bar_q_empty);
        }
        __syncwarp();
        if (prev >= 0) {
          ok = issue_pv(prev, prev_first);
          if (!ok) break;
        }
        prev = it;
        prev_first = (i == 0);
      }
      ++nseg;
    }
    if (ok && prev >= 0) issue_pv(prev, prev_first);
    // Nothing of ours may still run on the tensor core when TMEM is released.
    if (lane == 0) umma_commit(bar_final);
    __syncwarp();
    wait_warp(bar_final, 0, tmo, abort_flag, p.status, false);
  } else {
    // ------------------------------------------------------------------ softmax warps 0-3
    const int half = lane >> 4;
    const int h = 16 * warp + (lane & 15);
    const int branch = (G == 2) ? group * 2 + half : group;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * warp) << 16);
    const int tok0 = (G == 2) ? 0 : 32 * half;       // first tile position of this thread's scores
    const int ocol0 = (G == 2) ? 0 : half * (DBLK / 2);  // first output column of this thread
    SegmentWalker walk(p.prefix, p.N, total, R, range);
    Segment seg;
    int it = 0;
    bool ok = true;
    while (ok && walk.next(seg)) {
      const int L = p.lens[seg.seq];
      float m_used = -CUDART_INF_F, l_sum = 0.f;
      for (int i = 0; i < seg.ntiles; ++i, ++it) {
        const int t = seg.tile0 + i;
        ok = wait_warp(bar_s_full + 8 * (it & 1), (it >> 1) & 1, tmo, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        float v[C::S_COLS];
#pragma unroll
        for (int c0 = 0; c0 < C::S_COLS; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(lane_addr + C::O_COLS + (it & 1) * C::S_COLS + c0, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) v[c0 + k] = __uint_as_float(r[k]);
        }
        const int valid = min(C::T, L - C::T * t);
        float mx = -CUDART_INF_F;
#pragma unroll
        for (int c = 0; c < C::S_COLS; ++c) {
          const float x = (tok0 + c < valid) ? v[c] * p.scale_log2 : -CUDART_INF_F;
          v[c] = x;
          mx = fmaxf(mx, x);
        }
        if (G == 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
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
        const bool warp_rescale = __any_sync(kFull, rescale);
        if ((warp_rescale || NP == 1) && it > 0) {
          // O (rescale) and the single P buffer are only free once PV of tile it-1 is done
          ok = wait_warp(bar_pv_done + 8 * ((it - 1) & 1), ((it - 1) >> 1) & 1, tmo, abort_flag,
                         p.status);
          if (!ok) break;
          tc_fence_after();
        }
        if (warp_rescale) {
#pragma unroll 1
          for (int c0 = 0; c0 < C::O_COLS; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(lane_addr + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
            tmem_st32(lane_addr + c0, r);
          }
          tmem_wait_st();
        }
        // probabilities -> bf16 P tile (K-major, 128-byte swizzle), row h
        float sum = 0.f;
        uint32_t pk[C::S_COLS / 2];
#pragma unroll
        for (int c = 0; c < C::S_COLS; c += 2) {
          const float p0 = ex2_approx(v[c] - m_used);
          const float p1 = ex2_approx(v[c + 1] - m_used);
          sum += p0 + p1;
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
        if (G == 1) sum += __shfl_xor_sync(kFull, sum, 16);
        l_sum += sum;
        {
          uint8_t* prow = smem + C::OFF_P + (it % NP) * C::PBYTES + (G == 2 ? half * C::BOX : 0) + h * 128;
#pragma unroll
          for (int q = 0; q < C::S_COLS / 8; ++q) {
            const int chunk = tok0 / 8 + q;
            uint4 val = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            *reinterpret_cast<uint4*>(prow + ((chunk ^ (h & 7)) << 4)) = val;
          }
        }
        if (valid < C::T) {
          // Ragged last tile: zero the latent rows past the sequence end so that the zero
          // probabilities never multiply a non-finite value left in the cache.
          ok = wait_warp(bar_stage_full + 8 * (it % NS), (it / NS) & 1, tmo, abort_flag, p.status);
          if (!ok) break;
          uint8_t* stg = smem + C::OFF_STAGE + (it % NS) * C::STAGE;
          for (int k = threadIdx.x; k < C::NCB * 64 * 8; k += 128) {
            const int row = (k >> 3) & 63;
            if (row >= valid)
              *reinterpret_cast<uint4*>(stg + (k >> 9) * C::BOX + row * 128 + (k & 7) * 16) =
                  make_uint4(0u, 0u, 0u, 0u);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar_p_full + 8 * (it & 1));
      }
      if (!ok) break;
      // ------------------------------------------------ epilogue of the segment
      ok = wait_warp(bar_pv_done + 8 * ((it - 1) & 1), ((it - 1) >> 1) & 1, tmo, abort_flag,
                     p.status);
      if (!ok) break;
      tc_fence_after();
      const bool to_final = seg.whole && p.write_final;
      const bool live = h < p.H;
      float* dst;
      float scale;
      int ncols_out;
      if (to_final) {
        dst = p.out + ((int64_t)seg.seq * p.H + h) * p.out_width + (int64_t)branch * p.d_blk_out;
        scale = p.gamma / l_sum;
        ncols_out = p.d_blk_out;
      } else {
        const int64_t slot = (int64_t)range + seg.seq;
        dst = p.part_o + (slot * p.H + h) * p.dck + (int64_t)branch * DBLK;
        scale = 1.f;
        ncols_out = DBLK;
      }
#pragma unroll 1
      for (int c0 = 0; c0 < C::O_COLS; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lane_addr + c0, r);
        tmem_wait_ld();
        if (live) {
          const int cbase = ocol0 + c0;
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
      if (live && (G == 2 || half == 0)) {
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
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace mlra
