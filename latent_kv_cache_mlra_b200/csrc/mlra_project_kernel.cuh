// mlra_project_kernel.cuh -- K5: the per-head products of steps 1 and 3 of the absorbed decode.
//
// "Multi-Head Low-Rank Attention" (yunpan.plus page), section 1.3:
//   step 3 with the branch sum of sections 3 and 3.3 -- the value up-projection of every branch
//     output, summed over the branches.  With head h's projections side by side,
//     W_h = [W^UV_{h,1} | ... | W^UV_{h,B}] (d_head x d_latent), and o[s, h] the concatenated branch
//     outputs of step 2 (gamma applied):  y[s, h, :] = W_h o[s, h, :];
//   step 1 -- the absorbed query q~[s, h, b-block] = (W^UK_{h,b})^T q[s, h], i.e. the product with
//     the transpose of [W^UK_{h,1} | ... | W^UK_{h,B}] (d_head x d_latent).
// Both are x_out[s, h, :] = A_h x_in[s, h, :] with A_h of d_out x d_in.
// One CTA per (head, 64 rows of A_h, 64 sequences): a tcgen05 product with M = 64 rows of A_h,
// N = the sequences (padded to a multiple of 8), K = d_in, accumulated in TMEM.
//   * A is packed once (mlra_pack_kernel, at model load) into the product's shared-memory image:
//     per (head, 64-row tile) d_in / 64 boxes of [64 rows x 64 columns] bf16 in the 128-byte
//     swizzled K-major layout, contiguous, so each box arrives with one contiguous bulk copy.
//     The copies are issued first thing, before the wait on the previous kernel (A is never
//     written by it), so under programmatic serialization the weight stream overlaps its tail;
//   * x_in (fp32) is rounded to bf16 by all threads into the same swizzled K-major layout;
//   * one thread issues the d_in / 16 MMAs, a group of four boxes (one copy, one mbarrier) at a
//     time; the epilogue reads D with tcgen05.ld, transposes it through shared memory and writes
//     x_out in fp32 or bf16 with 16-byte stores (64 consecutive rows of one sequence).
// The work is bound by streaming A (H d_out d_in bf16) from HBM.
//
// Merge mode (step 3 fused behind the attention kernel, no combine kernel between them): the x
// row of a sequence split over several work ranges is merged from its partial results while it is
// staged (the combine's fold, mlra_merge.cuh), and block 0 writes the call's status word.
#pragma once
#include <cstdint>
#include <cuda.h>

#include <cuda_bf16.h>

#include "mlra_internal.h"
#include "mlra_merge.cuh"
#include "sm100_ptx.cuh"

namespace mlra {

// Threads per CTA: 128 for the plain products (warps 0-3 read the accumulator), 256 when the
// staging also merges split sequences (more loads in flight; warps 0-3 still read the accumulator).
constexpr int kProjThreads = 128, kProjMergeThreads = 256;
constexpr int kProjM = 64;     // rows of A_h per CTA
constexpr int kProjN = 64;     // sequences per CTA
constexpr int kProjBox = 8192; // one [64 x 64] bf16 box
constexpr int kProjGroup = 4;  // boxes per weight copy and per mbarrier (32 KB)

// A_h (d_out x d_in) -> the packed image: tile t = h * (d_out / 64) + m, box kb, row r: the
// 16-byte chunk j of columns kb * 64 + 8 j .. + 7 at byte r * 128 + 16 (j ^ (r & 7)).  The
// source w is [H, d_out, d_in] row-major (A_h = w[h]), or with `transpose` [H, d_in, d_out]
// (A_h = w[h]^T).
__global__ void __launch_bounds__(256) mlra_pack_kernel(const uint16_t* w, uint16_t* packed, int H,
                                                        int d_in, int d_out, int transpose) {
  const int KB = d_in / 64;
  const int64_t chunks = (int64_t)H * d_out * d_in / 8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < chunks;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t box = i >> 9;            // 512 chunks of 16 bytes per 8 KB box
    const int within = static_cast<int>(i & 511);
    const int r = within >> 3, jpos = within & 7, j = jpos ^ (r & 7);
    const int64_t t = box / KB;
    const int kb = static_cast<int>(box - t * KB);
    const int64_t row = t * kProjM + r;    // = h * d_out + m * 64 + r
    const int col = kb * 64 + j * 8;
    uint4 v;
    if (!transpose) {
      v = *reinterpret_cast<const uint4*>(w + row * d_in + col);
    } else {
      const int64_t h = row / d_out, o = row - h * d_out;
      uint16_t e[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) e[u] = w[(h * d_in + col + u) * d_out + o];
      v = make_uint4(e[0] | ((uint32_t)e[1] << 16), e[2] | ((uint32_t)e[3] << 16),
                     e[4] | ((uint32_t)e[5] << 16), e[6] | ((uint32_t)e[7] << 16));
    }
    *reinterpret_cast<uint4*>(packed + i * 8) = v;
  }
}

// shared memory: A boxes, x boxes, an mbarrier per group of A boxes (at most one per box) and
// one for the products, the TMEM address and a flag
inline int project_smem_bytes(int kb) { return 2 * kb * kProjBox + 8 * (kb + 1) + 16 + 1024; }

__device__ __forceinline__ bool project_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                             uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > timeout_ns) {
      if (status) atomicOr(status, kFlagTimeout);
      return false;
    }
  }
  return true;
}

template <int kThreads, bool kMerge>
__global__ void __launch_bounds__(kThreads, 1)
mlra_project_kernel(const __grid_constant__ ProjectParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int KB = p.d_in / 64;
  uint8_t* sW = smem;
  uint8_t* sX = smem + KB * kProjBox;
  const uint32_t bar_full = smem_u32(sX + KB * kProjBox);  // [groups]: W boxes of group g landed
  const uint32_t bar_done = bar_full + 8 * KB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sX + KB * kProjBox + 8 * (KB + 1));
  volatile uint32_t* issued_all = tmem_slot + 1;  // every product was issued (no time-out)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mtiles = p.d_out / kProjM;
  const int h = blockIdx.x / mtiles, m0 = (blockIdx.x % mtiles) * kProjM;
  const int n0 = blockIdx.y * kProjN;
  const int rows_n = min(kProjN, p.N - n0);
  const int npad = (rows_n + 7) / 8 * 8;

  const int ngroups = (KB + kProjGroup - 1) / kProjGroup;
  if (threadIdx.x == 0) {
    for (int g = 0; g < ngroups; ++g) mbar_init(bar_full + 8 * g, 1);
    mbar_init(bar_done, 1);
    fence_barrier_init();
    // The packed weights are constant (packed at load), never the output of the previous kernel
    // on the stream: their stream starts before the wait below, under that kernel's tail.  The
    // boxes of a group are contiguous in the packed image: one copy (and one mbarrier) each.
    const uint8_t* src = reinterpret_cast<const uint8_t*>(p.w_packed) +
                         ((int64_t)h * mtiles + m0 / kProjM) * KB * kProjBox;
    for (int g = 0; g < ngroups; ++g) {
      const int kb0 = g * kProjGroup;
      const uint32_t bytes = (uint32_t)(min(KB - kb0, kProjGroup) * kProjBox);
      mbar_arrive_expect_tx(bar_full + 8 * g, bytes);
      bulk_load(smem_u32(sW + kb0 * kProjBox), src + kb0 * kProjBox, bytes, bar_full + 8 * g);
    }
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // x comes from the previous kernel on the stream (programmatic serialization); the next kernel
  // may start its own prologue now (it waits for this grid before reading what it writes)
  pdl_wait_prerequisites();
  pdl_launch_dependents();
  // o[n0 + r, h, :] -> bf16, box kb holds columns 64 kb .. 64 kb + 63 of row r at 128 r, its
  // 16-byte chunk j at position j ^ (r & 7).  Only the npad rows the products read are staged
  // (rows past the batch as zeros); the loads of 8 chunks are issued before any is converted.
  constexpr int kU = 8;
  const int chunks = npad * KB * 8;
  if (kMerge && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < 32) {
    // the call's status word: the bits every attention CTA (and the prep kernel) raised
    uint32_t f = 0;
    for (int i = threadIdx.x; i < p.n_flag_slots; i += 32) f |= __ldcg(p.cta_flags + i);
    f = __reduce_or_sync(0xffffffffu, f);
    if (threadIdx.x == 0) *p.status = f;  // (a time-out of this kernel is ORed in after it)
  }
  if constexpr (kMerge) {
    // 8 columns (one branch) of row r per chunk: the attention kernel's final row, or the merge
    // of the sequence's parts.  Each thread takes two chunks at a time and keeps the loads of
    // both chunks' next kMergeBatch parts in flight (one memory round trip covers them).
    constexpr int kMergeBatch = 4;
    for (int base = threadIdx.x; base < chunks; base += 2 * kThreads) {
      int np[2], r0[2], s_[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int idx = base + c * kThreads;
        const int r = idx / (KB * 8);
        np[c] = 0;
        r0[c] = 0;
        s_[c] = n0 + r;
        if (idx < chunks && r < rows_n) {
          const int2 si = __ldcg(reinterpret_cast<const int2*>(p.seqs + s_[c]));
          np[c] = si.y - si.x + 1;
          r0[c] = si.x;
        } else {
          np[c] = -1;  // a padding row or past the chunks: zeros
        }
      }
      float4 a[2], b4[2];
      MergeState lo[2] = {merge_empty(), merge_empty()}, hi[2] = {merge_empty(), merge_empty()};
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        a[c] = b4[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        const int idx = base + c * kThreads;
        const int cidx = idx % (KB * 8);
        if (np[c] == 0 || np[c] == 1) {
          const float4* src = reinterpret_cast<const float4*>(p.x + ((int64_t)s_[c] * p.H + h) * p.d_in + cidx * 8);
          a[c] = __ldcg(src);
          b4[c] = __ldcg(src + 1);
        }
      }
      const int npmax = max(np[0], np[1]);
      for (int q0 = 0; npmax > 1 && q0 < npmax; q0 += kMergeBatch) {
        float2 ml[2][kMergeBatch];
        float4 va[2][kMergeBatch], vb[2][kMergeBatch];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int col = ((base + c * kThreads) % (KB * 8)) * 8;
          const int br = col / p.dblk;
#pragma unroll
          for (int u = 0; u < kMergeBatch; ++u) {
            if (np[c] > 1 && q0 + u < np[c]) {
              const int64_t row = ((int64_t)r0[c] + q0 + u + s_[c]) * p.H + h;
              ml[c][u] = __ldcg(reinterpret_cast<const float2*>(p.part_ml + (row * p.B + br) * 2));
              const float4* o = reinterpret_cast<const float4*>(p.part_o + row * p.d_in + col);
              va[c][u] = __ldcg(o);
              vb[c][u] = __ldcg(o + 1);
            }
          }
        }
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int u = 0; u < kMergeBatch; ++u)
            if (np[c] > 1 && q0 + u < np[c]) {
              merge_into(lo[c], ml[c][u].x, ml[c][u].y, va[c][u]);
              merge_into(hi[c], ml[c][u].x, ml[c][u].y, vb[c][u]);
            }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int idx = base + c * kThreads;
        if (idx >= chunks) continue;
        const int r = idx / (KB * 8), cidx = idx - r * (KB * 8);
        const int kb = cidx >> 3, j = cidx & 7;
        if (np[c] > 1) {
          const float sc = p.gamma / lo[c].l;
          a[c] = make_float4(lo[c].acc.x * sc, lo[c].acc.y * sc, lo[c].acc.z * sc, lo[c].acc.w * sc);
          b4[c] = make_float4(hi[c].acc.x * sc, hi[c].acc.y * sc, hi[c].acc.z * sc, hi[c].acc.w * sc);
        }
        *reinterpret_cast<uint4*>(sX + kb * kProjBox + r * 128 + ((j ^ (r & 7)) << 4)) =
            make_uint4(pack_bf16x2(a[c].x, a[c].y), pack_bf16x2(a[c].z, a[c].w),
                       pack_bf16x2(b4[c].x, b4[c].y), pack_bf16x2(b4[c].z, b4[c].w));
      }
    }
  }
  for (int base = kMerge ? chunks : threadIdx.x; base < chunks; base += kThreads * kU) {
    float4 va[kU], vb[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int idx = base + u * kThreads;
      const int r = idx / (KB * 8), cidx = idx - r * (KB * 8);
      va[u] = vb[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (idx < chunks && r < rows_n) {
        const float4* src = reinterpret_cast<const float4*>(
            p.x + ((int64_t)(n0 + r) * p.H + h) * p.d_in + cidx * 8);
        va[u] = __ldcg(src);
        vb[u] = __ldcg(src + 1);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int idx = base + u * kThreads;
      if (idx >= chunks) break;
      const int r = idx / (KB * 8), cidx = idx - r * (KB * 8);
      const int kb = cidx >> 3, j = cidx & 7;
      *reinterpret_cast<uint4*>(sX + kb * kProjBox + r * 128 + ((j ^ (r & 7)) << 4)) =
          make_uint4(pack_bf16x2(va[u].x, va[u].y), pack_bf16x2(va[u].z, va[u].w),
                     pack_bf16x2(vb[u].x, vb[u].y), pack_bf16x2(vb[u].z, vb[u].w));
    }
  }
  fence_proxy_async_smem();  // read by the MMA (async proxy)
  __syncthreads();

  bool ok = true;
  if (threadIdx.x == 0) {
    // the products of a group start as soon as it lands; within a group they are issued back to
    // back (a wait between two products costs more than the product)
    const uint32_t idesc = idesc_bf16_f32(kProjM, npad, false, false);
    for (int g = 0; ok && g < ngroups; ++g) {
      ok = project_wait(bar_full + 8 * g, 0, p.timeout_ns, p.status);
      if (!ok) break;
      tc_fence_after();
      for (int kb = g * kProjGroup; kb < min(KB, (g + 1) * kProjGroup); ++kb) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tmem, sw128_desc(smem_u32(sW + kb * kProjBox) + kk * 32, 16, 1024),
                    sw128_desc(smem_u32(sX + kb * kProjBox) + kk * 32, 16, 1024), idesc,
                    (kb | kk) ? 1u : 0u);
      }
    }
    *issued_all = ok ? 1u : 0u;
    umma_commit(bar_done);  // also after a time-out: it tracks whatever was issued
  }
  __syncthreads();
  // every thread waits for the products (bounded); the epilogue runs only if the whole block saw
  // them complete (it has block-wide barriers)
  const bool done = __syncthreads_and(project_wait(bar_done, 0, p.timeout_ns,
                                                   threadIdx.x == 0 ? p.status : nullptr)) != 0;
  if (done && *issued_all) {
    tc_fence_after();
    // D rows 16 w .. 16 w + 15 live in lanes 32 w + [0, 16); lane half q holds columns
    // 32 q .. 32 q + 31 (the sequences n0 + column).  They go through shared memory (the A boxes
    // are free now) as sT[column][row], so that each output row segment of 64 values leaves as
    // 16-byte stores: one scattered 4-byte store per value costs several times more.
    float* sT = reinterpret_cast<float*>(sW);  // [64][64] fp32 = 16 KB <= 2 * KB * 8 KB
    if (warp < 4) {  // the accumulator's sub-partitions
      uint32_t r[32];
      tmem_ld16x2_32(tmem + ((uint32_t)(32 * warp) << 16), r);
      tmem_wait_ld();
      const int q = lane >> 4, rr = 16 * warp + (lane & 15);
#pragma unroll
      for (int k = 0; k < 32; ++k) sT[(32 * q + k) * kProjM + rr] = __uint_as_float(r[k]);
    }
    __syncthreads();
    if (p.out_bf16) {
      // 8 rows (16 bytes) per store
      for (int it = threadIdx.x; it < rows_n * (kProjM / 8); it += kThreads) {
        const int col = it / (kProjM / 8), c8 = it % (kProjM / 8);
        const float4 a = *reinterpret_cast<const float4*>(sT + col * kProjM + 8 * c8);
        const float4 b = *reinterpret_cast<const float4*>(sT + col * kProjM + 8 * c8 + 4);
        const int64_t at = ((int64_t)(n0 + col) * p.H + h) * p.d_out + m0 + 8 * c8;
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.y) + at) =
            make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                       pack_bf16x2(b.z, b.w));
      }
    } else {
      // 4 rows (16 bytes) per store
      for (int it = threadIdx.x; it < rows_n * (kProjM / 4); it += kThreads) {
        const int col = it / (kProjM / 4), c4 = it % (kProjM / 4);
        const int64_t at = ((int64_t)(n0 + col) * p.H + h) * p.d_out + m0 + 4 * c4;
        *reinterpret_cast<float4*>(static_cast<float*>(p.y) + at) =
            *reinterpret_cast<const float4*>(sT + col * kProjM + 4 * c4);
      }
    }
  }
  if (threadIdx.x == 0 && !*issued_all)  // after a time-out: let the weight copies land (bounded)
    for (int g = 0; g < ngroups; ++g) project_wait(bar_full + 8 * g, 0, p.timeout_ns / 8, nullptr);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 64);
}

}  // namespace mlra
