// mlra_kernels.cu -- device kernels of the MLRA decode library and their launchers.
//   K0 mlra_prep_kernel      lengths -> clamped lengths, tile prefix sums, segment
//                            descriptors, empty-sequence outputs, status word reset
//   K1 mlra_decode_kernel    split-KV decode attention (mlra_decode_kernel.cuh)
//   K2 mlra_combine_kernel   merges the partial softmax states of split sequences
//   K3 mlra_repack_kernel    fp32 / odd-width inputs -> padded bf16 copies in the workspace
//   mlra_resolve_rows_kernel test hook for the cache-row addressing of K1
#include <cuda_bf16.h>
#include <math_constants.h>

#include "mlra_decode_kernel.cuh"
#include "mlra_merge.cuh"
#include "sm100_ptx.cuh"
#include "mlra_internal.h"
#include "mlra_plan.cuh"

namespace mlra {

// ----------------------------------------------------------------------------- K0
// One block.  seq_lens outside [0, limit] set kFlagBadLength and are clamped; the status word
// is rewritten so that it reports this call only.  prefix counts tiles of `tile` positions.
// Then the split plan for the decode and combine kernels: per work range its segment
// descriptors (range r's first descriptor sits at r + its first sequence, which keeps the
// ranges' descriptor blocks disjoint) and per sequence the ranges holding it.  Empty sequences
// get out = 0, lse = -inf here.  For up to kPrepSmemSeqs sequences the prefix and the lengths
// are also kept in shared memory, where the per-range searches read them.
constexpr int kPrepSmemSeqs = 4096;

__global__ void __launch_bounds__(1024) mlra_prep_kernel(const PrepParams p) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t carry;
  __shared__ uint32_t flags;
  extern __shared__ int32_t sh_plan[];  // [N + 1] prefix, [N] lens (when N <= kPrepSmemSeqs)
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int N = p.N;
  const bool in_smem = N <= kPrepSmemSeqs;
  int32_t* prefix = in_smem ? sh_plan : p.prefix;
  int32_t* lens = in_smem ? sh_plan + N + 1 : p.lens;
  pdl_launch_dependents();  // the decode kernel may start its prologue now
  if (tid == 0) {
    carry = 0;
    flags = 0;
    prefix[0] = 0;
  }
  __syncthreads();
  for (int base = 0; base < N; base += 1024) {
    const int i = base + tid;
    int tiles = 0;
    if (i < N) {
      int L = p.seq_lens[i];
      if (L < 0 || L > p.limit) {
        atomicOr(&flags, kFlagBadLength);
        L = L < 0 ? 0 : p.limit;
      }
      lens[i] = L;
      tiles = (L + p.tile - 1) / p.tile;
    }
    int x = tiles;  // inclusive warp scan
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int incl = x + (wid > 0 ? warp_tot[wid - 1] : 0) + carry;
    if (i < N) prefix[i + 1] = incl;
    __syncthreads();
    if (tid == 1023) carry = incl;
    __syncthreads();
  }
  // prefix and lens written above are visible to the whole block after the last __syncthreads
  const int64_t total = prefix[N];
  const int64_t R = effective_ranges(p.num_ranges, total);
  for (int r = tid; r < p.num_ranges; r += blockDim.x) {
    RangeInfo ri{0, 0};
    if (r < R && total > 0) {
      SegmentWalker walk(prefix, N, total, R, r);
      Segment seg;
      ri.first = -1;
      while (walk.next(seg)) {
        if (ri.first < 0) ri.first = r + seg.seq;
        SegDesc d;
        d.seq = seg.seq;
        d.tile0 = seg.tile0;
        d.ntiles = seg.ntiles;
        d.len_whole = lens[seg.seq] | (seg.whole ? (int32_t)0x80000000u : 0);
        p.segs[ri.first + ri.count] = d;
        ++ri.count;
      }
    }
    p.ranges[r] = ri;
  }
  for (int sq = tid; sq < N; sq += blockDim.x) {
    SeqInfo si{0, 0};
    if (total > 0) seq_parts(prefix, sq, total, R, &si.r0, &si.nparts);
    p.seqs[sq] = si;
  }
  for (int sq = wid; sq < N; sq += 32) {  // empty sequences (a warp each): out = 0, lse = -inf
    if (lens[sq] != 0) continue;
    float* row = p.out + (int64_t)sq * p.H * p.out_width;
    for (int i = lane; i < p.H * p.out_width; i += 32) row[i] = 0.f;
    if (p.lse)
      for (int i = lane; i < p.H * p.B; i += 32) p.lse[(int64_t)sq * p.H * p.B + i] = -CUDART_INF_F;
  }
  if (tid == 0) *p.status = flags;
}

cudaError_t launch_prep(const PrepParams& p, cudaStream_t st) {
  const size_t sh = p.N <= kPrepSmemSeqs ? (2 * (size_t)p.N + 1) * sizeof(int32_t) : 0;
  mlra_prep_kernel<<<1, 1024, sh, st>>>(p);
  return cudaGetLastError();
}

// ----------------------------------------------------------------------------- K1
template <int DBLK, int T, int NS>
static cudaError_t launch_decode_t(const CUtensorMap& tq, const CUtensorMap& tqr,
                                   const CUtensorMap& tc, const CUtensorMap& tkr,
                                   const DecodeParams& p, int grid, cudaStream_t st) {
  using C = DecodeCfg<DBLK, T, NS>;
  auto kern = mlra_decode_kernel<DBLK, T, NS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDecodeThreads);
  cfg.dynamicSmemBytes = C::SMEM_ALLOC;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlap with the prep kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tq, tqr, tc, tkr, p);
}

// (padded branch width, positions per tile, cache-tile stages)
#define MLRA_VARIANTS(X) \
  X(kV64, 64, 128, 4)    \
  X(kV128, 128, 128, 4)  \
  X(kV256, 256, 128, 2)  \
  X(kV512, 512, 64, 2)

int variant_smem_bytes(Variant v) {
  switch (v) {
#define X(id, D, T, NS) case id: return DecodeCfg<D, T, NS>::SMEM_ALLOC;
    MLRA_VARIANTS(X)
#undef X
    default: return 0;
  }
}

int variant_tile(Variant v) {
  switch (v) {
#define X(id, D, T, NS) case id: return T;
    MLRA_VARIANTS(X)
#undef X
    default: return 0;
  }
}

cudaError_t launch_decode(Variant v, const CUtensorMap& tq, const CUtensorMap& tqr,
                          const CUtensorMap& tc, const CUtensorMap& tkr, const DecodeParams& p,
                          int grid, cudaStream_t st) {
  switch (v) {
#define X(id, D, T, NS) case id: return launch_decode_t<D, T, NS>(tq, tqr, tc, tkr, p, grid, st);
    MLRA_VARIANTS(X)
#undef X
    default: return cudaErrorInvalidValue;
  }
}

// ----------------------------------------------------------------------------- K2
// Merge of split sequences.  For sequence s split into np parts (ranges r0 .. r0+np-1; part p
// in slot r0 + p + s), per head h and branch b the parts are folded as in mlra_merge.cuh;
// summed mode adds the branches' gamma o* / l*.  Launched with programmatic stream
// serialization: its blocks may be scheduled during the decode kernel and wait for it.
// Grid (N, ceil(H / HG), column chunks of 128), 256 threads = 8 warps = HG heads x G part groups.
// Lane t of a warp covers 4 columns (128 per warp); part group g takes parts g, g+G, ...; the G
// group states of a head are merged in shared memory.  Empty sequences were written by K0.
constexpr int kCombineWarps = 8;

__global__ void __launch_bounds__(kCombineWarps * 32) mlra_combine_kernel(const CombineParams p) {
  __shared__ MergeState part[kCombineWarps][32];
  const int s = blockIdx.x;
  const int G = p.groups, HG = kCombineWarps / G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * HG + warp / G, g = warp % G;
  const bool live_h = h < p.H;
  // padded column of this lane: branch mode over [0, dck), summed mode over [0, dblk_k)
  const int k = blockIdx.z * 128 + 4 * lane;
  const bool live = live_h && k < (p.summed ? p.dblk_k : p.dck);
  pdl_wait_prerequisites();  // the decode kernel's partials must be complete and visible
  const int2 si = __ldcg(reinterpret_cast<const int2*>(p.seqs + s));  // (r0, nparts)
  const int np = si.y;
  if (np == 0 || (np == 1 && p.final_written)) return;  // written by K0 / by the decode kernel
  const int width = p.summed ? p.d_blk_out : p.B * p.d_blk_out;
  float* out_row = p.out + ((int64_t)s * p.H + h) * width;
  const int64_t slot0 = (int64_t)si.x + s;
  const int b_lo = p.summed ? 0 : k / p.dblk_k;
  const int b_hi = p.summed ? p.B : b_lo + 1;
  MergeState tot = merge_empty();
  tot.acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int b = b_lo; b < b_hi; ++b) {  // block-uniform trip count (1 in branch mode)
    const int kb = p.summed ? b * p.dblk_k + k : k;
    MergeState st = merge_empty();
    if (live) st = fold_parts(p.part_ml, p.part_o, p.H, p.B, p.dck, slot0, np, g, G, h, b, kb);
    if (G > 1) {
      part[warp][lane] = st;
      __syncthreads();
      if (g == 0)
        for (int j = 1; j < G; ++j) {
          const MergeState o = part[warp + j][lane];
          merge_into(st, o.m, o.l, o.acc);
        }
      __syncthreads();  // part[] is rewritten by the next branch
    }
    if (!live || g != 0) continue;
    if (p.lse && (p.summed ? (blockIdx.z == 0 && lane == 0) : (k - b * p.dblk_k == 0)))
      p.lse[((int64_t)s * p.H + h) * p.B + b] = merged_lse(st);
    if (p.summed) {
      const float sc = p.gamma / st.l;
      tot.acc.x += st.acc.x * sc; tot.acc.y += st.acc.y * sc;
      tot.acc.z += st.acc.z * sc; tot.acc.w += st.acc.w * sc;
    } else {
      const int kk = k - b * p.dblk_k;
      if (kk < p.d_blk_out) store_merged(out_row + b * p.d_blk_out + kk, st, p.gamma, p.d_blk_out - kk);
    }
  }
  if (p.summed && live && g == 0 && k < p.d_blk_out) {
    tot.l = 1.f;
    store_merged(out_row + k, tot, 1.f, p.d_blk_out - k);
  }
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t st) {
  if (p.groups < 1 || p.groups > kCombineWarps || kCombineWarps % p.groups != 0)
    return cudaErrorInvalidValue;
  const int HG = kCombineWarps / p.groups;
  const int kspan = p.summed ? p.dblk_k : p.dck;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.N, (p.H + HG - 1) / HG, (kspan + 127) / 128);
  cfg.blockDim = dim3(kCombineWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlap the decode tail
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mlra_combine_kernel, p);
}

// ----------------------------------------------------------------------------- K3
template <typename Src>
__device__ __forceinline__ uint16_t to_bf16_bits(Src x);
template <>
__device__ __forceinline__ uint16_t to_bf16_bits<float>(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}
template <>
__device__ __forceinline__ uint16_t to_bf16_bits<uint16_t>(uint16_t x) {
  return x;
}

// Copies a [rows x cols] matrix (row pitch src_pitch) into a [rows x (B * dk)] bf16 matrix whose
// branch blocks of width d are padded with zeros to dk; with B == 1 and dk >= d it pads columns.
template <typename Src>
__device__ void repack_matrix(const Src* src, int64_t src_pitch, uint16_t* dst, int64_t rows,
                              int B, int d, int dk) {
  const int64_t width = (int64_t)B * dk;
  const int64_t n = rows * width;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / width;
    const int c = static_cast<int>(i - r * width);
    const int b = c / dk, k = c - b * dk;
    dst[i] = (k < d) ? to_bf16_bits<Src>(src[r * src_pitch + (int64_t)b * d + k]) : (uint16_t)0;
  }
}

template <typename Src>
__global__ void mlra_repack_kernel(const RepackParams p) {
  const int64_t nh = (int64_t)p.N * p.H;
  switch (blockIdx.y) {
    case 0: repack_matrix<Src>((const Src*)p.q_lat, (int64_t)p.B * p.d_blk, p.q_out, nh, p.B, p.d_blk, p.dblk_k); break;
    case 1: repack_matrix<Src>((const Src*)p.q_rope, p.d_rope, p.qr_out, nh, 1, p.d_rope, 64); break;
    case 2: repack_matrix<Src>((const Src*)p.c_kv, p.c_row_stride, p.c_out, p.rows, p.B, p.d_blk, p.dblk_k); break;
    default: repack_matrix<Src>((const Src*)p.k_rope, p.kr_row_stride, p.kr_out, p.rows, 1, p.d_rope, 64); break;
  }
}

cudaError_t launch_repack(const RepackParams& p, cudaStream_t st) {
  dim3 grid(296, 4);
  if (p.src_f32) mlra_repack_kernel<float><<<grid, 256, 0, st>>>(p);
  else mlra_repack_kernel<uint16_t><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

// ----------------------------------------------------------------------------- test hook
__global__ void mlra_resolve_rows_kernel(const int32_t* seq_lens, const int32_t* page_table, int N,
                                         int max_pages, int page_size, int max_seq_len,
                                         int64_t n_pages, int oob_row, int64_t* rows_out,
                                         int row_pitch) {
  const int s = blockIdx.x;
  const int L = min(seq_lens[s], row_pitch);
  for (int j = threadIdx.x; j < L; j += blockDim.x) {
    const int row0 = tile_row(page_table, max_pages, page_size, max_seq_len, n_pages, oob_row, s,
                              j / kTile, nullptr);
    rows_out[(int64_t)s * row_pitch + j] = (int64_t)row0 + (j % kTile);
  }
}

cudaError_t launch_resolve_rows(const int32_t* /*lens_or_null*/, const int32_t* seq_lens,
                                const int32_t* page_table, int N, int max_pages, int page_size,
                                int max_seq_len, int64_t n_pages, int oob_row, int64_t* rows_out,
                                int row_pitch, cudaStream_t st) {
  mlra_resolve_rows_kernel<<<N, 256, 0, st>>>(seq_lens, page_table, N, max_pages, page_size,
                                               max_seq_len, n_pages, oob_row, rows_out, row_pitch);
  return cudaGetLastError();
}

}  // namespace mlra
