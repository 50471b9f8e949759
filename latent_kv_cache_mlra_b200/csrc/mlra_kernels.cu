// mlra_kernels.cu -- device kernels of the MLRA decode library and their launchers.
//   K0 mlra_prep_kernel      (more than kSelfPlanMaxSeqs sequences) clamped lengths, the
//                            split plan as segment descriptors, empty-sequence outputs
//   K1 mlra_decode_kernel    split-KV decode attention (mlra_decode_kernel.cuh); plans its own
//                            work range for up to kSelfPlanMaxSeqs sequences
//   K2 mlra_combine_kernel   merges the partial softmax states of split sequences and writes
//                            the call's status word
//   K3 mlra_repack_kernel    fp32 / odd-width inputs -> padded bf16 copies in the workspace
//   K5 mlra_project_kernel   per-head products: step 1 (query absorption) and step 3 (value
//                            up-projection summed over the branches); mlra_pack_kernel packs
//                            their weights (mlra_project_kernel.cuh)
//   K7 mlra_rope_append_kernel  RoPE of the new token's query and key, cache append
//   mlra_resolve_rows_kernel test hook for the cache-row addressing of K1
#include <cuda_bf16.h>
#include <math_constants.h>

#include "mlra_decode_kernel.cuh"
#include "mlra_decode_m128_kernel.cuh"
#include "mlra_merge.cuh"
#include "mlra_project_kernel.cuh"
#include "sm100_ptx.cuh"
#include "mlra_internal.h"
#include "mlra_plan.cuh"

namespace mlra {

// ----------------------------------------------------------------------------- K0
// One block, for batches of more than kSelfPlanMaxSeqs sequences (smaller ones are planned by
// the decode kernel itself).  seq_lens outside [0, limit] set kFlagBadLength (in the kernel's
// status slot) and are clamped.  Tiles of `tile` positions are counted per
// sequence and scanned into the real and the virtual prefix of the split plan (mlra_plan.cuh).
// Then, per work range, its segment descriptors (range r's first descriptor sits at r + its first
// sequence, which keeps the ranges' descriptor blocks disjoint), per sequence the ranges holding
// it, and for empty sequences out = 0, lse = -inf.  The plan's arrays live in shared memory for
// up to kPrepSmemSeqs sequences, else in the workspace (p.scratch).
constexpr int kPrepSmemSeqs = 2400;  // 5 N + 2 ints <= 48 KB

__global__ void __launch_bounds__(1024) mlra_prep_kernel(const PrepParams p) {
  __shared__ int32_t warp_tot[2][32];
  __shared__ int32_t carry[2];
  __shared__ uint32_t flags;
  extern __shared__ int32_t sh_plan[];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int N = p.N;
  int32_t* base = N <= kPrepSmemSeqs ? sh_plan : p.scratch;
  int32_t* prefix = base;               // [N + 1]
  int32_t* vprefix = base + (N + 1);    // [N + 1]
  int32_t* lens = base + 2 * (N + 1);   // [N]
  int32_t* first_r = lens + N;          // [N] range holding the sequence's first tile
  int32_t* last_r = first_r + N;        // [N] range holding its last tile
  // Launched with programmatic stream serialization: the block may be resident before the
  // previous kernel on the stream (the previous call's combine) has finished.  Nothing is read
  // or written before that kernel's results are complete and visible.
  pdl_wait_prerequisites();
  pdl_launch_dependents();  // the decode kernel may start its prologue now
  if (tid == 0) {
    carry[0] = carry[1] = 0;
    flags = 0;
    prefix[0] = vprefix[0] = 0;
  }
  __syncthreads();
  for (int b0 = 0; b0 < N; b0 += 1024) {
    const int i = b0 + tid;
    int x[2] = {0, 0};  // tiles, virtual tiles
    if (i < N) {
      int L = virtual_len(p.seq_lens, i, p.q_per_seq, p.unit_tokens);
      if (L - (p.unit_tokens - 1) < 0 || L > p.limit) {  // (a unit's first token too short)
        atomicOr(&flags, kFlagBadLength);
        L = L < 0 ? 0 : (L > p.limit ? p.limit : L);
      }
      lens[i] = L;
      x[0] = (L + p.tile - 1) / p.tile;
      x[1] = x[0] > 0 ? x[0] + p.seg_cost : 0;
      first_r[i] = 0;
      last_r[i] = -1;
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {  // inclusive warp scans
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x[k], o);
        if (lane >= o) x[k] += y;
      }
      if (lane == 31) warp_tot[k][wid] = x[k];
    }
    __syncthreads();
    if (wid < 2) {
      int w = warp_tot[wid][lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[wid][lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int incl0 = x[0] + (wid > 0 ? warp_tot[0][wid - 1] : 0) + carry[0];
    const int incl1 = x[1] + (wid > 0 ? warp_tot[1][wid - 1] : 0) + carry[1];
    if (i < N) {
      prefix[i + 1] = incl0;
      vprefix[i + 1] = incl1;
    }
    __syncthreads();
    if (tid == 1023) {
      carry[0] = incl0;
      carry[1] = incl1;
    }
    __syncthreads();
  }
  // the arrays written above are visible to the whole block after the last __syncthreads
  PlanView pv;
  pv.prefix = prefix;
  pv.vprefix = vprefix;
  pv.n = N;
  pv.total = prefix[N];
  pv.vtotal = vprefix[N];
  pv.R = effective_ranges(p.num_ranges, pv.total);
  pv.cost = p.seg_cost;
  for (int r = tid; r < p.num_ranges; r += blockDim.x) {
    RangeInfo ri{0, 0};
    if (r < pv.R && pv.total > 0) {
      SegmentWalker walk(prefix, N, range_start(pv, r), range_start(pv, r + 1));
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
        if (seg.tile0 == 0) first_r[seg.seq] = r;
        if (seg.tile0 + seg.ntiles == prefix[seg.seq + 1] - prefix[seg.seq]) last_r[seg.seq] = r;
      }
    }
    p.ranges[r] = ri;
  }
  __syncthreads();
  for (int sq = tid; sq < N; sq += blockDim.x) {
    SeqInfo si;
    si.r0 = first_r[sq];
    si.r1 = last_r[sq];  // r0 - 1 for an empty sequence
    p.seqs[sq] = si;
  }
  for (int sq = wid; sq < N; sq += 32) {  // empty sequences (a warp each): out = 0, lse = -inf
    if (lens[sq] != 0) continue;
    float* row = p.out + (int64_t)sq * p.H * p.out_width;
    for (int i = lane; i < p.H * p.out_width; i += 32) row[i] = 0.f;
    if (p.lse)
      for (int i = lane; i < p.H * p.B; i += 32) p.lse[(int64_t)sq * p.H * p.B + i] = -CUDART_INF_F;
  }
  if (tid == 0) *p.flags = flags;  // folded into the status word by the combine kernel
}

cudaError_t launch_prep(const PrepParams& p, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(1024);
  cfg.dynamicSmemBytes = p.N <= kPrepSmemSeqs ? (5 * (size_t)p.N + 2) * sizeof(int32_t) : 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // hide the launch gap
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mlra_prep_kernel, p);
}

// ----------------------------------------------------------------------------- K1
template <int DBLK, int T, int NS>
static cudaError_t launch_decode_t(const CUtensorMap& tq, const CUtensorMap& tqr,
                                   const CUtensorMap& tc, const CUtensorMap& tkr,
                                   const CUtensorMap& tout, const CUtensorMap& tpart,
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
  return cudaLaunchKernelEx(&cfg, kern, tq, tqr, tc, tkr, tout, tpart, p);
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
                          const CUtensorMap& tc, const CUtensorMap& tkr, const CUtensorMap& tout,
                          const CUtensorMap& tpart, const DecodeParams& p, int grid,
                          cudaStream_t st) {
  switch (v) {
#define X(id, D, T, NS) \
  case id: return launch_decode_t<D, T, NS>(tq, tqr, tc, tkr, tout, tpart, p, grid, st);
    MLRA_VARIANTS(X)
#undef X
    default: return cudaErrorInvalidValue;
  }
}

// ----------------------------------------------------------------------------- K1M
constexpr int kM128Stages = 4;

cudaError_t launch_decode_m128(const CUtensorMap& tq, const CUtensorMap& tqr,
                               const CUtensorMap& tc, const CUtensorMap& tkr,
                               const DecodeParams& p, int grid, cudaStream_t st) {
  using C = DecodeM128Cfg<kM128Stages>;
  auto kern = mlra_decode_m128_kernel<kM128Stages>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDecodeM128Threads);
  cfg.dynamicSmemBytes = C::SMEM_ALLOC;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tq, tqr, tc, tkr, p);
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
  // The next call's prep kernel may be scheduled now: it waits for this grid before it reads
  // or writes anything.
  pdl_launch_dependents();
  pdl_wait_prerequisites();  // the decode kernel's partials must be complete and visible
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x < 32) {
    // the call's status word: the bits every decode CTA (and the prep kernel) raised
    uint32_t f = 0;
    for (int i = threadIdx.x; i < p.n_flag_slots; i += 32) f |= __ldcg(p.cta_flags + i);
    f = __reduce_or_sync(0xffffffffu, f);
    if (threadIdx.x == 0) *p.status = f;
  }
  const int2 si = __ldcg(reinterpret_cast<const int2*>(p.seqs + s));  // (r0, r1)
  const int np = si.y - si.x + 1;
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

// ----------------------------------------------------------------------------- K5
cudaError_t launch_pack(const void* w, void* packed, int H, int d_in, int d_out, bool transpose,
                        cudaStream_t st) {
  mlra_pack_kernel<<<592, 256, 0, st>>>(static_cast<const uint16_t*>(w),
                                        static_cast<uint16_t*>(packed), H, d_in, d_out,
                                        transpose ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_project(const ProjectParams& p, cudaStream_t st) {
  const int smem = project_smem_bytes(p.d_in / 64);
  auto kern = p.merge ? mlra_project_kernel<kProjMergeThreads, true>
                      : mlra_project_kernel<kProjThreads, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.H * (p.d_out / kProjM), (p.N + kProjN - 1) / kProjN);
  cfg.blockDim = dim3(p.merge ? kProjMergeThreads : kProjThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

// ----------------------------------------------------------------------------- K7
// Block (s, y) handles 256 of sequence s's items: the H * d_rope / 2 query pairs, then the
// d_rope / 2 key pairs, then the d_latent / 2 pairs of c_new (copied, not rotated).  The new token
// sits at position p = seq_lens[s]: its row follows the decode's addressing (page table, or
// s * max_seq_len + p).  Pair (2i, 2i+1) of the head queries and of the key is rotated by the
// angle p * base^(-2i/d_rope) (angle in double precision: p reaches 10^5 and more); the rotated
// query is written in bf16 for the decode, the rotated key and the latent in bf16 to the cache row.
// A position past the cache or an invalid page id flags the status word (block y = 0) and skips
// the append (the query is still rotated).  Each thread's input pair is loaded before the angles
// are computed, so the loads and the double-precision angle overlap.
constexpr int kRopeThreads = 256;

__global__ void __launch_bounds__(kRopeThreads) mlra_rope_append_kernel(const RopeAppendParams p) {
  __shared__ float2 rot[kMaxRopePairs];  // (cos, sin) of the d_rope / 2 angles of this position
  const int s = blockIdx.x;
  const int half = p.d_rope / 2;
  const int nq = p.H * half, nk = nq + half, items = nk + p.d_latent / 2;
  const int t = blockIdx.y * kRopeThreads + threadIdx.x;
  pdl_wait_prerequisites();  // the inputs come from the previous kernels on the stream
  pdl_launch_dependents();   // the decode kernel may start its prologue
  float2 x = make_float2(0.f, 0.f);
  if (t < nq)
    x = *reinterpret_cast<const float2*>(p.q_rope_in + (int64_t)s * p.H * p.d_rope + 2 * t);
  else if (t < nk)
    x = *reinterpret_cast<const float2*>(p.kr_new + (int64_t)s * p.d_rope + 2 * (t - nq));
  else if (t < items)
    x = *reinterpret_cast<const float2*>(p.c_new + (int64_t)s * p.d_latent + 2 * (t - nk));
  const int pos = p.seq_lens[s];
  if (threadIdx.x < half) {
    const double pd = pos > 0 ? (double)pos : 0.0;
    double sn, cs;
    sincos(pd * pow(p.base, -2.0 * threadIdx.x / p.d_rope), &sn, &cs);
    rot[threadIdx.x] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
  }
  int64_t row = -1;
  uint32_t bad = 0;
  if (pos < 0) {
    bad = kFlagBadLength;
  } else if (p.page_table != nullptr) {
    const int page = pos / p.page_size;
    if (page >= p.max_pages) {
      bad = kFlagBadLength;
    } else {
      const int pid = p.page_table[(int64_t)s * p.max_pages + page];
      if (pid < 0 || pid >= p.n_pages) bad = kFlagBadPage;
      else row = (int64_t)pid * p.page_size + pos % p.page_size;
    }
  } else {
    if (pos >= p.max_seq_len) bad = kFlagBadLength;
    else row = (int64_t)s * p.max_seq_len + pos;
  }
  if (bad && blockIdx.y == 0 && threadIdx.x == 0 && p.status) atomicOr(p.status, bad);
  __syncthreads();
  if (t >= items) return;
  float2 y = x;
  if (t < nk) {
    const float2 r = rot[t < nq ? t % half : t - nq];
    y = make_float2(x.x * r.x - x.y * r.y, x.x * r.y + x.y * r.x);
  }
  const uint32_t w = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y.x)) |
                     ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y.y)) << 16);
  uint16_t* dst = nullptr;
  if (t < nq) dst = p.q_rope_out + (int64_t)s * p.H * p.d_rope + 2 * t;
  else if (row < 0) dst = nullptr;
  else if (t < nk) dst = p.k_rope + row * p.kr_row_stride + 2 * (t - nq);
  else dst = p.c_kv + row * p.c_row_stride + 2 * (t - nk);
  if (dst) *reinterpret_cast<uint32_t*>(dst) = w;
}

cudaError_t launch_rope_append(const RopeAppendParams& p, cudaStream_t st) {
  const int items = p.H * (p.d_rope / 2) + p.d_rope / 2 + p.d_latent / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.N, (items + kRopeThreads - 1) / kRopeThreads);
  cfg.blockDim = dim3(kRopeThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mlra_rope_append_kernel, p);
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
