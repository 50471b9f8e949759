// mlra_kernels.cu -- device kernels of the MLRA decode library and their launchers.
//   K0 mlra_prep_kernel      lengths -> clamped lengths, tile prefix sums, status word reset
//   K1 mlra_decode_kernel    split-KV decode attention (mlra_decode_kernel.cuh)
//   K2 mlra_combine_kernel   merges the partial softmax states of split sequences
//   K3 mlra_repack_kernel    fp32 / odd-width inputs -> padded bf16 copies in the workspace
//   mlra_resolve_rows_kernel test hook for the cache-row addressing of K1
#include <cuda_bf16.h>
#include <math_constants.h>

#include "mlra_decode_kernel.cuh"
#include "sm100_ptx.cuh"
#include "mlra_internal.h"
#include "mlra_plan.cuh"

namespace mlra {

// ----------------------------------------------------------------------------- K0
// One block.  seq_lens outside [0, limit] set kFlagBadLength and are clamped; the status word
// is rewritten so that it reports this call only.  prefix counts tiles of `tile` positions.
__global__ void __launch_bounds__(1024) mlra_prep_kernel(const int32_t* seq_lens, int N, int limit,
                                                         int tile, int32_t* lens_out,
                                                         int32_t* prefix, uint32_t* status) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t carry;
  __shared__ uint32_t flags;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
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
      int L = seq_lens[i];
      if (L < 0 || L > limit) {
        atomicOr(&flags, kFlagBadLength);
        L = L < 0 ? 0 : limit;
      }
      lens_out[i] = L;
      tiles = (L + tile - 1) / tile;
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
  if (tid == 0) *status = flags;
}

cudaError_t launch_prep(const int32_t* seq_lens, int N, int limit, int tile, int32_t* lens_out,
                        int32_t* prefix, uint32_t* status, cudaStream_t st) {
  mlra_prep_kernel<<<1, 1024, 0, st>>>(seq_lens, N, limit, tile, lens_out, prefix, status);
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
// Grid (H, N, column chunks of 128), 128 threads.  For sequence s split into parts (ranges
// r0 .. r0+np-1, slot r + s), per branch b: m* = max_p m_p, l* = sum_p 2^(m_p - m*) l_p and
//   out = gamma * sum_p 2^(m_p - m*) o_p / l*,   lse = (m* + log2 l*) ln 2.
// Scores are kept in log2 units by K1.  The per-part weights gamma 2^(m_p - m*) / l* of every
// branch are computed once per block into shared memory.
__global__ void __launch_bounds__(128) mlra_combine_kernel(const CombineParams p) {
  const int h = blockIdx.x, s = blockIdx.y, chunk = blockIdx.z;
  pdl_wait_prerequisites();  // the decode kernel's partials must be complete and visible
  const int64_t total = p.prefix[p.N];
  int r0 = 0, np = 0;
  if (total > 0) seq_parts(p.prefix, s, total, effective_ranges(p.num_ranges, total), &r0, &np);
  if (np == 1 && p.final_written) return;
  const int width = p.summed ? p.d_blk_out : p.B * p.d_blk_out;
  const int c = chunk * 128 + threadIdx.x;
  float* out_row = p.out + ((int64_t)s * p.H + h) * width;
  if (np == 0) {
    if (c < width) out_row[c] = 0.f;
    if (p.lse && chunk == 0 && threadIdx.x < p.B)
      p.lse[((int64_t)s * p.H + h) * p.B + threadIdx.x] = -CUDART_INF_F;
    return;
  }
  extern __shared__ float sh[];  // m[np][B] (then the weights), l[np][B], m*[B], l*[B]
  float* wts = sh;
  float* lpart = sh + np * p.B;
  float* mstar = lpart + np * p.B;
  float* lstar = mstar + p.B;
  const int64_t slot0 = (int64_t)r0 + s;
  const int n_ml = np * p.B;
  // 1. every (part, branch) state in parallel
  for (int k = threadIdx.x; k < n_ml; k += blockDim.x) {
    const int q = k / p.B, b = k - q * p.B;
    const float2 ml = *reinterpret_cast<const float2*>(p.part_ml + (((slot0 + q) * p.H + h) * p.B + b) * 2);
    wts[k] = ml.x;
    lpart[k] = ml.y;
  }
  __syncthreads();
  // 2. per branch: m* = max_p m_p
  for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
    float m = -CUDART_INF_F;
    for (int q = 0; q < np; ++q) m = fmaxf(m, wts[q * p.B + b]);
    mstar[b] = m;
  }
  __syncthreads();
  // 3. w_p = 2^(m_p - m*) (unnormalised), in parallel
  for (int k = threadIdx.x; k < n_ml; k += blockDim.x) wts[k] = exp2f(wts[k] - mstar[k % p.B]);
  __syncthreads();
  // 4. l* = sum_p w_p l_p, then fold gamma / l* into the weights
  for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
    float l = 0.f;
    for (int q = 0; q < np; ++q) l += wts[q * p.B + b] * lpart[q * p.B + b];
    lstar[b] = l;
    if (p.lse && chunk == 0)
      p.lse[((int64_t)s * p.H + h) * p.B + b] = (mstar[b] + log2f(l)) * 0.69314718055994531f;
  }
  __syncthreads();
  for (int k = threadIdx.x; k < n_ml; k += blockDim.x) wts[k] *= p.gamma / lstar[k % p.B];
  __syncthreads();
  if (c >= width) return;
  const float* po = p.part_o + (slot0 * p.H + h) * p.dck;
  const int64_t pstride = (int64_t)p.H * p.dck;  // next part of the same (s, h)
  if (!p.summed) {
    const int b = c / p.d_blk_out;
    const float* src = po + b * p.dblk_k + (c - b * p.d_blk_out);
    float acc = 0.f;
#pragma unroll 4
    for (int q = 0; q < np; ++q) acc += wts[q * p.B + b] * src[q * pstride];
    out_row[c] = acc;
  } else {
    float acc = 0.f;
    for (int b = 0; b < p.B; ++b) {
      const float* src = po + b * p.dblk_k + c;
#pragma unroll 4
      for (int q = 0; q < np; ++q) acc += wts[q * p.B + b] * src[q * pstride];
    }
    out_row[c] = acc;
  }
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t st) {
  const int width = p.summed ? p.d_blk_out : p.B * p.d_blk_out;
  const size_t sh = (2 * (size_t)p.max_parts * p.B + 2 * p.B) * sizeof(float);
  if (sh > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(mlra_combine_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sh);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.H, p.N, (width + 127) / 128);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = sh;
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
