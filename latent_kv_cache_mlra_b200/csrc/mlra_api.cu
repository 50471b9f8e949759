// mlra_api.cu -- the C ABI declared in include/mlra.h: argument checks, the split plan,
// the workspace layout, TMA tensor maps and the launch sequence K3? -> K0 -> K1 -> K2.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <array>
#include <mutex>
#include <vector>

#include "mlra.h"
#include "mlra_internal.h"
#include "mlra_plan.cuh"

namespace {

using namespace mlra;

constexpr size_t kAlign = 256;
constexpr uint64_t kTimeoutNs = 1000ull * 1000ull * 1000ull;  // 1 s bound on every device wait

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Plan {
  bool repack = false;
  Variant variant = kV128;
  int dblk_k = 0;      // padded branch width seen by the kernel
  int tile = 0;        // KV positions per tile
  int n_groups = 1;    // CTAs per range (one per branch and 64-head group)
  int dck = 0;         // B * dblk_k
  int R = 0;           // work ranges
  int64_t slots = 0;   // partial slots = R + N - 1
  int limit = 0;       // bound on seq_lens
  int seg_cost = 0;    // tiles a sequence start costs a CTA (plan balance)
  bool self_plan = false;  // the decode kernel plans its ranges (no prep kernel)
  bool m128 = false;   // K1M: two query tokens x 64 heads per CTA (128 rows)
  int unit_tokens = 1; // query tokens per unit (virtual sequence)
  int64_t units = 0;   // virtual sequences of the plan
  int rows = 0;        // query rows per unit (heads, or 2 x 64 for K1M)
  size_t off_scratch = 0, off_ranges = 0, off_segs = 0, off_seqs = 0, off_flags = 0;
  size_t off_ml = 0, off_o = 0;
  size_t off_rq = 0, off_rqr = 0, off_rc = 0, off_rkr = 0, total = 0;
};

// Tiles of streaming that a sequence start inside a work range costs a CTA (the segment's
// epilogue and the next queries' load), measured at 2 to 3.5 tiles on B200.
constexpr int kSegmentCostTiles = 3;
constexpr int kCombineMaxGroups = 8;  // the combine kernel's warps per block

int device_sm_count(mlra_status* st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { *st = MLRA_ERR_CUDA; return 0; }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    *st = MLRA_ERR_CUDA;
    return 0;
  }
  *st = MLRA_OK;
  return sms;
}

mlra_status check_dims(const mlra_dims* d, bool paged) {
  if (!d) return MLRA_ERR_INVALID_ARG;
  if (d->batch < 1 || d->heads < 1 || d->num_branches < 1 || d->d_latent < 1 || d->d_rope < 1)
    return MLRA_ERR_INVALID_ARG;
  if (d->d_latent % d->num_branches != 0) return MLRA_ERR_INVALID_ARG;
  if (d->max_seq_len < 0 || d->cache_rows < 0 || d->num_ranges < 0) return MLRA_ERR_INVALID_ARG;
  if (d->c_row_stride < d->d_latent || d->kr_row_stride < d->d_rope) return MLRA_ERR_INVALID_ARG;
  if (d->dtype != MLRA_BF16 && d->dtype != MLRA_F32) return MLRA_ERR_INVALID_ARG;
  if (d->out_mode != MLRA_OUT_BRANCHES && d->out_mode != MLRA_OUT_SUMMED) return MLRA_ERR_INVALID_ARG;
  if (paged) {
    if (d->page_size < 1 || d->max_pages_per_seq < 1) return MLRA_ERR_INVALID_ARG;
    if ((int64_t)d->page_size * d->max_pages_per_seq > INT_MAX) return MLRA_ERR_INVALID_ARG;
  } else {
    if ((int64_t)d->batch * d->max_seq_len > d->cache_rows) return MLRA_ERR_INVALID_ARG;
  }
  if (d->heads > kMaxHeads || d->d_latent > 512 || d->d_rope > 64) return MLRA_ERR_UNSUPPORTED;
  if (paged && d->page_size % kTile != 0) return MLRA_ERR_UNSUPPORTED;
  if (d->cache_rows > (int64_t)INT_MAX - 2 * kTile) return MLRA_ERR_UNSUPPORTED;
  if (d->num_branches > 64) return MLRA_ERR_UNSUPPORTED;
  return MLRA_OK;
}

// Kernel variant and workspace layout.  sms == 0 requires dims->num_ranges > 0.  With q_len > 1
// query tokens per sequence the plan covers d->batch * q_len virtual sequences (virtual_len).
mlra_status make_plan(const mlra_dims* d, bool paged, int sms, Plan* pl, int q_len = 1) {
  mlra_status st = check_dims(d, paged);
  if (st != MLRA_OK) return st;
  if (q_len < 1 || (int64_t)d->batch * q_len > INT_MAX / 2) return MLRA_ERR_INVALID_ARG;
  const int64_t Nv = (int64_t)d->batch * q_len;
  const int B = d->num_branches, dblk = d->d_latent / B;
  const int dk = dblk <= 64 ? 64 : dblk <= 128 ? 128 : dblk <= 256 ? 256 : 512;
  if (B * dk > 512) return MLRA_ERR_UNSUPPORTED;
  const bool inplace_shape = (dk == dblk) && d->d_rope == 64;
  const bool inplace_align = d->c_row_stride % 8 == 0 && d->kr_row_stride % 8 == 0;
  if (d->dtype == MLRA_BF16 && inplace_shape && !inplace_align) return MLRA_ERR_UNSUPPORTED;
  pl->repack = !(d->dtype == MLRA_BF16 && inplace_shape);
  pl->dblk_k = dk;
  pl->variant = dk == 64 ? kV64 : dk == 128 ? kV128 : dk == 256 ? kV256 : kV512;
  pl->tile = variant_tile(pl->variant);
  // 128 query rows against each cache tile (K1M), for 128-wide branches read in place: an even
  // number of query tokens of 64 heads (two tokens per CTA), or one token of 128 heads (both head
  // groups in one CTA instead of two CTAs reading the same tiles)
  const bool m128_tokens = q_len >= 2 && q_len % 2 == 0 && d->heads == 64 && dk == 128 && !pl->repack;
  const bool m128_heads = q_len == 1 && d->heads == 128 && dk == 128 && !pl->repack;
  pl->m128 = m128_tokens || m128_heads;
  pl->unit_tokens = m128_tokens ? 2 : 1;
  pl->units = Nv / pl->unit_tokens;
  pl->rows = pl->m128 ? 128 : d->heads;
  pl->n_groups = pl->m128 ? B : B * ((d->heads + 63) / 64);  // CTAs per range
  if (pl->n_groups > 148) return MLRA_ERR_UNSUPPORTED;
  pl->dck = B * dk;
  if (d->num_ranges > 0) pl->R = d->num_ranges;
  else {
    if (sms <= 0) return MLRA_ERR_CUDA;
    pl->R = sms / pl->n_groups > 0 ? sms / pl->n_groups : 1;
  }
  if ((int64_t)pl->R * pl->n_groups > INT_MAX / 2) return MLRA_ERR_INVALID_ARG;
  pl->slots = (int64_t)pl->R + pl->units - 1;
  pl->limit = paged ? d->max_pages_per_seq * d->page_size : d->max_seq_len;
  if (!paged) pl->limit = d->max_seq_len;
  else if (d->max_seq_len > 0 && d->max_seq_len < pl->limit) pl->limit = d->max_seq_len;
  pl->seg_cost = kSegmentCostTiles;
  // the plan's (virtual) tile prefix must fit int32
  if (Nv * ((pl->limit + pl->tile - 1) / pl->tile + pl->seg_cost) > INT_MAX)
    return MLRA_ERR_INVALID_ARG;

  const int64_t N = pl->units, H = pl->rows;
  size_t off = kAlign;  // status word + padding
  pl->self_plan = N <= kSelfPlanMaxSeqs;
  pl->off_scratch = off; off = align_up(off + 4 * (5 * (size_t)N + 2));
  pl->off_flags = off; off = align_up(off + 4 * ((size_t)pl->R * pl->n_groups + 1));
  pl->off_ranges = off; off = align_up(off + sizeof(RangeInfo) * (size_t)pl->R);
  pl->off_segs = off; off = align_up(off + sizeof(SegDesc) * (size_t)pl->slots);
  pl->off_seqs = off; off = align_up(off + sizeof(SeqInfo) * (size_t)N);
  pl->off_ml = off; off = align_up(off + (size_t)pl->slots * H * B * 2 * sizeof(float));
  pl->off_o = off; off = align_up(off + (size_t)pl->slots * H * pl->dck * sizeof(float));
  if (pl->repack) {
    pl->off_rq = off; off = align_up(off + (size_t)N * H * pl->dck * 2);
    pl->off_rqr = off; off = align_up(off + (size_t)N * H * 64 * 2);
    pl->off_rc = off; off = align_up(off + (size_t)d->cache_rows * pl->dck * 2);
    pl->off_rkr = off; off = align_up(off + (size_t)d->cache_rows * 64 * 2);
  }
  pl->total = off;
  return MLRA_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link needed).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tensor map with boxes of 64 columns x box_rows rows and 128-byte swizzle.  dims/strides in
// elements.
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
              const uint64_t* strides_elems, uint32_t box_rows = 64) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[3], gstride[2];
  cuuint32_t box[3] = {64, box_rows, 1}, estr[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) gdim[i] = dims[i];
  for (int i = 0; i + 1 < rank; ++i) gstride[i] = strides_elems[i] * 2;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), gdim, gstride, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 store map over [dims[2]][dims[1]][dims[0]] (row pitches in elements), boxes of 32 x 16 x 1,
// 128-byte swizzle: the attention kernel's epilogue stores through it.
bool make_store_map(CUtensorMap* m, void* base, const uint64_t* dims, const uint64_t* pitches) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[3] = {dims[0], dims[1], dims[2]};
  cuuint64_t gstride[2] = {pitches[0] * 4, pitches[1] * 4};
  cuuint32_t box[3] = {32, 16, 1}, estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Scratch of mlra_decode_static_scratch.  In host code the name stands for the array only as a
// symbol: its device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_static_scratch[MLRA_STATIC_SCRATCH_BYTES];
constexpr int kMaxDevices = 256;
std::mutex g_static_scratch_mu;
void* g_static_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" {

int mlra_version(void) { return 0x000100; }

const char* mlra_status_string(mlra_status s) {
  switch (s) {
    case MLRA_OK: return "MLRA_OK";
    case MLRA_ERR_INVALID_ARG: return "MLRA_ERR_INVALID_ARG: invalid argument";
    case MLRA_ERR_UNSUPPORTED: return "MLRA_ERR_UNSUPPORTED: shape or layout not supported";
    case MLRA_ERR_CUDA: return "MLRA_ERR_CUDA: a CUDA call failed";
    case MLRA_ERR_TIMEOUT: return "MLRA_ERR_TIMEOUT: a device-side wait ran out";
    case MLRA_ERR_WORKSPACE: return "MLRA_ERR_WORKSPACE: workspace null, too small or misaligned";
    case MLRA_ERR_BAD_PAGE: return "MLRA_ERR_BAD_PAGE: page id outside the cache pool";
    case MLRA_ERR_BAD_LENGTH: return "MLRA_ERR_BAD_LENGTH: sequence length outside the cache";
    case MLRA_ERR_SCRATCH_LIMIT:
      return "MLRA_ERR_SCRATCH_LIMIT: the problem needs more scratch than the library's built-in "
             "buffer (MLRA_STATIC_SCRATCH_BYTES); use mlra_decode with a workspace";
  }
  return "MLRA: unknown status";
}

mlra_status mlra_workspace_size(const mlra_dims* dims, size_t* bytes_host) {
  if (!dims || !bytes_host) return MLRA_ERR_INVALID_ARG;
  const bool paged = dims->max_pages_per_seq > 0 && dims->page_size > 0;
  int sms = 0;
  if (dims->num_ranges == 0) {
    mlra_status st;
    sms = device_sm_count(&st);
    if (st != MLRA_OK) return st;
  }
  Plan pl;
  mlra_status st = make_plan(dims, paged, sms, &pl);
  if (st != MLRA_OK) return st;
  *bytes_host = pl.total;
  return MLRA_OK;
}

mlra_status mlra_query_plan(const mlra_dims* dims, mlra_plan_info* info) {
  if (!dims || !info) return MLRA_ERR_INVALID_ARG;
  const bool paged = dims->max_pages_per_seq > 0 && dims->page_size > 0;
  int sms = 0;
  if (dims->num_ranges == 0) {
    mlra_status st;
    sms = device_sm_count(&st);
    if (st != MLRA_OK) return st;
  }
  Plan pl;
  mlra_status st = make_plan(dims, paged, sms, &pl);
  if (st != MLRA_OK) return st;
  info->repack = pl.repack ? 1 : 0;
  info->launches = (pl.self_plan ? 2 : 3) + (pl.repack ? 1 : 0);
  info->num_ranges = pl.R;
  info->ctas = pl.R * pl.n_groups;
  info->kernel_branch_width = pl.dblk_k;
  info->branches_per_cta = 1;
  info->tile = pl.tile;
  info->partial_slots = pl.slots;
  info->segment_cost_tiles = pl.seg_cost;
  info->workspace_bytes = pl.total;
  return MLRA_OK;
}

mlra_status mlra_decode(const void* q_lat, const void* q_rope, const void* c_kv, const void* k_rope,
                        const int32_t* seq_lens, const int32_t* page_table, int B,
                        const mlra_scales* scales, float* out, float* lse, const mlra_dims* dims,
                        void* workspace, size_t ws_bytes, mlra_stream_t stream) {
  return mlra_decode_profiled(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table, B, scales, out,
                              lse, dims, workspace, ws_bytes, stream, nullptr, nullptr);
}

namespace {
mlra_status check_product(const void* a, const void* b, const void* c, int N, int H, int d_in,
                          int d_out);
// The decode call: q_len query tokens per caller sequence (1: single-token decode), run as
// dims->batch * q_len virtual sequences (virtual_len).
mlra_status decode_impl(const void* q_lat, const void* q_rope, const void* c_kv,
                        const void* k_rope, const int32_t* seq_lens, const int32_t* page_table,
                        int B, const mlra_scales* scales, float* out, float* lse,
                        const mlra_dims* dims, void* workspace, size_t ws_bytes,
                        mlra_stream_t stream, mlra_event_t k1_begin, mlra_event_t k1_end,
                        int q_len, const void* w_packed = nullptr, int d_head = 0,
                        float* y = nullptr) {
  // y != nullptr: step 3 follows in the same call (mlra_decode_project); `out` is then unused
  // and the attention kernel's final rows go to a region of the workspace
  const bool fused = y != nullptr;
  if (!q_lat || !q_rope || !c_kv || !k_rope || !seq_lens || !scales || !(out || fused) || !dims)
    return MLRA_ERR_INVALID_ARG;
  if (B != dims->num_branches) return MLRA_ERR_INVALID_ARG;
  if (!std::isfinite(scales->softmax_scale) || !std::isfinite(scales->branch_scale))
    return MLRA_ERR_INVALID_ARG;
  const bool paged = page_table != nullptr;
  mlra_status st = check_dims(dims, paged);
  if (st != MLRA_OK) return st;
  int sms = 0;
  if (dims->num_ranges == 0) {
    sms = device_sm_count(&st);
    if (st != MLRA_OK) return st;
  }
  Plan pl;
  st = make_plan(dims, paged, sms, &pl, q_len);
  if (st != MLRA_OK) return st;
  size_t need = pl.total;
  if (fused) {
    if (dims->out_mode != MLRA_OUT_BRANCHES || pl.repack || q_len != 1 || !w_packed)
      return MLRA_ERR_UNSUPPORTED;
    const mlra_status pst = check_product(w_packed, w_packed, y, dims->batch, dims->heads,
                                          dims->d_latent, d_head);
    if (pst != MLRA_OK) return pst;
    need = pl.total + align_up((size_t)dims->batch * dims->heads * dims->d_latent * sizeof(float));
    out = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + pl.total);
    lse = nullptr;
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 || ws_bytes < need)
    return MLRA_ERR_WORKSPACE;
  if (!pl.repack && !(aligned16(q_lat) && aligned16(q_rope) && aligned16(c_kv) && aligned16(k_rope)))
    return MLRA_ERR_UNSUPPORTED;
  if (!aligned16(out)) return MLRA_ERR_UNSUPPORTED;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  int32_t* plan_scratch = reinterpret_cast<int32_t*>(ws + pl.off_scratch);
  float* part_ml = reinterpret_cast<float*>(ws + pl.off_ml);
  float* part_o = reinterpret_cast<float*>(ws + pl.off_o);
  RangeInfo* ranges = reinterpret_cast<RangeInfo*>(ws + pl.off_ranges);
  SegDesc* segs = reinterpret_cast<SegDesc*>(ws + pl.off_segs);
  SeqInfo* seqs = reinterpret_cast<SeqInfo*>(ws + pl.off_seqs);
  // virtual sequences (units) and query rows per unit
  const int N = static_cast<int>(pl.units), H = pl.rows, dblk = dims->d_latent / B;
  const int64_t rows = dims->cache_rows;

  const void* kq = q_lat; const void* kqr = q_rope; const void* kc = c_kv; const void* kkr = k_rope;
  int64_t c_pitch = dims->c_row_stride, kr_pitch = dims->kr_row_stride, q_width = dims->d_latent;
  if (pl.repack) {
    RepackParams rp;
    rp.q_lat = q_lat; rp.q_rope = q_rope; rp.c_kv = c_kv; rp.k_rope = k_rope;
    rp.q_out = reinterpret_cast<uint16_t*>(ws + pl.off_rq);
    rp.qr_out = reinterpret_cast<uint16_t*>(ws + pl.off_rqr);
    rp.c_out = reinterpret_cast<uint16_t*>(ws + pl.off_rc);
    rp.kr_out = reinterpret_cast<uint16_t*>(ws + pl.off_rkr);
    rp.N = N; rp.H = H; rp.B = B; rp.d_blk = dblk; rp.dblk_k = pl.dblk_k; rp.d_rope = dims->d_rope;
    rp.rows = rows; rp.c_row_stride = dims->c_row_stride; rp.kr_row_stride = dims->kr_row_stride;
    rp.src_f32 = dims->dtype == MLRA_F32;
    if (launch_repack(rp, s) != cudaSuccess) return MLRA_ERR_CUDA;
    kq = rp.q_out; kqr = rp.qr_out; kc = rp.c_out; kkr = rp.kr_out;
    c_pitch = pl.dck; kr_pitch = 64; q_width = pl.dck;
  }

  CUtensorMap tq, tqr, tc, tkr;
  {
    const uint64_t dq[3] = {(uint64_t)q_width, (uint64_t)H, (uint64_t)N};
    const uint64_t sq[2] = {(uint64_t)q_width, (uint64_t)q_width * H};
    const uint64_t dqr[3] = {64, (uint64_t)H, (uint64_t)N};
    const uint64_t sqr[2] = {64, (uint64_t)64 * H};
    const uint64_t dcm[2] = {(uint64_t)q_width, (uint64_t)rows};
    const uint64_t scm[1] = {(uint64_t)c_pitch};
    const uint64_t dkr[2] = {64, (uint64_t)rows};
    const uint64_t skr[1] = {(uint64_t)kr_pitch};
    const uint32_t qbox = pl.m128 ? 128 : 64;  // one unit's query rows per box
    if (!make_map(&tq, kq, 3, dq, sq, qbox) || !make_map(&tqr, kqr, 3, dqr, sqr, qbox) ||
        !make_map(&tc, kc, 2, dcm, scm) || !make_map(&tkr, kkr, 2, dkr, skr))
      return MLRA_ERR_CUDA;
  }

  const bool summed = dims->out_mode == MLRA_OUT_SUMMED;
  const int out_width = summed ? dblk : dims->d_latent;  // floats per (sequence, head) row of out
  const int grid = pl.R * pl.n_groups;
  // store maps of the attention kernel's epilogue: partial outputs always, final outputs when
  // every branch block is whole 32-column boxes (else it stores them directly)
  CUtensorMap tpart, tout;
  const bool tma_out = !summed && dblk % 32 == 0 && out_width % 4 == 0;
  {
    const uint64_t dpart[3] = {(uint64_t)pl.dck, (uint64_t)H, (uint64_t)pl.slots};
    const uint64_t ppart[2] = {(uint64_t)pl.dck, (uint64_t)pl.dck * H};
    if (!make_store_map(&tpart, part_o, dpart, ppart)) return MLRA_ERR_CUDA;
    if (tma_out) {
      const uint64_t dout[3] = {(uint64_t)out_width, (uint64_t)H, (uint64_t)N};
      const uint64_t pout[2] = {(uint64_t)out_width, (uint64_t)out_width * H};
      if (!make_store_map(&tout, out, dout, pout)) return MLRA_ERR_CUDA;
    } else {
      tout = tpart;  // unused
    }
  }
  uint32_t* cta_flags = reinterpret_cast<uint32_t*>(ws + pl.off_flags);  // [grid] + prep's slot
  if (!pl.self_plan) {
    PrepParams pp;
    pp.seq_lens = seq_lens; pp.N = N; pp.limit = pl.limit; pp.tile = pl.tile; pp.num_ranges = pl.R;
    pp.seg_cost = pl.seg_cost; pp.scratch = plan_scratch;
    pp.q_per_seq = q_len / pl.unit_tokens; pp.unit_tokens = pl.unit_tokens;
    pp.ranges = ranges; pp.segs = segs; pp.seqs = seqs;
    pp.flags = cta_flags + grid;
    pp.out = out; pp.lse = lse; pp.H = H; pp.B = B; pp.out_width = out_width;
    if (launch_prep(pp, s) != cudaSuccess) return MLRA_ERR_CUDA;
  }

  DecodeParams p;
  p.ranges = ranges; p.segs = segs;
  p.self_plan = pl.self_plan ? 1 : 0;
  p.seq_lens = seq_lens; p.limit = pl.limit; p.tile = pl.tile; p.seg_cost = pl.seg_cost;
  p.seqs = seqs; p.cta_flags = cta_flags;
  p.page_table = page_table;
  p.out = out; p.lse = lse; p.part_o = part_o; p.part_ml = part_ml;
  p.N = N; p.H = H; p.B = B; p.d_blk_out = dblk; p.out_width = out_width; p.dck = pl.dck;
  p.n_groups = pl.n_groups; p.num_ranges = pl.R;
  p.page_size = paged ? dims->page_size : 0;
  p.max_pages = paged ? dims->max_pages_per_seq : 0;
  p.max_seq_len = dims->max_seq_len;
  p.n_pages = paged ? rows / dims->page_size : 0;
  p.oob_row = static_cast<int>(rows);
  p.q_per_seq = q_len / pl.unit_tokens;
  p.unit_tokens = pl.unit_tokens;
  p.scale_log2 = scales->softmax_scale * 1.4426950408889634f;
  p.gamma = scales->branch_scale;
  p.write_final = summed ? 0 : 1;
  p.tma_out = tma_out ? 1 : 0;
  p.timeout_ns = kTimeoutNs;
  // Test hook: with MLRA_TEST_FORCE_REPLAN set in the environment, the attention kernel treats
  // its speculative plan as stale and takes the re-plan path (results are unchanged).
  p.force_replan = std::getenv("MLRA_TEST_FORCE_REPLAN") != nullptr ? 1 : 0;
  // Test hook: with MLRA_TEST_FORCE_TIMEOUT set, the producer of every CTA that has a copy left
  // to issue after its speculative ones waits (1 ms) on a barrier nothing arrives at; the call
  // then reports MLRA_ERR_TIMEOUT and its outputs are undefined.
  p.force_timeout = std::getenv("MLRA_TEST_FORCE_TIMEOUT") != nullptr ? 1 : 0;
  if (k1_begin && cudaEventRecord(reinterpret_cast<cudaEvent_t>(k1_begin), s) != cudaSuccess)
    return MLRA_ERR_CUDA;
  const cudaError_t launched = pl.m128 ? launch_decode_m128(tq, tqr, tc, tkr, p, grid, s)
                                       : launch_decode(pl.variant, tq, tqr, tc, tkr, tout, tpart, p, grid, s);
  if (launched != cudaSuccess) return MLRA_ERR_CUDA;
  if (k1_end && cudaEventRecord(reinterpret_cast<cudaEvent_t>(k1_end), s) != cudaSuccess)
    return MLRA_ERR_CUDA;

  if (fused) {
    // step 3 merges the split sequences itself: no combine kernel
    ProjectParams pp3;
    pp3.w_packed = w_packed;
    pp3.x = out; pp3.y = y; pp3.status = status;
    pp3.N = N; pp3.H = H; pp3.d_in = dims->d_latent; pp3.d_out = d_head;
    pp3.out_bf16 = 0;
    pp3.timeout_ns = kTimeoutNs;
    pp3.merge = 1;
    pp3.seqs = seqs; pp3.part_ml = part_ml; pp3.part_o = part_o;
    pp3.B = B; pp3.dblk = dblk; pp3.gamma = scales->branch_scale;
    pp3.cta_flags = cta_flags; pp3.n_flag_slots = grid + (pl.self_plan ? 0 : 1);
    if (launch_project(pp3, s) != cudaSuccess) return MLRA_ERR_CUDA;
    return MLRA_OK;
  }
  CombineParams cp;
  cp.cta_flags = cta_flags; cp.n_flag_slots = grid + (pl.self_plan ? 0 : 1); cp.status = status;
  cp.seqs = seqs; cp.part_o = part_o; cp.part_ml = part_ml; cp.out = out; cp.lse = lse;
  cp.N = N; cp.H = H; cp.B = B; cp.dblk_k = pl.dblk_k; cp.dck = pl.dck; cp.d_blk_out = dblk;
  cp.summed = summed ? 1 : 0;
  // Part groups per head: the fewest that still give the combine about one block per attention
  // CTA (fewer, fuller warps fold several batches of parts each; too few blocks leave SMs idle:
  // one sequence split over every range needs G = 8, eight sequences G = 1 -- measured, MLA with
  // 8 sequences 85.6 -> 80.7 us per step against a parts-per-warp rule)
  {
    const int chunks = ((summed ? pl.dblk_k : pl.dck) + 127) / 128;
    int G = 1;
    while (G < kCombineMaxGroups &&
           (int64_t)N * ((H + kCombineMaxGroups / G - 1) / (kCombineMaxGroups / G)) * chunks < grid)
      G *= 2;
    cp.groups = G;
  }
  cp.final_written = summed ? 0 : 1;
  cp.gamma = scales->branch_scale;
  if (launch_combine(cp, s) != cudaSuccess) return MLRA_ERR_CUDA;
  return MLRA_OK;
}
}  // namespace

mlra_status mlra_decode_profiled(const void* q_lat, const void* q_rope, const void* c_kv,
                                 const void* k_rope, const int32_t* seq_lens,
                                 const int32_t* page_table, int B, const mlra_scales* scales,
                                 float* out, float* lse, const mlra_dims* dims, void* workspace,
                                 size_t ws_bytes, mlra_stream_t stream, mlra_event_t k1_begin,
                                 mlra_event_t k1_end) {
  return decode_impl(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table, B, scales, out, lse, dims,
                     workspace, ws_bytes, stream, k1_begin, k1_end, 1);
}

mlra_status mlra_decode_multi(const void* q_lat, const void* q_rope, const void* c_kv,
                              const void* k_rope, const int32_t* seq_lens,
                              const int32_t* page_table, int q_len, int B,
                              const mlra_scales* scales, float* out, float* lse,
                              const mlra_dims* dims, void* workspace, size_t ws_bytes,
                              mlra_stream_t stream) {
  if (q_len < 1) return MLRA_ERR_INVALID_ARG;
  return decode_impl(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table, B, scales, out, lse, dims,
                     workspace, ws_bytes, stream, nullptr, nullptr, q_len);
}

mlra_status mlra_workspace_size_multi(const mlra_dims* dims, int q_len, size_t* bytes_host) {
  if (!dims || !bytes_host || q_len < 1) return MLRA_ERR_INVALID_ARG;
  const bool paged = dims->max_pages_per_seq > 0 && dims->page_size > 0;
  int sms = 0;
  if (dims->num_ranges == 0) {
    mlra_status st;
    sms = device_sm_count(&st);
    if (st != MLRA_OK) return st;
  }
  Plan pl;
  mlra_status st = make_plan(dims, paged, sms, &pl, q_len);
  if (st != MLRA_OK) return st;
  *bytes_host = pl.total;
  return MLRA_OK;
}

mlra_status mlra_workspace_size_project(const mlra_dims* dims, size_t* bytes_host) {
  if (!dims || !bytes_host) return MLRA_ERR_INVALID_ARG;
  size_t base = 0;
  const mlra_status st = mlra_workspace_size(dims, &base);
  if (st != MLRA_OK) return st;
  *bytes_host = base + align_up((size_t)dims->batch * dims->heads * dims->d_latent * sizeof(float));
  return MLRA_OK;
}

mlra_status mlra_decode_project(const void* q_lat, const void* q_rope, const void* c_kv,
                                const void* k_rope, const int32_t* seq_lens,
                                const int32_t* page_table, int B, const mlra_scales* scales,
                                const void* w_packed, int d_head, float* y, const mlra_dims* dims,
                                void* workspace, size_t ws_bytes, mlra_stream_t stream) {
  if (!y) return MLRA_ERR_INVALID_ARG;
  return decode_impl(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table, B, scales, nullptr,
                     nullptr, dims, workspace, ws_bytes, stream, nullptr, nullptr, 1, w_packed,
                     d_head, y);
}

mlra_status mlra_decode_static_scratch(const void* q_lat, const void* q_rope, const void* c_kv,
                                       const void* k_rope, const int32_t* seq_lens,
                                       const int32_t* page_table, int B, const mlra_scales* scales,
                                       float* out, float* lse, const mlra_dims* dims,
                                       mlra_stream_t stream) {
  if (!dims) return MLRA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLRA_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_scratch_mu);
    if (!g_static_scratch_addr[dev]) {
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_static_scratch) != cudaSuccess || !addr) return MLRA_ERR_CUDA;
      g_static_scratch_addr[dev] = addr;
    }
    scratch = g_static_scratch_addr[dev];
  }
  const bool paged = page_table != nullptr;
  int sms = 0;
  mlra_status st = MLRA_OK;
  if (dims->num_ranges == 0) {
    sms = device_sm_count(&st);
    if (st != MLRA_OK) return st;
  }
  Plan pl;
  st = make_plan(dims, paged, sms, &pl);
  if (st != MLRA_OK) return st;
  if (pl.total > MLRA_STATIC_SCRATCH_BYTES) return MLRA_ERR_SCRATCH_LIMIT;
  return mlra_decode(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table, B, scales, out, lse, dims,
                     scratch, MLRA_STATIC_SCRATCH_BYTES, stream);
}

mlra_status mlra_read_status(const void* workspace, mlra_stream_t stream, uint32_t* flags_host) {
  if (!workspace || !flags_host) return MLRA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t f = 0;
  if (cudaMemcpyAsync(&f, workspace, sizeof(f), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MLRA_ERR_CUDA;
  *flags_host = f;
  if (f & kFlagTimeout) return MLRA_ERR_TIMEOUT;
  if (f & kFlagBadPage) return MLRA_ERR_BAD_PAGE;
  if (f & kFlagBadLength) return MLRA_ERR_BAD_LENGTH;
  return MLRA_OK;
}

namespace {
// Shared checks of the per-head products: widths in 64-column boxes, at most 512 input columns,
// 16-byte aligned arrays.
mlra_status check_product(const void* a, const void* b, const void* c, int N, int H, int d_in,
                          int d_out) {
  if (!a || !b || !c || N < 1 || H < 1 || d_in < 1 || d_out < 1) return MLRA_ERR_INVALID_ARG;
  if (d_in % 64 != 0 || d_in > 512 || d_out % 64 != 0) return MLRA_ERR_UNSUPPORTED;
  if ((int64_t)H * d_out > INT_MAX || (int64_t)N > 65535 * 64) return MLRA_ERR_UNSUPPORTED;
  if (!aligned16(a) || !aligned16(b) || !aligned16(c)) return MLRA_ERR_UNSUPPORTED;
  return MLRA_OK;
}

mlra_status run_product(const float* x, const void* w_packed, void* y, int N, int H, int d_in,
                        int d_out, bool out_bf16, uint32_t* status, mlra_stream_t stream) {
  const mlra_status st = check_product(x, w_packed, y, N, H, d_in, d_out);
  if (st != MLRA_OK) return st;
  ProjectParams p;
  p.w_packed = w_packed;
  p.x = x; p.y = y; p.status = status;
  p.N = N; p.H = H; p.d_in = d_in; p.d_out = d_out;
  p.out_bf16 = out_bf16 ? 1 : 0;
  p.timeout_ns = kTimeoutNs;
  p.merge = 0;
  p.seqs = nullptr; p.part_ml = nullptr; p.part_o = nullptr;
  p.B = 1; p.dblk = d_in; p.gamma = 1.f;
  p.cta_flags = nullptr; p.n_flag_slots = 0;
  if (launch_project(p, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MLRA_ERR_CUDA;
  return MLRA_OK;
}

mlra_status run_pack(const void* w, void* packed, int H, int d_in, int d_out, bool transpose,
                     mlra_stream_t stream) {
  const mlra_status st = check_product(w, packed, packed, 1, H, d_in, d_out);
  if (st != MLRA_OK) return st;
  if (launch_pack(w, packed, H, d_in, d_out, transpose, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return MLRA_ERR_CUDA;
  return MLRA_OK;
}
}  // namespace

mlra_status mlra_pack_wuv(const void* w_uv, void* w_packed, int H, int d_latent, int d_head,
                          mlra_stream_t stream) {
  return run_pack(w_uv, w_packed, H, d_latent, d_head, false, stream);
}

mlra_status mlra_project(const float* o, const void* w_packed, float* y, int N, int H, int d_latent,
                         int d_head, uint32_t* status, mlra_stream_t stream) {
  return run_product(o, w_packed, y, N, H, d_latent, d_head, false, status, stream);
}

mlra_status mlra_pack_wuk(const void* w_uk, void* w_packed, int H, int d_head, int d_latent,
                          mlra_stream_t stream) {
  return run_pack(w_uk, w_packed, H, d_head, d_latent, true, stream);
}

mlra_status mlra_absorb(const float* q_nope, const void* w_packed, void* q_lat, int N, int H,
                        int d_head, int d_latent, uint32_t* status, mlra_stream_t stream) {
  return run_product(q_nope, w_packed, q_lat, N, H, d_head, d_latent, true, status, stream);
}

mlra_status mlra_rope_append(const float* q_rope_in, const float* kr_new, const float* c_new,
                             const int32_t* seq_lens, const int32_t* page_table,
                             const mlra_dims* dims, void* c_kv, void* k_rope, void* q_rope_out,
                             double rope_base, uint32_t* status, mlra_stream_t stream) {
  if (!q_rope_in || !kr_new || !c_new || !seq_lens || !dims || !c_kv || !k_rope || !q_rope_out)
    return MLRA_ERR_INVALID_ARG;
  if (!(rope_base > 0.0) || !std::isfinite(rope_base)) return MLRA_ERR_INVALID_ARG;
  const bool paged = page_table != nullptr;
  const mlra_status st = check_dims(dims, paged);
  if (st != MLRA_OK) return st;
  if (dims->dtype != MLRA_BF16 || dims->d_rope % 2 != 0) return MLRA_ERR_UNSUPPORTED;
  // pairs are moved as 8-byte (fp32) and 4-byte (bf16) words
  if (!(aligned16(q_rope_in) && aligned16(kr_new) && aligned16(c_new) && aligned16(q_rope_out) &&
        aligned16(k_rope) && aligned16(c_kv)) ||
      dims->kr_row_stride % 2 != 0 || dims->d_latent % 2 != 0 || dims->c_row_stride % 2 != 0)
    return MLRA_ERR_UNSUPPORTED;
  RopeAppendParams p;
  p.q_rope_in = q_rope_in; p.kr_new = kr_new; p.c_new = c_new;
  p.seq_lens = seq_lens; p.page_table = page_table;
  p.max_pages = paged ? dims->max_pages_per_seq : 0;
  p.page_size = paged ? dims->page_size : 0;
  p.max_seq_len = dims->max_seq_len;
  p.n_pages = paged ? dims->cache_rows / dims->page_size : 0;
  p.c_kv = static_cast<uint16_t*>(c_kv);
  p.k_rope = static_cast<uint16_t*>(k_rope);
  p.c_row_stride = dims->c_row_stride;
  p.kr_row_stride = dims->kr_row_stride;
  p.q_rope_out = static_cast<uint16_t*>(q_rope_out);
  p.N = dims->batch; p.H = dims->heads; p.d_rope = dims->d_rope; p.d_latent = dims->d_latent;
  p.base = rope_base;
  p.status = status;
  if (launch_rope_append(p, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MLRA_ERR_CUDA;
  return MLRA_OK;
}

mlra_status mlra_debug_resolve_rows(const int32_t* seq_lens, const int32_t* page_table,
                                    const mlra_dims* dims, int64_t* rows_out, int row_pitch,
                                    mlra_stream_t stream) {
  if (!seq_lens || !rows_out || row_pitch < 0) return MLRA_ERR_INVALID_ARG;
  const bool paged = page_table != nullptr;
  mlra_status st = check_dims(dims, paged);
  if (st != MLRA_OK) return st;
  const int64_t rows = dims->cache_rows;
  if (launch_resolve_rows(nullptr, seq_lens, page_table, dims->batch,
                          paged ? dims->max_pages_per_seq : 0, paged ? dims->page_size : 0,
                          dims->max_seq_len, paged ? rows / dims->page_size : 0,
                          static_cast<int>(rows), rows_out, row_pitch,
                          reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MLRA_ERR_CUDA;
  return MLRA_OK;
}

namespace {
// The plan of the prep kernel, on the host: per sequence the first and last range holding it,
// and the segments in range order (optional).
mlra_status host_plan(const int32_t* tiles, int n, int num_ranges, int seg_cost,
                      std::vector<int32_t>* first_r, std::vector<int32_t>* last_r,
                      std::vector<std::array<int32_t, 4>>* segs) {
  if (!tiles || n < 1 || num_ranges < 1 || seg_cost < 0) return MLRA_ERR_INVALID_ARG;
  std::vector<int32_t> prefix(n + 1, 0), vprefix(n + 1, 0);
  for (int i = 0; i < n; ++i) {
    if (tiles[i] < 0) return MLRA_ERR_INVALID_ARG;
    const int64_t next = (int64_t)prefix[i] + tiles[i];
    const int64_t vnext = (int64_t)vprefix[i] + tiles[i] + (tiles[i] > 0 ? seg_cost : 0);
    if (vnext > INT_MAX) return MLRA_ERR_INVALID_ARG;
    prefix[i + 1] = static_cast<int32_t>(next);
    vprefix[i + 1] = static_cast<int32_t>(vnext);
  }
  PlanView pv;
  pv.prefix = prefix.data();
  pv.vprefix = vprefix.data();
  pv.n = n;
  pv.total = prefix[n];
  pv.vtotal = vprefix[n];
  pv.R = effective_ranges(num_ranges, pv.total);
  pv.cost = seg_cost;
  first_r->assign(n, 0);
  last_r->assign(n, -1);
  if (pv.total == 0) return MLRA_OK;
  for (int64_t r = 0; r < pv.R; ++r) {
    SegmentWalker walk(prefix.data(), n, range_start(pv, r), range_start(pv, r + 1));
    Segment seg;
    while (walk.next(seg)) {
      if (seg.tile0 == 0) (*first_r)[seg.seq] = static_cast<int32_t>(r);
      if (seg.tile0 + seg.ntiles == tiles[seg.seq]) (*last_r)[seg.seq] = static_cast<int32_t>(r);
      if (segs) segs->push_back({static_cast<int32_t>(r), seg.seq, seg.tile0, seg.ntiles});
    }
  }
  return MLRA_OK;
}
}  // namespace

mlra_status mlra_plan_host(const int32_t* tiles_host, int n, int num_ranges, int seg_cost,
                           int32_t* first_range_host, int32_t* num_parts_host) {
  if (!first_range_host || !num_parts_host) return MLRA_ERR_INVALID_ARG;
  std::vector<int32_t> first_r, last_r;
  const mlra_status st = host_plan(tiles_host, n, num_ranges, seg_cost, &first_r, &last_r, nullptr);
  if (st != MLRA_OK) return st;
  for (int s = 0; s < n; ++s) {
    first_range_host[s] = first_r[s];
    num_parts_host[s] = last_r[s] - first_r[s] + 1;
  }
  return MLRA_OK;
}

mlra_status mlra_plan_segments_host(const int32_t* tiles_host, int n, int num_ranges, int seg_cost,
                                    int32_t* range_host, int32_t* seq_host, int32_t* tile0_host,
                                    int32_t* ntiles_host, int max_segments, int* count_host) {
  if (!count_host || max_segments < 0) return MLRA_ERR_INVALID_ARG;
  std::vector<int32_t> first_r, last_r;
  std::vector<std::array<int32_t, 4>> segs;
  const mlra_status st = host_plan(tiles_host, n, num_ranges, seg_cost, &first_r, &last_r, &segs);
  if (st != MLRA_OK) return st;
  const int count = static_cast<int>(segs.size());
  for (int i = 0; i < count && i < max_segments; ++i) {
    if (range_host) range_host[i] = segs[i][0];
    if (seq_host) seq_host[i] = segs[i][1];
    if (tile0_host) tile0_host[i] = segs[i][2];
    if (ntiles_host) ntiles_host[i] = segs[i][3];
  }
  *count_host = count;
  return MLRA_OK;
}

}  // extern "C"
