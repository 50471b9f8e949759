// mlra_internal.h -- declarations shared by the host API (mlra_api.cu) and the kernels
// (mlra_kernels.cu).  Not part of the public C ABI.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace mlra {

constexpr uint32_t kFlagTimeout = 0x1u;
constexpr uint32_t kFlagBadPage = 0x2u;
constexpr uint32_t kFlagBadLength = 0x4u;
// Up to this many sequences the decode kernel plans its work range itself (no prep kernel).
constexpr int kSelfPlanMaxSeqs = 64;
constexpr int kMaxHeads = 128;        // query heads: groups of 64 per CTA
constexpr int kMaxRopePairs = 32;     // d_rope <= 64

// The split plan as the prep kernel writes it for the decode and combine kernels.
//   RangeInfo[r]  : descriptors segs[first, first + count) of work range r, in tile order
//   SegDesc       : one (range, sequence) overlap; its partial slot is r + seq
//   SeqInfo[s]    : ranges r0 .. r1 hold sequence s (its partial slots r + s); empty: r1 = r0 - 1
struct alignas(8) RangeInfo { int32_t first, count; };
struct alignas(16) SegDesc {
  int32_t seq, tile0, ntiles;  // tile0: first tile counted inside the sequence
  int32_t len_whole;           // bits 0-30: sequence length; bit 31: the segment is the whole sequence
};
struct alignas(8) SeqInfo { int32_t r0, r1; };

// Several query tokens per sequence (a speculative or chunked-prefill step): the q tokens of
// caller sequence s are grouped into units of `unit_tokens` (1, or 2 for the kernel with 128 query
// rows) and the decode runs N = (caller sequences) x units_per_seq virtual sequences,
// v = s units_per_seq + u for unit u, over s's cache rows.  Token t is at position
// seq_lens[s] - q + t and sees the positions up to its own (causal), i.e. its length is
// seq_lens[s] - (q - 1 - t); a unit's length is that of its last token,
//   seq_lens[s] - (units_per_seq - 1 - u) unit_tokens,
// and its first token's length is unit_tokens - 1 less.
__host__ __device__ inline int virtual_len(const int32_t* seq_lens, int v, int units_per_seq,
                                           int unit_tokens) {
  if (units_per_seq == 1) return seq_lens[v];
  return seq_lens[v / units_per_seq] - (units_per_seq - 1 - v % units_per_seq) * unit_tokens;
}

struct PrepParams {
  const int32_t* seq_lens;    // caller lengths [N / q_per_seq]
  int N, limit, tile, num_ranges;
  int q_per_seq;              // units (virtual sequences) per caller sequence (virtual_len)
  int unit_tokens;            // query tokens per unit (virtual_len)
  int seg_cost;               // tiles a sequence start costs a CTA (plan balance)
  int32_t* scratch;           // [5 N + 2] plan arrays when N is too large for shared memory
  RangeInfo* ranges;          // [num_ranges]
  SegDesc* segs;              // [num_ranges + N - 1]
  SeqInfo* seqs;              // [N]
  uint32_t* flags;            // this kernel's status bits (one of the combine kernel's slots)
  float* out;                 // rows of empty sequences are zeroed ...
  float* lse;                 // ... and their lse set to -inf (nullable)
  int H, B, out_width;        // out: [N, H, out_width], lse: [N, H, B]
};

// Parameters of the split-KV decode kernel (K1).
struct DecodeParams {
  // the plan: from the prep kernel (self_plan == 0) or made by each CTA from seq_lens
  const RangeInfo* ranges;    // [num_ranges] (prep kernel)
  const SegDesc* segs;
  int self_plan;              // 1: N <= kSelfPlanMaxSeqs, plan in-kernel
  const int32_t* seq_lens;    // caller lengths [N] (self_plan)
  int limit, tile, seg_cost;  // length bound, positions per tile, plan balance (self_plan)
  SeqInfo* seqs;              // [N] written by CTA 0 for the combine kernel (self_plan)
  uint32_t* cta_flags;        // [grid] status bits of each CTA, written at exit
  const int32_t* page_table;  // [N, max_pages] or nullptr (contiguous)
  float* out;                 // final output, row width out_width, or nullptr
  float* lse;                 // [N, H, B] or nullptr
  float* part_o;              // partial outputs [slots, H, dck]
  float* part_ml;             // partial (m, l) [slots, H, B, 2]
  int N, H, B;
  int d_blk_out;              // branch width of the caller's output
  int out_width;              // row width of out (d_latent)
  int dck;                    // latent width seen by the kernel (B * padded d_blk)
  int n_groups;               // CTAs per work range: B x (64-head groups), group g = (g / B, g % B)
  int num_ranges;
  int page_size, max_pages, max_seq_len;
  int64_t n_pages;            // pages in the pool (paged layout)
  int oob_row;                // tile row used for an invalid page id (reads zeros)
  int q_per_seq;              // units per caller sequence: virtual sequence v reads the cache
                              // rows of caller sequence v / q_per_seq (virtual_len)
  int unit_tokens;            // query tokens per unit (virtual_len)
  float scale_log2;           // softmax_scale * log2(e)
  float gamma;                // branch_scale
  int write_final;            // whole-sequence segments write `out` directly
  int tma_out;                // ... through the out tensor map (d_blk_out % 32 == 0)
  int force_replan;           // test hook: treat the speculative in-kernel plan as stale
  int force_timeout;          // test hook: the TMA producer's first wait runs out (short limit)
  uint64_t timeout_ns;        // bound on every wait inside the kernel
};

struct CombineParams {
  const SeqInfo* seqs;        // [N] (prep kernel, or the decode kernel's CTA 0)
  const uint32_t* cta_flags;  // [n_flag_slots] status bits of the decode CTAs (and the prep kernel)
  int n_flag_slots;
  uint32_t* status;           // the call's status word = OR of the slots
  const float* part_o;
  const float* part_ml;
  float* out;
  float* lse;
  int N, H, B;
  int dblk_k, dck;            // kernel branch width and latent width
  int d_blk_out;              // caller branch width
  int groups;                 // part groups per head (1, 2, 4 or 8): parts are split across warps
  int summed;                 // 1: out[s,h,:d_blk_out] = sum over branches
  int final_written;          // 1: sequences held in one part were written by K1
  float gamma;
};

// Per-head products (K5), steps 1 and 3: out[N, H, d_out] = A_h x[N, H, d_in] per head h.
struct ProjectParams {
  const void* w_packed;       // A in the packed image of mlra_pack_kernel
  const float* x;             // [N, H, d_in] fp32
  void* y;                    // [N, H, d_out], fp32 or bf16
  uint32_t* status;           // nullable: kFlagTimeout on a wait that ran out
  int N, H, d_in, d_out;
  int out_bf16;
  uint64_t timeout_ns;
  // Step 3 straight after the attention kernel (no combine kernel): x[s] is the attention
  // kernel's final output for sequences held in one part (or empty), else the merge of the
  // partial results of its parts, times gamma (mlra_merge.cuh).
  int merge;
  const SeqInfo* seqs;        // [N] parts r0 .. r1 of each sequence (slots r + s)
  const float* part_ml;       // [slots, H, B, 2]
  const float* part_o;        // [slots, H, d_in]
  int B, dblk;                // branches, branch width (d_in = B dblk)
  float gamma;
  const uint32_t* cta_flags;  // the attention kernel's status slots, ORed into *status
  int n_flag_slots;
};

// RoPE of the new token's query and key, and its append to the cache (K7).
struct RopeAppendParams {
  const float* q_rope_in;     // [N, H, d_rope] before rotation
  const float* kr_new;        // [N, d_rope] before rotation
  const float* c_new;         // [N, d_latent]
  const int32_t* seq_lens;    // [N]: the new token's position
  const int32_t* page_table;  // [N, max_pages] or nullptr (contiguous)
  int max_pages, page_size, max_seq_len;
  int64_t n_pages;
  uint16_t* c_kv;             // bf16 cache rows, pitch c_row_stride
  uint16_t* k_rope;           // bf16 cache rows, pitch kr_row_stride
  int64_t c_row_stride, kr_row_stride;
  uint16_t* q_rope_out;       // [N, H, d_rope] bf16
  int N, H, d_rope, d_latent;
  double base;                // RoPE base
  uint32_t* status;           // nullable: kFlagBadPage / kFlagBadLength for a skipped append
};

struct RepackParams {
  const void* q_lat; const void* q_rope; const void* c_kv; const void* k_rope;
  uint16_t* q_out; uint16_t* qr_out; uint16_t* c_out; uint16_t* kr_out;
  int N, H, B, d_blk, dblk_k, d_rope;
  int64_t rows, c_row_stride, kr_row_stride;
  int src_f32;
};

// Kernel variants of K1, one per padded branch width (one branch per CTA).
enum Variant { kV64 = 0, kV128, kV256, kV512, kNumVariants };

int variant_smem_bytes(Variant v);
int variant_tile(Variant v);  // KV positions per tile (64 or 128)
cudaError_t launch_prep(const PrepParams& p, cudaStream_t st);
// tout / tpart: fp32 store maps of out [N, H, out_width] and part_o [slots, H, dck], boxes of
// 16 heads x 32 columns, 128-byte swizzle
cudaError_t launch_decode(Variant v, const CUtensorMap& tq, const CUtensorMap& tqr,
                          const CUtensorMap& tc, const CUtensorMap& tkr, const CUtensorMap& tout,
                          const CUtensorMap& tpart, const DecodeParams& p, int grid,
                          cudaStream_t st);
// K1M: 128 query rows per CTA (two tokens x 64 heads), branch width 128; tq / tqr with boxes of
// 64 columns x 128 rows over [width, 128, units]
cudaError_t launch_decode_m128(const CUtensorMap& tq, const CUtensorMap& tqr,
                               const CUtensorMap& tc, const CUtensorMap& tkr,
                               const DecodeParams& p, int grid, cudaStream_t st);
cudaError_t launch_combine(const CombineParams& p, cudaStream_t st);
cudaError_t launch_repack(const RepackParams& p, cudaStream_t st);
cudaError_t launch_project(const ProjectParams& p, cudaStream_t st);
cudaError_t launch_pack(const void* w, void* packed, int H, int d_in, int d_out, bool transpose,
                        cudaStream_t st);
cudaError_t launch_rope_append(const RopeAppendParams& p, cudaStream_t st);
cudaError_t launch_resolve_rows(const int32_t* lens_or_null, const int32_t* seq_lens,
                                const int32_t* page_table, int N, int max_pages, int page_size,
                                int max_seq_len, int64_t n_pages, int oob_row, int64_t* rows_out,
                                int row_pitch, cudaStream_t st);

}  // namespace mlra
