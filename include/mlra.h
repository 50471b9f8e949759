/*
 * mlra.h -- C ABI of the B200 (sm_100a) MLRA decode-attention library.
 *
 * The operation ("Multi-Head Low-Rank Attention", yunpan.plus page):
 *   section 1.3  MLA's efficient decode in three steps -- (1) absorb the key up-projection
 *                into the query, (2) run MQA-style attention of the absorbed query against the
 *                cached latent vectors, (3) apply the value up-projection.  The core of this
 *                library is step 2 (mlra_decode, below); steps 1 and 3 (mlra_absorb,
 *                mlra_project), the new token's RoPE and cache append (mlra_rope_append) and
 *                several query tokens per sequence (mlra_decode_multi) follow further down.
 *   section 2    the per-head NoPE key is a sum of B block projections of the latent, so the
 *                latent c_t splits into B column blocks c_{t,b} of width d_blk = d_latent / B;
 *   section 3.1  MLRA moves that sum behind the attention: every branch b runs its own
 *                attention over its block with its own softmax over positions, and the RoPE
 *                key k^R_t is shared by all branches;
 *   section 3.3  the sum of the branch outputs is scaled.
 *
 * For sequence s, head h < heads, branch b < B and cached position j < seq_lens[s]:
 *
 *   score(j)          = softmax_scale * ( q_lat[s,h, b-block] . c_kv[row(s,j), b-block]
 *                                       + q_rope[s,h,:]       . k_rope[row(s,j), :] )
 *   p                 = softmax over j of score                 (one softmax per branch)
 *   out[s,h, b-block] = branch_scale * sum_j p(j) * c_kv[row(s,j), b-block]
 *   lse[s,h,b]        = log sum_j exp(score(j))                  (natural log)
 *
 * With num_branches = 1 this is plain MLA decode.  MLRA_OUT_SUMMED adds the B branch
 * outputs instead: out[s,h,:] = sum_b out[s,h,b-block] (width d_blk).
 *
 * Rows: with page_table == NULL the cache is contiguous, row(s,j) = s * max_seq_len + j;
 * otherwise row(s,j) = page_table[s * max_pages_per_seq + j / page_size] * page_size
 *                      + j % page_size.
 *
 * Conventions for every entry point:
 *   - Pointers named *_host are host memory; every other pointer is CUDA device memory.
 *   - The caller owns every buffer, including the workspace; the library never allocates
 *     device memory and keeps no pointer after a call returns.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     unless stated otherwise; nothing synchronises.
 *   - Argument errors are returned before any work is queued.  Problems found on the device
 *     (bad lengths, bad page ids, an internal wait that ran out) never trap: they set bits in
 *     a status word inside the workspace, read with mlra_read_status().
 *   - All functions are thread-safe; calls that share a workspace must not overlap on the GPU.
 */
#ifndef MLRA_H_
#define MLRA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mlra_stream_t; /* same type as cudaStream_t */

typedef enum {
  MLRA_OK = 0,
  MLRA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, inconsistent dims */
  MLRA_ERR_UNSUPPORTED = 2,  /* valid but not handled (see mlra_decode) */
  MLRA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  MLRA_ERR_TIMEOUT = 4,      /* a device-side bounded wait ran out (status word) */
  MLRA_ERR_WORKSPACE = 5,    /* workspace null, too small or misaligned */
  MLRA_ERR_BAD_PAGE = 6,     /* a page id outside [0, cache_rows / page_size) (status word) */
  MLRA_ERR_BAD_LENGTH = 7,   /* a sequence length < 0 or beyond the cache (status word) */
  MLRA_ERR_SCRATCH_LIMIT = 8 /* mlra_decode_static_scratch: the problem needs more scratch than
                                MLRA_STATIC_SCRATCH_BYTES */
} mlra_status;

typedef enum { MLRA_BF16 = 0, MLRA_F32 = 1 } mlra_dtype;
typedef enum { MLRA_OUT_BRANCHES = 0, MLRA_OUT_SUMMED = 1 } mlra_out_mode;

/* Device status bits (mlra_read_status).
 *
 * Test hooks, read from the environment at every decode call (unset in normal use):
 *   MLRA_TEST_FORCE_REPLAN   the attention kernel treats its speculative work plan as stale and
 *                            re-plans after its dependency wait; results are unchanged.
 *   MLRA_TEST_FORCE_TIMEOUT  each attention CTA with a copy left to issue after its speculative
 *                            ones waits 1 ms on a barrier nothing completes, so the call reports
 *                            MLRA_ERR_TIMEOUT / MLRA_FLAG_TIMEOUT; its outputs are undefined and
 *                            the next call on the same workspace is unaffected. */
#define MLRA_FLAG_TIMEOUT 0x1u
#define MLRA_FLAG_BAD_PAGE 0x2u
#define MLRA_FLAG_BAD_LENGTH 0x4u

typedef struct {
  float softmax_scale; /* sigma: multiplies the whole score (NoPE + RoPE terms) */
  float branch_scale;  /* gamma: multiplies every branch output (1/B for the MLRA sum) */
} mlra_scales;

typedef struct {
  int batch;              /* N >= 1 sequences, one query token each */
  int heads;              /* H, 1..128 (groups of 64 heads per CTA) */
  int num_branches;       /* B >= 1, divides d_latent */
  int d_latent;           /* d_c = B * d_blk, <= 512 */
  int d_rope;             /* d_R, 1..64 */
  int page_size;          /* P (paged layout, a multiple of 64); ignored when page_table == NULL */
  int max_pages_per_seq;  /* page_table row pitch (paged layout) */
  int max_seq_len;        /* contiguous layout: row pitch of a sequence; both layouts: bound on
                             seq_lens (paged: also <= max_pages_per_seq * page_size) */
  long long cache_rows;   /* rows in c_kv and k_rope (paged: the pool; contiguous: >= N * max_seq_len) */
  long long c_row_stride; /* elements between consecutive c_kv rows (>= d_latent) */
  long long kr_row_stride;/* elements between consecutive k_rope rows (>= d_rope); c_kv and
                             k_rope may be two column ranges of one row (e.g. 576-wide rows) */
  mlra_dtype dtype;       /* element type of q_lat, q_rope, c_kv, k_rope */
  mlra_out_mode out_mode;
  int num_ranges;         /* 0: one work range per SM (per branch group); > 0 forces the number
                             of equal tile ranges the batch is cut into (split-K control) */
} mlra_dims;

/* Bytes of workspace mlra_decode needs for `dims` (and the device's SM count when
 * dims->num_ranges == 0, queried on the current device).  Host only, synchronous.
 * Errors: MLRA_ERR_INVALID_ARG / MLRA_ERR_UNSUPPORTED as mlra_decode; MLRA_ERR_CUDA when the
 * SM count is needed and no device is available. */
mlra_status mlra_workspace_size(const mlra_dims* dims, size_t* bytes_host);

/* Step 2 of MLRA decode (see the top of this file).
 *   q_lat      [N, H, d_latent]   dims->dtype, contiguous: the absorbed queries q~ (section 1.3,
 *                                 step 1 output), branch b in columns [b*d_blk, (b+1)*d_blk)
 *   q_rope     [N, H, d_rope]     dims->dtype, contiguous: the RoPE queries q^R
 *   c_kv       [cache_rows, *]    dims->dtype, row pitch c_row_stride: latent cache c^KV
 *   k_rope     [cache_rows, *]    dims->dtype, row pitch kr_row_stride: shared RoPE key cache k^R
 *   seq_lens   [N]                int32, read on the device
 *   page_table [N, max_pages_per_seq] int32 page ids, or NULL for the contiguous layout
 *   B          must equal dims->num_branches (kept in the signature as a guard)
 *   scales     host pointer to {sigma, gamma}
 *   out        fp32 [N, H, d_latent] (MLRA_OUT_BRANCHES) or [N, H, d_latent / B] (SUMMED)
 *   lse        fp32 [N, H, B] or NULL
 *   workspace  >= mlra_workspace_size bytes, 256-byte aligned, caller-owned scratch
 * An empty sequence (seq_lens[s] == 0) gives out = 0 and lse = -inf.
 * bf16 inputs with d_blk in {64, 128, 256, 512}, d_rope == 64, 16-byte aligned rows and
 * base pointers are read in place.  Other shapes (and fp32 inputs) are first repacked into
 * padded bf16 copies inside the workspace (a full copy of the cache per call: meant for
 * small problems).  MLRA_ERR_UNSUPPORTED: H > 128, d_latent > 512, d_rope > 64, page_size not
 * a multiple of 64, misaligned bf16 rows.  Launch failures return MLRA_ERR_CUDA. */
mlra_status mlra_decode(const void* q_lat, const void* q_rope, const void* c_kv, const void* k_rope,
                        const int32_t* seq_lens, const int32_t* page_table, int B,
                        const mlra_scales* scales, float* out, float* lse, const mlra_dims* dims,
                        void* workspace, size_t ws_bytes, mlra_stream_t stream);

/* Same as mlra_decode, and records the caller's CUDA events `k1_begin` / `k1_end` (cudaEvent_t,
 * either may be NULL) on `stream` immediately before and after the split-KV attention kernel,
 * so that its duration can be timed alone (cudaEventElapsedTime).  Errors as mlra_decode;
 * a failing cudaEventRecord returns MLRA_ERR_CUDA. */
typedef struct CUevent_st* mlra_event_t; /* same type as cudaEvent_t */
mlra_status mlra_decode_profiled(const void* q_lat, const void* q_rope, const void* c_kv,
                                 const void* k_rope, const int32_t* seq_lens,
                                 const int32_t* page_table, int B, const mlra_scales* scales,
                                 float* out, float* lse, const mlra_dims* dims, void* workspace,
                                 size_t ws_bytes, mlra_stream_t stream, mlra_event_t k1_begin,
                                 mlra_event_t k1_end);

/* What mlra_decode will do for `dims` (same rules and SM-count query as mlra_workspace_size).
 * Host only, synchronous. */
typedef struct {
  int repack;             /* 1: inputs are first copied into padded bf16 buffers */
  int launches;           /* kernels launched per mlra_decode call */
  int num_ranges;         /* equal work ranges the batch's KV tiles are cut into */
  int ctas;               /* CTAs of the attention kernel (ranges x branch groups) */
  int kernel_branch_width;/* branch width after padding (64, 128, 256 or 512) */
  int branches_per_cta;   /* branches whose latent columns one attention CTA reads */
  int tile;               /* KV positions per tile (64 or 128) */
  long long partial_slots;/* partial-result slots in the workspace (num_ranges + N - 1) */
  int segment_cost_tiles; /* plan balance: tiles a sequence start costs a CTA (mlra_plan_host) */
  size_t workspace_bytes;
} mlra_plan_info;
mlra_status mlra_query_plan(const mlra_dims* dims, mlra_plan_info* info_host);

/* Decode for several query tokens per sequence (a speculative-decoding or chunked-prefill step):
 * the q_len newest tokens of every sequence attend the cache at once, each causally — token t of
 * sequence s sits at position seq_lens[s] - q_len + t (all q_len tokens are already in the cache,
 * seq_lens counts them) and attends positions 0 .. seq_lens[s] - q_len + t.  Per token this is the
 * single-token decode of mlra_decode (the pages' step 2) with the length
 * seq_lens[s] - (q_len - 1 - t) over sequence s's cache rows; the call runs dims->batch * q_len
 * such decodes in one launch sequence (each reads its own prefix of the cache: q_len reads of it).
 *   q_lat  [N, q_len, H, d_c], q_rope [N, q_len, H, d_R], contiguous, dtype as dims->dtype
 *   out    [N, q_len, H, width] fp32; lse nullable [N, q_len, H, B]
 *   dims   the caller's shapes with batch = N (not N * q_len)
 *   workspace  at least mlra_workspace_size_multi(dims, q_len) bytes
 * Everything else as mlra_decode.  A token whose length would be negative (seq_lens[s] < q_len - 1
 * - t) raises MLRA_FLAG_BAD_LENGTH and gets an empty output.
 * Errors as mlra_decode; MLRA_ERR_INVALID_ARG for q_len < 1. */
mlra_status mlra_decode_multi(const void* q_lat, const void* q_rope, const void* c_kv,
                              const void* k_rope, const int32_t* seq_lens,
                              const int32_t* page_table, int q_len, int B,
                              const mlra_scales* scales, float* out, float* lse,
                              const mlra_dims* dims, void* workspace, size_t ws_bytes,
                              mlra_stream_t stream);

/* Workspace bytes for mlra_decode_multi with q_len query tokens per sequence (dims->batch = N). */
mlra_status mlra_workspace_size_multi(const mlra_dims* dims, int q_len, size_t* bytes_host);

/* mlra_decode for callers that cannot hand the library any device memory: hosts that own every
 * device allocation through their own pool and give plug-ins no allocator, or serving paths that
 * must not allocate at all.  It takes the same arguments as mlra_decode minus the workspace and
 * uses instead a scratch array built into the library (MLRA_STATIC_SCRATCH_BYTES, allocated on a
 * device when the library's kernels are loaded there and kept until the process exits).  It
 * allocates nothing and frees nothing.  (This entry point is an addition of this library; the
 * method's pages have no counterpart.)
 *   - The first call on each device does a one-time set-up: with that device current it looks up
 *     the scratch array's device address.  Make that first call before any stream capture.
 *   - Every call on a device shares the one array, which keeps the last call's contents (nothing
 *     in it has to start at zero: each call rewrites what it later reads).  Calls that overlap on
 *     the GPU (other streams, other host threads) race on it: serialise them.
 *   - Problems whose workspace (mlra_workspace_size) exceeds MLRA_STATIC_SCRATCH_BYTES, including
 *     every problem that needs the fp32 / padded repack copies, return MLRA_ERR_SCRATCH_LIMIT
 *     before any work is queued.  Other errors as mlra_decode.  The device status word of these
 *     calls is not readable through mlra_read_status. */
#define MLRA_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)
mlra_status mlra_decode_static_scratch(const void* q_lat, const void* q_rope, const void* c_kv,
                                       const void* k_rope, const int32_t* seq_lens,
                                       const int32_t* page_table, int B, const mlra_scales* scales,
                                       float* out, float* lse, const mlra_dims* dims,
                                       mlra_stream_t stream);

/* Step 3 of the absorbed decode: the value up-projection of every branch output, summed over the
 * branches ("Multi-Head Low-Rank Attention", yunpan.plus page, section 1.3 step 3; the branch sum
 * of sections 3 and 3.3).  Head h's projections sit side by side,
 * W_h = [W^UV_{h,1} | ... | W^UV_{h,B}]:
 *     y[s, h, :] = W_h o[s, h, :]
 *   o        [N, H, d_latent] fp32 device: mlra_decode's output in MLRA_OUT_BRANCHES mode (gamma
 *            already applied)
 *   w_packed H * d_head * d_latent bf16 device: the weights W^UV as mlra_pack_wuv wrote them
 *   y        [N, H, d_head] fp32 device (written)
 *   status nullable device uint32: gets MLRA_FLAG_TIMEOUT if a bounded wait runs out
 * Products in bf16 (o is rounded to bf16) with fp32 accumulation.  Asynchronous on `stream`; the
 * kernel starts reading w_packed before it waits for the previous kernel on the stream
 * (programmatic serialization), so w_packed must not be written by a kernel that lets its
 * dependents start early (mlra_pack_wuv does not).
 * Errors: MLRA_ERR_INVALID_ARG for null pointers or sizes < 1; MLRA_ERR_UNSUPPORTED unless
 * d_latent is a multiple of 64 up to 512, d_head a multiple of 64 and all three arrays 16-byte
 * aligned; MLRA_ERR_CUDA when the launch fails.  The pages give no kernel for this step. */
mlra_status mlra_project(const float* o, const void* w_packed, float* y, int N, int H, int d_latent,
                         int d_head, uint32_t* status, mlra_stream_t stream);

/* Steps 2 and 3 of one attention layer in one call ("Multi-Head Low-Rank Attention", yunpan.plus
 * page, section 1.3 steps 2 and 3 with the branch sum of sections 3 and 3.3):
 *     y[s, h, :] = W_h o[s, h, :],   o = mlra_decode's output in MLRA_OUT_BRANCHES mode
 * The attention kernel runs as in mlra_decode; instead of the combine kernel and mlra_project, one
 * step-3 kernel merges the partial softmax states of the sequences the attention kernel split
 * while it stages o[s, h] for its product (one launch and the fp32 o round trip fewer).
 *   q_lat ... scales   as mlra_decode (bf16 inputs read in place; dims->out_mode must be
 *                      MLRA_OUT_BRANCHES)
 *   w_packed, d_head   as mlra_project (H * d_head * d_latent bf16 from mlra_pack_wuv)
 *   y                  [N, H, d_head] fp32 device (written)
 *   workspace          >= mlra_workspace_size_project(dims) bytes, 256-byte aligned; its status word
 *                      is read with mlra_read_status
 * No LSE output.  Errors: as mlra_decode and mlra_project; MLRA_ERR_UNSUPPORTED for summed mode,
 * fp32 inputs or padded branch widths (the repack path).  The pages give no kernel for this
 * fusion. */
mlra_status mlra_workspace_size_project(const mlra_dims* dims, size_t* bytes_host);
mlra_status mlra_decode_project(const void* q_lat, const void* q_rope, const void* c_kv,
                                const void* k_rope, const int32_t* seq_lens,
                                const int32_t* page_table, int B, const mlra_scales* scales,
                                const void* w_packed, int d_head, float* y, const mlra_dims* dims,
                                void* workspace, size_t ws_bytes, mlra_stream_t stream);

/* Packs the step-3 weights once for mlra_project (they are model weights: pack at load time).
 *   w_uv     [H, d_head, d_latent] bf16 device, row-major: W_h row k = w_uv[h, k, :]
 *   w_packed H * d_head * d_latent bf16 device (written; same size, caller-owned): per head and
 *            64-row tile, the d_latent / 64 blocks of 64 columns in the tensor-core image
 * Asynchronous on `stream`.  Errors as mlra_project (sizes, 16-byte alignment). */
mlra_status mlra_pack_wuv(const void* w_uv, void* w_packed, int H, int d_latent, int d_head,
                          mlra_stream_t stream);

/* Step 1 of the absorbed decode: each head's query absorbs the key up-projections of the B
 * branches ("Multi-Head Low-Rank Attention", yunpan.plus page, section 1.3 step 1; the block form
 * of section 2): q_lat[s, h, b-block] = (W^UK_{h,b})^T q_nope[s, h].
 *   q_nope   [N, H, d_head] fp32 device
 *   w_packed H * d_head * d_latent bf16 device, written by mlra_pack_wuk
 *   q_lat    [N, H, d_latent] bf16 device (written): mlra_decode's q_lat
 *   status   nullable device uint32: MLRA_FLAG_TIMEOUT if a bounded wait runs out
 * Products in bf16 (q_nope rounded) with fp32 accumulation, the result rounded to bf16.
 * Asynchronous on `stream`; w_packed is read early as in mlra_project.
 * Errors: MLRA_ERR_INVALID_ARG for null pointers or sizes < 1; MLRA_ERR_UNSUPPORTED unless d_head
 * is a multiple of 64 up to 512, d_latent a multiple of 64 and the arrays 16-byte aligned. */
mlra_status mlra_absorb(const float* q_nope, const void* w_packed, void* q_lat, int N, int H,
                        int d_head, int d_latent, uint32_t* status, mlra_stream_t stream);

/* Packs the step-1 weights once for mlra_absorb (model weights: pack at load time).
 *   w_uk     [H, d_head, d_latent] bf16 device, row-major: head h's key up-projections side by
 *            side, W^UK_{h,b} = w_uk[h, :, b*d_blk : (b+1)*d_blk]
 *   w_packed H * d_head * d_latent bf16 device (written): the transposes, in the tensor-core image
 * Errors as mlra_absorb. */
mlra_status mlra_pack_wuk(const void* w_uk, void* w_packed, int H, int d_head, int d_latent,
                          mlra_stream_t stream);

/* The new token of every sequence, before step 2: rotary position embedding of its RoPE query
 * (one per head) and of its RoPE key (shared by all heads and branches), and the append of its
 * latent and key to the cache.  The pages describe DeepSeek's decoupled RoPE without the rotation's
 * details; the rotation is the standard one: pair (2i, 2i+1) of a vector at position p turns by
 * p * rope_base^(-2i / d_rope).  The token's position is p = seq_lens[s] and its cache row follows
 * mlra_decode's addressing (page table, or s * max_seq_len + p); the caller then passes
 * seq_lens + 1 to mlra_decode.
 *   q_rope_in  [N, H, d_rope] fp32 device     kr_new [N, d_rope] fp32     c_new [N, d_latent] fp32
 *   seq_lens   [N] int32 device; page_table as for mlra_decode (NULL: contiguous)
 *   dims       the cache geometry as for mlra_decode (bf16 cache; batch, heads, d_latent, d_rope,
 *              page_size / max_pages_per_seq or max_seq_len, cache_rows, row strides)
 *   c_kv, k_rope  the bf16 caches (row `row` written)
 *   q_rope_out [N, H, d_rope] bf16 device (written): mlra_decode's q_rope
 *   status     nullable device uint32: MLRA_FLAG_BAD_LENGTH (position outside the sequence's
 *              cache space) or MLRA_FLAG_BAD_PAGE (invalid page id); that append is skipped
 * Errors: MLRA_ERR_INVALID_ARG for null pointers, a non-positive base or invalid dims;
 * MLRA_ERR_UNSUPPORTED for an fp32 cache, an odd d_rope, d_latent, kr_row_stride or c_row_stride,
 * or an array that is not 16-byte aligned. */
mlra_status mlra_rope_append(const float* q_rope_in, const float* kr_new, const float* c_new,
                             const int32_t* seq_lens, const int32_t* page_table,
                             const mlra_dims* dims, void* c_kv, void* k_rope, void* q_rope_out,
                             double rope_base, uint32_t* status, mlra_stream_t stream);

/* Reads the status word that the last mlra_decode on `workspace` left, after synchronising
 * `stream`.  *flags_host receives the MLRA_FLAG_* bits; the return value is MLRA_OK when no
 * bit is set, else the status of the most serious bit (timeout, bad page, bad length). */
mlra_status mlra_read_status(const void* workspace, mlra_stream_t stream, uint32_t* flags_host);

/* Test hook for the indexing logic (bit-exact): writes the cache row of every position
 * j < min(seq_lens[s], row_pitch) into rows_out[s * row_pitch + j] (int64, device), computed
 * by the same device function the decode kernel uses to address its TMA tiles.  Entries
 * past a sequence's length are left untouched.  Same dims rules as mlra_decode. */
mlra_status mlra_debug_resolve_rows(const int32_t* seq_lens, const int32_t* page_table,
                                    const mlra_dims* dims, int64_t* rows_out, int row_pitch,
                                    mlra_stream_t stream);

/* Host replica of the split plan (the same __host__ __device__ code the kernels run): tile
 * counts tiles_host[N] are cut into min(num_ranges, total tiles) contiguous ranges that balance
 * tiles plus seg_cost tiles per non-empty sequence (each range r starts at the virtual position
 * floor(r V / R) of the virtual length V = sum of (tiles + seg_cost) over non-empty sequences;
 * a position inside a sequence's seg_cost leading slots maps to the sequence's first tile).  The
 * attention kernel uses seg_cost = mlra_plan_info.segment_cost_tiles; 0 gives equal ranges.
 * Writes for every sequence the first range touching it and the number of ranges (partial
 * results) it is split into (0 for an empty sequence).  Errors: MLRA_ERR_INVALID_ARG for a
 * negative tile count or seg_cost, num_ranges < 1, n < 1, or a virtual length past INT_MAX.
 * Host only, synchronous; for tests and tooling. */
mlra_status mlra_plan_host(const int32_t* tiles_host, int n, int num_ranges, int seg_cost,
                           int32_t* first_range_host, int32_t* num_parts_host);

/* Host replica of the per-CTA segment walk of the attention kernel: for tile counts
 * tiles_host[N] and num_ranges CTAs (per branch group), lists every (range, sequence, first
 * tile, tile count) segment that the kernel's CTAs r = 0 .. num_ranges-1 process, in CTA order.
 * At most max_segments are written to the four *_host arrays; *count_host receives the total.
 * Host only, synchronous; for tests and tooling. */
mlra_status mlra_plan_segments_host(const int32_t* tiles_host, int n, int num_ranges, int seg_cost,
                                    int32_t* range_host, int32_t* seq_host, int32_t* tile0_host,
                                    int32_t* ntiles_host, int max_segments, int* count_host);

/* Human-readable name of a status code (static string). */
const char* mlra_status_string(mlra_status s);

/* Library version, e.g. 0x000100 for 0.1.0. */
int mlra_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLRA_H_ */
