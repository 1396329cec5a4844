/*
 * fa.h -- C ABI of the B200 (sm_100a) block-sparse attention library (libfa.so).
 *
 * Two operations, following the FlexAttention how-to
 * ("FlexAttention on Apple Silicon: block mask how-to", dreaming.press):
 *
 *   fa_create_block_mask  ~ create_block_mask(mask_mod, B=None, H=None, Q_LEN, KV_LEN)
 *                           ("Mask 1: causal", "Mask 2: sliding-window causal",
 *                            "Mask 3: document-packed"): classifies every 128x128 block of
 *                           the (Q_LEN x KV_LEN) score grid as empty, full or partial and
 *                           writes per-row block lists; one mask is broadcast over batch
 *                           and heads.
 *   fa_flex_attention_fwd ~ flex_attention(q, k, v, block_mask=, score_mod=)
 *                           ("Setup", "Bonus: a score_mod for soft-capping"):
 *                           out = softmax(Q K^T * scale + mask / score_mod) V computed tile by
 *                           tile on the tensor cores with an online softmax; empty blocks are
 *                           never touched.  The attention definition is the one of the SDPA
 *                           tutorial (qiita GeneLab_999, section 1).
 *
 * Conventions shared by every call
 *  - All tensor pointers are DEVICE pointers owned by the caller (for instance
 *    torch tensors).  The library never allocates device memory.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Argument errors are detected on the host before any launch and
 *    returned as a status; nothing is launched then.
 *  - Layouts are C-contiguous.  Q is (B, H, L, D); K and V are (B, H, S, D); out
 *    is (B, H, L, D) in the input dtype; lse is (B, H, L) float32.  D is 64 or 128.
 *  - Mask semantics: "true" means the (q, kv) pair is used (the SDPA boolean-mask
 *    convention, SDPA tutorial section 4).  Indices are absolute positions, so for
 *    L != S the causal diagonal is upper-left aligned.  Positions past L or S are
 *    never live.
 *  - A query row with no live key returns out = 0 and lse = -inf (SDPA returns 0
 *    for such rows, SDPA tutorial section 4).
 *  - Each call states the alignment its pointers need and checks it on the host.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,  /* bad pointer, size, enum value or mismatched shapes */
  FA_ERR_UNSUPPORTED = 2,  /* valid request outside what this library implements (e.g. D=96) */
  FA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed (no device, launch error ...) */
  FA_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up (reported by
                              fa_get_last_device_error) */
  FA_ERR_SCRATCH_TOO_SMALL = 5  /* fa_flex_attention_fwd_noalloc: the problem's block
                                   tables need more than FA_NOALLOC_SCRATCH_BYTES */
} fa_status;

typedef enum {
  FA_MASK_CAUSAL = 0,                /* q_idx >= kv_idx                                   */
  FA_MASK_SLIDING_WINDOW_CAUSAL = 1, /* q_idx >= kv_idx && q_idx - kv_idx < window        */
  FA_MASK_DOCUMENT_CAUSAL = 2,       /* q_idx >= kv_idx && doc_id[q_idx] == doc_id[kv_idx] */
  FA_MASK_BITMAP = 3                 /* bit kv_idx of row q_idx of a caller's bitmap
                                        (fa_create_block_mask_bitmap)                    */
} fa_mask_kind;

typedef enum {
  FA_SCORE_NONE = 0,
  FA_SCORE_TANH_SOFTCAP = 1          /* score -> softcap * tanh(score / softcap), on the scaled score */
} fa_score_kind;

typedef enum { FA_BF16 = 0, FA_FP16 = 1 } fa_dtype;

/* Block size of the mask tables; the only value this library accepts. */
#define FA_BLOCK 128
/* Largest Q_LEN / KV_LEN accepted (8192 blocks of 128). */
#define FA_MAX_LEN (8192 * 128)

/*
 * Block tables of one mask, broadcast over batch and heads.
 *
 * The caller allocates the five arrays on the device (8-byte aligned) and stores their pointers
 * here BEFORE calling fa_create_block_mask, which fills both the arrays and the
 * scalar fields.  Sizes: nQ = ceil(q_len / 128), nKV = ceil(kv_len / 128)
 * (fa_block_mask_dims computes them).
 *
 *   kv_num_blocks[nQ]           number of PARTIAL blocks of q-block row i
 *   kv_indices[nQ * nKV]        row i: its partial kv-block indices, ascending, then 0s
 *   full_kv_num_blocks[nQ]      number of FULL blocks of row i
 *   full_kv_indices[nQ * nKV]   row i: its full kv-block indices, ascending, then 0s
 *   q_order[2 * nQ]             the forward kernel's schedule: rank k lists the q-block
 *                               rows by descending live-block count (ties by ascending
 *                               row); q_order[2k] = row, q_order[2k+1] = its partial
 *                               count | full count << 16.  The persistent scheduler hands
 *                               out work in this order (heaviest rows first).
 *
 * A FULL block has all 128 x 128 pairs in range and allowed (the kernel skips the
 * mask there); a PARTIAL block has some but not all pairs live (the kernel evaluates
 * the mask per element); EMPTY blocks appear in neither list and are never read.
 * `doc_id` is kept (not copied): it must stay valid while the mask is used.
 */
typedef struct fa_block_mask {
  int32_t* kv_num_blocks;
  int32_t* kv_indices;
  int32_t* full_kv_num_blocks;
  int32_t* full_kv_indices;
  int32_t* q_order;
  int32_t q_len;
  int32_t kv_len;
  int32_t block;
  int32_t n_q_blocks;
  int32_t n_kv_blocks;
  int32_t kind;           /* fa_mask_kind */
  int32_t window;         /* sliding window W (kind 1), else 0 */
  const int32_t* doc_id;  /* device int32[max(q_len, kv_len)] (kind 2), else NULL */
  const uint32_t* bitmap; /* device bitmap (kind 3, see fa_create_block_mask_bitmap), else NULL */
  int32_t mask_batch;     /* 1: one mask for every batch element; B: one per element */
  int32_t mask_heads;     /* 1: one mask for every head; H: one per head */
} fa_block_mask;

/* nQ and nKV of a (q_len, kv_len) mask with the given block size.
 * Returns FA_ERR_INVALID_ARG for negative lengths, block != 128, lengths above
 * FA_MAX_LEN or NULL outputs.  Host only, no CUDA call. */
FA_API fa_status fa_block_mask_dims(int32_t q_len, int32_t kv_len, int32_t block,
                             int32_t* n_q_blocks, int32_t* n_kv_blocks);

/*
 * Build the block tables of a mask rule (FlexAttention how-to, "Mask 1..3").
 *   kind    fa_mask_kind.
 *   window  W >= 1 for FA_MASK_SLIDING_WINDOW_CAUSAL (ignored otherwise).
 *   doc_id  device int32 array of length max(q_len, kv_len) for
 *           FA_MASK_DOCUMENT_CAUSAL (one id per position, indexed by both q_idx and
 *           kv_idx as in the how-to's document_id tensor); ignored otherwise. Any
 *           int32 values are allowed (they need not be sorted).
 *   q_len, kv_len  >= 0 and <= FA_MAX_LEN;  block must be 128.
 *   bm      in: the five device array pointers (non-NULL when nQ > 0);
 *           out: every field filled.
 * Launches two kernels on `stream`; the tables are ready when the stream reaches
 * that point.  Returns FA_ERR_INVALID_ARG (nothing launched) on bad arguments,
 * FA_ERR_CUDA if a launch fails.
 */
FA_API fa_status fa_create_block_mask(int32_t kind, int32_t window, const int32_t* doc_id,
                               int32_t q_len, int32_t kv_len, int32_t block,
                               fa_block_mask* bm, void* stream);

/*
 * Block tables of per-(batch, head) masks (the how-to's create_block_mask(mask_mod,
 * B, H, Q_LEN, KV_LEN) with B and H given instead of None, "Mask 1: causal": the
 * mask may depend on b and h).  mask_batch is 1 (broadcast over the batch) or the
 * batch size B; mask_heads is 1 or the head count H; instance
 * n = (b or 0) * mask_heads + (h or 0) holds the tables of (b, h).
 *   kind      as fa_create_block_mask, or FA_MASK_BITMAP.
 *   doc_id    kind 2: device int32[instances][max(q_len, kv_len)], instance-major.
 *   bitmap    kind 3: device words [instances][q_len][4 * nKV], 16-byte aligned.
 *   bm        the five arrays sized for all instances: kv_num_blocks[inst * nQ],
 *             kv_indices[inst * nQ * nKV], full_* likewise, q_order[inst * 2 * nQ]
 *             (instance-major; each instance as fa_create_block_mask writes it).
 * The forward kernel reads instance n of a (b, h) unit; fa_block_mask_transpose
 * writes instance-major column lists.  Launches two kernels on `stream`.  Returns
 * FA_ERR_INVALID_ARG (nothing launched) on bad arguments, FA_ERR_CUDA if a launch
 * fails.  fa_create_block_mask and fa_create_block_mask_bitmap build one instance.
 */
FA_API fa_status fa_create_block_mask_bh(int32_t kind, int32_t window, const int32_t* doc_id,
                                  const uint32_t* bitmap, int32_t mask_batch,
                                  int32_t mask_heads, int32_t q_len, int32_t kv_len,
                                  int32_t block, fa_block_mask* bm, void* stream);

/*
 * Block tables of a tabulated mask_mod (the FlexAttention how-to's
 * create_block_mask takes any boolean function of (b, h, q_idx, kv_idx), "Mask 1:
 * causal"; here it is given as one bit per pair, broadcast over batch and heads).
 *   bitmap  device uint32 words, row-major (q_len, 4 * nKV), 16-byte aligned: pair
 *           (q, kv) is kept iff bit kv % 32 (least significant first) of word
 *           kv / 32 of row q is set.  Rows are padded to whole 128-key blocks; bits
 *           at kv >= kv_len are ignored.  Kept (not copied): it must stay valid while
 *           the mask is used, since the forward kernel reads it in PARTIAL blocks.
 *   q_len, kv_len, block, bm, stream   as for fa_create_block_mask.
 * Launches two kernels on `stream`.  Returns FA_ERR_INVALID_ARG (nothing launched)
 * on bad arguments, FA_ERR_CUDA if a launch fails.
 */
FA_API fa_status fa_create_block_mask_bitmap(const uint32_t* bitmap, int32_t q_len, int32_t kv_len,
                                      int32_t block, fa_block_mask* bm, void* stream);

/*
 * Column view of built tables (FlexAttention's BlockMask carries it for the
 * backward pass): for each kv block j, the q blocks i whose block (i, j) is
 * PARTIAL, ascending, and those whose block is FULL.
 *   bm                   tables from fa_create_block_mask / _bitmap (read only).
 *   q_num_blocks[nKV]            number of PARTIAL blocks in column j
 *   q_indices[nKV * nQ]          column j: their q-block indices, ascending, then 0s
 *   full_q_num_blocks[nKV]       number of FULL blocks in column j
 *   full_q_indices[nKV * nQ]     column j: their q-block indices, ascending, then 0s
 *   (per-(batch, head) tables: every array times mask_batch * mask_heads, instance-major)
 * Device arrays owned by the caller.  One kernel on `stream`, ordered after the
 * build on the same stream.  Returns FA_ERR_INVALID_ARG (nothing launched) on NULL
 * arguments, FA_ERR_CUDA if the launch fails; nKV == 0 or nQ == 0 launches nothing.
 */
FA_API fa_status fa_block_mask_transpose(const fa_block_mask* bm, int32_t* q_num_blocks,
                                  int32_t* q_indices, int32_t* full_q_num_blocks,
                                  int32_t* full_q_indices, void* stream);

/*
 * Host-side check of block tables (no CUDA call), for tables that did not come
 * from the builders above: the forward kernel trusts the tables it is given.  The
 * layout is that of the FlexAttention BlockMask (FlexAttention vs SDPA on M1 Max,
 * qiita kiarina, "役割とデータの流れ"): per q-block row, the PARTIAL and the FULL kv
 * blocks.  All pointers are HOST arrays (copies of the device tables), for
 * `instances` mask instances stored instance-major as fa_create_block_mask_bh
 * writes them (1 for a broadcast mask).
 * Checked per row: 0 <= partial, full <= 65535, partial + full <= nKV; each list's
 * indices in [0, nKV), strictly ascending; no block in both lists; unused entries
 * 0.  Per instance, q_order lists every row exactly once with its two counts, by
 * descending live count, ties by ascending row.
 * Returns FA_OK, or FA_ERR_INVALID_ARG for bad sizes / NULL arrays or tables that
 * break a rule; then, if first_bad is not NULL, *first_bad = instance * nQ + row of
 * the first offending row (-1 for a size or pointer error).
 */
FA_API fa_status fa_block_mask_validate(const int32_t* kv_num_blocks, const int32_t* kv_indices,
                                        const int32_t* full_kv_num_blocks,
                                        const int32_t* full_kv_indices, const int32_t* q_order,
                                        int32_t n_q_blocks, int32_t n_kv_blocks,
                                        int32_t instances, int64_t* first_bad);

/* Bytes of the device workspace fa_flex_attention_fwd needs (a small constant).
 * The caller allocates it, ZEROES IT ONCE, and may then reuse it for every call on
 * one stream; calls that run concurrently must use distinct workspaces. */
FA_API size_t fa_fwd_workspace_bytes(void);

/*
 * Block-sparse attention forward.
 *   q         device (B, H, L, D), dtype `dtype`.
 *   k, v      device (B, H, S, D), dtype `dtype`.
 *   dtype     FA_BF16 or FA_FP16 (Q, K, V and out share it; accumulation is fp32).
 *   B, H, L, S, D   sizes; D in {64, 128}; L == bm->q_len and S == bm->kv_len.
 *             B*H == 0 or L == 0 is a no-op returning FA_OK.
 *   bm        tables from fa_create_block_mask (device arrays stay owned by the caller).
 *   score_kind, softcap   FA_SCORE_NONE, or FA_SCORE_TANH_SOFTCAP with softcap > 0.
 *   scale     multiplier of Q K^T; <= 0 selects 1/sqrt(D).
 *   out       device (B, H, L, D), dtype `dtype`.
 *   lse       device (B, H, L) float32: natural-log softmax denominator
 *             m + ln(sum exp(s - m)); may be NULL.
 *   workspace device buffer of fa_fwd_workspace_bytes() bytes (see there).
 * Alignment (checked on the host; a misaligned pointer returns FA_ERR_INVALID_ARG
 * before any launch): q, k, v, out 16 bytes; bm->q_order and a tabulated mask's
 * bitmap 8 bytes; bm->kv_indices, bm->full_kv_indices, doc_id, lse and workspace 4
 * bytes.
 * The kernel is persistent (one CTA per SM) and processes (batch*head, q-block) work
 * units in the order of bm->q_order.  It trusts the tables' contents: tables that
 * did not come from the builders can be checked first with fa_block_mask_validate.
 * Returns FA_ERR_INVALID_ARG / FA_ERR_UNSUPPORTED (nothing launched) or FA_ERR_CUDA.
 * Device-side timeouts are reported by fa_get_last_device_error.
 */
FA_API fa_status fa_flex_attention_fwd(const void* q, const void* k, const void* v, int32_t dtype,
                                int32_t B, int32_t H, int32_t L, int32_t S, int32_t D,
                                const fa_block_mask* bm, int32_t score_kind, float softcap,
                                float scale, void* out, float* lse, void* workspace,
                                void* stream);

/*
 * Allocation-free variant of fa_create_block_mask + fa_flex_attention_fwd.
 * The pages have no counterpart: this entry point exists for callers that cannot
 * allocate device memory where they call attention -- an operator or plugin host
 * that passes only the input and output tensors (no allocator for the block
 * tables and the workspace the two calls above take from their caller), or a
 * serving loop that reserved its device memory up front, where cudaMalloc could
 * fail and would synchronise the whole device.
 *
 * Arguments are those of fa_create_block_mask (mask_kind, window, doc_id, with
 * block 128 and q_len = L, kv_len = S) and of fa_flex_attention_fwd, without `bm`
 * and `workspace`.  The block tables and the device error word live in one
 * file-scope device array of FA_NOALLOC_SCRATCH_BYTES (4 MiB) per device: the
 * tables take about 8 * nQ * nKV bytes, so square problems fit up to
 * L = S = 723 * 128 = 92544 (L = S = 32768 takes 0.5 MiB).  The call allocates
 * nothing and calls no allocating routine.  Each call clears the error word,
 * builds the tables, runs the forward, and, if `device_error` is not NULL (device
 * or pinned host int32), copies the error word there in stream order: 0 = success,
 * nonzero = a bounded device wait gave up and the outputs are invalid.  B*H == 0 or L == 0 is a no-op
 * returning FA_OK (nothing launched, *device_error untouched).
 *
 * Every call on a device shares that one array: calls whose GPU work may overlap
 * (different streams, or several host threads) race on it and must be ordered by
 * the caller.  The array keeps the last call's contents; each call clears the
 * error word and rebuilds the tables before the forward reads them.
 *
 * Set-up: the first call on a device (and the first after a cudaDeviceReset, which
 * replaces the device's context) looks up the array's device address with that
 * device current; in that lookup the CUDA runtime loads the library's device
 * module, which reserves the array's 4 MiB on the device.  Later calls read the
 * cached address.  Make that first call before any stream capture and outside
 * sections that must not wait on the device; after it, calls reserve nothing.
 * Returns FA_ERR_SCRATCH_TOO_SMALL (nothing launched) when the tables of an
 * (L, S) problem do not fit, the argument errors of the two calls above (nothing
 * launched), or FA_ERR_CUDA.
 */
#define FA_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
FA_API fa_status fa_flex_attention_fwd_noalloc(const void* q, const void* k, const void* v,
                                        int32_t dtype, int32_t B, int32_t H, int32_t L,
                                        int32_t S, int32_t D, int32_t mask_kind,
                                        int32_t window, const int32_t* doc_id,
                                        int32_t score_kind, float softcap, float scale,
                                        void* out, float* lse, int32_t* device_error,
                                        void* stream);

/*
 * Grouped-query attention forward (SDPA tutorial section 5: several query
 * heads share one K/V head, SDPA's enable_gqa).  As fa_flex_attention_fwd, except
 *   k, v      device (B, H_kv, S, D);
 *   H_kv      >= 1 and dividing H: query head h reads K/V head h / (H / H_kv)
 *             (consecutive query heads share a K/V head).
 * H_kv == H is fa_flex_attention_fwd.  Returns FA_ERR_INVALID_ARG (nothing
 * launched) if H_kv does not divide H, else as fa_flex_attention_fwd.
 */
FA_API fa_status fa_flex_attention_fwd_gqa(const void* q, const void* k, const void* v,
                                    int32_t dtype, int32_t B, int32_t H, int32_t H_kv, int32_t L,
                                    int32_t S, int32_t D, const fa_block_mask* bm,
                                    int32_t score_kind, float softcap, float scale, void* out,
                                    float* lse, void* workspace, void* stream);

/*
 * Decode against a KV cache (SDPA tutorial, section 4, pitfall 3): L new
 * queries after S - L cached keys.  Query i sits at key position S - L + i, so the
 * causal mask is aligned to the lower right (torch's causal_lower_right).
 *   q         device (B, H, L, D);   k, v  device (B, H_kv, S, D);  16-byte aligned.
 *   H_kv      >= 1 dividing H (grouped-query attention as in fa_flex_attention_fwd_gqa);
 *             (H / H_kv) * L <= FA_DECODE_MAX_ROWS (the query rows sharing one K/V
 *             head are processed together, reading K and V once).
 *   mask      fa_decode_mask; window W >= 1 for FA_DECODE_SLIDING_WINDOW
 *             (query i sees keys in (S - L + i - W, S - L + i]).
 *   score_kind, softcap, scale, dtype, D as for fa_flex_attention_fwd.
 *   out, lse  device (B, H, L, D) in dtype, 16-byte aligned / (B, H, L) fp32, 4-byte
 *             aligned (lse may be NULL).
 *   workspace device, at least fa_decode_workspace_bytes(B, H, H_kv, L, S, D) bytes,
 *             16-byte aligned; its first word is the device error word (zero it once;
 *             fa_get_last_device_error reads and clears it).  Calls that run
 *             concurrently need distinct workspaces.
 * Split-KV: the keys are cut into chunks processed by different CTAs, then merged.
 * Two kernels on `stream`.  B*H*L == 0 is a no-op.  Returns FA_ERR_INVALID_ARG /
 * FA_ERR_UNSUPPORTED (nothing launched) or FA_ERR_CUDA.
 */
typedef enum {
  FA_DECODE_FULL = 0,            /* every cached key */
  FA_DECODE_CAUSAL = 1,          /* kv_idx <= S - L + q_idx */
  FA_DECODE_SLIDING_WINDOW = 2   /* and S - L + q_idx - kv_idx < window */
} fa_decode_mask;
#define FA_DECODE_MAX_ROWS 32
FA_API size_t fa_decode_workspace_bytes(int32_t B, int32_t H, int32_t H_kv, int32_t L, int32_t S,
                                 int32_t D);
FA_API fa_status fa_flex_attention_decode(const void* q, const void* k, const void* v,
                                   int32_t dtype, int32_t B, int32_t H, int32_t H_kv, int32_t L,
                                   int32_t S, int32_t D, int32_t mask, int32_t window,
                                   int32_t score_kind, float softcap, float scale, void* out,
                                   float* lse, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * Backward pass (FlashAttention-2 article, "あえて再計算して転送を減らす":
 * the attention matrix is recomputed block by block from the inputs and the
 * forward's LSE rather than stored).  Gradients of the forward with the same
 * mask, score_mod and scale:
 *   q, out, dout  device (B, H, L, D);  k, v  device (B, H_kv, S, D);  dtype as forward.
 *   lse       device (B, H, L) fp32 from the forward (natural log; -inf rows get no gradient).
 *   bm        the forward's tables; per-(batch, head) tables (mask_batch 1 or B,
 *             mask_heads 1 or H, else FA_ERR_INVALID_ARG) as in the forward.
 *   q_num_blocks, q_indices, full_q_num_blocks, full_q_indices
 *             the column lists of bm from fa_block_mask_transpose (instance-major for
 *             per-(batch, head) tables, like bm's own arrays).
 *   dq        device (B, H, L, D);  dk, dv  device (B, H_kv, S, D);  in dtype, fully
 *             overwritten (tiles no row or column list reaches are written as zeros).
 *             With H_kv < H, dk and dv of a K/V head are the sums over the H / H_kv
 *             query heads that read it (h / (H / H_kv) == kv head).
 *   workspace device, at least fa_bwd_workspace_bytes(B, H, L) bytes: a 256-byte
 *             header whose first 4 bytes are the device error word, then the row sums
 *             of dO * O.  The caller ZEROES THE HEADER ONCE and may then reuse the
 *             buffer for every call on one stream; the row sums need no initial
 *             contents.  Calls that run concurrently need distinct workspaces.
 * Alignment (checked on the host; a misaligned pointer returns FA_ERR_INVALID_ARG
 * before any launch): q, k, v, out, dout, dq, dk, dv and workspace 16 bytes; lse
 * and every table pointer 4 bytes.  D 64 or 128; B * H * L and B * H_kv * S at most 2^33
 * (else FA_ERR_UNSUPPORTED).  Three kernels on `stream`: row sums of dO * O; dK and dV
 * per 128-key tile over its column lists and the query heads sharing its K/V head;
 * dQ per 128-query tile over its row lists.  Both gradient kernels run the products
 * on the tcgen05 tensor cores with fp32 accumulators in tensor memory; each output
 * tile has one owner (no atomics, deterministic).  Bounded device waits that run out
 * set the error word, which fa_get_last_device_error(workspace, stream) reports as
 * FA_ERR_TIMEOUT.  Returns FA_ERR_INVALID_ARG / FA_ERR_UNSUPPORTED (nothing
 * launched) or FA_ERR_CUDA.
 */
FA_API size_t fa_bwd_workspace_bytes(int32_t B, int32_t H, int32_t L);
FA_API fa_status fa_flex_attention_bwd(const void* q, const void* k, const void* v, const void* out,
                                const void* dout, const float* lse, int32_t dtype, int32_t B,
                                int32_t H, int32_t H_kv, int32_t L, int32_t S, int32_t D,
                                const fa_block_mask* bm, const int32_t* q_num_blocks,
                                const int32_t* q_indices, const int32_t* full_q_num_blocks,
                                const int32_t* full_q_indices, int32_t score_kind, float softcap,
                                float scale, void* dq, void* dk, void* dv, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * Testing hook for failure detection (no counterpart on the pages).  While `on`,
 * the forward kernel's MMA warp issues nothing and the decode and backward kernels
 * load no K/V tile, so the kernels' bounded waits run out after `wait_limit_ns` (0: the
 * default 2 s); each kernel stops, drains what it has in flight, frees TMEM and
 * returns, and fa_get_last_device_error on that call's workspace then reports
 * FA_ERR_TIMEOUT (the outputs of that call are invalid).  Nothing faults, traps or
 * hangs.  Process-wide; off by default.
 */
FA_API void fa_debug_set_mma_stall(int32_t on, uint64_t wait_limit_ns);

/* Synchronises `stream`, then reads and clears the error word that the forward,
 * decode or backward kernels keep at the start of `workspace`.  Returns
 * FA_ERR_TIMEOUT if a bounded device wait gave up since the last query (the outputs
 * of that call are then invalid), FA_ERR_CUDA if the stream reports an error,
 * FA_OK otherwise. */
FA_API fa_status fa_get_last_device_error(void* workspace, void* stream);

/* Static, human-readable name of a status code. */
FA_API const char* fa_status_string(int32_t status);

/* Number of SMs the forward kernel's persistent grid uses on the current device
 * (0 if no device).  Informational. */
FA_API int32_t fa_num_sms(void);

#ifdef __cplusplus
}
#endif

#endif  /* FA_H_ */
