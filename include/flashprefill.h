/*
 * flashprefill.h -- C ABI of the B200 (sm_100a) block-sparse causal prefill
 * attention library (FlashPrefill style).
 *
 * The method (sources: "FlashPrefill: Near-Zero-Cost Sparsity Discovery for
 * Ultra-Fast Long-Context Prefilling", zhichai.net summary, Method 1-3, and the
 * "FlashPrefill V2: Block-Sparse Prefill Attention for Long-Context LLM Serving"
 * abstract):
 *   1. fp_discover  -- mean-pool Q and K per block of B tokens, score every
 *      causal pair of pooled blocks, keep a block when exp(score - row max) >=
 *      alpha (per query head, union over the KV group's heads), always keep the
 *      sink and local-window blocks; emit a bit mask.
 *   2. fp_compact   -- turn each mask row into a contiguous ascending list of
 *      kept block indices ("index compaction -> physical jumps").
 *   3. fp_sparse_prefill / fp_paged_sparse_prefill -- flash attention with
 *      online softmax that visits only the listed KV blocks; all query heads of
 *      a KV group share each K/V tile (PackGQA); BF16 or FP8-e4m3; contiguous,
 *      varlen (continuous batching) or paged KV.
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller; the library
 *   allocates nothing and keeps no per-call state. Pointers to Q/K/V/O and to
 *   pools must be 16-byte aligned.
 * - Every call is asynchronous on the given CUDA stream (cudaStream_t, passed
 *   as void*; NULL = legacy default stream). Argument errors are returned
 *   before anything is launched. FP_ERR_CUDA reports a launch error.
 *   Device-side checks (bad cu_seqlens, page id or list entry, a pipeline wait
 *   that exceeded its time limit) never trap: they set a device status word
 *   that fp_get_device_status() reads and clears.
 * - Sequences ("requests") r = 0..R-1. Without cu_seqlens the batch is
 *   contiguous: R = batch, every request has max_seqlen tokens, Q is
 *   [R, L, Hq, d] and K/V are [R, L, Hkv, d] (row-major, d innermost). With
 *   cu_seqlens (device int32 [R+1], non-decreasing, cu[0] = 0,
 *   cu[R] = total_tokens) request r owns tokens cu[r] .. cu[r+1]-1 of a packed
 *   Q [total_tokens, Hq, d] (and of K/V [total_tokens, Hkv, d] when not
 *   paged); every length must be <= max_seqlen.
 * - Paged KV (page_table != NULL, requires cu_seqlens): K/V live in pools
 *   [num_pages, page_size, Hkv, d]; token t of request r is slot t % page_size
 *   of pool page page_table[r * max_pages_per_req + t / page_size].
 * - Chunked prefill with a cached prefix (kv_lens != NULL; needs cu_seqlens
 *   and page_table): request r has kv_lens[r] tokens in the paged KV cache and
 *   its queries are its LAST q_len_r = cu[r+1] - cu[r] tokens (positions
 *   p0 = kv_len - q_len .. kv_len - 1; q_len <= kv_len <= max_seqlen). Blocks
 *   are laid on the KV positions; a query block is pooled over the queries it
 *   holds, blocks before p0 get empty lists, and each query attends to kept
 *   keys at positions <= its own. Without kv_lens, kv_len = q_len (full prefill).
 * - Per-query-head selection (head_bits != NULL; G <= 8): fp_discover_compact
 *   also writes, for list entry n of row (r, g, i), the byte head_bits[base +
 *   n] (same offsets as idx) whose bit hh is set iff query head g*G + hh kept
 *   that block by its own threshold or the block is a sink/window block. The
 *   attention calls then still visit the group's list (the union, shared K/V
 *   tiles) but mask, for each query head, the blocks its own bit excludes,
 *   which gives every head exactly its own selection. fp_compact cannot
 *   produce the bits (the mask holds the union) and rejects head_bits.
 * - Block grid: per request, blocks of B = block tokens start at the request's
 *   first token; N_r = ceil(kv_len_r / B); Nmax = ceil(max_seqlen / B). Query
 *   head h uses KV head h / G with G = Hq / Hkv.
 * - Mask layout (uint32): word w of row (r, g, i) is
 *   mask[((r * Hkv + g) * Nmax + i) * Wmax + w], Wmax = ceil(Nmax / 32); bit b
 *   of word w is key block j = 32 w + b. Only j <= i can be set.
 * - List layout (int32): row (r, g, i) starts at
 *   idx[(r * Hkv + g) * Nmax * (Nmax + 1) / 2 + i * (i + 1) / 2] and holds
 *   cnt[(r * Hkv + g) * Nmax + i] strictly ascending block indices (capacity
 *   i + 1). Rows i >= N_r have cnt = 0.
 * - Thresholding happens in float32: keep iff s - rowmax >= ln(alpha), with
 *   s = softmax_scale * (pooled q . pooled k); the dot products are formed on
 *   the tensor cores from three-part bf16 splits of the float32 means, to
 *   float32 accuracy. Blocks whose exact probability lies within ~1e-5
 *   relative of alpha may be decided either way.
 */
#ifndef FLASHPREFILL_H_
#define FLASHPREFILL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FP_OK = 0,
  FP_ERR_INVALID_ARG = -1,  /* null pointer, bad size, alpha < 0 or not finite */
  FP_ERR_UNSUPPORTED = -2,  /* head_dim not 128 (or 64 with bf16), block not 64/128, G = hq / hkv not in
                               1..8 or 16, Nmax > 8192, page size not a power of two in
                               16..65536 */
  FP_ERR_ALIGNMENT = -3,    /* a tensor pointer is not 16-byte aligned */
  FP_ERR_WORKSPACE = -4,    /* workspace missing or smaller than fp_workspace_size */
  FP_ERR_CUDA = -5,         /* a CUDA runtime call or launch failed */
  FP_ERR_DEVICE = -6        /* the device status word is non-zero (see fp_get_device_status) */
} fp_status_t;

typedef enum { FP_BF16 = 0, FP_E4M3 = 1 } fp_dtype_t;

/* Device status bits (fp_get_device_status). */
#define FP_DEV_TIMEOUT 0x1u       /* a pipeline wait exceeded its limit; outputs invalid */
#define FP_DEV_BAD_SEQLENS 0x2u   /* cu_seqlens not monotone / out of range */
#define FP_DEV_BAD_PAGE 0x4u      /* page id outside [0, num_pages) */
#define FP_DEV_BAD_LIST 0x8u      /* list entry outside [0, i] or count > i+1 */

typedef struct {
  fp_dtype_t dtype;        /* element type of Q, K, V (O is always bf16) */
  int batch;               /* contiguous layout: number of sequences; varlen: number of requests R */
  int max_seqlen;          /* contiguous: tokens per sequence; varlen: upper bound on every length */
  int hq, hkv;             /* query heads, KV heads; hq % hkv == 0 */
  int head_dim;            /* 128, or 64 with bf16 inputs */
  int block;               /* B: 64 or 128 tokens */
  float alpha;             /* dynamic-threshold factor, finite and >= 0 */
  int sink_tokens;         /* leading tokens always kept: ceil(sink_tokens / B) blocks */
  int window_tokens;       /* local window: max(1, ceil(window_tokens / B)) blocks ending at the diagonal */
  float softmax_scale;     /* 0 -> 1 / sqrt(head_dim); used for scores and attention */
  const float* q_scale;    /* FP8 only: device float [hq], dequantisation scale per query head */
  const float* k_scale;    /* FP8 only: device float [hkv] */
  const float* v_scale;    /* FP8 only: device float [hkv] */
  const int32_t* cu_seqlens;  /* device int32 [batch + 1] or NULL (contiguous batch) */
  int total_tokens;           /* varlen: cu_seqlens[batch] (rows of the packed Q) */
  const int32_t* page_table;  /* device int32 [batch, max_pages_per_req] or NULL */
  int page_size;              /* paged: tokens per page (power of two, 16..65536) */
  int max_pages_per_req;
  int num_pages;              /* paged: pages in each pool */
  const int32_t* kv_lens;     /* chunked prefill: device int32 [batch] or NULL (see below) */
  uint8_t* head_bits;         /* per-head selection: device uint8 [fp_list_capacity(p)] or NULL (see below) */
} fp_params_t;

/* Bytes of device scratch fp_discover needs: the pooled Q and K, each pooled
 * float32 value stored as three bf16 parts (hi + mid + lo), plus what
 * fp_prefill adds: a work-queue counter (256 bytes) and the attention's claim
 * order (one int per work unit). */
size_t fp_workspace_size(const fp_params_t* p);
/* Number of uint32 words of the block mask: R * Hkv * Nmax * ceil(Nmax / 32). */
size_t fp_mask_words(const fp_params_t* p);
/* Number of int32 entries of the index lists: R * Hkv * Nmax * (Nmax + 1) / 2. */
size_t fp_list_capacity(const fp_params_t* p);
/* Number of int32 row counts: R * Hkv * Nmax. */
size_t fp_count_entries(const fp_params_t* p);

/*
 * Block pattern discovery (Method 1 "Instantaneous Pattern Discovery" and
 * Method 2 "Dynamic Threshold Pruning" of the FlashPrefill summary).
 * q: Q (bf16 or e4m3 per p->dtype, layout above); k: K, or the K pool when
 * p->page_table is set. mask: device uint32 [fp_mask_words(p)], fully
 * written (rows i >= N_r are zero). workspace: device scratch of
 * ws_bytes >= fp_workspace_size(p), 256-byte aligned; contents are
 * overwritten.
 */
fp_status_t fp_discover(const fp_params_t* p, const void* q, const void* k, uint32_t* mask,
                        void* workspace, size_t ws_bytes, void* stream);

/*
 * Index compaction (Method 3 "Index Compaction -> Physical Jumps"): mask ->
 * ascending lists. idx: device int32 [fp_list_capacity(p)]; cnt: device int32
 * [fp_count_entries(p)], fully written.
 */
fp_status_t fp_compact(const fp_params_t* p, const uint32_t* mask, int32_t* idx, int32_t* cnt,
                       void* stream);

/*
 * Discovery and compaction in one pass over the pooled scores: same outputs as
 * fp_discover followed by fp_compact (mask may be NULL to skip writing it).
 */
fp_status_t fp_discover_compact(const fp_params_t* p, const void* q, const void* k,
                                uint32_t* mask, int32_t* idx, int32_t* cnt, void* workspace,
                                size_t ws_bytes, void* stream);

/*
 * Block-sparse flash attention over the compacted lists ("FlashPrefill V2"
 * abstract: PackGQA, warp specialisation, ping-pong pipelining, FP8).
 * For each request r, query token t and head h:
 *   O[t, h] = sum_k softmax_k(scale * q_t,h . k_k) v_k over the keys k <= t of
 *   the blocks listed in row (r, h / G, t / B).
 * q, k, v: contiguous or varlen layout (no page table; p->page_table must be
 * NULL). o: device bf16, same layout as q. lse: NULL or device float
 * [hq, R * max_seqlen] (contiguous) / [hq, total_tokens] (varlen), natural-log
 * sum of exponentials of the scaled logits. S = Q K^T runs on the input type
 * (bf16, or e4m3 with float32 accumulation); the softmax weights P and V enter
 * O += P V as 16-bit values: bf16 for bf16 inputs, f16 for e4m3 inputs (V is
 * widened exactly from e4m3 to f16 on chip). O is normalised by the sum of the
 * rounded weights the PV product uses, and lse is the log of that same sum
 * (within 2^-8 relative of the exact sum for bf16, 2^-11 for f16). Rows
 * with cnt = 0 get O = 0 and lse = -inf. Output rows of tokens outside every
 * request are not written.
 */
fp_status_t fp_sparse_prefill(const fp_params_t* p, const void* q, const void* k, const void* v,
                              const int32_t* idx, const int32_t* cnt, void* o, float* lse,
                              void* stream);

/* As fp_sparse_prefill, with K/V read through p->page_table from the pools. */
fp_status_t fp_paged_sparse_prefill(const fp_params_t* p, const void* q, const void* k_pool,
                                    const void* v_pool, const int32_t* idx, const int32_t* cnt,
                                    void* o, float* lse, void* stream);

/*
 * The whole path in one call: discovery + compaction (as fp_discover_compact,
 * mask may be NULL) followed by the block-sparse attention (as
 * fp_sparse_prefill, or fp_paged_sparse_prefill when p->page_table is set;
 * k and v are then the pools). Between the two a one-CTA kernel sorts the
 * attention's work units (request, KV group, query block, M-tile pair) by
 * their list length, longest first; the attention is launched as a
 * programmatic dependent of it, so its prologue overlaps the sort, and claims
 * the units in that order from a device queue in the workspace instead of a
 * static stride. idx and cnt are required. workspace: fp_workspace_size(p)
 * bytes as for fp_discover. Outputs are identical to the three separate calls.
 */
fp_status_t fp_prefill(const fp_params_t* p, const void* q, const void* k, const void* v, uint32_t* mask,
                       int32_t* idx, int32_t* cnt, void* o, float* lse, void* workspace, size_t ws_bytes,
                       void* stream);

/*
 * Discovery and compaction without a caller-provided workspace: the same
 * kernels and outputs as fp_discover_compact, with the pooled-Q/K scratch
 * taken from a fixed device array inside the library. The paper has no
 * counterpart; this exists for callers that cannot allocate device memory,
 * such as a plugin inside a host engine that owns all device memory and
 * exposes no allocator, or a path that must not call cudaMalloc because it
 * can synchronise the device. It allocates nothing.
 * - Limit: fp_workspace_size(p) must not exceed fp_static_scratch_bytes()
 *   (32 MiB, enough for one 128K-token sequence with 32 query / 4 KV heads at
 *   block 128); larger problems return FP_ERR_WORKSPACE before any launch and
 *   fp_last_error() says how much was needed. The limit is checked against
 *   the whole fp_workspace_size, which also counts the attention's queue
 *   area that discovery does not use, so it errs on the safe side.
 * - The array exists on every GPU that loads the library, until exit. The
 *   first call on a device looks up the array's device address on that
 *   device (the device must be current) and keeps it for the life of the
 *   process; make that first call before any stream capture. A
 *   cudaDeviceReset() of that device invalidates the kept address: calling
 *   this entry point (or fp_get_device_status, which keeps the status word's
 *   address the same way) on a device after resetting it is not supported.
 * - All calls share the one array and it keeps the last call's contents
 *   (nothing in it needs to start at zero). Calls whose work overlaps on the
 *   GPU (e.g. on two streams at once) race on it: serialise them.
 */
fp_status_t fp_discover_compact_static(const fp_params_t* p, const void* q, const void* k,
                                       uint32_t* mask, int32_t* idx, int32_t* cnt, void* stream);

/* Size in bytes of the fixed scratch array fp_discover_compact_static uses. */
size_t fp_static_scratch_bytes(void);

/*
 * Synchronises `stream`, writes the device status bits (FP_DEV_*) of the
 * current device to *bits (may be NULL) and clears them. Returns FP_OK if no
 * bit was set, FP_ERR_DEVICE otherwise, FP_ERR_CUDA on a runtime error.
 */
fp_status_t fp_get_device_status(uint32_t* bits, void* stream);

/* Description of the CUDA call behind the calling thread's most recent
 * FP_ERR_CUDA (thread-local, valid until the next failing call; "" if none). */
const char* fp_last_error(void);

/* Static, human-readable name of a status code. */
const char* fp_status_string(fp_status_t s);

#ifdef __cplusplus
}
#endif

#endif /* FLASHPREFILL_H_ */
