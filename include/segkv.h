/*
 * segkv.h -- C ABI of libsegkv.so: head-wise segmented paged KV storage and attention
 * for NVIDIA B200 (sm_100a).
 *
 * The method ("RedKnot"): every (layer, KV head) owns its own paged KV storage holding
 * only the tokens that head needs.  A few "global" heads keep the full causal context;
 * the "local" majority keep a sliding window of W tokens (zhichai.net news item "What
 * Happened", items 1 and 3; hysenlabs.com write-up "The Three Core Mechanisms in
 * Detail", third mechanism: pages and their visibility organised per head and per
 * segment).  One variable-length attention pass serves every head over its own pages;
 * no attention mask is ever built.
 *
 * Conventions shared by every entry point
 *   - Positions are 0-based absolute token positions inside a sequence.
 *   - G = num_q_heads / num_kv_heads; query head h reads KV head h / G.
 *   - Visibility of a query at position p: global head  k <= p;
 *                                          local head   p - W < k <= p  (W keys, self included).
 *   - softmax_scale <= 0 selects 1/sqrt(head_dim).  lse = ln(sum over visible k of
 *     exp(softmax_scale * q.k)), fp32.
 *   - bf16 tensors are passed as void* to raw device memory, row-major, contiguous.
 *   - Streams are cudaStream_t values passed as void* (NULL = legacy default stream).
 *     Every call only enqueues work on that stream; nothing blocks except
 *     segkv_device_status.
 *   - Ownership: the caller owns every device buffer (pools, page table, free list,
 *     state, workspace, inputs, outputs).  The library owns the host handle, a host
 *     copy of the head classes, pinned staging for per-call metadata and CUDA events.
 *     It never calls cudaMalloc.
 *   - Errors: every int-returning call returns a segkv_status.  On a non-OK return
 *     nothing was enqueued and no state changed.  Device-side bounds or timeout
 *     violations set an error word instead (read it with segkv_device_status); kernels
 *     never trap.
 *   - A handle is not thread-safe.  Calls on one handle must be issued from one host
 *     thread, in stream order.
 *   - Tracing, read from the environment at the first call: SEGKV_LOG=1 writes one line to
 *     stderr for every call that returns an error, SEGKV_LOG=2 one line for every call
 *     (entry point, status, host time); SEGKV_NVTX=1 wraps every call in an NVTX range
 *     named after the entry point.  The entry points traced are those that can fail:
 *     create, reset, fork, append, the prefill, decode, router and relocation calls,
 *     segkv_device_status and segkv_debug_set.
 */
#ifndef SEGKV_H_
#define SEGKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct segkv segkv_t; /* opaque host handle */

typedef enum {
  SEGKV_OK = 0,
  SEGKV_ERR_INVALID_ARG = 1,    /* bad pointer, size, position or length */
  SEGKV_ERR_UNSUPPORTED = 2,    /* shape outside what the kernels implement */
  SEGKV_ERR_OUT_OF_PAGES = 3,   /* the free list would run out */
  SEGKV_ERR_RING_TOO_SMALL = 4, /* a local head's ring no longer holds a needed key */
  SEGKV_ERR_WORKSPACE = 5,      /* workspace too small or misaligned */
  SEGKV_ERR_CUDA = 6,           /* a CUDA runtime/driver call failed */
  SEGKV_ERR_DEVICE_BOUNDS = 7,  /* (device) page id outside the pool, or unallocated */
  SEGKV_ERR_DEVICE_TIMEOUT = 8  /* (device) a bounded pipeline wait gave up */
} segkv_status;

typedef struct {
  int num_layers;
  int num_q_heads;
  int num_kv_heads;   /* num_q_heads % num_kv_heads == 0; G = Hq/Hkv in {1,2,4,8,16,32,64,128} */
  int head_dim;       /* 64 or 128 */
  int page_size;      /* tokens per page: 16, 32 or 64 */
  int window;         /* W >= 1, keys a local head sees (self included) */
  int ring_pages;     /* R: pages of a local head's ring; 0 selects
                         min(ceil(max_seq_len/P), ceil((W + max_chunk - 1)/P) + 1) */
  int max_seqs;       /* sequence slots; seq ids are 0..max_seqs-1 */
  int max_seq_len;    /* longest sequence, tokens */
  int max_chunk;      /* longest query range of one prefill call (used for the default R) */
  const uint8_t *head_class; /* HOST [num_layers * num_kv_heads], 1 = global, 0 = local; copied */
  int num_pages;      /* N: physical pages in each pool */
  void *k_pool;       /* DEVICE bf16 [N, page_size, head_dim]; 16-byte aligned */
  void *v_pool;       /* DEVICE bf16 [N, page_size, head_dim]; 16-byte aligned */
  int32_t *page_table;       /* DEVICE int32 [num_layers, max_seqs, num_kv_heads, max_lp],
                                max_lp = ceil(max_seq_len / page_size); all -1 initially */
  const int32_t *free_list;  /* DEVICE int32 [N]: the order in which physical pages are handed out
                                (normally a permutation of 0..N-1) */
  int32_t *state;            /* DEVICE int32 [4]: [0] pages handed out, [1] error word; zero initially */
} segkv_config;

/* Validates the configuration and creates a handle.  Touches no GPU memory.
 * Returns INVALID_ARG / UNSUPPORTED for bad shapes. */
int segkv_create(const segkv_config *cfg, segkv_t **out);

/* Frees the host handle and its pinned staging.  Device buffers stay the caller's. */
void segkv_destroy(segkv_t *h);

/* Effective ring size R and page-table row length max_lp of a handle. */
int segkv_ring_pages(const segkv_t *h);
int segkv_max_lp(const segkv_t *h);

/* Tokens appended so far to (layer, seq) -- the host's view, updated at enqueue time. */
int segkv_seq_len(const segkv_t *h, int layer, int seq);

/* Pages handed out so far (host's view of state[0]). */
int segkv_pages_used(const segkv_t *h);

/* Bytes of device workspace any call with at most max_batch sequences and at most
 * max_tokens packed tokens needs.  Workspace must be 256-byte aligned; calls on the
 * same stream may share one workspace.  It includes a fixed area of 320 x 256 x
 * (head_dim + 1) x 4 bytes (about 42 MB at head_dim 128) for the partial results of
 * prefill items cut into key-range chunks (see segkv_prefill_attn). */
size_t segkv_workspace_bytes(const segkv_t *h, int max_batch, int max_tokens);

/* Empties every sequence: page table <- -1, state <- 0 (device, enqueued), lengths <- 0 (host). */
int segkv_reset(segkv_t *h, void *stream);

/*
 * Fork (hysenlabs.com write-up, "Experimental Features and Current Limitations": a shared KV
 * manager with forks and copy-on-write append): the empty sequence dst_seq takes src_seq's
 * page-table rows and length in every layer, so the two share those pages (reference
 * counted in the handle).  A later append to either one that touches a shared page first
 * gives that sequence a private copy (see segkv_append), so neither sees the other's new
 * tokens.  Enqueues one device-to-device copy of the page-table rows per layer.
 * Errors: INVALID_ARG (ids out of range, src == dst, dst not empty in some layer), CUDA.
 */
int segkv_fork(segkv_t *h, int src_seq, int dst_seq, void *stream);

/*
 * Appends tokens [start_pos[b], start_pos[b] + num_new[b]) of sequence seq_ids[b] to every
 * KV head of `layer`: the per-head page tables grow and the K/V rows are scattered into the
 * pages (zhichai.net news item "What Happened", item 3: per-(layer, head) segmented paged
 * storage).  start_pos[b] must equal segkv_seq_len(h, layer, seq_ids[b]); seq ids
 * in one call are distinct.  k_new / v_new: DEVICE bf16 [sum(num_new), Hkv, D],
 * sequences packed in call order.
 *   Page rule: every slot touched that is unallocated, or whose page another sequence
 *   shares after a fork, takes the next id of the free list, in the order (sequence in call
 *   order, KV head ascending, logical page ascending); a shared page's rows before the
 *   call's first token are copied into the new page (copy on write).  A global
 *   head stores logical page lp in slot lp; a local head in slot lp mod R and keeps only
 *   the last R logical pages ending at the call's last token (older tokens of the call
 *   are skipped: the ring would overwrite them).  The unwritten rows of a page the call
 *   starts are zeroed.
 *   Host arrays: seq_ids, start_pos, num_new [nseq].
 *   Errors: INVALID_ARG (continuity, range, duplicate ids), OUT_OF_PAGES, WORKSPACE.
 */
int segkv_append(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *start_pos,
                 const int32_t *num_new, const void *k_new, const void *v_new, void *ws, size_t ws_bytes,
                 void *stream);

/*
 * Causal variable-length prefill over the segmented storage (zhichai.net news item "What
 * Happened", item 3: one fused variable-length attention pass over every head's own
 * pages): for every query row and its query head,
 *   out = sum_visible softmax(scale * q.k) v   (bf16, RNE),  lse (fp32, natural log),
 *   visited[b, hq] += number of visible (q,k) pairs (u64, may be NULL).
 * Queries of sequence seq_ids[b] sit at positions [q_start_pos[b], q_start_pos[b] + q_len[b])
 * and every one of them must already be appended (q_start_pos + q_len <= seq len).
 * q, out: DEVICE bf16 [sum(q_len), Hq, D] packed in call order; lse: DEVICE fp32
 * [sum(q_len), Hq].  Host arrays: seq_ids, q_start_pos, q_len [nseq].
 * Scheduling: items (a pair of query tiles of one KV head) run longest first on one
 * persistent CTA per SM.  When the longest item exceeds the per-SM share of the call's
 * key tiles (a global head's item against short local ones), such items are cut into
 * chunks of consecutive key tiles (at least 8 tiles, at most 32 chunks an item); each
 * chunk writes its normalised fp32 O and lse to the workspace and a combine kernel
 * merges them (lse = log sum exp of the chunks' lse).  Results do not depend on the
 * schedule beyond rounding.
 * Errors: INVALID_ARG, RING_TOO_SMALL (a local head's ring dropped a key some query
 * needs), WORKSPACE, CUDA.
 */
int segkv_prefill_attn(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start_pos,
                       const int32_t *q_len, const void *q, float softmax_scale, void *out, float *lse,
                       uint64_t *visited, void *ws, size_t ws_bytes, void *stream);

/*
 * Fused append + prefill: the result of segkv_append (start_pos = q_start_pos, num_new =
 * q_len, K/V = k_new / v_new) followed by segkv_prefill_attn over the appended range, in one
 * kernel.  The keys of the range come from k_new / v_new as in segkv_prefill_attn_2src; once a
 * page of them has landed in shared memory, the work item whose query range holds the page's
 * first position also writes it to its pool page (a TMA store from shared memory) and records
 * it in the page table, so the append costs no kernel of its own (per-head storage grown as
 * it is attended: zhichai.net news item "What Happened", item 3).  Page tables, the cursor,
 * lengths, out, lse and visited equal those of the two calls; rows of a sequence's last page
 * past its last token hold finite values (the next packed sequence's rows, or zeros) where
 * segkv_append writes zeros -- no attention ever reads them unmasked.  Requires
 * q_start_pos[b] == segkv_seq_len(h, layer, seq_ids[b]), a multiple of the page size, and
 * (local heads) that the ring still holds every key the range's queries need after the
 * append (the condition of segkv_prefill_attn).  While a page is shared after a fork the call
 * runs as segkv_append then segkv_prefill_attn.
 * Errors: INVALID_ARG, RING_TOO_SMALL, OUT_OF_PAGES (nothing changed), WORKSPACE, CUDA.
 */
int segkv_prefill_append(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start_pos,
                         const int32_t *q_len, const void *q, const void *k_new, const void *v_new,
                         float softmax_scale, void *out, float *lse, uint64_t *visited, void *ws, size_t ws_bytes,
                         void *stream);

/*
 * Two-source prefill: the same attention as segkv_prefill_attn for a chunk that is NOT yet
 * appended.  The keys of each sequence's query range come from k_chunk / v_chunk (DEVICE
 * bf16 [sum(q_len), Hkv, D], packed like q); only the context before the range is read from
 * the pages.  A local head's ring then needs to hold just the W - 1 tokens before the chunk,
 * R = ceil((W - 1) / P) + 1 pages, whatever the chunk length (zhichai.net news item "What
 * Happened", item 3: storage holds only the tokens each head needs).  Append the chunk with
 * segkv_append afterwards; results equal appending first and calling segkv_prefill_attn,
 * bit for bit.  Requires q_start_pos[b] == segkv_seq_len(h, layer, seq_ids[b]), a multiple
 * of the page size.
 * Errors: INVALID_ARG (range not at the sequence's end or not page-aligned, pointers),
 * RING_TOO_SMALL, WORKSPACE, CUDA.
 */
int segkv_prefill_attn_2src(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start_pos,
                            const int32_t *q_len, const void *q, const void *k_chunk, const void *v_chunk,
                            float softmax_scale, void *out, float *lse, uint64_t *visited, void *ws,
                            size_t ws_bytes, void *stream);

/*
 * Longest-processing-time-first work list of the prefill call, before any item is cut into
 * key chunks (host only, no GPU).
 * Item = (b, kv head, query tile, cost); a query tile holds tile_pos = 256 / G consecutive
 * positions of all G query heads of the KV head; cost = number of key_tile-aligned key
 * tiles meeting [lo, q_last] (lo = 0 global, max(0, q_first - W + 1) local); order: cost
 * descending, item index ascending.  items_out: HOST int32 [cap][4].  *n_items receives
 * the count (also when cap is too small, which returns WORKSPACE).
 */
int segkv_plan_prefill(const segkv_t *h, int layer, int nseq, const int32_t *q_start_pos, const int32_t *q_len,
                       int32_t *items_out, int64_t cap, int64_t *n_items, int *tile_pos, int *key_tile);

/*
 * Decode: one query per sequence at position q_pos[b] (already appended), split-K over
 * the head's visible pages plus a log-sum-exp combine.
 * q, out: DEVICE bf16 [nseq, Hq, D]; lse DEVICE fp32 [nseq, Hq]; visited as for prefill.
 * num_splits: 0 = automatic, else the largest number of splits any head is cut into.
 */
int segkv_decode_attn(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_pos,
                      const void *q, float softmax_scale, int num_splits, void *out, float *lse, uint64_t *visited,
                      void *ws, size_t ws_bytes, void *stream);

/*
 * Decode step: appends one token to every sequence and decodes its query, in one pass.
 * For each b the token sits at position pos = segkv_seq_len(h, layer, seq_ids[b]); its K/V
 * rows are k_new / v_new[b] (DEVICE bf16 [nseq, Hkv, D]) and its query q[b] (DEVICE bf16
 * [nseq, Hq, D]).  Results, page tables and the allocation cursor equal those of
 * segkv_append (num_new = 1, start_pos = pos) followed by segkv_decode_attn (q_pos = pos),
 * bit for bit; lengths grow by one.  The append is folded into the decode kernel: the work
 * item that holds a head's last page writes the token's rows (and a page it starts) before
 * reading that page, so the step needs no append kernel and no second metadata upload
 * (the per-head storage it grows: zhichai.net news item "What Happened", item 3).
 * While a page is shared after a fork (segkv_fork), the step runs as the two calls above
 * (the append's copy on write first); an error of the second call then leaves the token
 * appended.
 * Errors: INVALID_ARG (a sequence at max_seq_len, bad pointers), RING_TOO_SMALL,
 * OUT_OF_PAGES (nothing changed), WORKSPACE, UNSUPPORTED (G > 16), CUDA.
 */
int segkv_decode_step(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const void *k_new, const void *v_new,
                      const void *q, float softmax_scale, int num_splits, void *out, float *lse, uint64_t *visited,
                      void *ws, size_t ws_bytes, void *stream);

/*
 * Attention as a router (zhichai.net news item "What Happened", item 2: the dense FFN runs
 * only on the top-k tokens by attention score, the rest take an identity path; hysenlabs.com
 * write-up, "The Three Core Mechanisms in Detail", second mechanism: token-level importance
 * scores).  The pages leave the score undefined; here a token's score is the attention mass
 * it receives from the call's queries:
 *   scores[j] = sum over query heads h and queries i of the call that see token j of
 *               exp(scale * q_{i,h} . k_j - lse_{i,h})        (fp32, >= 0),
 * for every token j of the call's query range (the FFN rows being routed); lse is the
 * output of segkv_prefill_attn for the same queries (DEVICE fp32 [sum(q_len), Hq]), q the
 * same queries (DEVICE bf16 [sum(q_len), Hq, D]).  scores: DEVICE fp32 [sum(q_len)], packed
 * like q.  Then, per sequence, the k[b] (HOST int32 [nseq], 0 <= k[b] <= q_len[b]) highest
 * scores, equal scores by lower position first: rows_out (DEVICE int32 [sum(k)]) receives
 * their packed rows, ascending within a sequence, sequences in call order.  The scores do
 * not depend on the schedule (each key's partial sums have their own slot and are added in
 * a fixed order).  Requires G = Hq / Hkv a power of two <= 16.
 * Errors: INVALID_ARG (ranges, k out of range, alignment), RING_TOO_SMALL (a scored token
 * is no longer stored in a local head), WORKSPACE, UNSUPPORTED, CUDA.
 */
int segkv_router_topk(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start_pos,
                      const int32_t *q_len, const void *q, const float *lse, float softmax_scale, const int32_t *k,
                      float *scores, int32_t *rows_out, void *ws, size_t ws_bytes, void *stream);

/*
 * Decode with no caller workspace and no allocation.  The pages have no counterpart to
 * this entry point; it exists for callers that cannot give the library device memory:
 * a serving engine that reserved the whole device for its own allocator at start-up, or
 * code running under a fixed memory budget where a cudaMalloc would fail or is not
 * allowed.  Arguments, results and errors are those of segkv_decode_attn, minus ws.
 *   Scratch: the split partials, the work list and the scheduler counter live in one
 *   fixed array of 64 MiB inside libsegkv.so (every GPU that loads the library holds it
 *   until the process exits); per-call metadata is staged in a fixed 1 MiB host buffer.
 *   A call that would need more returns SEGKV_ERR_WORKSPACE and names the sizes in
 *   segkv_last_error.  Nothing is allocated: no cudaMalloc, cudaFree or cudaHostAlloc.
 *   Set-up: segkv_create looks up the array's device address on the device current at
 *   that moment, which makes the 64 MiB resident there; create the handle before handing
 *   the rest of the device to another allocator.  A call on a device that no segkv_create
 *   saw does the look-up itself (once per device); make that first call before any stream
 *   capture.
 *   Every call shares the one array and the scheduler counter is re-zeroed by each call's
 *   metadata copy, so calls that overlap on the GPU (different streams, or different
 *   handles) race and give wrong results: issue them one after another on one stream.
 *   The host metadata buffer and the duplicate-id check's bitmap are shared by every
 *   handle of the process as well: calls from different host threads race there too, even
 *   on different handles.  Not thread-safe.
 */
int segkv_decode_attn_noalloc(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_pos,
                              const void *q, float softmax_scale, int num_splits, void *out, float *lse,
                              uint64_t *visited, void *stream);

/*
 * Query relocation for position-independent reuse of local-head KV ("RedKnot-MLA: Multi-
 * Head Offline-Online Reuse for DeepSeek-V4 Long-Context Serving", Summary: documents are
 * prefilled offline at canonical position zero; at serving time the queries are rotated by
 * the negative position offset).  For every packed token t, the query heads of `layer`'s
 * local KV heads are turned by the rotary angle of position -shift[t]: dimension pairs
 * (i, i + D/2) (interleaved = 0) or (2i, 2i + 1) (interleaved = 1) rotate by
 * -shift[t] * theta_base^(-2i/D).  A query rotated to its true position p and relocated by
 * delta then scores against a key stored at canonical position j as against that key at
 * j + delta (rotary scores depend only on position differences).  Query heads of global
 * KV heads are copied unchanged.
 *   q_in, q_out: DEVICE bf16 [n_tokens, Hq, D] (the same pointer relocates in place);
 *   shift: DEVICE int32 [n_tokens].  Angles are formed and reduced modulo 2 pi in fp64,
 *   the rotation is done in fp32 and rounded to bf16 (nearest even).
 * Errors: INVALID_ARG (pointers, alignment, theta_base <= 1, interleaved not 0/1),
 * UNSUPPORTED (more than 1024 query heads), CUDA.
 */
int segkv_relocate_q(segkv_t *h, int layer, int n_tokens, const int32_t *shift, const void *q_in, void *q_out,
                     float theta_base, int interleaved, void *stream);

/* Synchronizes `stream`, reads the device error word, clears it and returns it
 * (SEGKV_OK, SEGKV_ERR_DEVICE_BOUNDS or SEGKV_ERR_DEVICE_TIMEOUT), or SEGKV_ERR_CUDA. */
int segkv_device_status(segkv_t *h, void *stream);

/* What the last SEGKV_ERR_CUDA of this handle came from (the failing step and the CUDA
 * error name), or "" if none.  The string belongs to the handle. */
const char *segkv_last_error(const segkv_t *h);

/* Static description of a status code. */
const char *segkv_strerror(int status);

/* Test hooks.  The pages describe no such control; these exist so that the failure paths
 * and the scheduler's order independence can be exercised without faulting a GPU.
 *   SEGKV_DEBUG_WAIT_LIMIT: cycle limit of the bounded pipeline waits of every later launch
 *     of this handle (value >= 0; 0 restores the default of about two seconds).  A wait that
 *     runs out sets SEGKV_ERR_DEVICE_TIMEOUT in the error word; the kernel then lets its
 *     copies and MMAs in flight finish, frees its tensor memory and returns.
 *   SEGKV_DEBUG_STALL_NEXT_PREFILL: value 1 makes the next prefill launch of this handle wait
 *     first on a barrier that nothing arrives on, so that the wait runs out (one shot; the
 *     call's outputs are then undefined and segkv_device_status reports the timeout).
 *   SEGKV_DEBUG_PREFILL_ORDER: 0 runs a prefill call's work list longest first (the
 *     default); 1 runs it in reverse; any other value shuffles it with that seed.  Every item
 *     is computed by one CTA in a fixed key order, so outputs do not depend on it.
 * Returns INVALID_ARG for a null handle, an unknown key or a value out of range.  Not
 * thread-safe, like every call on a handle. */
enum {
  SEGKV_DEBUG_WAIT_LIMIT = 1,
  SEGKV_DEBUG_STALL_NEXT_PREFILL = 2,
  SEGKV_DEBUG_PREFILL_ORDER = 3
};
int segkv_debug_set(segkv_t *h, int key, long long value);

#ifdef __cplusplus
}
#endif

#endif /* SEGKV_H_ */
