// internal.h -- structures shared by the host runtime and the kernels of libsegkv.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace skv {

// Device error codes written to state[1] (first error wins); values match segkv_status.
constexpr int kErrDeviceBounds = 7;
constexpr int kErrDeviceTimeout = 8;

// Per-call metadata blobs are uploaded into the head of the caller's workspace with one
// host-to-device copy.  The first 64 bytes are scheduler counters that the upload zeroes.
constexpr int kHeaderBytes = 64;

struct AppendSeq {   // one sequence of an append call
  int32_t seq_id, start, count, tok_off;
};

struct PrefillSeq {  // one sequence of a prefill call
  int32_t seq_id, q_start, q_len, q_row0;
  int32_t kv_len, pad0, pad1, pad2;
};

struct DecodeSeq {   // one sequence of a decode call
  int32_t seq_id, q_pos, kv_len, pad;
};

// A work item is two int32 words: w0 = sequence index in the call,
// w1 = (global << 31) | (kv_head << 20) | tile_or_split.
__host__ __device__ inline int item_head(uint32_t w1) { return (int)((w1 >> 20) & 0x7FF); }
__host__ __device__ inline int item_tile(uint32_t w1) { return (int)(w1 & 0xFFFFF); }
__host__ __device__ inline bool item_global(uint32_t w1) { return (w1 >> 31) != 0; }
__host__ __device__ inline uint32_t make_item_w1(bool global, int head, int tile) {
  return ((uint32_t)global << 31) | ((uint32_t)head << 20) | (uint32_t)tile;
}

__host__ __device__ inline int max_i(int a, int b) { return a > b ? a : b; }

// Rank of logical page lp among the pages this call allocates for one (sequence, head),
// in ascending lp (the allocation order), or -1 when lp's slot was allocated before the
// call.  hb = slots the head held before the call.  A global head's slot is lp, so its new
// pages are lp >= hb.  A local head fills ring slots 0, 1, ... in order until it holds R, so
// a slot is new exactly when its index is >= hb; the call touches the last R pages
// [lp0, lp1], whose slots form a cyclic run starting at lp0 mod R.  (Used when the call
// copies no shared page: then "allocated" depends only on the sequence's length, also for a
// fork, which takes its source's length with its page-table rows.)
__host__ __device__ inline int new_page_rank(int lp, int lp0, int hb, bool global, int R) {
  if (global) return lp >= hb ? lp - hb : -1;
  if (lp % R < hb) return -1;
  const int s0 = lp0 % R, m = lp - lp0;  // new slots among lp0 .. lp-1
  if (s0 + m <= R) return max_i(0, s0 + m - max_i(s0, hb));
  return max_i(0, R - max_i(s0, hb)) + max_i(0, s0 + m - R - hb);
}

struct StorageGeom {  // what every kernel needs to resolve a logical position to a page
  int32_t *page_table;
  const int32_t *free_list;
  int32_t *state;
  void *k_pool, *v_pool;
  int num_pages, page, head_dim, hkv, hq, max_seqs, max_lp, ring, window;
  long long wait_limit;  // cycle limit of the kernels' bounded waits (0: about two seconds)
};

// -- launchers (each .cu file exposes one host function per kernel) --------------------
cudaError_t launch_reset(const StorageGeom &g, int num_layers, cudaStream_t st);

// The scatter, with the copy on write of shared pages folded in: plan_dev == NULL when no page
// of the call is shared; else plan_src_dev[i] = the free-list entry of the shared page whose
// rows before the call's first token the page of plan entry i copies first, or -1;
// max_pages = the most pages the call touches for one (sequence, head).
cudaError_t launch_append(const StorageGeom &g, int layer, const void *ws_meta, int nseq, const uint8_t *cls_dev,
                          const int32_t *pair_off_dev, const int32_t *plan_dev, const int32_t *plan_src_dev,
                          int cursor0, int new_pages, int max_pages, const void *k_new, const void *v_new,
                          cudaStream_t st);

// A prefill work item is four int32 words: w0 = sequence index in the call, w1 as above
// (tile = index of the item's pair of query tiles), w2 = (first key tile << 16) | last key
// tile of the item's key range, w3 = partial-result slot (-1: the item covers its whole key
// range and writes out/lse itself; else one chunk of a longer item's key range, whose
// normalised fp32 O and lse go to slot w3 for the combine kernel).
// A combine group is four int32 words: w0 = sequence index, w1 as above, w2 = first slot,
// w3 = number of chunks.
constexpr int kMaxPartSlots = 320;  // partial-result slots of one prefill call (>= 2 x 148 SMs)

struct PrefillLaunch {
  StorageGeom g;
  int layer, nseq, n_items, tile_pos, grid;
  const void *ws_meta;  // header + PrefillSeq[nseq] + items (int4) + combine groups (int4)
  int items_off;        // byte offset of the item array inside ws_meta
  int groups_off, n_groups;
  float *part_o;        // [slot][2 tiles][D / 4][128 rows] float4: each chunk's O, normalised
  float *part_lse;      // [slot][2 tiles][128 rows]: each chunk's lse (-inf: no visible key)
  const void *q;
  void *out;
  float *lse;
  unsigned long long *visited;
  float scale_log2;
  int two_src;  // 1: pages of each sequence's query range come from kcmap / vcmap, not the pool
  // Fused append (store == 1, with two_src): the item whose query range holds a chunk page's
  // first position also stores that page from shared memory into the pool (TMA store) and
  // records it in the page table; a page the call allocates takes free-list entry
  // cursor0 + pair_off[sequence * hkv + head] + new_page_rank.  Block 0 sets state[0] =
  // cursor0 + new_pages.
  int store;
  const int32_t *pair_off;
  int cursor0, new_pages;
  // Test hook: 1 makes the MMA thread first wait on a barrier nothing arrives on, so that its
  // bounded wait runs out and every role takes the abort and drain path.
  int stall_test;
};
// kcmap / vcmap: the two-source call's K/V tensors [tokens, hkv, D] (box 64 x 1 x page);
// unused (any valid map) when two_src == 0.
cudaError_t launch_prefill(const PrefillLaunch &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                           const CUtensorMap &vmap, const CUtensorMap &omap, const CUtensorMap &kcmap,
                           const CUtensorMap &vcmap, cudaStream_t st);
int prefill_smem_bytes(int head_dim);

struct DecodeLaunch {
  StorageGeom g;
  int layer, nseq, n_items, split_pages, max_splits, grid;
  const void *ws_meta;  // header + DecodeSeq[nseq] + nsplit[nseq*hkv] + items
  int nsplit_off, items_off;
  float *part_o, *part_lse;  // [nseq, hq, max_splits, D], [nseq, hq, max_splits]
  const void *q;
  void *out;
  float *lse;
  unsigned long long *visited;
  float scale_log2;
  // Decode step (newk != NULL): before attending, each (sequence, KV head) appends its token
  // at q_pos: newk[b * hkv + h] = free-list entry of a page the token starts (-1: the slot's
  // page is written in place); K/V rows from k_new / v_new [nseq, hkv, D]; block 0 sets the
  // allocation cursor state[0] = cursor_after.
  const int32_t *newk;
  const void *k_new, *v_new;
  int cursor_after;
};
cudaError_t launch_decode(const DecodeLaunch &p, const CUtensorMap &kmap, const CUtensorMap &vmap, cudaStream_t st);
int decode_smem_bytes(int head_dim);

// Attention-as-router scores.  A work item is four int32 words: w0 = sequence index in the
// call, w1 = (global << 31) | (kv_head << 20) | key tile (128 absolute positions), w2 = first
// query tile of the item, w3 = (chunk << 20) | number of query tiles.  Query tile t of key
// tile kt holds tile_pos positions from max(kt * 128, q_start) + t * tile_pos, all G heads.
// Reducing warps of the router kernel per TMEM lane quadrant; each sums 128 / groups of
// the 128 query columns, and each (chunk, column group) has its own partial slot.
constexpr int kRouterColGroups = 4;
struct RouterSeq {
  int32_t seq_id, q_start, q_len, q_row0;
  int32_t kv_len, pad0, pad1, pad2;
};
struct RouterLaunch {
  StorageGeom g;
  int layer, nseq, n_items, tile_pos, g_shift, grid, n_tokens;
  const void *ws_meta;  // header + RouterSeq[nseq] + items (int4)
  int items_off;
  const float *lse;     // [n_tokens, hq] natural-log lse of the queries
  float *part;          // [chunks][column groups][hkv][n_tokens]: received mass per key
  float scale_log2;
};
cudaError_t launch_router(const RouterLaunch &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                          cudaStream_t st);
int router_smem_bytes(int head_dim);

// scores[t] = sum over partial slots and KV heads of part (one thread per token), then the
// top-k per sequence (one CTA per sequence).  topk_meta: int4 per sequence (q_row0, q_len,
// k, first output row).
cudaError_t launch_topk(const float *part, int chunks, int hkv, int n_tokens, const int4 *topk_meta, int nseq,
                        int max_len, float *scores, int32_t *rows_out, cudaStream_t st);

struct RelocateLaunch {
  const int32_t *shift;  // DEVICE [n_tokens]: the position offset of each packed token
  const void *q_in;
  void *q_out;
  int hq, hkv, head_dim, interleaved;
  double theta[64];       // theta_i = base^(-2i/D) for i < D/2, in fp64
  uint32_t cls_bits[32];  // class of QUERY heads 0..1023 (their KV head's): bit set = global (passes unchanged)
};
cudaError_t launch_relocate_q(const RelocateLaunch &p, int n_tokens, cudaStream_t st);

}  // namespace skv
