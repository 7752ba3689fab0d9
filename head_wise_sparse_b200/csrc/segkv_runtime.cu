// segkv_runtime.cu -- host runtime of libsegkv: the C ABI declared in include/segkv.h.
//
// The runtime validates every call before anything is enqueued, keeps the host's view of
// sequence lengths and pages handed out (enough to reject a call that would overrun the
// free list or read a key a local head's ring already dropped), builds the per-call
// metadata (sequence table, longest-processing-time-first work list), uploads it with one
// host-to-device copy from pinned staging into the caller's workspace, and launches the
// kernels.  It never allocates device memory.
#include <cudaTypedefs.h>

#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <chrono>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <random>
#include <cstring>
#include <new>
#include <string>
#include <utility>
#include <vector>

#include "../../include/segkv.h"
#include "internal.h"

using namespace skv;

namespace {

constexpr int kPrefillTileRows = 128;  // rows of one prefill query tile (G heads x 128/G positions)
constexpr int kPrefillItemRows = 256;  // rows of one prefill work item (two query tiles)
constexpr int kPrefillKeyTile = 128;   // keys of a prefill key tile
constexpr int kDecodeStageKeys = 64;   // keys of a decode pipeline stage
constexpr int kMaxSplits = 32;         // most splits one decode head is cut into
constexpr int kRouterKeys = 128;       // keys of a router key tile
constexpr int kRouterMaxChunks = 8;    // most chunks one router key tile is cut into
constexpr int kStagingSlots = 4;
constexpr int kMaxChunks = 32;         // most chunks one prefill item is cut into

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int ceil_div(int a, int b) { return (a + b - 1) / b; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D bf16 tensor map, 128-byte swizzle, inner box of 64 elements (128 bytes).
bool make_map(CUtensorMap *m, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
              uint64_t stride2_bytes, uint32_t box1, uint32_t box2) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {64, box1, box2};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Staging {
  void *host = nullptr;
  size_t cap = 0;
  cudaEvent_t ev = nullptr;
  bool pending = false;
};

}  // namespace

struct segkv {
  segkv_config cfg;
  std::vector<uint8_t> cls;  // [layers * hkv]
  std::vector<int32_t> len;  // [layers * max_seqs]
  // Host mirror of the page table in free-list-index space: which free-list entry each
  // (layer, seq, head, slot) holds (-1: none), and how many slots hold each entry.  It lets
  // the host plan every allocation, including the copies on write after a fork.
  std::vector<int32_t> slot_k;  // [layers * max_seqs * hkv * max_lp]
  std::vector<int32_t> ref;     // [num_pages]
  std::vector<int32_t> ref_scratch;  // [num_pages]: a call's pending reference-count changes, 0 between calls
  long long n_shared = 0;       // entries with ref >= 2: while 0, no append copies a page
  int ring = 0, max_lp = 0, G = 0;
  long long pages_used = 0;
  Staging slot[kStagingSlots];
  int next_slot = 0;
  bool maps_ready = false;
  CUtensorMap kmap, vmap;
  int num_sms = 0;
  std::string last_error;  // which CUDA step failed last, and why
  // test hooks (segkv_debug_set): the kernels' wait limit in cycles (0: default), a one-shot
  // stall of the next prefill launch, and the order in which a prefill call's work list runs
  long long wait_limit = 0;
  int stall_next_prefill = 0;
  long long lpt_order = 0;
};

namespace {

int cuda_fail(segkv_t *h, const char *what, cudaError_t e) {
  h->last_error = std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
  return SEGKV_ERR_CUDA;
}
#define SEGKV_CUDA(h, what, expr)                    \
  do {                                               \
    const cudaError_t e_ = (expr);                   \
    if (e_ != cudaSuccess) return cuda_fail(h, what, e_); \
  } while (0)

StorageGeom geom(const segkv_t *h) {
  StorageGeom g;
  g.page_table = h->cfg.page_table;
  g.free_list = h->cfg.free_list;
  g.state = h->cfg.state;
  g.k_pool = h->cfg.k_pool;
  g.v_pool = h->cfg.v_pool;
  g.num_pages = h->cfg.num_pages;
  g.page = h->cfg.page_size;
  g.head_dim = h->cfg.head_dim;
  g.hkv = h->cfg.num_kv_heads;
  g.hq = h->cfg.num_q_heads;
  g.max_seqs = h->cfg.max_seqs;
  g.max_lp = h->max_lp;
  g.ring = h->ring;
  g.window = h->cfg.window;
  g.wait_limit = h->wait_limit;
  return g;
}

// Pinned staging slot big enough for `bytes`; waits for the copy that last used it.
int staging(segkv_t *h, size_t bytes, void **host) {
  Staging &s = h->slot[h->next_slot];
  if (s.pending) {
    SEGKV_CUDA(h, "staging event wait", cudaEventSynchronize(s.ev));
    s.pending = false;
  }
  if (!s.ev) SEGKV_CUDA(h, "staging event create", cudaEventCreateWithFlags(&s.ev, cudaEventDisableTiming));
  if (s.cap < bytes) {
    if (s.host) cudaFreeHost(s.host);
    s.host = nullptr;
    s.cap = 0;
    const size_t cap = std::max<size_t>(align_up(bytes, 4096), 64 << 10);
    SEGKV_CUDA(h, "pinned staging alloc", cudaHostAlloc(&s.host, cap, cudaHostAllocDefault));
    s.cap = cap;
  }
  *host = s.host;
  return SEGKV_OK;
}

int upload(segkv_t *h, void *ws, size_t bytes, cudaStream_t st) {
  Staging &s = h->slot[h->next_slot];
  SEGKV_CUDA(h, "metadata upload", cudaMemcpyAsync(ws, s.host, bytes, cudaMemcpyHostToDevice, st));
  SEGKV_CUDA(h, "staging event record", cudaEventRecord(s.ev, st));
  s.pending = true;
  h->next_slot = (h->next_slot + 1) % kStagingSlots;
  return SEGKV_OK;
}

int ensure_device_state(segkv_t *h) {
  if (h->maps_ready) return SEGKV_OK;
  int dev = 0;
  SEGKV_CUDA(h, "cudaGetDevice", cudaGetDevice(&dev));
  SEGKV_CUDA(h, "SM count", cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev));
  const segkv_config &c = h->cfg;
  const uint64_t rowb = (uint64_t)c.head_dim * 2, pageb = rowb * c.page_size;
  if (!make_map(&h->kmap, c.k_pool, c.head_dim, c.page_size, c.num_pages, rowb, pageb, c.page_size, 1) ||
      !make_map(&h->vmap, c.v_pool, c.head_dim, c.page_size, c.num_pages, rowb, pageb, c.page_size, 1)) {
    h->last_error = "pool tensor map encode failed";
    return SEGKV_ERR_CUDA;
  }
  h->maps_ready = true;
  return SEGKV_OK;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Common checks of a call's sequence list.
int check_seqs(const segkv_t *h, int layer, int nseq, const int32_t *seq_ids) {
  if (layer < 0 || layer >= h->cfg.num_layers || nseq < 1 || !seq_ids) return SEGKV_ERR_INVALID_ARG;
  if (nseq > h->cfg.max_seqs) return SEGKV_ERR_INVALID_ARG;
  std::vector<char> seen(h->cfg.max_seqs, 0);
  for (int b = 0; b < nseq; ++b) {
    const int s = seq_ids[b];
    if (s < 0 || s >= h->cfg.max_seqs || seen[s]) return SEGKV_ERR_INVALID_ARG;
    seen[s] = 1;
  }
  return SEGKV_OK;
}

// A local head can serve queries [q_lo, q_hi] only while its ring still holds key
// max(0, q_lo - W + 1): the ring holds the last R logical pages ending at the last token.
bool ring_covers(const segkv_t *h, int len, int q_lo) {
  const int P = h->cfg.page_size;
  const int need = std::max(0, q_lo - h->cfg.window + 1);
  return need / P >= (len - 1) / P - h->ring + 1;
}

bool layer_has_local(const segkv_t *h, int layer) {
  for (int k = 0; k < h->cfg.num_kv_heads; ++k)
    if (!h->cls[layer * h->cfg.num_kv_heads + k]) return true;
  return false;
}

struct PlanItem {
  int32_t b, h, t, cost;
};

// One launched work item: a whole item (slot -1) or a chunk [kt_a, kt_b] of its key tiles.
struct PlanChunk {
  int32_t b, h, t, kt_a, kt_b, slot;
};
struct SplitGroup {
  int32_t b, h, t, first_slot, n;
};

// Longest-processing-time-first list: enumerate (b, head, tile), cost = key tiles the
// tile touches, counting sort by cost descending (stable: ties keep enumeration order).
void plan_prefill_items(const segkv_t *h, int layer, int nseq, const int32_t *q_start, const int32_t *q_len,
                        std::vector<PlanItem> &out) {
  const int tile_pos = kPrefillItemRows / h->G, H = h->cfg.num_kv_heads, W = h->cfg.window;
  std::vector<PlanItem> items;
  int max_cost = 0;
  for (int b = 0; b < nseq; ++b)
    for (int k = 0; k < H; ++k) {
      const bool global = h->cls[layer * H + k] != 0;
      for (int t = 0; t * tile_pos < q_len[b]; ++t) {
        const int q_first = q_start[b] + t * tile_pos;
        const int q_last = q_start[b] + std::min((t + 1) * tile_pos, q_len[b]) - 1;
        const int lo = global ? 0 : std::max(0, q_first - W + 1);
        const int cost = q_last / kPrefillKeyTile - lo / kPrefillKeyTile + 1;
        items.push_back({b, k, t, cost});
        max_cost = std::max(max_cost, cost);
      }
    }
  std::vector<int64_t> start(max_cost + 2, 0);
  for (const PlanItem &it : items) start[it.cost]++;
  int64_t acc = 0;
  for (int c = max_cost; c >= 0; --c) {
    const int64_t n = start[c];
    start[c] = acc;
    acc += n;
  }
  out.assign(items.size(), PlanItem{0, 0, 0, 0});
  for (const PlanItem &it : items) out[start[it.cost]++] = it;
}

// Key tiles [kt_lo, kt_hi] an item of (sequence b, head k, tile pair t) touches.
void item_key_range(const segkv_t *h, int layer, int b, int k, int t, const int32_t *q_start, const int32_t *q_len,
                    int *kt_lo, int *kt_hi) {
  const int tile_pos = kPrefillItemRows / h->G, W = h->cfg.window;
  const bool global = h->cls[layer * h->cfg.num_kv_heads + k] != 0;
  const int q_first = q_start[b] + t * tile_pos;
  const int q_last = q_start[b] + std::min((t + 1) * tile_pos, q_len[b]) - 1;
  const int lo = global ? 0 : std::max(0, q_first - W + 1);
  *kt_lo = lo / kPrefillKeyTile;
  *kt_hi = q_last / kPrefillKeyTile;
}

// Cuts items longer than one SM's share of the work into chunks of contiguous key tiles,
// so that the longest-first schedule can balance: a global head's item can be far longer
// than total / SMs (for a 4096-query chunk at 128K context about twice as long).  Only
// when the longest item exceeds the per-SM share; chunks are at least 8 key tiles and at
// most kMaxPartSlots chunks are made.  The result is again sorted longest first (stable).
void split_long_items(const segkv_t *h, int layer, const int32_t *q_start, const int32_t *q_len,
                      const std::vector<PlanItem> &items, int grid, std::vector<PlanChunk> &chunks,
                      std::vector<SplitGroup> &groups) {
  long long total = 0;
  int max_cost = 0;
  for (const PlanItem &it : items) {
    total += it.cost;
    max_cost = std::max(max_cost, it.cost);
  }
  const long long fair = (total + grid - 1) / std::max(grid, 1);
  long long T = max_cost + 1;  // no split
  if (max_cost > fair) {
    // at least 8 key tiles a chunk, at most kMaxChunks chunks an item (the combine's limit)
    T = std::max<long long>({8, (fair + 1) / 2, (max_cost + kMaxChunks - 1) / kMaxChunks});
    for (;;) {
      long long slots = 0;
      for (const PlanItem &it : items)
        if (it.cost > T) slots += (it.cost + T - 1) / T;
      if (slots <= kMaxPartSlots) break;
      T = T + T / 4 + 1;
    }
  }
  chunks.clear();
  groups.clear();
  chunks.reserve(items.size() + (max_cost > T ? kMaxPartSlots : 0));
  if (max_cost <= T) {  // nothing to cut: the list keeps its longest-first order
    for (const PlanItem &it : items) {
      int a = 0, z = 0;
      item_key_range(h, layer, it.b, it.h, it.t, q_start, q_len, &a, &z);
      chunks.push_back({it.b, it.h, it.t, a, z, -1});
    }
    return;
  }
  int slot = 0;
  for (const PlanItem &it : items) {
    int a = 0, z = 0;
    item_key_range(h, layer, it.b, it.h, it.t, q_start, q_len, &a, &z);
    if (it.cost <= T) {
      chunks.push_back({it.b, it.h, it.t, a, z, -1});
      continue;
    }
    const int n = (int)((it.cost + T - 1) / T);
    groups.push_back({it.b, it.h, it.t, slot, n});
    for (int i = 0; i < n; ++i) {
      const int ca = a + (int)((long long)it.cost * i / n), cz = a + (int)((long long)it.cost * (i + 1) / n) - 1;
      chunks.push_back({it.b, it.h, it.t, ca, cz, slot++});
    }
  }
  std::stable_sort(chunks.begin(), chunks.end(),
                   [](const PlanChunk &x, const PlanChunk &y) { return x.kt_b - x.kt_a > y.kt_b - y.kt_a; });
}

// Prefill workspace: metadata (header, sequences, items, groups), then the partials.
size_t prefill_meta_bytes(int nseq, size_t n_items, size_t n_groups) {
  return align_up(align_up(kHeaderBytes + sizeof(PrefillSeq) * nseq, 16) + 16 * n_items + 16 * n_groups, 256);
}
size_t prefill_part_bytes(int head_dim) {
  return (size_t)kMaxPartSlots * 2 * 128 * ((size_t)head_dim + 1) * 4;
}

// Router workspace: header, sequences, items, per-sequence top-k rows, then the partials.
size_t router_meta_bytes(int nseq, size_t n_items) {
  return align_up(align_up(kHeaderBytes + sizeof(RouterSeq) * nseq, 16) + 16 * n_items + 16 * (size_t)nseq, 256);
}
size_t router_part_bytes(int chunks, int hkv, long long n_tokens) { return 4 * (size_t)chunks * hkv * n_tokens; }

// The token of a decode step, appended by the decode kernel itself: newk[b * hkv + h] =
// free-list entry of a page the token starts (-1: written in place), K/V rows on the device.
struct StepRows {
  const std::vector<int32_t> *newk;
  const void *k_new, *v_new;
  int cursor_after;
};

// Decode planning and launch.  With `step`, every sequence's length counts the step's token
// (not yet in the host's lengths) and the kernel appends it before attending.
int decode_common(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_pos, const void *q,
                  float softmax_scale, int num_splits, void *out, float *lse, uint64_t *visited, void *ws,
                  size_t ws_bytes, void *stream, const StepRows *step) {
  if (!h) return SEGKV_ERR_INVALID_ARG;
  int rc = check_seqs(h, layer, nseq, seq_ids);
  if (rc) return rc;
  if (!q_pos || num_splits < 0) return SEGKV_ERR_INVALID_ARG;
  if (h->G > 16) return SEGKV_ERR_UNSUPPORTED;
  if (!q || !out || !lse || !aligned(q, 16) || !aligned(out, 16) || !aligned(lse, 4)) return SEGKV_ERR_INVALID_ARG;
  const int P = h->cfg.page_size, H = h->cfg.num_kv_heads, Hq = h->cfg.num_q_heads, D = h->cfg.head_dim;
  const bool has_local = layer_has_local(h, layer);
  long long total_pages = 0;
  int max_pages = 0;
  for (int b = 0; b < nseq; ++b) {
    const int len = h->len[(size_t)layer * h->cfg.max_seqs + seq_ids[b]] + (step ? 1 : 0);
    if (q_pos[b] < 0 || q_pos[b] >= len) return SEGKV_ERR_INVALID_ARG;
    if (has_local && !ring_covers(h, len, q_pos[b])) return SEGKV_ERR_RING_TOO_SMALL;
    for (int k = 0; k < H; ++k) {
      const int lo = h->cls[layer * H + k] ? 0 : std::max(0, q_pos[b] - h->cfg.window + 1);
      const int n = q_pos[b] / P - lo / P + 1;
      total_pages += n;
      max_pages = std::max(max_pages, n);
    }
  }
  if ((rc = ensure_device_state(h))) return rc;
  // split size in pages: a multiple of the pages of one 64-key stage
  const int pps = kDecodeStageKeys / P;
  int split;
  if (num_splits > 0) {
    split = ceil_div(max_pages, std::min(num_splits, kMaxSplits));
  } else {
    const long long target = std::max<long long>(1, total_pages / (8LL * h->num_sms));
    split = 1;
    while (2LL * split <= target && split < 256) split *= 2;
  }
  split = std::max(split, ceil_div(max_pages, kMaxSplits));
  split = ceil_div(split, pps) * pps;
  const int max_splits = ceil_div(max_pages, split);
  const int nsplit_off = kHeaderBytes + (int)sizeof(DecodeSeq) * nseq;
  const int newk_off = nsplit_off + 4 * nseq * H;
  const int items_off = (int)align_up(newk_off + (step ? 4 * nseq * H : 0), 16);
  std::vector<int2> items;
  std::vector<int32_t> nsplit((size_t)nseq * H);
  for (int b = 0; b < nseq; ++b)
    for (int k = 0; k < H; ++k) {
      const bool global = h->cls[layer * H + k] != 0;
      const int lo = global ? 0 : std::max(0, q_pos[b] - h->cfg.window + 1);
      const int n = ceil_div(q_pos[b] / P - lo / P + 1, split);
      nsplit[(size_t)b * H + k] = n;
      for (int s = 0; s < n; ++s) items.push_back(make_int2(b, (int)make_item_w1(global, k, s)));
    }
  const size_t meta_bytes = items_off + 8 * items.size();
  const size_t part_o_off = align_up(meta_bytes, 256);
  const size_t part_lse_off = part_o_off + align_up(4 * (size_t)nseq * Hq * max_splits * D, 256);
  const size_t need = part_lse_off + 4 * (size_t)nseq * Hq * max_splits;
  if (!ws || !aligned(ws, 256) || ws_bytes < need) return SEGKV_ERR_WORKSPACE;
  void *host = nullptr;
  if ((rc = staging(h, meta_bytes, &host))) return rc;
  std::memset(host, 0, items_off);
  DecodeSeq *ds = reinterpret_cast<DecodeSeq *>(static_cast<char *>(host) + kHeaderBytes);
  for (int b = 0; b < nseq; ++b)
    ds[b] = DecodeSeq{seq_ids[b], q_pos[b], h->len[(size_t)layer * h->cfg.max_seqs + seq_ids[b]] + (step ? 1 : 0), 0};
  std::memcpy(static_cast<char *>(host) + nsplit_off, nsplit.data(), 4 * nsplit.size());
  if (step) std::memcpy(static_cast<char *>(host) + newk_off, step->newk->data(), 4 * step->newk->size());
  std::memcpy(static_cast<char *>(host) + items_off, items.data(), 8 * items.size());
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = upload(h, ws, meta_bytes, st))) return rc;
  DecodeLaunch p{};  // zeroed: fields a path does not set (the step append) stay off
  p.g = geom(h);
  p.layer = layer;
  p.nseq = nseq;
  p.n_items = (int)items.size();
  p.split_pages = split;
  p.max_splits = max_splits;
  p.grid = std::min<int>((int)items.size(), h->num_sms);
  p.ws_meta = ws;
  p.nsplit_off = nsplit_off;
  p.items_off = items_off;
  p.part_o = reinterpret_cast<float *>(static_cast<char *>(ws) + part_o_off);
  p.part_lse = reinterpret_cast<float *>(static_cast<char *>(ws) + part_lse_off);
  p.q = q;
  p.out = out;
  p.lse = lse;
  p.visited = reinterpret_cast<unsigned long long *>(visited);
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)D);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.newk = step ? reinterpret_cast<const int32_t *>(static_cast<const char *>(ws) + newk_off) : nullptr;
  p.k_new = step ? step->k_new : nullptr;
  p.v_new = step ? step->v_new : nullptr;
  p.cursor_after = step ? step->cursor_after : 0;
  SEGKV_CUDA(h, "decode launch", launch_decode(p, h->kmap, h->vmap, st));
  return SEGKV_OK;
}


}  // namespace

// ============================================================================== C ABI
extern "C" {

const char *segkv_strerror(int s) {
  switch (s) {
    case SEGKV_OK: return "ok";
    case SEGKV_ERR_INVALID_ARG: return "invalid argument";
    case SEGKV_ERR_UNSUPPORTED: return "unsupported shape";
    case SEGKV_ERR_OUT_OF_PAGES: return "out of pages";
    case SEGKV_ERR_RING_TOO_SMALL: return "local-head ring too small for the requested queries";
    case SEGKV_ERR_WORKSPACE: return "workspace too small or misaligned";
    case SEGKV_ERR_CUDA: return "CUDA error";
    case SEGKV_ERR_DEVICE_BOUNDS: return "device: page id out of range";
    case SEGKV_ERR_DEVICE_TIMEOUT: return "device: pipeline wait timed out";
    default: return "unknown status";
  }
}

namespace {
int noalloc_scratch(segkv_t *h, void **ptr);
}

}  // extern "C" (the tracing helper below is a template)

// ---------------------------------------------------------------------------- call tracing
// Every entry point that enqueues work or can fail runs through traced():
//   SEGKV_LOG=1   one stderr line for each call that returns an error (status, and the
//                 handle's last CUDA error text when there is one);
//   SEGKV_LOG=2   one stderr line for every call, with its host time;
//   SEGKV_NVTX=1  an NVTX range named after the entry point around the call (seen by
//                 profilers that record NVTX; the NVTX headers load nothing otherwise).
// Both variables are read once, at the first call.
namespace {
int env_level(const char *name) {
  const char *v = std::getenv(name);
  return v ? std::atoi(v) : 0;
}
template <class F>
int traced(const char *name, const segkv_t *h, F &&call) {
  static const int log = env_level("SEGKV_LOG");
  static const bool nvtx = env_level("SEGKV_NVTX") != 0;
  if (nvtx) nvtxRangePushA(name);
  const auto t0 = std::chrono::steady_clock::now();
  const int rc = call();
  const double us = std::chrono::duration<double, std::micro>(std::chrono::steady_clock::now() - t0).count();
  if (nvtx) nvtxRangePop();
  if (log >= 2 || (log >= 1 && rc != SEGKV_OK)) {
    const bool detail = rc == SEGKV_ERR_CUDA && h && !h->last_error.empty();
    std::fprintf(stderr, "[segkv] %s -> %d (%s)%s%s, %.1f us on the host\n", name, rc, segkv_strerror(rc),
                 detail ? ": " : "", detail ? h->last_error.c_str() : "", us);
  }
  return rc;
}
}  // namespace

extern "C" {

static int segkv_create_impl(const segkv_config *c, segkv_t **out) {
  if (!c || !out) return SEGKV_ERR_INVALID_ARG;
  *out = nullptr;
  if (c->num_layers < 1 || c->num_q_heads < 1 || c->num_kv_heads < 1 || c->max_seqs < 1 || c->max_seq_len < 1 ||
      c->window < 1 || c->num_pages < 1 || c->ring_pages < 0 || c->max_chunk < 0 || !c->head_class)
    return SEGKV_ERR_INVALID_ARG;
  if (!c->k_pool || !c->v_pool || !c->page_table || !c->free_list || !c->state) return SEGKV_ERR_INVALID_ARG;
  if (!aligned(c->k_pool, 16) || !aligned(c->v_pool, 16)) return SEGKV_ERR_INVALID_ARG;
  if (c->num_q_heads % c->num_kv_heads) return SEGKV_ERR_INVALID_ARG;
  const int G = c->num_q_heads / c->num_kv_heads;
  if (G > 128 || (G & (G - 1))) return SEGKV_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return SEGKV_ERR_UNSUPPORTED;
  if (c->page_size != 16 && c->page_size != 32 && c->page_size != 64) return SEGKV_ERR_UNSUPPORTED;
  if (c->num_kv_heads > 2047 || c->max_seq_len > (1 << 27)) return SEGKV_ERR_UNSUPPORTED;
  segkv_t *h = new (std::nothrow) segkv();
  if (!h) return SEGKV_ERR_INVALID_ARG;
  h->cfg = *c;
  h->G = G;
  h->max_lp = ceil_div(c->max_seq_len, c->page_size);
  if (c->ring_pages > 0) {
    h->ring = std::min(c->ring_pages, h->max_lp);
  } else {
    const int chunk = std::max(c->max_chunk, 1);
    h->ring = std::min(h->max_lp, ceil_div(c->window + chunk - 1, c->page_size) + 1);
  }
  h->cls.assign(c->head_class, c->head_class + (size_t)c->num_layers * c->num_kv_heads);
  for (uint8_t &x : h->cls) x = x ? 1 : 0;
  h->len.assign((size_t)c->num_layers * c->max_seqs, 0);
  h->slot_k.assign((size_t)c->num_layers * c->max_seqs * c->num_kv_heads * h->max_lp, -1);
  h->ref.assign((size_t)c->num_pages, 0);
  h->ref_scratch.assign((size_t)c->num_pages, 0);
  h->cfg.head_class = nullptr;
  // Set-up of the allocation-free decode: with a device current, look up (and so make
  // resident) the library's fixed scratch array on it now, before the caller hands the rest
  // of the device to its own allocator.  Without a device (a host-only process) there is
  // nothing to set up.
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    void *scratch = nullptr;
    if (noalloc_scratch(h, &scratch) != SEGKV_OK) {
      delete h;
      return SEGKV_ERR_CUDA;
    }
  } else {
    cudaGetLastError();  // clear the sticky "no device" status of the runtime
  }
  *out = h;
  return SEGKV_OK;
}
int segkv_create(const segkv_config *c, segkv_t **out) {
  return traced("segkv_create", nullptr, [&] { return segkv_create_impl(c, out); });
}

void segkv_destroy(segkv_t *h) {
  if (!h) return;
  for (Staging &s : h->slot) {
    if (s.pending) cudaEventSynchronize(s.ev);
    if (s.ev) cudaEventDestroy(s.ev);
    if (s.host) cudaFreeHost(s.host);
  }
  delete h;
}

int segkv_ring_pages(const segkv_t *h) { return h ? h->ring : -1; }
const char *segkv_last_error(const segkv_t *h) { return h ? h->last_error.c_str() : "no handle"; }

static int segkv_debug_set_impl(segkv_t *h, int key, long long value) {
  if (!h) return SEGKV_ERR_INVALID_ARG;
  switch (key) {
    case SEGKV_DEBUG_WAIT_LIMIT:
      if (value < 0) return SEGKV_ERR_INVALID_ARG;
      h->wait_limit = value;
      return SEGKV_OK;
    case SEGKV_DEBUG_STALL_NEXT_PREFILL:
      if (value != 0 && value != 1) return SEGKV_ERR_INVALID_ARG;
      h->stall_next_prefill = (int)value;
      return SEGKV_OK;
    case SEGKV_DEBUG_PREFILL_ORDER:
      if (value < 0) return SEGKV_ERR_INVALID_ARG;
      h->lpt_order = value;
      return SEGKV_OK;
    default:
      return SEGKV_ERR_INVALID_ARG;
  }
}
int segkv_debug_set(segkv_t *h, int key, long long value) {
  return traced("segkv_debug_set", h, [&] { return segkv_debug_set_impl(h, key, value); });
}
int segkv_max_lp(const segkv_t *h) { return h ? h->max_lp : -1; }
int segkv_pages_used(const segkv_t *h) { return h ? (int)h->pages_used : -1; }

int segkv_seq_len(const segkv_t *h, int layer, int seq) {
  if (!h || layer < 0 || layer >= h->cfg.num_layers || seq < 0 || seq >= h->cfg.max_seqs) return -1;
  return h->len[(size_t)layer * h->cfg.max_seqs + seq];
}

size_t segkv_workspace_bytes(const segkv_t *h, int max_batch, int max_tokens) {
  if (!h || max_batch < 1 || max_tokens < 0) return 0;
  const size_t H = h->cfg.num_kv_heads, Hq = h->cfg.num_q_heads, D = h->cfg.head_dim;
  const int tile_pos = kPrefillItemRows / h->G;
  // append: per (sequence, head) the plan offset, then one plan entry per touched page
  const size_t app = align_up(kHeaderBytes + sizeof(AppendSeq) * max_batch + align_up(H, 4) + 4 * (H * max_batch + 1),
                              16) +
                     sizeof(int4) * H * ((size_t)ceil_div(max_tokens, h->cfg.page_size) + 2 * max_batch);
  // prefill: items, the key-chunk groups and (fused append) one page offset per (sequence, head)
  const size_t pre = prefill_meta_bytes(max_batch, H * ((size_t)ceil_div(max_tokens, tile_pos) + max_batch) +
                                                      kMaxPartSlots + (H * max_batch + 3) / 4,
                                        kMaxPartSlots) +
                     prefill_part_bytes((int)D);
  // decode: split counts and (decode step) new page ids per (sequence, head), then the items
  const size_t dec_meta = align_up(kHeaderBytes + sizeof(DecodeSeq) * max_batch + 8 * max_batch * H +
                                       8 * max_batch * H * kMaxSplits + 16,
                                   256);
  const size_t dec = dec_meta + align_up(4 * (size_t)max_batch * Hq * kMaxSplits * D, 256) +
                     4 * (size_t)max_batch * Hq * kMaxSplits;
  const size_t rt = router_meta_bytes(max_batch, H * ((size_t)max_tokens / kRouterKeys + 2 * max_batch) *
                                                     kRouterMaxChunks) +
                    router_part_bytes(kRouterColGroups * kRouterMaxChunks, (int)H, max_tokens);
  return align_up(std::max(std::max(app, rt), std::max(pre, dec)), 256);
}

static int segkv_reset_impl(segkv_t *h, void *stream) {
  if (!h) return SEGKV_ERR_INVALID_ARG;
  SEGKV_CUDA(h, "reset launch", launch_reset(geom(h), h->cfg.num_layers, static_cast<cudaStream_t>(stream)));
  std::fill(h->len.begin(), h->len.end(), 0);
  std::fill(h->slot_k.begin(), h->slot_k.end(), -1);
  std::fill(h->ref.begin(), h->ref.end(), 0);
  h->n_shared = 0;
  h->pages_used = 0;
  return SEGKV_OK;
}
int segkv_reset(segkv_t *h, void *stream) {
  return traced("segkv_reset", h, [&] { return segkv_reset_impl(h, stream); });
}

static int segkv_fork_impl(segkv_t *h, int src_seq, int dst_seq, void *stream) {
  if (!h) return SEGKV_ERR_INVALID_ARG;
  const segkv_config &c = h->cfg;
  if (src_seq < 0 || dst_seq < 0 || src_seq >= c.max_seqs || dst_seq >= c.max_seqs || src_seq == dst_seq)
    return SEGKV_ERR_INVALID_ARG;
  for (int l = 0; l < c.num_layers; ++l)
    if (h->len[(size_t)l * c.max_seqs + dst_seq] != 0) return SEGKV_ERR_INVALID_ARG;
  const size_t row = (size_t)c.num_kv_heads * h->max_lp;  // one (layer, seq) block of the page table
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int l = 0; l < c.num_layers; ++l)
    SEGKV_CUDA(h, "fork page-table copy",
               cudaMemcpyAsync(c.page_table + ((size_t)l * c.max_seqs + dst_seq) * row,
                               c.page_table + ((size_t)l * c.max_seqs + src_seq) * row, row * sizeof(int32_t),
                               cudaMemcpyDeviceToDevice, st));
  for (int l = 0; l < c.num_layers; ++l) {
    const int32_t *a = &h->slot_k[((size_t)l * c.max_seqs + src_seq) * row];
    int32_t *b = &h->slot_k[((size_t)l * c.max_seqs + dst_seq) * row];
    for (size_t i = 0; i < row; ++i) {
      b[i] = a[i];
      if (a[i] >= 0 && ++h->ref[a[i]] == 2) h->n_shared++;
    }
    h->len[(size_t)l * c.max_seqs + dst_seq] = h->len[(size_t)l * c.max_seqs + src_seq];
  }
  return SEGKV_OK;
}
int segkv_fork(segkv_t *h, int src_seq, int dst_seq, void *stream) {
  return traced("segkv_fork", h, [&] { return segkv_fork_impl(h, src_seq, dst_seq, stream); });
}

static int segkv_append_impl(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *start_pos,
                 const int32_t *num_new, const void *k_new, const void *v_new, void *ws, size_t ws_bytes,
                 void *stream) {
  if (!h) return SEGKV_ERR_INVALID_ARG;
  int rc = check_seqs(h, layer, nseq, seq_ids);
  if (rc) return rc;
  if (!start_pos || !num_new) return SEGKV_ERR_INVALID_ARG;
  const int H = h->cfg.num_kv_heads;
  long long total = 0;
  for (int b = 0; b < nseq; ++b) {
    const int s = seq_ids[b];
    const int cur = h->len[(size_t)layer * h->cfg.max_seqs + s];
    if (num_new[b] < 0 || start_pos[b] != cur || (long long)cur + num_new[b] > h->cfg.max_seq_len)
      return SEGKV_ERR_INVALID_ARG;
    total += num_new[b];
  }
  if (total > (1LL << 30)) return SEGKV_ERR_UNSUPPORTED;
  if (total > 0 && (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16))) return SEGKV_ERR_INVALID_ARG;
  // Page plan, in the allocation order (sequence in call order, head ascending, logical page
  // ascending): for every page the call touches, the free-list index of a page it takes --
  // the slot is empty, or its page is shared with another sequence (copy on write: the
  // rows before the call's first token on that page are copied over) -- or -1 (the slot's
  // page is this sequence's alone and is written in place).
  const int P = h->cfg.page_size, R = h->ring, max_lp = h->max_lp;
  // Logical pages [lp0, lp1] the call touches for (sequence b, head k), and the mirror row.
  auto touched = [&](int b, int k, int &lp0, int &lp1, size_t &row, bool &global) {
    global = h->cls[layer * H + k] != 0;
    lp1 = (start_pos[b] + num_new[b] - 1) / P;
    lp0 = start_pos[b] / P;
    if (!global && lp1 - R + 1 > lp0) lp0 = lp1 - R + 1;
    row = (((size_t)layer * h->cfg.max_seqs + seq_ids[b]) * H + k) * max_lp;
  };
  std::vector<int32_t> pair_page((size_t)nseq * H + 1, 0);  // first plan entry of each pair
  std::vector<int32_t> pair_new((size_t)nseq * H + 1, 0);   // pages allocated for earlier pairs
  std::vector<int32_t> plan;
  std::vector<int32_t> plan_src;  // per plan entry: the shared page to copy rows from, else -1
  const bool copies = h->n_shared > 0;  // else every page is one sequence's: no copy, no plan
  // changes to the mirror, applied once the call is accepted; refcounts seen through them, so
  // a page one sequence of the call copies is no longer shared for a later one
  std::vector<std::pair<size_t, int32_t>> slot_set;
  std::vector<int32_t> ref_keys;  // entries whose count the call changes (pending in ref_scratch)
  struct ScratchClear {           // every exit leaves ref_scratch all zero again
    std::vector<int32_t> &scratch, &keys;
    ~ScratchClear() {
      for (const int32_t k : keys) scratch[k] = 0;
    }
  } scratch_clear{h->ref_scratch, ref_keys};
  auto ref_of = [&](int32_t k) { return h->ref[k] + h->ref_scratch[k]; };
  long long new_pages = 0;
  int max_pages = 0;  // the most pages one (sequence, head) of the call touches
  for (int b = 0; b < nseq; ++b)
    for (int k = 0; k < H; ++k) {
      pair_page[(size_t)b * H + k] = (int32_t)plan.size();
      pair_new[(size_t)b * H + k] = (int32_t)new_pages;
      if (num_new[b] == 0) continue;
      int lp0, lp1;
      size_t row;
      bool global;
      touched(b, k, lp0, lp1, row, global);
      max_pages = std::max(max_pages, lp1 - lp0 + 1);
      if (!copies) {  // a page is taken exactly for an empty slot
        for (int lp = lp0; lp <= lp1; ++lp) new_pages += h->slot_k[row + (global ? lp : lp % R)] < 0;
        continue;
      }
      const int first = start_pos[b];
      for (int lp = lp0; lp <= lp1; ++lp) {
        const size_t idx = row + (global ? lp : lp % R);
        const int32_t k_old = h->slot_k[idx];
        if (k_old >= 0 && ref_of(k_old) <= 1) {
          plan.push_back(-1);
          plan_src.push_back(-1);
          continue;
        }
        const int32_t k_new = (int32_t)(h->pages_used + new_pages++);
        const int copy_rows = (k_old >= 0 && lp == first / P) ? first % P : 0;
        plan.push_back(k_new);
        plan_src.push_back(copy_rows > 0 ? k_old : -1);
        slot_set.push_back({idx, k_new});
        if (k_old >= 0) {
          if (h->ref_scratch[k_old] == 0) ref_keys.push_back(k_old);
          h->ref_scratch[k_old] -= 1;
        }
      }
    }
  pair_page[(size_t)nseq * H] = (int32_t)plan.size();
  pair_new[(size_t)nseq * H] = (int32_t)new_pages;
  if (h->pages_used + new_pages > h->cfg.num_pages) return SEGKV_ERR_OUT_OF_PAGES;
  const size_t cls_off = kHeaderBytes + sizeof(AppendSeq) * nseq;
  const size_t off_off = cls_off + align_up(H, 4);
  const size_t plan_off = align_up(off_off + 4 * ((size_t)H * nseq + 1), 16);
  const size_t src_off = align_up(plan_off + 4 * plan.size(), 16);
  const size_t bytes = src_off + 4 * plan_src.size();
  if (!ws || !aligned(ws, 256) || ws_bytes < bytes) return SEGKV_ERR_WORKSPACE;
  if ((rc = ensure_device_state(h))) return rc;
  if (total == 0) return SEGKV_OK;
  void *host = nullptr;
  if ((rc = staging(h, bytes, &host))) return rc;
  std::memset(host, 0, kHeaderBytes);
  AppendSeq *as = reinterpret_cast<AppendSeq *>(static_cast<char *>(host) + kHeaderBytes);
  int tok = 0;
  for (int b = 0; b < nseq; ++b) {
    as[b] = AppendSeq{seq_ids[b], start_pos[b], num_new[b], tok};
    tok += num_new[b];
  }
  std::memcpy(static_cast<char *>(host) + cls_off, &h->cls[(size_t)layer * H], H);
  std::memcpy(static_cast<char *>(host) + off_off, copies ? pair_page.data() : pair_new.data(), 4 * pair_page.size());
  if (!plan.empty()) std::memcpy(static_cast<char *>(host) + plan_off, plan.data(), 4 * plan.size());
  if (!plan_src.empty()) std::memcpy(static_cast<char *>(host) + src_off, plan_src.data(), 4 * plan_src.size());
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = upload(h, ws, bytes, st))) return rc;
  const uint8_t *cls_dev = static_cast<const uint8_t *>(ws) + cls_off;
  const int32_t *off_dev = reinterpret_cast<const int32_t *>(static_cast<const char *>(ws) + off_off);
  const int32_t *plan_dev = reinterpret_cast<const int32_t *>(static_cast<const char *>(ws) + plan_off);
  const int32_t *src_dev = reinterpret_cast<const int32_t *>(static_cast<const char *>(ws) + src_off);
  SEGKV_CUDA(h, "append launch",
             launch_append(geom(h), layer, ws, nseq, cls_dev, off_dev, copies ? plan_dev : nullptr, src_dev,
                           (int)h->pages_used, (int)new_pages, max_pages, k_new, v_new, st));
  if (copies) {
    for (const auto &e : slot_set) {
      h->slot_k[e.first] = e.second;
      h->ref[e.second] = 1;
    }
    for (const int32_t k : ref_keys) {
      const int32_t before = h->ref[k];
      h->ref[k] += h->ref_scratch[k];
      if (before >= 2 && h->ref[k] < 2) h->n_shared--;
    }
  } else {  // the kernel's closed form: new pages in the allocation order
    int32_t k_new = (int32_t)h->pages_used;
    for (int b = 0; b < nseq; ++b)
      for (int k = 0; k < H && num_new[b] > 0; ++k) {
        int lp0, lp1;
        size_t row;
        bool global;
        touched(b, k, lp0, lp1, row, global);
        for (int lp = lp0; lp <= lp1; ++lp) {
          int32_t &slot = h->slot_k[row + (global ? lp : lp % R)];
          if (slot < 0) {
            slot = k_new;
            h->ref[k_new++] = 1;
          }
        }
      }
  }
  for (int b = 0; b < nseq; ++b) h->len[(size_t)layer * h->cfg.max_seqs + seq_ids[b]] += num_new[b];
  h->pages_used += new_pages;
  return SEGKV_OK;
}
int segkv_append(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *start_pos,
                 const int32_t *num_new, const void *k_new, const void *v_new, void *ws, size_t ws_bytes,
                 void *stream) {
  return traced("segkv_append", h, [&] { return segkv_append_impl(h, layer, nseq, seq_ids, start_pos, num_new, k_new, v_new, ws, ws_bytes, stream); });
}

static int segkv_plan_prefill_impl(const segkv_t *h, int layer, int nseq, const int32_t *q_start_pos, const int32_t *q_len,
                       int32_t *items_out, int64_t cap, int64_t *n_items, int *tile_pos, int *key_tile) {
  if (!h || layer < 0 || layer >= h->cfg.num_layers || nseq < 1 || !q_start_pos || !q_len)
    return SEGKV_ERR_INVALID_ARG;
  for (int b = 0; b < nseq; ++b)
    if (q_len[b] < 0 || q_start_pos[b] < 0) return SEGKV_ERR_INVALID_ARG;
  std::vector<PlanItem> items;
  plan_prefill_items(h, layer, nseq, q_start_pos, q_len, items);
  if (n_items) *n_items = (int64_t)items.size();
  if (tile_pos) *tile_pos = kPrefillItemRows / h->G;
  if (key_tile) *key_tile = kPrefillKeyTile;
  if ((int64_t)items.size() > cap || (!items_out && !items.empty())) return SEGKV_ERR_WORKSPACE;
  for (size_t i = 0; i < items.size(); ++i) {
    items_out[4 * i + 0] = items[i].b;
    items_out[4 * i + 1] = items[i].h;
    items_out[4 * i + 2] = items[i].t;
    items_out[4 * i + 3] = items[i].cost;
  }
  return SEGKV_OK;
}
int segkv_plan_prefill(const segkv_t *h, int layer, int nseq, const int32_t *q_start_pos, const int32_t *q_len,
                       int32_t *items_out, int64_t cap, int64_t *n_items, int *tile_pos, int *key_tile) {
  return traced("segkv_plan_prefill", h, [&] { return segkv_plan_prefill_impl(h, layer, nseq, q_start_pos, q_len, items_out, cap, n_items, tile_pos, key_tile); });
}

// Prefill, one-source (k_chunk == NULL: every key from the pages) or two-source (the keys of
// each sequence's query range from k_chunk / v_chunk, not yet appended); with `fused`, the
// kernel also appends those keys (segkv_prefill_append).
static int prefill_impl(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start_pos,
                        const int32_t *q_len, const void *q, const void *k_chunk, const void *v_chunk,
                        float softmax_scale, void *out, float *lse, uint64_t *visited, void *ws, size_t ws_bytes,
                        void *stream, bool fused = false) {
  if (!h) return SEGKV_ERR_INVALID_ARG;
  int rc = check_seqs(h, layer, nseq, seq_ids);
  if (rc) return rc;
  if (!q_start_pos || !q_len) return SEGKV_ERR_INVALID_ARG;
  const bool has_local = layer_has_local(h, layer), two = k_chunk != nullptr;
  long long tq = 0;
  for (int b = 0; b < nseq; ++b) {
    const int len = h->len[(size_t)layer * h->cfg.max_seqs + seq_ids[b]];
    if (q_len[b] < 0 || q_start_pos[b] < 0) return SEGKV_ERR_INVALID_ARG;
    if (two) {
      // the range starts where the stored sequence ends, on a page boundary
      if (q_start_pos[b] != len || q_start_pos[b] % h->cfg.page_size != 0 ||
          (long long)len + q_len[b] > h->cfg.max_seq_len)
        return SEGKV_ERR_INVALID_ARG;
    } else if ((long long)q_start_pos[b] + q_len[b] > len) {
      return SEGKV_ERR_INVALID_ARG;
    }
    if (q_len[b] > 0 && has_local && !ring_covers(h, len, q_start_pos[b])) return SEGKV_ERR_RING_TOO_SMALL;
    // fused: after the call the ring must still hold every key a query of the call needs
    // (the one-source rule), so no page the call overwrites in place is read by the call
    if (fused && q_len[b] > 0 && has_local && !ring_covers(h, len + q_len[b], q_start_pos[b]))
      return SEGKV_ERR_RING_TOO_SMALL;
    tq += q_len[b];
  }
  if (tq == 0) return SEGKV_OK;
  if (tq > (1LL << 30)) return SEGKV_ERR_UNSUPPORTED;
  if (!q || !out || !lse || !aligned(q, 16) || !aligned(out, 16) || !aligned(lse, 4)) return SEGKV_ERR_INVALID_ARG;
  if (two && (!v_chunk || !aligned(k_chunk, 16) || !aligned(v_chunk, 16))) return SEGKV_ERR_INVALID_ARG;
  const int H = h->cfg.num_kv_heads, P = h->cfg.page_size, R = h->ring;
  // fused append, page rule of segkv_append: every empty slot the call touches takes the next
  // free-list entry (sequence in call order, head ascending, page ascending); pair_off holds
  // the pages taken by earlier (sequence, head) pairs
  std::vector<int32_t> pair_off;
  long long new_pages = 0;
  auto touched = [&](int b, int k, int &lp0, int &lp1, size_t &row, bool &global) {
    global = h->cls[layer * H + k] != 0;
    lp1 = (q_start_pos[b] + q_len[b] - 1) / P;
    lp0 = q_start_pos[b] / P;
    if (!global && lp1 - R + 1 > lp0) lp0 = lp1 - R + 1;
    row = (((size_t)layer * h->cfg.max_seqs + seq_ids[b]) * H + k) * h->max_lp;
  };
  if (fused) {
    if (h->n_shared > 0) {
      // a page may be shared after a fork: the append's copy on write runs as its own call
      if ((rc = segkv_append(h, layer, nseq, seq_ids, q_start_pos, q_len, k_chunk, v_chunk, ws, ws_bytes, stream)))
        return rc;
      return prefill_impl(h, layer, nseq, seq_ids, q_start_pos, q_len, q, nullptr, nullptr, softmax_scale, out, lse,
                          visited, ws, ws_bytes, stream);
    }
    pair_off.assign((size_t)nseq * H, 0);
    for (int b = 0; b < nseq; ++b)
      for (int k = 0; k < H; ++k) {
        pair_off[(size_t)b * H + k] = (int32_t)new_pages;
        if (q_len[b] == 0) continue;
        int lp0, lp1;
        size_t row;
        bool global;
        touched(b, k, lp0, lp1, row, global);
        for (int lp = lp0; lp <= lp1; ++lp) new_pages += h->slot_k[row + (global ? lp : lp % R)] < 0;
      }
    if (h->pages_used + new_pages > h->cfg.num_pages) return SEGKV_ERR_OUT_OF_PAGES;
  }
  if ((rc = ensure_device_state(h))) return rc;
  std::vector<PlanItem> items;
  plan_prefill_items(h, layer, nseq, q_start_pos, q_len, items);
  std::vector<PlanChunk> chunks;
  std::vector<SplitGroup> groups;
  split_long_items(h, layer, q_start_pos, q_len, items, h->num_sms, chunks, groups);
  if (h->lpt_order != 0) {  // test hook: run the same work list in another order
    if (h->lpt_order == 1) {
      std::reverse(chunks.begin(), chunks.end());
    } else {
      std::mt19937_64 rng((uint64_t)h->lpt_order);
      std::shuffle(chunks.begin(), chunks.end(), rng);
    }
  }
  const int items_off = (int)align_up(kHeaderBytes + sizeof(PrefillSeq) * nseq, 16);
  const int groups_off = items_off + 16 * (int)chunks.size();
  const int pair_off_at = groups_off + 16 * (int)groups.size();
  const size_t pair_words = align_up(4 * pair_off.size(), 16) / 16;  // in 16-byte units
  const size_t bytes = pair_off_at + 16 * pair_words;
  const size_t meta = prefill_meta_bytes(nseq, chunks.size() + pair_words, groups.size());
  const size_t need = meta + prefill_part_bytes(h->cfg.head_dim);
  if (!ws || !aligned(ws, 256) || ws_bytes < need) return SEGKV_ERR_WORKSPACE;
  void *host = nullptr;
  if ((rc = staging(h, bytes, &host))) return rc;
  std::memset(host, 0, items_off);
  PrefillSeq *ps = reinterpret_cast<PrefillSeq *>(static_cast<char *>(host) + kHeaderBytes);
  int row0 = 0;
  for (int b = 0; b < nseq; ++b) {
    ps[b] = PrefillSeq{seq_ids[b], q_start_pos[b], q_len[b], row0,
                       h->len[(size_t)layer * h->cfg.max_seqs + seq_ids[b]], 0, 0, 0};
    row0 += q_len[b];
  }
  int4 *it = reinterpret_cast<int4 *>(static_cast<char *>(host) + items_off);
  for (size_t i = 0; i < chunks.size(); ++i) {
    const PlanChunk &c = chunks[i];
    it[i] = make_int4(c.b, (int)make_item_w1(h->cls[layer * H + c.h] != 0, c.h, c.t), (c.kt_a << 16) | c.kt_b,
                      c.slot);
  }
  int4 *gr = reinterpret_cast<int4 *>(static_cast<char *>(host) + groups_off);
  for (size_t i = 0; i < groups.size(); ++i) {
    const SplitGroup &g = groups[i];
    gr[i] = make_int4(g.b, (int)make_item_w1(h->cls[layer * H + g.h] != 0, g.h, g.t), g.first_slot, g.n);
  }
  if (!pair_off.empty()) std::memcpy(static_cast<char *>(host) + pair_off_at, pair_off.data(), 4 * pair_off.size());
  // query in (box: one 128-row tile, G heads x 128/G positions) and output out (box: the 32
  // rows one softmax warp stores, min(G, 32) heads x max(1, 32/G) positions), both [tokens, Hq, D]
  CUtensorMap qmap, omap;
  const int D = h->cfg.head_dim, Hq = h->cfg.num_q_heads, Hkv = h->cfg.num_kv_heads;
  if (!make_map(&qmap, q, D, Hq, (uint64_t)tq, (uint64_t)D * 2, (uint64_t)Hq * D * 2, h->G,
                kPrefillTileRows / h->G) ||
      !make_map(&omap, out, D, Hq, (uint64_t)tq, (uint64_t)D * 2, (uint64_t)Hq * D * 2, std::min(h->G, 32),
                std::max(1, 32 / h->G))) {
    h->last_error = "query/output tensor map encode failed";
    return SEGKV_ERR_CUDA;
  }
  CUtensorMap kcmap = h->kmap, vcmap = h->vmap;  // two-source: the call's K/V, one page-sized box per head
  if (two && (!make_map(&kcmap, k_chunk, D, Hkv, (uint64_t)tq, (uint64_t)D * 2, (uint64_t)Hkv * D * 2, 1,
                        h->cfg.page_size) ||
              !make_map(&vcmap, v_chunk, D, Hkv, (uint64_t)tq, (uint64_t)D * 2, (uint64_t)Hkv * D * 2, 1,
                        h->cfg.page_size))) {
    h->last_error = "chunk K/V tensor map encode failed";
    return SEGKV_ERR_CUDA;
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = upload(h, ws, bytes, st))) return rc;
  PrefillLaunch p{};
  p.g = geom(h);
  p.layer = layer;
  p.nseq = nseq;
  p.n_items = (int)chunks.size();
  p.tile_pos = kPrefillTileRows / h->G;
  p.grid = std::min<int>((int)chunks.size(), h->num_sms);
  p.ws_meta = ws;
  p.items_off = items_off;
  p.groups_off = groups_off;
  p.n_groups = (int)groups.size();
  p.part_o = reinterpret_cast<float *>(static_cast<char *>(ws) + meta);
  p.part_lse = p.part_o + (size_t)kMaxPartSlots * 2 * 128 * h->cfg.head_dim;
  p.q = q;
  p.out = out;
  p.lse = lse;
  p.visited = reinterpret_cast<unsigned long long *>(visited);
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)D);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.two_src = two ? 1 : 0;
  p.stall_test = h->stall_next_prefill;
  h->stall_next_prefill = 0;
  if (fused) {
    p.store = 1;
    p.pair_off = reinterpret_cast<const int32_t *>(static_cast<const char *>(ws) + pair_off_at);
    p.cursor0 = (int)h->pages_used;
    p.new_pages = (int)new_pages;
  }
  SEGKV_CUDA(h, "prefill launch", launch_prefill(p, qmap, h->kmap, h->vmap, omap, kcmap, vcmap, st));
  if (fused) {  // the host mirror follows the kernel's closed form, in the allocation order
    int32_t k_new = (int32_t)h->pages_used;
    for (int b = 0; b < nseq; ++b) {
      for (int k = 0; k < H && q_len[b] > 0; ++k) {
        int lp0, lp1;
        size_t row;
        bool global;
        touched(b, k, lp0, lp1, row, global);
        for (int lp = lp0; lp <= lp1; ++lp) {
          int32_t &slot = h->slot_k[row + (global ? lp : lp % R)];
          if (slot < 0) {
            slot = k_new;
            h->ref[k_new++] = 1;
          }
        }
      }
      h->len[(size_t)layer * h->cfg.max_seqs + seq_ids[b]] += q_len[b];
    }
    h->pages_used += new_pages;
  }
  return SEGKV_OK;
}

static int segkv_prefill_attn_impl(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start_pos,
                       const int32_t *q_len, const void *q, float softmax_scale, void *out, float *lse,
                       uint64_t *visited, void *ws, size_t ws_bytes, void *stream) {
  return prefill_impl(h, layer, nseq, seq_ids, q_start_pos, q_len, q, nullptr, nullptr, softmax_scale, out, lse,
                      visited, ws, ws_bytes, stream);
}
int segkv_prefill_attn(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start_pos,
                       const int32_t *q_len, const void *q, float softmax_scale, void *out, float *lse,
                       uint64_t *visited, void *ws, size_t ws_bytes, void *stream) {
  return traced("segkv_prefill_attn", h, [&] { return segkv_prefill_attn_impl(h, layer, nseq, seq_ids, q_start_pos, q_len, q, softmax_scale, out, lse, visited, ws, ws_bytes, stream); });
}

static int segkv_prefill_append_impl(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start_pos,
                         const int32_t *q_len, const void *q, const void *k_new, const void *v_new,
                         float softmax_scale, void *out, float *lse, uint64_t *visited, void *ws, size_t ws_bytes,
                         void *stream) {
  if (!k_new) return SEGKV_ERR_INVALID_ARG;
  return prefill_impl(h, layer, nseq, seq_ids, q_start_pos, q_len, q, k_new, v_new, softmax_scale, out, lse,
                      visited, ws, ws_bytes, stream, true);
}
int segkv_prefill_append(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start_pos,
                         const int32_t *q_len, const void *q, const void *k_new, const void *v_new,
                         float softmax_scale, void *out, float *lse, uint64_t *visited, void *ws, size_t ws_bytes,
                         void *stream) {
  return traced("segkv_prefill_append", h, [&] { return segkv_prefill_append_impl(h, layer, nseq, seq_ids, q_start_pos, q_len, q, k_new, v_new, softmax_scale, out, lse, visited, ws, ws_bytes, stream); });
}

static int segkv_prefill_attn_2src_impl(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start_pos,
                            const int32_t *q_len, const void *q, const void *k_chunk, const void *v_chunk,
                            float softmax_scale, void *out, float *lse, uint64_t *visited, void *ws,
                            size_t ws_bytes, void *stream) {
  if (!k_chunk) return SEGKV_ERR_INVALID_ARG;
  return prefill_impl(h, layer, nseq, seq_ids, q_start_pos, q_len, q, k_chunk, v_chunk, softmax_scale, out, lse,
                      visited, ws, ws_bytes, stream);
}
int segkv_prefill_attn_2src(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start_pos,
                            const int32_t *q_len, const void *q, const void *k_chunk, const void *v_chunk,
                            float softmax_scale, void *out, float *lse, uint64_t *visited, void *ws,
                            size_t ws_bytes, void *stream) {
  return traced("segkv_prefill_attn_2src", h, [&] { return segkv_prefill_attn_2src_impl(h, layer, nseq, seq_ids, q_start_pos, q_len, q, k_chunk, v_chunk, softmax_scale, out, lse, visited, ws, ws_bytes, stream); });
}

static int segkv_decode_attn_impl(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_pos,
                      const void *q, float softmax_scale, int num_splits, void *out, float *lse, uint64_t *visited,
                      void *ws, size_t ws_bytes, void *stream) {
  return decode_common(h, layer, nseq, seq_ids, q_pos, q, softmax_scale, num_splits, out, lse, visited, ws, ws_bytes,
                       stream, nullptr);
}
int segkv_decode_attn(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_pos,
                      const void *q, float softmax_scale, int num_splits, void *out, float *lse, uint64_t *visited,
                      void *ws, size_t ws_bytes, void *stream) {
  return traced("segkv_decode_attn", h, [&] { return segkv_decode_attn_impl(h, layer, nseq, seq_ids, q_pos, q, softmax_scale, num_splits, out, lse, visited, ws, ws_bytes, stream); });
}

static int segkv_decode_step_impl(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const void *k_new, const void *v_new,
                      const void *q, float softmax_scale, int num_splits, void *out, float *lse, uint64_t *visited,
                      void *ws, size_t ws_bytes, void *stream) {
  if (!h) return SEGKV_ERR_INVALID_ARG;
  int rc = check_seqs(h, layer, nseq, seq_ids);
  if (rc) return rc;
  if (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)) return SEGKV_ERR_INVALID_ARG;
  if (!q || !out || !lse || !aligned(q, 16) || !aligned(out, 16) || !aligned(lse, 4) || num_splits < 0)
    return SEGKV_ERR_INVALID_ARG;
  if (h->G > 16) return SEGKV_ERR_UNSUPPORTED;
  const int H = h->cfg.num_kv_heads, P = h->cfg.page_size, R = h->ring;
  std::vector<int32_t> pos((size_t)nseq);
  for (int b = 0; b < nseq; ++b) {
    pos[b] = h->len[(size_t)layer * h->cfg.max_seqs + seq_ids[b]];
    if (pos[b] + 1 > h->cfg.max_seq_len) return SEGKV_ERR_INVALID_ARG;
    if (layer_has_local(h, layer) && !ring_covers(h, pos[b] + 1, pos[b])) return SEGKV_ERR_RING_TOO_SMALL;
  }
  if (h->n_shared > 0) {
    // a page may be shared after a fork: the append's copy on write runs first, as its own call
    std::vector<int32_t> one((size_t)nseq, 1);
    if ((rc = segkv_append(h, layer, nseq, seq_ids, pos.data(), one.data(), k_new, v_new, ws, ws_bytes, stream)))
      return rc;
    return segkv_decode_attn(h, layer, nseq, seq_ids, pos.data(), q, softmax_scale, num_splits, out, lse, visited,
                             ws, ws_bytes, stream);
  }
  // the append's page rule for one token: a page starts at pos % P == 0 and takes a new
  // free-list entry unless it recycles a full ring's slot in place
  std::vector<int32_t> newk((size_t)nseq * H, -1);
  long long new_pages = 0;
  for (int b = 0; b < nseq; ++b)
    for (int k = 0; k < H; ++k) {
      const int lp = pos[b] / P;
      const size_t row = (((size_t)layer * h->cfg.max_seqs + seq_ids[b]) * H + k) * h->max_lp;
      const bool global = h->cls[layer * H + k] != 0;
      if (h->slot_k[row + (global ? lp : lp % R)] < 0) newk[(size_t)b * H + k] = (int32_t)(h->pages_used + new_pages++);
    }
  if (h->pages_used + new_pages > h->cfg.num_pages) return SEGKV_ERR_OUT_OF_PAGES;
  const StepRows step{&newk, k_new, v_new, (int)(h->pages_used + new_pages)};
  if ((rc = decode_common(h, layer, nseq, seq_ids, pos.data(), q, softmax_scale, num_splits, out, lse, visited, ws,
                          ws_bytes, stream, &step)))
    return rc;
  for (int b = 0; b < nseq; ++b) {
    for (int k = 0; k < H; ++k) {
      const int32_t kn = newk[(size_t)b * H + k];
      if (kn < 0) continue;
      const int lp = pos[b] / P;
      const size_t row = (((size_t)layer * h->cfg.max_seqs + seq_ids[b]) * H + k) * h->max_lp;
      h->slot_k[row + (h->cls[layer * H + k] ? lp : lp % R)] = kn;
      h->ref[kn] = 1;
    }
    h->len[(size_t)layer * h->cfg.max_seqs + seq_ids[b]] += 1;
  }
  h->pages_used += new_pages;
  return SEGKV_OK;
}
int segkv_decode_step(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const void *k_new, const void *v_new,
                      const void *q, float softmax_scale, int num_splits, void *out, float *lse, uint64_t *visited,
                      void *ws, size_t ws_bytes, void *stream) {
  return traced("segkv_decode_step", h, [&] { return segkv_decode_step_impl(h, layer, nseq, seq_ids, k_new, v_new, q, softmax_scale, num_splits, out, lse, visited, ws, ws_bytes, stream); });
}

static int segkv_router_topk_impl(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start_pos,
                      const int32_t *q_len, const void *q, const float *lse, float softmax_scale, const int32_t *k,
                      float *scores, int32_t *rows_out, void *ws, size_t ws_bytes, void *stream) {
  if (!h) return SEGKV_ERR_INVALID_ARG;
  int rc = check_seqs(h, layer, nseq, seq_ids);
  if (rc) return rc;
  if (!q_start_pos || !q_len || !k) return SEGKV_ERR_INVALID_ARG;
  const int G = h->G, P = h->cfg.page_size, H = h->cfg.num_kv_heads, W = h->cfg.window;
  if (G > 16 || (G & (G - 1)) != 0) return SEGKV_ERR_UNSUPPORTED;
  const bool has_local = layer_has_local(h, layer);
  long long tq = 0, tk = 0;
  for (int b = 0; b < nseq; ++b) {
    const int len = h->len[(size_t)layer * h->cfg.max_seqs + seq_ids[b]];
    if (q_len[b] < 0 || q_start_pos[b] < 0 || (long long)q_start_pos[b] + q_len[b] > len) return SEGKV_ERR_INVALID_ARG;
    if (k[b] < 0 || k[b] > q_len[b]) return SEGKV_ERR_INVALID_ARG;
    // every scored token must still be stored in every local head
    if (q_len[b] > 0 && has_local && q_start_pos[b] / P < (len - 1) / P - h->ring + 1) return SEGKV_ERR_RING_TOO_SMALL;
    tq += q_len[b];
    tk += k[b];
  }
  if (tq == 0) return SEGKV_OK;
  if (tq > (1LL << 30)) return SEGKV_ERR_UNSUPPORTED;
  if (!q || !lse || !scores || !aligned(q, 16) || !aligned(lse, 4) || !aligned(scores, 4)) return SEGKV_ERR_INVALID_ARG;
  if (tk > 0 && (!rows_out || !aligned(rows_out, 4))) return SEGKV_ERR_INVALID_ARG;
  if ((rc = ensure_device_state(h))) return rc;
  // items: (sequence, KV head, key tile, chunk of query tiles), longest first
  const int tile_pos = kRouterKeys / G;
  struct Span {
    int b, kt;
  };
  std::vector<Span> spans;
  long long total_tiles = 0;
  for (int b = 0; b < nseq; ++b) {
    if (q_len[b] == 0) continue;
    const int qs = q_start_pos[b], qe = qs + q_len[b];
    for (int kt = qs / kRouterKeys; kt <= (qe - 1) / kRouterKeys; ++kt) spans.push_back({b, kt});
  }
  std::vector<int4> items;
  std::vector<int32_t> cost;
  int max_n = 0;
  for (int pass = 0; pass < 2; ++pass) {
    const long long share = std::max<long long>(1, (total_tiles + 2LL * h->num_sms - 1) / (2LL * h->num_sms));
    for (const Span &sp : spans)
      for (int hh = 0; hh < H; ++hh) {
        const bool global = h->cls[layer * H + hh] != 0;
        const int qs = q_start_pos[sp.b], qe = qs + q_len[sp.b];
        const int k_lo = std::max(sp.kt * kRouterKeys, qs), k_hi = std::min(sp.kt * kRouterKeys + kRouterKeys - 1, qe - 1);
        const int q_hi = global ? qe - 1 : std::min(qe - 1, k_hi + W - 1);
        const int n = ceil_div(q_hi - k_lo + 1, tile_pos);
        if (pass == 0) {
          total_tiles += n;
          max_n = std::max(max_n, n);
          continue;
        }
        const int C = (int)std::min<long long>(kRouterMaxChunks, std::max<long long>(1, (n + share - 1) / share));
        for (int c = 0; c < C; ++c) {
          const int t0 = (int)((long long)n * c / C), t1 = (int)((long long)n * (c + 1) / C);
          if (t1 <= t0) continue;
          items.push_back(make_int4(sp.b, (int)make_item_w1(global, hh, sp.kt), t0, (c << 20) | (t1 - t0)));
        }
      }
  }
  // partial slots: (chunk, group of query columns) -- kRouterColGroups reducing warps share each key
  int chunks = 1;
  for (const int4 &it : items) chunks = std::max(chunks, ((int)((uint32_t)it.w >> 20)) + 1);
  const int slots = kRouterColGroups * chunks;
  {  // longest first, equal lengths in creation order: a counting sort on the tile count
    int max_nt = 0;
    for (const int4 &it : items) max_nt = std::max(max_nt, it.w & 0xFFFFF);
    std::vector<int32_t> start((size_t)max_nt + 2, 0);
    for (const int4 &it : items) ++start[(size_t)(max_nt - (it.w & 0xFFFFF)) + 1];
    for (size_t v = 1; v < start.size(); ++v) start[v] += start[v - 1];
    std::vector<int4> sorted(items.size());
    for (const int4 &it : items) sorted[(size_t)start[(size_t)(max_nt - (it.w & 0xFFFFF))]++] = it;
    items.swap(sorted);
  }
  const size_t items_off = align_up(kHeaderBytes + sizeof(RouterSeq) * nseq, 16);
  const size_t topk_off = items_off + 16 * items.size();
  const size_t bytes = topk_off + 16 * (size_t)nseq;
  const size_t part_off = router_meta_bytes(nseq, items.size());
  const size_t need = part_off + router_part_bytes(slots, H, tq);
  if (!ws || !aligned(ws, 256) || ws_bytes < need) return SEGKV_ERR_WORKSPACE;
  const int D = h->cfg.head_dim, Hq = h->cfg.num_q_heads;
  CUtensorMap qmap;
  if (!make_map(&qmap, q, D, Hq, (uint64_t)tq, (uint64_t)D * 2, (uint64_t)Hq * D * 2, G, tile_pos)) {
    h->last_error = "query tensor map encode failed";
    return SEGKV_ERR_CUDA;
  }
  void *host = nullptr;
  if ((rc = staging(h, bytes, &host))) return rc;
  std::memset(host, 0, items_off);
  RouterSeq *rs = reinterpret_cast<RouterSeq *>(static_cast<char *>(host) + kHeaderBytes);
  int4 *tm = reinterpret_cast<int4 *>(static_cast<char *>(host) + topk_off);
  int row0 = 0, out0 = 0;
  for (int b = 0; b < nseq; ++b) {
    rs[b] = RouterSeq{seq_ids[b], q_start_pos[b], q_len[b], row0, h->len[(size_t)layer * h->cfg.max_seqs + seq_ids[b]],
                      0, 0, 0};
    tm[b] = make_int4(row0, q_len[b], k[b], out0);
    row0 += q_len[b];
    out0 += k[b];
  }
  if (!items.empty())
    std::memcpy(static_cast<char *>(host) + items_off, items.data(), 16 * items.size());
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = upload(h, ws, bytes, st))) return rc;
  float *part = reinterpret_cast<float *>(static_cast<char *>(ws) + part_off);
  SEGKV_CUDA(h, "router partials clear", cudaMemsetAsync(part, 0, router_part_bytes(slots, H, tq), st));
  RouterLaunch p{};
  p.g = geom(h);
  p.layer = layer;
  p.nseq = nseq;
  p.n_items = (int)items.size();
  p.tile_pos = tile_pos;
  p.g_shift = 0;
  while ((1 << p.g_shift) < G) ++p.g_shift;
  p.grid = std::min<int>((int)items.size(), h->num_sms);
  p.n_tokens = (int)tq;
  p.ws_meta = ws;
  p.items_off = (int)items_off;
  p.lse = lse;
  p.part = part;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)D);
  p.scale_log2 = scale * 1.4426950408889634f;
  if (p.n_items > 0) SEGKV_CUDA(h, "router launch", launch_router(p, qmap, h->kmap, st));
  SEGKV_CUDA(h, "top-k launch",
             launch_topk(part, slots, H, (int)tq, reinterpret_cast<const int4 *>(static_cast<char *>(ws) + topk_off),
                         nseq, *std::max_element(q_len, q_len + nseq), scores, rows_out, st));
  return SEGKV_OK;
}
int segkv_router_topk(segkv_t *h, int layer, int nseq, const int32_t *seq_ids, const int32_t *q_start_pos,
                      const int32_t *q_len, const void *q, const float *lse, float softmax_scale, const int32_t *k,
                      float *scores, int32_t *rows_out, void *ws, size_t ws_bytes, void *stream) {
  return traced("segkv_router_topk", h, [&] { return segkv_router_topk_impl(h, layer, nseq, seq_ids, q_start_pos, q_len, q, lse, softmax_scale, k, scores, rows_out, ws, ws_bytes, stream); });
}

static int segkv_relocate_q_impl(segkv_t *h, int layer, int n_tokens, const int32_t *shift, const void *q_in, void *q_out,
                     float theta_base, int interleaved, void *stream) {
  if (!h) return SEGKV_ERR_INVALID_ARG;
  if (layer < 0 || layer >= h->cfg.num_layers || n_tokens < 0 || !(theta_base > 1.0f) ||
      (interleaved != 0 && interleaved != 1))
    return SEGKV_ERR_INVALID_ARG;
  if (n_tokens == 0) return SEGKV_OK;
  if (!shift || !q_in || !q_out || !aligned(shift, 4) || !aligned(q_in, 16) || !aligned(q_out, 16))
    return SEGKV_ERR_INVALID_ARG;
  const int H = h->cfg.num_kv_heads, Hq = h->cfg.num_q_heads;
  if (Hq > 1024 || n_tokens > (1 << 30)) return SEGKV_ERR_UNSUPPORTED;
  RelocateLaunch p{};
  p.shift = shift;
  p.q_in = q_in;
  p.q_out = q_out;
  p.hq = h->cfg.num_q_heads;
  p.hkv = H;
  p.head_dim = h->cfg.head_dim;
  p.interleaved = interleaved;
  const double log2_base = std::log2((double)theta_base);
  for (int i = 0; i < p.head_dim / 2; ++i) p.theta[i] = std::exp2(-2.0 * i / p.head_dim * log2_base);
  std::memset(p.cls_bits, 0, sizeof(p.cls_bits));
  for (int q = 0; q < Hq; ++q)
    if (h->cls[(size_t)layer * H + q / (Hq / H)]) p.cls_bits[q >> 5] |= 1u << (q & 31);
  SEGKV_CUDA(h, "relocate launch", launch_relocate_q(p, n_tokens, static_cast<cudaStream_t>(stream)));
  return SEGKV_OK;
}
int segkv_relocate_q(segkv_t *h, int layer, int n_tokens, const int32_t *shift, const void *q_in, void *q_out,
                     float theta_base, int interleaved, void *stream) {
  return traced("segkv_relocate_q", h, [&] { return segkv_relocate_q_impl(h, layer, n_tokens, shift, q_in, q_out, theta_base, interleaved, stream); });
}

static int segkv_device_status_impl(segkv_t *h, void *stream) {
  if (!h) return SEGKV_ERR_INVALID_ARG;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t word = 0;
  SEGKV_CUDA(h, "status sync", cudaStreamSynchronize(st));
  SEGKV_CUDA(h, "status read", cudaMemcpyAsync(&word, h->cfg.state + 1, sizeof(word), cudaMemcpyDeviceToHost, st));
  SEGKV_CUDA(h, "status clear", cudaMemsetAsync(h->cfg.state + 1, 0, sizeof(int32_t), st));
  SEGKV_CUDA(h, "status sync", cudaStreamSynchronize(st));
  return word;
}
int segkv_device_status(segkv_t *h, void *stream) {
  return traced("segkv_device_status", h, [&] { return segkv_device_status_impl(h, stream); });
}

}  // extern "C"

// ============================================================================== decode without allocation
// For callers that cannot hand the library a workspace: the split partials, the scheduler
// counter and the per-call metadata live in a fixed scratch array that this file owns.
namespace {

constexpr size_t kNoAllocScratchBytes = 64u << 20;  // device scratch, held by every GPU that loads the library
constexpr size_t kNoAllocMetaBytes = 1u << 20;      // host-side metadata, pageable
constexpr int kNoAllocMaxDevices = 64;
constexpr int kNoAllocMaxSeqSlots = 1 << 16;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
unsigned char g_noalloc_meta[kNoAllocMetaBytes];
uint64_t g_noalloc_seen[kNoAllocMaxSeqSlots / 64];
void *g_noalloc_dev_ptr[kNoAllocMaxDevices];

// Device address of the scratch array on the current device, looked up once per device
// (segkv_create does it for the device current there; a call on another device does it on
// its first call there).  The look-up loads the module that holds the array, so this is where
// its 64 MiB become resident on that device.
int noalloc_scratch(segkv_t *h, void **ptr) {
  int dev = 0;
  SEGKV_CUDA(h, "cudaGetDevice", cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNoAllocMaxDevices) {
    h->last_error = "fixed scratch: device index beyond the supported 64";
    return SEGKV_ERR_UNSUPPORTED;
  }
  if (!g_noalloc_dev_ptr[dev]) {
    void *p = nullptr;
    SEGKV_CUDA(h, "scratch symbol address", cudaGetSymbolAddress(&p, g_noalloc_scratch));
    g_noalloc_dev_ptr[dev] = p;
  }
  *ptr = g_noalloc_dev_ptr[dev];
  return SEGKV_OK;
}

}  // namespace

static int segkv_decode_attn_noalloc_impl(segkv_t *h, int layer, int nseq, const int32_t *seq_ids,
                                         const int32_t *q_pos, const void *q, float softmax_scale, int num_splits,
                                         void *out, float *lse, uint64_t *visited, void *stream) {
  if (!h) return SEGKV_ERR_INVALID_ARG;
  if (layer < 0 || layer >= h->cfg.num_layers || nseq < 1 || nseq > h->cfg.max_seqs || !seq_ids || !q_pos ||
      num_splits < 0)
    return SEGKV_ERR_INVALID_ARG;
  if (h->cfg.max_seqs > kNoAllocMaxSeqSlots) return SEGKV_ERR_UNSUPPORTED;
  if (h->G > 16) return SEGKV_ERR_UNSUPPORTED;
  if (!q || !out || !lse || !aligned(q, 16) || !aligned(out, 16) || !aligned(lse, 4)) return SEGKV_ERR_INVALID_ARG;
  // distinct sequence ids (a fixed bitmap, cleared again before returning)
  int rc = SEGKV_OK;
  int b_seen = 0;
  for (; b_seen < nseq; ++b_seen) {
    const int s = seq_ids[b_seen];
    if (s < 0 || s >= h->cfg.max_seqs || (g_noalloc_seen[s >> 6] >> (s & 63) & 1)) {
      rc = SEGKV_ERR_INVALID_ARG;
      break;
    }
    g_noalloc_seen[s >> 6] |= 1ull << (s & 63);
  }
  for (int b = 0; b < b_seen; ++b) g_noalloc_seen[seq_ids[b] >> 6] &= ~(1ull << (seq_ids[b] & 63));
  if (rc) return rc;
  const int P = h->cfg.page_size, H = h->cfg.num_kv_heads, Hq = h->cfg.num_q_heads, D = h->cfg.head_dim;
  const bool has_local = layer_has_local(h, layer);
  long long total_pages = 0;
  int max_pages = 0;
  for (int b = 0; b < nseq; ++b) {
    const int len = h->len[(size_t)layer * h->cfg.max_seqs + seq_ids[b]];
    if (q_pos[b] < 0 || q_pos[b] >= len) return SEGKV_ERR_INVALID_ARG;
    if (has_local && !ring_covers(h, len, q_pos[b])) return SEGKV_ERR_RING_TOO_SMALL;
    for (int k = 0; k < H; ++k) {
      const int lo = h->cls[layer * H + k] ? 0 : std::max(0, q_pos[b] - h->cfg.window + 1);
      const int n = q_pos[b] / P - lo / P + 1;
      total_pages += n;
      max_pages = std::max(max_pages, n);
    }
  }
  if ((rc = ensure_device_state(h))) return rc;
  // the same split rule as segkv_decode_attn
  const int pps = kDecodeStageKeys / P;
  int split;
  if (num_splits > 0) {
    split = ceil_div(max_pages, std::min(num_splits, kMaxSplits));
  } else {
    const long long target = std::max<long long>(1, total_pages / (8LL * h->num_sms));
    split = 1;
    while (2LL * split <= target && split < 256) split *= 2;
  }
  split = std::max(split, ceil_div(max_pages, kMaxSplits));
  split = ceil_div(split, pps) * pps;
  const int max_splits = ceil_div(max_pages, split);
  long long n_items = 0;
  for (int b = 0; b < nseq; ++b)
    for (int k = 0; k < H; ++k) {
      const int lo = h->cls[layer * H + k] ? 0 : std::max(0, q_pos[b] - h->cfg.window + 1);
      n_items += ceil_div(q_pos[b] / P - lo / P + 1, split);
    }
  const size_t nsplit_off = kHeaderBytes + sizeof(DecodeSeq) * nseq;
  const size_t items_off = align_up(nsplit_off + 4 * (size_t)nseq * H, 16);
  const size_t meta_bytes = items_off + 8 * (size_t)n_items;
  const size_t part_o_off = align_up(meta_bytes, 256);
  const size_t part_lse_off = part_o_off + align_up(4 * (size_t)nseq * Hq * max_splits * D, 256);
  const size_t need = part_lse_off + 4 * (size_t)nseq * Hq * max_splits;
  if (meta_bytes > kNoAllocMetaBytes || need > kNoAllocScratchBytes) {
    h->last_error = "decode needs " + std::to_string(need) + " bytes of scratch (metadata " +
                    std::to_string(meta_bytes) + "); the fixed scratch holds " +
                    std::to_string(kNoAllocScratchBytes) + " (metadata " + std::to_string(kNoAllocMetaBytes) + ")";
    return SEGKV_ERR_WORKSPACE;
  }
  void *scratch = nullptr;
  if ((rc = noalloc_scratch(h, &scratch))) return rc;
  // metadata: zeroed header (the scheduler counter), sequence table, split counts, items
  unsigned char *host = g_noalloc_meta;
  std::memset(host, 0, items_off);
  DecodeSeq *ds = reinterpret_cast<DecodeSeq *>(host + kHeaderBytes);
  int32_t *ns = reinterpret_cast<int32_t *>(host + nsplit_off);
  int2 *it = reinterpret_cast<int2 *>(host + items_off);
  long long w = 0;
  for (int b = 0; b < nseq; ++b) {
    ds[b] = DecodeSeq{seq_ids[b], q_pos[b], h->len[(size_t)layer * h->cfg.max_seqs + seq_ids[b]], 0};
    for (int k = 0; k < H; ++k) {
      const bool global = h->cls[layer * H + k] != 0;
      const int lo = global ? 0 : std::max(0, q_pos[b] - h->cfg.window + 1);
      const int n = ceil_div(q_pos[b] / P - lo / P + 1, split);
      ns[(size_t)b * H + k] = n;
      for (int s = 0; s < n; ++s) it[w++] = make_int2(b, (int)make_item_w1(global, k, s));
    }
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  // a copy from pageable memory has read the host buffer when it returns
  SEGKV_CUDA(h, "scratch metadata upload", cudaMemcpyAsync(scratch, host, meta_bytes, cudaMemcpyHostToDevice, st));
  DecodeLaunch p{};  // zeroed: fields a path does not set (the step append) stay off
  p.g = geom(h);
  p.layer = layer;
  p.nseq = nseq;
  p.n_items = (int)n_items;
  p.split_pages = split;
  p.max_splits = max_splits;
  p.grid = std::min<int>((int)n_items, h->num_sms);
  p.ws_meta = scratch;
  p.nsplit_off = (int)nsplit_off;
  p.items_off = (int)items_off;
  p.part_o = reinterpret_cast<float *>(static_cast<char *>(scratch) + part_o_off);
  p.part_lse = reinterpret_cast<float *>(static_cast<char *>(scratch) + part_lse_off);
  p.q = q;
  p.out = out;
  p.lse = lse;
  p.visited = reinterpret_cast<unsigned long long *>(visited);
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)D);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.newk = nullptr;  // a plain decode: no token to append
  SEGKV_CUDA(h, "decode launch", launch_decode(p, h->kmap, h->vmap, st));
  return SEGKV_OK;
}
extern "C" int segkv_decode_attn_noalloc(segkv_t *h, int layer, int nseq, const int32_t *seq_ids,
                                         const int32_t *q_pos, const void *q, float softmax_scale, int num_splits,
                                         void *out, float *lse, uint64_t *visited, void *stream) {
  return traced("segkv_decode_attn_noalloc", h, [&] { return segkv_decode_attn_noalloc_impl(h, layer, nseq, seq_ids, q_pos, q, softmax_scale, num_splits, out, lse, visited, stream); });
}
