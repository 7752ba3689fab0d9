// storage.cu -- per-head page tables and the KV append/scatter.
//
// The storage itself follows the pages' "per-(layer, head) segmented paged KV storage that
// physically stores only the tokens each head actually needs" (zhichai.net news item,
// "What Happened", item 3): a global head's page list grows with the sequence; a local
// head's list is a ring of R slots, so only the last R logical pages are ever stored.
#include <algorithm>

#include "device_common.cuh"

namespace skv {

// ---------------------------------------------------------------------------- reset
__global__ void __launch_bounds__(256) reset_kernel(int32_t *__restrict__ pt, long long n, int32_t *state) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) pt[i] = -1;
  if (blockIdx.x == 0 && threadIdx.x < 4) state[threadIdx.x] = 0;
}

cudaError_t launch_reset(const StorageGeom &g, int num_layers, cudaStream_t st) {
  const long long n = (long long)num_layers * g.max_seqs * g.hkv * g.max_lp;
  int grid = (int)((n + 255) / 256);
  if (grid > 1184) grid = 1184;
  if (grid < 1) grid = 1;
  reset_kernel<<<grid, 256, 0, st>>>(g.page_table, n, g.state);
  return cudaGetLastError();
}

// Logical page range [lp0, lp1] a call touches for one head: a global head every page
// of [first, last]; a local head only the last R pages ending at the call's last token.
__device__ __forceinline__ void touched_pages(int first, int last, int P, int R, bool global, int &lp0, int &lp1) {
  lp1 = last / P;
  lp0 = first / P;
  if (!global && lp1 - R + 1 > lp0) lp0 = lp1 - R + 1;
}

// ---------------------------------------------------------------------------- append

// ---------------------------------------------------------------------------- copy on write
// One thread per (job, row, 16-byte chunk): job j = (k_new, k_old, rows) copies rows
// [0, rows) of K and V from the page at free-list entry k_old (shared with another sequence
// after a fork) to the fresh page at entry k_new.  It runs before the append kernel on the
// same stream; the rows it writes lie before the call's first token on that page, so the
// two kernels never write the same row.
__global__ void __launch_bounds__(256) cow_copy_kernel(StorageGeom g, const int4 *__restrict__ jobs,
                                                       long long total) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int CH = g.head_dim / 8, P = g.page;
  const int c = (int)(i % CH);
  const int r = (int)((i / CH) % P);
  const int4 e = jobs[i / ((long long)CH * P)];
  if (r >= e.z) return;
  const int32_t dst = (e.x >= 0 && e.x < g.num_pages) ? g.free_list[e.x] : -1;
  const int32_t src = (e.y >= 0 && e.y < g.num_pages) ? g.free_list[e.y] : -1;
  if (dst < 0 || dst >= g.num_pages || src < 0 || src >= g.num_pages) {
    set_error(g.state, kErrDeviceBounds);
    return;
  }
  uint4 *kp = reinterpret_cast<uint4 *>(g.k_pool);
  uint4 *vp = reinterpret_cast<uint4 *>(g.v_pool);
  const long long from = ((long long)src * P + r) * CH + c, to = ((long long)dst * P + r) * CH + c;
  kp[to] = kp[from];
  vp[to] = vp[from];
}

// ---------------------------------------------------------------------------- scatter
// One thread per (token, KV head, 16-byte chunk).  Without a plan (plan == NULL: no page of
// the call is shared), a page the call allocates takes free-list entry
// cursor0 + pair_off[sequence, head] + new_page_rank (pair_off: pages the call allocates for
// earlier (sequence, head) pairs).  Otherwise the host lists every page the call touches, in
// the allocation order (sequence in call order, head ascending, logical page ascending):
// plan[pair_off[sequence, head] + (lp - lp0)] = the free-list entry the page takes (its slot
// was empty, or held a page shared after a fork, whose rows before the call were copied by
// cow_copy_kernel), or -1 (the slot's page is this sequence's alone: written in place).
// Each thread resolves its page, records a new id in the page table (the threads of one
// page write the same value) and moves its K and V chunk with 16-byte stores.  The thread
// holding the call's last token zeroes the rest of a page the call started or took, so
// every stored page holds finite values in every row.  Block 0 advances the allocation
// cursor.
__global__ void __launch_bounds__(256) append_kernel(StorageGeom g, int layer, const AppendSeq *__restrict__ seqs,
                                                     int nseq, const uint8_t *__restrict__ cls,
                                                     const int32_t *__restrict__ pair_off,
                                                     const int32_t *__restrict__ plan, int cursor0, int new_pages,
                                                     long long total, const uint4 *__restrict__ k_new,
                                                     const uint4 *__restrict__ v_new) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i == 0) g.state[0] = cursor0 + new_pages;
  if (i >= total) return;
  const int CH = g.head_dim / 8, H = g.hkv, P = g.page, R = g.ring;
  const int c = (int)(i % CH);
  const long long th = i / CH;
  const int h = (int)(th % H);
  const int t = (int)(th / H);
  int lo = 0, hi = nseq - 1;  // last sequence with tok_off <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (seqs[mid].tok_off <= t) lo = mid; else hi = mid - 1;
  }
  const AppendSeq s = seqs[lo];
  const int pos = s.start + (t - s.tok_off);
  const int first = s.start, last = s.start + s.count - 1;
  const bool global = cls[h] != 0;
  const int lp = pos / P, lp1 = last / P;
  int lp0 = first / P;
  if (!global && lp1 - R + 1 > lp0) lp0 = lp1 - R + 1;
  if (lp < lp0) return;  // the ring keeps only the last R pages
  const int slot = global ? lp : lp % R;
  int32_t *pt = g.page_table + ((((long long)layer * g.max_seqs + s.seq_id) * H + h) * g.max_lp + slot);
  int k;  // free-list entry of a page the call takes, else -1
  if (plan) {
    k = plan[pair_off[lo * H + h] + (lp - lp0)];
  } else {
    const int held = (s.start + P - 1) / P;
    const int rank = new_page_rank(lp, lp0, global ? held : min(held, R), global, R);
    k = rank >= 0 ? cursor0 + pair_off[lo * H + h] + rank : -1;
  }
  int32_t phys;
  if (k >= 0) {
    phys = k < g.num_pages ? g.free_list[k] : -1;
    if (phys >= 0 && phys < g.num_pages && c == 0) *pt = phys;
  } else {
    phys = *pt;
  }
  if (phys < 0 || phys >= g.num_pages) {
    set_error(g.state, kErrDeviceBounds);
    return;
  }
  uint4 *kp = reinterpret_cast<uint4 *>(g.k_pool);
  uint4 *vp = reinterpret_cast<uint4 *>(g.v_pool);
  const long long row = (long long)phys * P;
  kp[(row + pos % P) * CH + c] = k_new[th * CH + c];
  vp[(row + pos % P) * CH + c] = v_new[th * CH + c];
  const bool started = s.start == 0 || (s.start - 1) / P != lp;
  if (pos == last && (last + 1) % P != 0 && (started || k >= 0)) {
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int r = last % P + 1; r < P; ++r) {
      kp[(row + r) * CH + c] = z;
      vp[(row + r) * CH + c] = z;
    }
  }
}

cudaError_t launch_append(const StorageGeom &g, int layer, const void *ws_meta, int nseq, const uint8_t *cls_dev,
                          const int32_t *pair_off_dev, const int32_t *plan_dev, const int4 *jobs_dev, int n_jobs,
                          int cursor0, int new_pages, int total_tokens, const void *k_new, const void *v_new,
                          cudaStream_t st) {
  if (n_jobs > 0) {
    const long long copies = (long long)n_jobs * g.page * (g.head_dim / 8);
    cow_copy_kernel<<<(int)((copies + 255) / 256), 256, 0, st>>>(g, jobs_dev, copies);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const AppendSeq *seqs = reinterpret_cast<const AppendSeq *>(static_cast<const char *>(ws_meta) + kHeaderBytes);
  const long long total = (long long)total_tokens * g.hkv * (g.head_dim / 8);
  const int grid = (int)std::max<long long>(1, (total + 255) / 256);
  append_kernel<<<grid, 256, 0, st>>>(g, layer, seqs, nseq, cls_dev, pair_off_dev, plan_dev, cursor0, new_pages,
                                      total, reinterpret_cast<const uint4 *>(k_new),
                                      reinterpret_cast<const uint4 *>(v_new));
  return cudaGetLastError();
}

}  // namespace skv
