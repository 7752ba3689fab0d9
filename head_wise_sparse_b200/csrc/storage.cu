// storage.cu -- per-head page tables and the KV append/scatter.
//
// Storage per (layer, KV head), holding only the tokens that head reads (zhichai.net news
// item, "What Happened", item 3): a global head's page list grows with the sequence; a
// local head's list is a ring of R slots, so only the last R logical pages are ever stored.
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

// ---------------------------------------------------------------------------- scatter
// One warp per (sequence of the call, KV head, logical page the call touches): the warp
// resolves the page once and then moves the page's rows of K and V with 16-byte loads and
// stores, up to eight rows of each in flight per lane.  Without a plan (plan == NULL: no
// page of the call is shared), a page the call allocates takes free-list entry
// cursor0 + pair_off[sequence, head] + new_page_rank (pair_off: pages the call allocates for
// earlier (sequence, head) pairs).  Otherwise the host lists every page the call touches, in
// the allocation order (sequence in call order, head ascending, logical page ascending):
// plan[pair_off[sequence, head] + (lp - lp0)] = the free-list entry the page takes (its slot
// was empty, or held a page shared after a fork), or -1 (the slot's page is this sequence's
// alone: written in place); plan_src at the same index = the free-list entry of the shared
// page whose rows before the call's first token the warp copies first (copy on write), or -1.
// While a page is shared every sharer has the same length (sharing comes from a fork, and a
// sharer's first append takes it its own copy), so a sharer that copies the rows before that
// position and a later sharer of the same call that writes the page in place from it on
// touch disjoint rows.
// A local head keeps only the last R pages ending at the call's last token, so pages before
// them have no warp.  The warp holding the call's last page zeroes the rows after its last
// token on a page the call started or took, so every stored page holds finite values in
// every row.  Block (0, 0) advances the allocation cursor.
constexpr int kAppendWarps = 4;  // pages per CTA, one per warp
constexpr int kAppendBatch = 8;  // 16-byte chunks of K (and of V) in flight per lane

__global__ void __launch_bounds__(32 * kAppendWarps) append_kernel(
    StorageGeom g, int layer, const AppendSeq *__restrict__ seqs, int nseq, const uint8_t *__restrict__ cls,
    const int32_t *__restrict__ pair_off, const int32_t *__restrict__ plan, const int32_t *__restrict__ plan_src,
    int cursor0, int new_pages, const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new) {
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) g.state[0] = cursor0 + new_pages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = g.hkv, P = g.page, R = g.ring, CH = g.head_dim / 8;
  const int rows_per_step = 32 / CH, sub = lane / CH, c = lane % CH;  // a warp covers 32 / CH rows a step
  uint4 *kp = reinterpret_cast<uint4 *>(g.k_pool);
  uint4 *vp = reinterpret_cast<uint4 *>(g.v_pool);
  for (int pair = blockIdx.y; pair < nseq * H; pair += gridDim.y) {
    const int b = pair / H, h = pair % H;
    const AppendSeq s = seqs[b];
    if (s.count == 0) continue;
    const int first = s.start, last = s.start + s.count - 1;
    const bool global = cls[h] != 0;
    const int lp1 = last / P;
    int lp0 = first / P;
    if (!global && lp1 - R + 1 > lp0) lp0 = lp1 - R + 1;  // the ring keeps only the last R pages
    const int lp = lp0 + blockIdx.x * kAppendWarps + warp;
    if (lp > lp1) continue;
    const int r0 = max(first - lp * P, 0), r1 = min(last - lp * P, P - 1) + 1;  // rows this call writes
    const int slot = global ? lp : lp % R;
    int32_t *pt = g.page_table + ((((long long)layer * g.max_seqs + s.seq_id) * H + h) * g.max_lp + slot);
    int k;  // free-list entry of a page the call takes, else -1
    if (plan) {
      k = plan[pair_off[pair] + (lp - lp0)];
    } else {
      const int held = (first + P - 1) / P;
      const int rank = new_page_rank(lp, lp0, global ? held : min(held, R), global, R);
      k = rank >= 0 ? cursor0 + pair_off[pair] + rank : -1;
    }
    int32_t phys;
    if (k >= 0) {
      phys = k < g.num_pages ? g.free_list[k] : -1;
      if (phys >= 0 && phys < g.num_pages && lane == 0) *pt = phys;
    } else {
      phys = *pt;
    }
    if (phys < 0 || phys >= g.num_pages) {
      if (lane == 0) set_error(g.state, kErrDeviceBounds);
      continue;
    }
    const long long dst0 = (long long)phys * P;
    // copy on write: rows [0, r0) come from the shared page, in the same pass as the new rows
    const int ks = plan ? plan_src[pair_off[pair] + (lp - lp0)] : -1;
    long long old0 = 0;
    if (ks >= 0) {
      const int32_t old = ks < g.num_pages ? g.free_list[ks] : -1;
      if (old < 0 || old >= g.num_pages) {
        if (lane == 0) set_error(g.state, kErrDeviceBounds);
        continue;
      }
      old0 = (long long)old * P;
    }
    const int rb = ks >= 0 ? 0 : r0;  // first row this warp writes
    const long long src0 = ((long long)s.tok_off + (lp * P - first)) * H + h;  // source row of page row 0
    for (int base = rb; base < r1; base += rows_per_step * kAppendBatch) {
      uint4 kk[kAppendBatch], vv[kAppendBatch];
#pragma unroll
      for (int u = 0; u < kAppendBatch; ++u) {
        const int r = base + u * rows_per_step + sub;
        if (r < r1) {
          const long long from = r < r0 ? (old0 + r) * CH + c : (src0 + (long long)r * H) * CH + c;
          kk[u] = r < r0 ? kp[from] : k_new[from];
          vv[u] = r < r0 ? vp[from] : v_new[from];
        }
      }
#pragma unroll
      for (int u = 0; u < kAppendBatch; ++u) {
        const int r = base + u * rows_per_step + sub;
        if (r < r1) {
          kp[(dst0 + r) * CH + c] = kk[u];
          vp[(dst0 + r) * CH + c] = vv[u];
        }
      }
    }
    const bool started = first == 0 || (first - 1) / P != lp;  // no earlier token of the sequence on the page
    if (lp == lp1 && r1 < P && (started || k >= 0)) {
      const uint4 z = make_uint4(0, 0, 0, 0);
      for (int r = r1 + sub; r < P; r += rows_per_step) {
        kp[(dst0 + r) * CH + c] = z;
        vp[(dst0 + r) * CH + c] = z;
      }
    }
  }
}

cudaError_t launch_append(const StorageGeom &g, int layer, const void *ws_meta, int nseq, const uint8_t *cls_dev,
                          const int32_t *pair_off_dev, const int32_t *plan_dev, const int32_t *plan_src_dev,
                          int cursor0, int new_pages, int max_pages, const void *k_new, const void *v_new,
                          cudaStream_t st) {
  const AppendSeq *seqs = reinterpret_cast<const AppendSeq *>(static_cast<const char *>(ws_meta) + kHeaderBytes);
  const dim3 grid((unsigned)std::max(1, (max_pages + kAppendWarps - 1) / kAppendWarps),
                  (unsigned)std::min(std::max(1, nseq * g.hkv), 65535));
  append_kernel<<<grid, 32 * kAppendWarps, 0, st>>>(g, layer, seqs, nseq, cls_dev, pair_off_dev, plan_dev,
                                                    plan_src_dev, cursor0, new_pages,
                                                    reinterpret_cast<const uint4 *>(k_new),
                                                    reinterpret_cast<const uint4 *>(v_new));
  return cudaGetLastError();
}

}  // namespace skv
