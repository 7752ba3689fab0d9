// storage.cu -- per-head page-table builder and KV append/scatter (north star subsystem (1)).
//
// The storage itself follows the pages' "per-(layer, head) segmented paged KV storage that
// physically stores only the tokens each head actually needs" (zhichai.net news item,
// "What Happened", item 3): a global head's page list grows with the sequence; a local
// head's list is a ring of R slots, so only the last R logical pages are ever stored.
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

// ---------------------------------------------------------------------------- K1: page table
// One CTA.  Enumerates (sequence in call order, KV head ascending, logical page ascending),
// and hands the next free-list id to every unallocated slot, by block-wide prefix sums.
constexpr int kBuildThreads = 1024;
constexpr int kMaxPairs = 8192;

__device__ __forceinline__ int block_excl_scan(int v, int *warp_sums, int &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = (lane < (int)(blockDim.x >> 5)) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;  // inclusive
  }
  __syncthreads();
  const int base = warp ? warp_sums[warp - 1] : 0;
  total = warp_sums[(blockDim.x >> 5) - 1];
  __syncthreads();
  return base + x - v;
}

__global__ void __launch_bounds__(kBuildThreads) build_pages_kernel(StorageGeom g, int layer,
                                                                   const AppendSeq *__restrict__ seqs, int nseq,
                                                                   const uint8_t *__restrict__ cls) {
  __shared__ int prefix[kMaxPairs + 1];
  __shared__ int warp_sums[32];
  __shared__ int s_running;
  const int P = g.page, R = g.ring, H = g.hkv;
  const int pairs = nseq * H;

  // pages each (sequence, head) pair touches, then an exclusive scan over pairs
  int carry = 0;
  for (int base = 0; base < pairs; base += kBuildThreads) {
    const int p = base + threadIdx.x;
    int n = 0;
    if (p < pairs) {
      const AppendSeq s = seqs[p / H];
      if (s.count > 0) {
        int lp0, lp1;
        touched_pages(s.start, s.start + s.count - 1, P, R, cls[p % H] != 0, lp0, lp1);
        n = lp1 - lp0 + 1;
      }
    }
    int total;
    const int ex = block_excl_scan(n, warp_sums, total);
    if (p < pairs) prefix[p] = carry + ex;
    carry += total;
  }
  if (threadIdx.x == 0) {
    prefix[pairs] = carry;
    s_running = 0;
  }
  __syncthreads();
  const int E = prefix[pairs];
  const int cursor0 = g.state[0];

  for (int base = 0; base < E; base += kBuildThreads) {
    const int e = base + threadIdx.x;
    int need = 0;
    int32_t *slot_ptr = nullptr;
    if (e < E) {
      int lo = 0, hi = pairs - 1;  // last pair with prefix <= e
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= e) lo = mid; else hi = mid - 1;
      }
      const int p = lo, h = p % H;
      const AppendSeq s = seqs[p / H];
      const bool global = cls[h] != 0;
      int lp0, lp1;
      touched_pages(s.start, s.start + s.count - 1, P, R, global, lp0, lp1);
      const int lp = lp0 + (e - prefix[p]);
      const int slot = global ? lp : lp % R;
      slot_ptr = g.page_table + ((((long long)layer * g.max_seqs + s.seq_id) * H + h) * g.max_lp + slot);
      need = (*slot_ptr < 0) ? 1 : 0;
    }
    int total;
    const int rank = block_excl_scan(need, warp_sums, total);
    if (need) {
      const int k = cursor0 + s_running + rank;
      if (k < g.num_pages) *slot_ptr = g.free_list[k];
      else set_error(g.state, kErrDeviceBounds);
    }
    __syncthreads();
    if (threadIdx.x == 0) s_running += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) g.state[0] = cursor0 + s_running;
}

// ---------------------------------------------------------------------------- K2: scatter
// One thread per (token, KV head, 16-byte chunk): K and V rows move with 16-byte stores.
// The thread holding a call's last token also zeroes the rest of that page when the call
// started the page, so every stored page holds finite values in every row.
__global__ void __launch_bounds__(256) append_scatter_kernel(StorageGeom g, int layer,
                                                             const AppendSeq *__restrict__ seqs, int nseq,
                                                             const uint8_t *__restrict__ cls, long long total,
                                                             const uint4 *__restrict__ k_new,
                                                             const uint4 *__restrict__ v_new) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
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
  const int last = s.start + s.count - 1;
  const bool global = cls[h] != 0;
  const int lp = pos / P;
  if (!global && lp < last / P - R + 1) return;  // the ring keeps only the last R pages
  const int slot = global ? lp : lp % R;
  const int32_t phys = g.page_table[(((long long)layer * g.max_seqs + s.seq_id) * H + h) * g.max_lp + slot];
  if (phys < 0 || phys >= g.num_pages) {
    set_error(g.state, kErrDeviceBounds);
    return;
  }
  uint4 *kp = reinterpret_cast<uint4 *>(g.k_pool);
  uint4 *vp = reinterpret_cast<uint4 *>(g.v_pool);
  const long long row = (long long)phys * P;
  kp[(row + pos % P) * CH + c] = k_new[th * CH + c];
  vp[(row + pos % P) * CH + c] = v_new[th * CH + c];
  if (pos == last && (last + 1) % P != 0 && (s.start == 0 || (s.start - 1) / P != lp)) {
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int r = last % P + 1; r < P; ++r) {
      kp[(row + r) * CH + c] = z;
      vp[(row + r) * CH + c] = z;
    }
  }
}

cudaError_t launch_append(const StorageGeom &g, int layer, const void *ws_meta, int nseq, const uint8_t *cls_dev,
                          int total_tokens, const void *k_new, const void *v_new, cudaStream_t st) {
  const AppendSeq *seqs = reinterpret_cast<const AppendSeq *>(static_cast<const char *>(ws_meta) + kHeaderBytes);
  build_pages_kernel<<<1, kBuildThreads, 0, st>>>(g, layer, seqs, nseq, cls_dev);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || total_tokens == 0) return e;
  const long long total = (long long)total_tokens * g.hkv * (g.head_dim / 8);
  const int grid = (int)((total + 255) / 256);
  append_scatter_kernel<<<grid, 256, 0, st>>>(g, layer, seqs, nseq, cls_dev, total,
                                              reinterpret_cast<const uint4 *>(k_new),
                                              reinterpret_cast<const uint4 *>(v_new));
  return cudaGetLastError();
}

}  // namespace skv
