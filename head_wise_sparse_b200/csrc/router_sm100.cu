// router_sm100.cu -- attention as a router: the attention mass every token of a prefill call
// receives, and the k highest-scoring tokens of each sequence.
//
// What it computes (zhichai.net news item "What Happened", item 2: the dense FFN runs only on
// the top-k tokens by attention score, the other tokens take an identity path; hysenlabs.com
// write-up, "The Three Core Mechanisms in Detail", second mechanism: token-level importance
// scores choose the tokens that enter the FFN):
//   score[j] = sum over query heads h and over the call's queries i that see token j of
//              exp(scale q_{i,h}.k_j - lse_{i,h}),
// with lse from the prefill of the same queries; only the call's own tokens are scored.
//
// router_kernel.  Work item = (sequence, KV head, key tile of 128 absolute positions, chunk
// of query tiles).  S^T = K Q^T on the tensor cores: the key tile is the A operand (M = 128,
// so TMEM lane = key) and a query tile -- the G query heads of the KV head over 128/G
// consecutive positions -- the B operand (N = 128).  Each thread of the four reducing warps
// owns one key and sums its TMEM row of weights in registers: no cross-thread reduction.
// One exponential per visible pair bounds the kernel; the dot products ride the tensor core.
// CTA of 640 threads (96 registers each):
//   warp 0      producer: the key tile once per item into one of two buffers (pages resolved
//               through the head's page table), then the item's query tiles through a
//               4-deep ring, each with the 128 negated lse values of its columns (log2
//               domain, loaded one tile ahead; -inf marks a column past the sequence's
//               queries, whose weight is then exactly 0)
//   warp 1      lane 0 issues the MMAs into four 128-column S buffers in TMEM
//   warps 2, 3  idle
//   warps 4..19 four warps per TMEM lane quadrant, each summing 32 of the 128 columns of
//               its 32 keys (one key per thread); a key's sums over the item go to the
//               item's partial slot [chunk][column group][KV head][token], so the result
//               does not depend on the schedule
// score_sum_kernel.  One thread per token adds its partials in a fixed order (slot, then
// KV head) and writes the score.
// topk_kernel.  One CTA per sequence finds the k-th largest score by a radix select over
// the float bits (scores are >= 0, so their bit patterns are ordered like their values),
// and writes the selected rows in ascending order -- equal scores at the threshold by lower
// position -- with block scans.
#include <algorithm>

#include "device_common.cuh"

namespace skv {

namespace {

constexpr int kRKeys = 128;     // keys of a tile (M of the MMA, TMEM lanes)
constexpr int kRCols = 128;     // query rows of a tile (N of the MMA)
constexpr int kRStages = 4;     // query-tile ring depth
constexpr int kRSBufs = 4;      // S buffers in TMEM (4 x 128 columns: all of it)
constexpr int kRReducers = 4 * kRouterColGroups;  // reducing warps: kRouterColGroups per lane quadrant
constexpr int kRGroupCols = kRCols / kRouterColGroups;
constexpr int kRThreads = 128 + 32 * kRReducers;
static_assert(kRGroupCols % 32 == 0, "whole 32-column TMEM loads");
// With two groups (384 threads, 168 registers a thread at launch) the first warpgroup drops
// to 104 registers (the producer needs that many without spilling) and the two reducing
// warpgroups rise to 200: 128 x 104 + 256 x 200 = 64512 = 384 x 168.
constexpr bool kRSplitRegs = kRouterColGroups == 2;
constexpr int kRRegsLaunch = (65536 / kRThreads) / 8 * 8;
constexpr int kRRegsLow = 104, kRRegsHigh = (kRRegsLaunch * kRThreads - 128 * kRRegsLow) / 256 / 8 * 8;
static_assert(!kRSplitRegs || (kRRegsHigh == 200 && 128 * kRRegsLow + 256 * kRRegsHigh <= kRRegsLaunch * kRThreads),
              "register split exceeds the launch total");
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct RSmem {
  static constexpr int kTileBytes = kRKeys * D * 2;  // a K tile and each Q tile (128 rows)
  static constexpr int kQOff = 2 * kTileBytes;
  static constexpr int kLseOff = kQOff + kRStages * kTileBytes;
  static constexpr int kBarOff = kLseOff + kRStages * kRCols * 4;
  static constexpr int kBytes = 1024 + kBarOff + 512;
};

struct RBars {
  uint64_t k_full[2], k_empty[2];
  uint64_t q_full[kRStages], q_empty[kRStages], l_full[kRStages], l_empty[kRStages];
  uint64_t s_full[kRSBufs], s_empty[kRSBufs];
  uint64_t mma_done;
  uint64_t sched_full[4], sched_empty[4];
  int sched[4];
  uint32_t tmem_base;
  int abort_flag;
};

struct RItem {
  int b, h, kt, t0, nt, chunk, q_start, q_end, q_row0, seq_id, kv_len, k_lo;
  bool global;
};

__device__ __forceinline__ RItem decode_ritem(const RouterLaunch &p, const RouterSeq *seqs, const int4 *items,
                                              int idx) {
  const int4 w = items[idx];
  RItem it;
  it.b = w.x;
  const uint32_t w1 = (uint32_t)w.y;
  it.h = item_head(w1);
  it.kt = item_tile(w1);
  it.global = item_global(w1);
  it.t0 = w.z;
  it.nt = w.w & 0xFFFFF;
  it.chunk = (int)((uint32_t)w.w >> 20);
  const RouterSeq s = seqs[it.b];
  it.seq_id = s.seq_id;
  it.q_start = s.q_start;
  it.q_end = s.q_start + s.q_len;
  it.q_row0 = s.q_row0;
  it.kv_len = s.kv_len;
  it.k_lo = max(it.kt * kRKeys, s.q_start);  // query tile 0 starts at the tile's first scored key
  return it;
}

// ---------------------------------------------------------------------------- producer warp
template <int D>
__device__ __forceinline__ void router_producer(const CUtensorMap &qmap, const CUtensorMap &kmap,
                                                const RouterLaunch &p, RBars *bar, const RouterSeq *seqs,
                                                const int4 *items, uint8_t *k_s, uint8_t *q_s, float *lse_s,
                                                int *sched_next, int lane, int G, int32_t *state,
                                                volatile int *abort_flag) {
  using S = RSmem<D>;
  if (lane == 0) {
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&kmap);
  }
  const int P = p.g.page, PPT = kRKeys / P;
  int i = 0, qc = 0, k_loads = 0;
  bool ok = true;
  for (;;) {
    int idx = 0;
    if (lane == 0) idx = atomicAdd(sched_next, 1);
    idx = __shfl_sync(0xffffffffu, idx, 0);
    if (idx >= p.n_items) idx = -1;
    const int slot = i & 3;
    if (!(ok = warp_wait(&bar->sched_empty[slot], ((i >> 2) & 1) ^ 1, abort_flag, state))) break;
    if (lane == 0) {
      bar->sched[slot] = idx;
      mbar_arrive(&bar->sched_full[slot]);
    }
    if (idx < 0) {
      // no item left for this CTA: the partial-sum kernel may start its CTAs (they wait for
      // this grid to complete before reading the partials)
      if (lane == 0) pdl_launch_dependents();
      break;
    }
    const RItem it = decode_ritem(p, seqs, items, idx);
    const int kb = i & 1;  // K buffer of this item
    if (!(ok = warp_wait(&bar->k_empty[kb], ((i >> 1) & 1) ^ 1, abort_flag, state))) break;
    // the key tile: pages kt * PPT .. kt * PPT + PPT - 1, one per lane; pages not stored load zeros
    const long long row_base = (((long long)p.layer * p.g.max_seqs + it.seq_id) * p.g.hkv + it.h) * p.g.max_lp;
    const int last_lp = (it.kv_len - 1) / P;
    int pid = p.g.num_pages;
    if (lane < PPT) {
      const int lp = it.kt * PPT + lane;
      const bool stored = lp <= last_lp && (it.global || lp >= last_lp - p.g.ring + 1);
      if (stored) {
        const int32_t v = p.g.page_table[row_base + (it.global ? lp : lp % p.g.ring)];
        if (v >= 0 && v < p.g.num_pages) pid = v;
        else if (lp * P + P - 1 >= it.q_start && lp * P < it.q_end) set_error(state, kErrDeviceBounds);
      }
    }
    if (lane == 0) mbar_expect_tx(&bar->k_full[kb], S::kTileBytes);
    for (int j = 0; j < PPT; ++j) {
      const int phys = __shfl_sync(0xffffffffu, pid, j);
      if (lane == 0)
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_3d(k_s + kb * S::kTileBytes + hh * kRKeys * 128 + j * P * 128, &kmap, &bar->k_full[kb], hh * 64,
                      0, phys);
    }
    ++k_loads;
    // the negated log2-domain lse of column lane + 32 j of query tile t
    auto neg_lse = [&](int t, int j) -> float {
      const int qa = it.k_lo + (it.t0 + t) * p.tile_pos;
      const int col = lane + 32 * j;
      const int pos = qa + (col >> p.g_shift), hq = it.h * G + (col & (G - 1));
      return pos < it.q_end ? -kLog2e * p.lse[(long long)(it.q_row0 + pos - it.q_start) * p.g.hq + hq] : -INFINITY;
    };
    static_assert(kRCols == 128, "four lse values per lane");
    float nl0 = 0.f, nl1 = 0.f, nl2 = 0.f, nl3 = 0.f;
    if (it.nt > 0) {
      nl0 = neg_lse(0, 0);
      nl1 = neg_lse(0, 1);
      nl2 = neg_lse(0, 2);
      nl3 = neg_lse(0, 3);
    }
    for (int t = 0; t < it.nt; ++t, ++qc) {
      const int s = qc % kRStages;
      const uint32_t u = (uint32_t)(qc / kRStages);
      const int qa = it.k_lo + (it.t0 + t) * p.tile_pos;
      if (!(ok = warp_wait(&bar->q_empty[s], (u & 1) ^ 1, abort_flag, state))) break;
      if (!(ok = warp_wait(&bar->l_empty[s], (u & 1) ^ 1, abort_flag, state))) break;
      float *ls = lse_s + s * kRCols;
      ls[lane] = nl0;
      ls[lane + 32] = nl1;
      ls[lane + 64] = nl2;
      ls[lane + 96] = nl3;
      __syncwarp();
      if (t + 1 < it.nt) {  // in flight while the next stage frees up
        nl0 = neg_lse(t + 1, 0);
        nl1 = neg_lse(t + 1, 1);
        nl2 = neg_lse(t + 1, 2);
        nl3 = neg_lse(t + 1, 3);
      }
      if (lane == 0) {
        mbar_arrive(&bar->l_full[s]);
        mbar_expect_tx(&bar->q_full[s], S::kTileBytes);
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_3d(q_s + s * S::kTileBytes + hh * kRCols * 128, &qmap, &bar->q_full[s], hh * 64, it.h * G,
                      it.q_row0 + qa - it.q_start);
      }
    }
    if (!ok) break;
    ++i;
  }
  // drain: no copy of this CTA may still be in flight when it exits
  for (int k = k_loads - 1; k >= 0 && k >= k_loads - 2; --k) mbar_wait_drain(&bar->k_full[k & 1], (uint32_t)(k >> 1) & 1);
  for (int k = qc - 1; k >= 0 && k >= qc - kRStages; --k)
    mbar_wait_drain(&bar->q_full[k % kRStages], (uint32_t)(k / kRStages) & 1);
}

// ---------------------------------------------------------------------------- MMA thread
template <int D>
__device__ __forceinline__ void router_mma(const RouterLaunch &p, RBars *bar, const int4 *items, uint8_t *k_s,
                                           uint8_t *q_s, uint32_t tmem, int32_t *state, volatile int *abort_flag) {
  using S = RSmem<D>;
  constexpr uint32_t kIdesc = idesc_bf16(kRKeys, kRCols, 0, 0);
  constexpr uint32_t kHi = (1024u >> 4) | (1u << 14) | (2u << 29);
  auto desc = [](uint32_t lo) -> uint64_t { return ((uint64_t)kHi << 32) | lo; };
  const uint32_t k_lo = (smem_u32(k_s) >> 4) | (1u << 16);
  const uint32_t q_lo = (smem_u32(q_s) >> 4) | (1u << 16);
  int i = 0, qc = 0;
  bool ok = true;
  for (;;) {
    const int slot = i & 3;
    if (!(ok = mbar_wait(&bar->sched_full[slot], (i >> 2) & 1, abort_flag, state))) break;
    const int idx = bar->sched[slot];
    mbar_arrive(&bar->sched_empty[slot]);
    if (idx < 0) break;
    const int nt = items[idx].w & 0xFFFFF;
    const int kb = i & 1;
    if (!(ok = mbar_wait(&bar->k_full[kb], (i >> 1) & 1, abort_flag, state))) break;
    const uint32_t ka = k_lo + kb * (S::kTileBytes >> 4);
    for (int t = 0; t < nt; ++t, ++qc) {
      const int s = qc % kRStages, buf = qc % kRSBufs;
      if (!(ok = mbar_wait(&bar->q_full[s], (uint32_t)(qc / kRStages) & 1, abort_flag, state))) break;
      if (!(ok = mbar_wait(&bar->s_empty[buf], ((uint32_t)(qc / kRSBufs) & 1) ^ 1, abort_flag, state))) break;
      tc_fence_after();
      const uint32_t qb = q_lo + s * (S::kTileBytes >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        umma_ss(tmem + buf * kRCols, desc(ka + (kk >> 2) * (kRKeys * 128 >> 4) + (kk & 3) * 2),
                desc(qb + (kk >> 2) * (kRCols * 128 >> 4) + (kk & 3) * 2), kIdesc, kk > 0 ? 1u : 0u);
      umma_commit(&bar->s_full[buf]);
      umma_commit(&bar->q_empty[s]);
    }
    if (!ok) break;
    umma_commit(&bar->k_empty[kb]);
    ++i;
  }
  // every MMA issued by this thread must finish before TMEM is released
  umma_commit(&bar->mma_done);
  mbar_wait_drain(&bar->mma_done, 0);
}

// ---------------------------------------------------------------------------- reducing warps
// Warps 4 and up: warp w reads TMEM lane quadrant w mod 4 (32 keys, one per thread) and
// column group (w - 4) / 4 (kRGroupCols of the 128 query columns of each tile).
__device__ __forceinline__ void router_reduce(const RouterLaunch &p, RBars *bar, const RouterSeq *seqs,
                                              const int4 *items, const float *lse_s, uint32_t tmem, int warp,
                                              int lane, int32_t *state, volatile int *abort_flag) {
  constexpr int kHalf = kRGroupCols;
  const int q4 = warp & 3;
  const int half = (warp - 4) >> 2;  // column group
  const int row = q4 * 32 + lane;
  const uint32_t t_lane = tmem + ((uint32_t)(q4 * 32) << 16) + half * kHalf;
  const float sl2 = p.scale_log2;
  const int W = p.g.window;
  int i = 0, qc = 0;
  for (;;) {
    const int slot = i & 3;
    if (!warp_wait(&bar->sched_full[slot], (i >> 2) & 1, abort_flag, state)) break;
    const int idx = bar->sched[slot];
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar->sched_empty[slot]);
    if (idx < 0) break;
    const RItem it = decode_ritem(p, seqs, items, idx);
    const int k0 = it.kt * kRKeys, kp = k0 + row;
    float acc = 0.f;
    bool ok = true;
    for (int t = 0; t < it.nt; ++t, ++qc) {
      const int s = qc % kRStages, buf = qc % kRSBufs;
      if (!(ok = warp_wait(&bar->l_full[s], (uint32_t)(qc / kRStages) & 1, abort_flag, state))) break;
      if (!(ok = warp_wait(&bar->s_full[buf], (uint32_t)(qc / kRSBufs) & 1, abort_flag, state))) break;
      tc_fence_after();
      uint32_t r[kHalf];
#pragma unroll
      for (int j = 0; j < kHalf / 32; ++j)
        tmem_ld32(t_lane + buf * kRCols + 32 * j, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * j]));
      const int qa = it.k_lo + (it.t0 + t) * p.tile_pos, q_last = qa + p.tile_pos - 1;
      // every key of the tile sees every query of the tile, and every column is a query
      const bool full = qa >= k0 + kRKeys - 1 && q_last < it.q_end && (it.global || q_last - k0 < W);
      const float4 *nl = reinterpret_cast<const float4 *>(lse_s + s * kRCols + half * kHalf);
      // pairs of columns through the packed fp32 pipe: one fma.f32x2 forms two exponents, one
      // add.f32x2 adds two weights, so a column costs two issue slots besides its ex2
      const float2 sl2v = make_float2(sl2, sl2);
      float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
      tmem_ld_wait();
      if (full) {
        // (moving a quarter of these exponentials to an FMA-pipe polynomial measured 2 %
        // slower: the loop is bound by issue and latency, not by the MUFU)
#pragma unroll
        for (int c = 0; c < kHalf; c += 4) {
          const float4 l = nl[c / 4];
          const float2 x01 = ffma2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sl2v,
                                   make_float2(l.x, l.y));
          const float2 x23 = ffma2(make_float2(__uint_as_float(r[c + 2]), __uint_as_float(r[c + 3])), sl2v,
                                   make_float2(l.z, l.w));
          a01 = fadd2(a01, make_float2(fast_exp2(x01.x), fast_exp2(x01.y)));
          a23 = fadd2(a23, make_float2(fast_exp2(x23.x), fast_exp2(x23.y)));
        }
      } else {
        // key kp sees query position qpos iff kp <= qpos (and qpos - kp < W for a local head);
        // column c of this group holds position qa + ((col0 + c) >> g_shift), which never
        // decreases with c, so the visible columns are one range [c_lo, c_hi]
        const int col0 = half * kHalf;
        const int c_lo = max(kp - qa, 0) * (1 << p.g_shift) - col0;
        const int c_hi = it.global ? kHalf : min(kp + W - qa, p.tile_pos) * (1 << p.g_shift) - 1 - col0;
        auto w = [&](int c, float x) -> float { return (c >= c_lo && c <= c_hi) ? fast_exp2(x) : 0.f; };
#pragma unroll
        for (int c = 0; c < kHalf; c += 4) {
          const float4 l = nl[c / 4];
          const float2 x01 = ffma2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sl2v,
                                   make_float2(l.x, l.y));
          const float2 x23 = ffma2(make_float2(__uint_as_float(r[c + 2]), __uint_as_float(r[c + 3])), sl2v,
                                   make_float2(l.z, l.w));
          a01 = fadd2(a01, make_float2(w(c, x01.x), w(c + 1, x01.y)));
          a23 = fadd2(a23, make_float2(w(c + 2, x23.x), w(c + 3, x23.y)));
        }
      }
      acc += (a01.x + a01.y) + (a23.x + a23.y);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar->s_empty[buf]);
        mbar_arrive(&bar->l_empty[s]);
      }
    }
    if (!ok) break;
    if (kp >= it.q_start && kp < it.q_end)
      p.part[(((long long)it.chunk * kRouterColGroups + half) * p.g.hkv + it.h) * p.n_tokens + it.q_row0 +
             (kp - it.q_start)] = acc;
    ++i;
  }
}

template <int D>
__global__ void __launch_bounds__(kRThreads, 1)
    router_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                  const RouterLaunch p) {
  using S = RSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *k_s = base;
  uint8_t *q_s = base + S::kQOff;
  float *lse_s = reinterpret_cast<float *>(base + S::kLseOff);
  RBars *bar = reinterpret_cast<RBars *>(base + S::kBarOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const char *meta = static_cast<const char *>(p.ws_meta);
  int *sched_next = const_cast<int *>(reinterpret_cast<const int *>(meta));
  const RouterSeq *seqs = reinterpret_cast<const RouterSeq *>(meta + kHeaderBytes);
  const int4 *items = reinterpret_cast<const int4 *>(meta + p.items_off);
  const int G = p.g.hq / p.g.hkv;
  int32_t *state = p.g.state;
  volatile int *abort_flag = &bar->abort_flag;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar->k_full[b], 1);
      mbar_init(&bar->k_empty[b], 1);
    }
    for (int s = 0; s < kRStages; ++s) {
      mbar_init(&bar->q_full[s], 1);
      mbar_init(&bar->q_empty[s], 1);
      mbar_init(&bar->l_full[s], 1);
      mbar_init(&bar->l_empty[s], kRReducers);
    }
    for (int b = 0; b < kRSBufs; ++b) {
      mbar_init(&bar->s_full[b], 1);
      mbar_init(&bar->s_empty[b], kRReducers);
    }
    mbar_init(&bar->mma_done, 1);
    for (int s = 0; s < 4; ++s) {
      mbar_init(&bar->sched_full[s], 1);
      mbar_init(&bar->sched_empty[s], 1 + kRReducers);  // MMA thread + lane 0 of each reducing warp
    }
    bar->abort_flag = 0;
    set_wait_limit(p.g.wait_limit);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bar->tmem_base, kRSBufs * kRCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp >= 4) {
    if constexpr (kRSplitRegs) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRRegsHigh));
    router_reduce(p, bar, seqs, items, lse_s, tmem, warp, lane, state, abort_flag);
  } else {
    if constexpr (kRSplitRegs) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRRegsLow));
    if (warp == 0) {
      router_producer<D>(qmap, kmap, p, bar, seqs, items, k_s, q_s, lse_s, sched_next, lane, G, state, abort_flag);
    } else if (warp == 1 && lane == 0) {
      router_mma<D>(p, bar, items, k_s, q_s, tmem, state, abort_flag);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kRSBufs * kRCols);
  }
}

// ---------------------------------------------------------------------------- top-k
constexpr int kTopkThreads = 1024;

// Exclusive block scan of one 32-bit value per thread; also returns the block total.
__device__ __forceinline__ uint32_t block_scan_excl(uint32_t v, uint32_t *warp_tot, uint32_t &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = warp_tot[lane];
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    warp_tot[lane] = wi - w;  // exclusive prefix of the warp totals
    if (lane == 31) warp_tot[32] = wi;
  }
  __syncthreads();
  const uint32_t r = incl - v + warp_tot[warp];
  total = warp_tot[32];
  __syncthreads();  // warp_tot is reused by the next call
  return r;
}

// Launched as a programmatic dependent of the router kernel, and top-k as one of this kernel:
// each waits for its primary grid's memory before reading it.
__global__ void __launch_bounds__(64) score_sum_kernel(const float *__restrict__ part, int slots, int hkv,
                                                      int n_tokens, float *__restrict__ scores) {
  pdl_launch_dependents();  // top-k may start its CTAs; it waits for this grid to complete
  pdl_wait_primary();       // the router kernel's partials are complete and visible
  const int t = blockIdx.x * 64 + threadIdx.x;
  if (t >= n_tokens) return;
  const int n = slots * hkv;  // partial j = (slot, head) at part[j * n_tokens + t]
  float s = 0.f;
  int j = 0;
  for (; j + 8 <= n; j += 8) {  // eight loads in flight, added in order
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = part[(long long)(j + e) * n_tokens + t];
#pragma unroll
    for (int e = 0; e < 8; ++e) s += v[e];
  }
  for (; j < n; ++j) s += part[(long long)j * n_tokens + t];
  scores[t] = s;
}

// cache_cap: scores a CTA may keep in dynamic shared memory (a sequence with more tokens
// reads them from global memory in every pass).
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const int4 *__restrict__ meta,
                                                            const float *__restrict__ scores_g,
                                                            int32_t *__restrict__ rows_out, int cache_cap) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_tot[33];
  __shared__ uint32_t sel[2];
  extern __shared__ float cache[];
  const int4 m = meta[blockIdx.x];
  const int row0 = m.x, n = m.y, k = m.z, out0 = m.w;
  const int tid = threadIdx.x;
  if (k <= 0) return;
  pdl_wait_primary();  // the scores of score_sum_kernel are complete and visible
  const float *scores = scores_g + row0;
  if (n <= cache_cap) {
    for (int t = tid; t < n; t += kTopkThreads) cache[t] = scores[t];
    __syncthreads();
    scores = cache;
  }
  if (k >= n) {
    for (int t = tid; t < n; t += kTopkThreads) rows_out[out0 + t] = row0 + t;
    return;
  }
  // radix select of the k-th largest bit pattern, 8 bits per pass from the top
  const int lane = tid & 31;
  uint32_t prefix = 0, mask = 0, remaining = (uint32_t)k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (tid < 256) hist[tid] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kTopkThreads) {  // whole warps take part in the match
      const int t = base + tid;
      const uint32_t u = t < n ? __float_as_uint(scores[t]) : 0u;
      const bool in = t < n && (u & mask) == prefix;
      const uint32_t digit = in ? (u >> shift) & 255u : 256u;
      // lanes with the same digit add once, through their lowest lane
      const uint32_t same = __match_any_sync(0xffffffffu, digit);
      if (in && lane == __ffs(same) - 1) atomicAdd(&hist[digit], (uint32_t)__popc(same));
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns digits 255 - 8 l down to 248 - 8 l; a suffix scan over lanes finds the
      // digit at which the count of larger-or-equal candidates reaches `remaining`
      uint32_t own = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) own += hist[255 - 8 * lane - j];
      uint32_t incl = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t hit = __ballot_sync(0xffffffffu, incl >= remaining);
      const int l = __ffs(hit) - 1;  // the candidates always reach `remaining`
      if (lane == l) {
        uint32_t above = incl - own;
        int d = 255 - 8 * l;
        for (int j = 0; j < 7; ++j, --d) {
          if (above + hist[d] >= remaining) break;
          above += hist[d];
        }
        sel[0] = prefix | ((uint32_t)d << shift);
        sel[1] = remaining - above;
      }
    }
    __syncthreads();
    prefix = sel[0];
    remaining = sel[1];
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t thr = prefix, need_eq = remaining;  // take every score above thr, need_eq equal to it
  // thread tid owns the contiguous run [tid * per, tid * per + per): count its scores above
  // and at the threshold, one block scan of both counts, then write the run's rows in order
  // (a score above the threshold lands after every selected row before it; an equal one
  // only while fewer than need_eq equal ones came before it)
  const int per = (n + kTopkThreads - 1) / kTopkThreads, t0 = tid * per, t1 = min(t0 + per, n);
  uint32_t gt = 0, eq = 0;
  for (int t = t0; t < t1; ++t) {
    const uint32_t u = __float_as_uint(scores[t]);
    gt += u > thr ? 1u : 0u;
    eq += u == thr ? 1u : 0u;
  }
  uint32_t gt_total, eq_total;
  uint32_t gtb = block_scan_excl(gt, warp_tot, gt_total);
  uint32_t eqb = block_scan_excl(eq, warp_tot, eq_total);
  for (int t = t0; t < t1; ++t) {
    const uint32_t u = __float_as_uint(scores[t]);
    if (u > thr) {
      rows_out[out0 + gtb + min(eqb, need_eq)] = row0 + t;
      ++gtb;
    } else if (u == thr) {
      if (eqb < need_eq) rows_out[out0 + gtb + eqb] = row0 + t;
      ++eqb;
    }
  }
}

}  // namespace

int router_smem_bytes(int head_dim) { return head_dim == 64 ? RSmem<64>::kBytes : RSmem<128>::kBytes; }

template <int D>
static cudaError_t launch_router_d(const RouterLaunch &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                                   cudaStream_t st) {
  static bool attr_set = false;
  const int smem = RSmem<D>::kBytes;
  cudaError_t e;
  if (!attr_set) {
    if ((e = cudaFuncSetAttribute(router_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
    attr_set = true;
  }
  router_kernel<D><<<p.grid, kRThreads, smem, st>>>(qmap, kmap, p);
  return cudaGetLastError();
}

cudaError_t launch_router(const RouterLaunch &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                          cudaStream_t st) {
  return p.g.head_dim == 64 ? launch_router_d<64>(p, qmap, kmap, st) : launch_router_d<128>(p, qmap, kmap, st);
}

cudaError_t launch_topk(const float *part, int chunks, int hkv, int n_tokens, const int4 *topk_meta, int nseq,
                        int max_len, float *scores, int32_t *rows_out, cudaStream_t st) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((n_tokens + 63) / 64);
  cfg.blockDim = dim3(64);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, score_sum_kernel, part, chunks, hkv, n_tokens, scores);
  if (e != cudaSuccess) return e;
  // keep up to 16 384 scores (64 KiB) of a sequence in shared memory
  constexpr int kCacheCap = 16384;
  static bool attr_set = false;
  if (!attr_set) {
    if ((e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 4 * kCacheCap))) return e;
    attr_set = true;
  }
  const int cap = std::min(max_len, kCacheCap);
  cfg.gridDim = dim3(nseq);
  cfg.blockDim = dim3(kTopkThreads);
  cfg.dynamicSmemBytes = 4 * cap;
  return cudaLaunchKernelEx(&cfg, topk_kernel, topk_meta, static_cast<const float *>(scores), rows_out, cap);
}

}  // namespace skv
