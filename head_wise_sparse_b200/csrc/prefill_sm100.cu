// prefill_sm100.cu -- causal variable-length prefill over per-head paged KV storage,
// tcgen05 tensor cores with TMEM accumulators, TMA page loads, persistent LPT scheduling
// (one CTA per SM working through a longest-first list of items).
//
// What it computes (zhichai.net news item "What Happened", item 3): for every query row of
// every head, attention over exactly the keys that head keeps, with the head's visibility
// (global: k <= p; local: p - W < k <= p) decided from positions -- no mask tensor.
//
// Work item = two 128-row query tiles of one (sequence, KV head): each tile packs the G
// query heads of the KV head over 128/G consecutive positions (GQA group packing), and the
// two tiles cover 256/G consecutive positions.  Both tiles share every K/V tile load.
//
// One persistent CTA per SM, 384 threads (three warpgroups; one warp of each per SM
// sub-partition, so the softmax warps can hold a 128-column S row in registers):
//   warp 0      producer: takes the next item of the longest-first list (atomic counter),
//               decodes it once into a shared-memory ring the other roles read, pulls the
//               following item's Q rows into L2, loads both Q tiles, then streams K and V
//               tiles page by page through TMA
//               (a tile of BN = 128 keys is BN/P pages resolved through the head's page table)
//   warp 1      MMA issuer (one thread): for key tile j, per query tile t,
//               O_t += P_t(j-1) V(j-1) in two halves of 64 keys (each issued as soon as
//               the softmax has written that half of P_t(j-1)), then S_t(j) = Q_t K(j)^T,
//               all into TMEM
//   warps 2, 3  idle (they hand their registers to the softmax warpgroups)
//   warps 4..7  softmax of query tile 0, warps 8..11 softmax of query tile 1: one thread per
//               row; fp32 online softmax in the exp2 domain, O rescaled only when the row
//               maximum grows by more than 2^8; P (bf16) overwrites its S columns in TMEM,
//               each half of 64 keys signalled as soon as it is stored;
//               each row counts the key columns its mask keeps (the visited pairs);
//               the epilogue reads O_t out of TMEM (and frees it for the next item at once),
//               normalises it and writes bf16 out through a 128-byte-swizzled shared-memory
//               buffer, each warp storing its own 32 rows by TMA tile stores (64 columns at a
//               time; scattered per-thread row stores would flood the SM's L2 request path
//               that the K/V loads share), plus fp32 lse and visited counts.
// No warp waits at a barrier that another warp must reach after a bounded wait (the only
// block-wide barriers are at the start and the end), so an abort in any role lets every
// other role leave its loop.
// The two query tiles' chains (S -> softmax -> PV -> next S) interleave on the tensor core:
// while one tile's warpgroup runs its softmax, the other tile's MMAs run.
#include "device_common.cuh"

namespace skv {

namespace {

constexpr int kTileRows = 128;  // rows of one query tile (one TMEM accumulator)
constexpr int kBN = 128;        // keys of one key tile
constexpr int kStages = 2;      // K and V ring depth
constexpr int kThreads = 384;
// Registers per thread: 168 at launch (65536 / 384 rounded down to a multiple of 8);
// warpgroup 0 drops to 80 and the two softmax warpgroups rise to 208, which stays within the
// launch total: 128 x 80 + 256 x 208 <= 384 x 168 (setmaxnreg.inc can only take registers
// the block was launched with).
constexpr int kRegsLaunch = (65536 / kThreads) / 8 * 8;
constexpr int kRegsLow = 80, kRegsHigh = (kRegsLaunch * kThreads - 128 * kRegsLow) / 256 / 8 * 8;
static_assert(kRegsHigh == 208 && 128 * kRegsLow + 256 * kRegsHigh <= kRegsLaunch * kThreads,
              "register split exceeds the launch total");
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale when the max grows > 2^8

template <int D>
struct Smem {
  static constexpr int kQTileBytes = kTileRows * D * 2;
  static constexpr int kTileBytes = kBN * D * 2;
  static constexpr int kHalves = D / 64;
  static constexpr int kKOff = 2 * kQTileBytes;
  static constexpr int kVOff = kKOff + kStages * kTileBytes;
  // output staging: one buffer of 128 rows x 64 columns (16 KiB) per softmax warpgroup
  static constexpr int kOStageBytes = kTileRows * 128;
  static constexpr int kOOff = kVOff + kStages * kTileBytes;
  static constexpr int kBarOff = kOOff + 2 * kOStageBytes;
  static constexpr int kBytes = 1024 + kBarOff + 1024;
  // TMEM columns: S_t at 128 t, O_t at 256 + 128 t
  static constexpr uint32_t col_s(int t) { return 128u * t; }
  static constexpr uint32_t col_o(int t) { return 256u + 128u * t; }
};

struct Item {
  int b, h, t, q_first, q_last, lo_min, kt_lo, kt_hi, seq_id, kv_len, q_row, slot;
  int c_start, c_end, c_row0;  // the sequence's query range and its first packed row
  bool global;
};

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_lo[2], p_hi[2], pv_done[2], o_free[2];
  uint64_t mma_done, never;  // never: no one arrives (the stall test waits on it)
  uint64_t sched_full[4], sched_empty[4];
  int sched[4];
  Item sched_item[4];  // the producer decodes each item once; consumers read it here
  uint32_t tmem_base;
  int abort_flag;
};


// Item = (sequence b, KV head h, tile pair t): positions [q_start + 2 t tp, ...) of the
// sequence's queries, tp = 128 / G positions per query tile, over key tiles [kt_lo, kt_hi]
// (the item's whole key range, or one chunk of it when slot >= 0).
__device__ __forceinline__ Item decode_item(const PrefillLaunch &p, const PrefillSeq *seqs, const int4 *items,
                                            int idx) {
  const int4 w = items[idx];
  Item it;
  it.b = w.x;
  const uint32_t w1 = (uint32_t)w.y;
  it.h = item_head(w1);
  it.t = item_tile(w1);
  it.global = item_global(w1);
  const PrefillSeq s = seqs[it.b];
  const int pair = 2 * p.tile_pos;
  it.seq_id = s.seq_id;
  it.kv_len = s.kv_len;
  it.c_start = s.q_start;
  it.c_end = s.q_start + s.q_len;
  it.c_row0 = s.q_row0;
  it.q_first = s.q_start + it.t * pair;
  it.q_last = s.q_start + min((it.t + 1) * pair, s.q_len) - 1;
  it.q_row = s.q_row0 + it.t * pair;
  it.lo_min = it.global ? 0 : max(0, it.q_first - p.g.window + 1);
  it.kt_lo = (int)((uint32_t)w.z >> 16);
  it.kt_hi = w.z & 0xFFFF;
  it.slot = w.w;
  return it;
}

// ---------------------------------------------------------------------------- producer warp
template <int D, bool TWO, bool STORE>
__device__ __forceinline__ void producer_role(const CUtensorMap &qmap, const CUtensorMap &kmap,
                                              const CUtensorMap &vmap, const CUtensorMap &kcmap,
                                              const CUtensorMap &vcmap, const PrefillLaunch &p, Bars *bar,
                                              const PrefillSeq *seqs, const int4 *items, uint8_t *q_s, uint8_t *k_s,
                                              uint8_t *v_s, int *sched_next, int lane, int G, int32_t *state,
                                              volatile int *abort_flag) {
  using S = Smem<D>;
  if (lane == 0) {
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
    if constexpr (TWO) {
      tma_prefetch_desc(&kcmap);
      tma_prefetch_desc(&vcmap);
    }
  }
  const int P = p.g.page, PPT = kBN / P;
  // Two-source prefill (TWO, a template parameter so the one-source kernel carries none of
  // it): a page of the call's own query range comes from the caller's K/V tensors, packed
  // like q; only the context before the range is read from the pages.  Such a page's lane
  // holds -1 - (its first row in those tensors) instead of a page id.
  // Fused append (STORE): the item whose query range holds a chunk page's first position also
  // writes that page from shared memory to its pool page by TMA store, so every chunk page is
  // stored exactly once.  A tile's pages are stored one tile late, after the next tile's loads
  // are issued (by then they have landed, so the producer does not wait for its own loads),
  // with the pool ids worked out while the tile's own item was current; the last tile is
  // stored after the loop.  A stage is reloaded only after the stores that read it have read
  // it (bulk_wait_read_all before each K load).
  int i = 0, c = 0;
  // loads of the current tile / item already issued (bit 0: K, bit 1: V, bit 2: Q): with c and
  // i they say which loads the drain on the way out must wait for
  int issued = 0;
  int sp_prev = -1, c_prev = -1;  // STORE: lane j = pool id of page j of tile c_prev to store, else -1
  // STORE: writes the chunk pages of tile cs (lane j: page j's pool id in sp, else -1)
  auto store_tile = [&](int sp, int cs) -> bool {
    if (cs < 0 || !__ballot_sync(0xffffffffu, sp >= 0)) return true;
    const int st = cs % kStages;
    const uint32_t us = (uint32_t)(cs / kStages);
    if (!warp_wait(&bar->k_full[st], us & 1, abort_flag, state)) return false;
    for (int j = 0; j < PPT; ++j) {
      const int ph = __shfl_sync(0xffffffffu, sp, j);
      if (lane == 0 && ph >= 0)
        for (int hh = 0; hh < S::kHalves; ++hh)
          tma_store_3d(&kmap, k_s + st * S::kTileBytes + hh * kBN * 128 + j * P * 128, hh * 64, 0, ph);
    }
    if (!warp_wait(&bar->v_full[st], us & 1, abort_flag, state)) return false;
    for (int j = 0; j < PPT; ++j) {
      const int ph = __shfl_sync(0xffffffffu, sp, j);
      if (lane == 0 && ph >= 0)
        for (int hh = 0; hh < S::kHalves; ++hh)
          tma_store_3d(&vmap, v_s + st * S::kTileBytes + hh * kBN * 128 + j * P * 128, hh * 64, 0, ph);
    }
    if (lane == 0) bulk_commit();
    return true;
  };
  bool ok = true;
  // next item index, fetched one item ahead so its Q rows can be pulled into L2 early
  auto fetch = [&]() -> int {
    int v = 0;
    if (lane == 0) v = atomicAdd(sched_next, 1);
    v = __shfl_sync(0xffffffffu, v, 0);
    return v < p.n_items ? v : -1;
  };
  int idx = fetch();
  for (;;) {
    const int slot = i & 3;
    Item it;
    if (idx >= 0) it = decode_item(p, seqs, items, idx);
    if (!(ok = warp_wait(&bar->sched_empty[slot], ((i >> 2) & 1) ^ 1, abort_flag, state))) break;
    if (lane == 0) {
      bar->sched[slot] = idx;
      if (idx >= 0) bar->sched_item[slot] = it;
      mbar_arrive(&bar->sched_full[slot]);
    }
    if (idx < 0) break;
    const int next = fetch();
    if (next >= 0 && lane == 0) {
      const Item nt = decode_item(p, seqs, items, next);
      for (int t = 0; t < 2; ++t)
        for (int hh = 0; hh < S::kHalves; ++hh) tma_prefetch_l2_3d(&qmap, hh * 64, nt.h * G, nt.q_row + t * p.tile_pos);
    }
    if (!(ok = warp_wait(&bar->q_empty, (i & 1) ^ 1, abort_flag, state))) break;
    if (lane == 0) {
      mbar_expect_tx(&bar->q_full, 2 * S::kQTileBytes);
      for (int t = 0; t < 2; ++t)
        for (int hh = 0; hh < S::kHalves; ++hh)
          tma_load_3d(q_s + t * S::kQTileBytes + hh * kTileRows * 128, &qmap, &bar->q_full, hh * 64, it.h * G,
                      it.q_row + t * p.tile_pos);
    }
    issued |= 4;
    const long long row_base = (((long long)p.layer * p.g.max_seqs + it.seq_id) * p.g.hkv + it.h) * p.g.max_lp;
    const int last_lp = (it.kv_len - 1) / P;
    int lp_base = -(1 << 30), pid = p.g.num_pages;
    for (int kt = it.kt_lo; kt <= it.kt_hi; ++kt) {
      const int lp_first = kt * PPT;
      if (lp_first < lp_base || lp_first + PPT > lp_base + 32) {
        // resolve 32 logical pages at once, one per lane; pages not stored load zeros
        lp_base = lp_first;
        const int lp = lp_base + lane;
        pid = p.g.num_pages;
        const bool chunk = TWO && lp * P >= it.c_start && lp * P < it.c_end;
        const bool stored = !chunk && lp <= last_lp && (it.global || lp >= last_lp - p.g.ring + 1);
        if (stored) {
          const int32_t v = p.g.page_table[row_base + (it.global ? lp : lp % p.g.ring)];
          if (v >= 0 && v < p.g.num_pages) pid = v;
          else if ((long long)lp * P + P - 1 >= it.lo_min && lp * P <= it.q_last) set_error(state, kErrDeviceBounds);
        }
        if (chunk) pid = -1 - (it.c_row0 + lp * P - it.c_start);
      }
      const int s = c % kStages;
      const uint32_t u = (uint32_t)(c / kStages);
      if (!(ok = warp_wait(&bar->k_empty[s], (u & 1) ^ 1, abort_flag, state))) break;
      if constexpr (STORE) {
        if (lane == 0) bulk_wait_read_all();  // earlier stores from this stage have read it
      }
      if (lane == 0) mbar_expect_tx(&bar->k_full[s], S::kTileBytes);
      for (int j = 0; j < PPT; ++j) {
        const int phys = __shfl_sync(0xffffffffu, pid, lp_first + j - lp_base);
        if (lane == 0)
          for (int hh = 0; hh < S::kHalves; ++hh) {
            uint8_t *dst = k_s + s * S::kTileBytes + hh * kBN * 128 + j * P * 128;
            if (TWO && phys < 0)
              tma_load_3d(dst, &kcmap, &bar->k_full[s], hh * 64, it.h, -1 - phys);
            else
              tma_load_3d(dst, &kmap, &bar->k_full[s], hh * 64, 0, phys);
          }
      }
      issued |= 1;
      if (!(ok = warp_wait(&bar->v_empty[s], (u & 1) ^ 1, abort_flag, state))) break;
      if (lane == 0) mbar_expect_tx(&bar->v_full[s], S::kTileBytes);
      for (int j = 0; j < PPT; ++j) {
        const int phys = __shfl_sync(0xffffffffu, pid, lp_first + j - lp_base);
        if (lane == 0)
          for (int hh = 0; hh < S::kHalves; ++hh) {
            uint8_t *dst = v_s + s * S::kTileBytes + hh * kBN * 128 + j * P * 128;
            if (TWO && phys < 0)
              tma_load_3d(dst, &vcmap, &bar->v_full[s], hh * 64, it.h, -1 - phys);
            else
              tma_load_3d(dst, &vmap, &bar->v_full[s], hh * 64, 0, phys);
          }
      }
      issued |= 2;
      if constexpr (STORE) {
        if (!(ok = store_tile(sp_prev, c_prev))) break;  // the previous tile's pages
        // lane j: page j of this tile, if this item stores it (its id, else -1)
        int sp = -1;
        if (lane < PPT) {
          const int lp = lp_first + lane, pos = lp * P, R = p.g.ring;
          const int lp1 = (it.c_end - 1) / P, held = it.c_start / P;
          if (pos >= it.c_start && pos < it.c_end && pos >= it.q_first && pos <= it.q_last &&
              (it.global || lp >= lp1 - R + 1)) {
            const int lp0 = it.global ? held : max(held, lp1 - R + 1);
            const int rank = new_page_rank(lp, lp0, it.global ? held : min(held, R), it.global, R);
            const long long slot = row_base + (it.global ? lp : lp % R);
            const int k = rank >= 0 ? p.cursor0 + p.pair_off[it.b * p.g.hkv + it.h] + rank : -1;
            const int32_t phys = k >= 0 ? (k < p.g.num_pages ? p.g.free_list[k] : -1) : p.g.page_table[slot];
            if (phys >= 0 && phys < p.g.num_pages) {
              if (k >= 0) p.g.page_table[slot] = phys;
              sp = phys;
            } else {
              set_error(state, kErrDeviceBounds);
            }
          }
        }
        sp_prev = sp;
        c_prev = c;
      }
      ++c;
      issued &= 4;
    }
    if (!ok) break;
    ++i;
    issued = 0;
    idx = next;
  }
  if constexpr (STORE) {
    if (ok) store_tile(sp_prev, c_prev);  // the last tile's pages
  }
  // drain: no copy of this CTA may still be in flight when it exits.  On a stage only the last
  // load issued can still be in flight (each later load of a stage waited for the earlier one
  // to be consumed), likewise for the Q buffer.
  const int k_issued = c + (issued & 1), v_issued = c + ((issued >> 1) & 1), q_issued = i + ((issued >> 2) & 1);
  for (int k = k_issued - 1; k >= 0 && k >= k_issued - kStages; --k)
    mbar_wait_drain(&bar->k_full[k % kStages], (uint32_t)(k / kStages) & 1);
  for (int k = v_issued - 1; k >= 0 && k >= v_issued - kStages; --k)
    mbar_wait_drain(&bar->v_full[k % kStages], (uint32_t)(k / kStages) & 1);
  if (q_issued > 0) mbar_wait_drain(&bar->q_full, (uint32_t)(q_issued - 1) & 1);
  if constexpr (STORE) {
    if (lane == 0) bulk_wait_all();  // the pool holds every stored page before the CTA exits
  }
}

// ---------------------------------------------------------------------------- MMA thread
template <int D>
__device__ __forceinline__ void mma_role(const PrefillLaunch &p, Bars *bar, const PrefillSeq *seqs, const int4 *items,
                                         uint8_t *q_s, uint8_t *k_s, uint8_t *v_s, uint32_t tmem, int32_t *state,
                                         volatile int *abort_flag) {
  using S = Smem<D>;
  constexpr uint32_t kIdescQK = idesc_bf16(kTileRows, kBN, 0, 0);
  constexpr uint32_t kIdescPV = idesc_bf16(kTileRows, D, 0, 1);
  // Matrix descriptors differ only in their low word (start address and leading byte
  // offset); the high word (stride 1024 B, version 1, 128-byte swizzle) is shared.
  constexpr uint32_t kHi = (1024u >> 4) | (1u << 14) | (2u << 29);
  auto desc = [](uint32_t lo) -> uint64_t { return ((uint64_t)kHi << 32) | lo; };
  const uint32_t q_lo = (smem_u32(q_s) >> 4) | (1u << 16);
  const uint32_t k_lo = (smem_u32(k_s) >> 4) | (1u << 16);
  const uint32_t v_lo = (smem_u32(v_s) >> 4) | ((uint32_t)(kBN * 128 >> 4) << 16);
  int i = 0, c = 0;
  // stall test: a wait that runs out before any MMA is issued (nothing arrives on `never`)
  bool ok = !p.stall_test || mbar_wait(&bar->never, 0, abort_flag, state);
  // O_t += P_t(cc) V(cc); the first PV of an item overwrites O_t
  auto issue_pv = [&](int t, int cc, bool first, bool last) -> bool {
    const int s = cc % kStages;
    if (!mbar_wait(&bar->p_lo[t], cc & 1, abort_flag, state)) return false;
    if (t == 0 && !mbar_wait(&bar->v_full[s], (uint32_t)(cc / kStages) & 1, abort_flag, state)) return false;
    if (first && !mbar_wait(&bar->o_free[t], (i & 1) ^ 1, abort_flag, state)) return false;
    tc_fence_after();
    const uint32_t vb = v_lo + s * (S::kTileBytes >> 4);
    const uint32_t d_o = tmem + S::col_o(t), a_p = tmem + S::col_s(t);
    umma_ts(d_o, a_p, desc(vb), kIdescPV, first ? 0u : 1u);
#pragma unroll
    for (int kk = 1; kk < kBN / 32; ++kk) umma_ts(d_o, a_p + kk * 8, desc(vb + kk * 128), kIdescPV, 1u);
    if (!mbar_wait(&bar->p_hi[t], cc & 1, abort_flag, state)) return false;
    tc_fence_after();
#pragma unroll
    for (int kk = kBN / 32; kk < kBN / 16; ++kk) umma_ts(d_o, a_p + kk * 8, desc(vb + kk * 128), kIdescPV, 1u);
    if (last) umma_commit(&bar->pv_done[t]);
    return true;
  };
  // S_t(cc) = Q_t K(cc)^T
  auto issue_s = [&](int t, int cc) {
    const uint32_t kb = k_lo + (cc % kStages) * (S::kTileBytes >> 4);
    const uint32_t qb = q_lo + t * (S::kQTileBytes >> 4);
    const uint32_t d_s = tmem + S::col_s(t);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
      umma_ss(d_s, desc(qb + (kk >> 2) * (kTileRows * 128 >> 4) + (kk & 3) * 2),
              desc(kb + (kk >> 2) * (kBN * 128 >> 4) + (kk & 3) * 2), kIdescQK, kk > 0 ? 1u : 0u);
    umma_commit(&bar->s_full[t]);
  };
  while (ok) {
    const int slot = i & 3;
    if (!(ok = mbar_wait(&bar->sched_full[slot], (i >> 2) & 1, abort_flag, state))) break;
    const int idx = bar->sched[slot];
    const Item it = bar->sched_item[slot];
    mbar_arrive(&bar->sched_empty[slot]);
    if (idx < 0) break;
    const int n_tiles = it.kt_hi - it.kt_lo + 1;
    if (!(ok = mbar_wait(&bar->q_full, i & 1, abort_flag, state))) break;
    for (int j = 0; j < n_tiles && ok; ++j) {
      const int s = c % kStages;
      if (!(ok = mbar_wait(&bar->k_full[s], (uint32_t)(c / kStages) & 1, abort_flag, state))) break;
      tc_fence_after();
      for (int t = 0; t < 2; ++t) {
        if (j > 0 && !(ok = issue_pv(t, c - 1, j == 1, false))) break;
        issue_s(t, c);
      }
      if (!ok) break;
      umma_commit(&bar->k_empty[s]);
      if (j > 0) umma_commit(&bar->v_empty[(c - 1) % kStages]);
      if (j == n_tiles - 1) umma_commit(&bar->q_empty);
      ++c;
    }
    if (!ok) break;
    for (int t = 0; t < 2 && ok; ++t) ok = issue_pv(t, c - 1, n_tiles == 1, true);
    if (!ok) break;
    umma_commit(&bar->v_empty[(c - 1) % kStages]);
    ++i;
  }
  // every MMA issued by this thread must finish before TMEM is released
  umma_commit(&bar->mma_done);
  mbar_wait_drain(&bar->mma_done, 0);
}

// ---------------------------------------------------------------------------- softmax warpgroups
template <int D>
__device__ __forceinline__ void softmax_role(const CUtensorMap &omap, const PrefillLaunch &p, Bars *bar,
                                             const PrefillSeq *seqs, const int4 *items, uint8_t *o_stage,
                                             uint32_t tmem, int warp, int lane, int G, int32_t *state,
                                             volatile int *abort_flag) {
  using S = Smem<D>;
  const int tq = (warp - 4) >> 2;  // query tile of this warpgroup
  const int q4 = warp & 3;         // TMEM lane quadrant of this warp
  const int row = q4 * 32 + lane;
  const uint32_t t_lane = tmem + ((uint32_t)(q4 * 32) << 16);
  const uint32_t t_s = t_lane + S::col_s(tq), t_o = t_lane + S::col_o(tq);
  const float sl2 = p.scale_log2;
  // this warp's 32 rows of its warpgroup's staging buffer, and the first (head, position) of
  // those rows in the tile: the output map's box is the 32 rows one warp stores (min(G, 32)
  // heads x max(1, 32 / G) positions)
  uint8_t *stg = o_stage + tq * Smem<D>::kOStageBytes + q4 * 32 * 128;
  const int box_h = (q4 * 32) % G, box_p = (q4 * 32) / G, warp_last = (q4 * 32 + 31) / G;
  bool stored = false;  // a TMA store of this warp may still be reading its staging rows
  int i = 0, c = 0;
  for (;;) {
    const int slot = i & 3;
    if (!warp_wait(&bar->sched_full[slot], (i >> 2) & 1, abort_flag, state)) break;
    const int idx = bar->sched[slot];
    const Item it = bar->sched_item[slot];
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar->sched_empty[slot]);
    if (idx < 0) break;
    const int n_tiles = it.kt_hi - it.kt_lo + 1;
    const int pos_local = tq * p.tile_pos + row / G, g = row % G;
    const int p_raw = it.q_first + pos_local;
    const bool valid = p_raw <= it.q_last;
    const int pq = min(p_raw, it.q_last);  // rows past the sequence repeat its last query
    const int lo = it.global ? 0 : max(0, pq - p.g.window + 1);
    float m_used = -INFINITY, l = 0.f;
    uint32_t cnt = 0;  // key columns this row's mask keeps
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      if (!(ok = warp_wait(&bar->s_full[tq], c & 1, abort_flag, state))) break;
      tc_fence_after();
      static_assert(kBN == 128, "128-key tiles");
      float s[kBN];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(t_s + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[cc * 32]));
      tmem_ld_wait();
      const int k0 = (it.kt_lo + j) * kBN;
      // warp-uniform branch: only tiles that cut some row's window edge or diagonal mask
      if (__any_sync(0xffffffffu, k0 < lo || k0 + kBN - 1 > pq)) {
        // keep columns a..b of this tile: one unsigned compare per element, and count them
        const int a = lo - k0;
        const unsigned span = (unsigned)(pq - lo);
        uint32_t kept = 0;
#pragma unroll
        for (int jj = 0; jj < kBN; ++jj) {
          const bool keep = (unsigned)(jj - a) <= span;
          s[jj] = keep ? s[jj] : -INFINITY;
          kept += keep ? 1u : 0u;
        }
        cnt += kept;
      } else {
        cnt += kBN;  // every column of the tile is visible to every row of this warp
      }
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = fmax3(s[e], s[8 + e], s[16 + e]);
#pragma unroll
      for (int r = 0; r < 7; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = fmax3(mx8[e], s[24 + 16 * r + e], s[32 + 16 * r + e]);
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], s[120 + e]);
      const float mx = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(fmax3(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7]));
      const float m_new = mx * sl2;
      const bool grow = m_new > m_used + kRescaleThreshold;
      const bool rescale = grow && m_used != -INFINITY;
      if (__any_sync(0xffffffffu, rescale)) {
        const float alpha = rescale ? fast_exp2(m_used - m_new) : 1.0f;
        // 16 columns at a time: the whole S row is live here
#pragma unroll 1
        for (int cc = 0; cc < D / 16; ++cc) {
          uint32_t o[16];
          tmem_ld16(t_o + cc * 16, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st16(t_o + cc * 16, o);
        }
        l *= alpha;
      }
      if (grow) m_used = m_new;
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
      const float2 c2 = make_float2(sl2, sl2), nm2 = make_float2(neg_m, neg_m);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      // P in two halves of 64 keys (each stored as two quarters of 32 keys); the MMA thread
      // starts each half's PV as it lands
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 x = ffma2(make_float2(s[qq * 32 + 2 * e], s[qq * 32 + 2 * e + 1]), c2, nm2);
          const float2 pe = make_float2(fast_exp2(x.x), fast_exp2(x.y));
          acc[e & 3] = fadd2(acc[e & 3], pe);
          pk[e] = pack_bf16x2(pe.x, pe.y);
        }
        tmem_st16(t_s + qq * 16, pk);
        if (qq & 1) {
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(qq == 1 ? &bar->p_lo[tq] : &bar->p_hi[tq]);
        }
      }
      const float2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
      const float2 a = fadd2(a01, a23);
      l += a.x + a.y;
      ++c;
    }
    if (!ok) break;
    // epilogue: the item's last PV into O_t
    if (!warp_wait(&bar->pv_done[tq], (uint32_t)i & 1, abort_flag, state)) break;  // one phase per item
    tc_fence_after();
    const float inv_l = (valid && l > 0.f) ? 1.f / l : 0.f;
    const long long orow = (long long)(it.q_row + pos_local) * p.g.hq + it.h * G + g;
    if (it.slot >= 0) {
      // one chunk of a longer item: O normalised by this chunk's own sum and its lse go to
      // the chunk's slot (float4 columns, rows contiguous), merged by the combine kernel;
      // O streams out of TMEM 32 columns at a time
      float4 *po = reinterpret_cast<float4 *>(p.part_o) + ((long long)it.slot * 2 + tq) * (D / 4) * kTileRows + row;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(t_o + cc * 32, o);
        tmem_ld_wait();
#pragma unroll
        for (int v = 0; v < 8; ++v)
          po[(cc * 8 + v) * kTileRows] =
              make_float4(__uint_as_float(o[4 * v]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                          __uint_as_float(o[4 * v + 2]) * inv_l, __uint_as_float(o[4 * v + 3]) * inv_l);
      }
      tc_fence_before();
      mbar_arrive(&bar->o_free[tq]);
      p.part_lse[((long long)it.slot * 2 + tq) * kTileRows + row] =
          l > 0.f ? (m_used + fast_log2(l)) * 0.69314718055994531f : -INFINITY;
    } else {
      // O leaves TMEM 64 columns at a time, normalised and packed to bf16 on the way
      uint32_t w[D / 2];
#pragma unroll
      for (int hh = 0; hh < D / 64; ++hh) {
        uint32_t o[64];
        tmem_ld32(t_o + hh * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
        tmem_ld32(t_o + hh * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e)
          w[hh * 32 + e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
      }
      tc_fence_before();
      mbar_arrive(&bar->o_free[tq]);  // O_t is read: the next item's first PV may overwrite it
      if (it.q_first + tq * p.tile_pos + warp_last <= it.q_last) {
        // the warp's 32 rows are all real queries: stored by TMA from this warp's staging rows;
        // the last tile of a sequence may run past it (those rows belong to the next
        // sequence) and is stored row by row
#pragma unroll
        for (int hh = 0; hh < D / 64; ++hh) {
          if (stored) {
            if (lane == 0) bulk_wait_read_all();  // the previous store has read these rows
            __syncwarp();
          }
          // row r at r * 128 bytes, 16-byte chunk c at (c ^ (r mod 8)): the 128-byte swizzle
          // the output tensor map expects
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4 *>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                make_uint4(w[hh * 32 + 4 * c], w[hh * 32 + 4 * c + 1], w[hh * 32 + 4 * c + 2], w[hh * 32 + 4 * c + 3]);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&omap, stg, hh * 64, it.h * G + box_h, it.q_row + tq * p.tile_pos + box_p);
            bulk_commit();
          }
          stored = true;
        }
      } else if (valid) {
        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.out) + orow * D);
#pragma unroll
        for (int v = 0; v < D / 8; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
      }
    }
    if (valid && it.slot < 0) p.lse[orow] = (m_used + fast_log2(l)) * 0.69314718055994531f;
    if (p.visited) {
      // the key columns the row's mask kept in the item's key tiles (all of them unless chunked)
      unsigned long long n = valid ? (unsigned long long)cnt : 0ull;
      if (G < 32) {
        for (int off = G; off < 32; off <<= 1) n += __shfl_xor_sync(0xffffffffu, n, off);
        if (lane < G && n) atomicAdd(&p.visited[(long long)it.b * p.g.hq + it.h * G + lane], n);
      } else if (n) {
        atomicAdd(&p.visited[(long long)it.b * p.g.hq + it.h * G + g], n);
      }
    }
    ++i;
  }
  if (lane == 0) bulk_wait_all();  // no store of this warp outlives the CTA
}

template <int D, bool TWO, bool STORE>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap omap,
                   const __grid_constant__ CUtensorMap kcmap, const __grid_constant__ CUtensorMap vcmap,
                   const PrefillLaunch p) {
  using S = Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *q_s = base;
  uint8_t *k_s = base + S::kKOff;
  uint8_t *v_s = base + S::kVOff;
  uint8_t *o_stage = base + S::kOOff;
  Bars *bar = reinterpret_cast<Bars *>(base + S::kBarOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const char *meta = static_cast<const char *>(p.ws_meta);
  int *sched_next = const_cast<int *>(reinterpret_cast<const int *>(meta));
  const PrefillSeq *seqs = reinterpret_cast<const PrefillSeq *>(meta + kHeaderBytes);
  const int4 *items = reinterpret_cast<const int4 *>(meta + p.items_off);
  const int G = p.g.hq / p.g.hkv;
  int32_t *state = p.g.state;
  volatile int *abort_flag = &bar->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bar->q_full, 1);
    mbar_init(&bar->q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar->s_full[t], 1);
      mbar_init(&bar->p_lo[t], 128);
      mbar_init(&bar->p_hi[t], 128);
      mbar_init(&bar->pv_done[t], 1);
      mbar_init(&bar->o_free[t], 128);
    }
    mbar_init(&bar->mma_done, 1);
    mbar_init(&bar->never, 1);
    for (int s = 0; s < 4; ++s) {
      mbar_init(&bar->sched_full[s], 1);
      mbar_init(&bar->sched_empty[s], 9);  // MMA thread + lane 0 of each of the 8 softmax warps
    }
    bar->abort_flag = 0;
    set_wait_limit(p.g.wait_limit);
    fence_mbar_init();
    if (STORE && blockIdx.x == 0) state[0] = p.cursor0 + p.new_pages;
  }
  if (warp == 1) tmem_alloc(&bar->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp >= 4) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    if (lane == 0 && (warp & 3) == 0) tma_prefetch_desc(&omap);
    softmax_role<D>(omap, p, bar, seqs, items, o_stage, tmem, warp, lane, G, state, abort_flag);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    if (warp == 0) {
      producer_role<D, TWO, STORE>(qmap, kmap, vmap, kcmap, vcmap, p, bar, seqs, items, q_s, k_s, v_s, sched_next, lane, G, state,
                       abort_flag);
    } else if (warp == 1 && lane == 0) {
      mma_role<D>(p, bar, seqs, items, q_s, k_s, v_s, tmem, state, abort_flag);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merges the chunks of each split item: lse = log sum_i exp(lse_i), O = sum_i exp(lse_i -
// lse) O_i (each O_i normalised by its own chunk's sum), bf16 out rounded to nearest even.
// One CTA per (group, query tile), one thread per row.
template <int D>
__global__ void __launch_bounds__(kTileRows) prefill_combine_kernel(const PrefillLaunch p) {
  const char *meta = static_cast<const char *>(p.ws_meta);
  const PrefillSeq *seqs = reinterpret_cast<const PrefillSeq *>(meta + kHeaderBytes);
  const int4 gr = reinterpret_cast<const int4 *>(meta + p.groups_off)[blockIdx.x >> 1];
  const int tq = blockIdx.x & 1, row = threadIdx.x;
  const int G = p.g.hq / p.g.hkv, h = item_head((uint32_t)gr.y), tp = item_tile((uint32_t)gr.y);
  const PrefillSeq s = seqs[gr.x];
  const int pos_local = tq * p.tile_pos + row / G, g = row % G;
  if (tp * 2 * p.tile_pos + pos_local >= s.q_len) return;  // past the sequence's last query
  const long long orow = (long long)(s.q_row0 + tp * 2 * p.tile_pos + pos_local) * p.g.hq + h * G + g;
  float m = -INFINITY;
  for (int i = 0; i < gr.w; ++i) m = fmaxf(m, p.part_lse[((long long)(gr.z + i) * 2 + tq) * kTileRows + row]);
  float wsum = 0.f, w[32];  // the planner cuts an item into at most 32 chunks
  const int n = min(gr.w, 32);
  for (int i = 0; i < n; ++i) {
    const float li = p.part_lse[((long long)(gr.z + i) * 2 + tq) * kTileRows + row];
    w[i] = li == -INFINITY ? 0.f : expf(li - m);
    wsum += w[i];
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  const float4 *po = reinterpret_cast<const float4 *>(p.part_o);
  uint2 *dst = reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p.out) + orow * D);
  for (int v = 0; v < D / 4; ++v) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = 0; i < n; ++i) {
      const float4 x = po[(((long long)(gr.z + i) * 2 + tq) * (D / 4) + v) * kTileRows + row];
      a.x += w[i] * x.x;
      a.y += w[i] * x.y;
      a.z += w[i] * x.z;
      a.w += w[i] * x.w;
    }
    dst[v] = make_uint2(pack_bf16x2(a.x * inv, a.y * inv), pack_bf16x2(a.z * inv, a.w * inv));
  }
  p.lse[orow] = m + logf(wsum);
}

}  // namespace

int prefill_smem_bytes(int head_dim) { return head_dim == 64 ? Smem<64>::kBytes : Smem<128>::kBytes; }

template <int D, bool TWO, bool STORE>
static cudaError_t launch_prefill_d(const PrefillLaunch &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                                   const CUtensorMap &vmap, const CUtensorMap &omap, const CUtensorMap &kcmap,
                                   const CUtensorMap &vcmap, cudaStream_t st) {
  static bool attr_set = false;
  const int smem = prefill_smem_bytes(D);
  cudaError_t e;
  if (!attr_set) {
    if ((e = cudaFuncSetAttribute(prefill_kernel<D, TWO, STORE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smem)))
      return e;
    attr_set = true;
  }
  prefill_kernel<D, TWO, STORE><<<p.grid, kThreads, smem, st>>>(qmap, kmap, vmap, omap, kcmap, vcmap, p);
  if (p.n_groups > 0) prefill_combine_kernel<D><<<2 * p.n_groups, kTileRows, 0, st>>>(p);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_prefill_mode(const PrefillLaunch &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                                       const CUtensorMap &vmap, const CUtensorMap &omap, const CUtensorMap &kcmap,
                                       const CUtensorMap &vcmap, cudaStream_t st) {
  if (!p.two_src) return launch_prefill_d<D, false, false>(p, qmap, kmap, vmap, omap, kcmap, vcmap, st);
  if (!p.store) return launch_prefill_d<D, true, false>(p, qmap, kmap, vmap, omap, kcmap, vcmap, st);
  return launch_prefill_d<D, true, true>(p, qmap, kmap, vmap, omap, kcmap, vcmap, st);
}

cudaError_t launch_prefill(const PrefillLaunch &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                           const CUtensorMap &vmap, const CUtensorMap &omap, const CUtensorMap &kcmap,
                           const CUtensorMap &vcmap, cudaStream_t st) {
  return p.g.head_dim == 64 ? launch_prefill_mode<64>(p, qmap, kmap, vmap, omap, kcmap, vcmap, st)
                            : launch_prefill_mode<128>(p, qmap, kmap, vmap, omap, kcmap, vcmap, st);
}

}  // namespace skv
