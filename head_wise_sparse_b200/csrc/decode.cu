// decode.cu -- split-K decode over per-head paged KV storage plus a log-sum-exp combine
// (one query token per sequence).
//
// One query token per sequence.  A work item is (sequence, KV head, split): a run of
// consecutive logical pages of that head's visible range.  The item's G query heads
// (the GQA group) ride along as the 16 rows of a warp-level tensor-core tile, so every
// K/V byte is read from HBM once for all G heads.  The kernel is HBM-bound; the
// tensor-core instructions keep the arithmetic (8 FLOP per KV byte at G = 8) off the FP32
// pipe, whose rate would sit below the HBM rate.
//
// CTA (persistent, 160 threads): warp 4 streams 64-key stages (K and V pages) through TMA
// into a 6-deep ring; warps 0..3 each take 16 keys of every stage, keep their own running
// max / sum / output, and merge at the end of the item.  The merged partial (output
// normalised by its own sum, and its natural-log lse) goes to the workspace; the combine
// kernel folds the splits of each (sequence, query head).  It is chained to the split
// kernel by programmatic dependent launch, so its CTAs are resident and waiting when the
// split kernel ends.
//
// Decode step: the same kernel also appends the step's token.  Only the item holding a
// head's last page reads the row at q_pos, so that item's producer warp writes the K and V
// rows (and, for a page the token starts, the page-table entry and the zeroed rest of the
// page) before it loads the page; a proxy fence orders those stores before the TMA reads.
#include "device_common.cuh"

namespace skv {

namespace {

constexpr int kKeys = 64;  // keys per stage
constexpr int kStagesDec = 6;
constexpr int kThreadsDec = 160;

template <int D>
struct DSmem {
  static constexpr int kHalfBytes = kKeys * 128;  // one 64-column half of 64 keys
  static constexpr int kKVBytes = kKeys * D * 2;  // K (or V) of one stage
  static constexpr int kStageBytes = 2 * kKVBytes;
  static constexpr int kMergeOff = kStagesDec * kStageBytes;
  static constexpr int kMergeBytes = 4 * 16 * D * 4 + 4 * 16 * 2 * 4;
  static constexpr int kBarOff = kMergeOff + kMergeBytes;
  static constexpr int kBytes = 1024 + kBarOff + 256;
};

struct DBars {
  uint64_t full[kStagesDec], empty[kStagesDec];
  uint64_t sched_full[4], sched_empty[4];
  uint64_t merge[2];  // consumer-wide barriers around the merge of the four warps' partials
  int sched[4];
  int abort_flag;
};

struct DItem {
  int b, h, split, seq_id, q_pos, lo, hi, lp_a, lp_b, n_stages;
  bool global;
};

__device__ __forceinline__ DItem decode_ditem(const DecodeLaunch &p, const DecodeSeq *seqs, const int2 *items,
                                              int idx) {
  const int2 w = items[idx];
  DItem it;
  it.b = w.x;
  const uint32_t w1 = (uint32_t)w.y;
  it.h = item_head(w1);
  it.split = item_tile(w1);
  it.global = item_global(w1);
  const DecodeSeq s = seqs[it.b];
  it.seq_id = s.seq_id;
  it.q_pos = s.q_pos;
  it.hi = s.q_pos;
  it.lo = it.global ? 0 : max(0, s.q_pos - p.g.window + 1);
  const int P = p.g.page;
  it.lp_a = it.lo / P + it.split * p.split_pages;
  it.lp_b = min(it.lp_a + p.split_pages - 1, it.hi / P);
  const int pps = kKeys / P;
  it.n_stages = (it.lp_b - it.lp_a + 1 + pps - 1) / pps;
  return it;
}

// Decode step, producer warp of the item that holds the last page of (sequence, KV head):
// writes the token's K and V rows at q_pos and returns the page's id (num_pages after a
// bad page id, which sets the error word; the TMA then reads zeros).
template <int D>
__device__ int step_append(const DecodeLaunch &p, const DItem &it, long long row_base, int lane, int32_t *state) {
  constexpr int CH = D / 8;
  const int P = p.g.page, pos = it.q_pos, lp = pos / P;
  const long long slot = row_base + (it.global ? lp : lp % p.g.ring);
  const int k = p.newk[it.b * p.g.hkv + it.h];
  int32_t phys;
  if (k >= 0) phys = k < p.g.num_pages ? p.g.free_list[k] : -1;
  else phys = p.g.page_table[slot];
  if (phys < 0 || phys >= p.g.num_pages) {
    if (lane == 0) set_error(state, kErrDeviceBounds);
    return p.g.num_pages;
  }
  if (k >= 0 && lane == 0) p.g.page_table[slot] = phys;
  uint4 *kp = reinterpret_cast<uint4 *>(p.g.k_pool);
  uint4 *vp = reinterpret_cast<uint4 *>(p.g.v_pool);
  const long long src = ((long long)it.b * p.g.hkv + it.h) * CH;
  const long long row = (long long)phys * P + pos % P;
  for (int e = lane; e < 2 * CH; e += 32) {
    if (e < CH) kp[row * CH + e] = static_cast<const uint4 *>(p.k_new)[src + e];
    else vp[row * CH + e - CH] = static_cast<const uint4 *>(p.v_new)[src + e - CH];
  }
  if (pos % P == 0) {  // a page the token starts: the rows after it hold zeros
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int e = lane; e < (P - 1) * CH; e += 32) {
      kp[(row + 1) * CH + e] = z;
      vp[(row + 1) * CH + e] = z;
    }
  }
  fence_async_global();
  __syncwarp();
  return phys;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of (key row kr, 16-byte chunk dc) in a stage's K or V buffer laid out by TMA
// as [D/64 halves][64 keys][128 B] with the 128-byte swizzle (chunk ^= row % 8).
__device__ __forceinline__ uint32_t sw_off(int kr, int dc) {
  return (uint32_t)((dc >> 3) * (kKeys * 128) + kr * 128 + (((dc & 7) ^ (kr & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kThreadsDec, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                        const DecodeLaunch p) {
  using S = DSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *m_o = reinterpret_cast<float *>(base + S::kMergeOff);  // [4][16][D]
  float *m_ml = m_o + 4 * 16 * D;                               // [4][16][2]
  DBars *bar = reinterpret_cast<DBars *>(base + S::kBarOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const char *meta = static_cast<const char *>(p.ws_meta);
  int *sched_next = const_cast<int *>(reinterpret_cast<const int *>(meta));
  const DecodeSeq *seqs = reinterpret_cast<const DecodeSeq *>(meta + kHeaderBytes);
  const int2 *items = reinterpret_cast<const int2 *>(meta + p.items_off);
  const int G = p.g.hq / p.g.hkv;
  const int P = p.g.page;
  int32_t *state = p.g.state;
  volatile int *abort_flag = &bar->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesDec; ++s) {
      mbar_init(&bar->full[s], 1);
      mbar_init(&bar->empty[s], 4);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&bar->sched_full[s], 1);
      mbar_init(&bar->sched_empty[s], 4);
    }
    mbar_init(&bar->merge[0], 128);
    mbar_init(&bar->merge[1], 128);
    bar->abort_flag = 0;
    set_wait_limit(p.g.wait_limit);
    fence_mbar_init();
    if (p.newk && blockIdx.x == 0) state[0] = p.cursor_after;
    pdl_launch_dependents();  // the combine kernel may start its CTAs; they wait for this grid
  }
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
    }
    const int pps = kKeys / P;
    int i = 0, c = 0;
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
      if (idx < 0) break;
      const DItem it = decode_ditem(p, seqs, items, idx);
      const long long row_base = (((long long)p.layer * p.g.max_seqs + it.seq_id) * p.g.hkv + it.h) * p.g.max_lp;
      const int last_lp = it.hi / P;  // every key of the query is stored (host-validated)
      // decode step: the item holding the last page writes the token's row first
      const int last_phys = (p.newk && it.lp_b == last_lp) ? step_append<D>(p, it, row_base, lane, state) : -1;
      int lp_base = -(1 << 30), pid = p.g.num_pages;
      for (int j = 0; j < it.n_stages; ++j) {
        const int lp_first = it.lp_a + j * pps;
        if (lp_first < lp_base || lp_first + pps > lp_base + 32) {
          lp_base = lp_first;
          const int lp = lp_base + lane;
          pid = p.g.num_pages;
          if (last_phys >= 0 && lp == last_lp) {
            pid = last_phys;
          } else if (lp <= it.lp_b) {
            const int32_t v = p.g.page_table[row_base + (it.global ? lp : lp % p.g.ring)];
            if (v >= 0 && v < p.g.num_pages) pid = v;
            else set_error(state, kErrDeviceBounds);
          }
        }
        const int s = c % kStagesDec;
        const uint32_t u = (uint32_t)(c / kStagesDec);
        if (!(ok = warp_wait(&bar->empty[s], (u & 1) ^ 1, abort_flag, state))) break;
        uint8_t *kst = base + s * S::kStageBytes;
        uint8_t *vst = kst + S::kKVBytes;
        if (lane == 0) mbar_expect_tx(&bar->full[s], S::kStageBytes);
        for (int jp = 0; jp < pps; ++jp) {
          const int phys = __shfl_sync(0xffffffffu, pid, lp_first + jp - lp_base);
          if (lane == 0)
            for (int hh = 0; hh < D / 64; ++hh) {
              tma_load_3d(kst + hh * S::kHalfBytes + jp * P * 128, &kmap, &bar->full[s], hh * 64, 0, phys);
              tma_load_3d(vst + hh * S::kHalfBytes + jp * P * 128, &vmap, &bar->full[s], hh * 64, 0, phys);
            }
        }
        ++c;
      }
      if (!ok) break;
      ++i;
    }
    for (int k = c - 1; k >= 0 && k >= c - kStagesDec; --k)
      mbar_wait_drain(&bar->full[k % kStagesDec], (uint32_t)(k / kStagesDec) & 1);
  } else {
    // ------------------------------------------------------------------ consumers
    const float sl2 = p.scale_log2;
    const int qd = lane & 3, r0 = lane >> 2;
    const uint32_t stage0 = smem_u32(base);
    int i = 0, c = 0;
    for (;;) {
      const int slot = i & 3;
      if (!warp_wait(&bar->sched_full[slot], (i >> 2) & 1, abort_flag, state)) break;
      const int idx = bar->sched[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->sched_empty[slot]);
      if (idx < 0) break;
      const DItem it = decode_ditem(p, seqs, items, idx);
      // query fragments: rows = the G query heads of this KV head (rows >= G are zero)
      uint32_t qa[D / 16][4];
      {
        const uint32_t *q32 = static_cast<const uint32_t *>(p.q);
        const long long rowq0 = ((long long)it.b * p.g.hq + it.h * G + r0) * (D / 2);
        const long long rowq1 = rowq0 + 8LL * (D / 2);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          qa[ks][0] = r0 < G ? q32[rowq0 + ks * 8 + qd] : 0u;
          qa[ks][1] = r0 + 8 < G ? q32[rowq1 + ks * 8 + qd] : 0u;
          qa[ks][2] = r0 < G ? q32[rowq0 + ks * 8 + 4 + qd] : 0u;
          qa[ks][3] = r0 + 8 < G ? q32[rowq1 + ks * 8 + 4 + qd] : 0u;
        }
      }
      float acc[D / 8][4];
#pragma unroll
      for (int n = 0; n < D / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
      bool ok = true;
      for (int j = 0; j < it.n_stages; ++j) {
        const int s = c % kStagesDec;
        if (!(ok = warp_wait(&bar->full[s], (uint32_t)(c / kStagesDec) & 1, abort_flag, state))) break;
        const uint32_t kst = stage0 + s * S::kStageBytes;
        const uint32_t vst = kst + S::kKVBytes;
        const int key0 = (it.lp_a * P) + j * kKeys + warp * 16;  // absolute position of key row 0 of this warp
        // S = Q K^T over this warp's 16 keys
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
          const int mat = lane >> 3, rr = lane & 7;
          const int kr = warp * 16 + rr + ((mat >> 1) << 3);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kst + sw_off(kr, 2 * ks + (mat & 1)), b0, b1, b2, b3);
            mma_16816(sc[0], qa[ks], b0, b1);
            mma_16816(sc[1], qa[ks], b2, b3);
          }
        }
        // mask, scale to the log2 domain, online softmax per row
        float x[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int kp = key0 + nt * 8 + 2 * qd + (e & 1);
            x[nt][e] = (kp >= it.lo && kp <= it.hi) ? sc[nt][e] * sl2 : -INFINITY;
          }
        float mx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
        float mx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float ms0 = mn0 == -INFINITY ? 0.f : mn0, ms1 = mn1 == -INFINITY ? 0.f : mn1;
        const float a0 = fast_exp2(m0 - ms0), a1 = fast_exp2(m1 - ms1);
        m0 = mn0;
        m1 = mn1;
        float pr[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          pr[nt][0] = fast_exp2(x[nt][0] - ms0);
          pr[nt][1] = fast_exp2(x[nt][1] - ms0);
          pr[nt][2] = fast_exp2(x[nt][2] - ms1);
          pr[nt][3] = fast_exp2(x[nt][3] - ms1);
        }
        l0 = l0 * a0 + pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1];
        l1 = l1 * a1 + pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3];
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          acc[n][0] *= a0;
          acc[n][1] *= a0;
          acc[n][2] *= a1;
          acc[n][3] *= a1;
        }
        const uint32_t pa[4] = {pack_bf16x2(pr[0][0], pr[0][1]), pack_bf16x2(pr[0][2], pr[0][3]),
                                pack_bf16x2(pr[1][0], pr[1][1]), pack_bf16x2(pr[1][2], pr[1][3])};
        // O += P V over the same 16 keys
        {
          const int mat = lane >> 3, rr = lane & 7;
          const int kr = warp * 16 + rr + ((mat & 1) << 3);
#pragma unroll
          for (int dn = 0; dn < D / 8; dn += 2) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vst + sw_off(kr, dn + (mat >> 1)), b0, b1, b2, b3);
            mma_16816(acc[dn], pa, b0, b1);
            mma_16816(acc[dn + 1], pa, b2, b3);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->empty[s]);
        ++c;
      }
      // on abort the warp still passes both named barriers below, so no warp waits for it
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      // merge the four warps' partial results of this item
      float *mo = m_o + warp * 16 * D;
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        mo[r0 * D + n * 8 + 2 * qd] = acc[n][0];
        mo[r0 * D + n * 8 + 2 * qd + 1] = acc[n][1];
        mo[(r0 + 8) * D + n * 8 + 2 * qd] = acc[n][2];
        mo[(r0 + 8) * D + n * 8 + 2 * qd + 1] = acc[n][3];
      }
      if (qd == 0) {
        m_ml[(warp * 16 + r0) * 2 + 0] = m0;
        m_ml[(warp * 16 + r0) * 2 + 1] = l0;
        m_ml[(warp * 16 + r0 + 8) * 2 + 0] = m1;
        m_ml[(warp * 16 + r0 + 8) * 2 + 1] = l1;
      }
      if (!ok && lane == 0) *abort_flag = 1;
      mbar_arrive(&bar->merge[0]);
      if (!warp_wait(&bar->merge[0], i & 1, abort_flag, state)) break;
      const int t = threadIdx.x;
      const bool all_ok = ok && !*abort_flag;
      for (int e = t; all_ok && e < G * D && e < 16 * D; e += 128) {
        const int r = e / D, d = e % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, m_ml[(w * 16 + r) * 2]);
        float L = 0.f, o = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float mw = m_ml[(w * 16 + r) * 2];
          const float f = mw == -INFINITY ? 0.f : fast_exp2(mw - M);
          L += f * m_ml[(w * 16 + r) * 2 + 1];
          o += f * m_o[(w * 16 + r) * D + d];
        }
        const long long pr_idx = ((long long)it.b * p.g.hq + it.h * G + r) * p.max_splits + it.split;
        p.part_o[pr_idx * D + d] = o / L;
        if (d == 0) p.part_lse[pr_idx] = (M + fast_log2(L)) * 0.69314718055994531f;
      }
      if (t == 0 && all_ok && p.visited) {
        const int k_a = max(it.lo, it.lp_a * P), k_b = min(it.hi, it.lp_b * P + P - 1);
        const unsigned long long cnt = (unsigned long long)(k_b - k_a + 1);
        for (int g = 0; g < G; ++g) atomicAdd(&p.visited[(long long)it.b * p.g.hq + it.h * G + g], cnt);
      }
      mbar_arrive(&bar->merge[1]);
      if (!warp_wait(&bar->merge[1], i & 1, abort_flag, state) || !all_ok) break;
      ++i;
    }
  }
  __syncthreads();
}

// Folds the splits of each (sequence, query head): lse = m + ln(sum exp(lse_i - m)),
// out = sum exp(lse_i - lse) * out_i, rounded once to bf16.
template <int D>
__global__ void __launch_bounds__(128) lse_combine_kernel(const DecodeLaunch p, const int32_t *__restrict__ nsplit) {
  pdl_wait_primary();  // the split kernel's partials are complete and visible
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.nseq * p.g.hq) return;
  const int b = row / p.g.hq, hq = row % p.g.hq;
  const int G = p.g.hq / p.g.hkv;
  const int ns = nsplit[b * p.g.hkv + hq / G];
  const float *pl = p.part_lse + (long long)row * p.max_splits;
  float M = -INFINITY;
  for (int i = lane; i < ns; i += 32) M = fmaxf(M, pl[i]);
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float sum = 0.f;
  for (int i = lane; i < ns; i += 32) sum += expf(pl[i] - M);
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float lse = M + logf(sum);
  constexpr int PER = D / 32;
  float o[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) o[k] = 0.f;
  const float *po = p.part_o + (long long)row * p.max_splits * D;
  for (int i = 0; i < ns; ++i) {
    const float w = expf(pl[i] - lse);
#pragma unroll
    for (int k = 0; k < PER; ++k) o[k] += w * po[(long long)i * D + lane * PER + k];
  }
  __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out) + (long long)row * D + lane * PER;
#pragma unroll
  for (int k = 0; k < PER; ++k) out[k] = __float2bfloat16_rn(o[k]);
  if (lane == 0) p.lse[row] = lse;
}

}  // namespace

int decode_smem_bytes(int head_dim) { return head_dim == 64 ? DSmem<64>::kBytes : DSmem<128>::kBytes; }

template <int D>
cudaError_t launch_decode_d(const DecodeLaunch &p, const CUtensorMap &kmap, const CUtensorMap &vmap, int smem,
                            cudaStream_t st) {
  static bool attr_set = false;
  cudaError_t e;
  if (!attr_set) {
    if ((e = cudaFuncSetAttribute(decode_split_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)))
      return e;
    attr_set = true;
  }
  decode_split_kernel<D><<<p.grid, kThreadsDec, smem, st>>>(kmap, vmap, p);
  if ((e = cudaGetLastError())) return e;
  const int32_t *nsplit =
      reinterpret_cast<const int32_t *>(static_cast<const char *>(p.ws_meta) + p.nsplit_off);
  const int rows = p.nseq * p.g.hq;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((rows + 3) / 4);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, lse_combine_kernel<D>, p, nsplit);
}

cudaError_t launch_decode(const DecodeLaunch &p, const CUtensorMap &kmap, const CUtensorMap &vmap, cudaStream_t st) {
  const int smem = decode_smem_bytes(p.g.head_dim);
  return p.g.head_dim == 64 ? launch_decode_d<64>(p, kmap, vmap, smem, st)
                            : launch_decode_d<128>(p, kmap, vmap, smem, st);
}

}  // namespace skv
