// rope.cu -- query relocation for position-independent reuse of local-head KV.
//
// What it computes ("RedKnot-MLA: Multi-Head Offline-Online Reuse for DeepSeek-V4 Long-
// Context Serving", Summary): documents are prefilled offline at canonical position zero,
// and their local-head KV is reused at serving time by rotating the queries by the negative
// position offset.  A rotary score depends only on the difference of the query's and the
// key's positions, so a query at true position p, rotated by -delta, scores against a key
// cached at canonical position j exactly as against that key at j + delta.  The rotation:
// dimension pairs (i, i + D/2) (or (2i, 2i + 1) when interleaved) turn by the angle
// -delta * theta_i, theta_i = base^(-2i/D).  Global heads (recomputed at true positions)
// pass through unchanged.
//
// One CTA per block of tokens: as many tokens as make 512 16-byte units (two a thread), or
// one token (in passes of 512 units) when a token has more.  The grid holds every block and
// the hardware hands them to SMs as others finish, so the last wave stays short.  Each
// thread first issues the loads of its two units and the block's offsets, and only then are
// the block's angles formed, so the angle work overlaps the loads in flight: each token's D/2
// angles are formed and reduced modulo 2 pi in fp64 (offsets reach 10^5..10^6 positions,
// where an fp32 angle would be off by a good part of a radian), from frequencies the host
// computes in fp64; the reduced angle, within [-pi, pi], then goes to fp32 for its cosine and
// sine, which all heads of the token share through shared memory; each unit turns four pairs.
// HBM-bound: it reads and writes each query element once.
//
// Measured on the Llama-shaped queries (86 326 tokens x 64 heads x 128), this grid ran 16 %
// faster than one sized to the resident CTAs with each CTA taking blocks in turn (whose
// final pass leaves some CTAs with one block more than others), and on 8 192 tokens x 32
// heads as fast as a plain device copy of the same bytes.
#include <math.h>

#include <algorithm>

#include "device_common.cuh"

namespace skv {

namespace {

constexpr int kRopeThreads = 256;
constexpr int kRopeUnits = 2;  // 16-byte units a thread holds at once
constexpr int kRopeBlockUnits = kRopeThreads * kRopeUnits;

// Turns word j of a head row: rotate-half pairs element 2j (+1) with 2j + D/2 (+1); the
// interleaved layout holds the pairs (4j, 4j+1) and (4j+2, 4j+3) in words 2j and 2j+1.
__device__ __forceinline__ void turn(const __nv_bfloat162 a, const __nv_bfloat162 b, const float *cs, int half, int j,
                                     bool interleaved, __nv_bfloat162 &ra, __nv_bfloat162 &rb) {
  const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  const float c0 = cs[2 * j], c1 = cs[2 * j + 1], s0 = cs[half + 2 * j], s1 = cs[half + 2 * j + 1];
  if (!interleaved) {
    ra = __floats2bfloat162_rn(fa.x * c0 - fb.x * s0, fa.y * c1 - fb.y * s1);
    rb = __floats2bfloat162_rn(fb.x * c0 + fa.x * s0, fb.y * c1 + fa.y * s1);
  } else {
    ra = __floats2bfloat162_rn(fa.x * c0 - fa.y * s0, fa.y * c0 + fa.x * s0);
    rb = __floats2bfloat162_rn(fb.x * c1 - fb.y * s1, fb.y * c1 + fb.x * s1);
  }
}

template <int D>
__global__ void __launch_bounds__(kRopeThreads) relocate_q_kernel(RelocateLaunch p, int n_tokens, int tpb) {
  constexpr int half = D / 2;
  // a unit is 8 bf16x2 words of one head row: words 4g..4g+3 of the first half with their
  // partners in the second half (rotate half), or words 8g..8g+7 (interleaved)
  constexpr int gph = D / 16;  // units per head row
  extern __shared__ float cs_all[];                        // per token of the block: [D/2] cos, then [D/2] sin
  __shared__ int32_t shift_s[kRopeBlockUnits / (D / 16)];  // the block's offsets
  const int hq = p.hq;
  const float inv_hq = 1.0f / hq;
  const uint4 *in4 = reinterpret_cast<const uint4 *>(p.q_in);
  uint4 *out4 = reinterpret_cast<uint4 *>(p.q_out);
  const int t0 = blockIdx.x * tpb, nt = min(tpb, n_tokens - t0), units = nt * hq * gph;
  const long long base4 = (long long)t0 * hq * (D / 8);
  // 512 units a pass, more than one pass only when a token has more than 512 units
  // (hq * D > 8 192); the angles are formed while the first pass's loads are in flight
  for (int u0 = 0; u0 < units; u0 += kRopeBlockUnits) {
    uint4 A[kRopeUnits], B[kRopeUnits];
#pragma unroll
    for (int k = 0; k < kRopeUnits; ++k) {
      const int e = u0 + k * kRopeThreads + threadIdx.x;
      if (e < units) {
        const int row = e / gph, g4 = e % gph;  // row: head row of the block (token * hq + head)
        const long long row4 = base4 + (long long)row * (D / 8);
        A[k] = in4[row4 + (p.interleaved ? 2 * g4 : g4)];
        B[k] = in4[row4 + (p.interleaved ? 2 * g4 + 1 : gph + g4)];
      }
    }
    if (u0 == 0) {
      if (threadIdx.x < nt) shift_s[threadIdx.x] = p.shift[t0 + threadIdx.x];
      __syncthreads();
      // the angles: D/2 per token, formed and reduced modulo 2 pi in fp64, cos/sin in fp32
      for (int e = threadIdx.x; e < nt * half; e += blockDim.x) {
        const int tt = e / half, i = e % half;
        double a = -(double)shift_s[tt] * p.theta[i];
        a -= 6.283185307179586476925 * rint(a * 0.15915494309189533576888);  // reduce to [-pi, pi]
        float sn, cn;
        sincosf((float)a, &sn, &cn);
        cs_all[tt * D + i] = cn;
        cs_all[tt * D + half + i] = sn;
      }
      __syncthreads();
    }
#pragma unroll
    for (int k = 0; k < kRopeUnits; ++k) {
      const int e = u0 + k * kRopeThreads + threadIdx.x;
      if (e < units) {
        const int row = e / gph, g4 = e % gph;
        // token and head of the row: row / hq in fp32 is exact here (a block has at most
        // 1 024 rows, so (row + 0.5) / hq < 1 024; with hq <= 1 024 that quotient lies at
        // least 1/2048 from an integer, while the two roundings move it by less than 2^-13)
        const int tt = __float2int_rz(((float)row + 0.5f) * inv_hq), h = row - tt * hq;
        if (((p.cls_bits[h >> 5] >> (h & 31)) & 1u) == 0) {  // local head: turn; global: copy
          __nv_bfloat162 *a = reinterpret_cast<__nv_bfloat162 *>(&A[k]), *b = reinterpret_cast<__nv_bfloat162 *>(&B[k]);
          const float *cs = cs_all + tt * D;
          if (!p.interleaved) {
#pragma unroll
            for (int j = 0; j < 4; ++j) turn(a[j], b[j], cs, half, 4 * g4 + j, false, a[j], b[j]);
          } else {
            turn(a[0], a[1], cs, half, 4 * g4, true, a[0], a[1]);
            turn(a[2], a[3], cs, half, 4 * g4 + 1, true, a[2], a[3]);
            turn(b[0], b[1], cs, half, 4 * g4 + 2, true, b[0], b[1]);
            turn(b[2], b[3], cs, half, 4 * g4 + 3, true, b[2], b[3]);
          }
        }
        const long long row4 = base4 + (long long)row * (D / 8);
        out4[row4 + (p.interleaved ? 2 * g4 : g4)] = A[k];
        out4[row4 + (p.interleaved ? 2 * g4 + 1 : gph + g4)] = B[k];
      }
    }
  }
}

template <int D>
cudaError_t launch_relocate_d(const RelocateLaunch &p, int n_tokens, cudaStream_t st) {
  const int tpb = std::max(1, kRopeBlockUnits / (p.hq * (D / 16)));  // tokens per block
  relocate_q_kernel<D>
      <<<(n_tokens + tpb - 1) / tpb, kRopeThreads, tpb * D * sizeof(float), st>>>(p, n_tokens, tpb);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_relocate_q(const RelocateLaunch &p, int n_tokens, cudaStream_t st) {
  return p.head_dim == 64 ? launch_relocate_d<64>(p, n_tokens, st) : launch_relocate_d<128>(p, n_tokens, st);
}

}  // namespace skv
