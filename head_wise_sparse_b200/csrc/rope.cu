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
// One CTA per 8 tokens: each token's D/2 angles are formed and reduced modulo 2 pi in fp64
// (offsets reach 10^5..10^6 positions, where an fp32 angle would be off by a good part of a
// radian), their cos/sin shared through shared memory by all heads; each thread then turns
// two pairs at a time with packed bf16x2 loads and stores.  HBM-bound: it reads and writes
// each query element once.
#include <math.h>

#include "device_common.cuh"

namespace skv {

namespace {

constexpr int kRopeThreads = 256;
constexpr int kRopeTokens = 8;  // tokens per CTA

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

__global__ void __launch_bounds__(kRopeThreads) relocate_q_kernel(RelocateLaunch p, int n_tokens) {
  extern __shared__ float cs_all[];  // per token: [D/2] cos, then [D/2] sin
  const int D = p.head_dim, half = D / 2, G = p.hq / p.hkv;
  const int t0 = blockIdx.x * kRopeTokens;
  const int nt = min(kRopeTokens, n_tokens - t0);
  // the angles: D/2 per token, formed and reduced in fp64
  for (int e = threadIdx.x; e < nt * half; e += blockDim.x) {
    const int tt = e / half, i = e % half;
    const double theta = exp2(-2.0 * i / D * p.log2_base);
    double a = -(double)p.shift[t0 + tt] * theta;
    a -= 6.283185307179586476925 * rint(a * 0.15915494309189533576888);  // reduce to [-pi, pi]
    double sn, cn;
    sincos(a, &sn, &cn);
    cs_all[tt * D + i] = (float)cn;
    cs_all[tt * D + half + i] = (float)sn;
  }
  __syncthreads();
  // 16-byte units: a group is 8 bf16x2 words of one head row -- words 4g..4g+3 of the first
  // half with their partners in the second half (rotate half), or words 8g..8g+7 (interleaved)
  const int gph = D / 16;  // groups per head row
  const int groups = p.hq * gph;
  const uint4 *in4 = reinterpret_cast<const uint4 *>(p.q_in);
  uint4 *out4 = reinterpret_cast<uint4 *>(p.q_out);
#pragma unroll 2
  for (int e = threadIdx.x; e < nt * groups; e += blockDim.x) {
    const int tt = e / groups, r = e % groups;
    const int h = r / gph, g4 = r % gph;
    const int kv = h / G;
    const long long row4 = ((long long)(t0 + tt) * p.hq + h) * (D / 8);
    const int ia = p.interleaved ? 2 * g4 : g4, ib = p.interleaved ? 2 * g4 + 1 : gph + g4;
    uint4 A = in4[row4 + ia], B = in4[row4 + ib];
    if (((p.cls_bits[kv >> 5] >> (kv & 31)) & 1u) == 0) {  // local head: turn; global: copy
      __nv_bfloat162 *a = reinterpret_cast<__nv_bfloat162 *>(&A), *b = reinterpret_cast<__nv_bfloat162 *>(&B);
      const float *cs = cs_all + tt * D;
      if (!p.interleaved) {
#pragma unroll
        for (int k = 0; k < 4; ++k) turn(a[k], b[k], cs, half, 4 * g4 + k, false, a[k], b[k]);
      } else {
        turn(a[0], a[1], cs, half, 4 * g4, true, a[0], a[1]);
        turn(a[2], a[3], cs, half, 4 * g4 + 1, true, a[2], a[3]);
        turn(b[0], b[1], cs, half, 4 * g4 + 2, true, b[0], b[1]);
        turn(b[2], b[3], cs, half, 4 * g4 + 3, true, b[2], b[3]);
      }
    }
    out4[row4 + ia] = A;
    out4[row4 + ib] = B;
  }
}

}  // namespace

cudaError_t launch_relocate_q(const RelocateLaunch &p, int n_tokens, cudaStream_t st) {
  const int grid = (n_tokens + kRopeTokens - 1) / kRopeTokens;
  relocate_q_kernel<<<grid, kRopeThreads, kRopeTokens * p.head_dim * (int)sizeof(float), st>>>(p, n_tokens);
  return cudaGetLastError();
}

}  // namespace skv
