// K Compression Cache entries, as a CTA-wide device routine shared by the
// standalone update kernel and the fused plan kernel.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 2 and Knowl 5; "Sparse Attention Adaptation
// for Long Reasoning" (papernotes.org), key designs 2 and 4:
//   p   = [max | min | avg] of the b pre-RoPE keys of one full block (per channel)
//   y   = W_k[h] . p                          (d_gate x 3d, no bias)
//   out = bf16(RoPE_{n*b}(y))                 (rotate-half, theta_i = base^(-2i/d_gate))
// A call handles up to kKcompGroup consecutive blocks of one (b, h): 16-byte
// loads pool max/min/sum per channel, then one warp per output row of W_k[h]
// (L2-resident) serves all of the group's pooled vectors, then RoPE (angles in
// fp64) and the bf16 store.
#pragma once

#include "seer_device.cuh"
#include "seer_internal.h"

namespace seer {

constexpr int kKcompGroup = 8;   // blocks per group

template <int D, int DG, int NT>
struct KcompSmem {
  static constexpr int CH = D / 8;       // 16-byte chunks per key row
  static constexpr int RG = NT / CH;     // token row groups
  float red[3][RG][D];                   // per row-group max / min / sum
  float pooled[kKcompGroup][3 * D];
  float ys[kKcompGroup][DG];
};

// Number of full blocks of sequence b the cache may hold (bounded by the row length and,
// for a contiguous cache, by its token capacity).
template <int BLK>
__device__ __forceinline__ int kcomp_nfull(const KcompParams& p, int L) {
  int nfull = min(L / BLK, p.NB);
  if (!p.k.paged) {
    const long long cap_blocks = p.k.num_tokens / BLK;
    if (cap_blocks < nfull) nfull = (int)cap_blocks;
  }
  return nfull;
}

template <int D, int BLK, int DG, int NT>
__device__ void kcomp_group(const KcompParams& p, int b, int h, int g0, int ni, KcompSmem<D, DG, NT>& sm) {
  using SM = KcompSmem<D, DG, NT>;
  constexpr int CH = SM::CH, RG = SM::RG, P3 = 3 * D;
  static_assert(NT % CH == 0 && RG <= BLK, "whole row groups, each with a token of the block");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // ---------------- pooling, one block at a time
  for (int i = 0; i < ni; ++i) {
    const int n = g0 + i;
    const uint16_t* base;
    if (p.k.paged) {
      const int pg = n < p.k.max_pages ? p.k.block_table[(size_t)b * p.k.max_pages + n] : -1;
      if (pg < 0 || pg >= p.k.num_pages) {
        if (tid == 0) report(p.err, SEER_DEVERR_PAGE_INDEX);
        base = nullptr;
      } else {
        base = p.k.data + (size_t)pg * p.k.stride_b + (size_t)h * p.k.stride_h;
      }
    } else {
      base = p.k.data + (size_t)b * p.k.stride_b + (size_t)h * p.k.stride_h + (size_t)n * BLK * p.k.stride_t;
    }
    const int c = tid % CH, r = tid / CH;
    float mx[8], mn[8], smv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      mx[e] = -INFINITY;
      mn[e] = INFINITY;
      smv[e] = 0.f;
    }
    if (base) {
#pragma unroll 4
      for (int t = r; t < BLK; t += RG) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + (size_t)t * p.k.stride_t + c * 8));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float lo = bf16_lo(w[e]), hi = bf16_hi(w[e]);
          mx[2 * e] = fmaxf(mx[2 * e], lo);
          mn[2 * e] = fminf(mn[2 * e], lo);
          smv[2 * e] += lo;
          mx[2 * e + 1] = fmaxf(mx[2 * e + 1], hi);
          mn[2 * e + 1] = fminf(mn[2 * e + 1], hi);
          smv[2 * e + 1] += hi;
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      sm.red[0][r][c * 8 + e] = mx[e];
      sm.red[1][r][c * 8 + e] = mn[e];
      sm.red[2][r][c * 8 + e] = smv[e];
    }
    __syncthreads();
    for (int ch = tid; ch < D; ch += NT) {
      float a = -INFINITY, z = INFINITY, s = 0.f;
      for (int rr = 0; rr < RG; ++rr) {
        a = fmaxf(a, sm.red[0][rr][ch]);
        z = fminf(z, sm.red[1][rr][ch]);
        s += sm.red[2][rr][ch];
      }
      sm.pooled[i][ch] = a;
      sm.pooled[i][D + ch] = z;
      sm.pooled[i][2 * D + ch] = s * (1.0f / BLK);
    }
    __syncthreads();
  }
  // ---------------- y[i][r] = W_k[h][r] . pooled[i]; one warp per row, lanes along 3d
  const uint16_t* wk = p.w_k + (size_t)h * DG * P3;
  for (int row = warp; row < DG; row += NT / 32) {
    float acc[kKcompGroup];
#pragma unroll
    for (int i = 0; i < kKcompGroup; ++i) acc[i] = 0.f;
    const uint16_t* wr = wk + (size_t)row * P3;
#pragma unroll
    for (int k = 2 * lane; k < P3; k += 64) {
      const uint32_t w2 = __ldg(reinterpret_cast<const uint32_t*>(wr + k));
      const float w0 = bf16_lo(w2), w1 = bf16_hi(w2);
#pragma unroll
      for (int i = 0; i < kKcompGroup; ++i)
        if (i < ni) acc[i] += w0 * sm.pooled[i][k] + w1 * sm.pooled[i][k + 1];
    }
#pragma unroll
    for (int i = 0; i < kKcompGroup; ++i) {
      float v = acc[i];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0) sm.ys[i][row] = v;
    }
  }
  __syncthreads();
  // ---------------- RoPE at each block's first-token position, store bf16
  for (int e = tid; e < ni * (DG / 2); e += NT) {
    const int i = e / (DG / 2), j = e % (DG / 2);
    const int n = g0 + i;
    float c, s;
    rope_cos_sin((double)n * BLK * p.theta[j], c, s);
    const float x1 = sm.ys[i][j], x2 = sm.ys[i][j + DG / 2];
    uint16_t* dst = p.kcomp + (((size_t)b * p.Hkv + h) * p.NB + n) * DG;
    __nv_bfloat16 r1 = __float2bfloat16_rn(x1 * c - x2 * s);
    __nv_bfloat16 r2 = __float2bfloat16_rn(x2 * c + x1 * s);
    dst[j] = *reinterpret_cast<uint16_t*>(&r1);
    dst[j + DG / 2] = *reinterpret_cast<uint16_t*>(&r2);
  }
  __syncthreads();
}

// The new blocks of (b, h) are [v0, nfull); cluster rank r of kc takes groups r, r + kc, ...
template <int D, int BLK, int DG, int NT>
__device__ void kcomp_update_share(const KcompParams& p, int b, int h, int v0, int nfull, int rank, int kc,
                                   KcompSmem<D, DG, NT>& sm) {
  for (int g0 = v0 + rank * kKcompGroup; g0 < nfull; g0 += kc * kKcompGroup)
    kcomp_group<D, BLK, DG, NT>(p, b, h, g0, min(kKcompGroup, nfull - g0), sm);
}

}  // namespace seer
