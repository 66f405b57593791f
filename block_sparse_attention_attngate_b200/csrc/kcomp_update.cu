// K Compression Cache maintenance.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 2 and Knowl 5; "Sparse Attention Adaptation
// for Long Reasoning" (papernotes.org), key designs 2 and 4:
//   p   = [max | min | avg] of the b pre-RoPE keys of one full block (per channel)
//   y   = W_k[h] . p                          (d_gate x 3d, no bias)
//   out = bf16(RoPE_{n*b}(y))                 (rotate-half, theta_i = base^(-2i/d_gate))
// for every block n in [valid_blocks[b], floor(L_b / b)); then valid_blocks[b]
// advances (a second, one-CTA kernel, so no CTA of the first can observe the
// new value).  A CTA owns up to NI consecutive blocks of one (b, h) at a time,
// so one pass over W_k[h] (L2-resident, 96 KB at d=d_gate=128) serves NI
// blocks.  The read of the keys is the only HBM-sized traffic: prefill
// rebuilds are bandwidth-bound, per-step calls touch one block or none.
#include "seer_device.cuh"
#include "seer_internal.h"

namespace seer {
namespace {

constexpr int kThreads = 256;
constexpr int kNI = 8;  // blocks per group

template <int D, int BLK, int DG>
__global__ void __launch_bounds__(kThreads) kcomp_update_kernel(const KcompParams p) {
  constexpr int CH = D / 8;                 // 16-byte chunks per key row
  constexpr int RG = kThreads / CH;         // token row groups
  constexpr int P3 = 3 * D;
  static_assert(BLK % RG == 0, "row groups must tile the block");
  __shared__ float red[3][RG][D];           // per row-group max / min / sum
  __shared__ float pooled[kNI][P3];
  __shared__ float ys[kNI][DG];
  __shared__ double theta[DG / 2];

  const int b = blockIdx.z, h = blockIdx.y;
  const int L = max(p.seqlens[b], 0);
  int nfull = min(L / BLK, p.NB);
  if (!p.k.paged) {
    const long long cap_blocks = p.k.num_tokens / BLK;
    if (cap_blocks < nfull) nfull = (int)cap_blocks;
  }
  if (nfull < L / BLK && blockIdx.x == 0 && threadIdx.x == 0) report(p.err, SEER_DEVERR_COUNT);
  const int v0 = max(p.valid[b], 0);
  if (v0 >= nfull) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  for (int j = tid; j < DG / 2; j += kThreads) theta[j] = pow((double)p.rope_base, -2.0 * j / DG);

  const uint16_t* wk = p.w_k + (size_t)h * DG * P3;
  for (int g0 = v0 + blockIdx.x * kNI; g0 < nfull; g0 += gridDim.x * kNI) {
    const int ni = min(kNI, nfull - g0);
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
      float mx[8], mn[8], sm[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        mx[e] = -INFINITY;
        mn[e] = INFINITY;
        sm[e] = 0.f;
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
            sm[2 * e] += lo;
            mx[2 * e + 1] = fmaxf(mx[2 * e + 1], hi);
            mn[2 * e + 1] = fminf(mn[2 * e + 1], hi);
            sm[2 * e + 1] += hi;
          }
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        red[0][r][c * 8 + e] = mx[e];
        red[1][r][c * 8 + e] = mn[e];
        red[2][r][c * 8 + e] = sm[e];
      }
      __syncthreads();
      for (int ch = tid; ch < D; ch += kThreads) {
        float a = -INFINITY, z = INFINITY, s = 0.f;
        for (int rr = 0; rr < RG; ++rr) {
          a = fmaxf(a, red[0][rr][ch]);
          z = fminf(z, red[1][rr][ch]);
          s += red[2][rr][ch];
        }
        pooled[i][ch] = a;
        pooled[i][D + ch] = z;
        pooled[i][2 * D + ch] = s * (1.0f / BLK);
      }
      __syncthreads();
    }
    // ---------------- y[i][r] = W_k[h][r] . pooled[i]; one warp per row, lanes along 3d
    for (int row = warp; row < DG; row += kThreads / 32) {
      float acc[kNI];
#pragma unroll
      for (int i = 0; i < kNI; ++i) acc[i] = 0.f;
      const uint16_t* wr = wk + (size_t)row * P3;
#pragma unroll
      for (int k = 2 * lane; k < P3; k += 64) {
        const uint32_t w2 = __ldg(reinterpret_cast<const uint32_t*>(wr + k));
        const float w0 = bf16_lo(w2), w1 = bf16_hi(w2);
#pragma unroll
        for (int i = 0; i < kNI; ++i) acc[i] += w0 * pooled[i][k] + w1 * pooled[i][k + 1];
      }
#pragma unroll
      for (int i = 0; i < kNI; ++i) {
        float v = acc[i];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) ys[i][row] = v;
      }
    }
    __syncthreads();
    // ---------------- RoPE at each block's first-token position, store bf16
    for (int e = tid; e < ni * (DG / 2); e += kThreads) {
      const int i = e / (DG / 2), j = e % (DG / 2);
      const int n = g0 + i;
      double sn, cs;
      sincos((double)n * BLK * theta[j], &sn, &cs);
      const float c = (float)cs, s = (float)sn;
      const float x1 = ys[i][j], x2 = ys[i][j + DG / 2];
      uint16_t* dst = p.kcomp + (((size_t)b * p.Hkv + h) * p.NB + n) * DG;
      __nv_bfloat16 r1 = __float2bfloat16_rn(x1 * c - x2 * s);
      __nv_bfloat16 r2 = __float2bfloat16_rn(x2 * c + x1 * s);
      dst[j] = *reinterpret_cast<uint16_t*>(&r1);
      dst[j + DG / 2] = *reinterpret_cast<uint16_t*>(&r2);
    }
    __syncthreads();
  }
}

__global__ void kcomp_commit_kernel(const int32_t* seqlens, int32_t* valid, int B, int BLK, int NB) {
  for (int b = threadIdx.x; b < B; b += blockDim.x) valid[b] = min(max(seqlens[b], 0) / BLK, NB);
}

template <int D, int BLK, int DG>
cudaError_t launch_t(const KcompParams& p, int grid_x, cudaStream_t s) {
  dim3 grid(grid_x, p.Hkv, p.B);
  kcomp_update_kernel<D, BLK, DG><<<grid, kThreads, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  kcomp_commit_kernel<<<1, 256, 0, s>>>(p.seqlens, p.valid_out, p.B, BLK, p.NB);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_kcomp_update(const KcompParams& p, int D, int BLK, int DG, int grid_x, cudaStream_t s) {
#define SEER_K(d, blk, dg) \
  if (D == d && BLK == blk && DG == dg) return launch_t<d, blk, dg>(p, grid_x, s);
  SEER_K(64, 64, 64)
  SEER_K(64, 64, 128)
  SEER_K(64, 128, 64)
  SEER_K(64, 128, 128)
  SEER_K(128, 64, 64)
  SEER_K(128, 64, 128)
  SEER_K(128, 128, 64)
  SEER_K(128, 128, 128)
#undef SEER_K
  return cudaErrorInvalidValue;
}

}  // namespace seer
