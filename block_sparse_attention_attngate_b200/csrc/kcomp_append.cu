// K Compression Cache from running block statistics: the decode-time form of
// the cache update that needs no pre-RoPE copy of the whole context.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 2 and Knowl 5: each finished block of b keys
// gets one cache entry,
//   RoPE_{n*b}( W_k[h] . [max | min | avg] of the block's pre-RoPE keys ).
// max, min and avg over a block need only the running per-channel max, min and
// sum of its keys so far, so each (b, kv-head) keeps those (fp32, 3 x d) and
// folds in the key of every appended token; the token that completes block n
// writes entry n and advances the fill count.  The state of a sequence that
// resumes mid-block (after a prefill) is primed once from the key cache.
//
// One CTA per (b, kv-head), one thread per channel; a completing block's
// projection takes one warp per output row of W_k[h] (L2-resident), RoPE
// angles in fp64 as in the block-pooling update.
#include "seer_device.cuh"
#include "seer_internal.h"

namespace seer {
namespace {

constexpr int kThreads = 128;

template <int D, int BLK, int DG>
__global__ void __launch_bounds__(kThreads) kcomp_append_kernel(const AppendParams p) {
  __shared__ float pooled[3 * D];
  __shared__ float ys[DG];
  const int h = blockIdx.x, b = blockIdx.y, bh = b * p.Hkv + h;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();
  pdl_trigger();
  const int L = p.seqlens[b];
  if (L <= 0) return;   // nothing appended to this sequence
  const int n = (L - 1) / BLK, pos = (L - 1) - n * BLK;
  const bool fills = pos == BLK - 1;
  float* st = p.state + (size_t)bh * 3 * D;
  for (int c = tid; c < D; c += kThreads) {
    const uint16_t kb = p.k_new[(size_t)bh * D + c];
    const float k = __uint_as_float((uint32_t)kb << 16);
    float mx = k, mn = k, sm = k;   // a block's first token restarts the statistics
    if (pos != 0) {
      mx = fmaxf(st[c], k);
      mn = fminf(st[D + c], k);
      sm = st[2 * D + c] + k;
    }
    st[c] = mx;
    st[D + c] = mn;
    st[2 * D + c] = sm;
    if (fills) {
      pooled[c] = mx;
      pooled[D + c] = mn;
      pooled[2 * D + c] = sm * (1.0f / BLK);
    }
  }
  if (!fills) return;
  // the block's entry: the earlier entries must be in place and the row must hold it
  if (p.valid[bh] != n || n >= p.NB) {
    if (tid == 0) report(p.err, SEER_DEVERR_COUNT);
    return;
  }
  __syncthreads();
  // y = W_k[h] . pooled: one warp per row, lanes along 3d
  constexpr int P3 = 3 * D;
  const uint16_t* wk = p.w_k + (size_t)h * DG * P3;
  for (int row = warp; row < DG; row += kThreads / 32) {
    const uint16_t* wr = wk + (size_t)row * P3;
    float acc = 0.f;
#pragma unroll
    for (int k = 2 * lane; k < P3; k += 64) {
      const uint32_t w2 = __ldg(reinterpret_cast<const uint32_t*>(wr + k));
      acc += bf16_lo(w2) * pooled[k] + bf16_hi(w2) * pooled[k + 1];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) ys[row] = acc;
  }
  __syncthreads();
  // RoPE at the block's first-token position, bf16 store
  uint16_t* dst = p.kcomp + ((size_t)bh * p.NB + n) * DG;
  for (int j = tid; j < DG / 2; j += kThreads) {
    float c, s;
    rope_cos_sin((double)n * BLK * p.theta[j], c, s);
    const float x1 = ys[j], x2 = ys[j + DG / 2];
    __nv_bfloat16 r1 = __float2bfloat16_rn(x1 * c - x2 * s);
    __nv_bfloat16 r2 = __float2bfloat16_rn(x2 * c + x1 * s);
    dst[j] = *reinterpret_cast<uint16_t*>(&r1);
    dst[j + DG / 2] = *reinterpret_cast<uint16_t*>(&r2);
  }
  if (tid == 0) p.valid[bh] = n + 1;
}

// The running statistics of each sequence's current (incomplete) block, from the key cache:
// tokens [floor(L/b)*b, L).  A sequence at a block boundary gets the empty block's statistics,
// which its next append overwrites.
template <int D, int BLK>
__global__ void __launch_bounds__(kThreads) kcomp_state_init_kernel(const AppendParams p) {
  const int h = blockIdx.x, b = blockIdx.y, bh = b * p.Hkv + h;
  pdl_wait();
  pdl_trigger();
  const int L = max(p.seqlens[b], 0);
  const int t0 = (L / BLK) * BLK;
  const uint16_t* base = nullptr;   // the block's first key row
  if (L > t0) {
    if (p.k.paged) {
      const int nb = t0 / BLK;
      const int pg = nb < p.k.max_pages ? p.k.block_table[(size_t)b * p.k.max_pages + nb] : -1;
      if (pg < 0 || pg >= p.k.num_pages) {
        if (threadIdx.x == 0) report(p.err, SEER_DEVERR_PAGE_INDEX);
      } else {
        base = p.k.data + (size_t)pg * p.k.stride_b + (size_t)h * p.k.stride_h;
      }
    } else if (L <= p.k.num_tokens) {
      base = p.k.data + (size_t)b * p.k.stride_b + (size_t)h * p.k.stride_h + (size_t)t0 * p.k.stride_t;
    } else if (threadIdx.x == 0) {
      report(p.err, SEER_DEVERR_COUNT);
    }
  }
  float* st = p.state + (size_t)bh * 3 * D;
  for (int c = threadIdx.x; c < D; c += kThreads) {
    float mx = -INFINITY, mn = INFINITY, sm = 0.f;
    if (base)
      for (int t = 0; t < L - t0; ++t) {
        const float k = __uint_as_float((uint32_t)base[(size_t)t * p.k.stride_t + c] << 16);
        mx = fmaxf(mx, k);
        mn = fminf(mn, k);
        sm += k;
      }
    st[c] = mx;
    st[D + c] = mn;
    st[2 * D + c] = sm;
  }
}

template <int D, int BLK, int DG>
cudaError_t launch_append_t(const AppendParams& p, cudaStream_t s) {
  return launch_pdl(kcomp_append_kernel<D, BLK, DG>, dim3(p.Hkv, p.B), dim3(kThreads), 0, s, p);
}

template <int D, int BLK>
cudaError_t launch_init_t(const AppendParams& p, cudaStream_t s) {
  return launch_pdl(kcomp_state_init_kernel<D, BLK>, dim3(p.Hkv, p.B), dim3(kThreads), 0, s, p);
}

}  // namespace

cudaError_t launch_kcomp_append(const AppendParams& p, int D, int BLK, int DG, cudaStream_t s) {
#define SEER_K(d, blk, dg) \
  if (D == d && BLK == blk && DG == dg) return launch_append_t<d, blk, dg>(p, s);
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

cudaError_t launch_kcomp_state_init(const AppendParams& p, int D, int BLK, cudaStream_t s) {
  if (D == 64 && BLK == 64) return launch_init_t<64, 64>(p, s);
  if (D == 64 && BLK == 128) return launch_init_t<64, 128>(p, s);
  if (D == 128 && BLK == 64) return launch_init_t<128, 64>(p, s);
  if (D == 128 && BLK == 128) return launch_init_t<128, 128>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace seer
