// Decode ground truth: the block scores full attention would give, from the
// whole K cache -- the target the AttnGate is distilled towards, usable in
// place of the gate ("oracle" block selection).
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 3: for decoding, the attention map of the g
// query heads of a group over all L tokens is 1-D max-pooled over each
// block's columns, the g pooled rows are reduced by max, and the result is
// normalised to sum to 1.  With s_j[t] = scale * q_j . K[t] (and the usual
// softmax p_j[t] = exp(s_j[t] - lse_j)):
//   gt[n] = max_j max_{t in block n} p_j[t] / sum_n' (same)
//         = max_j exp(bmax_j[n] - lse_j) / sum_n' (same)
// so one streaming pass over K yields everything: per block and head the score
// maximum, per head the running (max, sum of exp).
//
// One CTA per chunk of kChunk consecutive blocks of one (b, h): a producer warp
// brings K tiles by TMA (128B swizzle, box 64 channels x b tokens) into a ring
// of mbarrier-guarded stages; four consumer warps own b/4 tokens of every
// block and compute S = Q K^T on mma.sync (the group's <= 8 query rows as a
// 16-row A fragment), in the log2 domain.  Each warp writes its per-head block
// maxima and, at the end of the chunk, its per-head (max, sum) to a
// workspace; the last chunk of the (b, h) to arrive (acquire-release counter)
// forms lse_j, the scores and their normalisation, and resets the counter.
// All waits are bounded.
#include "seer_device.cuh"
#include "seer_internal.h"

namespace seer {
namespace {

constexpr int kNW = 4;         // consumer warps
constexpr int kChunk = 16;     // blocks per CTA

template <int D, int BLK>
struct TruthShape {
  static constexpr int kTile = BLK * D * 2;
  static constexpr int kBox = BLK * 128;
  static constexpr int kNBox = D / 64;
  static constexpr int kTPW = BLK / kNW;
  static constexpr int kNT = kTPW / 8;
  static constexpr int kDK = D / 16;
  static constexpr int kStages = (6 * 16384) / kTile < 2 ? 2 : (6 * 16384) / kTile;   // ~96 KB of ring
  static constexpr int kThreads = (kNW + 1) * 32;
  static constexpr size_t kSmem = 1024 + (size_t)kStages * kTile + (2 * kStages + 1) * 8 + 64 + 8 * kNW * 4 +
                                  3 * kStages * 4;
};

__device__ __forceinline__ void coords(const int32_t perm[3], int t, int h, int bp, int& c1, int& c2, int& c3) {
  int c[3];
  c[perm[0]] = t;
  c[perm[1]] = h;
  c[perm[2]] = bp;
  c1 = c[0];
  c2 = c[1];
  c3 = c[2];
}

template <int D, int BLK>
__global__ void __launch_bounds__(TruthShape<D, BLK>::kThreads)
    truth_kernel(const __grid_constant__ CUtensorMap tmK, const TruthParams p) {
  using S = TruthShape<D, BLK>;
  constexpr int ST = S::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + (size_t)ST * S::kTile);
  uint64_t* empty = full + ST;
  uint64_t* cbar = empty + ST;
  volatile int* sh = reinterpret_cast<volatile int*>(cbar + 1);   // [0] abort, [1] last, [2] done
  float* red = reinterpret_cast<float*>(const_cast<int*>(sh) + 16);   // [kNW * 8] reduction scratch
  volatile int* loaded = sh + 16 + 8 * kNW;                          // [ST] the stage holds a tile
  volatile int* issued = loaded + ST;                                // [ST] tiles issued per stage
  volatile int* observed = issued + ST;                              // [ST] full phases observed

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z, bh = b * p.Hkv + h;
  const int g = p.g;
  if (tid == 0) {
    tma_prefetch_desc(&tmK);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kNW);
    }
    mbar_init(cbar, kNW);
    sh[0] = 0;
    sh[2] = 0;
    for (int s = 0; s < ST; ++s) issued[s] = observed[s] = 0;
    fence_barrier_init();
  }
  pdl_wait();
  pdl_trigger();
  const int L = max(p.seqlens[b], 0);
  const int nblk = min((L + BLK - 1) / BLK, p.NB);
  const int nch = (nblk + kChunk - 1) / kChunk;
  const int n0 = chunk * kChunk, n1 = min(nblk, n0 + kChunk);
  float* scores = p.scores + (size_t)bh * p.NB;
  float* lscores = p.log_scores ? p.log_scores + (size_t)bh * p.NB : nullptr;
  if (nblk == 0) {   // nothing to attend to: an all-zero row (chunk 0 writes it)
    if (chunk == 0)
      for (int n = tid; n < p.NB; n += S::kThreads) {
        scores[n] = 0.f;
        if (lscores) lscores[n] = -INFINITY;
      }
    return;
  }
  if (n0 >= n1) return;
  __syncthreads();   // barrier inits visible to every warp
  const int nit = n1 - n0;

  if (warp == kNW) {
    // ------------------------------------------------------------ producer warp
    if (lane == 0) {
      for (int it = 0; it < nit; ++it) {
        const int s = it % ST;
        if (it >= ST && !mbar_wait(&empty[s], ((it / ST) - 1) & 1)) {
          report(p.err, SEER_DEVERR_TIMEOUT);
          sh[0] = 1;
          break;
        }
        const int n = n0 + it;
        int tb = b, tt = n * BLK;
        if (p.k_paged) {
          const int pg = n < p.k_maxp ? p.k_table[(size_t)b * p.k_maxp + n] : -1;
          if (pg < 0 || pg >= p.k_pages) {
            report(p.err, SEER_DEVERR_PAGE_INDEX);
            loaded[s] = 0;
            mbar_arrive(&full[s]);   // an empty stage: the consumers skip it
            issued[s] = issued[s] + 1;
            continue;
          }
          tb = pg;
          tt = 0;
        }
        loaded[s] = 1;
        mbar_arrive_expect_tx(&full[s], S::kTile);
        int c1, c2, c3;
        coords(p.k_perm, tt, h, tb, c1, c2, c3);
#pragma unroll
        for (int bx = 0; bx < S::kNBox; ++bx)
          tma_load_4d(ring + (size_t)s * S::kTile + bx * S::kBox, &tmK, &full[s], bx * 64, c1, c2, c3);
        issued[s] = issued[s] + 1;
      }
      __threadfence_block();
      sh[2] = 1;
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gq = lane >> 2, tq = lane & 3;
  const bool live = gq < g;
  uint32_t qa[S::kDK][2];
  {
    const uint16_t* qrow = p.q + ((size_t)b * p.Hq + (size_t)h * g + (live ? gq : 0)) * D;
#pragma unroll
    for (int ks = 0; ks < S::kDK; ++ks) {
      qa[ks][0] = live ? __ldg(reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * tq)) : 0u;
      qa[ks][1] = live ? __ldg(reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 8 + 2 * tq)) : 0u;
    }
  }
  const float sl2 = p.scale_log2;
  const int tok_base = warp * S::kTPW;
  float m_run = -INFINITY, l_run = 0.f;
  float* bmax = p.bmax + (size_t)bh * p.NB * (kNW * kMaxGroup);
  bool alive = true;
  for (int it = 0; it < nit; ++it) {
    const int s = it % ST;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (it / ST) & 1))) {
      alive = false;
      break;
    }
    if (warp == 0 && lane == 0) observed[s] = observed[s] + 1;
    const int n = n0 + it;
    const int valid = loaded[s] ? min(BLK, L - n * BLK) : 0;   // a skipped tile scores nothing
    const uint32_t kt = smem_u32(ring + (size_t)s * S::kTile);
    float sacc[S::kNT][4];
#pragma unroll
    for (int j = 0; j < S::kNT; ++j) {
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t row = tok_base + j * 8 + (lane & 7);
#pragma unroll
      for (int kp = 0; kp < S::kDK / 2; ++kp) {
        const uint32_t chk = kp * 4 + (lane >> 3);
        uint32_t r0, r1, r2, r3;
        ldsm_x4(kt + (chk >> 3) * S::kBox + sw128(row, chk & 7), r0, r1, r2, r3);
        if (kp & 1) {
          mma_bf16_16816(sb, qa[2 * kp][0], 0u, qa[2 * kp][1], 0u, r0, r1);
          mma_bf16_16816(sb, qa[2 * kp + 1][0], 0u, qa[2 * kp + 1][1], 0u, r2, r3);
        } else {
          mma_bf16_16816(sa, qa[2 * kp][0], 0u, qa[2 * kp][1], 0u, r0, r1);
          mma_bf16_16816(sa, qa[2 * kp + 1][0], 0u, qa[2 * kp + 1][1], 0u, r2, r3);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[j][e] = sa[e] + sb[e];
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);   // the tile is in registers now
    // this lane: head gq, tokens 2tq, 2tq+1 of each 8-token tile; log2-domain scores
    float v[S::kNT][2];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < S::kNT; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tok = tok_base + j * 8 + 2 * tq + e;
        v[j][e] = tok < valid ? sacc[j][e] * sl2 : -INFINITY;
        mx = fmaxf(mx, v[j][e]);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    if (tq == 0 && live) bmax[((size_t)n * kNW + warp) * kMaxGroup + gq] = mx;
    const float m_new = fmaxf(m_run, mx);
    if (m_new != -INFINITY) {
      float ls = 0.f;
#pragma unroll
      for (int j = 0; j < S::kNT; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) ls += exp2f(v[j][e] - m_new);
      l_run = l_run * exp2f(m_run - m_new) + ls;
      m_run = m_new;
    }
  }
  if (!alive) {
    if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
    sh[0] = 1;
    if (warp == 0 && lane == 0) {
      // drain the copies still in flight (bounded) before shared memory is released
      const long long t0 = clock64();
      while (!sh[2] && clock64() - t0 < kWaitLimitCycles) {
      }
      for (int st = 0; st < ST; ++st)
        if (issued[st] > observed[st]) mbar_wait(&full[st], observed[st] & 1);
    }
    return;
  }
  // this warp's (max, sum) per head for the chunk
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  float* part = p.part + (((size_t)bh * p.nchunk + chunk) * kNW + warp) * kMaxGroup * 2;
  if (tq == 0 && live) {
    part[gq * 2] = m_run;
    part[gq * 2 + 1] = l_run;
  }
  uint32_t cph = 0;
  if (!warps_sync(cbar, cph)) {
    if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
    return;
  }
  if (tid == 0) sh[1] = atomic_add_acq_rel_gpu(&p.counters[bh], 1) == nch - 1;
  if (!warps_sync(cbar, cph)) {
    if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
    return;
  }
  if (!sh[1]) return;

  // ---------------------------------------------------------------- the (b, h)'s last chunk: finish
  constexpr int NT = kNW * 32;
  // lse_j (log2 domain) over every chunk's per-warp (max, sum)
  float* lse2 = red;   // [8]
  if (tid < g) {
    float M = -INFINITY;
    for (int c = 0; c < nch; ++c)
      for (int w = 0; w < kNW; ++w)
        M = fmaxf(M, __ldcg(p.part + (((size_t)bh * p.nchunk + c) * kNW + w) * kMaxGroup * 2 + tid * 2));
    float Z = 0.f;
    if (M != -INFINITY)
      for (int c = 0; c < nch; ++c)
        for (int w = 0; w < kNW; ++w) {
          const float* pp = p.part + (((size_t)bh * p.nchunk + c) * kNW + w) * kMaxGroup * 2 + tid * 2;
          const float m = __ldcg(pp), l = __ldcg(pp + 1);
          if (m != -INFINITY) Z += l * exp2f(m - M);
        }
    lse2[tid] = Z > 0.f ? M + log2f(Z) : INFINITY;   // +inf: no token of this head (cannot happen for nblk > 0)
  }
  if (!warps_sync(cbar, cph)) {
    if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
    return;
  }
  // raw[n] = max_j exp2(bmax_j[n] - lse2_j); the sum over n
  float part_sum = 0.f;
  for (int n = tid; n < nblk; n += NT) {
    float r = 0.f;
    for (int j = 0; j < g; ++j) {
      float bm = -INFINITY;
#pragma unroll
      for (int w = 0; w < kNW; ++w) bm = fmaxf(bm, __ldcg(bmax + ((size_t)n * kNW + w) * kMaxGroup + j));
      r = fmaxf(r, exp2f(bm - lse2[j]));
    }
    scores[n] = r;   // unnormalised for now; rescaled below by this thread
    part_sum += r;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) part_sum += __shfl_xor_sync(0xffffffffu, part_sum, off);
  if (lane == 0) red[8 + warp] = part_sum;
  if (!warps_sync(cbar, cph)) {
    if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
    return;
  }
  float total = 0.f;
#pragma unroll
  for (int w = 0; w < kNW; ++w) total += red[8 + w];
  const float inv = total > 0.f ? 1.f / total : 0.f;
  for (int n = tid; n < p.NB; n += NT) {
    const float gt = n < nblk ? scores[n] * inv : 0.f;
    scores[n] = gt;
    if (lscores) lscores[n] = gt > 0.f ? logf(gt) : -INFINITY;
  }
  if (tid == 0) p.counters[bh] = 0;
}

template <int D, int BLK>
cudaError_t launch_t(const CUtensorMap& tk, const TruthParams& p, cudaStream_t st) {
  using S = TruthShape<D, BLK>;
  auto kern = truth_kernel<D, BLK>;
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = ensure_smem_limit(kern, (int)S::kSmem, attr_done);
  if (e != cudaSuccess) return e;
  const dim3 grid(p.nchunk, p.Hkv, p.B);
  return launch_pdl(kern, grid, dim3(S::kThreads), S::kSmem, st, tk, p);
}

}  // namespace

int truth_chunk_blocks() { return kChunk; }
int truth_warps() { return kNW; }

cudaError_t launch_gate_truth(const CUtensorMap& tk, const TruthParams& p, int D, int BLK, cudaStream_t s) {
  if (D == 64 && BLK == 64) return launch_t<64, 64>(tk, p, s);
  if (D == 64 && BLK == 128) return launch_t<64, 128>(tk, p, s);
  if (D == 128 && BLK == 64) return launch_t<128, 64>(tk, p, s);
  if (D == 128 && BLK == 128) return launch_t<128, 128>(tk, p, s);
  return cudaErrorInvalidValue;
}

}  // namespace seer
