// Causal attention over whole sequences with the block-level target of every
// query position beside the output: the training-side ground truth, extracted
// inside the attention forward instead of from an explicit L x L map.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 3 (the target of query i: its softmax row,
// 1-D max-pooled over each block's columns, max over the GQA group's heads,
// normalised to sum to 1) and Knowl 4 (its extraction inside a
// FlashAttention-2 forward: each tile's row maximum r of the pre-softmax scores
// is stored; once the row's final maximum m and normaliser l are known, the
// block score is exp(r - m) / l).
//
// One CTA per (P query positions, kv head, sequence), GQA-packed: consumer warp
// w takes 16 consecutive positions of query head w mod g, so one K/V tile in
// shared memory serves the whole group.  A key tile is one block of b keys,
// so the tile's row maximum is the block's.  A producer warp streams K/V tiles
// (TMA, 128B swizzle, box 64 channels x b tokens) into an mbarrier ring; the
// consumers compute S = Q K^T and O += P V on mma.sync m16n8k16 (P taken from
// S's accumulators), keep the online softmax in the log2 domain and store each
// row's tile maximum to a block-major workspace.  Finally the CTA turns its
// positions' maxima into the target: max over the group of exp2(r - m) / l,
// normalised over the position's visible blocks, zero past them.
//
// The tensor cores are driven by the legacy warp-level mma path here; a
// tcgen05 / TMEM formulation of the same forward is the faster route on this
// GPU.  All waits are bounded.
#include "seer_device.cuh"
#include "seer_internal.h"

namespace seer {
namespace {

constexpr float kLn2 = 0.6931471805599453f;

template <int D, int BLK>
struct PrefillShape {
  static constexpr int kTile = BLK * D * 2;   // bytes of one K (or V) tile
  static constexpr int kBox = BLK * 128;      // bytes of one 64-channel box
  static constexpr int kNBox = D / 64;
  static constexpr int kStages = (98304 / (2 * kTile)) < 2 ? 2 : (98304 / (2 * kTile));
  static constexpr int kDK = D / 16;          // QK^T k-steps
  static constexpr int kSub = 64;             // keys per sub-tile (a 128-key block is two)
  static constexpr int kNT = kSub / 8;        // S n-tiles per sub-tile
  static constexpr int kKS = kSub / 16;       // PV k-steps per sub-tile
  static constexpr int kON = D / 8;           // O n-tiles
  static constexpr int kQWarp = 16 * D * 2;   // one warp's 16 query rows (swizzled 64-channel boxes)
  static constexpr int kMaxThreads = 9 * 32;  // <= 8 consumer warps + the producer
  static constexpr size_t kSmem = 1024 + (size_t)kStages * 2 * kTile + 8 * kQWarp + (2 * kStages + 1) * 8 +
                                  2 * 128 * 4 + 64 * 4;
};

__device__ __forceinline__ void map_coords(const int32_t perm[3], int t, int h, int bp, int& c1, int& c2, int& c3) {
  int c[3];
  c[perm[0]] = t;
  c[perm[1]] = h;
  c[perm[2]] = bp;
  c1 = c[0];
  c2 = c[1];
  c3 = c[2];
}

template <int D, int BLK>
__global__ void __launch_bounds__(PrefillShape<D, BLK>::kMaxThreads, 1)
    prefill_gt_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const PrefillParams p) {
  using S = PrefillShape<D, BLK>;
  constexpr int ST = S::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qsm = ring + (size_t)ST * 2 * S::kTile;   // [8 warps][kNBox][16 rows][128 B]
  uint64_t* full = reinterpret_cast<uint64_t*>(qsm + 8 * S::kQWarp);
  uint64_t* empty = full + ST;
  uint64_t* cbar = empty + ST;                        // the consumer warps' rendezvous
  float* ms = reinterpret_cast<float*>(cbar + 1);     // [g][P] final row maxima (log2 domain)
  float* ls = ms + 128;                                // [g][P] final row sums
  volatile int* sh = reinterpret_cast<volatile int*>(ls + 128);   // [0] abort, [1] producer done
  volatile int* issued = sh + 4;                                   // [ST]
  volatile int* observed = issued + 16;                            // [ST]

  const int g = p.g, Wp = 8 / g, CW = Wp * g, P = 16 * Wp;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int b = blockIdx.z, hk = blockIdx.y;
  // heaviest (latest) position tiles first
  const int p0 = ((int)gridDim.x - 1 - (int)blockIdx.x) * P;
  if (tid == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CW);
      issued[s] = observed[s] = 0;
    }
    mbar_init(cbar, CW);
    sh[0] = sh[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  const int Lr = max(p.seqlens[b], 0);
  const int L = min(Lr, min(p.T, p.kcap));
  if (Lr > L && blockIdx.x == 0 && hk == 0 && tid == 0) report(p.err, SEER_DEVERR_COUNT);
  if (p0 >= L) return;   // the whole CTA: no position of this tile exists
  const int pend = min(p0 + P, L);
  const int ntiles = (pend - 1) / BLK + 1;   // key tiles 0 .. ntiles-1 are visible to some row

  if (warp == CW) {
    // ------------------------------------------------------------ producer warp
    if (lane == 0) {
      for (int n = 0; n < ntiles; ++n) {
        const int s = n % ST;
        if (n >= ST && !mbar_wait(&empty[s], ((n / ST) - 1) & 1)) {
          report(p.err, SEER_DEVERR_TIMEOUT);
          sh[0] = 1;
          break;
        }
        mbar_arrive_expect_tx(&full[s], 2u * S::kTile);
        uint8_t* kdst = ring + (size_t)s * 2 * S::kTile;
        int c1, c2, c3;
        map_coords(p.k_perm, n * BLK, hk, b, c1, c2, c3);
#pragma unroll
        for (int bx = 0; bx < S::kNBox; ++bx) tma_load_4d(kdst + bx * S::kBox, &tmK, &full[s], bx * 64, c1, c2, c3);
        map_coords(p.v_perm, n * BLK, hk, b, c1, c2, c3);
#pragma unroll
        for (int bx = 0; bx < S::kNBox; ++bx)
          tma_load_4d(kdst + S::kTile + bx * S::kBox, &tmV, &full[s], bx * 64, c1, c2, c3);
        issued[s] = issued[s] + 1;
      }
      __threadfence_block();
      sh[1] = 1;
    }
    return;
  }
  if (warp > CW) return;

  // -------------------------------------------------------------- consumers
  const int hh = warp % g, pg = warp / g;
  const int h = hk * g + hh;                      // query head
  const int pw = p0 + 16 * pg;                    // this warp's first position
  const int gq = lane >> 2, tq = lane & 3;
  const int i_lo = pw + gq, i_hi = pw + gq + 8;   // this thread's two rows
  const size_t qrow = ((size_t)b * p.Hq + h) * p.T;
  // this warp's 16 query rows -> shared memory (128B-swizzled 64-channel boxes; rows past L zero)
  const uint32_t qw = smem_u32(qsm + warp * S::kQWarp);
  for (int e = lane; e < 16 * (D / 8); e += 32) {
    const int r = e / (D / 8), c = e - r * (D / 8);   // row, 16-byte chunk
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (pw + r < L) v = *reinterpret_cast<const uint4*>(p.q + (qrow + pw + r) * D + c * 8);
    *reinterpret_cast<uint4*>(qsm + warp * S::kQWarp + (c >> 3) * (16 * 128) + sw128(r, c & 7)) = v;
  }
  __syncwarp();
  float o[S::kON][4];
#pragma unroll
  for (int on = 0; on < S::kON; ++on) o[on][0] = o[on][1] = o[on][2] = o[on][3] = 0.f;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
  const float sl2 = p.scale_log2;
  const int wlast = min(pw + 15, L - 1);          // the warp's last existing position
  float* rws = p.rmax + ((size_t)b * p.Hq + h) * p.NB * p.T;   // [NB][T] tile row maxima
  bool alive = true;
  for (int n = 0; n < ntiles; ++n) {
    const int s = n % ST;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (n / ST) & 1))) {
      alive = false;
      break;
    }
    if (warp == 0 && lane == 0) observed[s] = observed[s] + 1;
    if (pw < L && n * BLK <= wlast) {
      const uint32_t kt = smem_u32(ring + (size_t)s * 2 * S::kTile);
      const uint32_t vt = kt + S::kTile;
      float rlo = -INFINITY, rhi = -INFINITY;   // the block's row maxima
#pragma unroll 1
      for (int half = 0; half < BLK / S::kSub; ++half) {
        const int tb = n * BLK + half * S::kSub;   // first key of the sub-tile
        // ---- S = Q K^T (16 rows x 64 keys): k-steps outermost, the 8 n-tiles' chains interleaved
        float sacc[S::kNT][4];
#pragma unroll
        for (int j = 0; j < S::kNT; ++j) sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < S::kDK; ++ks) {
          uint32_t a0, a1, a2, a3;
          {
            const uint32_t qr = (lane & 7) + (((lane >> 3) & 1) << 3), qc = 2 * ks + (lane >> 4);
            ldsm_x4(qw + (qc >> 3) * (16 * 128) + sw128(qr, qc & 7), a0, a1, a2, a3);
          }
#pragma unroll
          for (int j = 0; j < S::kNT; j += 2) {
            const uint32_t row = half * S::kSub + j * 8 + (lane & 7) + ((lane >> 4) << 3);
            const uint32_t chunk = 2 * ks + ((lane >> 3) & 1);
            uint32_t r0, r1, r2, r3;
            ldsm_x4(kt + (chunk >> 3) * S::kBox + sw128(row, chunk & 7), r0, r1, r2, r3);
            mma_bf16_16816(sacc[j], a0, a1, a2, a3, r0, r1);
            mma_bf16_16816(sacc[j + 1], a0, a1, a2, a3, r2, r3);
          }
        }
        // ---- causal mask (key t visible to row i iff t <= i), log2-domain scores, row maxima
        float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
        for (int j = 0; j < S::kNT; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int t = tb + j * 8 + 2 * tq + e;
            const float vlo = t <= i_lo ? sacc[j][e] * sl2 : -INFINITY;
            const float vhi = t <= i_hi ? sacc[j][2 + e] * sl2 : -INFINITY;
            sacc[j][e] = vlo;
            sacc[j][2 + e] = vhi;
            mx_lo = fmaxf(mx_lo, vlo);
            mx_hi = fmaxf(mx_hi, vhi);
          }
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
        rlo = fmaxf(rlo, mx_lo);
        rhi = fmaxf(rhi, mx_hi);
        // ---- online softmax
        const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
        const float mu_lo = mn_lo == -INFINITY ? 0.f : mn_lo, mu_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
        const float al_lo = exp2f(m_lo - mu_lo), al_hi = exp2f(m_hi - mu_hi);
        m_lo = mn_lo;
        m_hi = mn_hi;
        uint32_t pl[S::kNT], ph[S::kNT];
        float s_lo = 0.f, s_hi = 0.f;
#pragma unroll
        for (int j = 0; j < S::kNT; ++j) {
          pl[j] = pack_bf16(exp2f(sacc[j][0] - mu_lo), exp2f(sacc[j][1] - mu_lo));
          ph[j] = pack_bf16(exp2f(sacc[j][2] - mu_hi), exp2f(sacc[j][3] - mu_hi));
          s_lo += bf16_lo(pl[j]) + bf16_hi(pl[j]);
          s_hi += bf16_lo(ph[j]) + bf16_hi(ph[j]);
        }
        l_lo = l_lo * al_lo + s_lo;
        l_hi = l_hi * al_hi + s_hi;
#pragma unroll
        for (int on = 0; on < S::kON; ++on) {
          o[on][0] *= al_lo;
          o[on][1] *= al_lo;
          o[on][2] *= al_hi;
          o[on][3] *= al_hi;
        }
        // ---- O += P V (V rows past L may hold anything: zeroed so that 0 * V stays 0)
        const bool ragged = tb + S::kSub > L;
        const uint32_t mi = lane >> 3;
#pragma unroll
        for (int kk = 0; kk < S::kKS; ++kk) {
          const uint32_t a0 = pl[2 * kk], a1 = ph[2 * kk], a2 = pl[2 * kk + 1], a3 = ph[2 * kk + 1];
          const uint32_t row = half * S::kSub + kk * 16 + (lane & 7) + ((mi & 1) << 3);
          const int t0 = tb + kk * 16 + 2 * tq;   // tokens of this lane's B halves: t0, t0+1 / t0+8, t0+9
          const uint32_t m01 = (t0 < L ? 0x0000ffffu : 0u) | (t0 + 1 < L ? 0xffff0000u : 0u);
          const uint32_t m89 = (t0 + 8 < L ? 0x0000ffffu : 0u) | (t0 + 9 < L ? 0xffff0000u : 0u);
#pragma unroll
          for (int i = 0; i < S::kON / 2; ++i) {
            const uint32_t chunk = 2 * i + (mi >> 1);
            uint32_t v0, v1, v2, v3;
            ldsm_x4_trans(vt + (chunk >> 3) * S::kBox + sw128(row, chunk & 7), v0, v1, v2, v3);
            if (ragged) {
              v0 &= m01;
              v2 &= m01;
              v1 &= m89;
              v3 &= m89;
            }
            mma_bf16_16816(o[2 * i], a0, a1, a2, a3, v0, v1);
            mma_bf16_16816(o[2 * i + 1], a0, a1, a2, a3, v2, v3);
          }
        }
      }
      // the block's row maxima (the tile is one block of keys)
      if (tq == 0) {
        if (i_lo < L && n * BLK <= i_lo) rws[(size_t)n * p.T + i_lo] = rlo;
        if (i_hi < L && n * BLK <= i_hi) rws[(size_t)n * p.T + i_hi] = rhi;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  if (!__all_sync(0xffffffffu, alive)) {
    if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
    sh[0] = 1;
    if (warp == 0 && lane == 0) {
      // drain the copies still in flight (bounded) before shared memory is released
      const long long t0 = clock64();
      while (!sh[1] && clock64() - t0 < kWaitLimitCycles) {
      }
      for (int st = 0; st < ST; ++st)
        if (issued[st] > observed[st]) mbar_wait(&full[st], observed[st] & 1);
    }
    return;
  }

  // ---- output rows: O / l (bf16), LSE (natural log), and this head's row statistics
  l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
  l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
  l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
  l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
  const float inv_lo = l_lo > 0.f ? 1.f / l_lo : 0.f, inv_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
#pragma unroll
  for (int on = 0; on < S::kON; ++on) {
    const int c = on * 8 + 2 * tq;
    if (i_lo < L)
      *reinterpret_cast<uint32_t*>(p.o + (qrow + i_lo) * D + c) = pack_bf16(o[on][0] * inv_lo, o[on][1] * inv_lo);
    if (i_hi < L)
      *reinterpret_cast<uint32_t*>(p.o + (qrow + i_hi) * D + c) = pack_bf16(o[on][2] * inv_hi, o[on][3] * inv_hi);
  }
  if (tq == 0) {
    if (i_lo < L) {
      if (p.lse) p.lse[qrow + i_lo] = l_lo > 0.f ? (m_lo + log2f(l_lo)) * kLn2 : -INFINITY;
      ms[hh * P + (i_lo - p0)] = m_lo;
      ls[hh * P + (i_lo - p0)] = l_lo;
    }
    if (i_hi < L) {
      if (p.lse) p.lse[qrow + i_hi] = l_hi > 0.f ? (m_hi + log2f(l_hi)) * kLn2 : -INFINITY;
      ms[hh * P + (i_hi - p0)] = m_hi;
      ls[hh * P + (i_hi - p0)] = l_hi;
    }
  }
  // every consumer warp's row statistics and tile maxima are in place (bounded rendezvous; the
  // maxima other warps wrote are read back from L2)
  __threadfence();
  uint32_t cph = 0;
  if (!warps_sync(cbar, cph)) {
    if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
    return;
  }

  // ---- the target of each position: 8 threads per position, blocks strided by 8
  const int sub = tid & 7;
  const int nthr = CW * 32;
  float* gt_b = p.gt + ((size_t)b * p.Hkv + hk) * p.T * p.NB;
  const float* r_b = p.rmax + ((size_t)b * p.Hq + (size_t)hk * g) * p.NB * p.T;
  for (int base = 0; base < P; base += nthr / 8) {
    const int pi = base + tid / 8;
    const int i = p0 + pi;
    const bool live = pi < P && i < L;
    const int nb_i = live ? i / BLK + 1 : 0;   // blocks with a key visible to position i
    // a block's score, four blocks at a time with every load issued before any use (two passes:
    // the sum, then the normalised stores -- no store sits between a load and its successors)
    auto scores4 = [&](int n0, float (&v)[4]) {
      float r[4][kMaxGroup];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int j = 0; j < kMaxGroup; ++j)
          r[u][j] = (j < g && n0 + 8 * u < nb_i) ? __ldcg(r_b + ((size_t)j * p.NB + n0 + 8 * u) * p.T + i) : -INFINITY;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        v[u] = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxGroup; ++j)
          if (j < g && n0 + 8 * u < nb_i) v[u] = fmaxf(v[u], exp2f(r[u][j] - ms[j * P + pi]) / ls[j * P + pi]);
      }
    };
    float sum = 0.f;
    for (int n0 = sub; n0 < nb_i; n0 += 32) {
      float v[4];
      scores4(n0, v);
      sum += (v[0] + v[1]) + (v[2] + v[3]);
    }
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    sum += __shfl_xor_sync(0xffffffffu, sum, 4);
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    if (live) {
      for (int n0 = sub; n0 < nb_i; n0 += 32) {
        float v[4];
        scores4(n0, v);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (n0 + 8 * u < nb_i) gt_b[(size_t)i * p.NB + n0 + 8 * u] = v[u] * inv;
      }
      for (int n = (nb_i & ~7) + sub; n < p.NB; n += 8)
        if (n >= nb_i) gt_b[(size_t)i * p.NB + n] = 0.f;
    }
  }
}

template <int D, int BLK>
cudaError_t launch_t(const CUtensorMap& tk, const CUtensorMap& tv, const PrefillParams& p, int max_len,
                     cudaStream_t st) {
  using S = PrefillShape<D, BLK>;
  auto kern = prefill_gt_kernel<D, BLK>;
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = ensure_smem_limit(kern, (int)S::kSmem, attr_done);
  if (e != cudaSuccess) return e;
  const int wp = 8 / p.g, P = 16 * wp;
  const dim3 grid((max_len + P - 1) / P, p.Hkv, p.B);
  return launch_pdl(kern, grid, dim3((wp * p.g + 1) * 32), S::kSmem, st, tk, tv, p);
}

}  // namespace

cudaError_t launch_prefill_gt(const CUtensorMap& tk, const CUtensorMap& tv, const PrefillParams& p, int D, int BLK,
                              int max_len, cudaStream_t s) {
  if (D == 64 && BLK == 64) return launch_t<64, 64>(tk, tv, p, max_len, s);
  if (D == 64 && BLK == 128) return launch_t<64, 128>(tk, tv, p, max_len, s);
  if (D == 128 && BLK == 64) return launch_t<128, 64>(tk, tv, p, max_len, s);
  if (D == 128 && BLK == 128) return launch_t<128, 128>(tk, tv, p, max_len, s);
  return cudaErrorInvalidValue;
}

}  // namespace seer
