// Block-sparse flash decoding over the selected KV blocks, with the split
// log-sum-exp combine fused into the last CTA of each (batch, kv head).
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 6: grid (batch, heads_kv, num_split); the
// selected list [batch, heads_kv, max_selected_blocks] is split by its width,
// and the kernel visits only the active block indices.  The page's H100
// kernel pads the query group to 64 rows for wgmma; here the group (g <= 8
// query heads) stays a 16-row mma.sync fragment, because the work per KV byte
// is ~g multiply-adds and the bound is HBM, not the tensor pipe.
//
// CTA = one (split, kv head, batch).  Warp NW (the last) is the producer: one
// lane walks the split's block list and issues 128B-swizzled TMA tile loads
// of K and V into a STAGES-deep shared-memory ring (mbarrier complete_tx).
// Warps 0..NW-1 are consumers; each owns BLK/NW tokens of every block:
//   S   = Q K^T   (A = Q fragment in registers, B = K via ldmatrix)
//   P   = exp2(S*scale*log2e - m)   (fp32 online softmax per query head)
//   O^T += V^T P^T  (A = V via ldmatrix.trans, B = P straight from S's C fragment)
// The consumers' states merge in shared memory; with num_split > 1 each CTA
// writes a partial (o, lse) and the last arriving CTA of the (b, h) merges
// them and writes bf16 out.
#include "seer_device.cuh"
#include "seer_internal.h"

namespace seer {
namespace {

constexpr float kLn2 = 0.6931471805599453f;

template <int D, int BLK, int NW, int STAGES>
struct DecodeShape {
  static constexpr int kTile = BLK * D * 2;   // bytes of one K (or V) tile
  static constexpr int kBox = BLK * 128;      // bytes of one 64-channel box
  static constexpr int kNBox = D / 64;
  static constexpr int kTPW = BLK / NW;       // tokens per consumer warp per block
  static constexpr int kNT = kTPW / 8;        // 8-token S tiles per warp
  static constexpr int kKS = kTPW / 16;       // 16-token PV k-steps per warp
  static constexpr int kDK = D / 16;          // QK^T k-steps == PV m-tiles
  static constexpr int kThreads = (NW + 1) * 32;
  static constexpr int kRing = STAGES * 2 * kTile;
  static constexpr size_t kSmem = 1024 + kRing + STAGES * 16 + STAGES * 4 + 16;
  static_assert(kTPW % 16 == 0, "each consumer warp needs whole 16-token steps");
  static_assert(D % 64 == 0, "head_dim must be a multiple of 64");
  // merge scratch (reuses the ring): NW * 8 * D floats + m, l
  static_assert(NW * kMaxGroup * D * 4 + 2 * NW * kMaxGroup * 4 <= kRing, "merge buffer");
};

__device__ __forceinline__ void tile_coords(const int32_t perm[3], int t, int h, int bp, int& c1,
                                            int& c2, int& c3) {
  int c[3];
  c[perm[0]] = t;
  c[perm[1]] = h;
  c[perm[2]] = bp;
  c1 = c[0];
  c2 = c[1];
  c3 = c[2];
}

template <int D, int BLK, int NW, int STAGES>
__global__ void __launch_bounds__(DecodeShape<D, BLK, NW, STAGES>::kThreads)
    sparse_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  using S = DecodeShape<D, BLK, NW, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kRing);
  uint64_t* empty = full + STAGES;
  int* info = reinterpret_cast<int*>(empty + STAGES);
  volatile int* flags = info + STAGES;  // [0] abort, [1] last-CTA

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = max(p.seqlens[b], 0);
  const int nblk = (L + BLK - 1) / BLK;
  int count = p.cnt[b * p.Hkv + h];
  if (count > p.cap) {
    if (threadIdx.x == 0) report(p.err, SEER_DEVERR_COUNT);
    count = p.cap;
  }
  count = max(count, 0);
  const int pos0 = split * p.per_split;
  const int nit = max(0, min(pos0 + p.per_split, count) - pos0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NW);
    }
    flags[0] = 0;
    flags[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == NW) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nit > 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int32_t* list = p.idx + ((size_t)b * p.Hkv + h) * p.cap + pos0;
      for (int it = 0; it < nit; ++it) {
        const int s = it % STAGES;
        if (it >= STAGES && !mbar_wait(&empty[s], ((it / STAGES) - 1) & 1)) {
          report(p.err, SEER_DEVERR_TIMEOUT);
          flags[0] = 1;
          break;
        }
        if (flags[0]) break;
        const int n = list[it];
        bool ok = n >= 0 && n < nblk;
        if (!ok) report(p.err, SEER_DEVERR_BLOCK_INDEX);
        int kb = b, vb = b, kt = n * BLK, vt = n * BLK;
        if (ok && p.k_paged) {
          const int pg = n < p.k_maxp ? p.k_table[(size_t)b * p.k_maxp + n] : -1;
          if (pg < 0 || pg >= p.k_pages) {
            report(p.err, SEER_DEVERR_PAGE_INDEX);
            ok = false;
          }
          kb = pg;
          kt = 0;
        }
        if (ok && p.v_paged) {
          const int pg = n < p.v_maxp ? p.v_table[(size_t)b * p.v_maxp + n] : -1;
          if (pg < 0 || pg >= p.v_pages) {
            report(p.err, SEER_DEVERR_PAGE_INDEX);
            ok = false;
          }
          vb = pg;
          vt = 0;
        }
        info[s] = ok ? n : -1;
        if (ok) {
          uint8_t* kdst = ring + s * 2 * S::kTile;
          uint8_t* vdst = kdst + S::kTile;
          mbar_arrive_expect_tx(&full[s], 2 * S::kTile);
          int c1, c2, c3;
          tile_coords(p.k_perm, kt, h, kb, c1, c2, c3);
#pragma unroll
          for (int bx = 0; bx < S::kNBox; ++bx) tma_load_4d(kdst + bx * S::kBox, &tmK, &full[s], bx * 64, c1, c2, c3);
          tile_coords(p.v_perm, vt, h, vb, c1, c2, c3);
#pragma unroll
          for (int bx = 0; bx < S::kNBox; ++bx) tma_load_4d(vdst + bx * S::kBox, &tmV, &full[s], bx * 64, c1, c2, c3);
        } else {
          mbar_arrive(&full[s]);
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gq = lane >> 2, tq = lane & 3;
  const int g = p.g;
  uint32_t qa[S::kDK][2];
  {
    const bool live = gq < g;
    const uint16_t* qrow = p.q + ((size_t)b * p.Hq + (size_t)h * g + (live ? gq : 0)) * D;
#pragma unroll
    for (int ks = 0; ks < S::kDK; ++ks) {
      qa[ks][0] = live ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * tq) : 0u;
      qa[ks][1] = live ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 8 + 2 * tq) : 0u;
    }
  }
  float o[S::kDK][4];
#pragma unroll
  for (int i = 0; i < S::kDK; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  const float sl2 = p.scale_log2;
  const int tok_base = warp * S::kTPW;
  int consumed = 0;

  for (int it = 0; it < nit; ++it) {
    const int s = it % STAGES;
    // every lane observes the phase (acquire); the warp leaves together if any lane gave up
    const bool landed = __all_sync(0xffffffffu, mbar_wait(&full[s], (it / STAGES) & 1));
    if (!landed) {
      if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
      flags[0] = 1;
      break;
    }
    consumed = it + 1;
    const int n = info[s];
    if (n >= 0) {
      const uint32_t kt = smem_u32(ring + s * 2 * S::kTile);
      const uint32_t vt = kt + S::kTile;
      const int valid = min(BLK, L - n * BLK);
      // ---- S = Q K^T for this warp's tokens
      float sacc[S::kNT][4];
#pragma unroll
      for (int j = 0; j < S::kNT; ++j) {
        sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
        const uint32_t row = tok_base + j * 8 + (lane & 7);
#pragma unroll
        for (int kp = 0; kp < S::kDK / 2; ++kp) {
          const uint32_t chunk = kp * 4 + (lane >> 3);
          uint32_t r0, r1, r2, r3;
          ldsm_x4(kt + (chunk >> 3) * S::kBox + sw128(row, chunk & 7), r0, r1, r2, r3);
          mma_bf16_16816(sacc[j], qa[2 * kp][0], 0u, qa[2 * kp][1], 0u, r0, r1);
          mma_bf16_16816(sacc[j], qa[2 * kp + 1][0], 0u, qa[2 * kp + 1][1], 0u, r2, r3);
        }
      }
      // ---- online softmax (row = query head gq; this lane holds tokens 2tq, 2tq+1 of each tile)
      float sv[S::kNT][2];
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < S::kNT; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int tok = tok_base + j * 8 + 2 * tq + e;
          const float v = tok < valid ? sacc[j][e] * sl2 : -INFINITY;
          sv[j][e] = v;
          mx = fmaxf(mx, v);
        }
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run, mx);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = exp2f(m_run - m_use);
      m_run = m_new;
      uint32_t pb[S::kNT];
      float ls = 0.f;
#pragma unroll
      for (int j = 0; j < S::kNT; ++j) {
        pb[j] = pack_bf16(exp2f(sv[j][0] - m_use), exp2f(sv[j][1] - m_use));
        ls += bf16_lo(pb[j]) + bf16_hi(pb[j]);
      }
      l_run = l_run * alpha + ls;
      const float a0 = __shfl_sync(0xffffffffu, alpha, (2 * tq) * 4);
      const float a1 = __shfl_sync(0xffffffffu, alpha, (2 * tq + 1) * 4);
#pragma unroll
      for (int i = 0; i < S::kDK; ++i) {
        o[i][0] *= a0;
        o[i][1] *= a1;
        o[i][2] *= a0;
        o[i][3] *= a1;
      }
      // ---- O^T += V^T P^T
      const bool ragged = valid < BLK;
#pragma unroll
      for (int kk = 0; kk < S::kKS; ++kk) {
        const uint32_t b0 = pb[2 * kk], b1 = pb[2 * kk + 1];
        const int k0 = tok_base + kk * 16;
        const uint32_t mi = lane >> 3;
        const uint32_t row = k0 + (lane & 7) + ((mi >> 1) << 3);
        const int t_lo = k0 + 2 * tq;      // tokens of fragment halves: t_lo, t_lo+1, t_lo+8, t_lo+9
#pragma unroll
        for (int i = 0; i < S::kDK; ++i) {
          const uint32_t chunk = 2 * i + (mi & 1);
          uint32_t v0, v1, v2, v3;
          ldsm_x4_trans(vt + (chunk >> 3) * S::kBox + sw128(row, chunk & 7), v0, v1, v2, v3);
          if (ragged) {
            // rows past L may hold anything (even NaN): zero them so 0 * V stays 0
            const uint32_t m01 = (t_lo < valid ? 0x0000ffffu : 0u) | (t_lo + 1 < valid ? 0xffff0000u : 0u);
            const uint32_t m23 = (t_lo + 8 < valid ? 0x0000ffffu : 0u) | (t_lo + 9 < valid ? 0xffff0000u : 0u);
            v0 &= m01;
            v1 &= m01;
            v2 &= m23;
            v3 &= m23;
          }
          mma_bf16_16816(o[i], v0, v1, v2, v3, b0, b1);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // consumers of an aborted CTA drain the copies still in flight (bounded)
  if (flags[0] && warp == 0 && lane == 0) {
    for (int it = consumed; it < nit && it < consumed + STAGES; ++it)
      mbar_wait(&full[it % STAGES], (it / STAGES) & 1);
  }

  // -------------------------------------------------------------- merge the NW warps
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  asm volatile("bar.sync 1, %0;" ::"n"(NW * 32));   // ring no longer read by anyone
  float* Ow = reinterpret_cast<float*>(ring);                 // [NW][8][D]
  float* Mw = Ow + NW * kMaxGroup * D;                        // [NW][8]
  float* Lw = Mw + NW * kMaxGroup;                            // [NW][8]
  if (tq == 0 && gq < g) {
    Mw[warp * kMaxGroup + gq] = m_run;
    Lw[warp * kMaxGroup + gq] = l_run;
  }
#pragma unroll
  for (int i = 0; i < S::kDK; ++i) {
    const int d0 = i * 16 + gq;
    const int h0 = 2 * tq, h1 = 2 * tq + 1;
    float* base = Ow + warp * kMaxGroup * D;
    if (h0 < g) {
      base[h0 * D + d0] = o[i][0];
      base[h0 * D + d0 + 8] = o[i][2];
    }
    if (h1 < g) {
      base[h1 * D + d0] = o[i][1];
      base[h1 * D + d0 + 8] = o[i][3];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(NW * 32));

  const int tid = threadIdx.x;
  const int ns = p.ns;
  const size_t qh0 = (size_t)b * p.Hq + (size_t)h * g;   // first query head of the group
  for (int e = tid; e < g * D; e += NW * 32) {
    const int j = e / D, c = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, Mw[w * kMaxGroup + j]);
    float num = 0.f, den = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float sc = exp2f(Mw[w * kMaxGroup + j] - M);
        num += sc * Ow[(w * kMaxGroup + j) * D + c];
        den += sc * Lw[w * kMaxGroup + j];
      }
    }
    const bool any = den > 0.f;
    const float oval = any ? num / den : 0.f;
    const float lse = any ? (M + log2f(den)) * kLn2 : -INFINITY;
    if (ns == 1) {
      __nv_bfloat16 ob = __float2bfloat16_rn(oval);
      p.out[(qh0 + j) * D + c] = *reinterpret_cast<uint16_t*>(&ob);
      if (c == 0 && p.lse_out) p.lse_out[qh0 + j] = lse;
    } else {
      p.o_part[((qh0 + j) * ns + split) * D + c] = oval;
      if (c == 0) p.lse_part[(qh0 + j) * ns + split] = lse;
    }
  }
  if (ns == 1) return;

  // -------------------------------------------------------------- last CTA of (b, h) merges the splits
  __threadfence();
  asm volatile("bar.sync 1, %0;" ::"n"(NW * 32));
  if (tid == 0) {
    const int prev = atomicAdd(&p.counters[b * p.Hkv + h], 1);
    flags[1] = prev == ns - 1;
  }
  asm volatile("bar.sync 1, %0;" ::"n"(NW * 32));
  if (!flags[1]) return;
  __threadfence();
  for (int e = tid; e < g * D; e += NW * 32) {
    const int j = e / D, c = e % D;
    const float* lrow = p.lse_part + (qh0 + j) * ns;
    const float* orow = p.o_part + (qh0 + j) * ns * D + c;
    float M = -INFINITY;
    for (int s2 = 0; s2 < ns; ++s2) M = fmaxf(M, __ldcg(lrow + s2));
    float num = 0.f, den = 0.f;
    if (M != -INFINITY) {
      for (int s2 = 0; s2 < ns; ++s2) {
        const float w = expf(__ldcg(lrow + s2) - M);
        num += w * __ldcg(orow + (size_t)s2 * D);
        den += w;
      }
    }
    const bool any = den > 0.f;
    __nv_bfloat16 ob = __float2bfloat16_rn(any ? num / den : 0.f);
    p.out[(qh0 + j) * D + c] = *reinterpret_cast<uint16_t*>(&ob);
    if (c == 0 && p.lse_out) p.lse_out[qh0 + j] = any ? M + logf(den) : -INFINITY;
  }
  if (tid == 0) p.counters[b * p.Hkv + h] = 0;
}

template <int D, int BLK>
struct Choice;
// consumer warps / ring depth per shape (stage = 2 * BLK * D * 2 bytes)
template <> struct Choice<64, 64> { static constexpr int NW = 4, ST = 6; };
template <> struct Choice<64, 128> { static constexpr int NW = 4, ST = 4; };
template <> struct Choice<128, 64> { static constexpr int NW = 4, ST = 4; };
template <> struct Choice<128, 128> { static constexpr int NW = 4, ST = 3; };

template <int D, int BLK>
cudaError_t launch_t(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p, cudaStream_t st) {
  constexpr int NW = Choice<D, BLK>::NW, ST = Choice<D, BLK>::ST;
  using Sh = DecodeShape<D, BLK, NW, ST>;
  auto kern = sparse_decode_kernel<D, BLK, NW, ST>;
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = ensure_smem_limit(kern, (int)Sh::kSmem, attr_done);
  if (e != cudaSuccess) return e;
  dim3 grid(p.ns, p.Hkv, p.B);
  kern<<<grid, Sh::kThreads, Sh::kSmem, st>>>(tk, tv, p);
  return cudaGetLastError();
}

template <int D, int BLK>
int ctas_per_sm_t() {
  constexpr int NW = Choice<D, BLK>::NW, ST = Choice<D, BLK>::ST;
  using Sh = DecodeShape<D, BLK, NW, ST>;
  auto kern = sparse_decode_kernel<D, BLK, NW, ST>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Sh::kSmem) != cudaSuccess)
    return 1;
  int n = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, Sh::kThreads, Sh::kSmem) != cudaSuccess) return 1;
  return n > 0 ? n : 1;
}

}  // namespace

DecodeConfig decode_config(int D, int BLK) {
#define SEER_CFG(d, blk)                                                              \
  if (D == d && BLK == blk) {                                                         \
    using C = Choice<d, blk>;                                                         \
    return DecodeConfig{C::ST, C::NW, DecodeShape<d, blk, C::NW, C::ST>::kSmem};      \
  }
  SEER_CFG(64, 64)
  SEER_CFG(64, 128)
  SEER_CFG(128, 64)
  SEER_CFG(128, 128)
#undef SEER_CFG
  return DecodeConfig{0, 0, 0};
}

int decode_ctas_per_sm(int D, int BLK) {
  if (D == 64 && BLK == 64) return ctas_per_sm_t<64, 64>();
  if (D == 64 && BLK == 128) return ctas_per_sm_t<64, 128>();
  if (D == 128 && BLK == 64) return ctas_per_sm_t<128, 64>();
  if (D == 128 && BLK == 128) return ctas_per_sm_t<128, 128>();
  return 1;
}

cudaError_t launch_sparse_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p, int D,
                                 int BLK, cudaStream_t s) {
  if (D == 64 && BLK == 64) return launch_t<64, 64>(tk, tv, p, s);
  if (D == 64 && BLK == 128) return launch_t<64, 128>(tk, tv, p, s);
  if (D == 128 && BLK == 64) return launch_t<128, 64>(tk, tv, p, s);
  if (D == 128 && BLK == 128) return launch_t<128, 128>(tk, tv, p, s);
  return cudaErrorInvalidValue;
}

}  // namespace seer
