// AttnGate block logits of one (b, h) computed by a thread-block cluster, as a
// device routine shared by the standalone gate kernel and the fused plan kernel.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 1-2; "Sparse Attention Adaptation for Long
// Reasoning" (papernotes.org), key design 1 (one W_q per KV head merges the
// group's g query heads):
//   Q_gate = RoPE_{L-1}(W_q[h] . [q_0 | q_1 | ... | q_{g-1}])        (fp32)
//   logit[n] = <Q_gate, K_gate[n]> / sqrt(d_gate),  n < floor(L/b)
//
// CTA r of the KC-CTA cluster computes the RoPE pairs (i, i + d_gate/2) for i
// in its 1/KC of d_gate/2 (so each CTA streams only 2/KC of W_q[h]), writes
// them into every peer's shared memory (distributed shared memory), and after
// one cluster barrier each CTA holds the whole Q_gate and scores its 1/KC of
// the cache rows.  The cache rows of the CTA's slice are loaded before the
// projection so their latency overlaps it.  Rows n >= floor(L/b) get -inf.
#pragma once

#include <cooperative_groups.h>

#include "seer_device.cuh"
#include "seer_internal.h"

namespace seer {

template <int D, int DG, int KC>
struct GateSmem {
  float qs[kMaxGroup * D];             // concatenated group query (fp32)
  float yrow[DG / KC];
  alignas(16) float qg[DG];            // full Q_gate (filled by all cluster CTAs)
};

// All NT threads of every CTA of the cluster call this.  If `row0` is given (a
// distributed-shared-memory pointer into rank 0's row buffer), each logit is
// also stored there; the caller syncs the cluster before reading it.
template <int D, int DG, int KC, int NT>
__device__ void gate_cluster(const GateParams& p, int b, int h, int rank, cooperative_groups::cluster_group& cluster,
                             GateSmem<D, DG, KC>& sm, float* row0) {
  constexpr int HALF = DG / 2;
  constexpr int RPC = HALF / KC;           // rotation pairs per CTA
  constexpr int ROWS = 2 * RPC;            // projection rows per CTA
  constexpr int TPR = NT / ROWS;           // threads per projection row
  constexpr int WQ_IT = kMaxGroup * D / (TPR * 8);   // 16-byte W_q chunks per thread (at most)
  constexpr int LPR = DG / 8;              // lanes per cache row (16-byte chunks)
  constexpr int RPW = 32 / LPR;            // cache rows per warp step
  constexpr int RPS = (NT / 32) * RPW;     // cache rows per CTA step
  constexpr int PRE = 8;                   // CTA steps whose rows are loaded before the projection
  static_assert(TPR >= 4 && TPR <= 32 && (TPR & (TPR - 1)) == 0, "row split");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = p.g, GD = g * D;

  // ---- W_q chunks of this thread's projection row and the group query: independent of L, issued first
  const int lr = tid / TPR, tsub = tid % TPR;
  const int prow = lr < RPC ? rank * RPC + lr : HALF + rank * RPC + (lr - RPC);
  const uint16_t* wr = p.w_q + ((size_t)h * DG + prow) * GD;
  uint4 wv[WQ_IT];
#pragma unroll
  for (int it = 0; it < WQ_IT; ++it) {
    const int k = (it * TPR + tsub) * 8;
    wv[it] = k < GD ? __ldg(reinterpret_cast<const uint4*>(wr + k)) : make_uint4(0, 0, 0, 0);
  }
  const uint16_t* qsrc = p.q + ((size_t)b * p.Hq + (size_t)h * g) * D;   // g rows, head-major
  constexpr int QIT = (kMaxGroup * D + NT - 1) / NT;
  uint16_t qv16[QIT];
#pragma unroll
  for (int it = 0; it < QIT; ++it) {
    const int i = it * NT + tid;
    qv16[it] = i < GD ? qsrc[i] : (uint16_t)0;
  }

  const int L = max(p.seqlens[b], 0);
  const int nfull = min(L / p.BLK, p.NB);
  const int per = (nfull + KC - 1) / KC;
  const int n0 = rank * per, n1 = min(nfull, n0 + per);
  const int sub = lane % LPR, rw = lane / LPR;
  const uint16_t* kc = p.kcomp + ((size_t)b * p.Hkv + h) * p.NB * DG;

  // ---- cache rows of this CTA's slice: they do not depend on Q_gate
  uint4 kv[PRE];
#pragma unroll
  for (int st = 0; st < PRE; ++st) {
    const int n = n0 + st * RPS + warp * RPW + rw;
    kv[st] = n < n1 ? __ldg(reinterpret_cast<const uint4*>(kc + (size_t)n * DG + sub * 8)) : make_uint4(0, 0, 0, 0);
  }

#pragma unroll
  for (int it = 0; it < QIT; ++it) {
    const int i = it * NT + tid;
    if (i < GD) sm.qs[i] = __uint_as_float((uint32_t)qv16[it] << 16);
  }
  __syncthreads();
  {
    float acc = 0.f;
#pragma unroll
    for (int it = 0; it < WQ_IT; ++it) {
      const int k = (it * TPR + tsub) * 8;
      if (k < GD) {
        const uint32_t ww[4] = {wv[it].x, wv[it].y, wv[it].z, wv[it].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) acc += bf16_lo(ww[e]) * sm.qs[k + 2 * e] + bf16_hi(ww[e]) * sm.qs[k + 2 * e + 1];
      }
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (tsub == 0) sm.yrow[lr] = acc;
  }
  __syncthreads();

  // ---- RoPE at position L-1, broadcast the pairs to every CTA of the cluster
  if (tid < RPC) {
    const int j = rank * RPC + tid;
    float c, s;
    rope_cos_sin((double)(L - 1) * p.theta[j], c, s);
    const float x1 = sm.yrow[tid], x2 = sm.yrow[RPC + tid];
    const float r1 = x1 * c - x2 * s, r2 = x2 * c + x1 * s;
    for (int peer = 0; peer < KC; ++peer) {
      float* dst = cluster.map_shared_rank(sm.qg, peer);
      dst[j] = r1;
      dst[j + HALF] = r2;
    }
    if (p.q_gate) {
      float* o = p.q_gate + ((size_t)b * p.Hkv + h) * DG;
      o[j] = r1;
      o[j + HALF] = r2;
    }
  }
  cluster.sync();

  // ---- logits of this CTA's slice of full blocks
  float qv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qv[e] = sm.qg[sub * 8 + e];
  const float inv = rsqrtf((float)DG);
  float* lg = p.logits ? p.logits + ((size_t)b * p.Hkv + h) * p.NB : nullptr;
  auto score = [&](const uint4& v, int n) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc += bf16_lo(w[e]) * qv[2 * e] + bf16_hi(w[e]) * qv[2 * e + 1];
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (sub == 0 && n < n1) {
      if (lg) lg[n] = acc * inv;
      if (row0) row0[n] = acc * inv;
    }
  };
#pragma unroll
  for (int st = 0; st < PRE; ++st)
    if (n0 + st * RPS < n1) score(kv[st], n0 + st * RPS + warp * RPW + rw);
  for (int st = PRE; n0 + st * RPS < n1; ++st) {
    const int n = n0 + st * RPS + warp * RPW + rw;
    score(n < n1 ? __ldg(reinterpret_cast<const uint4*>(kc + (size_t)n * DG + sub * 8)) : make_uint4(0, 0, 0, 0), n);
  }
  if (lg)
    for (int n = nfull + rank * NT + tid; n < p.NB; n += KC * NT) lg[n] = -INFINITY;
}

}  // namespace seer
