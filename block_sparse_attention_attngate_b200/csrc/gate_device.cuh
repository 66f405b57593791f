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
// in its 1/KC of d_gate/2, so it needs only 2/KC of W_q[h]'s rows: two
// contiguous row blocks, bulk-copied into shared memory by one thread before
// the kernel waits for preceding work (weights are never written by work in
// flight on the stream), so they land while the previous kernel runs.  The
// CTA writes its pairs into every peer's shared memory (distributed shared
// memory); after one cluster barrier each CTA holds the whole Q_gate and
// scores its 1/KC of the cache rows.  The query and the cache rows of the
// CTA's slice are loaded up front so their latency overlaps the projection.
// Rows n >= floor(L/b) get -inf.
#pragma once

#include <cooperative_groups.h>

#include "seer_device.cuh"
#include "seer_internal.h"

namespace seer {

template <int D, int DG, int KC>
struct GateSmem {
  float part[8][DG / KC];              // projection partials of the k-ranges
  float yrow[DG / KC];
  alignas(16) float qg[DG];            // full Q_gate (filled by all cluster CTAs)
};

// W_q rows a CTA of a KC-CTA cluster holds in shared memory (padded by 16 bytes so the
// ldmatrix rows fall in distinct banks), and their bytes for group size g.
template <int DG, int KC>
__host__ __device__ constexpr int gate_wq_rows() {
  return DG / KC;
}
template <int D>
__host__ __device__ inline int gate_wq_stride(int g) {   // bf16 elements per shared row
  return g * D + 8;
}
template <int D, int DG, int KC>
__host__ __device__ inline size_t gate_wq_bytes(int g) {
  return (size_t)gate_wq_rows<DG, KC>() * gate_wq_stride<D>(g) * 2;
}

// One thread: arm the barrier `bar` and bulk-copy CTA `rank`'s W_q rows of head h into wq_s
// (shared row i, stride gate_wq_stride: W_q row rank*RPC + i for i < RPC, else
// d_gate/2 + rank*RPC + i - RPC).  Needs no preceding work; the caller syncs the CTA before
// anyone waits on the barrier, and neither `bar` nor wq_s may be reused until the gate has
// waited on it.
template <int D, int DG, int KC>
__device__ void gate_prefetch_wq(const GateParams& p, int h, int rank, uint64_t* bar, uint16_t* wq_s) {
  constexpr int HALF = DG / 2;
  constexpr int RPC = HALF / KC;
  const int GD = p.g * D, ST = gate_wq_stride<D>(p.g);
  const uint32_t row_bytes = (uint32_t)(GD * 2);
  mbar_init(bar, 1);
  fence_barrier_init();
  mbar_arrive_expect_tx(bar, 2 * RPC * row_bytes);
  const uint16_t* base = p.w_q + (size_t)h * DG * GD;
  for (int i = 0; i < 2 * RPC; ++i) {
    const int wrow = i < RPC ? rank * RPC + i : HALF + rank * RPC + (i - RPC);
    bulk_load(wq_s + (size_t)i * ST, base + (size_t)wrow * GD, row_bytes, bar);
  }
}

// Projection tiling: the CTA's 2*RPC = DG/KC W_q rows are MT m-tiles of 16; the 8 warps are
// MT m-tiles x KQ k-ranges, warp w taking m-tile w % MT and k-steps [kq*KS/KQ, (kq+1)*KS/KQ)
// of the KS = g*D/16 steps, kq = w / MT.
template <int DG, int KC>
struct GateTiling {
  static constexpr int kMT = DG / KC / 16;
  static constexpr int kKQ = 8 / kMT;
  static_assert(kMT >= 1 && kMT * 16 == DG / KC && 8 % kMT == 0, "projection rows: whole m-tiles");
};

// The query as the B operand of the projection's mma.sync.m16n8k16 (the query replicated into
// all 8 columns): each lane holds the two bf16 pairs of its fragment for each of its warp's
// k-steps.  Loaded early: it depends on nothing the gate computes.
template <int D, int DG, int KC, int NT>
struct GateQuery {
  using T = GateTiling<DG, KC>;
  static constexpr int kMaxSteps = (kMaxGroup * D / 16 + T::kKQ - 1) / T::kKQ;   // per warp, at most
  uint32_t b0[kMaxSteps], b1[kMaxSteps];
  __device__ void load(const GateParams& p, int b, int h) {
    const int KS = p.g * D / 16;
    const int kq = ((int)threadIdx.x >> 5) / T::kMT, t = (int)threadIdx.x & 3;
    const int ks0 = kq * KS / T::kKQ, ks1 = (kq + 1) * KS / T::kKQ;
    const uint16_t* qsrc = p.q + ((size_t)b * p.Hq + (size_t)h * p.g) * D;   // g rows, head-major
#pragma unroll
    for (int i = 0; i < kMaxSteps; ++i) {
      const bool on = ks0 + i < ks1;
      const int k = (ks0 + i) * 16 + 2 * t;
      b0[i] = on ? __ldg(reinterpret_cast<const uint32_t*>(qsrc + k)) : 0u;
      b1[i] = on ? __ldg(reinterpret_cast<const uint32_t*>(qsrc + k + 8)) : 0u;
    }
  }
};

// All NT threads of every CTA of the cluster call this, after gate_prefetch_wq (same wq_bar,
// wq_s).  L is the sequence length (current token included), q the preloaded query.  If `row0`
// is given (a distributed-shared-memory pointer into rank 0's row buffer), each logit is stored
// there instead of p.logits; the caller syncs the cluster before reading it.  If the W_q copy does not land
// within the wait bound the logits come out NaN (every CTA still takes the cluster barriers).
template <int D, int DG, int KC, int NT>
__device__ void gate_cluster(const GateParams& p, int b, int h, int rank, int L, const GateQuery<D, DG, KC, NT>& q,
                             cooperative_groups::cluster_group& cluster, GateSmem<D, DG, KC>& sm, uint64_t* wq_bar,
                             const uint16_t* wq_s, float* row0) {
  constexpr int HALF = DG / 2;
  constexpr int RPC = HALF / KC;           // rotation pairs per CTA
  constexpr int ROWS = 2 * RPC;            // projection rows per CTA
  using Tl = GateTiling<DG, KC>;
  static_assert(NT >= 256 && NT % 32 == 0, "projection: warps 0..7 (any further warps only score)");
  constexpr int LPR = DG / 8;              // lanes per cache row (16-byte chunks)
  constexpr int RPW = 32 / LPR;            // cache rows per warp step
  constexpr int RPS = (NT / 32) * RPW;     // cache rows per CTA step
  constexpr int PRE = 8;                   // CTA steps of rows held in registers at a time
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = p.g, GD = g * D;

  const int nfull = min(L / p.BLK, p.NB);
  const int per = (nfull + KC - 1) / KC;
  const int n0 = rank * per, n1 = min(nfull, n0 + per);
  const int sub = lane % LPR, rw = lane / LPR;
  const uint16_t* kc = p.kcomp + ((size_t)b * p.Hkv + h) * p.NB * DG;
  auto load_rows = [&](int st0, uint4 (&kv)[PRE]) {
#pragma unroll
    for (int st = 0; st < PRE; ++st) {
      const int n = n0 + (st0 + st) * RPS + warp * RPW + rw;
      kv[st] = n < n1 ? __ldg(reinterpret_cast<const uint4*>(kc + (size_t)n * DG + sub * 8)) : make_uint4(0, 0, 0, 0);
    }
  };

  // ---- the first PRE steps of this CTA's cache rows: they do not depend on Q_gate
  uint4 kv[PRE];
  load_rows(0, kv);

  const bool wq_ok = __syncthreads_and(mbar_wait(wq_bar, 0));
  {
    // projection on the tensor pipe: y[row] = W_q[row] . q for the CTA's ROWS rows, A from the
    // shared rows by ldmatrix; two accumulators halve the mma chain
    // warps past the first 8 get kq >= kKQ: no k-steps, and their (zero) partials land in slots
    // the sum below does not read
    const int mt = warp % Tl::kMT, kq = warp / Tl::kMT;
    const int KS = GD / 16, ST = gate_wq_stride<D>(g);
    const int ks0 = kq * KS / Tl::kKQ, ks1 = (kq + 1) * KS / Tl::kKQ;
    const uint32_t a_base = smem_u32(wq_s + (size_t)(mt * 16 + (lane & 15)) * ST + (lane >> 4) * 8);
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int i = 0; i < GateQuery<D, DG, KC, NT>::kMaxSteps; ++i) {
      if (ks0 + i < ks1) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(a_base + (uint32_t)((ks0 + i) * 16 * 2), a0, a1, a2, a3);
        mma_bf16_16816(acc[i & 1], a0, a1, a2, a3, q.b0[i], q.b1[i]);
      }
    }
    // every column of the product is y; lanes with lane % 4 == 0 hold column 0 of rows lane/4, +8
    if ((lane & 3) == 0) {
      sm.part[kq][mt * 16 + (lane >> 2)] = acc[0][0] + acc[1][0];
      sm.part[kq][mt * 16 + (lane >> 2) + 8] = acc[0][2] + acc[1][2];
    }
  }
  __syncthreads();
  if (tid < ROWS) {
    float y = 0.f;
#pragma unroll
    for (int k = 0; k < Tl::kKQ; ++k) y += sm.part[k][tid];
    sm.yrow[tid] = wq_ok ? y : __int_as_float(0x7fc00000);
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

  // ---- logits of this CTA's slice of full blocks: PRE rows per lane at a time, their partial
  // dot products first, then the LPR-lane reductions side by side
  float qv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qv[e] = sm.qg[sub * 8 + e];
  const float inv = rsqrtf((float)DG);
  // with a rank-0 row the caller writes the finished row out after its cluster barrier (stores
  // issued before a barrier with release semantics would have to complete first)
  float* lg = (p.logits && !row0) ? p.logits + ((size_t)b * p.Hkv + h) * p.NB : nullptr;
  for (int st0 = 0; n0 + st0 * RPS < n1; st0 += PRE) {
    uint4 kn[PRE];
    const bool more = n0 + (st0 + PRE) * RPS < n1;
    if (more) load_rows(st0 + PRE, kn);   // the next group's rows, in flight during this one
    float part[PRE];
#pragma unroll
    for (int st = 0; st < PRE; ++st) {
      const uint32_t w[4] = {kv[st].x, kv[st].y, kv[st].z, kv[st].w};
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) a += bf16_lo(w[e]) * qv[2 * e] + bf16_hi(w[e]) * qv[2 * e + 1];
      part[st] = a;
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) {
#pragma unroll
      for (int st = 0; st < PRE; ++st) part[st] += __shfl_xor_sync(0xffffffffu, part[st], off);
    }
    if (sub == 0) {
#pragma unroll
      for (int st = 0; st < PRE; ++st) {
        const int n = n0 + (st0 + st) * RPS + warp * RPW + rw;
        if (n < n1) {
          if (lg) lg[n] = part[st] * inv;
          if (row0) row0[n] = part[st] * inv;
        }
      }
    }
    if (!more) break;
#pragma unroll
    for (int st = 0; st < PRE; ++st) kv[st] = kn[st];
  }
  if (lg)
    for (int n = nfull + rank * NT + tid; n < p.NB; n += KC * NT) lg[n] = -INFINITY;
}

}  // namespace seer
