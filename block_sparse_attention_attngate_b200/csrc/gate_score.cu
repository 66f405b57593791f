// AttnGate block logits against the K Compression Cache.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 1-2; "Sparse Attention Adaptation for Long
// Reasoning" (papernotes.org), key design 1 (one W_q per KV head merges the
// group's g query heads):
//   Q_gate = RoPE_{L-1}(W_q[h] . [q_0 | q_1 | ... | q_{g-1}])        (fp32)
//   logit[n] = <Q_gate, K_gate[n]> / sqrt(d_gate),  n < floor(L/b)
//
// One thread-block cluster of CL CTAs per (b, h).  CTA r of the cluster
// computes the RoPE pairs (i, i + d_gate/2) for i in its slice of d_gate/2,
// so each CTA streams only 2/CL of W_q[h] and no CTA repeats the projection;
// it writes its pairs into every peer's shared memory (distributed shared
// memory), and after one cluster barrier each CTA holds the whole Q_gate and
// scores its slice of the cache rows.  Rows n >= floor(L/b) get -inf.
#include <cooperative_groups.h>

#include "seer_device.cuh"
#include "seer_internal.h"

namespace cg = cooperative_groups;

namespace seer {
namespace {

constexpr int kThreads = 256;
constexpr int kCL = 8;

template <int D, int DG>
__global__ void __cluster_dims__(kCL, 1, 1) __launch_bounds__(kThreads) gate_score_kernel(const GateParams p) {
  constexpr int HALF = DG / 2;
  constexpr int RPC = HALF / kCL;          // rotation pairs per CTA
  constexpr int ROWS = 2 * RPC;            // projection rows per CTA
  constexpr int TPR = kThreads / ROWS;     // threads per row
  static_assert(TPR >= 8 && TPR <= 32 && (TPR & (TPR - 1)) == 0, "row split");
  __shared__ float qs[kMaxGroup * D];      // concatenated group query (fp32)
  __shared__ float yrow[ROWS];
  __shared__ __align__(16) float qg[DG];   // full Q_gate (filled by all cluster CTAs)

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int g = p.g, GD = g * D;
  const int L = max(p.seqlens[b], 0);

  const uint16_t* qsrc = p.q + ((size_t)b * p.Hq + (size_t)h * g) * D;   // g rows, head-major
  for (int i = tid; i < GD; i += kThreads) {
    const uint16_t v = qsrc[i];
    qs[i] = __uint_as_float((uint32_t)v << 16);
  }
  __syncthreads();

  // ---- projection rows {rank*RPC + i} and {HALF + rank*RPC + i}
  {
    const int lr = tid / TPR, sub = tid % TPR;
    const int row = lr < RPC ? rank * RPC + lr : HALF + rank * RPC + (lr - RPC);
    const uint16_t* wr = p.w_q + ((size_t)h * DG + row) * GD;
    float acc = 0.f;
    for (int k = sub * 8; k < GD; k += TPR * 8) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(wr + k));
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) acc += bf16_lo(ww[e]) * qs[k + 2 * e] + bf16_hi(ww[e]) * qs[k + 2 * e + 1];
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (sub == 0) yrow[lr] = acc;
  }
  __syncthreads();

  // ---- RoPE at position L-1 (angle in fp64), broadcast the pairs to every CTA of the cluster
  if (tid < RPC) {
    const int j = rank * RPC + tid;
    const double theta = pow((double)p.rope_base, -2.0 * j / DG);
    double sn, cs;
    sincos((double)(L - 1) * theta, &sn, &cs);
    const float c = (float)cs, s = (float)sn;
    const float x1 = yrow[tid], x2 = yrow[RPC + tid];
    const float r1 = x1 * c - x2 * s, r2 = x2 * c + x1 * s;
    for (int peer = 0; peer < kCL; ++peer) {
      float* dst = cluster.map_shared_rank(qg, peer);
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

  // ---- logits of this CTA's slice of full blocks; DG/8 lanes per cache row
  constexpr int LPR = DG / 8;              // lanes per row (16-byte chunks)
  constexpr int RPW = 32 / LPR;            // rows per warp step
  const int nfull = min(L / p.BLK, p.NB);
  const int per = (nfull + kCL - 1) / kCL;
  const int n0 = rank * per, n1 = min(nfull, n0 + per);
  const int warp = tid >> 5, lane = tid & 31;
  const int sub = lane % LPR, rw = lane / LPR;
  float qv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qv[e] = qg[sub * 8 + e];
  const float inv = rsqrtf((float)DG);
  const uint16_t* kc = p.kcomp + ((size_t)b * p.Hkv + h) * p.NB * DG;
  float* lg = p.logits + ((size_t)b * p.Hkv + h) * p.NB;
  for (int nb = n0 + warp * RPW; nb < n1; nb += (kThreads / 32) * RPW) {
    const int n = nb + rw;
    float acc = 0.f;
    if (n < n1) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(kc + (size_t)n * DG + sub * 8));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) acc += bf16_lo(w[e]) * qv[2 * e] + bf16_hi(w[e]) * qv[2 * e + 1];
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (sub == 0 && n < n1) lg[n] = acc * inv;
  }
  for (int n = nfull + rank * kThreads + tid; n < p.NB; n += kCL * kThreads) lg[n] = -INFINITY;
}

template <int D, int DG>
cudaError_t launch_t(const GateParams& p, cudaStream_t s) {
  dim3 grid(kCL, p.Hkv, p.B);
  gate_score_kernel<D, DG><<<grid, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate_score(const GateParams& p, int D, int DG, cudaStream_t s) {
  if (D == 64 && DG == 64) return launch_t<64, 64>(p, s);
  if (D == 64 && DG == 128) return launch_t<64, 128>(p, s);
  if (D == 128 && DG == 64) return launch_t<128, 64>(p, s);
  if (D == 128 && DG == 128) return launch_t<128, 128>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace seer
