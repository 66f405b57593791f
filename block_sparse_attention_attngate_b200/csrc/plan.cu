// The per-step planning half of the decode in one launch: K Compression Cache
// update, AttnGate logits and block selection for each (b, h), run by one
// 4-CTA thread-block cluster per (b, h).
//
//   1. new full blocks of (b, h) (if any) -> cache rows      (kcomp_device.cuh)
//   2. Q_gate shared through distributed shared memory, each CTA scores its
//      1/4 of the cache rows, writing the logits into rank 0's row  (gate_device.cuh);
//      each CTA's W_q rows are bulk-copied before the kernel waits for the
//      preceding launch, so they land while it still runs
//   3. rank 0 selects the blocks from that row, keys in registers for rows of
//      up to 2048 blocks, in shared memory beyond that or for top-p (select_device.cuh)
// Equivalent to seer_kcomp_update + seer_gate_score + seer_select_blocks, with
// two kernel boundaries and the logits' round trip through global memory
// removed; the sources of each step are cited in its header.
#include <cooperative_groups.h>

#include <algorithm>

#include "gate_device.cuh"
#include "kcomp_device.cuh"
#include "select_device.cuh"

namespace cg = cooperative_groups;

namespace seer {
namespace {

constexpr int kThreads = 256;
#ifndef SEER_GATE_CLUSTER
#define SEER_GATE_CLUSTER 4   // CTAs per (b, h) cluster
#endif
constexpr int kCL = SEER_GATE_CLUSTER;

template <int D, int DG>
union PlanSmem {
  KcompSmem<D, DG, kThreads> k;
  GateSmem<D, DG, kCL> g;
};

template <int D, int BLK, int DG>
__global__ void __cluster_dims__(kCL, 1, 1) __launch_bounds__(kThreads) plan_kernel(const PlanParams p) {
  __shared__ PlanSmem<D, DG> sm;
  __shared__ union {
    SelectScratch sc;
    SelectRegsScratch sr;
  } ss;
  __shared__ uint64_t wq_bar;
  SelectScratch& sc = ss.sc;
  SelectRegsScratch& sr = ss.sr;
  // [NB] logits (rank 0), then a region used first for this CTA's W_q rows, then (rank 0) for
  // the selection keys / pairs
  extern __shared__ __align__(16) float row[];
  const int nb4 = (p.s.NB + 3) & ~3;
  uint16_t* wq_s = reinterpret_cast<uint16_t*>(row + nb4);
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int h = blockIdx.y, b = blockIdx.z, bh = b * p.g.Hkv + h;
  if (threadIdx.x == 0) gate_prefetch_wq<D, DG, kCL>(p.g, h, rank, &wq_bar, wq_s);   // weights: no wait needed
  // The parameters are fixed for the launch: bring them into the constant cache before the wait
  // (the RoPE table alone spans eight 64-byte lines), so no first use afterwards waits on memory.
  asm volatile("" ::"d"(p.g.theta[threadIdx.x % kMaxHalfGate]), "l"(p.g.q), "l"(p.g.kcomp), "l"(p.g.seqlens),
               "l"(p.s.idx), "l"(p.s.cnt), "l"(p.k.valid), "r"(p.s.NB), "r"(p.s.cap), "r"(p.s.kblocks),
               "d"(p.s.tau), "r"(p.update_cache));
  pdl_wait();
  pdl_trigger();
  GateQuery<D, DG, kCL, kThreads> q;
  q.load(p.g, b, h);
  const int L = max(p.g.seqlens[b], 0);
  int nfull_k = 0;
  if (p.update_cache) {
    nfull_k = kcomp_nfull<BLK>(p.k, L);
    const int v0 = max(p.k.valid[bh], 0);
    if (nfull_k > v0) {   // the same decision in every CTA of the cluster
      kcomp_update_share<D, BLK, DG, kThreads>(p.k, b, h, v0, nfull_k, rank, kCL, sm.k);
      __threadfence();    // the new rows are read by the other CTAs of the cluster below
      cluster.sync();
    }
  }
  gate_cluster<D, DG, kCL, kThreads>(p.g, b, h, rank, L, q, cluster, sm.g, &wq_bar, wq_s, cluster.map_shared_rank(row, 0));
  cluster.sync();   // rank 0's row is complete; every CTA has read the fill count
  if (rank != 0) return;
  const int nfull = min(L / p.s.BLK, p.s.NB);
  if (p.g.logits) {   // the optional logits output, off the cluster barriers' path
    float* lg = p.g.logits + (size_t)bh * p.s.NB;
    for (int n = threadIdx.x; n < p.s.NB; n += kThreads) lg[n] = n < nfull ? row[n] : -INFINITY;
  }
  uint32_t* keys = reinterpret_cast<uint32_t*>(row + nb4);   // the W_q rows are spent by now
  uint64_t* pairs = reinterpret_cast<uint64_t*>(keys + ((p.s.NB + 1) & ~1));
  int32_t* out = p.s.idx + (size_t)bh * p.s.cap;
  const bool partial = (L % p.s.BLK) != 0;
  int total;
  if (p.s.mode != 2 && p.s.NB <= 2 * kThreads) {
    total = select_row_regs<kThreads, 2>(row, nfull, partial, p.s.mode, p.s.kblocks, p.s.tau, sr, out, p.s.cap);
  } else if (p.s.mode != 2 && p.s.NB <= 4 * kThreads) {
    total = select_row_regs<kThreads, 4>(row, nfull, partial, p.s.mode, p.s.kblocks, p.s.tau, sr, out, p.s.cap);
  } else if (p.s.mode != 2 && p.s.NB <= 8 * kThreads) {
    total = select_row_regs<kThreads, 8>(row, nfull, partial, p.s.mode, p.s.kblocks, p.s.tau, sr, out, p.s.cap);
  } else {
    total = select_row<kThreads>(row, nfull, partial, p.s.mode, p.s.kblocks, p.s.tau, keys, pairs, sc, out, p.s.cap);
  }
  if (threadIdx.x == 0) {
    p.s.cnt[bh] = total;
    if (p.update_cache) p.k.valid_out[bh] = nfull_k;
  }
}

template <int D, int BLK, int DG>
cudaError_t launch_t(const PlanParams& p, cudaStream_t s) {
  auto kern = plan_kernel<D, BLK, DG>;
  static std::atomic<uint64_t> attr_done{0};
  const size_t row_max = (size_t)((kMaxBlocksRow + 3) & ~3) * 4;
  const size_t region_max = std::max(select_smem_bytes(kMaxBlocksRow, 2), gate_wq_bytes<D, DG, kCL>(kMaxGroup));
  cudaError_t e = ensure_smem_limit(kern, (int)(row_max + region_max), attr_done);
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)((p.s.NB + 3) & ~3) * 4 +
                      std::max(select_smem_bytes(p.s.NB, p.s.mode), gate_wq_bytes<D, DG, kCL>(p.g.g));
  dim3 grid(kCL, p.g.Hkv, p.g.B);
  return launch_pdl(kern, grid, dim3(kThreads), smem, s, p);
}

}  // namespace

cudaError_t launch_plan(const PlanParams& p, int D, int BLK, int DG, cudaStream_t s) {
#define SEER_P(d, blk, dg) \
  if (D == d && BLK == blk && DG == dg) return launch_t<d, blk, dg>(p, s);
  SEER_P(64, 64, 64)
  SEER_P(64, 64, 128)
  SEER_P(64, 128, 64)
  SEER_P(64, 128, 128)
  SEER_P(128, 64, 64)
  SEER_P(128, 64, 128)
  SEER_P(128, 128, 64)
  SEER_P(128, 128, 128)
#undef SEER_P
  return cudaErrorInvalidValue;
}

}  // namespace seer
