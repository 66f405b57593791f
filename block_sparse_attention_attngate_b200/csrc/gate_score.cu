// Standalone AttnGate logits: one 4-CTA cluster per (b, h) runs gate_cluster
// (gate_device.cuh, which cites the equations it implements).
#include "gate_device.cuh"

namespace cg = cooperative_groups;

namespace seer {
namespace {

constexpr int kThreads = 256;
#ifndef SEER_GATE_CLUSTER
#define SEER_GATE_CLUSTER 4   // CTAs per (b, h) cluster
#endif
constexpr int kCL = SEER_GATE_CLUSTER;

template <int D, int DG>
__global__ void __cluster_dims__(kCL, 1, 1) __launch_bounds__(kThreads) gate_score_kernel(const GateParams p) {
  __shared__ GateSmem<D, DG, kCL> sm;
  __shared__ uint64_t wq_bar;
  extern __shared__ uint4 wq_raw[];   // this CTA's W_q rows
  uint16_t* wq_s = reinterpret_cast<uint16_t*>(wq_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int b = blockIdx.z, h = blockIdx.y;
  if (threadIdx.x == 0) gate_prefetch_wq<D, DG, kCL>(p, h, rank, &wq_bar, wq_s);   // weights: no wait needed
  pdl_wait();
  pdl_trigger();
  GateQuery<D, DG, kCL, kThreads> q;
  q.load(p, b, h);
  const int L = max(p.seqlens[b], 0);
  gate_cluster<D, DG, kCL, kThreads>(p, b, h, rank, L, q, cluster, sm, &wq_bar, wq_s, nullptr);
}

template <int D, int DG>
cudaError_t launch_t(const GateParams& p, cudaStream_t s) {
  auto kern = gate_score_kernel<D, DG>;
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = ensure_smem_limit(kern, (int)gate_wq_bytes<D, DG, kCL>(kMaxGroup), attr_done);
  if (e != cudaSuccess) return e;
  dim3 grid(kCL, p.Hkv, p.B);
  return launch_pdl(kern, grid, dim3(kThreads), gate_wq_bytes<D, DG, kCL>(p.g), s, p);
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
