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
  cg::cluster_group cluster = cg::this_cluster();
  pdl_wait();
  pdl_trigger();
  gate_cluster<D, DG, kCL, kThreads>(p, blockIdx.z, blockIdx.y, (int)cluster.block_rank(), cluster, sm, nullptr);
}

template <int D, int DG>
cudaError_t launch_t(const GateParams& p, cudaStream_t s) {
  dim3 grid(kCL, p.Hkv, p.B);
  return launch_pdl(gate_score_kernel<D, DG>, grid, dim3(kThreads), 0, s, p);
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
