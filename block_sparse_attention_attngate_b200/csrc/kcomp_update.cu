// K Compression Cache maintenance in one launch: a cluster of kKcCluster CTAs
// per (b, h) shares the (b, h)'s new blocks; after the cluster barrier (every
// CTA of the cluster has read the fill count) rank 0 advances the fill count.
// See kcomp_device.cuh for the arithmetic and its sources.
#include <cooperative_groups.h>

#include "kcomp_device.cuh"

namespace cg = cooperative_groups;

namespace seer {
namespace {

constexpr int kThreads = 256;
constexpr int kKcCluster = 8;

template <int D, int BLK, int DG>
__global__ void __cluster_dims__(kKcCluster, 1, 1) __launch_bounds__(kThreads)
    kcomp_update_kernel(const KcompParams p) {
  __shared__ KcompSmem<D, DG, kThreads> sm;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int b = blockIdx.z, h = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  const int L = max(p.seqlens[b], 0);
  const int nfull = kcomp_nfull<BLK>(p, L);
  if (nfull < L / BLK && rank == 0 && threadIdx.x == 0) report(p.err, SEER_DEVERR_COUNT);
  const int v0 = max(p.valid[b * p.Hkv + h], 0);
  kcomp_update_share<D, BLK, DG, kThreads>(p, b, h, v0, nfull, rank, kKcCluster, sm);
  cluster.sync();   // every CTA of the (b, h) has read v0
  if (rank == 0 && threadIdx.x == 0) p.valid_out[b * p.Hkv + h] = nfull;
}

template <int D, int BLK, int DG>
cudaError_t launch_t(const KcompParams& p, cudaStream_t s) {
  dim3 grid(kKcCluster, p.Hkv, p.B);
  return launch_pdl(kcomp_update_kernel<D, BLK, DG>, grid, dim3(kThreads), 0, s, p);
}

}  // namespace

cudaError_t launch_kcomp_update(const KcompParams& p, int D, int BLK, int DG, int grid_x, cudaStream_t s) {
  (void)grid_x;
#define SEER_K(d, blk, dg) \
  if (D == d && BLK == blk && DG == dg) return launch_t<d, blk, dg>(p, s);
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

}  // namespace seer
