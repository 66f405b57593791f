// Standalone block selection: one CTA per (b, h) runs select_row (select_device.cuh)
// on its row of gate logits.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 5 (token budget top-k, threshold, forced
// partial block) and Knowl 14 (top-p).
#include "seer_device.cuh"
#include "seer_internal.h"
#include "select_device.cuh"

namespace seer {
namespace {

constexpr int kThreads = 512;

__global__ void __launch_bounds__(kThreads) select_kernel(const SelectParams p) {
  extern __shared__ uint32_t keys[];   // [NB] keys (even count), then top-p pairs
  __shared__ SelectScratch sc;
  const int h = blockIdx.x, b = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  const int L = max(p.seqlens[b], 0);
  const int nfull = min(L / p.BLK, p.NB);
  const bool partial = (L % p.BLK) != 0;
  const float* row = p.logits + ((size_t)b * p.Hkv + h) * p.NB;
  int32_t* out = p.idx + ((size_t)b * p.Hkv + h) * p.cap;
  uint64_t* pairs = reinterpret_cast<uint64_t*>(keys + ((p.NB + 1) & ~1));
  const int total = select_row<kThreads>(row, nfull, partial, p.mode, p.kblocks, p.tau, keys, pairs, sc, out, p.cap);
  if (threadIdx.x == 0) p.cnt[b * p.Hkv + h] = total;
}

// rows of at most kWarpSelectMax blocks (top-k, threshold): one warp per (b, h)
constexpr int kRowsPerCta = 4;
__global__ void __launch_bounds__(32 * kRowsPerCta) select_warp_kernel(const SelectParams p) {
  const int row_id = blockIdx.x * kRowsPerCta + (threadIdx.x >> 5);
  pdl_wait();
  pdl_trigger();
  if (row_id >= p.B * p.Hkv) return;
  const int b = row_id / p.Hkv;
  const int L = max(p.seqlens[b], 0);
  const int nfull = min(L / p.BLK, p.NB);
  const float* row = p.logits + (size_t)row_id * p.NB;
  int32_t* out = p.idx + (size_t)row_id * p.cap;
  const int total = select_row_warp<kWarpSelectMax / 32>(row, nfull, (L % p.BLK) != 0, p.mode, p.kblocks, p.tau, out,
                                                         p.cap);
  if ((threadIdx.x & 31) == 0) p.cnt[row_id] = total;
}

}  // namespace

cudaError_t launch_select(const SelectParams& p, cudaStream_t s) {
  if (p.NB <= kWarpSelectMax && p.mode != 2) {
    const int rows = p.B * p.Hkv;
    return launch_pdl(select_warp_kernel, dim3((rows + kRowsPerCta - 1) / kRowsPerCta), dim3(32 * kRowsPerCta), 0, s,
                      p);
  }
  const size_t smem = select_smem_bytes(p.NB, p.mode);
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = ensure_smem_limit(select_kernel, (int)select_smem_bytes(kMaxBlocksRow, 2), attr_done);
  if (e != cudaSuccess) return e;
  dim3 grid(p.Hkv, p.B);
  return launch_pdl(select_kernel, grid, dim3(kThreads), smem, s, p);
}

}  // namespace seer
