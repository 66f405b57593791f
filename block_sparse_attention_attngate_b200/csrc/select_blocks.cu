// Standalone block selection: one CTA per (b, h) selects from its row of gate
// logits (select_device.cuh): select_row_regs for top-k and threshold rows of up
// to 2048 blocks, select_row otherwise.
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

// top-k and threshold rows of up to 8 * kRegsThreads blocks: keys in registers
constexpr int kRegsThreads = 256;
template <int E>
__global__ void __launch_bounds__(kRegsThreads) select_regs_kernel(const SelectParams p) {
  __shared__ SelectRegsScratch sr;
  const int h = blockIdx.x, b = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  const int L = max(p.seqlens[b], 0);
  const int nfull = min(L / p.BLK, p.NB);
  const float* row = p.logits + ((size_t)b * p.Hkv + h) * p.NB;
  int32_t* out = p.idx + ((size_t)b * p.Hkv + h) * p.cap;
  const int total = select_row_regs<kRegsThreads, E>(row, nfull, (L % p.BLK) != 0, p.mode, p.kblocks, p.tau, sr,
                                                     out, p.cap);
  if (threadIdx.x == 0) p.cnt[b * p.Hkv + h] = total;
}

}  // namespace

cudaError_t launch_select(const SelectParams& p, cudaStream_t s) {
  const dim3 grid(p.Hkv, p.B);
  if (p.mode != 2) {
    if (p.NB <= 2 * kRegsThreads) return launch_pdl(select_regs_kernel<2>, grid, dim3(kRegsThreads), 0, s, p);
    if (p.NB <= 4 * kRegsThreads) return launch_pdl(select_regs_kernel<4>, grid, dim3(kRegsThreads), 0, s, p);
    if (p.NB <= 8 * kRegsThreads) return launch_pdl(select_regs_kernel<8>, grid, dim3(kRegsThreads), 0, s, p);
  }
  const size_t smem = select_smem_bytes(p.NB, p.mode);
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = ensure_smem_limit(select_kernel, (int)select_smem_bytes(kMaxBlocksRow, 2), attr_done);
  if (e != cudaSuccess) return e;
  return launch_pdl(select_kernel, grid, dim3(kThreads), smem, s, p);
}

}  // namespace seer
