// Internal launch interface between the C ABI layer (seer_api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "seer.h"

namespace seer {

// Launch `kern` on `s` with programmatic stream serialization (see pdl_wait /
// pdl_trigger in seer_device.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// Raise a kernel's dynamic shared-memory limit once per device (a host-side
// attribute call, kept out of CUDA-graph capture after the first use).
template <typename Kernel>
cudaError_t ensure_smem_limit(Kernel kern, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}


// ~1 s at 2 GHz: a wait that runs this long means a copy never landed (the default bound).
constexpr long long kWaitLimitCycles = 2000000000LL;
constexpr int kMaxGroup = 8;        // query heads per KV head
constexpr int kMaxBlocksRow = 8192; // max_blocks limit (selection keeps a row in shared memory)
constexpr int kMaxDecodeB = 4096;   // decode keeps the sequence lengths in shared memory
constexpr int kMaxDecodeBH = 4096;  // balanced decode keeps the list-length prefix in shared memory

// Where a K/V tile lives, for kernels that read it with plain loads.
struct KvPlain {
  const uint16_t* data;
  int64_t stride_b, stride_h, stride_t;   // elements
  const int32_t* block_table;             // paged only
  int32_t max_pages;
  int64_t num_pages;
  int64_t num_tokens;                     // contiguous only: token capacity
  int32_t paged;
};

// ---------------------------------------------------------------- kcomp update
constexpr int kMaxHalfGate = 64;    // d_gate / 2 rotation frequencies

struct KcompParams {
  double theta[kMaxHalfGate];   // base^(-2i/d_gate), computed on the host in fp64
  KvPlain k;
  const int32_t* seqlens;
  const int32_t* valid;
  int32_t* valid_out;
  const uint16_t* w_k;     // [Hkv, DG, 3D]
  uint16_t* kcomp;         // [B, Hkv, NB, DG]
  int32_t B, Hkv, NB;
  float rope_base;
  int32_t* err;
};
cudaError_t launch_kcomp_update(const KcompParams& p, int D, int BLK, int DG, int grid_x,
                                cudaStream_t s);

// ---------------------------------------------------------------- cache from running block statistics
struct AppendParams {
  double theta[kMaxHalfGate];   // base^(-2i/d_gate), computed on the host in fp64
  const uint16_t* k_new;   // [B, Hkv, D] pre-RoPE key of token seqlens[b]-1 (append)
  KvPlain k;               // pre-RoPE key cache (state init)
  const int32_t* seqlens;
  int32_t* valid;          // [B, Hkv] fill counts, read and advanced
  float* state;            // [B, Hkv, 3, D] running max / min / sum of the current block
  const uint16_t* w_k;     // [Hkv, DG, 3D]
  uint16_t* kcomp;         // [B, Hkv, NB, DG]
  int32_t B, Hkv, NB;
  int32_t* err;
};
cudaError_t launch_kcomp_append(const AppendParams& p, int D, int BLK, int DG, cudaStream_t s);
cudaError_t launch_kcomp_state_init(const AppendParams& p, int D, int BLK, cudaStream_t s);

// ---------------------------------------------------------------- prefill attention + block target
struct PrefillParams {
  const uint16_t* q;       // [B, Hq, T, D]
  uint16_t* o;             // [B, Hq, T, D]
  float* lse;              // [B, Hq, T] or null
  float* gt;               // [B, Hkv, T, NB]
  float* rmax;             // workspace [B, Hq, NB, T]: each row's tile maxima (log2 domain)
  float* rnorm;            // workspace [B, Hq, T]: each row's final m + log2(l) (tcgen05 path)
  const int32_t* seqlens;  // [B]
  int32_t k_perm[3], v_perm[3];
  int32_t B, Hq, Hkv, g, NB, T;
  int32_t kcap;            // tokens the K and V caches hold per sequence
  float scale_log2;
  int32_t* err;
};
cudaError_t launch_prefill_gt(const CUtensorMap& tk, const CUtensorMap& tv, const PrefillParams& p, int D, int BLK,
                              int max_len, cudaStream_t s);
// The same forward on tcgen05 / TMEM (prefill_tc.cu): head_dim 128, groups of 1, 2, 4 or 8.
bool prefill_tc_supported(int D, int BLK, int g);
// One persistent CTA per SM (sms = the device's SM count), items of 128 rows heaviest first.
cudaError_t launch_prefill_tc(const CUtensorMap& tk, const CUtensorMap& tv, const PrefillParams& p, int D, int BLK,
                              int max_len, int sms, cudaStream_t s);

// ---------------------------------------------------------------- gate score
struct GateParams {
  double theta[kMaxHalfGate];   // base^(-2i/d_gate), computed on the host in fp64
  const uint16_t* q;       // [B, Hq, D]
  const uint16_t* w_q;     // [Hkv, DG, g*D]
  const uint16_t* kcomp;   // [B, Hkv, NB, DG]
  const int32_t* seqlens;
  float* logits;           // [B, Hkv, NB]
  float* q_gate;           // [B, Hkv, DG] or null
  int32_t B, Hq, Hkv, g, NB, BLK;
  float rope_base;
};
cudaError_t launch_gate_score(const GateParams& p, int D, int DG, cudaStream_t s);

// ---------------------------------------------------------------- select
struct SelectParams {
  const float* logits;     // [B, Hkv, NB]
  const int32_t* seqlens;
  int32_t* idx;            // [B, Hkv, cap]
  int32_t* cnt;            // [B, Hkv]
  int32_t B, Hkv, NB, BLK, cap;
  int32_t mode;            // 0 top-k, 1 threshold, 2 top-p
  int32_t kblocks;         // top-k
  double tau;              // threshold / top-p mass
};
cudaError_t launch_select(const SelectParams& p, cudaStream_t s);

// ---------------------------------------------------------------- fused plan (cache update + gate + select)
struct PlanParams {
  KcompParams k;
  GateParams g;
  SelectParams s;
  int32_t update_cache;   // run the cache update first
};
cudaError_t launch_plan(const PlanParams& p, int D, int BLK, int DG, cudaStream_t s);

// ---------------------------------------------------------------- sparse decode
struct DecodeParams {
  const uint16_t* q;        // [B, Hq, D]
  const int32_t* idx;       // [B, Hkv, cap]
  const int32_t* cnt;       // [B, Hkv]
  const int32_t* seqlens;   // [B]
  const int32_t* k_table;   // paged block tables (may be equal)
  const int32_t* v_table;
  int32_t k_maxp, v_maxp;
  int64_t k_pages, v_pages;
  int32_t k_paged, v_paged;
  int32_t k_perm[3], v_perm[3];   // TMA dim (1..3) that holds token / head / batch-or-page
  int32_t B, Hq, Hkv, g;
  int32_t flat;             // 0: (split, kv head, batch) grid; one-wave ranges over 1: the concatenated
                            // lists (balanced), 2: every list padded to its capacity (capacity schedule)
  int32_t cap, ns, per_split;
  float scale_log2;         // softmax scale * log2(e)
  float* o_part;            // [B, Hq, ns, D]
  float* lse_part;          // [B, Hq, ns]
  int32_t* counters;        // [B, Hkv] split-arrival counters (zero between calls)
  uint16_t* out;            // [B, Hq, D] bf16
  float* lse_out;           // [B, Hq] or null
  int32_t* err;
  int32_t* ready;           // fused step: [B, Hkv] per-row list-ready flags (zero between calls); else null
  long long wait_limit;     // bound of every copy / hand-off wait, in SM cycles
  int32_t starve;           // debug: the producer issues no copy (every first wait runs out); 0 in use
};
cudaError_t launch_sparse_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                                 int D, int BLK, int grid_flat, cudaStream_t s);
int decode_ctas_per_sm(int D, int BLK);

// ---------------------------------------------------------------- fused decode step (plan + decode)
struct StepParams {
  DecodeParams d;   // capacity schedule (flat == 2), d.ready set
  PlanParams pl;
};
// Grid of the fused step on the current device: 2 x the co-resident clusters of two, at most one
// CTA per SM; 0 when the shape has no fused kernel or its shared memory does not fit.
int step_grid(int D, int BLK, int DG, int g, int NB, int mode, int B, int BH);
cudaError_t launch_decode_step(const CUtensorMap& tk, const CUtensorMap& tv, const StepParams& p, int D, int BLK,
                               int DG, int grid, cudaStream_t s);

// seer_sparse_decode in two stages: every argument check and the launch set-up (tensor maps,
// parameters), which enqueues nothing, then the launch itself.
struct DecodeLaunch {
  CUtensorMap tk, tv;
  DecodeParams p;
  int D, BLK, ctas;
  size_t need;   // workspace bytes the launch uses
};
seer_status prepare_sparse_decode(const seer_dims_t* dims, const void* q, const seer_kv_t* k, const seer_kv_t* v,
                                  const int32_t* block_idx, const int32_t* block_cnt, const int32_t* seqlens,
                                  int32_t capacity, int32_t num_split, void* workspace, size_t workspace_bytes,
                                  void* out, float* lse_out, int32_t* err_word, DecodeLaunch* launch);
seer_status launch_prepared_decode(const DecodeLaunch& launch, cudaStream_t s);

// ---------------------------------------------------------------- decode ground truth
struct TruthParams {
  const uint16_t* q;        // [B, Hq, D]
  const int32_t* seqlens;   // [B]
  const int32_t* k_table;   // paged block table or null
  int32_t k_maxp;
  int64_t k_pages;
  int32_t k_paged;
  int32_t k_perm[3];
  int32_t B, Hq, Hkv, g, NB, nchunk;
  int32_t nitems;           // B * Hkv * nchunk work items
  float scale_log2;         // softmax scale * log2(e)
  float* scores;            // [B, Hkv, NB]
  float* log_scores;        // [B, Hkv, NB] or null
  float* bmax;              // workspace [B*Hkv, NB, 8]: per head, the block's score maximum (log2 domain)
  float* part;              // workspace [B*Hkv, nchunk, 8, 2]: per head, the chunk's (max, sum of exp2)
  int32_t* counters;        // workspace [B*Hkv] (zero between calls)
  int32_t* err;
};
cudaError_t launch_gate_truth(const CUtensorMap& tk, const TruthParams& p, int D, int BLK, int sms, cudaStream_t s);
int truth_chunk_blocks();

// Record `msg` as the text seer_last_error() returns on this thread; returns `status`.
int set_last_error(int status, const char* msg);

}  // namespace seer
