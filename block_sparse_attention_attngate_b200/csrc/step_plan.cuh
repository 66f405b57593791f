// The planning phase of the fused decode step (decode_step_kernel): the K
// Compression Cache update, AttnGate logits and block selection of a few
// (b, h) rows, run by a thread-block cluster of two decode CTAs before they
// start streaming, and the per-row ready flags that hand each finished list
// to the CTAs that stream it.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary): Knowl 1-2 (gate), Knowl 5 (cache, top-k /
// threshold, the forced partial block), Knowl 6 (the block-sparse decode that
// consumes the lists).  The arithmetic is that of the standalone kernels
// (kcomp_device.cuh, gate_device.cuh, select_device.cuh), called here with the
// decode CTA's thread count.
//
// Hand-off.  Rank 0 of the planning cluster writes the row's list and count
// with ordinary stores, the CTA meets at a barrier, and one thread publishes
// ready[row] = 1 with a release store at GPU scope.  A streaming CTA's
// producer lane acquires ready[row] (a bounded spin) before it reads the list
// through L2.  The CTAs that stream a row reset its flag once the row is
// finished (the one whole piece, or the last-arriving piece that merges a
// split row), so every completed launch leaves the flags zero.
#pragma once

#include <cooperative_groups.h>

#include "gate_device.cuh"
#include "kcomp_device.cuh"
#include "select_device.cuh"

namespace seer {

constexpr int kStepCluster = 2;   // CTAs per planning cluster

template <int D, int DG, int NT>
struct StepPlanSmem {
  union {
    KcompSmem<D, DG, NT> k;               // cache update (before the gate)
    GateSmem<D, DG, kStepCluster> g;      // gate (after a cluster barrier that ends the update)
  } u;
  union {
    SelectScratch sc;
    SelectRegsScratch sr;
  } s;
  uint64_t wq_bar;
};

// Publish row `flag`'s list: every thread of the CTA wrote its entries before the barrier that
// precedes this call.
__device__ __forceinline__ void publish_ready(int32_t* flag) {
  __threadfence();
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flag), "r"(1) : "memory");
}

// Bounded acquire-wait for a row's list.  Gives up when the bound runs out or the CTA is
// aborting (*abort set); returns whether the list is ready.
__device__ __forceinline__ bool wait_ready(const int32_t* flag, const volatile int* abort) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
  if (v) return true;
  const long long t0 = clock64();
  do {
    if (*abort) return false;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v) return true;
  } while (clock64() - t0 < kWaitLimitCycles);
  return false;
}

// Bring `bytes` (a multiple of 16, 16-byte aligned) into L2.  Safe before the launch wait even
// for data the preceding kernel writes: only L2 is filled, and L2 is where those writes land.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  const char* c = static_cast<const char*>(p);
  for (uint32_t off = 0; off < bytes; off += 32768u) {
    const uint32_t n = bytes - off < 32768u ? bytes - off : 32768u;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(c + off), "r"(n) : "memory");
  }
}

// One thread, before the launch wait: row r's W_q rows for this CTA into wq_s (armed on
// ps.wq_bar), and this CTA's half of the row's cache entries and the group's query into L2.
template <int D, int DG, int NT>
__device__ void step_plan_prefetch(const PlanParams& pp, int r, int rank, uint16_t* wq_s,
                                   StepPlanSmem<D, DG, NT>& ps) {
  const int Hkv = pp.g.Hkv, b = r / Hkv, h = r - b * Hkv;
  gate_prefetch_wq<D, DG, kStepCluster>(pp.g, h, rank, &ps.wq_bar, wq_s);
  const int half = (pp.g.NB + 1) / 2;
  const int n0 = rank * half, n1 = min(pp.g.NB, n0 + half);
  if (n1 > n0)
    prefetch_l2(pp.g.kcomp + ((size_t)r * pp.g.NB + n0) * DG, (uint32_t)((n1 - n0) * DG * 2));
  if (rank == 0) prefetch_l2(pp.g.q + ((size_t)b * pp.g.Hq + (size_t)h * pp.g.g) * D, (uint32_t)(pp.g.g * D * 2));
}

// Plan rows [r_lo, r_hi) (row = b * Hkv + h).  Every NT threads of both CTAs of the cluster call
// this with the same rows, after the launch wait; the first row's W_q rows were requested by
// step_plan_prefetch (and the CTA synchronised since).  wq_s: the W_q rows' shared region;
// row: this CTA's logit row (rank 0's receives the logits); sel: shared scratch for the
// shared-memory selection path (keys / pairs); none of the three is touched by another CTA after
// the row's last cluster barrier.
template <int D, int BLK, int DG, int NT>
__device__ void step_plan_rows(const PlanParams& pp, int32_t* ready, int r_lo, int r_hi, uint16_t* wq_s, float* row,
                               uint8_t* sel, StepPlanSmem<D, DG, NT>& ps, cooperative_groups::cluster_group& cluster) {
  const int rank = (int)cluster.block_rank();
  const int Hkv = pp.g.Hkv;
  for (int r = r_lo; r < r_hi; ++r) {
    const int b = r / Hkv, h = r - b * Hkv;
    if (r > r_lo) {
      cluster.sync();   // both CTAs are done with the previous row's W_q rows, logit row and scratch
      if (threadIdx.x == 0) gate_prefetch_wq<D, DG, kStepCluster>(pp.g, h, rank, &ps.wq_bar, wq_s);
      __syncthreads();
    }
    GateQuery<D, DG, kStepCluster, NT> q;
    q.load(pp.g, b, h);
    const int L = max(pp.g.seqlens[b], 0);
    int nfull_k = 0;
    if (pp.update_cache) {
      nfull_k = kcomp_nfull<BLK>(pp.k, L);
      const int v0 = max(pp.k.valid[r], 0);
      if (nfull_k > v0) {   // the same decision in both CTAs
        kcomp_update_share<D, BLK, DG, NT>(pp.k, b, h, v0, nfull_k, rank, kStepCluster, ps.u.k);
        __threadfence();    // the new entries are read by the other CTA below
        cluster.sync();
      }
    }
    gate_cluster<D, DG, kStepCluster, NT>(pp.g, b, h, rank, L, q, cluster, ps.u.g, &ps.wq_bar, wq_s,
                                          cluster.map_shared_rank(row, 0));
    cluster.sync();   // rank 0's logit row is complete
    if (rank != 0) continue;
    const int nfull = min(L / pp.s.BLK, pp.s.NB);
    if (pp.g.logits) {
      float* lg = pp.g.logits + (size_t)r * pp.s.NB;
      for (int n = threadIdx.x; n < pp.s.NB; n += NT) lg[n] = n < nfull ? row[n] : -INFINITY;
    }
    int32_t* out = pp.s.idx + (size_t)r * pp.s.cap;
    const bool partial = (L % pp.s.BLK) != 0;
    int total;
    if (pp.s.mode != 2 && pp.s.NB <= 2 * NT) {
      total = select_row_regs<NT, 2>(row, nfull, partial, pp.s.mode, pp.s.kblocks, pp.s.tau, ps.s.sr, out, pp.s.cap);
    } else if (pp.s.mode != 2 && pp.s.NB <= 4 * NT) {
      total = select_row_regs<NT, 4>(row, nfull, partial, pp.s.mode, pp.s.kblocks, pp.s.tau, ps.s.sr, out, pp.s.cap);
    } else if (pp.s.mode != 2 && pp.s.NB <= 8 * NT) {
      total = select_row_regs<NT, 8>(row, nfull, partial, pp.s.mode, pp.s.kblocks, pp.s.tau, ps.s.sr, out, pp.s.cap);
    } else {
      uint32_t* keys = reinterpret_cast<uint32_t*>(sel);
      uint64_t* pairs = reinterpret_cast<uint64_t*>(keys + ((pp.s.NB + 1) & ~1));
      total = select_row<NT>(row, nfull, partial, pp.s.mode, pp.s.kblocks, pp.s.tau, keys, pairs, ps.s.sc, out,
                             pp.s.cap);
    }
    __syncthreads();   // every thread's list entries are written (and the scratch is free)
    if (threadIdx.x == 0) {
      pp.s.cnt[r] = total;
      if (pp.update_cache) pp.k.valid_out[r] = nfull_k;
      publish_ready(ready + r);
    }
  }
}

}  // namespace seer
