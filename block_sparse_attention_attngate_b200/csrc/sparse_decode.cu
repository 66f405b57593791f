// Block-sparse flash decoding over the selected KV blocks, and the split
// log-sum-exp combine.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 6: grid (batch, heads_kv, num_split); the
// selected list [batch, heads_kv, max_selected_blocks] is split by its width,
// and the kernel visits only the active block indices.  That grid is kept
// (num_split >= 1).  The one-wave schedules balance instead: the concatenation
// of every (b, h)'s selected list is cut into equal contiguous ranges, one per
// CTA of a grid with one CTA per SM, so ragged counts and small batches still
// keep every SM streaming -- by the lists' counts (num_split == 0, a scan of
// the counts first) or by their capacity (num_split == -1, no scan: positions
// past a count are skipped; its producer makes a dry pass over its issue loop
// before the launch dependency wait).
//
// The page's H100 kernel pads the query group to 64 rows for wgmma; here the
// group (g <= 8 query heads) stays a 16-row mma.sync fragment: the work per KV
// byte is ~g multiply-adds and the bound is HBM, not the tensor pipe.
//
// CTA structure.  Warp CW is the producer.  It resolves list positions 32 at a
// time (one lane each: binary search in the shared-memory prefix of the list
// lengths, one batched load of the block indices, fetched a chunk ahead), and
// its lane 0 issues 128B-swizzled TMA tile loads of each block's K and V into
// a STAGES-deep shared-memory ring (L2 evict-first: every tile is read once),
// plus a bulk copy of the group's q rows into one of two segment buffers when
// a segment starts; completion is counted on mbarriers.
//
// Warps 0..CW-1 are consumers, in NG groups of NWG warps.  Group k takes the
// ring iterations it == k (mod NG), so NG blocks are in compute at once and
// the per-block latency chain (ldmatrix -> mma -> softmax -> mma) is hidden;
// within a group each warp owns BLK/NWG tokens of the block:
//   S   = Q K^T        (A = Q from registers, B = K via ldmatrix)
//   P   = exp2(S*scale*log2e - m)   (fp32 online softmax per query head)
//   O^T += V^T P^T     (A = V via ldmatrix.trans, B = P from S's accumulator)
// A segment is a run of consecutive positions of one (b, h) inside one CTA;
// the consumers derive the segments from the same prefix the producer uses.
// At a segment's end all CW consumer warps meet once: each writes its state to
// shared memory, per-head merge weights are formed by CW*g threads, and every
// thread combines its outputs with CW independent multiply-adds.  A segment
// that is a whole (b, h) writes bf16 out directly; any other writes an fp32
// partial.  The CTA's first segment, if split, is handed to warp CW+1 (the
// epilogue warp), which publishes it (fence, arrival counter) and, if it was
// the (b, h)'s last piece to arrive, merges all of its partials, off the
// consumers' path; the CTA's last segment is published and, if last to
// arrive, merged by the consumers themselves.  All waits are bounded.
#include "seer_device.cuh"
#include "seer_internal.h"
#include "step_plan.cuh"

#include <algorithm>

namespace seer {
namespace {

constexpr float kLn2 = 0.6931471805599453f;

constexpr int kSegFirst = 1;  // first block of a segment (a q copy precedes it)

struct StageInfo {
  int n;       // block index, -1 = skip
  int pad[3];
};

template <int D, int BLK, int NWG, int NG, int STAGES>
struct DecodeShape {
  static constexpr int kTile = BLK * D * 2;   // bytes of one K (or V) tile
  static constexpr int kBox = BLK * 128;      // bytes of one 64-channel box
  static constexpr int kNBox = D / 64;
  static constexpr int kTPW = BLK / NWG;      // tokens per consumer warp per block
  static constexpr int kNT = kTPW / 8;        // 8-token S tiles per warp
  static constexpr int kKS = kTPW / 16;       // 16-token PV k-steps per warp
  static constexpr int kDK = D / 16;          // QK^T k-steps == PV m-tiles
  static constexpr int kCW = NWG * NG;        // consumer warps
  static constexpr int kThreads = (kCW + 2) * 32;   // consumers, producer, epilogue
  static constexpr int kRing = STAGES * 2 * kTile;
  static constexpr int kQBytes = kMaxGroup * D * 2;
  // merge area: Ow[CW][8][D], Mw[CW][8], Lw[CW][8], Wt[CW][8], Hs[8]
  static constexpr int kMergeFloats = kCW * kMaxGroup * D + 3 * kCW * kMaxGroup + kMaxGroup;
  static constexpr int kBars = (2 * STAGES + 7) * 8;   // full, empty, qfull[2], qempty[2], cbar, jbar[2]
  static constexpr int kEpi = 256;   // partial LSEs (segment-major) / merge weights, + per-head M, sum
  static constexpr int kSh = 32;     // shared scalars
  // fixed part; the list prefix and the sequence lengths follow (sized per launch)
  static constexpr size_t kSmemFixed = 1024 + kRing + 2 * kQBytes + (size_t)kMergeFloats * 4 + kBars +
                                       STAGES * sizeof(StageInfo) + 16 + (kEpi + 2 * kMaxGroup) * 4 +
                                       kSh * 4 + 2 * STAGES * 4;
  static_assert(kTPW % 16 == 0, "each consumer warp needs whole 16-token steps");
  static_assert(D % 64 == 0, "head_dim must be a multiple of 64");
  static_assert(STAGES % NG == 0, "each ring stage belongs to one consumer group");
  static_assert(kMergeFloats >= kEpi + 2 * kMaxGroup, "the merge area doubles as the final merge's scratch");
};

__device__ __forceinline__ void tile_coords(const int32_t perm[3], int t, int h, int bp, int& c1, int& c2,
                                            int& c3) {
  int c[3];
  c[perm[0]] = t;
  c[perm[1]] = h;
  c[perm[2]] = bp;
  c1 = c[0];
  c2 = c[1];
  c3 = c[2];
}

__device__ __forceinline__ int clamp_cnt(const DecodeParams& p, int i) {
  const int c = p.cnt[i];
  return c < 0 ? 0 : (c > p.cap ? p.cap : c);
}

// Balanced schedule: CTA c of G owns flattened positions [lo(c), lo(c+1)), lo(c) = floor(c*W/G).
// W < 2^30 and G <= 2^15 (host-checked): with W = qG + r, c*W/G = c*q + c*r/G and c*r < 2^30,
// so 32-bit integer arithmetic is exact (a 64-bit division is a long software sequence).
__device__ __forceinline__ int range_lo(int c, int W, int G) {
  const int q = W / G, r = W - (W / G) * G;
  return c * q + (c * r) / G;
}
// The CTA whose range holds position `pos` (0 <= pos < W): a float estimate of pos*G/W, then
// exact corrections against range_lo.
__device__ __forceinline__ int cta_of(int pos, int W, int G) {
  int c = min(G - 1, max(0, (int)((float)pos * (float)G / (float)W)));
  while (c + 1 < G && range_lo(c + 1, W, G) <= pos) ++c;
  while (c > 0 && range_lo(c, W, G) > pos) --c;
  return c;
}
// Last index i in [0, n) with pre[i] <= x (pre non-decreasing, pre[0] = 0 <= x).
__device__ __forceinline__ int bh_of(const int* pre, int n, int x) {
  int lo = 0, hi = n;   // invariant: pre[lo] <= x, answer in [lo, hi)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (pre[mid] <= x) lo = mid;
    else hi = mid;
  }
  return lo;
}

// A split segment handed to the epilogue warp.
struct Job {
  int bh, nseg, slot_first, cf;
};

// Partial slots: balanced schedule -- a CTA's first segment writes slot 2c, its last slot 2c+1
// (only those two can belong to a (b, h) that spans CTAs); grid schedule -- slot bh*ns + split.
__device__ __forceinline__ int split_slot(const DecodeParams& p, int bh, int k, int slot_first, int cf) {
  return k == 0 ? slot_first : (p.flat ? 2 * (cf + k) : bh * p.ns + k);
}

// Merge the nseg partials (o, lse) of one (b, h) into bf16 out (and lse_out), by the NT threads
// whose index is `t` (0 <= t < NT).  `wsc` is shared scratch of >= kEpi + 2*kMaxGroup floats;
// `sync()` is a barrier among those NT threads.  Partials are read with L2-coherent loads, four
// channels at a time; the outputs of the first MAXS pieces are requested together with every
// piece's LSE (one round trip up to MAXS pieces), and each piece's weight is formed once per head.
template <int D, int NT, int kEpi, typename Sync>
__device__ void merge_partials(const DecodeParams& p, int bh, int nseg, int slot_first, int cf, int t, float* wsc,
                               Sync sync) {
  const int g = p.g;
  const int b = bh / p.Hkv, h = bh - b * p.Hkv;
  const size_t qh0 = (size_t)b * p.Hq + (size_t)h * g;
  const int ng = nseg * g;
  constexpr int G4 = kMaxGroup * D / 4;              // float4 groups of the largest query group
  constexpr int EPT4 = (G4 + NT - 1) / NT;           // per thread
  constexpr int MAXS = EPT4 <= 2 ? 4 : 2;            // pieces whose outputs are requested together
  const int n4 = g * D / 4;
  if (ng <= kEpi) {
    auto load = [&](int k, int u) {
      const int q4 = u * NT + t;
      if (k >= nseg || q4 >= n4) return make_float4(0.f, 0.f, 0.f, 0.f);
      const int j = (4 * q4) / D, cc = 4 * q4 - j * D;
      const size_t sl = (size_t)split_slot(p, bh, k, slot_first, cf);
      return __ldcg(reinterpret_cast<const float4*>(p.o_part + (sl * g + j) * D + cc));
    };
    float4 ov[MAXS][EPT4];
#pragma unroll
    for (int k = 0; k < MAXS; ++k)
#pragma unroll
      for (int u = 0; u < EPT4; ++u) ov[k][u] = load(k, u);
    float* Mh = wsc + kEpi;
    float* Zh = Mh + kMaxGroup;
    for (int i = t; i < ng; i += NT)
      wsc[i] = __ldcg(p.lse_part + (size_t)split_slot(p, bh, i / g, slot_first, cf) * g + (i % g));
    sync();
    // per head: the largest LSE, the weight sum and, in place, each piece's weight
    if (t < g) {
      float M = -INFINITY;
      for (int k = 0; k < nseg; ++k) M = fmaxf(M, wsc[k * g + t]);
      float Z = 0.f;
      if (M != -INFINITY)
        for (int k = 0; k < nseg; ++k) Z += expf(wsc[k * g + t] - M);
      const float inv = Z > 0.f ? 1.f / Z : 0.f;
      for (int k = 0; k < nseg; ++k) wsc[k * g + t] = Z > 0.f ? expf(wsc[k * g + t] - M) * inv : 0.f;
      Mh[t] = M;
      Zh[t] = Z;
    }
    sync();
    float4 acc[EPT4];
#pragma unroll
    for (int u = 0; u < EPT4; ++u) {
      acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      const int q4 = u * NT + t;
      const int j = q4 < n4 ? (4 * q4) / D : 0;
#pragma unroll
      for (int k = 0; k < MAXS; ++k) {
        const float w = k < nseg ? wsc[k * g + j] : 0.f;
        acc[u].x += w * ov[k][u].x;
        acc[u].y += w * ov[k][u].y;
        acc[u].z += w * ov[k][u].z;
        acc[u].w += w * ov[k][u].w;
      }
    }
    // pieces past the first MAXS (another round trip per MAXS of them)
    for (int k0 = MAXS; k0 < nseg; k0 += MAXS) {
#pragma unroll
      for (int k = 0; k < MAXS; ++k)
#pragma unroll
        for (int u = 0; u < EPT4; ++u) ov[k][u] = load(k0 + k, u);
#pragma unroll
      for (int u = 0; u < EPT4; ++u) {
        const int q4 = u * NT + t;
        const int j = q4 < n4 ? (4 * q4) / D : 0;
#pragma unroll
        for (int k = 0; k < MAXS; ++k) {
          const float w = k0 + k < nseg ? wsc[(k0 + k) * g + j] : 0.f;
          acc[u].x += w * ov[k][u].x;
          acc[u].y += w * ov[k][u].y;
          acc[u].z += w * ov[k][u].z;
          acc[u].w += w * ov[k][u].w;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < EPT4; ++u) {
      const int q4 = u * NT + t;
      if (q4 < n4) {
        const int j = (4 * q4) / D, cc = 4 * q4 - j * D;
        uint2 pk;
        pk.x = pack_bf16(acc[u].x, acc[u].y);
        pk.y = pack_bf16(acc[u].z, acc[u].w);
        *reinterpret_cast<uint2*>(p.out + (qh0 + j) * D + cc) = pk;
        if (cc == 0 && p.lse_out) p.lse_out[qh0 + j] = Zh[j] > 0.f ? Mh[j] + logf(Zh[j]) : -INFINITY;
      }
    }
  } else {
    for (int e = t; e < g * D; e += NT) {
      const int j = e / D, cc = e % D;
      float M = -INFINITY;
      for (int k = 0; k < nseg; ++k)
        M = fmaxf(M, __ldcg(p.lse_part + (size_t)split_slot(p, bh, k, slot_first, cf) * g + j));
      float num = 0.f, den = 0.f;
      if (M != -INFINITY) {
        for (int k = 0; k < nseg; ++k) {
          const size_t sl = (size_t)split_slot(p, bh, k, slot_first, cf);
          const float w = expf(__ldcg(p.lse_part + sl * g + j) - M);
          num += w * __ldcg(p.o_part + (sl * g + j) * D + cc);
          den += w;
        }
      }
      const bool any = den > 0.f;
      __nv_bfloat16 ob = __float2bfloat16_rn(any ? num / den : 0.f);
      p.out[(qh0 + j) * D + cc] = *reinterpret_cast<uint16_t*>(&ob);
      if (cc == 0 && p.lse_out) p.lse_out[qh0 + j] = any ? M + logf(den) : -INFINITY;
    }
  }
}

// The decode, run by every thread of a CTA.  DG > 0 is the fused step (decode_step_kernel): the
// CTA's cluster first plans its rows (step_plan.cuh) and each list position waits for its row's
// ready flag; DG == 0 is the standalone decode over lists already in memory.
template <int D, int BLK, int NWG, int NG, int STAGES, int DG>
__device__ __forceinline__ void decode_body(const CUtensorMap* tmK, const CUtensorMap* tmV, const DecodeParams& p,
                                            const PlanParams* plan) {
  using S = DecodeShape<D, BLK, NWG, NG, STAGES>;
  constexpr int CW = S::kCW;
  constexpr bool FUSED = DG > 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* qseg = ring + S::kRing;                                   // [2] segment q rows
  float* Ow = reinterpret_cast<float*>(qseg + 2 * S::kQBytes);       // [CW][8][D]
  float* Mw = Ow + CW * kMaxGroup * D;                               // [CW][8]
  float* Lw = Mw + CW * kMaxGroup;                                   // [CW][8]
  float* Wt = Lw + CW * kMaxGroup;                                   // [CW][8] merge weights
  float* Hs = Wt + CW * kMaxGroup;                                   // [8] segment LSE
  uint64_t* full = reinterpret_cast<uint64_t*>(Ow + S::kMergeFloats);
  uint64_t* empty = full + STAGES;
  uint64_t* qfull = empty + STAGES;   // [2]
  uint64_t* qempty = qfull + 2;       // [2]
  uint64_t* cbar = qempty + 2;        // consumer-warp barrier
  uint64_t* jbar = cbar + 1;          // split first segment handed to the epilogue warp
  StageInfo* info = reinterpret_cast<StageInfo*>(jbar + 2);
  Job* job = reinterpret_cast<Job*>(info + STAGES);
  float* epi = reinterpret_cast<float*>(job + 1);   // [kEpi] + [2 * kMaxGroup]
  // sh[0] abort, sh[1] merge flag, sh[2] W, sh[3] G_eff, sh[4] p0, sh[5] p1, sh[6] first bh,
  // sh[7] its pre, sh[9] producer done, sh[10..12] first segment {cf, nseg, slot_first},
  // sh[13..15] last segment {cf, nseg, slot_first}, sh[16] last bh, sh[17] sh[10..15] ready
  volatile int* sh = reinterpret_cast<volatile int*>(epi + S::kEpi + 2 * kMaxGroup);
  volatile int* issued = sh + S::kSh;         // [STAGES] tiles issued per stage
  volatile int* observed = issued + STAGES;   // [STAGES] full phases observed per stage
  int* slen = const_cast<int*>(observed + STAGES);   // [B] sequence lengths
  int* pre = slen + p.B;                              // [BH + 1] list prefix (+ 16 ints of scan scratch)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tid = threadIdx.x;
  const int BH = p.B * p.Hkv;
  const int g = p.g;
  auto seq_len = [&](int b) { return p.flat == 2 ? max(__ldg(p.seqlens + b), 0) : slen[b]; };
  // fused step: the planning cluster's rows are those whose first list position falls in the
  // cluster's two ranges (capacity schedule: row r starts at position r * capacity)
  int r_lo = 0, r_hi = 0;
  uint8_t* plan_raw = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(pre + BH + 1 + 16) + 15) & ~uintptr_t(15));
  using PS = StepPlanSmem<D, (FUSED ? DG : 64), S::kThreads>;
  PS& ps = *reinterpret_cast<PS*>(plan_raw);
  if constexpr (FUSED) {
    const int W = BH * p.cap, Gd = min((int)gridDim.x, max(W, 1));
    const int c0 = (int)blockIdx.x & ~1;
    auto lo = [&](int c) { return c >= Gd ? W : range_lo(c, W, Gd); };
    r_lo = (lo(c0) + p.cap - 1) / p.cap;
    r_hi = min(BH, (lo(c0 + 2) + p.cap - 1) / p.cap);
  }
  if (tid == 0) {
    tma_prefetch_desc(tmK);
    tma_prefetch_desc(tmV);
    if constexpr (FUSED) {
      // the first row's W_q rows (weights: no wait needed) land while the previous kernel runs
      if (r_lo < r_hi)
        step_plan_prefetch<D, DG, S::kThreads>(*plan, r_lo, (int)blockIdx.x & 1, reinterpret_cast<uint16_t*>(ring),
                                               ps);
    }
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NWG);
      issued[s] = 0;
      observed[s] = 0;
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&qfull[k], 1);
      mbar_init(&qempty[k], CW);
    }
    mbar_init(cbar, CW);
    mbar_init(jbar, CW);
    sh[0] = 0;
    sh[9] = 0;
    fence_barrier_init();
  }
  __syncthreads();   // barrier inits visible to every warp (before the wait: off the critical path)
  // The parameters are fixed for the launch: bring the ones the first loads depend on into the
  // constant cache now, so their first use after the wait does not cost a memory round trip.
  asm volatile("" ::"l"(p.q), "l"(p.idx), "l"(p.cnt), "l"(p.seqlens), "l"(p.k_table), "l"(p.counters),
               "l"(p.err), "l"(p.out), "r"(p.cap), "r"(p.flat), "r"(p.B), "r"(p.Hkv), "r"(p.k_perm[0]),
               "r"(p.v_perm[2]), "r"(p.per_split), "f"(p.scale_log2));
  const bool fast = p.flat == 2;
  if constexpr (FUSED) {
    // every thread of the cluster plans its rows, then the CTA decodes; lists of rows planned
    // elsewhere are waited for per row (wait_ready), not per launch.  Both CTAs of the cluster
    // have started before either writes into the other's shared memory (arrive now, wait after
    // the launch dependency, so the barrier costs nothing on the critical path).
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    pdl_wait();
    pdl_trigger();
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    cooperative_groups::cluster_group cluster = cooperative_groups::this_cluster();
    step_plan_rows<D, BLK, DG, S::kThreads>(*plan, p.ready, r_lo, r_hi, reinterpret_cast<uint16_t*>(ring), Ow, ring,
                                             ps, cluster);
  } else if (!(fast && warp == CW)) {
    // (the capacity schedule's producer warp waits for the launch's inputs further down, after a
    // dry pass over its issue code)
    pdl_wait();
    pdl_trigger();
  }

  // ---------------------------------------------------------------- lengths, list prefix, this CTA's range
  // (the capacity schedule reads nothing here: its prefix is bh * capacity, the lengths are read
  // where they are used, and its producer warp computes its own range and starts at once -- the
  // other warps run this prologue behind a named barrier that leaves the producer out)
  int pp0 = 0, pnit = 0, pbh = 0;   // the producer's range start, length and (grid schedule) (b, h)
  auto cta_sync = [&]() {
    if (fast) asm volatile("bar.sync 1, %0;" ::"r"((CW + 1) * 32) : "memory");
    else __syncthreads();
  };
  if (fast && warp == CW) {
    const int W = BH * p.cap, G = min((int)gridDim.x, max(W, 1)), c = blockIdx.x;
    if (c < G && W > 0) {
      pp0 = range_lo(c, W, G);
      pnit = range_lo(c + 1, W, G) - pp0;
    }
  } else {
  if (p.flat != 2)
    for (int i = tid; i < p.B; i += S::kThreads) slen[i] = max(p.seqlens[i], 0);
  if (p.flat == 2) {
    const int t2 = warp < CW ? tid : tid - 32;   // the (CW+1)*32 threads other than the producer
    for (int i = t2; i <= BH; i += (CW + 1) * 32) pre[i] = i * p.cap;
    cta_sync();
  }
  if (p.flat == 1) {
    // each thread sums a contiguous run of counts, then one block-wide exclusive scan
    const int per_t = (BH + S::kThreads - 1) / S::kThreads;
    const int base = tid * per_t;
    int loc = 0;
    bool over = false;
    for (int j = 0; j < per_t; ++j) {
      const int i = base + j;
      if (i < BH) {
        loc += clamp_cnt(p, i);
        over |= p.cnt[i] > p.cap;
      }
    }
    if (over && blockIdx.x == 0) report(p.err, SEER_DEVERR_COUNT);
    int incl = loc;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    int* wsum = pre + BH + 1;   // scratch for the warp totals, just past the prefix
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    int run = before + incl - loc;
    for (int j = 0; j < per_t; ++j) {
      const int i = base + j;
      if (i < BH) {
        pre[i] = run;
        run += clamp_cnt(p, i);
      }
    }
    if (tid == S::kThreads - 1) pre[BH] = before + incl;
    __syncthreads();
  }
  if (p.flat) {
    if (tid == 0) {
      const int W = pre[BH];
      const int G = min((int)gridDim.x, max(W, 1));
      const int c = blockIdx.x;
      int p0 = 0, p1 = 0;
      if (c < G && W > 0) {
        p0 = range_lo(c, W, G);
        p1 = range_lo(c + 1, W, G);
      }
      // (b, h) of the first and last positions: the capacity schedule's prefix is bh * capacity
      const int bf = p1 > p0 ? (p.flat == 2 ? p0 / p.cap : bh_of(pre, BH, p0)) : 0;
      const int bl = p1 > p0 ? (p.flat == 2 ? (p1 - 1) / p.cap : bh_of(pre, BH, p1 - 1)) : 0;
      sh[2] = W;
      sh[3] = G;
      sh[4] = p0;
      sh[5] = p1;
      sh[6] = bf;
      sh[7] = pre[bf];
      sh[16] = bl;
      sh[17] = 0;   // split bookkeeping below is filled in by the epilogue warp, off the critical path
    }
  } else if (tid == 0) {
    const int bh = blockIdx.z * p.Hkv + blockIdx.y;
    const int c = clamp_cnt(p, bh);
    if (p.cnt[bh] > p.cap && blockIdx.x == 0) report(p.err, SEER_DEVERR_COUNT);
    const int a = min((int)blockIdx.x * p.per_split, c), e = min(a + p.per_split, c);
    const int nseg = (c + p.per_split - 1) / p.per_split;
    sh[2] = 0;
    sh[3] = 0;
    sh[4] = a;   // positions are local to the (b, h) in this schedule
    sh[5] = e;
    sh[6] = bh;
    sh[7] = 0;
    sh[16] = bh;
    sh[10] = sh[13] = 0;
    sh[11] = sh[14] = nseg;
    sh[12] = sh[15] = bh * p.ns;
    sh[17] = 1;
    pre[0] = c;  // the grid schedule keeps its one list length here
  }
  cta_sync();
  pp0 = sh[4];
  pnit = sh[5] - sh[4];
  pbh = sh[6];
  }
  const int nit = pnit;

  if (warp == CW + 1) {
    // ------------------------------------------------------------ epilogue warp
    if (p.flat && lane == 0) {
      // split bookkeeping of the CTA's first and last segments (a middle one is a whole (b, h)):
      // the CTA of the first piece, the piece count and the first piece's partial slot
      if (nit > 0) {
        const int W = sh[2], G = sh[3];
        const int bf = sh[6], bl = sh[16];
        const int cf_f = cta_of(pre[bf], W, G), cf_l = cta_of(pre[bl], W, G);
        sh[10] = cf_f;
        sh[11] = cta_of(pre[bf + 1] - 1, W, G) - cf_f + 1;
        sh[12] = 2 * cf_f + (range_lo(cf_f, W, G) != pre[bf] ? 1 : 0);
        sh[13] = cf_l;
        sh[14] = cta_of(pre[bl + 1] - 1, W, G) - cf_l + 1;
        sh[15] = 2 * cf_l + (range_lo(cf_l, W, G) != pre[bl] ? 1 : 0);
      }
      __threadfence_block();
      sh[17] = 1;
    }
    __syncwarp();
    // The CTA's first segment, when it is split across CTAs and is not also its last segment,
    // is published (and merged, if it arrives last) here.
    const bool expect = nit > 0 && p.flat && sh[16] != sh[6] && sh[11] > 1;
    if (expect) {
      if (!__all_sync(0xffffffffu, mbar_wait(jbar, 0, p.wait_limit))) {
        if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
        return;
      }
      const Job jb = job[0];
      int last = 0;
      // publish the consumers' partial (ordered before the hand-off) and learn whether this
      // segment is the (b, h)'s last to arrive; acquire the others' partials if so
      if (lane == 0) last = atomic_add_acq_rel_gpu(&p.counters[jb.bh], 1) == jb.nseg - 1;
      if (__shfl_sync(0xffffffffu, last, 0)) {
        merge_partials<D, 32, S::kEpi>(p, jb.bh, jb.nseg, jb.slot_first, jb.cf, lane, epi,
                                       [] { __syncwarp(); });
        __syncwarp();
        if (lane == 0) {
          p.counters[jb.bh] = 0;
          if constexpr (FUSED) p.ready[jb.bh] = 0;   // every piece of the row is done with its list
        }
      }
    }
    return;
  }

  if (warp == CW) {
    // ------------------------------------------------------------ producer warp
    const int p0 = pp0;
    const int fixed_bh = pbh;
    // resolve list position `it` of this CTA (one lane per position)
    bool dry = false;
    int ready_bh = -1;      // fused step: the row whose ready flag this lane last acquired
    bool ready_ok = false;
    auto resolve = [&](int it, int& n, int& bh, int& first, int& kb, int& kt, int& vb, int& vt) {
      n = -1;
      bh = fixed_bh;
      first = 0;
      kb = vb = kt = vt = 0;
      if (it >= nit) return;
      int pos;
      if (fast) {
        const int x = p0 + it;
        bh = x / p.cap;
        pos = x - bh * p.cap;
      } else if (p.flat) {
        const int x = p0 + it;
        bh = bh_of(pre, BH, x);
        pos = x - pre[bh];
      } else {
        pos = p0 + it;
      }
      first = (it == 0 || pos == 0) ? kSegFirst : 0;
      const int b = bh / p.Hkv;
      if constexpr (FUSED) {
        // the row's list is written in this launch: acquire its flag, then read through L2
        if (bh != ready_bh) {
          ready_ok = wait_ready(p.ready + bh, sh);
          if (!ready_ok) report(p.err, SEER_DEVERR_TIMEOUT);
          ready_bh = bh;
        }
        if (!ready_ok) return;
      }
      // the count (capacity schedule), the length and the block index, requested together
      const int c = p.flat == 2 ? (FUSED ? __ldcg(p.cnt + bh) : p.cnt[bh]) : p.cap;
      const int Lb = seq_len(b);
      const int blk = FUSED ? __ldcg(p.idx + (size_t)bh * p.cap + pos) : p.idx[(size_t)bh * p.cap + pos];
      if (p.flat == 2) {   // list positions past the count are padding
        if (pos == 0 && c > p.cap && !dry) report(p.err, SEER_DEVERR_COUNT);
        if (pos >= c) return;
      }
      const int nblk = (Lb + BLK - 1) / BLK;
      bool ok = blk >= 0 && blk < nblk;
      if (!ok && !dry) report(p.err, SEER_DEVERR_BLOCK_INDEX);
      kb = vb = b;
      kt = vt = blk * BLK;
      if (ok && p.k_paged) {
        const int pg = blk < p.k_maxp ? p.k_table[(size_t)b * p.k_maxp + blk] : -1;
        if (pg < 0 || pg >= p.k_pages) {
          if (!dry) report(p.err, SEER_DEVERR_PAGE_INDEX);
          ok = false;
        }
        kb = pg;
        kt = 0;
      }
      if (ok && p.v_paged) {
        const int pg = blk < p.v_maxp ? p.v_table[(size_t)b * p.v_maxp + blk] : -1;
        if (pg < 0 || pg >= p.v_pages) {
          if (!dry) report(p.err, SEER_DEVERR_PAGE_INDEX);
          ok = false;
        }
        vb = pg;
        vt = 0;
      }
      n = ok ? blk : -1;
    };
    const uint64_t stream_pol = l2_evict_first_policy();   // each K/V tile is read once
    const uint32_t qbytes = (uint32_t)(g * D * 2);
    // The capacity schedule's range needs none of the launch's inputs, so its producer makes a dry
    // pass over the resolve / issue loop before it waits for them (two positions; the lists are
    // read but the values are dropped, and no copy, barrier arrival or report is made).  Run for the
    // first time after the wait, this code delayed the first tile request by ~0.7 us more.
#pragma unroll 1
    for (int pass = (fast && !FUSED) ? 0 : 1; pass < 2; ++pass) {
      dry = pass == 0;
      if (fast && !dry && !FUSED) {
        pdl_wait();
        pdl_trigger();
      }
      int nq = 0;   // segments whose q copy was issued
      int cn_, cb_, cf_, ckb, ckt, cvb, cvt;   // current chunk (this lane's position)
      resolve(lane, cn_, cb_, cf_, ckb, ckt, cvb, cvt);
      bool abort = false;
      for (int chunk = 0; chunk * 32 < nit && !abort; ++chunk) {
        int nn, nb, nf, nkb, nkt, nvb, nvt;   // next chunk, fetched while this one issues
        resolve((chunk + 1) * 32 + lane, nn, nb, nf, nkb, nkt, nvb, nvt);
        const int count = min(dry ? 2 : 32, nit - chunk * 32);
        for (int j = 0; j < count; ++j) {
          const int it = chunk * 32 + j;
          const int n = __shfl_sync(0xffffffffu, cn_, j);
          const int bh = __shfl_sync(0xffffffffu, cb_, j);
          const int first = __shfl_sync(0xffffffffu, cf_, j);
          const int kb = __shfl_sync(0xffffffffu, ckb, j), kt = __shfl_sync(0xffffffffu, ckt, j);
          const int vb = __shfl_sync(0xffffffffu, cvb, j), vt = __shfl_sync(0xffffffffu, cvt, j);
          if (lane == 0 && !dry) {
            if (first) {
              // the segment's q rows -> segment buffer nq & 1, once the segment two back has read it
              const int k = nq & 1, u = nq >> 1;
              if (u >= 1 && !mbar_wait(&qempty[k], (u - 1) & 1, p.wait_limit)) {
                report(p.err, SEER_DEVERR_TIMEOUT);
                sh[0] = 1;
              }
              if (!sh[0] && !p.starve) {
                const int b = bh / p.Hkv, h = bh - b * p.Hkv;
                mbar_arrive_expect_tx(&qfull[k], qbytes);
                bulk_load(qseg + k * S::kQBytes, p.q + ((size_t)b * p.Hq + (size_t)h * g) * D, qbytes, &qfull[k]);
              }
              ++nq;
            }
            const int s = it % STAGES;
            if (!sh[0] && it >= STAGES && !mbar_wait(&empty[s], ((it / STAGES) - 1) & 1, p.wait_limit)) {
              report(p.err, SEER_DEVERR_TIMEOUT);
              sh[0] = 1;
            }
            if (!sh[0] && !p.starve) {
              info[s].n = n;
              if (n >= 0) {
                mbar_arrive_expect_tx(&full[s], 2u * S::kTile);
                const int h = bh % p.Hkv;
                uint8_t* kdst = ring + s * 2 * S::kTile;
                uint8_t* vdst = kdst + S::kTile;
                int c1, c2, c3;
                tile_coords(p.k_perm, kt, h, kb, c1, c2, c3);
  #pragma unroll
                for (int bx = 0; bx < S::kNBox; ++bx)
                  tma_load_4d_hint(kdst + bx * S::kBox, tmK, &full[s], bx * 64, c1, c2, c3, stream_pol);
                tile_coords(p.v_perm, vt, h, vb, c1, c2, c3);
  #pragma unroll
                for (int bx = 0; bx < S::kNBox; ++bx)
                  tma_load_4d_hint(vdst + bx * S::kBox, tmV, &full[s], bx * 64, c1, c2, c3, stream_pol);
              } else {
                mbar_arrive(&full[s]);
              }
              issued[s] = issued[s] + 1;
            }
          }
          if (__shfl_sync(0xffffffffu, (int)sh[0], 0)) {
            abort = true;
            break;
          }
        }
        cn_ = nn; cb_ = nb; cf_ = nf; ckb = nkb; ckt = nkt; cvb = nvb; cvt = nvt;
        if (dry) break;
      }
    }
    if (lane == 0) {
      __threadfence_block();
      sh[9] = 1;
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int cg = warp / NWG, wg = warp - cg * NWG;
  const int gq = lane >> 2, tq = lane & 3;
  const float sl2 = p.scale_log2;
  const int tok_base = wg * S::kTPW;
  const int p0 = sh[4], p1 = sh[5];
  uint32_t cphase = 0;
  bool alive = true;
  uint32_t qa[S::kDK][2];
  float o[S::kDK][4];

  int it0 = 0, seg = 0;
  while (it0 < nit) {
    // ---- this segment: [it0, it1) of (b, h) = bh
    int bh, it1;
    if (p.flat) {
      bh = bh_of(pre, BH, p0 + it0);
      it1 = min(p1, pre[bh + 1]) - p0;
    } else {
      bh = sh[6];
      it1 = nit;
    }
    // the group's q rows (rows >= g stay zero), then release the segment buffer
    if (!__all_sync(0xffffffffu, mbar_wait(&qfull[seg & 1], (seg >> 1) & 1, p.wait_limit))) {
      alive = false;
      break;
    }
    {
      const uint8_t* qs = qseg + (seg & 1) * S::kQBytes;
      const bool live = gq < g;
#pragma unroll
      for (int ks = 0; ks < S::kDK; ++ks) {
        qa[ks][0] = live ? *reinterpret_cast<const uint32_t*>(qs + (gq * D + ks * 16 + 2 * tq) * 2) : 0u;
        qa[ks][1] = live ? *reinterpret_cast<const uint32_t*>(qs + (gq * D + ks * 16 + 8 + 2 * tq) * 2) : 0u;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&qempty[seg & 1]);
#pragma unroll
    for (int i = 0; i < S::kDK; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    const int L = seq_len(bh / p.Hkv);

    for (int it = it0 + ((cg - it0 % NG) + NG) % NG; it < it1; it += NG) {
      const int s = it % STAGES;
      // every lane observes the phase (acquire); the warp leaves together if any lane gave up
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (it / STAGES) & 1, p.wait_limit))) {
        alive = false;
        break;
      }
      if (wg == 0 && lane == 0) observed[s] = observed[s] + 1;
      const int si_n = info[s].n;
      if (si_n >= 0) {
        const uint32_t kt = smem_u32(ring + s * 2 * S::kTile);
        const uint32_t vt = kt + S::kTile;
        const int valid = min(BLK, L - si_n * BLK);
        // ---- S = Q K^T for this warp's tokens (two accumulators per tile halve the mma chain)
        float sacc[S::kNT][4];
#pragma unroll
        for (int j = 0; j < S::kNT; ++j) {
          float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
          const uint32_t row = tok_base + j * 8 + (lane & 7);
#pragma unroll
          for (int kp = 0; kp < S::kDK / 2; ++kp) {
            const uint32_t chunk = kp * 4 + (lane >> 3);
            uint32_t r0, r1, r2, r3;
            ldsm_x4(kt + (chunk >> 3) * S::kBox + sw128(row, chunk & 7), r0, r1, r2, r3);
            if (kp & 1) {
              mma_bf16_16816(sb, qa[2 * kp][0], 0u, qa[2 * kp][1], 0u, r0, r1);
              mma_bf16_16816(sb, qa[2 * kp + 1][0], 0u, qa[2 * kp + 1][1], 0u, r2, r3);
            } else {
              mma_bf16_16816(sa, qa[2 * kp][0], 0u, qa[2 * kp][1], 0u, r0, r1);
              mma_bf16_16816(sa, qa[2 * kp + 1][0], 0u, qa[2 * kp + 1][1], 0u, r2, r3);
            }
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) sacc[j][e] = sa[e] + sb[e];
        }
        // ---- online softmax (row = query head gq; this lane holds tokens 2tq, 2tq+1 of each tile)
        float sv[S::kNT][2];
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < S::kNT; ++j) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int tok = tok_base + j * 8 + 2 * tq + e;
            const float v = tok < valid ? sacc[j][e] * sl2 : -INFINITY;
            sv[j][e] = v;
            mx = fmaxf(mx, v);
          }
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m_run, mx);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = exp2f(m_run - m_use);
        m_run = m_new;
        uint32_t pb[S::kNT];
        float ls = 0.f;
#pragma unroll
        for (int j = 0; j < S::kNT; ++j) {
          pb[j] = pack_bf16(exp2f(sv[j][0] - m_use), exp2f(sv[j][1] - m_use));
          ls += bf16_lo(pb[j]) + bf16_hi(pb[j]);
        }
        l_run = l_run * alpha + ls;
        const float a0 = __shfl_sync(0xffffffffu, alpha, (2 * tq) * 4);
        const float a1 = __shfl_sync(0xffffffffu, alpha, (2 * tq + 1) * 4);
#pragma unroll
        for (int i = 0; i < S::kDK; ++i) {
          o[i][0] *= a0;
          o[i][1] *= a1;
          o[i][2] *= a0;
          o[i][3] *= a1;
        }
        // ---- O^T += V^T P^T
        const bool ragged = valid < BLK;
#pragma unroll
        for (int kk = 0; kk < S::kKS; ++kk) {
          const uint32_t b0 = pb[2 * kk], b1 = pb[2 * kk + 1];
          const int k0 = tok_base + kk * 16;
          const uint32_t mi = lane >> 3;
          const uint32_t row = k0 + (lane & 7) + ((mi >> 1) << 3);
          const int t_lo = k0 + 2 * tq;   // tokens of the fragment halves: t_lo, t_lo+1, t_lo+8, t_lo+9
#pragma unroll
          for (int i = 0; i < S::kDK; ++i) {
            const uint32_t chunk = 2 * i + (mi & 1);
            uint32_t v0, v1, v2, v3;
            ldsm_x4_trans(vt + (chunk >> 3) * S::kBox + sw128(row, chunk & 7), v0, v1, v2, v3);
            if (ragged) {
              // rows past L may hold anything (even NaN): zero them so 0 * V stays 0
              const uint32_t m01 = (t_lo < valid ? 0x0000ffffu : 0u) | (t_lo + 1 < valid ? 0xffff0000u : 0u);
              const uint32_t m23 = (t_lo + 8 < valid ? 0x0000ffffu : 0u) | (t_lo + 9 < valid ? 0xffff0000u : 0u);
              v0 &= m01;
              v1 &= m01;
              v2 &= m23;
              v3 &= m23;
            }
            mma_bf16_16816(o[i], v0, v1, v2, v3, b0, b1);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (!__all_sync(0xffffffffu, alive)) {
      alive = false;
      break;
    }

    // ================================================================ segment flush
    const int b = bh / p.Hkv, h = bh - b * p.Hkv;
    const size_t qh0 = (size_t)b * p.Hq + (size_t)h * g;
    const bool first_seg = it0 == 0, last_seg = it1 == nit;
    if ((first_seg || last_seg) && !sh[17]) {
      // the epilogue warp publishes the split bookkeeping long before the first flush; wait if not
      const long long t0 = clock64();
      while (!sh[17] && clock64() - t0 < kWaitLimitCycles) {
      }
      if (!__all_sync(0xffffffffu, sh[17] != 0)) {
        alive = false;
        break;
      }
    }
    __threadfence_block();
    int nseg, slot_first, cf;   // pieces of this (b, h); the first piece's slot and CTA
    if (first_seg) {
      cf = sh[10];
      nseg = sh[11];
      slot_first = sh[12];
    } else if (last_seg) {
      cf = sh[13];
      nseg = sh[14];
      slot_first = sh[15];
    } else {
      cf = 0;
      nseg = 1;
      slot_first = 0;
    }
    const int slot = p.flat ? 2 * (int)blockIdx.x + (first_seg ? 0 : 1) : bh * p.ns + (int)blockIdx.x;
    // 1. each warp's state -> shared memory
    float lw = l_run;
    lw += __shfl_xor_sync(0xffffffffu, lw, 1);
    lw += __shfl_xor_sync(0xffffffffu, lw, 2);
    if (tq == 0 && gq < g) {
      Mw[warp * kMaxGroup + gq] = m_run;
      Lw[warp * kMaxGroup + gq] = lw;
    }
#pragma unroll
    for (int i = 0; i < S::kDK; ++i) {
      const int d0 = i * 16 + gq;
      const int h0 = 2 * tq, h1 = 2 * tq + 1;
      float* base = Ow + warp * kMaxGroup * D;
      if (h0 < g) {
        base[h0 * D + d0] = o[i][0];
        base[h0 * D + d0 + 8] = o[i][2];
      }
      if (h1 < g) {
        base[h1 * D + d0] = o[i][1];
        base[h1 * D + d0 + 8] = o[i][3];
      }
    }
    if (!warps_sync(cbar, cphase)) {
      alive = false;
      break;
    }
    // 2. per-head merge weights of the CW warp states, and the segment's LSE
    if (tid < CW * g) {
      const int w = tid / g, j = tid - (tid / g) * g;
      float M = -INFINITY;
#pragma unroll
      for (int w2 = 0; w2 < CW; ++w2) M = fmaxf(M, Mw[w2 * kMaxGroup + j]);
      float den = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w2 = 0; w2 < CW; ++w2) den += exp2f(Mw[w2 * kMaxGroup + j] - M) * Lw[w2 * kMaxGroup + j];
      }
      Wt[w * kMaxGroup + j] = den > 0.f ? exp2f(Mw[w * kMaxGroup + j] - M) / den : 0.f;
      if (w == 0) Hs[j] = den > 0.f ? (M + log2f(den)) * kLn2 : -INFINITY;
    }
    if (!warps_sync(cbar, cphase)) {
      alive = false;
      break;
    }
    // 3. combine: each output element is CW independent multiply-adds
    constexpr int EPT = (kMaxGroup * D + CW * 32 - 1) / (CW * 32);
#pragma unroll
    for (int u = 0; u < EPT; ++u) {
      const int e = u * CW * 32 + tid;
      if (e < g * D) {
        const int j = e / D, cc = e - j * D;
        float val = 0.f;
#pragma unroll
        for (int w = 0; w < CW; ++w) val += Wt[w * kMaxGroup + j] * Ow[(w * kMaxGroup + j) * D + cc];
        if (nseg <= 1) {
          __nv_bfloat16 ob = __float2bfloat16_rn(val);
          p.out[(qh0 + j) * D + cc] = *reinterpret_cast<uint16_t*>(&ob);
          if (cc == 0 && p.lse_out) p.lse_out[qh0 + j] = Hs[j];
        } else {
          p.o_part[((size_t)slot * g + j) * D + cc] = val;
          if (cc == 0) p.lse_part[(size_t)slot * g + j] = Hs[j];
        }
      }
    }
    if constexpr (FUSED) {
      if (nseg <= 1 && tid == 0) p.ready[bh] = 0;   // the row's only piece is done with its list
    }
    if (nseg > 1 && !last_seg) {
      // the CTA's split first segment: the epilogue warp publishes / merges it
      if (tid == 0) job[0] = Job{bh, nseg, slot_first, cf};
      __syncwarp();
      if (lane == 0) mbar_arrive(jbar);
    } else if (nseg > 1) {
      // the CTA's last segment: publish it and, if it arrived last, merge the (b, h) right here
      if (!warps_sync(cbar, cphase)) {
        alive = false;
        break;
      }
      if (tid == 0) sh[1] = atomic_add_acq_rel_gpu(&p.counters[bh], 1) == nseg - 1;
      if (!warps_sync(cbar, cphase)) {
        alive = false;
        break;
      }
      if (sh[1]) {
        bool ok = true;
        // scratch: the merge area (every warp has finished reading it) -- `epi` belongs to the epilogue warp
        merge_partials<D, CW * 32, S::kEpi>(p, bh, nseg, slot_first, cf, tid, Ow, [&] {
          ok = warps_sync(cbar, cphase) && ok;
        });
        if (!ok) {
          alive = false;
          break;
        }
        if (tid == 0) {
          p.counters[bh] = 0;
          if constexpr (FUSED) p.ready[bh] = 0;   // every piece of the row is done with its list
        }
      }
    }
    it0 = it1;
    ++seg;
    // the merge area is rewritten by the next segment's flush
    if (it0 < nit && !warps_sync(cbar, cphase)) {
      alive = false;
      break;
    }
  }
  if (!alive) {
    if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
    sh[0] = 1;
    // drain the copies still in flight (bounded) before the CTA's shared memory is released
    if (warp == 0 && lane == 0) {
      const long long t0 = clock64();
      while (!sh[9] && clock64() - t0 < kWaitLimitCycles) {
      }
      for (int s = 0; s < STAGES; ++s)
        if (issued[s] > observed[s]) mbar_wait(&full[s], observed[s] & 1, p.wait_limit);
    }
    return;
  }

  // (b, h) pairs with an empty list: zeros and lse = -inf (the capacity schedule's ranges cover
  // every (b, h), so an empty list already came out that way)
  if (p.flat == 2) return;
  const int first_bh = p.flat ? (int)blockIdx.x : (blockIdx.x == 0 ? (int)(blockIdx.z * p.Hkv + blockIdx.y) : BH);
  const int step_bh = p.flat ? (int)gridDim.x : BH;
  for (int bh = first_bh; bh < BH; bh += step_bh) {
    if (clamp_cnt(p, bh) != 0) continue;
    const int b = bh / p.Hkv, h = bh - b * p.Hkv;
    const size_t qh0 = (size_t)b * p.Hq + (size_t)h * g;
    for (int e = tid; e < g * D; e += CW * 32) {
      p.out[qh0 * D + e] = 0;
      if (e < g && p.lse_out) p.lse_out[qh0 + e] = -INFINITY;
    }
  }
}

template <int D, int BLK, int NWG, int NG, int STAGES>
__global__ void __launch_bounds__(DecodeShape<D, BLK, NWG, NG, STAGES>::kThreads, 1)
    sparse_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ DecodeParams p) {
  decode_body<D, BLK, NWG, NG, STAGES, 0>(&tmK, &tmV, p, nullptr);
}

// The fused decode step: plan (cache update, gate, selection) and decode in one launch, one CTA
// per SM in clusters of two (the pair that plans a row shares its gate through distributed
// shared memory).  Capacity schedule only.  Every CTA must be resident at once: the host sizes
// the grid by the co-resident cluster count, and every wait is bounded.
template <int D, int BLK, int DG, int NWG, int NG, int STAGES>
__global__ void __cluster_dims__(kStepCluster, 1, 1) __launch_bounds__(DecodeShape<D, BLK, NWG, NG, STAGES>::kThreads, 1)
    decode_step_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ StepParams sp) {
  decode_body<D, BLK, NWG, NG, STAGES, DG>(&tmK, &tmV, sp.d, &sp.pl);
}

// ring depth and consumer groups per shape (stage = 2 * BLK * D * 2 bytes; one CTA per SM)
#ifndef SEER_DECODE_STAGES_128_64
#define SEER_DECODE_STAGES_128_64 4
#endif
template <int D, int BLK>
struct Choice;
template <> struct Choice<64, 64> { static constexpr int NWG = 4, NG = 2, ST = 6; };
template <> struct Choice<64, 128> { static constexpr int NWG = 4, NG = 2, ST = 4; };
template <> struct Choice<128, 64> { static constexpr int NWG = 4, NG = 2, ST = SEER_DECODE_STAGES_128_64; };
template <> struct Choice<128, 128> { static constexpr int NWG = 4, NG = 2, ST = 2; };

template <int D, int BLK>
using ShapeOf = DecodeShape<D, BLK, Choice<D, BLK>::NWG, Choice<D, BLK>::NG, Choice<D, BLK>::ST>;

template <int D, int BLK>
size_t smem_bytes(int B, int BH) {
  return ShapeOf<D, BLK>::kSmemFixed + (size_t)(B + BH + 1 + 16) * 4;
}

template <int D, int BLK>
cudaError_t launch_t(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p, int grid_flat,
                     cudaStream_t st) {
  using C = Choice<D, BLK>;
  using Sh = ShapeOf<D, BLK>;
  auto kern = sparse_decode_kernel<D, BLK, C::NWG, C::NG, C::ST>;
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = ensure_smem_limit(kern, (int)smem_bytes<D, BLK>(kMaxDecodeB, kMaxDecodeBH), attr_done);
  if (e != cudaSuccess) return e;
  const size_t smem = smem_bytes<D, BLK>(p.B, p.B * p.Hkv);
  const dim3 grid = p.flat ? dim3(grid_flat, 1, 1) : dim3(p.ns, p.Hkv, p.B);
  return launch_pdl(kern, grid, dim3(Sh::kThreads), smem, st, tk, tv, p);
}

template <int D, int BLK>
int ctas_per_sm_t() {
  using C = Choice<D, BLK>;
  using Sh = ShapeOf<D, BLK>;
  auto kern = sparse_decode_kernel<D, BLK, C::NWG, C::NG, C::ST>;
  static std::atomic<uint64_t> attr_done{0};
  const int smax = (int)smem_bytes<D, BLK>(kMaxDecodeB, kMaxDecodeBH);
  if (ensure_smem_limit(kern, smax, attr_done) != cudaSuccess) return 1;
  int n = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, Sh::kThreads, smax) != cudaSuccess) return 1;
  return n > 0 ? n : 1;
}

template <int D, int BLK, int DG>
auto step_kernel() {
  using C = Choice<D, BLK>;
  return decode_step_kernel<D, BLK, DG, C::NWG, C::NG, C::ST>;
}

template <int D, int BLK, int DG>
size_t step_smem_bytes(int B, int BH) {
  return smem_bytes<D, BLK>(B, BH) + 16 + sizeof(StepPlanSmem<D, DG, ShapeOf<D, BLK>::kThreads>);
}

constexpr size_t kMaxDynSmem = 227 * 1024;

// Whether the planning phase's shared regions fit the decode's: the W_q rows in the ring and the
// q / merge areas before the barriers, the logit row in the merge area, the shared-memory
// selection's keys in the ring.
template <int D, int BLK, int DG>
bool step_fits(int g, int NB, int mode, int B, int BH) {
  using Sh = ShapeOf<D, BLK>;
  if (step_smem_bytes<D, BLK, DG>(B, BH) > kMaxDynSmem) return false;
  if (gate_wq_bytes<D, DG, kStepCluster>(g) > (size_t)Sh::kRing + 2 * Sh::kQBytes + (size_t)Sh::kMergeFloats * 4)
    return false;
  if ((size_t)NB * 4 > (size_t)Sh::kMergeFloats * 4) return false;
  const bool regs = mode != 2 && NB <= 8 * Sh::kThreads;
  if (!regs && select_smem_bytes(NB, mode) > (size_t)Sh::kRing) return false;
  return true;
}

template <int D, int BLK, int DG>
int step_grid_t(int g, int NB, int mode, int B, int BH) {
  if (!step_fits<D, BLK, DG>(g, NB, mode, B, BH)) return 0;
  auto kern = step_kernel<D, BLK, DG>();
  static std::atomic<uint64_t> attr_done{0};
  if (ensure_smem_limit(kern, (int)kMaxDynSmem, attr_done) != cudaSuccess) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kStepCluster * (sms / kStepCluster), 1, 1);
  cfg.blockDim = dim3(ShapeOf<D, BLK>::kThreads);
  cfg.dynamicSmemBytes = step_smem_bytes<D, BLK, DG>(B, BH);
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess) return 0;
  clusters = std::min(clusters, sms / kStepCluster);
  return clusters > 0 ? kStepCluster * clusters : 0;
}

template <int D, int BLK, int DG>
cudaError_t launch_step_t(const CUtensorMap& tk, const CUtensorMap& tv, const StepParams& p, int grid,
                          cudaStream_t st) {
  auto kern = step_kernel<D, BLK, DG>();
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = ensure_smem_limit(kern, (int)kMaxDynSmem, attr_done);
  if (e != cudaSuccess) return e;
  const size_t smem = step_smem_bytes<D, BLK, DG>(p.d.B, p.d.B * p.d.Hkv);
  return launch_pdl(kern, dim3(grid), dim3(ShapeOf<D, BLK>::kThreads), smem, st, tk, tv, p);
}

}  // namespace

int step_grid(int D, int BLK, int DG, int g, int NB, int mode, int B, int BH) {
#define SEER_S(d, blk, dg) \
  if (D == d && BLK == blk && DG == dg) return step_grid_t<d, blk, dg>(g, NB, mode, B, BH);
  SEER_S(64, 64, 64)
  SEER_S(64, 64, 128)
  SEER_S(64, 128, 64)
  SEER_S(64, 128, 128)
  SEER_S(128, 64, 64)
  SEER_S(128, 64, 128)
  SEER_S(128, 128, 64)
  SEER_S(128, 128, 128)
#undef SEER_S
  return 0;
}

cudaError_t launch_decode_step(const CUtensorMap& tk, const CUtensorMap& tv, const StepParams& p, int D, int BLK,
                               int DG, int grid, cudaStream_t s) {
#define SEER_S(d, blk, dg) \
  if (D == d && BLK == blk && DG == dg) return launch_step_t<d, blk, dg>(tk, tv, p, grid, s);
  SEER_S(64, 64, 64)
  SEER_S(64, 64, 128)
  SEER_S(64, 128, 64)
  SEER_S(64, 128, 128)
  SEER_S(128, 64, 64)
  SEER_S(128, 64, 128)
  SEER_S(128, 128, 64)
  SEER_S(128, 128, 128)
#undef SEER_S
  return cudaErrorInvalidValue;
}

int decode_ctas_per_sm(int D, int BLK) {
  if (D == 64 && BLK == 64) return ctas_per_sm_t<64, 64>();
  if (D == 64 && BLK == 128) return ctas_per_sm_t<64, 128>();
  if (D == 128 && BLK == 64) return ctas_per_sm_t<128, 64>();
  if (D == 128 && BLK == 128) return ctas_per_sm_t<128, 128>();
  return 1;
}

cudaError_t launch_sparse_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p, int D, int BLK,
                                 int grid_flat, cudaStream_t s) {
  if (D == 64 && BLK == 64) return launch_t<64, 64>(tk, tv, p, grid_flat, s);
  if (D == 64 && BLK == 128) return launch_t<64, 128>(tk, tv, p, grid_flat, s);
  if (D == 128 && BLK == 64) return launch_t<128, 64>(tk, tv, p, grid_flat, s);
  if (D == 128 && BLK == 128) return launch_t<128, 128>(tk, tv, p, grid_flat, s);
  return cudaErrorInvalidValue;
}

}  // namespace seer
