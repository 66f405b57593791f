// Block-sparse flash decoding over the selected KV blocks, and the split
// log-sum-exp combine.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 6: grid (batch, heads_kv, num_split); the
// selected list [batch, heads_kv, max_selected_blocks] is split by its width,
// and the kernel visits only the active block indices.  That grid is kept
// (num_split >= 1).  The default schedule (num_split == 0) balances instead:
// the concatenation of every (b, h)'s selected list is cut into equal
// contiguous ranges, one per CTA of a grid with one CTA per SM, so ragged
// counts and small batches still keep every SM streaming.
//
// The page's H100 kernel pads the query group to 64 rows for wgmma; here the
// group (g <= 8 query heads) stays a 16-row mma.sync fragment: the work per KV
// byte is ~g multiply-adds and the bound is HBM, not the tensor pipe.
//
// CTA structure.  Warp NW is the producer.  It resolves list positions 32 at a
// time (one lane each: binary search in the shared-memory prefix of the list
// lengths, one batched load of the block indices, fetched a chunk ahead), and
// its lane 0 issues 128B-swizzled TMA tile loads of each block's K and V --
// plus, at a segment's first block, a bulk copy of the group's q rows -- into
// a STAGES-deep shared-memory ring, completion counted on mbarriers.  Warps
// 0..NW-1 are consumers; each owns BLK/NW tokens of every block:
//   S   = Q K^T        (A = Q from registers, B = K via ldmatrix)
//   P   = exp2(S*scale*log2e - m)   (fp32 online softmax per query head)
//   O^T += V^T P^T     (A = V via ldmatrix.trans, B = P from S's accumulator)
// A segment is a run of consecutive positions of one (b, h) inside one CTA.
// At its last block the consumers merge their states in shared memory (two
// alternating merge buffers, one barrier per segment); a segment that is a
// whole (b, h) writes bf16 out directly, any other writes an fp32 partial and
// hands it to warp NW+1, the epilogue warp, which publishes it (fence, arrival
// counter) and, if it was the (b, h)'s last segment to arrive, merges all of
// its partials -- so the consumers never wait on a global round trip.
// All waits are bounded.
#include "seer_device.cuh"
#include "seer_internal.h"

namespace seer {
namespace {

constexpr float kLn2 = 0.6931471805599453f;

constexpr int kSegFirst = 1;  // first block of a segment (the q rows ride along)
constexpr int kSegLast = 2;   // last block of a segment

struct StageInfo {
  int n;       // block index, -1 = skip
  int bh;      // b * Hkv + h
  int flags;
  int pre;     // flattened position of the (b, h)'s first list entry (0 in the grid schedule)
  int cnt;     // the (b, h)'s list length (clamped to the capacity)
  int pad[3];
};

template <int D, int BLK, int NW, int STAGES>
struct DecodeShape {
  static constexpr int kTile = BLK * D * 2;   // bytes of one K (or V) tile
  static constexpr int kBox = BLK * 128;      // bytes of one 64-channel box
  static constexpr int kNBox = D / 64;
  static constexpr int kTPW = BLK / NW;       // tokens per consumer warp per block
  static constexpr int kNT = kTPW / 8;        // 8-token S tiles per warp
  static constexpr int kKS = kTPW / 16;       // 16-token PV k-steps per warp
  static constexpr int kDK = D / 16;          // QK^T k-steps == PV m-tiles
  static constexpr int kThreads = (NW + 2) * 32;   // consumers, producer, epilogue
  static constexpr int kRing = STAGES * 2 * kTile;
  static constexpr int kQBytes = kMaxGroup * D * 2;
  static constexpr int kMergeOne = NW * kMaxGroup * D * 4 + 2 * NW * kMaxGroup * 4;
  static constexpr int kBars = (2 * STAGES + 3) * 8;
  // fixed part; the list prefix and the sequence lengths follow (sized per launch)
  static constexpr int kEpi = 256;   // epilogue scratch: partial LSEs (segment-major) + per-head M, sum
  static constexpr size_t kSmemFixed = 1024 + kRing + STAGES * kQBytes + 2 * kMergeOne + kBars +
                                       STAGES * sizeof(StageInfo) + 2 * 16 + (kEpi + 2 * kMaxGroup) * 4 + 16 * 4;
  static_assert(kTPW % 16 == 0, "each consumer warp needs whole 16-token steps");
  static_assert(D % 64 == 0, "head_dim must be a multiple of 64");
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

// Balanced schedule: CTA c of G owns flattened positions [lo(c), lo(c+1)).
__device__ __forceinline__ long long range_lo(long long c, long long W, long long G) { return c * W / G; }
// The CTA whose range holds position `pos`.
__device__ __forceinline__ int cta_of(long long pos, long long W, long long G) {
  return (int)(((pos + 1) * G - 1) / W);
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

template <int D, int BLK, int NW, int STAGES>
__global__ void __launch_bounds__(DecodeShape<D, BLK, NW, STAGES>::kThreads)
    sparse_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const DecodeParams p) {
  using S = DecodeShape<D, BLK, NW, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* qbuf = ring + S::kRing;
  float* merge = reinterpret_cast<float*>(qbuf + STAGES * S::kQBytes);   // 2 x {Ow[NW][8][D], Mw[NW][8], Lw[NW][8]}
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(merge) + 2 * S::kMergeOne);
  uint64_t* empty = full + STAGES;
  uint64_t* cbar = empty + STAGES;   // consumer-warp barrier
  uint64_t* jbar = cbar + 1;         // [2] split-segment hand-off to the epilogue warp
  StageInfo* info = reinterpret_cast<StageInfo*>(jbar + 2);
  Job* job = reinterpret_cast<Job*>(info + STAGES);
  float* epi = reinterpret_cast<float*>(job + 2);   // [kEpi] + [2 * kMaxGroup]
  // sh[0] abort, sh[2] W, sh[3] G_eff, sh[4] p0, sh[5] p1, sh[6] first bh, sh[7] its pre
  volatile int* sh = reinterpret_cast<volatile int*>(epi + S::kEpi + 2 * kMaxGroup);
  int* slen = const_cast<int*>(reinterpret_cast<volatile int*>(sh + 16));   // [B] sequence lengths
  int* pre = slen + p.B;                                                       // [BH + 1] list prefix

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tid = threadIdx.x;
  const int BH = p.B * p.Hkv;
  const int g = p.g;
  if (tid == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NW);
    }
    mbar_init(cbar, NW);
    mbar_init(&jbar[0], NW);
    mbar_init(&jbar[1], NW);
    sh[0] = 0;
    fence_barrier_init();
  }
  pdl_wait();
  pdl_trigger();

  // ---------------------------------------------------------------- lengths, list prefix, this CTA's range
  for (int i = tid; i < p.B; i += S::kThreads) slen[i] = max(p.seqlens[i], 0);
  if (p.flat) {
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
    int* wsum = pre + BH + 1;   // scratch for NW+1 warp totals, just past the prefix
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
    if (tid == 0) {
      const int W = pre[BH];
      const long long G = min((long long)gridDim.x, (long long)max(W, 1));
      const long long c = blockIdx.x;
      long long p0 = 0, p1 = 0;
      if (c < G && W > 0) {
        p0 = range_lo(c, W, G);
        p1 = range_lo(c + 1, W, G);
      }
      const int bh0 = p1 > p0 ? bh_of(pre, BH, (int)p0) : 0;
      sh[2] = W;
      sh[3] = (int)G;
      sh[4] = (int)p0;
      sh[5] = (int)p1;
      sh[6] = bh0;
      sh[7] = pre[bh0];
    }
  } else if (tid == 0) {
    const int bh = blockIdx.z * p.Hkv + blockIdx.y;
    const int c = clamp_cnt(p, bh);
    if (p.cnt[bh] > p.cap && blockIdx.x == 0) report(p.err, SEER_DEVERR_COUNT);
    const int a = min((int)blockIdx.x * p.per_split, c), e = min(a + p.per_split, c);
    sh[2] = 0;
    sh[3] = 0;
    sh[4] = a;   // positions are local to the (b, h) in this schedule
    sh[5] = e;
    sh[6] = bh;
    sh[7] = 0;
    pre[0] = c;  // the grid schedule keeps its one list length here
  }
  __syncthreads();
  const int nit = sh[5] - sh[4];

  if (warp == NW + 1) {
    // ------------------------------------------------------------ epilogue warp
    // Which of this CTA's segments belong to a (b, h) split across CTAs (or splits)?
    bool expect[2] = {false, false};
    if (nit > 0) {
      if (p.flat) {
        const long long W = sh[2], G = sh[3];
        const int p0 = sh[4], p1 = sh[5];
        const int bf = sh[6];
        const int bl = bh_of(pre, BH, p1 - 1);
        auto split = [&](int x) { return cta_of(pre[x + 1] - 1, W, G) != cta_of(pre[x], W, G); };
        (void)p0;
        // the CTA's last segment is merged by the consumers themselves (it sets the kernel's tail)
        expect[0] = bl != bf && split(bf);
      }
    }
    for (int k = 0; k < 2; ++k) {
      if (!expect[k]) continue;
      if (!__all_sync(0xffffffffu, mbar_wait(&jbar[k], 0))) {
        if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
        break;
      }
      const Job jb = job[k];
      int last = 0;
      // publish the consumers' partial (ordered before the hand-off) and learn whether this
      // segment is the (b, h)'s last to arrive; acquire the others' partials if so
      if (lane == 0) last = atomic_add_acq_rel_gpu(&p.counters[jb.bh], 1) == jb.nseg - 1;
      if (!__shfl_sync(0xffffffffu, last, 0)) continue;
      const int b = jb.bh / p.Hkv, h = jb.bh - b * p.Hkv;
      const size_t qh0 = (size_t)b * p.Hq + (size_t)h * g;
      const int ng = jb.nseg * g;
      float* Mh = epi + S::kEpi;
      float* Zh = Mh + kMaxGroup;
      if (ng <= S::kEpi) {
        // partial LSEs -> shared (one round trip), per-head max and weight sum, then each lane
        // accumulates its outputs with one round of independent loads per segment
        for (int i0 = 0; i0 < ng; i0 += 32) {
          const int i = i0 + lane;
          if (i < ng)
            epi[i] = __ldcg(p.lse_part + (size_t)split_slot(p, jb.bh, i / g, jb.slot_first, jb.cf) * g + (i % g));
        }
        __syncwarp();
        if (lane < g) {
          float M = -INFINITY;
          for (int s2 = 0; s2 < jb.nseg; ++s2) M = fmaxf(M, epi[s2 * g + lane]);
          float Z = 0.f;
          if (M != -INFINITY)
            for (int s2 = 0; s2 < jb.nseg; ++s2) Z += expf(epi[s2 * g + lane] - M);
          Mh[lane] = M;
          Zh[lane] = Z;
        }
        __syncwarp();
        for (int i0 = 0; i0 < ng; i0 += 32) {
          const int i = i0 + lane;
          if (i < ng) {
            const float M = Mh[i % g];
            epi[i] = M != -INFINITY ? expf(epi[i] - M) : 0.f;
          }
        }
        __syncwarp();
        constexpr int EPT = kMaxGroup * D / 32;
        float acc[EPT];
#pragma unroll
        for (int t = 0; t < EPT; ++t) acc[t] = 0.f;
        for (int s2 = 0; s2 < jb.nseg; ++s2) {
          const size_t sl = (size_t)split_slot(p, jb.bh, s2, jb.slot_first, jb.cf);
#pragma unroll
          for (int t = 0; t < EPT; ++t) {
            const int e = t * 32 + lane;
            if (e < g * D) {
              const int j = e / D;
              acc[t] += epi[s2 * g + j] * __ldcg(p.o_part + (sl * g + j) * D + (e - j * D));
            }
          }
        }
#pragma unroll
        for (int t = 0; t < EPT; ++t) {
          const int e = t * 32 + lane;
          if (e < g * D) {
            const int j = e / D, cc = e - j * D;
            const float Z = Zh[j];
            __nv_bfloat16 ob = __float2bfloat16_rn(Z > 0.f ? acc[t] / Z : 0.f);
            p.out[(qh0 + j) * D + cc] = *reinterpret_cast<uint16_t*>(&ob);
            if (cc == 0 && p.lse_out) p.lse_out[qh0 + j] = Z > 0.f ? Mh[j] + logf(Z) : -INFINITY;
          }
        }
      } else {
        for (int e = lane; e < g * D; e += 32) {
          const int j = e / D, cc = e % D;
          float M = -INFINITY;
          for (int s2 = 0; s2 < jb.nseg; ++s2)
            M = fmaxf(M, __ldcg(p.lse_part + (size_t)split_slot(p, jb.bh, s2, jb.slot_first, jb.cf) * g + j));
          float num = 0.f, den = 0.f;
          if (M != -INFINITY) {
            for (int s2 = 0; s2 < jb.nseg; ++s2) {
              const size_t sl = (size_t)split_slot(p, jb.bh, s2, jb.slot_first, jb.cf);
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
      __syncwarp();
      if (lane == 0) p.counters[jb.bh] = 0;
    }
    return;
  }

  if (warp == NW) {
    // ------------------------------------------------------------ producer warp
    const int p0 = sh[4];
    const int fixed_bh = sh[6];
    // resolve list position `it` of this CTA (one lane per position)
    auto resolve = [&](int it, int& n, int& bh, int& flags, int& pr, int& cn, int& kb, int& kt, int& vb, int& vt) {
      n = -1;
      bh = fixed_bh;
      flags = 0;
      pr = 0;
      cn = 0;
      kb = vb = kt = vt = 0;
      if (it >= nit) return;
      int pos;
      if (p.flat) {
        const int x = p0 + it;
        bh = bh_of(pre, BH, x);
        pr = pre[bh];
        cn = pre[bh + 1] - pr;
        pos = x - pr;
      } else {
        cn = pre[0];
        pos = p0 + it;
      }
      flags = ((it == 0 || pos == 0) ? kSegFirst : 0) | ((it == nit - 1 || pos == cn - 1) ? kSegLast : 0);
      const int b = bh / p.Hkv;
      const int nblk = (slen[b] + BLK - 1) / BLK;
      const int blk = p.idx[(size_t)bh * p.cap + pos];
      bool ok = blk >= 0 && blk < nblk;
      if (!ok) report(p.err, SEER_DEVERR_BLOCK_INDEX);
      kb = vb = b;
      kt = vt = blk * BLK;
      if (ok && p.k_paged) {
        const int pg = blk < p.k_maxp ? p.k_table[(size_t)b * p.k_maxp + blk] : -1;
        if (pg < 0 || pg >= p.k_pages) {
          report(p.err, SEER_DEVERR_PAGE_INDEX);
          ok = false;
        }
        kb = pg;
        kt = 0;
      }
      if (ok && p.v_paged) {
        const int pg = blk < p.v_maxp ? p.v_table[(size_t)b * p.v_maxp + blk] : -1;
        if (pg < 0 || pg >= p.v_pages) {
          report(p.err, SEER_DEVERR_PAGE_INDEX);
          ok = false;
        }
        vb = pg;
        vt = 0;
      }
      n = ok ? blk : -1;
    };
    const uint64_t stream_pol = l2_evict_first_policy();   // each K/V tile is read once
    int cn_, cb_, cf_, cp_, cc_, ckb, ckt, cvb, cvt;   // current chunk (this lane's position)
    resolve(lane, cn_, cb_, cf_, cp_, cc_, ckb, ckt, cvb, cvt);
    bool abort = false;
    for (int chunk = 0; chunk * 32 < nit && !abort; ++chunk) {
      int nn, nb, nf, np, nc, nkb, nkt, nvb, nvt;   // next chunk, fetched while this one issues
      resolve((chunk + 1) * 32 + lane, nn, nb, nf, np, nc, nkb, nkt, nvb, nvt);
      const int count = min(32, nit - chunk * 32);
      for (int j = 0; j < count; ++j) {
        const int it = chunk * 32 + j;
        const int n = __shfl_sync(0xffffffffu, cn_, j);
        const int bh = __shfl_sync(0xffffffffu, cb_, j);
        const int flags = __shfl_sync(0xffffffffu, cf_, j);
        const int prv = __shfl_sync(0xffffffffu, cp_, j);
        const int cnv = __shfl_sync(0xffffffffu, cc_, j);
        const int kb = __shfl_sync(0xffffffffu, ckb, j), kt = __shfl_sync(0xffffffffu, ckt, j);
        const int vb = __shfl_sync(0xffffffffu, cvb, j), vt = __shfl_sync(0xffffffffu, cvt, j);
        if (lane == 0) {
          const int s = it % STAGES;
          if (it >= STAGES && !mbar_wait(&empty[s], ((it / STAGES) - 1) & 1)) {
            report(p.err, SEER_DEVERR_TIMEOUT);
            sh[0] = 1;
          }
          if (!sh[0]) {
            StageInfo& si = info[s];
            si.n = n;
            si.bh = bh;
            si.flags = flags;
            si.pre = prv;
            si.cnt = cnv;
            const bool first = flags & kSegFirst;
            const uint32_t qbytes = (uint32_t)(g * D * 2);
            const uint32_t tx = (n >= 0 ? 2u * S::kTile : 0u) + (first ? qbytes : 0u);
            if (tx) {
              mbar_arrive_expect_tx(&full[s], tx);
              if (first) {
                const int b = bh / p.Hkv, h = bh - b * p.Hkv;
                bulk_load(qbuf + s * S::kQBytes, p.q + ((size_t)b * p.Hq + (size_t)h * g) * D, qbytes, &full[s]);
              }
              if (n >= 0) {
                const int h = bh % p.Hkv;
                uint8_t* kdst = ring + s * 2 * S::kTile;
                uint8_t* vdst = kdst + S::kTile;
                int c1, c2, c3;
                tile_coords(p.k_perm, kt, h, kb, c1, c2, c3);
#pragma unroll
                for (int bx = 0; bx < S::kNBox; ++bx)
                  tma_load_4d_hint(kdst + bx * S::kBox, &tmK, &full[s], bx * 64, c1, c2, c3, stream_pol);
                tile_coords(p.v_perm, vt, h, vb, c1, c2, c3);
#pragma unroll
                for (int bx = 0; bx < S::kNBox; ++bx)
                  tma_load_4d_hint(vdst + bx * S::kBox, &tmV, &full[s], bx * 64, c1, c2, c3, stream_pol);
              }
            } else {
              mbar_arrive(&full[s]);
            }
          }
        }
        if (__shfl_sync(0xffffffffu, (int)sh[0], 0)) {
          abort = true;
          break;
        }
      }
      cn_ = nn; cb_ = nb; cf_ = nf; cp_ = np; cc_ = nc; ckb = nkb; ckt = nkt; cvb = nvb; cvt = nvt;
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gq = lane >> 2, tq = lane & 3;
  uint32_t qa[S::kDK][2];
  float o[S::kDK][4];
#pragma unroll
  for (int i = 0; i < S::kDK; ++i) {
    qa[i][0] = qa[i][1] = 0u;
    o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  }
  float m_run = -INFINITY, l_run = 0.f;
  const float sl2 = p.scale_log2;
  const int tok_base = warp * S::kTPW;
  int L = 0;
  int seg_start_it = 0;
  int consumed = 0;
  int nflush = 0;
  uint32_t cphase = 0;
  bool alive = true;

  for (int it = 0; it < nit; ++it) {
    const int s = it % STAGES;
    // every lane observes the phase (acquire); the warp leaves together if any lane gave up
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (it / STAGES) & 1))) {
      alive = false;
      break;
    }
    consumed = it + 1;
    const int si_n = info[s].n, si_bh = info[s].bh, si_flags = info[s].flags;
    const int si_pre = info[s].pre, si_cnt = info[s].cnt;
    if (si_flags & kSegFirst) {
      // new segment: the group's q rows (rows >= g stay zero) and a fresh state
      const uint8_t* qs = qbuf + s * S::kQBytes;
      const bool live = gq < g;
#pragma unroll
      for (int ks = 0; ks < S::kDK; ++ks) {
        qa[ks][0] = live ? *reinterpret_cast<const uint32_t*>(qs + (gq * D + ks * 16 + 2 * tq) * 2) : 0u;
        qa[ks][1] = live ? *reinterpret_cast<const uint32_t*>(qs + (gq * D + ks * 16 + 8 + 2 * tq) * 2) : 0u;
      }
#pragma unroll
      for (int i = 0; i < S::kDK; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
      m_run = -INFINITY;
      l_run = 0.f;
      L = slen[si_bh / p.Hkv];
      seg_start_it = it;
    }
    if (si_n >= 0) {
      const uint32_t kt = smem_u32(ring + s * 2 * S::kTile);
      const uint32_t vt = kt + S::kTile;
      const int valid = min(BLK, L - si_n * BLK);
      // ---- S = Q K^T for this warp's tokens
      float sacc[S::kNT][4];
#pragma unroll
      for (int j = 0; j < S::kNT; ++j) {
        sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
        const uint32_t row = tok_base + j * 8 + (lane & 7);
#pragma unroll
        for (int kp = 0; kp < S::kDK / 2; ++kp) {
          const uint32_t chunk = kp * 4 + (lane >> 3);
          uint32_t r0, r1, r2, r3;
          ldsm_x4(kt + (chunk >> 3) * S::kBox + sw128(row, chunk & 7), r0, r1, r2, r3);
          mma_bf16_16816(sacc[j], qa[2 * kp][0], 0u, qa[2 * kp][1], 0u, r0, r1);
          mma_bf16_16816(sacc[j], qa[2 * kp + 1][0], 0u, qa[2 * kp + 1][1], 0u, r2, r3);
        }
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
    if (!(si_flags & kSegLast)) continue;

    // ================================================================ segment flush
    const int bh = si_bh;
    const int b = bh / p.Hkv, h = bh - b * p.Hkv;
    const size_t qh0 = (size_t)b * p.Hq + (size_t)h * g;
    int nseg, slot, slot_first, cf = 0;   // segments of this (b, h); this segment's partial slot; the first one's
    if (p.flat) {
      const long long W = sh[2], G = sh[3];
      cf = cta_of(si_pre, W, G);
      nseg = cta_of(si_pre + si_cnt - 1, W, G) - cf + 1;
      slot = 2 * (int)blockIdx.x + (seg_start_it == 0 ? 0 : 1);
      slot_first = 2 * cf + (range_lo(cf, W, G) != si_pre ? 1 : 0);
    } else {
      nseg = (si_cnt + p.per_split - 1) / p.per_split;
      slot = bh * p.ns + (int)blockIdx.x;
      slot_first = bh * p.ns;
    }
    float* Ow = merge + (nflush & 1) * (S::kMergeOne / 4);
    float* Mw = Ow + NW * kMaxGroup * D;
    float* Lw = Mw + NW * kMaxGroup;
    ++nflush;
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
    for (int e = tid; e < g * D; e += NW * 32) {
      const int j = e / D, cc = e % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) M = fmaxf(M, Mw[w * kMaxGroup + j]);
      float num = 0.f, den = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          const float sc = exp2f(Mw[w * kMaxGroup + j] - M);
          num += sc * Ow[(w * kMaxGroup + j) * D + cc];
          den += sc * Lw[w * kMaxGroup + j];
        }
      }
      const bool any = den > 0.f;
      const float oval = any ? num / den : 0.f;
      const float lse = any ? (M + log2f(den)) * kLn2 : -INFINITY;
      if (nseg <= 1) {
        __nv_bfloat16 ob = __float2bfloat16_rn(oval);
        p.out[(qh0 + j) * D + cc] = *reinterpret_cast<uint16_t*>(&ob);
        if (cc == 0 && p.lse_out) p.lse_out[qh0 + j] = lse;
      } else {
        p.o_part[((size_t)slot * g + j) * D + cc] = oval;
        if (cc == 0) p.lse_part[(size_t)slot * g + j] = lse;
      }
    }
    if (nseg > 1 && it != nit - 1) {   // a split first segment: the epilogue warp publishes / merges it
      if (tid == 0) job[0] = Job{bh, nseg, slot_first, cf};
      __syncwarp();
      if (lane == 0) mbar_arrive(&jbar[0]);
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
        constexpr int EPC = (kMaxGroup * D + NW * 32 - 1) / (NW * 32);   // outputs per thread
        constexpr int MAXS = 4;                                           // segments merged from registers
        if (nseg <= MAXS) {
          float lv[MAXS][EPC], ov[MAXS][EPC];
#pragma unroll
          for (int s2 = 0; s2 < MAXS; ++s2) {
            const size_t sl = (size_t)split_slot(p, bh, s2 < nseg ? s2 : 0, slot_first, cf);
#pragma unroll
            for (int t = 0; t < EPC; ++t) {
              const int e = tid + t * NW * 32;
              const int j = e / D;
              const bool on = s2 < nseg && e < g * D;
              lv[s2][t] = on ? __ldcg(p.lse_part + sl * g + j) : -INFINITY;
              ov[s2][t] = on ? __ldcg(p.o_part + (sl * g + j) * D + (e - j * D)) : 0.f;
            }
          }
#pragma unroll
          for (int t = 0; t < EPC; ++t) {
            const int e = tid + t * NW * 32;
            if (e >= g * D) continue;
            const int j = e / D, cc = e - j * D;
            float M = -INFINITY;
#pragma unroll
            for (int s2 = 0; s2 < MAXS; ++s2) M = fmaxf(M, lv[s2][t]);
            float num = 0.f, den = 0.f;
            if (M != -INFINITY) {
#pragma unroll
              for (int s2 = 0; s2 < MAXS; ++s2) {
                const float w = s2 < nseg ? expf(lv[s2][t] - M) : 0.f;
                num += w * ov[s2][t];
                den += w;
              }
            }
            const bool any = den > 0.f;
            __nv_bfloat16 ob = __float2bfloat16_rn(any ? num / den : 0.f);
            p.out[(qh0 + j) * D + cc] = *reinterpret_cast<uint16_t*>(&ob);
            if (cc == 0 && p.lse_out) p.lse_out[qh0 + j] = any ? M + logf(den) : -INFINITY;
          }
        } else {
          for (int e = tid; e < g * D; e += NW * 32) {
            const int j = e / D, cc = e % D;
            float M = -INFINITY;
            for (int s2 = 0; s2 < nseg; ++s2)
              M = fmaxf(M, __ldcg(p.lse_part + (size_t)split_slot(p, bh, s2, slot_first, cf) * g + j));
            float num = 0.f, den = 0.f;
            if (M != -INFINITY) {
              for (int s2 = 0; s2 < nseg; ++s2) {
                const size_t sl = (size_t)split_slot(p, bh, s2, slot_first, cf);
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
        if (tid == 0) p.counters[bh] = 0;
      }
    }
  }
  if (!alive) {
    if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
    sh[0] = 1;
    // drain the copies still in flight (bounded) before the CTA's shared memory is released
    if (warp == 0 && lane == 0)
      for (int it = consumed; it < nit && it < consumed + STAGES; ++it) mbar_wait(&full[it % STAGES], (it / STAGES) & 1);
    return;
  }

  // (b, h) pairs with an empty list: zeros and lse = -inf
  const int first_bh = p.flat ? (int)blockIdx.x : (blockIdx.x == 0 ? (int)(blockIdx.z * p.Hkv + blockIdx.y) : BH);
  const int step_bh = p.flat ? (int)gridDim.x : BH;
  for (int bh = first_bh; bh < BH; bh += step_bh) {
    if (clamp_cnt(p, bh) != 0) continue;
    const int b = bh / p.Hkv, h = bh - b * p.Hkv;
    const size_t qh0 = (size_t)b * p.Hq + (size_t)h * g;
    for (int e = tid; e < g * D; e += NW * 32) {
      p.out[qh0 * D + e] = 0;
      if (e < g && p.lse_out) p.lse_out[qh0 + e] = -INFINITY;
    }
  }
}

// ring depth per shape (stage = 2 * BLK * D * 2 bytes; one CTA per SM)
#ifndef SEER_DECODE_STAGES_128_64
#define SEER_DECODE_STAGES_128_64 4
#endif
template <int D, int BLK>
struct Choice;
template <> struct Choice<64, 64> { static constexpr int NW = 4, ST = 6; };
template <> struct Choice<64, 128> { static constexpr int NW = 4, ST = 4; };
template <> struct Choice<128, 64> { static constexpr int NW = 4, ST = SEER_DECODE_STAGES_128_64; };
template <> struct Choice<128, 128> { static constexpr int NW = 4, ST = 2; };

template <int D, int BLK>
size_t smem_bytes(int B, int BH) {
  using C = Choice<D, BLK>;
  return DecodeShape<D, BLK, C::NW, C::ST>::kSmemFixed + (size_t)(B + BH + 1 + 8) * 4;
}

template <int D, int BLK>
cudaError_t launch_t(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p, int grid_flat,
                     cudaStream_t st) {
  constexpr int NW = Choice<D, BLK>::NW, ST = Choice<D, BLK>::ST;
  using Sh = DecodeShape<D, BLK, NW, ST>;
  auto kern = sparse_decode_kernel<D, BLK, NW, ST>;
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = ensure_smem_limit(kern, (int)smem_bytes<D, BLK>(kMaxDecodeB, kMaxDecodeBH), attr_done);
  if (e != cudaSuccess) return e;
  const size_t smem = smem_bytes<D, BLK>(p.B, p.B * p.Hkv);
  const dim3 grid = p.flat ? dim3(grid_flat, 1, 1) : dim3(p.ns, p.Hkv, p.B);
  return launch_pdl(kern, grid, dim3(Sh::kThreads), smem, st, tk, tv, p);
}

template <int D, int BLK>
int ctas_per_sm_t() {
  constexpr int NW = Choice<D, BLK>::NW, ST = Choice<D, BLK>::ST;
  using Sh = DecodeShape<D, BLK, NW, ST>;
  auto kern = sparse_decode_kernel<D, BLK, NW, ST>;
  static std::atomic<uint64_t> attr_done{0};
  const int smax = (int)smem_bytes<D, BLK>(kMaxDecodeB, kMaxDecodeBH);
  if (ensure_smem_limit(kern, smax, attr_done) != cudaSuccess) return 1;
  int n = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, Sh::kThreads, smax) != cudaSuccess) return 1;
  return n > 0 ? n : 1;
}

}  // namespace

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
