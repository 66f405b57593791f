// Decode ground truth: the block scores full attention would give, from the
// whole K cache -- the target the AttnGate is distilled towards, usable in
// place of the gate ("oracle" block selection).
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 3: for decoding, the attention map of the g
// query heads of a group over all L tokens is 1-D max-pooled over each
// block's columns, the g pooled rows are reduced by max, and the result is
// normalised to sum to 1.  With s_j[t] = scale * q_j . K[t] (and the usual
// softmax p_j[t] = exp(s_j[t] - lse_j)):
//   gt[n] = max_j max_{t in block n} p_j[t] / sum_n' (same)
//         = max_j exp(bmax_j[n] - lse_j) / sum_n' (same)
// so one streaming pass over K yields everything: per block and head the score
// maximum, per head the running (max, sum of exp).
//
// The work is the (b, h, chunk of kChunk consecutive blocks) items; a grid of
// one wave of persistent CTAs takes them in contiguous runs, so each CTA's
// TMA ring streams straight across chunk (and (b, h)) boundaries.  A producer
// warp brings K tiles (128B swizzle, box 64 channels x b tokens) into a ring
// of mbarrier-guarded stages, and the group's query rows into one of two
// buffers per item; four consumer warps own b/4 tokens of every block and
// compute S = Q K^T on mma.sync (the group's <= 8 query rows as a 16-row A
// fragment) in the log2 domain, leaving per-head block maxima and, at a
// chunk's end, per-head (max, sum) in a shared-memory hand-off slot.  An
// epilogue warp folds the four warps' values into one per head, writes them to
// the workspace, publishes the chunk (acquire-release counter) and, for the
// (b, h)'s last chunk to arrive, forms lse_j, the scores and their
// normalisation and resets the counter -- off the streaming path.  All waits
// are bounded.
#include "seer_device.cuh"
#include "seer_internal.h"

namespace seer {
namespace {

constexpr int kNW = 4;         // consumer warps
constexpr int kChunk = 16;     // blocks per work item
constexpr int kJobs = 2;       // chunk hand-off slots between the consumers and the epilogue warp
constexpr int kSlotFloats = kChunk * kNW * kMaxGroup + kNW * kMaxGroup * 2;   // block maxima, (max, sum)

template <int D, int BLK>
struct TruthShape {
  static constexpr int kTile = BLK * D * 2;
  static constexpr int kBox = BLK * 128;
  static constexpr int kNBox = D / 64;
  static constexpr int kTPW = BLK / kNW;
  static constexpr int kNT = kTPW / 8;
  static constexpr int kDK = D / 16;
  static constexpr int kStages = (6 * 16384) / kTile < 2 ? 2 : (6 * 16384) / kTile;   // ~96 KB of ring
  static constexpr int kQBytes = kMaxGroup * D * 2;
  static constexpr int kThreads = (kNW + 2) * 32;   // consumers, producer, epilogue
  static constexpr size_t kSmem = 1024 + (size_t)kStages * kTile + 2 * kQBytes + kJobs * kSlotFloats * 4 +
                                  (2 * kStages + 4 + 2 * kJobs) * 8 + kStages * 16 + kJobs * 16 + 64 * 4;
};

struct Stage {
  int bh, n, flags, nblk;   // flags: 1 first block of an item, 2 last block of an item; bits 8+: valid tokens
};

__device__ __forceinline__ void coords(const int32_t perm[3], int t, int h, int bp, int& c1, int& c2, int& c3) {
  int c[3];
  c[perm[0]] = t;
  c[perm[1]] = h;
  c[perm[2]] = bp;
  c1 = c[0];
  c2 = c[1];
  c3 = c[2];
}

// Item i -> (b, h) and chunk; its blocks [n0, n1) (empty when the chunk lies past ceil(L/b)).
__device__ __forceinline__ void item_of(const TruthParams& p, int i, int BLK, int& bh, int& chunk, int& n0, int& n1,
                                        int& nblk) {
  bh = i / p.nchunk;
  chunk = i - bh * p.nchunk;
  const int b = bh / p.Hkv;
  const int L = max(__ldg(p.seqlens + b), 0);
  nblk = min((L + BLK - 1) / BLK, p.NB);
  n0 = chunk * kChunk;
  n1 = min(nblk, n0 + kChunk);
}

// One warp: the (b, h)'s scores from every chunk's per-head (max, sum) and the per-head block maxima
// (workspace rows of kMaxGroup floats), with many loads in flight per lane.
__device__ void truth_finish(const TruthParams& p, int bh, int nblk, int lane) {
  const int g = p.g;
  const int nch = (nblk + kChunk - 1) / kChunk;
  // lse_j (log2 domain): lanes stride over the chunks, then a warp reduction per head
  float m[kMaxGroup], l[kMaxGroup];
#pragma unroll
  for (int j = 0; j < kMaxGroup; ++j) {
    m[j] = -INFINITY;
    l[j] = 0.f;
  }
  for (int c = lane; c < nch; c += 32) {
    const float4* pc = reinterpret_cast<const float4*>(p.part + ((size_t)bh * p.nchunk + c) * kMaxGroup * 2);
    float4 v[kMaxGroup / 2];
#pragma unroll
    for (int k = 0; k < kMaxGroup / 2; ++k) v[k] = __ldcg(pc + k);
#pragma unroll
    for (int k = 0; k < kMaxGroup / 2; ++k) {
      const float cm[2] = {v[k].x, v[k].z}, cl[2] = {v[k].y, v[k].w};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = 2 * k + e;
        const float mn = fmaxf(m[j], cm[e]);
        if (mn != -INFINITY) {
          l[j] = l[j] * exp2f(m[j] - mn) + cl[e] * exp2f(cm[e] - mn);
          m[j] = mn;
        }
      }
    }
  }
  float lse2[kMaxGroup];
#pragma unroll
  for (int j = 0; j < kMaxGroup; ++j) {
    float M = m[j];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float Z = M == -INFINITY ? 0.f : l[j] * exp2f(m[j] - M);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, off);
    lse2[j] = Z > 0.f ? M + log2f(Z) : INFINITY;   // +inf: no token of this head (not for nblk > 0)
  }
  // raw[n] = max_j exp2(bmax_j[n] - lse2_j), written unnormalised; the sum over n
  constexpr int U = 4;
  float* scores = p.scores + (size_t)bh * p.NB;
  const float* bmax = p.bmax + (size_t)bh * p.NB * kMaxGroup;
  float sum = 0.f;
  for (int nb = 0; nb < nblk; nb += 32 * U) {
    float4 lo[U], hi[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int n = nb + u * 32 + lane;
      if (n < nblk) {
        lo[u] = __ldcg(reinterpret_cast<const float4*>(bmax + (size_t)n * kMaxGroup));
        hi[u] = __ldcg(reinterpret_cast<const float4*>(bmax + (size_t)n * kMaxGroup + 4));
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int n = nb + u * 32 + lane;
      if (n < nblk) {
        const float bm[kMaxGroup] = {lo[u].x, lo[u].y, lo[u].z, lo[u].w, hi[u].x, hi[u].y, hi[u].z, hi[u].w};
        float r = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxGroup; ++j)
          if (j < g) r = fmaxf(r, exp2f(bm[j] - lse2[j]));
        scores[n] = r;
        sum += r;
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  float* lscores = p.log_scores ? p.log_scores + (size_t)bh * p.NB : nullptr;
  for (int nb = 0; nb < p.NB; nb += 32 * U) {
    float r[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int n = nb + u * 32 + lane;
      r[u] = n < nblk ? scores[n] : 0.f;   // this lane's own unnormalised value
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int n = nb + u * 32 + lane;
      if (n < p.NB) {
        const float gt = r[u] * inv;
        scores[n] = gt;
        if (lscores) lscores[n] = gt > 0.f ? logf(gt) : -INFINITY;
      }
    }
  }
}

template <int D, int BLK>
__global__ void __launch_bounds__(TruthShape<D, BLK>::kThreads, 1)
    truth_kernel(const __grid_constant__ CUtensorMap tmK, const TruthParams p) {
  using S = TruthShape<D, BLK>;
  constexpr int ST = S::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qbuf = ring + (size_t)ST * S::kTile;   // [2] item query rows
  float* slots = reinterpret_cast<float*>(qbuf + 2 * S::kQBytes);   // [kJobs][kSlotFloats]
  uint64_t* full = reinterpret_cast<uint64_t*>(slots + kJobs * kSlotFloats);
  uint64_t* empty = full + ST;
  uint64_t* qfull = empty + ST;     // [2]
  uint64_t* qempty = qfull + 2;     // [2]
  uint64_t* jfull = qempty + 2;     // [kJobs] chunk hand-off
  uint64_t* jempty = jfull + kJobs; // [kJobs]
  Stage* info = reinterpret_cast<Stage*>(jempty + kJobs);
  int4* job = reinterpret_cast<int4*>(info + ST);   // [kJobs] {bh, nblk, chunk, 1 = the consumers are done}
  // [0] abort, [2] producer done, [3] query loads issued, [4] query loads seen by warp 0
  volatile int* sh = reinterpret_cast<volatile int*>(job + kJobs);
  volatile int* issued = sh + 8;            // [ST]
  volatile int* observed = issued + ST;     // [ST]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int g = p.g;
  if (tid == 0) {
    tma_prefetch_desc(&tmK);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kNW);
      issued[s] = observed[s] = 0;
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&qfull[k], 1);
      mbar_init(&qempty[k], kNW);
    }
    for (int k = 0; k < kJobs; ++k) {
      mbar_init(&jfull[k], kNW);
      mbar_init(&jempty[k], 1);
    }
    sh[0] = sh[2] = sh[3] = sh[4] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  // this CTA's contiguous run of items
  const int G = gridDim.x, c = blockIdx.x;
  const int i0 = (int)((long long)c * p.nitems / G), i1 = (int)((long long)(c + 1) * p.nitems / G);

  if (warp == kNW) {
    // ------------------------------------------------------------ producer warp
    if (lane == 0) {
      int it = 0, nq = 0;
      bool stop = false;
      for (int i = i0; i < i1 && !stop; ++i) {
        int bh, chunk, n0, n1, nblk;
        item_of(p, i, BLK, bh, chunk, n0, n1, nblk);
        if (n0 >= n1) {
          if (nblk == 0 && chunk == 0) {   // an empty sequence: its row is all zero
            float* scores = p.scores + (size_t)bh * p.NB;
            for (int n = 0; n < p.NB; ++n) {
              scores[n] = 0.f;
              if (p.log_scores) p.log_scores[(size_t)bh * p.NB + n] = -INFINITY;
            }
          }
          continue;
        }
        const int b = bh / p.Hkv, h = bh - b * p.Hkv;
        {   // the item's query rows -> buffer nq & 1, once the item two back has read it
          const int k = nq & 1, u = nq >> 1;
          if (u >= 1 && !mbar_wait(&qempty[k], (u - 1) & 1)) {
            report(p.err, SEER_DEVERR_TIMEOUT);
            sh[0] = 1;
            break;
          }
          const uint32_t qbytes = (uint32_t)(g * D * 2);
          mbar_arrive_expect_tx(&qfull[k], qbytes);
          bulk_load(qbuf + k * S::kQBytes, p.q + ((size_t)b * p.Hq + (size_t)h * g) * D, qbytes, &qfull[k]);
          sh[3] = ++nq;
        }
        for (int n = n0; n < n1; ++n, ++it) {
          const int s = it % ST;
          if (it >= ST && !mbar_wait(&empty[s], ((it / ST) - 1) & 1)) {
            report(p.err, SEER_DEVERR_TIMEOUT);
            sh[0] = 1;
            stop = true;
            break;
          }
          const int flags = (n == n0 ? 1 : 0) | (n == n1 - 1 ? 2 : 0);
          const int L = __ldg(p.seqlens + b);
          int tb = b, tt = n * BLK;
          bool ok = true;
          if (p.k_paged) {
            const int pg = n < p.k_maxp ? p.k_table[(size_t)b * p.k_maxp + n] : -1;
            if (pg < 0 || pg >= p.k_pages) {
              report(p.err, SEER_DEVERR_PAGE_INDEX);
              ok = false;
            }
            tb = pg;
            tt = 0;
          }
          // a skipped tile scores nothing
          info[s] = Stage{bh, n, flags | ((ok ? min(BLK, L - n * BLK) : 0) << 8), nblk};
          if (ok) {
            mbar_arrive_expect_tx(&full[s], S::kTile);
            int c1, c2, c3;
            coords(p.k_perm, tt, h, tb, c1, c2, c3);
#pragma unroll
            for (int bx = 0; bx < S::kNBox; ++bx)
              tma_load_4d(ring + (size_t)s * S::kTile + bx * S::kBox, &tmK, &full[s], bx * 64, c1, c2, c3);
          } else {
            mbar_arrive(&full[s]);   // an empty stage: the consumers score nothing from it
          }
          issued[s] = issued[s] + 1;
        }
      }
      // the end marker: one more stage whose flags say so (no tile)
      if (!sh[0]) {
        const int s = it % ST;
        if (it < ST || mbar_wait(&empty[s], ((it / ST) - 1) & 1)) {
          info[s] = Stage{-1, 0, 0, 0};
          mbar_arrive(&full[s]);
          issued[s] = issued[s] + 1;
        } else {
          report(p.err, SEER_DEVERR_TIMEOUT);
          sh[0] = 1;
        }
      }
      __threadfence_block();
      sh[2] = 1;
    }
    return;
  }

  if (warp == kNW + 1) {
    // ------------------------------------------------------------ epilogue warp
    for (int j = 0;; ++j) {
      const int k = j % kJobs;
      if (!__all_sync(0xffffffffu, mbar_wait(&jfull[k], (j / kJobs) & 1))) {
        if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
        return;
      }
      const int4 jb = job[k];
      if (jb.w) return;   // the consumers are done (no reply expected)
      const int bh = jb.x, nblk = jb.y, chunk = jb.z;
      const int cnt = min(kChunk, nblk - chunk * kChunk);
      const float* sl = slots + k * kSlotFloats;
      // block maxima over the warps: lane -> block lane / 2, heads 4 (lane & 1) ..
      const int nl = lane >> 1, hh = (lane & 1) * 4;
      float4 bm = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      if (nl < cnt)
#pragma unroll
        for (int w = 0; w < kNW; ++w) {
          const float4 v = *reinterpret_cast<const float4*>(sl + (nl * kNW + w) * kMaxGroup + hh);
          bm = make_float4(fmaxf(bm.x, v.x), fmaxf(bm.y, v.y), fmaxf(bm.z, v.z), fmaxf(bm.w, v.w));
        }
      // (max, sum) over the warps: lane -> head
      float M = -INFINITY, Z = 0.f;
      if (lane < kMaxGroup) {
        const float* pw = sl + kChunk * kNW * kMaxGroup;
#pragma unroll
        for (int w = 0; w < kNW; ++w) M = fmaxf(M, pw[(w * kMaxGroup + lane) * 2]);
        if (M != -INFINITY)
#pragma unroll
          for (int w = 0; w < kNW; ++w) {
            const float wm = pw[(w * kMaxGroup + lane) * 2], wl = pw[(w * kMaxGroup + lane) * 2 + 1];
            if (wm != -INFINITY) Z += wl * exp2f(wm - M);
          }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&jempty[k]);   // the slot is free again
      if (nl < cnt)
        *reinterpret_cast<float4*>(p.bmax + ((size_t)bh * p.NB + chunk * kChunk + nl) * kMaxGroup + hh) = bm;
      if (lane < kMaxGroup)
        *reinterpret_cast<float2*>(p.part + (((size_t)bh * p.nchunk + chunk) * kMaxGroup + lane) * 2) =
            make_float2(M, Z);
      __threadfence();
      __syncwarp();
      // publish the chunk and learn whether it is the (b, h)'s last to arrive; acquire the others' if so
      int last = 0;
      if (lane == 0) last = atomic_add_acq_rel_gpu(&p.counters[bh], 1) == (nblk + kChunk - 1) / kChunk - 1;
      if (__shfl_sync(0xffffffffu, last, 0)) {
        truth_finish(p, bh, nblk, lane);
        __syncwarp();
        if (lane == 0) p.counters[bh] = 0;
      }
    }
  }

  // -------------------------------------------------------------- consumers
  const int gq = lane >> 2, tq = lane & 3;
  const bool live = gq < g;
  const float sl2 = p.scale_log2;
  const int tok_base = warp * S::kTPW;
  uint32_t qa[S::kDK][2];
  float m_run = -INFINITY, l_run = 0.f;
  int nq = 0, njob = 0;
  bool alive = true;
  for (int it = 0;; ++it) {
    const int s = it % ST;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (it / ST) & 1))) {
      alive = false;
      break;
    }
    if (warp == 0 && lane == 0) observed[s] = observed[s] + 1;
    const Stage si = info[s];
    if (si.bh < 0) {   // end marker
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      break;
    }
    const int js = njob % kJobs;
    float* sl = slots + js * kSlotFloats;
    if (si.flags & 1) {
      // a new item: a free hand-off slot, the item's query rows (then release their buffer), a fresh
      // (max, sum)
      if (njob >= kJobs && !__all_sync(0xffffffffu, mbar_wait(&jempty[js], ((njob / kJobs) - 1) & 1))) {
        alive = false;
        break;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&qfull[nq & 1], (nq >> 1) & 1))) {
        alive = false;
        break;
      }
      const uint8_t* qs = qbuf + (nq & 1) * S::kQBytes;
#pragma unroll
      for (int ks = 0; ks < S::kDK; ++ks) {
        qa[ks][0] = live ? *reinterpret_cast<const uint32_t*>(qs + (gq * D + ks * 16 + 2 * tq) * 2) : 0u;
        qa[ks][1] = live ? *reinterpret_cast<const uint32_t*>(qs + (gq * D + ks * 16 + 8 + 2 * tq) * 2) : 0u;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&qempty[nq & 1]);
      ++nq;
      if (warp == 0 && lane == 0) sh[4] = nq;
      m_run = -INFINITY;
      l_run = 0.f;
    }
    const int valid = si.flags >> 8;
    const uint32_t kt = smem_u32(ring + (size_t)s * S::kTile);
    float sacc[S::kNT][4];
#pragma unroll
    for (int j = 0; j < S::kNT; ++j) {
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t row = tok_base + j * 8 + (lane & 7);
#pragma unroll
      for (int kp = 0; kp < S::kDK / 2; ++kp) {
        const uint32_t chk = kp * 4 + (lane >> 3);
        uint32_t r0, r1, r2, r3;
        ldsm_x4(kt + (chk >> 3) * S::kBox + sw128(row, chk & 7), r0, r1, r2, r3);
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
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);   // the tile is in registers now
    // this lane: head gq, tokens 2tq, 2tq+1 of each 8-token tile; log2-domain scores
    float v[S::kNT][2];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < S::kNT; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tok = tok_base + j * 8 + 2 * tq + e;
        v[j][e] = tok < valid ? sacc[j][e] * sl2 : -INFINITY;
        mx = fmaxf(mx, v[j][e]);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    if (tq == 0 && live) sl[((si.n % kChunk) * kNW + warp) * kMaxGroup + gq] = mx;
    const float m_new = fmaxf(m_run, mx);
    if (m_new != -INFINITY) {
      float ls = 0.f;
#pragma unroll
      for (int j = 0; j < S::kNT; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) ls += exp2f(v[j][e] - m_new);
      l_run = l_run * exp2f(m_run - m_new) + ls;
      m_run = m_new;
    }
    if (si.flags & 2) {
      // the item's last block: this warp's (max, sum) per head, then hand the chunk over
      float lw = l_run;
      lw += __shfl_xor_sync(0xffffffffu, lw, 1);
      lw += __shfl_xor_sync(0xffffffffu, lw, 2);
      float* pw = sl + kChunk * kNW * kMaxGroup + (warp * kMaxGroup + gq) * 2;
      if (tq == 0 && live) {
        pw[0] = m_run;
        pw[1] = lw;
      }
      if (warp == 0 && lane == 0) job[js] = make_int4(si.bh, si.nblk, si.n / kChunk, 0);
      __syncwarp();
      if (lane == 0) mbar_arrive(&jfull[js]);
      ++njob;
    }
  }
  if (alive) {
    // tell the epilogue warp it is done
    const int k = njob % kJobs;
    if (njob >= kJobs && !__all_sync(0xffffffffu, mbar_wait(&jempty[k], ((njob / kJobs) - 1) & 1))) {
      alive = false;
    } else {
      if (warp == 0 && lane == 0) job[k] = make_int4(-1, 0, 0, 1);
      __syncwarp();
      if (lane == 0) mbar_arrive(&jfull[k]);
      return;
    }
  }
  if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
  sh[0] = 1;
  if (warp == 0 && lane == 0) {
    // drain the copies still in flight (bounded) before shared memory is released
    const long long t0 = clock64();
    while (!sh[2] && clock64() - t0 < kWaitLimitCycles) {
    }
    for (int st = 0; st < ST; ++st)
      if (issued[st] > observed[st]) mbar_wait(&full[st], observed[st] & 1);
    for (int u = sh[4]; u < sh[3]; ++u) mbar_wait(&qfull[u & 1], (u >> 1) & 1);
  }
}

template <int D, int BLK>
cudaError_t launch_t(const CUtensorMap& tk, TruthParams p, int sms, cudaStream_t st) {
  using S = TruthShape<D, BLK>;
  auto kern = truth_kernel<D, BLK>;
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = ensure_smem_limit(kern, (int)S::kSmem, attr_done);
  if (e != cudaSuccess) return e;
  static std::atomic<int> occ_cache{0};
  int occ = occ_cache.load();
  if (occ == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, S::kThreads, S::kSmem) != cudaSuccess || occ < 1)
      occ = 1;
    occ_cache.store(occ);
  }
  const int grid = std::max(1, std::min(p.nitems, sms * occ));
  return launch_pdl(kern, dim3(grid), dim3(S::kThreads), S::kSmem, st, tk, p);
}

}  // namespace

int truth_chunk_blocks() { return kChunk; }

cudaError_t launch_gate_truth(const CUtensorMap& tk, const TruthParams& p, int D, int BLK, int sms, cudaStream_t s) {
  if (D == 64 && BLK == 64) return launch_t<64, 64>(tk, p, sms, s);
  if (D == 64 && BLK == 128) return launch_t<64, 128>(tk, p, sms, s);
  if (D == 128 && BLK == 64) return launch_t<128, 64>(tk, p, sms, s);
  if (D == 128 && BLK == 128) return launch_t<128, 128>(tk, p, sms, s);
  return cudaErrorInvalidValue;
}

}  // namespace seer
