// The prefill forward with block targets on the 5th-generation tensor cores
// (tcgen05 / TMEM): causal attention over whole sequences, each query row's
// maximum pre-softmax score per key block kept on the way, and from those the
// block-level target of every position.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 3 (the target of query i: its softmax row,
// 1-D max-pooled over each block's columns, max over the GQA group's heads,
// normalised to sum to 1) and Knowl 4 (the extraction inside the attention
// forward: per key tile each row's maximum pre-softmax score r is stored; once
// the row's final maximum m and normaliser l are known, the block's score is
// exp(r - m) / l).  Same results as prefill_gt.cu (the warp-level mma form,
// kept for the shapes this kernel does not take: head_dim 64, groups that do
// not divide 128 rows).
//
// Work item: 128 query rows of one kv head of one sequence (the g heads of the
// group x 128/g consecutive positions, row r = head (r / P) at position
// p0 + (r % P)).  One persistent CTA per SM takes items in rounds, heaviest
// (latest positions) first, alternating direction each round; the pipelines
// below run on across items (the next item's Q is staged while the current
// item's last P.V runs, and its first P.V waits until the previous O has been
// read out of TMEM).  Key tiles of 128 keys (one or two blocks).
//   warp 0 and the last warp: producers, K tiles (three-stage ring, a stage
//              freed once S has read it) and V tiles (two stages, freed once
//              P.V has read them) by TMA (128-byte swizzle, boxes of 64
//              channels x b keys)
//   warp 1     allocates TMEM; one lane issues the MMAs: S_u = Q K_u^T into
//              TMEM buffer u % 3 (M = 128 rows, N = 128 keys, K = d; both
//              operands in shared memory) three tiles ahead -- S_{u+3} as soon
//              as the P.V of tile u has read that buffer -- and O += P_u V_u
//              into TMEM O (N = d, K = 128 keys; P read from TMEM, V from shared
//              memory), each group closed by a commit to an mbarrier
//   warps 2 .. 1 + 4 kNP: kNP threads per row (the row's TMEM lane; one
//              thread per 128 / kNP keys of the tile, the kNP exchanging their
//              maxima through shared memory): S by tcgen05.ld, causal mask, the
//              row maximum of each block (stored for the targets),
//              P = exp2(s - m_ref) as bf16 pairs by tcgen05.st over the first
//              64 columns of S_u's own buffer (both parts have read it: the
//              pair barrier), so tile u's exponentials overlap the P.V of
//              tile u - 1 and no P buffer is waited for,
//              V rows past the sequence zeroed (the cache may hold NaN there),
//              at the end O / l, the LSE and the row's log2 normaliser m + log2 l
// TMEM columns: S/P buffers 0-127, 128-255, 256-383; O 384-511.
// A second kernel (prefill_targets_kernel, launched behind it) forms the targets from the stored
// block maxima and normalisers: bandwidth-bound work that would otherwise hold each CTA's tensor
// cores idle at its end.
// The reference maximum m_ref moves only when a tile's maximum exceeds it by
// more than 8 (log2 units), so P stays <= 2^8 and O in TMEM is rescaled (ld,
// scale, st; after the P.V of the previous tile has landed) only then; l and
// the LSE use the same reference, so the results are those of the exact online
// softmax (l sums the probabilities before their rounding to bf16 for the P.V
// product).  All waits are bounded.
#include <algorithm>

#include "seer_device.cuh"
#include "seer_internal.h"

namespace seer {
namespace {

constexpr float kLn2f = 0.6931471805599453f;
constexpr int kD = 128;                 // head_dim of this kernel
constexpr int kM = 128;                 // query rows per CTA
constexpr int kKT = 128;                // keys per tile
constexpr int kBoxB = kM * 128;         // bytes of a 128-row x 64-channel (or 64-key) 128B-swizzled box
constexpr int kTileB = 2 * kBoxB;       // 32 KB: a K, V or Q tile (two boxes)
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kNP = 2;                  // softmax threads per row (each a 128 / kNP-key part of the tile)
constexpr int kSW = 4 * kNP;            // softmax warps (kNP per TMEM lane quarter)
constexpr int kVWarp = 2 + kSW;         // the V producer (after the softmax warps)
constexpr int kThreads = (kSW + 3) * 32;
constexpr int kSB = 3;                  // S / P buffers in TMEM (S_u and then P_u in buffer u % 3)
constexpr uint32_t kTmemCols = 512;     // buffers 0..127, 128..255, 256..383 (P in a buffer's first 64), O 384..511
constexpr float kLazy = 8.f;            // m_ref moves when a tile maximum exceeds it by more than this
constexpr size_t kSmem = 1024 + kTileB /* Q */ + (size_t)(kKStages + kVStages) * kTileB /* K, V */ +
                         256 /* barriers */ + 2 * kNP * kM * 4 /* the parts' tile maxima, two tiles */ +
                         kNP * kM * 4 /* each part's l */;

static_assert(kSmem <= 227 * 1024, "dynamic shared memory above the per-CTA limit");

// shared-memory matrix descriptors (sm_100 layout): start >> 4 in [0,14), leading byte offset
// >> 4 in [16,30), stride byte offset >> 4 in [32,46), version 1 at bit 46, 128-byte swizzle (2)
// in [61,64).  K-major operand in 128B-swizzled rows: stride offset = 8 rows (1024 B), leading
// offset unused.  MN-major operand (V as B of P.V, keys along K): leading offset = the next 64
// channels (one box), stride offset = the next 8 keys (1024 B).
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// kind::f16 instruction descriptor: D f32 (bits 4-5 = 1), A and B bf16 (7-9 = 1, 10-12 = 1),
// B major bit 16 (1 = MN-major), N / 8 in [17,23), M / 16 in [24,29)
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(acc));
}
// the same with A (M rows x 16 K elements, two bf16 per 32-bit column, the lower K index in the low
// half) read from tensor memory at `tmem_a`
__device__ __forceinline__ void umma_f16_ta(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc,
                                            uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(db), "r"(idesc), "r"(acc));
}
// arrive on `bar` once every MMA this thread issued so far has completed
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}
[[maybe_unused]] __device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31]));
}
// (used when kNP = 4: a part of 32 keys is 16 packed columns)
[[maybe_unused]] __device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])),
      "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])),
      "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31])));
}
// 2^x on the SFU (denormal results flushed to zero: a probability that small is zero in the sums)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// TMA coordinates 1..3 of (token t, head h, sequence bp): perm[k] is the dimension (0..2 for
// coordinates 1..3) that holds token / head / sequence (selects, not a runtime-indexed array)
__device__ __forceinline__ void kv_coords(const int32_t perm[3], int t, int h, int bp, int& c1, int& c2, int& c3) {
  auto at = [&](int d) { return perm[0] == d ? t : (perm[1] == d ? h : bp); };
  c1 = at(0);
  c2 = at(1);
  c3 = at(2);
}

// The work items (128 query rows of one KV head of one sequence: the group's g heads x 128 / g
// positions), heaviest (latest positions) first.
struct TcItem {
  int b, hk, p0, L, nt;
};

// Item `it` of the order (position tiles from the last, then KV head, then sequence); nt = 0 when
// none of its positions exists.
__device__ __forceinline__ TcItem tc_item(const PrefillParams& p, int P, int npt, int it) {
  TcItem w;
  const int per = p.Hkv * p.B, pr = it / per, rem = it - pr * per;
  w.hk = rem % p.Hkv;
  w.b = rem / p.Hkv;
  w.p0 = (npt - 1 - pr) * P;
  w.L = min(max(p.seqlens[w.b], 0), min(p.T, p.kcap));
  w.nt = w.p0 < w.L ? (min(w.p0 + P, w.L) - 1) / kKT + 1 : 0;
  return w;
}

// Round r of CTA c: item r * G + c on even rounds, r * G + (G - 1 - c) on odd ones, so that each
// CTA's items alternate between the heavy and the light end of a round.
__device__ __forceinline__ int tc_item_index(int r) {
  const int G = (int)gridDim.x, c = (int)blockIdx.x;
  return r * G + ((r & 1) ? G - 1 - c : c);
}

template <int BLK>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ PrefillParams p) {
  constexpr int NBT = kKT / BLK;   // blocks per key tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* qs = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kring = qs + kTileB;                        // [kKStages] K tiles
  uint8_t* vring = kring + (size_t)kKStages * kTileB;  // [kVStages] V tiles
  uint64_t* k_full = reinterpret_cast<uint64_t*>(vring + (size_t)kVStages * kTileB);
  uint64_t* k_empty = k_full + kKStages;
  uint64_t* v_full = k_empty + kKStages;
  uint64_t* v_empty = v_full + kVStages;
  uint64_t* s_full = v_empty + kVStages;   // [kSB] S_u in buffer u % kSB
  uint64_t* p_full = s_full + kSB;   // [kSB] P_u written over S_u
  uint64_t* p_free = p_full + kSB;   // [kSB] one completion per P.V (the buffer may take S_{u+kSB})
  uint64_t* o_fin = p_free + kSB;    // an item's last P.V done (one completion per item)
  uint64_t* o_drain = o_fin + 1;     // an item's O read out of TMEM (one completion per item)
  uint64_t* q_ready = o_drain + 1;   // an item's Q tile in shared memory (one completion per item)
  uint64_t* drain = q_ready + 1;
  uint64_t* pbar = drain + 1;        // [4] the kNP warps of each TMEM lane quarter
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pbar + 4);
  volatile int* sh = reinterpret_cast<volatile int*>(tmem_slot + 1);   // [0] abort
  float* xch = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(k_full) + 256);   // [tile & 1][part][row]
  float* lh = xch + 2 * kNP * kM;                                                    // [part][row] l

  const int g = p.g, P = kM / g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int npt = (p.T + P - 1) / P;               // position tiles per (KV head, sequence)
  const int n_items = npt * p.Hkv * p.B;
  const int rounds = (n_items + (int)gridDim.x - 1) / (int)gridDim.x;

  if (tid == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int k = 0; k < kSB; ++k) {
      mbar_init(&s_full[k], 1);
      mbar_init(&p_full[k], kSW);
      mbar_init(&p_free[k], 1);
    }
    for (int k = 0; k < 4; ++k) mbar_init(&pbar[k], kNP);
    mbar_init(o_fin, 1);
    mbar_init(o_drain, kSW);
    mbar_init(q_ready, kSW);
    mbar_init(drain, 1);
    sh[0] = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S[k] at 128 k, O at 256, P[k] at 384 + 64 k (computed, not indexed: a runtime index into
  // a local array would put it in local memory)
  const uint32_t tO = tmem + 384;
  auto tS = [tmem](uint32_t k) { return tmem + 128u * k; };   // buffer k: S, then P in its first 64 columns
  auto tP = [tmem](uint32_t k) { return tmem + 128u * k; };
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0 && tid == 0)
    for (int bb = 0; bb < p.B; ++bb)
      if (p.seqlens[bb] > min(p.T, p.kcap)) report(p.err, SEER_DEVERR_COUNT);

  if (warp == 0 || warp == kVWarp) {
    // ---------------------------------------------------------------- producers (K: warp 0, V: the last)
    const bool isK = warp == 0;
    const int NS = isK ? kKStages : kVStages;
    uint64_t* full = isK ? k_full : v_full;
    uint64_t* empty = isK ? k_empty : v_empty;
    uint8_t* ringb = isK ? kring : vring;
    const CUtensorMap* tm = isK ? &tmK : &tmV;
    const int32_t* perm = isK ? p.k_perm : p.v_perm;
    if (lane == 0) {
      uint32_t u = 0;   // tiles issued (over every item of this CTA)
      for (int r = 0; r < rounds && !sh[0]; ++r) {
        const int it = tc_item_index(r);
        if (it >= n_items) continue;
        const TcItem w = tc_item(p, P, npt, it);
        for (int n = 0; n < w.nt; ++n, ++u) {
          const uint32_t s = u % NS;
          if (u >= (uint32_t)NS && !mbar_wait(&empty[s], ((u / NS) - 1) & 1)) {
            report(p.err, SEER_DEVERR_TIMEOUT);
            sh[0] = 1;
          }
          if (sh[0]) break;
          mbar_arrive_expect_tx(&full[s], (uint32_t)kTileB);
          uint8_t* dst = ringb + (size_t)s * kTileB;
#pragma unroll
          for (int sub = 0; sub < NBT; ++sub) {
            // a 64-channel box of BLK keys; the tile's two channel halves are kBoxB apart, its blocks
            // BLK rows (BLK * 128 bytes) apart within a half
            int c1, c2, c3;
            kv_coords(perm, n * kKT + sub * BLK, w.hk, w.b, c1, c2, c3);
#pragma unroll
            for (int hx = 0; hx < 2; ++hx)
              tma_load_4d(dst + hx * kBoxB + sub * BLK * 128, tm, &full[s], hx * 64, c1, c2, c3);
          }
        }
      }
      // copies still landing when a consumer gave up: wait for them (bounded) before shared memory
      // is released; no later phase is ever armed on those stages
      for (uint32_t m = u > (uint32_t)NS ? u - NS : 0; m < u; ++m) mbar_wait(&full[m % NS], (m / NS) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16(kM, kKT, 0), id_o = idesc_bf16(kM, kD, 1);
      const uint32_t qa = smem_u32(qs);
      bool ok = true;
      uint32_t u0 = 0;   // tiles of the earlier items
      int items = 0;     // items started before this one
      // O += P_m V_m (m counts tiles over every item); the item's first P.V overwrites O, once the
      // previous item's O has been read out
      auto issue_pv = [&](uint32_t m, bool first) {
        const uint32_t sv = m % kVStages, pb = m % kSB;
        ok = ok && mbar_wait(&p_full[pb], (m / kSB) & 1) && mbar_wait(&v_full[sv], (m / kVStages) & 1);
        if (first && items > 0) ok = ok && mbar_wait(o_drain, (items - 1) & 1);
        if (!ok) return;
        tc_fence_after();
        const uint32_t vb = smem_u32(vring + (size_t)sv * kTileB);
#pragma unroll
        for (int kk = 0; kk < kKT / 16; ++kk)
          umma_f16_ta(tO, tP(pb) + kk * 8, desc_mnmajor(vb + kk * 2048, kBoxB), id_o, (!first || kk > 0) ? 1u : 0u);
        umma_commit(&v_empty[sv]);
        umma_commit(&p_free[pb]);
      };
      // S_u = Q K_u^T into buffer u % kSB, once K_u has landed and P_{u-kSB} (in that buffer) has
      // been consumed by its P.V
      auto issue_s = [&](uint32_t u) {
        const uint32_t sk = u % kKStages, k2 = u % kSB;
        ok = ok && mbar_wait(&k_full[sk], (u / kKStages) & 1);
        ok = ok && (u < (uint32_t)kSB || mbar_wait(&p_free[k2], ((u / kSB) - 1) & 1));
        if (!ok) return;
        tc_fence_after();
        const uint32_t kb = smem_u32(kring + (size_t)sk * kTileB);
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks)
          umma_f16(tS(k2), desc_kmajor(qa + (ks >> 2) * kBoxB + (ks & 3) * 32),
                   desc_kmajor(kb + (ks >> 2) * kBoxB + (ks & 3) * 32), id_s, ks > 0 ? 1u : 0u);
        umma_commit(&k_empty[sk]);
        umma_commit(&s_full[k2]);
      };
      // Issue order within an item: S_0 .. S_{kSB-1}, then for each tile n: P_n V_n and S_{n+kSB}
      // (into P_n's buffer once that P.V has read it).  S thus runs kSB tiles ahead of the softmax.
      for (int r = 0; r < rounds && ok; ++r) {
        const int it = tc_item_index(r);
        if (it >= n_items) continue;
        const TcItem w = tc_item(p, P, npt, it);
        if (w.nt == 0) continue;
        ok = mbar_wait(q_ready, items & 1);
        for (int n = 0; n < w.nt && n < kSB; ++n) issue_s(u0 + n);
        for (int n = 0; n < w.nt && ok; ++n) {
          issue_pv(u0 + n, n == 0);
          if (n + kSB < w.nt) issue_s(u0 + n + kSB);
        }
        if (ok) umma_commit(o_fin);
        u0 += w.nt;
        ++items;
      }
      if (!ok) {
        report(p.err, SEER_DEVERR_TIMEOUT);
        sh[0] = 1;
      }
      // every MMA issued so far retires before TMEM is released (bounded)
      umma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else {
    // ---------------------------------------------------------------- softmax warps (kNP per row)
    constexpr int HK = kKT / kNP;             // keys per thread (a part of the tile)
    constexpr int CP = kD / kNP;              // O channels per thread
    const int quarter = warp & 3;             // warp w reads TMEM lanes 32(w % 4) .. 32(w % 4) + 31
    const int part = (warp - 2) >> 2;         // warps 2-5: keys 0..HK-1 of each tile, warps 6-9 the next HK, ...
    const int row = 32 * quarter + lane;
    const int j = row / P, t = row - (row / P) * P;   // the row's head in the group and position offset
    const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
    const int st = tid - 64;                  // 0 .. 32 kSW - 1 over the softmax warps
    const float sl2 = p.scale_log2;
    uint32_t pph = 0;                         // the quarter barrier's phase
    // this thread's CP channels of an item's Q row (in the 128B-swizzled box of its 64 channels) ->
    // shared memory, zero past L; then the item's Q is announced
    auto load_q = [&](const TcItem& w) {
      const int i = w.p0 + t;
      const size_t qrow = ((size_t)w.b * p.Hq + (size_t)w.hk * g + j) * p.T;
#pragma unroll
      for (int c = 0; c < CP / 8; ++c) {
        const int ch = part * CP + c * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (i < w.L) v = *reinterpret_cast<const uint4*>(p.q + (qrow + i) * kD + ch);
        *reinterpret_cast<uint4*>(qs + (ch >> 6) * kBoxB + sw128(row, (ch & 63) >> 3)) = v;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    };
    // the next round (from r on) with an item that has work
    auto next_round = [&](int r) {
      for (; r < rounds; ++r) {
        const int it = tc_item_index(r);
        if (it < n_items && tc_item(p, P, npt, it).nt > 0) return r;
      }
      return rounds;
    };
    bool ok = true;
    uint32_t u0 = 0;   // tiles of the earlier items
    int items = 0;
    int r = next_round(0);
    if (r < rounds) load_q(tc_item(p, P, npt, tc_item_index(r)));
    while (r < rounds && ok) {
      const TcItem w = tc_item(p, P, npt, tc_item_index(r));
      const int L = w.L, h = w.hk * g + j, i = w.p0 + t;   // query head and position of the row
      const bool live = i < L;
      const int vis = min(i, L - 1);            // last key the row sees
      const size_t qrow = ((size_t)w.b * p.Hq + h) * p.T;
      float* rws = p.rmax + ((size_t)w.b * p.Hq + h) * p.NB * p.T;
      float m_ref = -INFINITY, l = 0.f;
      for (int n = 0; n < w.nt && ok; ++n) {
        const uint32_t u = u0 + n, k2 = u % kSB, sv = u % kVStages;
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[k2], (u / kSB) & 1));
        if (!ok) break;
        tc_fence_after();
        float x[HK];
#pragma unroll
        for (int c0 = 0; c0 < HK; c0 += 32) tmem_ld32(tS(k2) + lane_base + part * HK + c0, x + c0);
        tmem_wait_ld();
        // causal mask (key kt visible to row i iff kt <= min(i, L - 1)) where the tile needs one; the
        // maximum of this part (raw scores: the scale is positive)
        const int k0 = n * kKT + part * HK;     // first key of this part
        if (k0 + HK - 1 > vis) {
#pragma unroll
          for (int c = 0; c < HK; ++c) x[c] = (k0 + c <= vis) ? x[c] : -INFINITY;
        }
        // (eight independent running maxima: a single chain would be HK dependent max operations)
        float m8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) m8[e] = x[e];
#pragma unroll
        for (int c = 8; c < HK; c += 8)
#pragma unroll
          for (int e = 0; e < 8; ++e) m8[e] = fmaxf(m8[e], x[c + e]);
        float hm = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        hm *= sl2;   // log2 domain
        // the parts' maxima (double-buffered by tile parity: every part has read tile u - 2's values
        // before it arrived at tile u - 1's barrier)
        // (the pair barrier also orders this thread's completed S reads before the partner's P writes
        // over the same buffer)
        xch[((u & 1) * kNP + part) * kM + row] = hm;
        tc_fence_before();
        if (!warps_sync(&pbar[quarter], pph)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float pm[kNP];
#pragma unroll
        for (int q = 0; q < kNP; ++q) pm[q] = xch[((u & 1) * kNP + q) * kM + row];
        float mx = pm[0];
#pragma unroll
        for (int q = 1; q < kNP; ++q) mx = fmaxf(mx, pm[q]);
        // the row maximum of each block (PPB parts), written by the block's first part
        constexpr int PPB = BLK / HK;
#pragma unroll
        for (int sub = 0; sub < NBT; ++sub) {
          if (part != sub * PPB) continue;
          float bm = pm[sub * PPB];
#pragma unroll
          for (int q = 1; q < PPB; ++q) bm = fmaxf(bm, pm[sub * PPB + q]);
          const int blk = n * NBT + sub;
          if (live && blk * BLK <= i) rws[(size_t)blk * p.T + i] = bm;
        }
        // reference maximum: the item's first tile's, moved only when a tile exceeds it by more than
        // kLazy; then O (in TMEM, holding the item's tiles before this one) and l are rescaled
        float alpha = 1.f;
        bool move = false;
        if (n == 0) {
          m_ref = mx;
        } else if (mx > m_ref + kLazy) {
          alpha = ex2(m_ref - mx);
          m_ref = mx;
          move = true;
        }
        l *= alpha;
        // P_u goes over S_u in the same buffer (read by both parts: the pair barrier above).  A rescale
        // of O waits for the P.V of tile u - 1 (O then holds the item's earlier tiles and nothing
        // adds to it; that buffer's next completion needs P_{u-1+kSB}, not yet written, so a parity
        // wait is exact).
        const uint32_t pb = k2;
        if (__any_sync(0xffffffffu, move)) {
          ok = __all_sync(0xffffffffu, mbar_wait(&p_free[(u - 1) % kSB], ((u - 1) / kSB) & 1));
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < CP; c0 += 32) {
            float o[32];
            tmem_ld32(tO + lane_base + part * CP + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(tO + lane_base + part * CP + c0, o);
          }
          tmem_wait_st();
          tc_fence_before();
        }
        // P = exp2(s * scale - m_ref) (<= 2^kLazy; masked keys give 0) as bf16 pairs into this part's
        // HK / 2 columns of P[u % 2] in TMEM; l sums the same values
        const float mu = m_ref == -INFINITY ? 0.f : m_ref;
        {
          uint32_t pw[HK / 2];
          float s8[8];   // independent partial sums (one chain would be HK dependent adds)
#pragma unroll
          for (int e = 0; e < 8; ++e) s8[e] = 0.f;
#pragma unroll
          for (int e = 0; e < HK / 2; ++e) {
            const float a = ex2(fmaf(x[2 * e], sl2, -mu)), bb = ex2(fmaf(x[2 * e + 1], sl2, -mu));
            s8[e & 7] += a + bb;
            pw[e] = pack_bf16(a, bb);
          }
          if constexpr (HK == 64) tmem_st32u(tP(pb) + lane_base + part * (HK / 2), pw);
          else tmem_st16u(tP(pb) + lane_base + part * (HK / 2), pw);
          l += ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
        }
        if (n * kKT + kKT > L) {
          // V rows past L may hold anything (even NaN): zero them so that P = 0 there gives 0.  Wait for
          // the tile's copy here too (its phase is at most one behind, as for the MMA issuer); whole
          // 128-byte rows, so the swizzle does not matter.
          ok = __all_sync(0xffffffffu, mbar_wait(&v_full[sv], (u / kVStages) & 1));
          if (!ok) break;
          uint8_t* vt = vring + (size_t)sv * kTileB;
          const int r0 = max(0, L - n * kKT), nchunk = (kKT - r0) * 8;   // 16-byte chunks per channel half
          for (int e = st; e < 2 * nchunk; e += kSW * 32) {
            const int hx = e / nchunk, rr = r0 + (e - hx * nchunk) / 8, cc = e & 7;
            *reinterpret_cast<uint4*>(vt + hx * kBoxB + rr * 128 + cc * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[pb]);
      }
      if (!ok) break;
      // the next item's Q: every S of this item has completed (this thread saw the last one's
      // commit, which covers every earlier MMA), so the Q tile is free
      const int rn = next_round(r + 1);
      if (rn < rounds) load_q(tc_item(p, P, npt, tc_item_index(rn)));
      // this item's last P.V (one o_fin completion per item; the next needs this item's O read out)
      ok = __all_sync(0xffffffffu, mbar_wait(o_fin, items & 1));
      if (ok) {
        lh[part * kM + row] = l;
        ok = warps_sync(&pbar[quarter], pph);
      }
      if (!ok) break;
      float lt = 0.f;   // the row's l (all parts; one reference maximum)
#pragma unroll
      for (int q = 0; q < kNP; ++q) lt += lh[q * kM + row];
      tc_fence_after();
      float o[CP];
#pragma unroll
      for (int c0 = 0; c0 < CP; c0 += 32) tmem_ld32(tO + lane_base + part * CP + c0, o + c0);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_drain);   // O may be overwritten by the next item
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      if (live) {
#pragma unroll
        for (int e = 0; e < CP; e += 8) {
          uint4 v;
          v.x = pack_bf16(o[e] * inv, o[e + 1] * inv);
          v.y = pack_bf16(o[e + 2] * inv, o[e + 3] * inv);
          v.z = pack_bf16(o[e + 4] * inv, o[e + 5] * inv);
          v.w = pack_bf16(o[e + 6] * inv, o[e + 7] * inv);
          *reinterpret_cast<uint4*>(p.o + (qrow + i) * kD + part * CP + e) = v;
        }
        if (part == 0) {
          const float c = lt > 0.f ? m_ref + log2f(lt) : -INFINITY;   // log2 of the row's normaliser
          if (p.lse) p.lse[qrow + i] = c * kLn2f;
          p.rnorm[qrow + i] = c;
        }
      }
      u0 += w.nt;
      ++items;
      r = rn;
    }
    if (!ok) {
      if (lane == 0) report(p.err, SEER_DEVERR_TIMEOUT);
      sh[0] = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

// ---------------------------------------------------------------- the targets
// One CTA per (32 positions, kv head, sequence), 8 warps; lane t is position i0 + t while the
// scores are formed (the row maxima are position-contiguous per (head, block): 128-byte loads),
// and the block index while the rows are written (block-contiguous per position: 128-byte
// stores).  Score of block n for position i: max over the group's G heads j of exp2(r_j - c_j)
// (c = m + log2 l, the row's final log2 normaliser), for the blocks holding a key at or before i,
// normalised to sum to 1; 0 for the other blocks.  A thread keeps kTgU blocks x G heads (up to
// 32) of loads in flight (the maxima come from DRAM: the workspace is larger than L2).  Blocks are taken
// kTgChunk at a time through shared memory; with more blocks than one chunk the sum is a first
// pass of its own and each chunk's scores are formed again (from L2: the CTA's maxima are a few
// hundred KB at most).
constexpr int kTgPos = 32;
constexpr int kTgWarps = 8;
constexpr int kTgChunk = 256;

template <int BLK, int G>
__global__ void __launch_bounds__(kTgWarps * 32, 3)
    prefill_targets_kernel(const __grid_constant__ PrefillParams p) {
  constexpr int kTgU = G >= 8 ? 4 : 8;   // blocks per batch of loads (kTgU x G loads in flight per thread)
  __shared__ float vals[kTgChunk][kTgPos + 1];
  __shared__ float psum[kTgWarps][kTgPos];
  __shared__ float inv_s[kTgPos];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, hk = blockIdx.y, i0 = blockIdx.x * kTgPos;
  pdl_wait();   // the forward's row maxima and normalisers are complete
  pdl_trigger();
  const int L = min(max(p.seqlens[b], 0), min(p.T, p.kcap));
  if (i0 >= L) return;
  const int i = i0 + lane;
  const bool live = i < L;
  const int nb_i = live ? i / BLK + 1 : 0;                 // blocks with a key visible to position i
  const int nb_max = (min(i0 + kTgPos, L) - 1) / BLK + 1;  // the largest nb_i of the CTA
  const float* r_b = p.rmax + ((size_t)b * p.Hq + (size_t)hk * G) * p.NB * p.T + i;
  const size_t hstride = (size_t)p.NB * p.T;
  float c[G];
#pragma unroll
  for (int j = 0; j < G; ++j) c[j] = live ? __ldg(p.rnorm + ((size_t)b * p.Hq + (size_t)hk * G + j) * p.T + i) : 0.f;
  // scores of blocks n0 + kTgWarps * u (u < kTgU), every load issued before any use (one 64-bit
  // offset per block; the heads' offsets are fixed multiples of the head stride)
  auto scores = [&](int n0, float (&v)[kTgU]) {
    float r[kTgU][G];
#pragma unroll
    for (int u = 0; u < kTgU; ++u) {
      const int n = n0 + kTgWarps * u;
      const bool in = n < nb_i;
      const float* rn = r_b + (size_t)n * p.T;
#pragma unroll
      for (int j = 0; j < G; ++j) r[u][j] = in ? __ldcg(rn + j * hstride) : -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < kTgU; ++u) {
      float m = 0.f;
#pragma unroll
      for (int j = 0; j < G; ++j) m = fmaxf(m, ex2(r[u][j] - c[j]));   // masked blocks: ex2(-inf) = 0
      v[u] = m;
    }
  };
  // chunk [n_lo, n_hi): scores into vals (and into the sum when `add`)
  auto fill = [&](int n_lo, int n_hi, bool add, float& part) {
    for (int n0 = n_lo + warp; n0 < n_hi; n0 += kTgU * kTgWarps) {
      float v[kTgU];
      scores(n0, v);
#pragma unroll
      for (int u = 0; u < kTgU; ++u) {
        const int n = n0 + kTgWarps * u;
        if (n < n_hi) {
          vals[n - n_lo][lane] = v[u];
          if (add) part += v[u];
        }
      }
    }
  };
  const bool one = nb_max <= kTgChunk;
  float part = 0.f;
  if (one) {
    fill(0, nb_max, true, part);
  } else {
    for (int n0 = warp; n0 < nb_max; n0 += kTgU * kTgWarps) {
      float v[kTgU];
      scores(n0, v);
#pragma unroll
      for (int u = 0; u < kTgU; ++u) part += v[u];   // blocks past nb_i score 0
    }
  }
  psum[warp][lane] = part;
  __syncthreads();
  if (warp == 0) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kTgWarps; ++w) sum += psum[w][lane];
    inv_s[lane] = sum > 0.f ? 1.f / sum : 0.f;
  }
  __syncthreads();
  float* gt_b = p.gt + ((size_t)b * p.Hkv + hk) * p.T * p.NB;
  const int npos = min(kTgPos, L - i0);
  for (int n_lo = 0; n_lo < p.NB; n_lo += kTgChunk) {
    const int n_hi = min(p.NB, n_lo + kTgChunk);
    if (!one && n_lo < nb_max) {
      float unused = 0.f;
      fill(n_lo, min(n_hi, nb_max), false, unused);
      __syncthreads();
    }
    for (int t = warp; t < npos; t += kTgWarps) {
      const int nb_t = (i0 + t) / BLK + 1;
      const float inv = inv_s[t];
      float* row = gt_b + (size_t)(i0 + t) * p.NB;
      for (int n = n_lo + lane; n < n_hi; n += 32) __stcs(row + n, n < nb_t ? vals[n - n_lo][t] * inv : 0.f);
    }
    if (!one) __syncthreads();   // vals is refilled for the next chunk
  }
}

template <int BLK>
cudaError_t launch_targets(const PrefillParams& p, int max_len, cudaStream_t st) {
  const dim3 tgrid((max_len + kTgPos - 1) / kTgPos, p.Hkv, p.B);
  const dim3 blk(kTgWarps * 32);
  switch (p.g) {
    case 1: return launch_pdl(prefill_targets_kernel<BLK, 1>, tgrid, blk, 0, st, p);
    case 2: return launch_pdl(prefill_targets_kernel<BLK, 2>, tgrid, blk, 0, st, p);
    case 4: return launch_pdl(prefill_targets_kernel<BLK, 4>, tgrid, blk, 0, st, p);
    default: return launch_pdl(prefill_targets_kernel<BLK, 8>, tgrid, blk, 0, st, p);
  }
}

template <int BLK>
cudaError_t launch_tc_t(const CUtensorMap& tk, const CUtensorMap& tv, const PrefillParams& p, int max_len,
                        int sms, cudaStream_t st) {
  auto kern = prefill_tc_kernel<BLK>;
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = ensure_smem_limit(kern, (int)kSmem, attr_done);
  if (e != cudaSuccess) return e;
  const int P = kM / p.g;
  const long long items = (long long)((max_len + P - 1) / P) * p.Hkv * p.B;
  const dim3 grid((unsigned)std::min<long long>(items, std::max(sms, 1)));
  e = launch_pdl(kern, grid, dim3(kThreads), kSmem, st, tk, tv, p);
  if (e != cudaSuccess) return e;
  return launch_targets<BLK>(p, max_len, st);
}

}  // namespace

bool prefill_tc_supported(int D, int BLK, int g) {
  return D == kD && (BLK == 64 || BLK == 128) && (g == 1 || g == 2 || g == 4 || g == 8);
}

cudaError_t launch_prefill_tc(const CUtensorMap& tk, const CUtensorMap& tv, const PrefillParams& p, int D, int BLK,
                              int max_len, int sms, cudaStream_t s) {
  if (!prefill_tc_supported(D, BLK, p.g)) return cudaErrorInvalidValue;
  return BLK == 64 ? launch_tc_t<64>(tk, tv, p, max_len, sms, s) : launch_tc_t<128>(tk, tv, p, max_len, sms, s);
}

}  // namespace seer
