// Gate logits -> ascending lists of active blocks.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 5: a token budget B becomes k = ceil(B/b)
// blocks chosen by top-k on the un-softmaxed logits; or every block whose
// score S = softmax(logits) exceeds tau; the incomplete last block is always
// active.  Knowl 14 names nucleus (top-p) selection as the adaptive
// alternative: the fewest blocks whose S-mass reaches p.
//
// One CTA per (b, h); the row (<= 8192 logits) lives in shared memory as
// order-preserving uint32 keys.  Top-k finds the k-th largest key with a
// 4-pass 8-bit radix select (no sort), then keeps every key above it plus the
// lowest-index ties; top-p sorts (key, index) pairs with a bitonic network and
// walks the prefix mass in fp64; threshold evaluates S in fp64.  All modes
// end with an index-order compaction (block-wide scan), which yields ascending
// output and the lower-index tie rule.
#include "seer_device.cuh"
#include "seer_internal.h"

namespace seer {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.f) f = 0.f;  // -0 and +0 tie
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Block-wide exclusive scan of one int per thread; returns the prefix, *total = sum.
__device__ int block_excl_scan(int v, int* ws, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) ws[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kWarps ? ws[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += y;
    }
    if (lane < kWarps) ws[32 + lane] = w;   // inclusive warp prefix
  }
  __syncthreads();
  const int before = warp ? ws[32 + warp - 1] : 0;
  *total = ws[32 + kWarps - 1];
  __syncthreads();
  return before + x - v;
}

template <typename T>
__device__ T block_reduce(T v, T* ws, bool is_max) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const T y = __shfl_xor_sync(0xffffffffu, v, off);
    v = is_max ? (y > v ? y : v) : v + y;
  }
  if (lane == 0) ws[warp] = v;
  __syncthreads();
  if (warp == 0) {
    T w = lane < kWarps ? ws[lane] : (is_max ? ws[0] : T(0));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const T y = __shfl_xor_sync(0xffffffffu, w, off);
      w = is_max ? (y > w ? y : w) : w + y;
    }
    if (lane == 0) ws[0] = w;
  }
  __syncthreads();
  const T r = ws[0];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kThreads) select_kernel(const SelectParams p) {
  extern __shared__ uint32_t keys[];       // [NB] keys; top-p: [2 * pow2] u32 pairs
  __shared__ int ws[64];
  __shared__ double wsd[kWarps];
  __shared__ int hist[256];
  __shared__ int pick[2];                  // digit, remaining

  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x;
  const int L = max(p.seqlens[b], 0);
  const int nfull = min(L / p.BLK, p.NB);
  const bool partial = (L % p.BLK) != 0;
  const float* row = p.logits + ((size_t)b * p.Hkv + h) * p.NB;
  int32_t* out = p.idx + ((size_t)b * p.Hkv + h) * p.cap;

  for (int n = tid; n < nfull; n += kThreads) keys[n] = order_key(row[n]);
  __syncthreads();

  // Selection rule, evaluated per index n during the compaction:
  //   mode 0/2: key > T, or key == T and rank among ties < rem
  //   mode 1:   exp(x_n - m) / sum > tau   (fp64)
  uint32_t T = 0;
  int rem = 0;
  bool all = false;
  double mref = 0.0, ssum = 1.0;

  if (p.mode == 0) {
    const int k = min(p.kblocks, nfull);
    if (k >= nfull) {
      all = true;
    } else if (k > 0) {
      uint32_t prefix = 0, pmask = 0;
      int want = k;  // rank (from the top) of the key being located, within the prefix bucket
      for (int pass = 3; pass >= 0; --pass) {
        const int shift = pass * 8;
        for (int i = tid; i < 256; i += kThreads) hist[i] = 0;
        __syncthreads();
        for (int n = tid; n < nfull; n += kThreads) {
          const uint32_t u = keys[n];
          if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1);
        }
        __syncthreads();
        if (tid < 32) {
          // lane l owns digits 255-8l .. 248-8l (descending); suffix counts from the top
          int c[8], tot = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            c[e] = hist[255 - (8 * tid + e)];
            tot += c[e];
          }
          int incl = tot;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (tid >= off) incl += y;
          }
          int above = incl - tot;  // keys in digits larger than this lane's range
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (above < want && above + c[e] >= want) {
              pick[0] = 255 - (8 * tid + e);
              pick[1] = want - above;
            }
            above += c[e];
          }
        }
        __syncthreads();
        prefix |= (uint32_t)pick[0] << shift;
        pmask |= 255u << shift;
        want = pick[1];
        __syncthreads();
      }
      T = prefix;
      rem = want;  // ties at T to keep, lowest index first
    } else {
      T = 0xffffffffu;
      rem = 0;
    }
  } else if (p.mode == 1) {
    float mx = -INFINITY;
    for (int n = tid; n < nfull; n += kThreads) mx = fmaxf(mx, row[n]);
    mx = block_reduce<float>(mx, reinterpret_cast<float*>(ws), true);
    mref = (double)mx;
    double s = 0.0;
    for (int n = tid; n < nfull; n += kThreads) s += exp((double)row[n] - mref);
    ssum = block_reduce<double>(s, wsd, false);
  } else {
    // top-p: bitonic sort of (key desc, index asc) packed as 64-bit words
    int pw = 1;
    while (pw < nfull) pw <<= 1;
    uint64_t* pr = reinterpret_cast<uint64_t*>(keys + ((p.NB + 1) & ~1));
    for (int i = tid; i < pw; i += kThreads)
      pr[i] = i < nfull ? ((uint64_t)keys[i] << 32) | (uint32_t)(0xffffffffu - (uint32_t)i) : 0ull;
    __syncthreads();
    for (int kk = 2; kk <= pw; kk <<= 1) {
      for (int j = kk >> 1; j > 0; j >>= 1) {
        for (int i = tid; i < pw; i += kThreads) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const bool desc = (i & kk) == 0;
            const uint64_t a = pr[i], c = pr[ixj];
            if (desc ? a < c : a > c) {
              pr[i] = c;
              pr[ixj] = a;
            }
          }
        }
        __syncthreads();
      }
    }
    // scores in sorted order; cutoff = first position whose inclusive mass reaches p
    float mx = nfull > 0 ? key_value((uint32_t)(pr[0] >> 32)) : 0.f;
    mref = (double)mx;
    double s = 0.0;
    for (int n = tid; n < nfull; n += kThreads) s += exp((double)row[n] - mref);
    ssum = block_reduce<double>(s, wsd, false);
    // serial walk by warp 0 in chunks of 32 (prefix in fp64)
    if (tid < 32) {
      double run = 0.0;
      int cut = nfull;
      for (int base = 0; base < nfull && cut == nfull; base += 32) {
        const int i = base + tid;
        double v = 0.0;
        if (i < nfull) {
          const uint32_t idx = 0xffffffffu - (uint32_t)(pr[i] & 0xffffffffu);
          v = exp((double)row[idx] - mref) / ssum;
        }
        double incl = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const double y = __shfl_up_sync(0xffffffffu, incl, off);
          if (tid >= off) incl += y;
        }
        const double before = run + incl - v;   // mass before element i
        const unsigned stop = __ballot_sync(0xffffffffu, i < nfull && before >= p.tau);
        if (stop) cut = base + __ffs(stop) - 1;
        run += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (tid == 0) pick[0] = cut;   // number of blocks taken
    }
    __syncthreads();
    const int take = pick[0];
    // threshold key/ties for the compaction: everything sorted before `take`
    if (take >= nfull) {
      all = true;
    } else if (take == 0) {
      T = 0xffffffffu;
      rem = 0;
    } else {
      const uint64_t last = pr[take - 1];
      T = (uint32_t)(last >> 32);
      // ties at T taken = those sorted before `take` with key T
      int cnt = 0;
      for (int i = tid; i < take; i += kThreads) cnt += ((uint32_t)(pr[i] >> 32) == T);
      rem = block_reduce<int>(cnt, ws, false);
    }
    __syncthreads();
    // restore the keys array (the pairs region does not overlap it)
  }

  // ---------------- index-order compaction
  int running = 0;
  int eq_run = 0;
  for (int base = 0; base < nfull; base += kThreads) {
    const int n = base + tid;
    bool sel = false;
    if (n < nfull) {
      if (all) {
        sel = true;
      } else if (p.mode == 1) {
        sel = exp((double)row[n] - mref) / ssum > p.tau;
      }
    }
    if (p.mode != 1 && !all) {
      const uint32_t u = n < nfull ? keys[n] : 0u;
      const bool eq = n < nfull && u == T;
      int eq_tot;
      const int eq_before = eq_run + block_excl_scan(eq ? 1 : 0, ws, &eq_tot);
      eq_run += eq_tot;
      sel = n < nfull && (u > T || (eq && eq_before < rem));
    }
    int tot;
    const int pos = running + block_excl_scan(sel ? 1 : 0, ws, &tot);
    if (sel && pos < p.cap) out[pos] = n;
    running += tot;
  }
  if (partial) {
    if (tid == 0 && running < p.cap) out[running] = nfull;
    ++running;
  }
  const int total = min(running, p.cap);
  for (int i = total + tid; i < p.cap; i += kThreads) out[i] = -1;
  if (tid == 0) p.cnt[b * p.Hkv + h] = total;
}

}  // namespace

cudaError_t launch_select(const SelectParams& p, cudaStream_t s) {
  size_t smem = (size_t)((p.NB + 1) & ~1) * 4;
  if (p.mode == 2) {
    int pw = 1;
    while (pw < p.NB) pw <<= 1;
    smem += (size_t)pw * 8;
  }
  static std::atomic<uint64_t> attr_done{0};
  constexpr int kMaxSmem = kMaxBlocksRow * 4 + kMaxBlocksRow * 8;   // keys + top-p pairs
  cudaError_t e = ensure_smem_limit(select_kernel, kMaxSmem, attr_done);
  if (e != cudaSuccess) return e;
  dim3 grid(p.Hkv, p.B);
  select_kernel<<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace seer
