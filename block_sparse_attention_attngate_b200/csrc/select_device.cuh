// Block selection of one (b, h) row, as a CTA-wide device routine shared by the
// standalone selection kernel and the fused plan kernel.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (chapterpal.com summary), Knowl 5: a token budget B becomes k = ceil(B/b)
// blocks chosen by top-k on the un-softmaxed logits; or every block whose
// score S = softmax(logits) exceeds tau; the incomplete last block is always
// active.  Knowl 14 names nucleus (top-p) selection as the adaptive
// alternative: the fewest blocks whose S-mass reaches p.
//
// The row is held in shared memory as order-preserving uint32 keys.  Top-k
// finds the k-th largest key with a 4-pass 8-bit radix select (warp-aggregated
// histogram, early exit when a whole bucket is taken), then keeps every key
// above it plus the lowest-index ties; top-p sorts (key, index) pairs with a
// bitonic network and walks the prefix mass in fp64; threshold evaluates S in
// fp64.  All modes end with an index-order compaction (block-wide scans), which
// yields ascending output and the lower-index tie rule.
#pragma once

#include "seer_device.cuh"

namespace seer {

struct SelectScratch {
  int ws[64];
  double wsd[32];
  int hist[256];
  int pick[3];   // digit, remaining rank, bucket size
};

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.f) f = 0.f;  // -0 and +0 tie
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Block-wide exclusive scan of one int per thread; returns the prefix, *total = sum.
template <int NT>
__device__ int block_excl_scan(int v, int* ws, int* total) {
  constexpr int kWarps = NT / 32;
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

template <int NT, typename T>
__device__ T block_reduce(T v, T* ws, bool is_max) {
  constexpr int kWarps = NT / 32;
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

// Select blocks of one row.  All NT threads of the CTA call this.
//   row:   logits of the nfull full blocks (global or shared memory)
//   keys:  shared scratch of >= nfull uint32; pairs: shared scratch of >= pow2(nfull) uint64 (top-p only)
//   out:   the row of the index tensor (capacity entries); returns the count written.
template <int NT>
__device__ int select_row(const float* row, int nfull, bool partial, int mode, int kblocks, double tau,
                          uint32_t* keys, uint64_t* pairs, SelectScratch& sc, int32_t* out, int cap) {
  const int tid = threadIdx.x;
  for (int n = tid; n < nfull; n += NT) keys[n] = order_key(row[n]);
  __syncthreads();

  // Selection rule, evaluated per index n during the compaction:
  //   top-k / top-p: key > T, or key == T and rank among ties < rem
  //   threshold:     exp(x_n - m) / sum > tau   (fp64)
  uint32_t T = 0;
  int rem = 0;
  bool all = false;
  double mref = 0.0, ssum = 1.0;

  if (mode == 0) {
    const int k = min(kblocks, nfull);
    if (k >= nfull) {
      all = true;
    } else if (k > 0) {
      uint32_t prefix = 0, pmask = 0;
      int want = k;  // rank (from the top) of the key being located, within the prefix bucket
      bool whole_bucket = false;
      for (int pass = 3; pass >= 0 && !whole_bucket; --pass) {
        const int shift = pass * 8;
        for (int i = tid; i < 256; i += NT) sc.hist[i] = 0;
        __syncthreads();
        // warp-aggregated histogram: one shared atomic per distinct digit per warp
        for (int base = 0; base < nfull; base += NT) {
          const int n = base + tid;
          const uint32_t u = n < nfull ? keys[n] : 0u;
          const bool in = n < nfull && (u & pmask) == prefix;
          const uint32_t dig = in ? (u >> shift) & 255u : 256u;
          const unsigned same = __match_any_sync(0xffffffffu, dig);
          if (in && (threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(&sc.hist[dig], __popc(same));
        }
        __syncthreads();
        if (tid < 32) {
          // lane l owns digits 255-8l .. 248-8l (descending); counts above come from a lane scan
          int c[8], tot = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            c[e] = sc.hist[255 - (8 * tid + e)];
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
              sc.pick[0] = 255 - (8 * tid + e);
              sc.pick[1] = want - above;
              sc.pick[2] = c[e];
            }
            above += c[e];
          }
        }
        __syncthreads();
        prefix |= (uint32_t)sc.pick[0] << shift;
        pmask |= 255u << shift;
        want = sc.pick[1];
        // every key of the chosen bucket is selected: the bucket's lower bound settles it
        whole_bucket = sc.pick[2] == want && prefix > 0;
        __syncthreads();
      }
      if (whole_bucket) {
        T = prefix - 1;   // keys >= prefix (this bucket and above) are the top k
        rem = 0;
      } else {
        T = prefix;
        rem = want;  // ties at T to keep, lowest index first
      }
    } else {
      T = 0xffffffffu;
      rem = 0;
    }
  } else if (mode == 1) {
    float mx = -INFINITY;
    for (int n = tid; n < nfull; n += NT) mx = fmaxf(mx, row[n]);
    mx = block_reduce<NT, float>(mx, reinterpret_cast<float*>(sc.ws), true);
    mref = (double)mx;
    double s = 0.0;
    for (int n = tid; n < nfull; n += NT) s += exp((double)row[n] - mref);
    ssum = block_reduce<NT, double>(s, sc.wsd, false);
  } else {
    // top-p: bitonic sort of (key desc, index asc) packed as 64-bit words
    int pw = 1;
    while (pw < nfull) pw <<= 1;
    for (int i = tid; i < pw; i += NT)
      pairs[i] = i < nfull ? ((uint64_t)keys[i] << 32) | (uint32_t)(0xffffffffu - (uint32_t)i) : 0ull;
    __syncthreads();
    for (int kk = 2; kk <= pw; kk <<= 1) {
      for (int j = kk >> 1; j > 0; j >>= 1) {
        for (int i = tid; i < pw; i += NT) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const bool desc = (i & kk) == 0;
            const uint64_t a = pairs[i], c = pairs[ixj];
            if (desc ? a < c : a > c) {
              pairs[i] = c;
              pairs[ixj] = a;
            }
          }
        }
        __syncthreads();
      }
    }
    const float mx = nfull > 0 ? key_value((uint32_t)(pairs[0] >> 32)) : 0.f;
    mref = (double)mx;
    double s = 0.0;
    for (int n = tid; n < nfull; n += NT) s += exp((double)row[n] - mref);
    ssum = block_reduce<NT, double>(s, sc.wsd, false);
    // cutoff = first sorted position whose preceding mass reaches p (warp 0, chunks of 32, fp64)
    if (tid < 32) {
      double run = 0.0;
      int cut = nfull;
      for (int base = 0; base < nfull && cut == nfull; base += 32) {
        const int i = base + tid;
        double v = 0.0;
        if (i < nfull) {
          const uint32_t idx = 0xffffffffu - (uint32_t)(pairs[i] & 0xffffffffu);
          v = exp((double)row[idx] - mref) / ssum;
        }
        double incl = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const double y = __shfl_up_sync(0xffffffffu, incl, off);
          if (tid >= off) incl += y;
        }
        const double before = run + incl - v;   // mass before element i
        const unsigned stop = __ballot_sync(0xffffffffu, i < nfull && before >= tau);
        if (stop) cut = base + __ffs(stop) - 1;
        run += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (tid == 0) sc.pick[0] = cut;   // number of blocks taken
    }
    __syncthreads();
    const int take = sc.pick[0];
    if (take >= nfull) {
      all = true;
    } else if (take == 0) {
      T = 0xffffffffu;
      rem = 0;
    } else {
      T = (uint32_t)(pairs[take - 1] >> 32);
      // ties at T taken = those sorted before `take` with key T
      int cnt = 0;
      for (int i = tid; i < take; i += NT) cnt += ((uint32_t)(pairs[i] >> 32) == T);
      rem = block_reduce<NT, int>(cnt, sc.ws, false);
    }
    __syncthreads();
  }

  // ---------------- index-order compaction
  int running = 0;
  int eq_run = 0;
  for (int base = 0; base < nfull; base += NT) {
    const int n = base + tid;
    bool sel = false;
    if (n < nfull) {
      if (all) sel = true;
      else if (mode == 1) sel = exp((double)row[n] - mref) / ssum > tau;
    }
    if (mode != 1 && !all) {
      const uint32_t u = n < nfull ? keys[n] : 0u;
      const bool eq = n < nfull && u == T;
      int eq_tot;
      const int eq_before = eq_run + block_excl_scan<NT>(eq ? 1 : 0, sc.ws, &eq_tot);
      eq_run += eq_tot;
      sel = n < nfull && (u > T || (eq && eq_before < rem));
    }
    int tot;
    const int pos = running + block_excl_scan<NT>(sel ? 1 : 0, sc.ws, &tot);
    if (sel && pos < cap) out[pos] = n;
    running += tot;
  }
  if (partial) {
    if (tid == 0 && running < cap) out[running] = nfull;
    ++running;
  }
  const int total = min(running, cap);
  for (int i = total + tid; i < cap; i += NT) out[i] = -1;
  return total;
}

// ---------------------------------------------------------------- register-resident selection
// Top-k and threshold for rows of at most NT * E blocks, by the whole CTA with
// each thread holding E consecutive indices (n = tid * E + e) as keys in
// registers.  Top-k: 4-pass 8-bit radix select of the k-th largest key T (one
// shared atomic per key of the live bucket, bucket search by warp 0, two
// barriers a pass, early exit when a whole bucket is taken); threshold: max and
// sum of exp in fp64 by block reductions.  One block-wide scan of the packed
// (keys > T, keys == T) counts then places every kept index, so the output is
// ascending and ties at T go to the lowest indices: the same result as
// select_row for these modes.
struct SelectRegsScratch {
  int hist[2][256];
  int ws[64];
  double wsd[32];
  int pick[3];
};

template <int NT, int E>
__device__ int select_row_regs(const float* row, int nfull, bool partial, int mode, int kblocks, double tau,
                               SelectRegsScratch& sc, int32_t* out, int cap) {
  static_assert(NT >= 256 && NT % 32 == 0, "one thread per radix bucket");
  const int tid = threadIdx.x;
  const int n0 = tid * E;
  uint32_t key[E];
  float val[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int n = n0 + e;
    val[e] = n < nfull ? row[n] : 0.f;
    key[e] = n < nfull ? order_key(val[e]) : 0u;   // real keys are never 0
  }
  uint32_t T = 0;
  int rem = 0;          // ties at T to keep (top-k)
  bool all = false;
  double mref = 0.0, ssum = 1.0;
  if (mode == 0) {
    const int k = min(kblocks, nfull);
    if (k >= nfull) {
      all = true;
    } else if (k <= 0) {
      T = 0xffffffffu;
    } else {
      if (tid < 256) {
        sc.hist[0][tid] = 0;
        sc.hist[1][tid] = 0;
      }
      __syncthreads();
      uint32_t prefix = 0, pmask = 0;
      int want = k;
      bool whole = false;
      int cur = 0;
      for (int pass = 3; pass >= 0 && !whole; --pass, cur ^= 1) {
        const int shift = pass * 8;
#pragma unroll
        for (int e = 0; e < E; ++e)
          if (n0 + e < nfull && (key[e] & pmask) == prefix) atomicAdd(&sc.hist[cur][(key[e] >> shift) & 255u], 1);
        __syncthreads();
        if (tid < 32) {
          // lane l owns digits 255-8l .. 248-8l (descending); a lane scan gives the counts above
          int c[8], tot = 0;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            c[j] = sc.hist[cur][255 - (8 * tid + j)];
            tot += c[j];
          }
          int incl = tot;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (tid >= off) incl += y;
          }
          int above = incl - tot;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (above < want && above + c[j] >= want) {
              sc.pick[0] = 255 - (8 * tid + j);
              sc.pick[1] = want - above;
              sc.pick[2] = c[j];
            }
            above += c[j];
          }
        } else {
          // clear the other histogram for the next pass (threads 32 .. NT-1 cover the 256 buckets)
          for (int i = tid - 32; i < 256; i += NT - 32) sc.hist[cur ^ 1][i] = 0;
        }
        __syncthreads();
        prefix |= (uint32_t)sc.pick[0] << shift;
        pmask |= 255u << shift;
        want = sc.pick[1];
        whole = sc.pick[2] == want && prefix > 0;   // the whole bucket is taken: its lower bound settles it
      }
      if (whole) {
        T = prefix - 1;
        rem = 0;
      } else {
        T = prefix;
        rem = want;
      }
    }
  } else {
    float mx = -INFINITY;
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (n0 + e < nfull) mx = fmaxf(mx, val[e]);
    mx = block_reduce<NT, float>(mx, reinterpret_cast<float*>(sc.ws), true);
    mref = (double)mx;
    double s = 0.0;
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (n0 + e < nfull) s += exp((double)val[e] - mref);
    ssum = block_reduce<NT, double>(s, sc.wsd, false);
  }
  // packed counts: kept-for-sure (high 16 bits) and ties at T (low 16 bits); E * NT < 65536
  bool sel[E];
  int ngt = 0, neq = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const bool in = n0 + e < nfull;
    if (all) {
      sel[e] = in;
    } else if (mode == 0) {
      sel[e] = in && key[e] > T;
      neq += (in && key[e] == T) ? 1 : 0;
    } else {
      sel[e] = in && exp((double)val[e] - mref) / ssum > tau;
    }
    ngt += sel[e] ? 1 : 0;
  }
  int tot;
  const int pre = block_excl_scan<NT>((ngt << 16) | neq, sc.ws, &tot);
  const int eq_before = pre & 0xffff;
  int pos = (pre >> 16) + min(eq_before, rem);
  int eq_seen = eq_before;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    bool take = sel[e];
    if (!take && mode == 0 && !all && n0 + e < nfull && key[e] == T) take = eq_seen++ < rem;
    if (take) {
      if (pos < cap) out[pos] = n0 + e;
      ++pos;
    }
  }
  int running = (tot >> 16) + min(tot & 0xffff, rem);
  if (partial) {
    if (tid == 0 && running < cap) out[running] = nfull;
    ++running;
  }
  const int total = min(running, cap);
  for (int i = total + tid; i < cap; i += NT) out[i] = -1;
  return total;
}

// shared bytes select_row needs beyond SelectScratch: keys, plus pairs for top-p
__host__ __device__ inline size_t select_smem_bytes(int nb, int mode) {
  size_t s = (size_t)((nb + 1) & ~1) * 4;
  if (mode == 2) {
    int pw = 1;
    while (pw < nb) pw <<= 1;
    s += (size_t)pw * 8;
  }
  return s;
}

}  // namespace seer
