// C ABI of libseer (declared in include/seer.h): argument validation, TMA
// descriptor encoding (cached), launch-shape choices and kernel launches.
// Nothing here allocates device memory or synchronises the host.
#include <cstdint>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>

#include "seer.h"
#include "seer_internal.h"

namespace {

thread_local std::string g_err;

seer_status fail(seer_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

seer_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SEER_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

seer_status check_dims(const seer_dims_t* d) {
  if (!d) return fail(SEER_ERR_INVALID_ARG, "dims is NULL");
  if (d->batch < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1)
    return fail(SEER_ERR_INVALID_ARG, "batch, num_q_heads and num_kv_heads must be >= 1");
  if (d->num_q_heads % d->num_kv_heads != 0)
    return fail(SEER_ERR_INVALID_ARG, "num_q_heads (%d) is not a multiple of num_kv_heads (%d)",
                d->num_q_heads, d->num_kv_heads);
  const int g = d->num_q_heads / d->num_kv_heads;
  if (g > seer::kMaxGroup) return fail(SEER_ERR_UNSUPPORTED, "group size %d > %d", g, seer::kMaxGroup);
  if (d->head_dim != 64 && d->head_dim != 128)
    return fail(SEER_ERR_UNSUPPORTED, "head_dim %d not in {64, 128}", d->head_dim);
  if (d->gate_dim != 64 && d->gate_dim != 128)
    return fail(SEER_ERR_UNSUPPORTED, "gate_dim %d not in {64, 128}", d->gate_dim);
  if (d->block_size != 64 && d->block_size != 128)
    return fail(SEER_ERR_UNSUPPORTED, "block_size %d not in {64, 128}", d->block_size);
  if (d->max_blocks < 1 || d->max_blocks > seer::kMaxBlocksRow)
    return fail(SEER_ERR_UNSUPPORTED, "max_blocks %d not in [1, %d]", d->max_blocks, seer::kMaxBlocksRow);
  if (!(d->rope_base > 0.f) || !isfinite(d->rope_base)) return fail(SEER_ERR_INVALID_ARG, "rope_base must be > 0");
  if (!(d->softmax_scale >= 0.f) || !isfinite(d->softmax_scale))
    return fail(SEER_ERR_INVALID_ARG, "softmax_scale must be >= 0 (0 = 1/sqrt(head_dim))");
  return SEER_OK;
}

seer_status check_kv(const seer_dims_t* d, const seer_kv_t* kv, const char* name) {
  if (!kv) return fail(SEER_ERR_INVALID_ARG, "%s descriptor is NULL", name);
  if (!kv->data) return fail(SEER_ERR_INVALID_ARG, "%s data is NULL", name);
  if (!aligned16(kv->data)) return fail(SEER_ERR_INVALID_ARG, "%s data is not 16-byte aligned", name);
  if (kv->layout != SEER_KV_CONTIGUOUS && kv->layout != SEER_KV_PAGED)
    return fail(SEER_ERR_INVALID_ARG, "%s layout %d unknown", name, kv->layout);
  const int64_t D = d->head_dim;
  if (kv->stride_t < D || kv->stride_h < 1 || kv->stride_b < 1)
    return fail(SEER_ERR_INVALID_ARG, "%s strides (b=%lld h=%lld t=%lld) invalid for head_dim %lld", name,
                (long long)kv->stride_b, (long long)kv->stride_h, (long long)kv->stride_t, (long long)D);
  if ((kv->stride_t % 8) || (kv->stride_h % 8) || (kv->stride_b % 8))
    return fail(SEER_ERR_INVALID_ARG, "%s strides must be multiples of 8 elements (16 bytes)", name);
  if (kv->layout == SEER_KV_CONTIGUOUS) {
    if (kv->num_tokens < 1) return fail(SEER_ERR_INVALID_ARG, "%s num_tokens must be >= 1", name);
  } else {
    if (!kv->block_table) return fail(SEER_ERR_INVALID_ARG, "%s block_table is NULL (paged layout)", name);
    if (kv->num_pages < 1 || kv->max_pages_per_seq < 1)
      return fail(SEER_ERR_INVALID_ARG, "%s num_pages and max_pages_per_seq must be >= 1", name);
    if (kv->num_pages > INT32_MAX) return fail(SEER_ERR_UNSUPPORTED, "%s num_pages above 2^31", name);
  }
  return SEER_OK;
}

// ------------------------------------------------------------------ device facts (cached per device)
struct DevFacts {
  int sms = 0;
  int occ[2][2] = {{0, 0}, {0, 0}};  // decode CTAs/SM by [D==128][BLK==128]
};
std::mutex g_mu;
DevFacts g_dev[64];

seer_status device_facts(int* dev_out, DevFacts** f) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(SEER_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  DevFacts& df = g_dev[dev];
  if (df.sms == 0) {
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    df.sms = sms;
  }
  *dev_out = dev;
  *f = &df;
  return SEER_OK;
}

int decode_occ(DevFacts* df, int D, int BLK) {
  int& o = df->occ[D == 128][BLK == 128];
  if (o == 0) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (o == 0) o = seer::decode_ctas_per_sm(D, BLK);
  }
  return o;
}

// ------------------------------------------------------------------ TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;

seer_status encoder(EncodeTiledFn* fn) {
  std::call_once(g_encode_once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    g_encode_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (g_encode_err == cudaSuccess && q != cudaDriverEntryPointSuccess) g_encode_err = cudaErrorNotSupported;
    if (g_encode_err == cudaSuccess) g_encode = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!g_encode) return cuda_fail(g_encode_err == cudaSuccess ? cudaErrorNotSupported : g_encode_err,
                                  "resolving cuTensorMapEncodeTiled");
  *fn = g_encode;
  return SEER_OK;
}

struct MapKey {
  const void* data;
  int64_t ext[3], str[3];
  int D, BLK;
  bool operator==(const MapKey& o) const {
    if (data != o.data || D != o.D || BLK != o.BLK) return false;
    for (int i = 0; i < 3; ++i)
      if (ext[i] != o.ext[i] || str[i] != o.str[i]) return false;
    return true;
  }
};
struct MapEntry {
  MapKey key;
  CUtensorMap map;
  int perm[3];
  bool used = false;
};
constexpr int kMapCache = 128;
MapEntry g_maps[kMapCache];
int g_map_next = 0;

// Describe a K/V cache as a 4-D tensor (channel, then token / head / batch-or-page
// sorted by stride), box = 64 channels x BLK tokens, 128-byte swizzle.
seer_status tensor_map(const seer_dims_t* d, const seer_kv_t* kv, const char* name, CUtensorMap* out,
                       int perm[3]) {
  MapKey key;
  key.data = kv->data;
  key.D = d->head_dim;
  key.BLK = d->block_size;
  const bool paged = kv->layout == SEER_KV_PAGED;
  key.ext[0] = paged ? d->block_size : kv->num_tokens;  // role 0: token
  key.ext[1] = d->num_kv_heads;                          // role 1: head
  key.ext[2] = paged ? kv->num_pages : d->batch;         // role 2: batch or page
  key.str[0] = kv->stride_t;
  key.str[1] = kv->stride_h;
  key.str[2] = kv->stride_b;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    for (int i = 0; i < kMapCache; ++i) {
      if (g_maps[i].used && g_maps[i].key == key) {
        *out = g_maps[i].map;
        for (int r = 0; r < 3; ++r) perm[r] = g_maps[i].perm[r];
        return SEER_OK;
      }
    }
  }
  EncodeTiledFn enc;
  seer_status st = encoder(&enc);
  if (st != SEER_OK) return st;
  // order roles by stride (stable): TMA dims 1..3
  int order[3] = {0, 1, 2};
  for (int i = 1; i < 3; ++i)
    for (int j = i; j > 0 && key.str[order[j]] < key.str[order[j - 1]]; --j) {
      int t = order[j];
      order[j] = order[j - 1];
      order[j - 1] = t;
    }
  cuuint64_t gdim[4], gstr[3];
  cuuint32_t box[4], estr[4] = {1, 1, 1, 1};
  gdim[0] = (cuuint64_t)d->head_dim;
  box[0] = 64;
  for (int i = 0; i < 3; ++i) {
    const int role = order[i];
    perm[role] = i;
    if (key.ext[role] < 1 || key.ext[role] > (int64_t(1) << 32))
      return fail(SEER_ERR_INVALID_ARG, "%s extent out of range for a TMA descriptor", name);
    gdim[i + 1] = (cuuint64_t)key.ext[role];
    gstr[i] = (cuuint64_t)key.str[role] * 2;
    if (gstr[i] >= (cuuint64_t(1) << 40)) return fail(SEER_ERR_INVALID_ARG, "%s stride too large for TMA", name);
    box[i + 1] = role == 0 ? (cuuint32_t)d->block_size : 1u;
  }
  CUtensorMap map;
  CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(kv->data), gdim, gstr, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SEER_ERR_INVALID_ARG, "%s: cuTensorMapEncodeTiled failed (%d)", name, (int)r);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    MapEntry& e = g_maps[g_map_next];
    g_map_next = (g_map_next + 1) % kMapCache;
    e.key = key;
    e.map = map;
    for (int i = 0; i < 3; ++i) e.perm[i] = perm[i];
    e.used = true;
  }
  *out = map;
  return SEER_OK;
}

void rope_thetas(const seer_dims_t* d, double* theta) {
  const int half = d->gate_dim / 2;
  for (int i = 0; i < half; ++i) theta[i] = pow((double)d->rope_base, -2.0 * i / d->gate_dim);
}

seer_status select_args(const seer_dims_t* dims, int32_t mode, int32_t token_budget, float tau, int32_t capacity,
                        int32_t* kblocks) {
  if (mode != SEER_SELECT_TOPK && mode != SEER_SELECT_THRESHOLD && mode != SEER_SELECT_TOPP)
    return fail(SEER_ERR_INVALID_ARG, "unknown selection mode %d", mode);
  if (capacity < 1) return fail(SEER_ERR_INVALID_ARG, "capacity must be >= 1");
  *kblocks = 0;
  if (mode == SEER_SELECT_TOPK) {
    if (token_budget < 0) return fail(SEER_ERR_INVALID_ARG, "token_budget must be >= 0");
    int32_t k = (int32_t)(((int64_t)token_budget + dims->block_size - 1) / dims->block_size);
    if (k > dims->max_blocks) k = dims->max_blocks;
    if (capacity < k + 1 && capacity < dims->max_blocks)
      return fail(SEER_ERR_CAPACITY, "capacity %d < k+1 = %d (top-k plus the partial block)", capacity, k + 1);
    *kblocks = k;
  } else {
    if (!isfinite(tau)) return fail(SEER_ERR_INVALID_ARG, "tau must be finite");
    if (capacity < dims->max_blocks)
      return fail(SEER_ERR_CAPACITY, "capacity %d < max_blocks %d (threshold / top-p may select every block)",
                  capacity, dims->max_blocks);
  }
  return SEER_OK;
}

seer::KvPlain plain(const seer_kv_t* kv) {
  seer::KvPlain k;
  k.data = static_cast<const uint16_t*>(kv->data);
  k.stride_b = kv->stride_b;
  k.stride_h = kv->stride_h;
  k.stride_t = kv->stride_t;
  k.paged = kv->layout == SEER_KV_PAGED;
  k.block_table = kv->block_table;
  k.max_pages = kv->max_pages_per_seq;
  k.num_pages = kv->num_pages;
  k.num_tokens = kv->num_tokens;
  return k;
}

int32_t auto_split(const seer_dims_t* d, int32_t capacity, DevFacts* df) {
  const int64_t units = (int64_t)d->batch * d->num_kv_heads;
  const int64_t slots = (int64_t)df->sms * decode_occ(df, d->head_dim, d->block_size);
  int64_t ns = slots / units;                       // fill one wave, never spill into a second
  ns = ns < 1 ? 1 : ns;
  const int64_t max_ns = (capacity + 1) / 2;        // at least two list slots per split
  if (ns > max_ns) ns = max_ns;
  return (int32_t)(ns < 1 ? 1 : ns);
}

// CTAs of the balanced (num_split == 0) schedule: one per SM slot.
int flat_grid(const seer_dims_t* d, DevFacts* df) { return df->sms * decode_occ(df, d->head_dim, d->block_size); }

// Workspace: split-arrival counters [B*Hkv] int32 (zero before the first call, left zero) |
// lse partials [slots][g] | o partials [slots][g][d].  Balanced schedule: 2 partial slots per
// CTA (a CTA's first and last segment are the only ones that can belong to a (b, h) split
// across CTAs).  Grid schedule: num_split slots per (b, h).
size_t ws_layout(const seer_dims_t* d, int32_t ns, int flat_ctas, size_t* off_lse, size_t* off_o) {
  // ns <= 0: one of the one-wave schedules (balanced or capacity), 2 slots per CTA
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t g = (size_t)(d->num_q_heads / d->num_kv_heads);
  const size_t bh = (size_t)d->batch * d->num_kv_heads;
  const size_t slots = ns <= 0 ? 2 * (size_t)flat_ctas : bh * ns;
  const size_t rec = up(bh * 4);
  const size_t lse = up(slots * g * 4);
  const size_t o = slots * g * d->head_dim * 4;
  *off_lse = rec;
  *off_o = rec + lse;
  return ns == 1 ? 0 : rec + lse + o;
}

}  // namespace

int seer::set_last_error(int status, const char* msg) {
  g_err = msg ? msg : "";
  return status;
}

extern "C" {

const char* seer_last_error(void) { return g_err.c_str(); }

const char* seer_version(void) { return "libseer 0.1 (sm_100a)"; }

// process-wide bound and debug switch of the sparse decode's waits, read at each launch
namespace {
std::atomic<long long> g_wait_limit{seer::kWaitLimitCycles};
std::atomic<int32_t> g_debug{0};
}  // namespace

seer_status seer_set_wait_limit(int64_t cycles) {
  if (cycles == 0) cycles = seer::kWaitLimitCycles;
  if (cycles < SEER_WAIT_LIMIT_MIN || cycles > SEER_WAIT_LIMIT_MAX)
    return fail(SEER_ERR_INVALID_ARG, "wait limit %lld cycles outside [%lld, %lld] (0 = the default)",
                (long long)cycles, (long long)SEER_WAIT_LIMIT_MIN, (long long)SEER_WAIT_LIMIT_MAX);
  g_wait_limit.store(cycles);
  return SEER_OK;
}

int64_t seer_get_wait_limit(void) { return g_wait_limit.load(); }

seer_status seer_set_debug_flags(int32_t flags) {
  if (flags & ~SEER_DEBUG_STARVE_COPIES) return fail(SEER_ERR_INVALID_ARG, "unknown debug flags 0x%x", flags);
  g_debug.store(flags);
  return SEER_OK;
}

seer_status seer_kcomp_update(const seer_dims_t* dims, const seer_kv_t* k_nope, const int32_t* seqlens,
                              int32_t* valid_blocks, const void* w_k, void* kcomp, void* stream) {
  seer_status st = check_dims(dims);
  if (st != SEER_OK) return st;
  if ((st = check_kv(dims, k_nope, "k_nope")) != SEER_OK) return st;
  if (!seqlens || !valid_blocks || !w_k || !kcomp) return fail(SEER_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(w_k) || !aligned16(kcomp)) return fail(SEER_ERR_INVALID_ARG, "w_k / kcomp not 16-byte aligned");
  int dev;
  DevFacts* df;
  if ((st = device_facts(&dev, &df)) != SEER_OK) return st;
  seer::KcompParams p;
  rope_thetas(dims, p.theta);
  p.k = plain(k_nope);
  p.seqlens = seqlens;
  p.valid = valid_blocks;
  p.valid_out = valid_blocks;
  p.w_k = static_cast<const uint16_t*>(w_k);
  p.kcomp = static_cast<uint16_t*>(kcomp);
  p.B = dims->batch;
  p.Hkv = dims->num_kv_heads;
  p.NB = dims->max_blocks;
  p.rope_base = dims->rope_base;
  p.err = nullptr;
  const int units = dims->batch * dims->num_kv_heads;
  int gx = (2 * df->sms + units - 1) / units;
  const int groups = (dims->max_blocks + 7) / 8;
  gx = gx < 1 ? 1 : (gx > groups ? groups : gx);
  cudaError_t e = seer::launch_kcomp_update(p, dims->head_dim, dims->block_size, dims->gate_dim, gx,
                                            static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "kcomp_update launch");
  return SEER_OK;
}

size_t seer_prefill_gt_workspace_bytes(const seer_dims_t* dims, int32_t max_len) {
  if (check_dims(dims) != SEER_OK || max_len < 1) return 0;
  return (size_t)dims->batch * dims->num_q_heads * (dims->max_blocks + (size_t)1) * (size_t)max_len * sizeof(float);
}

seer_status seer_prefill_gt(const seer_dims_t* dims, const void* q, int32_t max_len, const seer_kv_t* k,
                            const seer_kv_t* v, const int32_t* seqlens, void* out, float* lse_out, float* gt,
                            void* workspace, size_t workspace_bytes, int32_t* err_word, void* stream) {
  seer_status st = check_dims(dims);
  if (st != SEER_OK) return st;
  if ((st = check_kv(dims, k, "k")) != SEER_OK) return st;
  if ((st = check_kv(dims, v, "v")) != SEER_OK) return st;
  if (k->layout != SEER_KV_CONTIGUOUS || v->layout != SEER_KV_CONTIGUOUS)
    return fail(SEER_ERR_UNSUPPORTED, "prefill attention takes contiguous K/V caches");
  if (!q || !seqlens || !out || !gt || !workspace) return fail(SEER_ERR_INVALID_ARG, "NULL pointer argument");
  if (max_len < 1) return fail(SEER_ERR_INVALID_ARG, "max_len must be >= 1");
  if ((int64_t)dims->max_blocks * dims->block_size < max_len)
    return fail(SEER_ERR_INVALID_ARG, "max_blocks * block_size < max_len");
  if (!aligned16(q) || !aligned16(out) || !aligned16(gt) || !aligned16(workspace) || (lse_out && !aligned16(lse_out)))
    return fail(SEER_ERR_INVALID_ARG, "pointer not 16-byte aligned");
  const size_t need = seer_prefill_gt_workspace_bytes(dims, max_len);
  if (workspace_bytes < need)
    return fail(SEER_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", workspace_bytes, need);
  int dev;
  DevFacts* df;
  if ((st = device_facts(&dev, &df)) != SEER_OK) return st;
  CUtensorMap tk, tv;
  seer::PrefillParams p{};
  if ((st = tensor_map(dims, k, "k", &tk, p.k_perm)) != SEER_OK) return st;
  if ((st = tensor_map(dims, v, "v", &tv, p.v_perm)) != SEER_OK) return st;
  p.q = static_cast<const uint16_t*>(q);
  p.o = static_cast<uint16_t*>(out);
  p.lse = lse_out;
  p.gt = gt;
  p.rmax = static_cast<float*>(workspace);
  p.rnorm = p.rmax + (size_t)dims->batch * dims->num_q_heads * dims->max_blocks * (size_t)max_len;
  p.seqlens = seqlens;
  p.B = dims->batch;
  p.Hq = dims->num_q_heads;
  p.Hkv = dims->num_kv_heads;
  p.g = dims->num_q_heads / dims->num_kv_heads;
  p.NB = dims->max_blocks;
  p.T = max_len;
  const int64_t cap = k->num_tokens < v->num_tokens ? k->num_tokens : v->num_tokens;
  p.kcap = cap > max_len ? max_len : (int32_t)cap;
  const float scale = dims->softmax_scale > 0.f ? dims->softmax_scale : 1.0f / sqrtf((float)dims->head_dim);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.err = err_word;
  // the tcgen05 / TMEM kernel where it takes the shape, the warp-level mma kernel otherwise
  cudaError_t e = seer::prefill_tc_supported(dims->head_dim, dims->block_size, p.g)
                      ? seer::launch_prefill_tc(tk, tv, p, dims->head_dim, dims->block_size, max_len, df->sms,
                                                static_cast<cudaStream_t>(stream))
                      : seer::launch_prefill_gt(tk, tv, p, dims->head_dim, dims->block_size, max_len,
                                                static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prefill_gt launch");
  return SEER_OK;
}

size_t seer_kcomp_state_bytes(const seer_dims_t* dims) {
  if (check_dims(dims) != SEER_OK) return 0;
  return (size_t)dims->batch * dims->num_kv_heads * 3 * dims->head_dim * sizeof(float);
}

seer_status seer_kcomp_append(const seer_dims_t* dims, const void* k_new, const int32_t* seqlens, float* state,
                              int32_t* valid_blocks, const void* w_k, void* kcomp, int32_t* err_word,
                              void* stream) {
  seer_status st = check_dims(dims);
  if (st != SEER_OK) return st;
  if (!k_new || !seqlens || !state || !valid_blocks || !w_k || !kcomp)
    return fail(SEER_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(k_new) || !aligned16(state) || !aligned16(w_k) || !aligned16(kcomp))
    return fail(SEER_ERR_INVALID_ARG, "k_new / state / w_k / kcomp not 16-byte aligned");
  seer::AppendParams p{};
  rope_thetas(dims, p.theta);
  p.k_new = static_cast<const uint16_t*>(k_new);
  p.seqlens = seqlens;
  p.valid = valid_blocks;
  p.state = state;
  p.w_k = static_cast<const uint16_t*>(w_k);
  p.kcomp = static_cast<uint16_t*>(kcomp);
  p.B = dims->batch;
  p.Hkv = dims->num_kv_heads;
  p.NB = dims->max_blocks;
  p.err = err_word;
  cudaError_t e = seer::launch_kcomp_append(p, dims->head_dim, dims->block_size, dims->gate_dim,
                                            static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "kcomp_append launch");
  return SEER_OK;
}

seer_status seer_kcomp_state_init(const seer_dims_t* dims, const seer_kv_t* k_nope, const int32_t* seqlens,
                                  float* state, int32_t* err_word, void* stream) {
  seer_status st = check_dims(dims);
  if (st != SEER_OK) return st;
  if ((st = check_kv(dims, k_nope, "k_nope")) != SEER_OK) return st;
  if (!seqlens || !state) return fail(SEER_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(state)) return fail(SEER_ERR_INVALID_ARG, "state not 16-byte aligned");
  seer::AppendParams p{};
  p.k = plain(k_nope);
  p.seqlens = seqlens;
  p.state = state;
  p.B = dims->batch;
  p.Hkv = dims->num_kv_heads;
  p.NB = dims->max_blocks;
  p.err = err_word;
  cudaError_t e = seer::launch_kcomp_state_init(p, dims->head_dim, dims->block_size,
                                                static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "kcomp_state_init launch");
  return SEER_OK;
}

seer_status seer_gate_score(const seer_dims_t* dims, const void* q_nope, const void* w_q, const void* kcomp,
                            const int32_t* seqlens, float* logits, float* q_gate_out, void* stream) {
  seer_status st = check_dims(dims);
  if (st != SEER_OK) return st;
  if (!q_nope || !w_q || !kcomp || !seqlens || !logits) return fail(SEER_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(q_nope) || !aligned16(w_q) || !aligned16(kcomp) || !aligned16(logits) ||
      (q_gate_out && !aligned16(q_gate_out)))
    return fail(SEER_ERR_INVALID_ARG, "pointer not 16-byte aligned");
  seer::GateParams p;
  rope_thetas(dims, p.theta);
  p.q = static_cast<const uint16_t*>(q_nope);
  p.w_q = static_cast<const uint16_t*>(w_q);
  p.kcomp = static_cast<const uint16_t*>(kcomp);
  p.seqlens = seqlens;
  p.logits = logits;
  p.q_gate = q_gate_out;
  p.B = dims->batch;
  p.Hq = dims->num_q_heads;
  p.Hkv = dims->num_kv_heads;
  p.g = dims->num_q_heads / dims->num_kv_heads;
  p.NB = dims->max_blocks;
  p.BLK = dims->block_size;
  p.rope_base = dims->rope_base;
  cudaError_t e = seer::launch_gate_score(p, dims->head_dim, dims->gate_dim, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gate_score launch");
  return SEER_OK;
}

seer_status seer_select_blocks(const seer_dims_t* dims, const float* logits, const int32_t* seqlens, int32_t mode,
                               int32_t token_budget, float tau, int32_t* block_idx, int32_t* block_cnt,
                               int32_t capacity, void* stream) {
  seer_status st = check_dims(dims);
  if (st != SEER_OK) return st;
  if (!logits || !seqlens || !block_idx || !block_cnt) return fail(SEER_ERR_INVALID_ARG, "NULL pointer argument");
  int32_t kblocks = 0;
  if ((st = select_args(dims, mode, token_budget, tau, capacity, &kblocks)) != SEER_OK) return st;
  seer::SelectParams p;
  p.logits = logits;
  p.seqlens = seqlens;
  p.idx = block_idx;
  p.cnt = block_cnt;
  p.B = dims->batch;
  p.Hkv = dims->num_kv_heads;
  p.NB = dims->max_blocks;
  p.BLK = dims->block_size;
  p.cap = capacity;
  p.mode = mode;
  p.kblocks = kblocks;
  p.tau = (double)tau;
  cudaError_t e = seer::launch_select(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "select_blocks launch");
  return SEER_OK;
}

}  // extern "C"

namespace {

// Argument checks and kernel parameters of seer_decode_plan (shared with seer_decode_step).
seer_status plan_params(const seer_dims_t* dims, const seer_kv_t* k_nope, const int32_t* seqlens,
                        int32_t* valid_blocks, const void* w_k, void* kcomp, const void* q_nope, const void* w_q,
                        float* logits_out, float* q_gate_out, int32_t mode, int32_t token_budget, float tau,
                        int32_t* block_idx, int32_t* block_cnt, int32_t capacity, seer::PlanParams* pp) {
  seer_status st = check_dims(dims);
  if (st != SEER_OK) return st;
  if (!seqlens || !kcomp || !q_nope || !w_q || !block_idx || !block_cnt)
    return fail(SEER_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(kcomp) || !aligned16(q_nope) || !aligned16(w_q) || (logits_out && !aligned16(logits_out)) ||
      (q_gate_out && !aligned16(q_gate_out)))
    return fail(SEER_ERR_INVALID_ARG, "pointer not 16-byte aligned");
  const bool update = valid_blocks != nullptr;
  if (update) {
    if ((st = check_kv(dims, k_nope, "k_nope")) != SEER_OK) return st;
    if (!w_k || !aligned16(w_k)) return fail(SEER_ERR_INVALID_ARG, "w_k is NULL or not 16-byte aligned");
  }
  int32_t kblocks = 0;
  if ((st = select_args(dims, mode, token_budget, tau, capacity, &kblocks)) != SEER_OK) return st;
  seer::PlanParams& p = *pp;
  p.update_cache = update;
  rope_thetas(dims, p.k.theta);
  if (update) p.k.k = plain(k_nope);
  else memset(&p.k.k, 0, sizeof(p.k.k));
  p.k.seqlens = seqlens;
  p.k.valid = valid_blocks;
  p.k.valid_out = valid_blocks;
  p.k.w_k = static_cast<const uint16_t*>(w_k);
  p.k.kcomp = static_cast<uint16_t*>(kcomp);
  p.k.B = dims->batch;
  p.k.Hkv = dims->num_kv_heads;
  p.k.NB = dims->max_blocks;
  p.k.rope_base = dims->rope_base;
  p.k.err = nullptr;
  rope_thetas(dims, p.g.theta);
  p.g.q = static_cast<const uint16_t*>(q_nope);
  p.g.w_q = static_cast<const uint16_t*>(w_q);
  p.g.kcomp = static_cast<const uint16_t*>(kcomp);
  p.g.seqlens = seqlens;
  p.g.logits = logits_out;
  p.g.q_gate = q_gate_out;
  p.g.B = dims->batch;
  p.g.Hq = dims->num_q_heads;
  p.g.Hkv = dims->num_kv_heads;
  p.g.g = dims->num_q_heads / dims->num_kv_heads;
  p.g.NB = dims->max_blocks;
  p.g.BLK = dims->block_size;
  p.g.rope_base = dims->rope_base;
  p.s.logits = nullptr;
  p.s.seqlens = seqlens;
  p.s.idx = block_idx;
  p.s.cnt = block_cnt;
  p.s.B = dims->batch;
  p.s.Hkv = dims->num_kv_heads;
  p.s.NB = dims->max_blocks;
  p.s.BLK = dims->block_size;
  p.s.cap = capacity;
  p.s.mode = mode;
  p.s.kblocks = kblocks;
  p.s.tau = (double)tau;
  return SEER_OK;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" {

seer_status seer_decode_plan(const seer_dims_t* dims, const seer_kv_t* k_nope, const int32_t* seqlens,
                             int32_t* valid_blocks, const void* w_k, void* kcomp, const void* q_nope,
                             const void* w_q, float* logits_out, float* q_gate_out, int32_t mode,
                             int32_t token_budget, float tau, int32_t* block_idx, int32_t* block_cnt,
                             int32_t capacity, void* stream) {
  seer::PlanParams p;
  const seer_status st = plan_params(dims, k_nope, seqlens, valid_blocks, w_k, kcomp, q_nope, w_q, logits_out,
                                     q_gate_out, mode, token_budget, tau, block_idx, block_cnt, capacity, &p);
  if (st != SEER_OK) return st;
  cudaError_t e = seer::launch_plan(p, dims->head_dim, dims->block_size, dims->gate_dim, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode_plan launch");
  return SEER_OK;
}

size_t seer_decode_step_workspace_bytes(const seer_dims_t* dims, int32_t capacity) {
  if (check_dims(dims) != SEER_OK || capacity < 1) return 0;
  return up256((size_t)dims->batch * dims->num_kv_heads * 4) + seer_sparse_decode_workspace_bytes(dims, capacity, -1);
}

int32_t seer_decode_step_supported(const seer_dims_t* dims, int32_t mode, int32_t capacity) {
  if (check_dims(dims) != SEER_OK || capacity < 1) return 0;
  if ((int64_t)dims->batch * dims->num_kv_heads > seer::kMaxDecodeBH) return 0;
  if ((int64_t)dims->batch * dims->num_kv_heads * capacity >= (int64_t)1 << 30) return 0;
  const int bh = dims->batch * dims->num_kv_heads;
  return seer::step_grid(dims->head_dim, dims->block_size, dims->gate_dim, dims->num_q_heads / dims->num_kv_heads,
                         dims->max_blocks, mode, dims->batch, bh) > 0;
}

seer_status seer_decode_step(const seer_dims_t* dims, const seer_kv_t* k_nope, const int32_t* seqlens,
                             int32_t* valid_blocks, const void* w_k, void* kcomp, const void* q_nope,
                             const void* w_q, float* logits_out, float* q_gate_out, int32_t mode,
                             int32_t token_budget, float tau, int32_t* block_idx, int32_t* block_cnt,
                             int32_t capacity, const void* q, const seer_kv_t* k, const seer_kv_t* v,
                             void* workspace, size_t workspace_bytes, void* out, float* lse_out,
                             int32_t* err_word, void* stream) {
  seer::StepParams sp;
  seer_status st = plan_params(dims, k_nope, seqlens, valid_blocks, w_k, kcomp, q_nope, w_q, logits_out, q_gate_out,
                               mode, token_budget, tau, block_idx, block_cnt, capacity, &sp.pl);
  if (st != SEER_OK) return st;
  if (!workspace || !aligned16(workspace)) return fail(SEER_ERR_INVALID_ARG, "workspace is NULL or not 16-byte aligned");
  const size_t flags = up256((size_t)dims->batch * dims->num_kv_heads * 4);
  const size_t need = seer_decode_step_workspace_bytes(dims, capacity);
  if (workspace_bytes < need)
    return fail(SEER_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", workspace_bytes, need);
  const int bh = dims->batch * dims->num_kv_heads;
  const int grid = (int64_t)bh * capacity >= (int64_t)1 << 30
                       ? 0
                       : seer::step_grid(dims->head_dim, dims->block_size, dims->gate_dim,
                                         dims->num_q_heads / dims->num_kv_heads, dims->max_blocks, mode, dims->batch, bh);
  if (grid <= 0)
    return fail(SEER_ERR_UNSUPPORTED, "no fused step for this shape (shared memory or cluster residency); call "
                                      "seer_decode_plan and seer_sparse_decode instead");
  seer::DecodeLaunch L;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  st = seer::prepare_sparse_decode(dims, q, k, v, block_idx, block_cnt, seqlens, capacity, -1, ws + flags,
                                   workspace_bytes - flags, out, lse_out, err_word, &L);
  if (st != SEER_OK) return st;
  if (L.ctas < grid) return fail(SEER_ERR_UNSUPPORTED, "fused step grid %d above the decode's %d", grid, L.ctas);
  sp.d = L.p;
  sp.d.ready = reinterpret_cast<int32_t*>(ws);
  sp.d.starve = 0;   // the debug switch covers the two-launch decode only
  sp.pl.k.err = err_word;
  cudaError_t e = seer::launch_decode_step(L.tk, L.tv, sp, dims->head_dim, dims->block_size, dims->gate_dim, grid,
                                           static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode_step launch");
  return SEER_OK;
}

int32_t seer_sparse_decode_auto_split(const seer_dims_t* dims, int32_t capacity) {
  if (check_dims(dims) != SEER_OK || capacity < 1) return 1;
  int dev;
  DevFacts* df;
  if (device_facts(&dev, &df) != SEER_OK) return 1;
  return auto_split(dims, capacity, df);
}

size_t seer_sparse_decode_workspace_bytes(const seer_dims_t* dims, int32_t capacity, int32_t num_split) {
  if (check_dims(dims) != SEER_OK || capacity < 1 || num_split < -1) return 0;
  const int32_t ns = num_split > capacity ? capacity : num_split;
  int ctas = 0;
  if (ns <= 0) {
    int dev;
    DevFacts* df;
    if (device_facts(&dev, &df) != SEER_OK) return 0;
    ctas = flat_grid(dims, df);
  }
  size_t a, b;
  return ws_layout(dims, ns, ctas, &a, &b);
}

}  // extern "C"

namespace seer {

seer_status prepare_sparse_decode(const seer_dims_t* dims, const void* q, const seer_kv_t* k, const seer_kv_t* v,
                                  const int32_t* block_idx, const int32_t* block_cnt, const int32_t* seqlens,
                                  int32_t capacity, int32_t num_split, void* workspace, size_t workspace_bytes,
                                  void* out, float* lse_out, int32_t* err_word, DecodeLaunch* L) {
  seer_status st = check_dims(dims);
  if (st != SEER_OK) return st;
  if ((st = check_kv(dims, k, "k")) != SEER_OK) return st;
  if ((st = check_kv(dims, v, "v")) != SEER_OK) return st;
  if (!q || !block_idx || !block_cnt || !seqlens || !out) return fail(SEER_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(q) || !aligned16(out)) return fail(SEER_ERR_INVALID_ARG, "q / out not 16-byte aligned");
  if (capacity < 1) return fail(SEER_ERR_INVALID_ARG, "capacity must be >= 1");
  if (num_split < -1) return fail(SEER_ERR_INVALID_ARG, "num_split must be >= -1");
  int dev;
  DevFacts* df;
  if ((st = device_facts(&dev, &df)) != SEER_OK) return st;
  if (dims->batch > seer::kMaxDecodeB) return fail(SEER_ERR_UNSUPPORTED, "batch %d > %d", dims->batch, seer::kMaxDecodeB);
  int32_t ns = num_split > capacity ? capacity : num_split;
  if (ns <= 0 && dims->batch * dims->num_kv_heads > seer::kMaxDecodeBH)
    return fail(SEER_ERR_UNSUPPORTED, "one-wave schedules need batch*num_kv_heads <= %d; pass num_split >= 1",
                seer::kMaxDecodeBH);
  if (ns <= 0 && (int64_t)dims->batch * dims->num_kv_heads * capacity >= (int64_t)1 << 30)
    return fail(SEER_ERR_UNSUPPORTED, "one-wave schedules need batch*num_kv_heads*capacity < 2^30");
  const int ctas = ns <= 0 ? flat_grid(dims, df) : 0;
  size_t off_lse, off_o;
  const size_t need = ws_layout(dims, ns, ctas, &off_lse, &off_o);
  if (need > 0) {
    if (!workspace) return fail(SEER_ERR_INVALID_ARG, "workspace is NULL (num_split %d needs %zu bytes)", ns, need);
    if (workspace_bytes < need)
      return fail(SEER_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed for num_split %d", workspace_bytes, need, ns);
    if (!aligned16(workspace)) return fail(SEER_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  }
  DecodeParams& p = L->p;
  if ((st = tensor_map(dims, k, "k", &L->tk, p.k_perm)) != SEER_OK) return st;
  if ((st = tensor_map(dims, v, "v", &L->tv, p.v_perm)) != SEER_OK) return st;
  p.q = static_cast<const uint16_t*>(q);
  p.idx = block_idx;
  p.cnt = block_cnt;
  p.seqlens = seqlens;
  p.k_paged = k->layout == SEER_KV_PAGED;
  p.v_paged = v->layout == SEER_KV_PAGED;
  p.k_table = k->block_table;
  p.v_table = v->block_table;
  p.k_maxp = k->max_pages_per_seq;
  p.v_maxp = v->max_pages_per_seq;
  p.k_pages = k->num_pages;
  p.v_pages = v->num_pages;
  p.B = dims->batch;
  p.Hq = dims->num_q_heads;
  p.Hkv = dims->num_kv_heads;
  p.g = dims->num_q_heads / dims->num_kv_heads;
  p.cap = capacity;
  p.flat = ns == 0 ? 1 : (ns == -1 ? 2 : 0);
  p.ns = ns > 0 ? ns : 0;
  p.per_split = ns > 0 ? (capacity + ns - 1) / ns : capacity;
  const float scale = dims->softmax_scale > 0.f ? dims->softmax_scale : 1.0f / sqrtf((float)dims->head_dim);
  p.scale_log2 = scale * 1.4426950408889634f;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.counters = need ? reinterpret_cast<int32_t*>(ws) : nullptr;
  p.lse_part = need ? reinterpret_cast<float*>(ws + off_lse) : nullptr;
  p.o_part = need ? reinterpret_cast<float*>(ws + off_o) : nullptr;
  p.out = static_cast<uint16_t*>(out);
  p.lse_out = lse_out;
  p.err = err_word;
  p.ready = nullptr;
  p.wait_limit = g_wait_limit.load();
  p.starve = (g_debug.load() & SEER_DEBUG_STARVE_COPIES) ? 1 : 0;
  L->D = dims->head_dim;
  L->BLK = dims->block_size;
  L->ctas = ctas;
  L->need = need;
  return SEER_OK;
}

// Capacity schedule with short shares (at most this many list positions per CTA): the grid is cut
// to a whole multiple of the row count, so every row splits at the same points and no CTA carries a
// segment flush in mid-stream (measured: 90 %- and 95 %-sparse rows 1-5 % of the copy peak faster);
// with longer shares every SM's bandwidth counts for more (the 50 %-sparse and dense rows lose 6-9 %
// with the cut).  The workspace stays sized for the full grid.
constexpr int kShortShare = 28;

int decode_grid(const DecodeParams& p, int ctas) {
  const long long bh = (long long)p.B * p.Hkv;
  if (p.flat != 2 || bh > ctas) return ctas;
  const int whole = (int)(ctas / bh * bh);
  return bh * p.cap <= (long long)kShortShare * whole ? whole : ctas;
}

seer_status launch_prepared_decode(const DecodeLaunch& L, cudaStream_t s) {
  cudaError_t e = launch_sparse_decode(L.tk, L.tv, L.p, L.D, L.BLK, decode_grid(L.p, L.ctas), s);
  if (e != cudaSuccess) return cuda_fail(e, "sparse_decode launch");
  return SEER_OK;
}

}  // namespace seer

extern "C" {

seer_status seer_sparse_decode(const seer_dims_t* dims, const void* q, const seer_kv_t* k, const seer_kv_t* v,
                               const int32_t* block_idx, const int32_t* block_cnt, const int32_t* seqlens,
                               int32_t capacity, int32_t num_split, void* workspace, size_t workspace_bytes,
                               void* out, float* lse_out, int32_t* err_word, void* stream) {
  seer::DecodeLaunch L;
  const seer_status st = seer::prepare_sparse_decode(dims, q, k, v, block_idx, block_cnt, seqlens, capacity, num_split,
                                                     workspace, workspace_bytes, out, lse_out, err_word, &L);
  if (st != SEER_OK) return st;
  return seer::launch_prepared_decode(L, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- decode ground truth

namespace {
// counters [BH] | per-chunk (max, sum) [BH][nchunk][8][2] | block maxima [BH][NB][8] (8 = the largest group)
size_t truth_layout(const seer_dims_t* d, int* nchunk, size_t* off_part, size_t* off_bmax) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t bh = (size_t)d->batch * d->num_kv_heads;
  const int nc = (d->max_blocks + seer::truth_chunk_blocks() - 1) / seer::truth_chunk_blocks();
  const size_t w = seer::kMaxGroup;
  *nchunk = nc;
  *off_part = up(bh * 4);
  *off_bmax = *off_part + up(bh * nc * w * 2 * 4);
  return *off_bmax + bh * d->max_blocks * w * 4;
}
}  // namespace

size_t seer_gate_truth_workspace_bytes(const seer_dims_t* dims) {
  if (check_dims(dims) != SEER_OK) return 0;
  int nc;
  size_t a, b;
  return truth_layout(dims, &nc, &a, &b);
}

seer_status seer_gate_truth(const seer_dims_t* dims, const void* q, const seer_kv_t* k, const int32_t* seqlens,
                            float* scores, float* log_scores, void* workspace, size_t workspace_bytes,
                            int32_t* err_word, void* stream) {
  seer_status st = check_dims(dims);
  if (st != SEER_OK) return st;
  if ((st = check_kv(dims, k, "k")) != SEER_OK) return st;
  if (!q || !seqlens || !scores || !workspace) return fail(SEER_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(q) || !aligned16(scores) || (log_scores && !aligned16(log_scores)) || !aligned16(workspace))
    return fail(SEER_ERR_INVALID_ARG, "pointer not 16-byte aligned");
  int nc;
  size_t off_part, off_bmax;
  const size_t need = truth_layout(dims, &nc, &off_part, &off_bmax);
  if (workspace_bytes < need)
    return fail(SEER_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", workspace_bytes, need);
  int dev;
  DevFacts* df;
  if ((st = device_facts(&dev, &df)) != SEER_OK) return st;
  CUtensorMap tk;
  seer::TruthParams p;
  if ((st = tensor_map(dims, k, "k", &tk, p.k_perm)) != SEER_OK) return st;
  p.q = static_cast<const uint16_t*>(q);
  p.seqlens = seqlens;
  p.k_paged = k->layout == SEER_KV_PAGED;
  p.k_table = k->block_table;
  p.k_maxp = k->max_pages_per_seq;
  p.k_pages = k->num_pages;
  p.B = dims->batch;
  p.Hq = dims->num_q_heads;
  p.Hkv = dims->num_kv_heads;
  p.g = dims->num_q_heads / dims->num_kv_heads;
  p.NB = dims->max_blocks;
  p.nchunk = nc;
  p.nitems = dims->batch * dims->num_kv_heads * nc;
  const float scale = dims->softmax_scale > 0.f ? dims->softmax_scale : 1.0f / sqrtf((float)dims->head_dim);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.scores = scores;
  p.log_scores = log_scores;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.counters = reinterpret_cast<int32_t*>(ws);
  p.part = reinterpret_cast<float*>(ws + off_part);
  p.bmax = reinterpret_cast<float*>(ws + off_bmax);
  p.err = err_word;
  cudaError_t e = seer::launch_gate_truth(tk, p, dims->head_dim, dims->block_size, df->sms,
                                          static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gate_truth launch");
  return SEER_OK;
}

}  // extern "C"
