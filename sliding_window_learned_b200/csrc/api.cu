// api.cu -- the C ABI of libattnsink.so (declared in include/attnsink.h):
// argument validation, the device status word, the decode workspace pool and
// TMA descriptor encoding.  Every compute step runs in the kernels; nothing
// here touches tensor data on the host.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/attnsink.h"
#include "api_internal.h"
#include "kernels.h"

namespace attnsink {

// Device status word: [0] = first error code, [1] = location of the failing
// wait, [2..3] = the bounded waits' limit in ns (one 64-bit value; 0 = the
// default).  Kernels receive its address; attn_sink_get_status reads and
// clears [0..1]; attn_sink_set_wait_limit_ns sets [2..3].
__device__ __align__(8) int g_status[4];

namespace {
thread_local char t_last_error[256] = "";
}  // namespace

void clear_error() { t_last_error[0] = '\0'; }

int fail(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof t_last_error, fmt, ap);
  va_end(ap);
  return code;
}

int fail_cuda(cudaError_t e, const char *what) {
  return fail(e == cudaErrorMemoryAllocation ? ATTN_ENOMEM : ATTN_ECUDA, "%s: %s", what,
              cudaGetErrorString(e));
}

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Injected workspace-allocation failures still to deliver
// (attn_sink_fail_workspace_allocs).
std::atomic<int> g_fail_allocs{0};
int *g_status_ptr[kMaxDevices];
cudaMemPool_t g_pool[kMaxDevices];
bool g_pool_ready[kMaxDevices];

}  // namespace

// True (and one fewer to come) while injected allocation failures are pending.
bool take_injected_alloc_failure() {
  int n = g_fail_allocs.load();
  while (n > 0)
    if (g_fail_allocs.compare_exchange_weak(n, n - 1)) return true;
  return false;
}

int current_device(int *dev) {
  const cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  if (*dev < 0 || *dev >= kMaxDevices) return fail(ATTN_EUNSUPPORTED, "device index %d", *dev);
  return ATTN_OK;
}

int status_ptr(int **out) {
  int dev;
  int rc = current_device(&dev);
  if (rc) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_status);
    if (e != cudaSuccess) return fail_cuda(e, "cudaGetSymbolAddress(status)");
    g_status_ptr[dev] = static_cast<int *>(p);
  }
  *out = g_status_ptr[dev];
  return ATTN_OK;
}

namespace {

// A private stream-ordered pool per device that keeps freed blocks cached, so
// repeated decode calls reuse their workspace without new mappings.
int workspace_pool(cudaMemPool_t *out) {
  int dev;
  int rc = current_device(&dev);
  if (rc) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_pool_ready[dev]) {
    cudaMemPoolProps props;
    memset(&props, 0, sizeof props);
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaError_t e = cudaMemPoolCreate(&g_pool[dev], &props);
    if (e != cudaSuccess) return fail_cuda(e, "cudaMemPoolCreate");
    uint64_t keep = ~0ull;
    e = cudaMemPoolSetAttribute(g_pool[dev], cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) return fail_cuda(e, "cudaMemPoolSetAttribute");
    g_pool_ready[dev] = true;
  }
  *out = g_pool[dev];
  return ATTN_OK;
}

// ------------------------------------------------------------ validation
const char *dtype_name(int32_t d) {
  switch (d) {
    case ATTN_DTYPE_BF16: return "bf16";
    case ATTN_DTYPE_F32: return "f32";
    case ATTN_DTYPE_I32: return "i32";
    case ATTN_DTYPE_E4M3: return "e4m3";
    default: return "unknown";
  }
}

int check_tensor(const attn_tensor *t, const char *name, int32_t dtype, int ndim, bool tma) {
  if (!t) return fail(ATTN_EINVAL, "%s: null tensor", name);
  if (t->dtype != dtype)
    return fail(ATTN_EINVAL, "%s: dtype %s, expected %s", name, dtype_name(t->dtype), dtype_name(dtype));
  if (t->ndim != ndim) return fail(ATTN_EINVAL, "%s: ndim %d, expected %d", name, t->ndim, ndim);
  int64_t numel = 1;
  for (int d = 0; d < ndim; ++d) {
    if (t->shape[d] < 0) return fail(ATTN_EINVAL, "%s: negative size in dim %d", name, d);
    numel *= t->shape[d];
  }
  if (numel > 0 && !t->data) return fail(ATTN_EINVAL, "%s: null data pointer", name);
  if (reinterpret_cast<uintptr_t>(t->data) % 16 != 0)
    return fail(ATTN_EINVAL, "%s: data pointer not 16-byte aligned", name);
  if (t->stride[ndim - 1] != 1 && t->shape[ndim - 1] > 1)
    return fail(ATTN_EINVAL, "%s: innermost stride must be 1", name);
  for (int d = 0; d < ndim - 1; ++d) {
    if (t->stride[d] <= 0) return fail(ATTN_EINVAL, "%s: stride of dim %d must be positive", name, d);
    const int64_t per16 = dtype == ATTN_DTYPE_E4M3 ? 16 : 8;   // elements per 16 bytes
    if (tma && t->stride[d] % per16 != 0)
      return fail(ATTN_EINVAL, "%s: stride of dim %d must be a multiple of %lld elements (16 bytes)", name,
                  d, (long long)per16);
  }
  return ATTN_OK;
}

bool finite_pos(float x) { return isfinite(x) && x > 0.f; }

int prep_fwd(const attn_tensor *q, const attn_tensor *k, const attn_tensor *v,
             const attn_tensor *sinks, int32_t window, float scale, attn_tensor *out,
             attn_tensor *lse, bool tma, FwdArgs *a) {
  int rc;
  if ((rc = check_tensor(q, "q", ATTN_DTYPE_BF16, 4, tma))) return rc;
  if ((rc = check_tensor(k, "k", ATTN_DTYPE_BF16, 4, tma))) return rc;
  if ((rc = check_tensor(v, "v", ATTN_DTYPE_BF16, 4, tma))) return rc;
  if ((rc = check_tensor(sinks, "sinks", ATTN_DTYPE_F32, 1, false))) return rc;
  if ((rc = check_tensor(out, "out", ATTN_DTYPE_BF16, 4, tma))) return rc;
  const int64_t B = q->shape[0], L = q->shape[1], Hq = q->shape[2], D = q->shape[3];
  const int64_t Hkv = k->shape[2];
  if (k->shape[0] != B || k->shape[1] != L || k->shape[3] != D)
    return fail(ATTN_EINVAL, "k shape does not match q");
  for (int d = 0; d < 4; ++d)
    if (v->shape[d] != k->shape[d]) return fail(ATTN_EINVAL, "v shape does not match k");
  for (int d = 0; d < 4; ++d)
    if (out->shape[d] != q->shape[d]) return fail(ATTN_EINVAL, "out shape does not match q");
  if (sinks->shape[0] != Hq) return fail(ATTN_EINVAL, "sinks must have Hq = %lld entries", (long long)Hq);
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return fail(ATTN_EINVAL, "Hq must be a positive multiple of Hkv");
  if (window < 1) return fail(ATTN_EINVAL, "window must be >= 1");
  if (!finite_pos(scale)) return fail(ATTN_EINVAL, "scale must be finite and > 0");
  if (lse) {
    if ((rc = check_tensor(lse, "lse", ATTN_DTYPE_F32, 3, false))) return rc;
    if (lse->shape[0] != B || lse->shape[1] != Hq || lse->shape[2] != L)
      return fail(ATTN_EINVAL, "lse must be [B, Hq, L]");
  }
  if (B > 65535 || Hq > 65535 || L > (1LL << 30))
    return fail(ATTN_EUNSUPPORTED, "B and Hq must be <= 65535 and L <= 2^30");
  a->q = q->data;
  a->k = k->data;
  a->v = v->data;
  a->sinks = static_cast<const float *>(sinks->data);
  a->out = out->data;
  a->lse = lse ? static_cast<float *>(lse->data) : nullptr;
  a->B = static_cast<int>(B);
  a->L = static_cast<int>(L);
  a->Hq = static_cast<int>(Hq);
  a->Hkv = static_cast<int>(Hkv);
  a->D = static_cast<int>(D);
  a->W = window;
  a->scale = scale;
  for (int d = 0; d < 3; ++d) {
    a->q_s[d] = q->stride[d];
    a->k_s[d] = k->stride[d];
    a->v_s[d] = v->stride[d];
    a->o_s[d] = out->stride[d];
  }
  a->lse_s[0] = lse ? lse->stride[0] : 0;
  a->lse_s[1] = lse ? lse->stride[1] : 0;
  if (sinks->shape[0] > 1 && sinks->stride[0] != 1) return fail(ATTN_EINVAL, "sinks must be contiguous");
  return ATTN_OK;
}

// Validates the packed variable-length forward's arguments and fills `a`.
int prep_fwd_varlen(const attn_tensor *q, const attn_tensor *k, const attn_tensor *v,
                    const attn_tensor *cu_seqlens, int32_t max_seqlen, const attn_tensor *sinks,
                    int32_t window, float scale, attn_tensor *out, attn_tensor *lse, FwdArgs *a) {
  int rc;
  if ((rc = check_tensor(q, "q", ATTN_DTYPE_BF16, 3, true))) return rc;
  if ((rc = check_tensor(k, "k", ATTN_DTYPE_BF16, 3, true))) return rc;
  if ((rc = check_tensor(v, "v", ATTN_DTYPE_BF16, 3, true))) return rc;
  if ((rc = check_tensor(cu_seqlens, "cu_seqlens", ATTN_DTYPE_I32, 1, false))) return rc;
  if ((rc = check_tensor(sinks, "sinks", ATTN_DTYPE_F32, 1, false))) return rc;
  if ((rc = check_tensor(out, "out", ATTN_DTYPE_BF16, 3, true))) return rc;
  const int64_t T = q->shape[0], Hq = q->shape[1], D = q->shape[2];
  const int64_t Hkv = k->shape[1];
  if (k->shape[0] != T || k->shape[2] != D) return fail(ATTN_EINVAL, "k shape does not match q");
  for (int d = 0; d < 3; ++d) {
    if (v->shape[d] != k->shape[d]) return fail(ATTN_EINVAL, "v shape does not match k");
    if (out->shape[d] != q->shape[d]) return fail(ATTN_EINVAL, "out shape does not match q");
  }
  if (cu_seqlens->shape[0] < 1) return fail(ATTN_EINVAL, "cu_seqlens needs B + 1 >= 1 entries");
  if (cu_seqlens->shape[0] > 1 && cu_seqlens->stride[0] != 1) return fail(ATTN_EINVAL, "cu_seqlens must be contiguous");
  if (sinks->shape[0] != Hq) return fail(ATTN_EINVAL, "sinks must have Hq = %lld entries", (long long)Hq);
  if (sinks->shape[0] > 1 && sinks->stride[0] != 1) return fail(ATTN_EINVAL, "sinks must be contiguous");
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return fail(ATTN_EINVAL, "Hq must be a positive multiple of Hkv");
  if (window < 1) return fail(ATTN_EINVAL, "window must be >= 1");
  if (max_seqlen < 0) return fail(ATTN_EINVAL, "max_seqlen must be >= 0");
  if (!finite_pos(scale)) return fail(ATTN_EINVAL, "scale must be finite and > 0");
  if (lse) {
    if ((rc = check_tensor(lse, "lse", ATTN_DTYPE_F32, 2, false))) return rc;
    if (lse->shape[0] != Hq || lse->shape[1] != T) return fail(ATTN_EINVAL, "lse must be [Hq, T]");
  }
  const int64_t B = cu_seqlens->shape[0] - 1;
  if (B > 65535 || Hq > 65535 || T > (1LL << 30))
    return fail(ATTN_EUNSUPPORTED, "B and Hq must be <= 65535 and T <= 2^30");
  a->q = q->data;
  a->k = k->data;
  a->v = v->data;
  a->sinks = static_cast<const float *>(sinks->data);
  a->out = out->data;
  a->lse = lse ? static_cast<float *>(lse->data) : nullptr;
  a->B = static_cast<int>(B);
  a->L = max_seqlen;
  a->T = static_cast<int>(T);
  a->Hq = static_cast<int>(Hq);
  a->Hkv = static_cast<int>(Hkv);
  a->D = static_cast<int>(D);
  a->W = window;
  a->scale = scale;
  a->cu_seqlens = static_cast<const int *>(cu_seqlens->data);
  // one batch slice of T rows: its (unused) batch stride spans the slice
  const attn_tensor *ts[4] = {q, k, v, out};
  int64_t *ss[4] = {a->q_s, a->k_s, a->v_s, a->o_s};
  for (int x = 0; x < 4; ++x) {
    ss[x][0] = (T > 0 ? T : 1) * ts[x]->stride[0];
    ss[x][1] = ts[x]->stride[0];
    ss[x][2] = ts[x]->stride[1];
  }
  a->lse_s[0] = 0;
  a->lse_s[1] = lse ? lse->stride[0] : 0;
  return ATTN_OK;
}

}  // namespace

// TMA descriptor for a [d3, d2, d1, d0] bf16 tensor, box {64, 1, box_rows, 1},
// 128-byte swizzle, zero fill out of range.  Encoded descriptors are kept in
// a small least-recently-used cache keyed by everything that determines them
// (address, sizes, strides, box), so repeated calls on the same buffers skip
// the driver call.
namespace {
struct TmaKey {
  const void *base;
  int64_t d[4], s[3];
  int box, elem;
  bool operator==(const TmaKey &o) const {
    return base == o.base && box == o.box && elem == o.elem && memcmp(d, o.d, sizeof d) == 0 &&
           memcmp(s, o.s, sizeof s) == 0;
  }
};
struct TmaEntry {
  TmaKey key;
  alignas(64) CUtensorMap map;
  uint64_t used;
  bool valid;
};
constexpr int kTmaCacheSize = 64;
TmaEntry g_tma_cache[kTmaCacheSize];
uint64_t g_tma_tick = 0;
std::mutex g_tma_mu;
}  // namespace

typedef CUresult (*tma_encode_fn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda); null if the driver does not provide it.
static tma_encode_fn tma_encode() {
  static tma_encode_fn encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<tma_encode_fn>(fn);
  });
  return encode;
}

static bool tma_cache_get(const TmaKey &key, void *map_out) {
  std::lock_guard<std::mutex> lk(g_tma_mu);
  for (TmaEntry &e : g_tma_cache)
    if (e.valid && e.key == key) {
      e.used = ++g_tma_tick;
      memcpy(map_out, &e.map, sizeof(CUtensorMap));
      return true;
    }
  return false;
}

static void tma_cache_put(const TmaKey &key, const CUtensorMap &map) {
  std::lock_guard<std::mutex> lk(g_tma_mu);
  TmaEntry *victim = &g_tma_cache[0];
  for (TmaEntry &e : g_tma_cache) {
    if (!e.valid) {
      victim = &e;
      break;
    }
    if (e.used < victim->used) victim = &e;
  }
  victim->key = key;
  memcpy(&victim->map, &map, sizeof(CUtensorMap));
  victim->used = ++g_tma_tick;
  victim->valid = true;
}

cudaError_t make_tma_bshd(void *map_out, const void *base, int64_t d3, int64_t d2, int64_t d1,
                          int64_t d0, const int64_t strides_el[3], int box_rows, int elem_bytes) {
  const tma_encode_fn encode = tma_encode();
  if (!encode) return cudaErrorNotSupported;
  TmaKey key;
  key.base = base;
  key.d[0] = d0;
  key.d[1] = d1;
  key.d[2] = d2;
  key.d[3] = d3;
  key.s[0] = strides_el[0];
  key.s[1] = strides_el[1];
  key.s[2] = strides_el[2];
  key.box = box_rows;
  key.elem = elem_bytes;
  if (tma_cache_get(key, map_out)) return cudaSuccess;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d0), static_cast<cuuint64_t>(d1),
                              static_cast<cuuint64_t>(d2), static_cast<cuuint64_t>(d3)};
  // byte strides of dims 1..3 (innermost first): head, position, batch
  const cuuint64_t eb = static_cast<cuuint64_t>(elem_bytes);
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(strides_el[2]) * eb,
                                 static_cast<cuuint64_t>(strides_el[1]) * eb,
                                 static_cast<cuuint64_t>(strides_el[0]) * eb};
  // 128 bytes of the innermost dimension per box row (the swizzle span); an
  // f32 map instead spans the whole row, unswizzled
  const bool f32 = elem_bytes == 4;
  if (f32 && (d0 > 256 || (d0 * 4) % 16 != 0)) return cudaErrorInvalidValue;
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(f32 ? d0 : 128 / elem_bytes), 1,
                             static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  alignas(64) CUtensorMap map;
  const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : f32         ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                               : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUresult r = encode(&map, dt, 4, const_cast<void *>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE,
                            f32 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  memcpy(map_out, &map, sizeof(CUtensorMap));
  tma_cache_put(key, map);
  return cudaSuccess;
}

cudaError_t make_tma_pages5d(void *map_out, const void *base, int64_t npages, int64_t page, int64_t H,
                             int64_t D, const int64_t strides_el[3]) {
  const tma_encode_fn encode = tma_encode();
  if (!encode) return cudaErrorNotSupported;
  if (D % 64 != 0 || page < 1 || page > 256) return cudaErrorInvalidValue;
  TmaKey key;
  key.base = base;
  key.d[0] = D;
  key.d[1] = H;
  key.d[2] = page;
  key.d[3] = npages;
  key.s[0] = strides_el[0];
  key.s[1] = strides_el[1];
  key.s[2] = strides_el[2];
  key.box = static_cast<int>(page);
  key.elem = -5;                     // (the 5-D page view; no 4-D map has this)
  if (tma_cache_get(key, map_out)) return cudaSuccess;
  const cuuint64_t dims[5] = {64, static_cast<cuuint64_t>(page), static_cast<cuuint64_t>(D / 64),
                              static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(npages)};
  // byte strides of dims 1..4: position in page, chunk, head, page
  const cuuint64_t strides[4] = {static_cast<cuuint64_t>(strides_el[1]) * 2, 128,
                                 static_cast<cuuint64_t>(strides_el[2]) * 2,
                                 static_cast<cuuint64_t>(strides_el[0]) * 2};
  const cuuint32_t box[5] = {64, static_cast<cuuint32_t>(page), static_cast<cuuint32_t>(D / 64), 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  alignas(64) CUtensorMap map;
  const CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  memcpy(map_out, &map, sizeof(CUtensorMap));
  tma_cache_put(key, map);
  return cudaSuccess;
}

// Validates the decode arguments and fills `out_args`; `*empty` is set when
// there is nothing to compute (B == 0 or Hq == 0).
int prep_decode(const attn_tensor *q, const attn_tensor *kcache, const attn_tensor *vcache,
                const attn_tensor *seqlens, const attn_tensor *sinks, int32_t window, float scale,
                int32_t chunk, attn_tensor *out, DecodeArgs *out_args, bool *empty) {
  int rc;
  *empty = false;
  if ((rc = check_tensor(q, "q", ATTN_DTYPE_BF16, 3, false))) return rc;
  if ((rc = check_tensor(kcache, "kcache", ATTN_DTYPE_BF16, 4, true))) return rc;
  if ((rc = check_tensor(vcache, "vcache", ATTN_DTYPE_BF16, 4, true))) return rc;
  if ((rc = check_tensor(seqlens, "seqlens", ATTN_DTYPE_I32, 1, false))) return rc;
  if ((rc = check_tensor(sinks, "sinks", ATTN_DTYPE_F32, 1, false))) return rc;
  if ((rc = check_tensor(out, "out", ATTN_DTYPE_BF16, 3, false))) return rc;
  const int64_t B = q->shape[0], Hq = q->shape[1], D = q->shape[2];
  const int64_t Smax = kcache->shape[1], Hkv = kcache->shape[2];
  if (kcache->shape[0] != B || kcache->shape[3] != D) return fail(ATTN_EINVAL, "kcache shape does not match q");
  for (int d = 0; d < 4; ++d)
    if (vcache->shape[d] != kcache->shape[d]) return fail(ATTN_EINVAL, "vcache shape does not match kcache");
  for (int d = 0; d < 3; ++d)
    if (out->shape[d] != q->shape[d]) return fail(ATTN_EINVAL, "out shape does not match q");
  if (seqlens->shape[0] != B) return fail(ATTN_EINVAL, "seqlens must have B entries");
  if (sinks->shape[0] != Hq) return fail(ATTN_EINVAL, "sinks must have Hq entries");
  if ((B > 1 && seqlens->stride[0] != 1) || (Hq > 1 && sinks->stride[0] != 1))
    return fail(ATTN_EINVAL, "seqlens and sinks must be contiguous");
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return fail(ATTN_EINVAL, "Hq must be a positive multiple of Hkv");
  if (window < 1) return fail(ATTN_EINVAL, "window must be >= 1");
  if (!finite_pos(scale)) return fail(ATTN_EINVAL, "scale must be finite and > 0");
  if (chunk < 0 || chunk % 64 != 0) return fail(ATTN_EINVAL, "chunk must be 0 or a positive multiple of 64");
  if (D != 64 && D != 128 && D != 256) return fail(ATTN_EUNSUPPORTED, "head dim %lld not supported", (long long)D);
  if (Hq / Hkv > (D == 256 ? 8 : 16)) return fail(ATTN_EUNSUPPORTED, "Hq/Hkv too large for this head dim");
  if ((reinterpret_cast<uintptr_t>(q->data) % 4) || q->stride[0] % 2 || q->stride[1] % 2)
    return fail(ATTN_EINVAL, "q rows must be 4-byte aligned");
  if (B > (1 << 20) || Smax > (1LL << 30)) return fail(ATTN_EUNSUPPORTED, "B or Smax too large");
  if (B == 0 || Hq == 0) {
    *empty = true;
    return ATTN_OK;
  }
  DecodeArgs &a = *out_args;
  a.q = q->data;
  a.kc = kcache->data;
  a.vc = vcache->data;
  a.seqlens = static_cast<const int *>(seqlens->data);
  a.sinks = static_cast<const float *>(sinks->data);
  a.out = out->data;
  a.B = static_cast<int>(B);
  a.Smax = static_cast<int>(Smax);
  a.Hq = static_cast<int>(Hq);
  a.Hkv = static_cast<int>(Hkv);
  a.D = static_cast<int>(D);
  a.W = window;
  a.scale = scale;
  const int64_t vis = window < Smax ? window : Smax;
  if (chunk == 0) {
    // keep every sequence within 32 splits (the exact small-split combine)
    int64_t c = ((vis + 31) / 32 + 63) / 64 * 64;
    chunk = static_cast<int32_t>(c < 256 ? 256 : c);
  }
  a.chunk = chunk;
  for (int d = 0; d < 2; ++d) {
    a.q_s[d] = q->stride[d];
    a.o_s[d] = out->stride[d];
  }
  for (int d = 0; d < 3; ++d) {
    a.kc_s[d] = kcache->stride[d];
    a.vc_s[d] = vcache->stride[d];
  }
  return ATTN_OK;
}

// Validates the backward's arguments and fills `a`.
int prep_bwd(const attn_tensor *q, const attn_tensor *k, const attn_tensor *v, const attn_tensor *o,
             const attn_tensor *lse, const attn_tensor *dout, const attn_tensor *sinks, int32_t window,
             float scale, attn_tensor *dq, attn_tensor *dk, attn_tensor *dv, attn_tensor *dsink, BwdArgs *a) {
  int rc;
  if ((rc = check_tensor(q, "q", ATTN_DTYPE_BF16, 4, true))) return rc;
  if ((rc = check_tensor(k, "k", ATTN_DTYPE_BF16, 4, true))) return rc;
  if ((rc = check_tensor(v, "v", ATTN_DTYPE_BF16, 4, true))) return rc;
  if ((rc = check_tensor(dout, "dout", ATTN_DTYPE_BF16, 4, true))) return rc;
  if (!o || (o->dtype != ATTN_DTYPE_BF16 && o->dtype != ATTN_DTYPE_F32))
    return fail(ATTN_EINVAL, "o: dtype must be bf16 or f32");
  if ((rc = check_tensor(o, "o", o->dtype, 4, false))) return rc;
  if ((rc = check_tensor(lse, "lse", ATTN_DTYPE_F32, 3, false))) return rc;
  if ((rc = check_tensor(sinks, "sinks", ATTN_DTYPE_F32, 1, false))) return rc;
  if ((rc = check_tensor(dq, "dq", ATTN_DTYPE_BF16, 4, true))) return rc;
  if ((rc = check_tensor(dk, "dk", ATTN_DTYPE_BF16, 4, true))) return rc;
  if ((rc = check_tensor(dv, "dv", ATTN_DTYPE_BF16, 4, true))) return rc;
  if ((rc = check_tensor(dsink, "dsink", ATTN_DTYPE_F32, 1, false))) return rc;
  const int64_t B = q->shape[0], L = q->shape[1], Hq = q->shape[2], D = q->shape[3], Hkv = k->shape[2];
  for (int d = 0; d < 4; ++d) {
    if (o->shape[d] != q->shape[d] || dout->shape[d] != q->shape[d] || dq->shape[d] != q->shape[d])
      return fail(ATTN_EINVAL, "o, dout and dq must have q's shape");
    if (v->shape[d] != k->shape[d] || dk->shape[d] != k->shape[d] || dv->shape[d] != k->shape[d])
      return fail(ATTN_EINVAL, "v, dk and dv must have k's shape");
  }
  if (k->shape[0] != B || k->shape[1] != L || k->shape[3] != D) return fail(ATTN_EINVAL, "k shape does not match q");
  if (lse->shape[0] != B || lse->shape[1] != Hq || lse->shape[2] != L) return fail(ATTN_EINVAL, "lse must be [B, Hq, L]");
  if (sinks->shape[0] != Hq || dsink->shape[0] != Hq) return fail(ATTN_EINVAL, "sinks and dsink must have Hq entries");
  if ((Hq > 1 && (sinks->stride[0] != 1 || dsink->stride[0] != 1)))
    return fail(ATTN_EINVAL, "sinks and dsink must be contiguous");
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return fail(ATTN_EINVAL, "Hq must be a positive multiple of Hkv");
  if (window < 1) return fail(ATTN_EINVAL, "window must be >= 1");
  if (!finite_pos(scale)) return fail(ATTN_EINVAL, "scale must be finite and > 0");
  if (D != 64 && D != 128) return fail(ATTN_EUNSUPPORTED, "backward: head dim %lld not supported (64, 128)", (long long)D);
  if (B > 65535 || Hkv > 65535 || L > (1LL << 28)) return fail(ATTN_EUNSUPPORTED, "B, Hkv or L too large");
  a->q = q->data;
  a->k = k->data;
  a->v = v->data;
  a->o = o->data;
  a->dout = dout->data;
  a->lse = static_cast<const float *>(lse->data);
  a->sinks = static_cast<const float *>(sinks->data);
  a->dq = dq->data;
  a->dk = dk->data;
  a->dv = dv->data;
  a->dsink = static_cast<float *>(dsink->data);
  a->B = static_cast<int>(B);
  a->L = static_cast<int>(L);
  a->Hq = static_cast<int>(Hq);
  a->Hkv = static_cast<int>(Hkv);
  a->D = static_cast<int>(D);
  a->W = window;
  a->scale = scale;
  a->o_f32 = o->dtype == ATTN_DTYPE_F32;
  for (int d = 0; d < 3; ++d) {
    a->q_s[d] = q->stride[d];
    a->k_s[d] = k->stride[d];
    a->v_s[d] = v->stride[d];
    a->o_s[d] = o->stride[d];
    a->do_s[d] = dout->stride[d];
    a->dq_s[d] = dq->stride[d];
    a->dk_s[d] = dk->stride[d];
    a->dv_s[d] = dv->stride[d];
  }
  a->lse_s[0] = lse->stride[0];
  a->lse_s[1] = lse->stride[1];
  return status_ptr(&a->status);
}

// Validates the paged-cache decode arguments and fills `out_args` (kc/vc are
// the page pools, Smax = pages per sequence * page size); `*empty` as above.
int prep_decode_paged(const attn_tensor *q, const attn_tensor *kpages, const attn_tensor *vpages,
                      const attn_tensor *block_table, const attn_tensor *seqlens,
                      const attn_tensor *sinks, int32_t window, float scale, attn_tensor *out,
                      DecodeArgs *out_args, bool *empty) {
  int rc;
  *empty = false;
  if ((rc = check_tensor(q, "q", ATTN_DTYPE_BF16, 3, false))) return rc;
  if ((rc = check_tensor(kpages, "kpages", ATTN_DTYPE_BF16, 4, true))) return rc;
  if ((rc = check_tensor(vpages, "vpages", ATTN_DTYPE_BF16, 4, true))) return rc;
  if ((rc = check_tensor(block_table, "block_table", ATTN_DTYPE_I32, 2, false))) return rc;
  if ((rc = check_tensor(seqlens, "seqlens", ATTN_DTYPE_I32, 1, false))) return rc;
  if ((rc = check_tensor(sinks, "sinks", ATTN_DTYPE_F32, 1, false))) return rc;
  if ((rc = check_tensor(out, "out", ATTN_DTYPE_BF16, 3, false))) return rc;
  const int64_t B = q->shape[0], Hq = q->shape[1], D = q->shape[2];
  const int64_t NB = kpages->shape[0], P = kpages->shape[1], Hkv = kpages->shape[2];
  const int64_t MP = block_table->shape[1];
  if (kpages->shape[3] != D) return fail(ATTN_EINVAL, "kpages head dim does not match q");
  for (int d = 0; d < 4; ++d)
    if (vpages->shape[d] != kpages->shape[d]) return fail(ATTN_EINVAL, "vpages shape does not match kpages");
  for (int d = 0; d < 3; ++d)
    if (out->shape[d] != q->shape[d]) return fail(ATTN_EINVAL, "out shape does not match q");
  if (block_table->shape[0] != B) return fail(ATTN_EINVAL, "block_table must have B rows");
  if (seqlens->shape[0] != B) return fail(ATTN_EINVAL, "seqlens must have B entries");
  if (sinks->shape[0] != Hq) return fail(ATTN_EINVAL, "sinks must have Hq entries");
  if ((B > 1 && seqlens->stride[0] != 1) || (Hq > 1 && sinks->stride[0] != 1))
    return fail(ATTN_EINVAL, "seqlens and sinks must be contiguous");
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return fail(ATTN_EINVAL, "Hq must be a positive multiple of Hkv");
  if (P < 16 || P > 65536 || (P & (P - 1)))
    return fail(ATTN_EUNSUPPORTED, "page size %lld must be a power of two in [16, 65536]", (long long)P);
  if (window < 1) return fail(ATTN_EINVAL, "window must be >= 1");
  if (!finite_pos(scale)) return fail(ATTN_EINVAL, "scale must be finite and > 0");
  if (D != 64 && D != 128 && D != 256) return fail(ATTN_EUNSUPPORTED, "head dim %lld not supported", (long long)D);
  if (Hq / Hkv > (D == 256 ? 8 : 16)) return fail(ATTN_EUNSUPPORTED, "Hq/Hkv too large for this head dim");
  if ((reinterpret_cast<uintptr_t>(q->data) % 4) || q->stride[0] % 2 || q->stride[1] % 2)
    return fail(ATTN_EINVAL, "q rows must be 4-byte aligned");
  if (B > (1 << 20) || NB > (1LL << 31) - 1 || MP * P > (1LL << 30))
    return fail(ATTN_EUNSUPPORTED, "B, the pool or pages per sequence * page size too large");
  if (B == 0 || Hq == 0) {
    *empty = true;
    return ATTN_OK;
  }
  DecodeArgs &a = *out_args;
  a.q = q->data;
  a.kc = kpages->data;
  a.vc = vpages->data;
  a.seqlens = static_cast<const int *>(seqlens->data);
  a.sinks = static_cast<const float *>(sinks->data);
  a.out = out->data;
  a.B = static_cast<int>(B);
  a.Smax = static_cast<int>(MP * P);
  a.Hq = static_cast<int>(Hq);
  a.Hkv = static_cast<int>(Hkv);
  a.D = static_cast<int>(D);
  a.W = window;
  a.scale = scale;
  // keep every sequence within 32 splits; the range may start 63 keys early
  const int64_t vis = (window < a.Smax ? window : a.Smax) + 63;
  int64_t c = ((vis + 31) / 32 + 63) / 64 * 64;
  a.chunk = static_cast<int32_t>(c < 256 ? 256 : c);
  for (int d = 0; d < 2; ++d) {
    a.q_s[d] = q->stride[d];
    a.o_s[d] = out->stride[d];
  }
  for (int d = 0; d < 3; ++d) {
    a.kc_s[d] = kpages->stride[d];
    a.vc_s[d] = vpages->stride[d];
  }
  a.block_table = static_cast<const int *>(block_table->data);
  a.bt_s0 = block_table->stride[0];
  a.page = static_cast<int>(P);
  a.npages = static_cast<int>(NB);
  a.max_pages = static_cast<int>(MP);
  return ATTN_OK;
}

// Validates the FP8-cache decode arguments: as prep_decode, with e4m3 caches
// and the two [Hkv] f32 descale vectors.
int prep_decode_fp8(const attn_tensor *q, const attn_tensor *kcache, const attn_tensor *vcache,
                    const attn_tensor *k_descale, const attn_tensor *v_descale,
                    const attn_tensor *seqlens, const attn_tensor *sinks, int32_t window, float scale,
                    attn_tensor *out, DecodeArgs *out_args, bool *empty) {
  int rc;
  if ((rc = check_tensor(kcache, "kcache", ATTN_DTYPE_E4M3, 4, true))) return rc;
  if ((rc = check_tensor(vcache, "vcache", ATTN_DTYPE_E4M3, 4, true))) return rc;
  if ((rc = check_tensor(k_descale, "k_descale", ATTN_DTYPE_F32, 1, false))) return rc;
  if ((rc = check_tensor(v_descale, "v_descale", ATTN_DTYPE_F32, 1, false))) return rc;
  const int64_t Hkv = kcache->shape[2], D = kcache->shape[3];
  if (k_descale->shape[0] != Hkv || v_descale->shape[0] != Hkv)
    return fail(ATTN_EINVAL, "k_descale and v_descale must have Hkv = %lld entries", (long long)Hkv);
  if ((Hkv > 1 && (k_descale->stride[0] != 1 || v_descale->stride[0] != 1)))
    return fail(ATTN_EINVAL, "descales must be contiguous");
  if (D != 128 && D != 256) return fail(ATTN_EUNSUPPORTED, "FP8 cache: head dim %lld not supported (128, 256)", (long long)D);
  // the remaining checks are those of the bf16 decode, on shape-only copies
  attn_tensor kc = *kcache, vc = *vcache;
  kc.dtype = vc.dtype = ATTN_DTYPE_BF16;
  for (int d = 0; d < 3; ++d) {
    if (kc.stride[d] % 16 != 0 || vc.stride[d] % 16 != 0)
      return fail(ATTN_EINVAL, "FP8 cache strides must be multiples of 16 elements");
  }
  if ((rc = prep_decode(q, &kc, &vc, seqlens, sinks, window, scale, 0, out, out_args, empty))) return rc;
  // whole tiles per split, so that no tile reads into the next split's keys
  out_args->fp8 = true;
  const int tile = decode_tile_keys(*out_args);
  out_args->chunk = (out_args->chunk + tile - 1) / tile * tile;
  out_args->k_descale = static_cast<const float *>(k_descale->data);
  out_args->v_descale = static_cast<const float *>(v_descale->data);
  return ATTN_OK;
}

}  // namespace attnsink

using namespace attnsink;

extern "C" {

const char *attn_sink_strerror(int code) {
  switch (code) {
    case ATTN_OK: return "success";
    case ATTN_EINVAL: return "invalid argument";
    case ATTN_EUNSUPPORTED: return "unsupported configuration";
    case ATTN_ECUDA: return "CUDA runtime error";
    case ATTN_ENOMEM: return "workspace allocation failed";
    case ATTN_ETIMEOUT: return "device-side wait timed out";
    default: return "unknown error";
  }
}

const char *attn_sink_last_error(void) { return t_last_error; }

int attn_sink_fwd(const attn_tensor *q, const attn_tensor *k, const attn_tensor *v,
                  const attn_tensor *sinks, int32_t window, float scale, attn_tensor *out,
                  attn_tensor *lse, void *stream) {
  t_last_error[0] = '\0';
  FwdArgs a;
  int rc = prep_fwd(q, k, v, sinks, window, scale, out, lse, true, &a);
  if (rc) return rc;
  if (a.D != 64 && a.D != 128 && a.D != 256)
    return fail(ATTN_EUNSUPPORTED, "head dim %d not supported (64, 128, 256)", a.D);
  if (a.B == 0 || a.L == 0) return ATTN_OK;
  if ((rc = status_ptr(&a.status))) return rc;
  const cudaError_t e = launch_fwd_tc(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : fail_cuda(e, "attn_sink_fwd launch");
}

int attn_sink_fwd_max_logit(const attn_tensor *q, const attn_tensor *k, const attn_tensor *v,
                            const attn_tensor *sinks, int32_t window, float scale, attn_tensor *out,
                            attn_tensor *lse, attn_tensor *max_logit, void *stream) {
  t_last_error[0] = '\0';
  FwdArgs a;
  int rc = prep_fwd(q, k, v, sinks, window, scale, out, lse, true, &a);
  if (rc) return rc;
  if (a.D != 64 && a.D != 128 && a.D != 256)
    return fail(ATTN_EUNSUPPORTED, "head dim %d not supported (64, 128, 256)", a.D);
  if ((rc = check_tensor(max_logit, "max_logit", ATTN_DTYPE_F32, 2, false))) return rc;
  if (max_logit->shape[0] != a.B || max_logit->shape[1] != a.Hq)
    return fail(ATTN_EINVAL, "max_logit must be [B, Hq]");
  if (a.B == 0 || a.Hq == 0) return ATTN_OK;
  a.max_logit = static_cast<float *>(max_logit->data);
  a.ml_sb = max_logit->stride[0];
  if (a.L == 0) {
    // no position anywhere: every maximum is -inf and there is nothing else
    const cudaError_t e = launch_max_logit_init(a.max_logit, a.ml_sb, a.B, a.Hq,
                                                static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ATTN_OK : fail_cuda(e, "attn_sink_fwd_max_logit launch");
  }
  if ((rc = status_ptr(&a.status))) return rc;
  const cudaError_t e = launch_fwd_tc(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : fail_cuda(e, "attn_sink_fwd_max_logit launch");
}

int attn_sink_fwd_varlen(const attn_tensor *q, const attn_tensor *k, const attn_tensor *v,
                         const attn_tensor *cu_seqlens, int32_t max_seqlen,
                         const attn_tensor *sinks, int32_t window, float scale, attn_tensor *out,
                         attn_tensor *lse, void *stream) {
  t_last_error[0] = '\0';
  FwdArgs a;
  int rc = prep_fwd_varlen(q, k, v, cu_seqlens, max_seqlen, sinks, window, scale, out, lse, &a);
  if (rc) return rc;
  if (a.D != 64 && a.D != 128 && a.D != 256)
    return fail(ATTN_EUNSUPPORTED, "head dim %d not supported (64, 128, 256)", a.D);
  if (a.B == 0 || a.T == 0 || a.L == 0) return ATTN_OK;
  if ((rc = status_ptr(&a.status))) return rc;
  const cudaError_t e = launch_fwd_tc(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : fail_cuda(e, "attn_sink_fwd_varlen launch");
}

int attn_sink_fwd_cudacore(const attn_tensor *q, const attn_tensor *k, const attn_tensor *v,
                           const attn_tensor *sinks, int32_t window, float scale,
                           attn_tensor *out, attn_tensor *lse, void *stream) {
  t_last_error[0] = '\0';
  FwdArgs a;
  int rc = prep_fwd(q, k, v, sinks, window, scale, out, lse, false, &a);
  if (rc) return rc;
  if (a.D % 32 != 0 || a.D < 32 || a.D > 256)
    return fail(ATTN_EUNSUPPORTED, "head dim %d not supported (multiple of 32, <= 256)", a.D);
  if (a.B == 0 || a.L == 0) return ATTN_OK;
  if ((rc = status_ptr(&a.status))) return rc;
  const cudaError_t e = launch_fwd_cudacore(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : fail_cuda(e, "attn_sink_fwd_cudacore launch");
}

int attn_sink_decode_chunked(const attn_tensor *q, const attn_tensor *kcache,
                             const attn_tensor *vcache, const attn_tensor *seqlens,
                             const attn_tensor *sinks, int32_t window, float scale,
                             int32_t chunk, attn_tensor *out, void *stream) {
  t_last_error[0] = '\0';
  DecodeArgs a;
  bool empty;
  int rc = prep_decode(q, kcache, vcache, seqlens, sinks, window, scale, chunk, out, &a, &empty);
  if (rc || empty) return rc;
  if ((rc = status_ptr(&a.status))) return rc;
  cudaMemPool_t pool;
  if ((rc = workspace_pool(&pool))) return rc;
  const size_t bytes = decode_workspace_bytes(a);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void *ws = nullptr;
  if (take_injected_alloc_failure()) return fail(ATTN_ENOMEM, "decode workspace allocation failed (injected)");
  cudaError_t e = cudaMallocFromPoolAsync(&ws, bytes, pool, st);
  if (e != cudaSuccess) return fail_cuda(e, "decode workspace allocation");
  e = launch_decode(a, ws, st);
  const cudaError_t ef = cudaFreeAsync(ws, st);
  if (e != cudaSuccess) return fail_cuda(e, "attn_sink_decode launch");
  if (ef != cudaSuccess) return fail_cuda(ef, "decode workspace release");
  return ATTN_OK;
}

int attn_sink_decode(const attn_tensor *q, const attn_tensor *kcache, const attn_tensor *vcache,
                     const attn_tensor *seqlens, const attn_tensor *sinks, int32_t window,
                     float scale, attn_tensor *out, void *stream) {
  return attn_sink_decode_chunked(q, kcache, vcache, seqlens, sinks, window, scale, 0, out, stream);
}

int attn_sink_decode_paged(const attn_tensor *q, const attn_tensor *kpages,
                           const attn_tensor *vpages, const attn_tensor *block_table,
                           const attn_tensor *seqlens, const attn_tensor *sinks, int32_t window,
                           float scale, attn_tensor *out, void *stream) {
  t_last_error[0] = '\0';
  DecodeArgs a;
  bool empty;
  int rc = prep_decode_paged(q, kpages, vpages, block_table, seqlens, sinks, window, scale, out, &a,
                             &empty);
  if (rc || empty) return rc;
  if ((rc = status_ptr(&a.status))) return rc;
  cudaMemPool_t pool;
  if ((rc = workspace_pool(&pool))) return rc;
  const size_t bytes = decode_workspace_bytes(a);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void *ws = nullptr;
  if (take_injected_alloc_failure()) return fail(ATTN_ENOMEM, "decode workspace allocation failed (injected)");
  cudaError_t e = cudaMallocFromPoolAsync(&ws, bytes, pool, st);
  if (e != cudaSuccess) return fail_cuda(e, "decode workspace allocation");
  e = launch_decode(a, ws, st);
  const cudaError_t ef = cudaFreeAsync(ws, st);
  if (e != cudaSuccess) return fail_cuda(e, "attn_sink_decode_paged launch");
  if (ef != cudaSuccess) return fail_cuda(ef, "decode workspace release");
  return ATTN_OK;
}

int attn_sink_decode_fp8(const attn_tensor *q, const attn_tensor *kcache, const attn_tensor *vcache,
                         const attn_tensor *k_descale, const attn_tensor *v_descale,
                         const attn_tensor *seqlens, const attn_tensor *sinks, int32_t window,
                         float scale, attn_tensor *out, void *stream) {
  t_last_error[0] = '\0';
  DecodeArgs a;
  bool empty;
  int rc = prep_decode_fp8(q, kcache, vcache, k_descale, v_descale, seqlens, sinks, window, scale, out, &a,
                           &empty);
  if (rc || empty) return rc;
  if ((rc = status_ptr(&a.status))) return rc;
  cudaMemPool_t pool;
  if ((rc = workspace_pool(&pool))) return rc;
  const size_t bytes = decode_workspace_bytes(a);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void *ws = nullptr;
  if (take_injected_alloc_failure()) return fail(ATTN_ENOMEM, "decode workspace allocation failed (injected)");
  cudaError_t e = cudaMallocFromPoolAsync(&ws, bytes, pool, st);
  if (e != cudaSuccess) return fail_cuda(e, "decode workspace allocation");
  e = launch_decode(a, ws, st);
  const cudaError_t ef = cudaFreeAsync(ws, st);
  if (e != cudaSuccess) return fail_cuda(e, "attn_sink_decode_fp8 launch");
  if (ef != cudaSuccess) return fail_cuda(ef, "decode workspace release");
  return ATTN_OK;
}

int attn_sink_bwd(const attn_tensor *q, const attn_tensor *k, const attn_tensor *v, const attn_tensor *o,
                  const attn_tensor *lse, const attn_tensor *dout, const attn_tensor *sinks, int32_t window,
                  float scale, attn_tensor *dq, attn_tensor *dk, attn_tensor *dv, attn_tensor *dsink,
                  void *stream) {
  t_last_error[0] = '\0';
  BwdArgs a;
  int rc = prep_bwd(q, k, v, o, lse, dout, sinks, window, scale, dq, dk, dv, dsink, &a);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (a.B == 0 || a.L == 0) {
    const cudaError_t e = cudaMemsetAsync(a.dsink, 0, sizeof(float) * a.Hq, st);
    return e == cudaSuccess ? ATTN_OK : fail_cuda(e, "attn_sink_bwd");
  }
  cudaMemPool_t pool;
  if ((rc = workspace_pool(&pool))) return rc;
  void *ws = nullptr;
  if (take_injected_alloc_failure()) return fail(ATTN_ENOMEM, "backward workspace allocation failed (injected)");
  cudaError_t e = cudaMallocFromPoolAsync(&ws, bwd_workspace_bytes(a), pool, st);
  if (e != cudaSuccess) return fail_cuda(e, "backward workspace allocation");
  e = launch_bwd(a, ws, st);
  const cudaError_t ef = cudaFreeAsync(ws, st);
  if (e != cudaSuccess) return fail_cuda(e, "attn_sink_bwd launch");
  if (ef != cudaSuccess) return fail_cuda(ef, "backward workspace release");
  return ATTN_OK;
}

int attn_sink_set_wait_limit_ns(uint64_t ns) {
  t_last_error[0] = '\0';
  int *dptr = nullptr;
  int rc = status_ptr(&dptr);
  if (rc) return rc;
  const unsigned long long v = ns;
  const cudaError_t e = cudaMemcpy(dptr + 2, &v, sizeof v, cudaMemcpyHostToDevice);
  return e == cudaSuccess ? ATTN_OK : fail_cuda(e, "wait limit");
}

int attn_sink_fail_workspace_allocs(int32_t count) {
  t_last_error[0] = '\0';
  if (count < 0) return fail(ATTN_EINVAL, "count must be >= 0");
  g_fail_allocs.store(count);
  return ATTN_OK;
}

int attn_sink_get_status(void *stream) {
  t_last_error[0] = '\0';
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "cudaStreamSynchronize");
  int *dptr;
  int rc = status_ptr(&dptr);
  if (rc) return rc;
  int h[2] = {0, 0};
  e = cudaMemcpy(h, dptr, sizeof h, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail_cuda(e, "status read");
  if (h[0] != 0) {
    const int zero[2] = {0, 0};
    e = cudaMemcpy(dptr, zero, sizeof zero, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return fail_cuda(e, "status reset");
    return fail(h[0], "device wait timed out at location %d", h[1]);
  }
  return ATTN_OK;
}

}  // extern "C"
