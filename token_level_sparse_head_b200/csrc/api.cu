// C ABI of libsas (declared in include/sas.h): host-side validation, workspace layout and
// kernel launches.  Nothing here allocates device memory or synchronises, except the
// debugging call sas_check_workspace.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <array>
#include <mutex>
#include <unordered_map>

#include <cuda.h>  // driver types only (CUcontext, CUresult); no driver library is linked

#include "sas.h"
#include "sas_kernels.h"

namespace sas {

namespace {
using PfnCtxGetCurrent = CUresult (*)(CUcontext*);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long*);
struct CtxQuery {
  PfnCtxGetCurrent get_current = nullptr;
  PfnCtxGetId get_id = nullptr;
  cudaError_t status = cudaErrorNotSupported;
  CtxQuery() {
    cudaDriverEntryPointQueryResult q1, q2;
    cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", reinterpret_cast<void**>(&get_current),
                                            cudaEnableDefault, &q1);
    if (e == cudaSuccess)
      e = cudaGetDriverEntryPoint("cuCtxGetId", reinterpret_cast<void**>(&get_id), cudaEnableDefault, &q2);
    if (e != cudaSuccess) status = e;
    else if (q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess) status = cudaErrorNotSupported;
    else status = cudaSuccess;
  }
};
}  // namespace

// Id of the context current on this thread (driver entry points resolved once, thread-safely,
// through the runtime, so the library links no driver library); 0 when there is none yet.
cudaError_t current_context_id(unsigned long long* id) {
  static const CtxQuery q;
  if (q.status != cudaSuccess) return q.status;
  CUcontext ctx = nullptr;
  if (q.get_current(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
  *id = 0;
  if (ctx != nullptr && q.get_id(ctx, id) != CUDA_SUCCESS) return cudaErrorUnknown;
  return cudaSuccess;
}

// Kernel attributes belong to the context: the limit set for a kernel is remembered per device
// together with the id of the context it was set in, and set again in a new context.
cudaError_t prepare_kernel(const void* kern, int smem_bytes, bool nonportable_cluster) {
  constexpr int kDevices = 64;
  struct Allowed {
    int bytes;
    bool nonportable;
    unsigned long long ctx_id;
  };
  static std::mutex mu;
  static std::unordered_map<const void*, std::array<Allowed, kDevices>> allowed;  // per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  unsigned long long ctx_id = 0;
  e = current_context_id(&ctx_id);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  Allowed* lim = nullptr;
  if (dev >= 0 && dev < kDevices) {
    auto it = allowed.find(kern);
    if (it == allowed.end()) {
      std::array<Allowed, kDevices> none;
      none.fill(Allowed{-1, false, 0});
      it = allowed.emplace(kern, none).first;
    }
    lim = &it->second[dev];
    if (ctx_id != 0 && lim->ctx_id == ctx_id && lim->bytes >= smem_bytes && (lim->nonportable || !nonportable_cluster))
      return cudaSuccess;
  }
  // Never lower a limit already set in this context (another launch of the kernel may need it).
  const int bytes = (lim != nullptr && ctx_id != 0 && lim->ctx_id == ctx_id && lim->bytes > smem_bytes) ? lim->bytes
                                                                                                     : smem_bytes;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && nonportable_cluster)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess && lim != nullptr) {
    if (ctx_id == 0) current_context_id(&ctx_id);  // the call above made the primary context current
    if (lim->ctx_id != ctx_id) {
      lim->bytes = -1;
      lim->nonportable = false;
    }
    if (bytes > lim->bytes) lim->bytes = bytes;
    if (nonportable_cluster) lim->nonportable = true;
    lim->ctx_id = ctx_id;
  }
  return e;
}

int ctas_per_sm(const void* kern, int threads, int smem_bytes) {
  struct Key {
    const void* k;
    int dev, threads, smem;
    bool operator==(const Key& o) const { return k == o.k && dev == o.dev && threads == o.threads && smem == o.smem; }
  };
  struct Hash {
    size_t operator()(const Key& x) const {
      return std::hash<const void*>()(x.k) ^ ((size_t)x.dev << 48) ^ ((size_t)x.threads << 32) ^ (size_t)x.smem;
    }
  };
  static std::mutex mu;
  static std::unordered_map<Key, int, Hash> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  const Key key{kern, dev, threads, smem_bytes};
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, (size_t)smem_bytes) != cudaSuccess || n < 1) n = 1;
  cache.emplace(key, n);
  return n;
}

}  // namespace sas

namespace {

thread_local char g_detail[512] = {0};

sas_status fail(sas_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
  return s;
}

sas_status cuda_fail(cudaError_t e, const char* where) {
  return fail(SAS_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cap_of(const sas_shape* s) { return s->page_size ? s->max_pages * s->page_size : s->n_cap; }

sas_status check_shape(const sas_shape* s) {
  if (s == nullptr) return fail(SAS_ERR_INVALID_ARG, "shape is NULL");
  if (s->B < 1 || s->Hq < 1 || s->Hkv < 1) return fail(SAS_ERR_INVALID_ARG, "B, Hq, Hkv must be >= 1");
  if (s->Hq % s->Hkv) return fail(SAS_ERR_INVALID_ARG, "Hq (%d) is not a multiple of Hkv (%d)", s->Hq, s->Hkv);
  if (s->d != 64 && s->d != 128) return fail(SAS_ERR_UNSUPPORTED, "head dim d=%d (supported: 64, 128)", s->d);
  if (s->r != 16 && s->r != 32 && s->r != 64) return fail(SAS_ERR_UNSUPPORTED, "rank r=%d (supported: 16, 32, 64)", s->r);
  if (s->r > s->d) return fail(SAS_ERR_INVALID_ARG, "rank r=%d exceeds d=%d", s->r, s->d);
  if (s->kproj_dtype != SAS_KPROJ_BF16 && s->kproj_dtype != SAS_KPROJ_FP8_E4M3)
    return fail(SAS_ERR_UNSUPPORTED, "kproj_dtype %d", s->kproj_dtype);
  if (s->kproj_dtype == SAS_KPROJ_FP8_E4M3) {
    if (s->kproj_scale == nullptr) return fail(SAS_ERR_INVALID_ARG, "FP8 projected cache needs kproj_scale");
    if ((reinterpret_cast<uintptr_t>(s->kproj_scale) & 3u) != 0)
      return fail(SAS_ERR_INVALID_ARG, "kproj_scale is not 4-byte aligned");
  }
  if (s->page_size == 0) {
    if (s->n_cap < 4 || (s->n_cap % 4)) return fail(SAS_ERR_INVALID_ARG, "n_cap=%d must be a positive multiple of 4", s->n_cap);
    if ((long long)s->B * s->Hkv * s->n_cap >= (1LL << 32)) return fail(SAS_ERR_UNSUPPORTED, "cache rows exceed 2^32");
  } else if (s->page_size == 64) {
    if (s->max_pages < 1 || s->num_pages < 1) return fail(SAS_ERR_INVALID_ARG, "paged layout needs max_pages, num_pages >= 1");
    if ((long long)s->num_pages * s->Hkv * 64 >= (1LL << 32)) return fail(SAS_ERR_UNSUPPORTED, "cache rows exceed 2^32");
  } else {
    return fail(SAS_ERR_UNSUPPORTED, "page_size=%d (supported: 0 contiguous, 64 paged)", s->page_size);
  }
  if (cap_of(s) > SAS_MAX_CAPACITY) return fail(SAS_ERR_UNSUPPORTED, "capacity %d exceeds %d", cap_of(s), SAS_MAX_CAPACITY);
  if ((long long)s->B * s->Hkv > 65535) return fail(SAS_ERR_UNSUPPORTED, "B*Hkv exceeds 65535");
  return SAS_OK;
}

sas_status check_ptr(const void* p, const char* name, bool required = true) {
  if (p == nullptr) return required ? fail(SAS_ERR_INVALID_ARG, "%s is NULL", name) : SAS_OK;
  if (!aligned16(p)) return fail(SAS_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return SAS_OK;
}

#define SAS_TRY(expr)                 \
  do {                                \
    const sas_status _s = (expr);     \
    if (_s != SAS_OK) return _s;      \
  } while (0)

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

constexpr size_t kErrBytes = 256;

sas::AttendParams attend_plan(const sas_shape* s, int count_max, bool dense) {
  sas::AttendParams a = {};
  a.B = s->B; a.Hq = s->Hq; a.Hkv = s->Hkv; a.G = s->Hq / s->Hkv; a.d = s->d;
  a.cap = cap_of(s);
  sas::plan_attend(a, count_max, dense);
  return a;
}

// Workspace: [0,256) error word | key histograms | attention partials | score keys.
// The histograms sit at a fixed offset: they must stay zero between calls (the selection clears
// them after use), whatever other calls (dense decode, other budgets) share the workspace;
// partials and keys are rewritten by every call.
struct WsLayout {
  size_t hist, partials, keys, total;
};

WsLayout ws_layout(const sas::AttendParams& a, bool with_keys) {
  WsLayout w;
  size_t o = kErrBytes;
  w.hist = o;
  o += (size_t)a.B * a.Hkv * sas::kHistBins * 4;
  w.partials = o;
  o += (sas::attend_workspace_floats(a) * 4 + 255) & ~(size_t)255;
  w.keys = o;
  if (with_keys) o += ((size_t)a.B * a.Hkv * a.cap * 4 + 255) & ~(size_t)255;
  w.total = o;
  return w;
}

size_t ws_bytes_for(const sas::AttendParams& a, bool with_keys) { return ws_layout(a, with_keys).total; }

void bind_workspace(sas::AttendParams& a, void* ws) {
  unsigned char* w = static_cast<unsigned char*>(ws);
  const WsLayout L = ws_layout(a, false);
  a.err = reinterpret_cast<uint32_t*>(w);
  a.partials = reinterpret_cast<float*>(w + L.partials);
}

sas_status check_cache_ptrs(const sas_shape* s, const int32_t* page_table, const int32_t* seqlens) {
  SAS_TRY(check_ptr(seqlens, "seqlens"));
  if (s->page_size) SAS_TRY(check_ptr(page_table, "page_table"));
  return SAS_OK;
}

struct SelectPlan {
  sas::ScoreParams sp;
  sas::SelectParams sl;
};

sas_status plan_selection(const sas_shape* s, const void* q, const float* M, const void* Kproj,
                          const int32_t* page_table, const int32_t* seqlens, const int32_t* k, int32_t k_max,
                          float lambda, const float* log_g, int32_t* idx_out, float* scores_out, void* ws,
                          SelectPlan* out) {
  const sas::AttendParams a = attend_plan(s, k_max, false);
  const WsLayout L = ws_layout(a, true);
  unsigned char* w = static_cast<unsigned char*>(ws);
  const int sms = num_sms();

  sas::ScoreParams& sp = out->sp;
  sp = {};
  sp.q = static_cast<const __nv_bfloat16*>(q);
  sp.M = M;
  sp.kproj = Kproj;
  sp.fp8 = s->kproj_dtype == SAS_KPROJ_FP8_E4M3 ? 1 : 0;
  sp.kproj_scale = s->kproj_scale;
  sp.page_table = s->page_size ? page_table : nullptr;
  sp.seqlens = seqlens;
  sp.kvec = k;
  sp.log_g = (lambda != 0.0f) ? log_g : nullptr;
  sp.keys = reinterpret_cast<uint32_t*>(w + L.keys);
  sp.hist = reinterpret_cast<uint32_t*>(w + L.hist);
  sp.scores_out = scores_out;
  sp.err = reinterpret_cast<uint32_t*>(w);
  sp.B = s->B; sp.Hq = s->Hq; sp.Hkv = s->Hkv; sp.G = s->Hq / s->Hkv; sp.d = s->d; sp.r = s->r;
  sp.cap = cap_of(s);
  sp.max_pages = s->max_pages; sp.num_pages = s->num_pages; sp.paged = s->page_size ? 1 : 0;
  sp.k_max = k_max;
  sp.sigma = 1.0f / sqrtf((float)s->d);
  sp.lam = lambda;
  sas::plan_score(sp, sms);

  sas::SelectParams& sl = out->sl;
  sl = {};
  sl.keys = sp.keys;
  sl.hist = sp.hist;
  sl.seqlens = seqlens;
  sl.kvec = k;
  sl.idx_out = idx_out;
  sl.err = sp.err;
  sl.B = s->B; sl.Hkv = s->Hkv; sl.cap = sp.cap; sl.k_max = k_max;
  if (!sas::plan_select(sl, sms)) return fail(SAS_ERR_UNSUPPORTED, "no selection plan for this shape");
  return SAS_OK;
}

sas_status run_score(const SelectPlan& pl, cudaStream_t st) {
  const cudaError_t e = sas::launch_score(pl.sp, st);
  return e == cudaSuccess ? SAS_OK : cuda_fail(e, "score kernel launch");
}

sas_status run_select(const SelectPlan& pl, cudaStream_t st) {
  const cudaError_t e = sas::launch_select(pl.sl, st);
  return e == cudaSuccess ? SAS_OK : cuda_fail(e, "select kernel launch");
}

sas_status do_select(const sas_shape* s, const void* q, const float* M, const void* Kproj,
                     const int32_t* page_table, const int32_t* seqlens, const int32_t* k, int32_t k_max,
                     float lambda, const float* log_g, int32_t* idx_out, float* scores_out, void* ws,
                     cudaStream_t st) {
  SelectPlan pl;
  SAS_TRY(plan_selection(s, q, M, Kproj, page_table, seqlens, k, k_max, lambda, log_g, idx_out, scores_out, ws, &pl));
  SAS_TRY(run_score(pl, st));
  return run_select(pl, st);
}

sas_status do_attend(const sas_shape* s, const void* q, const void* K, const void* V, const int32_t* page_table,
                     const int32_t* seqlens, const int32_t* idx, const int32_t* k, int32_t count_max,
                     float lambda, const float* log_g, float* out, void* ws, cudaStream_t st) {
  sas::AttendParams a = attend_plan(s, count_max, idx == nullptr);
  bind_workspace(a, ws);
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.K = static_cast<const __nv_bfloat16*>(K);
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.page_table = s->page_size ? page_table : nullptr;
  a.seqlens = seqlens;
  a.idx = idx;
  a.kvec = k;
  a.log_g = (idx != nullptr && lambda != 0.0f) ? log_g : nullptr;
  a.out = out;
  a.sms = num_sms();
  a.max_pages = s->max_pages; a.num_pages = s->num_pages; a.paged = s->page_size ? 1 : 0;
  a.k_max = count_max;
  a.sigma = 1.0f / sqrtf((float)s->d);
  a.lam = lambda;
  const cudaError_t e = sas::launch_attend(a, st);
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch");
  return SAS_OK;
}

}  // namespace

extern "C" {

int sas_abi_version(void) { return SAS_ABI_VERSION; }

const char* sas_status_string(sas_status s) {
  switch (s) {
    case SAS_OK: return "SAS_OK";
    case SAS_ERR_INVALID_ARG: return "SAS_ERR_INVALID_ARG";
    case SAS_ERR_UNSUPPORTED: return "SAS_ERR_UNSUPPORTED";
    case SAS_ERR_CUDA: return "SAS_ERR_CUDA";
    case SAS_ERR_DEVICE_CHECK: return "SAS_ERR_DEVICE_CHECK";
  }
  return "SAS_UNKNOWN_STATUS";
}

const char* sas_last_error_detail(void) { return g_detail; }

size_t sas_decode_workspace_bytes(const sas_shape* shape, int32_t k_max) {
  if (check_shape(shape) != SAS_OK || k_max < 1) return 0;
  return ws_bytes_for(attend_plan(shape, k_max, false), true);
}

size_t sas_dense_workspace_bytes(const sas_shape* shape) {
  if (check_shape(shape) != SAS_OK) return 0;
  return ws_bytes_for(attend_plan(shape, cap_of(shape), true), false);
}

sas_status sas_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
  SAS_TRY(check_ptr(workspace, "workspace"));
  if (ws_bytes < kErrBytes) return fail(SAS_ERR_INVALID_ARG, "workspace smaller than %zu bytes", kErrBytes);
  const cudaError_t e = cudaMemsetAsync(workspace, 0, ws_bytes, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SAS_OK : cuda_fail(e, "workspace memset");
}

sas_status sas_check_workspace(void* workspace, size_t ws_bytes, void* stream, uint32_t* code_out,
                               uint32_t* where_out) {
  SAS_TRY(check_ptr(workspace, "workspace"));
  if (ws_bytes < kErrBytes) return fail(SAS_ERR_INVALID_ARG, "workspace smaller than %zu bytes", kErrBytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t w[2] = {0, 0};
  cudaError_t e = cudaMemcpyAsync(w, workspace, sizeof(w), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof(w), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "reading the workspace error word");
  if (code_out) *code_out = w[0];
  if (where_out) *where_out = w[1];
  return w[0] ? SAS_ERR_DEVICE_CHECK : SAS_OK;
}

sas_status sas_build_proj_cache(const sas_shape* shape, const void* K, const float* M, void* Kproj,
                                const int32_t* page_table, const int32_t* seqlens, void* stream) {
  SAS_TRY(check_shape(shape));
  SAS_TRY(check_ptr(K, "K"));
  SAS_TRY(check_ptr(M, "M"));
  SAS_TRY(check_ptr(Kproj, "Kproj"));
  SAS_TRY(check_cache_ptrs(shape, page_table, seqlens));
  sas::ProjParams p = {};
  p.K = static_cast<const __nv_bfloat16*>(K);
  p.M = M;
  p.Kproj = Kproj;
  p.fp8 = shape->kproj_dtype == SAS_KPROJ_FP8_E4M3 ? 1 : 0;
  p.kproj_scale = shape->kproj_scale;
  p.page_table = shape->page_size ? page_table : nullptr;
  p.seqlens = seqlens;
  p.err = nullptr;
  p.B = shape->B; p.Hkv = shape->Hkv; p.d = shape->d; p.r = shape->r; p.cap = cap_of(shape);
  p.max_pages = shape->max_pages; p.num_pages = shape->num_pages; p.paged = shape->page_size ? 1 : 0;
  p.append = 0;
  const cudaError_t e = sas::launch_proj(p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SAS_OK : cuda_fail(e, "projection build launch");
}

sas_status sas_append_proj(const sas_shape* shape, const void* K_new, const float* M, void* Kproj,
                           const int32_t* page_table, const int32_t* seqlens, void* stream) {
  SAS_TRY(check_shape(shape));
  SAS_TRY(check_ptr(K_new, "K_new"));
  SAS_TRY(check_ptr(M, "M"));
  SAS_TRY(check_ptr(Kproj, "Kproj"));
  SAS_TRY(check_cache_ptrs(shape, page_table, seqlens));
  sas::ProjParams p = {};
  p.K = static_cast<const __nv_bfloat16*>(K_new);
  p.M = M;
  p.Kproj = Kproj;
  p.fp8 = shape->kproj_dtype == SAS_KPROJ_FP8_E4M3 ? 1 : 0;
  p.kproj_scale = shape->kproj_scale;
  p.page_table = shape->page_size ? page_table : nullptr;
  p.seqlens = seqlens;
  p.B = shape->B; p.Hkv = shape->Hkv; p.d = shape->d; p.r = shape->r; p.cap = cap_of(shape);
  p.max_pages = shape->max_pages; p.num_pages = shape->num_pages; p.paged = shape->page_size ? 1 : 0;
  p.append = 1;
  const cudaError_t e = sas::launch_proj(p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SAS_OK : cuda_fail(e, "projection append launch");
}

sas_status sas_select_topk(const sas_shape* shape, const void* q, const float* M, const void* Kproj,
                           const int32_t* page_table, const int32_t* seqlens, const int32_t* k, int32_t k_max,
                           float lambda, const float* log_g, int32_t* idx_out, float* scores_out, void* workspace,
                           size_t ws_bytes, void* stream) {
  SAS_TRY(check_shape(shape));
  if (k_max < 1) return fail(SAS_ERR_INVALID_ARG, "k_max must be >= 1");
  SAS_TRY(check_ptr(q, "q"));
  SAS_TRY(check_ptr(M, "M"));
  SAS_TRY(check_ptr(Kproj, "Kproj"));
  SAS_TRY(check_ptr(k, "k"));
  SAS_TRY(check_ptr(idx_out, "idx_out"));
  SAS_TRY(check_ptr(scores_out, "scores_out", false));
  SAS_TRY(check_cache_ptrs(shape, page_table, seqlens));
  if (lambda != 0.0f) SAS_TRY(check_ptr(log_g, "log_g"));
  SAS_TRY(check_ptr(workspace, "workspace"));
  if (ws_bytes < sas_decode_workspace_bytes(shape, k_max)) return fail(SAS_ERR_INVALID_ARG, "workspace too small");
  return do_select(shape, q, M, Kproj, page_table, seqlens, k, k_max, lambda, log_g, idx_out, scores_out,
                   workspace, static_cast<cudaStream_t>(stream));
}

sas_status sas_score_scan(const sas_shape* shape, const void* q, const float* M, const void* Kproj,
                          const int32_t* page_table, const int32_t* seqlens, const int32_t* k, int32_t k_max,
                          float lambda, const float* log_g, float* scores_out, void* workspace, size_t ws_bytes,
                          void* stream) {
  SAS_TRY(check_shape(shape));
  if (k_max < 1) return fail(SAS_ERR_INVALID_ARG, "k_max must be >= 1");
  SAS_TRY(check_ptr(q, "q"));
  SAS_TRY(check_ptr(M, "M"));
  SAS_TRY(check_ptr(Kproj, "Kproj"));
  SAS_TRY(check_ptr(k, "k"));
  SAS_TRY(check_ptr(scores_out, "scores_out", false));
  SAS_TRY(check_cache_ptrs(shape, page_table, seqlens));
  if (lambda != 0.0f) SAS_TRY(check_ptr(log_g, "log_g"));
  SAS_TRY(check_ptr(workspace, "workspace"));
  if (ws_bytes < sas_decode_workspace_bytes(shape, k_max)) return fail(SAS_ERR_INVALID_ARG, "workspace too small");
  SelectPlan pl;
  SAS_TRY(plan_selection(shape, q, M, Kproj, page_table, seqlens, k, k_max, lambda, log_g, nullptr, scores_out,
                         workspace, &pl));
  return run_score(pl, static_cast<cudaStream_t>(stream));
}

sas_status sas_select_from_scores(const sas_shape* shape, const int32_t* seqlens, const int32_t* k, int32_t k_max,
                                  int32_t* idx_out, void* workspace, size_t ws_bytes, void* stream) {
  SAS_TRY(check_shape(shape));
  if (k_max < 1) return fail(SAS_ERR_INVALID_ARG, "k_max must be >= 1");
  SAS_TRY(check_ptr(seqlens, "seqlens"));
  SAS_TRY(check_ptr(k, "k"));
  SAS_TRY(check_ptr(idx_out, "idx_out"));
  SAS_TRY(check_ptr(workspace, "workspace"));
  if (ws_bytes < sas_decode_workspace_bytes(shape, k_max)) return fail(SAS_ERR_INVALID_ARG, "workspace too small");
  SelectPlan pl;
  SAS_TRY(plan_selection(shape, nullptr, nullptr, nullptr, nullptr, seqlens, k, k_max, 0.0f, nullptr, idx_out,
                         nullptr, workspace, &pl));
  return run_select(pl, static_cast<cudaStream_t>(stream));
}

sas_status sas_sparse_attention(const sas_shape* shape, const void* q, const void* K, const void* V,
                                const int32_t* page_table, const int32_t* seqlens, const int32_t* idx,
                                const int32_t* k, int32_t k_max, float lambda, const float* log_g, float* out,
                                void* workspace, size_t ws_bytes, void* stream) {
  SAS_TRY(check_shape(shape));
  if (k_max < 1) return fail(SAS_ERR_INVALID_ARG, "k_max must be >= 1");
  SAS_TRY(check_ptr(q, "q"));
  SAS_TRY(check_ptr(K, "K"));
  SAS_TRY(check_ptr(V, "V"));
  SAS_TRY(check_ptr(idx, "idx"));
  SAS_TRY(check_ptr(k, "k"));
  SAS_TRY(check_ptr(out, "out"));
  SAS_TRY(check_cache_ptrs(shape, page_table, seqlens));
  if (lambda != 0.0f) SAS_TRY(check_ptr(log_g, "log_g"));
  SAS_TRY(check_ptr(workspace, "workspace"));
  if (ws_bytes < sas_decode_workspace_bytes(shape, k_max)) return fail(SAS_ERR_INVALID_ARG, "workspace too small");
  return do_attend(shape, q, K, V, page_table, seqlens, idx, k, k_max, lambda, log_g, out, workspace,
                   static_cast<cudaStream_t>(stream));
}

sas_status sas_decode_step(const sas_shape* shape, const void* q, const float* M, const void* Kproj, const void* K,
                           const void* V, const int32_t* page_table, const int32_t* seqlens, const int32_t* k,
                           int32_t k_max, float lambda, const float* log_g, float* out, int32_t* idx_out,
                           void* workspace, size_t ws_bytes, void* stream) {
  SAS_TRY(check_shape(shape));
  if (k_max < 1) return fail(SAS_ERR_INVALID_ARG, "k_max must be >= 1");
  SAS_TRY(check_ptr(q, "q"));
  SAS_TRY(check_ptr(M, "M"));
  SAS_TRY(check_ptr(Kproj, "Kproj"));
  SAS_TRY(check_ptr(K, "K"));
  SAS_TRY(check_ptr(V, "V"));
  SAS_TRY(check_ptr(k, "k"));
  SAS_TRY(check_ptr(out, "out"));
  SAS_TRY(check_ptr(idx_out, "idx_out"));
  SAS_TRY(check_cache_ptrs(shape, page_table, seqlens));
  if (lambda != 0.0f) SAS_TRY(check_ptr(log_g, "log_g"));
  SAS_TRY(check_ptr(workspace, "workspace"));
  if (ws_bytes < sas_decode_workspace_bytes(shape, k_max)) return fail(SAS_ERR_INVALID_ARG, "workspace too small");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SAS_TRY(do_select(shape, q, M, Kproj, page_table, seqlens, k, k_max, lambda, log_g, idx_out, nullptr,
                    workspace, st));
  return do_attend(shape, q, K, V, page_table, seqlens, idx_out, k, k_max, lambda, log_g, out, workspace, st);
}

sas_status sas_dense_decode(const sas_shape* shape, const void* q, const void* K, const void* V,
                            const int32_t* page_table, const int32_t* seqlens, float* out, void* workspace,
                            size_t ws_bytes, void* stream) {
  SAS_TRY(check_shape(shape));
  SAS_TRY(check_ptr(q, "q"));
  SAS_TRY(check_ptr(K, "K"));
  SAS_TRY(check_ptr(V, "V"));
  SAS_TRY(check_ptr(out, "out"));
  SAS_TRY(check_cache_ptrs(shape, page_table, seqlens));
  SAS_TRY(check_ptr(workspace, "workspace"));
  if (ws_bytes < sas_dense_workspace_bytes(shape)) return fail(SAS_ERR_INVALID_ARG, "workspace too small");
  return do_attend(shape, q, K, V, page_table, seqlens, nullptr, nullptr, cap_of(shape), 0.0f, nullptr, out,
                   workspace, static_cast<cudaStream_t>(stream));
}

sas_status sas_gather_selected(const sas_shape* shape, const void* K, const void* V, const int32_t* page_table,
                               const int32_t* seqlens, const int32_t* idx, const int32_t* k, int32_t k_max,
                               void* Kg, void* Vg, int32_t* counts, void* stream) {
  SAS_TRY(check_shape(shape));
  if (k_max < 1) return fail(SAS_ERR_INVALID_ARG, "k_max must be >= 1");
  SAS_TRY(check_ptr(K, "K"));
  SAS_TRY(check_ptr(V, "V"));
  SAS_TRY(check_ptr(idx, "idx"));
  SAS_TRY(check_ptr(k, "k"));
  SAS_TRY(check_ptr(Kg, "Kg"));
  SAS_TRY(check_ptr(Vg, "Vg"));
  SAS_TRY(check_ptr(counts, "counts"));
  SAS_TRY(check_cache_ptrs(shape, page_table, seqlens));
  sas::GatherParams p = {};
  p.K = static_cast<const __nv_bfloat16*>(K);
  p.V = static_cast<const __nv_bfloat16*>(V);
  p.page_table = shape->page_size ? page_table : nullptr;
  p.seqlens = seqlens;
  p.idx = idx;
  p.kvec = k;
  p.Kg = static_cast<__nv_bfloat16*>(Kg);
  p.Vg = static_cast<__nv_bfloat16*>(Vg);
  p.counts = counts;
  p.B = shape->B; p.Hkv = shape->Hkv; p.d = shape->d; p.cap = cap_of(shape);
  p.max_pages = shape->max_pages; p.num_pages = shape->num_pages; p.paged = shape->page_size ? 1 : 0;
  p.k_max = k_max;
  const cudaError_t e = sas::launch_gather(p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SAS_OK : cuda_fail(e, "gather kernel launch");
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// sas_decode_step_static_scratch: the decode step on a fixed scratch array that belongs to the
// library, for callers that cannot provide a workspace.  The array is part of this file's
// device image, so no allocation call is ever made for it: the CUDA driver places it when the
// image is loaded on a device.  One array per device, shared by every call on that device.
// ---------------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_static_scratch[SAS_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mutex;
// Per device: the address of g_static_scratch and the id of the CUDA context it was looked up
// in.  A device reset (or any teardown of the primary context) loads the library's device image
// again, possibly elsewhere, so the address is looked up again whenever the context changes.
struct ScratchEntry {
  void* ptr;
  unsigned long long ctx_id;
};
ScratchEntry g_scratch[kMaxScratchDevices] = {};

// Address of this device's copy of g_static_scratch, looked up with the device current the first
// time and again after the device's context has been replaced; cached otherwise.
sas_status static_scratch_ptr(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxScratchDevices)
    return fail(SAS_ERR_UNSUPPORTED, "device ordinal %d: the static scratch supports devices 0..%d", dev,
                kMaxScratchDevices - 1);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  unsigned long long id = 0;
  e = sas::current_context_id(&id);
  if (e != cudaSuccess) return cuda_fail(e, "querying the current context");
  ScratchEntry& ent = g_scratch[dev];
  if (ent.ptr == nullptr || id == 0 || id != ent.ctx_id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);  // makes the device's primary context current
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the static scratch");
    if (id == 0) {
      e = sas::current_context_id(&id);
      if (e != cudaSuccess) return cuda_fail(e, "querying the current context");
    }
    ent.ptr = p;
    ent.ctx_id = id;
  }
  *out = ent.ptr;
  return SAS_OK;
}

}  // namespace

extern "C" {

sas_status sas_decode_step_static_scratch(const sas_shape* shape, const void* q, const float* M,
                                          const void* Kproj, const void* K, const void* V,
                                          const int32_t* page_table, const int32_t* seqlens, const int32_t* k,
                                          int32_t k_max, float lambda, const float* log_g, float* out,
                                          int32_t* idx_out, void* stream) {
  SAS_TRY(check_shape(shape));
  if (k_max < 1) return fail(SAS_ERR_INVALID_ARG, "k_max must be >= 1");
  const size_t need = sas_decode_workspace_bytes(shape, k_max);
  if (need > (size_t)SAS_STATIC_SCRATCH_BYTES)
    return fail(SAS_ERR_UNSUPPORTED,
                "this shape and k_max need %zu bytes of scratch, more than the %zu-byte static scratch; "
                "call sas_decode_step with a caller workspace instead",
                need, (size_t)SAS_STATIC_SCRATCH_BYTES);
  SAS_TRY(check_ptr(q, "q"));
  SAS_TRY(check_ptr(M, "M"));
  SAS_TRY(check_ptr(Kproj, "Kproj"));
  SAS_TRY(check_ptr(K, "K"));
  SAS_TRY(check_ptr(V, "V"));
  SAS_TRY(check_ptr(k, "k"));
  SAS_TRY(check_ptr(out, "out"));
  SAS_TRY(check_ptr(idx_out, "idx_out"));
  SAS_TRY(check_cache_ptrs(shape, page_table, seqlens));
  if (lambda != 0.0f) SAS_TRY(check_ptr(log_g, "log_g"));

  void* ws = nullptr;
  SAS_TRY(static_scratch_ptr(&ws));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The error word and the per-head histograms must start at zero; a previous call may have
  // been cut short, so every call clears them.  The score keys and the attention partials that
  // follow are written before they are read.
  const WsLayout L = ws_layout(attend_plan(shape, k_max, false), true);
  const cudaError_t e = cudaMemsetAsync(ws, 0, L.partials, st);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the static scratch");
  SAS_TRY(do_select(shape, q, M, Kproj, page_table, seqlens, k, k_max, lambda, log_g, idx_out, nullptr, ws, st));
  return do_attend(shape, q, K, V, page_table, seqlens, idx_out, k, k_max, lambda, log_g, out, ws, st);
}

}  // extern "C"
