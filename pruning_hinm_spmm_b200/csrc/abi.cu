// C ABI of the HiNM hot path: argument checks, workspace sizing and dispatch to the
// kernels.  Every entry point returns an hinm_status and never throws.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>
#include <algorithm>

#include "../../include/hinm.h"
#include "hinm_internal.h"

namespace {

thread_local std::string g_last_error;

hinm_status fail(hinm_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

hinm_status ok() {
  g_last_error.clear();
  return HINM_OK;
}

hinm_status cuda_fail(cudaError_t e, const char* where) {
  return fail(HINM_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE_PTR(p)                                                            \
  do {                                                                            \
    if ((p) == nullptr) return fail(HINM_ERR_INVALID_ARG, "%s is NULL", #p);      \
    if (!aligned16(p)) return fail(HINM_ERR_ALIGNMENT, "%s is not 16-byte aligned", #p); \
  } while (0)

#define REQUIRE_ALIGNED_OR_NULL(p)                                                \
  do {                                                                            \
    if ((p) != nullptr && !aligned16(p))                                          \
      return fail(HINM_ERR_ALIGNMENT, "%s is not 16-byte aligned", #p);           \
  } while (0)

hinm_status check_mkt(int M, int K, int T) {
  if (T != 64 && T != 128) return fail(HINM_ERR_SHAPE, "T=%d: tile height must be 64 or 128", T);
  if (M <= 0 || M % T != 0) return fail(HINM_ERR_SHAPE, "M=%d must be a positive multiple of T=%d", M, T);
  if (K < 4 || K > hinm::kMaxK || K % 4 != 0)
    return fail(HINM_ERR_SHAPE, "K=%d must be a multiple of 4 in [4, %d]", K, hinm::kMaxK);
  if ((long long)M * (long long)K >= (1ll << 31))
    return fail(HINM_ERR_SHAPE, "M*K=%lld exceeds 2^31 elements", (long long)M * K);
  if (M / T > 65535) return fail(HINM_ERR_SHAPE, "M/T=%d tiles exceeds 65535", M / T);
  return HINM_OK;
}

hinm_status check_n(int N) {
  if (N <= 0 || N % 8 != 0) return fail(HINM_ERR_SHAPE, "N=%d must be a positive multiple of 8", N);
  if (N > (1 << 24)) return fail(HINM_ERR_SHAPE, "N=%d too large", N);
  return HINM_OK;
}

hinm_status check_search_params(double t_s, double alpha) {
  if (!std::isfinite(t_s) || t_s < 0.0 || t_s > 1.0)
    return fail(HINM_ERR_INVALID_ARG, "t_s=%g must be in [0, 1]", t_s);
  if (!std::isfinite(alpha) || alpha <= 0.0)
    return fail(HINM_ERR_INVALID_ARG, "alpha=%g must be a positive finite step", alpha);
  return HINM_OK;
}

// One status word per device, its address resolved with cudaGetSymbolAddress on first use
// in each context.
__device__ int g_device_status;
hinm::SymbolCache g_status_cache;

// cuCtxGetCurrent, resolved through the runtime (the library does not link the driver).
typedef int (*CtxGetCurrentFn)(void**);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

void* current_context() {
  void* ctx = nullptr;
  CtxGetCurrentFn fn = ctx_get_current_fn();
  if (!fn || fn(&ctx) != 0) return nullptr;
  return ctx;
}

}  // namespace

namespace hinm {

void* current_cuda_context() { return current_context(); }

// The address of a __device__ symbol belongs to the module loaded in one context: after
// cudaDeviceReset (or any re-creation of the primary context) the module is loaded again
// and the symbol can move.  The cache keeps, per device, the context the address was
// resolved in and resolves it again when the current context differs.
cudaError_t resolve_symbol(SymbolCache& c, const void* symbol, void** out) {
  *out = nullptr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= SymbolCache::kDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(c.mu);
  void* ctx = current_context();
  if (c.ptr[dev] && ctx && ctx == c.ctx[dev]) {
    *out = c.ptr[dev];
    return cudaSuccess;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, symbol);  // makes the device's primary context current if none is
  if (e != cudaSuccess) return e;
  c.ptr[dev] = p;
  c.ctx[dev] = ctx ? ctx : current_context();
  *out = p;
  return cudaSuccess;
}

}  // namespace hinm

namespace hinm {

// Closed form of the three region counts (see hinm.h).  Evaluated left to right in
// double precision with no fused multiply-add (the host build uses -ffp-contract=off).
bool counts_from_vs_host(int K, double t_s, double v_s, int out[3]) {
  const double x = 2.0 * (t_s - v_s) * K / 4.0;
  const double fl = std::floor(x + 0.5);
  if (!std::isfinite(fl)) return false;
  const long long n24 = 4ll * (long long)fl;
  const double tk = t_s * K;
  if (tk != std::floor(tk)) return false;
  const long long n0 = (long long)tk - n24 / 2;
  const long long n4 = (long long)K - n0 - n24;
  if (n24 < 0 || n0 < 0 || n4 < 0) return false;
  out[0] = (int)n0;
  out[1] = (int)n24;
  out[2] = (int)n4;
  return true;
}

int search_candidates_host(int K, double t_s, double alpha, Candidate* out, int cap) {
  const double lower = std::fmax(0.0, 2.0 * t_s - 1.0);
  const double mm = std::floor((t_s - lower) / alpha);
  const long long m_max = (long long)mm;
  int n = 0;
  for (long long m = 0; m <= m_max && n < cap; ++m) {
    const double v_s = t_s - (double)m * alpha;
    int c[3];
    if (!counts_from_vs_host(K, t_s, v_s, c)) {
      if (m == 0) return -1;
      break;
    }
    out[n++] = Candidate{c[0], c[1], c[2]};
  }
  return n;
}

int* device_status_ptr() {
  void* p = nullptr;
  if (resolve_symbol(g_status_cache, &g_device_status, &p) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

namespace {
// A function attribute lives in the module of one context: a re-created context (after
// cudaDeviceReset) starts without it, so the record is kept per device and context.
struct SmemAttr {
  int dev;
  void* ctx;
  const void* fn;
  int bytes;  // the largest limit set so far
};
std::mutex g_attr_mu;
SmemAttr g_attr_done[1024];
int g_attr_count = 0;
}  // namespace

cudaError_t set_max_dynamic_smem(const void* fn, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_attr_mu);
  void* ctx = current_context();
  int slot = -1;
  for (int i = 0; i < g_attr_count; ++i)
    if (g_attr_done[i].dev == dev && g_attr_done[i].ctx == ctx && g_attr_done[i].fn == fn)
      slot = i;
  if (ctx && slot >= 0 && g_attr_done[slot].bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (!ctx) return cudaSuccess;  // no context known: set again on every call
  if (slot >= 0) g_attr_done[slot].bytes = bytes;
  else if (g_attr_count < (int)(sizeof(g_attr_done) / sizeof(g_attr_done[0])))
    g_attr_done[g_attr_count++] = SmemAttr{dev, ctx, fn, bytes};
  return cudaSuccess;
}

}  // namespace hinm

// =====================================================================================
extern "C" {

const char* hinm_status_string(int st) {
  switch (st) {
    case HINM_OK: return "HINM_OK";
    case HINM_ERR_INVALID_ARG: return "HINM_ERR_INVALID_ARG";
    case HINM_ERR_SHAPE: return "HINM_ERR_SHAPE";
    case HINM_ERR_ALIGNMENT: return "HINM_ERR_ALIGNMENT";
    case HINM_ERR_UNSUPPORTED: return "HINM_ERR_UNSUPPORTED";
    case HINM_ERR_CUDA: return "HINM_ERR_CUDA";
    case HINM_ERR_DEVICE_TIMEOUT: return "HINM_ERR_DEVICE_TIMEOUT";
    case HINM_ERR_BAD_MASK: return "HINM_ERR_BAD_MASK";
    case HINM_ERR_WORKSPACE: return "HINM_ERR_WORKSPACE";
    default: return "HINM_ERR_UNKNOWN";
  }
}

const char* hinm_last_error(void) { return g_last_error.c_str(); }

int hinm_abi_version(void) { return HINM_ABI_VERSION; }

hinm_status hinm_counts_from_vs(int K, double t_s, double v_s, int32_t* out_host) {
  if (!out_host) return fail(HINM_ERR_INVALID_ARG, "out_host is NULL");
  if (K <= 0) return fail(HINM_ERR_SHAPE, "K=%d must be positive", K);
  if (!std::isfinite(t_s) || !std::isfinite(v_s) || t_s < 0 || t_s > 1 || v_s < 0 || v_s > 1)
    return fail(HINM_ERR_INVALID_ARG, "t_s=%g, v_s=%g must be finite and in [0, 1]", t_s, v_s);
  int c[3];
  if (!hinm::counts_from_vs_host(K, t_s, v_s, c))
    return fail(HINM_ERR_INVALID_ARG,
                "boundary (t_s=%g, v_s=%g) gives no valid counts for K=%d (t_s*K must be whole, "
                "v_s >= 2 t_s - 1)", t_s, v_s, K);
  out_host[0] = c[0];
  out_host[1] = c[1];
  out_host[2] = c[2];
  return ok();
}

hinm_status hinm_importance_workspace_size(int M, int K, int N, size_t* bytes_host) {
  if (!bytes_host) return fail(HINM_ERR_INVALID_ARG, "bytes_host is NULL");
  if (M <= 0 || K <= 0 || N <= 0) return fail(HINM_ERR_SHAPE, "sizes must be positive");
  *bytes_host = hinm::importance_workspace_bytes(K);
  return ok();
}

hinm_status hinm_importance(const void* W, const void* X, int M, int K, int N, float* I_out,
                            void* workspace, size_t workspace_bytes, void* stream) {
  REQUIRE_PTR(W);
  REQUIRE_PTR(X);
  REQUIRE_PTR(I_out);
  if (M <= 0 || K <= 0 || K % 4 != 0 || (long long)M * K >= (1ll << 31))
    return fail(HINM_ERR_SHAPE, "M=%d, K=%d: need M > 0 and K a positive multiple of 4", M, K);
  hinm_status st = check_n(N);
  if (st != HINM_OK) return st;
  const size_t need = hinm::importance_workspace_bytes(K);
  if (!workspace || workspace_bytes < need)
    return fail(HINM_ERR_WORKSPACE, "workspace %zu bytes, need %zu", workspace_bytes, need);
  REQUIRE_PTR(workspace);
  cudaError_t e = hinm::launch_importance(static_cast<const uint16_t*>(W),
                                          static_cast<const uint16_t*>(X), M, K, N, I_out,
                                          static_cast<float*>(workspace),
                                          static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hinm_importance launch");
  return ok();
}

hinm_status hinm_tile_stats_size(int M, int K, int T, size_t* bytes_host) {
  if (!bytes_host) return fail(HINM_ERR_INVALID_ARG, "bytes_host is NULL");
  hinm_status st = check_mkt(M, K, T);
  if (st != HINM_OK) return st;
  *bytes_host = hinm::tile_stats_bytes(M, K, T);
  return ok();
}

hinm_status hinm_importance_stats(const void* W, const void* X, int M, int K, int N, int T,
                                  float* I_out, void* stats_out, size_t stats_bytes,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  REQUIRE_PTR(W);
  REQUIRE_PTR(X);
  REQUIRE_ALIGNED_OR_NULL(I_out);
  REQUIRE_PTR(stats_out);
  hinm_status st = check_mkt(M, K, T);
  if (st != HINM_OK) return st;
  st = check_n(N);
  if (st != HINM_OK) return st;
  if (stats_bytes < hinm::tile_stats_bytes(M, K, T))
    return fail(HINM_ERR_INVALID_ARG, "stats %zu bytes, need %zu", stats_bytes,
                hinm::tile_stats_bytes(M, K, T));
  (void)workspace;  // the channel energies live in stats_out
  (void)workspace_bytes;
  cudaError_t e = hinm::launch_importance_stats(
      static_cast<const uint16_t*>(W), static_cast<const uint16_t*>(X), M, K, N, T, I_out,
      stats_out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hinm_importance_stats launch");
  return ok();
}

hinm_status hinm_importance_noalloc(const void* W, const void* X, int M, int K, int N,
                                    float* I_out, void* stream) {
  REQUIRE_PTR(W);
  REQUIRE_PTR(X);
  REQUIRE_PTR(I_out);
  if (M <= 0 || K <= 0 || K % 4 != 0 || (long long)M * K >= (1ll << 31))
    return fail(HINM_ERR_SHAPE, "M=%d, K=%d: need M > 0 and K a positive multiple of 4", M, K);
  if (K > hinm::kNoAllocMaxK)
    return fail(HINM_ERR_SHAPE, "K=%d exceeds the static scratch (%d channels)", K,
                hinm::kNoAllocMaxK);
  hinm_status st = check_n(N);
  if (st != HINM_OK) return st;
  float* scratch = nullptr;
  cudaError_t e = hinm::noalloc_energy_scratch(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, "hinm_importance_noalloc scratch address");
  e = hinm::launch_importance(static_cast<const uint16_t*>(W), static_cast<const uint16_t*>(X),
                              M, K, N, I_out, scratch, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hinm_importance_noalloc launch");
  return ok();
}

hinm_status hinm_search_num_candidates(int K, double t_s, double alpha, int32_t* n_host) {
  if (!n_host) return fail(HINM_ERR_INVALID_ARG, "n_host is NULL");
  if (K < 4 || K > hinm::kMaxK) return fail(HINM_ERR_SHAPE, "K=%d out of range", K);
  hinm_status st = check_search_params(t_s, alpha);
  if (st != HINM_OK) return st;
  hinm::Candidate c[hinm::kMaxCandidates];
  const int n = hinm::search_candidates_host(K, t_s, alpha, c, hinm::kMaxCandidates);
  if (n < 0) return fail(HINM_ERR_INVALID_ARG, "t_s*K = %g is not a whole number", t_s * K);
  *n_host = n;
  return ok();
}

hinm_status hinm_search_workspace_size(int M, int K, int T, double t_s, double alpha,
                                       size_t* bytes_host) {
  if (!bytes_host) return fail(HINM_ERR_INVALID_ARG, "bytes_host is NULL");
  hinm_status st = check_mkt(M, K, T);
  if (st != HINM_OK) return st;
  st = check_search_params(t_s, alpha);
  if (st != HINM_OK) return st;
  hinm::Candidate c[hinm::kMaxCandidates];
  const int n = hinm::search_candidates_host(K, t_s, alpha, c, hinm::kMaxCandidates);
  if (n < 0) return fail(HINM_ERR_INVALID_ARG, "t_s*K = %g is not a whole number", t_s * K);
  *bytes_host = hinm::search_workspace_bytes(M, K, T, n);
  return ok();
}

namespace {

// hinm_boundary_search(_stats): stats (with its size) or nullptr
// The importance as the search and the mask read it: I, or W with the channel energies that
// hinm_importance_stats stored in the statistics.
hinm::ImpSrc imp_src(const float* I, const void* W, const void* stats, int M, int K, int T) {
  hinm::ImpSrc q{I, nullptr, nullptr};
  if (!I) {
    q.W = static_cast<const uint16_t*>(W);
    q.s = reinterpret_cast<const float*>(static_cast<const char*>(stats) +
                                         hinm::tile_stats_s_offset(M, K, T));
  }
  return q;
}

hinm_status search_impl(const float* I, const void* W, const void* stats, size_t stats_bytes,
                        const int32_t* perm, int perm_per_tile, int M, int K, int T, double t_s,
                        double alpha,
                        int32_t* counts_out, double* vs_out, int32_t* rank_out,
                        double* retained_out, void* workspace, size_t workspace_bytes,
                        void* stream) {
  REQUIRE_ALIGNED_OR_NULL(I);
  REQUIRE_ALIGNED_OR_NULL(W);
  if (!I && (!W || !stats))
    return fail(HINM_ERR_INVALID_ARG, "I is NULL: W and stats are needed to recompute it");
  REQUIRE_ALIGNED_OR_NULL(perm);
  REQUIRE_PTR(counts_out);
  REQUIRE_PTR(vs_out);
  REQUIRE_ALIGNED_OR_NULL(rank_out);
  REQUIRE_ALIGNED_OR_NULL(retained_out);
  hinm_status st = check_mkt(M, K, T);
  if (st != HINM_OK) return st;
  st = check_search_params(t_s, alpha);
  if (st != HINM_OK) return st;
  if (stats && stats_bytes < hinm::tile_stats_bytes(M, K, T))
    return fail(HINM_ERR_INVALID_ARG, "stats %zu bytes, need %zu", stats_bytes,
                hinm::tile_stats_bytes(M, K, T));
  hinm::Candidate c[hinm::kMaxCandidates];
  const int n = hinm::search_candidates_host(K, t_s, alpha, c, hinm::kMaxCandidates);
  if (n < 0) return fail(HINM_ERR_INVALID_ARG, "t_s*K = %g is not a whole number", t_s * K);
  const double lower = std::fmax(0.0, 2.0 * t_s - 1.0);
  if (std::floor((t_s - lower) / alpha) + 1 > hinm::kMaxCandidates && n == hinm::kMaxCandidates)
    return fail(HINM_ERR_UNSUPPORTED, "alpha=%g gives more than %d candidates", alpha,
                hinm::kMaxCandidates);
  const size_t need = hinm::search_workspace_bytes(M, K, T, n);
  if (!workspace || workspace_bytes < need)
    return fail(HINM_ERR_WORKSPACE, "workspace %zu bytes, need %zu", workspace_bytes, need);
  REQUIRE_PTR(workspace);
  if (perm_per_tile != 0 && perm_per_tile != 1)
    return fail(HINM_ERR_INVALID_ARG, "perm_per_tile=%d must be 0 or 1", perm_per_tile);
  const hinm::ImpSrc src = imp_src(I, W, stats, M, K, T);
  cudaError_t e = hinm::launch_boundary_search(src, stats, perm, perm_per_tile ? (long long)K : 0ll,
                                               M, K, T, t_s, alpha, c, n,
                                               counts_out, vs_out, rank_out, retained_out,
                                               workspace, hinm::device_status_ptr(),
                                               static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hinm_boundary_search launch");
  return ok();
}

}  // namespace

hinm_status hinm_boundary_search(const float* I, const int32_t* perm, int M, int K, int T,
                                 double t_s, double alpha, int32_t* counts_out, double* vs_out,
                                 int32_t* rank_out, double* retained_out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  REQUIRE_PTR(I);
  return search_impl(I, nullptr, nullptr, 0, perm, 0, M, K, T, t_s, alpha, counts_out, vs_out,
                     rank_out, retained_out, workspace, workspace_bytes, stream);
}

hinm_status hinm_boundary_search_stats(const float* I, const void* stats, size_t stats_bytes,
                                       const int32_t* perm, int M, int K, int T, double t_s,
                                       double alpha, int32_t* counts_out, double* vs_out,
                                       int32_t* rank_out, double* retained_out,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  REQUIRE_PTR(I);
  REQUIRE_PTR(stats);
  return search_impl(I, nullptr, stats, stats_bytes, perm, 0, M, K, T, t_s, alpha, counts_out,
                     vs_out, rank_out, retained_out, workspace, workspace_bytes, stream);
}

hinm_status hinm_boundary_search_ex(const float* I, const void* W, const void* stats,
                                    size_t stats_bytes, const int32_t* perm, int perm_per_tile,
                                    int M, int K, int T, double t_s, double alpha,
                                    int32_t* counts_out, double* vs_out, int32_t* rank_out,
                                    double* retained_out, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  return search_impl(I, W, stats, stats ? stats_bytes : 0, perm, perm_per_tile, M, K, T, t_s,
                     alpha, counts_out, vs_out, rank_out, retained_out, workspace,
                     workspace_bytes, stream);
}

hinm_status hinm_mask_workspace_size(int M, int K, int T, size_t* bytes_host) {
  if (!bytes_host) return fail(HINM_ERR_INVALID_ARG, "bytes_host is NULL");
  hinm_status st = check_mkt(M, K, T);
  if (st != HINM_OK) return st;
  *bytes_host = hinm::mask_workspace_bytes(M, K, T);
  return ok();
}

hinm_status hinm_mask(const float* I, const int32_t* perm, const int32_t* counts,
                      const int32_t* rank, int M, int K, int T, uint32_t* bitmask_out,
                      int8_t* region_out, void* workspace, size_t workspace_bytes,
                      void* stream) {
  REQUIRE_PTR(I);
  return hinm_mask_ex(I, nullptr, nullptr, 0, perm, 0, counts, rank, M, K, T, bitmask_out,
                      region_out, workspace, workspace_bytes, stream);
}

hinm_status hinm_mask_ex(const float* I, const void* W, const void* stats, size_t stats_bytes,
                         const int32_t* perm, int perm_per_tile, const int32_t* counts,
                         const int32_t* rank, int M, int K, int T, uint32_t* bitmask_out,
                         int8_t* region_out, void* workspace, size_t workspace_bytes,
                         void* stream) {
  REQUIRE_ALIGNED_OR_NULL(I);
  REQUIRE_ALIGNED_OR_NULL(W);
  if (!I && (!W || !stats))
    return fail(HINM_ERR_INVALID_ARG, "I is NULL: W and stats are needed to recompute it");
  if (perm_per_tile != 0 && perm_per_tile != 1)
    return fail(HINM_ERR_INVALID_ARG, "perm_per_tile=%d must be 0 or 1", perm_per_tile);
  REQUIRE_ALIGNED_OR_NULL(perm);
  REQUIRE_PTR(counts);
  REQUIRE_ALIGNED_OR_NULL(rank);
  REQUIRE_PTR(bitmask_out);
  REQUIRE_PTR(region_out);
  hinm_status st = check_mkt(M, K, T);
  if (st != HINM_OK) return st;
  const size_t need = hinm::mask_workspace_bytes(M, K, T);
  if (!workspace || workspace_bytes < need)
    return fail(HINM_ERR_WORKSPACE, "workspace %zu bytes, need %zu", workspace_bytes, need);
  REQUIRE_PTR(workspace);
  if (!I && stats_bytes < hinm::tile_stats_bytes(M, K, T))
    return fail(HINM_ERR_INVALID_ARG, "stats %zu bytes, need %zu", stats_bytes,
                hinm::tile_stats_bytes(M, K, T));
  const hinm::ImpSrc src = imp_src(I, W, stats, M, K, T);
  cudaError_t e = hinm::launch_mask(src, perm, perm_per_tile ? (long long)K : 0ll, counts, rank, M,
                                    K, T, bitmask_out, region_out,
                                    workspace, hinm::device_status_ptr(),
                                    static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hinm_mask launch");
  return ok();
}

hinm_status hinm_compress_size(const int32_t* counts_host, int M, int K, int T,
                               hinm_layout_sizes* out_host) {
  if (!out_host) return fail(HINM_ERR_INVALID_ARG, "out_host is NULL");
  hinm_status st = check_mkt(M, K, T);
  if (st != HINM_OK) return st;
  const int nt = M / T;
  long long nd = 0, ns = 0;
  if (counts_host) {
    for (int t = 0; t < nt; ++t) {
      const int n0 = counts_host[3 * t], n24 = counts_host[3 * t + 1], n4 = counts_host[3 * t + 2];
      if (n0 < 0 || n24 < 0 || n4 < 0 || n0 + n24 + n4 != K || n24 % 4 != 0)
        return fail(HINM_ERR_INVALID_ARG, "tile %d: counts (%d, %d, %d) invalid for K=%d", t, n0,
                    n24, n4, K);
      nd += (n4 + hinm::kDenseBK - 1) / hinm::kDenseBK;
      ns += (n24 + hinm::kSparseBK - 1) / hinm::kSparseBK;
    }
  } else {
    nd = (long long)nt * ((K + hinm::kDenseBK - 1) / hinm::kDenseBK + 1);
    ns = (long long)nt * ((K + hinm::kSparseBK - 1) / hinm::kSparseBK + 1);
  }
  if (nd == 0) nd = 1;  // keep every buffer non-empty so pointers can be checked
  if (ns == 0) ns = 1;
  out_host->max_dense_blocks = (int32_t)nd;
  out_host->max_sparse_blocks = (int32_t)ns;
  out_host->tile_info_bytes = (size_t)nt * 4 * sizeof(int32_t);
  out_host->vals_dense_bytes = (size_t)nd * hinm::kBlockBytes;
  out_host->vals_sparse_bytes = (size_t)ns * hinm::kBlockBytes;
  out_host->meta_bytes = (size_t)ns * hinm::kMetaWords * sizeof(uint32_t);
  out_host->idx_dense_bytes = (size_t)nd * hinm::kDenseBK * sizeof(int32_t);
  out_host->idx_sparse_bytes = (size_t)ns * hinm::kSparseBK * sizeof(int32_t);
  out_host->run_dense_bytes = (size_t)nd * sizeof(int32_t);
  out_host->run_sparse_bytes = (size_t)ns * sizeof(int32_t);
  return ok();
}

hinm_status hinm_compress_workspace_size(int M, int K, int T, size_t* bytes_host) {
  if (!bytes_host) return fail(HINM_ERR_INVALID_ARG, "bytes_host is NULL");
  hinm_status st = check_mkt(M, K, T);
  if (st != HINM_OK) return st;
  *bytes_host = hinm::compress_workspace_bytes(M, K, T);
  return ok();
}

static hinm_status check_layout(const hinm_layout* L) {
  if (!L) return fail(HINM_ERR_INVALID_ARG, "layout is NULL");
  if (L->layout_version != HINM_LAYOUT_VERSION)
    return fail(HINM_ERR_INVALID_ARG, "layout_version %d, expected %d", L->layout_version,
                HINM_LAYOUT_VERSION);
  hinm_status st = check_mkt(L->M, L->K, L->T);
  if (st != HINM_OK) return st;
  if (L->num_tiles != L->M / L->T)
    return fail(HINM_ERR_SHAPE, "num_tiles=%d != M/T=%d", L->num_tiles, L->M / L->T);
  if (L->max_dense_blocks < 1 || L->max_sparse_blocks < 1)
    return fail(HINM_ERR_SHAPE, "layout capacities must be >= 1 block");
  REQUIRE_PTR(L->tile_info);
  REQUIRE_PTR(L->vals_dense);
  REQUIRE_PTR(L->vals_sparse);
  REQUIRE_PTR(L->meta);
  REQUIRE_PTR(L->idx_dense);
  REQUIRE_PTR(L->idx_sparse);
  REQUIRE_PTR(L->run_dense);
  REQUIRE_PTR(L->run_sparse);
  return HINM_OK;
}

hinm_status hinm_compress(const void* W, const uint32_t* bitmask, const int8_t* region,
                          const int32_t* perm, const int32_t* counts, int M, int K, int T,
                          const hinm_layout* layout, void* workspace, size_t workspace_bytes,
                          void* stream) {
  return hinm_compress_ex(W, bitmask, region, perm, 0, counts, M, K, T, layout, workspace,
                          workspace_bytes, stream);
}

hinm_status hinm_compress_ex(const void* W, const uint32_t* bitmask, const int8_t* region,
                             const int32_t* perm, int perm_per_tile, const int32_t* counts,
                             int M, int K, int T, const hinm_layout* layout, void* workspace,
                             size_t workspace_bytes, void* stream) {
  REQUIRE_PTR(W);
  if (perm_per_tile != 0 && perm_per_tile != 1)
    return fail(HINM_ERR_INVALID_ARG, "perm_per_tile=%d must be 0 or 1", perm_per_tile);
  REQUIRE_PTR(bitmask);
  REQUIRE_PTR(region);
  REQUIRE_ALIGNED_OR_NULL(perm);
  REQUIRE_PTR(counts);
  hinm_status st = check_mkt(M, K, T);
  if (st != HINM_OK) return st;
  st = check_layout(layout);
  if (st != HINM_OK) return st;
  if (layout->M != M || layout->K != K || layout->T != T)
    return fail(HINM_ERR_SHAPE, "layout is %dx%d T=%d, call is %dx%d T=%d", layout->M, layout->K,
                layout->T, M, K, T);
  const size_t need = hinm::compress_workspace_bytes(M, K, T);
  if (!workspace || workspace_bytes < need)
    return fail(HINM_ERR_WORKSPACE, "workspace %zu bytes, need %zu", workspace_bytes, need);
  REQUIRE_PTR(workspace);
  cudaError_t e = hinm::launch_compress(static_cast<const uint16_t*>(W), bitmask, region, perm,
                                        perm_per_tile ? (long long)K : 0ll, counts, M, K, T, *layout, workspace,
                                        hinm::device_status_ptr(),
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hinm_compress launch");
  return ok();
}

namespace {
// The band of a gyro input round: n % 4 == 0, 4 <= n <= K, distinct entries in [0, K).
hinm_status check_band(int T, int K, const int32_t* band, int n) {
  if (T <= 0 || K < 4 || n < 4 || n % 4 != 0 || n > K)
    return fail(HINM_ERR_SHAPE, "T=%d, K=%d, n=%d: need T > 0, n a positive multiple of 4, n <= K",
                T, K, n);
  std::vector<char> seen(K, 0);
  for (int i = 0; i < n; ++i) {
    if (band[i] < 0 || band[i] >= K)
      return fail(HINM_ERR_INVALID_ARG, "band[%d]=%d outside [0, K)", i, band[i]);
    if (seen[band[i]]) return fail(HINM_ERR_INVALID_ARG, "band[%d]=%d repeated", i, band[i]);
    seen[band[i]] = 1;
  }
  return HINM_OK;
}
// G distinct items in [0, count) and, for each, k distinct sub-items in [0, sub).
hinm_status check_samples(const int32_t* items, int count, const int32_t* sub, int subcount,
                          int G, int k, const char* what) {
  if (G < 1 || G > count || k < 1 || k > subcount)
    return fail(HINM_ERR_INVALID_ARG, "%s: G=%d, k=%d: need 1 <= G <= %d, 1 <= k <= %d", what, G,
                k, count, subcount);
  std::vector<char> seen(count, 0);
  for (int i = 0; i < G; ++i) {
    if (items[i] < 0 || items[i] >= count || seen[items[i]])
      return fail(HINM_ERR_INVALID_ARG, "%s[%d]=%d: need distinct values in [0, %d)", what, i,
                  items[i], count);
    seen[items[i]] = 1;
    for (int j = 0; j < k; ++j) {
      const int v = sub[(size_t)i * k + j];
      if (v < 0 || v >= subcount)
        return fail(HINM_ERR_INVALID_ARG, "%s sample [%d][%d]=%d outside [0, %d)", what, i, j, v,
                    subcount);
      for (int q = 0; q < j; ++q)
        if (sub[(size_t)i * k + q] == v)
          return fail(HINM_ERR_INVALID_ARG, "%s sample [%d] repeats %d", what, i, v);
    }
  }
  return HINM_OK;
}
}  // namespace

hinm_status hinm_gyro_input_round_host(const float* I_tile, int T, int K, int32_t* band, int n,
                                       const int32_t* groups, const int32_t* slots, int G, int k,
                                       int kmeans_iters, double* cost_out) {
  if (!I_tile || !band || !groups || !slots)
    return fail(HINM_ERR_INVALID_ARG, "I_tile, band, groups and slots must not be NULL");
  hinm_status st = check_band(T, K, band, n);
  if (st != HINM_OK) return st;
  st = check_samples(groups, n / 4, slots, 4, G, k, "groups");
  if (st != HINM_OK) return st;
  if (kmeans_iters < 0) return fail(HINM_ERR_INVALID_ARG, "kmeans_iters=%d < 0", kmeans_iters);
  // the costs and the K-means need finite values: every importance the round reads
  for (int r = 0; r < T; ++r)
    for (int i = 0; i < n; ++i)
      if (!std::isfinite(I_tile[(size_t)r * K + band[i]]))
        return fail(HINM_ERR_INVALID_ARG, "I_tile[%d][%d] is not finite", r, band[i]);
  if (!hinm::gyro_input_round(I_tile, T, K, band, groups, slots, G, k, kmeans_iters, cost_out))
    return fail(HINM_ERR_INVALID_ARG, "the assignment could not be formed");
  return ok();
}

hinm_status hinm_gyro_band_cost_host(const float* I_tile, int T, int K, const int32_t* band,
                                     int n, double* cost_host) {
  if (!I_tile || !band || !cost_host)
    return fail(HINM_ERR_INVALID_ARG, "I_tile, band and cost_host must not be NULL");
  hinm_status st = check_band(T, K, band, n);
  if (st != HINM_OK) return st;
  *cost_host = hinm::gyro_band_cost(I_tile, T, K, band, n);
  return ok();
}

hinm_status hinm_gyro_cost_matrix(const float* I, int M, int K, int T, const int32_t* bands,
                                  int band_len, const int32_t* groups, const int32_t* slots,
                                  const int32_t* clusters, int G, int k, double* cost_out,
                                  void* stream) {
  REQUIRE_PTR(I);
  REQUIRE_PTR(bands);
  REQUIRE_PTR(groups);
  REQUIRE_PTR(slots);
  REQUIRE_PTR(clusters);
  REQUIRE_PTR(cost_out);
  if (T <= 0 || M <= 0 || M % T != 0 || K < 4)
    return fail(HINM_ERR_SHAPE, "M=%d, K=%d, T=%d: need M a positive multiple of T, K >= 4", M,
                K, T);
  if (band_len < 4 || band_len % 4 != 0 || band_len > K)
    return fail(HINM_ERR_SHAPE, "band_len=%d: need a multiple of 4 in [4, K]", band_len);
  if (k < 1 || k > 4 || G < 1 || G > band_len / 4)
    return fail(HINM_ERR_INVALID_ARG, "G=%d, k=%d: need 1 <= k <= 4, 1 <= G <= band_len/4", G, k);
  cudaError_t e = hinm::launch_gyro_cost(I, K, T, M / T, bands, band_len, groups, slots, clusters,
                                         G, k, cost_out, hinm::device_status_ptr(),
                                         static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hinm_gyro_cost_matrix launch");
  return ok();
}

hinm_status hinm_gyro_output_round_host(const float* I, int M, int K, int T, const int32_t* n0,
                                        int32_t* row_order, const int32_t* tiles,
                                        const int32_t* rows, int G, int k, int kmeans_iters,
                                        double* cost_out) {
  if (!I || !n0 || !row_order || !tiles || !rows)
    return fail(HINM_ERR_INVALID_ARG, "I, n0, row_order, tiles and rows must not be NULL");
  if (T <= 0 || M <= 0 || M % T != 0 || K <= 0)
    return fail(HINM_ERR_SHAPE, "M=%d, K=%d, T=%d: need M a positive multiple of T", M, K, T);
  const int nt = M / T;
  std::vector<char> seen(M, 0);
  for (int i = 0; i < M; ++i) {
    if (row_order[i] < 0 || row_order[i] >= M || seen[row_order[i]])
      return fail(HINM_ERR_INVALID_ARG, "row_order[%d]=%d: need a permutation of 0..M-1", i,
                  row_order[i]);
    seen[row_order[i]] = 1;
  }
  for (int t = 0; t < nt; ++t)
    if (n0[t] < 0 || n0[t] > K) return fail(HINM_ERR_INVALID_ARG, "n0[%d]=%d outside [0, K]", t, n0[t]);
  hinm_status st = check_samples(tiles, nt, rows, T, G, k, "tiles");
  if (st != HINM_OK) return st;
  if (kmeans_iters < 0) return fail(HINM_ERR_INVALID_ARG, "kmeans_iters=%d < 0", kmeans_iters);
  for (int i = 0; i < G; ++i)
    for (int r = 0; r < T; ++r) {
      const float* row = I + (size_t)row_order[(size_t)tiles[i] * T + r] * K;
      for (int c = 0; c < K; ++c)
        if (!std::isfinite(row[c]))
          return fail(HINM_ERR_INVALID_ARG, "I[%d][%d] is not finite",
                      row_order[(size_t)tiles[i] * T + r], c);
    }
  if (!hinm::gyro_output_round(I, M, K, T, n0, row_order, tiles, rows, G, k, kmeans_iters,
                               cost_out))
    return fail(HINM_ERR_INVALID_ARG, "the assignment could not be formed");
  return ok();
}

hinm_status hinm_hard_concrete_forward(const float* log_alpha, const float* eps, long long n,
                                      float tau, float* z_out, uint8_t* hard_out,
                                      double* sums_out, void* stream) {
  REQUIRE_PTR(log_alpha);
  REQUIRE_PTR(eps);
  REQUIRE_PTR(z_out);
  REQUIRE_ALIGNED_OR_NULL(hard_out);
  REQUIRE_ALIGNED_OR_NULL(sums_out);
  if (n <= 0 || n % 4 != 0)
    return fail(HINM_ERR_SHAPE, "n=%lld must be a positive multiple of 4", n);
  if (!(tau > 0.0f) || !std::isfinite(tau))
    return fail(HINM_ERR_INVALID_ARG, "tau=%g must be positive and finite", (double)tau);
  cudaError_t e = hinm::launch_hard_concrete(log_alpha, eps, n, tau, z_out, hard_out, sums_out,
                                             static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hinm_hard_concrete_forward launch");
  return ok();
}

hinm_status hinm_translate_index(const hinm_layout* layout, const int32_t* row_of_channel,
                                void* stream) {
  hinm_status st = check_layout(layout);
  if (st != HINM_OK) return st;
  REQUIRE_PTR(row_of_channel);
  cudaError_t e = hinm::launch_translate_index(*layout, row_of_channel, hinm::device_status_ptr(),
                                               static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hinm_translate_index launch");
  return ok();
}

hinm_status hinm_spmm(const hinm_layout* layout, const void* X, int N, float* Y_out,
                      void* stream) {
  return hinm_spmm_ex(layout, X, N, Y_out, 0, stream);
}

hinm_status hinm_spmm_ex(const hinm_layout* layout, const void* X, int N, float* Y_out,
                         int flags, void* stream) {
  return hinm_spmm_epilogue(layout, X, N, Y_out, nullptr, HINM_ACT_NONE, 0, flags, stream);
}

hinm_status hinm_spmm_epilogue(const hinm_layout* layout, const void* X, int N, void* Y_out,
                               const float* bias, int activation, int out_bf16, int flags,
                               void* stream) {
  if (flags & ~HINM_SPMM_TILE_PAIRS) return fail(HINM_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (activation < HINM_ACT_NONE || activation > HINM_ACT_GELU)
    return fail(HINM_ERR_INVALID_ARG, "unknown activation %d", activation);
  REQUIRE_ALIGNED_OR_NULL(bias);
  hinm_status st = check_layout(layout);
  if (st != HINM_OK) return st;
  REQUIRE_PTR(X);
  REQUIRE_PTR(Y_out);
  st = check_n(N);
  if (st != HINM_OK) return st;
  hinm::SpmmOut out{out_bf16 ? nullptr : static_cast<float*>(Y_out),
                     out_bf16 ? static_cast<uint16_t*>(Y_out) : nullptr, bias, activation};
  cudaError_t e = hinm::launch_spmm(*layout, static_cast<const uint16_t*>(X), N, out,
                                    (flags & HINM_SPMM_TILE_PAIRS) != 0,
                                    hinm::device_status_ptr(), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hinm_spmm launch");
  return ok();
}

hinm_status hinm_selftest_wait_timeout(unsigned long long limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 2000000000ull)
    return fail(HINM_ERR_INVALID_ARG, "limit_ns=%llu: need 0 < limit_ns <= 2e9", limit_ns);
  int* status = hinm::device_status_ptr();
  if (!status) return fail(HINM_ERR_CUDA, "no device status word");
  cudaError_t e =
      hinm::launch_wait_timeout_selftest(limit_ns, status, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hinm_selftest_wait_timeout launch");
  return ok();
}

hinm_status hinm_device_status(void* stream, int32_t* status_host) {
  if (!status_host) return fail(HINM_ERR_INVALID_ARG, "status_host is NULL");
  int* p = hinm::device_status_ptr();
  if (!p) return fail(HINM_ERR_CUDA, "cannot resolve the device status word");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, p, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && v != 0) {
    const int zero = 0;
    e = cudaMemcpyAsync(p, &zero, sizeof(int), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "hinm_device_status");
  *status_host = v;
  return ok();
}

}  // extern "C"
