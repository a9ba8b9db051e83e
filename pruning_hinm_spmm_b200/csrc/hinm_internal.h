// Internal interface between the C ABI (abi.cu) and the kernels of the HiNM hot path.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "../../include/hinm.h"

namespace hinm {

// The importance matrix as the search and the mask read it: I itself, or (I null) W and
// the channel energies s, from which each value is recomputed bit for bit as
// fl32(fl32(w^2) s_c) (device helpers in stage_rows.cuh).
struct ImpSrc {
  const float* I;
  const uint16_t* W;
  const float* s;
};

// Device status word codes (a subset of hinm_status) written by kernels.
constexpr int kStatusOk = 0;

// Geometry of the compressed layout (see hinm.h, a5).
constexpr int kBlockRows = 128;     // rows per compressed block
constexpr int kDenseBK = 64;        // dense vectors per dense block
constexpr int kSparseBK = 128;      // 2:4 vectors per sparse block (32 groups)
constexpr int kBlockBytes = 16384;  // 128 rows x 128 bytes
constexpr int kMetaWords = 512;     // 128 lanes x 4 words
constexpr int kMaxK = 16384;        // rank sort runs in one CTA's shared memory
constexpr int kMaxCandidates = 64;  // boundary-search candidates per call

struct Candidate {
  int n0, n24, n4;
};

// Host-side closed form (hinm.h, counts).  Returns false on an invalid boundary.
bool counts_from_vs_host(int K, double t_s, double v_s, int out[3]);
// Candidate list of the boundary search; returns the number of candidates (>= 1) or
// -1 when the start boundary itself is invalid.
int search_candidates_host(int K, double t_s, double alpha, Candidate* out, int cap);

// Device address of a __device__ symbol of this library in the current context: resolved
// with cudaGetSymbolAddress once per (device, context) and cached.
struct SymbolCache {
  static constexpr int kDevices = 64;
  std::mutex mu;
  void* ctx[kDevices] = {};
  void* ptr[kDevices] = {};
};
cudaError_t resolve_symbol(SymbolCache& c, const void* symbol, void** out);

// Address of the library's status word on the current device (resolve_symbol).
int* device_status_ptr();

// The CUDA context current on this thread (cuCtxGetCurrent), or nullptr when none is or the
// driver entry point is unavailable.  Handles the library keeps (symbol addresses, function
// attributes, the search's side stream) belong to one context and are made again when it
// changes.
void* current_cuda_context();

// Raises kernel `fn`'s maximum dynamic shared memory on the current device to at least
// `bytes`, calling the runtime only when the limit grows in the current context (the
// attribute belongs to the context's module, and a process may drive several devices).
// Thread-safe; call it before the first launch on each device (and before stream capture).
cudaError_t set_max_dynamic_smem(const void* fn, int bytes);

// Workspace carving helper: 256-byte aligned sub-buffers.
struct Carve {
  char* base;
  size_t off;
  template <class T>
  T* take(size_t count) {
    off = (off + 255) & ~size_t(255);
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off += count * sizeof(T);
    return p;
  }
};

// ---- launchers (all asynchronous on `s`) ----
size_t importance_workspace_bytes(int K);
cudaError_t launch_importance(const uint16_t* W, const uint16_t* X, int M, int K, int N,
                              float* I, float* s_scratch, cudaStream_t s);
// Tile statistics of the boundary search made with I: V (fp64 [M/T][K], channel order) at
// offset 0, the tile maxima (int [M/T]) at tile_stats_v_bytes(), then the channel energies
// s_c (fp32 [K]) at tile_stats_s_offset(), from which I can be recomputed.  I may be null
// (the importance is then not materialized).
size_t tile_stats_v_bytes(int M, int K, int T);
size_t tile_stats_s_offset(int M, int K, int T);
size_t tile_stats_bytes(int M, int K, int T);
cudaError_t launch_importance_stats(const uint16_t* W, const uint16_t* X, int M, int K, int N,
                                    int T, float* I, void* stats, cudaStream_t s);

// Workspace-free variant: channel energies in a static per-device array of kNoAllocMaxK
// floats (64 KiB).
constexpr int kNoAllocMaxK = 16384;
cudaError_t noalloc_energy_scratch(float** out);

size_t search_workspace_bytes(int M, int K, int T, int ncand);
// perm: the working order, [K] shared by every tile (perm_stride 0) or [M/T][K] one per tile
// (perm_stride K), or nullptr (identity).
// stats: from launch_importance_stats for this I and T, or nullptr (computed here from I)
cudaError_t launch_boundary_search(const ImpSrc& I, const void* stats, const int32_t* perm,
                                   long long perm_stride, int M, int K, int T, double t_s, double alpha,
                                   const Candidate* cands, int ncand, int32_t* counts_out,
                                   double* vs_out, int32_t* rank_out, double* retained_out,
                                   void* ws, int* status, cudaStream_t s);

size_t mask_workspace_bytes(int M, int K, int T);
cudaError_t launch_mask(const ImpSrc& I, const int32_t* perm, long long perm_stride,
                        const int32_t* counts,
                        const int32_t* rank, int M, int K, int T, uint32_t* bitmask,
                        int8_t* region, void* ws, int* status, cudaStream_t s);

size_t compress_workspace_bytes(int M, int K, int T);
cudaError_t launch_compress(const uint16_t* W, const uint32_t* bitmask, const int8_t* region,
                            const int32_t* perm, long long perm_stride, const int32_t* counts, int M, int K, int T,
                            const hinm_layout& L, void* ws, int* status, cudaStream_t s);

cudaError_t launch_wait_timeout_selftest(unsigned long long limit_ns, int* status,
                                         cudaStream_t s);

// tile_pairs: the caller's hint that tiles select the same X rows (HINM_SPMM_TILE_PAIRS)
// Gyro-permutation rounds (host; arguments checked by the caller) and the device cost
// matrices of the input rounds.
double gyro_band_cost(const float* I, int T, int K, const int32_t* band, int n);
bool gyro_input_round(const float* I, int T, int K, int32_t* band, const int32_t* groups,
                      const int32_t* slots, int G, int k, int kmeans_iters, double* cost_out);
bool gyro_output_round(const float* I, int M, int K, int T, const int32_t* n0, int32_t* order,
                       const int32_t* tiles, const int32_t* rows, int G, int k, int kmeans_iters,
                       double* cost_out);
cudaError_t launch_gyro_cost(const float* I, int K, int T, int nt, const int32_t* bands, int nb,
                             const int32_t* groups, const int32_t* slots,
                             const int32_t* clusters, int G, int k, double* cost, int* status,
                             cudaStream_t s);

cudaError_t launch_hard_concrete(const float* log_alpha, const float* eps, long long n, float tau,
                                 float* z, uint8_t* hard, double* sums, cudaStream_t s);

cudaError_t launch_translate_index(const hinm_layout& L, const int32_t* row_of_channel,
                                   int* status, cudaStream_t s);

// The SpMM's output: y = act(acc + bias[row]) stored as fp32 to Y, or as bf16 to Yb when Yb
// is set (then Y is unused); bias per output row or nullptr; act one of HINM_ACT_*.
// tile_pairs: the caller's hint that tiles select the same X rows (HINM_SPMM_TILE_PAIRS).
struct SpmmOut {
  float* Y;
  uint16_t* Yb;
  const float* bias;
  int act;
};
cudaError_t launch_spmm(const hinm_layout& L, const uint16_t* X, int N, const SpmmOut& o,
                        bool tile_pairs, int* status, cudaStream_t s);

// Shared by the rank users (search and mask): V (fp64 column sums per tile) and the rank
// of every working position.
// tile_pmax (int [M/T]) receives each tile's largest fp32 exponent; scratch holds
// rank_scratch_bytes() bytes.
size_t rank_scratch_bytes(int M, int K, int T);
cudaError_t launch_vector_rank(const ImpSrc& I, const int32_t* perm, long long perm_stride, int M,
                               int K, int T,
                               double* V, int32_t* rank, int* tile_pmax, void* scratch,
                               cudaStream_t s);

}  // namespace hinm
