/*
 * hinm.h -- C ABI of the B200 (sm_100a) hierarchical N:M (HiNM) hot path:
 *
 *     Y = W_HiNM . X
 *
 * W (M x K, bf16) is cut into tiles of T output rows.  In every tile each input channel
 * restricted to the tile's rows (a "vector") is assigned to one of three regions --
 * dense 4:4, 2:4, or pruned 0:4 -- and the 2:4 vectors keep 2 of every 4 per row.  The
 * product runs on the compressed dense values, the compressed 2:4 values with their
 * 2-bit metadata, and an index of surviving vectors with the input-channel permutation
 * folded in.
 *
 * Sources (page title, section):
 *   [P1] "FlexHiNM-GP: Flexible Hierarchical Pruning via Region Allocation and Channel
 *        Permutation" (papernotes.org notes): 整体框架, 关键设计 1 (three regions, closed
 *        form t_s = v_s + (1 - v_s) p_s / 2, scan of v_s from t_s downward stopping at
 *        the first drop of retained second-order importance), 关键设计 2 (channel
 *        permutation folded into the HiNM index), 关键设计 4 (dense part + 2:4 part
 *        gathered by the precomputed index, summed into one output).
 *   [P2] "面向Transformer的块稀疏剪枝：N:M稀疏模式在硬件加速上的优势" (rkmt.cn), section 二:
 *        keep 2 of every 4 consecutive elements along the input dimension.
 *   [P3] "结构化稀疏与剪枝:2:4 稀疏模式为何能让 GPU 矩阵吞吐翻倍" (geek-doc.cn), section 三:
 *        2 stored values per group plus 2-bit positions; section 五: layer uses W ⊙ M.
 *
 * Conventions shared by every call
 *   - Matrices are row-major and dense: W is M x K, X is K x N, Y is M x N, I is M x K.
 *     bf16 arguments are passed as 16-bit bit patterns (const void*).
 *   - Pointers are DEVICE pointers unless the name ends in _host.  The caller owns all
 *     memory; the library never allocates, frees or synchronises, except the *_size
 *     helpers and hinm_counts_from_vs, which run on the host only.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Work is enqueued asynchronously on it.  The first boundary search on a device also
 *     creates one stream and two events of the library's own (remade if the device's
 *     context is made again); part of every search runs there, forked from and joined
 *     back to `stream` with events, so stream capture sees one graph.
 *   - Kernels are launched with programmatic stream serialization: a launch may begin
 *     while the previous kernel in the stream is still running, but each kernel waits for
 *     the stream's earlier work to finish before it touches memory, so stream order holds
 *     as usual.
 *   - Argument checks run on the host before any launch; a failed check returns an error
 *     status and launches nothing.  hinm_last_error() then describes it.
 *   - Faults detected on the device (a malformed mask in hinm_compress, a wait that
 *     timed out inside a kernel) set a library-owned device status word; kernels then
 *     finish without hanging or trapping.  hinm_device_status() reads and clears it.
 *   - Supported sizes: T in {64, 128}; M % T == 0; 4 <= K <= 16384 and K % 4 == 0;
 *     N % 8 == 0 (16-byte rows for the tensor-memory-accelerator copies); all device
 *     pointers 16-byte aligned; X must be finite (padding multiplies row 0 of X by 0).
 *   - No exception crosses the ABI.
 */
#ifndef HINM_H_
#define HINM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HINM_ABI_VERSION 1
#define HINM_LAYOUT_VERSION 2

typedef enum {
  HINM_OK = 0,
  HINM_ERR_INVALID_ARG = 1,      /* null pointer, NaN parameter, bad enum */
  HINM_ERR_SHAPE = 2,            /* sizes violate the supported-size rules above */
  HINM_ERR_ALIGNMENT = 3,        /* a device pointer is not 16-byte aligned */
  HINM_ERR_UNSUPPORTED = 4,      /* a valid request this library does not implement */
  HINM_ERR_CUDA = 5,             /* a CUDA runtime call failed (launch, memcpy, ...) */
  HINM_ERR_DEVICE_TIMEOUT = 6,   /* device status: a bounded wait gave up */
  HINM_ERR_BAD_MASK = 7,         /* device status: a 2:4 group without exactly 2 kept */
  HINM_ERR_WORKSPACE = 8         /* workspace pointer null or smaller than required */
} hinm_status;

/* Region codes written by hinm_mask (one int8 per tile and input channel). */
#define HINM_REGION_PRUNED 0     /* 0:4 -- vector removed */
#define HINM_REGION_24 1         /* 2:4 -- 2 of every 4 kept per row */
#define HINM_REGION_DENSE 2      /* 4:4 -- vector kept whole */

/* Static description of the strings/versions. */
const char* hinm_status_string(int status);
const char* hinm_last_error(void);          /* detail of the last error on this host thread */
int hinm_abi_version(void);

/* ---------------------------------------------------------------------------------
 * a1. Importance  ([P1] 关键设计 1: second-order importance; 关键设计 2: the importance
 * matrix D)
 *   s_c    = sum_{n=0..N-1} x_cn^2, accumulated in fp64 with n ascending, rounded to fp32
 *   I[i,c] = fl32( fl32(w_ic^2) * s_c )
 * W: bf16 [M][K]; X: bf16 [K][N]; I_out: fp32 [M][K] (written in full).
 * workspace: hinm_importance_workspace_size() bytes (holds s, one fp32 per channel).
 * -------------------------------------------------------------------------------- */
hinm_status hinm_importance_workspace_size(int M, int K, int N, size_t* bytes_host);
hinm_status hinm_importance(const void* W, const void* X, int M, int K, int N,
                            float* I_out, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Workspace-free variant of hinm_importance.  The method's description has no counterpart:
 * this is a deployment convenience for callers that cannot hand the library memory.
 *   Same arguments, layout and result as hinm_importance, without the workspace.  The
 *   channel energies s live in a static per-device array of the library (16384 fp32,
 *   64 KiB); K > 16384 returns HINM_ERR_SHAPE.  The call allocates nothing (no
 *   cudaMalloc / cudaFree, no allocating library routine).  Nothing in the scratch has
 *   to start at zero: every s_c is written before it is read, in stream order.
 *   Calls that overlap on one device (other streams or host threads) share the scratch
 *   and race: order them.  The first call on each device resolves the scratch address
 *   (cudaGetSymbolAddress, device current) and caches it for that device's current
 *   context; a call from a new context (e.g. after cudaDeviceReset) resolves it again.
 *   Make the first call in a context before any stream capture.
 *   Errors: as hinm_importance, plus HINM_ERR_CUDA if the address cannot be resolved.
 */
hinm_status hinm_importance_noalloc(const void* W, const void* X, int M, int K, int N,
                                    float* I_out, void* stream);

/* Importance with the boundary search's tile statistics made in the same pass.  The
 * method's description has no counterpart: the statistics are the search's own first step
 * (a2 below), computed here while I is written so that the search does not read I for them.
 *   I_out: as hinm_importance (bit for bit), or NULL: I is then not written (the _ex search
 *   and mask recompute it from W and these statistics).  stats_out (device,
 *   hinm_tile_stats_size() bytes, caller-owned): V[t][c] = sum over the tile's rows
 *   (ascending, fp64) of I[row, c] by input channel c, each tile's largest importance and
 *   the channel energies s_c; an opaque layout that only the search and the mask read.
 *   The workspace is not used (it may be NULL).  T as for the search (64 or 128).
 *   Errors: as hinm_importance, plus HINM_ERR_SHAPE for T, HINM_ERR_INVALID_ARG for a NULL
 *   or too small stats_out. */
hinm_status hinm_tile_stats_size(int M, int K, int T, size_t* bytes_host);
hinm_status hinm_importance_stats(const void* W, const void* X, int M, int K, int N, int T,
                                  float* I_out, void* stats_out, size_t stats_bytes,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * Region counts for a fixed boundary (host only).  ([P1] 关键设计 1, closed form)
 *   n_24 = 4 * floor(2 (t_s - v_s) K / 4 + 1/2), n_0 = t_s K - n_24 / 2,
 *   n_4 = K - n_0 - n_24.   t_s K must be whole and every count >= 0.
 * out_host[3] = { n_0, n_24, n_4 }.
 * -------------------------------------------------------------------------------- */
hinm_status hinm_counts_from_vs(int K, double t_s, double v_s, int32_t* out_host);

/* ---------------------------------------------------------------------------------
 * a2 + a3. Boundary search  ([P1] 整体框架: every tile runs it; 关键设计 1)
 * Per tile t:
 *   V[t,j]  = sum over the tile's rows (ascending, fp64) of I[row, perm[j]]
 *   rank    = working positions ordered by (V descending, j ascending)
 *   for m = 0..m_max, v_s = t_s - m * alpha, counts from the closed form above;
 *     m_max = floor((t_s - max(0, 2 t_s - 1)) / alpha), trailing candidates with a
 *     negative count dropped; dense = first n_4 ranks, 2:4 = next n_24 (grouped by 4 in
 *     ascending working position, top-2 of I per row, lower position wins ties);
 *     R(m) = exact sum of the importance of every kept element, rounded once to fp64.
 *   Result: the first m with R(m+1) < R(m), else m_max.
 * I: fp32 [M][K]; perm: int32 [K] (NULL = identity), working position j holds channel
 * perm[j]; counts_out: int32 [M/T][3] = {n_0, n_24, n_4}; vs_out: fp64 [M/T];
 * rank_out (NULL allowed): int32 [M/T][K], rank of working position j.
 * retained_out (NULL allowed): fp64 [M/T][n_cand], R(m) of every tile and candidate
 * (n_cand from hinm_search_num_candidates).
 * alpha > 0, 0 <= t_s <= 1.  workspace: hinm_search_workspace_size() bytes.
 * -------------------------------------------------------------------------------- */
hinm_status hinm_search_num_candidates(int K, double t_s, double alpha, int32_t* n_host);
hinm_status hinm_search_workspace_size(int M, int K, int T, double t_s, double alpha,
                                       size_t* bytes_host);
hinm_status hinm_boundary_search(const float* I, const int32_t* perm, int M, int K, int T,
                                 double t_s, double alpha, int32_t* counts_out,
                                 double* vs_out, int32_t* rank_out, double* retained_out,
                                 void* workspace, size_t workspace_bytes, void* stream);
/* hinm_boundary_search with the tile statistics that hinm_importance_stats made with this
 * I (same M, K, T): the same results, without the search's own pass over I for V.  stats
 * from another I or T give meaningless results (nothing checks that they match).
 * Errors: as hinm_boundary_search, plus HINM_ERR_INVALID_ARG for a NULL or too small
 * stats. */
hinm_status hinm_boundary_search_stats(const float* I, const void* stats, size_t stats_bytes,
                                       const int32_t* perm, int M, int K, int T, double t_s,
                                       double alpha, int32_t* counts_out, double* vs_out,
                                       int32_t* rank_out, double* retained_out,
                                       void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * a4. Mask  ([P1] 亮点与洞察: high -> dense, middle -> 2:4, low -> pruned;
 *            [P2] 二: 2 of every 4; [P3] 五: M has W's shape)
 * counts: int32 [M/T][3] (device; n_24 % 4 == 0, n_0 + n_24 + n_4 == K);
 * rank: int32 [M/T][K] from hinm_boundary_search, or NULL to recompute it from I.
 * bitmask_out: uint32 [M][ceil(K/32)], bit b of word w of row i = channel 32w+b kept
 * (bits past K are 0).  region_out: int8 [M/T][K] by original channel (HINM_REGION_*).
 * workspace: hinm_mask_workspace_size() bytes.
 * -------------------------------------------------------------------------------- */
hinm_status hinm_mask_workspace_size(int M, int K, int T, size_t* bytes_host);
hinm_status hinm_mask(const float* I, const int32_t* perm, const int32_t* counts,
                      const int32_t* rank, int M, int K, int T, uint32_t* bitmask_out,
                      int8_t* region_out, void* workspace, size_t workspace_bytes,
                      void* stream);

/* ---------------------------------------------------------------------------------
 * a5. Compressed HiNM layout  ([P1] 关键设计 2/4, [P3] 三)
 * Per tile: dense vectors (ascending working position) in blocks of 64, 2:4 vectors in
 * blocks of 128 (32 groups of 4).  Every block is 128 rows (rows >= T are zero) and is
 * stored exactly as the tensor cores read it from shared memory:
 *   value block  16384 B: bf16 (r, k) at r*128 + ((k/8) XOR (r%8))*16 + (k%8)*2
 *                (dense: k = vector in block; 2:4: k = 2*group + slot, slot 0 = lower
 *                kept position);
 *   meta block    2048 B: 128 lanes x 4 uint32 words; word w of lane L, bits
 *                [16s+4q, 16s+4q+4) = a | b<<2 (a < b, kept positions 0..3) of group
 *                8w + 4((L/8)%2) + q of row 16(L/16) + 8s + L%8;
 *   index         int32 per vector = perm[j] (input channel), 0 for padding;
 *   run           int32 per block = index[0] if the block's indices are one ascending
 *                 run index[0], index[0]+1, ..., else -1 (such blocks of X load as a tile).
 * Padding: value 0, nibble 0x4, index 0.
 * tile_info[t] = { dense blocks, sparse blocks, first dense block, first sparse block }.
 * -------------------------------------------------------------------------------- */
typedef struct {
  int32_t layout_version;     /* must be HINM_LAYOUT_VERSION */
  int32_t M, K, T, num_tiles; /* num_tiles = M / T */
  int32_t max_dense_blocks;   /* capacity of vals_dense / idx_dense in blocks */
  int32_t max_sparse_blocks;  /* capacity of vals_sparse / meta / idx_sparse in blocks */
  int32_t* tile_info;         /* device int32 [num_tiles][4] (written by hinm_compress) */
  uint16_t* vals_dense;       /* device bf16 [max_dense_blocks][8192] */
  uint16_t* vals_sparse;      /* device bf16 [max_sparse_blocks][8192] */
  uint32_t* meta;             /* device uint32 [max_sparse_blocks][512] */
  int32_t* idx_dense;         /* device int32 [max_dense_blocks][64] */
  int32_t* idx_sparse;        /* device int32 [max_sparse_blocks][128] */
  int32_t* run_dense;         /* device int32 [max_dense_blocks] */
  int32_t* run_sparse;        /* device int32 [max_sparse_blocks] */
} hinm_layout;

typedef struct {
  int32_t max_dense_blocks, max_sparse_blocks;
  size_t tile_info_bytes, vals_dense_bytes, vals_sparse_bytes, meta_bytes,
      idx_dense_bytes, idx_sparse_bytes, run_dense_bytes, run_sparse_bytes;
} hinm_layout_sizes;

/* Buffer sizes.  counts_host (int32 [M/T][3], host) gives exact sizes; NULL gives the
 * worst case over all valid counts (ceil(K/64)+1 dense and ceil(K/128)+1 sparse blocks
 * per tile), which needs no device-to-host copy of the search result. */
hinm_status hinm_compress_size(const int32_t* counts_host, int M, int K, int T,
                               hinm_layout_sizes* out_host);
hinm_status hinm_compress_workspace_size(int M, int K, int T, size_t* bytes_host);
/* W: bf16 [M][K]; bitmask/region: from hinm_mask; counts: device int32 [M/T][3].
 * `layout` (host struct) holds caller-allocated device buffers of the sizes above.
 * A 2:4 group whose row does not have exactly 2 kept bits sets HINM_ERR_BAD_MASK in the
 * device status word (that group is then packed from its first two kept bits). */
hinm_status hinm_compress(const void* W, const uint32_t* bitmask, const int8_t* region,
                          const int32_t* perm, const int32_t* counts, int M, int K, int T,
                          const hinm_layout* layout, void* workspace,
                          size_t workspace_bytes, void* stream);

/* Per-tile working orders  ([P1] 关键设计 2: the input-channel permutation is found inside
 * each tile, and it is folded into the tile's HiNM index).  The _ex forms of the search,
 * the mask and compress take perm_per_tile: 0 = perm is one order int32 [K] for every tile
 * (the calls above), 1 = perm is int32 [M/T][K], row t the working order of tile t (each
 * row a permutation of 0..K-1; a bad row sets HINM_ERR_INVALID_ARG in the device status
 * word, as for the shared order).  Working position j of tile t holds channel perm[t][j]:
 * the tile's 2:4 groups are 4 consecutive 2:4 channels in that order, and compress folds
 * perm[t] into tile t's index, so the SpMM needs nothing else.  The same perm and flag must
 * be given to the three calls.  Other arguments, results and errors as the calls above;
 * hinm_boundary_search_ex covers both search forms (stats may be NULL).
 * The importance need not be materialized: with I NULL, the search and the mask recompute
 * every value they read from W (device bf16 [M][K]) and the channel energies that
 * hinm_importance_stats stored in `stats` (for this W, X and T), as fl32(fl32(w^2) s_c) --
 * the same bits as I -- reading 2 bytes per weight instead of 4.  With I given, W may be
 * NULL.  Errors: HINM_ERR_INVALID_ARG for I NULL without W and stats. */
hinm_status hinm_boundary_search_ex(const float* I, const void* W, const void* stats,
                                    size_t stats_bytes, const int32_t* perm, int perm_per_tile,
                                    int M, int K, int T, double t_s, double alpha,
                                    int32_t* counts_out, double* vs_out, int32_t* rank_out,
                                    double* retained_out, void* workspace,
                                    size_t workspace_bytes, void* stream);
hinm_status hinm_mask_ex(const float* I, const void* W, const void* stats, size_t stats_bytes,
                         const int32_t* perm, int perm_per_tile, const int32_t* counts,
                         const int32_t* rank, int M, int K, int T, uint32_t* bitmask_out,
                         int8_t* region_out, void* workspace, size_t workspace_bytes,
                         void* stream);
hinm_status hinm_compress_ex(const void* W, const uint32_t* bitmask, const int8_t* region,
                             const int32_t* perm, int perm_per_tile, const int32_t* counts,
                             int M, int K, int T, const hinm_layout* layout, void* workspace,
                             size_t workspace_bytes, void* stream);

/* Gyro-permutation  ([P1] 关键设计 2: channel permutation reorders input and output
 * channels without changing the product, so that important weights land where they are
 * kept; the pipeline is output-channel permutation -> column-vector pruning -> in-tile
 * input-channel permutation, and each round samples vectors per tile, clusters them with a
 * balanced K-means and assigns the clusters by the Hungarian algorithm on the pruning-cost
 * matrix, smaller cost better; iterated to refine).  Offline, once per layer; its outputs
 * are the permutations the hot path takes: a per-tile working order (perm_per_tile of
 * hinm_boundary_search_ex / hinm_mask_ex / hinm_compress_ex) and an output-row order.
 * All costs are row-ascending fp64 sums of fp32 importances, so the host calls, the device
 * call and an fp64 reference agree bit for bit.
 *
 * In-tile input-channel round.  band: the tile's 2:4-region channels in working order
 * (groups = 4 consecutive entries), host int32 [n], n % 4 == 0, 4 <= n <= K, distinct
 * entries in [0, K), refined in place.  The caller's random draws choose G distinct groups
 * (groups: host int32 [G], in [0, n/4)) and k distinct slots in each (slots: host int32
 * [G][k], in [0, 4), 1 <= k <= 4); the S = G k sampled vectors (sample i k + j = the vector
 * in slot slots[i][j] of group groups[i]) leave their slots.  Reading of the pages: their
 * features are their importance columns over the tile's rows; a balanced K-means (seeded
 * by source group; Lloyd steps whose assignment is the min-cost assignment of the samples
 * to G clusters x k seats under the squared distance; at most kmeans_iters steps, stopping
 * when the partition repeats) groups them into G clusters of k; cost[c][i] = the pruning
 * cost of group groups[i] (per row the two smallest of its four values) with its sampled
 * slots, ascending, holding cluster c's vectors in ascending sample order; the min-cost
 * assignment places the clusters, and the result is kept only if the sampled groups' total
 * cost does not rise.  cost_out (NULL allowed): host fp64 [2] = {before, after}.
 * I_tile: host fp32 [T][K], the tile's importance rows by channel; every value the round
 * reads must be finite.  Errors (before any work): HINM_ERR_SHAPE, HINM_ERR_INVALID_ARG. */
hinm_status hinm_gyro_input_round_host(const float* I_tile, int T, int K, int32_t* band, int n,
                                       const int32_t* groups, const int32_t* slots, int G, int k,
                                       int kmeans_iters, double* cost_out);

/* Pruning cost of a whole band (fp64 sum over its groups, ascending): host. */
hinm_status hinm_gyro_band_cost_host(const float* I_tile, int T, int K, const int32_t* band,
                                     int n, double* cost_host);

/* The input rounds' cost matrices of every tile of a layer on the GPU (the G x G x T part):
 *   cost_out[t][c][i] = pruning cost of tile t's group groups[t][i] with its slots
 *   slots[t][i][0..k) (ascending) holding the vectors of cluster c, clusters[t][c][0..k)
 *   (ascending sample indices p in [0, G k), sample p = slot slots[t][p/k][p%k] of group
 *   groups[t][p/k]).
 * I: device fp32 [M][K] (tile t = rows t T .. t T + T - 1); bands: device int32
 * [M/T][band_len]; groups [M/T][G], slots [M/T][G][k], clusters [M/T][G][k]: device int32;
 * cost_out: device fp64 [M/T][G][G].  1 <= k <= 4, 1 <= G <= band_len / 4.  A channel
 * outside [0, K) is read as channel 0 and reported as HINM_ERR_INVALID_ARG in the device
 * status word; the other indices must be valid (they are not checked on the device). */
hinm_status hinm_gyro_cost_matrix(const float* I, int M, int K, int T, const int32_t* bands,
                                  int band_len, const int32_t* groups, const int32_t* slots,
                                  const int32_t* clusters, int G, int k, double* cost_out,
                                  void* stream);

/* Output-channel round over a layer's tiles, on the host.  row_order: host int32 [M], a
 * permutation of 0..M-1 listing the output channels in their current order (tile t holds
 * row_order[t T .. t T + T - 1]), refined in place.  The caller's draws choose G distinct
 * tiles (tiles: host int32 [G]) and k distinct positions in each (rows: host int32 [G][k],
 * in [0, T)).  Reading: the S = G k output channels leave their positions; their features
 * are their importance rows; the balanced K-means (as above) groups them into G clusters of
 * k; cost[c][i] = the column-vector pruning cost of tile tiles[i] with its sampled
 * positions, ascending, holding cluster c's channels: the sum of the tile's n0[tile]
 * smallest vector scores (column sums over the tile's rows in their order, fp64; ties by
 * channel), summed ascending; the min-cost assignment places the clusters, kept only if the
 * sampled tiles' total cost does not rise.  The layer then computes W[row_order] and yields
 * Y[row_order]; hinm_translate_index with the inverse order lets the next layer read it.
 * I: host fp32 [M][K] (rows = output channels, by channel); n0: host int32 [M/T], in
 * [0, K].  cost_out (NULL allowed): host fp64 [2] = {before, after}.
 * Errors (before any work): HINM_ERR_SHAPE, HINM_ERR_INVALID_ARG. */
hinm_status hinm_gyro_output_round_host(const float* I, int M, int K, int T, const int32_t* n0,
                                        int32_t* row_order, const int32_t* tiles,
                                        const int32_t* rows, int G, int k, int kmeans_iters,
                                        double* cost_out);

/* Hard-Concrete soft 2:4 mask, forward  ([P1] 关键设计 3: each group of 4 has learnable
 * logits log alpha; with noise eps ~ U(0, 1) the soft mask is
 *   s = sigmoid((log eps - log(1 - eps) + log alpha) / tau),
 * stretched to (-0.1, 1.1) and clipped to [0, 1]; the regularisers are mean(z) and the mean
 * over groups of |sum of the group's z - 2|; the hardened mask thresholds z at 0.5).
 *   z_i = min(1, max(0, 1.2 s_i - 0.1)) (fp32, with CUDA's logf and expf; the noise logit
 *   as logf of eps / (1 - eps))
 * log_alpha, eps: device fp32 [n], n % 4 == 0, groups = 4 consecutive elements; eps is the
 * caller's noise (eps = 1/2 everywhere gives the deterministic mask; eps = 0 or 1 give
 * z = 0 or 1; NaN in, NaN out).  tau > 0.
 * z_out: fp32 [n].  hard_out (NULL allowed): uint8 [n], 1 where z > 0.5.
 * sums_out (NULL allowed): fp64 [2] = { sum z, sum over groups |sum z - 2| } (zeroed by the
 * call, then added to in an unspecified order: the last bits may differ between calls).
 * Errors: HINM_ERR_SHAPE (n), HINM_ERR_INVALID_ARG (tau, NULL), HINM_ERR_ALIGNMENT. */
hinm_status hinm_hard_concrete_forward(const float* log_alpha, const float* eps, long long n,
                                       float tau, float* z_out, uint8_t* hard_out,
                                       double* sums_out, void* stream);

/* Cross-layer index translation  ([P1] 关键设计 2: channel reordering leaves the result
 * unchanged, and the translation between layers is folded into the HiNM index).
 * For an X whose rows arrive reordered -- row r holds input channel sigma[r], e.g. the
 * previous layer's output in its own permuted row order -- rewrites the layout in place:
 * every vector index c becomes row_of_channel[c] (= sigma^-1[c]) and every block's run flag
 * is recomputed.  hinm_spmm(translated layout, reordered X) then equals hinm_spmm(layout,
 * X) bit for bit, with no reordering of X at run time.
 * row_of_channel: device int32 [K], a permutation of 0..K-1 (an entry outside [0, K) sets
 * HINM_ERR_INVALID_ARG in the device status word and maps to row 0; a repeated entry is not
 * detected and gives a different product).  Values, metadata and tile_info are untouched. */
hinm_status hinm_translate_index(const hinm_layout* layout, const int32_t* row_of_channel,
                                 void* stream);

/* ---------------------------------------------------------------------------------
 * a6. SpMM  ([P1] 关键设计 4: Y = dense part + 2:4 part, one output)
 *   Y[t*T + r, n] = sum over dense vectors v of Wd[r, v] * X[idx_d(v), n]
 *                 + sum over 2:4 groups of the 2 kept values times their gathered X rows,
 * accumulated in fp32 on the tensor cores (dense and sparse MMA into one accumulator).
 * X: bf16 [K][N]; Y_out: fp32 [M][N] (written in full).
 * -------------------------------------------------------------------------------- */
hinm_status hinm_spmm(const hinm_layout* layout, const void* X, int N, float* Y_out,
                      void* stream);

/* hinm_spmm with flags (0 = hinm_spmm).  Same arguments, layout, result and errors; an
 * unknown flag bit returns HINM_ERR_INVALID_ARG.
 *   HINM_SPMM_TILE_PAIRS: a performance hint from a caller that knows its tiles select the
 *   same X rows, i.e. every tile has one region (all 2:4 or all dense) and the permutation
 *   is ascending, so that every block of X is one run of rows.  With T == 128 and N >= 1024
 *   the SpMM then takes tiles two at a time (2p, 2p+1) on 240-column blocks: where both
 *   tiles' blocks are the same runs (checked on the device, pair by pair) one copy of each
 *   X block feeds the tensor-core products of both.  A pair that differs runs tile by tile:
 *   the result is the same, only slower.  Otherwise ignored. */
#define HINM_SPMM_TILE_PAIRS 1
hinm_status hinm_spmm_ex(const hinm_layout* layout, const void* X, int N, float* Y_out,
                         int flags, void* stream);

/* hinm_spmm_ex with a fused epilogue (an extension of a6: the pages merge the two
 * parts into one output and name no epilogue; [reading] per output row bias, an activation
 * and a bf16 output, applied to the fp32 accumulator before the one store of Y):
 *   y[i, n] = act(acc[i, n] + bias[i])   (bias NULL: 0; act HINM_ACT_*)
 * stored as fp32 to Y_out (fp32 [M][N]) or, with out_bf16 != 0, as bf16 (round to nearest
 * even) to Y_out (bf16 [M][N]), which halves the bytes of Y.  ReLU max(x, 0); SiLU
 * x / (1 + exp(-x)); GELU x (1 + erf(x / sqrt 2)) / 2 -- with CUDA's expf and erff.
 * bias: device fp32 [M] or NULL.  Errors: as hinm_spmm_ex, plus HINM_ERR_INVALID_ARG for an
 * unknown activation. */
#define HINM_ACT_NONE 0
#define HINM_ACT_RELU 1
#define HINM_ACT_SILU 2
#define HINM_ACT_GELU 3
hinm_status hinm_spmm_epilogue(const hinm_layout* layout, const void* X, int N, void* Y_out,
                               const float* bias, int activation, int out_bf16, int flags,
                               void* stream);

/* Diagnostic with no counterpart in the pages: launches one small kernel whose bounded
 * wait cannot complete (it waits on an mbarrier nothing arrives at), so that after about
 * limit_ns nanoseconds it records HINM_ERR_DEVICE_TIMEOUT and returns, exercising the
 * timeout path of every pipelined kernel.  0 < limit_ns <= 2e9, else HINM_ERR_INVALID_ARG.
 * Read the result with hinm_device_status(); the context stays usable. */
hinm_status hinm_selftest_wait_timeout(unsigned long long limit_ns, void* stream);

/* Reads the device status word into *status_host (0 = no fault; else an hinm_status)
 * and clears it.  Synchronises `stream`. */
hinm_status hinm_device_status(void* stream, int32_t* status_host);

#ifdef __cplusplus
}
#endif

#endif /* HINM_H_ */
