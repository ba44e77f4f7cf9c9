/*
 * msa.h - modality-aware permutation sparse attention for long-context prefill
 * on NVIDIA B200 (sm_100a).  C ABI of libmsa.so.
 *
 * The method (MMInference, ICML 2025, building on MInference 1.0, NeurIPS 2024):
 * every attention head is assigned a sparse pattern offline; online, for each
 * prefill, a sparse index is estimated per head from the last 64 queries (or
 * from 64-token mean-pooled blocks), Q/K/V are permuted so the selected entries
 * become contiguous, block-sparse causal attention runs over only those blocks,
 * and the output is permuted back.  The four steps are the four calls
 *   msa_estimate -> msa_permute -> msa_sparse_prefill -> msa_unpermute,
 * or, with the permutation realised as index-based loading inside the attention
 * kernel, the two calls
 *   msa_estimate -> msa_sparse_prefill_indexed.
 *
 * Conventions shared by every call
 *  - Tensors are bf16, d = 128 contiguous elements per row.  Q and O are
 *    [Hq, L, 128], K and V are [Hkv, L, 128], addressed through msa_strides
 *    (element strides between heads and between rows), so [L, H, 128] works
 *    as well.  Base pointers must be 16-byte aligned and strides multiples of
 *    8 elements.  Query head h reads key/value head h / (Hq / Hkv).
 *  - Causality is always j <= i in ORIGINAL token positions.
 *  - All device pointers are owned by the caller; the library never allocates
 *    or frees device memory.  Scratch lives in one caller-provided workspace of
 *    msa_workspace_bytes() bytes (msa_workspace_bytes_indexed() for the two-call
 *    path), 256-byte aligned, which carries the estimated indices and permuted
 *    tensors from one call to the next: pass the same workspace to the calls of
 *    one prefill and do not reuse it for another prefill until the last call has
 *    completed on the stream.
 *  - Calls are asynchronous and stream-ordered on the cudaStream_t passed as
 *    `stream` (NULL = legacy default stream); only the inspection calls
 *    (msa_read_indices, msa_read_tiles, msa_tile_stats, msa_mask_pairs) and
 *    msa_device_status synchronise.
 *  - Argument errors are returned before any launch.  Conditions found on the
 *    device (a bounded wait that expired, an index outside its buffer) are
 *    recorded in the workspace and reported by msa_device_status; kernels never
 *    trap.
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1,   /* null pointer, unknown kind, negative budget, ... */
  MSA_ERR_SHAPE = 2,         /* d != 128, L % 64 != 0, Hq % Hkv != 0, segments not tiling [0, L) */
  MSA_ERR_ALIGN = 3,         /* pointer not 16-byte (workspace: 256-byte) aligned, stride not a multiple of 8 */
  MSA_ERR_WORKSPACE = 4,     /* workspace smaller than the call needs (msa_workspace_bytes[_indexed]()) */
  MSA_ERR_UNSUPPORTED = 5,   /* a valid problem outside this build's limits (see msa_status_string) */
  MSA_ERR_CUDA = 6,          /* a CUDA runtime/driver call failed */
  MSA_ERR_TIMEOUT = 7,       /* device: a bounded wait expired (reported by msa_device_status) */
  MSA_ERR_DEVICE_BOUNDS = 8, /* device: an index fell outside its buffer (reported by msa_device_status) */
  MSA_ERR_STATE = 9          /* calls out of order for this workspace */
} msa_status;

/* modality of a token */
enum { MSA_TEXT = 0, MSA_VIDEO = 1 };

/* Sparse pattern of one attention head (MInference 1.0, "Approach"; MMInference, "key machinery").
 *  DENSE   : causal attention, no sparsity.
 *  ASHAPE  : attention sinks + local window: j < sink or i - j < local (static, no estimation).
 *  VSLASH  : vertical lines V (keys) and slash lines S (offsets i - j), top k_v / k_s of the
 *            last-64-query attention reduced per key / per offset.
 *  BLOCK   : 64x64 blocks; per query block the top-k key blocks of the mean-pooled logits.
 *  GRID    : video grid (MMInference Algorithm 1): stride s and phases P searched online from
 *            the last 64 video queries; queries and keys on the (s, P) lines attend / are attended
 *            densely, text queries attend densely, plus a local band of `local` (default 64).
 *  QBOUND  : Q-boundary (Algorithm 2): vertical-slash per query modality.  With the head flag
 *            MSA_HEAD_PER_SEGMENT: vertical-slash per modality segment, each segment's lines
 *            estimated from its own last 64 queries (all of them if shorter) and serving only
 *            that segment's queries (the MMInference review page's "last 64 queries of each
 *            modality segment", read literally; the default estimates once per modality, from
 *            its last segment, and extrapolates across the others, "key machinery").
 *  BOUND2D : 2D-boundary (Algorithm 3): per (query modality, key modality) pair; intra-modality
 *            pairs are vertical-slash in within-modality ranks, cross pairs vertical only. */
typedef enum {
  MSA_DENSE = 0,
  MSA_ASHAPE = 1,
  MSA_VSLASH = 2,
  MSA_BLOCK = 3,
  MSA_GRID = 4,
  MSA_QBOUND = 5,
  MSA_BOUND2D = 6
} msa_kind;

#define MSA_MAX_STRIDES 8

typedef struct {
  int32_t kind;        /* msa_kind */
  int32_t sink;        /* ASHAPE: sink tokens */
  int32_t local;       /* ASHAPE: local window; GRID: local band (0 = 64) */
  int32_t k_v;         /* VSLASH/QBOUND: vertical lines; BOUND2D: scaled per key modality, max(1, round(k_v n_b / L)) */
  int32_t k_s;         /* VSLASH/QBOUND: slash lines;    BOUND2D: max(1, round(k_s n_a / L)) per query modality */
  int32_t topk_blocks; /* BLOCK: key blocks per query block (> 0), else block_budget is used */
  double block_budget; /* BLOCK: keep ceil(block_budget * (b + 1)) blocks in query block b */
  int32_t n_strides;   /* GRID: candidate strides (1..MSA_MAX_STRIDES) */
  int32_t strides[MSA_MAX_STRIDES];
  int32_t n_phases;    /* GRID: phases kept (> 0), else max(1, floor(grid_budget * s / 2)) */
  int32_t flags;       /* MSA_HEAD_* options (0: none) */
  double grid_budget;
} msa_head_cfg;

/* msa_head_cfg.flags: QBOUND only, one index per modality segment (see MSA_QBOUND) */
#define MSA_HEAD_PER_SEGMENT 1

typedef struct {
  int64_t start, len; /* token range [start, start + len) */
  int32_t modality;   /* MSA_TEXT or MSA_VIDEO */
  int32_t _pad;
} msa_segment;

typedef struct {
  int64_t L;                   /* sequence length, a multiple of 64 */
  int32_t Hq, Hkv, d;          /* d must be 128; Hq a multiple of Hkv */
  float scale;                 /* softmax scale, e.g. 1/sqrt(128) */
  int32_t n_segments;          /* ordered segments tiling [0, L) */
  const msa_segment* segments; /* host pointer, copied by msa_plan_create */
  const msa_head_cfg* heads;   /* host pointer [Hq], copied by msa_plan_create */
} msa_problem;

/* element strides of the four tensors; the 128-element d axis is contiguous */
typedef struct {
  int64_t q_head, q_row;
  int64_t k_head, k_row;
  int64_t v_head, v_row;
  int64_t o_head, o_row;
} msa_strides;

typedef struct msa_plan msa_plan;

/* Validates the problem and sizes the workspace.  Host only: no device work, no
 * allocation on the device.  On success *out owns a host copy of every table. */
msa_status msa_plan_create(const msa_problem* problem, msa_plan** out);
void msa_plan_destroy(msa_plan* plan);

/* Bytes of device workspace one prefill with this plan needs (msa_permute, msa_sparse_prefill
 * and msa_unpermute). */
size_t msa_workspace_bytes(const msa_plan* plan);

/* Bytes of device workspace the index-based path needs (msa_estimate or msa_set_indices, then
 * msa_sparse_prefill_indexed): the same layout without its trailing permuted Q and O copies. */
size_t msa_workspace_bytes_indexed(const msa_plan* plan);

/* Online index estimation (MInference 1.0 "Approach": last-64-query vertical/slash sums,
 * 64-block mean pooling; MMInference "key machinery": grid stride/phase search, per-modality
 * estimation from the 64 latest queries of every modality), followed by the
 * per-head row classes, gathered-key lists, line bitmaps and executed-tile lists.
 * Reads Q and K (device), writes only the workspace (ws_bytes >= msa_workspace_bytes_indexed;
 * the same holds for msa_set_indices). */
msa_status msa_estimate(msa_plan* plan, const void* Q, const void* K, const msa_strides* strides, void* ws,
                        size_t ws_bytes, void* stream);

/* Host-provided index sets instead of msa_estimate (indices reused across prefills, or fixed
 * ones).  One msa_head_indices per query head; fields a head's kind does not use are ignored.
 * Lists are host pointers, sorted ascending, copied before the call returns. */
typedef struct {
  int32_t stride;          /* GRID: chosen stride */
  int32_t n_phases;        /* GRID: phases (< stride) */
  const int32_t* phases;
  int32_t n_v[2][2];       /* vertical lines, token positions: VSLASH [0][0]; QBOUND [a][0] for query
                              modality a over all keys; BOUND2D [a][b] keys of modality b */
  const int32_t* v[2][2];
  int32_t n_s[2];          /* slash lines (offsets): VSLASH [0]; QBOUND [a]; BOUND2D [a] in ranks */
  const int32_t* s[2];
  const int32_t* blk_ptr;  /* BLOCK: CSR over query blocks, blk_ptr[L/64 + 1] */
  const int32_t* blk_idx;  /* BLOCK: selected key blocks (each row ascending, c <= b) */
  /* QBOUND with MSA_HEAD_PER_SEGMENT: lines of each segment k (n_seg = the problem's segment
   * count): vertical positions seg_v[k][0 .. seg_nv[k]) and slash offsets seg_s[k][0 .. seg_ns[k]) */
  int32_t n_seg;
  const int32_t* seg_nv;
  const int32_t* const* seg_v;
  const int32_t* seg_ns;
  const int32_t* const* seg_s;
} msa_head_indices;

msa_status msa_set_indices(msa_plan* plan, const msa_head_indices* heads, void* ws, size_t ws_bytes,
                           void* stream);

/* Permutation (MMInference "core discovery": row-wise grouping of same-modality queries,
 * column-wise gathering of selected keys, 2D modality-pair grouping).  Gathers permuted Q
 * rows, gathered K/V lines and modality-grouped K/V into the workspace. */
msa_status msa_permute(msa_plan* plan, const void* Q, const void* K, const void* V, const msa_strides* strides,
                       void* ws, size_t ws_bytes, void* stream);

/* Block-sparse causal flash attention over the executed tiles (MMInference "key machinery":
 * kernels that load only the permuted blocks and keep the tensor-core compute dense;
 * "Grid-Shape Flash Attention", Algorithm 5).  Writes the permuted output into the workspace
 * and, if lse != NULL, the natural-log softmax normaliser per query, lse[h * L + i] (fp32,
 * -inf for a query with no allowed key; such a query's output row is 0). */
msa_status msa_sparse_prefill(msa_plan* plan, const void* Q, const void* K, const void* V,
                              const msa_strides* strides, void* ws, size_t ws_bytes, float* lse, void* stream);

/* Scatters the permuted output back to original token order into O (bf16, device):
 * O[h][pos(r)] = O_perm[h][r] for every permuted row r.  The MMInference review page ("core
 * discovery") requires the permutation to leave a head's output unchanged; this inverse
 * gather is what makes the permuted computation return rows in the caller's order.  Output
 * rows of identity (unpermuted) heads are copied as they are.  Layout and strides as for Q in
 * msa_permute; asynchronous on `stream`. */
msa_status msa_unpermute(msa_plan* plan, const void* ws, size_t ws_bytes, void* O, const msa_strides* strides,
                         void* stream);

/* Index-based sparse prefill, in place of msa_permute + msa_sparse_prefill + msa_unpermute
 * (MMInference "core discovery": the permutations are realised as index-based sparse loading
 * inside the attention kernel).  The query rows of permuted row classes are gathered by row
 * index from Q into the kernel's query tiles, and every output row is written straight to O
 * (bf16, device, strides->o_head / o_row) at its original position; the gathered key lines and
 * the modality-grouped keys are still copied into the workspace first (one pass over K / V).
 * Same values as the three-call path (same operations in the same order).  lse as for
 * msa_sparse_prefill.  ws_bytes >= msa_workspace_bytes_indexed; asynchronous on `stream`;
 * MSA_ERR_STATE if the workspace holds no indices of this plan. */
msa_status msa_sparse_prefill_indexed(msa_plan* plan, const void* Q, const void* K, const void* V, void* O,
                                      const msa_strides* strides, void* ws, size_t ws_bytes, float* lse,
                                      void* stream);

/* ---- inspection (synchronising) ---- */

/* Copies head `head`'s raw index sets to the host as a flat int32 record:
 *   kind, stride, n_phases, phases[n_phases],
 *   for a in {0,1}, b in {0,1}: n_v[a][b], v[a][b][...],
 *   for a in {0,1}: n_s[a], s[a][...],
 *   nb, blk_ptr[nb + 1], blk_idx[blk_ptr[nb]]          (nb = 0 unless BLOCK)
 *   n_seg, then per segment k: n_v, v[...], n_s, s[...]  (n_seg = 0 unless QBOUND with
 *                                                         MSA_HEAD_PER_SEGMENT)
 * `*len` is the capacity of `out` in int32 on entry and the record length on return
 * (MSA_ERR_INVALID_ARG with the needed length if too small). */
msa_status msa_read_indices(const msa_plan* plan, const void* ws, int32_t head, int32_t* out, int64_t* len,
                            void* stream);

/* Executed-tile statistics of the last msa_estimate / msa_set_indices in this workspace:
 * tiles[0] = executed 128x128 tiles, tiles[1] = work items (128-query tiles) with work.
 * Executed block FLOPs = 4 * 128 * 128 * 128 * tiles[0]. */
msa_status msa_tile_stats(const msa_plan* plan, const void* ws, int64_t tiles[2], void* stream);

/* Executed 128 x 128 tiles of each query head (host int64 [Hq]) under the tile lists of the last
 * msa_estimate / msa_set_indices in `ws` (the FLOPs accounting of the MInference 1.0 and MMInference
 * pages, per head: how much of the dense causal work each head's pattern executes).  Reads the
 * per-item tile counts on `stream` and synchronises it. */
msa_status msa_tile_stats_heads(const msa_plan* plan, const void* ws, int64_t* tiles, void* stream);

/* Allowed (query, key) pairs of each query head under the masks of the last msa_estimate /
 * msa_set_indices in this workspace: causal in original positions and the head's pattern, each
 * pair once (MInference / MMInference: the token-level masks of the A-shape, vertical-slash,
 * block-sparse, grid, Q-boundary and 2D-boundary heads).  counts: host int64 [Hq].  Useful
 * FLOPs = 4 * d * sum(counts); the executed block FLOPs of msa_tile_stats also count the masked
 * entries of the executed tiles.  Runs a counting kernel over the tile lists with the attention
 * kernel's mask logic on `stream` and synchronises it; MSA_ERR_STATE if the workspace holds no
 * indices of this plan. */
msa_status msa_mask_pairs(const msa_plan* plan, void* ws, int64_t* counts, void* stream);

/* How msa_sparse_prefill divides its work (host only, no device access): out[0] = work units,
 * out[1] = key chunks, out[2] = unit bands (0 when the keys are not chunked).  When one head's
 * K and V exceed about 96 MB (L > 192K tokens) the keys are cut into chunks of 131072 (the
 * environment variable MSA_ATTN_CHUNK_KEYS, a multiple of 128, read at msa_plan_create,
 * overrides the chunk size; 0 turns chunking off): the units of a band of work items then run
 * chunk by chunk so that the units in flight share one chunk of K and V in L2, and a work
 * item's online-softmax state passes from chunk to chunk through an accumulator slot in the
 * workspace.  Alternate bands share two sets of slots; a unit writes a slot only after every
 * unit of the band that used it before has finished.  Bands are runs of up to 1024 query-tile
 * slots of one KV head, key source and head kind, merged up to at least 2048 units
 * (MSA_ATTN_BAND_SLOTS and MSA_ATTN_MIN_BAND_UNITS, read at msa_plan_create, override the two
 * numbers).  The result does not depend on the chunking or the bands beyond rounding. */
msa_status msa_attention_units(const msa_plan* plan, int64_t out[3]);

/* Dumps the work list of head `head` for tests: for each of its 128-query work items the
 * query positions covered (-1 for padding) and, for every executed tile, its key source
 * (0 = keys in original order, 1 = modality-grouped keys, 2 = gathered keys; plus 8 when every
 * query of the item attends to all 128 keys, so that the kernel applies no mask) and the original
 * positions of its 128 keys (-1 where a column holds no key, or a key the tile's mask leaves
 * to a gathered tile).  Flat int32 record:
 *   n_items, then per item: class, n_rows, rows[128], n_tiles, n_tiles x (src, keys[128]).
 * `*len` as for msa_read_indices. */
msa_status msa_read_tiles(const msa_plan* plan, const void* ws, int32_t head, int32_t* out, int64_t* len,
                          void* stream);

/* Synchronises `stream` and returns the first device-side error recorded in `ws` (MSA_OK if
 * none) and clears it.  The status word is reset by msa_estimate and msa_set_indices (the plan
 * tables they upload include it); a workspace no call has used yet has no defined status. */
msa_status msa_device_status(const msa_plan* plan, void* ws, void* stream);

/* Failure-detection self-test.  Every pipeline wait in the library's kernels is bounded by the
 * global timer; on expiry the kernel records MSA_ERR_TIMEOUT in the workspace's status word and
 * unwinds (no trap), leaving the context usable.  This call launches one kernel on `stream` whose
 * bounded wait (the same helper) waits for a barrier no thread arrives at, gives up after
 * `limit_us` microseconds (1 .. 1000000) and records the timeout the same way; the next
 * msa_device_status then returns MSA_ERR_TIMEOUT.  Asynchronous. */
msa_status msa_selftest_timeout(const msa_plan* plan, void* ws, uint32_t limit_us, void* stream);

const char* msa_status_string(msa_status status);

/* ---- attention analysis ----
 *
 * Share of the dense attention weights needed for a given recall (MMInference summary page,
 * attention analysis: in video-language models 95 % of the attention mass lies in 1.79 % of the
 * weights, against 5.78 % in language models).  For sample s, query row i = rows[s] of query
 * head h = heads[s]: the dense causal weights w_j = softmax_j(q_i . k_j * scale), j <= i, taken
 * in descending order; counts[s] = the fewest of them whose sum reaches recall * sum_j w_j
 * (the share is counts[s] / (i + 1)).  Q [Hq][L][128] and K [Hkv][L][128] bf16 on the device
 * with the q_* and k_* element strides of `strides` (multiples of 8; pointers 16-byte
 * aligned); query head h reads KV head h / (Hq / Hkv).  heads, rows: device int32 [n]; counts:
 * device int64 [n], -1 for a sample whose head or row is out of range.  recall in (0, 1].
 * Logits in fp32, weights and sums in fp64.  Asynchronous on `stream`; allocates nothing. */
msa_status msa_weight_share(const void* Q, const void* K, int64_t L, int32_t Hq, int32_t Hkv,
                            const msa_strides* strides, float scale, const int32_t* heads, const int32_t* rows,
                            int32_t n, double recall, int64_t* counts, void* stream);

/* ---- allocation-free variant ----
 *
 * Vertical-slash index estimation of ONE query head (the vertical and slash lines of its last
 * 64 queries, with the kernels, tile and key chunking msa_estimate uses for a one-head
 * vertical-slash plan, so the lines are the same) for callers
 * that cannot allocate device memory or provide a workspace: code running inside another
 * framework's memory manager, or serving loops where cudaMalloc and its implicit device
 * synchronisation are not allowed.  This call has no counterpart in the method's description;
 * it exists for those callers.
 *  - Inputs: Q and K of the head, bf16 [L][128] on the device with row strides q_row_stride /
 *    k_row_stride (elements, multiples of 8; pointers 16-byte aligned); softmax scale.
 *  - Outputs (device, caller-owned): v_out[k_v] vertical-line key positions and s_out[k_s]
 *    slash-line offsets, each ascending; counts_out[2] = number written to each.
 *  - Scratch: a fixed 1.2 MB array compiled into the library (every GPU that loads libmsa.so
 *    holds it until the process exits); L must be a multiple of 64 and at most 65536, larger L
 *    returns MSA_ERR_UNSUPPORTED; k_v, k_s in [1, L].
 *  - The first call on a device looks up the array's device address (a runtime call, no
 *    allocation); make that first call before any stream capture on that device.
 *  - Every call shares the one array and keeps its last contents: calls that may overlap on the
 *    GPU (different streams, or different threads) race and must be serialised by the caller.
 *  - Nothing is allocated or freed: no cudaMalloc, cudaFree or allocating library routine. */
msa_status msa_vslash_estimate_static(const void* Q, const void* K, int64_t L, int64_t q_row_stride,
                                      int64_t k_row_stride, float scale, int32_t k_v, int32_t k_s, int32_t* v_out,
                                      int32_t* s_out, int32_t* counts_out, void* stream);

/* Number of CUDA kernels this library has launched since it was loaded (all plans, all
 * threads); lets a caller count the kernels of one call by differencing. */
uint64_t msa_kernel_launches(void);

#ifdef __cplusplus
}
#endif
#endif /* MSA_H_ */
