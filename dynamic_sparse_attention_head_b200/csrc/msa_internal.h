// Internal data model of libmsa: plan-time tables (built on the host, uploaded into the
// workspace) and the device-written dynamic state.  Shared by host and device code.
#pragma once
#include <stdint.h>

#include "../../include/msa.h"

namespace msa {

constexpr int D = 128;          // head dimension
constexpr int TILE = 128;       // query / key tile of the attention kernel
constexpr int UNIT = 64;        // key unit of the tile builder (window starts are unit aligned)
constexpr int LASTQ = 64;       // estimation rows per row set
constexpr int BLK = 64;         // block-sparse block
constexpr int GRID_BAND = 64;   // default local band of grid heads
constexpr int MAX_CLASSES_PER_HEAD = 2;
constexpr int32_t POS_PAD = 0x7fffffff;  // position of a padding key (never causal)
// Executed-tile id: source in bits 28-31, first key row in bits 0-26, and bit 27 set when every
// row of the work item attends to all 128 keys of the tile (no element mask needed).
constexpr uint32_t TILE_FULL = 1u << 27;
constexpr int HDR_NEXT_ITEM = 2;  // header word: next work item of the attention kernel
constexpr uint32_t TILE_ROW_MASK = TILE_FULL - 1u;

// key sources of a tile
enum : int32_t { SRC_K = 0, SRC_K2D = 1, SRC_X = 2 };

// class flags
enum : int32_t {
  CF_DENSE = 1,      // rows attend every causal key of the identity region
  CF_PERMUTED = 2,   // rows come from a row list (Q read from the permuted copy)
  CF_RANK = 4,       // coordinates are within-modality ranks (2D-boundary)
  CF_SLASH = 8,      // slash bitmap / list present
  CF_EXCL = 16,      // exclusion bitmap present (keys served by gathered tiles)
  CF_BLOCK = 32,     // block-sparse bitmap present
  CF_X = 64,         // gathered key list present
  CF_DYNROWS = 128,  // row count decided on the device (grid heads)
  CF_SINK = 256,     // sink prefix
  CF_BAND = 512,     // local band
  CF_SEGIDX = 1024   // the class's vertical / slash lists are its own (one class per segment)
};

// Device error bits recorded in the workspace header.
enum : uint32_t { DEV_ERR_TIMEOUT = 1u, DEV_ERR_BOUNDS = 2u };

struct ClassStatic {
  int32_t head, kvh, kind, flags;
  int32_t modality;        // QBOUND/BOUND2D: query modality; GRID: 0 = dense rows, 1 = other video rows
  int32_t sink, band;      // sink prefix length, local band width (coordinates)
  int32_t k_src;           // SRC_K or SRC_K2D for the identity region
  int32_t kc_lo, kc_hi;    // coordinate range of the identity region
  int32_t krow_lo;         // source row holding coordinate kc_lo
  int32_t max_rows;        // capacity of the row list / row count of static classes
  int32_t rows_static;     // row count when known at plan time, -1 if written on device
  int32_t x_cap;           // gathered-key capacity (multiple of 128)
  int32_t x_row0;          // first row of this class in the head's gathered K/V slice
  int32_t qrow0_static;    // first row in the head's permuted Q / O slice (static classes)
  int32_t item0, n_items;  // work items [item0, item0 + n_items)
  int32_t tile_cap;        // tile capacity per work item
  int32_t seg;             // CF_SEGIDX: the segment whose queries the class holds, else -1
  int64_t rows_off;        // int32 [max_rows] original positions of the rows (CF_PERMUTED)
  int64_t x_pos_off;       // int32 [x_cap] positions of gathered keys, POS_PAD padded
  int64_t slash_list_off;  // int32 slash offsets (sorted) - raw list
  int64_t slash_bits_off;  // uint32 bitmap over offsets [0, L)
  int64_t excl_bits_off;   // uint32 bitmap over identity coordinates [0, L)
  int64_t blk_bits_off;    // uint32 [nb][blk_wpr] block-sparse selection bits
  int64_t tile_base;       // first tile slot of item slot 0 (item slot s starts at tile_base + s * tile_cap)
  int32_t blk_wpr;         // words per block-bitmap row
  int32_t dyn;             // index into the ClassDyn array
  // CF_SEGIDX: the class's raw lists (positions, offsets) and their counts (int32 [2]: n_v, n_s)
  int64_t segv_off, segs_off, segcnt_off;
  int32_t segv_cap, segs_cap;
};

// Written on the device every prefill.
struct ClassDyn {
  int32_t nrows;     // rows of the class
  int32_t qrow0;     // first row in the permuted Q / O slice of the head
  int32_t x_len;     // gathered keys (before padding)
  int32_t n_slash;   // slash offsets
};

// Raw index slots of one head (the estimator's / msa_set_indices' output).
struct HeadStatic {
  int32_t kind, kvh;
  int32_t class0, n_classes;
  int32_t q_rows;            // rows of this head's permuted Q / O slice (0: not permuted)
  int32_t x_rows;            // rows of this head's gathered K/V slice
  int32_t grid_n_cand;
  int32_t grid_band;
  int32_t grid_cand[MSA_MAX_STRIDES];
  int32_t grid_np[MSA_MAX_STRIDES];  // phases kept for each candidate stride
  int32_t rawv_cap[2][2];
  int32_t raws_cap[2];
  int64_t rawv_off[2][2];    // int32 lists (positions)
  int64_t raws_off[2];       // int32 lists (offsets)
  int64_t counts_off;        // int32 [8]: n_v[0][0], n_v[0][1], n_v[1][0], n_v[1][1], n_s[0], n_s[1], stride, n_phases
  int64_t phases_off;        // int32 [max stride]
  int32_t blk_kmax, blk_nb;
  int32_t blk_fixed, _pad1;  // BLOCK: fixed top-k per row (> 0), else blk_budget
  double blk_budget;
  int64_t blk_list_off;      // int32 [nb][kmax]
  int64_t blk_cnt_off;       // int32 [nb]
  int64_t qbar_off;          // fp32 [nb][128] pooled queries (BLOCK heads)
  int64_t q_slice;           // head slot of the permuted Q / O tensors (-1 none)
  int64_t x_slice;           // head slot of the gathered K/V tensors (-1 none)
};

// One set of estimation rows: up to 64 queries of one head against one key source.
struct RowSet {
  int32_t head, kvh, k_src, n_rows;
  int32_t key_hi;            // scan source rows [0, key_hi)
  int32_t slash_lo, slash_hi;// source rows whose keys take part in the slash sums
  int32_t span;              // max(rcs) - min(rcs)
  int32_t rows[LASTQ];       // original positions of the rows
  int32_t rcs[LASTQ];        // slash coordinate of each row in source-row units
  int64_t v_off, s_off;      // fp32 [L] vertical sums (by source row), slash sums (by offset)
  int64_t mz_off;            // fp32 [n_chunks][LASTQ][2] partial (max, sum) of pass 1
  int64_t stat_off;          // fp32 [LASTQ][2] row max and 1/sum
  int32_t n_chunks, chunk;   // key chunks of the sweep
  int32_t cls;               // class whose own lists this row set's index fills (CF_SEGIDX), else -1
  int32_t _pad;
};

// One tile of the last-query sweep: up to two row sets of one KV head and key source, stacked
// as the 128 rows (row set 0: rows 0-63, row set 1: rows 64-127) of one tensor-core tile, so
// that their logits come from one MMA per key block and K is streamed once for both.
struct LqTile {
  int32_t rs[2];             // row set indices (rs[1] = -1: rows 64-127 are padding)
  int32_t kvh, k_src;
  int32_t key_hi;            // keys [0, key_hi) of the source (the larger of the two row sets')
  int32_t n_chunks;          // key chunks (the larger of the two row sets')
};

struct TopkJob {
  int64_t score_off;         // fp32 scores
  int32_t lo, hi;            // candidate index range [lo, hi)
  int32_t k;                 // kept
  int32_t map_k2d;           // 1: candidates are modality-grouped key rows, write positions
  int64_t out_off;           // int32 output list (sorted ascending)
  int64_t cnt_off;           // int32 count
};

struct WorkItem {
  int32_t cls, slot;         // class, 128-row slot within the class
};

// Units of work of the attention kernel when the keys are chunked: the tiles of one work item
// whose keys lie in one key chunk (gathered-key tiles count as chunk 0).  The work items are cut
// into bands (consecutive items of the plan order); a band's units run chunk-major, so that the
// units in flight read one chunk of K/V, and a long item carries its online-softmax state
// (unnormalised O, running max and sum) from chunk to chunk through an accumulator slot.
// Band b holds items [item0, item0 + n) and units [unit0, unit0 + n * n_kchunks): unit
// unit0 + c n + i is chunk c of item item0 + i, accumulator slot acc0 + i.
struct UnitBand {
  int32_t item0, n, acc0, unit0;
};
// fp32 per accumulator row: O[128], running max (log2), running sum, padding to a multiple of
// four so that every row starts on a 16-byte boundary (rows are moved with 16-byte accesses)
constexpr int ACC_ROW = D + 4;
static_assert(ACC_ROW % 4 == 0, "accumulator rows must be 16-byte aligned");

// Byte offsets of the workspace regions.
struct Layout {
  int64_t header;            // uint32 [64]: [0] error bits, [1] ready flags, [2] attention work-item counter, [8..] stats
  int64_t classes;           // ClassStatic [n_classes]
  int64_t heads;             // HeadStatic [Hq]
  int64_t rowsets;           // RowSet [n_rowsets]
  int64_t lq_tiles;          // LqTile [n_lqtiles]
  int64_t jobs;              // TopkJob [n_jobs]
  int64_t items;             // WorkItem [n_items]
  int64_t segs;              // int32 [n_segments][3] start, len, modality
  int64_t class_dyn;         // ClassDyn [n_classes]
  int64_t item_ntiles;       // int32 [n_items]
  int64_t bands;             // UnitBand [n_bands] (chunked keys only)
  int64_t cstart;            // int32 [n_items][n_kchunks + 1]: first tile of each key chunk (chunked keys only)
  int64_t chunk_done;        // uint32 [n_items]: chunks of the item whose state is in its accumulator,
                             // then uint32 [n_bands]: finished units of each band
  int64_t acc;               // fp32 [n_acc][128][ACC_ROW]: per-item online-softmax state between chunks
  int64_t tiles;             // uint32 [total tile capacity]: (src << 28) | TILE_FULL? | first key row
  int64_t mask_pairs;        // uint64 [Hq]: allowed (query, key) pairs per head (msa_mask_pairs)
  int64_t modality;          // uint8 [L]
  int64_t rank;              // int32 [L]
  int64_t perm2d;            // int32 [L] modality-grouped order (text then video) -> position
  int64_t mod_rows[2];       // int32 lists of text / video positions (views into perm2d)
  int64_t kbar;              // fp32 [Hkv][nb][128] pooled keys
  int64_t qp;                // bf16 [n_qslices][q_rows][128] permuted Q
  int64_t op;                // bf16 [n_qslices][q_rows][128] permuted O (+ identity heads)
  int64_t xk, xv;            // bf16 [n_xslices][x_rows][128] gathered K / V
  int64_t k2d, v2d;          // bf16 [Hkv][L][128] modality-grouped K / V
  int64_t indexed_total;     // bytes msa_sparse_prefill_indexed uses: every region before qp
  int64_t total;
};

}  // namespace msa
