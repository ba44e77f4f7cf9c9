// Host launchers of the libmsa kernels (one translation unit each).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "msa_internal.h"

namespace msa {

struct DevPlan {
  uint8_t* ws;
  Layout lay;
  int64_t L;
  int32_t Hq, Hkv, LP;
  int32_t n_classes, n_heads, n_rowsets, n_jobs, n_items, n_segs;
  int32_t n_units;     // attention work units (= n_items when the keys are not chunked)
  int32_t n_kchunks;   // key chunks of the attention kernel (1: not chunked)
  int32_t chunk_keys;  // keys per chunk (a multiple of 128)
  int32_t n_bands;     // unit bands (chunked keys only)
  int32_t x_rows;      // rows per gathered K/V slice
  int32_t n_qslices, n_xslices;
  int32_t has2d, has_block;
  int32_t n_block_heads;  // query heads of kind MSA_BLOCK
  int32_t nb;          // L / 64
  int64_t n_text;      // text tokens (they lead the modality-grouped order)
  int32_t tb_words;    // unit-bitmap words per tile-builder warp
  int32_t max_chunks;  // most key chunks of any row set
  int32_t n_lqtiles;   // tiles of the last-query sweep (pairs of row sets)
  int32_t lq_ring;     // slash ring entries per row set in the second sweep pass (power of two)
  float scale;
  const int32_t* class_kind;  // host copy: kind of each class
};

int sm_count();  // SMs of the current device

// One-time setup per device (function attributes such as the dynamic shared-memory limit are
// per device): pending until marked for device `dev`.
inline bool device_pending(const std::atomic<uint64_t>& flags, int dev) {
  return dev < 0 || dev >= 64 || !((flags.load(std::memory_order_acquire) >> dev) & 1u);
}
inline void mark_device(std::atomic<uint64_t>& flags, int dev) {
  if (dev >= 0 && dev < 64) flags.fetch_or(1ull << dev, std::memory_order_release);
}
// bumps the library-wide kernel launch counter by n
void count_launches(int n);

// layout of modalities / ranks / modality-grouped order from the segment table
cudaError_t launch_layout(const DevPlan& dp, cudaStream_t st);
// last-64-query sweeps (two passes) and top-k jobs
// Modality-grouped copy of K (text rows, then video rows) for the 2D-boundary heads.
cudaError_t launch_group_k(const DevPlan& dp, const void* K, const msa_strides& s, cudaStream_t st);
cudaError_t launch_lastq(const DevPlan& dp, const void* Q, const void* K, const msa_strides& s, cudaStream_t st);
// Slash-ring entries per row set the second sweep pass needs for row sets spanning max_span
// coordinates (a power of two), and the shared memory of each pass.
int lastq_ring_entries(int32_t max_span);
// Key chunk of the sweep for tiles reaching the given keys (one CTA per tile and chunk).
int32_t lastq_pick_chunk(const int32_t* tile_key_hi, int n_tiles);
size_t lastq_smem_bytes(int pass, int ring);
cudaError_t launch_topk_jobs(const DevPlan& dp, cudaStream_t st);
// block-sparse pooled estimation
cudaError_t launch_block_estimate(const DevPlan& dp, const void* Q, const void* K, const msa_strides& s,
                                  cudaStream_t st);
// grid stride / phase search
cudaError_t launch_grid_detect(const DevPlan& dp, cudaStream_t st);
// raw index sets -> row classes, gathered lists, bitmaps, then the tile lists
cudaError_t launch_materialize(const DevPlan& dp, cudaStream_t st);
cudaError_t launch_tiles(const DevPlan& dp, cudaStream_t st);
// gathers
// with_q: also the permuted Q copy (the index-based prefill gathers Q rows itself)
cudaError_t launch_permute(const DevPlan& dp, const void* Q, const void* K, const void* V, const msa_strides& s,
                           bool with_q, cudaStream_t st);
cudaError_t launch_unpermute(const DevPlan& dp, void* O, const msa_strides& s, cudaStream_t st);
// attention
// O null: the output goes to the permuted O copy in the workspace (msa_unpermute scatters it);
// otherwise the Q rows of permuted classes are gathered by index and every output row is
// written to O at its original position.
cudaError_t launch_attention(const DevPlan& dp, const void* Q, const void* K, const void* V, const msa_strides& s,
                             float* lse, void* O, cudaStream_t st);
// failure-detection self-test: one bounded wait that expires after limit_ns, recorded in *status
cudaError_t launch_wait_probe(uint32_t* status, uint64_t limit_ns, cudaStream_t st);
// allowed (query, key) pairs per head over the tile lists, into the workspace's mask_pairs
cudaError_t launch_mask_count(const DevPlan& dp, cudaStream_t st);

}  // namespace msa
