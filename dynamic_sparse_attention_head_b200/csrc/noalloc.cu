// Allocation-free vertical-slash index estimation of one query head.
//
// Some callers cannot allocate device memory at the point where they need the estimate:
// plug-ins that run inside another framework's memory manager, or serving loops that must not
// call cudaMalloc (it may synchronise the device).  This entry point needs no workspace from
// them: its scratch is a file-scope __device__ array of fixed size, so every GPU that loads the
// library holds NOALLOC_BYTES of device memory until the process exits.  The caller passes only
// the inputs (Q and K of the head) and the outputs (the two index lists and their counts).
//
// It runs the same kernels as msa_estimate (two-pass last-64-query sweep, deterministic
// top-k) with the same key chunking, on a one-head plan whose workspace is the static array,
// so its lines are those msa_estimate finds for a one-head vertical-slash plan.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "kernels.h"
#include "msa_internal.h"

namespace msa {

namespace {

constexpr int64_t NOALLOC_MAX_L = 65536;
constexpr int64_t NOALLOC_MIN_CHUNK = 256;  // the sweep's smallest key chunk
// header + tables (2 KB) + v, s (4 B per key each) + chunk partials + row stats + the two lists
constexpr size_t NOALLOC_BYTES = 4096 + 2 * 4 * NOALLOC_MAX_L + (NOALLOC_MAX_L / NOALLOC_MIN_CHUNK) * LASTQ * 2 * 4 +
                                 LASTQ * 2 * 4 + 2 * 4 * NOALLOC_MAX_L + 512;

__device__ __align__(256) uint8_t g_noalloc_scratch[NOALLOC_BYTES];

// Device address of the scratch array on each device, looked up once per device.
std::mutex g_mu;
void* g_scratch_addr[64] = {nullptr};

cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

inline int64_t up256(int64_t x) { return (x + 255) / 256 * 256; }

struct Tables {
  RowSet rs;
  LqTile tile;
  TopkJob jv, js;
};

// Writes the one-head tables into the scratch (kernel parameters carry them: no host copies).
__global__ void noalloc_setup_kernel(uint8_t* ws, Layout lay, Tables t) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    *reinterpret_cast<RowSet*>(ws + lay.rowsets) = t.rs;
    *reinterpret_cast<LqTile*>(ws + lay.lq_tiles) = t.tile;
    reinterpret_cast<TopkJob*>(ws + lay.jobs)[0] = t.jv;
    reinterpret_cast<TopkJob*>(ws + lay.jobs)[1] = t.js;
    reinterpret_cast<uint32_t*>(ws + lay.header)[0] = 0u;
  }
}

// Copies the selected lists and their counts to the caller's buffers.
__global__ void noalloc_copy_kernel(const uint8_t* ws, int64_t v_off, int64_t s_off, int64_t cnt_off,
                                    int32_t cap_v, int32_t cap_s, int32_t* v_out, int32_t* s_out,
                                    int32_t* counts_out) {
  const int32_t* cnt = reinterpret_cast<const int32_t*>(ws + cnt_off);
  const int32_t nv = min(cnt[0], cap_v), ns = min(cnt[1], cap_s);
  const int32_t* v = reinterpret_cast<const int32_t*>(ws + v_off);
  const int32_t* s = reinterpret_cast<const int32_t*>(ws + s_off);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < max(nv, ns); i += gridDim.x * blockDim.x) {
    if (i < nv) v_out[i] = v[i];
    if (i < ns) s_out[i] = s[i];
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    counts_out[0] = nv;
    counts_out[1] = ns;
  }
}

}  // namespace

}  // namespace msa

using namespace msa;

extern "C" msa_status msa_vslash_estimate_static(const void* Q, const void* K, int64_t L, int64_t q_row_stride,
                                                 int64_t k_row_stride, float scale, int32_t k_v, int32_t k_s,
                                                 int32_t* v_out, int32_t* s_out, int32_t* counts_out,
                                                 void* stream) {
  if (!Q || !K || !v_out || !s_out || !counts_out) return MSA_ERR_INVALID_ARG;
  if (L < 64 || L % 64 != 0) return MSA_ERR_SHAPE;
  if (L > NOALLOC_MAX_L) return MSA_ERR_UNSUPPORTED;  // the static scratch holds L <= 65536
  if (k_v < 1 || k_s < 1 || k_v > L || k_s > L || !(scale > 0.f)) return MSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K)) % 16) return MSA_ERR_ALIGN;
  if (q_row_stride % 8 || k_row_stride % 8 || q_row_stride < D || k_row_stride < D) return MSA_ERR_ALIGN;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return MSA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // one-head layout inside the scratch; the sweep's key chunk by msa_estimate's rule
  const int32_t key_hi = (int32_t)L;
  const int32_t chunk = lastq_pick_chunk(&key_hi, 1);
  const int32_t n_chunks = (int32_t)((L + chunk - 1) / chunk);
  Layout lay{};
  int64_t off = 0;
  lay.header = off;
  off += 256;
  lay.rowsets = off;
  off = up256(off + (int64_t)sizeof(RowSet));
  lay.lq_tiles = off;
  off = up256(off + (int64_t)sizeof(LqTile));
  lay.jobs = off;
  off = up256(off + 2 * (int64_t)sizeof(TopkJob));
  const int64_t cnt_off = off;
  off += 256;
  const int64_t v_off = off;
  off = up256(off + 4 * L);
  const int64_t s_off = off;
  off = up256(off + 4 * L);
  const int64_t mz_off = off;
  off = up256(off + (int64_t)n_chunks * LASTQ * 2 * 4);
  const int64_t stat_off = off;
  off = up256(off + LASTQ * 2 * 4);
  const int64_t lv_off = off;
  off = up256(off + 4 * (int64_t)k_v);
  const int64_t ls_off = off;
  off = up256(off + 4 * (int64_t)k_s);
  if (off > (int64_t)NOALLOC_BYTES) return MSA_ERR_UNSUPPORTED;

  Tables t{};
  RowSet& r = t.rs;
  r.head = 0;
  r.kvh = 0;
  r.k_src = SRC_K;
  r.n_rows = LASTQ;
  for (int i = 0; i < LASTQ; ++i) r.rows[i] = r.rcs[i] = (int32_t)(L - LASTQ + i);
  r.span = LASTQ - 1;
  r.key_hi = (int32_t)L;
  r.slash_lo = 0;
  r.slash_hi = (int32_t)L;
  r.v_off = v_off;
  r.s_off = s_off;
  r.mz_off = mz_off;
  r.stat_off = stat_off;
  r.chunk = chunk;
  r.n_chunks = n_chunks;
  r.cls = -1;
  t.tile.rs[0] = 0;
  t.tile.rs[1] = -1;
  t.tile.kvh = 0;
  t.tile.k_src = SRC_K;
  t.tile.key_hi = (int32_t)L;
  t.tile.n_chunks = n_chunks;
  t.jv.score_off = v_off;
  t.jv.lo = 0;
  t.jv.hi = (int32_t)L;
  t.jv.k = k_v;
  t.jv.out_off = lv_off;
  t.jv.cnt_off = cnt_off;
  t.js.score_off = s_off;
  t.js.lo = 0;
  t.js.hi = (int32_t)L;
  t.js.k = k_s;
  t.js.out_off = ls_off;
  t.js.cnt_off = cnt_off + 4;

  DevPlan dp{};
  dp.ws = static_cast<uint8_t*>(scratch);
  dp.lay = lay;
  dp.L = L;
  dp.Hq = 1;
  dp.Hkv = 1;
  dp.n_rowsets = 1;
  dp.n_jobs = 2;
  dp.max_chunks = n_chunks;
  dp.n_lqtiles = 1;
  dp.lq_ring = lastq_ring_entries(LASTQ - 1);  // consecutive rows: span 63
  dp.scale = scale;
  dp.has2d = 0;
  msa_strides s{};
  s.q_head = 0;
  s.q_row = q_row_stride;
  s.k_head = 0;
  s.k_row = k_row_stride;

  count_launches(1);
  noalloc_setup_kernel<<<1, 32, 0, st>>>(dp.ws, lay, t);
  if (cudaGetLastError() != cudaSuccess) return MSA_ERR_CUDA;
  if (launch_lastq(dp, Q, K, s, st) != cudaSuccess) return MSA_ERR_CUDA;
  if (launch_topk_jobs(dp, st) != cudaSuccess) return MSA_ERR_CUDA;
  count_launches(1);
  noalloc_copy_kernel<<<std::max<int64_t>(1, std::min<int64_t>(64, (std::max(k_v, k_s) + 255) / 256)), 256, 0, st>>>(
      dp.ws, lv_off, ls_off, cnt_off, k_v, k_s, v_out, s_out, counts_out);
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}
