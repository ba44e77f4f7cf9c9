// Index-side kernels: token layout, grid stride/phase search, materialisation of the
// per-class row lists / gathered-key lists / line bitmaps, and the executed-tile builder.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "kernels.h"
#include "msa_internal.h"

namespace msa {

namespace {

template <typename T>
__host__ __device__ __forceinline__ T* at(const DevPlan& dp, int64_t off) {
  return reinterpret_cast<T*>(dp.ws + off);
}
__device__ __forceinline__ const ClassStatic& cls(const DevPlan& dp, int c) {
  return at<const ClassStatic>(dp, dp.lay.classes)[c];
}
__device__ __forceinline__ const HeadStatic& head(const DevPlan& dp, int h) {
  return at<const HeadStatic>(dp, dp.lay.heads)[h];
}
__device__ __forceinline__ ClassDyn& dyn(const DevPlan& dp, int c) { return at<ClassDyn>(dp, dp.lay.class_dyn)[c]; }

__device__ __forceinline__ void flag_bounds(const DevPlan& dp) {
  atomicOr(at<uint32_t>(dp, dp.lay.header), DEV_ERR_BOUNDS);
}

// ---------------------------------------------------------------------------------------
// token layout: modality, within-modality rank, modality-grouped order (text, then video)
// ---------------------------------------------------------------------------------------
__global__ void layout_kernel(DevPlan dp, int64_t n_text) {
  const int32_t* seg = at<const int32_t>(dp, dp.lay.segs);
  uint8_t* mod = at<uint8_t>(dp, dp.lay.modality);
  int32_t* rank = at<int32_t>(dp, dp.lay.rank);
  int32_t* perm = at<int32_t>(dp, dp.lay.perm2d);
  // segment s starts a run; rank base = tokens of the same modality in earlier segments
  for (int s = blockIdx.x; s < dp.n_segs; s += gridDim.x) {
    const int32_t st = seg[3 * s], len = seg[3 * s + 1], m = seg[3 * s + 2];
    __shared__ int32_t base_sh;
    if (threadIdx.x == 0) {
      int32_t b = 0;
      for (int q = 0; q < s; ++q)
        if (seg[3 * q + 2] == m) b += seg[3 * q + 1];
      base_sh = b;
    }
    __syncthreads();
    const int32_t base = base_sh;
    const int64_t region = (m == MSA_TEXT) ? 0 : n_text;
    for (int32_t i = threadIdx.x; i < len; i += blockDim.x) {
      const int32_t t = st + i;
      mod[t] = (uint8_t)m;
      rank[t] = base + i;
      perm[region + base + i] = t;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------------------
// per-class dynamic state of classes whose rows are known at plan time
// ---------------------------------------------------------------------------------------
__global__ void dyn_init_kernel(DevPlan dp) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= dp.n_classes) return;
  const ClassStatic& cs = cls(dp, c);
  ClassDyn& d = dyn(dp, cs.dyn);
  d.nrows = cs.rows_static < 0 ? 0 : cs.rows_static;
  d.qrow0 = cs.qrow0_static;
  d.x_len = 0;
  d.n_slash = 0;
}

// ---------------------------------------------------------------------------------------
// vertical-slash style classes (VSLASH, QBOUND, BOUND2D): gathered list, slash and
// exclusion bitmaps.  One CTA per class.
// ---------------------------------------------------------------------------------------
__global__ void mat_lists_kernel(DevPlan dp) {
  const int c = blockIdx.x;
  const ClassStatic& cs = cls(dp, c);
  if (!(cs.kind == MSA_VSLASH || cs.kind == MSA_QBOUND || cs.kind == MSA_BOUND2D)) return;
  const HeadStatic& hs = head(dp, cs.head);
  const int32_t* counts = at<const int32_t>(dp, hs.counts_off);
  const int a = (cs.kind == MSA_VSLASH) ? 0 : cs.modality;
  const int nwords = (int)((dp.L + 31) >> 5);
  uint32_t* sbits = at<uint32_t>(dp, cs.slash_bits_off);
  uint32_t* ebits = at<uint32_t>(dp, cs.excl_bits_off);
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) {
    sbits[w] = 0u;
    ebits[w] = 0u;
  }
  __syncthreads();
  // a class with its own lists (one class per segment) or the head's lists of modality a
  const bool own = (cs.flags & CF_SEGIDX) != 0;
  const int32_t* ccnt = own ? at<const int32_t>(dp, cs.segcnt_off) : nullptr;
  // slash lines
  const int32_t ns = own ? ccnt[1] : (hs.raws_cap[a] > 0 ? counts[4 + a] : 0);
  const int32_t* sl = at<const int32_t>(dp, own ? cs.segs_off : hs.raws_off[a]);
  for (int i = threadIdx.x; i < ns; i += blockDim.x) {
    const int32_t o = sl[i];
    if (o < 0 || o >= dp.L) { flag_bounds(dp); continue; }
    atomicOr(&sbits[o >> 5], 1u << (o & 31));
  }
  // gathered keys: VSLASH [0][0]; QBOUND [a][0]; BOUND2D merge of [a][0] and [a][1]
  int32_t* xp = at<int32_t>(dp, cs.x_pos_off);
  const int32_t* ra = at<const int32_t>(dp, own ? cs.segv_off : hs.rawv_off[a][0]);
  const int32_t na = own ? ccnt[0] : (hs.rawv_cap[a][0] > 0 ? counts[a * 2] : 0);
  const int32_t* rb = at<const int32_t>(dp, hs.rawv_off[a][1]);
  const int32_t nb_ = (cs.kind == MSA_BOUND2D && hs.rawv_cap[a][1] > 0) ? counts[a * 2 + 1] : 0;
  const int32_t nx = na + nb_;
  if (nx > cs.x_cap) {
    if (threadIdx.x == 0) flag_bounds(dp);
    return;
  }
  const int32_t* rank = at<const int32_t>(dp, dp.lay.rank);
  for (int i = threadIdx.x; i < na; i += blockDim.x) {
    const int32_t v = ra[i];
    int lo = 0, hi = nb_;  // elements of b strictly below v
    while (lo < hi) {
      int m = (lo + hi) >> 1;
      if (rb[m] < v) lo = m + 1;
      else hi = m;
    }
    xp[i + lo] = v;
    if (cs.kind != MSA_BOUND2D || a == 0) {
      const int32_t e = (cs.kind == MSA_BOUND2D) ? rank[v] : v;  // own-modality keys leave the identity region
      atomicOr(&ebits[e >> 5], 1u << (e & 31));
    }
  }
  for (int i = threadIdx.x; i < nb_; i += blockDim.x) {
    const int32_t v = rb[i];
    int lo = 0, hi = na;  // elements of a not above v
    while (lo < hi) {
      int m = (lo + hi) >> 1;
      if (ra[m] <= v) lo = m + 1;
      else hi = m;
    }
    xp[i + lo] = v;
    if (a == 1) {
      const int32_t e = rank[v];
      atomicOr(&ebits[e >> 5], 1u << (e & 31));
    }
  }
  for (int i = nx + threadIdx.x; i < cs.x_cap; i += blockDim.x) xp[i] = POS_PAD;
  if (threadIdx.x == 0) {
    ClassDyn& d = dyn(dp, cs.dyn);
    d.x_len = nx;
    d.n_slash = ns;
  }
}

// ---------------------------------------------------------------------------------------
// Grid stride / phase search (MMInference Algorithm 1, "key machinery"): the column sums v
// of the last 64 video queries are averaged over the video keys of each (stride, phase);
// the stride with the highest best-phase mean wins (ties: the smaller stride), then its
// n_p best phases are kept (ties: the smaller phase).  One CTA per grid head.
// ---------------------------------------------------------------------------------------
__global__ void grid_detect_kernel(DevPlan dp) {
  const int h = blockIdx.x;
  const HeadStatic& hs = head(dp, h);
  if (hs.kind != MSA_GRID) return;
  __shared__ float sc_best[4096];
  __shared__ float sc_cur[4096];
  __shared__ float red_v[32];
  __shared__ int red_i[32];
  __shared__ int best_s_sh;
  __shared__ float best_val_sh;
  const RowSet* rs = nullptr;
  for (int r = 0; r < dp.n_rowsets; ++r) {
    const RowSet& x = at<const RowSet>(dp, dp.lay.rowsets)[r];
    if (x.head == h) rs = &x;
  }
  const bool have_v = rs && rs->n_rows > 0;
  const float* v = have_v ? at<const float>(dp, rs->v_off) : nullptr;
  const int32_t* seg = at<const int32_t>(dp, dp.lay.segs);
  if (threadIdx.x == 0) {
    best_s_sh = -1;
    best_val_sh = 0.f;
  }
  __syncthreads();
  for (int ci = 0; ci < hs.grid_n_cand; ++ci) {
    const int s = hs.grid_cand[ci];
    float my_best = -INFINITY;
    for (int p = threadIdx.x; p < s; p += blockDim.x) {
      float sum = 0.f;
      int cnt = 0;
      for (int g = 0; g < dp.n_segs; ++g) {
        if (seg[3 * g + 2] != MSA_VIDEO) continue;
        const int st = seg[3 * g], len = seg[3 * g + 1];
        if (p >= len) continue;
        cnt += (len - p + s - 1) / s;
        if (!have_v) continue;
        // four independent partial sums (loads in flight), combined in a fixed order
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        int t = p;
        for (; t + 3 * s < len; t += 4 * s) {
          a0 += v[st + t];
          a1 += v[st + t + s];
          a2 += v[st + t + 2 * s];
          a3 += v[st + t + 3 * s];
        }
        for (; t < len; t += s) a0 += v[st + t];
        sum += (a0 + a1) + (a2 + a3);
      }
      const float mean = cnt > 0 ? sum / (float)cnt : 0.f;
      sc_cur[p] = mean;
      my_best = fmaxf(my_best, mean);
    }
    // block max of the best-phase means
    for (int o = 16; o; o >>= 1) {
      float ov = __shfl_xor_sync(0xFFFFFFFFu, my_best, o);
      my_best = fmaxf(my_best, ov);
    }
    if ((threadIdx.x & 31) == 0) red_v[threadIdx.x >> 5] = my_best;
    __syncthreads();
    if (threadIdx.x == 0) {
      float m = -INFINITY;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red_v[w]);
      if (best_s_sh < 0 || m > best_val_sh) {
        best_s_sh = ci;
        best_val_sh = m;
      }
    }
    __syncthreads();
    if (best_s_sh == ci)
      for (int p = threadIdx.x; p < s; p += blockDim.x) sc_best[p] = sc_cur[p];
    __syncthreads();
  }
  const int ci = best_s_sh;
  const int s = hs.grid_cand[ci];
  const int np = hs.grid_np[ci];
  int32_t* phases = at<int32_t>(dp, hs.phases_off);
  // n_p rounds of (max score, smallest phase) selection
  for (int k = 0; k < np; ++k) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int p = threadIdx.x; p < s; p += blockDim.x) {
      const float x = sc_best[p];
      if (x > bv || (x == bv && p < bi)) {
        bv = x;
        bi = p;
      }
    }
    for (int o = 16; o; o >>= 1) {
      float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
      int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if ((threadIdx.x & 31) == 0) {
      red_v[threadIdx.x >> 5] = bv;
      red_i[threadIdx.x >> 5] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float b = -INFINITY;
      int i = 0x7fffffff;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w)
        if (red_v[w] > b || (red_v[w] == b && red_i[w] < i)) {
          b = red_v[w];
          i = red_i[w];
        }
      phases[k] = i;
      sc_best[i] = -INFINITY;  // taken
      // a phase scoring -inf can only be a taken one; keep the order of the rest
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    // sort the phases ascending (n_p is small)
    for (int i = 1; i < np; ++i) {
      int x = phases[i], j = i - 1;
      while (j >= 0 && phases[j] > x) {
        phases[j + 1] = phases[j];
        --j;
      }
      phases[j + 1] = x;
    }
    int32_t* counts = at<int32_t>(dp, hs.counts_off);
    counts[6] = s;
    counts[7] = np;
  }
}

// ---------------------------------------------------------------------------------------
// grid classes: row lists of both classes, gathered grid keys, exclusion bitmap.
// ---------------------------------------------------------------------------------------

// Grid heads, materialised in two launches over GM_BLOCKS blocks per head (each block a run of
// whole 32-position words): positions whose in-segment offset mod the stride is one of the
// selected phases (video only) are the gathered keys of the head's video class and excluded from
// its identity tiles; query rows split into class 0 (text rows and those grid positions) and
// class 1 (the other video rows), all lists in ascending position order.
constexpr int GM_BLOCKS = 32;
constexpr int GM_THREADS = 256;

struct GridCtx {
  int s, np;
  int64_t b0, b1;  // this block's positions
};

// The block's positions and the phase bitmap of the head (shared memory); false: not a grid head.
__device__ __forceinline__ bool grid_block(const DevPlan& dp, const HeadStatic& hs, uint32_t* pset, GridCtx& g) {
  if (hs.kind != MSA_GRID) return false;
  const int32_t* counts = at<const int32_t>(dp, hs.counts_off);
  g.s = counts[6];
  g.np = counts[7];
  const int32_t* phases = at<const int32_t>(dp, hs.phases_off);
  for (int i = threadIdx.x; i < 128; i += blockDim.x) pset[i] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < g.np; i += blockDim.x) {
    const int ph = phases[i];
    if (ph >= 0 && ph < 4096) atomicOr(&pset[ph >> 5], 1u << (ph & 31));
  }
  __syncthreads();
  const int64_t words = (dp.L + 31) >> 5;
  const int64_t per = (words + GM_BLOCKS - 1) / GM_BLOCKS;
  g.b0 = min((int64_t)blockIdx.x * per, words) << 5;
  g.b1 = min(((int64_t)blockIdx.x + 1) * per, words) << 5;
  return true;
}

// One 32-position word of a block (lane = position t = w0 + lane): the grid mark and the class.
// Returns ballots: marks, class-0 rows, class-1 rows.
__device__ __forceinline__ void grid_word(const DevPlan& dp, const uint32_t* pset, int s, int64_t w0, uint32_t& gb,
                                          uint32_t& c0b, uint32_t& c1b) {
  const int lane = threadIdx.x & 31;
  const int64_t t = w0 + lane;
  const bool valid = t < dp.L;
  bool g = false, text = false;
  if (valid) {
    const uint8_t m = at<const uint8_t>(dp, dp.lay.modality)[t];
    text = m == MSA_TEXT;
    if (m == MSA_VIDEO) {
      // segment of t: the last whose start is <= t
      const int32_t* seg = at<const int32_t>(dp, dp.lay.segs);
      int lo = 0, hi = dp.n_segs - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (seg[3 * mid] <= t) lo = mid;
        else hi = mid - 1;
      }
      const int ph = (int)((t - seg[3 * lo]) % s);
      g = (pset[ph >> 5] >> (ph & 31)) & 1u;
    }
  }
  gb = __ballot_sync(0xFFFFFFFFu, g);
  c0b = __ballot_sync(0xFFFFFFFFu, valid && (g || text));
  c1b = __ballot_sync(0xFFFFFFFFu, valid && !(g || text));
}

// Pass 1: per block, the number of grid marks, class-0 rows and class-1 rows.
__global__ void __launch_bounds__(GM_THREADS) grid_count_kernel(DevPlan dp) {
  const HeadStatic& hs = head(dp, blockIdx.y);
  __shared__ uint32_t pset[128];  // phase bitmap, strides <= 4096
  __shared__ int sums[GM_THREADS / 32][3];
  GridCtx g;
  if (!grid_block(dp, hs, pset, g)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  int n[3] = {0, 0, 0};
  for (int64_t w0 = g.b0 + 32 * warp; w0 < g.b1; w0 += 32 * nw) {
    uint32_t gb, c0b, c1b;
    grid_word(dp, pset, g.s, w0, gb, c0b, c1b);
    n[0] += __popc(gb);
    n[1] += __popc(c0b);
    n[2] += __popc(c1b);
  }
  if (lane == 0)
    for (int i = 0; i < 3; ++i) sums[warp][i] = n[i];
  __syncthreads();
  if (threadIdx.x < 3) {
    int v = 0;
    for (int w = 0; w < nw; ++w) v += sums[w][threadIdx.x];
    at<int32_t>(dp, hs.counts_off)[16 + 3 * blockIdx.x + threadIdx.x] = v;
  }
}

// Pass 2: each block writes its marks, rows and exclusion words at the offsets of the blocks
// before it; warps take consecutive runs of words, so every list stays in position order.
__global__ void __launch_bounds__(GM_THREADS) grid_write_kernel(DevPlan dp) {
  const int h = blockIdx.y;
  const HeadStatic& hs = head(dp, h);
  __shared__ uint32_t pset[128];
  __shared__ int wsum[GM_THREADS / 32][3];
  __shared__ int base[3], tot[3];
  GridCtx g;
  if (!grid_block(dp, hs, pset, g)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int32_t* bc = at<const int32_t>(dp, hs.counts_off) + 16;
  if (threadIdx.x < 3) {
    int before = 0, all = 0;
    for (int b = 0; b < GM_BLOCKS; ++b) {
      const int v = bc[3 * b + threadIdx.x];
      if (b < (int)blockIdx.x) before += v;
      all += v;
    }
    base[threadIdx.x] = before;
    tot[threadIdx.x] = all;
  }
  // this warp's run of words
  const int64_t nwords = (g.b1 - g.b0) >> 5;
  const int64_t wper = (nwords + nw - 1) / nw;
  const int64_t wa = g.b0 + 32 * min((int64_t)warp * wper, nwords), wb = g.b0 + 32 * min((int64_t)(warp + 1) * wper, nwords);
  int n[3] = {0, 0, 0};
  for (int64_t w0 = wa; w0 < wb; w0 += 32) {
    uint32_t gb, c0b, c1b;
    grid_word(dp, pset, g.s, w0, gb, c0b, c1b);
    n[0] += __popc(gb);
    n[1] += __popc(c0b);
    n[2] += __popc(c1b);
  }
  if (lane == 0)
    for (int i = 0; i < 3; ++i) wsum[warp][i] = n[i];
  __syncthreads();
  const ClassStatic& c0 = cls(dp, hs.class0);
  const ClassStatic& c1 = cls(dp, hs.class0 + 1);
  if (tot[0] > c1.x_cap) {
    if (threadIdx.x == 0) flag_bounds(dp);
    return;
  }
  int off[3];
  for (int i = 0; i < 3; ++i) {
    off[i] = base[i];
    for (int w = 0; w < warp; ++w) off[i] += wsum[w][i];
  }
  int32_t* rows0 = at<int32_t>(dp, c0.rows_off);
  int32_t* rows1 = at<int32_t>(dp, c1.rows_off);
  int32_t* xg = at<int32_t>(dp, c1.x_pos_off);
  uint32_t* ex = at<uint32_t>(dp, c1.excl_bits_off);
  const uint32_t lt = (1u << lane) - 1u;
  for (int64_t w0 = wa; w0 < wb; w0 += 32) {
    uint32_t gb, c0b, c1b;
    grid_word(dp, pset, g.s, w0, gb, c0b, c1b);
    const int64_t t = w0 + lane;
    if ((gb >> lane) & 1u) xg[off[0] + __popc(gb & lt)] = (int32_t)t;
    if ((c0b >> lane) & 1u) rows0[off[1] + __popc(c0b & lt)] = (int32_t)t;
    if ((c1b >> lane) & 1u) rows1[off[2] + __popc(c1b & lt)] = (int32_t)t;
    if (lane == 0) ex[w0 >> 5] = gb;
    off[0] += __popc(gb);
    off[1] += __popc(c0b);
    off[2] += __popc(c1b);
  }
  if (blockIdx.x == GM_BLOCKS - 1) {
    for (int i = tot[0] + threadIdx.x; i < c1.x_cap; i += blockDim.x) xg[i] = POS_PAD;
    if (threadIdx.x == 0) {
      ClassDyn& d0 = dyn(dp, c0.dyn);
      d0.nrows = tot[1];
      d0.qrow0 = 0;
      d0.x_len = 0;
      d0.n_slash = 0;
      ClassDyn& d1 = dyn(dp, c1.dyn);
      d1.nrows = tot[2];
      d1.qrow0 = (tot[1] + TILE - 1) / TILE * TILE;
      d1.x_len = tot[0];
      d1.n_slash = 0;
    }
  }
}

// ---------------------------------------------------------------------------------------
// block-sparse selection bitmaps: one warp per query block row
// ---------------------------------------------------------------------------------------
__global__ void block_bits_kernel(DevPlan dp, int c) {
  const ClassStatic& cs = cls(dp, c);
  const HeadStatic& hs = head(dp, cs.head);
  const int nb = hs.blk_nb;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  uint32_t* bits = at<uint32_t>(dp, cs.blk_bits_off);
  const int32_t* lists = at<const int32_t>(dp, hs.blk_list_off);
  const int32_t* cnt = at<const int32_t>(dp, hs.blk_cnt_off);
  for (int b = warp; b < nb; b += nwarps) {
    uint32_t* row = bits + (size_t)b * cs.blk_wpr;
    for (int w = lane; w < cs.blk_wpr; w += 32) row[w] = 0u;
    __syncwarp();
    const int n = cnt[b];
    for (int i = lane; i < n; i += 32) {
      const int kb = lists[(size_t)b * hs.blk_kmax + i];
      if (kb < 0 || kb > b) {
        flag_bounds(dp);
        continue;
      }
      atomicOr(&row[kb >> 5], 1u << (kb & 31));
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------------------
// Tile builder: one warp per 128-query work item.  Gathered-key tiles first (the keys of
// the class's gathered list at positions <= the last query), then the identity region:
// every condition of the class marks the 64-key units it needs (causal bound included),
// and the marked units are covered greedily by disjoint 128-key windows starting on a
// marked unit.  Windows may cover unneeded keys; the attention kernel's element mask
// removes them, and disjointness guarantees no key is counted twice for a row.
// ---------------------------------------------------------------------------------------
constexpr int TB_WARPS = 8;

__device__ __forceinline__ void mark_units(uint32_t* bm, int64_t a, int64_t b, int32_t kc_lo, int64_t hi_clip) {
  if (a < kc_lo) a = kc_lo;
  if (b > hi_clip) b = hi_clip;
  if (a > b) return;
  const int64_t ua = (a - kc_lo) >> 6, ub = (b - kc_lo) >> 6;
  for (int64_t u = ua; u <= ub;) {
    const int64_t w = u >> 5;
    const int lo = (int)(u & 31);
    const int hi = (int)(ub - (w << 5) < 31 ? ub - (w << 5) : 31);
    const uint32_t m = (hi - lo == 31) ? 0xFFFFFFFFu : (((1u << (hi - lo + 1)) - 1u) << lo);
    atomicOr(&bm[w], m);
    u = (w + 1) << 5;
  }
}

// Window starts of one bitmap word for the greedy cover (see tiles_kernel): the marked units at
// an even distance from the start of their run; cin: the first unit is covered by the window
// before the word.  Runs that start at even positions are found by adding their start bits (the
// carry clears exactly the run).
__device__ __forceinline__ uint32_t window_starts(uint32_t x, uint32_t cin) {
  if (cin) x &= ~1u;
  const uint32_t even = 0x55555555u;
  const uint32_t rs = x & ~(x << 1);              // run starts
  const uint32_t re = x & ~(x + (rs & even));     // units of runs that start at even positions
  return (re & even) | (x & ~re & ~even);
}

__global__ void __launch_bounds__(TB_WARPS * 32) tiles_kernel(DevPlan dp, int bm_words) {
  extern __shared__ uint32_t tb_smem[];
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* bm = tb_smem + (size_t)wl * (bm_words + 2 * TILE);
  int32_t* run_lo = reinterpret_cast<int32_t*>(bm + bm_words);
  int32_t* run_hi = run_lo + TILE;
  const int wpb = blockDim.x >> 5;
  const int gw = blockIdx.x * wpb + wl, nw = gridDim.x * wpb;
  const WorkItem* items = at<const WorkItem>(dp, dp.lay.items);
  int32_t* ntiles = at<int32_t>(dp, dp.lay.item_ntiles);
  uint32_t* tiles = at<uint32_t>(dp, dp.lay.tiles);
  for (int item = gw; item < dp.n_items; item += nw) {
    const WorkItem wi = items[item];
    const ClassStatic& cs = cls(dp, wi.cls);
    const ClassDyn cd = dyn(dp, cs.dyn);
    const int nrows = cd.nrows;
    const int row0 = wi.slot * TILE;
    if (row0 >= nrows) {
      if (lane == 0) ntiles[item] = 0;
      if (dp.n_kchunks > 1)
        for (int c = lane; c <= dp.n_kchunks; c += 32) at<int32_t>(dp, dp.lay.cstart)[(int64_t)item * (dp.n_kchunks + 1) + c] = 0;
      continue;
    }
    const int nval = min(TILE, nrows - row0);
    const int32_t* rl = at<const int32_t>(dp, cs.rows_off);
    const bool perm = (cs.flags & CF_PERMUTED) != 0;
    const bool rank = (cs.flags & CF_RANK) != 0;
    auto pos_of = [&](int r) -> int32_t { return perm ? rl[r] : r; };
    auto coord_of = [&](int r) -> int32_t { return rank ? r : pos_of(r); };
    const int32_t qpos_max = pos_of(row0 + nval - 1);
    const int32_t qc_min = coord_of(row0), qc_max = coord_of(row0 + nval - 1);
    uint32_t* out = tiles + cs.tile_base + (int64_t)wi.slot * cs.tile_cap;
    int nt = 0;
    // ---- gathered keys
    if (cs.flags & CF_X) {
      const int32_t* xp = at<const int32_t>(dp, cs.x_pos_off);
      int lo = 0, hi = cd.x_len;
      while (lo < hi) {
        int m = (lo + hi) >> 1;
        if (xp[m] <= qpos_max) lo = m + 1;
        else hi = m;
      }
      const int ntx = (lo + TILE - 1) / TILE;
      for (int i = lane; i < ntx; i += 32) out[i] = ((uint32_t)SRC_X << 28) | (uint32_t)(cs.x_row0 + i * TILE);
      nt = ntx;
    }
    // ---- identity region
    const int64_t hi_clip = ((int64_t)qc_max < (int64_t)cs.kc_hi - 1) ? (int64_t)qc_max : (int64_t)cs.kc_hi - 1;
    const int64_t umax = hi_clip >= cs.kc_lo ? ((hi_clip - cs.kc_lo) >> 6) : -1;
    const int wmax = (int)((umax + 32) >> 5);  // words in use
    if (wmax > bm_words) {
      if (lane == 0) {
        flag_bounds(dp);
        ntiles[item] = 0;
      }
      if (dp.n_kchunks > 1)
        for (int c = lane; c <= dp.n_kchunks; c += 32) at<int32_t>(dp, dp.lay.cstart)[(int64_t)item * (dp.n_kchunks + 1) + c] = 0;
      continue;
    }
    for (int w = lane; w < wmax; w += 32) bm[w] = 0u;
    // runs of consecutive coordinates among the tile's rows
    int nruns = 0;
    {
      int ne = 0;
      for (int base = 0; base < nval; base += 32) {
        const int r = base + lane;
        bool start = false, end = false;
        int32_t c = 0;
        if (r < nval) {
          c = coord_of(row0 + r);
          start = (r == 0) || (coord_of(row0 + r - 1) != c - 1);
          end = (r == nval - 1) || (coord_of(row0 + r + 1) != c + 1);
        }
        const uint32_t bs = __ballot_sync(0xFFFFFFFFu, start), be = __ballot_sync(0xFFFFFFFFu, end);
        const uint32_t lt = (1u << lane) - 1u;
        if (start) run_lo[nruns + __popc(bs & lt)] = c;
        if (end) run_hi[ne + __popc(be & lt)] = c;
        nruns += __popc(bs);
        ne += __popc(be);
      }
      __syncwarp();
    }
    const int32_t kc_lo = cs.kc_lo;
    if (umax >= 0) {
      if (cs.flags & CF_DENSE) {
        if (lane == 0) mark_units(bm, kc_lo, hi_clip, kc_lo, hi_clip);
      } else {
        if ((cs.flags & CF_SINK) && lane == 0) mark_units(bm, kc_lo, (int64_t)cs.sink - 1, kc_lo, hi_clip);
        if (cs.flags & CF_BAND)
          for (int i = lane; i < nruns; i += 32)
            mark_units(bm, (int64_t)run_lo[i] - cs.band + 1, run_hi[i], kc_lo, hi_clip);
        if (cs.flags & CF_SLASH) {
          // each lane takes a run of the (ascending) offsets; for one run of rows their key ranges
          // descend, and two ranges less than a unit apart mark the same units as their hull (no
          // unit fits in the gap), so the lane merges them and marks each merged range once
          const int32_t* sl = at<const int32_t>(dp, cs.slash_list_off);
          const int per = (cd.n_slash + 31) >> 5;
          const int i0 = min(lane * per, cd.n_slash), i1 = min(i0 + per, cd.n_slash);
          for (int r = 0; r < nruns; ++r) {
            int64_t lo = 1, hi = 0;  // merged key range (empty)
            for (int i = i0; i < i1; ++i) {
              const int64_t o = sl[i];
              int64_t a = run_lo[r] - o, b = run_hi[r] - o;  // clipped first: the gap rule holds inside
              if (a < kc_lo) a = kc_lo;
              if (b > hi_clip) b = hi_clip;
              if (a > b) continue;
              if (lo <= hi && b >= lo - UNIT && a <= hi + UNIT) {
                lo = a < lo ? a : lo;
                hi = b > hi ? b : hi;
              } else {
                if (lo <= hi) mark_units(bm, lo, hi, kc_lo, hi_clip);
                lo = a;
                hi = b;
              }
            }
            if (lo <= hi) mark_units(bm, lo, hi, kc_lo, hi_clip);
          }
        }
        if (cs.flags & CF_BLOCK) {
          const HeadStatic& hs = head(dp, cs.head);
          const int32_t* lists = at<const int32_t>(dp, hs.blk_list_off);
          const int32_t* cnt = at<const int32_t>(dp, hs.blk_cnt_off);
          for (int qb = qc_min >> 6; qb <= (qc_max >> 6); ++qb) {
            const int n = cnt[qb];
            for (int i = lane; i < n; i += 32) {
              const int64_t kb = lists[(size_t)qb * hs.blk_kmax + i];
              mark_units(bm, kb * BLK, kb * BLK + BLK - 1, kc_lo, hi_clip);
            }
          }
        }
      }
    }
    __syncwarp();
    // ---- greedy cover of the marked units by disjoint 2-unit windows, scanning units upwards: a
    // window starts at every marked unit not covered by the window before it, which is every
    // marked unit at an even distance from the start of its run of marked units.  Each lane
    // takes a run of words; the one bit of state between words (the last window covers the next
    // word's first unit) goes across the lanes by a scan of the words' carry maps.
    {
      const int per = (wmax + 31) >> 5;
      const int w0 = min(lane * per, wmax), w1 = min(w0 + per, wmax);
      uint32_t f0 = 0u, f1 = 1u;  // carry out of this lane's words for carry in 0 / 1
      for (int w = w0; w < w1; ++w) {
        const uint32_t x = bm[w];
        f0 = window_starts(x, f0) >> 31;
        f1 = window_starts(x, f1) >> 31;
      }
      // inclusive scan of the maps (composition: earlier lanes' map first)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t g0 = __shfl_up_sync(0xFFFFFFFFu, f0, o), g1 = __shfl_up_sync(0xFFFFFFFFu, f1, o);
        if (lane >= o) {
          const uint32_t h0 = g0 ? f1 : f0, h1 = g1 ? f1 : f0;
          f0 = h0;
          f1 = h1;
        }
      }
      uint32_t cin = __shfl_up_sync(0xFFFFFFFFu, f0, 1);  // the chain starts with carry 0
      if (lane == 0) cin = 0u;
      // windows of this lane's words, then their places in the list
      int cnt = 0;
      uint32_t c = cin;
      for (int w = w0; w < w1; ++w) {
        const uint32_t st = window_starts(bm[w], c);
        c = st >> 31;
        cnt += __popc(st);
      }
      int base = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, base, o);
        if (lane >= o) base += v;
      }
      const int total = __shfl_sync(0xFFFFFFFFu, base, 31);
      base = nt + base - cnt;
      c = cin;
      for (int w = w0; w < w1; ++w) {
        uint32_t st = window_starts(bm[w], c);
        c = st >> 31;
        while (st) {
          const int b = __ffs(st) - 1;
          st &= st - 1u;
          const int64_t u = ((int64_t)w << 5) + b;
          if (base < cs.tile_cap) out[base] = ((uint32_t)cs.k_src << 28) | (uint32_t)(cs.krow_lo + u * UNIT);
          ++base;
        }
      }
      nt += total;
      if (lane == 0) {
        if (nt > cs.tile_cap) flag_bounds(dp);
        ntiles[item] = min(nt, cs.tile_cap);
      }
      nt = min(nt, cs.tile_cap);
    }
    __syncwarp();
    // ---- tiles that every row of the item attends to in full (sufficient conditions only)
    const int32_t qpos_min = pos_of(row0);
    for (int i = lane; i < nt; i += 32) {
      const uint32_t t = out[i];
      const int src = (int)(t >> 28);
      const int32_t krow = (int32_t)(t & TILE_ROW_MASK);
      bool full;
      if (src == SRC_X) {  // gathered keys ascend by position; padding is never causal
        full = at<const int32_t>(dp, cs.x_pos_off)[krow - cs.x_row0 + TILE - 1] <= qpos_min;
      } else {
        const int64_t kc0 = (int64_t)cs.kc_lo + (krow - cs.krow_lo), kc1 = kc0 + TILE - 1;
        full = kc1 <= qc_min && kc1 < cs.kc_hi;  // causal for the first row, inside the region
        if (full && !(cs.flags & CF_DENSE)) {
          bool cover = ((cs.flags & CF_SINK) && kc1 < cs.sink) ||
                       ((cs.flags & CF_BAND) && kc0 >= (int64_t)qc_max - cs.band + 1);
          if (!cover && (cs.flags & CF_BLOCK)) {
            const uint32_t* bits = at<const uint32_t>(dp, cs.blk_bits_off);
            cover = true;
            for (int qb = qc_min >> 6; qb <= (qc_max >> 6) && cover; ++qb)
              for (int64_t kb = kc0 >> 6; kb <= (kc1 >> 6) && cover; ++kb)
                cover = (bits[(size_t)qb * cs.blk_wpr + (kb >> 5)] >> (kb & 31)) & 1u;
          }
          full = cover;
        }
        if (full && (cs.flags & CF_EXCL)) {
          const uint32_t* ex = at<const uint32_t>(dp, cs.excl_bits_off);
          for (int64_t w = kc0 >> 5; w <= (kc1 >> 5) && full; ++w) {
            const int lo = (w << 5) < kc0 ? (int)(kc0 - (w << 5)) : 0;
            const int hi = ((w << 5) + 31) > kc1 ? (int)(kc1 - (w << 5)) : 31;
            const uint32_t m = (hi - lo == 31) ? 0xFFFFFFFFu : (((1u << (hi - lo + 1)) - 1u) << lo);
            full = (ex[w] & m) == 0u;
          }
        }
      }
      if (full) out[i] = t | TILE_FULL;
    }
    __syncwarp();
    // ---- first tile of each key chunk (gathered-key tiles count as chunk 0; the list is in
    // chunk order: gathered tiles first, then identity windows by ascending key row)
    if (dp.n_kchunks > 1) {
      int32_t* cst = at<int32_t>(dp, dp.lay.cstart) + (int64_t)item * (dp.n_kchunks + 1);
      for (int c = lane; c <= dp.n_kchunks; c += 32) {
        int lo = 0, hi = nt;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          const uint32_t t = out[mid];
          const int tc = ((t >> 28) == SRC_X) ? 0 : (int)((t & TILE_ROW_MASK) / dp.chunk_keys);
          if (tc < c) lo = mid + 1;
          else hi = mid;
        }
        cst[c] = (c == dp.n_kchunks) ? nt : lo;
      }
    }
    __syncwarp();
  }
}

}  // namespace

int sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  cudaGetDevice(&dev);
  int n = (dev >= 0 && dev < 64) ? cached[dev].load(std::memory_order_relaxed) : 0;
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

cudaError_t launch_layout(const DevPlan& dp, cudaStream_t st) {
  count_launches(1);
  layout_kernel<<<std::min(dp.n_segs, 4096), 256, 0, st>>>(dp, dp.n_text);
  return cudaGetLastError();
}

cudaError_t launch_grid_detect(const DevPlan& dp, cudaStream_t st) {
  count_launches(1);
  grid_detect_kernel<<<dp.Hq, 1024, 0, st>>>(dp);
  return cudaGetLastError();
}

cudaError_t launch_materialize(const DevPlan& dp, cudaStream_t st) {
  count_launches(4);
  dyn_init_kernel<<<(dp.n_classes + 127) / 128, 128, 0, st>>>(dp);
  mat_lists_kernel<<<dp.n_classes, 512, 0, st>>>(dp);
  grid_count_kernel<<<dim3(GM_BLOCKS, dp.Hq), GM_THREADS, 0, st>>>(dp);
  grid_write_kernel<<<dim3(GM_BLOCKS, dp.Hq), GM_THREADS, 0, st>>>(dp);
  for (int c = 0; c < dp.n_classes; ++c)
    if (dp.class_kind[c] == MSA_BLOCK) {
      count_launches(1);
      block_bits_kernel<<<std::max(1, std::min(dp.nb / 8, 1024)), 256, 0, st>>>(dp, c);
    }
  return cudaGetLastError();
}

cudaError_t launch_tiles(const DevPlan& dp, cudaStream_t st) {
  const int bm_words = dp.tb_words;
  const size_t per_warp = (size_t)(bm_words + 2 * TILE) * 4;
  int warps = TB_WARPS;
  while (warps > 1 && per_warp * warps > 200 * 1024) --warps;
  const size_t smem = per_warp * warps;
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  static size_t configured = 0;
  if (smem > 48 * 1024 && smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(tiles_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  const int blocks = std::max(1, std::min((dp.n_items + warps - 1) / warps, sm_count() * 8));
  count_launches(1);
  tiles_kernel<<<blocks, warps * 32, smem, st>>>(dp, bm_words);
  return cudaGetLastError();
}

}  // namespace msa
