// Block-sparse causal flash attention over executed 128x128 tiles, sm_100a.
//
// MMInference ("key machinery"): block-sparse FlashAttention-style kernels load only the
// permuted blocks and keep the tensor-core compute dense; "Grid-Shape Flash Attention"
// (Algorithm 5) is the FlashAttention-2 online softmax over those blocks.  Here:
//  - one persistent CTA per SM walks 128-query work items;
//  - warp 0 streams Q, K and V tiles with TMA (128-byte swizzle) into a 2-stage ring;
//  - warp 1 (one elected thread) issues tcgen05.mma: S = Q K^T into one of two TMEM
//    buffers, then O += P V with O resident in TMEM for the whole work item;
//  - warps 2..9 form two warpgroups, each owning TMEM lanes 0..127 (one query row per thread)
//    and one 64-key half of every tile: they read S with
//    tcgen05.ld, apply the element mask (causal in original positions + the head's
//    pattern), run the online softmax in fp32 (exp2 on MUFU, lazy rescale of O when the
//    running max grows by more than 2^8), write P as bf16 into shared memory in the
//    K-major 128B-swizzled layout the MMA reads, and finally normalise O.
// Every wait is bounded; on a timeout the CTA records DEV_ERR_TIMEOUT and unwinds.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <algorithm>

#include "kernels.h"

#include "msa_internal.h"
#include "ptx.cuh"

namespace msa {

struct AttnParams {
  const uint8_t* ws;
  Layout lay;
  int32_t L, Hq, Hkv, LP;
  int32_t n_items;
  float scale_log2;        // softmax scale * log2(e)
  float* lse;              // [Hq][L] or null
};

constexpr int ATT_THREADS = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 softmax (two warpgroups)
constexpr int K_STAGES = 2;  // K tiles are loaded ahead of V tiles
constexpr int V_STAGES = 2;
constexpr uint32_t TILE_BYTES = 128 * 128 * 2;  // one 128x128 bf16 tile
constexpr uint32_t ATOM_BYTES = 128 * 128;      // one [128 rows][64 cols] 128B-swizzled atom

struct __align__(1024) AttnSmem {
  uint8_t q[TILE_BYTES];
  uint8_t k[K_STAGES][TILE_BYTES];
  uint8_t v[V_STAGES][TILE_BYTES];
  uint8_t p[TILE_BYTES];
  uint64_t q_full, q_empty;
  uint64_t k_full[K_STAGES], k_empty[K_STAGES];
  uint64_t v_full[V_STAGES], v_empty[V_STAGES];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], pv_done[2], o_free, drain;
  float xm[2][128];  // [key half][row] running max of the half (log2 units)
  float xl[2][128];  // [key half][row] running sum of the half
  uint32_t tmem_base;
  int abort;
};

static_assert(sizeof(AttnSmem) <= 232448, "attention shared memory exceeds 227 KB per CTA");

constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O = 256;  // O of key half g at TM_O + 128 g

__device__ __forceinline__ const ClassStatic& class_of(const AttnParams& p, int c) {
  return reinterpret_cast<const ClassStatic*>(p.ws + p.lay.classes)[c];
}

// Item geometry shared by all roles.
struct ItemInfo {
  int cls, head, kvh;
  int nrows, row0, qrow0;  // rows in class, first row of the item, first row of class in Q/O slice
  int ntiles;
  int64_t tile0;
  int q_src;               // 0: original Q, 1: permuted Q
  int q_slice, x_slice;
};

__device__ __forceinline__ bool load_item(const AttnParams& p, int item, ItemInfo& it) {
  const WorkItem wi = reinterpret_cast<const WorkItem*>(p.ws + p.lay.items)[item];
  const ClassStatic& cs = class_of(p, wi.cls);
  const ClassDyn cd = reinterpret_cast<const ClassDyn*>(p.ws + p.lay.class_dyn)[cs.dyn];
  const HeadStatic& hs = reinterpret_cast<const HeadStatic*>(p.ws + p.lay.heads)[cs.head];
  it.cls = wi.cls;
  it.head = cs.head;
  it.kvh = cs.kvh;
  it.nrows = (cs.flags & CF_DYNROWS) ? cd.nrows : cs.rows_static;
  it.qrow0 = (cs.flags & CF_DYNROWS) ? cd.qrow0 : cs.qrow0_static;
  it.row0 = wi.slot * TILE;
  it.ntiles = reinterpret_cast<const int32_t*>(p.ws + p.lay.item_ntiles)[item];
  it.tile0 = cs.tile_base + (int64_t)wi.slot * cs.tile_cap;
  it.q_src = (cs.flags & CF_PERMUTED) ? 1 : 0;
  it.q_slice = (int)hs.q_slice;
  it.x_slice = (int)hs.x_slice;
  if (it.row0 >= it.nrows) it.ntiles = -1;  // no rows: item skipped by every role
  return it.ntiles >= 0;
}

// Per-row state of the element mask.
struct RowCtx {
  int valid, qpos, qcoord;
  int flags, sink, band, kc_lo, kc_hi, krow_lo, x_row0, nwords, blk_wpr;
  const uint32_t* slash;
  const uint32_t* excl;
  const uint32_t* blk;
  const int32_t* xpos;
};

__device__ __forceinline__ void prefix_mask2(uint32_t (&m)[2], int n) {
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    int k = n - 32 * w;
    m[w] = k >= 32 ? 0xFFFFFFFFu : (k <= 0 ? 0u : ((1u << k) - 1u));
  }
}

// Mask words of one query row against key columns [64 half, 64 half + 64) of a tile, in two
// steps so the bitmap loads of the next tile are in flight while the current tile is
// processed: mask_prefetch issues the loads, mask_finish combines them.
struct MaskRaw {
  int src, krow, kc0;
  uint32_t sl[3], ex[3], bk0, bk1;
};

__device__ __forceinline__ uint32_t ldg_word(const uint32_t* bm, int nwords, int w) {
  return (w >= 0 && w < nwords) ? __ldg(bm + w) : 0u;
}

__device__ __forceinline__ void mask_prefetch(const RowCtx& rc, uint32_t tile, int half, MaskRaw& r) {
  r.src = (int)(tile >> 28);
  r.krow = (int)(tile & 0x0FFFFFFFu);
  r.kc0 = rc.kc_lo + (r.krow - rc.krow_lo) + 64 * half;
  if (!rc.valid || r.src == SRC_X) return;
  if (rc.flags & CF_SLASH) {
    const int w0 = (rc.qcoord - r.kc0 - 63) >> 5;
#pragma unroll
    for (int i = 0; i < 3; ++i) r.sl[i] = ldg_word(rc.slash, rc.nwords, w0 + i);
  }
  if (rc.flags & CF_EXCL) {
    const int w0 = r.kc0 >> 5;
#pragma unroll
    for (int i = 0; i < 3; ++i) r.ex[i] = ldg_word(rc.excl, rc.nwords, w0 + i);
  }
  if (rc.flags & CF_BLOCK) {
    const uint32_t* row = rc.blk + (size_t)(rc.qcoord >> 6) * rc.blk_wpr;
    const int nbk = (rc.kc_hi + 63) >> 6;
    const int b0 = r.kc0 >> 6, b1 = b0 + 1;  // a 64-column half touches at most two blocks
    r.bk0 = b0 < nbk ? (__ldg(row + (b0 >> 5)) >> (b0 & 31)) & 1u : 0u;
    r.bk1 = b1 < nbk ? (__ldg(row + (b1 >> 5)) >> (b1 & 31)) & 1u : 0u;
  }
}

__device__ __forceinline__ void mask_finish(const RowCtx& rc, const MaskRaw& r, int half, uint32_t (&m)[2]) {
  if (!rc.valid) {
    m[0] = m[1] = 0u;
    return;
  }
  if (r.src == SRC_X) {
    // gathered keys are sorted by position: the allowed ones are a prefix
    const int32_t* kp = rc.xpos + (r.krow - rc.x_row0) + 64 * half;
    int lo = 0, hi = 64;
    while (lo < hi) {
      int mid = (lo + hi) >> 1;
      if (__ldg(kp + mid) <= rc.qpos) lo = mid + 1;
      else hi = mid;
    }
    prefix_mask2(m, lo);
    return;
  }
  const int kc0 = r.kc0;
  prefix_mask2(m, min(rc.qcoord - kc0 + 1, rc.kc_hi - kc0));  // causal and inside the region
  if (!(rc.flags & CF_DENSE)) {
    uint32_t any[2] = {0u, 0u};
    if (rc.flags & CF_SINK) {
      uint32_t t[2];
      prefix_mask2(t, rc.sink - kc0);
      any[0] |= t[0];
      any[1] |= t[1];
    }
    if (rc.flags & CF_BAND) {
      uint32_t t[2];
      prefix_mask2(t, rc.qcoord - rc.band + 1 - kc0);  // columns below qcoord - band + 1 are outside
      any[0] |= ~t[0];
      any[1] |= ~t[1];
    }
    if (rc.flags & CF_SLASH) {
      // column c has offset qcoord - kc0 - c: bits [base, base + 64) reversed
      const int sh = (rc.qcoord - kc0 - 63) & 31;
      const uint32_t b0 = __funnelshift_r(r.sl[0], r.sl[1], sh), b1 = __funnelshift_r(r.sl[1], r.sl[2], sh);
      any[0] |= __brev(b1);
      any[1] |= __brev(b0);
    }
    if (rc.flags & CF_BLOCK) {
      // columns before the next 64-boundary of the coordinate lie in block kc0 >> 6
      const int split = 64 - (kc0 & 63);
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int lo = split - 32 * w;  // columns of word w inside the first block
        const uint32_t low = lo >= 32 ? 0xFFFFFFFFu : (lo <= 0 ? 0u : ((1u << lo) - 1u));
        any[w] |= (r.bk0 ? low : 0u) | (r.bk1 ? ~low : 0u);
      }
    }
    m[0] &= any[0];
    m[1] &= any[1];
  }
  if (rc.flags & CF_EXCL) {
    const int sh = kc0 & 31;
    m[0] &= ~__funnelshift_r(r.ex[0], r.ex[1], sh);
    m[1] &= ~__funnelshift_r(r.ex[1], r.ex[2], sh);
  }
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void issue_kv(const CUtensorMap* tk, const CUtensorMap* tv, const CUtensorMap* tk2,
                                         const CUtensorMap* tv2, const CUtensorMap* txk, const CUtensorMap* txv,
                                         bool is_v, uint32_t tile, const ItemInfo& it, uint8_t* dst,
                                         uint64_t* bar) {
  const int src = (int)(tile >> 28);
  const int row = (int)(tile & 0x0FFFFFFFu);
  const CUtensorMap* m;
  int c2;
  if (src == SRC_X) {
    m = is_v ? txv : txk;
    c2 = it.x_slice;
  } else if (src == SRC_K2D) {
    m = is_v ? tv2 : tk2;
    c2 = it.kvh;
  } else {
    m = is_v ? tv : tk;
    c2 = it.kvh;
  }
  mbar_arrive_expect_tx(bar, TILE_BYTES);
  tma_load_3d(dst, m, bar, 0, row, c2);
  tma_load_3d(dst + ATOM_BYTES, m, bar, 64, row, c2);
}

__global__ void __launch_bounds__(ATT_THREADS, 1)
    msa_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQp,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmK2, const __grid_constant__ CUtensorMap tmV2,
                    const __grid_constant__ CUtensorMap tmXK, const __grid_constant__ CUtensorMap tmXV,
                    const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw);
  if (smem_addr(smem_raw) & 1023u) {  // the 128-byte swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicOr(reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(p.ws + p.lay.header)), DEV_ERR_BOUNDS);
    return;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort = &sm.abort;
  uint32_t* err = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(p.ws + p.lay.header));

  if (threadIdx.x == 0) {
    sm.abort = 0;
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < K_STAGES; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < V_STAGES; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.s_free[b], 256);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&sm.p_full[g], 128);
      mbar_init(&sm.pv_done[g], 1);
    }
    mbar_init(&sm.o_free, 256);
    mbar_init(&sm.drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc<TMEM_COLS>(&sm.tmem_base);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      uint32_t k_issued = 0, v_issued = 0, q_uses = 0;
      const uint32_t* tiles = reinterpret_cast<const uint32_t*>(p.ws + p.lay.tiles);
      bool ok = true;
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        ItemInfo it;
        if (!load_item(p, item, it) || it.ntiles == 0) continue;
        if (q_uses > 0 && !mbar_wait(&sm.q_empty, (q_uses - 1) & 1, abort)) { ok = false; break; }
        ++q_uses;
        mbar_arrive_expect_tx(&sm.q_full, TILE_BYTES);
        if (it.q_src) {
          tma_load_3d(sm.q, &tmQp, &sm.q_full, 0, it.qrow0 + it.row0, it.q_slice);
          tma_load_3d(sm.q + ATOM_BYTES, &tmQp, &sm.q_full, 64, it.qrow0 + it.row0, it.q_slice);
        } else {
          tma_load_3d(sm.q, &tmQ, &sm.q_full, 0, it.row0, it.head);
          tma_load_3d(sm.q + ATOM_BYTES, &tmQ, &sm.q_full, 64, it.row0, it.head);
        }
        auto issue_k = [&](int t) -> bool {
          const uint32_t st = k_issued % K_STAGES, use = k_issued / K_STAGES;
          if (use > 0 && !mbar_wait(&sm.k_empty[st], (use - 1) & 1, abort)) return false;
          issue_kv(&tmK, &tmV, &tmK2, &tmV2, &tmXK, &tmXV, false, __ldg(tiles + it.tile0 + t), it, sm.k[st],
                   &sm.k_full[st]);
          ++k_issued;
          return true;
        };
        auto issue_v = [&](int t) -> bool {
          const uint32_t st = v_issued % V_STAGES, use = v_issued / V_STAGES;
          if (use > 0 && !mbar_wait(&sm.v_empty[st], (use - 1) & 1, abort)) return false;
          issue_kv(&tmK, &tmV, &tmK2, &tmV2, &tmXK, &tmXV, true, __ldg(tiles + it.tile0 + t), it, sm.v[st],
                   &sm.v_full[st]);
          ++v_issued;
          return true;
        };
        const int lead = min(K_STAGES - 1, it.ntiles);
        for (int t = 0; t < lead && ok; ++t) ok = issue_k(t);
        for (int t = 0; t < it.ntiles && ok; ++t) {
          if (t + lead < it.ntiles) ok = issue_k(t + lead);
          if (ok) ok = issue_v(t);
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA goes away
        for (uint32_t c = (k_issued > K_STAGES ? k_issued - K_STAGES : 0); c < k_issued; ++c)
          mbar_wait(&sm.k_full[c % K_STAGES], (c / K_STAGES) & 1, abort, 100000000ull);
        for (uint32_t c = (v_issued > V_STAGES ? v_issued - V_STAGES : 0); c < v_issued; ++c)
          mbar_wait(&sm.v_full[c % V_STAGES], (c / V_STAGES) & 1, abort, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, 0, 1);
      const uint32_t q_addr = smem_addr(sm.q), p_addr = smem_addr(sm.p);
      uint32_t k_used = 0, v_used = 0, s_count = 0, q_uses = 0, p_uses = 0, items_done = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        ItemInfo it;
        if (!load_item(p, item, it) || it.ntiles == 0) continue;
        if (!mbar_wait(&sm.q_full, q_uses & 1, abort)) { ok = false; break; }
        ++q_uses;
        auto do_pv = [&](int t) -> bool {
          const uint32_t st = v_used % V_STAGES, use = v_used / V_STAGES;
          if (!mbar_wait(&sm.v_full[st], use & 1, abort)) return false;
          if (t == 0 && items_done > 0 && !mbar_wait(&sm.o_free, (items_done - 1) & 1, abort)) return false;
          const uint32_t v_addr = smem_addr(sm.v[st]);
          // O_g += P[:, 64g:64g+64] V[64g:64g+64, :] for each key half g, as soon as its P is ready
          for (int g = 0; g < 2; ++g) {
            if (!mbar_wait(&sm.p_full[g], p_uses & 1, abort)) return false;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = smem_desc_sw128(p_addr + g * ATOM_BYTES + kk * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(v_addr + g * 8192 + kk * 2048, ATOM_BYTES, 1024);
              umma_ss(tmem + TM_O + 128 * g, ad, bd, IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&sm.pv_done[g]);
          }
          ++p_uses;
          umma_commit(&sm.v_empty[st]);
          ++v_used;
          return true;
        };
        for (int t = 0; t < it.ntiles && ok; ++t) {
          const uint32_t st = k_used % K_STAGES, use = k_used / K_STAGES;
          const uint32_t sb = s_count & 1, su = s_count >> 1;
          if (!mbar_wait(&sm.k_full[st], use & 1, abort)) { ok = false; break; }
          if (su > 0 && !mbar_wait(&sm.s_free[sb], (su - 1) & 1, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = smem_addr(sm.k[st]);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * ATOM_BYTES + (kk & 3) * 32;
            umma_ss(tmem + (sb ? TM_S1 : TM_S0), smem_desc_sw128(q_addr + off, 16, 1024),
                    smem_desc_sw128(k_addr + off, 16, 1024), IDESC_QK, kk > 0 ? 1u : 0u);
          }
          umma_commit(&sm.s_full[sb]);
          umma_commit(&sm.k_empty[st]);
          if (t == it.ntiles - 1) umma_commit(&sm.q_empty);
          ++k_used;
          ++s_count;
          if (t > 0 && !do_pv(t - 1)) { ok = false; break; }
        }
        if (ok && !do_pv(it.ntiles - 1)) ok = false;
        ++items_done;
      }
      // wait for every MMA issued by this thread before the tensor memory is released
      umma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, abort, 100000000ull);
    }
  } else {
    // ------------------------------------------------------------------ softmax / epilogue
    // Two independent warpgroups: warpgroup g owns key columns [64g, 64g + 64) of every S
    // tile with its own running max / sum and its own accumulator O_g = sum P_g V_g in TMEM;
    // the halves are combined once per work item.  Thread t owns query row t (TMEM lane t).
    const int g = (warp - 2) >> 2;  // warps 2-5: key half 0, warps 6-9: key half 1
    const int t = (warp & 3) * 32 + lane;  // a warp may only touch TMEM lanes 32 (warp % 4) .. + 31
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t o_own = lane_base + TM_O + 128 * g;
    __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(const_cast<uint8_t*>(p.ws + p.lay.op));
    const uint32_t* tiles = reinterpret_cast<const uint32_t*>(p.ws + p.lay.tiles);
    uint32_t s_count = 0, pv_waits = 0, items_done = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      ItemInfo it;
      if (!load_item(p, item, it)) continue;
      const ClassStatic& cs = class_of(p, it.cls);
      const int r = it.row0 + t;
      RowCtx rc;
      rc.valid = r < it.nrows;
      const int32_t* rows = reinterpret_cast<const int32_t*>(p.ws + cs.rows_off);
      rc.qpos = rc.valid ? ((cs.flags & CF_PERMUTED) ? __ldg(rows + r) : r) : 0;
      rc.qcoord = (cs.flags & CF_RANK) ? r : rc.qpos;
      rc.flags = cs.flags;
      rc.sink = cs.sink;
      rc.band = cs.band;
      rc.kc_lo = cs.kc_lo;
      rc.kc_hi = cs.kc_hi;
      rc.krow_lo = cs.krow_lo;
      rc.x_row0 = cs.x_row0;
      rc.nwords = (p.L + 31) >> 5;
      rc.blk_wpr = cs.blk_wpr;
      rc.slash = reinterpret_cast<const uint32_t*>(p.ws + cs.slash_bits_off);
      rc.excl = reinterpret_cast<const uint32_t*>(p.ws + cs.excl_bits_off);
      rc.blk = reinterpret_cast<const uint32_t*>(p.ws + cs.blk_bits_off);
      rc.xpos = reinterpret_cast<const int32_t*>(p.ws + cs.x_pos_off);
      const size_t orow = ((size_t)it.head * p.LP + it.qrow0 + r) * D + 64 * g;

      if (it.ntiles == 0) {
        if (rc.valid) {
          uint4* dst = reinterpret_cast<uint4*>(op + orow);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
          if (p.lse && g == 0) p.lse[(size_t)it.head * p.L + rc.qpos] = -INFINITY;
        }
        continue;
      }

      float m_used = -INFINITY, l = 0.f;
      uint32_t mk[2];
      MaskRaw raw;
      mask_prefetch(rc, __ldg(tiles + it.tile0), g, raw);
      mask_finish(rc, raw, g, mk);
      for (int tt = 0; tt < it.ntiles; ++tt) {
        const bool has_next = tt + 1 < it.ntiles;
        if (has_next) mask_prefetch(rc, __ldg(tiles + it.tile0 + tt + 1), g, raw);

        const uint32_t sb = s_count & 1, su = s_count >> 1;
        if (!mbar_wait(&sm.s_full[sb], su & 1, abort)) { ok = false; break; }
        tc_fence_after();
        float s[64];
        {
          const uint32_t scol = lane_base + (sb ? TM_S1 : TM_S0) + 64 * g;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t rr[32];
            tmem_ld32(scol + 32 * c, rr);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) s[32 * c + j] = __uint_as_float(rr[j]);
          }
        }
        tc_fence_before();
        mbar_arrive(&sm.s_free[sb]);
        ++s_count;

#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = ((mk[c >> 5] >> (c & 31)) & 1u) ? s[c] : -INFINITY;
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 64; c += 8) {
#pragma unroll
          for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], s[c + 2 * q], s[c + 2 * q + 1]);
        }
        const float mxs = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * p.scale_log2;
        float alpha = 1.f;
        bool resc = false;
        if (mxs > m_used + 8.f) {  // also true on the first finite max
          alpha = (m_used == -INFINITY) ? 0.f : ex2(m_used - mxs);
          m_used = mxs;
          resc = true;
        }

        // the previous P_g V_g must be complete before P_g is overwritten or O_g rescaled
        if (tt > 0) {
          if (!mbar_wait(&sm.pv_done[g], pv_waits & 1, abort)) { ok = false; break; }
          ++pv_waits;
          tc_fence_after();
          if (__any_sync(0xFFFFFFFFu, resc)) {
            const float f = resc ? alpha : 1.f;
#pragma unroll 1
            for (int c = 0; c < 8; ++c) {  // 16 columns at a time: S stays live in registers
              uint32_t oo[16];
              tmem_ld16(o_own + 16 * c, oo);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 16; ++j) oo[j] = __float_as_uint(__uint_as_float(oo[j]) * f);
              tmem_st16(o_own + 16 * c, oo);
            }
            tmem_wait_st();
          }
        }
        const float nb = (m_used == -INFINITY) ? 0.f : -m_used;
        float rs4[4] = {0.f, 0.f, 0.f, 0.f};
        // P row t, K-major 128B swizzle: atom g holds keys 64g..64g+63; chunk j -> j ^ (t & 7)
        uint8_t* prow = sm.p + g * ATOM_BYTES + t * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float a = ex2(fmaf(s[32 * h + 2 * c], p.scale_log2, nb));
            const float b = ex2(fmaf(s[32 * h + 2 * c + 1], p.scale_log2, nb));
            rs4[c & 3] += a + b;
            pk[c] = pack_bf16x2(a, b);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 v = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            *reinterpret_cast<uint4*>(prow + (((4 * h + j) ^ (t & 7)) << 4)) = v;
          }
        }
        l = l * alpha + ((rs4[0] + rs4[1]) + (rs4[2] + rs4[3]));
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sm.p_full[g]);
        if (has_next) mask_finish(rc, raw, g, mk);
      }
      if (!ok) break;
      // epilogue: both halves' last P V done, then O = (c0 O_0 + c1 O_1) / (c0 l0 + c1 l1)
      if (!mbar_wait(&sm.pv_done[g], pv_waits & 1, abort)) { ok = false; break; }
      ++pv_waits;
      sm.xm[g][t] = m_used;
      sm.xl[g][t] = l;
      tc_fence_before();
      named_bar_sync(1, 256);
      tc_fence_after();
      const float m0 = sm.xm[0][t], m1 = sm.xm[1][t];
      const float M = fmaxf(m0, m1);
      const float c0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - M);
      const float c1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M);
      const float ltot = c0 * sm.xl[0][t] + c1 * sm.xl[1][t];
      named_bar_sync(1, 256);  // both halves read before the next item's values land
      const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
      const float f0 = c0 * inv, f1 = c1 * inv;
      uint4* dst = reinterpret_cast<uint4*>(op + orow);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t oa[32], ob[32];
        tmem_ld32(lane_base + TM_O + 64 * g + 32 * c, oa);
        tmem_ld32(lane_base + TM_O + 128 + 64 * g + 32 * c, ob);
        tmem_wait_ld();
        if (c == 1) {
          tc_fence_before();
          mbar_arrive(&sm.o_free);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k = 8 * j + 2 * e;
            w[e] = pack_bf16x2(__uint_as_float(oa[k]) * f0 + __uint_as_float(ob[k]) * f1,
                               __uint_as_float(oa[k + 1]) * f0 + __uint_as_float(ob[k + 1]) * f1);
          }
          if (rc.valid) dst[4 * c + j] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      ++items_done;
      if (rc.valid && p.lse && g == 0)
        p.lse[(size_t)it.head * p.L + rc.qpos] = (ltot > 0.f) ? (M + __log2f(ltot)) * 0.6931471805599453f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && sm.abort) atomicOr(err, DEV_ERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<TMEM_COLS>(tmem);
  }
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3D map over [heads][rows][128] bf16 with element strides; boxes of 128 rows x 64 columns,
// 128-byte swizzle; rows beyond `rows` read as zero.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t heads, int64_t row_stride,
              int64_t head_stride) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)std::max<int64_t>(heads, 1)};
  cuuint64_t strides[2] = {(cuuint64_t)(row_stride * 2), (cuuint64_t)(std::max<int64_t>(head_stride, rows * row_stride) * 2)};
  if (heads > 1) strides[1] = (cuuint64_t)(head_stride * 2);
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attention(const DevPlan& dp, const void* Q, const void* K, const void* V, const msa_strides& s,
                             float* lse, cudaStream_t st) {
  CUtensorMap mq, mqp, mk, mv, mk2, mv2, mxk, mxv;
  const uint8_t* ws = dp.ws;
  bool ok = make_map(&mq, Q, dp.L, dp.Hq, s.q_row, s.q_head) && make_map(&mk, K, dp.L, dp.Hkv, s.k_row, s.k_head) &&
            make_map(&mv, V, dp.L, dp.Hkv, s.v_row, s.v_head) &&
            make_map(&mqp, ws + dp.lay.qp, dp.LP, std::max(dp.n_qslices, 1), D, (int64_t)dp.LP * D) &&
            make_map(&mxk, ws + dp.lay.xk, dp.x_rows, std::max(dp.n_xslices, 1), D, (int64_t)dp.x_rows * D) &&
            make_map(&mxv, ws + dp.lay.xv, dp.x_rows, std::max(dp.n_xslices, 1), D, (int64_t)dp.x_rows * D);
  if (ok && dp.has2d) {
    ok = make_map(&mk2, ws + dp.lay.k2d, dp.L, dp.Hkv, D, dp.L * D) &&
         make_map(&mv2, ws + dp.lay.v2d, dp.L, dp.Hkv, D, dp.L * D);
  } else {
    mk2 = mk;
    mv2 = mv;
  }
  if (!ok) return cudaErrorInvalidValue;
  AttnParams p;
  p.ws = ws;
  p.lay = dp.lay;
  p.L = (int32_t)dp.L;
  p.Hq = dp.Hq;
  p.Hkv = dp.Hkv;
  p.LP = dp.LP;
  p.n_items = dp.n_items;
  p.scale_log2 = dp.scale * 1.4426950408889634f;
  p.lse = lse;
  const size_t smem = sizeof(AttnSmem);
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(msa_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int grid = std::max(1, std::min(dp.n_items, sm_count()));
  count_launches(1);
  msa_attn_kernel<<<grid, ATT_THREADS, smem, st>>>(mq, mqp, mk, mv, mk2, mv2, mxk, mxv, p);
  return cudaGetLastError();
}

}  // namespace msa
