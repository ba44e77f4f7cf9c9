// Block-sparse causal flash attention over executed 128x128 tiles, sm_100a.
//
// MMInference ("key machinery"): block-sparse FlashAttention-style kernels load only the
// permuted blocks and keep the tensor-core compute dense; "Grid-Shape Flash Attention"
// (Algorithm 5) is the FlashAttention-2 online softmax over those blocks.  Here:
//  - one persistent CTA per SM runs two independent streams of work units (a 128-query work
//    item, or, for long sequences whose keys are cut into chunks, the item's tiles of one key
//    chunk); each stream takes the next unit from a global counter when it needs one (plan
//    order: grouped so that the units in flight share one head's K/V in L2, longest first);
//  - a unit after its item's first key chunk resumes the item's online softmax from an
//    accumulator in the workspace (unnormalised O, running max and sum), handed over between
//    units through a per-item counter (release / acquire);
//  - warps 0 and 2 stream the Q, K and V tiles of stream 0 and 1 with TMA (128-byte
//    swizzle) into single-buffered slots of their own; in the index-based instantiation
//    (msa_attn_kernel<true>) the whole warp also gathers the query rows of permuted classes
//    from the caller's Q by row index (cp.async into the swizzled Q slot);
//  - warps 1 and 3 (one thread each) issue the tcgen05.mma of stream 0 and 1:
//    S_s = Q_s K^T into stream s's TMEM columns, then O_s += P_s V with P_s read from TMEM
//    and O_s resident in TMEM for the whole unit; a group [PV(j), QK(j + 1)] is issued under
//    a lock shared by the two issuers, so the tensor pipe receives whole groups back to back
//    and the streams settle half a cycle apart: one stream's MMAs run while the other
//    stream computes its softmax;
//  - warps 4..7 (stream 0) and 8..11 (stream 1) each own TMEM lanes 0..127, one query row per
//    thread and all 128 keys of every tile: they read S with tcgen05.ld, apply the element
//    mask (causal in original positions + the head's pattern), run the online softmax in fp32
//    (exp2 on MUFU, lazy rescale of O when the running max grows by more than 2^8), write P
//    as packed bf16 over the first 64 columns of S with tcgen05.st, and finally normalise O
//    into the permuted O copy (or, index-based, into the caller's O at the original position).
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
  uint32_t* next_item;     // work-unit counter, zero at launch
  int32_t n_units, n_kchunks, n_bands;
  uint32_t* chunk_done;    // per item: chunks whose state is in its accumulator (chunked keys)
  uint32_t* band_done;     // per band: units finished (chunked keys)
  float* acc;              // accumulator slots [slot][128][ACC_ROW] (chunked keys)
  // index-based prefill (od not null): the Q rows of permuted classes are gathered from the
  // caller's Q by row index, and every output row goes to the caller's O at its original
  // position; otherwise Q comes from the permuted copy and O goes to the permuted O copy
  const __nv_bfloat16* qg;
  int64_t qg_head, qg_row;
  __nv_bfloat16* od;
  int64_t od_head, od_row;
};

// warpgroup 0: warps 0 / 2 TMA of stream 0 / 1, warps 1 / 3 MMA of stream 0 / 1; warpgroups
// 1 / 2: softmax of stream 0 / 1
constexpr int ATT_THREADS = 384;
// Register split (setmaxnreg): launched at 168 per thread (384 x 168 = 64512), warpgroup 0 gives
// back to 72 and the softmax warpgroups grow to 216: 128 x 72 + 256 x 216 = 64512.
constexpr int REG_CTRL = 72, REG_SOFTMAX = 216;
static_assert(128 * REG_CTRL + 256 * REG_SOFTMAX <= ATT_THREADS * 168, "register split exceeds the launch allocation");
constexpr int N_STREAMS = 2;
constexpr int IQ_DEPTH = 4;
// readers of a queue entry: the MMA issuer, the V loads of the TMA thread, 128 softmax threads
constexpr uint32_t IQ_READERS = 130;
constexpr uint32_t TILE_BYTES = 128 * 128 * 2;  // one 128x128 bf16 tile
constexpr uint32_t ATOM_BYTES = 128 * 128;      // one [128 rows][64 cols] 128B-swizzled atom

// Per-row state of the element mask.
struct RowCtx {
  int valid, qpos, qcoord;
  int flags, sink, band, kc_lo, kc_hi, krow_lo, x_row0, nwords, blk_wpr;
  const uint32_t* slash;
  const uint32_t* excl;
  const uint32_t* blk;
  const int32_t* xpos;
};

struct __align__(1024) AttnSmem {
  uint8_t q[N_STREAMS][TILE_BYTES];
  uint8_t k[N_STREAMS][TILE_BYTES];
  uint8_t v[N_STREAMS][TILE_BYTES];
  uint64_t q_full[N_STREAMS], q_empty[N_STREAMS];
  uint64_t k_full[N_STREAMS], k_empty[N_STREAMS];
  uint64_t v_full[N_STREAMS], v_empty[N_STREAMS];
  uint64_t qg_full[N_STREAMS];  // Q gathered by the producer warp (index-based prefill)
  uint64_t s_full[N_STREAMS], p_full[N_STREAMS];
  uint64_t o_full[N_STREAMS], o_free[N_STREAMS];
  // work-item queue of each stream: ids taken from the global counter by the stream's TMA
  // thread, read by its MMA issuer and softmax warpgroup (-1 ends the stream)
  int32_t iq[N_STREAMS][IQ_DEPTH][4];  // item, key chunk, accumulator slot, band
  uint64_t iq_full[N_STREAMS][IQ_DEPTH], iq_empty[N_STREAMS][IQ_DEPTH];
  // softmax warpgroup handshakes around the accumulator of chunked items
  uint64_t acc_in[N_STREAMS], acc_out[N_STREAMS];
  uint64_t drain[N_STREAMS];
  RowCtx rctx[256];  // mask state of the row of each softmax thread (read off the critical path)
  uint32_t tmem_base;
  int abort;
  int issue_lock;
};

static_assert(sizeof(AttnSmem) <= 232448, "attention shared memory exceeds 227 KB per CTA");

constexpr uint32_t TMEM_COLS = 512;
// stream s: S (fp32, 128 columns; P as packed bf16 pairs over its first 64) at 256 s,
// O (fp32, 128 columns) at 256 s + 128
constexpr uint32_t TM_STREAM = 256, TM_OOFF = 128;

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

// One queue entry: the unit's item and key chunk.  it.tile0 / it.ntiles are narrowed to the
// unit's tiles; k = key chunks of the item before this one that have tiles (their state is in
// the item's accumulator), last = no tiles of the item after this unit, total = the item's
// tiles.  False: the item has no rows (every role skips it).
struct UnitInfo {
  int item, chunk, acc, band, k, total;
  bool last;
};

__device__ __forceinline__ bool load_unit(const AttnParams& p, const int32_t* e, ItemInfo& it, UnitInfo& u) {
  u.item = e[0];
  u.chunk = e[1];
  u.acc = e[2];
  u.band = e[3];
  if (!load_item(p, u.item, it)) return false;
  u.total = it.ntiles;
  u.k = 0;
  u.last = true;
  if (p.n_kchunks > 1 && it.ntiles > 0) {
    const int32_t* cs = reinterpret_cast<const int32_t*>(p.ws + p.lay.cstart) + (int64_t)u.item * (p.n_kchunks + 1);
    const int t0 = cs[u.chunk], t1 = cs[u.chunk + 1];
    for (int c = 0; c < u.chunk; ++c) u.k += cs[c + 1] > cs[c] ? 1 : 0;
    u.last = t1 == it.ntiles;
    it.tile0 += t0;
    it.ntiles = t1 - t0;
  }
  return true;
}

// Unit id -> (item, key chunk, accumulator slot, band).
__device__ __forceinline__ void unit_entry(const AttnParams& p, int u, int32_t (&e)[4]) {
  if (p.n_kchunks == 1) {
    e[0] = u;
    e[1] = 0;
    e[2] = -1;
    e[3] = -1;
    return;
  }
  const UnitBand* b = reinterpret_cast<const UnitBand*>(p.ws + p.lay.bands);
  int lo = 0, hi = p.n_bands - 1;  // last band with unit0 <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (b[mid].unit0 <= u) lo = mid;
    else hi = mid - 1;
  }
  const UnitBand bd = b[lo];
  const int local = u - bd.unit0;
  e[0] = bd.item0 + local % bd.n;
  e[1] = local / bd.n;
  e[2] = bd.acc0 + local % bd.n;
  e[3] = lo;
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* a) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(uint32_t* a, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void red_release_add(uint32_t* a, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(a), "r"(v) : "memory");
}

// Accumulator slots of band b are those of bands b - 2, b - 4, ... (two buffers, alternate
// bands).  Every unit counts itself finished in its band's counter once it no longer touches its
// slot; a unit of band b >= 2 waits (bounded) until every unit of every earlier band of the same
// parity has finished before its item's first write to the slot.  (Band b - 2 alone is not
// enough: a band whose items all end in their first chunk with keys never writes a slot, so it
// can finish while the band before it still uses the buffer.)  Earlier bands' units were all
// handed out before any of band b, and a stream runs its units in the order it took them, so
// the oldest unfinished unit never waits on a newer one.  known0 / known1: bands of even / odd
// index below it are already known finished (a stream's bands only increase).
__device__ __forceinline__ void band_unit_done(const AttnParams& p, const UnitInfo& u) {
  if (p.band_done && u.band >= 0) red_release_add(p.band_done + u.band, 1u);
}
__device__ __forceinline__ bool band_wait_previous(const AttnParams& p, const UnitInfo& u, int& known0,
                                                   int& known1, volatile int* abort) {
  if (!p.band_done || u.band < 2) return true;
  const bool odd = (u.band & 1) != 0;
  const UnitBand* bands = reinterpret_cast<const UnitBand*>(p.ws + p.lay.bands);
  const uint64_t t0 = global_ns();
  for (int b = odd ? known1 : known0; b <= u.band - 2; b += 2) {
    const uint32_t need = (uint32_t)bands[b].n * (uint32_t)p.n_kchunks;
    while (ld_acquire(p.band_done + b) < need) {
      if (*abort) return false;
      if (global_ns() - t0 > 1000000000ull) {
        *abort = 1;
        return false;
      }
    }
  }
  if (odd) known1 = u.band;
  else known0 = u.band;
  return true;
}


// Bits [0, n) of the 32-column word w of a 128-column row (n clipped to [0, 128]).
__device__ __forceinline__ uint32_t low_bits(int n, int w) {
  const int k = n - 32 * w;
  return k >= 32 ? 0xFFFFFFFFu : (k <= 0 ? 0u : ((1u << k) - 1u));
}

__device__ __forceinline__ void prefix_mask4(uint32_t (&m)[4], int n) {
#pragma unroll
  for (int w = 0; w < 4; ++w) m[w] = low_bits(n, w);
}

// Mask words of one query row against the 128 key columns of a tile, in two steps so the
// bitmap loads are in flight while the thread waits for S: mask_prefetch issues the loads,
// mask_finish combines them.
struct MaskRaw {
  int src, krow, kc0;
  uint32_t sl[5], ex[5], bk[3];
};

__device__ __forceinline__ uint32_t ldg_word(const uint32_t* bm, int nwords, int w) {
  return (w >= 0 && w < nwords) ? __ldg(bm + w) : 0u;
}

__device__ __forceinline__ void mask_prefetch(const RowCtx& rc, uint32_t tile, MaskRaw& r) {
  r.src = (int)(tile >> 28);
  r.krow = (int)(tile & TILE_ROW_MASK);
  r.kc0 = rc.kc_lo + (r.krow - rc.krow_lo);
  if (!rc.valid || r.src == SRC_X) return;
  if (rc.flags & CF_SLASH) {
    const int w0 = (rc.qcoord - r.kc0 - 127) >> 5;
#pragma unroll
    for (int i = 0; i < 5; ++i) r.sl[i] = ldg_word(rc.slash, rc.nwords, w0 + i);
  }
  if (rc.flags & CF_EXCL) {
    const int w0 = r.kc0 >> 5;
#pragma unroll
    for (int i = 0; i < 5; ++i) r.ex[i] = ldg_word(rc.excl, rc.nwords, w0 + i);
  }
  if (rc.flags & CF_BLOCK) {
    const uint32_t* row = rc.blk + (size_t)(rc.qcoord >> 6) * rc.blk_wpr;
    const int nbk = (rc.kc_hi + 63) >> 6;
    const int b0 = r.kc0 >> 6;  // 128 columns touch at most three 64-blocks
#pragma unroll
    for (int i = 0; i < 3; ++i) r.bk[i] = (b0 + i) < nbk ? (__ldg(row + ((b0 + i) >> 5)) >> ((b0 + i) & 31)) & 1u : 0u;
  }
}

__device__ __forceinline__ void mask_finish(const RowCtx& rc, const MaskRaw& r, uint32_t (&m)[4]) {
  if (!rc.valid) {
    m[0] = m[1] = m[2] = m[3] = 0u;
    return;
  }
  if (r.src == SRC_X) {
    // gathered keys are sorted by position: the allowed ones are a prefix
    const int32_t* kp = rc.xpos + (r.krow - rc.x_row0);
    int lo = 0, hi = 128;
    while (lo < hi) {
      int mid = (lo + hi) >> 1;
      if (__ldg(kp + mid) <= rc.qpos) lo = mid + 1;
      else hi = mid;
    }
    prefix_mask4(m, lo);
    return;
  }
  const int kc0 = r.kc0;
  prefix_mask4(m, min(rc.qcoord - kc0 + 1, rc.kc_hi - kc0));  // causal and inside the region
  if (!(rc.flags & CF_DENSE)) {
    uint32_t any[4] = {0u, 0u, 0u, 0u};
    if (rc.flags & CF_SINK) {
#pragma unroll
      for (int w = 0; w < 4; ++w) any[w] |= low_bits(rc.sink - kc0, w);
    }
    if (rc.flags & CF_BAND) {  // columns below qcoord - band + 1 are outside the band
#pragma unroll
      for (int w = 0; w < 4; ++w) any[w] |= ~low_bits(rc.qcoord - rc.band + 1 - kc0, w);
    }
    if (rc.flags & CF_SLASH) {
      // column c has offset qcoord - kc0 - c: bits [base, base + 128) of the offset bitmap,
      // base = qcoord - kc0 - 127, in reverse column order
      const int sh = (rc.qcoord - kc0 - 127) & 31;
#pragma unroll
      for (int w = 0; w < 4; ++w) any[w] |= __brev(__funnelshift_r(r.sl[3 - w], r.sl[4 - w], sh));
    }
    if (rc.flags & CF_BLOCK) {
      // columns [0, split) lie in block kc0 >> 6, [split, split + 64) in the next one, the
      // rest in the one after
      const int split = 64 - (kc0 & 63);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t a = low_bits(split, w), b = low_bits(split + 64, w);
        any[w] |= (r.bk[0] ? a : 0u) | (r.bk[1] ? (b & ~a) : 0u) | (r.bk[2] ? ~b : 0u);
      }
    }
#pragma unroll
    for (int w = 0; w < 4; ++w) m[w] &= any[w];
  }
  if (rc.flags & CF_EXCL) {
    const int sh = kc0 & 31;
#pragma unroll
    for (int w = 0; w < 4; ++w) m[w] &= ~__funnelshift_r(r.ex[w], r.ex[w + 1], sh);
  }
}

// Mask state of query row `t` of an item (row it.row0 + t of its class).
__device__ __forceinline__ void fill_row_ctx(const AttnParams& p, const ItemInfo& it, const ClassStatic& cs, int t,
                                             RowCtx& rc) {
  const int r = it.row0 + t;
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
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ void issue_kv(const CUtensorMap* tk, const CUtensorMap* tv, const CUtensorMap* tk2,
                                         const CUtensorMap* tv2, const CUtensorMap* txk, const CUtensorMap* txv,
                                         bool is_v, uint32_t tile, const ItemInfo& it, uint8_t* dst,
                                         uint64_t* bar) {
  const int src = (int)(tile >> 28);
  const int row = (int)(tile & TILE_ROW_MASK);
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

// No-progress guard of the polling roles: true (and *abort raised) after one second without
// progress, or as soon as another role has aborted.
struct Watchdog {
  uint64_t t0 = 0;
  int idle = 0;
  __device__ __forceinline__ void progress() { idle = 0; }
  __device__ __forceinline__ bool expired(volatile int* abort) {
    if (++idle < 64) return false;
    if (idle == 64) t0 = global_ns();
    if (*abort) return true;
    if (global_ns() - t0 > 1000000000ull) {
      *abort = 1;
      return true;
    }
    return false;
  }
};

// Exclusive right to issue tcgen05.mma, held for one group at a time (see mma_stream).
__device__ __forceinline__ bool issue_lock(int* lock, volatile int* abort) {
  if (atomicCAS(lock, 0, 1) == 0) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    for (int i = 0; i < 32; ++i)
      if (atomicCAS(lock, 0, 1) == 0) return true;
    if (*abort) return false;
    if (global_ns() - t0 > 1000000000ull) {
      *abort = 1;
      return false;
    }
  }
}
__device__ __forceinline__ void issue_unlock(int* lock) { atomicExch(lock, 0); }

// MMA issuer of one stream (one thread).  Per item: QK(0), then the groups [PV(j), QK(j + 1)]
// and finally PV(n - 1).  QK(j + 1) may overwrite P(j) in TMEM because the tcgen05.mma
// operations of one thread run in issue order.  Each stream has its own issuer, so one
// stream never waits for the other's softmax; a group is issued under a lock shared by the two
// issuers, so the tensor pipe receives whole groups back to back instead of interleaved.  A
// stream whose group follows the other's gets its S one group later and starts its softmax
// then: the streams settle half a cycle apart, and one stream's MMAs run while the other
// computes its softmax.
template <bool INDEXED>
__device__ __forceinline__ void mma_stream(const AttnParams& p, AttnSmem& sm, uint32_t tmem, int s,
                                           volatile int* abort) {
  constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, 0, 1);
  const uint32_t s_col = tmem + TM_STREAM * s;
  uint32_t q_use = 0, qg_use = 0, k_use = 0, v_use = 0, done = 0;
  auto qk = [&](bool last) {
    tc_fence_after();
    uint32_t q_addr = smem_addr(sm.q[s]), k_addr = smem_addr(sm.k[s]);
    // keep the descriptors from being hoisted out of the loop: the issuer has 72 registers
    asm volatile("" : "+r"(q_addr), "+r"(k_addr));
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t off = (kk >> 2) * ATOM_BYTES + (kk & 3) * 32;
      umma_ss(s_col, smem_desc_sw128(q_addr + off, 16, 1024), smem_desc_sw128(k_addr + off, 16, 1024), IDESC_QK,
              kk > 0 ? 1u : 0u);
    }
    umma_commit(&sm.s_full[s]);
    umma_commit(&sm.k_empty[s]);
    if (last) umma_commit(&sm.q_empty[s]);
    ++k_use;
  };
  for (uint32_t qi = 0;; ++qi) {
    const uint32_t slot = qi % IQ_DEPTH;
    if (!mbar_wait(&sm.iq_full[s][slot], (qi / IQ_DEPTH) & 1, abort)) return;
    const int32_t e[4] = {sm.iq[s][slot][0], sm.iq[s][slot][1], sm.iq[s][slot][2], sm.iq[s][slot][3]};
    mbar_arrive(&sm.iq_empty[s][slot]);
    if (e[0] < 0) break;
    ItemInfo it;
    UnitInfo un;
    if (!load_unit(p, e, it, un) || it.ntiles == 0) continue;
    const int n = it.ntiles;
    const bool cont = un.k > 0;  // O starts from the item's accumulator (loaded by the softmax)
    if (INDEXED && it.q_src) {  // Q gathered by index by the producer warp
      if (!mbar_wait(&sm.qg_full[s], qg_use & 1, abort)) return;
      ++qg_use;
    } else {
      if (!mbar_wait(&sm.q_full[s], q_use & 1, abort)) return;
      ++q_use;
    }
    if (!mbar_wait(&sm.k_full[s], k_use & 1, abort)) return;
    if (!issue_lock(&sm.issue_lock, abort)) return;
    qk(n == 1);
    issue_unlock(&sm.issue_lock);
    for (int j = 0; j < n; ++j) {
      if (j == 0 && done > 0 && !mbar_wait(&sm.o_free[s], (done - 1) & 1, abort)) return;
      if (!mbar_wait(&sm.v_full[s], v_use & 1, abort)) return;
      if (!mbar_wait(&sm.p_full[s], v_use & 1, abort)) return;
      if (j + 1 < n && !mbar_wait(&sm.k_full[s], k_use & 1, abort)) return;
      if (!issue_lock(&sm.issue_lock, abort)) return;
      tc_fence_after();
      {  // O_s += P_s V_j
        uint32_t v_addr = smem_addr(sm.v[s]);
        asm volatile("" : "+r"(v_addr));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // 16 keys per step: 8 TMEM columns of P, 2 KB of V
          umma_ts(s_col + TM_OOFF, s_col + 8 * kk, smem_desc_sw128(v_addr + kk * 2048, ATOM_BYTES, 1024), IDESC_PV,
                  (cont || j > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&sm.v_empty[s]);
      ++v_use;
      if (j + 1 < n) qk(j + 2 == n);  // S_s = Q_s K_{j+1}^T
      issue_unlock(&sm.issue_lock);
    }
    umma_commit(&sm.o_full[s]);
    ++done;
  }
}

// INDEXED: the index-based prefill (Q rows of permuted classes gathered by row index, output
// rows written at their original positions), compiled separately so that the other path keeps
// its code unchanged.
template <bool INDEXED>
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
    sm.issue_lock = 0;
    for (int s = 0; s < N_STREAMS; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.q_empty[s], 1);
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
      mbar_init(&sm.qg_full[s], 1);
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 128);
      mbar_init(&sm.o_full[s], 1);
      mbar_init(&sm.o_free[s], 128);
      mbar_init(&sm.drain[s], 1);
      for (int i = 0; i < IQ_DEPTH; ++i) {
        mbar_init(&sm.iq_full[s][i], 1);
        mbar_init(&sm.iq_empty[s][i], IQ_READERS);
      }
      mbar_init(&sm.acc_in[s], 1);
      mbar_init(&sm.acc_out[s], 128);
    }
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc<TMEM_COLS>(&sm.tmem_base);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp < 4) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_CTRL));
   if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------------ TMA producers
    // Warp 0 loads stream 0, warp 2 stream 1: two independent load sequences each, polled in
    // turn: Q then the K tiles of every item (slot freed by the QK MMA), and the V tiles
    // (slot freed by the PV MMA).  One lane runs the loop; in the index-based instantiation the
    // whole warp runs it in step (lane 0 takes every decision that reads shared state and
    // broadcasts it, and alone issues the copies and arrivals), so that the 32 lanes can gather
    // the query rows of permuted classes.
    if (INDEXED || lane == 0) {
      const bool leader = !INDEXED || lane == 0;
      // lane 0's value of a condition, for every lane of the warp (index-based instantiation)
      auto uni = [&](bool x) -> bool {
        if constexpr (INDEXED) return __shfl_sync(0xFFFFFFFFu, (int)x, 0) != 0;
        return x;
      };
      auto wsync = [&]() {
        if constexpr (INDEXED) __syncwarp();
      };
      const int s = warp >> 1;
      if (leader) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
      }
      const uint32_t* tiles = reinterpret_cast<const uint32_t*>(p.ws + p.lay.tiles);
      // Work items come from the global counter in plan order (most keys first), one at a
      // time into the stream's queue: the Q/K loads take them as they come, the V loads
      // follow the same sequence from the queue.
      uint32_t published = 0;
      bool ended = false;
      auto publish = [&]() -> bool {
        const uint32_t slot = published % IQ_DEPTH, use = published / IQ_DEPTH;
        if (ended || uni(use > 0 && !mbar_test(&sm.iq_empty[s][slot], (use - 1) & 1))) return false;
        int32_t e0 = -1;
        if (leader) {
          const int id = (int)atomicAdd(p.next_item, 1u);
          int32_t e[4] = {-1, 0, -1, -1};
          if (id < p.n_units) unit_entry(p, id, e);
          e0 = e[0];
          sm.iq[s][slot][0] = e[0];
          sm.iq[s][slot][1] = e[1];
          sm.iq[s][slot][2] = e[2];
          sm.iq[s][slot][3] = e[3];
          mbar_arrive(&sm.iq_full[s][slot]);
        }
        if constexpr (INDEXED) {
          __syncwarp();  // the entry is visible to the whole warp
          e0 = sm.iq[s][slot][0];
        }
        ended = e0 < 0;
        ++published;
        return true;
      };
      uint32_t qk_q = 0, v_q = 0;  // queue positions of the items the two load sequences are on
      int qk_op = -1, v_j = -1;    // -1: no item yet
      ItemInfo qk_it, v_it;
      bool qk_live = true, v_live = true;
      uint32_t q_iss = 0, qt_iss = 0, k_iss = 0, v_iss = 0;  // qt_iss: Q tiles loaded by TMA
      Watchdog wd;
      while (qk_live || v_live) {
        if (qk_live && qk_op < 0) {  // next item of the Q/K loads
          if (published <= qk_q && publish()) wd.progress();
          if (published > qk_q) {
            const int32_t* e = sm.iq[s][qk_q % IQ_DEPTH];
            UnitInfo un;
            if (e[0] < 0) qk_live = false;
            else if (!load_unit(p, e, qk_it, un) || qk_it.ntiles == 0) ++qk_q;
            else qk_op = 0;
          }
        }
        if (qk_live && qk_op >= 0) {
          if (qk_op == 0) {
            // the slot is free once the stream's previous item's last QK is complete
            // (q_empty completes once per item)
            if (uni(q_iss == 0 || mbar_test(&sm.q_empty[s], (q_iss - 1) & 1))) {
              if (INDEXED && qk_it.q_src) {
                // the item's query rows from the caller's Q by row index (zeros past the class)
                // into the 128-byte-swizzled layout the MMA reads: 16-byte chunk c of row r at
                // chunk c ^ (r & 7); half-warp per row, 64 copies per lane
                const ClassStatic& cs = class_of(p, qk_it.cls);
                const int32_t* rows = reinterpret_cast<const int32_t*>(p.ws + cs.rows_off);
                const uint32_t qs = smem_addr(sm.q[s]);
                const int ch = lane & 15, a = ch >> 3, c = ch & 7;
#pragma unroll 2
                for (int r = lane >> 4; r < TILE; r += 2) {
                  const int cr = qk_it.row0 + r;
                  const bool valid = cr < qk_it.nrows;
                  const int pos = valid ? __ldg(rows + cr) : 0;
                  const __nv_bfloat16* src = p.qg + (size_t)qk_it.head * p.qg_head + (size_t)pos * p.qg_row + a * 64 + c * 8;
                  cp_async16_zfill(qs + a * ATOM_BYTES + (uint32_t)r * 128u + ((uint32_t)(c ^ (r & 7)) << 4), src,
                                   valid ? 16u : 0u);
                }
                cp_async_wait_all();
                fence_proxy_async_smem();
                wsync();
                if (leader) mbar_arrive(&sm.qg_full[s]);
              } else {
                if (leader) {
                  mbar_arrive_expect_tx(&sm.q_full[s], TILE_BYTES);
                  if (qk_it.q_src) {
                    tma_load_3d(sm.q[s], &tmQp, &sm.q_full[s], 0, qk_it.qrow0 + qk_it.row0, qk_it.q_slice);
                    tma_load_3d(sm.q[s] + ATOM_BYTES, &tmQp, &sm.q_full[s], 64, qk_it.qrow0 + qk_it.row0,
                                qk_it.q_slice);
                  } else {
                    tma_load_3d(sm.q[s], &tmQ, &sm.q_full[s], 0, qk_it.row0, qk_it.head);
                    tma_load_3d(sm.q[s] + ATOM_BYTES, &tmQ, &sm.q_full[s], 64, qk_it.row0, qk_it.head);
                  }
                }
                ++qt_iss;
              }
              ++q_iss;
              qk_op = 1;
              wd.progress();
            }
          } else if (uni(k_iss == 0 || mbar_test(&sm.k_empty[s], (k_iss - 1) & 1))) {
            const int j = qk_op - 1;
            if (leader)
              issue_kv(&tmK, &tmV, &tmK2, &tmV2, &tmXK, &tmXV, false, __ldg(tiles + qk_it.tile0 + j), qk_it, sm.k[s],
                       &sm.k_full[s]);
            ++k_iss;
            wd.progress();
            if (j + 1 == qk_it.ntiles) {
              ++qk_q;
              qk_op = -1;
            } else {
              qk_op = j + 2;
            }
          }
        }
        if (v_live && v_j < 0 && published > v_q) {  // next item of the V loads
          const uint32_t slot = v_q % IQ_DEPTH;
          const int32_t* e = sm.iq[s][slot];
          UnitInfo un;
          if (e[0] < 0) {
            if (leader) mbar_arrive(&sm.iq_empty[s][slot]);
            v_live = false;
          } else if (!load_unit(p, e, v_it, un) || v_it.ntiles == 0) {
            if (leader) mbar_arrive(&sm.iq_empty[s][slot]);
            ++v_q;
          } else {
            v_j = 0;
          }
        }
        if (v_live && v_j >= 0 && uni(v_iss == 0 || mbar_test(&sm.v_empty[s], (v_iss - 1) & 1))) {
          if (leader)
            issue_kv(&tmK, &tmV, &tmK2, &tmV2, &tmXK, &tmXV, true, __ldg(tiles + v_it.tile0 + v_j), v_it, sm.v[s],
                     &sm.v_full[s]);
          ++v_iss;
          wd.progress();
          if (++v_j == v_it.ntiles) {
            if (leader) mbar_arrive(&sm.iq_empty[s][v_q % IQ_DEPTH]);
            ++v_q;
            v_j = -1;
          }
        }
        if (uni(wd.expired(abort))) {
          // let the copies already issued land before the CTA goes away: these waits ignore the
          // CTA's abort flag (which is set by now) and give up only after their own limit
          if (leader) {
            int drain_flag = 0;
            if (qt_iss) mbar_wait(&sm.q_full[s], (qt_iss - 1) & 1, &drain_flag, 100000000ull);
            if (k_iss) mbar_wait(&sm.k_full[s], (k_iss - 1) & 1, &drain_flag, 100000000ull);
            if (v_iss) mbar_wait(&sm.v_full[s], (v_iss - 1) & 1, &drain_flag, 100000000ull);
          }
          wsync();
          break;
        }
      }
    }
   } else {
    // ------------------------------------------------------------------ MMA issuers
    // warp 1: stream 0, warp 3: stream 1
    if (lane == 0) {
      mma_stream<INDEXED>(p, sm, tmem, warp >> 1, abort);
      // wait for every MMA issued by this thread before the tensor memory is released; the wait
      // ignores the CTA's abort flag (MMAs in flight must finish even after a timeout elsewhere)
      // and gives up only after its own limit
      umma_commit(&sm.drain[warp >> 1]);
      int drain_flag = 0;
      mbar_wait(&sm.drain[warp >> 1], 0, &drain_flag, 100000000ull);
    }
   }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REG_SOFTMAX));
    // ------------------------------------------------------------------ softmax / epilogue
    const int s = (warp - 4) >> 2;         // warps 4-7: stream 0, warps 8-11: stream 1
    const int t = (warp & 3) * 32 + lane;  // a warp may only touch TMEM lanes 32 (warp % 4) .. + 31
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16) + TM_STREAM * s;
    const uint32_t s_own = lane_base, o_own = lane_base + TM_OOFF;
    __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(const_cast<uint8_t*>(p.ws + p.lay.op));
    const uint32_t* tiles = reinterpret_cast<const uint32_t*>(p.ws + p.lay.tiles);
    uint32_t s_count = 0, items_done = 0, acc_ins = 0, acc_outs = 0;
    int bands_known0 = 0, bands_known1 = 1;  // unit bands of each parity known finished below these
    bool ok = true;
    for (uint32_t qi = 0; ok; ++qi) {
      const uint32_t slot = qi % IQ_DEPTH;
      if (!mbar_wait(&sm.iq_full[s][slot], (qi / IQ_DEPTH) & 1, abort)) break;
      const int32_t e[4] = {sm.iq[s][slot][0], sm.iq[s][slot][1], sm.iq[s][slot][2], sm.iq[s][slot][3]};
      mbar_arrive(&sm.iq_empty[s][slot]);
      if (e[0] < 0) break;
      ItemInfo it;
      UnitInfo un;
      // units that skip their work touch no accumulator slot: counted finished at once
      if (!load_unit(p, e, it, un)) { if (t == 0) band_unit_done(p, un); continue; }
      if (un.total > 0 && it.ntiles == 0) { if (t == 0) band_unit_done(p, un); continue; }  // no keys in this chunk
      if (un.total == 0 && un.chunk != 0) { if (t == 0) band_unit_done(p, un); continue; }  // written once
      const ClassStatic& cs = class_of(p, it.cls);
      const int r = it.row0 + t;
      RowCtx& rc = sm.rctx[threadIdx.x - 128];
      fill_row_ctx(p, it, cs, t, rc);
      const size_t orow = ((size_t)it.head * p.LP + it.qrow0 + r) * D;

      // the unit's output row: the caller's O at the original position (index-based), or the
      // permuted O copy
      auto out_row = [&]() -> uint4* {
        return reinterpret_cast<uint4*>(INDEXED ? p.od + (size_t)it.head * p.od_head + (size_t)rc.qpos * p.od_row
                                                : op + orow);
      };
      if (it.ntiles == 0) {
        if (rc.valid) {
          uint4* dst = out_row();
#pragma unroll
          for (int i = 0; i < 16; ++i) dst[i] = make_uint4(0, 0, 0, 0);
          if (p.lse) p.lse[(size_t)it.head * p.L + rc.qpos] = -INFINITY;
        }
        if (t == 0) band_unit_done(p, un);
        continue;
      }

      float m_used = -INFINITY, l = 0.f;
      // A unit after the item's first key chunk resumes from the item's accumulator: the
      // previous chunk's unit releases it (chunk_done) once every row is stored.
      const bool cont = un.k > 0;
      float* arow = p.acc ? p.acc + ((int64_t)un.acc * TILE + t) * ACC_ROW : nullptr;
      if (cont) {
        if (t == 0) {
          const uint64_t t0 = global_ns();
          while (ld_acquire(p.chunk_done + un.item) < (uint32_t)un.k) {
            if (*abort || global_ns() - t0 > 1000000000ull) {
              *abort = 1;
              break;
            }
          }
          mbar_arrive(&sm.acc_in[s]);
        }
        if (!mbar_wait(&sm.acc_in[s], acc_ins & 1, abort)) { ok = false; break; }
        ++acc_ins;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t oa[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(arow + 32 * c + 4 * j));
            oa[4 * j] = __float_as_uint(v.x);
            oa[4 * j + 1] = __float_as_uint(v.y);
            oa[4 * j + 2] = __float_as_uint(v.z);
            oa[4 * j + 3] = __float_as_uint(v.w);
          }
          tmem_st32(o_own + 32 * c, oa);
        }
        m_used = __ldcg(arow + D);
        l = __ldcg(arow + D + 1);
        tmem_wait_st();
      }
      // The element mask of a tile is built before its S is waited for (for the first tile
      // here, for the others right after the previous tile's P is handed over), so that the
      // bitmap loads and the bit arithmetic overlap the tensor core's work.  Tiles flagged full
      // need no mask (the flag is the same for the whole warp).
      uint32_t mk[4];
      bool full;
      auto build_mask = [&](uint32_t t) {
        full = (t & TILE_FULL) != 0u;
        if (!full) {
          MaskRaw raw;
          mask_prefetch(rc, t, raw);
          mask_finish(rc, raw, mk);
        }
      };
      build_mask(__ldg(tiles + it.tile0));
      for (int tt = 0; tt < it.ntiles; ++tt) {
        const uint32_t tile_next = (tt + 1 < it.ntiles) ? __ldg(tiles + it.tile0 + tt + 1) : 0u;
        if (!mbar_wait(&sm.s_full[s], s_count & 1, abort)) { ok = false; break; }
        ++s_count;
        tc_fence_after();
        float sv[128];
        {  // the whole S row in one load (measured faster than four 32-column loads)
          uint32_t rr[128];
          tmem_ld128(s_own, rr);
#pragma unroll
          for (int j = 0; j < 128; ++j) sv[j] = __uint_as_float(rr[j]);
        }
        if (!full) {
          tmem_wait_ld();
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            if (__all_sync(0xFFFFFFFFu, mk[w] == 0xFFFFFFFFu)) continue;  // word open for the whole warp
#pragma unroll
            for (int c = 32 * w; c < 32 * w + 32; ++c) sv[c] = ((mk[w] >> (c & 31)) & 1u) ? sv[c] : -INFINITY;
          }
        } else {
          tmem_wait_ld();
        }
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
#pragma unroll
          for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], sv[c + 2 * q], sv[c + 2 * q + 1]);
        }
        const float mxs = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * p.scale_log2;
        float alpha = 1.f;
        bool resc = false;
        if (mxs > m_used + 8.f) {  // also true on the first finite max
          alpha = (m_used == -INFINITY) ? 0.f : ex2(m_used - mxs);
          m_used = mxs;
          resc = true;
        }
        // S_s(tt) complete implies the previous P V of this stream is complete (same issuer,
        // issue order), so O_s may be rescaled here
        if ((tt > 0 || cont) && __any_sync(0xFFFFFFFFu, resc)) {
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
        }
        const float nb = (m_used == -INFINITY) ? 0.f : -m_used;
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nb2 = make_float2(nb, nb);
        float2 rs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        // P row t over S columns [0, 64): column c holds keys 2c (low half) and 2c + 1.
        // Exponent arguments and the row sum use the packed two-lane fp32 FMA / add.
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float2 x = __ffma2_rn(make_float2(sv[32 * h + 2 * c], sv[32 * h + 2 * c + 1]), sc2, nb2);
            const float2 e = make_float2(ex2(x.x), ex2(x.y));
            rs2[c & 1] = __fadd2_rn(rs2[c & 1], e);
            pk[c] = pack_bf16x2(e.x, e.y);
          }
          tmem_st16(s_own + 16 * h, pk);
        }
        l = l * alpha + ((rs2[0].x + rs2[1].x) + (rs2[0].y + rs2[1].y));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sm.p_full[s]);
        if (tt + 1 < it.ntiles) build_mask(tile_next);
      }
      if (!ok) break;
      // epilogue: the unit's last P V done, then O = O_s / l, or the state into the accumulator
      if (!mbar_wait(&sm.o_full[s], items_done & 1, abort)) { ok = false; break; }
      ++items_done;
      tc_fence_after();
      if (!un.last) {
        // the item's first write to its slot: the earlier bands that used the slot must be done
        // (each thread takes the counters with acquire itself; a continued item's slot was
        // claimed by its first unit, in the same band)
        if (!cont && !band_wait_previous(p, un, bands_known0, bands_known1, abort)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t oa[32];
          tmem_ld32(o_own + 32 * c, oa);
          tmem_wait_ld();
          if (c == 3) {
            tc_fence_before();
            mbar_arrive(&sm.o_free[s]);
          }
#pragma unroll
          for (int j = 0; j < 8; ++j)
            __stcg(reinterpret_cast<float4*>(arow + 32 * c + 4 * j),
                   make_float4(__uint_as_float(oa[4 * j]), __uint_as_float(oa[4 * j + 1]),
                               __uint_as_float(oa[4 * j + 2]), __uint_as_float(oa[4 * j + 3])));
        }
        __stcg(arow + D, m_used);
        __stcg(arow + D + 1, l);
        __threadfence();
        mbar_arrive(&sm.acc_out[s]);
        if (t == 0) {
          if (!mbar_wait(&sm.acc_out[s], acc_outs & 1, abort)) { ok = false; break; }
          __threadfence();
          st_release(p.chunk_done + un.item, (uint32_t)un.k + 1u);
          band_unit_done(p, un);
        }
        ++acc_outs;
        continue;
      }
      // the item's last unit: its slot was read (when continued) before its first P was handed
      // to the tensor core, and this thread has seen the last P V of the unit, which needed
      // every row's P: the slot is free
      if (t == 0) band_unit_done(p, un);
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint4* dst = out_row();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t oa[32];
        tmem_ld32(o_own + 32 * c, oa);
        tmem_wait_ld();
        if (c == 3) {
          tc_fence_before();
          mbar_arrive(&sm.o_free[s]);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k = 8 * j + 2 * e;
            w[e] = pack_bf16x2(__uint_as_float(oa[k]) * inv, __uint_as_float(oa[k + 1]) * inv);
          }
          if (rc.valid) dst[4 * c + j] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      if (rc.valid && p.lse)
        p.lse[(size_t)it.head * p.L + rc.qpos] = (l > 0.f) ? (m_used + __log2f(l)) * 0.6931471805599453f : -INFINITY;
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

// Allowed (query, key) pairs of every head: the attention kernel's element mask evaluated over
// each work item's whole tile list (one thread per query row), full tiles counted as 128 per
// valid row, summed per head.  Keys that a gathered tile serves are excluded from the identity
// tiles, so every pair is counted once.
__global__ void __launch_bounds__(TILE) mask_count_kernel(const AttnParams p, unsigned long long* counts) {
  const uint32_t* tiles = reinterpret_cast<const uint32_t*>(p.ws + p.lay.tiles);
  for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
    ItemInfo it;
    if (!load_item(p, item, it)) continue;
    RowCtx rc;
    fill_row_ctx(p, it, class_of(p, it.cls), threadIdx.x, rc);
    unsigned long long n = 0;
    for (int tt = 0; tt < it.ntiles; ++tt) {
      const uint32_t tile = __ldg(tiles + it.tile0 + tt);
      if (tile & TILE_FULL) {
        n += rc.valid ? TILE : 0;
        continue;
      }
      MaskRaw raw;
      uint32_t mk[4];
      mask_prefetch(rc, tile, raw);
      mask_finish(rc, raw, mk);
      n += __popc(mk[0]) + __popc(mk[1]) + __popc(mk[2]) + __popc(mk[3]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n += __shfl_down_sync(0xFFFFFFFFu, n, o);
    if ((threadIdx.x & 31) == 0 && n) atomicAdd(counts + it.head, n);
  }
}

}  // namespace

cudaError_t launch_mask_count(const DevPlan& dp, cudaStream_t st) {
  AttnParams p{};
  p.ws = dp.ws;
  p.lay = dp.lay;
  p.L = (int32_t)dp.L;
  p.Hq = dp.Hq;
  p.Hkv = dp.Hkv;
  p.LP = dp.LP;
  p.n_items = dp.n_items;
  auto* counts = reinterpret_cast<unsigned long long*>(const_cast<uint8_t*>(dp.ws + dp.lay.mask_pairs));
  if (cudaError_t e = cudaMemsetAsync(counts, 0, 8 * (size_t)dp.Hq, st)) return e;
  if (dp.n_items == 0) return cudaSuccess;
  const int grid = std::max(1, std::min(dp.n_items, sm_count() * 8));
  count_launches(1);
  mask_count_kernel<<<grid, TILE, 0, st>>>(p, counts);
  return cudaGetLastError();
}

cudaError_t launch_attention(const DevPlan& dp, const void* Q, const void* K, const void* V, const msa_strides& s,
                             float* lse, void* O, cudaStream_t st) {
  CUtensorMap mq, mqp, mk, mv, mk2, mv2, mxk, mxv;
  const uint8_t* ws = dp.ws;
  bool ok = make_map(&mq, Q, dp.L, dp.Hq, s.q_row, s.q_head) && make_map(&mk, K, dp.L, dp.Hkv, s.k_row, s.k_head) &&
            make_map(&mv, V, dp.L, dp.Hkv, s.v_row, s.v_head) &&
            (O ? make_map(&mqp, Q, dp.L, dp.Hq, s.q_row, s.q_head)  // unused: Q rows are gathered
               : make_map(&mqp, ws + dp.lay.qp, dp.LP, std::max(dp.n_qslices, 1), D, (int64_t)dp.LP * D)) &&
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
  // work items are handed out by a counter in the workspace header, zeroed here
  p.next_item = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(ws + dp.lay.header)) + HDR_NEXT_ITEM;
  if (cudaError_t e = cudaMemsetAsync(p.next_item, 0, sizeof(uint32_t), st)) return e;
  p.n_units = dp.n_units;
  p.n_kchunks = dp.n_kchunks;
  p.n_bands = dp.n_bands;
  p.chunk_done = nullptr;
  p.band_done = nullptr;
  p.acc = nullptr;
  p.qg = static_cast<const __nv_bfloat16*>(Q);
  p.qg_head = s.q_head;
  p.qg_row = s.q_row;
  p.od = static_cast<__nv_bfloat16*>(O);
  p.od_head = s.o_head;
  p.od_row = s.o_row;
  if (dp.n_kchunks > 1) {
    p.chunk_done = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(ws + dp.lay.chunk_done));
    p.band_done = p.chunk_done + dp.n_items;
    p.acc = reinterpret_cast<float*>(const_cast<uint8_t*>(ws + dp.lay.acc));
    if (cudaError_t e = cudaMemsetAsync(p.chunk_done, 0, sizeof(uint32_t) * ((size_t)dp.n_items + (size_t)dp.n_bands), st))
      return e;
  }
  const size_t smem = sizeof(AttnSmem);
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev)) return e;
  if (device_pending(configured, dev)) {
    cudaError_t e = cudaFuncSetAttribute(msa_attn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(msa_attn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    mark_device(configured, dev);
  }
  const int grid = std::max(1, std::min((dp.n_units + N_STREAMS - 1) / N_STREAMS, sm_count()));
  count_launches(1);
  if (O)
    msa_attn_kernel<true><<<grid, ATT_THREADS, smem, st>>>(mq, mqp, mk, mv, mk2, mv2, mxk, mxv, p);
  else
    msa_attn_kernel<false><<<grid, ATT_THREADS, smem, st>>>(mq, mqp, mk, mv, mk2, mv2, mxk, mxv, p);
  return cudaGetLastError();
}

}  // namespace msa
