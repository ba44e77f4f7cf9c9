// Last-query sweep of the online index estimation on the tensor cores (MInference 1.0 page,
// "Approach": the vertical and slash lines of a head come from the attention of its final 64
// queries; MMInference review page, "core discovery": video-aware heads take those 64 queries
// per modality, and "key machinery": 2D-boundary heads measure slash lines in within-modality
// coordinates).
//
// For each row set R (<= 64 estimation queries of one head, with row positions i_r and slash
// coordinates rc_r) the causal softmax A[r, j] = exp(x_rj - m_r) / Z_r of the logits
// x_rj = q_r . k_j * scale over the keys j <= i_r is reduced to
//   v[j] = sum_r A[r, j]                 (vertical sums, by key)
//   s[o] = sum_r A[r, j] with rc_r - kc_j = o, kc_j the key's slash coordinate   (slash sums)
// in two passes over K: pass 1 finds each row's max and normaliser per key chunk (combined in
// chunk order afterwards), pass 2 forms the probabilities and sums them.
//
// Design for sm_100a: two row sets of one KV head and key source form the 128 rows of one
// tile (LqTile), so K is streamed once for both; one CTA per (tile, key chunk).  A producer
// warp streams 64-key blocks of K with TMA (128-byte swizzle, no multicast) into a ring of
// stages; one thread issues tcgen05.mma (M = 128 query rows, N = 64 keys, K = 128, bf16 in,
// fp32 accumulate) into one of two S buffers in tensor memory; four softmax warps, one thread
// per query row, read their row of S with tcgen05.ld and do the per-element work in fp32
// (exp2 on MUFU).  Pass 2 stages each block's probabilities in shared memory (row pitch 65
// words: the row-wise writes, the column sums and the diagonal sums are all free of bank
// conflicts) and reduces columns (vertical) and diagonals (slash) with one thread per column
// / diagonal pair of its row set, in a fixed order, so results are deterministic.  A chunk
// owns the vertical sums of its keys and the slash sums of the offsets whose last-row key lies
// in it; it re-reads the `span` keys below it to complete those offsets, and carries partial
// slash sums from block to block in a small ring indexed by offset.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "kernels.h"
#include "msa_internal.h"
#include "ptx.cuh"

namespace msa {

namespace {

template <typename T>
__host__ __device__ __forceinline__ T* at(const DevPlan& dp, int64_t off) {
  return reinterpret_cast<T*>(dp.ws + off);
}

constexpr float LOG2E = 1.4426950408889634f;
constexpr int LQ_KB = 64;                       // keys per block (MMA N)
constexpr int LQ_THREADS = 320;                 // warp 0 TMA, warp 1 MMA, warps 2-9 softmax
constexpr int LQ_SOFTMAX = 256;                 // softmax threads: two per query row
constexpr uint32_t Q_ATOM = 128 * 128;          // [128 rows][64 cols] bf16, 128-byte swizzled
constexpr uint32_t K_ATOM = LQ_KB * 128;        // [64 rows][64 cols]
constexpr uint32_t K_STAGE = 2 * K_ATOM;        // one 64-key block, all 128 columns
constexpr int P_PITCH = LQ_KB + 1;              // staged probabilities: row pitch in words
constexpr int TM_COLS = 2 * LQ_KB;              // two S buffers of 64 fp32 columns
constexpr uint32_t IDESC = idesc_bf16_f32(128, LQ_KB, 0, 0);
constexpr int LQ_RING_MAX = 8192;               // row sets span at most 4096 coordinates

// K stages: pass 1 fits two CTAs per SM with four, pass 2 (which adds 35 KB of staging) with two
template <int PASS>
struct LqShape {
  static constexpr int STAGES = PASS == 1 ? 4 : 2;
};

// Shared memory of one CTA.  The tiles come first (1024-byte aligned for the swizzle); pass 2
// adds the staged probabilities and the slash rings (sized at launch) after the barriers.
template <int PASS>
struct __align__(1024) LqtSmem {
  uint8_t q[2 * Q_ATOM];
  uint8_t k[LqShape<PASS>::STAGES][K_STAGE];
  uint64_t k_full[LqShape<PASS>::STAGES], k_empty[LqShape<PASS>::STAGES];
  uint64_t s_full[2], s_free[2], q_ready, drain;
  uint32_t tmem_base;
  int abort;
};

// tcgen05.wait::ld with the loaded registers as operands, so that no use of them can be
// scheduled before the wait
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
        "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
        "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}

__device__ __forceinline__ float lq_fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Barrier of the 128 softmax threads of one row set (named barriers 1 and 2).
__device__ __forceinline__ void set_sync(int set) {
  if (set == 0) asm volatile("bar.sync 1, 128;" ::: "memory");
  else asm volatile("bar.sync 2, 128;" ::: "memory");
}

// The tile's key range processed by chunk `chunk`: keys [c0, c1), of which the chunk owns
// [own0, own1); c0 reaches `span64` keys below the chunk so that the slash offsets whose
// last-row key lies in the chunk are complete.  Block boundaries are multiples of 64 from c0.
struct ChunkKeys {
  int64_t own0, own1, c0, c1;
};

__device__ __forceinline__ ChunkKeys chunk_keys(const RowSet& a, const RowSet* b, int chunk, bool pass2) {
  ChunkKeys k;
  k.own0 = (int64_t)chunk * a.chunk;
  const int64_t hi = b ? max(a.key_hi, b->key_hi) : a.key_hi;
  k.own1 = min(k.own0 + (int64_t)a.chunk, hi);
  int64_t back = 0;
  if (pass2) {
    if (a.slash_hi > a.slash_lo) back = max(back, (int64_t)((a.span + 63) / 64 * 64));
    if (b && b->slash_hi > b->slash_lo) back = max(back, (int64_t)((b->span + 63) / 64 * 64));
  }
  k.c0 = max((int64_t)0, k.own0 - back);
  k.c1 = k.own1;
  return k;
}

}  // namespace

namespace {

// Pass-2 additions to the shared memory, placed after LqtSmem: staged probabilities of each
// row set's block, its rows' slash coordinates, and its slash ring (ring entries per set at
// launch).
struct LqtSmem2 {
  float p[2][64 * P_PITCH];   // probabilities of row sets with non-consecutive coordinates
  int32_t rcs[2][64];
  float vst[2][2][2][64];     // [block parity][set][row half][column]: column sums of a half
  float dst[2][2][4][64];     // [block parity][set][quarter][diagonal + 32]: diagonal sums
};

// Butterfly reduce-scatter over the 32 lanes of a warp: lane l returns the sum over all lanes of
// v[l], that is column l of the warp's 32 x 32 block (lane = row) summed over its rows, in a
// fixed order.  Each step keeps the half of the columns named by one lane bit and adds the
// partner lane's copy of it.
__device__ __forceinline__ float warp_column_sums(const float (&v)[32], int lane) {
  constexpr unsigned F = 0xFFFFFFFFu;
  float a[16], b[8], c[4], d[2];
  const bool u16 = lane & 16, u8 = lane & 8, u4 = lane & 4, u2 = lane & 2, u1 = lane & 1;
#pragma unroll
  for (int i = 0; i < 16; ++i) a[i] = (u16 ? v[i + 16] : v[i]) + __shfl_xor_sync(F, u16 ? v[i] : v[i + 16], 16);
#pragma unroll
  for (int i = 0; i < 8; ++i) b[i] = (u8 ? a[i + 8] : a[i]) + __shfl_xor_sync(F, u8 ? a[i] : a[i + 8], 8);
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = (u4 ? b[i + 4] : b[i]) + __shfl_xor_sync(F, u4 ? b[i] : b[i + 4], 4);
#pragma unroll
  for (int i = 0; i < 2; ++i) d[i] = (u2 ? c[i + 2] : c[i]) + __shfl_xor_sync(F, u2 ? c[i] : c[i + 2], 2);
  return (u1 ? d[1] : d[0]) + __shfl_xor_sync(F, u1 ? d[0] : d[1], 1);
}

// Diagonal sums of the warp's 32 x 32 block (lane = row r, register c = column): lane l returns
// the sum along r - c = l in `hi` and along r - c = l - 32 in `lo` (empty for lane 0).  Step c
// reads column c of row (l + c) mod 32, so every lane collects its diagonals in registers.
__device__ __forceinline__ void warp_diagonal_sums(const float (&v)[32], int lane, float& hi, float& lo) {
  float h0 = 0.f, h1 = 0.f, l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const float x = __shfl_sync(0xFFFFFFFFu, v[c], (lane + c) & 31);
    if (lane + c < 32) {
      if (c & 1) h1 += x;
      else h0 += x;
    } else {
      if (c & 1) l1 += x;
      else l0 += x;
    }
  }
  hi = h0 + h1;
  lo = l0 + l1;
}

// bar.red.or over the 128 threads of one row set: true if any of them passes true.
template <int ID>
__device__ __forceinline__ bool bar_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(ID)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool set_any(int set, bool v) { return set == 0 ? bar_any<1>(v) : bar_any<2>(v); }

template <int PASS>
__global__ void __launch_bounds__(LQ_THREADS, 2)
    lastq_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmK2, const DevPlan dp,
             const __nv_bfloat16* __restrict__ Q, int64_t qh, int64_t qr) {
  using Smem = LqtSmem<PASS>;
  constexpr int ST = LqShape<PASS>::STAGES;
  extern __shared__ __align__(1024) uint8_t lq_smem[];
  Smem& sm = *reinterpret_cast<Smem*>(lq_smem);
  uint32_t* err = at<uint32_t>(dp, dp.lay.header);
  if (smem_addr(lq_smem) & 1023u) {  // the swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicOr(err, DEV_ERR_BOUNDS);
    return;
  }
  const LqTile tile = at<const LqTile>(dp, dp.lay.lq_tiles)[blockIdx.y];
  const int chunk = blockIdx.x;
  if (chunk >= tile.n_chunks) return;
  const RowSet* rsets = at<const RowSet>(dp, dp.lay.rowsets);
  const RowSet& ra = rsets[tile.rs[0]];
  const RowSet* rb = tile.rs[1] >= 0 ? &rsets[tile.rs[1]] : nullptr;
  const ChunkKeys ck = chunk_keys(ra, rb, chunk, PASS == 2);
  const int nblk = (int)((ck.c1 - ck.c0 + LQ_KB - 1) / LQ_KB);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &sm.abort;

  if (threadIdx.x == 0) {
    sm.abort = 0;
    for (int s = 0; s < ST; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.s_free[b], LQ_SOFTMAX);
    }
    mbar_init(&sm.q_ready, LQ_SOFTMAX);
    mbar_init(&sm.drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc<TM_COLS>(&sm.tmem_base);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && nblk > 0) {
      const CUtensorMap* m = tile.k_src == SRC_K2D ? &tmK2 : &tmK;
      tma_prefetch_desc(m);
      int issued = 0;
      for (int b = 0; b < nblk; ++b) {
        const int st = b % ST;
        if (b >= ST && !mbar_wait(&sm.k_empty[st], ((b / ST) - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&sm.k_full[st], K_STAGE);
        const int row = (int)(ck.c0 + (int64_t)b * LQ_KB);
        tma_load_3d(sm.k[st], m, &sm.k_full[st], 0, row, tile.kvh);
        tma_load_3d(sm.k[st] + K_ATOM, m, &sm.k_full[st], 64, row, tile.kvh);
        issued = b + 1;
      }
      // the copies still in flight land before the CTA goes away (own limit; ignores abort)
      int drain_flag = 0;
      for (int b = max(0, issued - ST); b < issued; ++b)
        mbar_wait(&sm.k_full[b % ST], (b / ST) & 1, &drain_flag, 100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      if (nblk > 0 && mbar_wait(&sm.q_ready, 0, abort)) {
        const uint32_t qa = smem_addr(sm.q);
        for (int b = 0; b < nblk; ++b) {
          const int st = b % ST, buf = b & 1;
          if (!mbar_wait(&sm.k_full[st], (b / ST) & 1, abort)) break;
          if (b >= 2 && !mbar_wait(&sm.s_free[buf], ((b >> 1) - 1) & 1, abort)) break;
          tc_fence_after();
          const uint32_t ka = smem_addr(sm.k[st]);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tmem + (uint32_t)(buf * LQ_KB), smem_desc_sw128(qa + (kk >> 2) * Q_ATOM + (kk & 3) * 32, 16, 1024),
                    smem_desc_sw128(ka + (kk >> 2) * K_ATOM + (kk & 3) * 32, 16, 1024), IDESC, kk > 0 ? 1u : 0u);
          umma_commit(&sm.k_empty[st]);
          umma_commit(&sm.s_full[buf]);
        }
      }
      // every MMA issued here completes before the tensor memory is released (own limit)
      umma_commit(&sm.drain);
      int drain_flag = 0;
      mbar_wait(&sm.drain, 0, &drain_flag, 100000000ull);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    // eight warps, two per row: warp w reaches TMEM lanes 32 (w % 4) .. + 31 only, so warps
    // 2-5 take columns 0-31 of their 32 rows and warps 6-9 columns 32-63 of the same rows
    const int qd = warp & 3;
    const int hc = (warp - 2) >> 2;  // column half of this warp
    const int m = qd * 32 + lane;
    const int set = m >> 6, rr = m & 63;
    const int ts = hc * 64 + rr;     // thread of the row set (0 .. 127)
    const RowSet* rs = set == 0 ? &ra : rb;
    const int t256 = threadIdx.x - 64;
    // the tile's 128 query rows into the swizzled Q tile (16-byte copies, zero rows as padding)
    for (int i = t256; i < 128 * 16; i += LQ_SOFTMAX) {
      const int r = i >> 4, c = i & 15;
      const RowSet* s_ = r < 64 ? &ra : rb;
      const int rl = r & 63;
      const bool valid = s_ != nullptr && rl < s_->n_rows;
      const __nv_bfloat16* src = valid ? Q + (int64_t)s_->head * qh + (int64_t)s_->rows[rl] * qr + c * 8 : Q;
      const uint32_t dst = smem_addr(sm.q) + (uint32_t)(c >> 3) * Q_ATOM + (uint32_t)r * 128u +
                           ((uint32_t)((c & 7) ^ (r & 7)) << 4);
      cp_async16_zfill(dst, src, valid ? 16u : 0u);
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    mbar_arrive(&sm.q_ready);

    const bool have = rs != nullptr && rr < rs->n_rows;
    const int32_t pr = have ? rs->rows[rr] : -1;  // a padding row has no causal key
    const float sl2 = dp.scale * LOG2E;
    const bool k2d = tile.k_src == SRC_K2D;
    const int32_t* perm = k2d ? at<const int32_t>(dp, dp.lay.perm2d) : nullptr;
    const uint32_t s_lane = tmem + ((uint32_t)(qd * 32) << 16) + (uint32_t)(32 * hc);

    // the row's 32 logits of block b (this warp's column half) in log2 units, -inf where the key
    // is not causal; key positions: modality-grouped keys through perm2d, else the row itself
    auto load_logits = [&](int b, float (&x)[32]) -> bool {
      const int buf = b & 1;
      const int64_t j0 = ck.c0 + (int64_t)b * LQ_KB + 32 * hc;
      int32_t pos, pmax;
      if (!k2d) {
        pos = (int32_t)(j0 + lane);
        pmax = (int32_t)(j0 + 31);
      } else {
        pos = j0 + lane < dp.L ? __ldg(perm + j0 + lane) : 0x7fffffff;
        pmax = pos;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) pmax = max(pmax, __shfl_xor_sync(0xFFFFFFFFu, pmax, o));
      }
      // the warp decides together (the loads below are warp-collective)
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.s_full[buf], (b >> 1) & 1, abort))) return false;
      tc_fence_after();
      uint32_t sa[32];
      tmem_ld32(s_lane + (uint32_t)(buf * LQ_KB), sa);
      tmem_wait_ld_regs(sa);
      tc_fence_before();
      mbar_arrive(&sm.s_free[buf]);
#pragma unroll
      for (int c = 0; c < 32; ++c) x[c] = __uint_as_float(sa[c]) * sl2;
      if (__any_sync(0xFFFFFFFFu, pmax > pr)) {  // some key of the half is after some row of the warp
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (__shfl_sync(0xFFFFFFFFu, pos, c) > pr) x[c] = -INFINITY;
      }
      return true;
    };

    if constexpr (PASS == 1) {
      float mrun = -INFINITY, z = 0.f;  // over this thread's 32 columns of each block
      for (int b = 0; b < nblk; ++b) {
        float x[32];
        if (!load_logits(b, x)) break;
        // the half-block max in eight independent chains, then the sum of the exponentials in
        // four chains (short dependency chains: the loop is latency-bound)
        float m8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) m8[q] = lq_fmax3(x[q], x[8 + q], fmaxf(x[16 + q], x[24 + q]));
        const float bm = fmaxf(lq_fmax3(m8[0], m8[1], m8[2]), lq_fmax3(m8[3], lq_fmax3(m8[4], m8[5], m8[6]), m8[7]));
        const float nm = fmaxf(mrun, bm);
        if (nm == -INFINITY) continue;
        z = (mrun == -INFINITY) ? 0.f : z * ex2(mrun - nm);
        mrun = nm;
        float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 32; ++c) a[c & 3] += ex2(x[c] - mrun);
        z += (a[0] + a[1]) + (a[2] + a[3]);
      }
      // the two halves of each row: the second half's (max, sum) through shared memory, combined
      // by the first half's thread (columns 0-31 first, then 32-63)
      float* xch = reinterpret_cast<float*>(lq_smem + sizeof(Smem));
      if (hc == 1) {
        xch[2 * m] = mrun;
        xch[2 * m + 1] = z;
      }
      asm volatile("bar.sync 3, %0;" ::"n"(LQ_SOFTMAX) : "memory");
      if (hc == 0) {
        const float m1 = xch[2 * m], z1 = xch[2 * m + 1];
        const float M = fmaxf(mrun, m1);
        float Z = 0.f;
        if (M > -INFINITY) Z = (mrun > -INFINITY ? z * ex2(mrun - M) : 0.f) + (m1 > -INFINITY ? z1 * ex2(m1 - M) : 0.f);
        if (rs != nullptr && chunk < rs->n_chunks) {
          float* mz = at<float>(dp, rs->mz_off) + (int64_t)chunk * LASTQ * 2;
          mz[2 * rr] = M;
          mz[2 * rr + 1] = Z;
        }
      }
    } else {
      LqtSmem2& s2 = *reinterpret_cast<LqtSmem2*>(lq_smem + sizeof(Smem));
      float* ring = reinterpret_cast<float*>(lq_smem + sizeof(Smem) + sizeof(LqtSmem2)) + set * dp.lq_ring;
      const int R = dp.lq_ring;
      float* P = s2.p[set];
      // the row set's slash geometry
      const bool slash = rs != nullptr && rs->slash_hi > rs->slash_lo;
      int32_t min_rc = 0x7fffffff, max_rc = -0x7fffffff;
      bool contig = true;
      if (rs != nullptr) {
        for (int r = 0; r < rs->n_rows; ++r) {
          const int32_t c = rs->rcs[r];
          min_rc = min(min_rc, c);
          max_rc = max(max_rc, c);
          contig = contig && c == rs->rcs[0] + r;
        }
        if (hc == 0) s2.rcs[set][rr] = rr < rs->n_rows ? rs->rcs[rr] : 0;
      }
      for (int i = ts; i < R; i += 128) ring[i] = 0.f;
      const float* st = have ? at<const float>(dp, rs->stat_off) : nullptr;
      const float Mr = have ? st[2 * rr] : -INFINITY, Ir = have ? st[2 * rr + 1] : 0.f;
      const bool live = have && Mr > -INFINITY;
      const int64_t own0 = ck.own0, own1 = rs != nullptr ? min(ck.own0 + (int64_t)ra.chunk, (int64_t)rs->key_hi) : 0;
      float* vout = rs != nullptr ? at<float>(dp, rs->v_off) : nullptr;
      float* sout = slash ? at<float>(dp, rs->s_off) : nullptr;
      const int32_t slo = slash ? rs->slash_lo : 0, shi = slash ? rs->slash_hi : 0;
      const int n_rows = rs != nullptr ? rs->n_rows : 0;
      const int64_t rc0 = rs != nullptr ? rs->rcs[0] : 0;
      const int64_t own_end = ck.own0 + ra.chunk;  // offsets owned: last-row key in [own0, own_end)
      set_sync(set);  // ring and row coordinates in place

      const int rh = rr >> 5;      // row half of the set held by this warp
      const int w4 = rh * 2 + hc;  // the warp's quarter (row half, column half) of the set's block

      for (int b = 0; b < nblk; ++b) {
        const int64_t j0 = ck.c0 + (int64_t)b * LQ_KB;
        const int sb = b & 1;  // staging parity: a block's staging is rewritten two blocks later,
                               // after every thread of the set has passed the barrier between
        float p[32];
        const bool got = load_logits(b, p);
        if (got) {
#pragma unroll
          for (int c = 0; c < 32; ++c) p[c] = live ? ex2(p[c] - Mr) * Ir : 0.f;
          // vertical: column 32 hc + lane of the block summed over the warp's 32 rows
          s2.vst[sb][set][rh][32 * hc + lane] = warp_column_sums(p, lane);
          if (slash) {
            if (!(j0 >= slo && j0 + LQ_KB <= shi)) {  // keys outside the slash range count zero
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                const int64_t j = j0 + 32 * hc + c;
                if (j < slo || j >= shi) p[c] = 0.f;
              }
            }
            if (contig) {
              float hi, lo;
              warp_diagonal_sums(p, lane, hi, lo);
              s2.dst[sb][set][w4][lane + 32] = hi;
              s2.dst[sb][set][w4][lane] = lo;
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c) P[rr * P_PITCH + 32 * hc + c] = p[c];
            }
          }
        }
        if (set_any(set, !got)) break;  // every thread of the set leaves together
        // the set's 128 threads combine the four quarters in a fixed order
        if (ts < 64) {
          const int64_t j = j0 + ts;
          if (vout != nullptr && j >= own0 && j < own1) vout[j] = s2.vst[sb][set][0][ts] + s2.vst[sb][set][1][ts];
        }
        if (slash && contig) {
          // consecutive row coordinates: offset rc0 - j0 + d collects the block's diagonal
          // d = r - c (-63 .. 63), held by quarter (h, c') at d - 32 (h - c'); thread ts takes
          // d = ts - 64, adds it to the ring and writes the offset out once its last-row key is
          // in this block
          const int d = ts - 64;
          float a = 0.f;
          if (d >= -32 && d < 32) a += s2.dst[sb][set][0][d + 32];
          if (d < 0) a += s2.dst[sb][set][1][d + 64];
          if (d >= 0) a += s2.dst[sb][set][2][d];
          if (d >= -32 && d < 32) a += s2.dst[sb][set][3][d + 32];
          const int64_t o = rc0 - j0 + d;
          float& e = ring[o & (R - 1)];
          const float tot = e + a;
          const int64_t kk = (int64_t)max_rc - o - j0;  // the offset's last-row key, from j0
          if (kk >= 0 && kk < LQ_KB) {
            if (j0 + kk >= own0 && j0 + kk < own_end && o >= 0 && o < dp.L) sout[o] = tot;
            e = 0.f;
          } else {
            e = tot;
          }
        } else if (slash) {
          // any row coordinates: one thread per offset touched by the block, rows in order
          const int64_t olo = (int64_t)min_rc - (j0 + LQ_KB - 1), ohi = (int64_t)max_rc - j0;
          for (int64_t o = olo + ts; o <= ohi; o += 128) {
            float a = 0.f;
            for (int r = 0; r < n_rows; ++r) {
              const int64_t c = (int64_t)s2.rcs[set][r] - o - j0;
              if (c >= 0 && c < LQ_KB) a += P[r * P_PITCH + (int)c];
            }
            ring[o & (R - 1)] += a;
          }
          set_sync(set);  // block's sums in the ring; P may be overwritten
          if (ts < 64) {
            // offsets whose last-row key is j0 + ts are complete: written if the chunk owns them
            const int64_t o = (int64_t)max_rc - (j0 + ts);
            float& e = ring[o & (R - 1)];
            if (j0 + ts >= own0 && j0 + ts < own_end && o >= 0 && o < dp.L) sout[o] = e;
            e = 0.f;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && sm.abort) atomicOr(err, DEV_ERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<TM_COLS>(tmem);
  }
}

// Row max / inverse normaliser over the chunks, in chunk order.
__global__ void lastq_combine(DevPlan dp) {
  const RowSet& rs = at<const RowSet>(dp, dp.lay.rowsets)[blockIdx.x];
  const int r = threadIdx.x;
  if (r >= LASTQ) return;
  const float* mz = at<const float>(dp, rs.mz_off);
  float M = -INFINITY;
  for (int c = 0; c < rs.n_chunks; ++c) M = fmaxf(M, mz[(int64_t)c * LASTQ * 2 + 2 * r]);
  float Z = 0.f;
  if (M > -INFINITY)
    for (int c = 0; c < rs.n_chunks; ++c) {
      const float m = mz[(int64_t)c * LASTQ * 2 + 2 * r];
      if (m > -INFINITY) Z += mz[(int64_t)c * LASTQ * 2 + 2 * r + 1] * ex2(m - M);
    }
  float* st = at<float>(dp, rs.stat_off);
  st[2 * r] = M;
  st[2 * r + 1] = Z > 0.f ? 1.f / Z : 0.f;
}

PFN_cuTensorMapEncodeTiled_v12000 lq_encode_fn() {
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

// 3D map over [heads][rows][128] bf16 (element strides); boxes of 64 rows x 64 columns with
// the 128-byte swizzle; rows outside [0, rows) read as zero.
bool lq_make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t heads, int64_t row_stride,
                 int64_t head_stride) {
  auto fn = lq_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)std::max<int64_t>(heads, 1)};
  cuuint64_t strides[2] = {(cuuint64_t)(row_stride * 2),
                           (cuuint64_t)(std::max<int64_t>(head_stride, rows * row_stride) * 2)};
  if (heads > 1) strides[1] = (cuuint64_t)(head_stride * 2);
  cuuint32_t box[3] = {64, (cuuint32_t)LQ_KB, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

// Shared memory the two passes launch with (pass 2 with `ring` slash-ring entries per row set).
size_t lastq_smem_bytes(int pass, int ring) {
  if (pass == 1) return sizeof(LqtSmem<1>) + 2 * sizeof(float) * 128;  // + the row halves' exchange
  return sizeof(LqtSmem<2>) + sizeof(LqtSmem2) + 2 * sizeof(float) * (size_t)ring;
}

int32_t lastq_pick_chunk(const int32_t* tile_key_hi, int n_tiles) {
  // the largest power of two from 8192 down to 256 keys that still gives eight CTAs per SM (four
  // waves of the two resident CTAs, so that the last wave's tail is short), while the look-back
  // of pass 2 (the rows' span below each chunk) stays small against the chunk
  auto ctas = [&](int32_t ch) {
    int64_t n = 0;
    for (int i = 0; i < n_tiles; ++i) n += (tile_key_hi[i] + ch - 1) / ch;
    return n;
  };
  int32_t chunk = 8192;
  while (chunk > 256 && ctas(chunk) < 8LL * sm_count()) chunk /= 2;
  return chunk;
}

int lastq_ring_entries(int32_t max_span) {
  int r = 128;
  while (r < max_span + 2 * LQ_KB && r < LQ_RING_MAX) r <<= 1;
  return r;
}

cudaError_t launch_lastq(const DevPlan& dp, const void* Q, const void* K, const msa_strides& s, cudaStream_t st) {
  cudaError_t e;
  if (dp.n_lqtiles <= 0) return cudaSuccess;
  if (dp.has2d && (e = launch_group_k(dp, K, s, st)) != cudaSuccess) return e;
  if (dp.lq_ring < 128 || dp.lq_ring > LQ_RING_MAX || (dp.lq_ring & (dp.lq_ring - 1))) return cudaErrorInvalidValue;
  const size_t smem1 = lastq_smem_bytes(1, 0), smem2 = lastq_smem_bytes(2, dp.lq_ring);
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (device_pending(configured, dev)) {
    if ((e = cudaFuncSetAttribute(lastq_tc<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(lastq_tc<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)lastq_smem_bytes(2, LQ_RING_MAX))) != cudaSuccess)
      return e;
    mark_device(configured, dev);
  }
  CUtensorMap mk, mk2;
  bool ok = lq_make_map(&mk, K, dp.L, dp.Hkv, s.k_row, s.k_head);
  if (ok)
    ok = dp.has2d ? lq_make_map(&mk2, dp.ws + dp.lay.k2d, dp.L, dp.Hkv, D, dp.L * D)
                  : lq_make_map(&mk2, K, dp.L, dp.Hkv, s.k_row, s.k_head);
  if (!ok) return cudaErrorInvalidValue;
  const dim3 grid(dp.max_chunks, dp.n_lqtiles);
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(Q);
  count_launches(3);
  lastq_tc<1><<<grid, LQ_THREADS, smem1, st>>>(mk, mk2, dp, q, s.q_head, s.q_row);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  lastq_combine<<<dp.n_rowsets, LASTQ, 0, st>>>(dp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  lastq_tc<2><<<grid, LQ_THREADS, smem2, st>>>(mk, mk2, dp, q, s.q_head, s.q_row);
  return cudaGetLastError();
}

}  // namespace msa
