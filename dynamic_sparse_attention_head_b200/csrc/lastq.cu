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
// warp streams key blocks of K with TMA (128-byte swizzle, no multicast) into a ring of
// stages; one thread issues tcgen05.mma (bf16 in, fp32 accumulate, K = 128) into one of two
// accumulator buffers in tensor memory; eight softmax warps read them with tcgen05.ld and do
// the per-element work in fp32 (exp2 on MUFU).
//   Pass 1 computes S = Q K^T (M = 128 query rows, N = 64 keys): a thread holds 32 keys of one
// query row, so the row max and sum stay in registers.
//   Pass 2 computes S^T = K Q^T (M = 128 keys, N = 128 query rows): a thread holds one key and
// the 64 rows of one row set, so its vertical sum is a sum over its own registers; the
// diagonals (key - row = const) are gathered across the warp's lanes by shuffles (column c of
// lane l moves to lane l - c, so each lane collects whole diagonals), staged per warp and
// combined by the row set's 128 threads in a fixed order, so results are deterministic.  A
// chunk owns the vertical sums of its keys and the slash sums of the offsets whose last-row key
// lies in it; it re-reads the `span` keys below it to complete those offsets, and carries
// partial slash sums from block to block in a small ring indexed by offset.
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
constexpr int LQ_THREADS = 320;                 // warp 0 TMA, warp 1 MMA, warps 2-9 softmax
constexpr int LQ_SOFTMAX = 256;                 // softmax threads
constexpr uint32_t Q_ATOM = 128 * 128;          // [128 rows][64 cols] bf16, 128-byte swizzled
constexpr uint32_t BOX = 64 * 128;              // one TMA box: [64 rows][64 cols] bf16
constexpr int LQ_RING_MAX = 8192;               // row sets span at most 4096 coordinates

// pass 1: 64-key blocks, four stages, S buffers of 64 columns
constexpr int P1_KB = 64;
constexpr int P1_STAGES = 4;
constexpr uint32_t P1_STAGE = 2 * BOX;          // [2 column halves][64 keys][64 cols]
constexpr int P1_TMEM = 2 * P1_KB;


// pass 2: 128-key blocks, two stages, S^T buffers of 128 columns (one per query row)
constexpr int P2_KB = 128;
constexpr int P2_STAGES = 2;
constexpr uint32_t P2_ATOM = P2_KB * 128;       // [128 keys][64 cols]
constexpr uint32_t P2_STAGE = 2 * P2_ATOM;
constexpr int P2_TMEM = 2 * 128;

constexpr int P2_DIAG = 96;                     // staged diagonals per warp (32 keys x 64 rows)

struct __align__(1024) Lq1Smem {
  uint8_t q[2 * Q_ATOM];
  uint8_t k[P1_STAGES][P1_STAGE];
  uint64_t k_full[P1_STAGES], k_empty[P1_STAGES];
  uint64_t s_full[2], s_free[2], q_ready, drain;
  uint32_t tmem_base;
  int abort;
  float xch[128][2];  // the second column half's (max, sum) of each row
};

struct __align__(1024) Lq2Smem {
  uint8_t q[2 * Q_ATOM];
  uint8_t k[P2_STAGES][P2_STAGE];
  uint64_t k_full[P2_STAGES], k_empty[P2_STAGES];
  uint64_t s_full[2], s_free[2], q_ready, drain;
  uint32_t tmem_base;
  int abort;
  float nm2[128];                   // per tile row: -(max + log2(normaliser)), -inf: no probability
  int32_t pos[128];                 // per tile row: position (causal bound of its keys)
  int32_t rcs[128];                 // per tile row: slash coordinate
  float stg[2][2][4][P2_DIAG];      // [block parity][set][key quarter][entry]: diagonal sums
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

// Column c (register) of lane l moves to lane l - c: `lo` adds it when l + c < 32 (the value
// of lane l + c), `hi` when l + c >= 32 (the value of lane l + c - 32).  Shifting by c and by
// 32 - c moves every value exactly once; each shuffle's own in-range predicate picks the sum.
template <int C>
__device__ __forceinline__ void diag_step(float v, float& lo, float& hi) {
  if constexpr (C == 0) {
    lo += v;
  } else {
    asm("{\n\t.reg .pred p, q;\n\t.reg .f32 t, u;\n\t"
        "shfl.sync.down.b32 t|p, %2, %3, 0x1f, 0xffffffff;\n\t"
        "shfl.sync.up.b32 u|q, %2, %4, 0x0, 0xffffffff;\n\t"
        "@p add.f32 %0, %0, t;\n\t"
        "@q add.f32 %1, %1, u;\n\t}"
        : "+f"(lo), "+f"(hi)
        : "f"(v), "n"(C), "n"(32 - C));
  }
}

template <int C>
struct DiagUnroll {
  __device__ __forceinline__ static void run(const float (&v)[32], float& lo, float& hi) {
    DiagUnroll<C - 1>::run(v, lo, hi);
    diag_step<C - 1>(v[C - 1], lo, hi);
  }
};
template <>
struct DiagUnroll<0> {
  __device__ __forceinline__ static void run(const float (&)[32], float&, float&) {}
};

// The tile's key range processed by chunk `chunk`: keys [c0, c1), of which the chunk owns
// [own0, own1); in pass 2, c0 reaches the rows' span (rounded up to a block) below the chunk so
// that the slash offsets whose last-row key lies in the chunk are complete.
struct ChunkKeys {
  int64_t own0, own1, c0, c1;
};

__device__ __forceinline__ ChunkKeys chunk_keys(const RowSet& a, const RowSet* b, int chunk, int back_round) {
  ChunkKeys k;
  k.own0 = (int64_t)chunk * a.chunk;
  const int64_t hi = b ? max(a.key_hi, b->key_hi) : a.key_hi;
  k.own1 = min(k.own0 + (int64_t)a.chunk, hi);
  int64_t back = 0;
  if (back_round > 0) {
    const int64_t r = back_round;
    if (a.slash_hi > a.slash_lo) back = max(back, (a.span + r - 1) / r * r);
    if (b && b->slash_hi > b->slash_lo) back = max(back, (b->span + r - 1) / r * r);
  }
  k.c0 = max((int64_t)0, k.own0 - back);
  k.c1 = k.own1;
  return k;
}

// The tile's 128 query rows into the swizzled Q tile (16-byte copies by the 256 softmax
// threads, zero rows as padding).
__device__ __forceinline__ void load_q_tile(uint8_t* qs, const RowSet& ra, const RowSet* rb,
                                            const __nv_bfloat16* __restrict__ Q, int64_t qh, int64_t qr, int t256) {
  for (int i = t256; i < 128 * 16; i += LQ_SOFTMAX) {
    const int r = i >> 4, c = i & 15;
    const RowSet* s_ = r < 64 ? &ra : rb;
    const int rl = r & 63;
    const bool valid = s_ != nullptr && rl < s_->n_rows;
    const __nv_bfloat16* src = valid ? Q + (int64_t)s_->head * qh + (int64_t)s_->rows[rl] * qr + c * 8 : Q;
    const uint32_t dst = smem_addr(qs) + (uint32_t)(c >> 3) * Q_ATOM + (uint32_t)r * 128u +
                         ((uint32_t)((c & 7) ^ (r & 7)) << 4);
    cp_async16_zfill(dst, src, valid ? 16u : 0u);
  }
  cp_async_wait_all();
  fence_proxy_async_smem();
}

}  // namespace

namespace {
// Barriers and tensor memory of a sweep CTA (thread 0 initialises, warp 1 allocates).
template <int ST, int TM>
__device__ __forceinline__ void lq_setup(uint64_t* k_full, uint64_t* k_empty, uint64_t* s_full, uint64_t* s_free,
                                         uint64_t* q_ready, uint64_t* drain, int* abort, uint32_t* tmem_slot) {
  if (threadIdx.x == 0) {
    *abort = 0;
    for (int s = 0; s < ST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], LQ_SOFTMAX);
    }
    mbar_init(q_ready, LQ_SOFTMAX);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if ((threadIdx.x >> 5) == 1) tmem_alloc<TM>(tmem_slot);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

// TMA producer (one thread): key blocks of KB rows, both 64-column halves, into ST stages laid
// out [column half][KB rows][128 B]; the copies still in flight land before it returns.
template <int KB, int ST>
__device__ __forceinline__ void lq_produce(uint8_t* k0, uint64_t* k_full, uint64_t* k_empty, const CUtensorMap* m,
                                           int64_t c0, int nblk, int kvh, volatile int* abort) {
  constexpr uint32_t ATOM = KB * 128;
  tma_prefetch_desc(m);
  int issued = 0;
  for (int b = 0; b < nblk; ++b) {
    const int st = b % ST;
    if (b >= ST && !mbar_wait(&k_empty[st], ((b / ST) - 1) & 1, abort)) break;
    mbar_arrive_expect_tx(&k_full[st], 2 * ATOM);
    const int row = (int)(c0 + (int64_t)b * KB);
    uint8_t* dst = k0 + (size_t)st * 2 * ATOM;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int r = 0; r < KB / 64; ++r) tma_load_3d(dst + h * ATOM + r * BOX, m, &k_full[st], 64 * h, row + 64 * r, kvh);
    issued = b + 1;
  }
  int drain_flag = 0;  // own limit; ignores abort
  for (int b = max(0, issued - ST); b < issued; ++b) mbar_wait(&k_full[b % ST], (b / ST) & 1, &drain_flag, 100000000ull);
}

// MMA issuer (one thread): per block, eight K = 16 steps into accumulator buffer b & 1.
// KEYS_AS_ROWS: D = K Q^T (M = KB keys, N = 128 query rows), else D = Q K^T (M = 128, N = KB).
// Every MMA issued completes before it returns.
template <int KB, int ST, bool KEYS_AS_ROWS>
__device__ __forceinline__ void lq_issue(uint32_t tmem, uint32_t qa, uint32_t k0, uint64_t* k_full, uint64_t* k_empty,
                                         uint64_t* s_full, uint64_t* s_free, uint64_t* q_ready, uint64_t* drain,
                                         int nblk, volatile int* abort) {
  constexpr uint32_t ATOM = KB * 128;
  constexpr uint32_t DCOLS = KEYS_AS_ROWS ? 128 : KB;
  constexpr uint32_t IDESC = KEYS_AS_ROWS ? idesc_bf16_f32(KB, 128, 0, 0) : idesc_bf16_f32(128, KB, 0, 0);
  if (nblk > 0 && mbar_wait(q_ready, 0, abort)) {
    for (int b = 0; b < nblk; ++b) {
      const int st = b % ST, buf = b & 1;
      if (!mbar_wait(&k_full[st], (b / ST) & 1, abort)) break;
      if (b >= 2 && !mbar_wait(&s_free[buf], ((b >> 1) - 1) & 1, abort)) break;
      tc_fence_after();
      const uint32_t ka = k0 + (uint32_t)st * 2 * ATOM;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t qd = smem_desc_sw128(qa + (kk >> 2) * Q_ATOM + (kk & 3) * 32, 16, 1024);
        const uint64_t kd = smem_desc_sw128(ka + (kk >> 2) * ATOM + (kk & 3) * 32, 16, 1024);
        umma_ss(tmem + (uint32_t)buf * DCOLS, KEYS_AS_ROWS ? kd : qd, KEYS_AS_ROWS ? qd : kd, IDESC, kk > 0 ? 1u : 0u);
      }
      umma_commit(&k_empty[st]);
      umma_commit(&s_full[buf]);
    }
  }
  umma_commit(drain);
  int drain_flag = 0;  // own limit
  mbar_wait(drain, 0, &drain_flag, 100000000ull);
}

// Pass 1: per row and key chunk, the max and the sum of the exponentials (log2 units).
__global__ void __launch_bounds__(LQ_THREADS, 2)
    lastq_stats(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmK2, const DevPlan dp,
                const __nv_bfloat16* __restrict__ Q, int64_t qh, int64_t qr) {
  extern __shared__ __align__(1024) uint8_t lq_smem[];
  Lq1Smem& sm = *reinterpret_cast<Lq1Smem*>(lq_smem);
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
  const ChunkKeys ck = chunk_keys(ra, rb, chunk, 0);
  const int nblk = (int)((ck.c1 - ck.c0 + P1_KB - 1) / P1_KB);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &sm.abort;
  lq_setup<P1_STAGES, P1_TMEM>(sm.k_full, sm.k_empty, sm.s_full, sm.s_free, &sm.q_ready, &sm.drain, &sm.abort,
                               &sm.tmem_base);
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    if (lane == 0 && nblk > 0)
      lq_produce<P1_KB, P1_STAGES>(&sm.k[0][0], sm.k_full, sm.k_empty, tile.k_src == SRC_K2D ? &tmK2 : &tmK, ck.c0,
                                   nblk, tile.kvh, abort);
  } else if (warp == 1) {
    if (lane == 0)
      lq_issue<P1_KB, P1_STAGES, false>(tmem, smem_addr(sm.q), smem_addr(&sm.k[0][0]), sm.k_full, sm.k_empty,
                                        sm.s_full, sm.s_free, &sm.q_ready, &sm.drain, nblk, abort);
  } else {
    // eight warps, two per row: warp w reaches TMEM lanes 32 (w % 4) .. + 31 only, so warps
    // 2-5 take columns 0-31 of their 32 rows and warps 6-9 columns 32-63 of the same rows
    const int qd = warp & 3;
    const int hc = (warp - 2) >> 2;  // column half of this warp
    const int m = qd * 32 + lane;
    const int set = m >> 6, rr = m & 63;
    const RowSet* rs = set == 0 ? &ra : rb;
    load_q_tile(sm.q, ra, rb, Q, qh, qr, threadIdx.x - 64);
    mbar_arrive(&sm.q_ready);

    const bool have = rs != nullptr && rr < rs->n_rows;
    const int32_t pr = have ? rs->rows[rr] : -1;  // a padding row has no causal key
    const float sl2 = dp.scale * LOG2E;
    const bool k2d = tile.k_src == SRC_K2D;
    const int32_t* perm = k2d ? at<const int32_t>(dp, dp.lay.perm2d) : nullptr;
    const uint32_t s_lane = tmem + ((uint32_t)(qd * 32) << 16) + (uint32_t)(32 * hc);

    // over this thread's 32 columns of each block: running max of the raw logits, the same max
    // in log2 units (mrun * sl2, the value every exponent is taken against) and the sum
    float mrun = -INFINITY, ml2 = -INFINITY, z = 0.f;
    const float2 sl2v = make_float2(sl2, sl2);
    // modality-grouped keys: this lane's key position in block b, through perm2d (loaded one
    // block ahead, so that the load overlaps the work on the block before)
    auto grouped_pos = [&](int b) -> int32_t {
      const int64_t j = ck.c0 + (int64_t)b * P1_KB + 32 * hc + lane;
      return j < dp.L ? __ldg(perm + j) : 0x7fffffff;
    };
    int32_t pos_next = k2d && nblk > 0 ? grouped_pos(0) : 0;
    for (int b = 0; b < nblk; ++b) {
      // the row's 32 raw logits of block b (this warp's column half), -inf where the key is not
      // causal; key positions: modality-grouped keys through perm2d, else the row itself
      const int buf = b & 1;
      const int64_t j0 = ck.c0 + (int64_t)b * P1_KB + 32 * hc;
      int32_t pos, pmax;
      if (!k2d) {
        pos = (int32_t)(j0 + lane);
        pmax = (int32_t)(j0 + 31);
      } else {
        pos = pos_next;
        if (b + 1 < nblk) pos_next = grouped_pos(b + 1);
        pmax = pos;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) pmax = max(pmax, __shfl_xor_sync(0xFFFFFFFFu, pmax, o));
      }
      // the warp decides together (the loads below are warp-collective)
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.s_full[buf], (b >> 1) & 1, abort))) break;
      tc_fence_after();
      uint32_t sa[32];
      tmem_ld32(s_lane + (uint32_t)(buf * P1_KB), sa);
      tmem_wait_ld_regs(sa);
      tc_fence_before();
      mbar_arrive(&sm.s_free[buf]);
      float x[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) x[c] = __uint_as_float(sa[c]);
      if (__any_sync(0xFFFFFFFFu, pmax > pr)) {  // some key of the half is after some row of the warp
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (__shfl_sync(0xFFFFFFFFu, pos, c) > pr) x[c] = -INFINITY;
      }
      // the half-block max in eight independent chains, then the sum of the exponentials in
      // pairs (short dependency chains: the loop is latency-bound)
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = lq_fmax3(x[q], x[8 + q], fmaxf(x[16 + q], x[24 + q]));
      const float bm = fmaxf(lq_fmax3(m8[0], m8[1], m8[2]), lq_fmax3(m8[3], lq_fmax3(m8[4], m8[5], m8[6]), m8[7]));
      if (!(bm > mrun)) {
        if (mrun == -INFINITY) continue;  // nothing causal yet
      } else {
        const float nl2 = bm * sl2;
        z = (mrun == -INFINITY) ? 0.f : z * ex2(ml2 - nl2);
        mrun = bm;
        ml2 = nl2;
      }
      const float2 neg = make_float2(-ml2, -ml2);
      float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 32; c += 4) {
        const float2 t0 = __ffma2_rn(make_float2(x[c], x[c + 1]), sl2v, neg);
        const float2 t1 = __ffma2_rn(make_float2(x[c + 2], x[c + 3]), sl2v, neg);
        a0 = __fadd2_rn(a0, make_float2(ex2(t0.x), ex2(t0.y)));
        a1 = __fadd2_rn(a1, make_float2(ex2(t1.x), ex2(t1.y)));
      }
      const float2 a = __fadd2_rn(a0, a1);
      z += a.x + a.y;
    }
    mrun = ml2;  // the row's max in log2 units from here on
    // the two halves of each row: the second half's (max, sum) through shared memory, combined
    // by the first half's thread (columns 0-31 first, then 32-63)
    if (hc == 1) {
      sm.xch[m][0] = mrun;
      sm.xch[m][1] = z;
    }
    asm volatile("bar.sync 3, %0;" ::"n"(LQ_SOFTMAX) : "memory");
    if (hc == 0) {
      const float m1 = sm.xch[m][0], z1 = sm.xch[m][1];
      const float M = fmaxf(mrun, m1);
      float Z = 0.f;
      if (M > -INFINITY) Z = (mrun > -INFINITY ? z * ex2(mrun - M) : 0.f) + (m1 > -INFINITY ? z1 * ex2(m1 - M) : 0.f);
      if (rs != nullptr && chunk < rs->n_chunks) {
        float* mz = at<float>(dp, rs->mz_off) + (int64_t)chunk * LASTQ * 2;
        mz[2 * rr] = M;
        mz[2 * rr + 1] = Z;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && sm.abort) atomicOr(err, DEV_ERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<P1_TMEM>(tmem);
  }
}

// One half (32 query rows) of a pass-2 thread's key: the probabilities p = exp2(s * sl2 + nm2)
// (nm2 = -(max + log2 Z) of the row), their sum into va, and, with DIAG, the diagonals into
// lo / hi (see diag_step).  With MASK: rows the key is not causal for count zero (key position
// kp after the row's position), and so do all slash contributions of a key outside the slash
// range (dz).  The probabilities (zero outside the slash range) are left in sv for the caller.
template <bool MASK, bool DIAG>
__device__ __forceinline__ void lq2_half(uint32_t (&sv)[32], const float* nm2, const int32_t* pos, float2 sl2v,
                                         int32_t kp, bool dz, float2 (&va)[2], float& lo, float& hi) {
  float p[32];
#pragma unroll
  for (int c = 0; c < 32; c += 2) {
    const float2 t = __ffma2_rn(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl2v,
                                make_float2(nm2[c], nm2[c + 1]));
    float x0 = ex2(t.x), x1 = ex2(t.y);
    if (MASK) {
      x0 = kp > pos[c] ? 0.f : x0;
      x1 = kp > pos[c + 1] ? 0.f : x1;
    }
    va[(c >> 1) & 1] = __fadd2_rn(va[(c >> 1) & 1], make_float2(x0, x1));
    p[c] = MASK && dz ? 0.f : x0;
    p[c + 1] = MASK && dz ? 0.f : x1;
  }
  if (DIAG) DiagUnroll<32>::run(p, lo, hi);
#pragma unroll
  for (int c = 0; c < 32; ++c) sv[c] = __float_as_uint(p[c]);
}

// Pass 2: the probabilities exp2(x - max - log2 Z) of the tile's rows against each key;
// vertical sums by key and slash sums by offset.
__global__ void __launch_bounds__(LQ_THREADS, 2)
    lastq_sums(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmK2, const DevPlan dp,
               const __nv_bfloat16* __restrict__ Q, int64_t qh, int64_t qr) {
  extern __shared__ __align__(1024) uint8_t lq_smem[];
  Lq2Smem& sm = *reinterpret_cast<Lq2Smem*>(lq_smem);
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
  const ChunkKeys ck = chunk_keys(ra, rb, chunk, 64);
  const int nblk = (int)((ck.c1 - ck.c0 + P2_KB - 1) / P2_KB);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &sm.abort;
  lq_setup<P2_STAGES, P2_TMEM>(sm.k_full, sm.k_empty, sm.s_full, sm.s_free, &sm.q_ready, &sm.drain, &sm.abort,
                               &sm.tmem_base);
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    if (lane == 0 && nblk > 0)
      lq_produce<P2_KB, P2_STAGES>(&sm.k[0][0], sm.k_full, sm.k_empty, tile.k_src == SRC_K2D ? &tmK2 : &tmK, ck.c0,
                                   nblk, tile.kvh, abort);
  } else if (warp == 1) {
    if (lane == 0)
      lq_issue<P2_KB, P2_STAGES, true>(tmem, smem_addr(sm.q), smem_addr(&sm.k[0][0]), sm.k_full, sm.k_empty,
                                       sm.s_full, sm.s_free, &sm.q_ready, &sm.drain, nblk, abort);
  } else {
    // eight warps: warp w reaches TMEM lanes (keys) 32 (w % 4) .. + 31 only; warps 2-5 take
    // the columns (query rows) of row set 0, warps 6-9 those of row set 1
    const int q4 = warp & 3;          // key quarter of the block
    const int set = (warp - 2) >> 2;  // row set
    const int ts = q4 * 32 + lane;    // thread of the row set (0 .. 127)
    const int t256 = threadIdx.x - 64;
    const RowSet* rs = set == 0 ? &ra : rb;
    load_q_tile(sm.q, ra, rb, Q, qh, qr, t256);
    mbar_arrive(&sm.q_ready);
    if (t256 < 128) {
      // per tile row: -(max + log2 Z) from the pass-1 statistics, position, slash coordinate
      const int r = t256 & 63;
      const RowSet* s_ = t256 < 64 ? &ra : rb;
      const bool have = s_ != nullptr && r < s_->n_rows;
      float nm2 = -INFINITY;
      if (have) {
        const float* st = at<const float>(dp, s_->stat_off);
        if (st[2 * r] > -INFINITY) nm2 = -(st[2 * r] + st[2 * r + 1]);
      }
      sm.nm2[t256] = nm2;
      sm.pos[t256] = have ? s_->rows[r] : -1;
      sm.rcs[t256] = have ? s_->rcs[r] : 0;
    }
    const int R = dp.lq_ring;
    float* ring = reinterpret_cast<float*>(lq_smem + sizeof(Lq2Smem)) + set * R;
    for (int i = ts; i < R; i += 128) ring[i] = 0.f;
    // the row set's geometry
    const bool slash = rs != nullptr && rs->slash_hi > rs->slash_lo;
    int32_t min_rc = 0x7fffffff, max_rc = -0x7fffffff, min_pos = 0x7fffffff;
    bool contig = true;
    if (rs != nullptr)
      for (int r = 0; r < rs->n_rows; ++r) {
        const int32_t c = rs->rcs[r];
        min_rc = min(min_rc, c);
        max_rc = max(max_rc, c);
        min_pos = min(min_pos, rs->rows[r]);
        contig = contig && c == rs->rcs[0] + r;
      }
    // key and offset coordinates fit in 32 bits (L < 2^31)
    const int32_t own0 = (int32_t)ck.own0;
    const int32_t own1 = rs != nullptr ? (int32_t)min(ck.own0 + (int64_t)ra.chunk, (int64_t)rs->key_hi) : 0;
    const int32_t own_end = (int32_t)min(ck.own0 + (int64_t)ra.chunk, (int64_t)dp.L);  // offsets owned: last-row key in [own0, own_end)
    float* vout = rs != nullptr ? at<float>(dp, rs->v_off) : nullptr;
    float* sout = slash ? at<float>(dp, rs->s_off) : nullptr;
    const int32_t slo = slash ? rs->slash_lo : 0, shi = slash ? rs->slash_hi : 0;
    const int32_t rc0 = rs != nullptr ? rs->rcs[0] : 0;
    const int32_t L32 = (int32_t)dp.L;
    const float sl2 = dp.scale * LOG2E;
    const bool k2d = tile.k_src == SRC_K2D;
    const int32_t* perm = k2d ? at<const int32_t>(dp, dp.lay.perm2d) : nullptr;
    const uint32_t t_lane = tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(64 * set);
    const float* m2s = sm.nm2 + 64 * set;
    const float2 sl2v = make_float2(sl2, sl2);
    const int32_t* poss = sm.pos + 64 * set;
    const int32_t* rcss = sm.rcs + 64 * set;
    asm volatile("bar.sync 3, %0;" ::"n"(LQ_SOFTMAX) : "memory");  // tables and rings in place

    for (int b = 0; b < nblk; ++b) {
      const int32_t j0 = (int32_t)ck.c0 + b * P2_KB;
      const int32_t k = j0 + 32 * q4 + lane;  // this thread's key (source row)
      const int buf = b & 1;
      const int sb = b & 1;  // staging parity: rewritten two blocks later, after every thread of
                             // the set has passed the barrier between
      // the warp decides together (the loads below are warp-collective)
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.s_full[buf], (b >> 1) & 1, abort));
      float2 va[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      float d0 = 0.f, d1 = 0.f, d2 = 0.f;  // diagonals -32 q4 - lane, + 32, + 64 of the block
      if (ok) tc_fence_after();
      if (rs == nullptr) {
        if (ok) mbar_arrive(&sm.s_free[buf]);
      } else {
        const bool live = ok;
        int32_t kp = 0x7fffffff;  // the key's position
        if (live) kp = !k2d ? k : (k < L32 ? __ldg(perm + k) : 0x7fffffff);
        const bool dzero = slash && !(k >= slo && k < shi);  // key outside the slash range
        // warp-uniform: some row is before some key of the warp, or some key is outside the range
        const bool masked = __any_sync(0xFFFFFFFFu, kp > min_pos || dzero);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // rows 32 h .. 32 h + 31 of the set; the buffer is released after the second load
          uint32_t sv[32];
          if (live) {
            tmem_ld32(t_lane + (uint32_t)(buf * 128 + 32 * h), sv);
            tmem_wait_ld_regs(sv);
            if (h == 1) {
              tc_fence_before();
              mbar_arrive(&sm.s_free[buf]);
            }
          }
          const float* m2h = m2s + 32 * h;
          const int32_t* posh = poss + 32 * h;
          if (slash && contig) {
            if (live) {
              float& lo = h == 0 ? d0 : d1;
              float& hi = h == 0 ? d1 : d2;
              if (masked) lq2_half<true, true>(sv, m2h, posh, sl2v, kp, dzero, va, lo, hi);
              else lq2_half<false, true>(sv, m2h, posh, sl2v, kp, dzero, va, lo, hi);
            }
          } else if (!slash) {
            if (live) {
              if (masked) lq2_half<true, false>(sv, m2h, posh, sl2v, kp, dzero, va, d0, d0);
              else lq2_half<false, false>(sv, m2h, posh, sl2v, kp, dzero, va, d0, d0);
            }
          } else {
            // any row coordinates: the set's four warps add their keys' slash values to the ring
            // in turn (within a warp the 32 keys of one row reach 32 distinct offsets), rows in
            // order; every warp of the set takes part in the barriers
            if (live) lq2_half<true, false>(sv, m2h, posh, sl2v, kp, dzero, va, d0, d0);
#pragma unroll 1
            for (int qq = 0; qq < 4; ++qq) {
              set_sync(set);
              if (live && q4 == qq)
#pragma unroll
                for (int c = 0; c < 32; ++c) ring[(rcss[32 * h + c] - k) & (R - 1)] += __uint_as_float(sv[c]);
            }
          }
        }
        if (live && k >= own0 && k < own1) vout[k] = (va[0].x + va[0].y) + (va[1].x + va[1].y);
        if (live && slash && contig) {
          sm.stg[sb][set][q4][lane] = d2;
          sm.stg[sb][set][q4][32 + lane] = d1;
          sm.stg[sb][set][q4][64 + lane] = d0;
        }
      }
      if (set_any(set, !ok)) break;  // every thread of the set leaves together
      if (slash && contig) {
        // consecutive row coordinates: offset rc0 - j0 + d collects the block's diagonal
        // d = row - key (-127 .. 63), held by key quarter qq at entry 64 - 32 qq - d; quarters
        // in order, then the ring; an offset is written out once its last-row key is in the block
        for (int e = ts; e < 192; e += 128) {
          const int d = e - 128;
          float a = 0.f;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const int t = 64 - 32 * qq - d;
            if (t >= 0 && t < P2_DIAG) a += sm.stg[sb][set][qq][t];
          }
          const int32_t o = rc0 - j0 + d;
          float& ent = ring[o & (R - 1)];
          const float tot = ent + a;
          const int32_t kk = max_rc - o - j0;  // the offset's last-row key, from j0
          if (kk >= 0 && kk < P2_KB) {
            if (j0 + kk >= own0 && j0 + kk < own_end && o >= 0) sout[o] = tot;
            ent = 0.f;
          } else {
            ent = tot;
          }
        }
      } else if (slash) {
        // offsets whose last-row key is j0 + ts are complete: written if the chunk owns them
        const int32_t o = max_rc - (j0 + ts);
        float& ent = ring[o & (R - 1)];
        if (j0 + ts >= own0 && j0 + ts < own_end && o >= 0) sout[o] = ent;
        ent = 0.f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && sm.abort) atomicOr(err, DEV_ERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<P2_TMEM>(tmem);
  }
}

// Row max and log2 of the normaliser over the chunks, in chunk order (max -inf: no causal key).
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
  st[2 * r] = Z > 0.f ? M : -INFINITY;
  st[2 * r + 1] = Z > 0.f ? log2f(Z) : 0.f;
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
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

// Shared memory the two passes launch with (pass 2 with `ring` slash-ring entries per row set).
size_t lastq_smem_bytes(int pass, int ring) {
  if (pass == 1) return sizeof(Lq1Smem);
  return sizeof(Lq2Smem) + 2 * sizeof(float) * (size_t)ring;
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
  // the offsets one pass-2 block touches (span + 2 blocks of keys) map to distinct entries
  int r = 256;
  while (r < max_span + 2 * P2_KB && r < LQ_RING_MAX) r <<= 1;
  return r;
}

cudaError_t launch_lastq(const DevPlan& dp, const void* Q, const void* K, const msa_strides& s, cudaStream_t st) {
  cudaError_t e;
  if (dp.n_lqtiles <= 0) return cudaSuccess;
  if (dp.has2d && (e = launch_group_k(dp, K, s, st)) != cudaSuccess) return e;
  if (dp.lq_ring < 256 || dp.lq_ring > LQ_RING_MAX || (dp.lq_ring & (dp.lq_ring - 1))) return cudaErrorInvalidValue;
  const size_t smem1 = lastq_smem_bytes(1, 0), smem2 = lastq_smem_bytes(2, dp.lq_ring);
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (device_pending(configured, dev)) {
    if ((e = cudaFuncSetAttribute(lastq_stats, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(lastq_sums, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  lastq_stats<<<grid, LQ_THREADS, smem1, st>>>(mk, mk2, dp, q, s.q_head, s.q_row);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  lastq_combine<<<dp.n_rowsets, LASTQ, 0, st>>>(dp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  lastq_sums<<<grid, LQ_THREADS, smem2, st>>>(mk, mk2, dp, q, s.q_head, s.q_row);
  return cudaGetLastError();
}

}  // namespace msa
