// Online index estimation (MInference 1.0 "Approach"; MMInference "key machinery" and
// "core discovery"):
//  - last-64-query sweep: for each row set (<= 64 queries of one head) the causal softmax
//    over all keys is reduced to vertical sums v[key] and slash sums s[offset].  Pass 1
//    finds each row's max and normaliser, pass 2 accumulates the probabilities.  Every
//    sum has a fixed order, so results are deterministic; chunks of 1024 keys own their
//    v entries and the slash offsets whose last-row key falls in the chunk (they recompute
//    the `span` keys below the chunk instead of exchanging partial sums).
//  - deterministic top-k (radix select on the order-preserving uint32 image of fp32;
//    ties go to the lower index), output sorted ascending;
//  - block-sparse: 64-token mean pooling of Q and K, pooled logits, per-row top-k.
// The logits come from bf16 mma.sync with fp32 accumulation: this stage streams K once per
// pass and is bound by HBM bandwidth / MUFU exp throughput, not by the tensor pipe.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

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

// ---------------------------------------------------------------------------------------
// modality-grouped copy of K (or V): dst[h][r] = src[h][perm2d[r]]
// ---------------------------------------------------------------------------------------
__global__ void group_rows_kernel(DevPlan dp, const __nv_bfloat16* src, int64_t sh, int64_t sr,
                                  __nv_bfloat16* dst) {
  const int32_t* perm = at<const int32_t>(dp, dp.lay.perm2d);
  const int64_t total = (int64_t)dp.Hkv * dp.L;
  const int sub = threadIdx.x & 15;  // 16 lanes x 16 bytes per row
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4; i < total;
       i += ((int64_t)gridDim.x * blockDim.x) >> 4) {
    const int64_t h = i / dp.L, r = i % dp.L;
    const uint4* s = reinterpret_cast<const uint4*>(src + h * sh + (int64_t)perm[r] * sr);
    uint4* d = reinterpret_cast<uint4*>(dst + (h * dp.L + r) * D);
    d[sub] = s[sub];
  }
}

// ---------------------------------------------------------------------------------------
// last-query sweep
// ---------------------------------------------------------------------------------------
constexpr int LQ_THREADS = 128;
constexpr int KB = 64;       // keys per block
constexpr int PAD = 136;     // bf16 row pitch in shared memory (272 bytes: conflict-free fragments)
constexpr int SACC_MAX = 4096 + 1024 + 4096 + 64;  // largest accumulator: span 4096, chunk 1024

struct LqSmem {
  __nv_bfloat16 q[LASTQ * PAD];
  __nv_bfloat16 k[2][KB * PAD];
  float a[LASTQ * (KB + 1)];
  int32_t kpos[2][KB];
  int32_t rows[LASTQ];
  int32_t rcs[LASTQ];
  float stat[LASTQ][2];
};

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = smem_addr(dst);
  const int n = valid ? 16 : 0;  // zero-fill when invalid
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

struct KeySrc {
  const __nv_bfloat16* base;
  int64_t row_stride;
  const int32_t* pos;  // null: position = row
};

__device__ __forceinline__ void load_kblock(LqSmem& sm, int buf, const KeySrc& ks, int64_t j0, int64_t key_hi) {
  for (int i = threadIdx.x; i < KB * 16; i += LQ_THREADS) {
    const int r = i >> 4, c = i & 15;
    const int64_t j = j0 + r;
    const bool ok = j >= 0 && j < key_hi;
    const __nv_bfloat16* src = ks.base + (ok ? j : 0) * ks.row_stride + c * 8;
    cp_async16(&sm.k[buf][r * PAD + c * 8], src, ok);
  }
  for (int r = threadIdx.x; r < KB; r += LQ_THREADS) {
    const int64_t j = j0 + r;
    sm.kpos[buf][r] = (j >= 0 && j < key_hi) ? (ks.pos ? ks.pos[j] : (int32_t)j) : POS_PAD;
  }
}

// logits of this warp's 16 rows against the 64 keys of a block: c[nt][*] for key 8nt + 2t (+1)
__device__ __forceinline__ void block_logits(const LqSmem& sm, int buf, const uint32_t (&af)[8][4],
                                             float (&c)[8][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) c[nt][0] = c[nt][1] = c[nt][2] = c[nt][3] = 0.f;
  const __nv_bfloat16* kb = sm.k[buf];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const __nv_bfloat16* row = kb + (nt * 8 + g) * PAD + ks * 16 + 2 * t;
      const uint32_t b0 = *reinterpret_cast<const uint32_t*>(row);
      const uint32_t b1 = *reinterpret_cast<const uint32_t*>(row + 8);
      mma_bf16(c[nt], af[ks], b0, b1);
    }
  }
}

__device__ __forceinline__ void load_q(LqSmem& sm, const RowSet& rs, const __nv_bfloat16* Q, int64_t qh,
                                       int64_t qr) {
  for (int i = threadIdx.x; i < LASTQ * 16; i += LQ_THREADS) {
    const int r = i >> 4, c = i & 15;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < rs.n_rows)
      v = *reinterpret_cast<const uint4*>(Q + (int64_t)rs.head * qh + (int64_t)rs.rows[r] * qr + c * 8);
    *reinterpret_cast<uint4*>(&sm.q[r * PAD + c * 8]) = v;
  }
  for (int r = threadIdx.x; r < LASTQ; r += LQ_THREADS) {
    sm.rows[r] = r < rs.n_rows ? rs.rows[r] : -1;  // -1: no key is causal for a padding row
    sm.rcs[r] = r < rs.n_rows ? rs.rcs[r] : 0;
  }
}

__device__ __forceinline__ void load_afrag(const LqSmem& sm, uint32_t (&af)[8][4]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const __nv_bfloat16* q0 = sm.q + (warp * 16 + g) * PAD;
  const __nv_bfloat16* q8 = q0 + 8 * PAD;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    af[ks][0] = *reinterpret_cast<const uint32_t*>(q0 + ks * 16 + 2 * t);
    af[ks][1] = *reinterpret_cast<const uint32_t*>(q8 + ks * 16 + 2 * t);
    af[ks][2] = *reinterpret_cast<const uint32_t*>(q0 + ks * 16 + 8 + 2 * t);
    af[ks][3] = *reinterpret_cast<const uint32_t*>(q8 + ks * 16 + 8 + 2 * t);
  }
}

__device__ __forceinline__ KeySrc key_src(const DevPlan& dp, const RowSet& rs, const void* K, int64_t kh,
                                          int64_t kr) {
  KeySrc s;
  if (rs.k_src == SRC_K2D) {
    s.base = at<const __nv_bfloat16>(dp, dp.lay.k2d) + (int64_t)rs.kvh * dp.L * D;
    s.row_stride = D;
    s.pos = at<const int32_t>(dp, dp.lay.perm2d);
  } else {
    s.base = static_cast<const __nv_bfloat16*>(K) + (int64_t)rs.kvh * kh;
    s.row_stride = kr;
    s.pos = nullptr;
  }
  return s;
}

// Pass 1: per (row set, chunk) the running max / normaliser of each row (log2 domain).
__global__ void __launch_bounds__(LQ_THREADS) lastq_pass1(DevPlan dp, const __nv_bfloat16* Q, int64_t qh,
                                                          int64_t qr, const void* K, int64_t kh, int64_t kr) {
  extern __shared__ uint8_t lq_raw[];
  LqSmem& sm = *reinterpret_cast<LqSmem*>(lq_raw);
  const RowSet& rs = at<const RowSet>(dp, dp.lay.rowsets)[blockIdx.y];
  const int chunk = blockIdx.x;
  if (chunk >= rs.n_chunks) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  load_q(sm, rs, Q, qh, qr);
  const KeySrc ks = key_src(dp, rs, K, kh, kr);
  const int64_t c0 = (int64_t)chunk * rs.chunk, c1 = std::min<int64_t>(c0 + rs.chunk, rs.key_hi);
  const int nblk = (int)((c1 - c0 + KB - 1) / KB);
  load_kblock(sm, 0, ks, c0, c1);
  cp_async_commit();
  __syncthreads();
  uint32_t af[8][4];
  load_afrag(sm, af);
  const int r0 = warp * 16 + g, r1 = r0 + 8;
  const int32_t p0 = sm.rows[r0], p1 = sm.rows[r1];
  float m0 = -INFINITY, z0 = 0.f, m1 = -INFINITY, z1 = 0.f;
  for (int b = 0; b < nblk; ++b) {
    if (b + 1 < nblk) load_kblock(sm, (b + 1) & 1, ks, c0 + (int64_t)(b + 1) * KB, c1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    float c[8][4];
    block_logits(sm, b & 1, af, c);
    // the block's logits of both rows (log2 units; -inf where not causal), the rows' block
    // maxima over the quad, then one rescale of the running sums and one exp2 per element
    float bm0 = -INFINITY, bm1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int32_t kp = sm.kpos[b & 1][nt * 8 + 2 * t + (e & 1)];
        const bool top = e < 2;
        const float x = (kp > (top ? p0 : p1)) ? -INFINITY : (c[nt][e] * dp.scale) * LOG2E;
        c[nt][e] = x;
        if (top) bm0 = fmaxf(bm0, x);
        else bm1 = fmaxf(bm1, x);
      }
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      bm0 = fmaxf(bm0, __shfl_xor_sync(0xFFFFFFFFu, bm0, o));
      bm1 = fmaxf(bm1, __shfl_xor_sync(0xFFFFFFFFu, bm1, o));
    }
    const float n0 = fmaxf(m0, bm0), n1 = fmaxf(m1, bm1);
    if (n0 > -INFINITY) z0 = (m0 == -INFINITY) ? 0.f : z0 * ex2(m0 - n0);
    if (n1 > -INFINITY) z1 = (m1 == -INFINITY) ? 0.f : z1 * ex2(m1 - n1);
    m0 = n0;
    m1 = n1;
    const float s0 = (m0 == -INFINITY) ? 0.f : -m0, s1 = (m1 == -INFINITY) ? 0.f : -m1;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      z0 += ex2(c[nt][0] + s0) + ex2(c[nt][1] + s0);
      z1 += ex2(c[nt][2] + s1) + ex2(c[nt][3] + s1);
    }
    __syncthreads();
  }
  // combine the 4 lanes of each quad (fixed order)
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    const float om0 = __shfl_xor_sync(0xFFFFFFFFu, m0, o), oz0 = __shfl_xor_sync(0xFFFFFFFFu, z0, o);
    const float om1 = __shfl_xor_sync(0xFFFFFFFFu, m1, o), oz1 = __shfl_xor_sync(0xFFFFFFFFu, z1, o);
    float M = fmaxf(m0, om0);
    z0 = (M == -INFINITY) ? 0.f : z0 * ex2(m0 - M) + oz0 * ex2(om0 - M);
    m0 = M;
    M = fmaxf(m1, om1);
    z1 = (M == -INFINITY) ? 0.f : z1 * ex2(m1 - M) + oz1 * ex2(om1 - M);
    m1 = M;
  }
  if (t == 0) {
    float* mz = at<float>(dp, rs.mz_off) + (int64_t)chunk * LASTQ * 2;
    mz[2 * r0] = m0;
    mz[2 * r0 + 1] = z0;
    mz[2 * r1] = m1;
    mz[2 * r1 + 1] = z1;
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

// Pass 2: probabilities, vertical sums of owned keys, slash sums of owned offsets.
__global__ void __launch_bounds__(LQ_THREADS) lastq_pass2(DevPlan dp, const __nv_bfloat16* Q, int64_t qh,
                                                          int64_t qr, const void* K, int64_t kh, int64_t kr) {
  extern __shared__ uint8_t lq_raw[];
  LqSmem& sm = *reinterpret_cast<LqSmem*>(lq_raw);
  float* sacc = reinterpret_cast<float*>(lq_raw + sizeof(LqSmem));
  const RowSet& rs = at<const RowSet>(dp, dp.lay.rowsets)[blockIdx.y];
  const int chunk = blockIdx.x;
  if (chunk >= rs.n_chunks) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  load_q(sm, rs, Q, qh, qr);
  const float* stg = at<const float>(dp, rs.stat_off);
  for (int r = threadIdx.x; r < LASTQ; r += LQ_THREADS) {
    sm.stat[r][0] = stg[2 * r];
    sm.stat[r][1] = stg[2 * r + 1];
  }
  const KeySrc ks = key_src(dp, rs, K, kh, kr);
  const bool slash = rs.slash_hi > rs.slash_lo;
  const int span64 = slash ? (rs.span + KB - 1) / KB * KB : 0;
  const int64_t own0 = (int64_t)chunk * rs.chunk, own1 = std::min<int64_t>(own0 + rs.chunk, rs.key_hi);
  const int64_t c0 = std::max<int64_t>(0, own0 - span64);
  const int nblk = (int)((own1 - c0 + KB - 1) / KB);
  int32_t min_rc = 0x7fffffff, max_rc = -0x7fffffff;
  bool contig = true;  // row coordinates rcs[r] = rcs[0] + r: each offset is one diagonal of a block
  for (int r = 0; r < rs.n_rows; ++r) {
    min_rc = min(min_rc, rs.rcs[r]);
    max_rc = max(max_rc, rs.rcs[r]);
    contig = contig && rs.rcs[r] == rs.rcs[0] + r;
  }
  const int64_t obase = (int64_t)min_rc - (own0 + rs.chunk - 1);
  const int64_t ocount = (int64_t)max_rc - c0 - obase + 1;
  if (slash)
    for (int64_t i = threadIdx.x; i < ocount && i < dp.sacc_n; i += LQ_THREADS) sacc[i] = 0.f;
  load_kblock(sm, 0, ks, c0, own1);
  cp_async_commit();
  __syncthreads();
  uint32_t af[8][4];
  load_afrag(sm, af);
  const int r0 = warp * 16 + g, r1 = r0 + 8;
  const int32_t p0 = sm.rows[r0], p1 = sm.rows[r1];
  const float M0 = sm.stat[r0][0], I0 = sm.stat[r0][1], M1 = sm.stat[r1][0], I1 = sm.stat[r1][1];
  float* vout = at<float>(dp, rs.v_off);
  for (int b = 0; b < nblk; ++b) {
    const int64_t j0 = c0 + (int64_t)b * KB;
    if (b + 1 < nblk) load_kblock(sm, (b + 1) & 1, ks, j0 + KB, own1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    float c[8][4];
    block_logits(sm, b & 1, af, c);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = nt * 8 + 2 * t + (e & 1);
        const bool top = e < 2;
        const int32_t kp = sm.kpos[b & 1][col];
        const int32_t rp = top ? p0 : p1;
        float a = 0.f;
        if (kp <= rp) {
          const float x = (c[nt][e] * dp.scale) * LOG2E;
          a = ex2(x - (top ? M0 : M1)) * (top ? I0 : I1);
        }
        sm.a[(top ? r0 : r1) * (KB + 1) + col] = a;
      }
    }
    __syncthreads();
    // vertical sums of owned keys
    if (threadIdx.x < KB) {
      const int col = threadIdx.x;
      const int64_t j = j0 + col;
      if (j >= own0 && j < own1) {
        float s = 0.f;
        for (int r = 0; r < LASTQ; ++r) s += sm.a[r * (KB + 1) + col];
        vout[j] = s;
      }
    }
    // slash sums: offsets touched by this block, rows in order
    if (slash && contig) {
      // offset o = rcs[0] + d - j0 collects the elements (r, r - d) of diagonal d; one thread
      // per diagonal, rows ascending (the order of the general loop below)
      const bool inside = j0 >= rs.slash_lo && j0 + KB <= rs.slash_hi;
      const int n_rows = rs.n_rows;
      for (int dd = threadIdx.x; dd < n_rows + KB - 1; dd += LQ_THREADS) {
        const int d = dd - (KB - 1);
        const int64_t si = (int64_t)min_rc + d - j0 - obase;
        if (si < 0 || si >= dp.sacc_n) continue;
        const int r_lo = max(0, d), r_hi = min(n_rows, KB + d);
        float acc = 0.f;
        if (inside) {
          for (int r = r_lo; r < r_hi; ++r) acc += sm.a[r * (KB + 1) + (r - d)];
        } else {
          for (int r = r_lo; r < r_hi; ++r) {
            const int64_t j = j0 + (r - d);
            if (j < rs.slash_lo || j >= rs.slash_hi) continue;
            acc += sm.a[r * (KB + 1) + (r - d)];
          }
        }
        sacc[si] += acc;
      }
    } else if (slash) {
      const int64_t olo = (int64_t)min_rc - (j0 + KB - 1), ohi = (int64_t)max_rc - j0;
      for (int64_t o = olo + threadIdx.x; o <= ohi; o += LQ_THREADS) {
        const int64_t si = o - obase;
        if (si < 0 || si >= dp.sacc_n) continue;
        float s = 0.f;
        for (int r = 0; r < rs.n_rows; ++r) {
          const int64_t cc = (int64_t)sm.rcs[r] - o - j0;
          if (cc < 0 || cc >= KB) continue;
          const int64_t j = j0 + cc;
          if (j < rs.slash_lo || j >= rs.slash_hi) continue;
          s += sm.a[r * (KB + 1) + (int)cc];
        }
        sacc[si] += s;
      }
    }
    __syncthreads();
  }
  if (slash) {
    float* sout = at<float>(dp, rs.s_off);
    // owned offsets: the last row's key max_rc - o lies in [own0, own0 + chunk)
    for (int64_t i = threadIdx.x; i < rs.chunk; i += LQ_THREADS) {
      const int64_t j = own0 + i;
      const int64_t o = (int64_t)max_rc - j;
      if (o < 0 || o >= dp.L) continue;
      const int64_t si = o - obase;
      sout[o] = (si >= 0 && si < dp.sacc_n) ? sacc[si] : 0.f;
    }
  }
}

// ---------------------------------------------------------------------------------------
// top-k selection
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int NT>
__device__ __forceinline__ int block_scan_excl(int x, int* sh, int* total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int v = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xFFFFFFFFu, v, o);
    if (lane >= o) v += y;
  }
  if (lane == 31) sh[w] = v;
  __syncthreads();
  if (w == 0) {
    int s = lane < NW ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xFFFFFFFFu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < NW) sh[lane] = s;
  }
  __syncthreads();
  const int before = w ? sh[w - 1] : 0;
  *total = sh[NW - 1];
  __syncthreads();
  return before + v - x;
}

// Selects the k largest keys of n (ties: lower index) and writes their indices, ascending.
// `key(i)` returns the order key of candidate i.  NT threads cooperate.
template <int NT, typename KeyF, typename OutF>
__device__ void select_topk(int n, int k, KeyF key, OutF emit, uint32_t* hist, int* scan_sh) {
  if (k <= 0 || n <= 0) return;
  if (k >= n) {
    for (int i = threadIdx.x; i < n; i += NT) emit(i, i);
    return;
  }
  uint32_t prefix = 0, pmask = 0;
  int remaining = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += NT) hist[i] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += NT) {
      const uint32_t u = key(i);
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int cum = 0, sel = 0;
      for (int d = 255; d >= 0; --d) {
        const int h = (int)hist[d];
        if (cum + h >= remaining) {
          sel = d;
          break;
        }
        cum += h;
      }
      hist[256] = (uint32_t)sel;
      hist[257] = (uint32_t)(remaining - cum);
    }
    __syncthreads();
    prefix |= hist[256] << shift;
    pmask |= 255u << shift;
    remaining = (int)hist[257];
    __syncthreads();
  }
  const uint32_t T = prefix;  // key of the k-th largest; `remaining` ties at T are kept
  const int per = (n + NT - 1) / NT;
  const int i0 = min(n, (int)threadIdx.x * per), i1 = min(n, i0 + per);
  int gt = 0, eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t u = key(i);
    gt += u > T;
    eq += u == T;
  }
  int tg, te;
  const int gt_before = block_scan_excl<NT>(gt, scan_sh, &tg);
  const int eq_before = block_scan_excl<NT>(eq, scan_sh, &te);
  int o = gt_before + min(eq_before, remaining);
  int eq_seen = eq_before;
  for (int i = i0; i < i1; ++i) {
    const uint32_t u = key(i);
    if (u > T) {
      emit(o++, i);
    } else if (u == T && eq_seen < remaining) {
      emit(o++, i);
      ++eq_seen;
    } else if (u == T) {
      ++eq_seen;
    }
  }
}

constexpr int TK_THREADS = 1024;

__global__ void __launch_bounds__(TK_THREADS) topk_jobs_kernel(DevPlan dp) {
  __shared__ uint32_t hist[258];
  __shared__ int scan_sh[32];
  const TopkJob& jb = at<const TopkJob>(dp, dp.lay.jobs)[blockIdx.x];
  const float* sc = at<const float>(dp, jb.score_off) + jb.lo;
  int32_t* out = at<int32_t>(dp, jb.out_off);
  const int32_t* perm = at<const int32_t>(dp, dp.lay.perm2d);
  const int n = max(0, jb.hi - jb.lo);
  const int lo = jb.lo;
  const bool map = jb.map_k2d != 0;
  select_topk<TK_THREADS>(
      n, jb.k, [&](int i) { return order_key(sc[i]); },
      [&](int o, int i) { out[o] = map ? perm[lo + i] : lo + i; }, hist, scan_sh);
  if (threadIdx.x == 0) *at<int32_t>(dp, jb.cnt_off) = min(jb.k, n);
}

// ---------------------------------------------------------------------------------------
// block-sparse estimation
// ---------------------------------------------------------------------------------------
// mean of each 64-row block, fp32, rows summed in order
// Mean of each 64-row block of K (grid rows y < Hkv: KV head y) and of Q (rows y >= Hkv: the
// (y - Hkv)-th block-sparse query head), one launch for both.  One CTA of 256 threads per
// block: 16 lanes cover a 256-byte row with 16-byte loads, 16 row groups take rows g, g + 16,
// g + 32, g + 48, and the 16 partial sums of each column are added in row-group order.
constexpr int POOL_THREADS = 256;
__global__ void __launch_bounds__(POOL_THREADS) pool_kernel(DevPlan dp, const __nv_bfloat16* Q, int64_t qh,
                                                            int64_t qr, const __nv_bfloat16* K, int64_t kh,
                                                            int64_t kr) {
  __shared__ float part[16][D + 4];
  const bool q_side = (int)blockIdx.y >= dp.Hkv;
  int h = blockIdx.y;
  if (q_side) {
    const HeadStatic* hs = at<const HeadStatic>(dp, dp.lay.heads);
    int seen = -1;
    for (h = 0; h < dp.Hq; ++h)
      if (hs[h].kind == MSA_BLOCK && ++seen == (int)blockIdx.y - dp.Hkv) break;
    if (h >= dp.Hq) return;
  }
  float* out = q_side ? at<float>(dp, at<const HeadStatic>(dp, dp.lay.heads)[h].qbar_off)
                      : at<float>(dp, dp.lay.kbar) + (int64_t)h * dp.nb * D;
  const __nv_bfloat16* X = q_side ? Q + (int64_t)h * qh : K + (int64_t)h * kh;
  const int64_t xr = q_side ? qr : kr;
  const int sub = threadIdx.x & 15, g = threadIdx.x >> 4;
  auto load = [&](int b, uint4 (&v)[4]) {
    const __nv_bfloat16* src = X + (int64_t)b * BLK * xr + sub * 8;
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __ldg(reinterpret_cast<const uint4*>(src + (int64_t)(g + 16 * i) * xr));
  };
  uint4 nxt[4];
  if ((int)blockIdx.x < dp.nb) load(blockIdx.x, nxt);
  for (int b = blockIdx.x; b < dp.nb; b += gridDim.x) {
    uint4 v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = nxt[i];
    if (b + (int)gridDim.x < dp.nb) load(b + gridDim.x, nxt);  // next block's rows in flight meanwhile
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&v[i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p2[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) part[g][sub * 8 + e] = acc[e];
    __syncthreads();
    if (threadIdx.x < D) {
      float t = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) t += part[j][threadIdx.x];
      out[(int64_t)b * D + threadIdx.x] = t * (1.f / BLK);
    }
    __syncthreads();
  }
}

constexpr int BT_THREADS = 256;

// one CTA per (query block, block-sparse head): pooled logits of key blocks c <= b, then top-k
__global__ void __launch_bounds__(BT_THREADS) block_topk_kernel(DevPlan dp) {
  extern __shared__ uint32_t bt_keys[];
  __shared__ uint32_t hist[258];
  __shared__ int scan_sh[32];
  __shared__ __align__(16) float qb[D];
  const int b = blockIdx.x;
  int h = 0;  // the blockIdx.y-th block-sparse head
  {
    const HeadStatic* all = at<const HeadStatic>(dp, dp.lay.heads);
    int seen = -1;
    for (h = 0; h < dp.Hq; ++h)
      if (all[h].kind == MSA_BLOCK && ++seen == (int)blockIdx.y) break;
    if (h >= dp.Hq) return;
  }
  const HeadStatic& hs = at<const HeadStatic>(dp, dp.lay.heads)[h];
  const float* qbar = at<const float>(dp, hs.qbar_off) + (int64_t)b * D;
  const float* kbar = at<const float>(dp, dp.lay.kbar) + (int64_t)hs.kvh * dp.nb * D;
  if (threadIdx.x < D) qb[threadIdx.x] = qbar[threadIdx.x];
  __syncthreads();
  const int n = b + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float4 q4 = reinterpret_cast<const float4*>(qb)[lane];
  for (int c = warp; c < n; c += BT_THREADS / 32) {
    const float4 k4 = reinterpret_cast<const float4*>(kbar + (int64_t)c * D)[lane];
    float s = q4.x * k4.x + q4.y * k4.y + q4.z * k4.z + q4.w * k4.w;
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    if (lane == 0) bt_keys[c] = order_key(s * dp.scale);
  }
  __syncthreads();
  // k per row: fixed top-k or ceil(budget * (b + 1)), clipped to [1, b + 1] and the capacity
  int k = hs.blk_fixed > 0 ? hs.blk_fixed : (int)ceil(hs.blk_budget * (double)(b + 1));
  k = min(max(1, min(k, n)), hs.blk_kmax);
  int32_t* out = at<int32_t>(dp, hs.blk_list_off) + (int64_t)b * hs.blk_kmax;
  select_topk<BT_THREADS>(
      n, k, [&](int i) { return bt_keys[i]; }, [&](int o, int i) { out[o] = i; }, hist, scan_sh);
  if (threadIdx.x == 0) at<int32_t>(dp, hs.blk_cnt_off)[b] = k;
}

}  // namespace

// ---------------------------------------------------------------------------------------
cudaError_t launch_group_k(const DevPlan& dp, const void* K, const msa_strides& s, cudaStream_t st) {
  count_launches(1);
  group_rows_kernel<<<sm_count() * 8, 256, 0, st>>>(dp, static_cast<const __nv_bfloat16*>(K), s.k_head, s.k_row,
                                                   at<__nv_bfloat16>(dp, dp.lay.k2d));
  return cudaGetLastError();
}

cudaError_t launch_group_v(const DevPlan& dp, const void* V, const msa_strides& s, cudaStream_t st) {
  count_launches(1);
  group_rows_kernel<<<sm_count() * 8, 256, 0, st>>>(dp, static_cast<const __nv_bfloat16*>(V), s.v_head, s.v_row,
                                                   at<__nv_bfloat16>(dp, dp.lay.v2d));
  return cudaGetLastError();
}

cudaError_t launch_lastq(const DevPlan& dp, const void* Q, const void* K, const msa_strides& s, cudaStream_t st) {
  cudaError_t e;
  if (dp.has2d && (e = launch_group_k(dp, K, s, st)) != cudaSuccess) return e;
  const size_t smem1 = sizeof(LqSmem);
  const size_t smem2 = sizeof(LqSmem) + sizeof(float) * SACC_MAX;
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (device_pending(configured, dev)) {
    if ((e = cudaFuncSetAttribute(lastq_pass1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(lastq_pass2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2)) != cudaSuccess)
      return e;
    mark_device(configured, dev);
  }
  if (dp.sacc_n < 0 || dp.sacc_n > SACC_MAX) return cudaErrorInvalidValue;
  const size_t smem2_used = sizeof(LqSmem) + sizeof(float) * (size_t)dp.sacc_n;
  const dim3 grid(dp.max_chunks, dp.n_rowsets);
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(Q);
  count_launches(3);
  lastq_pass1<<<grid, LQ_THREADS, smem1, st>>>(dp, q, s.q_head, s.q_row, K, s.k_head, s.k_row);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  lastq_combine<<<dp.n_rowsets, LASTQ, 0, st>>>(dp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  lastq_pass2<<<grid, LQ_THREADS, smem2_used, st>>>(dp, q, s.q_head, s.q_row, K, s.k_head, s.k_row);
  return cudaGetLastError();
}

cudaError_t launch_topk_jobs(const DevPlan& dp, cudaStream_t st) {
  count_launches(1);
  topk_jobs_kernel<<<dp.n_jobs, TK_THREADS, 0, st>>>(dp);
  return cudaGetLastError();
}

cudaError_t launch_block_estimate(const DevPlan& dp, const void* Q, const void* K, const msa_strides& s,
                                  cudaStream_t st) {
  // about eight 256-thread blocks per SM in all, each walking several 64-row blocks
  const int gx = std::max(1, std::min(dp.nb, sm_count() * 8 / std::max(1, dp.Hkv + dp.n_block_heads)));
  count_launches(2);
  pool_kernel<<<dim3(gx, dp.Hkv + dp.n_block_heads), POOL_THREADS, 0, st>>>(
      dp, static_cast<const __nv_bfloat16*>(Q), s.q_head, s.q_row, static_cast<const __nv_bfloat16*>(K), s.k_head,
      s.k_row);
  const size_t smem = sizeof(uint32_t) * (size_t)dp.nb;
  static size_t configured = 0;
  if (smem > 48 * 1024 && smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(block_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  block_topk_kernel<<<dim3(dp.nb, std::max(1, dp.n_block_heads)), BT_THREADS, smem, st>>>(dp);
  return cudaGetLastError();
}

}  // namespace msa
