// Online index estimation (MInference 1.0 "Approach"; MMInference "key machinery" and
// "core discovery"), the parts besides the last-query sweep (lastq.cu):
//  - the modality-grouped copy of K that 2D-boundary heads estimate and attend over;
//  - deterministic top-k (radix select on the order-preserving uint32 image of fp32;
//    ties go to the lower index), output sorted ascending;
//  - block-sparse: 64-token mean pooling of Q and K, pooled logits, per-row top-k.
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
