// Share of the dense attention weights a query row needs for a given recall (MMInference
// summary page, attention analysis: in video-language models 95 % of the attention mass lies in
// 1.79 % of the weights, against 5.78 % in language models).
//
// For query row i of head h, the dense causal weights w_j = softmax_j(q_i . k_j * scale),
// j <= i, sorted descending; the count is the fewest weights whose sum reaches recall * sum_j w_j
// (ties broken arbitrarily: equal weights are interchangeable).  One CTA per sampled row finds
// it without sorting: a radix select over the order-preserving 32-bit image of the logits,
// descending, with a histogram of counts and weight sums per 8-bit digit (four passes that
// recompute the logits), gives the logit at which the running sum from the top crosses the
// target; the count is the number of larger logits plus the fewest copies of that logit needed.
// Logits in fp32 (fp32 dot product), weights and sums in fp64.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "msa_internal.h"

namespace msa {

namespace {

constexpr int WS_THREADS = 256;

__device__ __forceinline__ uint32_t ws_key(float f) {  // order-preserving image of an fp32 value
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ws_unkey(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

struct WsArgs {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  int64_t q_head, q_row, k_head, k_row;
  int64_t L;
  int32_t Hq, group;
  float scale;
  const int32_t* heads;
  const int32_t* rows;
  double recall;
  long long* counts;
};

__global__ void __launch_bounds__(WS_THREADS) weight_share_kernel(const WsArgs a) {
  __shared__ float q[D];
  __shared__ unsigned long long h_cnt[256];
  __shared__ double h_w[256];
  __shared__ float red_f[WS_THREADS / 32];
  __shared__ double red_d[WS_THREADS / 32];
  __shared__ uint32_t sel_bin;
  __shared__ double sel_acc;
  __shared__ unsigned long long sel_cnt;
  const int s = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int32_t h = a.heads[s], i = a.rows[s];
  if (h < 0 || h >= a.Hq || i < 0 || i >= a.L) {  // out of range: reported as -1
    if (t == 0) a.counts[s] = -1;
    return;
  }
  const __nv_bfloat16* qr = a.Q + (int64_t)h * a.q_head + (int64_t)i * a.q_row;
  const __nv_bfloat16* kb = a.K + (int64_t)(h / a.group) * a.k_head;
  if (t < D) q[t] = __bfloat162float(qr[t]);
  __syncthreads();
  auto logit = [&](int64_t j) -> float {
    const uint4* kr = reinterpret_cast<const uint4*>(kb + j * a.k_row);
    float acc = 0.f;
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {
      const uint4 v = __ldg(kr + c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc = fmaf(q[8 * c + 2 * e], __uint_as_float(w[e] << 16), acc);
        acc = fmaf(q[8 * c + 2 * e + 1], __uint_as_float(w[e] & 0xFFFF0000u), acc);
      }
    }
    return acc * a.scale;
  };
  // pass 0: the row's max logit and its softmax normaliser
  float mx = -INFINITY;
  for (int64_t j = t; j <= i; j += WS_THREADS) mx = fmaxf(mx, logit(j));
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  if (lane == 0) red_f[warp] = mx;
  __syncthreads();
  mx = red_f[0];
  for (int w = 1; w < WS_THREADS / 32; ++w) mx = fmaxf(mx, red_f[w]);
  double z = 0.0;
  for (int64_t j = t; j <= i; j += WS_THREADS) z += exp((double)logit(j) - (double)mx);
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xFFFFFFFFu, z, o);
  if (lane == 0) red_d[warp] = z;
  __syncthreads();
  z = 0.0;
  for (int w = 0; w < WS_THREADS / 32; ++w) z += red_d[w];
  const double target = a.recall * z;
  // radix select from the most significant digit: the key at which the running weight sum,
  // taken from the largest logits down, first reaches the target
  uint32_t prefix = 0u, mask = 0u;
  double above = 0.0;             // weight of the keys above the current digit's range
  unsigned long long n_above = 0; // their number
  for (int d = 3; d >= 0; --d) {
    h_cnt[t] = 0ull;
    h_w[t] = 0.0;
    __syncthreads();
    for (int64_t j = t; j <= i; j += WS_THREADS) {
      const float x = logit(j);
      const uint32_t u = ws_key(x);
      if ((u & mask) != prefix) continue;
      const int bin = (int)((u >> (8 * d)) & 255u);
      atomicAdd(&h_cnt[bin], 1ull);
      atomicAdd(&h_w[bin], exp((double)x - (double)mx));
    }
    __syncthreads();
    if (t == 0) {
      double acc = above;
      unsigned long long cnt = n_above;
      int b = 255, last = -1;
      for (; b >= 0; --b) {
        if (h_cnt[b] == 0ull) continue;
        last = b;
        if (acc + h_w[b] >= target) break;
        acc += h_w[b];
        cnt += h_cnt[b];
      }
      if (b < 0) {  // rounding left the target just out of reach: the last non-empty bin
        b = last;
        acc -= h_w[b];
        cnt -= h_cnt[b];
      }
      sel_bin = (uint32_t)b;
      sel_acc = acc;
      sel_cnt = cnt;
    }
    __syncthreads();
    prefix |= sel_bin << (8 * d);
    mask |= 255u << (8 * d);
    above = sel_acc;
    n_above = sel_cnt;
    __syncthreads();
  }
  if (t == 0) {
    // every key equal to `prefix` has the same weight; take the fewest that reach the target
    const double w = exp((double)ws_unkey(prefix) - (double)mx);
    const unsigned long long tie = h_cnt[prefix & 255u];
    unsigned long long need = w > 0.0 ? (unsigned long long)ceil((target - above) / w) : tie;
    if (need < 1ull) need = 1ull;
    if (need > tie) need = tie;
    a.counts[s] = (long long)(n_above + need);
  }
}

}  // namespace

}  // namespace msa

using namespace msa;

extern "C" msa_status msa_weight_share(const void* Q, const void* K, int64_t L, int32_t Hq, int32_t Hkv,
                                       const msa_strides* strides, float scale, const int32_t* heads,
                                       const int32_t* rows, int32_t n, double recall, int64_t* counts,
                                       void* stream) {
  if (!Q || !K || !strides || !heads || !rows || !counts || n < 0) return MSA_ERR_INVALID_ARG;
  if (!(recall > 0.0 && recall <= 1.0) || !(scale > 0.f)) return MSA_ERR_INVALID_ARG;
  if (L <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return MSA_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K)) % 16) return MSA_ERR_ALIGN;
  if (strides->q_row % 8 || strides->k_row % 8 || strides->q_head % 8 || strides->k_head % 8) return MSA_ERR_ALIGN;
  if (n == 0) return MSA_OK;
  WsArgs a;
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.K = static_cast<const __nv_bfloat16*>(K);
  a.q_head = strides->q_head;
  a.q_row = strides->q_row;
  a.k_head = strides->k_head;
  a.k_row = strides->k_row;
  a.L = L;
  a.Hq = Hq;
  a.group = Hq / Hkv;
  a.scale = scale;
  a.heads = heads;
  a.rows = rows;
  a.recall = recall;
  a.counts = reinterpret_cast<long long*>(counts);
  count_launches(1);
  weight_share_kernel<<<n, WS_THREADS, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}
