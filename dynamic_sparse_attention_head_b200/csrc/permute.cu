// Permutation gathers (MMInference "core discovery": row-wise permutation groups
// same-modality queries, column-wise permutation gathers the selected keys, 2D permutation
// groups keys by modality) and the inverse scatter of the output.  Bandwidth-bound row
// copies: 16 lanes move one 256-byte row with 16-byte vector loads and stores.
#include <cuda_bf16.h>
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

__device__ __forceinline__ void copy_row(uint4* dst, const uint4* src, int sub) {
  dst[sub] = src ? __ldg(src + sub) : make_uint4(0, 0, 0, 0);
}

// Permuted Q of every head with row classes: slice rows [qrow0, qrow0 + padded(nrows)).
__global__ void permute_q_kernel(DevPlan dp, const __nv_bfloat16* Q, int64_t qh, int64_t qr) {
  const int h = blockIdx.y;
  const HeadStatic& hs = at<const HeadStatic>(dp, dp.lay.heads)[h];
  if (hs.q_slice < 0) return;
  __nv_bfloat16* dst = at<__nv_bfloat16>(dp, dp.lay.qp) + hs.q_slice * (int64_t)dp.LP * D;
  const int sub = threadIdx.x & 15;
  const int64_t lane_row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
  const int64_t stride = ((int64_t)gridDim.x * blockDim.x) >> 4;
  for (int c = hs.class0; c < hs.class0 + hs.n_classes; ++c) {
    const ClassStatic& cs = at<const ClassStatic>(dp, dp.lay.classes)[c];
    if (!(cs.flags & CF_PERMUTED)) continue;
    const ClassDyn cd = at<const ClassDyn>(dp, dp.lay.class_dyn)[cs.dyn];
    const int32_t* rl = at<const int32_t>(dp, cs.rows_off);
    const int64_t padded = (int64_t)(cd.nrows + TILE - 1) / TILE * TILE;
    for (int64_t r = lane_row; r < padded; r += stride) {
      const uint4* src = r < cd.nrows ? reinterpret_cast<const uint4*>(Q + h * qh + (int64_t)rl[r] * qr) : nullptr;
      copy_row(reinterpret_cast<uint4*>(dst + (cd.qrow0 + r) * D), src, sub);
    }
  }
}

// Gathered key / value rows of every class with a gathered list, zero padded to 128.
__global__ void gather_x_kernel(DevPlan dp, const __nv_bfloat16* K, int64_t kh, int64_t kr, const __nv_bfloat16* V,
                                int64_t vh, int64_t vr) {
  const int h = blockIdx.y;
  const HeadStatic& hs = at<const HeadStatic>(dp, dp.lay.heads)[h];
  if (hs.x_slice < 0) return;
  const int64_t slice = hs.x_slice * (int64_t)dp.x_rows * D;
  __nv_bfloat16* xk = at<__nv_bfloat16>(dp, dp.lay.xk) + slice;
  __nv_bfloat16* xv = at<__nv_bfloat16>(dp, dp.lay.xv) + slice;
  const int sub = threadIdx.x & 15;
  const int64_t lane_row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
  const int64_t stride = ((int64_t)gridDim.x * blockDim.x) >> 4;
  for (int c = hs.class0; c < hs.class0 + hs.n_classes; ++c) {
    const ClassStatic& cs = at<const ClassStatic>(dp, dp.lay.classes)[c];
    if (!(cs.flags & CF_X)) continue;
    const ClassDyn cd = at<const ClassDyn>(dp, dp.lay.class_dyn)[cs.dyn];
    const int32_t* xp = at<const int32_t>(dp, cs.x_pos_off);
    const int64_t padded = (int64_t)(cd.x_len + TILE - 1) / TILE * TILE;
    for (int64_t i = lane_row; i < padded; i += stride) {
      const int64_t p = i < cd.x_len ? xp[i] : -1;
      const int64_t row = (cs.x_row0 + i) * D;
      copy_row(reinterpret_cast<uint4*>(xk + row),
               p >= 0 ? reinterpret_cast<const uint4*>(K + (int64_t)hs.kvh * kh + p * kr) : nullptr, sub);
      copy_row(reinterpret_cast<uint4*>(xv + row),
               p >= 0 ? reinterpret_cast<const uint4*>(V + (int64_t)hs.kvh * vh + p * vr) : nullptr, sub);
    }
  }
}

// Modality-grouped K and V (2D-boundary heads): dst[h][r] = src[h][perm2d[r]]
__global__ void group_kv_kernel(DevPlan dp, const __nv_bfloat16* K, int64_t kh, int64_t kr, const __nv_bfloat16* V,
                                int64_t vh, int64_t vr) {
  const int32_t* perm = at<const int32_t>(dp, dp.lay.perm2d);
  __nv_bfloat16* k2 = at<__nv_bfloat16>(dp, dp.lay.k2d);
  __nv_bfloat16* v2 = at<__nv_bfloat16>(dp, dp.lay.v2d);
  const int64_t total = (int64_t)dp.Hkv * dp.L;
  const int sub = threadIdx.x & 15;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4; i < total;
       i += ((int64_t)gridDim.x * blockDim.x) >> 4) {
    const int64_t h = i / dp.L, r = i % dp.L;
    const int64_t p = perm[r];
    copy_row(reinterpret_cast<uint4*>(k2 + i * D), reinterpret_cast<const uint4*>(K + h * kh + p * kr), sub);
    copy_row(reinterpret_cast<uint4*>(v2 + i * D), reinterpret_cast<const uint4*>(V + h * vh + p * vr), sub);
  }
}

// O[h][pos(r)] = O_perm[h][qrow0 + r] for every class row.
__global__ void unpermute_kernel(DevPlan dp, __nv_bfloat16* O, int64_t oh, int64_t orow) {
  const int h = blockIdx.y;
  const HeadStatic& hs = at<const HeadStatic>(dp, dp.lay.heads)[h];
  const __nv_bfloat16* op = at<const __nv_bfloat16>(dp, dp.lay.op) + (int64_t)h * dp.LP * D;
  const int sub = threadIdx.x & 15;
  const int64_t lane_row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
  const int64_t stride = ((int64_t)gridDim.x * blockDim.x) >> 4;
  for (int c = hs.class0; c < hs.class0 + hs.n_classes; ++c) {
    const ClassStatic& cs = at<const ClassStatic>(dp, dp.lay.classes)[c];
    const ClassDyn cd = at<const ClassDyn>(dp, dp.lay.class_dyn)[cs.dyn];
    const bool perm = (cs.flags & CF_PERMUTED) != 0;
    const int32_t* rl = at<const int32_t>(dp, cs.rows_off);
    for (int64_t r = lane_row; r < cd.nrows; r += stride) {
      const int64_t pos = perm ? rl[r] : r;
      copy_row(reinterpret_cast<uint4*>(O + h * oh + pos * orow),
               reinterpret_cast<const uint4*>(op + (cd.qrow0 + r) * D), sub);
    }
  }
}

}  // namespace

cudaError_t launch_permute(const DevPlan& dp, const void* Q, const void* K, const void* V, const msa_strides& s,
                           bool with_q, cudaStream_t st) {
  const int bx = std::max(1, sm_count() * 4 / std::max(1, dp.Hq)) ;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(Q);
  const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(K);
  const __nv_bfloat16* v = static_cast<const __nv_bfloat16*>(V);
  if (with_q && dp.n_qslices > 0) {
    count_launches(1);
    permute_q_kernel<<<dim3(bx * 2, dp.Hq), 256, 0, st>>>(dp, q, s.q_head, s.q_row);
  }
  if (dp.n_xslices > 0) {
    count_launches(1);
    gather_x_kernel<<<dim3(bx, dp.Hq), 256, 0, st>>>(dp, k, s.k_head, s.k_row, v, s.v_head, s.v_row);
  }
  if (dp.has2d) {
    count_launches(1);
    group_kv_kernel<<<sm_count() * 8, 256, 0, st>>>(dp, k, s.k_head, s.k_row, v, s.v_head, s.v_row);
  }
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const DevPlan& dp, void* O, const msa_strides& s, cudaStream_t st) {
  const int bx = std::max(1, sm_count() * 8 / std::max(1, dp.Hq));
  count_launches(1);
  unpermute_kernel<<<dim3(bx, dp.Hq), 256, 0, st>>>(dp, static_cast<__nv_bfloat16*>(O), s.o_head, s.o_row);
  return cudaGetLastError();
}

}  // namespace msa
