// Gated RMS-norm on the delta-rule layer output (Agnes-3.0-Flash Preview model
// card, 架构 table: "gated RMS-norm"):
//   y = x / sqrt(mean(x^2) + eps) * w * SiLU(z)      per 128-channel row.
//
// HBM-bound: x and z are read once, y written once. 16 threads own one row
// (8 channels = one 16-byte bf16 vector each); the sum of squares is a
// 16-lane shuffle reduction. A 16-thread group handles kRowsPerGroup rows
// (interleaved, so a warp reads two adjacent rows at a time) and issues all of
// their loads before it computes.
#include "gdn_common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kNormThreads = 256;
constexpr int kGroups = kNormThreads / 16;
// rows per 16-thread group: all of their x and z vectors stay in registers
template <class Tx, class Tz>
__host__ __device__ constexpr int rows_per_group() {
  return sizeof(Tx) + sizeof(Tz) == 4 ? 4 : 2;
}

template <class Tx, class Tz, class Tw, class Ty>
__global__ void __launch_bounds__(kNormThreads, 3)
gated_rmsnorm_kernel(const Tx* __restrict__ x, const Tz* __restrict__ z,
                     const Tw* __restrict__ w, int64_t rows, float eps,
                     Ty* y) {
  constexpr int kRowsPerGroup = rows_per_group<Tx, Tz>();
  const int sub = threadIdx.x & 15;          // 8-channel slice of the row
  const int64_t r0 = (int64_t)blockIdx.x * (kGroups * kRowsPerGroup) + (threadIdx.x >> 4);
  Raw8<Tx> xr[kRowsPerGroup];
  Raw8<Tz> zr[kRowsPerGroup];
#pragma unroll
  for (int j = 0; j < kRowsPerGroup; ++j) {
    const int64_t r = r0 + (int64_t)j * kGroups;
    xr[j].zero();
    zr[j].zero();
    if (r < rows) {
      xr[j].load(x + r * kHeadDim + sub * 8);
      zr[j].load(z + r * kHeadDim + sub * 8);
    }
  }
  float wf[8];
  load8(w + sub * 8, wf);
#pragma unroll
  for (int j = 0; j < kRowsPerGroup; ++j) {
    const int64_t r = r0 + (int64_t)j * kGroups;
    float xf[8], zf[8];
    xr[j].to_f32(xf);
    zr[j].to_f32(zf);
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(xf[e], xf[e], ss);
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = rsqrtf(ss * (1.0f / kHeadDim) + eps);
    float out[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = xf[e] * inv * wf[e] * silu(zf[e]);
    if (r < rows) store8(y + r * kHeadDim + sub * 8, out);
  }
}

template <class Tx, class Tz, class Tw, class Ty>
cudaError_t launch_typed(const NormArgs& a) {
  constexpr int kRowsPerBlock = kGroups * rows_per_group<Tx, Tz>();
  const int64_t blocks = (a.rows + kRowsPerBlock - 1) / kRowsPerBlock;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  gated_rmsnorm_kernel<Tx, Tz, Tw, Ty><<<(unsigned)blocks, kNormThreads, 0, a.stream>>>(
      static_cast<const Tx*>(a.x), static_cast<const Tz*>(a.z),
      static_cast<const Tw*>(a.w), a.rows, a.eps, static_cast<Ty*>(a.y));
  return cudaGetLastError();
}

template <class Tx, class Tz, class Tw>
cudaError_t pick_y(const NormArgs& a) {
  return a.y_dtype == GDN_F32 ? launch_typed<Tx, Tz, Tw, float>(a)
                              : launch_typed<Tx, Tz, Tw, __nv_bfloat16>(a);
}
template <class Tx, class Tz>
cudaError_t pick_w(const NormArgs& a) {
  return a.w_dtype == GDN_F32 ? pick_y<Tx, Tz, float>(a)
                              : pick_y<Tx, Tz, __nv_bfloat16>(a);
}
template <class Tx>
cudaError_t pick_z(const NormArgs& a) {
  return a.z_dtype == GDN_F32 ? pick_w<Tx, float>(a)
                              : pick_w<Tx, __nv_bfloat16>(a);
}

}  // namespace

cudaError_t launch_gated_rmsnorm(const NormArgs& a) {
  if (a.rows == 0) return cudaSuccess;
  return a.x_dtype == GDN_F32 ? pick_z<float>(a) : pick_z<__nv_bfloat16>(a);
}

}  // namespace gdn
