// The float32 outputs of the block transforms, computed in double:
//
//   kq_transform            y = x K          (per 32-block, bf16 x)
//   kq_inverse_transform    x = y K^-1       (float32 y)
//   kq_fold_weight          W' = W K^-T      (bf16 W)
//   kq_transform16, kq_fold_weight16: the same with 16-element blocks
//
// (KroQuant review, "What carries the argument": K = G1 (x) ... (x) G5 with
// G = L U = [[b, c], [a b, a c + 1/b]], det G = 1, G^-1 = [[g11, -g01],
// [-g10, g00]]; the fold is Eq. 1's W T^-T.)  Every factor entry is formed
// in double from the float32 parameters (the inputs and the products a b,
// a c are exact there; 1/b is the correctly rounded double quotient), the
// five butterfly stages run in double and the result is rounded once to
// float32.  So the outputs carry the float32 rounding of a value within
// about 1e-15 of the sum of the terms' magnitudes: relative error at most
// 2^-24 except where a sum cancels by ten decimal orders.  The quantizer
// keeps its own float32 path; these calls serve round trips, the weight
// fold and the calibration's straight-through pass, which read the
// transformed values themselves.
//
// Layout: lane l of a warp takes unit j = 32 blockIdx.y + l (a 32-element
// block, or two 16-element blocks), holds its factors in registers and walks
// rows r = 4 blockIdx.x + warp, + 4 gridDim.x, ...; a warp's 32 lanes read
// 32 consecutive units of one row.  The arithmetic is about 320 double
// multiply-adds a unit (two a pair and stage) against 64 + 128 bytes of
// traffic.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "kq.h"
#include "kq_device.cuh"
#include "kq_internal.h"

namespace kq {
namespace {

enum ExactKind { kExactForward = 0, kExactInverse = 1, kExactFold = 2 };

constexpr int kExactThreads = 128;
constexpr int kExactRowsPerCta = kExactThreads / 32;

// Factor k of a block as the 2x2 matrix the row vector is multiplied by:
// f[0] f[1] / f[2] f[3] = row 0 / row 1.
template <int kKind>
__device__ __forceinline__ void exact_factor(float a, float b, float c, double (&f)[4]) {
  const double da = a, db = b, dc = c;
  const double g00 = db, g01 = dc, g10 = da * db, g11 = __fma_rn(da, dc, 1.0 / db);
  if (kKind == kExactForward) {
    f[0] = g00; f[1] = g01; f[2] = g10; f[3] = g11;
  } else if (kKind == kExactInverse) {
    f[0] = g11; f[1] = -g01; f[2] = -g10; f[3] = g00;
  } else {
    f[0] = g11; f[1] = -g10; f[2] = -g01; f[3] = g00;
  }
}

// kNf factors per block (5: one 32-block a unit; 4: two 16-blocks a unit,
// 24 parameters).  kF32In: float32 input (the inverse transform), else bf16.
template <int kNf, int kKind, bool kF32In>
__global__ void __launch_bounds__(kExactThreads)
    exact_transform_kernel(const void* __restrict__ x, int64_t M, int units,
                           const float* __restrict__ params, float* __restrict__ y) {
  constexpr int kSub = 32 >> kNf;                  // blocks per unit
  constexpr int kLen = 1 << kNf;                   // elements per block
  pdl_wait_then_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int j = blockIdx.y * 32 + lane;
  if (j >= units) return;
  double f[kSub][kNf][4];
  const float* p = params + (int64_t)j * (3 * kNf * kSub);
#pragma unroll
  for (int s = 0; s < kSub; ++s)
#pragma unroll
    for (int k = 0; k < kNf; ++k) {
      const float* q = p + 3 * (kNf * s + k);
      exact_factor<kKind>(q[0], q[1], q[2], f[s][k]);
    }
  for (int64_t r = (int64_t)blockIdx.x * kExactRowsPerCta + warp; r < M;
       r += (int64_t)gridDim.x * kExactRowsPerCta) {
    const int64_t g = r * units + j;
    double v[32];
    if constexpr (kF32In) {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(x) + g * 32);
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const float4 w = __ldcs(src + t);
        v[4 * t] = w.x; v[4 * t + 1] = w.y; v[4 * t + 2] = w.z; v[4 * t + 3] = w.w;
      }
    } else {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + g * 32);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint4 w = __ldcs(src + t);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[8 * t + 2 * i] = __uint_as_float(ws[i] << 16);
          v[8 * t + 2 * i + 1] = __uint_as_float(ws[i] & 0xFFFF0000u);
        }
      }
    }
    // Factor k acts on index bit kNf - 1 - k of its block: each pair of
    // indices that differ in that bit, as the row vector (v0, v1) times it.
#pragma unroll
    for (int s = 0; s < kSub; ++s)
#pragma unroll
      for (int k = 0; k < kNf; ++k) {
        const int h = 1 << (kNf - 1 - k);
#pragma unroll
        for (int i = 0; i < kLen; ++i) {
          if (i & h) continue;
          const double v0 = v[kLen * s + i], v1 = v[kLen * s + i + h];
          v[kLen * s + i] = __fma_rn(v1, f[s][k][2], v0 * f[s][k][0]);
          v[kLen * s + i + h] = __fma_rn(v1, f[s][k][3], v0 * f[s][k][1]);
        }
      }
    float4* dst = reinterpret_cast<float4*>(y + g * 32);
#pragma unroll
    for (int t = 0; t < 8; ++t)
      __stcs(dst + t, make_float4(__double2float_rn(v[4 * t]), __double2float_rn(v[4 * t + 1]),
                                  __double2float_rn(v[4 * t + 2]),
                                  __double2float_rn(v[4 * t + 3])));
  }
}

template <int kNf, int kKind, bool kF32In>
int launch_exact(const void* x, int64_t M, int64_t d, const float* params, float* y,
                 cudaStream_t st) {
  const DeviceInfo* di = nullptr;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != KQ_OK) return rc;
  const int64_t units = d / kBlock;
  const int64_t gy = (units + 31) / 32;
  if (gy > 65535) return KQ_ERR_INVALID;
  // About six CTAs of 128 threads per SM in all (three are resident at a
  // time), at most one row per warp.
  const int64_t want = std::max<int64_t>(1, (int64_t)di->sms * 6 / gy);
  const int64_t gx = std::min<int64_t>(want, (M + kExactRowsPerCta - 1) / kExactRowsPerCta);
  cudaError_t e = launch_pdl(exact_transform_kernel<kNf, kKind, kF32In>,
                             dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)),
                             dim3(kExactThreads), 0, st, x, M, static_cast<int>(units), params, y);
  if (e != cudaSuccess) return record_cuda_error(e);
  return KQ_OK;
}

}  // namespace

int exact_transform(int kind, int nf, bool f32_in, const void* x, int64_t M, int64_t d,
                    const float* params, float* y, cudaStream_t st) {
  if (nf == 5 && kind == kExactForward && !f32_in)
    return launch_exact<5, kExactForward, false>(x, M, d, params, y, st);
  if (nf == 5 && kind == kExactInverse && f32_in)
    return launch_exact<5, kExactInverse, true>(x, M, d, params, y, st);
  if (nf == 5 && kind == kExactFold && !f32_in)
    return launch_exact<5, kExactFold, false>(x, M, d, params, y, st);
  if (nf == 4 && kind == kExactForward && !f32_in)
    return launch_exact<4, kExactForward, false>(x, M, d, params, y, st);
  if (nf == 4 && kind == kExactFold && !f32_in)
    return launch_exact<4, kExactFold, false>(x, M, d, params, y, st);
  return KQ_ERR_INVALID;
}

}  // namespace kq
