// Warp-per-block variant of the Kronecker quantizer (KQ_IMPL_WARP), kept as a
// measured comparator of the thread-per-block kernels.
//
// Lane l of a warp holds element l of a 32-element block.  The five factors
// act on the five bits of the in-block index (G1 on bit 4), so stage k mixes
// lane l with lane l ^ (1 << (4 - k)) through one __shfl_xor_sync:
//   y_l = x_l * G[bit][bit] + x_partner * G[1 - bit][bit]      (row vector)
// with bit = bit (4 - k) of l.  The block maximum is a five-step xor-shuffle
// reduction, every lane forms the E8M0 scale, and the even lane of each pair
// converts its two elements to one byte of E2M1 codes.
//
// A warp keeps one column block j (its ten coefficients stay in registers)
// and walks groups of kRows rows, whose independent shuffle chains overlap.
#include <algorithm>
#include <cstdint>

#include "kq_device.cuh"
#include "kq_internal.h"

namespace kq {
namespace {

constexpr int kWarpThreads = 256;          // 8 warps per CTA
constexpr int kRows = 4;                   // rows in flight per warp
constexpr int kWarpsPerSm = 48;            // target resident warps per SM

__global__ void __launch_bounds__(kWarpThreads)
    warp_kron_kernel(const uint16_t* __restrict__ x, int64_t M, int32_t nb,
                     const float* __restrict__ params, uint8_t* __restrict__ q,
                     uint8_t* __restrict__ scales, int64_t tw) {
  pdl_wait_then_trigger();
  const int lane = threadIdx.x & 31;
  // tw warps take part (a multiple of nb where possible); the rest of the
  // last CTA has no work.
  const int64_t gw = (int64_t)blockIdx.x * (kWarpThreads / 32) + (threadIdx.x >> 5);
  if (gw >= tw) return;
  const int64_t groups = (M + kRows - 1) / kRows;
  const int64_t tasks = groups * nb;
  const int64_t d = (int64_t)nb * kBlock;
  float c_own[kFactors], c_other[kFactors];
  int cur_j = -1;
  for (int64_t t = gw; t < tasks; t += tw) {
    const int j = static_cast<int>(t % nb);
    const int64_t row0 = (t / nb) * kRows;
    if (j != cur_j) {
      // This lane's two coefficients per factor, formed in double and
      // rounded once: G[bit][bit] for its own element, G[1 - bit][bit] for
      // its partner's.
      const float* p = params + (int64_t)j * 15;
#pragma unroll
      for (int k = 0; k < kFactors; ++k) {
        const double a = p[3 * k], b = p[3 * k + 1], c = p[3 * k + 2];
        const double g00 = b, g01 = c, g10 = a * b, g11 = __fma_rn(a, c, recip_d(b));
        const int bit = (lane >> (4 - k)) & 1;
        c_own[k] = static_cast<float>(bit ? g11 : g00);
        c_other[k] = static_cast<float>(bit ? g01 : g10);
      }
      cur_j = j;
    }
    float v[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int64_t row = row0 + r;
      const uint16_t h = row < M ? __ldg(x + row * d + (int64_t)j * kBlock + lane) : 0;
      v[r] = __uint_as_float(static_cast<uint32_t>(h) << 16);
    }
#pragma unroll
    for (int k = 0; k < kFactors; ++k) {
      const int m = 1 << (4 - k);
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const float o = __shfl_xor_sync(0xFFFFFFFFu, v[r], m);
        v[r] = __fmaf_rn(o, c_other[k], __fmul_rn(v[r], c_own[k]));
      }
    }
    float amax[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) amax[r] = fabsf(v[r]);
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1)
#pragma unroll
      for (int r = 0; r < kRows; ++r)
        amax[r] = fmaxf(amax[r], __shfl_xor_sync(0xFFFFFFFFu, amax[r], m));
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int field = static_cast<int>(__float_as_uint(amax[r]) >> 23);
      const int sbyte = field > 2 ? field - 2 : 0;
      const float inv_x = __uint_as_float(static_cast<uint32_t>(254 - sbyte) << 23);
      const float s = __fmul_rn(v[r], inv_x);
      const float s_hi = __shfl_xor_sync(0xFFFFFFFFu, s, 1);
      const int64_t row = row0 + r;
      if (row < M) {
        if ((lane & 1) == 0) {
          uint32_t byte;
          asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\t"
              "cvt.u32.u8 %0, b;\n\t}"
              : "=r"(byte)
              : "f"(s_hi), "f"(s));
          q[row * (d / 2) + (int64_t)j * 16 + (lane >> 1)] = static_cast<uint8_t>(byte);
        }
        if (lane == 0) scales[row * nb + j] = static_cast<uint8_t>(sbyte);
      }
    }
  }
}

}  // namespace

int launch_warp_kron(const uint16_t* x, int64_t M, int64_t d, const float* params, uint8_t* q,
                     uint8_t* scales, cudaStream_t st) {
  const DeviceInfo* di = nullptr;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != KQ_OK) return rc;
  const int64_t nb = d / kBlock;
  if (nb > (int64_t(1) << 30)) return KQ_ERR_INVALID;
  // A whole number of warps per column block where the device holds at
  // least one per block, so that every warp keeps its coefficients.
  const int64_t want = (int64_t)di->sms * kWarpsPerSm;
  const int64_t groups = (M + kRows - 1) / kRows;
  int64_t warps = nb <= want ? nb * std::max<int64_t>(1, std::min<int64_t>(want / nb, groups))
                             : want;
  const int64_t ctas = (warps + kWarpThreads / 32 - 1) / (kWarpThreads / 32);
  cudaError_t e = launch_pdl(warp_kron_kernel, dim3(static_cast<unsigned>(ctas)),
                             dim3(kWarpThreads), 0, st, x, M, static_cast<int32_t>(nb), params,
                             q, scales, warps);
  if (e != cudaSuccess) return record_cuda_error(e);
  return KQ_OK;
}

}  // namespace kq
