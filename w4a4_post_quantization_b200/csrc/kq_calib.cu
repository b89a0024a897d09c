// Kernels of the straight-through calibration of the Kronecker transform on
// one linear layer (KroQuant review, "What carries the argument" and the
// free-parameter ledger: the transform is learned per layer by minimizing
// the quantized output error plus per-operand regularization, Adam with a
// straight-through estimator, from the Hadamard initialization).
//
//   kq_transform_params_grad  dL/dtheta of Z = X K(theta) per 32-block from
//                             Z (already computed), its quantized value and
//                             the output-side gradient; K = T or T^-T
//   kq_residual               R = scale (Y - Y_ref) and sum (Y - Y_ref)^2
//   kq_adam_step              Adam on the parameters
//
// Parameter gradient.  The five factor stages of K act on different bits of
// the in-block index and commute, so stage k can be taken last: its input is
// Z with stage k undone (F_k^-1 on bit 5 - k; det F_k = 1), and
// dL/dF_k[p][q] = sum over rows and index pairs of u_p G_q.  One thread owns
// one block of one row at a time and accumulates the 5 x 4 sums over its
// rows; a CTA tree-sums its row lanes in a fixed order and writes a partial
// per block, and the last CTA to finish sums the partials in a fixed order
// and applies dF/d(a, b, c), so the result does not depend on timing.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "kq.h"
#include "kq_device.cuh"
#include "kq_internal.h"

namespace kq {
namespace {

constexpr int kGradBlocksPerCta = 32;          // one warp across 32 blocks
constexpr int kGradRowLanes = 8;               // rows in flight per CTA
constexpr int kGradThreads = kGradBlocksPerCta * kGradRowLanes;
constexpr int kGradAcc = 5 * 4 + 1;            // factor sums + the regularizer sum

// Entries of stage k's matrix M_k^-1 (row-vector form), the one that undoes
// it: for F = G, G^-1 = [[g11, -g01], [-g10, g00]]; for F = (G^-1)^T,
// F^-1 = G^T = [[g00, g10], [g01, g11]].
template <bool kInvT>
__device__ __forceinline__ void undo_entries(const float* p, int k, float& m00, float& m01,
                                             float& m10, float& m11) {
  const float a = p[3 * k], b = p[3 * k + 1], c = p[3 * k + 2];
  const float g00 = b, g01 = c, g10 = a * b, g11 = __fmaf_rn(a, c, 1.0f / b);
  if (kInvT) {
    m00 = g00; m01 = g10; m10 = g01; m11 = g11;
  } else {
    m00 = g11; m01 = -g01; m10 = -g10; m11 = g00;
  }
}

// d F / d(a, b, c) contracted with the 2x2 sums s[p][q] = dL/dF[p][q].
template <bool kInvT>
__device__ __forceinline__ void chain_params(const float* p, int k, const float (&s)[4],
                                             float* out) {
  const float a = p[3 * k], b = p[3 * k + 1], c = p[3 * k + 2];
  const float s00 = s[0], s01 = s[1], s10 = s[2], s11 = s[3];
  const float ib2 = 1.0f / (b * b);
  if (kInvT) {
    // F = [[a c + 1/b, -a b], [-c, b]]
    out[0] = s00 * c - s01 * b;
    out[1] = -s00 * ib2 - s01 * a + s11;
    out[2] = s00 * a - s10;
  } else {
    // F = [[b, c], [a b, a c + 1/b]]
    out[0] = s10 * b + s11 * c;
    out[1] = s00 + s10 * a - s11 * ib2;
    out[2] = s01 + s11 * a;
  }
}

struct GradArgs {
  int64_t M;
  int32_t nb, rows_per_split;
  float two_lambda;
  const float* z;           // [M][d] the transformed operand (X T or W T^-T)
  const float* zq;          // [M][d] its quantized value
  const float* g;           // [M][d] dL_out / dZq
  const float* params;      // [nb][5][3]
  float* partial;           // [gridDim.y][nb][kGradAcc]
  unsigned int* counter;
  float* dparams;           // [nb][5][3] out
  float* reg;               // out: sum (zq - z)^2
};

template <bool kInvT>
__global__ void __launch_bounds__(kGradThreads)
    params_grad_kernel(const GradArgs a) {
  __shared__ float red[kGradRowLanes][kGradBlocksPerCta][kGradAcc];
  __shared__ bool last;
  pdl_wait_then_trigger();     // programmatic dependent launch: no global access before
  const int bl = threadIdx.x % kGradBlocksPerCta, rl = threadIdx.x / kGradBlocksPerCta;
  const int j = blockIdx.x * kGradBlocksPerCta + bl;
  float acc[kGradAcc];
#pragma unroll
  for (int t = 0; t < kGradAcc; ++t) acc[t] = 0.f;
  if (j < a.nb) {
    float m[5][4];
#pragma unroll
    for (int k = 0; k < 5; ++k)
      undo_entries<kInvT>(a.params + (int64_t)j * 15, k, m[k][0], m[k][1], m[k][2], m[k][3]);
    const int64_t r0 = (int64_t)blockIdx.y * a.rows_per_split;
    const int64_t r1 = a.M < r0 + a.rows_per_split ? a.M : r0 + a.rows_per_split;
    const int64_t d = (int64_t)a.nb * 32;
    for (int64_t r = r0 + rl; r < r1; r += kGradRowLanes) {
      const float4* pz = reinterpret_cast<const float4*>(a.z + r * d + 32 * j);
      const float4* pq = reinterpret_cast<const float4*>(a.zq + r * d + 32 * j);
      const float4* pg = reinterpret_cast<const float4*>(a.g + r * d + 32 * j);
      float z[32], G[32];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const float4 vz = __ldg(pz + t), vq = __ldg(pq + t), vg = __ldg(pg + t);
        const float zz[4] = {vz.x, vz.y, vz.z, vz.w}, qq[4] = {vq.x, vq.y, vq.z, vq.w};
        const float gg[4] = {vg.x, vg.y, vg.z, vg.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          z[4 * t + e] = zz[e];
          const float dq = zz[e] - qq[e];
          G[4 * t + e] = __fmaf_rn(a.two_lambda, dq, gg[e]);
          acc[20] = __fmaf_rn(dq, dq, acc[20]);
        }
      }
#pragma unroll
      for (int k = 0; k < 5; ++k) {
        const int bit = 4 - k;                    // factor k + 1 acts on bit 4 - k
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (i & (1 << bit)) continue;
          const int h = i | (1 << bit);
          // the stage's input at this pair: (z_lo, z_hi) M_k^-1
          const float ulo = __fmaf_rn(z[h], m[k][2], z[i] * m[k][0]);
          const float uhi = __fmaf_rn(z[h], m[k][3], z[i] * m[k][1]);
          acc[4 * k + 0] = __fmaf_rn(ulo, G[i], acc[4 * k + 0]);
          acc[4 * k + 1] = __fmaf_rn(ulo, G[h], acc[4 * k + 1]);
          acc[4 * k + 2] = __fmaf_rn(uhi, G[i], acc[4 * k + 2]);
          acc[4 * k + 3] = __fmaf_rn(uhi, G[h], acc[4 * k + 3]);
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kGradAcc; ++t) red[rl][bl][t] = acc[t];
  __syncthreads();
  // Row lanes summed in a fixed order; one partial per (split, block).
  if (rl == 0 && j < a.nb) {
    float* out = a.partial + ((int64_t)blockIdx.y * a.nb + j) * kGradAcc;
    for (int t = 0; t < kGradAcc; ++t) {
      float v = red[0][bl][t];
      for (int q = 1; q < kGradRowLanes; ++q) v += red[q][bl][t];
      out[t] = v;
    }
  }
  // The last CTA to finish reduces the partials over the row splits.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int total = gridDim.x * gridDim.y;
    last = atomicAdd(a.counter, 1u) == total - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int jj = threadIdx.x; jj < a.nb; jj += blockDim.x) {
    float s[kGradAcc];
    for (int t = 0; t < kGradAcc; ++t) s[t] = 0.f;
    for (int y = 0; y < (int)gridDim.y; ++y) {
      const float* pp = a.partial + ((int64_t)y * a.nb + jj) * kGradAcc;
      for (int t = 0; t < kGradAcc; ++t) s[t] += __ldcg(pp + t);
    }
    for (int k = 0; k < 5; ++k) {
      const float sk[4] = {s[4 * k], s[4 * k + 1], s[4 * k + 2], s[4 * k + 3]};
      chain_params<kInvT>(a.params + (int64_t)jj * 15, k, sk, a.dparams + (int64_t)jj * 15 + 3 * k);
    }
    a.partial[(int64_t)jj * kGradAcc + 20] = s[20];   // split 0 keeps the block's reg sum
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = 0.f;
    for (int jj = 0; jj < a.nb; ++jj) r += a.partial[(int64_t)jj * kGradAcc + 20];
    *a.reg = r;
    *a.counter = 0u;                             // ready for the next call
  }
}

constexpr int kResThreads = 256;

// out = scale (y - ref), and sum (y - ref)^2 accumulated in double: each
// CTA's sum to a partial, the last CTA adds the partials in a fixed order.
__global__ void __launch_bounds__(kResThreads)
    residual_kernel(const float* y, const float* ref, int64_t n, float scale, float* out,
                    double* partial, unsigned int* counter, double* sumsq) {
  __shared__ double red[kResThreads];
  __shared__ bool last;
  pdl_wait_then_trigger();     // programmatic dependent launch: no global access before
  double acc = 0.0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const double dr = (double)y[i] - (double)ref[i];     // exact
    acc += dr * dr;
    out[i] = scale * (y[i] - ref[i]);
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = kResThreads / 2; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    partial[blockIdx.x] = red[0];
    __threadfence();
    last = atomicAdd(counter, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (last && threadIdx.x == 0) {
    __threadfence();
    double t = 0.0;
    for (unsigned int b = 0; b < gridDim.x; ++b) t += __ldcg(partial + b);
    *sumsq = t;
    *counter = 0u;
  }
}

// Adam with bias correction; the gradient is the sum of two parts.
// The coefficients come from the host, the complements 1 - beta formed in
// double there (1 - float(0.999) is 1.3e-5 away from 0.001).
__global__ void adam_kernel(float* p, const float* g0, const float* g1, float* m, float* v,
                            int64_t n, float lr, float beta1, float cbeta1, float beta2,
                            float cbeta2, float eps, float corr1, float corr2) {
  pdl_wait_then_trigger();     // programmatic dependent launch: no global access before
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float g = g0[i] + (g1 ? g1[i] : 0.f);
    const float mi = __fmaf_rn(beta1, m[i], cbeta1 * g);
    const float vi = __fmaf_rn(beta2, v[i], cbeta2 * (g * g));
    m[i] = mi;
    v[i] = vi;
    p[i] -= lr * (mi / corr1) / (sqrtf(vi / corr2) + eps);
  }
}

}  // namespace
}  // namespace kq

using namespace kq;

namespace {

bool al(const void* p, uintptr_t n) { return reinterpret_cast<uintptr_t>(p) % n == 0; }

// Row splits of the gradient kernel: about four CTAs per SM in all.
int grad_splits(int64_t M, int nb, int sms) {
  const int64_t col_ctas = (nb + kGradBlocksPerCta - 1) / kGradBlocksPerCta;
  const int64_t want = std::max<int64_t>(1, (int64_t)sms * 4 / col_ctas);
  return static_cast<int>(std::min<int64_t>(std::min<int64_t>(want, 65535),
                                            std::max<int64_t>(1, M / kGradRowLanes)));
}

}  // namespace

extern "C" size_t kq_transform_params_grad_workspace_bytes(int64_t M, int64_t d) {
  if (M < 1 || d < 32 || d % 32 != 0) return 0;
  const DeviceInfo* di = nullptr;
  int dev = 0;
  const int sms = device_info(&di, &dev) == KQ_OK ? di->sms : 148;
  const int nb = static_cast<int>(d / 32);
  return 256 + (size_t)grad_splits(M, nb, sms) * nb * kGradAcc * sizeof(float);
}

extern "C" int kq_transform_params_grad(const float* z, const float* zq, const float* g,
                                        int64_t M, int64_t d, const float* params,
                                        int inverse_transpose, float lambda, float* dparams,
                                        float* reg, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  if (M < 1 || d < 32 || d % 32 != 0 || d / 32 > (1 << 24)) return KQ_ERR_INVALID;
  if (M > 0 && d > (int64_t(1) << 40) / M) return KQ_ERR_INVALID;
  if (!z || !zq || !g || !params || !dparams || !reg || !workspace) return KQ_ERR_INVALID;
  if (!al(z, 16) || !al(zq, 16) || !al(g, 16) || !al(params, 4) || !al(dparams, 4) ||
      !al(reg, 4) || !al(workspace, 256) || !std::isfinite(lambda))
    return KQ_ERR_INVALID;
  const DeviceInfo* di = nullptr;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != KQ_OK) return rc;
  const int nb = static_cast<int>(d / 32);
  const int splits = grad_splits(M, nb, di->sms);
  if (workspace_bytes < 256 + (size_t)splits * nb * kGradAcc * sizeof(float))
    return KQ_ERR_INVALID;
  GradArgs a{};
  a.M = M;
  a.nb = nb;
  a.rows_per_split = static_cast<int32_t>((M + splits - 1) / splits);
  a.two_lambda = 2.0f * lambda;
  a.z = z;
  a.zq = zq;
  a.g = g;
  a.params = params;
  a.counter = static_cast<unsigned int*>(workspace);
  a.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + 256);
  a.dparams = dparams;
  a.reg = reg;
  const dim3 grid((nb + kGradBlocksPerCta - 1) / kGradBlocksPerCta, splits);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = inverse_transpose
                      ? launch_pdl(params_grad_kernel<true>, grid, dim3(kGradThreads), 0, st, a)
                      : launch_pdl(params_grad_kernel<false>, grid, dim3(kGradThreads), 0, st, a);
  if (e != cudaSuccess) return record_cuda_error(e);
  return KQ_OK;
}

extern "C" size_t kq_residual_workspace_bytes(void) { return 256 + 4096 * sizeof(double); }

extern "C" int kq_residual(const float* y, const float* y_ref, int64_t n, float scale, float* out,
                           double* sumsq, void* workspace, size_t workspace_bytes, void* stream) {
  if (n < 1 || !y || !y_ref || !out || !sumsq || !workspace) return KQ_ERR_INVALID;
  if (!al(workspace, 256) || !al(sumsq, 8) || !std::isfinite(scale)) return KQ_ERR_INVALID;
  if (workspace_bytes < kq_residual_workspace_bytes()) return KQ_ERR_INVALID;
  const DeviceInfo* di = nullptr;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != KQ_OK) return rc;
  const int64_t want = (n + kResThreads - 1) / kResThreads;
  const int grid = static_cast<int>(std::min<int64_t>(want, std::min(4096, di->sms * 8)));
  cudaError_t e = launch_pdl(residual_kernel, dim3(grid), dim3(kResThreads), 0,
                             static_cast<cudaStream_t>(stream), y, y_ref, n, scale, out,
                             reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) + 256),
                             static_cast<unsigned int*>(workspace), sumsq);
  if (e != cudaSuccess) return record_cuda_error(e);
  return KQ_OK;
}

extern "C" int kq_adam_step(float* params, const float* grad0, const float* grad1, float* m,
                            float* v, int64_t n, int step, double lr, double beta1, double beta2,
                            double eps, void* stream) {
  if (n < 1 || step < 1 || !params || !grad0 || !m || !v) return KQ_ERR_INVALID;
  if (!(beta1 >= 0.0 && beta1 < 1.0 && beta2 >= 0.0 && beta2 < 1.0 && eps > 0.0) ||
      !std::isfinite(lr))
    return KQ_ERR_INVALID;
  const DeviceInfo* di = nullptr;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != KQ_OK) return rc;
  const float corr1 = static_cast<float>(1.0 - std::pow(beta1, step));
  const float corr2 = static_cast<float>(1.0 - std::pow(beta2, step));
  const int grid = static_cast<int>(std::min<int64_t>((n + 255) / 256, di->sms * 4));
  cudaError_t e = launch_pdl(
      adam_kernel, dim3(grid), dim3(256), 0, static_cast<cudaStream_t>(stream), params, grad0,
      grad1, m, v, n, static_cast<float>(lr), static_cast<float>(beta1),
      static_cast<float>(1.0 - beta1), static_cast<float>(beta2),
      static_cast<float>(1.0 - beta2), static_cast<float>(eps), corr1, corr2);
  if (e != cudaSuccess) return record_cuda_error(e);
  return KQ_OK;
}
