// kq_quantize_host_static: the host-memory quantizer for callers that cannot
// allocate device memory.  A serving process that has already reserved
// nearly all of the GPU's memory for its own pool can see cudaMalloc fail,
// and cudaMalloc / cudaFree may synchronise the whole device, which a
// latency-bound caller cannot afford.  This entry point therefore takes no
// workspace and allocates nothing: the rows pass through a staging area that
// is part of the library image itself.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "kq.h"

namespace kq {
int record_cuda_error(cudaError_t e);   // kq_kernels.cu: sets kq_last_cuda_error
}

namespace {

constexpr size_t kStagingBytes = KQ_STATIC_STAGING_BYTES;
constexpr int kMaxDevices = 64;

// The staging area.  Each GPU on which this part of the library is loaded
// keeps these 16 MiB until the process exits.  In host code the name stands
// for a host-side handle, not a device address: the address is looked up
// per device below.
static __device__ __align__(256) uint8_t g_staging[kStagingBytes];

std::mutex g_mu;
void* g_staging_ptr[kMaxDevices] = {};

// Device address of g_staging on the current device, looked up once per
// device (with that device current).
int staging_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return kq::record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return KQ_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_staging_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_staging);
    if (e != cudaSuccess) return kq::record_cuda_error(e);
    g_staging_ptr[dev] = p;
  }
  *out = g_staging_ptr[dev];
  return KQ_OK;
}

size_t up256(size_t n) { return (n + 255) / 256 * 256; }

// Staging bytes for `rows` rows of width d: x, codes and scales, each
// rounded up to 256 bytes.
size_t chunk_bytes(int64_t rows, int64_t d) {
  return up256(rows * d * 2) + up256(rows * d / 2) + up256(rows * d / 32);
}

}  // namespace

extern "C" int kq_quantize_host_static(const uint16_t* x_host, int64_t M, int64_t d,
                                       const float* params, uint8_t* q_host,
                                       uint8_t* scales_host, void* stream) {
  if (M < 0 || d < 32 || d % 32 != 0) return KQ_ERR_INVALID;
  if (M == 0) return KQ_OK;
  if (d > (int64_t(1) << 40) / M) return KQ_ERR_INVALID;
  if (!x_host || !params || !q_host || !scales_host) return KQ_ERR_INVALID;
  // Rows per chunk; a row too wide for the staging area is rejected.
  if (chunk_bytes(1, d) > kStagingBytes) return KQ_ERR_INVALID;
  int64_t rows = static_cast<int64_t>((kStagingBytes - 768) / (d * 2 + d / 2 + d / 32));
  rows = std::max<int64_t>(1, std::min(rows, M));
  while (rows > 1 && chunk_bytes(rows, d) > kStagingBytes) --rows;

  void* base = nullptr;
  int rc = staging_address(&base);
  if (rc != KQ_OK) return rc;
  uint8_t* stage = static_cast<uint8_t*>(base);
  uint16_t* xs = reinterpret_cast<uint16_t*>(stage);
  uint8_t* qs = stage + up256(rows * d * 2);
  uint8_t* ss = qs + up256(rows * d / 2);
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // One stream, in order: copy a chunk in, quantize it, copy it out.  Every
  // staged byte is written before it is read, so nothing needs clearing.
  for (int64_t r0 = 0; r0 < M; r0 += rows) {
    const int64_t nr = std::min(rows, M - r0);
    cudaError_t e = cudaMemcpyAsync(xs, x_host + r0 * d, nr * d * 2, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return kq::record_cuda_error(e);
    rc = kq_quantize(xs, nr, d, params, qs, ss, st);
    if (rc != KQ_OK) return rc;
    e = cudaMemcpyAsync(q_host + r0 * (d / 2), qs, nr * (d / 2), cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return kq::record_cuda_error(e);
    e = cudaMemcpyAsync(scales_host + r0 * (d / 32), ss, nr * (d / 32), cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return kq::record_cuda_error(e);
  }
  return KQ_OK;
}
