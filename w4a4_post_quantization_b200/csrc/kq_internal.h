// Host-side helpers shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "kq.h"

namespace kq {

constexpr int kMaxDevices = 64;

// Remembers a failed CUDA call for kq_last_cuda_error; returns KQ_ERR_CUDA.
int record_cuda_error(cudaError_t e);

struct DeviceInfo {
  bool ready = false;
  int status = KQ_OK;
  int sms = 0;
  int smem_optin = 0;
  int smem_per_sm = 0;
};

// Properties of the current device (cached) and its index; KQ_ERR_DEVICE if
// it is not an sm_100 part.
int device_info(const DeviceInfo** out, int* dev_out);

// The driver's cuTensorMapEncodeTiled (valid after a successful device_info).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Device address of the library's device-side error word on device `dev`.
int device_error_word(int dev, int** out);

// The float32 outputs of the block transforms computed in double
// (kq_exact.cu): kind 0 = x K, 1 = x K^-1, 2 = x K^-T; nf = 5 (32-element
// blocks) or 4 (16-element blocks, two a 32-element unit); f32_in: float32
// input (else bf16).  Shapes and pointers checked by the caller.
int exact_transform(int kind, int nf, bool f32_in, const void* x, int64_t M, int64_t d,
                    const float* params, float* y, cudaStream_t st);

// Sets the dynamic shared-memory limit of one kernel once per device.
template <auto kKernel>
int allow_smem(int bytes, int dev) {
  static std::mutex mu;
  static int done[kMaxDevices] = {0};
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev] < bytes) {
    cudaError_t e = cudaFuncSetAttribute(kKernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return record_cuda_error(e);
    done[dev] = bytes;
  }
  return KQ_OK;
}

// Launches `kernel` with programmatic stream serialization, so that its
// set-up overlaps the tail of the previous kernel of the stream (the kernel
// executes griddepcontrol.wait before its first global read or write); a
// plain launch where the runtime refuses the attribute.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    kernel<<<grid, block, smem, st>>>(args...);
    e = cudaGetLastError();
  }
  return e;
}

// Launchers defined in other translation units.
int launch_mma_kron(const uint16_t* x, int64_t M, int64_t d, const float* params, uint8_t* q,
                    uint8_t* scales, float* y, cudaStream_t st);
int launch_warp_kron(const uint16_t* x, int64_t M, int64_t d, const float* params, uint8_t* q,
                     uint8_t* scales, cudaStream_t st);

}  // namespace kq
