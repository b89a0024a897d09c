// Quantization of activations that live in host memory: rows are moved in
// chunks through a device workspace, with the host-to-device copy of one
// chunk, the quantizer on the previous one and the device-to-host copy of the
// one before that running at the same time (two copy streams owned by the
// library, ordered against the caller's stream by events).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "kq.h"

namespace kq {
int record_cuda_error(cudaError_t e);   // kq_kernels.cu: sets kq_last_cuda_error
}

namespace {

constexpr int kMaxDevices = 64;
constexpr int kSlots = 2;

struct Pipe {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr;
  cudaEvent_t loaded[kSlots] = {}, computed[kSlots] = {}, drained[kSlots] = {};
};

std::mutex g_pipe_mu[kMaxDevices];
Pipe g_pipe[kMaxDevices];

int fail(cudaError_t e) { return kq::record_cuda_error(e); }

// Streams and events of this device's pipeline, created on first use.
int pipe_for(int dev, Pipe** out) {
  Pipe& p = g_pipe[dev];
  if (!p.ready) {
    cudaError_t e = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming);
    for (int s = 0; s < kSlots && e == cudaSuccess; ++s) {
      e = cudaEventCreateWithFlags(&p.loaded[s], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.computed[s], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.drained[s], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) return fail(e);
    p.ready = true;
  }
  *out = &p;
  return KQ_OK;
}

// Device bytes of one slot for `rows` rows of width d: x, codes, scales,
// each rounded up to 256 bytes.
size_t slot_bytes(int64_t rows, int64_t d) {
  auto up = [](size_t n) { return (n + 255) / 256 * 256; };
  return up(rows * d * 2) + up(rows * d / 2) + up(rows * d / 32);
}

}  // namespace

extern "C" size_t kq_quantize_host_workspace_bytes(int64_t d, int64_t rows_per_chunk) {
  if (d < 32 || d % 32 != 0 || rows_per_chunk < 1) return 0;
  return kSlots * slot_bytes(rows_per_chunk, d);
}

extern "C" int kq_quantize_host(const uint16_t* x_host, int64_t M, int64_t d,
                                const float* params, uint8_t* q_host, uint8_t* scales_host,
                                void* workspace, size_t workspace_bytes, void* stream) {
  if (M < 0 || d < 32 || d % 32 != 0) return KQ_ERR_INVALID;
  if (M == 0) return KQ_OK;
  if (M > 0 && d > (int64_t(1) << 40) / M) return KQ_ERR_INVALID;
  if (!x_host || !params || !q_host || !scales_host || !workspace) return KQ_ERR_INVALID;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return KQ_ERR_INVALID;
  // Rows per chunk: as many as two slots of the workspace hold (2.53125 bytes
  // per element plus up to 3 x 255 bytes of rounding per slot).
  const size_t per_slot = workspace_bytes / kSlots;
  int64_t rows = per_slot > 768 ? static_cast<int64_t>((per_slot - 768) / (d * 2 + d / 2 + d / 32)) : 1;
  rows = std::max<int64_t>(1, rows);
  while (rows > 1 && kSlots * slot_bytes(rows, d) > workspace_bytes) --rows;
  if (kSlots * slot_bytes(rows, d) > workspace_bytes) return KQ_ERR_INVALID;
  rows = std::min(rows, M);

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(e);
  if (dev < 0 || dev >= kMaxDevices) return KQ_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_pipe_mu[dev]);
  Pipe* p = nullptr;
  int rc = pipe_for(dev, &p);
  if (rc != KQ_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t sb = slot_bytes(rows, d);
  const size_t xb = (rows * d * 2 + 255) / 256 * 256, qb = (rows * d / 2 + 255) / 256 * 256;

  // Everything below runs after the work already queued on the caller's stream.
  if ((e = cudaEventRecord(p->start, st)) != cudaSuccess) return fail(e);
  if ((e = cudaStreamWaitEvent(p->in, p->start, 0)) != cudaSuccess) return fail(e);
  if ((e = cudaStreamWaitEvent(p->out, p->start, 0)) != cudaSuccess) return fail(e);

  const int64_t n_chunks = (M + rows - 1) / rows;
  for (int64_t c = 0; c < n_chunks; ++c) {
    const int s = static_cast<int>(c % kSlots);
    const int64_t r0 = c * rows, nr = std::min(rows, M - r0);
    uint16_t* xs = reinterpret_cast<uint16_t*>(ws + s * sb);
    uint8_t* qs = ws + s * sb + xb;
    uint8_t* ss = ws + s * sb + xb + qb;
    // Load: the slot's x is free once the quantizer of chunk c - 2 is done.
    if (c >= kSlots && (e = cudaStreamWaitEvent(p->in, p->computed[s], 0)) != cudaSuccess)
      return fail(e);
    if ((e = cudaMemcpyAsync(xs, x_host + r0 * d, nr * d * 2, cudaMemcpyHostToDevice, p->in)) !=
        cudaSuccess)
      return fail(e);
    if ((e = cudaEventRecord(p->loaded[s], p->in)) != cudaSuccess) return fail(e);
    // Quantize on the caller's stream, once the chunk is in and the slot's
    // outputs of chunk c - 2 have been copied out.
    if ((e = cudaStreamWaitEvent(st, p->loaded[s], 0)) != cudaSuccess) return fail(e);
    if (c >= kSlots && (e = cudaStreamWaitEvent(st, p->drained[s], 0)) != cudaSuccess)
      return fail(e);
    rc = kq_quantize(xs, nr, d, params, qs, ss, st);
    if (rc != KQ_OK) return rc;
    if ((e = cudaEventRecord(p->computed[s], st)) != cudaSuccess) return fail(e);
    // Drain the codes and scales.
    if ((e = cudaStreamWaitEvent(p->out, p->computed[s], 0)) != cudaSuccess) return fail(e);
    if ((e = cudaMemcpyAsync(q_host + r0 * (d / 2), qs, nr * (d / 2), cudaMemcpyDeviceToHost,
                             p->out)) != cudaSuccess)
      return fail(e);
    if ((e = cudaMemcpyAsync(scales_host + r0 * (d / 32), ss, nr * (d / 32),
                             cudaMemcpyDeviceToHost, p->out)) != cudaSuccess)
      return fail(e);
    if ((e = cudaEventRecord(p->drained[s], p->out)) != cudaSuccess) return fail(e);
  }
  // The caller's stream completes only after the last copies out.
  for (int s = 0; s < kSlots && s < n_chunks; ++s)
    if ((e = cudaStreamWaitEvent(st, p->drained[s], 0)) != cudaSuccess) return fail(e);
  return KQ_OK;
}
