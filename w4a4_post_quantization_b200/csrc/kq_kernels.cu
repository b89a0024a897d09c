// Kernels of the KroQuant quantizer library and their launchers.
//
// Hot path (kq_quantize): the panel kernel.  One thread owns one 32-element
// block of a row at a time and keeps its column block, so its factors stay
// in registers.  A CTA (one per SM, persistent) owns a column panel of W
// blocks and walks the panel's row tiles; x is staged into shared memory by
// 3-D TMA boxes (64-byte swizzle, so that the thread-per-block reads are
// bank-conflict free) through a ring of stages guarded by mbarriers.  A
// producer warp issues the loads; 12 to 16 consumer warps run the scaled
// shear butterfly, the diagonal, the block maximum, the E8M0 scale and the
// E2M1 conversion, and store 16 bytes of codes and one scale byte per block.
// The flat-tile TMA kernel and the direct kernel below serve the shapes the
// panel does not fit, and the measurements.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <mutex>
#include <type_traits>

#include "kq.h"
#include "kq_device.cuh"
#include "kq_internal.h"

namespace kq {

__device__ int g_device_error = 0;

thread_local int t_last_cuda_error = 0;

// Remembers a failed CUDA call for kq_last_cuda_error; returns KQ_ERR_CUDA.
int record_cuda_error(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return KQ_ERR_CUDA;
}

// kXfKron16: 16-element Kronecker blocks (four factors each) with a scale
// per 16 elements; a thread owns a unit of two adjacent 16-blocks.
// kXfKronInvT: the weight-side fold W T^-T, factors (G_k^-1)^T.
// kXfKron16InvT: the weight-side fold with 16-element blocks.
enum Xform {
  kXfKron = 0, kXfHadamard = 1, kXfSmooth = 2, kXfKron16 = 3, kXfKronInvT = 4, kXfKron16InvT = 5
};

// Transforms made of five 2x2 factors per 32-block, and of four per 16-block.
__host__ __device__ constexpr bool kron5(int xf) { return xf == kXfKron || xf == kXfKronInvT; }
__host__ __device__ constexpr bool kron4(int xf) { return xf == kXfKron16 || xf == kXfKron16InvT; }
enum Out { kOutMx4 = 0, kOutF32 = 1 };

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = 32 * kConsumerWarps;       // threads = blocks per tile
constexpr int kTmaThreads = kConsumers + 32;          // + one producer warp
constexpr int kTile = kConsumers;                     // 32-blocks per TMA tile
constexpr int kTileBytes = kTile * kBlock * 2;        // bf16 tile, 16 KiB
constexpr int kMaxStages = 8;
constexpr int kTmaMaxNb = 512;                        // blocks per row the TMA kernel tables
constexpr int kDirectThreads = 256;                   // = column blocks per direct-kernel panel

struct LaunchArgs {
  int64_t G;            // 32-blocks in this launch (rows * nb)
  int32_t nb;           // 32-blocks per row
  int32_t n_tiles;      // ceil(G / kTile)
  int32_t stages;       // TMA ring depth
  const float* aux;     // params [nb][5][3] (Kronecker) or inv_s [nb*32] (smooth)
  uint8_t* q;           // [G][16] packed codes
  uint8_t* scales;      // [G] scale bytes
  float* y;             // [G][32] float32 output (kOutF32)
};

// ------------------------------------------------------------ table build
// Per-CTA shared table: for the Kronecker transform kTabStride floats per
// column block (the G_k entries), for smooth the 32 reciprocal scales.
template <int kXf>
__device__ __forceinline__ void build_table(float* tab, const LaunchArgs& a, int j0, int jn,
                                            int t, int nt) {
  if (kXf == kXfKron) {
    for (int j = t; j < jn; j += nt) kron_entry(tab + j * kTabStride, a.aux + (j0 + j) * 15);
  } else if (kXf == kXfSmooth) {
    const float4* src = reinterpret_cast<const float4*>(a.aux + (int64_t)j0 * kBlock);
    float4* dst = reinterpret_cast<float4*>(tab);
    for (int i = t; i < jn * (kBlock / 4); i += nt) {
      const int j = i >> 3, c = i & 7;           // block j's chunk c -> position c ^ (j & 7)
      dst[8 * j + (c ^ (j & 7))] = src[i];
    }
  }
}

template <int kXf>
__device__ __forceinline__ void apply_xform(f2 (&u)[16], const float* tab, int j) {
  if (kXf == kXfKron) kron_apply(u, tab + j * kTabStride);
  else if (kXf == kXfHadamard) hadamard_apply(u);
  else smooth_apply(u, tab + j * kBlock, j);
}

template <int kOut>
__device__ __forceinline__ void store_block(const f2 (&u)[16], const LaunchArgs& a, int64_t g) {
  if (kOut == kOutMx4) {
    const Mx4Block r = mxfp4_block(u);
    __stcs(reinterpret_cast<uint4*>(a.q + g * 16), r.codes);
    a.scales[g] = static_cast<uint8_t>(r.scale);
  } else {
    float4* dst = reinterpret_cast<float4*>(a.y + g * kBlock);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float x0, x1, x2, x3;
      unpack2(u[2 * i], x0, x1);
      unpack2(u[2 * i + 1], x2, x3);
      __stcs(dst + i, make_float4(x0, x1, x2, x3));
    }
  }
}

__host__ __device__ constexpr int table_floats(int xf, int nb) {
  return xf == kXfKron ? nb * kTabStride : (xf == kXfSmooth ? nb * kBlock : 0);
}

// ------------------------------------------------------------ TMA kernel
template <int kXf, int kOut>
__global__ void __launch_bounds__(kTmaThreads, 1)
    tma_kernel(const __grid_constant__ CUtensorMap xmap, const LaunchArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // Stage buffers first, 1 KiB aligned: the 64-byte swizzle pattern repeats
  // every 512 bytes and is a function of the shared-memory address.
  uint8_t* base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = base;
  float* tab = reinterpret_cast<float*>(base + a.stages * kTileBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(tab + table_floats(kXf, a.nb));
  uint64_t* empty = full + a.stages;
  pdl_wait_then_trigger();     // programmatic dependent launch: no global access before

  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  const int S = a.stages;
  const int n_local =
      blockIdx.x < a.n_tiles ? (a.n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

  if (tid >= kConsumers) {
    // Producer warp: one lane streams the CTA's tiles through the ring.
    if (tid == kConsumers) {
      tma_prefetch_map(&xmap);
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < n_local; ++i) {
        const int s = i % S;
        if (i >= S && !mbar_wait(&empty[s], ((i / S) - 1) & 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[s], kTileBytes);
        tma_load_2d(stages + s * kTileBytes, &xmap, 0, (blockIdx.x + i * gridDim.x) * kTile,
                    &full[s]);
        issued = i + 1;
      }
      if (!ok) {
        atomicOr(&g_device_error, kErrProducerWait);
        // Let the copies still in flight land before the CTA exits.
        for (int i = issued > S ? issued - S : 0; i < issued; ++i)
          mbar_wait(&full[i % S], (i / S) & 1);
      }
    }
    return;
  }

  // Consumers: build the coefficient table, then one 32-block per tile each.
  build_table<kXf>(tab, a, 0, a.nb, tid, kConsumers);
  asm volatile("bar.sync 1, %0;" ::"r"(kConsumers) : "memory");

  const int64_t step = (int64_t)gridDim.x * kTile;
  int64_t g = (int64_t)blockIdx.x * kTile + tid;
  int j = static_cast<int>(g % a.nb);
  const int jstep = static_cast<int>(step % a.nb);
  // Row tid of a tile holds its 4 chunks of 16 bytes at chunk ^ ((tid >> 1) & 3).
  const uint32_t swz = (tid >> 1) & 3;
  for (int i = 0; i < n_local; ++i) {
    const int s = i % S;
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], (i / S) & 1))) {
      if ((tid & 31) == 0) atomicOr(&g_device_error, kErrConsumerWait);
      break;
    }
    const uint8_t* row = stages + s * kTileBytes + tid * (kBlock * 2);
    uint4 c[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) c[q] = *reinterpret_cast<const uint4*>(row + 16 * (q ^ swz));
    // Hand the stage back: the reads above must be ordered before the TMA
    // load that will overwrite it (generic -> async proxy), then one arrival
    // per warp.
    fence_proxy_async_smem();
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive(&empty[s]);
    if (g < a.G) {
      f2 u[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        u[4 * q + 0] = bf16x2_to_f2(c[q].x);
        u[4 * q + 1] = bf16x2_to_f2(c[q].y);
        u[4 * q + 2] = bf16x2_to_f2(c[q].z);
        u[4 * q + 3] = bf16x2_to_f2(c[q].w);
      }
      apply_xform<kXf>(u, tab, j);
      store_block<kOut>(u, a, g);
    }
    g += step;
    j += jstep;
    if (j >= a.nb) j -= a.nb;
  }
}

// ------------------------------------------------------------ panel kernel
// CTA c owns the column panel c % panels (W consecutive 32-blocks of every
// row) and walks its row tiles; consumer thread t < W*R keeps column block
// j = panel*W + t % W for the whole kernel (its factors stay in registers)
// and handles rows t / W + r*R, r < kRpt, of every tile.  A tile is the TMA
// box {32 elements, W blocks, kRpt*R rows} of the 3-D view x[M][nb][32].
struct PanelArgs {
  int64_t M;            // rows
  int32_t nb;           // 32-blocks per row
  int32_t W;            // panel width in 32-blocks (divides nb)
  int32_t R;            // thread rows per tile (a tile holds kRpt * R rows)
  int32_t panels;       // nb / W
  int32_t row_tiles;    // ceil(M / (kRpt * R))
  int32_t stages;       // TMA ring depth
  int32_t tile_bytes;   // W * kRpt * R * 64 (one TMA box)
  int32_t stage_bytes;  // tile_bytes rounded up to 1 KiB: every stage starts on
                        // a multiple of the 512-byte 64B-swizzle period
  const float* aux;     // params [nb][5][3] (Kronecker) or inv_s [nb*32] (smooth)
  uint8_t* q;
  uint8_t* scales;
  float* y;
  int32_t scale_tiles_k;  // 0: scales row-major; else the tiled layout with this
                          // many 4-scale columns (128-row x 4-scale tiles)
};

// Offset of (row, scale column j) in the tiled scale layout: 128-row x
// 4-scale tiles of 512 bytes, row r = r0 + 32 r1 and scale i at byte
// 16 r0 + 4 r1 + i.
__device__ __forceinline__ int64_t tiled_scale_offset(int64_t row, int j, int tiles_k) {
  const int r = static_cast<int>(row & 127);
  return ((row >> 7) * tiles_k + (j >> 2)) * 512 + 16 * (r & 31) + 4 * (r >> 5) + (j & 3);
}

// Launch shape of the panel kernel: consumer warps, rows per consumer thread
// per tile, and CTAs per SM it is compiled for.
template <int kCW_, int kRpt_, int kMinBlocks_>
struct PanelCfg {
  static constexpr int kCW = kCW_;
  static constexpr int kRpt = kRpt_;
  static constexpr int kMinBlocks = kMinBlocks_;
  static constexpr int kCons = 32 * kCW_;
  static constexpr int kThreads = kCons + 32;
};

// Hands a stage back to the producer: the generic->async proxy fence orders
// this thread's shared-memory reads of the stage before the TMA load that
// will overwrite it (without it, lanes were seen reading the next tile's
// data); then one arrival per warp.
__device__ __forceinline__ void release_stage(uint64_t* bar, int lane) {
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

template <int kXf, int kOut, class Cfg, int kForm, class SD, class PF>
__device__ __forceinline__ void panel_consume(const PanelArgs& a, const uint8_t* stages,
                                              uint64_t* full, uint64_t* empty, int n_local,
                                              int k0, int cpp, int tid, bool active, int rho,
                                              int j, const SD& sd, const PF& pf) {
  constexpr int kRpt = Cfg::kRpt;
  const int S = a.stages;
  const int lane = tid & 31;
  // Byte offsets of this thread's 16-byte chunks inside a stage: row
  // ridx = (rho + r R) W + (t mod W) holds chunk q at q ^ ((ridx >> 1) & 3).
  uint32_t off[kRpt][4];
#pragma unroll
  for (int r = 0; r < kRpt; ++r) {
    const int ridx = (rho + r * a.R) * a.W + (tid % a.W);
    const uint32_t swz = (ridx >> 1) & 3;
#pragma unroll
    for (int q = 0; q < 4; ++q) off[r][q] = ridx * (kBlock * 2) + 16 * (q ^ swz);
  }
  const int64_t tile_rows = (int64_t)kRpt * a.R;
  int64_t row = k0 * tile_rows + rho;
  const int64_t row_step = (int64_t)cpp * tile_rows;
  int s = 0;
  uint32_t phase = 0;
  for (int i = 0; i < n_local; ++i) {
    // Every lane waits; the warp gives up only as a whole, so that no lane
    // leaves while the others sit in a warp-wide operation.
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], phase))) {
      if (lane == 0) atomicOr(&g_device_error, kErrConsumerWait);
      return;
    }
    const uint8_t* st = stages + s * a.stage_bytes;
    uint4 c[kRpt][4];
#pragma unroll
    for (int r = 0; r < kRpt; ++r)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        c[r][q] = active ? *reinterpret_cast<const uint4*>(st + off[r][q]) : make_uint4(0, 0, 0, 0);
    release_stage(&empty[s], lane);
    if (++s == S) {
      s = 0;
      phase ^= 1;
    }
    const int64_t row_i = row;
    row += row_step;
    if (!active) continue;
#pragma unroll
    for (int r = 0; r < kRpt; ++r) {
      const int64_t rr = row_i + (int64_t)r * a.R;
      if (rr >= a.M) break;
      f2 u[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        u[4 * q + 0] = bf16x2_to_f2(c[r][q].x);
        u[4 * q + 1] = bf16x2_to_f2(c[r][q].y);
        u[4 * q + 2] = bf16x2_to_f2(c[r][q].z);
        u[4 * q + 3] = bf16x2_to_f2(c[r][q].w);
      }
      if constexpr (kron4(kXf)) {
        if constexpr (kForm == 1) {
          plain_apply16(u, pf);
        } else {
          shear_apply16(u, sd);
          diag_mul(u, sd.delta);
        }
      } else if constexpr (kron5(kXf) && kForm == 1) {
        plain_apply(u, pf);
      } else if constexpr (kXf == kXfHadamard) {
        hadamard_apply(u);
      } else {
        if constexpr (kron5(kXf)) shear_apply(u, sd);
        diag_mul(u, sd.delta);
      }
      const int64_t g = rr * a.nb + j;
      if constexpr (kOut == kOutMx4 && kron4(kXf)) {
        // Two scale bytes per unit, block 0 at the lower address.
        const Mx4Block b = mxfp4_block16x2(u);
        __stcs(reinterpret_cast<uint4*>(a.q + g * 16), b.codes);
        if (a.scale_tiles_k == 0) {
          reinterpret_cast<uint16_t*>(a.scales)[g] = static_cast<uint16_t>(b.scale);
        } else {
          // Tiled layout, scale columns 2 j and 2 j + 1 (one 4-byte word
          // half); an odd count of units leaves half a 4-scale column of
          // padding, zeroed by the row's last unit.
          const int64_t o = tiled_scale_offset(rr, 2 * j, a.scale_tiles_k);
          *reinterpret_cast<uint16_t*>(a.scales + o) = static_cast<uint16_t>(b.scale);
          if (j == a.nb - 1 && (j & 1) == 0) *reinterpret_cast<uint16_t*>(a.scales + o + 2) = 0;
        }
      } else if constexpr (kOut == kOutMx4) {
        const Mx4Block b = mxfp4_block(u);
        __stcs(reinterpret_cast<uint4*>(a.q + g * 16), b.codes);
        if (a.scale_tiles_k == 0) {
          a.scales[g] = static_cast<uint8_t>(b.scale);
        } else {
          const int64_t o = tiled_scale_offset(rr, j, a.scale_tiles_k);
          a.scales[o] = static_cast<uint8_t>(b.scale);
          // The last block of a row also zeroes the row's padding scales:
          // they multiply zero codes in the product and must be finite.
          if (j == a.nb - 1)
            for (int t = (j & 3) + 1; t < 4; ++t) a.scales[o + t - (j & 3)] = 0;
        }
      } else {
        float4* dst = reinterpret_cast<float4*>(a.y + g * kBlock);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          float x0, x1, x2, x3;
          unpack2(u[2 * t], x0, x1);
          unpack2(u[2 * t + 1], x2, x3);
          __stcs(dst + t, make_float4(x0, x1, x2, x3));
        }
      }
    }
  }
}

template <int kXf, int kOut, class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads, Cfg::kMinBlocks)
    panel_kernel(const __grid_constant__ CUtensorMap xmap, const PanelArgs a) {
  constexpr int kRpt = Cfg::kRpt;
  constexpr int kCons = Cfg::kCons;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = base;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + a.stages * a.stage_bytes);
  uint64_t* empty = full + a.stages;
  const int tid = threadIdx.x;
  const int S = a.stages;
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], Cfg::kCW);
    }
    fence_mbar_init();
  }
  __syncthreads();
  // Programmatic dependent launch: the set-up above overlaps the previous
  // kernel of the stream; every global read and write of this grid comes
  // after the wait.  The next kernel may then start its own set-up as soon
  // as SMs free up (it waits the same way before touching memory).
  pdl_wait_then_trigger();

  const int panel = blockIdx.x % a.panels;
  const int cpp = gridDim.x / a.panels;           // CTAs per panel
  const int k0 = blockIdx.x / a.panels;           // first row tile of this CTA
  const int n_local = k0 < a.row_tiles ? (a.row_tiles - k0 + cpp - 1) / cpp : 0;
  const bool active = tid < a.W * a.R;
  const int j = panel * a.W + (tid % a.W);

  // Parameters first.  Each consumer thread reads its unit's parameters (or
  // reciprocal scales) into registers, and the whole CTA waits until they
  // have arrived before the producer issues the first tile loads: issued
  // behind the tiles' DRAM traffic, these few L2 reads were measured to
  // return several microseconds late, and every thread's coefficients wait
  // for them.
  constexpr int kUnitParams = kron5(kXf) ? 15 : kron4(kXf) ? 24 : kXf == kXfSmooth ? 32 : 0;
  float prm[kUnitParams > 0 ? kUnitParams : 1];
  float arrived = 0.0f;
  if constexpr (kUnitParams > 0) {
    if (tid < kCons && active) {
      const float* src = a.aux + (int64_t)j * kUnitParams;
      if constexpr (kXf == kXfSmooth) {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const float4 v = reinterpret_cast<const float4*>(src)[t];
          prm[4 * t] = v.x;
          prm[4 * t + 1] = v.y;
          prm[4 * t + 2] = v.z;
          prm[4 * t + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int t = 0; t < kUnitParams; ++t) prm[t] = src[t];
      }
      // A value that depends on every load: the barrier below then waits
      // for them.
#pragma unroll
      for (int t = 0; t < kUnitParams; ++t) arrived += prm[t];
    }
  }
  // The first tile alone goes out beside the parameter reads (one tile per
  // SM adds little to their wait), the rest after them.
  if (tid == kCons && n_local > 0) {
    tma_prefetch_map(&xmap);
    mbar_arrive_expect_tx(&full[0], a.tile_bytes);
    tma_load_3d(stages, &xmap, 0, panel * a.W, k0 * (kRpt * a.R), &full[0]);
  }
  asm volatile("bar.sync 2, %0;" ::"r"(Cfg::kThreads), "f"(arrived) : "memory");

  if (tid >= kCons) {
    if (tid == kCons) {
      int issued = n_local > 0 ? 1 : 0;
      bool ok = true;
      int s = issued % S;
      uint32_t phase = 0;                 // parity of the empty-barrier phase to wait for
      const int row_step = cpp * (kRpt * a.R);
      int row0 = k0 * (kRpt * a.R) + issued * row_step;
      for (int i = issued; i < n_local; ++i) {
        if (i >= S && !mbar_wait(&empty[s], phase)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[s], a.tile_bytes);
        tma_load_3d(stages + s * a.stage_bytes, &xmap, 0, panel * a.W, row0, &full[s]);
        row0 += row_step;
        issued = i + 1;
        if (++s == S) {
          s = 0;
          if (i >= S) phase ^= 1;
        }
      }
      if (!ok) {
        atomicOr(&g_device_error, kErrProducerWait);
        for (int i = issued > S ? issued - S : 0; i < issued; ++i)
          mbar_wait(&full[i % S], (i / S) & 1);
      }
    }
    return;
  }

  const int rho = tid / a.W;
  using SD = std::conditional_t<kron4(kXf), ShearDiag16, ShearDiag>;
  using PF = std::conditional_t<kron4(kXf), PlainFactors16, PlainFactors>;
  SD sd;
  PF pf;
  int plain = 0;
  if constexpr (kron5(kXf) || kron4(kXf)) {
    // Parameters per thread unit: 5 x 3 for a 32-block, 2 x 4 x 3 for a pair
    // of 16-blocks.
    const float* p = prm;
    if constexpr (kron5(kXf)) {
      if (active) plain = load_shear_diag<kXf == kXfKronInvT>(sd, p) ? 0 : 1;
    } else {
      if (active) plain = load_shear_diag16<kXf == kXfKron16InvT>(sd, p) ? 0 : 1;
    }
    // One form for the whole CTA: the plain one if any of its blocks needs it.
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.s32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\tselp.s32 %0, 1, 0, q;\n\t}"
        : "=r"(plain)
        : "r"(plain), "r"(kCons)
        : "memory");
    if (plain && active) {
      if constexpr (kron5(kXf)) load_plain<kXf == kXfKronInvT>(pf, p);
      else load_plain16<kXf == kXfKron16InvT>(pf, p);
    }
  } else if constexpr (kXf == kXfSmooth) {
    if (active) {
#pragma unroll
      for (int t = 0; t < 16; ++t) sd.delta[t] = pack2(prm[2 * t], prm[2 * t + 1]);
    }
  }
  if (plain)
    panel_consume<kXf, kOut, Cfg, 1>(a, stages, full, empty, n_local, k0, cpp, tid, active, rho,
                                      j, sd, pf);
  else
    panel_consume<kXf, kOut, Cfg, 0>(a, stages, full, empty, n_local, k0, cpp, tid, active, rho,
                                      j, sd, pf);
}

// ---------------------------------------------------------- direct kernel
// Grid (row groups, column panels of kDirectThreads blocks); thread t of
// panel p handles column block 256 p + t of rows blockIdx.x, +gridDim.x, ...
// (four 16-byte bf16 loads per block).
template <int kXf, int kOut>
__global__ void __launch_bounds__(kDirectThreads)
    direct_kernel(const uint16_t* __restrict__ xin, int64_t M, const LaunchArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* tab = reinterpret_cast<float*>(smem_raw);
  pdl_wait_then_trigger();     // programmatic dependent launch: no global access before
  const int j0 = blockIdx.y * kDirectThreads;
  const int jn = min(kDirectThreads, a.nb - j0);
  build_table<kXf>(tab, a, j0, jn, threadIdx.x, blockDim.x);
  __syncthreads();
  const int t = threadIdx.x;
  if (t >= jn) return;
  for (int64_t r = blockIdx.x; r < M; r += gridDim.x) {
    const int64_t g = r * a.nb + j0 + t;
    f2 u[16];
    const uint4* src = reinterpret_cast<const uint4*>(xin + g * kBlock);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 c = __ldg(src + q);
      u[4 * q + 0] = bf16x2_to_f2(c.x);
      u[4 * q + 1] = bf16x2_to_f2(c.y);
      u[4 * q + 2] = bf16x2_to_f2(c.z);
      u[4 * q + 3] = bf16x2_to_f2(c.w);
    }
    apply_xform<kXf>(u, tab, t);
    store_block<kOut>(u, a, g);
  }
}

// ------------------------------------------------------ wait self-test
// Waits on an mbarrier that nothing ever completes, with a short bound, and
// reports the expiry through the device error word: the same give-up path
// every pipeline wait takes, exercised without any fault.
__global__ void wait_selftest_kernel(int polls) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t addr = smem_addr(&bar);
    bool done = false;
    for (int i = 0; i < polls && !done; ++i) {
      uint32_t d;
      asm volatile(
          "{\n\t.reg .pred p;\n\t"
          "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(d)
          : "r"(addr), "r"(0u), "r"(1000u)
          : "memory");
      done = d != 0;
    }
    if (!done) atomicOr(&g_device_error, kErrSelfTest);
  }
}

// ------------------------------------------------------- dequantize kernel
__global__ void __launch_bounds__(256)
    dequant_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ scales, int64_t G,
                   float* __restrict__ y) {
  __shared__ float lut[16];
  pdl_wait_then_trigger();     // programmatic dependent launch: no global access before
  if (threadIdx.x < 16) {
    const int c = threadIdx.x, e = (c >> 1) & 3, m = c & 1;
    const float mag = e == 0 ? 0.5f * m : ldexpf(1.0f + 0.5f * m, e - 1);
    lut[c] = (c & 8) ? -mag : mag;
  }
  __syncthreads();
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < G;
       g += (int64_t)gridDim.x * blockDim.x) {
    const uint4 c = __ldcs(reinterpret_cast<const uint4*>(q + g * 16));
    const uint32_t s = scales[g];
    const float x = s == 255 ? __uint_as_float(0x7FC00000u)
                             : (s == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(s << 23));
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    float4* dst = reinterpret_cast<float4*>(y + g * kBlock);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = lut[(w[k] >> (4 * i)) & 15] * x;
      __stcs(dst + 2 * k, make_float4(v[0], v[1], v[2], v[3]));
      __stcs(dst + 2 * k + 1, make_float4(v[4], v[5], v[6], v[7]));
    }
  }
}

// =================================================================== host
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
int* g_error_word[kMaxDevices] = {};

int device_info(const DeviceInfo** out, int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return KQ_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.ready) {
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return record_cuda_error(e);
    di.status = prop.major == 10 ? KQ_OK : KQ_ERR_DEVICE;
    di.sms = prop.multiProcessorCount;
    di.smem_optin = static_cast<int>(prop.sharedMemPerBlockOptin);
    di.smem_per_sm = static_cast<int>(prop.sharedMemPerMultiprocessor);
    if (!g_encode) {
      cudaDriverEntryPointQueryResult qr;
      void* fn = nullptr;
      e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                           &qr);
      if (e != cudaSuccess || qr != cudaDriverEntryPointSuccess || !fn)
        return record_cuda_error(e != cudaSuccess ? e : cudaErrorNotSupported);
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    di.ready = true;
  }
  *out = &di;
  *dev_out = dev;
  return di.status;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() { return g_encode; }

int device_error_word(int dev, int** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_error_word[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_device_error);
    if (e != cudaSuccess) return record_cuda_error(e);
    g_error_word[dev] = static_cast<int*>(p);
  }
  *out = g_error_word[dev];
  return KQ_OK;
}

namespace {

int cuda_fail(cudaError_t e) { return record_cuda_error(e); }

bool aligned(const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

int check_shape(int64_t M, int64_t d) {
  if (M < 0 || d < kBlock || d % kBlock != 0) return KQ_ERR_INVALID;
  if (M > 0 && d > (int64_t(1) << 40) / M) return KQ_ERR_INVALID;
  return KQ_OK;
}

template <int kXf, int kOut>
int launch_tma(const uint16_t* x, int64_t M, int64_t d, LaunchArgs a, cudaStream_t st,
               const DeviceInfo& di, int dev) {
  const int nb = static_cast<int>(d / kBlock);
  if (nb > kTmaMaxNb) return KQ_ERR_INVALID;
  const int tab_bytes = table_floats(kXf, nb) * 4;
  const int fixed = 1024 + tab_bytes + 2 * kMaxStages * 8;
  const int stages = std::min(kMaxStages, (di.smem_optin - fixed) / kTileBytes);
  if (stages < 2) return KQ_ERR_INVALID;
  const int smem = 1024 + stages * kTileBytes + tab_bytes + 2 * stages * 8;
  int rc = allow_smem<tma_kernel<kXf, kOut>>(smem, dev);
  if (rc != KQ_OK) return rc;
  // Rows per launch keep the tile coordinate (an int32) in range.
  const int64_t rows_per_launch = ((int64_t(1) << 30) / nb);
  for (int64_t r0 = 0; r0 < M; r0 += rows_per_launch) {
    const int64_t rows = std::min(rows_per_launch, M - r0);
    LaunchArgs la = a;
    la.G = rows * nb;
    la.nb = nb;
    la.n_tiles = static_cast<int32_t>((la.G + kTile - 1) / kTile);
    la.stages = stages;
    const int64_t off = r0 * nb;          // in 32-blocks
    if (la.q) la.q += off * 16;
    if (la.scales) la.scales += off;
    if (la.y) la.y += off * kBlock;
    CUtensorMap map;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kBlock), static_cast<cuuint64_t>(la.G)};
    const cuuint64_t strides[1] = {kBlock * 2};
    const cuuint32_t box[2] = {kBlock, kTile};
    const cuuint32_t estr[2] = {1, 1};
    CUresult cr = g_encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                           const_cast<uint16_t*>(x + off * kBlock), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    const int grid = std::min(la.n_tiles, di.sms);
    cudaError_t le = launch_pdl(tma_kernel<kXf, kOut>, dim3(grid), dim3(kTmaThreads), smem, st,
                                map, la);
    if (le != cudaSuccess) return cuda_fail(le);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return KQ_OK;
}

// Panel shape for nb blocks per row: W divides nb, R = thread rows per tile,
// W * R <= cons, and W <= 256 and rpt * R <= 256 (TMA box dimension limit).
// Score: the share of busy consumer threads times the share of SMs that a
// grid made of whole panels (nb / W CTAs each) keeps busy; the best score
// wins, then the wider panel.  Returns the busy-thread share of the winner.
double panel_shape(int nb, int cons, int rpt, int sms, int* W_out, int* R_out) {
  double best = -1.0, best_use = 0.0;
  for (int W = std::min(std::min(nb, cons), 256); W >= 1; --W) {
    if (nb % W) continue;
    const int R = std::min(cons / W, 256 / rpt);
    const double use = double(W * R) / cons;
    const int panels = nb / W;
    const double sm_use = panels >= sms ? 1.0 : double(sms / panels * panels) / sms;
    const double score = use * sm_use;
    if (score > best + 1e-9) {
      best = score;
      best_use = use;
      *W_out = W;
      *R_out = R;
    }
  }
  return best_use;
}

// Panel-kernel shapes measured on B200 (interleaved medians on the
// 16384 x 12288 stress input, GB/s): 12 consumer warps x 2 rows 5526,
// 15 x 2 5405, 14 x 2 4971, 8 x 2 4972, 15 x 1 5441, 16 x 1 with the diagonal
// in shared memory 4978, 8 x 3 4740, 10 x 3 4601.  More warps hide latency until the register budget
// (ceil(warps / 4) warps share one scheduler's 16K registers) forces spills.
using PanelV0 = PanelCfg<12, 2, 1>;
using PanelV1 = PanelCfg<8, 2, 1>;
using PanelV2 = PanelCfg<15, 1, 1>;
using PanelV4 = PanelCfg<16, 1, 1>;
constexpr int kPanelMaxStages = 6;

template <class Cfg>
double panel_use(int nb, int sms, int* W, int* R) {
  return panel_shape(nb, Cfg::kCons, Cfg::kRpt, sms * Cfg::kMinBlocks, W, R);
}

// Launch shape by the work per SM.  Measured on B200, back to back over cold
// copies of x, microseconds per launch with 12 x 2 / 15 x 1 / 16 x 1
// consumer warps x rows: 8192 x 1152 9.24 / 8.69 / 8.61; 8192 x 4608
// 22.6 / 22.0 / 22.1; 4096 x 2240 9.23 / 8.60 / 8.27; 4096 x 5600
// 16.2 / 15.6 / 15.5; 4608 x 3072 11.3 / 11.3 / 10.9; 4608 x 12288
// 30.5 / 30.1 / 50.9; 16384 x 12288 87.1 / 88.6 / 152.  Up to about 24K
// blocks per SM the one-row shapes win (a shorter chain per tile, more
// warps); above that two rows per thread do.  16 x 1 is taken for rows of up
// to 256 blocks (it runs the 384-block rows on 128-block panels, measured
// slow) where its panel keeps 90 % of the 512 threads busy, 15 x 1 where its
// panel keeps three quarters of 480 busy; else the two-row shape, whose 384
// threads divide more widths.  The 16-element variant (two blocks of four
// factors a thread, a heavier set-up) keeps the two-row shape at every size
// (measured: the one-row shapes lose at 8192 x 4608, 4096 x 5600 and
// 4608 x 3072).
int auto_panel_variant(int64_t M, int nb, int sms, bool one_row_ok) {
  int W = 0, R = 0;
  if (!one_row_ok || M * nb > static_cast<int64_t>(sms) * 24576) return 0;
  if (nb <= 256 && panel_use<PanelV4>(nb, sms, &W, &R) >= 0.9) return 4;
  return panel_use<PanelV2>(nb, sms, &W, &R) >= 0.75 ? 2 : 0;
}

// KQ_PANEL_VARIANT (0, 1, 2 or 4) forces one compiled shape (read at every
// call; for tuning measurements only).
int panel_variant(int64_t M, int nb, int sms, bool one_row_ok = true) {
  const char* e = getenv("KQ_PANEL_VARIANT");
  return e ? atoi(e) : auto_panel_variant(M, nb, sms, one_row_ok);
}

template <int kXf, int kOut, class Cfg>
int launch_panel_cfg(const uint16_t* x, int64_t M, int64_t d, const float* aux, uint8_t* q,
                     uint8_t* scales, float* y, cudaStream_t st, const DeviceInfo& di, int dev,
                     int32_t scale_tiles_k) {
  constexpr int kRpt = Cfg::kRpt;
  const int nb = static_cast<int>(d / kBlock);
  PanelArgs a{};
  // The 16-element variant and the weight fold have no other kernel, so
  // they take any shape.
  const double min_use =
      (kron4(kXf) || kXf == kXfKronInvT || scale_tiles_k > 0) ? 0.0 : 0.5;
  if (panel_use<Cfg>(nb, di.sms, &a.W, &a.R) < min_use) return KQ_ERR_INVALID;
  a.M = M;
  a.nb = nb;
  a.panels = nb / a.W;
  a.tile_bytes = a.W * kRpt * a.R * kBlock * 2;
  a.stage_bytes = (a.tile_bytes + 1023) / 1024 * 1024;
  // Shared memory per CTA: the opt-in limit, or an equal share of the SM.
  const int budget = Cfg::kMinBlocks == 1 ? di.smem_optin
                                          : di.smem_per_sm / Cfg::kMinBlocks - 1024;
  a.stages = std::min(kPanelMaxStages,
                      (budget - 1024 - 2 * kPanelMaxStages * 8) / a.stage_bytes);
  if (a.stages < 2) return KQ_ERR_INVALID;
  const int64_t tile_rows = (int64_t)kRpt * a.R;
  const int64_t row_tiles = (M + tile_rows - 1) / tile_rows;
  if (M > (int64_t(1) << 31) - 1 - tile_rows || row_tiles > (int64_t(1) << 30))
    return KQ_ERR_INVALID;
  a.row_tiles = static_cast<int32_t>(row_tiles);
  a.aux = aux;
  a.q = q;
  a.scales = scales;
  a.y = y;
  a.scale_tiles_k = scale_tiles_k;
  const int smem = 1024 + a.stages * a.stage_bytes + 2 * a.stages * 8;
  int rc = allow_smem<panel_kernel<kXf, kOut, Cfg>>(smem, dev);
  if (rc != KQ_OK) return rc;
  CUtensorMap map;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kBlock), static_cast<cuuint64_t>(nb),
                              static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[2] = {kBlock * 2, static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[3] = {kBlock, static_cast<cuuint32_t>(a.W),
                             static_cast<cuuint32_t>(tile_rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult cr = g_encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(x), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  // A multiple of the panel count, up to the resident CTAs of the device.
  const int64_t resident = (int64_t)di.sms * Cfg::kMinBlocks;
  const int64_t per_panel = std::max<int64_t>(1, std::min<int64_t>(resident / a.panels, row_tiles));
  const int grid = static_cast<int>(per_panel * a.panels);
  cudaError_t e = launch_pdl(panel_kernel<kXf, kOut, Cfg>, dim3(static_cast<unsigned>(grid)),
                             dim3(Cfg::kThreads), static_cast<size_t>(smem), st, map, a);
  if (e != cudaSuccess) return cuda_fail(e);
  return KQ_OK;
}

template <int kXf, int kOut>
int launch_panel(const uint16_t* x, int64_t M, int64_t d, const float* aux, uint8_t* q,
                 uint8_t* scales, float* y, cudaStream_t st, const DeviceInfo& di, int dev,
                 int32_t scale_tiles_k = 0) {
  switch (panel_variant(M, static_cast<int>(d / kBlock), di.sms, !kron4(kXf))) {
    case 1:
      return launch_panel_cfg<kXf, kOut, PanelV1>(x, M, d, aux, q, scales, y, st, di, dev,
                                                  scale_tiles_k);
    case 2:
      return launch_panel_cfg<kXf, kOut, PanelV2>(x, M, d, aux, q, scales, y, st, di, dev,
                                                  scale_tiles_k);
    case 4:
      return launch_panel_cfg<kXf, kOut, PanelV4>(x, M, d, aux, q, scales, y, st, di, dev,
                                                  scale_tiles_k);
    default:
      return launch_panel_cfg<kXf, kOut, PanelV0>(x, M, d, aux, q, scales, y, st, di, dev,
                                                  scale_tiles_k);
  }
}

bool panel_fits(int64_t M, int nb, int sms) {
  int W = 0, R = 0;
  switch (panel_variant(M, nb, sms)) {
    case 1: return panel_use<PanelV1>(nb, sms, &W, &R) >= 0.75;
    case 2: return panel_use<PanelV2>(nb, sms, &W, &R) >= 0.75;
    case 4: return panel_use<PanelV4>(nb, sms, &W, &R) >= 0.75;
    default: return panel_use<PanelV0>(nb, sms, &W, &R) >= 0.75;
  }
}

template <int kXf, int kOut>
int launch_direct(const uint16_t* x, int64_t M, int64_t d, LaunchArgs a, cudaStream_t st,
                  const DeviceInfo& di, int dev) {
  const int nb = static_cast<int>(d / kBlock);
  const int panels = (nb + kDirectThreads - 1) / kDirectThreads;
  const int smem = table_floats(kXf, std::min(nb, kDirectThreads)) * 4;
  int rc = allow_smem<direct_kernel<kXf, kOut>>(std::max(smem, 1), dev);
  if (rc != KQ_OK) return rc;
  a.nb = nb;
  a.G = M * nb;
  const int64_t want = std::max<int64_t>(1, (int64_t)di.sms * 8 / panels);
  const int rows = static_cast<int>(std::min<int64_t>(M, std::min<int64_t>(want, 65535)));
  dim3 grid(rows, panels);
  {
    cudaError_t le = launch_pdl(direct_kernel<kXf, kOut>, grid, dim3(kDirectThreads), smem,
                                st, x, M, a);
    if (le != cudaSuccess) return cuda_fail(le);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return KQ_OK;
}

template <int kXf, int kOut>
int run(const uint16_t* x, int64_t M, int64_t d, const float* aux, uint8_t* q, uint8_t* scales,
        float* y, int impl, void* stream) {
  const DeviceInfo* di = nullptr;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != KQ_OK) return rc;
  LaunchArgs a{};
  a.aux = aux;
  a.q = q;
  a.scales = scales;
  a.y = y;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t nb = d / kBlock;
  if constexpr (kron4(kXf) || kXf == kXfKronInvT) {
    // Only the panel kernel carries the 16-element variant and the fold.
    if (impl != KQ_IMPL_PANEL || nb > 65535) return KQ_ERR_INVALID;
    return launch_panel<kXf, kOut>(x, M, d, aux, q, scales, y, st, *di, dev);
  } else {
    if (impl == KQ_IMPL_AUTO) {
      if (nb <= 65535 && panel_fits(M, static_cast<int>(nb), di->sms) && M < (int64_t(1) << 30))
        impl = KQ_IMPL_PANEL;
      else
        impl = nb <= kTmaMaxNb ? KQ_IMPL_TMA : KQ_IMPL_DIRECT;
    }
    if (impl == KQ_IMPL_WARP) {
      if (kXf != kXfKron || kOut != kOutMx4) return KQ_ERR_INVALID;
      return launch_warp_kron(x, M, d, aux, q, scales, st);
    }
    if (impl == KQ_IMPL_MMA) {
      if (kXf != kXfKron) return KQ_ERR_INVALID;
      return launch_mma_kron(x, M, d, aux, kOut == kOutMx4 ? q : nullptr,
                             kOut == kOutMx4 ? scales : nullptr, kOut == kOutF32 ? y : nullptr, st);
    }
    if (impl == KQ_IMPL_PANEL) {
      if (nb > 65535) return KQ_ERR_INVALID;
      return launch_panel<kXf, kOut>(x, M, d, aux, q, scales, y, st, *di, dev);
    }
    if (impl == KQ_IMPL_TMA) return launch_tma<kXf, kOut>(x, M, d, a, st, *di, dev);
    if (impl == KQ_IMPL_DIRECT) return launch_direct<kXf, kOut>(x, M, d, a, st, *di, dev);
    return KQ_ERR_INVALID;
  }
}

// The panel kernel with scales written in the tiled layout (4-scale
// columns: d/32 scales a row, or d/16 for the 16-element variants).
template <int kXf>
int run_tiled(const uint16_t* x, int64_t M, int64_t d, const float* params, uint8_t* q,
              uint8_t* scales_tiled, void* stream) {
  const DeviceInfo* di = nullptr;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != KQ_OK) return rc;
  const int64_t nb = d / kBlock;
  if (nb > 65535) return KQ_ERR_INVALID;
  const int64_t ns = kron4(kXf) ? 2 * nb : nb;
  return launch_panel<kXf, kOutMx4>(x, M, d, params, q, scales_tiled, nullptr,
                                    static_cast<cudaStream_t>(stream), *di, dev,
                                    static_cast<int32_t>((ns + 3) / 4));
}

int check_quant_args(const uint16_t* x, int64_t M, int64_t d, const void* aux, bool need_aux,
                     const uint8_t* q, const uint8_t* scales) {
  int rc = check_shape(M, d);
  if (rc != KQ_OK || M == 0) return rc;
  if (!x || !q || !scales || (need_aux && !aux)) return KQ_ERR_INVALID;
  if (!aligned(x, 16) || !aligned(q, 16) || (need_aux && !aligned(aux, 4))) return KQ_ERR_INVALID;
  return KQ_OK;
}

}  // namespace
}  // namespace kq

// ================================================================= C ABI
using namespace kq;

extern "C" int kq_quantize_ex(const uint16_t* x, int64_t M, int64_t d, const float* params,
                              uint8_t* q_packed, uint8_t* scales, int impl, void* stream) {
  int rc = check_quant_args(x, M, d, params, true, q_packed, scales);
  if (rc != KQ_OK || M == 0) return rc;
  if (impl < KQ_IMPL_AUTO || impl > KQ_IMPL_MMA) return KQ_ERR_INVALID;
  return run<kXfKron, kOutMx4>(x, M, d, params, q_packed, scales, nullptr, impl, stream);
}

extern "C" int kq_quantize(const uint16_t* x, int64_t M, int64_t d, const float* params,
                           uint8_t* q_packed, uint8_t* scales, void* stream) {
  return kq_quantize_ex(x, M, d, params, q_packed, scales, KQ_IMPL_AUTO, stream);
}

extern "C" int kq_quantize_hadamard(const uint16_t* x, int64_t M, int64_t d, uint8_t* q_packed,
                                    uint8_t* scales, void* stream) {
  int rc = check_quant_args(x, M, d, nullptr, false, q_packed, scales);
  if (rc != KQ_OK || M == 0) return rc;
  return run<kXfHadamard, kOutMx4>(x, M, d, nullptr, q_packed, scales, nullptr, KQ_IMPL_AUTO,
                                   stream);
}

extern "C" int kq_quantize_smooth(const uint16_t* x, int64_t M, int64_t d, const float* inv_s,
                                  uint8_t* q_packed, uint8_t* scales, void* stream) {
  int rc = check_quant_args(x, M, d, inv_s, true, q_packed, scales);
  if (rc != KQ_OK || M == 0) return rc;
  if (!aligned(inv_s, 16)) return KQ_ERR_INVALID;
  return run<kXfSmooth, kOutMx4>(x, M, d, inv_s, q_packed, scales, nullptr, KQ_IMPL_AUTO, stream);
}

extern "C" int kq_transform(const uint16_t* x, int64_t M, int64_t d, const float* params,
                            float* y, void* stream) {
  int rc = check_shape(M, d);
  if (rc != KQ_OK || M == 0) return rc;
  if (!x || !params || !y || !aligned(x, 16) || !aligned(y, 16) || !aligned(params, 4))
    return KQ_ERR_INVALID;
  return exact_transform(0, 5, false, x, M, d, params, y, static_cast<cudaStream_t>(stream));
}

extern "C" int kq_quantize16(const uint16_t* x, int64_t M, int64_t d, const float* params16,
                             uint8_t* q_packed, uint8_t* scales16, void* stream) {
  int rc = check_quant_args(x, M, d, params16, true, q_packed, scales16);
  if (rc != KQ_OK || M == 0) return rc;
  if (!aligned(scales16, 2) || d / kBlock > 65535) return KQ_ERR_INVALID;
  return run<kXfKron16, kOutMx4>(x, M, d, params16, q_packed, scales16, nullptr, KQ_IMPL_PANEL,
                                 stream);
}

extern "C" int kq_transform16(const uint16_t* x, int64_t M, int64_t d, const float* params16,
                              float* y, void* stream) {
  int rc = check_shape(M, d);
  if (rc != KQ_OK || M == 0) return rc;
  if (!x || !params16 || !y || !aligned(x, 16) || !aligned(y, 16) || !aligned(params16, 4) ||
      d / kBlock > 65535)
    return KQ_ERR_INVALID;
  return exact_transform(0, 4, false, x, M, d, params16, y, static_cast<cudaStream_t>(stream));
}

extern "C" int kq_quantize16_tiled(const uint16_t* x, int64_t M, int64_t d,
                                   const float* params16, uint8_t* q_packed,
                                   uint8_t* scales16_tiled, void* stream) {
  int rc = check_quant_args(x, M, d, params16, true, q_packed, scales16_tiled);
  if (rc != KQ_OK || M == 0) return rc;
  if (!aligned(scales16_tiled, 16)) return KQ_ERR_INVALID;
  return run_tiled<kXfKron16>(x, M, d, params16, q_packed, scales16_tiled, stream);
}

extern "C" int kq_quantize_weight16(const uint16_t* w, int64_t N, int64_t d,
                                    const float* params16, uint8_t* q_packed, uint8_t* scales16,
                                    void* stream) {
  int rc = check_quant_args(w, N, d, params16, true, q_packed, scales16);
  if (rc != KQ_OK || N == 0) return rc;
  if (!aligned(scales16, 2) || d / kBlock > 65535) return KQ_ERR_INVALID;
  return run<kXfKron16InvT, kOutMx4>(w, N, d, params16, q_packed, scales16, nullptr,
                                     KQ_IMPL_PANEL, stream);
}

extern "C" int kq_quantize_weight16_tiled(const uint16_t* w, int64_t N, int64_t d,
                                          const float* params16, uint8_t* q_packed,
                                          uint8_t* scales16_tiled, void* stream) {
  int rc = check_quant_args(w, N, d, params16, true, q_packed, scales16_tiled);
  if (rc != KQ_OK || N == 0) return rc;
  if (!aligned(scales16_tiled, 16)) return KQ_ERR_INVALID;
  return run_tiled<kXfKron16InvT>(w, N, d, params16, q_packed, scales16_tiled, stream);
}

extern "C" int kq_fold_weight16(const uint16_t* w, int64_t N, int64_t d, const float* params16,
                                float* w_folded, void* stream) {
  int rc = check_shape(N, d);
  if (rc != KQ_OK || N == 0) return rc;
  if (!w || !params16 || !w_folded || !aligned(w, 16) || !aligned(w_folded, 16) ||
      !aligned(params16, 4) || d / kBlock > 65535)
    return KQ_ERR_INVALID;
  return exact_transform(2, 4, false, w, N, d, params16, w_folded,
                         static_cast<cudaStream_t>(stream));
}

extern "C" int kq_quantize_weight(const uint16_t* w, int64_t N, int64_t d, const float* params,
                                  uint8_t* q_packed, uint8_t* scales, void* stream) {
  int rc = check_quant_args(w, N, d, params, true, q_packed, scales);
  if (rc != KQ_OK || N == 0) return rc;
  if (d / kBlock > 65535) return KQ_ERR_INVALID;
  return run<kXfKronInvT, kOutMx4>(w, N, d, params, q_packed, scales, nullptr, KQ_IMPL_PANEL,
                                   stream);
}

extern "C" int kq_fold_weight(const uint16_t* w, int64_t N, int64_t d, const float* params,
                              float* w_folded, void* stream) {
  int rc = check_shape(N, d);
  if (rc != KQ_OK || N == 0) return rc;
  if (!w || !params || !w_folded || !aligned(w, 16) || !aligned(w_folded, 16) ||
      !aligned(params, 4) || d / kBlock > 65535)
    return KQ_ERR_INVALID;
  return exact_transform(2, 5, false, w, N, d, params, w_folded,
                         static_cast<cudaStream_t>(stream));
}

extern "C" int kq_quantize_tiled(const uint16_t* x, int64_t M, int64_t d, const float* params,
                                 uint8_t* q_packed, uint8_t* scales_tiled, void* stream) {
  int rc = check_quant_args(x, M, d, params, true, q_packed, scales_tiled);
  if (rc != KQ_OK || M == 0) return rc;
  return run_tiled<kXfKron>(x, M, d, params, q_packed, scales_tiled, stream);
}

extern "C" int kq_quantize_weight_tiled(const uint16_t* w, int64_t N, int64_t d,
                                        const float* params, uint8_t* q_packed,
                                        uint8_t* scales_tiled, void* stream) {
  int rc = check_quant_args(w, N, d, params, true, q_packed, scales_tiled);
  if (rc != KQ_OK || N == 0) return rc;
  return run_tiled<kXfKronInvT>(w, N, d, params, q_packed, scales_tiled, stream);
}

extern "C" int kq_inverse_transform(const float* y, int64_t M, int64_t d, const float* params,
                                    float* x, void* stream) {
  int rc = check_shape(M, d);
  if (rc != KQ_OK || M == 0) return rc;
  if (!y || !params || !x || !aligned(y, 16) || !aligned(x, 16) || !aligned(params, 4))
    return KQ_ERR_INVALID;
  return exact_transform(1, 5, true, y, M, d, params, x, static_cast<cudaStream_t>(stream));
}

extern "C" int kq_dequantize(const uint8_t* q_packed, const uint8_t* scales, int64_t M, int64_t d,
                             float* y, void* stream) {
  int rc = check_shape(M, d);
  if (rc != KQ_OK || M == 0) return rc;
  if (!q_packed || !scales || !y || !aligned(q_packed, 16) || !aligned(y, 16)) return KQ_ERR_INVALID;
  const DeviceInfo* di = nullptr;
  int dev = 0;
  rc = device_info(&di, &dev);
  if (rc != KQ_OK) return rc;
  const int64_t G = M * (d / kBlock);
  const int64_t want = (G + 255) / 256;
  const int grid = static_cast<int>(std::min<int64_t>(want, (int64_t)di->sms * 8));
  {
    cudaError_t le = launch_pdl(dequant_kernel, dim3(grid), dim3(256), 0,
                                static_cast<cudaStream_t>(stream), q_packed, scales, G, y);
    if (le != cudaSuccess) return cuda_fail(le);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return KQ_OK;
}

extern "C" int kq_selftest_wait_timeout(void* stream) {
  const DeviceInfo* di = nullptr;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != KQ_OK) return rc;
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(64);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return KQ_OK;
}

extern "C" const char* kq_status_string(int status) {
  switch (status) {
    case KQ_OK: return "ok";
    case KQ_ERR_INVALID: return "invalid argument";
    case KQ_ERR_CUDA: return "CUDA error";
    case KQ_ERR_DEVICE: return "unsupported device (needs sm_100)";
    case KQ_ERR_TIMEOUT: return "a bounded device wait gave up";
    default: return "unknown status";
  }
}

extern "C" int kq_last_cuda_error(void) { return t_last_cuda_error; }

extern "C" int kq_device_status(int* flags) {
  if (!flags) return KQ_ERR_INVALID;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e);
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  *flags = v;
  return KQ_OK;
}

extern "C" int kq_version(void) { return (1 << 16) | 0; }
