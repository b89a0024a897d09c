// Tensor-core variant of the Kronecker transform (the paper's "K1" kernel:
// precomputed dense 32x32 blocks applied as small GEMMs), for sm_100a:
//
//   y[128 rows, block j] = x[128 rows, 32] . K^(j)      (tcgen05.mma, kind::f16)
//
// K^(j) is materialised per CTA in double and split exactly into three bf16
// terms K = K_hi + K_mid + K_lo (about 24 significant bits together), so
// three bf16 MMAs accumulating in float32 TMEM reproduce a float32 transform
// of the bf16 activations (which are exact in bf16).  Each CTA owns a panel
// of Wb column blocks and walks its 128-row tiles:
//   warp 0      TMA: x tile as [Wb blocks][128 rows][64 B], 64-byte swizzle,
//               one 3-D box per block
//   warp 1      allocates TMEM; one lane issues 6 MMAs per block per tile
//               into one of two TMEM accumulator sets
//   warps 2..9  epilogue: tcgen05.ld of a row's 32 outputs per block, then
//               the same MXFP4 quantizer as the CUDA-core kernels; code tiles
//               leave through shared memory by TMA store
#include <cuda_bf16.h>

#include <algorithm>

#include "kq_device.cuh"
#include "kq_internal.h"
#include "kq_tc.cuh"

namespace kq {
namespace {

constexpr int kTileRows = 128;                       // UMMA M
constexpr int kMaxWb = 8;                            // 2 x 8 x 32 TMEM columns = 512
// Epilogue width measured on B200 (16384 x 12288 stress input): 8 warps
// 90 us, 12 warps 154 us and 16 warps 119 us (both spill registers).
constexpr int kEpiWarps = 8;                         // 2 per TMEM lane quarter
constexpr int kEpiGroups = kEpiWarps / 4;             // column groups per quarter
constexpr int kMaxPer = (kMaxWb + kEpiGroups - 1) / kEpiGroups;   // blocks per warp
constexpr int kMmaThreads = 32 * (2 + kEpiWarps);
constexpr int kBMatBytes = 32 * 64;                  // one 32x32 bf16 operand
constexpr int kMmaMaxStages = 4;

// Instruction descriptor: D f32, A and B bf16, both K-major, N = 32, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((32u >> 3) << 17) |
                            ((uint32_t(kTileRows) >> 4) << 24);

struct MmaArgs {
  int64_t M;
  int32_t nb, Wb, panels, row_tiles, stages, tmem_cols, out_f32;
  int32_t tma_store;    // codes leave through shared memory and a TMA store (Wb 4 or 8)
  const float* params;
  uint8_t* q;
  uint8_t* scales;
  float* y;
  int* err;
};

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(kIdesc), "r"(acc)
      : "memory");
}

// The three bf16 terms of K^(j)^T for the panel, written in the K-major
// 64-byte-swizzled layout the MMA reads: operand (w, t) is 32 rows n of
// 64 bytes (k = 0..31), chunk k/8 of row n at chunk (k/8) ^ ((n >> 1) & 3).
__device__ void build_b_operands(uint8_t* bmat, double* gtab, const float* params, int j0, int Wb,
                                 int tid, int nt) {
  // G_k entries per block, row-vector form, in double: [w][k][g00 g01 g10 g11].
  for (int i = tid; i < Wb * kFactors; i += nt) {
    const int w = i / kFactors, k = i % kFactors;
    const float* p = params + (int64_t)(j0 + w) * 15 + 3 * k;
    const double a = p[0], b = p[1], c = p[2];
    double* g = gtab + 4 * i;
    g[0] = b;
    g[1] = c;
    g[2] = a * b;
    g[3] = __fma_rn(a, c, 1.0 / b);
  }
  __syncthreads();
  for (int e = tid; e < Wb * 1024; e += nt) {
    const int w = e >> 10, n = (e >> 5) & 31, k = e & 31;
    double v = 1.0;
#pragma unroll
    for (int f = 0; f < kFactors; ++f) {
      const int sh = 4 - f;
      v *= gtab[4 * (w * kFactors + f) + 2 * ((k >> sh) & 1) + ((n >> sh) & 1)];
    }
    const __nv_bfloat16 hi = __double2bfloat16(v);
    const double r1 = v - static_cast<double>(__bfloat162float(hi));
    const __nv_bfloat16 mid = __double2bfloat16(r1);
    const double r2 = r1 - static_cast<double>(__bfloat162float(mid));
    const __nv_bfloat16 lo = __double2bfloat16(r2);
    const uint32_t off = n * 64 + ((((k >> 3) ^ ((n >> 1) & 3))) << 4) + (k & 7) * 2;
    *reinterpret_cast<__nv_bfloat16*>(bmat + (w * 3 + 0) * kBMatBytes + off) = hi;
    *reinterpret_cast<__nv_bfloat16*>(bmat + (w * 3 + 1) * kBMatBytes + off) = mid;
    *reinterpret_cast<__nv_bfloat16*>(bmat + (w * 3 + 2) * kBMatBytes + off) = lo;
  }
}

__global__ void __launch_bounds__(kMmaThreads, 1)
    mma_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap qmap,
               const MmaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int Wb = a.Wb, S = a.stages;
  const int stage_bytes = Wb * kTileRows * kBlock * 2;
  uint8_t* stages = base;
  uint8_t* bmat = base + S * stage_bytes;
  const int out_bytes = kTileRows * Wb * 16;           // one tile of codes
  uint8_t* outbuf = bmat + Wb * 3 * kBMatBytes;          // 2 tiles when a.tma_store
  double* gtab = reinterpret_cast<double*>(outbuf + (a.tma_store ? 2 * out_bytes : 0));
  uint64_t* full = reinterpret_cast<uint64_t*>(gtab + kMaxWb * kFactors * 4);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int panel = blockIdx.x % a.panels;
  const int cpp = gridDim.x / a.panels;
  const int k0 = blockIdx.x / a.panels;
  const int n_local = k0 < a.row_tiles ? (a.row_tiles - k0 + cpp - 1) / cpp : 0;
  const int j0 = panel * Wb;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(a.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  build_b_operands(bmat, gtab, a.params, j0, Wb, tid, kMmaThreads);
  fence_proxy_async_smem();            // B operands: generic writes -> tensor core reads
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_map(&xmap);
      int s = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < n_local; ++i) {
        if (i >= S && !mbar_wait(&empty[s], phase)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[s], stage_bytes);
        // One box per column block: 128 rows x 64 B, contiguous in its slot.
        for (int w = 0; w < Wb; ++w)
          tma_load_3d(stages + s * stage_bytes + w * (kTileRows * 64), &xmap, 0, j0 + w,
                      (k0 + i * cpp) * kTileRows, &full[s]);
        issued = i + 1;
        if (++s == S) {
          s = 0;
          if (i >= S) phase ^= 1;
        }
      }
      if (!ok) {
        atomicOr(a.err, kErrProducerWait);
        for (int i = issued > S ? issued - S : 0; i < issued; ++i)
          mbar_wait(&full[i % S], (i / S) & 1);
      }
    }
    return;
  }

  if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint64_t bdesc0 = smem_desc_sw64(smem_addr(bmat));
      int s = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < n_local && ok; ++i) {
        const int b = i & 1;
        ok = mbar_wait(&full[s], phase);
        if (ok && i >= 2) ok = mbar_wait(&acc_empty[b], ((i >> 1) - 1) & 1);
        if (!ok) break;
        tmem_fence_after();
        // Descriptors step by (bytes >> 4) in their low 14 bits.
        uint64_t da = smem_desc_sw64(smem_addr(stages + s * stage_bytes));
        uint64_t db = bdesc0;
        uint32_t d = tmem_base + b * (Wb * 32);
        for (int w = 0; w < Wb; ++w) {
#pragma unroll
          for (int t = 0; t < 3; ++t) {
            mma_bf16(d, da, db + t * (kBMatBytes >> 4), t != 0);
            mma_bf16(d, da + (32 >> 4), db + t * (kBMatBytes >> 4) + (32 >> 4), 1);
          }
          da += (kTileRows * 64) >> 4;
          db += (3 * kBMatBytes) >> 4;
          d += 32;
        }
        mma_commit(&empty[s]);         // the stage is free once these MMAs have read it
        mma_commit(&acc_full[b]);      // and the accumulators are ready
        if (++s == S) {
          s = 0;
          phase ^= 1;
        }
      }
      if (!ok) atomicOr(a.err, kErrConsumerWait);
      // Every issued MMA completes before the accumulators are released.
      mma_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue
    const int e = warp - 2;
    const int quarter = warp & 3;                  // TMEM lanes 32*quarter .. +31
    const int group = e / 4;
    const int per = (Wb + kEpiGroups - 1) / kEpiGroups;   // <= kMaxPer blocks per warp
    const int w0 = min(Wb, group * per), nw = min(Wb, w0 + per) - w0;
    const bool issuer = tid == 64;                 // warp 2, lane 0: TMA stores
    const int rloc = quarter * 32 + lane;          // row within the tile
    for (int i = 0; i < n_local; ++i) {
      const int b = i & 1;
      bool ok;
      if (a.tma_store) {
        // The output tile buffer i & 1 is free once the store of tile i - 2
        // has read it; one AND-barrier also makes a timeout CTA-uniform.
        const bool mine = mbar_wait(&acc_full[b], (i >> 1) & 1);
        if (issuer) bulk_wait_read_1();
        ok = bar_and(3, 32 * kEpiWarps, mine);
      } else {
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&acc_full[b], (i >> 1) & 1));
      }
      if (!ok) {
        if (lane == 0) atomicOr(a.err, kErrConsumerWait);
        break;
      }
      tmem_fence_after();
      // All of this warp's blocks in flight at once, one wait, then the
      // accumulators go straight back to the MMA warp.
      uint32_t r[kMaxPer][32];
      const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16) + b * (Wb * 32) + w0 * 32;
#pragma unroll
      for (int v = 0; v < kMaxPer; ++v)
        if (v < nw) tmem_ld32(taddr + v * 32, r[v]);
      tmem_wait_ld();
      tmem_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
      const int64_t row0 = (int64_t)(k0 + (int64_t)i * cpp) * kTileRows;
      const int64_t row = row0 + rloc;
      uint8_t* ob = outbuf + b * out_bytes;
      uint32_t sc = 0;                               // this row's scale bytes, low byte first
#pragma unroll
      for (int v = 0; v < kMaxPer; ++v) {
        if (v >= nw) break;
        f2 u[16];
#pragma unroll
        for (int m = 0; m < 16; ++m)
          u[m] = pack2(__uint_as_float(r[v][2 * m]), __uint_as_float(r[v][2 * m + 1]));
        const int64_t g = row * a.nb + j0 + w0 + v;
        if (a.out_f32) {
          if (row < a.M) {
            float4* dst = reinterpret_cast<float4*>(a.y + g * kBlock);
#pragma unroll
            for (int t = 0; t < 8; ++t)
              __stcs(dst + t, make_float4(__uint_as_float(r[v][4 * t]), __uint_as_float(r[v][4 * t + 1]),
                                          __uint_as_float(r[v][4 * t + 2]),
                                          __uint_as_float(r[v][4 * t + 3])));
          }
          continue;
        }
        const Mx4Block blk = mxfp4_block(u);
        sc |= blk.scale << (8 * v);
        if (a.tma_store) {
          // 16-byte chunk c of tile row rloc, swizzled like the TMA store map.
          const int c = w0 + v;
          const int phys = Wb == 8 ? (c ^ (rloc & 7)) : (c ^ ((rloc >> 1) & 3));
          *reinterpret_cast<uint4*>(ob + rloc * (Wb * 16) + phys * 16) = blk.codes;
        } else if (row < a.M) {
          __stcs(reinterpret_cast<uint4*>(a.q + g * 16), blk.codes);
        }
      }
      if (!a.out_f32 && row < a.M && nw > 0) {
        uint8_t* sp = a.scales + row * a.nb + j0 + w0;
        if (nw == 4 && (reinterpret_cast<uintptr_t>(sp) & 3) == 0) {
          *reinterpret_cast<uint32_t*>(sp) = sc;
        } else if (nw == 2 && (reinterpret_cast<uintptr_t>(sp) & 1) == 0) {
          *reinterpret_cast<uint16_t*>(sp) = static_cast<uint16_t>(sc);
        } else {
          for (int v = 0; v < nw; ++v) sp[v] = static_cast<uint8_t>(sc >> (8 * v));
        }
      }
      if (a.tma_store) {
        fence_proxy_async_smem();                    // generic writes -> TMA store reads
        asm volatile("bar.sync 4, %0;" ::"r"(32 * kEpiWarps) : "memory");
        if (issuer) {
          tma_store_2d(&qmap, ob, j0 * 16, static_cast<int>(row0));
          bulk_commit();
        }
      }
    }
    if (a.tma_store && issuer) bulk_wait_all();
  }
  // Warps 1..9 meet here; then warp 1 returns the TMEM columns.
  asm volatile("bar.sync 2, %0;" ::"r"(kMmaThreads - 32) : "memory");
  if (warp == 1) {
    tmem_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(a.tmem_cols)
                 : "memory");
  }
}

}  // namespace

// Panel width for nb blocks per row: Wb divides nb, 2 <= Wb <= 8, the grid
// (panels x CTAs per panel) keeps the most SMs busy; ties go to widths 8 and
// 4 (whose code tiles leave by TMA store), then to the wider panel.
// Returns 0 if no width fits.
int mma_panel_width(int nb, int sms) {
  int best = 0;
  double best_use = 0.0;
  for (int Wb = std::min(nb, kMaxWb); Wb >= 2; --Wb) {
    if (nb % Wb) continue;
    const int panels = nb / Wb;
    if (panels > sms) continue;
    const double use = double(sms / panels * panels) / sms + ((Wb == 8 || Wb == 4) ? 1e-3 : 0.0);
    if (use > best_use + 1e-9) {
      best_use = use;
      best = Wb;
    }
  }
  return best;
}

int launch_mma_kron(const uint16_t* x, int64_t M, int64_t d, const float* params, uint8_t* q,
                    uint8_t* scales, float* y, cudaStream_t st) {
  const DeviceInfo* di = nullptr;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != KQ_OK) return rc;
  const int nb = static_cast<int>(d / kBlock);
  MmaArgs a{};
  a.Wb = mma_panel_width(nb, di->sms);
  if (a.Wb == 0 || M > (int64_t(1) << 31) - 1 - kTileRows) return KQ_ERR_INVALID;
  rc = device_error_word(dev, &a.err);
  if (rc != KQ_OK) return rc;
  a.M = M;
  a.nb = nb;
  a.panels = nb / a.Wb;
  a.row_tiles = static_cast<int32_t>((M + kTileRows - 1) / kTileRows);
  a.params = params;
  a.q = q;
  a.scales = scales;
  a.y = y;
  a.out_f32 = y != nullptr;
  int cols = 32;
  while (cols < 2 * a.Wb * 32) cols *= 2;
  a.tmem_cols = cols;
  a.tma_store = (q != nullptr) && (a.Wb == 8 || a.Wb == 4);
  const int stage_bytes = a.Wb * kTileRows * kBlock * 2;
  const int fixed = 1024 + a.Wb * 3 * kBMatBytes + (a.tma_store ? 2 * kTileRows * a.Wb * 16 : 0) +
                    kMaxWb * kFactors * 4 * 8 + (2 * kMmaMaxStages + 5) * 8 + 16;
  a.stages = std::min(kMmaMaxStages, (di->smem_optin - fixed) / stage_bytes);
  if (a.stages < 2) return KQ_ERR_INVALID;
  const int smem = fixed + a.stages * stage_bytes;
  rc = allow_smem<mma_kernel>(smem, dev);
  if (rc != KQ_OK) return rc;
  // x as [M][nb][32]: a box {32, 1 block, 128 rows} lands in shared memory as
  // 128 rows of 64 B, one K-major operand; Wb boxes fill a stage.
  CUtensorMap map;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kBlock), static_cast<cuuint64_t>(nb),
                              static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[2] = {kBlock * 2, static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[3] = {kBlock, 1, kTileRows};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult cr = tensor_map_encoder()(
      &map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(x), dims, strides, box, estr,
      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return record_cuda_error(cudaErrorInvalidValue);
  // Codes as [M][d/2] bytes; a box is one tile: Wb * 16 bytes x 128 rows,
  // with the swizzle whose span is exactly one box row.
  CUtensorMap qmap = map;
  if (a.tma_store) {
    const cuuint64_t qdims[2] = {static_cast<cuuint64_t>(nb) * 16, static_cast<cuuint64_t>(M)};
    const cuuint64_t qstrides[1] = {static_cast<cuuint64_t>(nb) * 16};
    const cuuint32_t qbox[2] = {static_cast<cuuint32_t>(a.Wb * 16), kTileRows};
    const cuuint32_t qestr[2] = {1, 1};
    cr = tensor_map_encoder()(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, qdims, qstrides, qbox,
                              qestr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              a.Wb == 8 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return record_cuda_error(cudaErrorInvalidValue);
  }
  const int per_panel = std::max(1, std::min(di->sms / a.panels, a.row_tiles));
  mma_kernel<<<per_panel * a.panels, kMmaThreads, smem, st>>>(map, qmap, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return record_cuda_error(e);
  return KQ_OK;
}

}  // namespace kq
