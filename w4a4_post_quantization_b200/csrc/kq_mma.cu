// Tensor-core variant of the Kronecker quantizer (KQ_IMPL_MMA): the paper's
// "K1" design, dense 32x32 blocks applied as small GEMMs, written for sm_100a.
//
//   y[128 rows, block j] = x[128 rows, 32] . K^(j)      (tcgen05.mma, kind::f16)
//
// K^(j) is formed per CTA (each entry a product of five factor entries in
// double, rounded once to float32) and split exactly into three bf16 terms
// K = K_hi + K_mid + K_lo, so three bf16 MMAs accumulating in float32 TMEM
// give a float32 transform of the bf16 activations (which are exact in bf16).
// A CTA owns a panel of Wb column blocks and walks its 128-row tiles:
//   warp 0      TMA: a stage holds one 128-row x 64-byte box per block
//               (64-byte swizzle), the K-major A operand of that block
//   warp 1      allocates TMEM; one lane issues 6 MMAs per block and tile
//               into one of up to four TMEM accumulator sets
//   warps 2-17  epilogue, four groups of four warps (one per TMEM lane
//               quarter): group g takes blocks g, g + 4 of a tile; a thread
//               holds one token row's 32 outputs of a block (tcgen05.ld),
//               releases the accumulator at once, and runs the same MXFP4
//               epilogue as the CUDA-core kernels.  Codes go through a
//               swizzled shared-memory tile and leave by one TMA store per
//               tile; scale bytes are gathered per row and stored by the
//               first group.
// The transform's flops run on the tensor cores, so a thread spends a few
// instructions per element (the E2M1 epilogue) instead of the butterfly's.
#include <cuda_bf16.h>

#include <algorithm>

#include "kq_device.cuh"
#include "kq_internal.h"
#include "kq_tc.cuh"

namespace kq {
namespace {

constexpr int kTileRows = 128;                        // UMMA M
constexpr int kMaxWb = 8;                             // blocks per panel
constexpr int kEpiWarps = 16;
constexpr int kEpiGroups = kEpiWarps / 4;             // groups of four lane quarters
constexpr int kMaxPer = (kMaxWb + kEpiGroups - 1) / kEpiGroups;   // blocks per warp and tile
constexpr int kMmaThreads = 32 * (2 + kEpiWarps);
constexpr int kIssuer = 64;                           // warp 2, lane 0: TMA stores
constexpr int kBMatBytes = 32 * 64;                   // one 32x32 bf16 operand
constexpr int kABoxBytes = kTileRows * 64;            // one block's x tile
constexpr int kMaxStages = 8;
constexpr int kMaxAcc = 4;
constexpr int kTmemCols = 512;

// Instruction descriptor: D f32, A and B bf16, both K-major, N = 32, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((32u >> 3) << 17) |
                            ((uint32_t(kTileRows) >> 4) << 24);

// Swizzle of the code staging tile (rows of Wb * 16 bytes), matching the TMA
// store map: 128-byte for Wb = 8, 64-byte for 4, 32-byte for 2, none else.
enum { kSwzNone = 0, kSwz32 = 1, kSwz64 = 2, kSwz128 = 3 };

struct MmaArgs {
  int64_t M;
  int32_t nb, Wb, panels, row_tiles, stages, nacc, swz, out_f32;
  const float* params;
  uint8_t* scales;
  float* y;
  int* err;
};

// Shared-memory layout (from a 1 KiB aligned base).
struct Layout {
  uint32_t stage_bytes, b_off, codes_off, code_bytes, sc_off, bar_off, total;
  __host__ __device__ Layout(int Wb, int S) {
    stage_bytes = Wb * kABoxBytes;
    b_off = S * stage_bytes;
    codes_off = b_off + Wb * 3 * kBMatBytes;           // a multiple of 1 KiB
    code_bytes = kTileRows * Wb * 16;                  // one code tile
    sc_off = codes_off + 2 * code_bytes;               // two scale tiles of 128 x Wb
    const uint32_t g_off = sc_off + 2 * kTileRows * Wb;
    bar_off = (g_off + Wb * kFactors * 4 * 4 + 7) / 8 * 8;   // after the factor table
    total = bar_off + (2 * kMaxStages + 2 * kMaxAcc + 2) * 8 + 16;
  }
};

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(kIdesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void bar_sync_n(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// G_k entries of the panel's blocks, row-vector form, formed in double and
// rounded once: gtab[w][k] = (g00, g01, g10, g11).
__device__ __forceinline__ void build_factor_table(float* gtab, const float* params, int j0,
                                                   int Wb, int tid) {
  if (tid < Wb * kFactors) {
    const int w = tid / kFactors, k = tid % kFactors;
    const float* p = params + (int64_t)(j0 + w) * 15 + 3 * k;
    const double a = p[0], b = p[1], c = p[2];
    float* g = gtab + 4 * tid;
    g[0] = static_cast<float>(b);
    g[1] = static_cast<float>(c);
    g[2] = static_cast<float>(a * b);
    g[3] = static_cast<float>(__fma_rn(a, c, recip_d(b)));
  }
}

// The three bf16 terms of K^(j)^T for the panel, in the K-major 64-byte
// swizzled layout the MMA reads: operand (w, t) is 32 rows n of 64 bytes
// (k = 0..31), chunk k/8 of row n at chunk (k/8) ^ ((n >> 1) & 3).
__device__ void build_b_operands(uint8_t* bmat, const float* gtab, int Wb, int tid, int nt) {
  for (int e = tid; e < Wb * 1024; e += nt) {
    const int w = e >> 10, n = (e >> 5) & 31, k = e & 31;
    double v = 1.0;
#pragma unroll
    for (int f = 0; f < kFactors; ++f) {
      const int sh = 4 - f;
      v *= gtab[4 * (w * kFactors + f) + 2 * ((k >> sh) & 1) + ((n >> sh) & 1)];
    }
    // An exact split of the float32 entry: 8 + 8 + 8 significant bits.
    const float vf = static_cast<float>(v);
    const __nv_bfloat16 hi = __float2bfloat16_rn(vf);
    const float r1 = vf - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    const uint32_t off = n * 64 + ((((k >> 3) ^ ((n >> 1) & 3))) << 4) + (k & 7) * 2;
    *reinterpret_cast<__nv_bfloat16*>(bmat + (w * 3 + 0) * kBMatBytes + off) = hi;
    *reinterpret_cast<__nv_bfloat16*>(bmat + (w * 3 + 1) * kBMatBytes + off) = mid;
    *reinterpret_cast<__nv_bfloat16*>(bmat + (w * 3 + 2) * kBMatBytes + off) = lo;
  }
}

// 16-byte chunk that block w of tile row r occupies in the code staging tile.
__device__ __forceinline__ int code_chunk(int w, int r, int swz) {
  switch (swz) {
    case kSwz128: return w ^ (r & 7);
    case kSwz64: return w ^ ((r >> 1) & 3);
    case kSwz32: return w ^ ((r >> 2) & 1);
    default: return w;
  }
}

__global__ void __launch_bounds__(kMmaThreads, 1)
    mma_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap qmap,
               const MmaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int Wb = a.Wb, S = a.stages, NA = a.nacc;
  const Layout L(Wb, S);
  uint8_t* stages = base;
  uint8_t* bmat = base + L.b_off;
  uint8_t* codes = base + L.codes_off;
  uint8_t* sstage = base + L.sc_off;
  float* gtab = reinterpret_cast<float*>(base + L.sc_off + 2 * kTileRows * Wb);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + L.bar_off);
  uint64_t* empty = full + kMaxStages;
  uint64_t* acc_full = empty + kMaxStages;
  uint64_t* acc_empty = acc_full + kMaxAcc;
  uint64_t* mma_done = acc_empty + kMaxAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 2);

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
    for (int b = 0; b < NA; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  // Programmatic dependent launch: the set-up above overlaps the previous
  // kernel; every global access below comes after the wait.
  pdl_wait_then_trigger();
  // The parameters first, before any tile load: issued behind the tiles'
  // DRAM traffic, these few L2 reads return microseconds late.
  build_factor_table(gtab, a.params, j0, Wb, tid);
  __syncthreads();
  // The first stages' loads go out now and arrive while the B operands are
  // formed.
  const int pre = min(S, n_local);
  if (tid == 0) {
    tma_prefetch_map(&xmap);
    for (int i = 0; i < pre; ++i) {
      mbar_arrive_expect_tx(&full[i], L.stage_bytes);
      const int row0 = (k0 + i * cpp) * kTileRows;
      for (int w = 0; w < Wb; ++w)
        tma_load_3d(stages + i * L.stage_bytes + w * kABoxBytes, &xmap, 0, j0 + w, row0,
                    &full[i]);
    }
  }
  build_b_operands(bmat, gtab, Wb, tid, kMmaThreads);
  fence_proxy_async_smem();            // B operands: generic writes -> tensor core reads
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      // Tiles 0 .. pre-1 went out before the B operands were formed.
      int s = pre % S, issued = pre;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = pre; i < n_local; ++i) {
        if (i >= S && !mbar_wait(&empty[s], phase)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[s], L.stage_bytes);
        const int row0 = (k0 + i * cpp) * kTileRows;
        for (int w = 0; w < Wb; ++w)
          tma_load_3d(stages + s * L.stage_bytes + w * kABoxBytes, &xmap, 0, j0 + w, row0,
                      &full[s]);
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
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint64_t bdesc0 = smem_desc_sw64(smem_addr(bmat));
      int s = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < n_local && ok; ++i) {
        const int b = i % NA;
        ok = mbar_wait(&full[s], phase);
        if (ok && i >= NA) ok = mbar_wait(&acc_empty[b], ((i / NA) - 1) & 1);
        if (!ok) break;
        tmem_fence_after();
        // Descriptors step by (bytes >> 4) in their low 14 bits.
        uint64_t da = smem_desc_sw64(smem_addr(stages + s * L.stage_bytes));
        uint64_t db = bdesc0;
        uint32_t d = tmem_base + b * (Wb * 32);
        for (int w = 0; w < Wb; ++w) {
#pragma unroll
          for (int t = 0; t < 3; ++t) {
            mma_bf16(d, da, db + t * (kBMatBytes >> 4), t != 0);
            mma_bf16(d, da + (32 >> 4), db + t * (kBMatBytes >> 4) + (32 >> 4), 1);
          }
          da += kABoxBytes >> 4;
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
    const int quarter = warp & 3;                  // TMEM lanes 32 * quarter .. + 31
    const int group = (warp - 2) >> 2;
    const int rloc = quarter * 32 + lane;          // row within the tile
    constexpr int kEpiThreads = 32 * kEpiWarps;
    for (int i = 0; i < n_local; ++i) {
      const int b = i % NA, ob = i & 1;
      // Code tile ob is free once the store of tile i - 2 has read it; the
      // AND over all epilogue threads also makes a timeout CTA-uniform.
      const bool mine = mbar_wait(&acc_full[b], (i / NA) & 1);
      if (tid == kIssuer) bulk_wait_read_1();
      if (!bar_and(1, kEpiThreads, mine)) {
        if (lane == 0) atomicOr(a.err, kErrConsumerWait);
        break;
      }
      tmem_fence_after();
      uint32_t r[kMaxPer][32];
      const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16) + b * (Wb * 32);
#pragma unroll
      for (int v = 0; v < kMaxPer; ++v) {
        const int w = group + kEpiGroups * v;
        if (w < Wb) tmem_ld32(taddr + w * 32, r[v]);
      }
      tmem_wait_ld();
      tmem_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
      const int64_t row0 = (int64_t)(k0 + (int64_t)i * cpp) * kTileRows;
      const int64_t row = row0 + rloc;
      uint8_t* ct = codes + ob * L.code_bytes + rloc * (Wb * 16);
      uint8_t* st = sstage + ob * (kTileRows * Wb) + rloc * Wb;
#pragma unroll
      for (int v = 0; v < kMaxPer; ++v) {
        const int w = group + kEpiGroups * v;
        if (w >= Wb) break;
        if (a.out_f32) {
          if (row < a.M) {
            float4* dst = reinterpret_cast<float4*>(a.y + (row * a.nb + j0 + w) * kBlock);
#pragma unroll
            for (int t = 0; t < 8; ++t)
              __stcs(dst + t, make_float4(__uint_as_float(r[v][4 * t]),
                                          __uint_as_float(r[v][4 * t + 1]),
                                          __uint_as_float(r[v][4 * t + 2]),
                                          __uint_as_float(r[v][4 * t + 3])));
          }
          continue;
        }
        f2 u[16];
#pragma unroll
        for (int m = 0; m < 16; ++m)
          u[m] = pack2(__uint_as_float(r[v][2 * m]), __uint_as_float(r[v][2 * m + 1]));
        const Mx4Block blk = mxfp4_block(u);
        *reinterpret_cast<uint4*>(ct + 16 * code_chunk(w, rloc, a.swz)) = blk.codes;
        st[w] = static_cast<uint8_t>(blk.scale);
      }
      if (a.out_f32) continue;
      fence_proxy_async_smem();                    // generic writes -> TMA store reads
      bar_sync_n(2, kEpiThreads);
      if (tid == kIssuer) {
        tma_store_2d(&qmap, codes + ob * L.code_bytes, j0 * 16, static_cast<int>(row0));
        bulk_commit();
      }
      if (group == 0 && row < a.M) {
        // This row's Wb scale bytes, gathered from the four groups.
        uint8_t* dst = a.scales + row * a.nb + j0;
        const uintptr_t addr = reinterpret_cast<uintptr_t>(dst);
        if (Wb == 8 && (addr & 7) == 0) {
          *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(st);
        } else if (Wb == 4 && (addr & 3) == 0) {
          *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<const uint32_t*>(st);
        } else {
          for (int w = 0; w < Wb; ++w) dst[w] = st[w];
        }
      }
    }
    if (tid == kIssuer) bulk_wait_all();
  }
  // Warps 1..17 meet here; then warp 1 returns the TMEM columns.
  __syncwarp();
  if (warp >= 1) bar_sync_n(3, kMmaThreads - 32);
  if (warp == 1) {
    tmem_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

// Panel width for nb blocks per row: Wb divides nb, 1 <= Wb <= 8, and the
// grid (panels x CTAs per panel, one CTA per SM) keeps the most SMs busy.
// Among equal ones, widths of 4 and more come first (every epilogue group
// then has a block of each tile), the smaller first (more stages fit).
// Returns 0 if no width fits (more panels than SMs).
int mma_panel_width(int nb, int sms) {
  static const int kOrder[kMaxWb] = {4, 5, 6, 7, 8, 3, 2, 1};
  int best = 0;
  double best_use = 0.0;
  for (int Wb : kOrder) {
    if (Wb > nb || nb % Wb) continue;
    const int panels = nb / Wb;
    if (panels > sms) continue;
    const double use = double(sms / panels * panels) / sms;
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
  a.scales = scales;
  a.y = y;
  a.out_f32 = y != nullptr;
  a.nacc = std::min(kMaxAcc, kTmemCols / (a.Wb * 32));
  a.swz = a.Wb == 8 ? kSwz128 : a.Wb == 4 ? kSwz64 : a.Wb == 2 ? kSwz32 : kSwzNone;
  const int fixed = 1024 + static_cast<int>(Layout(a.Wb, 0).total);
  a.stages = std::min(kMaxStages, (di->smem_optin - fixed) / (a.Wb * kABoxBytes));
  if (a.stages < 2) return KQ_ERR_INVALID;
  // At least half of the SM's shared memory, so that no second CTA (of this
  // grid or of the next launch) shares the SM and waits for its TMEM.
  const int smem = std::max(1024 + static_cast<int>(Layout(a.Wb, a.stages).total),
                            di->smem_per_sm / 2 + 1024);
  if (smem > di->smem_optin) return KQ_ERR_INVALID;
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
  // with the swizzle whose span is one box row where one exists.
  CUtensorMap qmap = map;
  if (!a.out_f32) {
    const cuuint64_t qdims[2] = {static_cast<cuuint64_t>(nb) * 16, static_cast<cuuint64_t>(M)};
    const cuuint64_t qstrides[1] = {static_cast<cuuint64_t>(nb) * 16};
    const cuuint32_t qbox[2] = {static_cast<cuuint32_t>(a.Wb * 16), kTileRows};
    const cuuint32_t qestr[2] = {1, 1};
    const CUtensorMapSwizzle sw = a.swz == kSwz128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : a.swz == kSwz64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                  : a.swz == kSwz32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                    : CU_TENSOR_MAP_SWIZZLE_NONE;
    cr = tensor_map_encoder()(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, qdims, qstrides, qbox,
                              qestr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return record_cuda_error(cudaErrorInvalidValue);
  }
  const int per_panel = std::max(1, std::min(di->sms / a.panels, a.row_tiles));
  cudaError_t e = launch_pdl(mma_kernel, dim3(static_cast<unsigned>(per_panel * a.panels)),
                             dim3(kMmaThreads), static_cast<size_t>(smem), st, map, qmap, a);
  if (e != cudaSuccess) return record_cuda_error(e);
  return KQ_OK;
}

}  // namespace kq
