// W4A4 MXFP4 GEMM on the 5th-generation tensor cores (sm_100a):
//
//   C[M][N] = A[M][K] . B[N][K]^T
//
// with A and B as the quantizer writes them: packed E2M1 codes (element 2i
// in the low nibble of byte i) and one E8M0 scale byte per 32 elements along
// K, row-major.  This is the product the transformed layer computes
// (KroQuant review, "Circularity Check", Eq. 1: A = Q(x T), B = Q(W T^-T)).
//
// One CTA computes a 128 x 256 tile of C and walks K in tiles of 256:
//   warp 0      TMA: A tile [128 rows][128 B] and B tile [256 rows][128 B],
//               128-byte swizzle, into a ring of stages
//   warps 6..9  scale loaders, one per stage: the tile's E8M0 bytes from the
//               row-major scale arrays into shared memory in the tensor
//               core's scale layout (128-row x 4-scale chunks of 512 bytes:
//               row r, scale i at byte 16 (r mod 32) + 4 (r div 32) + i).
//               With scales already in that tiled layout
//               (kq_gemm_mxfp4_tiled) there are no scale warps: warp 0 adds
//               one bulk copy per 512-byte chunk run to each stage's loads,
//               since four-byte scale words scattered over rows cost as many
//               L2 requests as the codes themselves.
//   warp 1      allocates TMEM; one lane copies the stage's scales into TMEM
//               (tcgen05.cp) and issues four block-scaled MMAs
//               (tcgen05.mma kind::mxf4, K = 64 each) into a float32
//               accumulator of 256 TMEM columns
//   warps 2..5  epilogue: tcgen05.ld of the accumulator rows, stores to C
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <type_traits>
#include <cstdlib>

#include "kq.h"
#include "kq_device.cuh"
#include "kq_internal.h"
#include "kq_tc.cuh"

namespace kq {
namespace {

constexpr int kBM = 128;                       // UMMA M: rows of A per tile
constexpr int kBN = 256;                       // UMMA N: rows of B per tile
constexpr int kBK = 256;                       // K elements per stage
constexpr int kBKBytes = kBK / 2;              // 128 bytes of codes per row
constexpr int kMmaK = 64;                      // K elements per MMA
constexpr int kStages = 4;
constexpr int kATile = kBM * kBKBytes;         // 16 KiB
constexpr int kBTile = kBN * kBKBytes;         // 32 KiB
constexpr int kSfChunk = 512;                  // 128 rows x 4 scale bytes
constexpr int kChunksPerStage = kBK / 128;     // 2 chunks of 4 scales per row
constexpr int kSfaBytes = kChunksPerStage * kSfChunk;
constexpr int kSfbBytes = kChunksPerStage * (kBN / 128) * kSfChunk;
constexpr int kStageBytes = kATile + kBTile + kSfaBytes + kSfbBytes;
static_assert(kStageBytes % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + (2 * kStages + 2) * 8 + 16;
constexpr int kOutBoxBytes = kBM * 128;        // one store box: 128 rows x 128 bytes
static_assert(kBN * 4 / 128 * kOutBoxBytes <= kStages * kStageBytes, "output tile in the stages");

constexpr int kSfWarp0 = 6;                    // warps 6..9 load scales, one stage each
constexpr int kSfWarps = kStages;
constexpr int kGemmThreads = 32 * (kSfWarp0 + kSfWarps);
constexpr int kBandN = 16;                     // column tiles per raster band
// Scale words (4 bytes) per stage: 2 per row of A and of B.
constexpr int kSfWordsPerStage = (kBM + kBN) * kChunksPerStage;
constexpr int kSfWordsPerLane = kSfWordsPerStage / 32;

// TMEM: the accumulator in columns [0, 256), then per stage 4 columns per
// scale chunk of A and 8 per chunk of B (two 128-row groups).
constexpr int kSfColsA = 4 * kChunksPerStage;
constexpr int kSfColsB = 8 * kChunksPerStage;
constexpr int kSfCol0 = kBN;
constexpr int kTmemCols = 512;
static_assert(kSfCol0 + kStages * (kSfColsA + kSfColsB) <= kTmemCols, "TMEM columns");

// Instruction descriptor, block-scaled kinds: A and B E2M1 (format 1 of
// kind::mxf4), K-major, N = bn, E8M0 scales, M = 128, dense K = 64.  The
// scale-factor ids (byte of the 32-bit TMEM word holding the first scale of
// the MMA's K range) go in bits 29-30 (A) and 4-5 (B).
__host__ __device__ constexpr uint32_t idesc_mxf4(int bn) {
  return (1u << 7) | (1u << 10) | (uint32_t(bn >> 3) << 17) | (1u << 23) |
         (uint32_t(kBM >> 4) << 24);
}

struct GemmArgs {
  int32_t M, N, K;
  int32_t k_tiles, m_tiles, n_tiles;
  int32_t sf_tiles_k, sf_tiles_n;   // tiled scales: 4-scale columns, B row tiles
  int32_t tma_store;                // the epilogue stages the tile and stores it by TMA
  int32_t sf_stride;        // scale bytes per row: K / 32
  int32_t out_bf16;
  const uint8_t* sa;
  const uint8_t* sb;
  void* c;
  int* err;
};

__device__ __forceinline__ void mma_mxf4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t tsfa, uint32_t tsfb,
                                         uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;"
      "\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(tsfa), "r"(tsfb)
      : "memory");
}

// The same MMA over a CTA pair (M = 256): issued by the even CTA, A rows and
// accumulator rows 0..127 in it and 128..255 in the odd one, B's N rows split
// 128 / 128 between their shared memories, each CTA's scales in its TMEM.
__device__ __forceinline__ void mma_mxf4_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t tsfa, uint32_t tsfb,
                                              uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;"
      "\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(tsfa), "r"(tsfb)
      : "memory");
}

// Untiled bulk copy of `bytes` (a multiple of 16, 16-byte aligned ends)
// from global memory into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes),
      "r"(smem_addr(bar))
      : "memory");
}

// Four scale bytes of row `row` (of `rows`) starting at scale index k0, as one
// little-endian word; indices at or past `nsf` (and rows past the end) read
// as 0 (2^-127, finite: those codes are zero-filled by the TMA loads).
template <bool kAligned>
__device__ __forceinline__ uint32_t load_sf_word(const uint8_t* s, int64_t row, int rows, int k0,
                                                 int nsf) {
  if (row >= rows || k0 >= nsf) return 0u;
  const uint8_t* p = s + row * nsf + k0;
  if (kAligned) return __ldg(reinterpret_cast<const uint32_t*>(p));
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (k0 + i < nsf) w |= static_cast<uint32_t>(__ldg(p + i)) << (8 * i);
  return w;
}

// Byte offset of (row r of a 128-row group, 4-scale word) inside a chunk.
__device__ __forceinline__ int sf_chunk_offset(int r) { return 16 * (r & 31) + 4 * (r >> 5); }

// This lane's scale words of k-tile kt: word w = lane + 32 i of the stage is
// (A row w / 2, chunk w mod 2) for w < 256, then (B row (w - 256) / 2, ...).
template <bool kAligned>
__device__ __forceinline__ void load_sf_words(uint32_t (&v)[kSfWordsPerLane], const GemmArgs& a,
                                              int m0, int n0, int kt, int lane) {
  const int kb = kt * (kBK / 32);
#pragma unroll
  for (int i = 0; i < kSfWordsPerLane; ++i) {
    const int w = lane + 32 * i, c = w & 1;
    if (w < kBM * kChunksPerStage)
      v[i] = load_sf_word<kAligned>(a.sa, (int64_t)m0 + (w >> 1), a.M, kb + 4 * c, a.sf_stride);
    else
      v[i] = load_sf_word<kAligned>(a.sb, (int64_t)n0 + ((w - kBM * kChunksPerStage) >> 1), a.N,
                                    kb + 4 * c, a.sf_stride);
  }
}

// Scale modes: row-major scale bytes loaded by the scale warps (4-byte
// words when every row's scales are 4-byte aligned, bytes otherwise), or
// the tiled layout (128-row x 4-scale tiles of 512 bytes), which the
// producer thread copies straight into the stage with bulk copies.
// kSfTiled16: tiled scales with one scale per 16 elements along K (the
// 16-element variant), MMAs of kind::mxf4nvf4 with block16 scaling.
enum SfMode { kSfRowWords = 0, kSfRowBytes = 1, kSfTiled = 2, kSfTiled16 = 3 };

// Per-stage scale geometry: 4-scale chunks of 128 rows per stage (two for
// scales per 32, four for scales per 16), their bytes and TMEM columns.
template <int kSfMode>
struct StageGeom {
  static constexpr int kChunks = kSfMode == kSfTiled16 ? 4 : kChunksPerStage;
  static constexpr int kSfa = kChunks * kSfChunk;
  static constexpr int kSfb = kChunks * (kBN / 128) * kSfChunk;
  static constexpr int kStage = kATile + kBTile + kSfa + kSfb;
  static constexpr int kColsA = 4 * kChunks;
  static constexpr int kColsB = 8 * kChunks;
  static constexpr int kSmem = 1024 + kStages * kStage + (2 * kStages + 2) * 8 + 16;
  static_assert(kStage % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
  static_assert(kSfCol0 + kStages * (kColsA + kColsB) <= kTmemCols, "TMEM columns");
  static_assert(kSmem <= 232448, "shared memory");
};

// Block-scaled MMA with a scale per 16 elements: four E8M0 scales of each
// row per K = 64 (the whole 32-bit TMEM word, scale-factor id 0).
__device__ __forceinline__ void mma_mxf4_b16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t tsfa, uint32_t tsfb,
                                             uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;"
      "\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(tsfa), "r"(tsfb)
      : "memory");
}

// The kN MMAs (K = 64 each) of one k-tile: 64 codes = 32 bytes per MMA, so
// the descriptors' start address steps by 2 (x16 B).  Scales per 32: two per
// row and MMA, bytes 0-1 or 2-3 of the chunk's 32-bit word (scale-factor
// id); scales per 16: four per row and MMA, chunk kk, the whole word.
// kBNt: the tile's N (B rows), 256 or 128; B's scales take 4 TMEM columns
// per 128-row group and chunk.
template <int kSfMode, int kN, int kBNt = kBN>
__device__ __forceinline__ void ktile_mmas(uint32_t tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t tsfa, uint32_t tsfb, int kt) {
  constexpr uint32_t kId = idesc_mxf4(kBNt);
  constexpr int kBCols = 4 * (kBNt / 128);
#pragma unroll
  for (int kk = 0; kk < kN; ++kk) {
    if constexpr (kSfMode == kSfTiled16) {
      mma_mxf4_b16(tmem, adesc + 2 * kk, bdesc + 2 * kk, kId, tsfa + 4 * kk,
                   tsfb + kBCols * kk, (kt | kk) != 0);
    } else {
      const uint32_t sf_id = 2u * (kk & 1);
      const uint32_t idesc = kId | (sf_id << 29) | (sf_id << 4);
      mma_mxf4(tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, tsfa + 4 * (kk >> 1),
               tsfb + kBCols * (kk >> 1), (kt | kk) != 0);
    }
  }
}

// A k-tile's MMAs; a last k-tile that ends inside the stage issues none
// over its zero fill (K elements left: rem).
template <int kSfMode, int kBNt = kBN>
__device__ __forceinline__ void issue_ktile(uint32_t tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t tsfa, uint32_t tsfb, int kt, int rem) {
  static_assert(kBK / kMmaK == 4, "four MMAs per k-tile");
  if (rem > 3 * kMmaK)
    ktile_mmas<kSfMode, 4, kBNt>(tmem, adesc, bdesc, tsfa, tsfb, kt);
  else if (rem > 2 * kMmaK)
    ktile_mmas<kSfMode, 3, kBNt>(tmem, adesc, bdesc, tsfa, tsfb, kt);
  else if (rem > kMmaK)
    ktile_mmas<kSfMode, 2, kBNt>(tmem, adesc, bdesc, tsfa, tsfb, kt);
  else
    ktile_mmas<kSfMode, 1, kBNt>(tmem, adesc, bdesc, tsfa, tsfb, kt);
}

template <int kSfMode>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_mxf4_kernel(const __grid_constant__ CUtensorMap amap,
                     const __grid_constant__ CUtensorMap bmap,
                     const __grid_constant__ CUtensorMap cmap, const GemmArgs a) {
  using Geo = StageGeom<kSfMode>;
  constexpr bool kTiledSf = kSfMode == kSfTiled || kSfMode == kSfTiled16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kStages * Geo::kStage);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* mma_done = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Tile order: bands of kBandN column tiles; inside a band the row tile
  // changes every kBandN CTAs, so a band's slice of B stays in L2 while all
  // row tiles pass over it and each A tile is read by neighbouring CTAs.
  int m0, n0;
  {
    const int t = blockIdx.x;
    const int band = t / (kBandN * a.m_tiles);
    const int r = t - band * kBandN * a.m_tiles;
    const int width = min(kBandN, a.n_tiles - band * kBandN);
    m0 = (r / width) * kBM;
    n0 = (band * kBandN + r % width) * kBN;
  }
  const int nk = a.k_tiles;

  if (kTiledSf) {
    // Chunks past the end of K are not copied; their codes are zero, and
    // the scales there must only be finite.
    for (int s = 0; s < kStages; ++s)
      for (int i = tid; i < (Geo::kSfa + Geo::kSfb) / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(base + s * Geo::kStage + kATile + kBTile)[i] =
            make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      // TMA bytes, plus the stage's scale warp unless the scales come by
      // bulk copy with the codes.
      mbar_init(&full[s], kTiledSf ? 1 : 2);
      mbar_init(&empty[s], 1);                     // tcgen05.commit of the stage's MMAs
    }
    mbar_init(acc_full, 1);
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Programmatic dependent launch: no global access before this.
  pdl_wait_then_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA codes
    if (lane == 0) {
      tma_prefetch_map(&amap);
      tma_prefetch_map(&bmap);
      int s = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kt = 0; kt < nk; ++kt) {
        if (kt >= kStages && !mbar_wait(&empty[s], phase)) {
          ok = false;
          break;
        }
        uint8_t* st = base + s * Geo::kStage;
        if (kTiledSf) {
          // This k-tile's scale columns 2 kt, 2 kt + 1 (those that exist) of
          // the A row tile and of the (up to) two B row tiles.
          const int avail = min(Geo::kChunks, a.sf_tiles_k - Geo::kChunks * kt);
          const int b_tiles = min(kBN / 128, a.sf_tiles_n - n0 / 128);
          const uint32_t sf_bytes = (uint32_t)(avail * (1 + b_tiles)) * kSfChunk;
          mbar_arrive_expect_tx(&full[s], kATile + kBTile + sf_bytes);
          uint8_t* sfa = st + kATile + kBTile;
          bulk_load(sfa, a.sa + ((int64_t)(m0 / 128) * a.sf_tiles_k + Geo::kChunks * kt) *
                                  kSfChunk, avail * kSfChunk, &full[s]);
          for (int g = 0; g < b_tiles; ++g)
            bulk_load(sfa + Geo::kSfa + g * Geo::kChunks * kSfChunk,
                      a.sb + ((int64_t)(n0 / 128 + g) * a.sf_tiles_k + Geo::kChunks * kt) *
                                 kSfChunk, avail * kSfChunk, &full[s]);
        } else {
          mbar_arrive_expect_tx(&full[s], kATile + kBTile);
        }
        tma_load_2d(st, &amap, kt * kBKBytes, m0, &full[s]);
        tma_load_2d(st + kATile, &bmap, kt * kBKBytes, n0, &full[s]);
        issued = kt + 1;
        if (++s == kStages) {
          s = 0;
          if (kt >= kStages) phase ^= 1;
        }
      }
      if (!ok) {
        atomicOr(a.err, kErrProducerWait);
        for (int i = issued > kStages ? issued - kStages : 0; i < issued; ++i)
          mbar_wait(&full[i % kStages], (i / kStages) & 1);
      }
    }
    return;
  }

  if (!kTiledSf && warp >= kSfWarp0) {
    // ---------------------------------------------------------- scale loader
    // Loader warp sw owns stage sw (k-tiles sw, sw + 4, ...), so a stage's
    // scales have four k-tiles of MMA time to arrive; all of a stage's
    // loads are in flight together before the stores.
    const int sw = warp - kSfWarp0;
    const int s = sw;
    uint8_t* sfa = base + s * Geo::kStage + kATile + kBTile;
    uint8_t* sfb = sfa + Geo::kSfa;
    for (int kt = sw, n = 0; kt < nk; kt += kStages, ++n) {
      uint32_t cur[kSfWordsPerLane];
      load_sf_words<kSfMode == kSfRowWords>(cur, a, m0, n0, kt, lane);
      if (n >= 1 && !__all_sync(0xFFFFFFFFu, mbar_wait(&empty[s], (n - 1) & 1))) {
        if (lane == 0) atomicOr(a.err, kErrProducerWait);
        break;
      }
#pragma unroll
      for (int i = 0; i < kSfWordsPerLane; ++i) {
        const int w = lane + 32 * i, c = w & 1;
        if (w < kBM * kChunksPerStage) {
          const int r = w >> 1;
          *reinterpret_cast<uint32_t*>(sfa + c * kSfChunk + sf_chunk_offset(r)) = cur[i];
        } else {
          const int r = (w - kBM * kChunksPerStage) >> 1;
          *reinterpret_cast<uint32_t*>(sfb + (2 * (r >> 7) + c) * kSfChunk +
                                       sf_chunk_offset(r & 127)) = cur[i];
        }
      }
      fence_proxy_async_smem();      // generic stores -> tcgen05.cp reads
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[s]);
    }
    return;
  }

  if (warp == 1) {
    // -------------------------------------------------- scale copies + MMA
    if (lane == 0) {
      int s = 0;
      uint32_t phase = 0;
      // One k-tile: its stage's scales into TMEM, its MMAs (all four in a
      // full k-tile, so that path has no branch; a last k-tile that ends
      // inside the stage issues none over its zero fill), the stage freed.
      auto ktile = [&](int kt, auto full_tile) -> bool {
        if (!mbar_wait(&full[s], phase)) return false;
        tmem_fence_after();
        const uint8_t* st = base + s * Geo::kStage;
        const uint8_t* sfa = st + kATile + kBTile;
        const uint8_t* sfb = sfa + Geo::kSfa;
        const uint32_t tsfa = tmem_base + kSfCol0 + s * (Geo::kColsA + Geo::kColsB);
        const uint32_t tsfb = tsfa + Geo::kColsA;
#pragma unroll
        for (int c = 0; c < Geo::kChunks; ++c) {
          tmem_cp_32x128b_x4(tsfa + 4 * c, smem_desc_rows16(smem_addr(sfa + c * kSfChunk)));
#pragma unroll
          for (int g = 0; g < kBN / 128; ++g)
            tmem_cp_32x128b_x4(tsfb + 8 * c + 4 * g,
                               smem_desc_rows16(smem_addr(sfb + (Geo::kChunks * g + c) * kSfChunk)));
        }
        const uint64_t adesc = smem_desc_sw128(smem_addr(st));
        const uint64_t bdesc = smem_desc_sw128(smem_addr(st + kATile));
        if constexpr (decltype(full_tile)::value)
          ktile_mmas<kSfMode, kBK / kMmaK>(tmem_base, adesc, bdesc, tsfa, tsfb, kt);
        else
          issue_ktile<kSfMode>(tmem_base, adesc, bdesc, tsfa, tsfb, kt, a.K - kt * kBK);
        mma_commit(&empty[s]);         // stage (codes and scales) free once read
        if (++s == kStages) {
          s = 0;
          phase ^= 1;
        }
        return true;
      };
      const int nk_full = a.K % kBK == 0 ? nk : nk - 1;
      bool ok = true;
      int kt = 0;
      for (; ok && kt < nk_full; ++kt) ok = ktile(kt, std::true_type{});
      if (ok && kt < nk) ok = ktile(kt, std::false_type{});
      if (!ok) atomicOr(a.err, kErrConsumerWait);
      mma_commit(acc_full);
      // Every issued MMA completes before the columns are released.
      mma_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue
    const int quarter = warp & 3;                  // TMEM lanes 32 quarter .. +31
    const int row = m0 + quarter * 32 + lane;
    const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, 0));
    if (!ok) {
      if (lane == 0) atomicOr(a.err, kErrConsumerWait);
    } else if (a.tma_store) {
      // Every MMA has completed, so the stage buffers are free: the tile
      // goes there as 128-byte-swizzled boxes of 128 rows x 128 bytes
      // (row r's 16-byte chunk c at c ^ (r mod 8)), then out by TMA stores
      // that clip at the matrix edges.
      tmem_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16);
      const int r = quarter * 32 + lane;
      const int cols_per_box = a.out_bf16 ? 64 : 32;
#pragma unroll 1
      for (int v = 0; v < kBN / 32; ++v) {
        uint32_t x[32];
        tmem_ld32(taddr + 32 * v, x);
        tmem_wait_ld();
        const int col = 32 * v;
        uint8_t* box = base + (col / cols_per_box) * kOutBoxBytes + r * 128;
        if (a.out_bf16) {
          const int c0 = (col % 64) / 8;           // first 16-byte chunk of these 32 columns
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t wv[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const __nv_bfloat162 p = __floats2bfloat162_rn(__uint_as_float(x[8 * q + 2 * h]),
                                                            __uint_as_float(x[8 * q + 2 * h + 1]));
              wv[h] = *reinterpret_cast<const uint32_t*>(&p);
            }
            *reinterpret_cast<uint4*>(box + 16 * ((c0 + q) ^ (r & 7))) =
                make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<uint4*>(box + 16 * (q ^ (r & 7))) =
                make_uint4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
        }
      }
      fence_proxy_async_smem();                    // generic stores -> TMA store reads
      asm volatile("bar.sync 3, %0;" ::"r"(4 * 32) : "memory");
      if (warp == 2 && lane == 0) {
        for (int b = 0; b < kBN / cols_per_box; ++b)
          tma_store_2d(&cmap, base + b * kOutBoxBytes, n0 + b * cols_per_box, m0);
        bulk_commit();
        bulk_wait_all();
      }
    } else {
      tmem_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16);
      const bool vec = (a.N & 7) == 0;
#pragma unroll 1
      for (int v = 0; v < kBN / 32; ++v) {
        uint32_t r[32];
        tmem_ld32(taddr + 32 * v, r);
        tmem_wait_ld();
        const int col = n0 + 32 * v;
        if (row >= a.M || col >= a.N) continue;
        if (a.out_bf16) {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.c) + (int64_t)row * a.N + col;
          if (vec && col + 32 <= a.N) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t wv[4];
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const __nv_bfloat162 p = __floats2bfloat162_rn(__uint_as_float(r[8 * q + 2 * h]),
                                                              __uint_as_float(r[8 * q + 2 * h + 1]));
                wv[h] = *reinterpret_cast<const uint32_t*>(&p);
              }
              *reinterpret_cast<uint4*>(dst + 8 * q) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (col + i < a.N) dst[i] = __float2bfloat16_rn(__uint_as_float(r[i]));
          }
        } else {
          float* dst = static_cast<float*>(a.c) + (int64_t)row * a.N + col;
          if (vec && col + 32 <= a.N) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<float4*>(dst + 4 * q) =
                  make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                              __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (col + i < a.N) dst[i] = __uint_as_float(r[i]);
          }
        }
      }
    }
    tmem_fence_before();
  }
  // Warps 1..5 meet here; then warp 1 returns the TMEM columns.
  asm volatile("bar.sync 2, %0;" ::"r"(5 * 32) : "memory");
  if (warp == 1) {
    tmem_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Row-major packed codes [rows][K/2] as a 2-D byte tensor; a box is
// `box_rows` rows of 128 bytes (256 codes), 128-byte swizzle.
bool encode_codes_map(CUtensorMap* map, const uint8_t* q, int64_t rows, int64_t K, int box_rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  const cuuint32_t box[2] = {kBKBytes, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return tensor_map_encoder()(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(q), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// Persistent variant (tiled scales): one CTA per SM walks the banded tile
// order with four stages and a separate 16 KiB staging box, so the producer
// runs on into the next tile while the epilogue drains.  With bf16 output an
// epilogue thread holds its row's 256 outputs as 128 registers of bf16
// pairs, so the accumulator is released as soon as it has been read and the
// MMAs of tile i + 1 start while tile i's four boxes still leave by TMA.
constexpr int kStagingBytes = kOutBoxBytes;              // 16 KiB: four 4 KiB boxes
constexpr int kPBoxRows = 32;                            // rows of one output box
constexpr int kPThreads = 32 * 6;

// Geometry of the persistent kernel per scale mode and tile width N:
//   N = 256, one accumulator of 256 TMEM columns: four stages of 51 KiB with
//   scales per 32, three of 54 KiB with scales per 16 (four do not fit
//   beside the staging box);
//   N = 128 (scales per 32), two accumulators of 128 columns, so that the
//   MMAs of tile i + 1 run while the epilogue drains tile i: six stages of
//   34 KiB.
template <int kSfMode, int kBNt = kBN>
struct PGeom {
  static constexpr int kChunks = kSfMode == kSfTiled16 ? 4 : kChunksPerStage;
  static constexpr int kGroups = kBNt / 128;               // 128-row groups of B
  static constexpr int kBTile = kBNt * kBKBytes;
  static constexpr int kSfa = kChunks * kSfChunk;
  static constexpr int kSfb = kChunks * kGroups * kSfChunk;
  static constexpr int kStage = kATile + kBTile + kSfa + kSfb;
  static constexpr int kColsA = 4 * kChunks;
  static constexpr int kColsB = 4 * kGroups * kChunks;
  static constexpr int kAcc = kBNt == 128 ? 2 : 1;         // accumulators
  static constexpr int kSfCol0 = kAcc * kBNt;
  static constexpr int kStages = kBNt == 128 ? 6 : (kSfMode == kSfTiled16 ? 3 : 4);
  static constexpr int kSmem = 1024 + kStages * kStage + kStagingBytes +
                               (2 * kStages + 2 * kAcc + 2) * 8 + 16;
  static_assert(kStage % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
  static_assert(kSmem <= 232448, "shared memory");
  static_assert(kSfCol0 + kStages * (kColsA + kColsB) <= kTmemCols, "TMEM columns");
};

// L2 policies: the operand tiles are read again by other tiles of the band
// (kept), the output is written once (evicted first), so that the output
// stream does not push the operands out of L2.
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, int c0, int c1,
                                                 uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar)), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap* map, const void* src, int c0,
                                                  int c1, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1],"
      " %4;" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(smem_addr(src)), "r"(c0), "r"(c1), "l"(pol)
      : "memory");
}

// Tile t of the banded order (bands of kBandN column tiles, the row tile
// changing fastest), for tiles of bn columns.
__device__ __forceinline__ void tile_origin(const GemmArgs& a, int t, int& m0, int& n0,
                                            int bn = kBN) {
  const int band = t / (kBandN * a.m_tiles);
  const int r = t - band * kBandN * a.m_tiles;
  const int width = min(kBandN, a.n_tiles - band * kBandN);
  m0 = (r / width) * kBM;
  n0 = (band * kBandN + r % width) * bn;
}

template <int kSfMode, int kBNt>
__global__ void __launch_bounds__(kPThreads, 1)
    gemm_mxf4_persistent(const __grid_constant__ CUtensorMap amap,
                         const __grid_constant__ CUtensorMap bmap,
                         const __grid_constant__ CUtensorMap cmap, const GemmArgs a) {
  using P = PGeom<kSfMode, kBNt>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* staging = base + P::kStages * P::kStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + kStagingBytes);
  uint64_t* empty = full + P::kStages;
  uint64_t* acc_full = empty + P::kStages;
  uint64_t* acc_empty = acc_full + P::kAcc;
  uint64_t* mma_done = acc_empty + P::kAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_tiles_total = a.m_tiles * a.n_tiles;
  const int nk = a.k_tiles;

  for (int st = 0; st < P::kStages; ++st)
    for (int i = tid; i < (P::kSfa + P::kSfb) / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(base + st * P::kStage + kATile + P::kBTile)[i] =
          make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (tid == 0) {
    for (int st = 0; st < P::kStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);
    }
    for (int b = 0; b < P::kAcc; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);           // one arrival per epilogue warp
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Set-up above overlaps the previous kernel of the stream (programmatic
  // dependent launch); operands are read and C written only after this.
  pdl_wait_then_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_map(&amap);
      tma_prefetch_map(&bmap);
      const uint64_t pol_keep = policy_evict_last();
      int s = 0, issued = 0, g = 0;          // g: k-tiles issued over all tiles
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles_total && ok; t += gridDim.x) {
        int m0, n0;
        tile_origin(a, t, m0, n0, kBNt);
        const int b_tiles = min(P::kGroups, a.sf_tiles_n - n0 / 128);
        for (int kt = 0; kt < nk; ++kt, ++g) {
          if (g >= P::kStages && !mbar_wait(&empty[s], phase)) {
            ok = false;
            break;
          }
          uint8_t* stg = base + s * P::kStage;
          const int avail = min(P::kChunks, a.sf_tiles_k - P::kChunks * kt);
          mbar_arrive_expect_tx(&full[s], kATile + P::kBTile +
                                              (uint32_t)(avail * (1 + b_tiles)) * kSfChunk);
          uint8_t* sfa = stg + kATile + P::kBTile;
          bulk_load(sfa, a.sa + ((int64_t)(m0 / 128) * a.sf_tiles_k + P::kChunks * kt) *
                                  kSfChunk, avail * kSfChunk, &full[s]);
          for (int gb = 0; gb < b_tiles; ++gb)
            bulk_load(sfa + P::kSfa + gb * P::kChunks * kSfChunk,
                      a.sb + ((int64_t)(n0 / 128 + gb) * a.sf_tiles_k + P::kChunks * kt) *
                                 kSfChunk, avail * kSfChunk, &full[s]);
          tma_load_2d_hint(stg, &amap, kt * kBKBytes, m0, &full[s], pol_keep);
          tma_load_2d_hint(stg + kATile, &bmap, kt * kBKBytes, n0, &full[s], pol_keep);
          issued = g + 1;
          if (++s == P::kStages) {
            s = 0;
            if (g >= P::kStages) phase ^= 1;
          }
        }
      }
      if (!ok) {
        atomicOr(a.err, kErrProducerWait);
        for (int i = issued > P::kStages ? issued - P::kStages : 0; i < issued; ++i)
          mbar_wait(&full[i % P::kStages], (i / P::kStages) & 1);
      }
    }
    return;
  }

  if (warp == 1) {
    // -------------------------------------------------- scale copies + MMA
    if (lane == 0) {
      int s = 0, i = 0;
      uint32_t phase = 0;
      uint32_t tacc = tmem_base;             // the accumulator of the current tile
      bool ok = true;
      // One k-tile: its stage's scales into TMEM, its MMAs (all four in a
      // full k-tile, so that path has no branch; a last k-tile that ends
      // inside the stage issues none over its zero fill), the stage freed.
      auto ktile = [&](int kt, auto full_tile) -> bool {
        if (!mbar_wait(&full[s], phase)) return false;
        tmem_fence_after();
        const uint8_t* stg = base + s * P::kStage;
        const uint8_t* sfa = stg + kATile + P::kBTile;
        const uint8_t* sfb = sfa + P::kSfa;
        const uint32_t tsfa = tmem_base + P::kSfCol0 + s * (P::kColsA + P::kColsB);
        const uint32_t tsfb = tsfa + P::kColsA;
#pragma unroll
        for (int c = 0; c < P::kChunks; ++c) {
          tmem_cp_32x128b_x4(tsfa + 4 * c, smem_desc_rows16(smem_addr(sfa + c * kSfChunk)));
#pragma unroll
          for (int gb = 0; gb < P::kGroups; ++gb)
            tmem_cp_32x128b_x4(tsfb + 4 * P::kGroups * c + 4 * gb,
                               smem_desc_rows16(smem_addr(sfb + (P::kChunks * gb + c) * kSfChunk)));
        }
        const uint64_t adesc = smem_desc_sw128(smem_addr(stg));
        const uint64_t bdesc = smem_desc_sw128(smem_addr(stg + kATile));
        if constexpr (decltype(full_tile)::value)
          ktile_mmas<kSfMode, kBK / kMmaK, kBNt>(tacc, adesc, bdesc, tsfa, tsfb, kt);
        else
          issue_ktile<kSfMode, kBNt>(tacc, adesc, bdesc, tsfa, tsfb, kt, a.K - kt * kBK);
        mma_commit(&empty[s]);
        if (++s == P::kStages) {
          s = 0;
          phase ^= 1;
        }
        return true;
      };
      for (int t = blockIdx.x; t < n_tiles_total && ok; t += gridDim.x, ++i) {
        // Accumulator i mod kAcc is free once the epilogue has read tile
        // i - kAcc.
        const int b = i % P::kAcc;
        if (i >= P::kAcc && !mbar_wait(&acc_empty[b], ((i / P::kAcc) - 1) & 1)) {
          ok = false;
          break;
        }
        tacc = tmem_base + b * kBNt;
        tmem_fence_after();
        const int nk_full = a.K % kBK == 0 ? nk : nk - 1;
        int kt = 0;
        for (; ok && kt < nk_full; ++kt) ok = ktile(kt, std::true_type{});
        if (ok && kt < nk) ok = ktile(kt, std::false_type{});
        if (ok) mma_commit(&acc_full[b]);
      }
      if (!ok) atomicOr(a.err, kErrConsumerWait);
      mma_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Rows of TMEM lane quarter (warp mod 4).  Each warp sends its 32 rows
    // on its own: a 4 KiB slice of the staging area holds one box of 32 rows
    // x 128 bytes (128-byte swizzle: row r's 16-byte chunk c at c ^ (r mod
    // 8)), stored by the warp's first lane, so the four warps' stores
    // proceed side by side with no barrier between them.
    const int quarter = warp & 3;
    const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16);
    uint8_t* wstage = staging + quarter * (kPBoxRows * 128);
    const uint64_t pol_stream = policy_evict_first();
    uint8_t* srow = wstage + lane * 128;
    // Box `col` of this warp's rows: wait until its previous store has read
    // the slice, fill it, store it.
    auto store_box = [&](int m0, int col, const uint32_t (&wv)[32]) {
      if (lane == 0) bulk_wait_read_0();
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(srow + 16 * (c ^ (lane & 7))) =
            make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d_hint(&cmap, wstage, col, m0 + quarter * kPBoxRows, pol_stream);
        bulk_commit();
      }
    };
    int i = 0;
    for (int t = blockIdx.x; t < n_tiles_total; t += gridDim.x, ++i) {
      int m0, n0;
      tile_origin(a, t, m0, n0, kBNt);
      const int b = i % P::kAcc;
      const uint32_t tb = taddr + b * kBNt;
      // One AND-barrier makes a timeout the same for the four warps.
      const bool got = mbar_wait(&acc_full[b], (i / P::kAcc) & 1);
      if (!bar_and(3, 4 * 32, got)) {
        if (lane == 0) atomicOr(a.err, kErrConsumerWait);
        break;
      }
      tmem_fence_after();
      if (a.out_bf16) {
        // The row's 256 columns in two rounds of four loads with one wait
        // each, so that the loads' latencies overlap and the accumulator is
        // released sooner.
        constexpr int kLdPerWait = 4;
        uint32_t h[kBNt / 2];                     // the row as bf16 pairs
#pragma unroll
        for (int v0 = 0; v0 < kBNt / 32; v0 += kLdPerWait) {
          uint32_t x[kLdPerWait][32];
#pragma unroll
          for (int u = 0; u < kLdPerWait; ++u) tmem_ld32(tb + 32 * (v0 + u), x[u]);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < kLdPerWait; ++u)
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const __nv_bfloat162 p = __floats2bfloat162_rn(__uint_as_float(x[u][2 * q]),
                                                             __uint_as_float(x[u][2 * q + 1]));
              h[16 * (v0 + u) + q] = *reinterpret_cast<const uint32_t*>(&p);
            }
        }
        // Every column has been read: the MMAs of the next tile may start.
        tmem_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
#pragma unroll
        for (int ob = 0; ob < kBNt / 64; ++ob) {
          uint32_t wv[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) wv[k] = h[32 * ob + k];
          store_box(m0, n0 + 64 * ob, wv);
        }
      } else {
        // float32: eight boxes of 32 columns, each read out of TMEM as it
        // goes; the accumulator is released after the last read.
#pragma unroll 1
        for (int ob = 0; ob < kBNt / 32; ++ob) {
          uint32_t x[32];
          tmem_ld32(tb + 32 * ob, x);
          tmem_wait_ld();
          if (ob == kBNt / 32 - 1) {
            tmem_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
          }
          store_box(m0, n0 + 32 * ob, x);
        }
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
    tmem_fence_before();
  }
  asm volatile("bar.sync 2, %0;" ::"r"(5 * 32) : "memory");
  if (warp == 1) {
    tmem_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// CTA-pair kernel (tiled scales per 32): clusters of two CTAs walk the banded
// order of 256 x 256 output tiles with tcgen05.mma.cta_group::2 (M = 256).
// Each CTA loads its 128 rows of A and its 128 rows of B, so B costs each SM
// half the bytes per flop of a one-CTA tile, plus the scales of its A rows
// and of all 256 B rows (the MMA reads B's scales from each CTA's own TMEM).
// The even CTA (rank 0) issues the scale copies, the MMAs and the commits;
// the commits arrive on the barriers of both CTAs, and every TMA load of the
// pair counts its bytes on rank 0's stage barrier.  No load uses cluster
// multicast.  Every cross-CTA wait is bounded; both CTAs always reach the
// final TMEM release.
constexpr int kQBN = 128;                                     // B rows per CTA
constexpr int kQBTile = kQBN * kBKBytes;                      // 16 KiB
constexpr int kQStage = kATile + kQBTile + kSfaBytes + kSfbBytes;   // 35 KiB
constexpr int kQStages = 6;
constexpr int kQBoxRows = 64;                                 // staging box: 64 rows x 128 B
constexpr int kQStaging = kQBoxRows * 128;
constexpr int kQSmem = 1024 + kQStages * kQStage + kQStaging + (2 * kQStages + 4) * 8 + 16;
constexpr int kQTile = 2 * kBM;                               // 256 rows and columns a tile
static_assert(kQStage % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
static_assert(kQSmem <= 232448, "shared memory");
static_assert(kSfCol0 + kQStages * (kSfColsA + kSfColsB) <= kTmemCols, "TMEM columns");
// M = 256 over the pair, N = 256.
constexpr uint32_t kIdescMxf4Pair = (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) |
                                    (1u << 23) | (uint32_t(kQTile >> 4) << 24);
// Bytes one k-tile brings into the pair: codes of 128 A rows and 128 B rows,
// the A scales of 128 rows and the B scales of 256 rows, per CTA.
constexpr uint32_t kQTxBytes = 2u * kQStage;

struct PairArgs {
  int32_t K, k_tiles, m_tiles, n_tiles;     // tiles of 256 x 256
  int32_t out_bf16;
  int* err;
};

__device__ __forceinline__ void pair_tile_origin(const PairArgs& a, int t, int& m0, int& n0) {
  const int band = t / (kBandN * a.m_tiles);
  const int r = t - band * kBandN * a.m_tiles;
  const int width = min(kBandN, a.n_tiles - band * kBandN);
  m0 = (r / width) * kQTile;
  n0 = (band * kBandN + r % width) * kQTile;
}

__global__ void __launch_bounds__(kPThreads, 1)
    gemm_mxf4_pair(const __grid_constant__ CUtensorMap amap,
                   const __grid_constant__ CUtensorMap bmap,
                   const __grid_constant__ CUtensorMap sfamap,
                   const __grid_constant__ CUtensorMap sfbmap,
                   const __grid_constant__ CUtensorMap cmap, const PairArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* staging = base + kQStages * kQStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + kQStaging);
  uint64_t* empty = full + kQStages;
  uint64_t* acc_full = empty + kQStages;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int n_tiles_total = a.m_tiles * a.n_tiles;
  const int nk = a.k_tiles;

  if (tid == 0) {
    for (int st = 0; st < kQStages; ++st) {
      mbar_init(&full[st], 1);               // rank 0's producer, plus the pair's bytes
      mbar_init(&empty[st], 1);              // rank 0's commit, multicast
    }
    mbar_init(acc_full, 1);                  // rank 0's commit, multicast
    mbar_init(acc_empty, 8);                 // the four epilogue warps of each CTA
    fence_mbar_init_cluster();
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, kTmemCols);
  tmem_fence_before();
  cluster_sync();                            // barriers of both CTAs initialised
  tmem_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_map(&amap);
      tma_prefetch_map(&bmap);
      tma_prefetch_map(&sfamap);
      tma_prefetch_map(&sfbmap);
      int s = 0, g = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = pair; t < n_tiles_total && ok; t += n_pairs) {
        int m0, n0;
        pair_tile_origin(a, t, m0, n0);
        const int am0 = m0 + (int)rank * kBM, bn0 = n0 + (int)rank * kQBN;
        for (int kt = 0; kt < nk; ++kt, ++g) {
          if (g >= kQStages && !mbar_wait(&empty[s], phase)) {
            ok = false;
            break;
          }
          uint8_t* stg = base + s * kQStage;
          const uint32_t fb = cluster_addr(&full[s], 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[s], kQTxBytes);
          uint8_t* sfa = stg + kATile + kQBTile;
          // Scales: chunks 2 kt, 2 kt + 1 of this CTA's A row tile and of
          // the tile's two B row tiles (zero past the ends).
          tma_load_4d_pair(sfa, &sfamap, 0, 0, 2 * kt, am0 / 128, fb);
          tma_load_4d_pair(sfa + kSfaBytes, &sfbmap, 0, 0, 2 * kt, n0 / 128, fb);
          tma_load_2d_pair(stg, &amap, kt * kBKBytes, am0, fb);
          tma_load_2d_pair(stg + kATile, &bmap, kt * kBKBytes, bn0, fb);
          if (++s == kQStages) {
            s = 0;
            if (g >= kQStages) phase ^= 1;
          }
        }
      }
      if (!ok) atomicOr(a.err, kErrProducerWait);
    }
  } else if (warp == 1) {
    // -------------------------------------------------- scale copies + MMA
    if (rank == 0 && lane == 0) {
      int s = 0, i = 0;
      uint32_t phase = 0;
      bool ok = true;
      auto ktile = [&](int kt, auto full_tile) -> bool {
        if (!mbar_wait(&full[s], phase)) return false;
        tmem_fence_after();
        const uint8_t* stg = base + s * kQStage;
        const uint8_t* sfa = stg + kATile + kQBTile;
        const uint8_t* sfb = sfa + kSfaBytes;
        const uint32_t tsfa = tmem_base + kSfCol0 + s * (kSfColsA + kSfColsB);
        const uint32_t tsfb = tsfa + kSfColsA;
#pragma unroll
        for (int c = 0; c < kChunksPerStage; ++c) {
          tmem_cp_pair_32x128b_x4(tsfa + 4 * c, smem_desc_rows16(smem_addr(sfa + c * kSfChunk)));
#pragma unroll
          for (int gb = 0; gb < kBN / 128; ++gb)
            tmem_cp_pair_32x128b_x4(tsfb + 8 * c + 4 * gb,
                                    smem_desc_rows16(smem_addr(sfb + (2 * gb + c) * kSfChunk)));
        }
        const uint64_t adesc = smem_desc_sw128(smem_addr(stg));
        const uint64_t bdesc = smem_desc_sw128(smem_addr(stg + kATile));
        const int n_mma = decltype(full_tile)::value
                              ? kBK / kMmaK
                              : min(kBK / kMmaK, (a.K - kt * kBK + kMmaK - 1) / kMmaK);
#pragma unroll
        for (int kk = 0; kk < kBK / kMmaK; ++kk) {
          if (!decltype(full_tile)::value && kk >= n_mma) break;
          const uint32_t sf_id = 2u * (kk & 1);
          const uint32_t idesc = kIdescMxf4Pair | (sf_id << 29) | (sf_id << 4);
          mma_mxf4_pair(tmem_base, adesc + 2 * kk, bdesc + 2 * kk, idesc, tsfa + 4 * (kk >> 1),
                        tsfb + 8 * (kk >> 1), (kt | kk) != 0);
        }
        mma_commit_pair(&empty[s]);
        if (++s == kQStages) {
          s = 0;
          phase ^= 1;
        }
        return true;
      };
      for (int t = pair; t < n_tiles_total && ok; t += n_pairs, ++i) {
        // The accumulators are free once both CTAs' epilogues read tile i - 1.
        if (i >= 1 && !mbar_wait_cluster(acc_empty, (i - 1) & 1)) {
          ok = false;
          break;
        }
        tmem_fence_after();
        const int nk_full = a.K % kBK == 0 ? nk : nk - 1;
        int kt = 0;
        for (; ok && kt < nk_full; ++kt) ok = ktile(kt, std::true_type{});
        if (ok && kt < nk) ok = ktile(kt, std::false_type{});
        mma_commit_pair(acc_full);           // also after a failed wait: epilogues go on
      }
      if (!ok) atomicOr(a.err, kErrConsumerWait);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // This CTA's 128 accumulator rows (TMEM lane quarter = warp mod 4),
    // through the staging box as 128-byte-swizzled boxes of 128 rows x 128
    // bytes, one box at a time.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16);
    const bool issuer = warp == 2 && lane == 0;
    const uint32_t acc_empty0 = cluster_addr(acc_empty, 0);
    constexpr int kParts = kBM / kQBoxRows;         // row boxes per column box
    const int part = r / kQBoxRows;
    uint8_t* srow = staging + (r - part * kQBoxRows) * 128;
    auto epi_sync = [] { asm volatile("bar.sync 3, %0;" ::"r"(4 * 32) : "memory"); };
    auto store_box = [&](int row0, int col, const uint32_t (&wv)[32]) {
#pragma unroll
      for (int pp = 0; pp < kParts; ++pp) {
        if (issuer) bulk_wait_read_0();
        epi_sync();
        if (part == pp) {
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(srow + 16 * (c ^ (r & 7))) =
                make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
        }
        fence_proxy_async_smem();
        epi_sync();
        if (issuer) {
          tma_store_2d(&cmap, staging, col, row0 + pp * kQBoxRows);
          bulk_commit();
        }
      }
    };
    bool ok = true;
    int i = 0;
    for (int t = pair; t < n_tiles_total; t += n_pairs, ++i) {
      int m0, n0;
      pair_tile_origin(a, t, m0, n0);
      const int row0 = m0 + (int)rank * kBM;
      // One AND-barrier makes a timeout the same for the four warps, which
      // then stop (one bounded wait per failure, not one per tile).
      ok = bar_and(3, 4 * 32, mbar_wait(acc_full, i & 1));
      if (!ok) break;
      tmem_fence_after();
      if (a.out_bf16) {
        uint32_t h[kBN / 2];
#pragma unroll
        for (int v = 0; v < kBN / 32; ++v) {
          uint32_t x[32];
          tmem_ld32(taddr + 32 * v, x);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const __nv_bfloat162 p =
                __floats2bfloat162_rn(__uint_as_float(x[2 * q]), __uint_as_float(x[2 * q + 1]));
            h[16 * v + q] = *reinterpret_cast<const uint32_t*>(&p);
          }
        }
        tmem_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty0);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          uint32_t wv[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) wv[k] = h[32 * b + k];
          store_box(row0, n0 + 64 * b, wv);
        }
      } else {
#pragma unroll 1
        for (int b = 0; b < kBN / 32; ++b) {
          uint32_t x[32];
          tmem_ld32(taddr + 32 * b, x);
          tmem_wait_ld();
          if (b == kBN / 32 - 1) {
            tmem_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty0);
          }
          store_box(row0, n0 + 32 * b, x);
        }
      }
    }
    if (!ok && lane == 0) atomicOr(a.err, kErrConsumerWait);
    if (issuer) bulk_wait_all();
    tmem_fence_before();
  }
  // Neither CTA leaves, nor frees its TMEM, before the other has made all its
  // arrivals on its barriers and the MMAs on its memory have completed: every
  // wait above is bounded, so both CTAs get here.
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    tmem_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace
}  // namespace kq

using namespace kq;

namespace kq {
namespace {

// The persistent kernel for the tiled layout with TMA stores (measured
// ahead of the one-tile-per-CTA kernel at every K from 1152 to 16384);
// KQ_GEMM_PERSISTENT=0/1 forces either (measurements, tests).
bool persistent_gemm() {
  const char* e = getenv("KQ_GEMM_PERSISTENT");
  return e ? atoi(e) != 0 : true;
}

// The same choice for scales per 16 (three persistent stages against the
// one-tile-per-CTA kernel's four); KQ_GEMM16_PERSISTENT=0/1 forces either.
bool persistent_gemm16() {
  const char* e = getenv("KQ_GEMM16_PERSISTENT");
  return e ? atoi(e) != 0 : true;
}

// Tile width of the persistent kernel with scales per 32: 256 columns with
// one accumulator, or 128 with two (the next tile's MMAs overlap the
// epilogue's drain, at twice the A traffic per flop).  KQ_GEMM_BN=128/256
// forces either (measurements, tests).
int gemm_tile_n(int64_t K) {
  const char* e = getenv("KQ_GEMM_BN");
  if (e) return atoi(e) == 128 ? 128 : 256;
  (void)K;
  return 256;
}

// The CTA-pair kernel for scales per 32 (KQ_GEMM_PAIR=1 selects it).
bool pair_gemm() {
  const char* e = getenv("KQ_GEMM_PAIR");
  return e ? atoi(e) != 0 : false;
}

// Tiled scales [row tiles][4-scale columns][512 bytes] as a 4-D byte tensor
// {256, 2, columns, row tiles}; a box {256, 2, 2, box_tiles} is the two
// columns of one k-tile for box_tiles row tiles (zeros past either end).
bool encode_scales_map(CUtensorMap* map, const uint8_t* sf, int64_t row_tiles, int64_t cols,
                       int box_tiles) {
  const cuuint64_t dims[4] = {256, 2, static_cast<cuuint64_t>(cols),
                              static_cast<cuuint64_t>(row_tiles)};
  const cuuint64_t strides[3] = {256, 512, static_cast<cuuint64_t>(cols) * 512};
  const cuuint32_t box[4] = {256, 2, 2, static_cast<cuuint32_t>(box_tiles)};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return tensor_map_encoder()(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<uint8_t*>(sf),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launches the CTA-pair kernel: clusters of two, as many as can be resident.
int launch_gemm_pair(const CUtensorMap& amap, const uint8_t* qb, const uint8_t* sa,
                     const uint8_t* sb, const CUtensorMap& cmap, const GemmArgs& g,
                     const DeviceInfo* di, int dev, cudaStream_t st) {
  CUtensorMap bmap, sfamap, sfbmap;
  if (!encode_codes_map(&bmap, qb, g.N, g.K, kQBN) ||
      !encode_scales_map(&sfamap, sa, (g.M + 127) / 128, g.sf_tiles_k, 1) ||
      !encode_scales_map(&sfbmap, sb, g.sf_tiles_n, g.sf_tiles_k, 2))
    return record_cuda_error(cudaErrorInvalidValue);
  PairArgs pa{};
  pa.K = g.K;
  pa.k_tiles = g.k_tiles;
  pa.m_tiles = (g.M + kQTile - 1) / kQTile;
  pa.n_tiles = (g.N + kQTile - 1) / kQTile;
  pa.out_bf16 = g.out_bf16;
  pa.err = g.err;
  int rc = allow_smem<gemm_mxf4_pair>(kQSmem, dev);
  if (rc != KQ_OK) return rc;
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = kQSmem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * (di->sms / 2)));
  int clusters = 0;
  cudaError_t e = cudaOccupancyMaxActiveClusters(&clusters, gemm_mxf4_pair, &cfg);
  if (e != cudaSuccess || clusters < 1) return record_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidConfiguration);
  const int64_t tiles = (int64_t)pa.m_tiles * pa.n_tiles;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * std::min<int64_t>(tiles, clusters)));
  e = cudaLaunchKernelEx(&cfg, gemm_mxf4_pair, amap, bmap, sfamap, sfbmap, cmap, pa);
  if (e != cudaSuccess) return record_cuda_error(e);
  return KQ_OK;
}

int launch_gemm(const uint8_t* qa, const uint8_t* sa, const uint8_t* qb, const uint8_t* sb,
                int64_t M, int64_t N, int64_t K, void* c, int c_dtype, void* stream,
                bool tiled, int scale_block = 32) {
  if (M < 0 || N < 0 || K < 32 || K % 32 != 0) return KQ_ERR_INVALID;
  if (c_dtype != KQ_OUT_F32 && c_dtype != KQ_OUT_BF16) return KQ_ERR_INVALID;
  if (M == 0 || N == 0) return KQ_OK;
  if (M > (int64_t(1) << 31) - kBM || N > (int64_t(1) << 31) - kBN || K > (int64_t(1) << 31) - kBK)
    return KQ_ERR_INVALID;
  if (((M + kBM - 1) / kBM) * ((N + kBN - 1) / kBN) > (int64_t(1) << 31) - 1) return KQ_ERR_INVALID;
  if (!qa || !sa || !qb || !sb || !c) return KQ_ERR_INVALID;
  auto al = [](const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; };
  if (!al(qa, 16) || !al(qb, 16) || !al(c, 16)) return KQ_ERR_INVALID;
  if (tiled && (!al(sa, 16) || !al(sb, 16))) return KQ_ERR_INVALID;
  const DeviceInfo* di = nullptr;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != KQ_OK) return rc;
  GemmArgs a{};
  rc = device_error_word(dev, &a.err);
  if (rc != KQ_OK) return rc;
  a.M = static_cast<int32_t>(M);
  a.N = static_cast<int32_t>(N);
  a.K = static_cast<int32_t>(K);
  a.k_tiles = static_cast<int32_t>((K + kBK - 1) / kBK);
  a.m_tiles = static_cast<int32_t>((M + kBM - 1) / kBM);
  a.n_tiles = static_cast<int32_t>((N + kBN - 1) / kBN);
  a.sf_stride = static_cast<int32_t>(K / 32);
  a.sf_tiles_k = static_cast<int32_t>((K / scale_block + 3) / 4);
  a.sf_tiles_n = static_cast<int32_t>((N + 127) / 128);
  a.out_bf16 = c_dtype == KQ_OUT_BF16;
  a.sa = sa;
  a.sb = sb;
  a.c = c;
  CUtensorMap amap, bmap, cmap;
  if (!encode_codes_map(&amap, qa, M, K, kBM) || !encode_codes_map(&bmap, qb, N, K, kBN))
    return record_cuda_error(cudaErrorInvalidValue);
  // TMA-store epilogue when the output row pitch is a multiple of 16 bytes.
  const int esize = c_dtype == KQ_OUT_BF16 ? 2 : 4;
  a.tma_store = (N * esize) % 16 == 0;
  const bool pair = tiled && a.tma_store && scale_block == 32 && pair_gemm();
  cmap = amap;
  if (a.tma_store) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * esize};
    // Output boxes of 128 bytes x 128 rows (per-tile kernel), the pair
    // kernel's rows, or 32 rows (persistent kernels: one box per warp).
    const bool pers = scale_block == 16 ? persistent_gemm16()
                                        : (!pair && tiled && persistent_gemm());
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esize),
                               static_cast<cuuint32_t>(pair ? kQBoxRows
                                                            : pers ? kPBoxRows : kBM)};
    const cuuint32_t estr[2] = {1, 1};
    if (tensor_map_encoder()(&cmap,
                             esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                        : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                             2, c, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return record_cuda_error(cudaErrorInvalidValue);
  }
  const dim3 grid(static_cast<unsigned>(a.m_tiles * a.n_tiles));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (scale_block == 16 && a.tma_store && persistent_gemm16()) {
    rc = allow_smem<gemm_mxf4_persistent<kSfTiled16, kBN>>(PGeom<kSfTiled16>::kSmem, dev);
    if (rc != KQ_OK) return rc;
    const int pgrid = static_cast<int>(std::min<int64_t>((int64_t)a.m_tiles * a.n_tiles, di->sms));
    cudaError_t le = launch_pdl(gemm_mxf4_persistent<kSfTiled16, kBN>, dim3(pgrid),
                                dim3(kPThreads), PGeom<kSfTiled16>::kSmem, st, amap, bmap, cmap,
                                a);
    if (le != cudaSuccess) return record_cuda_error(le);
  } else if (scale_block == 16) {
    using G = StageGeom<kSfTiled16>;
    rc = allow_smem<gemm_mxf4_kernel<kSfTiled16>>(G::kSmem, dev);
    if (rc != KQ_OK) return rc;
    cudaError_t le = launch_pdl(gemm_mxf4_kernel<kSfTiled16>, grid, dim3(32 * kSfWarp0), G::kSmem,
                                st, amap, bmap, cmap, a);
    if (le != cudaSuccess) return record_cuda_error(le);
  } else if (pair) {
    return launch_gemm_pair(amap, qb, sa, sb, cmap, a, di, dev, st);
  } else if (tiled && a.tma_store && persistent_gemm()) {
    cudaError_t le;
    if (gemm_tile_n(K) == 128) {
      // Tiles of 128 columns with two accumulators.
      a.n_tiles = static_cast<int32_t>((N + 127) / 128);
      if (!encode_codes_map(&bmap, qb, N, K, 128)) return record_cuda_error(cudaErrorInvalidValue);
      rc = allow_smem<gemm_mxf4_persistent<kSfTiled, 128>>(PGeom<kSfTiled, 128>::kSmem, dev);
      if (rc != KQ_OK) return rc;
      const int pgrid =
          static_cast<int>(std::min<int64_t>((int64_t)a.m_tiles * a.n_tiles, di->sms));
      le = launch_pdl(gemm_mxf4_persistent<kSfTiled, 128>, dim3(pgrid), dim3(kPThreads),
                      PGeom<kSfTiled, 128>::kSmem, st, amap, bmap, cmap, a);
    } else {
      rc = allow_smem<gemm_mxf4_persistent<kSfTiled, kBN>>(PGeom<kSfTiled>::kSmem, dev);
      if (rc != KQ_OK) return rc;
      const int pgrid =
          static_cast<int>(std::min<int64_t>((int64_t)a.m_tiles * a.n_tiles, di->sms));
      le = launch_pdl(gemm_mxf4_persistent<kSfTiled, kBN>, dim3(pgrid), dim3(kPThreads),
                      PGeom<kSfTiled>::kSmem, st, amap, bmap, cmap, a);
    }
    if (le != cudaSuccess) return record_cuda_error(le);
  } else if (tiled) {
    // No scale warps: six warps.
    rc = allow_smem<gemm_mxf4_kernel<kSfTiled>>(kSmemBytes, dev);
    if (rc != KQ_OK) return rc;
    cudaError_t le = launch_pdl(gemm_mxf4_kernel<kSfTiled>, grid, dim3(32 * kSfWarp0), kSmemBytes,
                                st, amap, bmap, cmap, a);
    if (le != cudaSuccess) return record_cuda_error(le);
  } else if ((a.sf_stride % 4 == 0) && al(sa, 4) && al(sb, 4)) {
    rc = allow_smem<gemm_mxf4_kernel<kSfRowWords>>(kSmemBytes, dev);
    if (rc != KQ_OK) return rc;
    cudaError_t le = launch_pdl(gemm_mxf4_kernel<kSfRowWords>, grid, dim3(kGemmThreads),
                                kSmemBytes, st, amap, bmap, cmap, a);
    if (le != cudaSuccess) return record_cuda_error(le);
  } else {
    rc = allow_smem<gemm_mxf4_kernel<kSfRowBytes>>(kSmemBytes, dev);
    if (rc != KQ_OK) return rc;
    cudaError_t le = launch_pdl(gemm_mxf4_kernel<kSfRowBytes>, grid, dim3(kGemmThreads),
                                kSmemBytes, st, amap, bmap, cmap, a);
    if (le != cudaSuccess) return record_cuda_error(le);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return record_cuda_error(e);
  return KQ_OK;
}

// One thread per 4-byte word of the tiled layout: word t of tile
// (row tile, column) holds row 32 (t mod 4) + t / 4 of the tile, scales
// 4 column .. 4 column + 3.
__global__ void scales_tile_kernel(const uint8_t* s, int64_t rows, int64_t ns, int64_t col_tiles,
                                   int64_t words, uint32_t* out) {
  for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < words;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tile = w >> 7;
    const int t = static_cast<int>(w & 127);
    const int64_t row = (tile / col_tiles) * 128 + 32 * (t & 3) + (t >> 2);
    const int64_t k0 = (tile % col_tiles) * 4;
    uint32_t v = 0;
    if (row < rows)
      for (int i = 0; i < 4; ++i)
        if (k0 + i < ns) v |= static_cast<uint32_t>(s[row * ns + k0 + i]) << (8 * i);
    out[w] = v;
  }
}

}  // namespace
}  // namespace kq

extern "C" int kq_gemm_mxfp4(const uint8_t* qa, const uint8_t* sa, const uint8_t* qb,
                             const uint8_t* sb, int64_t M, int64_t N, int64_t K, void* c,
                             int c_dtype, void* stream) {
  return launch_gemm(qa, sa, qb, sb, M, N, K, c, c_dtype, stream, false);
}

extern "C" int kq_gemm_mxfp4_tiled(const uint8_t* qa, const uint8_t* sa_tiled, const uint8_t* qb,
                                   const uint8_t* sb_tiled, int64_t M, int64_t N, int64_t K,
                                   void* c, int c_dtype, void* stream) {
  return launch_gemm(qa, sa_tiled, qb, sb_tiled, M, N, K, c, c_dtype, stream, true);
}

extern "C" int kq_gemm_mxfp4_16_tiled(const uint8_t* qa, const uint8_t* sa16_tiled,
                                      const uint8_t* qb, const uint8_t* sb16_tiled, int64_t M,
                                      int64_t N, int64_t K, void* c, int c_dtype, void* stream) {
  return launch_gemm(qa, sa16_tiled, qb, sb16_tiled, M, N, K, c, c_dtype, stream, true, 16);
}

extern "C" size_t kq_scales16_tiled_bytes(int64_t rows, int64_t K) {
  if (rows < 1 || K < 32 || K % 32 != 0) return 0;
  return static_cast<size_t>((rows + 127) / 128) * static_cast<size_t>((K / 16 + 3) / 4) * 512;
}

extern "C" size_t kq_scales_tiled_bytes(int64_t rows, int64_t K) {
  if (rows < 1 || K < 32 || K % 32 != 0) return 0;
  return static_cast<size_t>((rows + 127) / 128) * static_cast<size_t>((K / 32 + 3) / 4) * 512;
}

extern "C" int kq_scales_to_tiled(const uint8_t* scales, int64_t rows, int64_t K, uint8_t* tiled,
                                  void* stream) {
  if (rows < 0 || K < 32 || K % 32 != 0) return KQ_ERR_INVALID;
  if (rows == 0) return KQ_OK;
  if (rows > (int64_t(1) << 40) / K) return KQ_ERR_INVALID;
  if (!scales || !tiled || reinterpret_cast<uintptr_t>(tiled) % 16 != 0) return KQ_ERR_INVALID;
  const DeviceInfo* di = nullptr;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != KQ_OK) return rc;
  const int64_t words = static_cast<int64_t>(kq_scales_tiled_bytes(rows, K) / 4);
  const int grid = static_cast<int>(std::min<int64_t>((words + 255) / 256, di->sms * 8));
  scales_tile_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      scales, rows, K / 32, (K / 32 + 3) / 4, words, reinterpret_cast<uint32_t*>(tiled));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return record_cuda_error(e);
  return KQ_OK;
}
