// LayerNorm + AdaLN modulation fused with the Kronecker transform and the
// MXFP4 quantizer:
//
//   h = (x - mean) / sqrt(var + eps) * (1 + scale[b]) + shift[b],
//   codes, scales = MXFP4(h T)
//
// with mean and (biased) variance over each row's d channels and row m in
// sample b = m / tokens_per_sample.  This is the normalization that keeps
// the transform from being folded offline (KroQuant review, "Core claim" and
// the axiom ledger; handbook page "Quantization: where diffusion differs from
// an LLM": AdaLN scales and shifts the activations per timestep), done in the
// same pass that quantizes, so that x is read from HBM once.
//
// A CTA owns whole rows: R rows of nb = d/32 blocks per group, one thread
// per (row, block), R = floor(384 / nb).  Each group arrives by TMA (3-D boxes
// {32, Wb, R} of the view x[M][nb][32], 64-byte swizzle) into a ring of
// stages; thread 0 refills a stage right after the group's statistics
// barrier, by which every thread has read it, so no producer warp or empty
// barrier is needed and 12 warps keep 168 registers.  Row statistics: each
// thread's 32 values give a sum and a sum of squared deviations; shuffle sums
// over the lanes of the same row in a warp (a segment) give the segment's
// mean and, from the block means' deviations, its M2 (Chan's decomposition
// M2 = sum M2_i + n_i (m_i - m)^2, with no divisions); the segment's first
// lane writes a slot, and after one named barrier every thread combines its
// row's slots in a fixed order, so the result does not depend on timing.
//
// The transform is taken with its diagonal first: every factor is
// G = diag(g00, g11) [[1, g01/g00], [g10/g11, 1]], so K = D S with
// D = (x) diag(g00, g11) and S the product of five unit-diagonal shears.  D
// then merges with the modulation: h D = t alpha + beta with t = (x - mean)
// rstd, alpha = (1 + scale[b]) D and beta = shift[b] D, per sample and
// channel, followed by the shear stages.  A thread keeps column block j for
// the whole kernel, so it recomputes its block's alpha and beta only when its
// rows enter a new sample, into a slice of shared memory that only it reads.
// On wide rows a thread's two rows of a group share one pass over that slice
// when they belong to the same sample.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "kq.h"
#include "kq_device.cuh"
#include "kq_internal.h"
#include "kq_tc.cuh"

namespace kq {
namespace {

constexpr int kAdaWarps = 12;                     // 3 warps per scheduler: 168 registers
constexpr int kAdaCons = 32 * kAdaWarps;          // threads, all consumers
constexpr int kAdaMaxStages = 8;
constexpr int kAdaHalves = 2;                     // rows of a group a thread takes
constexpr int kAdaMaxRows = 256;                  // TMA box limit on a group's rows
constexpr int kAdaMaxHalfRows = kAdaMaxRows / kAdaHalves;
constexpr int kAdaSlots = kAdaWarps + kAdaMaxHalfRows;   // segment slots per half
constexpr int kAdaSlotBufs = 4;
// Rows of at least this many blocks (d >= 3072) take the paired apply:
// one pass over the modulation table for a thread's two rows when they
// belong to one sample.  Narrower rows keep the one-row apply, whose
// register allocation does not spill (the paired form was measured 2-4 %
// slower there and 1-3 % faster on wider rows).
constexpr int kAdaPairMinBlocks = 96;

struct AdaArgs {
  int64_t M;
  int64_t tokens;            // rows per sample
  int32_t nb, R, Wb, boxes;
  int32_t groups, stages, stage_bytes, box_bytes, tx_bytes;
  float eps;
  const float* params;       // [nb][5][3]
  const uint32_t* shift;     // bf16 [B][d], read as bf16 pairs
  const uint32_t* scale;
  uint8_t* q;
  uint8_t* scales;
  int32_t scale_tiles_k;     // 0: row-major scales; else the tiled layout (4-scale columns)
  float* y;
  int* err;
};


// Sum of a block's 32 values, and of their squared deviations from the
// block's own mean (two passes over the registers).
__device__ __forceinline__ void block_sums(const f2 (&u)[16], float& sum, float& m2) {
  f2 s = add2(u[0], u[1]);
#pragma unroll
  for (int m = 2; m < 16; m += 2) s = add2(s, add2(u[m], u[m + 1]));
  float s0, s1;
  unpack2(s, s0, s1);
  sum = s0 + s1;
  const float mean = sum * (1.0f / 32.0f);
  const f2 mean2 = pack2(mean, mean);
  f2 q0 = pack2(0.f, 0.f), q1 = q0;
#pragma unroll
  for (int m = 0; m < 16; m += 2) {
    const f2 d0 = sub2(u[m], mean2), d1 = sub2(u[m + 1], mean2);
    q0 = fma2(d0, d0, q0);
    q1 = fma2(d1, d1, q1);
  }
  float a0, a1, b0, b1;
  unpack2(q0, a0, a1);
  unpack2(q1, b0, b1);
  m2 = (a0 + a1) + (b0 + b1);
}

// Sums of two values over this lane's segment (the lanes of the warp in
// the same row), left in the segment's first lane: shuffle-down steps that
// stay inside the segment (bit k of `inside` says whether lane + 2^k is in
// it), the two values side by side.
__device__ __forceinline__ void segment_sum2(float& v0, float& v1, uint32_t inside) {
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    const float o0 = __shfl_down_sync(0xFFFFFFFFu, v0, 1 << k);
    const float o1 = __shfl_down_sync(0xFFFFFFFFu, v1, 1 << k);
    if (inside & (1u << k)) {
      v0 += o0;
      v1 += o1;
    }
  }
}

// The shear form with its diagonal first: per factor
// G = diag(g00, g11) [[1, r01], [r10, 1]] with r01 = g01 / g00 and
// r10 = g10 / g11, applied to a row vector v as
// (v_lo + r10 v_hi, v_hi + r01 v_lo) after v has been scaled by the diagonal.
// |diag| |S| = |G| entrywise, so each stage keeps the float32 error within a
// few ulp of the magnitudes of the terms of the plain product.
struct ShearIn {
  f2 r10[4], r01[4];     // stages on index bits 4..1, both halves equal
  float r10b, r01b;      // stage on bit 0
};

// Fills the form for the block with parameters p[15]; false if the block
// must take the plain four-term stages instead (an entry outside the float32
// set-up range, a vanishing diagonal entry, or intermediate growth above the
// bound of the output-side shear form).  In float32, as for the output-side
// form: r01 = c / b and r10 = a b / g11 by one corrected division each, the
// latter from the exact split of a b and the pair form of g11.
__device__ __forceinline__ bool load_shear_in(ShearIn& f, const float* p) {
  bool ok = true;
  float growth = 1.0f;
  float r10[kFactors], r01[kFactors];
#pragma unroll
  for (int k = 0; k < kFactors; ++k) {
    const float a = p[3 * k + 0], b = p[3 * k + 1], c = p[3 * k + 2];
    float hi, lo;
    g11_pair(a, b, c, hi, lo);
    ok = ok && in_setup_range(b) && in_setup_range(hi) && fabsf(a) <= 0x1p100f &&
         fabsf(c) <= 0x1p100f;
    const float ab = __fmul_rn(a, b);
    r10[k] = div_pair(ab, hi, lo, __fmaf_rn(a, b, -ab));
    r01[k] = div_pair(c, b, 0.0f);
    growth = __fmul_rn(growth, fmaxf(1.0f + fabsf(r10[k]), 1.0f + fabsf(r01[k])));
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f.r10[k] = pack2(r10[k], r10[k]);
    f.r01[k] = pack2(r01[k], r01[k]);
  }
  f.r10b = r10[4];
  f.r01b = r01[4];
  return ok && growth <= static_cast<float>(kShearGrowthMax);
}

__device__ __forceinline__ void shear_in_apply(f2 (&u)[16], const ShearIn& f) {
  shear_stage<8>(u, f.r10[0], f.r01[0]);
  shear_stage<4>(u, f.r10[1], f.r01[1]);
  shear_stage<2>(u, f.r10[2], f.r01[2]);
  shear_stage<1>(u, f.r10[3], f.r01[3]);
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    float lo, hi;
    unpack2(u[m], lo, hi);
    u[m] = pack2(__fmaf_rn(f.r10b, hi, lo), __fmaf_rn(f.r01b, lo, hi));
  }
}

// Entries 2m and 2m + 1 of the diagonal (x) diag(g00_k, g11_k) of the block
// with parameters p[15], factor k on index bit 4 - k (float32 set-up).
__device__ __forceinline__ void diag_pairs(const float* p, f2 (&dl)[16]) {
  float d0[kFactors], d1[kFactors];
#pragma unroll
  for (int k = 0; k < kFactors; ++k) {
    float lo;
    d0[k] = p[3 * k + 1];
    g11_pair(p[3 * k + 0], p[3 * k + 1], p[3 * k + 2], d1[k], lo);
  }
  delta_tree<kFactors>(d0, d1, dl);
}

// Writes alpha = (1 + scale) delta and beta = shift delta of this thread's
// block for one sample into its slice of the modulation table: chunk c
// (four channels) of alpha at tab[c * kAdaCons + tid], of beta at
// tab[(8 + c) * kAdaCons + tid], so that a warp's 16-byte reads of one chunk
// are consecutive.  delta = 1 for the plain form.  p: the block's 15
// parameters; vs / vc: the sample's shift / scale of the block, 32 bf16 each.
template <int kForm>
__device__ __forceinline__ void write_modulation(const float* p, const uint4 (&vs)[4],
                                                 const uint4 (&vc)[4], int tid, float4* tab) {
  f2 dl[16];
  if (kForm == 0) {
    diag_pairs(p, dl);
  } else {
#pragma unroll
    for (int m = 0; m < 16; ++m) dl[m] = pack2(1.0f, 1.0f);
  }
  const f2 one2 = pack2(1.0f, 1.0f);
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint32_t ws[4] = {vs[t].x, vs[t].y, vs[t].z, vs[t].w};
    const uint32_t wc[4] = {vc[t].x, vc[t].y, vc[t].z, vc[t].w};
    float al[8], be[8];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const f2 dd = dl[4 * t + w];
      const f2 av = mul2(add2(bf16x2_to_f2(wc[w]), one2), dd);
      const f2 bv = mul2(bf16x2_to_f2(ws[w]), dd);
      unpack2(av, al[2 * w], al[2 * w + 1]);
      unpack2(bv, be[2 * w], be[2 * w + 1]);
    }
    tab[(2 * t) * kAdaCons + tid] = make_float4(al[0], al[1], al[2], al[3]);
    tab[(2 * t + 1) * kAdaCons + tid] = make_float4(al[4], al[5], al[6], al[7]);
    tab[(8 + 2 * t) * kAdaCons + tid] = make_float4(be[0], be[1], be[2], be[3]);
    tab[(8 + 2 * t + 1) * kAdaCons + tid] = make_float4(be[4], be[5], be[6], be[7]);
  }
}

// The sample's shift and scale words of block j.
__device__ __forceinline__ void read_modulation(const AdaArgs& a, int64_t b, int j, uint4 (&vs)[4],
                                                uint4 (&vc)[4]) {
  const uint4* ps = reinterpret_cast<const uint4*>(a.shift + (b * a.nb + j) * 16);
  const uint4* pc = reinterpret_cast<const uint4*>(a.scale + (b * a.nb + j) * 16);
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    vs[t] = __ldg(ps + t);
    vc[t] = __ldg(pc + t);
  }
}

// The modulation of sample b, read from global memory at a sample change
// (16 bytes of shift and of scale at a time: the main loop's registers are
// tight).
template <int kForm>
__device__ __forceinline__ void load_modulation(const AdaArgs& a, int64_t b, int j, int tid,
                                                float4* tab) {
  f2 dl[16];
  if (kForm == 0) {
    diag_pairs(a.params + (int64_t)j * 15, dl);
  } else {
#pragma unroll
    for (int m = 0; m < 16; ++m) dl[m] = pack2(1.0f, 1.0f);
  }
  const uint4* ps = reinterpret_cast<const uint4*>(a.shift + (b * a.nb + j) * 16);
  const uint4* pc = reinterpret_cast<const uint4*>(a.scale + (b * a.nb + j) * 16);
  const f2 one2 = pack2(1.0f, 1.0f);
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint4 vs = __ldg(ps + t), vc = __ldg(pc + t);
    const uint32_t ws[4] = {vs.x, vs.y, vs.z, vs.w};
    const uint32_t wc[4] = {vc.x, vc.y, vc.z, vc.w};
    float al[8], be[8];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const f2 dd = dl[4 * t + w];
      const f2 av = mul2(add2(bf16x2_to_f2(wc[w]), one2), dd);
      const f2 bv = mul2(bf16x2_to_f2(ws[w]), dd);
      unpack2(av, al[2 * w], al[2 * w + 1]);
      unpack2(bv, be[2 * w], be[2 * w + 1]);
    }
    tab[(2 * t) * kAdaCons + tid] = make_float4(al[0], al[1], al[2], al[3]);
    tab[(2 * t + 1) * kAdaCons + tid] = make_float4(al[4], al[5], al[6], al[7]);
    tab[(8 + 2 * t) * kAdaCons + tid] = make_float4(be[0], be[1], be[2], be[3]);
    tab[(8 + 2 * t + 1) * kAdaCons + tid] = make_float4(be[4], be[5], be[6], be[7]);
  }
}

// Thread 0 issues the TMA load of a group into a stage.
__device__ __forceinline__ void adaln_issue(const AdaArgs& a, const CUtensorMap* xmap,
                                            uint8_t* stage, uint64_t* bar, int g) {
  mbar_arrive_expect_tx(bar, a.tx_bytes);
  for (int b = 0; b < a.boxes; ++b)
    tma_load_3d(stage + b * a.box_bytes, xmap, 0, b * a.Wb, g * kAdaHalves * a.R, bar);
}

// The loop of one thread over its CTA's groups, software-pipelined by one
// group: the statistics of group i + 1 (slots written, arrival on a
// statistics mbarrier) are produced before group i is normalized, so no
// warp waits for the whole CTA inside a group.  Slots rotate through four
// buffers, enough that a warp writing group i + 3's slots can only have got
// there after every warp finished reading group i - 1's.  A group is 2 R
// rows and a thread takes block j of rows rr and R + rr, so the two rows'
// reductions run side by side and a group's latency is paid once per 64
// elements of each thread.
template <int kOut, int kForm, bool kPair>
__device__ __forceinline__ void adaln_consume(const AdaArgs& a, const CUtensorMap* xmap,
                                              uint8_t* stages, uint64_t* full, uint64_t* statbar,
                                              float4* slots, float4* modtab, int tid,
                                              const ShearIn& si, const PlainFactors& pf,
                                              int64_t b_end_first) {
  const int lane = tid & 31, warp = tid >> 5;
  const int nb = a.nb, R = a.R;
  const bool active = tid < R * nb;
  const int rr = active ? tid / nb : R;         // inactive threads form their own "row"
  const int j = tid - rr * nb;
  // Byte offsets of this thread's four 16-byte chunks of row h R + rr inside
  // a stage: box j / Wb, line (h R + rr) Wb + j mod Wb, chunk q at
  // q ^ ((line >> 1) & 3).
  uint32_t off[kAdaHalves][4];
#pragma unroll
  for (int h = 0; h < kAdaHalves; ++h) {
    const int line = (h * R + rr) * a.Wb + (j % a.Wb);
    const uint32_t boff = (j / a.Wb) * a.box_bytes;
#pragma unroll
    for (int q = 0; q < 4; ++q) off[h][q] = boff + line * 64 + 16 * (q ^ ((line >> 1) & 3));
  }
  // Segments: the lanes of a warp that share a row.  Slot of (row, warp) is
  // warp + row, unique and increasing along the rows.
  const int w_first = active ? (rr * nb) >> 5 : 0;
  const int w_last = active ? ((rr + 1) * nb - 1) >> 5 : -1;
  const int n_slots = w_last - w_first + 1;
  const int prev_rr = (tid > 0 && tid - 1 < R * nb) ? (tid - 1) / nb : -1;
  const bool head = active && (lane == 0 || prev_rr != rr);
  const float inv_d = 1.0f / static_cast<float>(nb * 32);
  const int seg_lo = active ? max(32 * warp, rr * nb) : tid;
  const int seg_hi = active ? min(32 * (warp + 1), (rr + 1) * nb) : tid + 1;
  const int head_lane = seg_lo - 32 * warp;
  const float seg_n = 32.0f * static_cast<float>(seg_hi - seg_lo);
  const float inv_seg_n = 1.0f / seg_n;
  uint32_t inside = 0;
#pragma unroll
  for (int k = 0; k < 5; ++k)
    if (tid + (1 << k) < seg_hi) inside |= 1u << k;
  // Rows this warp's active lanes belong to: with at most two, the row
  // combine runs lane-parallel (blocks per row >= 32, every DiT width).
  const int row_lo = min((32 * warp) / nb, R - 1);
  const int row_hi = min((32 * warp + 31) / nb, R - 1);
  const int n_rows_here = 32 * warp < R * nb ? row_hi - row_lo + 1 : 0;
  const bool lane_parallel = nb >= 32;

  const int S = a.stages;
  const int n_local = (int)blockIdx.x < a.groups
                          ? (a.groups - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  int issued = min(S, n_local);                   // meaningful in thread 0

  // Group k's data from its stage: waits for the TMA, reads, and orders the
  // reads before the stage's refill.
  auto read_group = [&](int k, uint4 (&c)[kAdaHalves][4]) -> bool {
    const bool got = __all_sync(0xFFFFFFFFu, mbar_wait(&full[k % S], (k / S) & 1));
    const uint8_t* st = stages + (k % S) * a.stage_bytes;
#pragma unroll
    for (int h = 0; h < kAdaHalves; ++h)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        c[h][q] = active ? *reinterpret_cast<const uint4*>(st + off[h][q]) : make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    return got;
  };
  // Group k's slots: segment sums of the block sums give the segment mean,
  // then the block M2 plus 32 (block mean - segment mean)^2 summed over the
  // segment is the segment's M2.  Rows past M hold zeros (TMA fill).
  auto post_stats = [&](int k, const uint4 (&c)[kAdaHalves][4]) {
    float bsum[kAdaHalves], bm2[kAdaHalves];
#pragma unroll
    for (int h = 0; h < kAdaHalves; ++h) {
      f2 u[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        u[4 * q + 0] = bf16x2_to_f2(c[h][q].x);
        u[4 * q + 1] = bf16x2_to_f2(c[h][q].y);
        u[4 * q + 2] = bf16x2_to_f2(c[h][q].z);
        u[4 * q + 3] = bf16x2_to_f2(c[h][q].w);
      }
      bsum[h] = 0.f;
      bm2[h] = 0.f;
      if (active) block_sums(u, bsum[h], bm2[h]);
    }
    float s0 = bsum[0], s1 = bsum[1];
    segment_sum2(s0, s1, inside);
    const float m0 = __shfl_sync(0xFFFFFFFFu, s0, head_lane) * inv_seg_n;
    const float m1 = __shfl_sync(0xFFFFFFFFu, s1, head_lane) * inv_seg_n;
    const float d0 = __fmaf_rn(bsum[0], 1.0f / 32.0f, -m0);
    const float d1 = __fmaf_rn(bsum[1], 1.0f / 32.0f, -m1);
    float q0 = __fmaf_rn(32.0f * d0, d0, bm2[0]), q1 = __fmaf_rn(32.0f * d1, d1, bm2[1]);
    segment_sum2(q0, q1, inside);
    if (head) {
      float4* sb = slots + (k & 3) * (kAdaHalves * kAdaSlots) + warp + rr;
      sb[0] = make_float4(m0, q0, seg_n, 0.f);
      sb[kAdaSlots] = make_float4(m1, q1, seg_n, 0.f);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&statbar[k & 1]);
  };

  int64_t b_end = b_end_first;                    // first row past this thread's sample
  uint4 cn[kAdaHalves][4];
  bool ok = n_local > 0;
  int read = 0;                                   // groups whose data arrived
  if (ok) {
    ok = read_group(0, cn);
    read = ok ? 1 : 0;
    post_stats(0, cn);
  }
  for (int i = 0; ok && i < n_local; ++i) {
    uint4 cc[kAdaHalves][4];
#pragma unroll
    for (int h = 0; h < kAdaHalves; ++h)
#pragma unroll
      for (int q = 0; q < 4; ++q) cc[h][q] = cn[h][q];
    if (i + 1 < n_local) {
      ok = read_group(i + 1, cn);
      read += ok ? 1 : 0;
      post_stats(i + 1, cn);
    }
    // Every warp has posted group i's slots and read its stage.
    ok = __all_sync(0xFFFFFFFFu, mbar_wait(&statbar[i & 1], (i >> 1) & 1)) && ok;
    if (!ok) break;
    if (tid == 0 && i + S < n_local) {
      adaln_issue(a, xmap, stages + (i % S) * a.stage_bytes, &full[i % S],
                  (int)blockIdx.x + (i + S) * (int)gridDim.x);
      ++issued;
    }
    // Each row's segments in a fixed order: mean = sum n_k m_k / d, then
    // M2 = sum M2_k + n_k (m_k - mean)^2; the two halves side by side.
    const float4* sbuf = slots + (i & 3) * (kAdaHalves * kAdaSlots);
    float mean[kAdaHalves] = {0.f, 0.f}, m2[kAdaHalves] = {0.f, 0.f};
    if (lane_parallel) {
      // Lane k takes slot k of the warp's first (then last) row; xor sums
      // give every lane the same totals.
      for (int t = 0; t < n_rows_here; ++t) {
        const int r = t == 0 ? row_lo : row_hi;
        const int base = ((r * nb) >> 5) + r, cnt = (((r + 1) * nb - 1) >> 5) - ((r * nb) >> 5) + 1;
        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 v0 = lane < cnt ? sbuf[base + lane] : z4;
        const float4 v1 = lane < cnt ? sbuf[kAdaSlots + base + lane] : z4;
        float ms0 = v0.z * v0.x, ms1 = v1.z * v1.x;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          ms0 += __shfl_xor_sync(0xFFFFFFFFu, ms0, o);
          ms1 += __shfl_xor_sync(0xFFFFFFFFu, ms1, o);
        }
        const float mr0 = ms0 * inv_d, mr1 = ms1 * inv_d;
        const float dk0 = v0.x - mr0, dk1 = v1.x - mr1;
        float q0 = __fmaf_rn(v0.z * dk0, dk0, v0.y), q1 = __fmaf_rn(v1.z * dk1, dk1, v1.y);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          q0 += __shfl_xor_sync(0xFFFFFFFFu, q0, o);
          q1 += __shfl_xor_sync(0xFFFFFFFFu, q1, o);
        }
        if (rr == r) {
          mean[0] = mr0;
          m2[0] = q0;
          mean[1] = mr1;
          m2[1] = q1;
        }
      }
    } else {
#pragma unroll
      for (int h = 0; h < kAdaHalves; ++h) {
        const float4* rs = sbuf + h * kAdaSlots + w_first + rr;
        float msum = 0.f;
        for (int k = 0; k < n_slots; ++k) msum = __fmaf_rn(rs[k].z, rs[k].x, msum);
        mean[h] = msum * inv_d;
        for (int k = 0; k < n_slots; ++k) {
          const float4 v = rs[k];
          const float dk = v.x - mean[h];
          m2[h] += __fmaf_rn(v.z * dk, dk, v.y);
        }
      }
    }
    // Transform and encode one modulated row block.
    auto emit = [&](int64_t row, f2 (&u)[16]) {
      if (kForm == 1) {
        plain_apply(u, pf);
      } else {
        shear_in_apply(u, si);
      }
      const int64_t gi = row * nb + j;
      if (kOut == 0) {
        const Mx4Block blk = mxfp4_block(u);
        __stcs(reinterpret_cast<uint4*>(a.q + gi * 16), blk.codes);
        if (a.scale_tiles_k == 0) {
          a.scales[gi] = static_cast<uint8_t>(blk.scale);
        } else {
          // Tiled layout: 128-row x 4-scale tiles, row r = r0 + 32 r1 and
          // scale i at byte 16 r0 + 4 r1 + i; the row's last block also
          // zeroes the padding of its 4-scale column.
          const int rl = static_cast<int>(row & 127);
          const int64_t o = ((row >> 7) * a.scale_tiles_k + (j >> 2)) * 512 + 16 * (rl & 31) +
                            4 * (rl >> 5) + (j & 3);
          a.scales[o] = static_cast<uint8_t>(blk.scale);
          if (j == nb - 1)
            for (int t = (j & 3) + 1; t < 4; ++t) a.scales[o + t - (j & 3)] = 0;
        }
      } else {
        float4* dst = reinterpret_cast<float4*>(a.y + gi * 32);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          float x0, x1, x2, x3;
          unpack2(u[2 * t], x0, x1);
          unpack2(u[2 * t + 1], x2, x3);
          __stcs(dst + t, make_float4(x0, x1, x2, x3));
        }
      }
    };
    const int64_t row0 =
        ((int64_t)blockIdx.x + (int64_t)i * gridDim.x) * (kAdaHalves * R) + rr;
    if (!active || row0 >= a.M) continue;
    if (row0 >= b_end) {                          // rows only grow: a new sample
      const int64_t b = row0 / a.tokens;
      b_end = (b + 1) * a.tokens;
      load_modulation<kForm>(a, b, j, tid, modtab);
    }
    const int64_t row1 = row0 + R;
    const float rstd0 = rsqrtf(__fmaf_rn(m2[0], inv_d, a.eps));
    const f2 r20 = pack2(rstd0, rstd0), nm0 = pack2(-mean[0] * rstd0, -mean[0] * rstd0);
    if (kPair && row1 < a.M && row1 < b_end) {
      // Both rows in one sample: one pass over the modulation table for
      // both (half the table reads; the second row's modulated values wait
      // in registers while the first is transformed and encoded).
      const float rstd1 = rsqrtf(__fmaf_rn(m2[1], inv_d, a.eps));
      const f2 r21 = pack2(rstd1, rstd1), nm1 = pack2(-mean[1] * rstd1, -mean[1] * rstd1);
      f2 u0[16], u1[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 al0 = modtab[(2 * q) * kAdaCons + tid];
        const float4 al1 = modtab[(2 * q + 1) * kAdaCons + tid];
        const float4 be0 = modtab[(8 + 2 * q) * kAdaCons + tid];
        const float4 be1 = modtab[(8 + 2 * q + 1) * kAdaCons + tid];
        const f2 A0 = pack2(al0.x, al0.y), A1 = pack2(al0.z, al0.w);
        const f2 A2 = pack2(al1.x, al1.y), A3 = pack2(al1.z, al1.w);
        const f2 B0 = pack2(be0.x, be0.y), B1 = pack2(be0.z, be0.w);
        const f2 B2 = pack2(be1.x, be1.y), B3 = pack2(be1.z, be1.w);
        u0[4 * q + 0] = fma2(fma2(bf16x2_to_f2(cc[0][q].x), r20, nm0), A0, B0);
        u0[4 * q + 1] = fma2(fma2(bf16x2_to_f2(cc[0][q].y), r20, nm0), A1, B1);
        u0[4 * q + 2] = fma2(fma2(bf16x2_to_f2(cc[0][q].z), r20, nm0), A2, B2);
        u0[4 * q + 3] = fma2(fma2(bf16x2_to_f2(cc[0][q].w), r20, nm0), A3, B3);
        u1[4 * q + 0] = fma2(fma2(bf16x2_to_f2(cc[1][q].x), r21, nm1), A0, B0);
        u1[4 * q + 1] = fma2(fma2(bf16x2_to_f2(cc[1][q].y), r21, nm1), A1, B1);
        u1[4 * q + 2] = fma2(fma2(bf16x2_to_f2(cc[1][q].z), r21, nm1), A2, B2);
        u1[4 * q + 3] = fma2(fma2(bf16x2_to_f2(cc[1][q].w), r21, nm1), A3, B3);
      }
      emit(row0, u0);
      emit(row1, u1);
      continue;
    }
#pragma unroll
    for (int h = 0; h < kAdaHalves; ++h) {
    const int64_t row = row0 + (int64_t)h * R;
    if (row >= a.M) continue;
    if (row >= b_end) {                           // rows only grow: a new sample
      const int64_t b = row / a.tokens;
      b_end = (b + 1) * a.tokens;
      load_modulation<kForm>(a, b, j, tid, modtab);
    }
    const float rstd = h == 0 ? rstd0 : rsqrtf(__fmaf_rn(m2[h], inv_d, a.eps));
    const f2 r2 = pack2(rstd, rstd), nmr2 = pack2(-mean[h] * rstd, -mean[h] * rstd);
    f2 u[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 al0 = modtab[(2 * q) * kAdaCons + tid];
      const float4 al1 = modtab[(2 * q + 1) * kAdaCons + tid];
      const float4 be0 = modtab[(8 + 2 * q) * kAdaCons + tid];
      const float4 be1 = modtab[(8 + 2 * q + 1) * kAdaCons + tid];
      u[4 * q + 0] = fma2(fma2(bf16x2_to_f2(cc[h][q].x), r2, nmr2), pack2(al0.x, al0.y),
                          pack2(be0.x, be0.y));
      u[4 * q + 1] = fma2(fma2(bf16x2_to_f2(cc[h][q].y), r2, nmr2), pack2(al0.z, al0.w),
                          pack2(be0.z, be0.w));
      u[4 * q + 2] = fma2(fma2(bf16x2_to_f2(cc[h][q].z), r2, nmr2), pack2(al1.x, al1.y),
                          pack2(be1.x, be1.y));
      u[4 * q + 3] = fma2(fma2(bf16x2_to_f2(cc[h][q].w), r2, nmr2), pack2(al1.z, al1.w),
                          pack2(be1.z, be1.w));
    }
    emit(row, u);
    }
  }
  if (!ok) {
    if (lane == 0) atomicOr(a.err, kErrConsumerWait);
    // Let this CTA's loads still in flight land before it leaves.
    if (tid == 0)
      for (int k = read; k < issued; ++k) mbar_wait(&full[k % S], (k / S) & 1);
  }
}

template <int kOut, bool kPair>
__global__ void __launch_bounds__(kAdaCons, 1)
    adaln_kernel(const __grid_constant__ CUtensorMap xmap, const AdaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = base;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + a.stages * a.stage_bytes);
  uint64_t* statbar = full + kAdaMaxStages;
  float4* slots = reinterpret_cast<float4*>(statbar + 2);            // 16-byte aligned
  float4* modtab = slots + kAdaSlotBufs * kAdaHalves * kAdaSlots;  // [16][kAdaCons]
  const int tid = threadIdx.x;
  const int S = a.stages;
  // Programmatic dependent launch: nothing global is read or written before
  // the previous kernel of the stream has completed.
  pdl_wait_then_trigger();
  if (tid == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
    mbar_init(&statbar[0], kAdaWarps);
    mbar_init(&statbar[1], kAdaWarps);
    fence_mbar_init();
    tma_prefetch_map(&xmap);
    // The first group alone goes out beside the parameter reads (one group
    // per SM adds little to their wait), the rest after them.
    if ((int)blockIdx.x < a.groups) adaln_issue(a, &xmap, stages, &full[0], (int)blockIdx.x);
  }

  const bool active = tid < a.R * a.nb;
  const int j = active ? tid % a.nb : 0;
  // Parameters and the first sample's modulation first: issued behind the
  // tiles' DRAM traffic, these few L2 reads return microseconds late, and
  // the first group's apply waits for them.  The CTA waits until they have
  // arrived, then the first groups' loads go out.
  float prm[15];
  uint4 vs[4], vc[4];
  int64_t b_first = -1;
  float arrived = 0.0f;
  if (active) {
#pragma unroll
    for (int t = 0; t < 15; ++t) prm[t] = a.params[(int64_t)j * 15 + t];
    const int64_t row0 = (int64_t)blockIdx.x * (kAdaHalves * a.R) + tid / a.nb;
    if ((int)blockIdx.x < a.groups && row0 < a.M) {
      b_first = row0 / a.tokens;
      read_modulation(a, b_first, j, vs, vc);
#pragma unroll
      for (int t = 0; t < 4; ++t)
        arrived += __uint_as_float((vs[t].x ^ vs[t].w) & 0x007FFFFFu) +
                   __uint_as_float((vc[t].x ^ vc[t].w) & 0x007FFFFFu);
    }
#pragma unroll
    for (int t = 0; t < 15; ++t) arrived += prm[t];
  }
  asm volatile("bar.sync 2, %0;" ::"r"(kAdaCons), "f"(arrived) : "memory");
  // The raw words wait in this thread's slice of the table until the form
  // is known (their registers are needed for the set-up).
  if (b_first >= 0)
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      reinterpret_cast<uint4*>(modtab)[t * kAdaCons + tid] = vs[t];
      reinterpret_cast<uint4*>(modtab)[(4 + t) * kAdaCons + tid] = vc[t];
    }
  if (tid == 0) {
    // The next S - 1 groups of this CTA.
    for (int s = 1; s < S; ++s) {
      const int64_t g = (int64_t)blockIdx.x + (int64_t)s * gridDim.x;
      if (g < a.groups) adaln_issue(a, &xmap, stages + s * a.stage_bytes, &full[s], (int)g);
    }
  }
  ShearIn si;
  PlainFactors pf;
  int plain = 0;
  if (active) plain = load_shear_in(si, prm) ? 0 : 1;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.s32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\tselp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(plain)
      : "r"(plain), "r"(kAdaCons)
      : "memory");
  // The first sample's table, from the words read above; the consumer
  // loop reloads it only when its rows enter another sample.
  const int64_t b_end_first = b_first >= 0 ? (b_first + 1) * a.tokens : 0;
  if (b_first >= 0)
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      vs[t] = reinterpret_cast<const uint4*>(modtab)[t * kAdaCons + tid];
      vc[t] = reinterpret_cast<const uint4*>(modtab)[(4 + t) * kAdaCons + tid];
    }
  if (plain) {
    if (active) load_plain(pf, prm);
    if (b_first >= 0) write_modulation<1>(prm, vs, vc, tid, modtab);
    adaln_consume<kOut, 1, kPair>(a, &xmap, stages, full, statbar, slots, modtab, tid, si, pf,
                           b_end_first);
  } else {
    if (b_first >= 0) write_modulation<0>(prm, vs, vc, tid, modtab);
    adaln_consume<kOut, 0, kPair>(a, &xmap, stages, full, statbar, slots, modtab, tid, si, pf,
                           b_end_first);
  }
}

template <int kOut, bool kPair>
int launch_adaln_kernel(const CUtensorMap& map, const AdaArgs& a, int grid, int smem, int dev,
                        cudaStream_t st) {
  int rc = allow_smem<adaln_kernel<kOut, kPair>>(smem, dev);
  if (rc != KQ_OK) return rc;
  cudaError_t e =
      launch_pdl(adaln_kernel<kOut, kPair>, dim3(grid), dim3(kAdaCons), smem, st, map, a);
  if (e != cudaSuccess) return record_cuda_error(e);
  return KQ_OK;
}

// Launches the fused kernel; the shapes were checked by the caller.
int launch_adaln(const uint16_t* x, int64_t M, int64_t d, const uint16_t* shift,
                 const uint16_t* scale, int64_t tokens, float eps, const float* params,
                 uint8_t* q, uint8_t* scales, float* y, cudaStream_t st, bool tiled = false) {
  const DeviceInfo* di = nullptr;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != KQ_OK) return rc;
  const int nb = static_cast<int>(d / kBlock);
  if (nb > kAdaCons) return KQ_ERR_INVALID;
  AdaArgs a{};
  rc = device_error_word(dev, &a.err);
  if (rc != KQ_OK) return rc;
  a.M = M;
  a.tokens = tokens;
  a.nb = nb;
  a.R = std::min(kAdaCons / nb, kAdaMaxHalfRows);   // rows per half of a group
  // Boxes of at most 256 blocks; the last may run past the row and is
  // zero-filled there.
  a.boxes = (nb + 255) / 256;
  a.Wb = (nb + a.boxes - 1) / a.boxes;
  const int box_raw = kAdaHalves * a.R * a.Wb * kBlock * 2;
  a.box_bytes = (box_raw + 1023) / 1024 * 1024;
  a.stage_bytes = a.boxes * a.box_bytes;
  a.tx_bytes = a.boxes * box_raw;
  const int group_rows = kAdaHalves * a.R;
  const int64_t groups = (M + group_rows - 1) / group_rows;
  if (M > (int64_t(1) << 31) - 1 - group_rows || groups > (int64_t(1) << 30))
    return KQ_ERR_INVALID;
  a.groups = static_cast<int32_t>(groups);
  a.eps = eps;
  a.params = params;
  a.shift = reinterpret_cast<const uint32_t*>(shift);
  a.scale = reinterpret_cast<const uint32_t*>(scale);
  a.q = q;
  a.scales = scales;
  a.scale_tiles_k = tiled ? (nb + 3) / 4 : 0;
  a.y = y;
  // Barriers, four slot buffers and the modulation table (alpha and beta,
  // 256 bytes a thread).
  const int fixed =
      1024 + (kAdaMaxStages + 2) * 8 + kAdaSlotBufs * kAdaHalves * kAdaSlots * 16 +
      16 * kAdaCons * 16;
  a.stages = std::min(kAdaMaxStages, (di->smem_optin - fixed) / a.stage_bytes);
  if (a.stages < 2) return KQ_ERR_INVALID;
  const int smem = a.stages * a.stage_bytes + fixed;
  CUtensorMap map;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kBlock), static_cast<cuuint64_t>(nb),
                              static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[2] = {kBlock * 2, static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[3] = {kBlock, static_cast<cuuint32_t>(a.Wb),
                             static_cast<cuuint32_t>(kAdaHalves * a.R)};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult cr = tensor_map_encoder()(
      &map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(x), dims, strides, box,
      estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return record_cuda_error(cudaErrorInvalidValue);
  const int grid = static_cast<int>(std::min<int64_t>(groups, di->sms));
  if (y) {
    rc = launch_adaln_kernel<1, false>(map, a, grid, smem, dev, st);
  } else if (nb >= kAdaPairMinBlocks) {
    rc = launch_adaln_kernel<0, true>(map, a, grid, smem, dev, st);
  } else {
    rc = launch_adaln_kernel<0, false>(map, a, grid, smem, dev, st);
  }
  if (rc != KQ_OK) return rc;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return record_cuda_error(e);
  return KQ_OK;
}

}  // namespace
}  // namespace kq

using namespace kq;

namespace {

int check_adaln(const uint16_t* x, int64_t M, int64_t d, const uint16_t* shift,
                const uint16_t* scale, int64_t tokens, float eps, const float* params) {
  if (M < 0 || d < kBlock || d % kBlock != 0 || d / kBlock > kAdaCons) return KQ_ERR_INVALID;
  if (M > 0 && d > (int64_t(1) << 40) / M) return KQ_ERR_INVALID;
  if (tokens < 1 || !(eps >= 0.0f) || !(eps < 3.0e38f)) return KQ_ERR_INVALID;
  if (M == 0) return KQ_OK;
  if (!x || !shift || !scale || !params) return KQ_ERR_INVALID;
  auto al = [](const void* p, uintptr_t n) { return reinterpret_cast<uintptr_t>(p) % n == 0; };
  if (!al(x, 16) || !al(shift, 16) || !al(scale, 16) || !al(params, 4)) return KQ_ERR_INVALID;
  return KQ_OK;
}

}  // namespace

extern "C" int kq_quantize_adaln(const uint16_t* x, int64_t M, int64_t d, const uint16_t* shift,
                                 const uint16_t* scale, int64_t tokens_per_sample, float eps,
                                 const float* params, uint8_t* q_packed, uint8_t* scales,
                                 void* stream) {
  int rc = check_adaln(x, M, d, shift, scale, tokens_per_sample, eps, params);
  if (rc != KQ_OK || M == 0) return rc;
  if (!q_packed || !scales || reinterpret_cast<uintptr_t>(q_packed) % 16 != 0)
    return KQ_ERR_INVALID;
  return launch_adaln(x, M, d, shift, scale, tokens_per_sample, eps, params, q_packed, scales,
                      nullptr, static_cast<cudaStream_t>(stream));
}

extern "C" int kq_quantize_adaln_tiled(const uint16_t* x, int64_t M, int64_t d,
                                       const uint16_t* shift, const uint16_t* scale,
                                       int64_t tokens_per_sample, float eps, const float* params,
                                       uint8_t* q_packed, uint8_t* scales_tiled, void* stream) {
  int rc = check_adaln(x, M, d, shift, scale, tokens_per_sample, eps, params);
  if (rc != KQ_OK || M == 0) return rc;
  if (!q_packed || !scales_tiled || reinterpret_cast<uintptr_t>(q_packed) % 16 != 0)
    return KQ_ERR_INVALID;
  return launch_adaln(x, M, d, shift, scale, tokens_per_sample, eps, params, q_packed,
                      scales_tiled, nullptr, static_cast<cudaStream_t>(stream), true);
}

extern "C" int kq_transform_adaln(const uint16_t* x, int64_t M, int64_t d, const uint16_t* shift,
                                  const uint16_t* scale, int64_t tokens_per_sample, float eps,
                                  const float* params, float* y, void* stream) {
  int rc = check_adaln(x, M, d, shift, scale, tokens_per_sample, eps, params);
  if (rc != KQ_OK || M == 0) return rc;
  if (!y || reinterpret_cast<uintptr_t>(y) % 16 != 0) return KQ_ERR_INVALID;
  return launch_adaln(x, M, d, shift, scale, tokens_per_sample, eps, params, nullptr, nullptr, y,
                      static_cast<cudaStream_t>(stream));
}
