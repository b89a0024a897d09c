// Device-side building blocks of the quantizer kernels (sm_100a only):
// PTX wrappers for mbarriers, TMA, packed float32x2 arithmetic and the E2M1
// conversion, the three block transforms and the shared MXFP4 epilogue.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a (B200) only"
#endif

namespace kq {

constexpr int kBlock = 32;           // elements per MX block and per Kronecker block
constexpr int kFactors = 5;          // 32 = 2^5: one 2x2 factor per index bit
constexpr int kTabStride = 44;       // floats per block in a Kronecker coefficient table

// Bits of the device error word (kq_device_status).
constexpr int kErrConsumerWait = 1;
constexpr int kErrProducerWait = 2;
constexpr int kErrSelfTest = 4;

// A bounded mbarrier wait polls at most kWaitPolls times, each poll suspending
// for at most kWaitHintNs: about four seconds in all, far above any real wait.
constexpr int kWaitPolls = 4000;
constexpr uint32_t kWaitHintNs = 1000000;

// --------------------------------------------------------------- addresses
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA) accesses: needed before a stage that was read with
// ordinary loads is handed back to be overwritten by a TMA load.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// Waits for the phase of the given parity to complete; gives up (returns
// false) after kWaitPolls suspended polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_addr(bar);
  for (int poll = 0; poll < kWaitPolls; ++poll) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(addr), "r"(parity), "r"(kWaitHintNs)
        : "memory");
    if (done) return true;
  }
  return false;
}

// Programmatic dependent launch: waits until the previous kernel of the
// stream has completed and its memory is visible (every thread, before its
// first global read or write), then lets the next kernel start its set-up.
__device__ __forceinline__ void pdl_wait_then_trigger() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled bulk tensor load into this CTA's shared memory (no multicast).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
      : "memory");
}

// 3-D tiled bulk tensor load into this CTA's shared memory (no multicast).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
      : "memory");
}

// ----------------------------------------------------- packed float32 x 2
// A pair of floats in one 64-bit register pair; the first float is the low
// half.  Blackwell executes add/mul/fma on both halves with one instruction.
typedef unsigned long long f2;

__device__ __forceinline__ f2 pack2(float lo, float hi) {
  f2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack2(f2 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
  f2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
  f2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2 add2(f2 a, f2 b) {
  f2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2 sub2(f2 a, f2 b) {
  f2 d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Two bf16 values (element 2m in the low half-word) widened exactly to f32.
__device__ __forceinline__ f2 bf16x2_to_f2(uint32_t w) {
  return pack2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// ----------------------------------------------------------- E2M1 convert
// Eight floats (already divided by the block scale) to eight E2M1 codes,
// element 0 in the low nibble of the low byte.  Round to nearest even,
// saturating to +-6.
__device__ __forceinline__ uint32_t e2m1x8(float v0, float v1, float v2, float v3, float v4,
                                           float v5, float v6, float v7) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return r;
}

// 1/v in double to about 2^-46 relative: the float32 reciprocal refined by
// one Newton step in double (the seed's relative error e becomes e^2), in
// place of a full double division; the exact division where v lies outside
// the range in which the float seed is a normal number.  The coefficients
// built from it are rounded to float32, so the result matches the exact
// quotient's except within 2^-46 of a float32 rounding boundary.
__device__ __forceinline__ double recip_d(double v) {
  const double av = fabs(v);
  if (!(av > 0x1p-120 && av < 0x1p120)) return 1.0 / v;
  const double r0 = static_cast<double>(__frcp_rn(static_cast<float>(v)));
  const double e = __fma_rn(-v, r0, 1.0);
  return __fma_rn(r0, e, r0);
}

// ------------------------------------------------------ block transforms
// A 32-element block lives in u[16]; u[m] holds elements 2m (low) and 2m+1.
//
// One butterfly stage applies a 2x2 factor G to every index pair that differs
// only in bit p, as a row vector times G:
//     y_lo = x_lo G00 + x_hi G10,   y_hi = x_lo G01 + x_hi G11.
// For p >= 1 the two members of a pair sit in different registers and two
// neighbouring pairs share a packed register, so one packed instruction does
// two pairs; for p = 0 the pair shares one register and runs scalar.

// Coefficients of stage s (bit 4 - s) in a table entry, as float4s:
//   e[2s]   = (G00, G00, G10, G10)
//   e[2s+1] = (G01, G01, G11, G11)
template <int kHalfDist>
__device__ __forceinline__ void stage_packed(f2 (&u)[16], float4 c0, float4 c1) {
  const f2 g00 = pack2(c0.x, c0.y), g10 = pack2(c0.z, c0.w);
  const f2 g01 = pack2(c1.x, c1.y), g11 = pack2(c1.z, c1.w);
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    if (m & kHalfDist) continue;
    const f2 lo = u[m], hi = u[m + kHalfDist];
    u[m] = fma2(g10, hi, mul2(g00, lo));
    u[m + kHalfDist] = fma2(g11, hi, mul2(g01, lo));
  }
}

__device__ __forceinline__ void stage_bit0(f2 (&u)[16], float4 c0, float4 c1) {
  const float g00 = c0.x, g10 = c0.z, g01 = c1.x, g11 = c1.z;
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    float lo, hi;
    unpack2(u[m], lo, hi);
    const float ylo = __fmaf_rn(g10, hi, __fmul_rn(g00, lo));
    const float yhi = __fmaf_rn(g11, hi, __fmul_rn(g01, lo));
    u[m] = pack2(ylo, yhi);
  }
}

// y = x K with K = G1 (x) ... (x) G5, from a table entry of kTabStride floats.
__device__ __forceinline__ void kron_apply(f2 (&u)[16], const float* entry) {
  const float4* e = reinterpret_cast<const float4*>(entry);
  stage_packed<8>(u, e[0], e[1]);   // G1, index bit 4
  stage_packed<4>(u, e[2], e[3]);   // G2, bit 3
  stage_packed<2>(u, e[4], e[5]);   // G3, bit 2
  stage_packed<1>(u, e[6], e[7]);   // G4, bit 1
  stage_bit0(u, e[8], e[9]);        // G5, bit 0
}

// Fills one table entry from the (a, b, c) parameters of a block; the four
// entries of each G_k are formed in double and rounded once to float.
__device__ __forceinline__ void kron_entry(float* entry, const float* p) {
#pragma unroll
  for (int k = 0; k < kFactors; ++k) {
    const double a = p[3 * k + 0], b = p[3 * k + 1], c = p[3 * k + 2];
    const double g00 = b, g01 = c, g10 = a * b, g11 = __fma_rn(a, c, recip_d(b));
    const float f00 = (float)g00, f01 = (float)g01, f10 = (float)g10, f11 = (float)g11;
    float4* e = reinterpret_cast<float4*>(entry + 8 * k);
    e[0] = make_float4(f00, f00, f10, f10);
    e[1] = make_float4(f01, f01, f11, f11);
  }
}

// --------------------------------------------- register-resident factors
// The factors of one column block, held in registers by a thread that keeps
// the same block for the whole kernel.
//
// Scaled-shear form: with row-vector factors G = [[g00, g01], [g10, g11]],
//     G = S D,   S = [[1, r01], [r10, 1]],   D = diag(g00, g11),
//     r10 = g10 / g00 = a,   r01 = g01 / g11 = c / (a c + 1/b),
// and by the mixed-product rule K = (S1 (x) ... (x) S5)(D1 (x) ... (x) D5):
// five stages of one multiply-add per output, then one multiply by the
// diagonal delta_i = prod_k (bit_k(i) ? g11_k : g00_k).  Since |S||D| = |G|
// entrywise, the rounding error stays bounded by the same |x| |K| as the
// plain four-term stage.  It needs every g11 != 0 and a bounded growth of
// the intermediate values; blocks that miss that use the plain form.
struct ShearDiag {
  f2 r10[4], r01[4];     // stages on index bits 4..1, both halves equal
  float r10b, r01b;      // stage on bit 0
  f2 delta[16];          // (delta_2m, delta_2m+1)
};

struct PlainFactors {
  f2 g00[4], g10[4], g01[4], g11[4];   // bits 4..1
  float h00, h10, h01, h11;            // bit 0
};

// Bound on the growth of the shear form's intermediate values over the five
// stages (prod_k max(1 + |r10|, 1 + |r01|)): with inputs below 2^100 they
// stay inside the float32 range.
constexpr double kShearGrowthMax = 16777216.0;   // 2^24

// The four entries of G_k (row-vector form) from (a, b, c), in double; with
// kInvT those of (G_k^-1)^T = [[g11, -g10], [-g01, g00]] (det G_k = 1), the
// factor of the weight-side fold W T^-T.
template <bool kInvT = false>
__device__ __forceinline__ void factor_entries(const float* p, int k, double& g00, double& g01,
                                               double& g10, double& g11) {
  const double a = p[3 * k + 0], b = p[3 * k + 1], c = p[3 * k + 2];
  const double e00 = b, e01 = c, e10 = a * b, e11 = __fma_rn(a, c, recip_d(b));
  if (kInvT) {
    g00 = e11;
    g01 = -e10;
    g10 = -e01;
    g11 = e00;
  } else {
    g00 = e00;
    g01 = e01;
    g10 = e10;
    g11 = e11;
  }
}

// ------------------------------------------- float32 factor set-up
// The shear form's coefficients are formed in float32 arithmetic, a few
// operations per factor on the full-rate pipes: double-precision set-up
// (conversions to and from double, double products) was measured to take
// about 2 us at the start of every CTA, on the critical path of the small
// DiT shapes.  The entries that are not exact products come out within about
// one float32 ulp of the exact values:
//   g11 = a c + 1/b   as an unevaluated pair hi + lo (error ~2^-44 |1/b|),
//   c / g11           from the pair by one corrected division,
//   delta_i           a product of five float entries, four roundings.
// Any block whose entries leave [2^-100, 2^100] takes the plain form, whose
// coefficients are still formed in double (factor_entries).

// The hardware's approximate reciprocal (within about an ulp; inputs are
// kept inside [2^-100, 2^100] by the callers, so flushing of subnormals
// never applies).
__device__ __forceinline__ float rcp_approx(float v) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

// g11 = a c + 1/b as hi + lo: an approximate reciprocal r of b and its
// residual e = 1 - b r, exact in float32 since r is within about an ulp of
// 1/b, so that 1/b = r (1 + e + e^2 + ...) = r + r e to about 2^-46
// relative; the product a c split exactly by an fma (Dekker's product); the
// two large terms added by a two-sum (Knuth), the small ones after.
__device__ __forceinline__ void g11_pair(float a, float b, float c, float& hi, float& lo) {
  const float r = rcp_approx(b);
  const float e = __fmaf_rn(-b, r, 1.0f);
  const float pc = __fmul_rn(a, c);
  const float pe = __fmaf_rn(a, c, -pc);
  const float s = __fadd_rn(pc, r);
  const float v = __fsub_rn(s, pc);
  const float t = __fadd_rn(__fsub_rn(pc, __fsub_rn(s, v)), __fsub_rn(r, v));
  const float rest = __fadd_rn(t, __fmaf_rn(r, e, pe));
  hi = __fadd_rn(s, rest);
  lo = __fsub_rn(rest, __fsub_rn(hi, s));
}

// (n + nl) / (hi + lo): the quotient q = n r by an approximate reciprocal r
// of hi, then one correction by its residual n + nl - q (hi + lo) (Newton's
// step for a quotient, as in Markstein's division), which leaves it within
// about an ulp.
__device__ __forceinline__ float div_pair(float n, float hi, float lo, float nl = 0.0f) {
  const float rh = rcp_approx(hi);
  const float q = __fmul_rn(n, rh);
  const float rem = __fmaf_rn(-q, lo, __fmaf_rn(-q, hi, n) + nl);
  return __fmaf_rn(rem, rh, q);
}

__device__ __forceinline__ bool in_setup_range(float v) {
  const float av = fabsf(v);
  return av >= 0x1p-100f && av <= 0x1p100f;
}

// Diagonal entries (g00_k, g11_k) and shear ratios (r10_k, r01_k) of the
// factors of one block, in float32; false if the block must take the plain
// form (an entry outside the set-up range, a vanishing diagonal entry, or
// intermediate growth above kShearGrowthMax).  nf factors, p[3 nf].  For
// G_k itself r10 = g10 / g00 = a exactly; for (G_k^-1)^T (kInvT) the
// entries are [[g11, -a b], [-c, b]], so r01 = -a exactly and
// r10 = -c / g11.
template <bool kInvT, int nf>
__device__ __forceinline__ bool shear_factors(const float* p, float (&d0)[nf], float (&d1)[nf],
                                              float (&r10)[nf], float (&r01)[nf]) {
  bool ok = true;
  float growth = 1.0f;
#pragma unroll
  for (int k = 0; k < nf; ++k) {
    const float a = p[3 * k + 0], b = p[3 * k + 1], c = p[3 * k + 2];
    float hi, lo;
    g11_pair(a, b, c, hi, lo);
    ok = ok && in_setup_range(b) && in_setup_range(hi) && fabsf(a) <= 0x1p100f &&
         fabsf(c) <= 0x1p100f;
    const float q = div_pair(c, hi, lo);
    if (kInvT) {
      d0[k] = hi;
      d1[k] = b;
      r10[k] = -q;
      r01[k] = -a;
    } else {
      d0[k] = b;
      d1[k] = hi;
      r10[k] = a;
      r01[k] = q;
    }
    growth = __fmul_rn(growth, fmaxf(1.0f + fabsf(r10[k]), 1.0f + fabsf(r01[k])));
  }
  // NaN fails the comparison as well.
  return ok && growth <= static_cast<float>(kShearGrowthMax);
}

// delta pairs (delta_2m, delta_2m+1) of a block of 2^nf elements from its
// factors' diagonal entries, factor k on index bit nf - 1 - k: a product
// tree from the last factor up, two entries per packed multiply.
template <int nf>
__device__ __forceinline__ void delta_tree(const float (&d0)[nf], const float (&d1)[nf],
                                           f2* out) {
  constexpr int kPairs = 1 << (nf - 1);
  f2 t[kPairs];
  t[0] = pack2(d0[nf - 1], d1[nf - 1]);
#pragma unroll
  for (int k = nf - 2; k >= 0; --k) {
    // Entries with bit (nf - 2 - k) of m clear take d0[k], set d1[k]; bit
    // nf - 2 - k of m is the most significant of the bits built so far.
    const f2 lo = pack2(d0[k], d0[k]), hi = pack2(d1[k], d1[k]);
#pragma unroll
    for (int m = 0; m < (1 << (nf - 2 - k)); ++m) {
      t[m + (1 << (nf - 2 - k))] = mul2(t[m], hi);
      t[m] = mul2(t[m], lo);
    }
  }
#pragma unroll
  for (int m = 0; m < kPairs; ++m) out[m] = t[m];
}

// Fills the shear form for the block with parameters p[15]; returns false if
// the block must use the plain form instead.
template <bool kInvT = false>
__device__ __forceinline__ bool load_shear_diag(ShearDiag& f, const float* p) {
  float d0[kFactors], d1[kFactors], r10[kFactors], r01[kFactors];
  const bool ok = shear_factors<kInvT, kFactors>(p, d0, d1, r10, r01);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f.r10[k] = pack2(r10[k], r10[k]);
    f.r01[k] = pack2(r01[k], r01[k]);
  }
  f.r10b = r10[4];
  f.r01b = r01[4];
  delta_tree<kFactors>(d0, d1, f.delta);
  return ok;
}

template <bool kInvT = false>
__device__ __forceinline__ void load_plain(PlainFactors& f, const float* p) {
#pragma unroll
  for (int k = 0; k < kFactors; ++k) {
    double g00, g01, g10, g11;
    factor_entries<kInvT>(p, k, g00, g01, g10, g11);
    const float f00 = (float)g00, f01 = (float)g01, f10 = (float)g10, f11 = (float)g11;
    if (k < 4) {
      f.g00[k] = pack2(f00, f00);
      f.g01[k] = pack2(f01, f01);
      f.g10[k] = pack2(f10, f10);
      f.g11[k] = pack2(f11, f11);
    } else {
      f.h00 = f00; f.h01 = f01; f.h10 = f10; f.h11 = f11;
    }
  }
}

template <int kHalfDist>
__device__ __forceinline__ void shear_stage(f2 (&u)[16], f2 r10, f2 r01) {
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    if (m & kHalfDist) continue;
    const f2 lo = u[m], hi = u[m + kHalfDist];
    u[m] = fma2(r10, hi, lo);
    u[m + kHalfDist] = fma2(r01, lo, hi);
  }
}

// The shear stages; the diagonal is applied by the caller.
__device__ __forceinline__ void shear_apply(f2 (&u)[16], const ShearDiag& f) {
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

// Per-element diagonal multiply (the shear form's D, or SmoothQuant's 1/s).
__device__ __forceinline__ void diag_mul(f2 (&u)[16], const f2 (&delta)[16]) {
#pragma unroll
  for (int m = 0; m < 16; ++m) u[m] = mul2(u[m], delta[m]);
}

template <int kHalfDist>
__device__ __forceinline__ void plain_stage(f2 (&u)[16], f2 g00, f2 g10, f2 g01, f2 g11) {
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    if (m & kHalfDist) continue;
    const f2 lo = u[m], hi = u[m + kHalfDist];
    u[m] = fma2(g10, hi, mul2(g00, lo));
    u[m + kHalfDist] = fma2(g11, hi, mul2(g01, lo));
  }
}

__device__ __forceinline__ void plain_apply(f2 (&u)[16], const PlainFactors& f) {
  plain_stage<8>(u, f.g00[0], f.g10[0], f.g01[0], f.g11[0]);
  plain_stage<4>(u, f.g00[1], f.g10[1], f.g01[1], f.g11[1]);
  plain_stage<2>(u, f.g00[2], f.g10[2], f.g01[2], f.g11[2]);
  plain_stage<1>(u, f.g00[3], f.g10[3], f.g01[3], f.g11[3]);
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    float lo, hi;
    unpack2(u[m], lo, hi);
    u[m] = pack2(__fmaf_rn(f.h10, hi, __fmul_rn(f.h00, lo)),
                 __fmaf_rn(f.h11, hi, __fmul_rn(f.h01, lo)));
  }
}

// -------------------------------------------- 16-element blocks, in pairs
// The 16-element variant keeps two adjacent 16-blocks in one 32-element unit:
// u[0..7] is block 0, u[8..15] block 1, each with its own four factors
// (index bits 3..0 of the block, G1 on bit 3).
struct ShearDiag16 {
  f2 r10[2][3], r01[2][3];   // per block: stages on index bits 3, 2, 1
  float r10b[2], r01b[2];    // per block: bit 0
  f2 delta[16];              // (delta_2m, delta_2m+1), block 0 then block 1
};

struct PlainFactors16 {
  f2 g00[2][3], g10[2][3], g01[2][3], g11[2][3];
  float h00[2], h10[2], h01[2], h11[2];
};

constexpr int kFactors16 = 4;

// p: the 2 x 4 x 3 parameters of the unit's two blocks; kInvT as for
// load_shear_diag.
template <bool kInvT = false>
__device__ __forceinline__ bool load_shear_diag16(ShearDiag16& f, const float* p) {
  bool ok = true;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float d0[kFactors16], d1[kFactors16], r10[kFactors16], r01[kFactors16];
    ok = shear_factors<kInvT, kFactors16>(p + 12 * h, d0, d1, r10, r01) && ok;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      f.r10[h][k] = pack2(r10[k], r10[k]);
      f.r01[h][k] = pack2(r01[k], r01[k]);
    }
    f.r10b[h] = r10[3];
    f.r01b[h] = r01[3];
    delta_tree<kFactors16>(d0, d1, f.delta + 8 * h);
  }
  return ok;
}

template <bool kInvT = false>
__device__ __forceinline__ void load_plain16(PlainFactors16& f, const float* p) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int k = 0; k < kFactors16; ++k) {
      double g00, g01, g10, g11;
      factor_entries<kInvT>(p + 12 * h, k, g00, g01, g10, g11);
      const float f00 = (float)g00, f01 = (float)g01, f10 = (float)g10, f11 = (float)g11;
      if (k < 3) {
        f.g00[h][k] = pack2(f00, f00);
        f.g01[h][k] = pack2(f01, f01);
        f.g10[h][k] = pack2(f10, f10);
        f.g11[h][k] = pack2(f11, f11);
      } else {
        f.h00[h] = f00; f.h01[h] = f01; f.h10[h] = f10; f.h11[h] = f11;
      }
    }
  }
}

// One stage on registers u[kOff .. kOff + 8) (one 16-block).
template <int kHalfDist, int kOff>
__device__ __forceinline__ void shear_stage8(f2 (&u)[16], f2 r10, f2 r01) {
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    if (m & kHalfDist) continue;
    const f2 lo = u[kOff + m], hi = u[kOff + m + kHalfDist];
    u[kOff + m] = fma2(r10, hi, lo);
    u[kOff + m + kHalfDist] = fma2(r01, lo, hi);
  }
}

template <int kHalfDist, int kOff>
__device__ __forceinline__ void plain_stage8(f2 (&u)[16], f2 g00, f2 g10, f2 g01, f2 g11) {
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    if (m & kHalfDist) continue;
    const f2 lo = u[kOff + m], hi = u[kOff + m + kHalfDist];
    u[kOff + m] = fma2(g10, hi, mul2(g00, lo));
    u[kOff + m + kHalfDist] = fma2(g11, hi, mul2(g01, lo));
  }
}

__device__ __forceinline__ void shear_apply16(f2 (&u)[16], const ShearDiag16& f) {
  shear_stage8<4, 0>(u, f.r10[0][0], f.r01[0][0]);
  shear_stage8<2, 0>(u, f.r10[0][1], f.r01[0][1]);
  shear_stage8<1, 0>(u, f.r10[0][2], f.r01[0][2]);
  shear_stage8<4, 8>(u, f.r10[1][0], f.r01[1][0]);
  shear_stage8<2, 8>(u, f.r10[1][1], f.r01[1][1]);
  shear_stage8<1, 8>(u, f.r10[1][2], f.r01[1][2]);
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const int h = m >> 3;
    float lo, hi;
    unpack2(u[m], lo, hi);
    u[m] = pack2(__fmaf_rn(f.r10b[h], hi, lo), __fmaf_rn(f.r01b[h], lo, hi));
  }
}

__device__ __forceinline__ void plain_apply16(f2 (&u)[16], const PlainFactors16& f) {
  plain_stage8<4, 0>(u, f.g00[0][0], f.g10[0][0], f.g01[0][0], f.g11[0][0]);
  plain_stage8<2, 0>(u, f.g00[0][1], f.g10[0][1], f.g01[0][1], f.g11[0][1]);
  plain_stage8<1, 0>(u, f.g00[0][2], f.g10[0][2], f.g01[0][2], f.g11[0][2]);
  plain_stage8<4, 8>(u, f.g00[1][0], f.g10[1][0], f.g01[1][0], f.g11[1][0]);
  plain_stage8<2, 8>(u, f.g00[1][1], f.g10[1][1], f.g01[1][1], f.g11[1][1]);
  plain_stage8<1, 8>(u, f.g00[1][2], f.g10[1][2], f.g01[1][2], f.g11[1][2]);
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const int h = m >> 3;
    float lo, hi;
    unpack2(u[m], lo, hi);
    u[m] = pack2(__fmaf_rn(f.h10[h], hi, __fmul_rn(f.h00[h], lo)),
                 __fmaf_rn(f.h11[h], hi, __fmul_rn(f.h01[h], lo)));
  }
}

// Fixed block Hadamard H_32 (Sylvester order: H2 = [[1,1],[1,-1]] on every
// bit), then the orthonormal factor 1/sqrt(32) as one float32 multiply.
__device__ __forceinline__ void hadamard_apply(f2 (&u)[16]) {
#pragma unroll
  for (int hd = 8; hd >= 1; hd >>= 1) {
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      if (m & hd) continue;
      const f2 lo = u[m], hi = u[m + hd];
      u[m] = add2(lo, hi);
      u[m + hd] = sub2(lo, hi);
    }
  }
  const float s = 0.17677669529663688f;   // 1/sqrt(32) rounded to float32
  const f2 s2 = pack2(s, s);
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    float lo, hi;
    unpack2(u[m], lo, hi);
    u[m] = mul2(pack2(lo + hi, lo - hi), s2);
  }
}

// Per-channel scaling y[c] = x[c] * inv_s[c]; ``inv`` points at the block's
// 32 reciprocal scales in shared memory, stored as 8 chunks of 4 with chunk i
// at position i ^ (j & 7), so that eight threads with consecutive blocks j
// read eight different bank groups.
__device__ __forceinline__ void smooth_apply(f2 (&u)[16], const float* inv, int j) {
  const float4* v = reinterpret_cast<const float4*>(inv);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 s = v[i ^ (j & 7)];
    u[2 * i] = mul2(u[2 * i], pack2(s.x, s.y));
    u[2 * i + 1] = mul2(u[2 * i + 1], pack2(s.z, s.w));
  }
}

// ------------------------------------------------------------ MXFP4 epilogue
// Shared E8M0 scale of the block and the 16 bytes of packed codes.
struct Mx4Block {
  uint4 codes;
  uint32_t scale;
};

// Three-input maximum (sm_100).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Largest magnitude of the 32 values: a tree of three-input maxima (fewer
// instructions on B200 than two-input maxima with folded |.|, measured).
__device__ __forceinline__ float block_amax(const f2 (&u)[16]) {
  float a[32];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    unpack2(u[i], a[2 * i], a[2 * i + 1]);
    a[2 * i] = fabsf(a[2 * i]);
    a[2 * i + 1] = fabsf(a[2 * i + 1]);
  }
  float b[11];
#pragma unroll
  for (int i = 0; i < 10; ++i) b[i] = max3(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
  b[10] = fmaxf(a[30], a[31]);
  const float c0 = max3(b[0], b[1], b[2]), c1 = max3(b[3], b[4], b[5]);
  const float c2 = max3(b[6], b[7], b[8]), c3 = fmaxf(b[9], b[10]);
  return fmaxf(max3(c0, c1, c2), c3);
}

// Scale byte of a block from its largest magnitude, and 2^-e as a float.
__device__ __forceinline__ uint32_t e8m0_from_amax(float amax, f2& inv_x2) {
  const int field = static_cast<int>(__float_as_uint(amax) >> 23);
  const int sbyte = field > 2 ? field - 2 : 0;
  const float inv_x = __uint_as_float(static_cast<uint32_t>(254 - sbyte) << 23);
  inv_x2 = pack2(inv_x, inv_x);
  return static_cast<uint32_t>(sbyte);
}

// Two 16-element blocks (u[0..7], u[8..15]): 16 bytes of codes (block 0 in
// the first 8) and the two scale bytes (block 0 in bits 0..7).
__device__ __forceinline__ Mx4Block mxfp4_block16x2(const f2 (&u)[16]) {
  uint32_t w[4];
  uint32_t scales = 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float a[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      unpack2(u[8 * h + i], a[2 * i], a[2 * i + 1]);
      a[2 * i] = fabsf(a[2 * i]);
      a[2 * i + 1] = fabsf(a[2 * i + 1]);
    }
    const float b0 = max3(a[0], a[1], a[2]), b1 = max3(a[3], a[4], a[5]);
    const float b2 = max3(a[6], a[7], a[8]), b3 = max3(a[9], a[10], a[11]);
    const float b4 = max3(a[12], a[13], a[14]);
    const float amax = fmaxf(max3(b0, b1, b2), max3(b3, b4, a[15]));
    f2 s2;
    scales |= e8m0_from_amax(amax, s2) << (8 * h);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) unpack2(mul2(u[8 * h + 4 * k + i], s2), v[2 * i], v[2 * i + 1]);
      w[2 * h + k] = e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
    }
  }
  Mx4Block r;
  r.codes = make_uint4(w[0], w[1], w[2], w[3]);
  r.scale = scales;
  return r;
}

__device__ __forceinline__ Mx4Block mxfp4_block(const f2 (&u)[16]) {
  float m[1];
  m[0] = block_amax(u);
  // floor(log2(amax)) is the biased exponent field minus 127, so the scale
  // byte e + 127 = field - 2, clamped at 0 (zero and subnormal maxima too).
  const int field = static_cast<int>(__float_as_uint(m[0]) >> 23);
  const int sbyte = field > 2 ? field - 2 : 0;
  // 2^-e as a normal float32: biased exponent 127 - e = 254 - sbyte.
  const float inv_x = __uint_as_float(static_cast<uint32_t>(254 - sbyte) << 23);
  const f2 s2 = pack2(inv_x, inv_x);
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) unpack2(mul2(u[4 * k + i], s2), v[2 * i], v[2 * i + 1]);
    w[k] = e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
  }
  Mx4Block r;
  r.codes = make_uint4(w[0], w[1], w[2], w[3]);
  r.scale = static_cast<uint32_t>(sbyte);
  return r;
}

}  // namespace kq
