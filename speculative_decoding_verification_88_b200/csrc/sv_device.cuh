// sv_device.cuh -- device primitives of the verify kernels (sm_100a):
// mbarrier + 1-D bulk copy (TMA) wrappers with bounded waits, Philox4x32-10,
// the uniform and Gumbel mappings, bf16 unpacking and 64-bit argmax keys.
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

#include "sv_internal.h"

namespace sv {

constexpr unsigned int kFlagInvalidToken = 1u;
constexpr unsigned int kFlagResidualFallback = 2u;
constexpr unsigned int kFlagTimeout = 4u;
constexpr unsigned int kFlagInvalidRow = 8u;
constexpr unsigned int kFlagCapacity = 16u;
constexpr unsigned int kFlagInvalidTree = 32u;
constexpr unsigned int kFlagBounds = 64u;  // bounds-checked builds only

// A device wait gives up after this long (ns) and raises kFlagTimeout.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

constexpr float kLn2 = 0.693147180559945309f;
constexpr float kLog2e = 1.442695040888963407f;

// ------------------------------------------------------------ bounds checks
// A build with SV_DEBUG_BOUNDS defined checks every global index the kernels
// form (logit offsets of each chunk and gather, workspace slots, tokens,
// outputs) against the extent of its buffer.  A violation raises
// kFlagBounds in the status word, records the first offending source line in
// the control block's first spare word, and the access is skipped, so that an
// index error shows up as a status bit rather than a fault.  Release builds
// compile every check to `true`.
#ifdef SV_DEBUG_BOUNDS
static __device__ __noinline__ void bounds_fail(Ctrl* ctrl, int line) {
  atomicOr(&ctrl->flags, kFlagBounds);
  atomicCAS(&ctrl->pad[0], 0u, static_cast<unsigned int>(line));
}
#define SV_IN(ctrl, idx, n)                                                      \
  ((static_cast<long long>(idx) >= 0 && static_cast<long long>(idx) < static_cast<long long>(n)) \
       ? true                                                                    \
       : (::sv::bounds_fail((ctrl), __LINE__), false))
// [lo, lo + len) inside [0, n)
#define SV_IN_RANGE(ctrl, lo, len, n)                                            \
  ((static_cast<long long>(lo) >= 0 &&                                           \
    static_cast<long long>(lo) + static_cast<long long>(len) <= static_cast<long long>(n)) \
       ? true                                                                    \
       : (::sv::bounds_fail((ctrl), __LINE__), false))
#else
#define SV_IN(ctrl, idx, n) true
#define SV_IN_RANGE(ctrl, lo, len, n) true
#endif

// ------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2f(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (Blackwell f32x2 FMA / add): two lanes of arithmetic per
// instruction.
__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
  unsigned long long d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ void unpack2(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long sub2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long splat2(float x) { return pack2(x, x); }

// Largest of three (sm_100 three-input max; a NaN operand is ignored, like fmaxf).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}


__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_u32(unsigned int* p, unsigned int v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// 64-bit atomic OR with acquire-release semantics at GPU scope.
__device__ __forceinline__ unsigned long long atom_or_acq_rel_u64(unsigned long long* p,
                                                                 unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.acq_rel.gpu.global.or.b64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v)
               : "memory");
  return old;
}

__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned int ld_relaxed_u32(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// With a preceding relaxed load that saw a release store, makes the writer's
// earlier stores visible to this thread's later accesses.
__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Programmatic dependent launch: a grid lets the next grid on its stream be
// scheduled (once every block of it has executed this or exited), and the
// dependent grid waits until its prerequisite grid has completed and that
// grid's memory operations are visible.  Without a programmatic launch the
// wait returns at once.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Every kernel of this library starts with dep_enter(): it waits until the
// kernel before it on the stream has completed and that kernel's memory is
// visible, then lets the next kernel be scheduled.  A launch with
// programmatic stream serialization (launch_k) can thus overlap its
// scheduling with the previous kernel's tail without reading anything early;
// launched otherwise, or after work that is not a kernel, the wait returns at
// once.  Dependents are let go only after the wait, and only once every block
// of this grid has started, so a waiting grid never holds an SM that the grid
// it waits for still needs.
__device__ __forceinline__ void dep_enter() {
  griddep_wait();
  griddep_launch_dependents();
}

// SV_PDL 1: only the finalize grid of the one-grid argmax path is launched
// as a programmatic dependent (of its streaming grid); 2: every kernel; 0:
// none.  A graph of the four bench calls (greedy B = 64, stochastic B = 64
// and B = 256, multi-candidate B = 16) measured 243.4 / 240.5 / 247.7 us per
// step with 0 / 1 / 2.
#ifndef SV_PDL
#define SV_PDL 1
#endif
template <typename... KArgs, typename... Args>
cudaError_t launch_k(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t st, Args... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Orders this thread's generic-proxy accesses to global memory before its
// later async-proxy (bulk copy) accesses, and the reverse.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ bool aborted(const Ctrl* ctrl) {
  return (*reinterpret_cast<const volatile unsigned int*>(&ctrl->flags) & kFlagTimeout) != 0;
}

// Wait for phase `parity` of an mbarrier, at most kWaitLimitNs, and give up
// early once another wait in the grid has timed out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Ctrl* ctrl) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (unsigned int spin = 1;; ++spin) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((spin & 255u) == 0u) {
      if (aborted(ctrl)) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        atomicOr(&ctrl->flags, kFlagTimeout);
        return false;
      }
    }
  }
}

// 1-D bulk copy global -> shared, completing `bytes` of transaction on `bar`.
// dst, src 16-byte aligned; bytes a positive multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// ------------------------------------------------------------ Philox4x32-10
// Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3"
// (SC'11): ten rounds of two 32x32->64 multiplies, the high halves xored with
// the other counter words and the round key; Weyl key schedule.

__device__ __forceinline__ uint4 philox10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    // one 32x32->64 multiply per product gives both halves
    const unsigned long long p0 = static_cast<unsigned long long>(c.x) * 0xD2511F53u;
    const unsigned long long p1 = static_cast<unsigned long long>(c.z) * 0xCD9E8D57u;
    c = make_uint4(static_cast<uint32_t>(p1 >> 32) ^ c.y ^ k0, static_cast<uint32_t>(p1),
                   static_cast<uint32_t>(p0 >> 32) ^ c.w ^ k1, static_cast<uint32_t>(p0));
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

// The same generator with its ten round keys (k + r W, r = 0..9, the Weyl
// schedule summed) computed once, for loops that draw many counters under
// one key.
struct PhiloxKeys {
  uint32_t k0[10], k1[10];
};
__device__ __forceinline__ PhiloxKeys philox_keys(uint32_t k0, uint32_t k1) {
  PhiloxKeys k;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    k.k0[r] = k0 + static_cast<uint32_t>(r) * 0x9E3779B9u;
    k.k1[r] = k1 + static_cast<uint32_t>(r) * 0xBB67AE85u;
  }
  return k;
}
__device__ __forceinline__ uint4 philox10(uint4 c, const PhiloxKeys& k) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const unsigned long long p0 = static_cast<unsigned long long>(c.x) * 0xD2511F53u;
    const unsigned long long p1 = static_cast<unsigned long long>(c.z) * 0xCD9E8D57u;
    c = make_uint4(static_cast<uint32_t>(p1 >> 32) ^ c.y ^ k.k0[r], static_cast<uint32_t>(p1),
                   static_cast<uint32_t>(p0 >> 32) ^ c.w ^ k.k1[r], static_cast<uint32_t>(p0));
  }
  return c;
}

enum : uint32_t { kTagAccept = 0u, kTagCorrection = 1u, kTagBonus = 2u };

// Acceptance uniform in [0, 1): 24 bits, exact in fp32.
__device__ __forceinline__ float accept_uniform(uint32_t w) {
  return static_cast<float>(w >> 8) * 0x1p-24f;
}

// Exponential variates for the Gumbel-max draws, kept in NEGATIVE LOG2 UNITS:
//   e = lg2 u' = -E / ln 2,   E = -ln u',   u' = ((w >> 9) + 1/2) 2^-23 in (0, 1).
// Every comparison the draws enter (r / E of the exponential race, l/T - ln E
// of a Gumbel score) is invariant under this fixed rescaling, so no ln 2
// factor is ever applied.
//
// u' and v = 1 - u' are formed exactly from bits: the float with exponent 0
// and mantissa j is 1 + j 2^-23, and subtracting 1 - 2^-24 from a float in
// [1, 2) is exact (Sterbenz); the complemented mantissa 2^23 - 1 - j gives v.
//
// e must be accurate relative to its own size, also when it is tiny (u' near
// 1), because small E are the ones that win.  So:
//   v <  1/8 (w >= 0xE0000000):  lg2(1 - v) = -v g(v), g(v) = -ln(1 - v) / (v ln 2),
//              with g the degree-4 polynomial that interpolates it at the five
//              Chebyshev nodes of [0, 1/8] (relative error 1.4e-8; 1.37e-7,
//              about 2 ulp, after the fp32 Horner steps);
//   v >= 1/8:  the hardware lg2 of u', whose absolute error (about 2^-22.6)
//              is below 1e-6 relative here, since |lg2 u'| >= 0.19.
constexpr float kOneMinusHalfUlp = 1.0f - 0x1p-24f;
constexpr float kG0 = -1.44269506f, kG1 = -0.72133995f, kG2 = -0.48137748f,
                kG3 = -0.35020793f, kG4 = -0.37898599f;  // -g(v) coefficients
constexpr uint32_t kSeriesWords = 0xE0000000u;  // w >= this  <=>  v < 1/8

__device__ __forceinline__ float bits_1j(uint32_t w) { return __uint_as_float(0x3f800000u + (w >> 9)); }
__device__ __forceinline__ float bits_1jc(uint32_t w) { return __uint_as_float(0x3fffffffu - (w >> 9)); }

__device__ __forceinline__ float neg_exp1_log2(uint32_t w) {
  const float u = bits_1j(w) - kOneMinusHalfUlp;
  const float v = bits_1jc(w) - kOneMinusHalfUlp;
  float t = fmaf(v, kG4, kG3);
  t = fmaf(v, t, kG2);
  t = fmaf(v, t, kG1);
  t = fmaf(v, t, kG0);
  return w >= kSeriesWords ? v * t : lg2f(u);
}

// The same for two words at once (f32x2 arithmetic; identical values).
__device__ __forceinline__ void neg_exp1_log2_x2(uint32_t w0, uint32_t w1, float& e0, float& e1) {
  const unsigned long long c = splat2(-kOneMinusHalfUlp);
  float u0, u1;
  unpack2(add2(pack2(bits_1j(w0), bits_1j(w1)), c), u0, u1);
  const unsigned long long v = add2(pack2(bits_1jc(w0), bits_1jc(w1)), c);
  unsigned long long t = fma2(v, splat2(kG4), splat2(kG3));
  t = fma2(v, t, splat2(kG2));
  t = fma2(v, t, splat2(kG1));
  t = fma2(v, t, splat2(kG0));
  float s0, s1;
  unpack2(mul2(v, t), s0, s1);
  e0 = w0 >= kSeriesWords ? s0 : lg2f(u0);
  e1 = w1 >= kSeriesWords ? s1 : lg2f(u1);
}

// 2^y for y <= 0, two at a time on the FMA pipe, to take part of the
// exponentials off the special-function unit.  y is clamped at -126 (2^-126
// is negligible against a sum that holds a term equal to 1), split as
// y = j + f with j = rint(y) (adding and removing 1.5 * 2^23 rounds to an
// integer) and f in [-1/2, 1/2]; 2^f is the degree-5 polynomial that
// interpolates it at the six Chebyshev nodes of [-1/2, 1/2] (relative error
// 1.0e-7, 2.2e-7 with fp32 rounding); 2^j enters by adding j to the exponent
// field (the low bits of y + 1.5 * 2^23 hold j, shifted up by 23).
__device__ __forceinline__ unsigned long long ex2_poly_x2(float y0, float y1) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const unsigned long long y = pack2(fmaxf(y0, -126.0f), fmaxf(y1, -126.0f));
  const unsigned long long t = add2(y, splat2(kRound));
  const unsigned long long f = sub2(y, sub2(t, splat2(kRound)));
  unsigned long long q = fma2(f, splat2(1.339086337e-03f), splat2(9.676031918e-03f));
  q = fma2(f, q, splat2(5.550357114e-02f));
  q = fma2(f, q, splat2(2.402210749e-01f));
  q = fma2(f, q, splat2(6.931471880e-01f));
  q = fma2(f, q, splat2(1.000000075e+00f));
  float q0, q1, t0, t1;
  unpack2(q, q0, q1);
  unpack2(t, t0, t1);
  return pack2(__uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23)),
               __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23)));
}

// Gumbel noise in log2 units: g / ln 2 = -lg2 E = -lg2(-e ln 2); the constant
// -lg2(ln 2) is dropped, as it shifts every score of a row alike.
__device__ __forceinline__ float gumbel_log2(float e) { return -lg2f(-e); }

__device__ __forceinline__ uint32_t word_of(const uint4& v, int j) {
  return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
}

// ------------------------------------------------------------ elements

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static constexpr int kBytes = 4;
  static constexpr int kPerVec = 4;  // elements per 16-byte vector
};
template <>
struct Elem<uint16_t> {
  static constexpr int kBytes = 2;
  static constexpr int kPerVec = 8;
};

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

template <typename T>
__device__ __forceinline__ float load_elem(const void* base, long long off) {
  return to_f32(__ldg(reinterpret_cast<const T*>(base) + off));
}

// Unpack one 16-byte vector into floats (8 for bf16, 4 for f32).
__device__ __forceinline__ void unpack(const uint4& v, float (&f)[8]) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
  f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
  f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}
__device__ __forceinline__ void unpack(const uint4& v, float (&f)[4]) {
  f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
}

__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Max of the elements of one 16-byte vector.
template <typename T>
__device__ __forceinline__ float vec_max(const uint4& v);
template <>
__device__ __forceinline__ float vec_max<uint16_t>(const uint4& v) {
  const uint32_t m = bmax2(bmax2(v.x, v.y), bmax2(v.z, v.w));
  return fmaxf(bf16_lo(m), bf16_hi(m));
}
template <>
__device__ __forceinline__ float vec_max<float>(const uint4& v) {
  return fmaxf(fmaxf(__uint_as_float(v.x), __uint_as_float(v.y)),
               fmaxf(__uint_as_float(v.z), __uint_as_float(v.w)));
}

// ------------------------------------------------------------ argmax keys
// 64-bit key ordered like (value, -index): larger value wins, and among
// equal values the lower index wins.  -0 is folded into +0.  Every real
// value (including -inf) gives a nonzero key; 0 means "no candidate".

__device__ __forceinline__ uint32_t orderable(float v) {
  uint32_t b = __float_as_uint(v == 0.0f ? 0.0f : v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ unsigned long long make_key(float v, int idx) {
  return (static_cast<unsigned long long>(orderable(v)) << 32) |
         static_cast<unsigned long long>(~static_cast<uint32_t>(idx));
}

__device__ __forceinline__ int key_index(unsigned long long key) {
  return static_cast<int>(~static_cast<uint32_t>(key & 0xffffffffull));
}

// (value, index) pair preferred by an argmax with lowest-index tie-break.
__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// Warp-wide maximum of a float (sm_100 redux; a NaN operand is ignored).
__device__ __forceinline__ float warp_max(float v) {
  float m;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(m) : "f"(v));
  return m;
}

// Warp-wide argmax in the order of better(): the largest value, and among
// lanes holding it (-0 and +0 alike) the lowest index.  Every lane gets it.
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
  const float m = warp_max(v);
  const unsigned int cand = v == m ? static_cast<unsigned int>(i) : 0xffffffffu;
  unsigned int r;
  asm volatile("redux.sync.min.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(cand));
  v = m;
  i = static_cast<int>(r);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Merge softmax statistics (m in log2 units, s = sum 2^(z - m)).
__device__ __forceinline__ void merge_stats(float& M, float& S, float m, float s) {
  if (m == -INFINITY) return;
  if (M == -INFINITY) {
    M = m;
    S = s;
  } else if (m > M) {
    S = S * ex2f(M - m) + s;
    M = m;
  } else {
    S += s * ex2f(m - M);
  }
}

}  // namespace sv
