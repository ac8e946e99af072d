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

// A device wait gives up after this long (ns) and raises kFlagTimeout.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

constexpr float kLn2 = 0.693147180559945309f;
constexpr float kLog2e = 1.442695040888963407f;

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
    const uint32_t lo0 = 0xD2511F53u * c.x;
    const uint32_t hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

enum : uint32_t { kTagAccept = 0u, kTagCorrection = 1u, kTagBonus = 2u };

// Acceptance uniform in [0, 1): 24 bits, exact in fp32.
__device__ __forceinline__ float accept_uniform(uint32_t w) {
  return static_cast<float>(w >> 8) * 0x1p-24f;
}

// Exponential variate E = -ln u', u' = ((w >> 9) + 0.5) 2^-23 in (0, 1).  Both
// u' and v = 1 - u' are exact in fp32.  E must be accurate relative to its own
// size, also when it is tiny (u' near 1), because small E are the ones that win
// a Gumbel-max.  So:
//   v <  1/8:  -ln(1 - v) = v + v^2/2 + ... + v^7/7, Taylor series written in
//              Horner form (truncation below 7e-8 relative);
//   v >= 1/8:  -ln(u') = -lg2(u') ln 2 with the hardware lg2, whose absolute
//              error (about 2^-22.6) is below 1e-6 relative here, since
//              |lg2 u'| >= 0.19.
__device__ __forceinline__ float exp1_variate(uint32_t w) {
  const uint32_t j = w >> 9;
  const float u = (static_cast<float>(j) + 0.5f) * 0x1p-23f;
  const float v = (static_cast<float>(0x7fffffu - j) + 0.5f) * 0x1p-23f;
  float t = fmaf(v, 1.0f / 7.0f, 1.0f / 6.0f);
  t = fmaf(v, t, 0.2f);
  t = fmaf(v, t, 0.25f);
  t = fmaf(v, t, 1.0f / 3.0f);
  t = fmaf(v, t, 0.5f);
  t = fmaf(v, t, 1.0f);
  const float series = v * t;
  const float viaLog = -lg2f(u) * kLn2;
  return v < 0.125f ? series : viaLog;
}

// Gumbel noise g = -ln(-ln u') = -ln E.
__device__ __forceinline__ float gumbel(uint32_t w) { return -lg2f(exp1_variate(w)) * kLn2; }

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

__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    if (better(ov, oi, v, i)) {
      v = ov;
      i = oi;
    }
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
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
