// sv_math_probe.cu -- test-only probes of the verify kernels' hand-written
// fast-math helpers (built by the tests, never part of libspecverify.so).
//
// The helpers come from the library's own device header, so the probes run
// exactly the code the kernels run:
//   ex2_poly_x2     2^y for y <= 0 on the FMA pipe (degree-5 Chebyshev
//                   interpolant of 2^f on [-1/2, 1/2], 2^j added to the
//                   exponent field), two values at a time
//   ex2f            the special-function unit's 2^x
//   neg_exp1_log2   lg2 u' of the Gumbel uniform u' = ((w >> 9) + 1/2) 2^-23,
//                   by the degree-4 series for v = 1 - u' < 1/8 and the
//                   hardware lg2 elsewhere; and its two-at-a-time form
#include <cstdint>

#include "sv_device.cuh"

namespace {

__global__ void ex2_probe_kernel(const float* __restrict__ y, float* __restrict__ poly,
                                 float* __restrict__ mufu, long long n) {
  const long long j = 2 * (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x);
  if (j >= n) return;
  const float y0 = y[j], y1 = j + 1 < n ? y[j + 1] : 0.0f;
  float a, b;
  sv::unpack2(sv::ex2_poly_x2(y0, y1), a, b);
  poly[j] = a;
  mufu[j] = sv::ex2f(y0);
  if (j + 1 < n) {
    poly[j + 1] = b;
    mufu[j + 1] = sv::ex2f(y1);
  }
}

__global__ void exp1_probe_kernel(const uint32_t* __restrict__ w, float* __restrict__ one,
                                  float* __restrict__ two, long long n) {
  const long long j = 2 * (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x);
  if (j >= n) return;
  const uint32_t w0 = w[j], w1 = j + 1 < n ? w[j + 1] : 0u;
  float e0, e1;
  sv::neg_exp1_log2_x2(w0, w1, e0, e1);
  one[j] = sv::neg_exp1_log2(w0);
  two[j] = e0;
  if (j + 1 < n) {
    one[j + 1] = sv::neg_exp1_log2(w1);
    two[j + 1] = e1;
  }
}

}  // namespace

// poly[j] = ex2_poly_x2 of y[j], mufu[j] = ex2f(y[j]); device arrays of n floats.
extern "C" int sv_probe_ex2(const float* y, float* poly, float* mufu, long long n, void* stream) {
  if (n <= 0) return 0;
  const long long pairs = (n + 1) / 2;
  ex2_probe_kernel<<<static_cast<unsigned int>((pairs + 255) / 256), 256, 0,
                     static_cast<cudaStream_t>(stream)>>>(y, poly, mufu, n);
  return cudaGetLastError() == cudaSuccess ? 0 : 4;
}

// one[j] = neg_exp1_log2(w[j]), two[j] = the same from neg_exp1_log2_x2.
extern "C" int sv_probe_exp1(const uint32_t* w, float* one, float* two, long long n,
                             void* stream) {
  if (n <= 0) return 0;
  const long long pairs = (n + 1) / 2;
  exp1_probe_kernel<<<static_cast<unsigned int>((pairs + 255) / 256), 256, 0,
                      static_cast<cudaStream_t>(stream)>>>(w, one, two, n);
  return cudaGetLastError() == cudaSuccess ? 0 : 4;
}
