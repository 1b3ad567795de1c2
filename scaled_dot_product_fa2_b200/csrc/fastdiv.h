// fastdiv.h -- division by a divisor fixed at launch, as a multiply-high and
// a shift (T. Granlund and P. Montgomery, "Division by invariant integers
// using multiplication", PLDI 1994, the unsigned case): for 1 <= d < 2^31
// and 0 <= n < 2^31,
//     n / d == (umulhi(m, n) + n) >> l,
//     l = ceil(log2 d),  m = floor(2^32 (2^l - d) / d) + 1  (m < 2^32).
// The sum cannot overflow 32 bits because umulhi(m, n) <= n < 2^31.
// Host and device code share this header; make_fastdiv runs on the host.
#pragma once
#include <cstdint>

#ifdef __CUDACC__
#define SDPA_HOST_DEVICE __host__ __device__ __forceinline__
#else
#define SDPA_HOST_DEVICE inline
#endif

namespace sdpa {

struct FastDiv {
  uint32_t m;  // multiplier
  uint32_t l;  // shift
};

// d in [1, 2^31).
inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while ((uint64_t{1} << l) < d) ++l;
  const uint64_t m = ((uint64_t{1} << 32) * ((uint64_t{1} << l) - d)) / d + 1;
  return FastDiv{static_cast<uint32_t>(m), l};
}

// n / d for n in [0, 2^31).
SDPA_HOST_DEVICE uint32_t fastdiv(uint32_t n, FastDiv f) {
#ifdef __CUDA_ARCH__
  const uint32_t t = __umulhi(f.m, n);
#else
  const uint32_t t = static_cast<uint32_t>((uint64_t{f.m} * n) >> 32);
#endif
  return (t + n) >> f.l;
}

}  // namespace sdpa
