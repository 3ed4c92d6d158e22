// selfcheck.cuh -- inputs of the start-up self-check, generated on the device.
//
// Every element i of tensor `tid` is drawn from r = SplitMix64(base + tid * 2^32 + i),
// SplitMix64 being the output function of Steele, Lea & Flood, "Fast splittable
// pseudorandom number generators" (OOPSLA 2014): z = c + 0x9E3779B97F4A7C15,
// z = (z ^ z >> 30) * 0xBF58476D1CE4E5B9, z = (z ^ z >> 27) * 0x94D049BB133111EB,
// r = z ^ z >> 31.  The expected results were computed on the CPU from the same
// definition, so a wrong byte here shows up as a failed check.
#pragma once
#include <cstdint>

namespace moe {

constexpr uint64_t SELFCHECK_BASE = 0x5EED000000000000ull;

enum SelfcheckKind {
  SC_BF16 = 0,   // sign r>>63, exponent e0 + ((r>>56) & 3), mantissa r & 0x7F
  SC_BYTE = 1,   // r & 0xFF (MXFP4 code pairs)
  SC_E8M0 = 2,   // 120 + r % 8
  SC_E4M3 = 3,   // r & 0xFF, the two NaN codes replaced by 0
  SC_POW2 = 4    // fp32 2^-(8 + r % 6)
};

__device__ __forceinline__ uint64_t splitmix64(uint64_t c) {
  uint64_t z = c + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void k_selfcheck_fill(void* dst, uint32_t n, int kind, uint32_t tid, int e0) {
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const uint64_t r = splitmix64(SELFCHECK_BASE + (static_cast<uint64_t>(tid) << 32) + i);
    switch (kind) {
      case SC_BF16:
        static_cast<uint16_t*>(dst)[i] = static_cast<uint16_t>(((r >> 63) << 15) |
                                                               ((e0 + ((r >> 56) & 3)) << 7) | (r & 0x7F));
        break;
      case SC_BYTE:
        static_cast<uint8_t*>(dst)[i] = static_cast<uint8_t>(r & 0xFF);
        break;
      case SC_E8M0:
        static_cast<uint8_t*>(dst)[i] = static_cast<uint8_t>(120 + r % 8);
        break;
      case SC_E4M3: {
        const uint8_t q = static_cast<uint8_t>(r & 0xFF);
        static_cast<uint8_t*>(dst)[i] = (q & 0x7F) == 0x7F ? 0 : q;
        break;
      }
      default:
        static_cast<uint32_t*>(dst)[i] = static_cast<uint32_t>(127 - 8 - r % 6) << 23;
        break;
    }
  }
}

}  // namespace moe
