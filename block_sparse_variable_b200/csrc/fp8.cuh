// fp8.cuh -- e4m3 packing for the FP8 forward (GenericBlockSparseAttention
// article, quantization table, quantType 5: P is cast to fp8 before P V).
#pragma once

#include <stdint.h>

namespace bsa {

// four fp32 values -> four e4m3 bytes, round to nearest even, saturating to
// +-448; a in the lowest byte (element order along K in a 32-bit TMEM column)
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  // cvt ... e4m3x2.f32 d, x, y puts x in the upper byte and y in the lower
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return uint32_t(lo) | (uint32_t(hi) << 16);
}

}  // namespace bsa
