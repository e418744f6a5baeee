// Warp-level tensor-core MMA (mma.sync), for kernels whose operands are formed in
// registers (the weight-streaming GEMM, the small-batch router).  sm_100a.
#pragma once

#include <stdint.h>

namespace moe {

// D += A B with mma.sync m16n8k16 (fp32 accumulators), fp16 or bf16 operands.  Lane
// (g, t) = (lane / 4, lane % 4) holds A rows g and g + 8 at K columns (2t, 2t + 1) in a0 /
// a1 and (2t + 8, 2t + 9) in a2 / a3, B column g at K rows (2t, 2t + 1) in b0 and (2t + 8,
// 2t + 9) in b1 (lower K index in the low half), and C rows g / g + 8 at columns 2t, 2t + 1.
template <bool BF16>
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

}  // namespace moe
