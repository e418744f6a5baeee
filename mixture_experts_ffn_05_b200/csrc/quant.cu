// Per-output-row symmetric int8 quantisation of bf16 weights ("Gemma-4 26B-A4B (MoE,
// int8 experts) on AWS Inferentia2", "How it works": per-channel symmetric INT8 expert
// weights).  In fp32, the precision the rounding decision is taken in:
//   s = max|w| / 127   (s = 1 for an all-zero row)
//   q = round-half-even(w / s), clamped to [-127, 127]
// One warp per row; cols a multiple of 8.
#include "common.cuh"
#include "internal.h"

namespace moe {

__global__ void __launch_bounds__(256) quantize_int8_kernel(int64_t rows, int cols,
                                                            const uint16_t* __restrict__ w,
                                                            int8_t* __restrict__ q,
                                                            float* __restrict__ scales) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  pdl_wait();
  if (r >= rows) return;
  const int lane = threadIdx.x & 31;
  const uint4* wr = reinterpret_cast<const uint4*>(w + r * cols);
  const int nch = cols >> 3;
  float amax = 0.f;
  for (int c = lane; c < nch; c += 32) {
    float f[8];
    unpack8(__ldg(wr + c), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
  }
  amax = warp_max(amax);
  const float s = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 1.0f;
  if (lane == 0) scales[r] = s;
  uint2* qr = reinterpret_cast<uint2*>(q + r * cols);
  for (int c = lane; c < nch; c += 32) {
    float f[8];
    unpack8(__ldg(wr + c), f);
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float v = rintf(__fdiv_rn(f[i], s));
      v = fminf(127.f, fmaxf(-127.f, v));
      const uint32_t b = static_cast<uint32_t>(static_cast<int32_t>(v)) & 0xFFu;
      packed[i >> 2] |= b << (8 * (i & 3));
    }
    qr[c] = make_uint2(packed[0], packed[1]);
  }
}

// Per-output-row E4M3 quantisation of bf16 weights (the FP8-dynamic variant of the "Gemma
// 4 26B-A4B IT" recipe page, "Quantized Variants": E4M3 weights), in fp32:
//   s = max|w| / 448   (s = 1 for an all-zero row)
//   q = E4M3 code of (w / s), rounded to nearest even, saturating at +-448
// One warp per row; cols a multiple of 8.
__global__ void __launch_bounds__(256) quantize_fp8_kernel(int64_t rows, int cols,
                                                           const uint16_t* __restrict__ w,
                                                           uint8_t* __restrict__ q,
                                                           float* __restrict__ scales) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  pdl_wait();
  if (r >= rows) return;
  const int lane = threadIdx.x & 31;
  const uint4* wr = reinterpret_cast<const uint4*>(w + r * cols);
  const int nch = cols >> 3;
  float amax = 0.f;
  for (int c = lane; c < nch; c += 32) {
    float f[8];
    unpack8(__ldg(wr + c), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
  }
  amax = warp_max(amax);
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  if (lane == 0) scales[r] = s;
  uint2* qr = reinterpret_cast<uint2*>(q + r * cols);
  for (int c = lane; c < nch; c += 32) {
    float f[8];
    unpack8(__ldg(wr + c), f);
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i)
      packed[i >> 2] |= static_cast<uint32_t>(e4m3_bits_sat(__fdiv_rn(f[i], s))) << (8 * (i & 3));
    qr[c] = make_uint2(packed[0], packed[1]);
  }
}

cudaError_t launch_quantize_fp8(const uint16_t* w, int64_t rows, int cols, uint8_t* q,
                                float* scales, cudaStream_t s) {
  const int64_t blocks = (rows + 7) / 8;
  quantize_fp8_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(rows, cols, w, q, scales);
  return cudaGetLastError();
}

cudaError_t launch_quantize_int8(const uint16_t* w, int64_t rows, int cols, int8_t* q,
                                 float* scales, cudaStream_t s) {
  const int64_t blocks = (rows + 7) / 8;
  quantize_int8_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(rows, cols, w, q, scales);
  return cudaGetLastError();
}

}  // namespace moe
