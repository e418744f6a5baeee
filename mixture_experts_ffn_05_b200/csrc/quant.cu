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

// NVFP4 quantisation of bf16 weight matrices (the "NVFP4 (4-bit) quantized weights" of the
// "Gemma 4 26B-A4B IT" recipe page's variant list), weight-only, in fp32:
//   t = max|W| / (448 * 6) over the whole matrix (t = 1 for an all-zero matrix)
//   per block of 16 consecutive elements of a row: b = E4M3(max|block| / 6 / t), rounded to
//   nearest even and saturating; codes E2M1(w / (b t)), nearest, ties to even, saturating
//   at +-6 (a block whose scale is zero gets code 0 throughout).
// E2M1 values: 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives; code = sign << 3 | index.
// Packed 8 codes to a 32-bit word: nibbles 0-3 hold elements 0, 2, 4, 6 of the word's 8,
// nibbles 4-7 elements 1, 3, 5, 7 (the order the weight-streaming kernel widens them in).

// Pass 1: tensor_amax[m] = max |w| over matrix m, as float bits (zeroed beforehand; the
// bits of non-negative floats order like the floats).
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(int64_t per_matrix_chunks,
                                                         int64_t total_chunks,
                                                         const uint16_t* __restrict__ w,
                                                         unsigned* __restrict__ amax_bits) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  float a = 0.f;
  int64_t m = -1;
  if (i < total_chunks) {
    m = i / per_matrix_chunks;
    float f[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(w) + i), f);
#pragma unroll
    for (int j = 0; j < 8; ++j) a = fmaxf(a, fabsf(f[j]));
  }
  // a warp's chunks may straddle two matrices: combine only lanes of the same matrix
  const int64_t m0 = __shfl_sync(0xffffffffu, m, 0);
  const bool uniform = __all_sync(0xffffffffu, m == m0);
  if (uniform) {
    a = warp_max(a);
    if ((threadIdx.x & 31) == 0 && m0 >= 0) atomicMax(amax_bits + m0, __float_as_uint(a));
  } else if (m >= 0) {
    atomicMax(amax_bits + m, __float_as_uint(a));
  }
}

// E2M1 magnitude index of a >= 0 (round to nearest, ties to the even index, saturating).
__device__ __forceinline__ uint32_t e2m1_index(float a) {
  return static_cast<uint32_t>(a > 0.25f) + static_cast<uint32_t>(a >= 0.75f) +
         static_cast<uint32_t>(a > 1.25f) + static_cast<uint32_t>(a >= 1.75f) +
         static_cast<uint32_t>(a > 2.5f) + static_cast<uint32_t>(a >= 3.5f) +
         static_cast<uint32_t>(a > 5.0f);
}

// Pass 2: one thread per block of 16 elements: its E4M3 scale and 16 packed codes.
__global__ void __launch_bounds__(256) nvfp4_quant_kernel(int64_t blocks_per_matrix,
                                                          int64_t total_blocks,
                                                          const uint16_t* __restrict__ w,
                                                          const float* __restrict__ amax,
                                                          uint8_t* __restrict__ q,
                                                          uint8_t* __restrict__ bscale) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= total_blocks) return;
  const float am = amax[i / blocks_per_matrix];
  const float t = am > 0.f ? __fdiv_rn(am, 2688.0f) : 1.0f;
  const uint4* src = reinterpret_cast<const uint4*>(w) + 2 * i;
  float f[16];
  {
    float lo[8], hi[8];
    unpack8(__ldg(src), lo);
    unpack8(__ldg(src + 1), hi);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      f[j] = lo[j];
      f[8 + j] = hi[j];
    }
  }
  float bmax = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) bmax = fmaxf(bmax, fabsf(f[j]));
  const uint8_t bcode = e4m3_bits_sat(__fdiv_rn(__fdiv_rn(bmax, 6.0f), t));
  const __half bh = __nv_cvt_fp8_to_halfraw(bcode, __NV_E4M3);  // exact
  const float bval = __half2float(bh);
  const float bs = __fmul_rn(bval, t);
  uint32_t code[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float quot = bs > 0.f ? __fdiv_rn(f[j], bs) : 0.f;
    code[j] = (signbit(quot) ? 8u : 0u) | e2m1_index(fabsf(quot));
  }
  uint32_t word[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t* c = code + 8 * h;
    word[h] = c[0] | (c[2] << 4) | (c[4] << 8) | (c[6] << 12) | (c[1] << 16) | (c[3] << 20) |
              (c[5] << 24) | (c[7] << 28);
  }
  reinterpret_cast<uint2*>(q)[i] = make_uint2(word[0], word[1]);
  bscale[i] = bcode;
}

// Pass 3: the matrix scales from the maxima, in place: t = amax / 2688, 1 for a zero matrix.
__global__ void __launch_bounds__(256) nvfp4_tscale_kernel(int64_t matrices, float* __restrict__ ts) {
  const int64_t m = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (m >= matrices) return;
  const float am = ts[m];
  ts[m] = am > 0.f ? __fdiv_rn(am, 2688.0f) : 1.0f;
}

cudaError_t launch_quantize_nvfp4(const uint16_t* w, int64_t matrices, int64_t rows, int cols,
                                  uint8_t* q, uint8_t* bscale, float* tensor_scale,
                                  cudaStream_t s) {
  const int64_t per_matrix = rows * cols;
  cudaError_t e = cudaMemsetAsync(tensor_scale, 0, static_cast<size_t>(matrices) * sizeof(float), s);
  if (e != cudaSuccess) return e;
  const int64_t chunks = matrices * per_matrix / 8;
  nvfp4_amax_kernel<<<static_cast<unsigned>((chunks + 255) / 256), 256, 0, s>>>(
      per_matrix / 8, chunks, w, reinterpret_cast<unsigned*>(tensor_scale));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t blocks = matrices * per_matrix / 16;
  nvfp4_quant_kernel<<<static_cast<unsigned>((blocks + 255) / 256), 256, 0, s>>>(
      per_matrix / 16, blocks, w, tensor_scale, q, bscale);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  nvfp4_tscale_kernel<<<static_cast<unsigned>((matrices + 255) / 256), 256, 0, s>>>(matrices,
                                                                                 tensor_scale);
  return cudaGetLastError();
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
