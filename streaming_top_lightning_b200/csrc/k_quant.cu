// Per-row E4M3 quantisation for the FP8 score path.
//
// The StreamIndex abstract's reference list cites "FP8 Formats for Deep
// Learning" (the E4M3 format) and "Microscaling Data Formats for Deep
// Learning"; the abstract itself fixes no scaling.  This library scales each
// row by its own absolute maximum: scale = amax / 448 (448 = largest finite
// E4M3), code = E4M3(x / scale) rounded to nearest even and saturated.  Both
// divisions are IEEE round-to-nearest (__fdiv_rn), so the codes are a fixed
// function of the input bits.  One warp per row; HBM-bound.
#include "si_kernels.h"

namespace si {

constexpr int kQuantWarps = 8;

__global__ void __launch_bounds__(kQuantWarps * 32)
    k_quant_rows(const uint16_t* __restrict__ x, int64_t rows, int cols, uint8_t* __restrict__ x8,
                 float* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const uint16_t* xr = x + row * cols;
  // pass 1: amax over the row, 8 bf16 per 16-byte load
  float amax = 0.0f;
  for (int c = lane * 8; c < cols; c += 32 * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(xr + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      amax = fmaxf(amax, fabsf(__uint_as_float(w[i] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  const float s = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
  if (lane == 0) scale[row] = s;
  // pass 2: codes, two per conversion (first element in the low byte)
  for (int c = lane * 8; c < cols; c += 32 * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(xr + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint16_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __fdiv_rn(__uint_as_float(w[i] << 16), s);
      const float hi = __fdiv_rn(__uint_as_float(w[i] & 0xFFFF0000u), s);
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out[i]) : "f"(hi), "f"(lo));
    }
    uint2 o;
    o.x = (uint32_t)out[0] | ((uint32_t)out[1] << 16);
    o.y = (uint32_t)out[2] | ((uint32_t)out[3] << 16);
    *reinterpret_cast<uint2*>(x8 + row * cols + c) = o;
  }
}

cudaError_t launch_quantize_fp8(const uint16_t* x, int64_t rows, int cols, uint8_t* x8,
                                float* scale, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int64_t blocks = (rows + kQuantWarps - 1) / kQuantWarps;
  k_quant_rows<<<(unsigned)blocks, kQuantWarps * 32, 0, stream>>>(x, rows, cols, x8, scale);
  return cudaGetLastError();
}

}  // namespace si
