// Per-row E4M3 quantisation for the FP8 score path.
//
// The StreamIndex abstract's reference list cites "FP8 Formats for Deep
// Learning" (the E4M3 format) and "Microscaling Data Formats for Deep
// Learning"; the abstract itself fixes no scaling.  This library scales each
// row by its own absolute maximum: scale = amax / 448 (448 = largest finite
// E4M3), code = E4M3(x / scale) rounded to nearest even and saturated.  Both
// divisions are IEEE round-to-nearest (__fdiv_rn), so the codes are a fixed
// function of the input bits.  Rows of 64, 128 or 256 values are read once by
// a group of 8, 16 or 32 lanes; other lengths take one warp per row.  HBM-bound.
#include "si_kernels.h"

namespace si {

constexpr int kQuantWarps = 8;

// Codes of 8 consecutive bf16 values (one 16-byte word) for scale s, two per
// conversion (first element in the low byte).
SI_DEV uint2 e4m3_codes8(const uint4 v, float s) {
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
  return o;
}

SI_DEV float amax8(const uint4 v, float amax) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    amax = fmaxf(amax, fabsf(__uint_as_float(w[i] << 16)));
    amax = fmaxf(amax, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
  }
  return amax;
}

// Short rows (cols = 8 * G with G a power of two <= 32): a group of G lanes
// holds one row, 8 values per lane, read once; a warp covers 32/G rows.
template <int G>
__global__ void __launch_bounds__(kQuantWarps * 32)
    k_quant_short(const uint16_t* __restrict__ x, int64_t rows, uint8_t* __restrict__ x8,
                  float* __restrict__ scale) {
  constexpr int cols = 8 * G;
  const int lane = threadIdx.x & 31;
  const int64_t row =
      ((int64_t)blockIdx.x * kQuantWarps + (threadIdx.x >> 5)) * (32 / G) + lane / G;
  const int c = (lane % G) * 8;
  const bool live = row < rows;
  const uint4 v = live ? *reinterpret_cast<const uint4*>(x + row * cols + c) : make_uint4(0, 0, 0, 0);
  float amax = amax8(v, 0.0f);
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  const float s = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
  if (!live) return;
  if (lane % G == 0) scale[row] = s;
  *reinterpret_cast<uint2*>(x8 + row * cols + c) = e4m3_codes8(v, s);
}

// Any row length: one warp per row, two passes over the row.
__global__ void __launch_bounds__(kQuantWarps * 32)
    k_quant_rows(const uint16_t* __restrict__ x, int64_t rows, int cols, uint8_t* __restrict__ x8,
                 float* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const uint16_t* xr = x + row * cols;
  float amax = 0.0f;
  for (int c = lane * 8; c < cols; c += 32 * 8)
    amax = amax8(*reinterpret_cast<const uint4*>(xr + c), amax);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  const float s = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
  if (lane == 0) scale[row] = s;
  for (int c = lane * 8; c < cols; c += 32 * 8)
    *reinterpret_cast<uint2*>(x8 + row * cols + c) =
        e4m3_codes8(*reinterpret_cast<const uint4*>(xr + c), s);
}

template <int G>
static cudaError_t launch_short(const uint16_t* x, int64_t rows, uint8_t* x8, float* scale,
                                cudaStream_t stream) {
  const int64_t per_block = (int64_t)kQuantWarps * (32 / G);
  const int64_t blocks = (rows + per_block - 1) / per_block;
  k_quant_short<G><<<(unsigned)blocks, kQuantWarps * 32, 0, stream>>>(x, rows, x8, scale);
  return cudaGetLastError();
}

cudaError_t launch_quantize_fp8(const uint16_t* x, int64_t rows, int cols, uint8_t* x8,
                                float* scale, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  switch (cols) {
    case 64: return launch_short<8>(x, rows, x8, scale, stream);
    case 128: return launch_short<16>(x, rows, x8, scale, stream);
    case 256: return launch_short<32>(x, rows, x8, scale, stream);
    default: break;
  }
  const int64_t blocks = (rows + kQuantWarps - 1) / kQuantWarps;
  k_quant_rows<<<(unsigned)blocks, kQuantWarps * 32, 0, stream>>>(x, rows, cols, x8, scale);
  return cudaGetLastError();
}

}  // namespace si
