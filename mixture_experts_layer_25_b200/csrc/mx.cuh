// MX (MXFP8) element rule shared by the quantisers and the fused GEMM
// epilogues: E4M3 codes with one E8M0 scale per 32 elements along K.
//
// Olmo-core 3 オープン混合エキスパート学習インフラストラクチャ, section
// "MXFP8による精度最適化": MXFP8 for the expert feed-forward compute.  Rule
// (OCP MX): X = 2^(floor(log2 amax) - 8), code = RNE-saturating E4M3 of v/X,
// an all-zero block gets scale byte 0.  For a bf16 (or bf16-valued fp32)
// block maximum, floor(log2 amax) is the exponent field of amax minus 127,
// so the scale byte is max(expfield(amax) - 8, 0), and 1/X is the fp32
// number with exponent field 254 - byte (exact power-of-two scaling).
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

// byte offset of the scale of (MN index mn, K block kb) in the tensor-core
// layout: 512-byte blocks of 128 MN indices x 4 K blocks
__device__ __forceinline__ size_t mx_sf_offset(int mn, int kb, int kchunks) {
  return ((size_t)(mn >> 7) * kchunks + (kb >> 2)) * 512 + (mn & 31) * 16 + ((mn >> 5) & 3) * 4 +
         (kb & 3);
}

__device__ __forceinline__ uint32_t mx_scale_byte(float amax) {
  const int ef = (__float_as_uint(amax) >> 23) & 0xFF;
  return ef > 8 ? (uint32_t)(ef - 8) : 0u;
}

__device__ __forceinline__ float mx_inv_scale(uint32_t byte) {
  return __uint_as_float((254u - byte) << 23);
}


// two values scaled by (power-of-two, so exact) factors -> two E4M3 codes;
// one packed fp32 multiply for the pair
__device__ __forceinline__ uint32_t mx_encode2s(float a, float b, float sa, float sb) {
  const float2 q = __fmul2_rn(make_float2(a, b), make_float2(sa, sb));
  return (uint32_t)__nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3);
}

// 8 values -> 8 E4M3 codes (memory order)
__device__ __forceinline__ uint2 mx_encode8(const float* f, float inv) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = mx_encode2s(f[2 * i], f[2 * i + 1], inv, inv);
  return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// scale byte of a block whose largest magnitude has the bf16 bit pattern
// `bits` (sign clear): the exponent field sits in bits 7..14
__device__ __forceinline__ uint32_t mx_scale_byte_bf16(uint32_t bits) {
  const int ef = (int)(bits >> 7) & 0xFF;
  return ef > 8 ? (uint32_t)(ef - 8) : 0u;
}

// lane-wise maximum of two pairs of non-negative bf16 numbers
__device__ __forceinline__ uint32_t mx_max_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// A warp's 32 x 32 block of bf16 numbers (lane = row, v[j] = column j as
// fp32, w[i] = columns 2i | 2i+1 as a bf16 pair, low half first) quantised
// both ways: cr = the lane's row codes (blocks of 32 along the row), cc =
// its codes under the column scales (blocks of 32 rows down each column),
// 4 codes per word in column order; br = the row's scale byte, bc = the
// scale byte of column `lane`.  The magnitudes are compared as bf16 pairs;
// the column maxima come from a transposing butterfly over the lanes (each
// of five exchange rounds halves the words a lane holds, so that lane L
// ends with column L's maximum over the 32 rows).  The 32 reciprocal
// column scales reach every lane through inv_s (32 floats of this warp's
// shared memory).
__device__ __forceinline__ void mx_quant_block32_regs(const float* v, const uint32_t* w,
                                                      uint32_t* cr, uint32_t* cc, uint32_t& br,
                                                      uint32_t& bc, float* inv_s) {
  const int lane = threadIdx.x & 31;
  uint32_t a[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) a[i] = w[i] & 0x7fff7fffu;
  uint32_t m = a[0];
#pragma unroll
  for (int i = 1; i < 16; ++i) m = mx_max_bf16x2(m, a[i]);
  br = mx_scale_byte_bf16(max(m & 0xffffu, m >> 16));
  const float inv = mx_inv_scale(br);
#pragma unroll
  for (int n = 16, s = 16; s >= 2; n >>= 1, s >>= 1) {
    // words [0, n/2) cover the lower half of this lane's columns, [n/2, n)
    // the upper; lanes with bit s keep the upper half
    const bool up = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const uint32_t send = up ? a[i] : a[i + n / 2];
      const uint32_t keep = up ? a[i + n / 2] : a[i];
      a[i] = mx_max_bf16x2(keep, __shfl_xor_sync(0xffffffffu, send, s));
    }
  }
  const uint32_t pm = mx_max_bf16x2(a[0], __shfl_xor_sync(0xffffffffu, a[0], 1));
  bc = mx_scale_byte_bf16((lane & 1) ? pm >> 16 : pm & 0xffffu);
  __syncwarp();
  inv_s[lane] = mx_inv_scale(bc);
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float4 ic = *reinterpret_cast<const float4*>(inv_s + j);
    cr[j / 4] = mx_encode2s(v[j], v[j + 1], inv, inv) |
                (mx_encode2s(v[j + 2], v[j + 3], inv, inv) << 16);
    cc[j / 4] = mx_encode2s(v[j], v[j + 1], ic.x, ic.y) |
                (mx_encode2s(v[j + 2], v[j + 3], ic.z, ic.w) << 16);
  }
}

// mx_quant_block32_regs with the codes written to two [32 rows x 32 bytes]
// shared-memory boxes (row r at r * 32; box_r: row codes, box_c: column
// codes) and the scale bytes to global memory: the row scale of (row,
// col0/32) with K = the row length (row_kchunks = K / 128), the column
// scale of (col0 + lane, row0/32) with K = the padded row count
// (col_kchunks = A_pad_max / 128).  inv_s: as in mx_quant_block32_regs.
__device__ __forceinline__ void mx_quant_block32(const float* v, const uint32_t* w,
                                                 uint8_t* box_r, uint8_t* box_c,
                                                 uint8_t* scales_r, int row, int col0,
                                                 int row_kchunks, uint8_t* scales_c, int row0,
                                                 int col_kchunks, float* inv_s) {
  const int lane = threadIdx.x & 31;
  uint32_t cr[8], cc[8], br, bc;
  mx_quant_block32_regs(v, w, cr, cc, br, bc, inv_s);
  *reinterpret_cast<uint4*>(box_r + lane * 32) = make_uint4(cr[0], cr[1], cr[2], cr[3]);
  *reinterpret_cast<uint4*>(box_r + lane * 32 + 16) = make_uint4(cr[4], cr[5], cr[6], cr[7]);
  *reinterpret_cast<uint4*>(box_c + lane * 32) = make_uint4(cc[0], cc[1], cc[2], cc[3]);
  *reinterpret_cast<uint4*>(box_c + lane * 32 + 16) = make_uint4(cc[4], cc[5], cc[6], cc[7]);
  scales_r[mx_sf_offset(row, col0 >> 5, row_kchunks)] = (uint8_t)br;
  scales_c[mx_sf_offset(col0 + lane, row0 >> 5, col_kchunks)] = (uint8_t)bc;
}

}  // namespace moe
