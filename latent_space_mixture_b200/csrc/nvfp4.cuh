// NVFP4 on the device: E2M1 elements, 16-element micro-blocks along the GEMM
// reduction axis, E4M3 block scales, FP32 global scale ("NVIDIA Nemotron 3:
// Efficient and Open Intelligence", section 三 "NVFP4 训练"; "Nemotron-3 Super
// 精读报告", section 5.3).  Rounding is round-to-nearest-even with saturation
// (the cvt instructions below), the scale arithmetic IEEE float32 in a fixed
// order so that the codes are reproducible:
//   six_g = 6 g; sbf = amax / six_g; s = E4M3(sbf); denom = s g;
//   r = 1 / denom (rounded once per block); q = E2M1(x * r), or 0 when
//   denom == 0.
//
// Scale-factor layout consumed by tcgen05.mma ... block_scale (block16): an
// "atom" of 512 bytes covers 128 rows x 64 reduction elements (4 scales per
// row); the scale of row m (0..127) and 16-block k1 (0..3) is byte
// (m % 32) * 16 + (m / 32) * 4 + k1.  A matrix's atoms are stored with the
// 64-wide reduction chunk fastest.
#pragma once
#include <cuda_fp8.h>
#include <cstdint>

namespace lmoe {

constexpr int NVFP4_BLOCK = 16;
constexpr int SF_ATOM_BYTES = 512;

__device__ __forceinline__ int sf_atom_offset(int m, int k1) {
  return (m & 31) * 16 + ((m >> 5) & 3) * 4 + k1;
}

// Two floats to two E2M1 codes in one byte: `lo` in bits 0-3, `hi` in bits 4-7
// (the lower reduction index in the lower nibble).
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u16.u8 %0, t;\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// Eight floats times r to eight E2M1 codes in one word: element i in bits
// 4i..4i+3 (the byte layout of e2m1x2, four bytes packed lowest first).
__device__ __forceinline__ uint32_t e2m1x8(const float* x, float r) {
  uint32_t w;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(w)
      : "f"(__fmul_rn(x[0], r)), "f"(__fmul_rn(x[1], r)), "f"(__fmul_rn(x[2], r)),
        "f"(__fmul_rn(x[3], r)), "f"(__fmul_rn(x[4], r)), "f"(__fmul_rn(x[5], r)),
        "f"(__fmul_rn(x[6], r)), "f"(__fmul_rn(x[7], r)));
  return w;
}

__device__ __forceinline__ uint8_t e4m3_code(float x) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float e4m3_value(uint8_t code) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
  return __half2float(__half(h));
}

// E2M1 code (bit 3 = sign) -> value: magnitudes 0, 0.5, 1, 1.5 (codes 0-3,
// code / 2), 2, 3 (codes 4-5, code - 2), 4, 6 (codes 6-7, 2 code - 8)
__device__ __forceinline__ float e2m1_value(uint32_t code) {
  const int m = static_cast<int>(code & 7);
  const float v = m < 4 ? 0.5f * static_cast<float>(m)
                        : static_cast<float>(m < 6 ? m - 2 : 2 * m - 8);
  return (code & 8) ? -v : v;
}

// Codes of 16 elements under a given E4M3 scale code (the arithmetic of
// nvfp4_block after its scale choice).
__device__ __forceinline__ void nvfp4_codes_with_scale(const float (&x)[16], float g, uint8_t sc,
                                                       uint8_t (&out)[8]) {
  const float denom = __fmul_rn(e4m3_value(sc), g);
  const float r = denom > 0.0f ? __fdiv_rn(1.0f, denom) : 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    out[i] = static_cast<uint8_t>(e2m1x2(__fmul_rn(x[2 * i], r), __fmul_rn(x[2 * i + 1], r)));
}

// Continue a float32 squared-error sum over 16 elements quantised with scale
// code sc, in element order: err += (x - q * denom)^2, every step rounded
// (no fused multiply-add), as the MSE scale search of the weight quantiser.
__device__ __forceinline__ float nvfp4_sq_error(const float (&x)[16], float g, uint8_t sc,
                                                float err) {
  const float denom = __fmul_rn(e4m3_value(sc), g);
  const float r = denom > 0.0f ? __fdiv_rn(1.0f, denom) : 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t b = e2m1x2(__fmul_rn(x[2 * i], r), __fmul_rn(x[2 * i + 1], r));
    const float d0 = __fsub_rn(x[2 * i], __fmul_rn(e2m1_value(b & 15), denom));
    err = __fadd_rn(err, __fmul_rn(d0, d0));
    const float d1 = __fsub_rn(x[2 * i + 1], __fmul_rn(e2m1_value(b >> 4), denom));
    err = __fadd_rn(err, __fmul_rn(d1, d1));
  }
  return err;
}

// Quantise one 16-element block: returns the E4M3 scale code and writes the 8
// packed bytes of codes.
__device__ __forceinline__ uint8_t nvfp4_block(const float (&x)[16], float g, uint8_t (&out)[8]) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  const float six_g = __fmul_rn(6.0f, g);
  const float sbf = six_g > 0.0f ? __fdiv_rn(amax, six_g) : 0.0f;
  const uint8_t sc = e4m3_code(sbf);
  const float denom = __fmul_rn(e4m3_value(sc), g);
  const float r = denom > 0.0f ? __fdiv_rn(1.0f, denom) : 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    out[i] = static_cast<uint8_t>(e2m1x2(__fmul_rn(x[2 * i], r), __fmul_rn(x[2 * i + 1], r)));
  return sc;
}

// ---------------------------------------------------------------------------
// Scale tables of one static global scale g (NVFP4_TAB floats, built once by
// launch_scale_tables): thr[k] (k = 1..126) is the smallest float amax whose
// block scale code E4M3(f32(amax / f32(6 g))) is at least k, thr[0] = 0 and
// thr[127] = infinity; rtab[k] = f32(1 / f32(E4M3value(k) g)), or 0 when that
// product is 0; inv6g = f32(1 / f32(6 g)).  The code is a monotone step
// function of amax, so counting thresholds reproduces it exactly; a product
// with inv6g lands within one code of it, and one comparison corrects it.
constexpr int NVFP4_TAB = 256;   // thr [0, 128), rtab [128, 255), inv6g [255]

// (The five table entries the correction may need are loaded together, so
// that the lookup costs one load latency.)
__device__ __forceinline__ uint8_t nvfp4_scale_tab(float amax, const float* __restrict__ tab,
                                                   float* r) {
  int code = e4m3_code(__fmul_rn(amax, tab[255]));
  code = code > 126 ? 126 : code;
  const float t0 = tab[code], t1 = tab[code + 1];
  const float r_dn = tab[128 + (code > 0 ? code - 1 : 0)], r_0 = tab[128 + code],
              r_up = tab[128 + code + 1];
  const bool up = amax >= t1, dn = !up && amax < t0;
  *r = up ? r_up : dn ? r_dn : r_0;
  return static_cast<uint8_t>(code + (up ? 1 : 0) - (dn ? 1 : 0));
}

// ---------------------------------------------------------------------------
// Gradient-path pieces of the NVFP4 training recipe ("Nemotron-3 Super 精读报告",
// section 5.3: a random Hadamard transform on the inputs of the weight-gradient
// GEMMs, stochastic rounding of gradient tensors; section 9.3: stochastic
// rounding is unbiased in expectation).
//
// Random bits: SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom
// number generators", OOPSLA 2014) used as a counter-based generator: counter
// i gives mix(seed + (i + 1) * 0x9E3779B97F4A7C15).  Element (row, col) of a
// [rows][cols] tensor takes counter row * cols + col; the transform's signs
// take counters 0..15 (sign -1 when bit 63 is set); a uniform in [0, 1) is
// the top 24 bits times 2^-24.

// SplitMix64 output for counter ctr, up to its last step z ^ (z >> 31): that
// step leaves bits 33..63 unchanged, and only the top 24 bits (uniforms) and
// bit 63 (the transform's signs) are used.
constexpr uint64_t SPLITMIX_GAMMA = 0x9E3779B97F4A7C15ull;

// the mixing steps from the state z = seed + (ctr + 1) gamma
__device__ __forceinline__ uint64_t splitmix64_mix_high(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  return (z ^ (z >> 27)) * 0x94D049BB133111EBull;
}

__device__ __forceinline__ uint64_t splitmix64_high(uint64_t seed, uint64_t ctr) {
  return splitmix64_mix_high(seed + (ctr + 1ull) * SPLITMIX_GAMMA);
}

// a uniform in [0, 1) from the state of a counter (consecutive counters'
// states differ by gamma, so a run of them costs one multiply less each)
__device__ __forceinline__ float uniform24_z(uint64_t z) {
  return static_cast<float>(static_cast<uint32_t>(splitmix64_mix_high(z) >> 40)) *
         5.9604644775390625e-8f;   // 2^-24
}

__device__ __forceinline__ float uniform24(uint64_t seed, uint64_t ctr) {
  return uniform24_z(seed + (ctr + 1ull) * SPLITMIX_GAMMA);
}

// Stochastic rounding of v to an E2M1 code (bit 3 = sign): the upper grid
// neighbour with probability (|v| - lo) / (hi - lo), the lower otherwise;
// |v| >= 6 saturates.  The probability is exact in float32 (hi - lo is a
// power of two, |v| - lo is exact).
// The grid step is 0.5 below 2, 1 below 4 and 2 below 6, so lo = floor(|v| /
// step) step, |v| - lo (exact: lo <= |v| < 2 lo or lo = 0) and its quotient
// by the step (a power of two) are all exact products, without a division.
__device__ __forceinline__ uint32_t e2m1_sr(float v, float u) {
  const float mag = fabsf(v);
  uint32_t code;
  if (mag >= 6.0f) {
    code = 7;
  } else {
    const bool b0 = mag < 2.0f, b1 = mag < 4.0f;
    const float inv = b0 ? 2.0f : b1 ? 1.0f : 0.5f;      // 1 / step
    const float k = floorf(mag * inv);
    const float p = __fsub_rn(mag * inv, k);              // (|v| - lo) / step
    const int lo = b0 ? static_cast<int>(k) : b1 ? static_cast<int>(k) + 2 : 6;
    code = static_cast<uint32_t>(u < p ? lo + 1 : lo);
  }
  return code | (signbit(v) ? 8u : 0u);
}

// y = (1/4) H16 (s * x) on one 16-element block, in place: signs s from
// counters 0..15 of `seed` (rht16_signs: bit j set for sign -1), float32
// butterflies (stages 1, 2, 4, 8: (a, b) -> (a + b, a - b)), then the exact
// product by 0.25.
__device__ __forceinline__ uint32_t rht16_signs(uint64_t seed) {
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j)
    m |= static_cast<uint32_t>(splitmix64_high(seed, static_cast<uint64_t>(j)) >> 63) << j;
  return m;
}

__device__ __forceinline__ void rht16_masked(float (&b)[16], uint32_t signs) {
#pragma unroll
  for (int j = 0; j < 16; ++j)
    if ((signs >> j) & 1u) b[j] = -b[j];
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j & h) continue;
      const float a = b[j], c = b[j + h];
      b[j] = __fadd_rn(a, c);
      b[j + h] = __fsub_rn(a, c);
    }
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) b[j] = b[j] * 0.25f;
}

__device__ __forceinline__ void rht16_block(float (&b)[16], uint64_t seed) {
  rht16_masked(b, rht16_signs(seed));
}

}  // namespace lmoe
