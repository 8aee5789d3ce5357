// NVFP4 kernels of the LatentMoE expert path: quantisation of the expert
// weights at layer creation (per-expert FP32 global scale, E4M3 block scales,
// E2M1 codes), a standalone row quantiser, and the gather of quantised
// latent rows into expert order.  Format: "NVIDIA Nemotron 3: Efficient and
// Open Intelligence", section 三 "NVFP4 训练"; "Nemotron-3 Super 精读报告",
// section 5.3 (blocks along the GEMM reduction axis).
#include <cuda_bf16.h>

#include "kernels.h"
#include "launch.cuh"
#include "nvfp4.cuh"
#include "ptx.cuh"

namespace lmoe {

// amax[e] = max |W[e]| over a [E][rows_per][K] bf16 tensor (amax pre-zeroed;
// non-negative floats order like their bit patterns, so atomicMax on ints).
__global__ void __launch_bounds__(256) k_amax_expert(const __nv_bfloat16* __restrict__ w,
                                                     int64_t per_expert, float* amax) {
  const int e = blockIdx.y;
  const __nv_bfloat162* p =
      reinterpret_cast<const __nv_bfloat162*>(w + static_cast<int64_t>(e) * per_expert);
  const int64_t n2 = per_expert / 2;
  float m = 0.0f;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n2;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float2 f = __bfloat1622float2(p[i]);
    m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  __shared__ float wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.0f;
    for (int i = 0; i < 8; ++i) b = fmaxf(b, wm[i]);
    atomicMax(reinterpret_cast<int*>(amax + e), __float_as_int(b));
  }
}

// One thread per (row, 16-element block) of a [E * rows_per][K] bf16 matrix:
// codes into [row][Kp/2] bytes, scale into the 512-byte atoms
// [row / 128][Kp / 64], global scale g[e] = amax[e] / (6 * 448).
__global__ void __launch_bounds__(256) k_quant_weight(const __nv_bfloat16* __restrict__ w,
                                                      int64_t rows, int rows_per, int K, int Kp,
                                                      const float* __restrict__ amax,
                                                      uint8_t* __restrict__ codes,
                                                      uint8_t* __restrict__ atoms,
                                                      float* __restrict__ gscale) {
  const int kb16 = K / 16;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= rows * kb16) return;
  const int64_t row = i / kb16;
  const int blk = static_cast<int>(i - row * kb16);
  const int e = static_cast<int>(row / rows_per);
  const float g = __fdiv_rn(amax[e], 6.0f * 448.0f);
  if (blk == 0 && row % rows_per == 0) gscale[e] = g;
  float x[16];
  const __nv_bfloat162* src = reinterpret_cast<const __nv_bfloat162*>(w + row * K + blk * 16);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float2 f = __bfloat1622float2(src[j]);
    x[2 * j] = f.x;
    x[2 * j + 1] = f.y;
  }
  uint8_t q[8];
  const uint8_t sc = nvfp4_block(x, g, q);
  uint8_t* dst = codes + row * (Kp / 2) + blk * 8;
  *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(q);
  const int kc = blk / 4, k1 = blk % 4;
  atoms[((row / 128) * (Kp / 64) + kc) * SF_ATOM_BYTES + sf_atom_offset(static_cast<int>(row % 128), k1)] = sc;
}

// Weight variants ("Nemotron-3 Super 精读报告", section 5.3: 2D block scaling
// of weights; section 9.2: weight block scales chosen by minimum MSE).  One
// thread per scale unit: a (row, 16-block) in 1D, a (16-row group, 16-block)
// in 2D, whose 16 rows share the scale.  MSE: the candidates are the E4M3
// codes from 8 below to 2 above the max-based code (clipped to 1..126), the
// error is the float32 sum in row-major element order, ties go to the higher
// code, an all-zero unit keeps code 0.
template <bool TWO_D, bool MSE>
__global__ void __launch_bounds__(128) k_quant_weight_var(const __nv_bfloat16* __restrict__ w,
                                                          int64_t rows, int rows_per, int K,
                                                          int Kp, const float* __restrict__ amax,
                                                          uint8_t* __restrict__ codes,
                                                          uint8_t* __restrict__ atoms,
                                                          float* __restrict__ gscale) {
  constexpr int R = TWO_D ? 16 : 1;   // rows per unit
  const int kb16 = K / 16;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= (rows / R) * kb16) return;
  const int64_t row0 = (i / kb16) * R;
  const int blk = static_cast<int>(i - (i / kb16) * kb16);
  const int e = static_cast<int>(row0 / rows_per);
  const float g = __fdiv_rn(amax[e], 6.0f * 448.0f);
  if (blk == 0 && row0 % rows_per == 0) gscale[e] = g;
  auto load = [&](int r, float (&x)[16]) {
    const __nv_bfloat162* src =
        reinterpret_cast<const __nv_bfloat162*>(w + (row0 + r) * K + blk * 16);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 f = __bfloat1622float2(src[j]);
      x[2 * j] = f.x;
      x[2 * j + 1] = f.y;
    }
  };
  float x[16];
  float m = 0.0f;
  for (int r = 0; r < R; ++r) {
    load(r, x);
#pragma unroll
    for (int j = 0; j < 16; ++j) m = fmaxf(m, fabsf(x[j]));
  }
  const float six_g = __fmul_rn(6.0f, g);
  const uint8_t c0 = e4m3_code(six_g > 0.0f ? __fdiv_rn(m, six_g) : 0.0f);
  uint8_t sc = c0;
  if (MSE && c0 != 0) {
    float best = __int_as_float(0x7f800000);   // +inf
    const int lo = c0 > 9 ? c0 - 8 : 1, hi = c0 < 124 ? c0 + 2 : 126;
    for (int c = lo; c <= hi; ++c) {
      float err = 0.0f;
      for (int r = 0; r < R; ++r) {
        load(r, x);
        err = nvfp4_sq_error(x, g, static_cast<uint8_t>(c), err);
      }
      if (err <= best) {
        best = err;
        sc = static_cast<uint8_t>(c);
      }
    }
  }
  const int kc = blk / 4, k1 = blk % 4;
  for (int r = 0; r < R; ++r) {
    const int64_t row = row0 + r;
    load(r, x);
    uint8_t q[8];
    nvfp4_codes_with_scale(x, g, sc, q);
    *reinterpret_cast<uint2*>(codes + row * (Kp / 2) + blk * 8) = *reinterpret_cast<const uint2*>(q);
    atoms[((row / 128) * (Kp / 64) + kc) * SF_ATOM_BYTES + sf_atom_offset(static_cast<int>(row % 128), k1)] = sc;
  }
}

cudaError_t launch_quant_weights(const void* w, int E, int rows_per, int K, int Kp, float* amax,
                                 uint8_t* codes, uint8_t* atoms, float* gscale, int variant,
                                 cudaStream_t st) {
  if (cudaMemsetAsync(amax, 0, E * sizeof(float), st) != cudaSuccess) return cudaGetLastError();
  const int64_t per = static_cast<int64_t>(rows_per) * K;
  k_amax_expert<<<dim3(64, E), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(w), per, amax);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t rows = static_cast<int64_t>(E) * rows_per;
  const __nv_bfloat16* wb = static_cast<const __nv_bfloat16*>(w);
  const bool two_d = variant & QUANT_W_2D, mse = variant & QUANT_W_MSE;
  if (!two_d && !mse) {
    const int64_t n = rows * (K / 16);
    k_quant_weight<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(
        wb, rows, rows_per, K, Kp, amax, codes, atoms, gscale);
    return cudaGetLastError();
  }
  if (two_d && rows_per % 16) return cudaErrorInvalidValue;
  const int64_t n = (two_d ? rows / 16 : rows) * (K / 16);
  const unsigned blocks = static_cast<unsigned>((n + 127) / 128);
  if (two_d && mse)
    k_quant_weight_var<true, true><<<blocks, 128, 0, st>>>(wb, rows, rows_per, K, Kp, amax, codes, atoms, gscale);
  else if (two_d)
    k_quant_weight_var<true, false><<<blocks, 128, 0, st>>>(wb, rows, rows_per, K, Kp, amax, codes, atoms, gscale);
  else
    k_quant_weight_var<false, true><<<blocks, 128, 0, st>>>(wb, rows, rows_per, K, Kp, amax, codes, atoms, gscale);
  return cudaGetLastError();
}

// FP8 (E4M3) W8A8 expert weights ("Nemotron-3 Super 精读报告", section 9.1):
// one float32 scale per expert matrix, s = amax / 448, r = 1 / s (rounded
// once), code = E4M3(x * r) round-to-nearest-even, saturating.  Thread per 8
// consecutive elements of a [E * rows_per][K] bf16 matrix.
__global__ void __launch_bounds__(256) k_quant_w8(const __nv_bfloat16* __restrict__ w,
                                                  int64_t n8, int64_t per_expert,
                                                  const float* __restrict__ amax,
                                                  uint8_t* __restrict__ codes,
                                                  float* __restrict__ scale) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const int e = static_cast<int>(i * 8 / per_expert);
  const float s = __fdiv_rn(amax[e], 448.0f);
  if (i * 8 == static_cast<int64_t>(e) * per_expert) scale[e] = s;
  const float r = s > 0.0f ? __fdiv_rn(1.0f, s) : 0.0f;
  const uint4 raw = reinterpret_cast<const uint4*>(w)[i];
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
  uint8_t q[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __bfloat1622float2(p[j]);
    q[2 * j] = e4m3_code(__fmul_rn(f.x, r));
    q[2 * j + 1] = e4m3_code(__fmul_rn(f.y, r));
  }
  reinterpret_cast<uint2*>(codes)[i] = *reinterpret_cast<const uint2*>(q);
}

cudaError_t launch_quant_w8(const void* w, int E, int rows_per, int K, float* amax, uint8_t* codes,
                            float* scale, cudaStream_t st) {
  if (cudaMemsetAsync(amax, 0, E * sizeof(float), st) != cudaSuccess) return cudaGetLastError();
  const int64_t per = static_cast<int64_t>(rows_per) * K;
  k_amax_expert<<<dim3(64, E), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(w), per, amax);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t n8 = static_cast<int64_t>(E) * per / 8;
  k_quant_w8<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(w), n8, per, amax, codes, scale);
  return cudaGetLastError();
}

// The scale tables of global scale g (nvfp4.cuh, NVFP4_TAB floats): a thread
// per entry; a threshold is found by bisection over the bit patterns of the
// non-negative floats, with the quantiser's own float32 operations.
__global__ void k_scale_tables(float g, float* __restrict__ tab) {
  const int k = threadIdx.x;
  const float six_g = __fmul_rn(6.0f, g);
  if (k == 0) {
    tab[0] = 0.0f;
  } else if (k < 127) {
    uint32_t lo = 0, hi = 0x7F800000u;   // code(lo) < k <= code(hi)
    while (hi - lo > 1) {
      const uint32_t mid = lo + (hi - lo) / 2;
      const float a = __uint_as_float(mid);
      const int c = e4m3_code(six_g > 0.0f ? __fdiv_rn(a, six_g) : 0.0f);
      if (c >= k) hi = mid;
      else lo = mid;
    }
    tab[k] = __uint_as_float(hi);
  } else if (k == 127) {
    tab[127] = __uint_as_float(0x7F800000u);
  } else if (k < 255) {
    const float denom = __fmul_rn(e4m3_value(static_cast<uint8_t>(k - 128)), g);
    tab[k] = denom > 0.0f ? __fdiv_rn(1.0f, denom) : 0.0f;
  } else {
    tab[255] = six_g > 0.0f ? __fdiv_rn(1.0f, six_g) : 0.0f;
  }
}

cudaError_t launch_scale_tables(float g, float* tab, cudaStream_t st) {
  k_scale_tables<<<1, NVFP4_TAB, 0, st>>>(g, tab);
  return cudaGetLastError();
}

// Row quantiser with canonical outputs: codes [rows][cols/2], scales [rows][cols/16].
__global__ void __launch_bounds__(256) k_quant_rows(const float* __restrict__ x, int64_t rows,
                                                    int cols, float g, uint8_t* __restrict__ codes,
                                                    uint8_t* __restrict__ scales) {
  const int nb = cols / 16;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= rows * nb) return;
  const int64_t row = i / nb;
  const int blk = static_cast<int>(i - row * nb);
  float v[16];
  const float4* src = reinterpret_cast<const float4*>(x + row * cols + blk * 16);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 f = src[j];
    v[4 * j] = f.x;
    v[4 * j + 1] = f.y;
    v[4 * j + 2] = f.z;
    v[4 * j + 3] = f.w;
  }
  uint8_t q[8];
  scales[row * nb + blk] = nvfp4_block(v, g, q);
  *reinterpret_cast<uint2*>(codes + row * (cols / 2) + blk * 8) = *reinterpret_cast<const uint2*>(q);
}

cudaError_t launch_quant_rows(const float* x, int64_t rows, int cols, float g, uint8_t* codes,
                              uint8_t* scales, cudaStream_t st) {
  const int64_t n = rows * (cols / 16);
  if (n <= 0) return cudaSuccess;
  k_quant_rows<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(x, rows, cols, g, codes,
                                                                        scales);
  return cudaGetLastError();
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

// One thread per 16-element block: y = (1/4) H16 (s * x) as float32
// butterflies (stages 1, 2, 4, 8: (a, b) -> (a + b, a - b)).
__global__ void __launch_bounds__(256) k_rht16(const float* __restrict__ x, int64_t nblocks,
                                               uint64_t seed, float* __restrict__ y) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= nblocks) return;
  float b[16];
  const float4* src = reinterpret_cast<const float4*>(x + i * 16);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 f = src[j];
    b[4 * j] = f.x;
    b[4 * j + 1] = f.y;
    b[4 * j + 2] = f.z;
    b[4 * j + 3] = f.w;
  }
  rht16_block(b, seed);
  float4* dst = reinterpret_cast<float4*>(y + i * 16);
#pragma unroll
  for (int j = 0; j < 4; ++j) dst[j] = make_float4(b[4 * j], b[4 * j + 1], b[4 * j + 2], b[4 * j + 3]);
}

cudaError_t launch_rht16(const float* x, int64_t rows, int cols, uint64_t seed, float* y,
                         cudaStream_t st) {
  const int64_t n = rows * (cols / 16);
  if (n <= 0) return cudaSuccess;
  k_rht16<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(x, n, seed, y);
  return cudaGetLastError();
}

// NVFP4 rows with stochastically rounded elements: the block scale of the
// round-to-nearest quantiser (nvfp4_block's arithmetic), then e2m1_sr of
// f32(x * r) with the uniform of the element's counter.
__global__ void __launch_bounds__(256) k_quant_rows_sr(const float* __restrict__ x, int64_t rows,
                                                       int cols, float g, uint64_t seed,
                                                       uint8_t* __restrict__ codes,
                                                       uint8_t* __restrict__ scales) {
  const int nb = cols / 16;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= rows * nb) return;
  const int64_t row = i / nb;
  const int blk = static_cast<int>(i - row * nb);
  float v[16];
  const float4* src = reinterpret_cast<const float4*>(x + row * cols + blk * 16);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 f = src[j];
    v[4 * j] = f.x;
    v[4 * j + 1] = f.y;
    v[4 * j + 2] = f.z;
    v[4 * j + 3] = f.w;
  }
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
  const float six_g = __fmul_rn(6.0f, g);
  const float sbf = six_g > 0.0f ? __fdiv_rn(amax, six_g) : 0.0f;
  const uint8_t sc = e4m3_code(sbf);
  const float denom = __fmul_rn(e4m3_value(sc), g);
  const float r = denom > 0.0f ? __fdiv_rn(1.0f, denom) : 0.0f;
  const uint64_t c0 = static_cast<uint64_t>(row) * cols + blk * 16;
  uint8_t q[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t lo = e2m1_sr(__fmul_rn(v[2 * j], r), uniform24(seed, c0 + 2 * j));
    const uint32_t hi = e2m1_sr(__fmul_rn(v[2 * j + 1], r), uniform24(seed, c0 + 2 * j + 1));
    q[j] = static_cast<uint8_t>(lo | (hi << 4));
  }
  scales[row * nb + blk] = sc;
  *reinterpret_cast<uint2*>(codes + row * (cols / 2) + blk * 8) = *reinterpret_cast<const uint2*>(q);
}

cudaError_t launch_quant_rows_sr(const float* x, int64_t rows, int cols, float g, uint64_t seed,
                                 uint8_t* codes, uint8_t* scales, cudaStream_t st) {
  const int64_t n = rows * (cols / 16);
  if (n <= 0) return cudaSuccess;
  k_quant_rows_sr<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(x, rows, cols, g, seed,
                                                                           codes, scales);
  return cudaGetLastError();
}

// Quantised latent rows into expert order: codes u_q[tok] -> u_perm_q[r]
// (row pitch Kp/2 bytes) and the row's scales [tok][l/16] into the B-operand
// atoms of its token block: atom (block, kc), row j of the block.
__global__ void __launch_bounds__(256) k_gather_q(const uint8_t* __restrict__ uq,
                                                  const uint8_t* __restrict__ usf,
                                                  const int32_t* __restrict__ perm,
                                                  const int32_t* __restrict__ rblock, int64_t rows,
                                                  int K, int l, int lp,
                                                  uint8_t* __restrict__ u_perm_q,
                                                  uint8_t* __restrict__ atoms) {
  pdl_wait();
  pdl_trigger();
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  const int c16 = l / 32;   // 16-byte chunks of codes per row
  const int kc = l / 64;    // 64-element chunks (4 scales each)
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += nwarps) {
    const int64_t tok = perm[r] / K;
    const uint4* src = reinterpret_cast<const uint4*>(uq + tok * (l / 2));
    uint4* dst = reinterpret_cast<uint4*>(u_perm_q + r * (lp / 2));
    for (int i = lane; i < c16; i += 32) dst[i] = src[i];
    const int rb = rblock[r];
    const int b = rb >> 8, j = rb & 255;
    const uint32_t* ssrc = reinterpret_cast<const uint32_t*>(usf + tok * (l / 16));
    for (int c = lane; c < kc; c += 32) {
      const int64_t off = (static_cast<int64_t>(b) * (lp / 64) + c) * SF_ATOM_BYTES +
                          (j & 31) * 16 + ((j >> 5) & 3) * 4;
      *reinterpret_cast<uint32_t*>(atoms + off) = ssrc[c];
    }
  }
}

cudaError_t launch_gather_q(const uint8_t* uq, const uint8_t* usf, const int32_t* perm,
                            const int32_t* rblock, int64_t rows, int K, int l, int lp,
                            uint8_t* u_perm_q, uint8_t* atoms, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  int64_t blocks = (rows + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  return launch_pdl(k_gather_q, static_cast<unsigned>(blocks), 256, 0, st, uq, usf, perm, rblock,
                    rows, K, l, lp, u_perm_q, atoms);
}

}  // namespace lmoe
