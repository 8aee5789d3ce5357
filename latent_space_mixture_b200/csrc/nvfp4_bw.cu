// Non-GEMM kernels of the routed experts' backward pass under the NVFP4
// training recipe ("Nemotron-3 Super 精读报告", section 5.3: every linear
// layer's fprop, dgrad and wgrad GEMMs in NVFP4; weights with 2D block
// scales, so one 16 x 16 block's scale serves W and its transpose;
// activations and gradients with 1D blocks along each GEMM's reduction axis;
// a random Hadamard transform on the inputs of the weight-gradient GEMMs and
// stochastic rounding of the gradient tensors).
//
// Layouts.  Routed rows are in expert order (expert, then token, then slot).
// The weight-gradient GEMMs reduce over an expert's rows, so their operands
// are transposed: [features][columns], expert e's rows at columns
// [po256[e], po256[e] + c_e), each segment padded with zeros to a multiple
// of 256 (the FP4 MMA's K step).  The transform takes 16-column blocks from
// each segment's start.  A stochastically rounded element takes the counter
// of its place in the same layout padded to 16 instead, [po16[e] + j]: row f
// of a tensor of total 16-padded width W16 uses counters f W16 + col16.
// Global scales are amax / (6 * 448) over the whole tensor, from a device
// scalar that the producing kernels raise with atomicMax.
#include <cuda_bf16.h>

#include "kernels.h"
#include "launch.cuh"
#include "nvfp4.cuh"
#include "ptx.cuh"

namespace lmoe {

using bf16 = __nv_bfloat16;

// non-negative floats order like their bit patterns; the atomic only when the
// value would raise the current maximum (most warps' do not)
__device__ __forceinline__ void atomic_max_nonneg(float* p, float v) {
  if (__float_as_int(v) > *reinterpret_cast<volatile int*>(p))
    atomicMax(reinterpret_cast<int*>(p), __float_as_int(v));
}

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// global scale of a tensor from its amax: f32(amax / f32(6 * 448))
__device__ __forceinline__ float gscale_of(float amax) { return __fdiv_rn(amax, 2688.0f); }

// 16 scaled values -> 8 bytes of codes and the E4M3 scale code; stochastic
// rounding with counters c0 + i (SR), else round to nearest (nvfp4_block).
template <bool SR>
__device__ __forceinline__ uint8_t quant16(const float (&v)[16], float g, uint64_t seed,
                                           uint64_t c0, uint8_t (&q)[8]) {
  if constexpr (!SR) {
    return nvfp4_block(v, g, q);
  } else {
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
    if (amax == 0.0f) {
      // every element rounds to a zero of its own sign: no random bits needed
#pragma unroll
      for (int j = 0; j < 8; ++j)
        q[j] = static_cast<uint8_t>((signbit(v[2 * j]) ? 8u : 0u) |
                                    (signbit(v[2 * j + 1]) ? 128u : 0u));
      return 0;
    }
    const float six_g = __fmul_rn(6.0f, g);
    const float sbf = six_g > 0.0f ? __fdiv_rn(amax, six_g) : 0.0f;
    const uint8_t sc = e4m3_code(sbf);
    const float denom = __fmul_rn(e4m3_value(sc), g);
    const float r = denom > 0.0f ? __fdiv_rn(1.0f, denom) : 0.0f;
    // counters c0 .. c0 + 15: their states step by gamma
    uint64_t z = seed + (c0 + 1ull) * SPLITMIX_GAMMA;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t lo = e2m1_sr(__fmul_rn(v[2 * j], r), uniform24_z(z));
      z += SPLITMIX_GAMMA;
      const uint32_t hi = e2m1_sr(__fmul_rn(v[2 * j + 1], r), uniform24_z(z));
      z += SPLITMIX_GAMMA;
      q[j] = static_cast<uint8_t>(lo | (hi << 4));
    }
    return sc;
  }
}

// ---------------------------------------------------------------------------
// bf16 rows [rows][cols] -> NVFP4 codes (row pitch code_pitch bytes) and
// canonical scales [rows][cols/16], round to nearest, host global scale g.

__global__ void __launch_bounds__(256) k_quant_rows_bf16(const bf16* __restrict__ x, int64_t rows,
                                                         int cols, float g,
                                                         uint8_t* __restrict__ codes,
                                                         int code_pitch,
                                                         uint8_t* __restrict__ scales) {
  pdl_wait();
  pdl_trigger();
  const int nb = cols / 16;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= rows * nb) return;
  const int64_t row = i / nb;
  const int blk = static_cast<int>(i - row * nb);
  const uint4* src = reinterpret_cast<const uint4*>(x + row * cols + blk * 16);
  float v[16];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const uint4 raw = src[j];
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(p[k]);
      v[8 * j + 2 * k] = f.x;
      v[8 * j + 2 * k + 1] = f.y;
    }
  }
  uint8_t q[8];
  scales[row * nb + blk] = nvfp4_block(v, g, q);
  *reinterpret_cast<uint2*>(codes + row * code_pitch + blk * 8) = *reinterpret_cast<const uint2*>(q);
}

cudaError_t launch_quant_rows_bf16(const void* x, int64_t rows, int cols, float g, uint8_t* codes,
                                   int code_pitch, uint8_t* scales, cudaStream_t st) {
  const int64_t n = rows * (cols / 16);
  if (n <= 0) return cudaSuccess;
  return launch_pdl(k_quant_rows_bf16, static_cast<unsigned>((n + 255) / 256), 256, 0, st,
                    static_cast<const bf16*>(x), rows, cols, g, codes, code_pitch, scales);
}

// ---------------------------------------------------------------------------
// The output-gradient rows of the experts: out[r] = f32(w_r dv[token of r])
// ([R][l] fp32, rows in expert order), and their amax.  A warp per row.

__global__ void __launch_bounds__(256) k_rows_scaled(const bf16* __restrict__ dv,
                                                     const int32_t* __restrict__ perm,
                                                     const float* __restrict__ wrow, int64_t R,
                                                     int K, int l, float* __restrict__ out,
                                                     float* amax) {
  pdl_wait();
  pdl_trigger();
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= R) return;
  const int64_t tok = perm[r] / K;
  const float w = wrow[r];
  const uint4* src = reinterpret_cast<const uint4*>(dv + tok * l);
  float4* dst = reinterpret_cast<float4*>(out + r * l);
  float m = 0.0f;
  for (int c = lane; c < l / 8; c += 32) {
    const uint4 raw = src[c];
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
    float o[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(p[k]);
      o[2 * k] = __fmul_rn(w, f.x);
      o[2 * k + 1] = __fmul_rn(w, f.y);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(o[k]));
    dst[2 * c] = make_float4(o[0], o[1], o[2], o[3]);
    dst[2 * c + 1] = make_float4(o[4], o[5], o[6], o[7]);
  }
  m = warp_max_f(m);
  if (lane == 0) atomic_max_nonneg(amax, m);
}

cudaError_t launch_rows_scaled(const void* dv, const int32_t* perm, const float* wrow, int64_t R,
                               int K, int l, float* out, float* amax, cudaStream_t st) {
  if (R <= 0) return cudaSuccess;
  return launch_pdl(k_rows_scaled, static_cast<unsigned>((R + 7) / 8), 256, 0, st,
                    static_cast<const bf16*>(dv), perm, wrow, R, K, l, out, amax);
}

// ---------------------------------------------------------------------------
// fp32 rows [rows][cols] -> codes (row pitch code_pitch) and canonical scales
// [rows][cols/16] with the global scale of the tensor's amax (device), which
// is also written to *g_out; stochastic rounding with counter row * cols + col.

template <bool SR>
__global__ void __launch_bounds__(256) k_quant_rows_dev(const float* __restrict__ x, int64_t rows,
                                                        int cols, const float* amax, uint64_t seed,
                                                        uint8_t* __restrict__ codes,
                                                        int code_pitch,
                                                        uint8_t* __restrict__ scales,
                                                        float* g_out) {
  pdl_wait();
  pdl_trigger();
  const int nb = cols / 16;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const float g = gscale_of(*amax);
  if (i == 0) *g_out = g;
  if (i >= rows * nb) return;
  const int64_t row = i / nb;
  const int blk = static_cast<int>(i - row * nb);
  const float4* src = reinterpret_cast<const float4*>(x + row * cols + blk * 16);
  float v[16];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 f = src[j];
    v[4 * j] = f.x;
    v[4 * j + 1] = f.y;
    v[4 * j + 2] = f.z;
    v[4 * j + 3] = f.w;
  }
  uint8_t q[8];
  scales[row * nb + blk] =
      quant16<SR>(v, g, seed, static_cast<uint64_t>(row) * cols + blk * 16, q);
  *reinterpret_cast<uint2*>(codes + row * code_pitch + blk * 8) = *reinterpret_cast<const uint2*>(q);
}

cudaError_t launch_quant_rows_dev(const float* x, int64_t rows, int cols, const float* amax,
                                  bool sr, uint64_t seed, uint8_t* codes, int code_pitch,
                                  uint8_t* scales, float* g_out, cudaStream_t st) {
  const int64_t n = rows * (cols / 16);
  const unsigned blocks = static_cast<unsigned>(n > 0 ? (n + 255) / 256 : 1);
  return sr ? launch_pdl(k_quant_rows_dev<true>, blocks, 256, 0, st, x, rows, cols, amax, seed,
                         codes, code_pitch, scales, g_out)
            : launch_pdl(k_quant_rows_dev<false>, blocks, 256, 0, st, x, rows, cols, amax, seed,
                         codes, code_pitch, scales, g_out);
}

// ---------------------------------------------------------------------------
// Canonical scales of expert-order rows [R][nkb] -> the B-operand scale atoms
// of their token blocks ([block][kp64][512], rblock[r] = (block << 8) | row in
// block).  A thread per row and group of 4 scales (one 64-element chunk).

__global__ void __launch_bounds__(256) k_atoms_rblock(const uint8_t* __restrict__ scales,
                                                      const int32_t* __restrict__ rblock,
                                                      int64_t R, int nkb, int kp64,
                                                      uint8_t* __restrict__ atoms) {
  pdl_wait();
  pdl_trigger();
  const int ng = nkb / 4;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= R * ng) return;
  const int64_t r = i / ng;
  const int c = static_cast<int>(i - r * ng);
  const int rb = rblock[r];
  const int b = rb >> 8, j = rb & 255;
  const int64_t off = (static_cast<int64_t>(b) * kp64 + c) * SF_ATOM_BYTES + sf_atom_offset(j, 0);
  *reinterpret_cast<uint32_t*>(atoms + off) =
      *reinterpret_cast<const uint32_t*>(scales + r * nkb + 4 * c);
}

cudaError_t launch_atoms_rblock(const uint8_t* scales, const int32_t* rblock, int64_t R, int nkb,
                                int kp64, uint8_t* atoms, cudaStream_t st) {
  const int64_t n = R * (nkb / 4);
  if (n <= 0) return cudaSuccess;
  return launch_pdl(k_atoms_rblock, static_cast<unsigned>((n + 255) / 256), 256, 0, st, scales,
                    rblock, R, nkb, kp64, atoms);
}

// ---------------------------------------------------------------------------
// dL/dw of every routed (token, slot): dw[t][k] = o[inv[t][k]] . dv[t], o the
// experts' unweighted outputs (bf16 rows), fp32 in a fixed order (lane
// partial sums, then a butterfly).  A warp per (token, slot).

__global__ void __launch_bounds__(256) k_dw_rows(const bf16* __restrict__ O,
                                                 const int32_t* __restrict__ inv,
                                                 const bf16* __restrict__ dv, int64_t T, int K,
                                                 int l, float* __restrict__ dw) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (i >= T * K) return;
  const int64_t t = i / K;
  const uint4* a = reinterpret_cast<const uint4*>(O + static_cast<int64_t>(inv[i]) * l);
  const uint4* b = reinterpret_cast<const uint4*>(dv + t * l);
  float s = 0.0f;
  for (int c = lane; c < l / 8; c += 32) {
    const uint4 ra = a[c], rb = b[c];
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&ra);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&rb);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 fa = __bfloat1622float2(pa[k]), fb = __bfloat1622float2(pb[k]);
      s = fmaf(fa.x, fb.x, s);
      s = fmaf(fa.y, fb.y, s);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) dw[i] = s;
}

cudaError_t launch_dw_rows(const void* O, const int32_t* inv, const void* dv, int64_t T, int K,
                           int l, float* dw, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  return launch_pdl(k_dw_rows, static_cast<unsigned>((T * K + 7) / 8), 256, 0, st,
                    static_cast<const bf16*>(O), inv, static_cast<const bf16*>(dv), T, K, l, dw);
}

// ---------------------------------------------------------------------------
// Segment offsets of the transposed operands from the rows per expert:
// po16 / po256 [N + 1] (columns; each segment padded to 16 / 256), kofs
// [N + 1] = po256 / 256 (FP4 k-steps) and grp [po256[N] / 64], the expert of
// each 64-column group.  One CTA: thread 0 scans (N <= 1024), then thread e
// fills expert e's groups.

__global__ void __launch_bounds__(1024) k_seg_offsets(const int32_t* __restrict__ counts, int N,
                                                      int32_t* __restrict__ po16,
                                                      int32_t* __restrict__ po256,
                                                      int32_t* __restrict__ kofs,
                                                      int32_t* __restrict__ grp) {
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) {
    int32_t a = 0, b = 0;
    for (int e = 0; e < N; ++e) {
      po16[e] = a;
      po256[e] = b;
      kofs[e] = b / 256;
      a += (counts[e] + 15) / 16 * 16;
      b += (counts[e] + 255) / 256 * 256;
    }
    po16[N] = a;
    po256[N] = b;
    kofs[N] = b / 256;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < N; e += blockDim.x)
    for (int g = po256[e] / 64; g < po256[e + 1] / 64; ++g) grp[g] = e;
}

cudaError_t launch_seg_offsets(const int32_t* counts, int N, int32_t* po16, int32_t* po256,
                               int32_t* kofs, int32_t* grp, cudaStream_t st) {
  return launch_pdl(k_seg_offsets, 1, 1024, 0, st, counts, N, po16, po256, kofs, grp);
}

// ---------------------------------------------------------------------------
// Transposed, transformed, quantised operand of a weight-gradient GEMM, in
// two passes over its source and no intermediate tensor.  Element
// (f, po256[e] + j) is expert e's row j of feature f (zero past its c_e
// rows); each 16-column block goes through the random Hadamard transform of
// seed_rht.
//   pass 1 (STORE false): the transformed tensor's amax (atomicMax into
//          *amax);
//   pass 2 (STORE true): its NVFP4 codes [F][pitch / 2], canonical scales
//          [F][pitch / 16] and scale atoms [F / 128][pitch / 64][512] under
//          the global scale of *amax (also written to *g_out); stochastic
//          rounding (SR) with the counters of the 16-padded layout: element
//          (f, po256[e] + j) uses f W16 + po16[e] + j, W16 = po16[N] (the
//          padding past a segment's 16-row multiple is zero, which rounds to
//          zero whatever its counter).
// Sources (rows in expert order unless stated):
//   SRC 0: fp32 rows [R][F];
//   SRC 1: bf16 token rows [T][F], routed row r reading token perm[r] / K;
//   SRC 2: NVFP4 rows, codes [R][code_pitch] and B-operand scale atoms
//          ([block][Fp/64][512] by rblock), dequantised with global scale g.
// A CTA per (128 features, 64-column group): the group's source rows are
// staged in shared memory with coalesced loads, then two threads take one
// feature (a column of the tile), 32 columns each, so a thread's 16 bytes of
// codes and 2 scales are contiguous.  A 64-column group lies inside one segment (the segments are
// 256-aligned); groups past the layout's width (po256[N], on the device) do
// nothing.

// The CTA's source tile, rows [0, nr) x features [f0, f0 + 128) of its
// 64-row group, as floats in shared memory (rows read with coalesced vector
// loads; NVFP4 rows dequantised 8 codes at a time).
constexpr int TQ_PITCH = 129;
constexpr int TQ_THREADS = 256;   // two threads per feature, 32 columns each

// E2M1 code -> value with the eight magnitudes x 2 (0, 1, 2, 3, 4, 6, 8, 12)
// as the nibbles of one word: a shift, a mask and a conversion (the same
// values as e2m1_value, -0 for code 8 included)
__device__ __forceinline__ float e2m1_value_nib(uint32_t code) {
  const float m = static_cast<float>((0xC8643210u >> (4u * (code & 7u))) & 15u) * 0.5f;
  return (code & 8u) ? -m : m;
}

// One 64-column group of the CTA: its expert, first row of the segment in
// the group, rows with data (nr, may be <= 0).
struct TqGroup {
  int col0, e, j0, nr;
  int64_t rbase;
};

__device__ __forceinline__ TqGroup tq_group(int g, const int32_t* __restrict__ grp,
                                            const int32_t* __restrict__ offsets,
                                            const int32_t* __restrict__ counts,
                                            const int32_t* __restrict__ po256) {
  TqGroup q;
  q.col0 = g * 64;
  q.e = grp[g];
  q.j0 = q.col0 - po256[q.e];
  q.nr = min(64, counts[q.e] - q.j0);
  q.rbase = static_cast<int64_t>(offsets[q.e]) + q.j0;
  return q;
}

// The group's source rows x features [f0, f0 + 128) in flight in registers
// (issued a group ahead), then written to the shared tile as floats.
template <int SRC>
struct TqRegs;
template <>
struct TqRegs<0> {   // fp32 rows: 32 float4 per row, 8 per thread
  float4 x[8];
};
template <>
struct TqRegs<1> {   // bf16 token rows: 16 x 8 elements per row, 4 per thread
  uint4 raw[4];
};
template <>
struct TqRegs<2> {   // NVFP4 rows: 16 words of 8 codes per row, 4 per thread, and
  uint32_t w[4];     // (threads < 128) one word of 4 block scales (row t/2,
  uint32_t sc;       // 64-feature chunk t%2: adjacent in the row's atom)
};

template <int SRC>
__device__ __forceinline__ void tq_issue(TqRegs<SRC>& r, const TSrc& s, int64_t rbase, int nr,
                                         int f0, int F) {
  const int t = threadIdx.x;
  if constexpr (SRC == 0) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = t + TQ_THREADS * k, row = i >> 5, f = f0 + 4 * (i & 31);
      r.x[k] = (row < nr && f < F) ? *reinterpret_cast<const float4*>(
                                         static_cast<const float*>(s.p) + (rbase + row) * F + f)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else if constexpr (SRC == 1) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = t + TQ_THREADS * k, row = i >> 4, f = f0 + 8 * (i & 15);
      r.raw[k] = make_uint4(0u, 0u, 0u, 0u);
      if (row < nr && f < F) {
        const int64_t tok = s.perm[rbase + row] / s.K;
        r.raw[k] = *reinterpret_cast<const uint4*>(static_cast<const bf16*>(s.p) + tok * F + f);
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = t + TQ_THREADS * k, row = i >> 4, f = f0 + 8 * (i & 15);
      r.w[k] = (row < nr && f < F)
                   ? *reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(s.p) +
                                                        (rbase + row) * s.code_pitch + f / 2)
                   : 0u;
    }
    r.sc = 0u;
    if (t < 128) {
      const int row = t >> 1, f = f0 + 64 * (t & 1);
      if (row < nr && f < F) {
        const int rb = s.rblock[rbase + row];
        const int b = rb >> 8, j = rb & 255;
        r.sc = *reinterpret_cast<const uint32_t*>(
            s.atoms + (static_cast<int64_t>(b) * s.fp64 + f / 64) * SF_ATOM_BYTES +
            sf_atom_offset(j, 0));
      }
    }
  }
}

// nr is uniform over the CTA (the NVFP4 branch has a barrier inside)
template <int SRC>
__device__ __forceinline__ void tq_commit(const TqRegs<SRC>& r, const TSrc& s, int nr,
                                          float (*tile)[TQ_PITCH], uint32_t (*scw)[2]) {
  const int t = threadIdx.x;
  if constexpr (SRC == 0) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = t + TQ_THREADS * k, row = i >> 5, q = i & 31;
      if (row < nr) {
        tile[row][4 * q] = r.x[k].x;
        tile[row][4 * q + 1] = r.x[k].y;
        tile[row][4 * q + 2] = r.x[k].z;
        tile[row][4 * q + 3] = r.x[k].w;
      }
    }
  } else if constexpr (SRC == 1) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = t + TQ_THREADS * k, row = i >> 4, q = i & 15;
      if (row < nr) {
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&r.raw[k]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float2 v = __bfloat1622float2(p2[c]);
          tile[row][8 * q + 2 * c] = v.x;
          tile[row][8 * q + 2 * c + 1] = v.y;
        }
      }
    }
  } else {
    if (t < 128 && (t >> 1) < nr) scw[t >> 1][t & 1] = r.sc;
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = t + TQ_THREADS * k, row = i >> 4, q = i & 15;
      if (row < nr) {
        const uint32_t sc = (scw[row][q >> 3] >> (8 * ((q & 7) >> 1))) & 255u;
        const float scv = e4m3_value(static_cast<uint8_t>(sc));
#pragma unroll
        for (int c = 0; c < 8; ++c)   // (code x scale) x g, the dequantisation order
          tile[row][8 * q + c] =
              __fmul_rn(__fmul_rn(e2m1_value_nib((r.w[k] >> (4 * c)) & 15u), scv), s.g);
      }
    }
  }
}

// 64-column groups per CTA: the next group's loads are in flight while this
// one is transformed and quantised.  The stochastically rounding pass keeps
// one group per CTA: its random bits need registers, and those that would
// hold a group in flight would cost it occupancy.
template <bool SR>
struct TqGroups {
  static constexpr int value = SR ? 1 : 4;
};

template <int SRC, bool SR, bool STORE>
__global__ void __launch_bounds__(TQ_THREADS) k_tq(TSrc s, const int32_t* __restrict__ offsets,
                                                   const int32_t* __restrict__ counts,
                                                   const int32_t* __restrict__ po16,
                                                   const int32_t* __restrict__ po256,
                                                   const int32_t* __restrict__ grp, int N, int F,
                                                   int64_t pitch, uint64_t seed_rht, float* amax,
                                                   uint64_t seed_sr, uint8_t* __restrict__ codes,
                                                   uint8_t* __restrict__ scales,
                                                   uint8_t* __restrict__ atoms, float* g_out) {
  __shared__ float tile[64][TQ_PITCH];
  __shared__ uint32_t scw[64][2];
  pdl_wait();
  pdl_trigger();
  const int width = po256[N];
  constexpr int TQ_GROUPS = TqGroups<SR>::value;
  const int g0 = blockIdx.y * TQ_GROUPS;
  if (g0 * 64 >= width) return;
  const int f0 = blockIdx.x * 128;
  const int f = f0 + (threadIdx.x & 127);
  const int hv = threadIdx.x >> 7;   // this thread's 32 of a group's 64 columns
  const uint32_t signs = rht16_signs(seed_rht);
  float g = 0.0f;
  if constexpr (STORE) {
    g = gscale_of(*amax);
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *g_out = g;
  }
  const uint64_t w16 = SR ? static_cast<uint64_t>(po16[N]) : 0;
  float m = 0.0f;
  TqGroup cur = tq_group(g0, grp, offsets, counts, po256);
  TqRegs<SRC> regs;
  if (cur.nr > 0) tq_issue<SRC>(regs, s, cur.rbase, cur.nr, f0, F);
  for (int gi = 0; gi < TQ_GROUPS; ++gi) {
    __syncthreads();   // the previous group's transform has read the tile
    if (cur.nr > 0) tq_commit<SRC>(regs, s, cur.nr, tile, scw);
    __syncthreads();
    const bool more = gi + 1 < TQ_GROUPS && (g0 + gi + 1) * 64 < width;
    TqGroup nxt = cur;
    if (more) {
      nxt = tq_group(g0 + gi + 1, grp, offsets, counts, po256);
      if (nxt.nr > 0) tq_issue<SRC>(regs, s, nxt.rbase, nxt.nr, f0, F);
    }
    if (f < F) {
      uint32_t cw[4];
      uint32_t sw = 0;
#pragma unroll
      for (int b2 = 0; b2 < 2; ++b2) {
        const int bk = 2 * hv + b2;   // 16-column block of the group
        if (16 * bk >= cur.nr) {
          // past the segment's rows: zeros, scale 0
          cw[2 * b2] = cw[2 * b2 + 1] = 0u;
          continue;
        }
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          v[i] = (16 * bk + i < cur.nr) ? tile[16 * bk + i][threadIdx.x & 127] : 0.0f;
        rht16_masked(v, signs);
        if constexpr (!STORE) {
#pragma unroll
          for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
        } else {
          const uint64_t c0 =
              SR ? static_cast<uint64_t>(f) * w16 + po16[cur.e] + cur.j0 + 16 * bk : 0;
          uint8_t q[8];
          const uint8_t sc = quant16<SR>(v, g, seed_sr, c0, q);
          cw[2 * b2] = *reinterpret_cast<const uint32_t*>(q);
          cw[2 * b2 + 1] = *reinterpret_cast<const uint32_t*>(q + 4);
          sw |= static_cast<uint32_t>(sc) << (8 * b2);
        }
      }
      if constexpr (STORE) {
        const int c32 = cur.col0 + 32 * hv;
        *reinterpret_cast<uint4*>(codes + f * (pitch / 2) + c32 / 2) =
            make_uint4(cw[0], cw[1], cw[2], cw[3]);
        *reinterpret_cast<uint16_t*>(scales + f * (pitch / 16) + c32 / 16) =
            static_cast<uint16_t>(sw);
        *reinterpret_cast<uint16_t*>(
            atoms + ((static_cast<int64_t>(f) >> 7) * (pitch / 64) + cur.col0 / 64) * SF_ATOM_BYTES +
            sf_atom_offset(f & 127, 2 * hv)) = static_cast<uint16_t>(sw);
      }
    }
    if (!more) break;
    cur = nxt;
  }
  if constexpr (!STORE) {
    m = warp_max_f(m);
    if ((threadIdx.x & 31) == 0) atomic_max_nonneg(amax, m);
  }
}

template <int SRC, bool SR, bool STORE>
static cudaError_t launch_tq_v(const TSrc& s, const int32_t* offsets, const int32_t* counts,
                               const int32_t* po16, const int32_t* po256, const int32_t* grp,
                               int N, int F,
                               int64_t pitch, uint64_t seed_rht, float* amax, uint64_t seed_sr,
                               uint8_t* codes, uint8_t* scales, uint8_t* atoms, float* g_out,
                               cudaStream_t st) {
  const int64_t groups = pitch / 64;
  constexpr int per = TqGroups<SR>::value;
  const dim3 grid(static_cast<unsigned>((F + 127) / 128),
                  static_cast<unsigned>((groups + per - 1) / per));
  return launch_pdl(k_tq<SRC, SR, STORE>, grid, TQ_THREADS, 0, st, s, offsets, counts, po16,
                    po256, grp, N, F, pitch, seed_rht, amax, seed_sr, codes, scales, atoms, g_out);
}

cudaError_t launch_tq_amax(int src_kind, const TSrc& s, const int32_t* offsets,
                           const int32_t* counts, const int32_t* po16, const int32_t* po256,
                           const int32_t* grp, int N, int F, int64_t pitch, uint64_t seed_rht, float* amax,
                           cudaStream_t st) {
  switch (src_kind) {
    case 0: return launch_tq_v<0, false, false>(s, offsets, counts, po16, po256, grp, N, F, pitch,
                                                seed_rht, amax, 0, nullptr, nullptr, nullptr,
                                                nullptr, st);
    case 1: return launch_tq_v<1, false, false>(s, offsets, counts, po16, po256, grp, N, F, pitch,
                                                seed_rht, amax, 0, nullptr, nullptr, nullptr,
                                                nullptr, st);
    default: return launch_tq_v<2, false, false>(s, offsets, counts, po16, po256, grp, N, F, pitch,
                                                 seed_rht, amax, 0, nullptr, nullptr, nullptr,
                                                 nullptr, st);
  }
}

cudaError_t launch_tq_quant(int src_kind, bool sr, const TSrc& s, const int32_t* offsets,
                            const int32_t* counts, const int32_t* po16, const int32_t* po256,
                            const int32_t* grp, int N, int F, int64_t pitch, uint64_t seed_rht, float* amax,
                            uint64_t seed_sr, uint8_t* codes, uint8_t* scales, uint8_t* atoms,
                            float* g_out, cudaStream_t st) {
  // the recipe's four operands: gradients (SRC 0) stochastically rounded,
  // activations (SRC 1, 2) rounded to nearest
  if (src_kind == 0 && sr)
    return launch_tq_v<0, true, true>(s, offsets, counts, po16, po256, grp, N, F, pitch, seed_rht,
                                      amax, seed_sr, codes, scales, atoms, g_out, st);
  if (src_kind == 1 && !sr)
    return launch_tq_v<1, false, true>(s, offsets, counts, po16, po256, grp, N, F, pitch, seed_rht,
                                       amax, 0, codes, scales, atoms, g_out, st);
  if (src_kind == 2 && !sr)
    return launch_tq_v<2, false, true>(s, offsets, counts, po16, po256, grp, N, F, pitch, seed_rht,
                                       amax, 0, codes, scales, atoms, g_out, st);
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------
// Weight gradients of experts that no row chose: zero (the GEMM has no tiles
// for an empty K range).  grid.y = expert.

__global__ void __launch_bounds__(256) k_zero_empty(const int32_t* __restrict__ counts,
                                                    int64_t per, float* __restrict__ dw) {
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.y;
  if (counts[e] != 0) return;
  float4* p = reinterpret_cast<float4*>(dw + static_cast<int64_t>(e) * per);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < per / 4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

cudaError_t launch_zero_empty(const int32_t* counts, int N, int64_t per, float* dw,
                              cudaStream_t st) {
  return launch_pdl(k_zero_empty, dim3(16, static_cast<unsigned>(N)), 256, 0, st, counts, per, dw);
}

// ---------------------------------------------------------------------------
// The transposed copy of a 2D-block NVFP4 weight matrix, at layer creation:
// W [E][R][C] (codes [E*R][Cp/2], atoms [E*R/128][Cp/64][512]) -> W^T
// [E][C][R] (codes [E*C][Rp/2], atoms [E*C/128][Rp/64][512]).  A 16 x 16
// block's one scale serves both.  A thread per (expert, transposed row c,
// 16-element block b of W's rows); rows past R are zero.

__global__ void __launch_bounds__(256) k_transpose_w2d(const uint8_t* __restrict__ codes,
                                                       const uint8_t* __restrict__ atoms, int E,
                                                       int R, int C, int Cp, int Rp,
                                                       uint8_t* __restrict__ tcodes,
                                                       uint8_t* __restrict__ tatoms) {
  const int nb = Rp / 16;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(E) * C * nb) return;
  const int b = static_cast<int>(i % nb);
  const int64_t ec = i / nb;             // e * C + c
  const int e = static_cast<int>(ec / C);
  const int c = static_cast<int>(ec - static_cast<int64_t>(e) * C);
  uint8_t q[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  uint8_t sc = 0;
  if (16 * b < R) {
    const int64_t row0 = static_cast<int64_t>(e) * R + 16 * b;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const uint8_t byte = codes[(row0 + k) * (Cp / 2) + c / 2];
      const uint32_t nib = (c & 1) ? (byte >> 4) : (byte & 15);
      q[k / 2] |= static_cast<uint8_t>(nib << (4 * (k & 1)));
    }
    sc = atoms[((row0 >> 7) * (Cp / 64) + c / 64) * SF_ATOM_BYTES +
               sf_atom_offset(static_cast<int>(row0 & 127), (c & 63) >> 4)];
  }
  *reinterpret_cast<uint2*>(tcodes + ec * (Rp / 2) + 8 * b) = *reinterpret_cast<const uint2*>(q);
  tatoms[((ec >> 7) * (Rp / 64) + b / 4) * SF_ATOM_BYTES +
         sf_atom_offset(static_cast<int>(ec & 127), b & 3)] = sc;
}

cudaError_t launch_transpose_w2d(const uint8_t* codes, const uint8_t* atoms, int E, int R, int C,
                                 int Cp, int Rp, uint8_t* tcodes, uint8_t* tatoms,
                                 cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(E) * C * (Rp / 16);
  if (n <= 0) return cudaSuccess;
  k_transpose_w2d<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(codes, atoms, E, R, C,
                                                                          Cp, Rp, tcodes, tatoms);
  return cudaGetLastError();
}

}  // namespace lmoe
