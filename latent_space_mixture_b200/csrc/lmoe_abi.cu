// C ABI of the LatentMoE layer forward and backward passes (declarations and
// contracts in include/lmoe.h).  Host orchestration only: every step of the
// layer runs in the kernels of gemm_tc.cuh, gemm_pair.cuh, gemm_bw.cuh,
// routing.cu, nvfp4.cu and backward.cu.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "gemm_bw.cuh"
#include "gemm_pair.cuh"
#include "gemm_tc.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "lmoe.h"

using bf16 = __nv_bfloat16;

namespace lmoe {

// ---------------------------------------------------------------------------
// epilogues of the four contractions

// x -> [W_r; W_dn; W_s1] x: router logits (fp32), latent u (bf16) and the
// shared-expert hidden sqrelu(W_s1 x) (bf16, into columns [l, l+h_s) of vh).
// Features [0, N) are logits, [N, N+lu) u and the rest the shared hidden;
// lu = 0 for the standard MoE (no W_dn rows, u = x).
struct EpiX {
  static constexpr int kWarps = 4;
  float* logits;
  bf16* u;
  bf16* vh;
  int N, lu, l, ldvh;
  uint8_t* uq;    // NVFP4 experts: u codes [T][l/2] (nullptr for BF16 experts)
  uint8_t* usf;   //   and its E4M3 block scales [T][l/16]
  float g_u;      //   static global scale of u
  const float* tab_u;   //   its scale tables (nvfp4_scale_tab)
  uint8_t* u8;    // FP8 experts: u codes [T][l] (nullptr otherwise)
  float r_u8;     //   1 / s_u (rounded once)
  __half* u16;    // W4A16 experts: u in f16 [T][l] (nullptr otherwise)
  __device__ __forceinline__ void store8(const TileInfo&, long row, int feat, const float* v,
                                         bool valid) const {
    if (uq) {
      // every lane takes part in the 16-block pair exchange; only u lanes store
      uint8_t sc;
      const uint32_t codes = nvfp4_pair_tab(v, tab_u, &sc);
      if (valid && feat >= N && feat < N + lu) {
        const int f = feat - N;
        *reinterpret_cast<uint32_t*>(uq + row * (lu / 2) + f / 2) = codes;
        if ((f & 15) == 0) usf[row * (lu / 16) + f / 16] = sc;
      }
    }
    if (!valid) return;
    if (u8 && feat >= N && feat < N + lu) {
      uint8_t q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = e4m3_code(__fmul_rn(v[i], r_u8));
      *reinterpret_cast<uint2*>(u8 + row * lu + (feat - N)) = *reinterpret_cast<const uint2*>(q);
    }
    if (u16 && feat >= N && feat < N + lu) store8_f16(u16 + row * lu + (feat - N), v);
    if (feat < N) {
      float4* p = reinterpret_cast<float4*>(logits + row * N + feat);
      p[0] = make_float4(v[0], v[1], v[2], v[3]);
      p[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else if (feat < N + lu) {
      store8_bf16(u + row * lu + (feat - N), v);
    } else {
      float a[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = sqrelu(v[i]);
      store8_bf16(vh + row * ldvh + l + (feat - N - lu), a);
    }
  }
};

// shared expert FC1 alone (W_s1 x, on the side stream of an overlapped
// forward): sqrelu into columns [l, l + h_s) of vh
struct EpiS1 {
  static constexpr int kWarps = 4;
  bf16* vh;
  int l, ldvh;
  __device__ __forceinline__ void store8(const TileInfo&, long row, int feat, const float* v,
                                         bool valid) const {
    if (!valid) return;
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = sqrelu(v[i]);
    store8_bf16(vh + row * ldvh + l + feat, a);
  }
};

// expert FC1: H[row] = sqrelu(W1[e] u[row])
struct EpiH {
  static constexpr int kWarps = 4;
  bf16* H;
  int h;
  __device__ __forceinline__ void store8(const TileInfo&, long row, int feat, const float* v,
                                         bool valid) const {
    if (!valid) return;
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = sqrelu(v[i]);
    store8_bf16(H + row * h + feat, a);
  }
};

// expert FC2 times the router weight of the row: O[row] = w[row] W2[e] H[row]
struct EpiO {
  static constexpr int kWarps = 4;
  bf16* O;
  const float* wrow;
  int l;
  __device__ __forceinline__ void store8(const TileInfo&, long row, int feat, const float* v,
                                         bool valid) const {
    if (!valid) return;
    // no weights: an expert shard returns the unweighted outputs
    const float w = wrow ? wrow[row] : 1.0f;
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = v[i] * w;
    store8_bf16(O + row * l + feat, a);
  }
};

// [W_upl | W_s2] [v ; hs]: routed branch plus shared branch in one K loop.
// Standard MoE (no W_upl): the GEMM is W_s2 hs and the epilogue adds v
// (resid, row pitch ldr) before the store.
struct EpiY {
  static constexpr int kWarps = 4;
  bf16* y;
  int d;
  const bf16* resid;
  int ldr;
  float* yf = nullptr;             // fp32 output [T][d] instead of y (the side stream's W_s2 hs)
  const float* residf = nullptr;   // fp32 residual [T][d], added before y's one rounding
  __device__ __forceinline__ void store8(const TileInfo&, long row, int feat, const float* v,
                                         bool valid) const {
    if (!valid) return;
    if (yf) {
      float4* p = reinterpret_cast<float4*>(yf + row * d + feat);
      p[0] = make_float4(v[0], v[1], v[2], v[3]);
      p[1] = make_float4(v[4], v[5], v[6], v[7]);
      return;
    }
    if (residf) {
      const float4* p = reinterpret_cast<const float4*>(residf + row * d + feat);
      const float4 r0 = p[0], r1 = p[1];
      const float a[8] = {v[0] + r0.x, v[1] + r0.y, v[2] + r0.z, v[3] + r0.w,
                          v[4] + r1.x, v[5] + r1.y, v[6] + r1.z, v[7] + r1.w};
      store8_bf16(y + row * d + feat, a);
      return;
    }
    if (resid) {
      const uint4 raw = *reinterpret_cast<const uint4*>(resid + row * ldr + feat);
      const __nv_bfloat162* r2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
      float a[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(r2[i]);
        a[2 * i] = v[2 * i] + f.x;
        a[2 * i + 1] = v[2 * i + 1] + f.y;
      }
      store8_bf16(y + row * d + feat, a);
    } else {
      store8_bf16(y + row * d + feat, v);
    }
  }
};

// NVFP4 expert FC1: H = sqrelu(g_W1[e] g_u * acc), quantised with the static
// global scale g_h into codes [R][hp/2] and the B-operand scale atoms of the
// second grouped GEMM ([token block][hp/64][512 B], row = index in the block).
struct EpiHq {
  // epilogue warps at >= 128-row token blocks: quantising H is ~9x the FP4 MMAs
  static constexpr int kWarps = 16;
  static constexpr int kVec = 16;   // a whole 16-element NVFP4 block per lane
  uint8_t* Hq;
  uint8_t* sfh;
  const float* gw1;
  float g_u, g_h;
  int hp;   // h rounded up to 256 (row pitch hp/2 bytes)
  const float* tab_h;    // scale tables of g_h (nvfp4_scale_tab)
  bf16* a16 = nullptr;   // NVFP4 training: the pre-activation a = W1[e] u, bf16 [R][ha]
  int ha = 0;
  static constexpr bool kTokMajor = true;
  // 32 consecutive features of one token row (token-major accumulators): two
  // NVFP4 blocks, 16 bytes of codes and two adjacent scale bytes
  __device__ __forceinline__ void store32(const TileInfo& t, long row, int feat, const float* v,
                                          bool valid) const {
    if (!valid) return;
    const float s = __fmul_rn(gw1[t.e], g_u);
    float a[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) a[i] = sqrelu(v[i] * s);
    uint32_t w[4];
    uint8_t sc[2];
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmaxf(amax, a[16 * b + i]);   // a >= 0
      float r;
      sc[b] = nvfp4_scale_tab(amax, tab_h, &r);
      w[2 * b] = e2m1x8(a + 16 * b, r);
      w[2 * b + 1] = e2m1x8(a + 16 * b + 8, r);
    }
    *reinterpret_cast<uint4*>(Hq + row * (hp / 2) + feat / 2) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint16_t*>(
        sfh + (static_cast<long>(t.tb) * (hp / 64) + feat / 64) * SF_ATOM_BYTES +
        sf_atom_offset(static_cast<int>(row - t.row0), (feat & 63) >> 4)) =
        static_cast<uint16_t>(sc[0] | (sc[1] << 8));
    if (a16) {
      float pre[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) pre[i] = v[i] * s;
#pragma unroll
      for (int i = 0; i < 4; ++i) store8_bf16(a16 + row * ha + feat + 8 * i, pre + 8 * i);
    }
  }
  __device__ __forceinline__ void store8(const TileInfo& t, long row, int feat, const float* v,
                                         bool valid) const {
    const float s = __fmul_rn(gw1[t.e], g_u);
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = sqrelu(v[i] * s);
    uint8_t sc;
    const uint32_t codes = nvfp4_pair_tab(a, tab_h, &sc);
    if (!valid) return;
    if (a16) {
      float pre[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) pre[i] = v[i] * s;
      store8_bf16(a16 + row * ha + feat, pre);
    }
    *reinterpret_cast<uint32_t*>(Hq + row * (hp / 2) + feat / 2) = codes;
    if ((feat & 15) == 0)
      sfh[(static_cast<long>(t.tb) * (hp / 64) + feat / 64) * SF_ATOM_BYTES +
          sf_atom_offset(static_cast<int>(row - t.row0), (feat & 63) >> 4)] = sc;
  }
  // one 16-element block of a row: the block's scale from the tables of g_h,
  // no lane exchange (the same codes as store8)
  __device__ __forceinline__ void store16(const TileInfo& t, long row, int feat, const float* v,
                                          bool valid) const {
    if (!valid) return;
    const float s = __fmul_rn(gw1[t.e], g_u);
    float a[16];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      a[i] = sqrelu(v[i] * s);
      amax = fmaxf(amax, fabsf(a[i]));
    }
    float r;
    const uint8_t sc = nvfp4_scale_tab(amax, tab_h, &r);
    uint32_t w0 = 0, w1 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      w0 |= e2m1x2(__fmul_rn(a[2 * i], r), __fmul_rn(a[2 * i + 1], r)) << (8 * i);
      w1 |= e2m1x2(__fmul_rn(a[8 + 2 * i], r), __fmul_rn(a[8 + 2 * i + 1], r)) << (8 * i);
    }
    *reinterpret_cast<uint2*>(Hq + row * (hp / 2) + feat / 2) = make_uint2(w0, w1);
    sfh[(static_cast<long>(t.tb) * (hp / 64) + feat / 64) * SF_ATOM_BYTES +
        sf_atom_offset(static_cast<int>(row - t.row0), (feat & 63) >> 4)] = sc;
    if (a16) {
      float pre[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) pre[i] = v[i] * s;
      store8_bf16(a16 + row * ha + feat, pre);
      store8_bf16(a16 + row * ha + feat + 8, pre + 8);
    }
  }
};

// NVFP4 expert FC2 times the router weight: O = w g_W2[e] g_h * acc (bf16)
struct EpiOq {
  // epilogue warps at >= 128-row token blocks
  static constexpr int kWarps = 8;
  bf16* O;
  const float* wrow;
  const float* gw2;
  float g_h;
  int l;
  static constexpr bool kTokMajor = true;
  __device__ __forceinline__ void store32(const TileInfo& t, long row, int feat, const float* v,
                                          bool valid) const {
    if (!valid) return;
    const float s = __fmul_rn(__fmul_rn(gw2[t.e], g_h), wrow ? wrow[row] : 1.0f);
    float a[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) a[i] = v[i] * s;
#pragma unroll
    for (int i = 0; i < 4; ++i) store8_bf16(O + row * l + feat + 8 * i, a + 8 * i);
  }
  __device__ __forceinline__ void store8(const TileInfo& t, long row, int feat, const float* v,
                                         bool valid) const {
    if (!valid) return;
    // no weights: the experts' unweighted outputs (the NVFP4 backward's o)
    const float s = __fmul_rn(__fmul_rn(gw2[t.e], g_h), wrow ? wrow[row] : 1.0f);
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = v[i] * s;
    store8_bf16(O + row * l + feat, a);
  }
};

// NVFP4 backward, data gradient of FC2: dg = g_W2[e] g_do * acc (the FP4
// product W2q^T Q(do)), and the pre-activation gradient da = dg 2 max(a, 0)
// in fp32 [R][h], with its amax (a warp maximum, then one atomic per warp).
struct EpiDA {
  static constexpr int kWarps = 8;
  float* da;
  const bf16* a16;
  const float* gw2;
  const float* g_do;   // device scalar
  int h;
  float* amax;
  static constexpr bool kTokMajor = true;
  static constexpr bool kPre32 = true;
  // the chunk's 32 saved pre-activations, loaded before the accumulator wait
  __device__ __forceinline__ void pre32(const TileInfo&, long row, int feat, bool valid,
                                        uint4 (&p)[4]) const {
    const uint4* ap = reinterpret_cast<const uint4*>(a16 + row * h + feat);
#pragma unroll
    for (int c = 0; c < 4; ++c) p[c] = valid ? ap[c] : make_uint4(0u, 0u, 0u, 0u);
  }
  __device__ __forceinline__ void store32(const TileInfo& t, long row, int feat, const float* v,
                                          bool valid, const uint4 (&pa)[4]) const {
    float m = 0.0f;
    if (valid) {
      const float s = __fmul_rn(gw2[t.e], *g_do);
      float4* p = reinterpret_cast<float4*>(da + row * h + feat);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 raw = pa[c];
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
        float o[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 a = __bfloat1622float2(a2[i]);
          o[2 * i] = __fmul_rn(__fmul_rn(v[8 * c + 2 * i] * s, 2.0f), fmaxf(a.x, 0.0f));
          o[2 * i + 1] = __fmul_rn(__fmul_rn(v[8 * c + 2 * i + 1] * s, 2.0f), fmaxf(a.y, 0.0f));
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(o[i]));
        p[2 * c] = make_float4(o[0], o[1], o[2], o[3]);
        p[2 * c + 1] = make_float4(o[4], o[5], o[6], o[7]);
      }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0 && __float_as_int(m) > *reinterpret_cast<volatile int*>(amax))
      atomicMax(reinterpret_cast<int*>(amax), __float_as_int(m));
  }
  __device__ __forceinline__ void store8(const TileInfo& t, long row, int feat, const float* v,
                                         bool valid) const {
    float m = 0.0f;
    if (valid) {
      const float s = __fmul_rn(gw2[t.e], *g_do);
      const uint4 raw = *reinterpret_cast<const uint4*>(a16 + row * h + feat);
      const __nv_bfloat162* ap = reinterpret_cast<const __nv_bfloat162*>(&raw);
      float o[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 a = __bfloat1622float2(ap[i]);
        o[2 * i] = __fmul_rn(__fmul_rn(v[2 * i] * s, 2.0f), fmaxf(a.x, 0.0f));
        o[2 * i + 1] = __fmul_rn(__fmul_rn(v[2 * i + 1] * s, 2.0f), fmaxf(a.y, 0.0f));
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(o[i]));
      float4* p = reinterpret_cast<float4*>(da + row * h + feat);
      p[0] = make_float4(o[0], o[1], o[2], o[3]);
      p[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    // the atomic only when it would raise the maximum
    if ((threadIdx.x & 31) == 0 && __float_as_int(m) > *reinterpret_cast<volatile int*>(amax))
      atomicMax(reinterpret_cast<int*>(amax), __float_as_int(m));
  }
};

// NVFP4 backward, data gradient of FC1: du rows = g_W1[e] g_da * acc (bf16)
struct EpiDU {
  static constexpr int kWarps = 8;
  bf16* du;
  const float* gw1;
  const float* g_da;   // device scalar
  int l;
  static constexpr bool kTokMajor = true;
  __device__ __forceinline__ void store32(const TileInfo& t, long row, int feat, const float* v,
                                          bool valid) const {
    if (!valid) return;
    const float s = __fmul_rn(gw1[t.e], *g_da);
    float o[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i] = v[i] * s;
#pragma unroll
    for (int i = 0; i < 4; ++i) store8_bf16(du + row * l + feat + 8 * i, o + 8 * i);
  }
  __device__ __forceinline__ void store8(const TileInfo& t, long row, int feat, const float* v,
                                         bool valid) const {
    if (!valid) return;
    const float s = __fmul_rn(gw1[t.e], *g_da);
    float o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = v[i] * s;
    store8_bf16(du + row * l + feat, o);
  }
};

// NVFP4 weight gradient of one expert (group): out[e][row][feat] =
// g_a g_b * acc, fp32, row = B row, feat = A row; stored by TMA through the
// map m of out ([E * rows][cols] fp32, 32 x 32 boxes, 128-byte swizzle).
struct EpiWq {
  static constexpr int kWarps = 8;
  float* out;
  int rows, cols;
  const float* g_a;   // device scalars
  const float* g_b;
  CUtensorMap m;
  static constexpr bool kTokMajor = true;
  static constexpr bool kTmaBoxes = true;
  __device__ __forceinline__ float scale(const TileInfo&) const { return __fmul_rn(*g_a, *g_b); }
  __device__ __forceinline__ void target(const TileInfo& t, long row, int feat,
                                         const CUtensorMap** mp, int* x, int* y) const {
    *mp = &m;
    *x = feat;
    *y = t.e * rows + static_cast<int>(row);
  }
  __device__ __forceinline__ void store8(const TileInfo& t, long row, int feat, const float* v,
                                         bool valid) const {
    if (!valid) return;
    const float s = __fmul_rn(*g_a, *g_b);
    float4* p = reinterpret_cast<float4*>(out + (static_cast<long>(t.e) * rows + row) * cols + feat);
    p[0] = make_float4(v[0] * s, v[1] * s, v[2] * s, v[3] * s);
    p[1] = make_float4(v[4] * s, v[5] * s, v[6] * s, v[7] * s);
  }
};

// FP8 expert FC1: H = E4M3(sqrelu(s_W1[e] s_u * acc) / s_h), codes [R][h]
struct EpiH8 {
  // epilogue warps at >= 128-row token blocks
  static constexpr int kWarps = 8;
  uint8_t* H8;
  const float* sw1;
  float s_u, r_h;
  int h;
  __device__ __forceinline__ void store8(const TileInfo& t, long row, int feat, const float* v,
                                         bool valid) const {
    if (!valid) return;
    const float s = __fmul_rn(sw1[t.e], s_u);
    uint8_t q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = e4m3_code(__fmul_rn(sqrelu(v[i] * s), r_h));
    *reinterpret_cast<uint2*>(H8 + row * h + feat) = *reinterpret_cast<const uint2*>(q);
  }
};

// FP8 expert FC2: O = w * s_W2[e] s_h * acc
struct EpiO8 {
  // epilogue warps at >= 128-row token blocks
  static constexpr int kWarps = 8;
  bf16* O;
  const float* wrow;
  const float* sw2;
  float s_h;
  int l;
  __device__ __forceinline__ void store8(const TileInfo& t, long row, int feat, const float* v,
                                         bool valid) const {
    if (!valid) return;
    const float s = __fmul_rn(__fmul_rn(sw2[t.e], s_h), wrow[row]);
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = v[i] * s;
    store8_bf16(O + row * l + feat, a);
  }
};

// W4A16 expert FC1: H = sqrelu(g_W1[e] * acc) in f16 (the MMA summed the
// FP4 codes times their block scales; the global scale comes here)
struct EpiH16 {
  static constexpr int kWarps = 4;
  __half* H16;
  const float* gw1;
  int h;
  __device__ __forceinline__ void store8(const TileInfo& t, long row, int feat, const float* v,
                                         bool valid) const {
    if (!valid) return;
    const float g = gw1[t.e];
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = sqrelu(v[i] * g);
    store8_f16(H16 + row * h + feat, a);
  }
};

// W4A16 expert FC2: O = w * g_W2[e] * acc
struct EpiO16 {
  static constexpr int kWarps = 4;
  bf16* O;
  const float* wrow;
  const float* gw2;
  int l;
  __device__ __forceinline__ void store8(const TileInfo& t, long row, int feat, const float* v,
                                         bool valid) const {
    if (!valid) return;
    const float s = __fmul_rn(gw2[t.e], wrow[row]);
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = v[i] * s;
    store8_bf16(O + row * l + feat, a);
  }
};

// ---------------------------------------------------------------------------
// epilogues of the backward contractions (gemm_bw.cuh; rows are tokens or
// routed rows for the data gradients, rows of dW for the weight gradients)

// dy -> dy [W_upl | W_s2]: dv (bf16, [T][l]) and the gradient of the shared
// hidden pre-activation, (dy W_s2) * 2 max(a, 0) with max(a, 0) =
// sqrt(sqrelu(a)) from the forward's hs (columns [l, l+h_s) of vh), into
// columns [N+l, N+l+h_s) of dxh.
struct EpiDVH {
  static constexpr bool kAux = true;   // reads hs
  static constexpr bool kTma = false;
  bf16* dv;
  bf16* dxh;
  const bf16* vh;
  int l, ldvh, ldx, N;
  __device__ __forceinline__ uint4 fetch(long row, int feat, bool valid) const {
    if (!valid || feat < l) return make_uint4(0u, 0u, 0u, 0u);
    return *reinterpret_cast<const uint4*>(vh + row * ldvh + feat);
  }
  __device__ __forceinline__ void store8(const BwTile&, long row, int feat, const float* v,
                                         bool valid, const uint4 raw) const {
    if (!valid) return;
    if (feat < l) {
      store8_bf16(dv + row * l + feat, v);
      return;
    }
    const __nv_bfloat162* hp = reinterpret_cast<const __nv_bfloat162*>(&raw);
    float a[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 g = __bfloat1622float2(hp[i]);
      a[2 * i] = v[2 * i] * (2.0f * sqrtf(g.x));
      a[2 * i + 1] = v[2 * i + 1] * (2.0f * sqrtf(g.y));
    }
    store8_bf16(dxh + row * ldx + N + feat, a);
  }
};

// plain bf16 store of the product (du rows in expert order; dx)
struct EpiStore {
  static constexpr bool kAux = false;
  static constexpr bool kTma = false;
  bf16* out;
  int ld;
  __device__ __forceinline__ void store8(const BwTile&, long row, int feat, const float* v,
                                         bool valid) const {
    if (valid) store8_bf16(out + row * ld + feat, v);
  }
};

// Weight gradients (fp32) leave through TMA stores of 32 x 32 boxes: target()
// names the tensor map and the box coordinates of the chunk of 32 dW rows
// starting at `row` and the 32 features starting at `feat`.

// d[W_r; W_dn; W_s1] = dxh^T x: rows [0, r1) to m0, [r1, r2) to m1, the rest
// to m2 (maps of [rows][d] fp32; r1, r2 multiples of 32)
struct EpiWRows {
  static constexpr bool kAux = false;
  static constexpr bool kTma = true;
  CUtensorMap m0, m1, m2;
  int r1, r2;
  __device__ __forceinline__ void target(const BwTile&, long row, int feat, const CUtensorMap** m,
                                         int* x, int* y) const {
    *x = feat;
    if (row < r1) {
      *m = &m0;
      *y = static_cast<int>(row);
    } else if (row < r2) {
      *m = &m1;
      *y = static_cast<int>(row - r1);
    } else {
      *m = &m2;
      *y = static_cast<int>(row - r2);
    }
  }
};

// d[W_upl | W_s2] = dy^T [v | hs]: features [0, c1) to m0 ([d][l]), the rest
// to m1 ([d][h_s]); c1 a multiple of 32
struct EpiWCols {
  static constexpr bool kAux = false;
  static constexpr bool kTma = true;
  CUtensorMap m0, m1;
  int c1;
  __device__ __forceinline__ void target(const BwTile&, long row, int feat, const CUtensorMap** m,
                                         int* x, int* y) const {
    *y = static_cast<int>(row);
    if (feat < c1) {
      *m = &m0;
      *x = feat;
    } else {
      *m = &m1;
      *x = feat - c1;
    }
  }
};

// per-expert weight gradient dW[e] ([E * rows_per][cols] fp32)
struct EpiWExp {
  static constexpr bool kAux = false;
  static constexpr bool kTma = true;
  CUtensorMap m;
  int rows_per;
  __device__ __forceinline__ void target(const BwTile& t, long row, int feat, const CUtensorMap** mp,
                                         int* x, int* y) const {
    *mp = &m;
    *x = feat;
    *y = t.e * rows_per + static_cast<int>(row);
  }
};

template <int BN>
struct BwStages {
  static constexpr int value = BN == 256 ? 4 : BN == 128 ? 6 : 10;
};

template <int BN, bool B_MN, class Epi>
cudaError_t set_bw_smem() {
  constexpr int S = BwStages<BN>::value;
  return cudaFuncSetAttribute(k_gemm_bw<BN, S, B_MN, Epi>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              BwLayout<BN, S, B_MN, Epi::kTma>::SMEM_BYTES);
}

template <int BN, bool B_MN, class Epi>
cudaError_t launch_bw(const CUtensorMap& A, const CUtensorMap& B16, const CUtensorMap& B64,
                      const BwSource& src, const Epi& epi, int grid, int* err,
                      unsigned long long limit, cudaStream_t st) {
  constexpr int S = BwStages<BN>::value;
  return launch_pdl(k_gemm_bw<BN, S, B_MN, Epi>, grid, GEMM_THREADS,
                    BwLayout<BN, S, B_MN, Epi::kTma>::SMEM_BYTES, st, A, B16, B64, src, epi, err,
                    limit);
}

// data-gradient GEMM with a K-major token-row B operand of BN rows per block
template <class Epi>
cudaError_t launch_bw_dgrad(int bn, const CUtensorMap& A, const CUtensorMap& B16,
                            const CUtensorMap& B64, const BwSource& src, const Epi& epi, int grid,
                            int* err, unsigned long long limit, cudaStream_t st) {
  switch (bn) {
    case 256: return launch_bw<256, false>(A, B16, B64, src, epi, grid, err, limit, st);
    case 128: return launch_bw<128, false>(A, B16, B64, src, epi, grid, err, limit, st);
    default: return launch_bw<32, false>(A, B16, B64, src, epi, grid, err, limit, st);
  }
}

template <class Epi>
cudaError_t set_bw_dgrad_smem() {
  cudaError_t e;
  if ((e = set_bw_smem<256, false, Epi>()) != cudaSuccess) return e;
  if ((e = set_bw_smem<128, false, Epi>()) != cudaSuccess) return e;
  return set_bw_smem<32, false, Epi>();
}

// token-block width of the dense data-gradient GEMMs
static int bw_dense_bn(int64_t T) { return T >= 2048 ? 256 : T >= 512 ? 128 : 32; }

// GEMM variants: (BN, operand kind) -> pipeline stages (FP8 stages hold
// 128-byte rows like bf16 ones)
template <int BN, int KIND>
struct Stages {
  static constexpr int value = BN == 256 ? 4 : BN == 128 ? 6 : 10;
};
template <>
struct Stages<128, KIND_NVFP4> {
  static constexpr int value = 6;
};
template <>
struct Stages<32, KIND_NVFP4> {
  static constexpr int value = 8;
};
// W4A16 stages hold two K sub-tiles plus the raw FP4 codes and scale atoms
template <>
struct Stages<128, KIND_W4A16> {
  static constexpr int value = 2;
};
template <>
struct Stages<32, KIND_W4A16> {
  static constexpr int value = 4;
};

// the ring depth of a variant: its default, or what fits beside the staging
// of a wider epilogue
template <int BN, class Epi, int KIND>
struct StagesOf {
  static constexpr int EPIW = GemmEpiWarps<BN, Epi>::value;
  static constexpr int STG = GemmStg<BN, Epi, KIND>::value;
  static constexpr int value = gemm_fit_stages<BN, KIND, EPIW, STG>(Stages<BN, KIND>::value);
  using L = GemmLayout<BN, value, KIND, EPIW, STG>;
};

template <int BN, class Epi, int KIND = KIND_BF16>
cudaError_t set_gemm_smem() {
  using S = StagesOf<BN, Epi, KIND>;
  return cudaFuncSetAttribute(k_gemm_tc<BN, S::value, Epi, KIND>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, S::L::SMEM_BYTES);
}

// B operand: the same matrix under two tensor maps (16-row and 64-row boxes)
struct BMaps {
  CUtensorMap b16, b64;
};

template <int BN, class Epi, int KIND = KIND_BF16>
cudaError_t launch_gemm(const CUtensorMap& A, const BMaps& B, const TileSource& src,
                        const Epi& epi, int grid, int* err, unsigned long long limit,
                        cudaStream_t st) {
  using S = StagesOf<BN, Epi, KIND>;
  return launch_pdl(k_gemm_tc<BN, S::value, Epi, KIND>, grid, S::L::THREADS, S::L::SMEM_BYTES, st,
                    A, B.b16, B.b64, src, epi, err, limit);
}

// CTA-pair variant: 256 x 256 tiles, 3 stages of K = 128 (64 KB per CTA)
constexpr int PAIR_BN = 256;
constexpr int PAIR_STAGES = 3;
constexpr int PAIR_KSUB = 2;

template <class Epi>
cudaError_t set_pair_smem() {
  return cudaFuncSetAttribute(k_gemm_pair<PAIR_BN, PAIR_STAGES, PAIR_KSUB, Epi>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              PairLayout<PAIR_BN, PAIR_STAGES, PAIR_KSUB>::SMEM_BYTES);
}

template <class Epi>
cudaError_t launch_gemm_pair(const CUtensorMap& A, const BMaps& B, const TileSource& src,
                             const Epi& epi, int npairs, int* err, unsigned long long limit,
                             cudaStream_t st) {
  return launch_pair_pdl(k_gemm_pair<PAIR_BN, PAIR_STAGES, PAIR_KSUB, Epi>, 2 * npairs,
                         GEMM_THREADS, PairLayout<PAIR_BN, PAIR_STAGES, PAIR_KSUB>::SMEM_BYTES, st,
                         A, B.b16, B.b64, src, epi, err, limit);
}

template <int KIND, class Epi>
cudaError_t launch_gemm_q(int bn, const CUtensorMap& A, const BMaps& B, const TileSource& src,
                          const Epi& epi, int grid, int* err, unsigned long long limit,
                          cudaStream_t st) {
  if constexpr (KIND == KIND_FP8)
    if (bn == 256) return launch_gemm<256, Epi, KIND>(A, B, src, epi, grid, err, limit, st);
  if (bn == 128) return launch_gemm<128, Epi, KIND>(A, B, src, epi, grid, err, limit, st);
  return launch_gemm<32, Epi, KIND>(A, B, src, epi, grid, err, limit, st);
}

template <class Epi>
cudaError_t launch_gemm_bn(int bn, const CUtensorMap& A, const BMaps& B, const TileSource& src,
                           const Epi& epi, int grid, int* err, unsigned long long limit,
                           cudaStream_t st) {
  switch (bn) {
    case 256: return launch_gemm<256>(A, B, src, epi, grid, err, limit, st);
    case 128: return launch_gemm<128>(A, B, src, epi, grid, err, limit, st);
    default: return launch_gemm<32>(A, B, src, epi, grid, err, limit, st);
  }
}

template <class Epi>
cudaError_t launch_reduce(const float* part, int ksplit, int T, int F, const Epi& epi,
                          cudaStream_t st) {
  const long threads = static_cast<long>(T) * (F / 8);
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  return launch_pdl(k_splitk_reduce<Epi>, blocks, 256, 0, st, part, ksplit, T, F, epi);
}

// the x-GEMM's split-K reduction with the router's top-K fused (N <= 1024)
template <class Epi>
cudaError_t launch_reduce_route(const float* part, int ksplit, int T, int F, int N,
                                const Epi& epi, const float* bias, int K, float* logits,
                                int32_t* topk_idx, float* topk_w, cudaStream_t st) {
  const int rblocks = (T + 7) / 8;
  const long threads = static_cast<long>(T) * ((F - N) / 8);
  const unsigned blocks = static_cast<unsigned>(rblocks + (threads + 255) / 256);
  if (N <= 32 * 4)
    return launch_pdl(k_splitk_reduce_route<Epi, 4>, blocks, 256, 0, st, part, ksplit, T, F, N,
                      epi, bias, K, logits, topk_idx, topk_w, rblocks);
  if (N <= 32 * 16)
    return launch_pdl(k_splitk_reduce_route<Epi, 16>, blocks, 256, 0, st, part, ksplit, T, F, N,
                      epi, bias, K, logits, topk_idx, topk_w, rblocks);
  return launch_pdl(k_splitk_reduce_route<Epi, 32>, blocks, 256, 0, st, part, ksplit, T, F, N,
                    epi, bias, K, logits, topk_idx, topk_w, rblocks);
}

template <class Epi>
cudaError_t set_smem_all() {
  cudaError_t e;
  if ((e = set_gemm_smem<256, Epi>()) != cudaSuccess) return e;
  if ((e = set_gemm_smem<128, Epi>()) != cudaSuccess) return e;
  return set_gemm_smem<32, Epi>();
}

// ---------------------------------------------------------------------------
// tensor maps (driver entry point fetched through the runtime)

typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode() {
  static PFN_encodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  });
  return fn;
}

// 2-D bf16 row-major [rows][cols] matrix, box of 64 columns x box_rows rows,
// 128-byte swizzle; out-of-range rows read as zero.
static bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                     uint32_t box_rows) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// as make_map, for a [rows][cols] window of a matrix whose rows are `pitch`
// elements apart
static bool make_map_strided(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                             uint64_t pitch, uint32_t box_rows) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D byte matrix [rows][cols] of packed FP4 codes read as (32 x W4_KSUB)-byte
// x 128-row tiles without swizzle (the W4A16 converter reads them row by row)
static bool make_map_codes(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {32 * W4_KSUB, GEMM_BM};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D byte matrix [rows][cols] (packed NVFP4 codes), box of 128 bytes x
// box_rows rows, 128-byte swizzle.
static bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                        uint32_t box_rows) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 row-major [rows][cols] matrix written by TMA stores of 32 x 32
// boxes, no swizzle (cols * 4 a multiple of 16 bytes); out-of-range elements
// of a box are not written.
// fp32 [rows][cols] output map with 32 x 32 boxes stored from 128-byte-swizzled
// shared memory (the token-major epilogues' boxes)
static bool make_map_f32_out_sw(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 4};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool make_map_f32_out(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 4};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) cudaSetDevice(dev);
    else prev = -1;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

static size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

}  // namespace lmoe

using namespace lmoe;

// names of the kernels one forward launches, in launch order (the two
// split-K reductions run only for small token counts)
static const char* const kKernelNames[] = {
    "xgemm(router|W_dn|W_s1)", "route(sigmoid+bias+topK)", "hist", "scan", "scatter",
    "gather(u->expert order)", "grouped_gemm1(W1,sqrelu)", "grouped_gemm2(W2,*w)",
    "combine", "ygemm([W_upl|W_s2])", "xgemm split-K reduce + route(sigmoid+bias+topK)",
    "ygemm split-K reduce",
    // backward
    "bw dgrad [W_upl|W_s2]^T (dv, dhs)", "bw gather(w dv -> expert order)",
    "bw dgrad W2^T (dg)", "bw dgrad W1^T (du rows)", "bw combine(du)", "bw route(dz)",
    "bw dgrad [W_r;W_dn;W_s1]^T (dx)", "bw wgrad [W_upl|W_s2]", "bw wgrad W2",
    "bw wgrad W1", "bw wgrad [W_r;W_dn;W_s1]", "bw act'(da = dg 2 sqrt(g), dw)",
    // overlapped forward: the shared expert on the side stream
    "shared W_s1 (side stream)", "shared W_s2 (side stream)",
    // the routed experts' NVFP4 backward (its GEMMs keep the labels above)
    "bw4 dL/dw = o . dv", "bw4 w dv rows -> NVFP4 (SR)", "bw4 da rows -> NVFP4 (SR)",
    "bw4 wgrad W2 operands (g^T, do^T)", "bw4 wgrad W1 operands (u^T, da^T)",
    "bw4 zero gradients of experts without rows",
    // forward, at most 256 tokens
    "segments (hist+scan+scatter, one block)"};
static constexpr int kNumKernels = 33;
static_assert(sizeof(kKernelNames) / sizeof(kKernelNames[0]) == kNumKernels, "kernel labels");

// Dense-GEMM plan for T tokens: token-block width and number of K slices.
// Enough tiles to fill the GPU first by narrower token blocks (while one
// block still spans 128 rows), else by splitting K, so that every weight byte
// is read once and no token block is re-read more than necessary.
struct DensePlan {
  int bn, ksplit;
};
static DensePlan plan_dense(int64_t T, int fb, int kblocks, int sms) {
  for (int bn : {256, 128})
    if (((T + bn - 1) / bn) * fb >= sms) return {bn, 1};
  const int bn = T <= 32 ? 32 : (T <= 128 ? 128 : 256);
  const int64_t tiles = ((T + bn - 1) / bn) * fb;
  int64_t ks = sms / tiles;   // one wave: tiles * ks <= sms
  if (ks > 8) ks = 8;
  if (ks > kblocks / 4) ks = kblocks / 4;
  if (ks < 1) ks = 1;
  return {bn, static_cast<int>(ks)};
}

struct lmoe_handle {
  lmoe_config cfg;
  int dev = 0;
  int sms = 148;
  // weights
  bf16* w_x = nullptr;     // [N+l+h_s][d]
  float* bias = nullptr;   // [N]
  bf16* w1 = nullptr;      // [N][h][l]
  bf16* w2 = nullptr;      // [N][l][h]
  bf16* w_y = nullptr;     // [d][l+h_s]
  // workspace
  float* logits = nullptr;
  int32_t* topk_idx = nullptr;
  float* topk_w = nullptr;
  int32_t* chunk = nullptr;
  int32_t* counts = nullptr;
  int32_t* offsets = nullptr;
  int32_t* perm = nullptr;
  int32_t* inv = nullptr;
  float* wrow = nullptr;
  int4* blocks = nullptr;
  int32_t* nblocks = nullptr;
  bf16* u = nullptr;
  bf16* u_perm = nullptr;
  bf16* H = nullptr;
  bf16* O = nullptr;
  bf16* vh = nullptr;      // [max_tokens][l+h_s]: v | hs
  bf16* x_dev = nullptr;   // staging for lmoe_forward_host
  bf16* y_dev = nullptr;
  float* part = nullptr;   // split-K partials of the dense GEMMs
  int64_t part_floats = 0; // its capacity
  int* err = nullptr;
  // NVFP4 experts: quantised weights, activations and their scale atoms
  bool fp4 = false;
  int lp = 0, hp = 0;          // l, h rounded up to 256 (K of the two grouped GEMMs)
  float g_u = 0.f, g_h = 0.f;  // static global scales of u and of the expert hidden
  uint8_t* w1q = nullptr;      // [N*h][lp/2]
  uint8_t* w1sf = nullptr;     // [N*h/128][lp/64][512]
  float* gw1 = nullptr;        // [N]
  uint8_t* w2q = nullptr;      // [N*l][hp/2]
  uint8_t* w2sf = nullptr;     // [N*l/128][hp/64][512]
  float* gw2 = nullptr;        // [N]
  float* amax = nullptr;       // [N] scratch of the weight quantisation
  float* stab = nullptr;       // scale tables of g_u, then of g_h (2 x NVFP4_TAB)
  uint8_t* uq = nullptr;       // [T][l/2]
  uint8_t* usf = nullptr;      // [T][l/16]
  uint8_t* upq = nullptr;      // [T*K][lp/2] expert order
  uint8_t* sfbu = nullptr;     // [token blocks][lp/64][512]
  uint8_t* Hq = nullptr;       // [T*K][hp/2]
  uint8_t* sfbh = nullptr;     // [token blocks][hp/64][512]
  int32_t* rblock = nullptr;   // [T*K] (token block << 8) | row in block
  CUtensorMap tm_w1q, tm_w2q;
  BMaps tm_upq, tm_Hq;
  // FP8 (E4M3) W8A8 experts: codes and per-tensor scales
  bool fp8 = false;
  float r_u8 = 0.f, r_h8 = 0.f;  // 1 / s_u, 1 / s_h (rounded once); s in g_u, g_h
  uint8_t* w1f8 = nullptr;     // [N*h][l]
  uint8_t* w2f8 = nullptr;     // [N*l][h]
  float* sw1 = nullptr;        // [N] amax / 448
  float* sw2 = nullptr;        // [N]
  uint8_t* uf8 = nullptr;      // [T][l]
  uint8_t* upf8 = nullptr;     // [T*K][l] expert order
  uint8_t* Hf8 = nullptr;      // [T*K][h]
  CUtensorMap tm_w1f8, tm_w2f8;
  BMaps tm_upf8, tm_Hf8;
  // W4A16 experts: the NVFP4 weights above, read as raw code tiles (32 B x
  // 128 rows, no swizzle) and expanded to f16 in the GEMM; u and H in f16
  bool w4 = false;
  __half* u16 = nullptr;       // [T][l]
  CUtensorMap tm_w1c, tm_w2c;
  // backward workspace (LMOE_FLAG_BACKWARD)
  bool bw = false;
  bf16* dv = nullptr;        // [Tm_b][l]   dL/dv
  bf16* dog = nullptr;       // [rows_b][l] w_r dv rows in expert order
  bf16* da = nullptr;        // [rows_b][h] gradient of the expert pre-activation
  bf16* dup = nullptr;       // [rows_b][l] W1[e]^T da rows in expert order
  float* dwacc = nullptr;    // [rows]      sum_h g dg per routed row
  bf16* dxh = nullptr;       // [Tm_b][N+l+h_s] dz | du | d(shared pre-activation)
  bf16* dy_dev = nullptr;    // [64][d]     staging of dy for T < 64
  CUtensorMap tm_wx64, tm_wy64, tm_w1_64, tm_w2_64;   // weights in 64-row boxes
  BMaps tm_dog, tm_da, tm_dxh;
  // NVFP4 training (NVFP4 experts, 2D weight blocks, LMOE_FLAG_BACKWARD):
  // transposed weights, the backward's rows and transposed operands
  bool bw4 = false;
  uint8_t* w1qT = nullptr;     // [N*l][hp/2] codes of W1[e]^T
  uint8_t* w1qT_sf = nullptr;  // [N*l/128][hp/64][512]
  uint8_t* w2qT = nullptr;     // [N*h][lp/2] codes of W2[e]^T
  uint8_t* w2qT_sf = nullptr;  // [N*h/128][lp/64][512]
  bf16* a16 = nullptr;         // [rows_b][h] pre-activations W1[e] u
  float* do32 = nullptr;       // [rows][l] w dv rows
  uint8_t* doq = nullptr;      // [rows_b][lp/2]
  uint8_t* doS = nullptr;      // [rows][l/16]
  uint8_t* sfbdo = nullptr;    // [token blocks][lp/64][512]
  float* da32 = nullptr;       // [rows][h]
  uint8_t* daq = nullptr;      // [rows_b][hp/2]
  uint8_t* daS = nullptr;      // [rows][h/16]
  uint8_t* sfbda = nullptr;    // [token blocks][hp/64][512]
  int32_t* po16 = nullptr;     // [N+1] columns, segments padded to 16
  int32_t* po256 = nullptr;    // [N+1] columns, segments padded to 256
  int32_t* kofs = nullptr;     // [N+1] FP4 k-steps of po256
  int32_t* grp = nullptr;      // [rp_cap / 64] expert of each 64-column group
  float* scal = nullptr;       // [16]: amax 0..7, global scales 8..15
  int64_t rp_cap = 0;          // columns of the transposed operands
  // transposed operands: 0 do^T (B of dW2), 1 g^T (A of dW2), 2 u^T (A of
  // dW1), 3 da^T (B of dW1): codes [F][rp_cap/2], scales [F][rp_cap/16], atoms
  uint8_t* tq[4] = {};
  uint8_t* ts[4] = {};
  uint8_t* ta[4] = {};
  CUtensorMap tm_w1qT, tm_w2qT, tm_tA[4];
  BMaps tm_doq, tm_daq, tm_tB[4];
  int64_t bw4_T = -1;          // T of the last lmoe_experts_backward_nvfp4
  uint64_t bw_seed = 0;        // random bits of the next NVFP4 lmoe_backward
  // overlapped forward (BF16 experts bound by HBM): the shared expert's two
  // GEMMs on a side stream over a share of the SMs
  cudaStream_t side_st = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  float* ys = nullptr;         // [max_tokens][d] W_s2 hs (fp32)
  CUtensorMap tm_ws1, tm_ws2;  // W_s1 rows of w_x; W_s2 columns of w_y
  BMaps tm_hs;                 // hs columns of vh
  std::vector<void*> allocs;
  CUtensorMap tm_wx, tm_w1, tm_w2, tm_wy;
  BMaps tm_uperm, tm_H, tm_vh;
  int64_t last_T = 0;
  // expert parallelism: a layer handle without expert weights (dispatch and
  // combine only), or an expert shard (experts [first_expert, + n_experts))
  bool ep_dense = false;
  bool shard = false;
  int first_expert = 0;
  int64_t max_rows = 0;       // shard: rows one lmoe_experts_forward accepts
  bool pairs = true;   // CTA-pair GEMMs for large token counts (LMOE_PAIR=0: off)
  bool proj = true;    // latent projections (false: standard MoE, u = x, r = v)
  int lx = 0;          // W_dn rows in w_x and W_upl columns in w_y (l, or 0)
  unsigned long long wait_limit_ns = 2000000000ull;
  // profiling
  bool prof = false;
  std::vector<cudaEvent_t> ev;      // pairs
  std::vector<int> ev_kernel;
  size_t ev_used = 0;
  double prof_ms[kNumKernels] = {};
  int64_t prof_n[kNumKernels] = {};
};

// A zero-byte request leaves the pointer null, so that a buffer of an unused
// path can never be mistaken for a live one.
static int alloc_dev(lmoe_handle* h, void** p, size_t bytes) {
  if (bytes == 0) {
    *p = nullptr;
    return LMOE_OK;
  }
  if (cudaMalloc(p, bytes < 256 ? 256 : bytes) != cudaSuccess) {
    cudaGetLastError();
    return LMOE_ERR_OOM;
  }
  h->allocs.push_back(*p);
  return LMOE_OK;
}

static void free_all(lmoe_handle* h) {
  for (void* p : h->allocs) cudaFree(p);
  h->allocs.clear();
  if (h->side_st) cudaStreamDestroy(h->side_st);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  h->side_st = nullptr;
  h->ev_fork = h->ev_join = nullptr;
  for (cudaEvent_t e : h->ev) cudaEventDestroy(e);
  h->ev.clear();
}

static int check_cfg(const lmoe_config* c) {
  if (!c) return LMOE_ERR_INVALID_ARG;
  if (c->d <= 0 || c->latent <= 0 || c->n_experts <= 0 || c->top_k <= 0 ||
      c->expert_hidden <= 0 || c->shared_hidden <= 0 || c->max_tokens < 1 ||
      (c->flags & ~(LMOE_FLAG_NO_PROJECTION | LMOE_FLAG_NVFP4_WEIGHT_2D |
                    LMOE_FLAG_NVFP4_WEIGHT_MSE | LMOE_FLAG_BACKWARD | LMOE_FLAG_EP_DENSE)) != 0)
    return LMOE_ERR_INVALID_ARG;
  if ((c->flags & LMOE_FLAG_EP_DENSE) &&
      ((c->flags & (LMOE_FLAG_NO_PROJECTION | LMOE_FLAG_BACKWARD)) ||
       c->expert_format != LMOE_FMT_BF16))
    return LMOE_ERR_UNSUPPORTED;
  if ((c->flags & (LMOE_FLAG_NVFP4_WEIGHT_2D | LMOE_FLAG_NVFP4_WEIGHT_MSE)) &&
      c->expert_format != LMOE_FMT_NVFP4 && c->expert_format != LMOE_FMT_W4A16)
    return LMOE_ERR_INVALID_ARG;
  if ((c->flags & LMOE_FLAG_NO_PROJECTION) &&
      (c->latent != c->d || c->expert_format != LMOE_FMT_BF16))
    return LMOE_ERR_UNSUPPORTED;
  if ((c->flags & LMOE_FLAG_BACKWARD) &&
      ((c->flags & LMOE_FLAG_NO_PROJECTION) ||
       !(c->expert_format == LMOE_FMT_BF16 ||
         (c->expert_format == LMOE_FMT_NVFP4 && (c->flags & LMOE_FLAG_NVFP4_WEIGHT_2D)))))
    return LMOE_ERR_UNSUPPORTED;
  if (c->top_k > c->n_experts) return LMOE_ERR_INVALID_ARG;
  if (c->expert_format != LMOE_FMT_BF16 && c->expert_format != LMOE_FMT_NVFP4 &&
      c->expert_format != LMOE_FMT_FP8 && c->expert_format != LMOE_FMT_W4A16)
    return LMOE_ERR_INVALID_ARG;
  if (c->expert_format != LMOE_FMT_BF16 && (c->latent % 128 || c->expert_hidden % 128))
    return LMOE_ERR_UNSUPPORTED;
  if (c->d % 64 || c->latent % 64 || c->expert_hidden % 64 || c->shared_hidden % 64)
    return LMOE_ERR_UNSUPPORTED;
  if (c->n_experts % 32 || c->n_experts > 1024 || c->top_k > 32) return LMOE_ERR_UNSUPPORTED;
  const int64_t rows = c->max_tokens * c->top_k;
  if (rows >= (int64_t(1) << 31) - 65536) return LMOE_ERR_UNSUPPORTED;
  if (int64_t(c->n_experts) * c->expert_hidden >= (int64_t(1) << 31)) return LMOE_ERR_UNSUPPORTED;
  if (int64_t(c->n_experts) * c->latent >= (int64_t(1) << 31)) return LMOE_ERR_UNSUPPORTED;
  return LMOE_OK;
}

// grouped-GEMM token-block width for a forward of T tokens (NVFP4 tiles have
// at most 128 token rows: one scale atom)
static int grouped_bn(const lmoe_config& c, int64_t T) {
  const double avg = double(T) * c.top_k / c.n_experts;
  if (avg <= 40.0) return 32;
  // NVFP4 B tiles carry one scale atom (<= 128 rows); W4A16 stages at 256
  // rows would leave one stage of shared memory
  if (avg <= 160.0 || c.expert_format == LMOE_FMT_NVFP4 || c.expert_format == LMOE_FMT_W4A16)
    return 128;
  return 256;
}

extern "C" {

const char* lmoe_strerror(int code) {
  switch (code) {
    case LMOE_OK: return "ok";
    case LMOE_ERR_INVALID_ARG: return "invalid argument";
    case LMOE_ERR_UNSUPPORTED: return "unsupported layer shape or format";
    case LMOE_ERR_OOM: return "device allocation failed";
    case LMOE_ERR_CUDA: return "CUDA call failed";
    case LMOE_ERR_TIMEOUT: return "a bounded device wait ran out";
    case LMOE_ERR_DEVICE: return "a kernel flagged invalid data";
    default: return "unknown error";
  }
}

int lmoe_create(const lmoe_config* cfg, const lmoe_weights* w, lmoe_handle** out) {
  if (!out) return LMOE_ERR_INVALID_ARG;
  *out = nullptr;
  int rc = check_cfg(cfg);
  if (rc != LMOE_OK) return rc;
  const bool proj = !(cfg->flags & LMOE_FLAG_NO_PROJECTION);
  const bool ep_dense = (cfg->flags & LMOE_FLAG_EP_DENSE) != 0;
  if (!w || !w->w_router || (!ep_dense && (!w->w1 || !w->w2)) || !w->w_s1 || !w->w_s2 ||
      (proj && (!w->w_dn || !w->w_upl)))
    return LMOE_ERR_INVALID_ARG;
  if ((cfg->expert_format == LMOE_FMT_NVFP4 || cfg->expert_format == LMOE_FMT_FP8) &&
      !(w->act_gscale_latent > 0.0f && w->act_gscale_hidden > 0.0f &&
        w->act_gscale_latent < 3.0e38f && w->act_gscale_hidden < 3.0e38f))
    return LMOE_ERR_INVALID_ARG;
  if (!get_encode()) return LMOE_ERR_CUDA;

  lmoe_handle* h = new (std::nothrow) lmoe_handle();
  if (!h) return LMOE_ERR_OOM;
  h->cfg = *cfg;
  if (cudaGetDevice(&h->dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, h->dev) != cudaSuccess) {
    delete h;
    return LMOE_ERR_CUDA;
  }
  const lmoe_config& c = h->cfg;
  const int64_t N = c.n_experts, d = c.d, l = c.latent, hh = c.expert_hidden,
                hs = c.shared_hidden, K = c.top_k, Tm = c.max_tokens;
  h->proj = proj;
  h->lx = proj ? static_cast<int>(l) : 0;
  const int64_t lx = h->lx;
  const int64_t rows = Tm * K;
  const int64_t C = (Tm + 31) / 32;
  // operand buffers read by TMA hold at least one box of rows
  const int64_t rows_b = rows < 256 ? 256 : rows;
  const int64_t Tm_b = Tm < 256 ? 256 : Tm;
  const int64_t d_a = d < GEMM_BM ? GEMM_BM : d;
  const bool w4 = c.expert_format == LMOE_FMT_W4A16;
  const bool fp4 = c.expert_format == LMOE_FMT_NVFP4;   // NVFP4 activations too
  const bool fp8 = c.expert_format == LMOE_FMT_FP8;
  h->ep_dense = ep_dense;
  const bool bfx = !fp4 && !fp8 && !w4 && !ep_dense;   // BF16 experts held by this handle
  const bool qw4 = fp4 || w4;             // NVFP4-quantised expert weights
  h->fp4 = fp4;
  h->fp8 = fp8;
  h->w4 = w4;
  h->lp = static_cast<int>((l + 255) / 256 * 256);
  h->hp = static_cast<int>((hh + 255) / 256 * 256);
  const int64_t lp = h->lp, hp = h->hp;
  const int64_t nb_max = rows / 32 + N + 1;   // token blocks of >= 32 rows, one partial per expert
  // bytes of the bf16 expert path buffers that NVFP4 replaces
  const int64_t bf16_only = bfx ? 1 : 0;
  const int64_t act16 = (bfx || w4) ? 1 : 0;   // 16-bit expert activations (u_perm, H)
  // largest split-K partials buffer over the token counts this handle
  // accepts, for the same feature and K extents the forward pass plans with
  // (x-GEMM: N + lx + h_s features over K = d; y-GEMM: d features over
  // K = lx + h_s)
  int64_t part_floats = 0;
  {
    const int fbx = static_cast<int>((N + lx + hs + 127) / 128);
    const int fby = static_cast<int>((d + 127) / 128);
    const int64_t tmax = Tm < 256LL * h->sms ? Tm : 256LL * h->sms;
    for (int64_t T = 1; T <= tmax; ++T) {
      const DensePlan px = plan_dense(T, fbx, static_cast<int>(d / 64), h->sms);
      const DensePlan py = plan_dense(T, fby, static_cast<int>((lx + hs) / 64), h->sms);
      if (px.ksplit > 1 && px.ksplit * T * (N + lx + hs) > part_floats)
        part_floats = px.ksplit * T * (N + lx + hs);
      if (py.ksplit > 1 && py.ksplit * T * d > part_floats) part_floats = py.ksplit * T * d;
    }
  }
  h->part_floats = part_floats;
  const int64_t max_blocks = rows / 32 + N + 1;
  // the BF16 backward's workspace, or the NVFP4 training backward's
  const int64_t bwd = ((c.flags & LMOE_FLAG_BACKWARD) && bfx) ? 1 : 0;
  const int64_t bw4 = ((c.flags & LMOE_FLAG_BACKWARD) && fp4) ? 1 : 0;
  const int64_t bwx = (bwd || bw4) ? 1 : 0;   // the dense GEMMs' backward
  h->bw = bwd != 0;
  h->bw4 = bw4 != 0;
  // transposed operands of the NVFP4 weight gradients: every expert's rows
  // padded to 256 columns; the transform kernels take a 16-column block per
  // grid row (at most 65535)
  const int64_t rp_cap = bw4 ? (rows + 255 * N + 255) / 256 * 256 : 0;
  if (rp_cap / 16 > 65535) {
    delete h;
    return LMOE_ERR_UNSUPPORTED;
  }
  h->rp_cap = rp_cap;
  const int64_t tf[4] = {l, hh, l, hh};   // features of the transposed operands
  struct Req {
    void** p;
    size_t bytes;
  } reqs[] = {
      {(void**)&h->w_x, size_t((N + lx + hs) * d * 2)},
      {(void**)&h->bias, size_t(N * 4)},
      {(void**)&h->w1, size_t(bf16_only * N * hh * l * 2)},
      {(void**)&h->w2, size_t(bf16_only * N * l * hh * 2)},
      {(void**)&h->w_y, size_t(d_a * (lx + hs) * 2)},
      {(void**)&h->logits, size_t(Tm * N * 4)},
      {(void**)&h->topk_idx, size_t(rows * 4)},
      {(void**)&h->topk_w, size_t(rows * 4)},
      {(void**)&h->chunk, size_t(C * N * 4)},
      {(void**)&h->counts, size_t(N * 4)},
      {(void**)&h->offsets, size_t((N + 1) * 4)},
      {(void**)&h->perm, size_t(rows * 4)},
      {(void**)&h->inv, size_t(rows * 4)},
      {(void**)&h->wrow, size_t(rows * 4)},
      {(void**)&h->blocks, size_t(max_blocks * 16)},
      {(void**)&h->nblocks, size_t(4)},
      {(void**)&h->u, size_t(Tm * lx * 2)},
      {(void**)&h->u_perm, size_t(act16 * rows_b * l * 2)},
      {(void**)&h->H, size_t(act16 * rows_b * hh * 2)},
      {(void**)&h->O, size_t(rows * l * 2)},
      {(void**)&h->vh, size_t(Tm_b * (l + hs) * 2)},
      {(void**)&h->x_dev, size_t(Tm_b * d * 2)},
      {(void**)&h->y_dev, size_t(Tm * d * 2)},
      {(void**)&h->part, size_t(part_floats * 4)},
      {(void**)&h->err, size_t(4)},
      {(void**)&h->w1q, size_t(qw4 * N * hh * lp / 2)},
      {(void**)&h->w1sf, size_t(qw4 * (N * hh / 128) * (lp / 64) * 512)},
      {(void**)&h->gw1, size_t(qw4 * N * 4)},
      {(void**)&h->w2q, size_t(qw4 * N * l * hp / 2)},
      {(void**)&h->w2sf, size_t(qw4 * (N * l / 128) * (hp / 64) * 512)},
      {(void**)&h->gw2, size_t(qw4 * N * 4)},
      {(void**)&h->amax, size_t((qw4 || fp8) * N * 4)},
      {(void**)&h->u16, size_t(w4 * Tm * l * 2)},
      {(void**)&h->stab, size_t(fp4 * 2 * NVFP4_TAB * 4)},
      {(void**)&h->uq, size_t(fp4 * Tm * l / 2)},
      {(void**)&h->usf, size_t(fp4 * Tm * l / 16)},
      {(void**)&h->upq, size_t(fp4 * rows_b * lp / 2)},
      {(void**)&h->sfbu, size_t(fp4 * nb_max * (lp / 64) * 512)},
      {(void**)&h->Hq, size_t(fp4 * rows_b * hp / 2)},
      {(void**)&h->sfbh, size_t(fp4 * nb_max * (hp / 64) * 512)},
      {(void**)&h->rblock, size_t(fp4 * rows * 4)},
      {(void**)&h->w1f8, size_t(fp8 * N * hh * l)},
      {(void**)&h->w2f8, size_t(fp8 * N * l * hh)},
      {(void**)&h->sw1, size_t(fp8 * N * 4)},
      {(void**)&h->sw2, size_t(fp8 * N * 4)},
      {(void**)&h->uf8, size_t(fp8 * Tm * l)},
      {(void**)&h->upf8, size_t(fp8 * rows_b * l)},
      {(void**)&h->Hf8, size_t(fp8 * rows_b * hh)},
      {(void**)&h->dv, size_t(bwx * Tm_b * l * 2)},
      {(void**)&h->dog, size_t(bwd * rows_b * l * 2)},
      {(void**)&h->da, size_t(bwd * rows_b * hh * 2)},
      {(void**)&h->dup, size_t(bwd * rows_b * l * 2)},
      {(void**)&h->dwacc, size_t(bwx * rows * 4)},
      {(void**)&h->dxh, size_t(bwx * Tm_b * (N + l + hs) * 2)},
      {(void**)&h->dy_dev, size_t(bwx * GEMM_BROWS_BIG * d * 2)},
      {(void**)&h->ys, size_t((bfx && proj) ? Tm * d * 4 : 0)},
      {(void**)&h->w1qT, size_t(bw4 * N * l * hp / 2)},
      {(void**)&h->w1qT_sf, size_t(bw4 * (N * l / 128) * (hp / 64) * 512)},
      {(void**)&h->w2qT, size_t(bw4 * N * hh * lp / 2)},
      {(void**)&h->w2qT_sf, size_t(bw4 * (N * hh / 128) * (lp / 64) * 512)},
      {(void**)&h->a16, size_t(bw4 * rows_b * hh * 2)},
      {(void**)&h->do32, size_t(bw4 * rows * l * 4)},
      {(void**)&h->doq, size_t(bw4 * rows_b * lp / 2)},
      {(void**)&h->doS, size_t(bw4 * rows * l / 16)},
      {(void**)&h->sfbdo, size_t(bw4 * nb_max * (lp / 64) * 512)},
      {(void**)&h->da32, size_t(bw4 * rows * hh * 4)},
      {(void**)&h->daq, size_t(bw4 * rows_b * hp / 2)},
      {(void**)&h->daS, size_t(bw4 * rows * hh / 16)},
      {(void**)&h->sfbda, size_t(bw4 * nb_max * (hp / 64) * 512)},
      {(void**)&h->po16, size_t(bw4 * (N + 1) * 4)},
      {(void**)&h->po256, size_t(bw4 * (N + 1) * 4)},
      {(void**)&h->kofs, size_t(bw4 * (N + 1) * 4)},
      {(void**)&h->grp, size_t(bw4 * (rp_cap / 64) * 4)},
      {(void**)&h->scal, size_t(bw4 * 64)},
      {(void**)&h->tq[0], size_t(bw4 * tf[0] * rp_cap / 2)},
      {(void**)&h->tq[1], size_t(bw4 * tf[1] * rp_cap / 2)},
      {(void**)&h->tq[2], size_t(bw4 * tf[2] * rp_cap / 2)},
      {(void**)&h->tq[3], size_t(bw4 * tf[3] * rp_cap / 2)},
      {(void**)&h->ts[0], size_t(bw4 * tf[0] * rp_cap / 16)},
      {(void**)&h->ts[1], size_t(bw4 * tf[1] * rp_cap / 16)},
      {(void**)&h->ts[2], size_t(bw4 * tf[2] * rp_cap / 16)},
      {(void**)&h->ts[3], size_t(bw4 * tf[3] * rp_cap / 16)},
      {(void**)&h->ta[0], size_t(bw4 * tf[0] * rp_cap / 16)},
      {(void**)&h->ta[1], size_t(bw4 * tf[1] * rp_cap / 16)},
      {(void**)&h->ta[2], size_t(bw4 * tf[2] * rp_cap / 16)},
      {(void**)&h->ta[3], size_t(bw4 * tf[3] * rp_cap / 16)},
  };
  for (auto& r : reqs) {
    if ((rc = alloc_dev(h, r.p, r.bytes)) != LMOE_OK) {
      free_all(h);
      delete h;
      return rc;
    }
  }
  bool ok = true;
  // weights, re-laid: [W_r; W_dn; W_s1] and [W_upl | W_s2]
  ok &= cudaMemcpy(h->w_x, w->w_router, N * d * 2, cudaMemcpyDeviceToDevice) == cudaSuccess;
  if (proj)
    ok &= cudaMemcpy(h->w_x + N * d, w->w_dn, l * d * 2, cudaMemcpyDeviceToDevice) == cudaSuccess;
  ok &= cudaMemcpy(h->w_x + (N + lx) * d, w->w_s1, hs * d * 2, cudaMemcpyDeviceToDevice) ==
        cudaSuccess;
  if (bfx) {
    ok &= cudaMemcpy(h->w1, w->w1, N * hh * l * 2, cudaMemcpyDeviceToDevice) == cudaSuccess;
    ok &= cudaMemcpy(h->w2, w->w2, N * l * hh * 2, cudaMemcpyDeviceToDevice) == cudaSuccess;
  } else if (ep_dense) {
    // no expert weights: the experts live in expert shards (lmoe_experts_create)
  } else if (fp8) {
    // per-tensor scales: s = amax / 448 per expert matrix; activations static
    h->g_u = w->act_gscale_latent;
    h->g_h = w->act_gscale_hidden;
    h->r_u8 = 1.0f / h->g_u;
    h->r_h8 = 1.0f / h->g_h;
    ok &= cudaMemset(h->upf8, 0, rows_b * l) == cudaSuccess;
    ok &= cudaMemset(h->Hf8, 0, rows_b * hh) == cudaSuccess;
    ok &= launch_quant_w8(w->w1, static_cast<int>(N), static_cast<int>(hh), static_cast<int>(l),
                          h->amax, h->w1f8, h->sw1, 0) == cudaSuccess;
    ok &= launch_quant_w8(w->w2, static_cast<int>(N), static_cast<int>(l), static_cast<int>(hh),
                          h->amax, h->w2f8, h->sw2, 0) == cudaSuccess;
    ok &= make_map_u8(&h->tm_w1f8, h->w1f8, N * hh, l, GEMM_BM);
    ok &= make_map_u8(&h->tm_w2f8, h->w2f8, N * l, hh, GEMM_BM);
    ok &= make_map_u8(&h->tm_upf8.b16, h->upf8, rows_b, l, GEMM_BROWS);
    ok &= make_map_u8(&h->tm_upf8.b64, h->upf8, rows_b, l, GEMM_BROWS_BIG);
    ok &= make_map_u8(&h->tm_Hf8.b16, h->Hf8, rows_b, hh, GEMM_BROWS);
    ok &= make_map_u8(&h->tm_Hf8.b64, h->Hf8, rows_b, hh, GEMM_BROWS_BIG);
    ok &= set_gemm_smem<256, EpiH8, KIND_FP8>() == cudaSuccess;
    ok &= set_gemm_smem<256, EpiO8, KIND_FP8>() == cudaSuccess;
    ok &= set_gemm_smem<128, EpiH8, KIND_FP8>() == cudaSuccess;
    ok &= set_gemm_smem<32, EpiH8, KIND_FP8>() == cudaSuccess;
    ok &= set_gemm_smem<128, EpiO8, KIND_FP8>() == cudaSuccess;
    ok &= set_gemm_smem<32, EpiO8, KIND_FP8>() == cudaSuccess;
  } else {
    // padding (K beyond l or h, unused atoms) must read as zero
    h->g_u = w->act_gscale_latent;
    h->g_h = w->act_gscale_hidden;
    ok &= cudaMemset(h->w1q, 0, N * hh * lp / 2) == cudaSuccess;
    ok &= cudaMemset(h->w1sf, 0, (N * hh / 128) * (lp / 64) * 512) == cudaSuccess;
    ok &= cudaMemset(h->w2q, 0, N * l * hp / 2) == cudaSuccess;
    ok &= cudaMemset(h->w2sf, 0, (N * l / 128) * (hp / 64) * 512) == cudaSuccess;
    if (fp4) {
      ok &= cudaMemset(h->upq, 0, rows_b * lp / 2) == cudaSuccess;
      ok &= cudaMemset(h->sfbu, 0, nb_max * (lp / 64) * 512) == cudaSuccess;
      ok &= cudaMemset(h->Hq, 0, rows_b * hp / 2) == cudaSuccess;
      ok &= cudaMemset(h->sfbh, 0, nb_max * (hp / 64) * 512) == cudaSuccess;
    }
    const int wvar = ((c.flags & LMOE_FLAG_NVFP4_WEIGHT_2D) ? QUANT_W_2D : 0) |
                     ((c.flags & LMOE_FLAG_NVFP4_WEIGHT_MSE) ? QUANT_W_MSE : 0);
    ok &= launch_quant_weights(w->w1, static_cast<int>(N), static_cast<int>(hh), static_cast<int>(l),
                               static_cast<int>(lp), h->amax, h->w1q, h->w1sf, h->gw1, wvar,
                               0) == cudaSuccess;
    ok &= launch_quant_weights(w->w2, static_cast<int>(N), static_cast<int>(l), static_cast<int>(hh),
                               static_cast<int>(hp), h->amax, h->w2q, h->w2sf, h->gw2, wvar,
                               0) == cudaSuccess;
    if (fp4) {
      ok &= launch_scale_tables(h->g_u, h->stab, 0) == cudaSuccess;
      ok &= launch_scale_tables(h->g_h, h->stab + NVFP4_TAB, 0) == cudaSuccess;
      ok &= make_map_u8(&h->tm_w1q, h->w1q, N * hh, lp / 2, GEMM_BM);
      ok &= make_map_u8(&h->tm_w2q, h->w2q, N * l, hp / 2, GEMM_BM);
      ok &= make_map_u8(&h->tm_upq.b16, h->upq, rows_b, lp / 2, GEMM_BROWS);
      ok &= make_map_u8(&h->tm_upq.b64, h->upq, rows_b, lp / 2, GEMM_BROWS_BIG);
      ok &= make_map_u8(&h->tm_Hq.b16, h->Hq, rows_b, hp / 2, GEMM_BROWS);
      ok &= make_map_u8(&h->tm_Hq.b64, h->Hq, rows_b, hp / 2, GEMM_BROWS_BIG);
      ok &= set_gemm_smem<128, EpiHq, KIND_NVFP4>() == cudaSuccess;
      ok &= set_gemm_smem<32, EpiHq, KIND_NVFP4>() == cudaSuccess;
      ok &= set_gemm_smem<128, EpiOq, KIND_NVFP4>() == cudaSuccess;
      ok &= set_gemm_smem<32, EpiOq, KIND_NVFP4>() == cudaSuccess;
      if (bw4) {
        // the dgrad GEMMs read W^T: a 2D block's scale serves both orientations
        ok &= cudaMemset(h->doq, 0, rows_b * lp / 2) == cudaSuccess;
        ok &= cudaMemset(h->daq, 0, rows_b * hp / 2) == cudaSuccess;
        ok &= cudaMemset(h->sfbdo, 0, nb_max * (lp / 64) * 512) == cudaSuccess;
        ok &= cudaMemset(h->sfbda, 0, nb_max * (hp / 64) * 512) == cudaSuccess;
        ok &= launch_transpose_w2d(h->w1q, h->w1sf, static_cast<int>(N), static_cast<int>(hh),
                                   static_cast<int>(l), static_cast<int>(lp),
                                   static_cast<int>(hp), h->w1qT, h->w1qT_sf, 0) == cudaSuccess;
        ok &= launch_transpose_w2d(h->w2q, h->w2sf, static_cast<int>(N), static_cast<int>(l),
                                   static_cast<int>(hh), static_cast<int>(hp),
                                   static_cast<int>(lp), h->w2qT, h->w2qT_sf, 0) == cudaSuccess;
        ok &= make_map_u8(&h->tm_w1qT, h->w1qT, N * l, hp / 2, GEMM_BM);
        ok &= make_map_u8(&h->tm_w2qT, h->w2qT, N * hh, lp / 2, GEMM_BM);
        ok &= make_map_u8(&h->tm_doq.b16, h->doq, rows_b, lp / 2, GEMM_BROWS);
        ok &= make_map_u8(&h->tm_doq.b64, h->doq, rows_b, lp / 2, GEMM_BROWS_BIG);
        ok &= make_map_u8(&h->tm_daq.b16, h->daq, rows_b, hp / 2, GEMM_BROWS);
        ok &= make_map_u8(&h->tm_daq.b64, h->daq, rows_b, hp / 2, GEMM_BROWS_BIG);
        for (int i = 0; i < 4; ++i) {
          ok &= make_map_u8(&h->tm_tA[i], h->tq[i], tf[i], rp_cap / 2, GEMM_BM);
          ok &= make_map_u8(&h->tm_tB[i].b16, h->tq[i], tf[i], rp_cap / 2, GEMM_BROWS);
          ok &= make_map_u8(&h->tm_tB[i].b64, h->tq[i], tf[i], rp_cap / 2, GEMM_BROWS_BIG);
        }
        ok &= set_gemm_smem<128, EpiDA, KIND_NVFP4>() == cudaSuccess;
        ok &= set_gemm_smem<32, EpiDA, KIND_NVFP4>() == cudaSuccess;
        ok &= set_gemm_smem<128, EpiDU, KIND_NVFP4>() == cudaSuccess;
        ok &= set_gemm_smem<32, EpiDU, KIND_NVFP4>() == cudaSuccess;
        ok &= set_gemm_smem<128, EpiWq, KIND_NVFP4>() == cudaSuccess;
      }
    } else {
      // W4A16: code tiles of one k-step (64 elements = 32 bytes) x 128 rows
      ok &= make_map_codes(&h->tm_w1c, h->w1q, N * hh, lp / 2);
      ok &= make_map_codes(&h->tm_w2c, h->w2q, N * l, hp / 2);
      ok &= set_gemm_smem<128, EpiH16, KIND_W4A16>() == cudaSuccess;
      ok &= set_gemm_smem<32, EpiH16, KIND_W4A16>() == cudaSuccess;
      ok &= set_gemm_smem<128, EpiO16, KIND_W4A16>() == cudaSuccess;
      ok &= set_gemm_smem<32, EpiO16, KIND_W4A16>() == cudaSuccess;
    }
  }
  if (proj)
    ok &= cudaMemcpy2D(h->w_y, (lx + hs) * 2, w->w_upl, l * 2, l * 2, d,
                       cudaMemcpyDeviceToDevice) == cudaSuccess;
  ok &= cudaMemcpy2D(h->w_y + lx, (lx + hs) * 2, w->w_s2, hs * 2, hs * 2, d,
                     cudaMemcpyDeviceToDevice) == cudaSuccess;
  if (w->router_bias)
    ok &= cudaMemcpy(h->bias, w->router_bias, N * 4, cudaMemcpyDeviceToDevice) == cudaSuccess;
  else
    ok &= cudaMemset(h->bias, 0, N * 4) == cudaSuccess;
  ok &= cudaMemset(h->err, 0, 4) == cudaSuccess;
  ok &= cudaMemset(h->vh, 0, Tm_b * (l + hs) * 2) == cudaSuccess;
  if (bfx || w4) {
    ok &= cudaMemset(h->u_perm, 0, rows_b * l * 2) == cudaSuccess;
    ok &= cudaMemset(h->H, 0, rows_b * hh * 2) == cudaSuccess;
  }
  ok &= cudaMemset(h->x_dev, 0, Tm_b * d * 2) == cudaSuccess;
  if (d_a > d)
    ok &= cudaMemset(h->w_y + d * (lx + hs), 0, (d_a - d) * (lx + hs) * 2) == cudaSuccess;
  // tensor maps of the fixed operands
  ok &= make_map(&h->tm_wx, h->w_x, N + lx + hs, d, GEMM_BM);
  if (bfx) {
    ok &= make_map(&h->tm_w1, h->w1, N * hh, l, GEMM_BM);
    ok &= make_map(&h->tm_w2, h->w2, N * l, hh, GEMM_BM);
  }
  ok &= make_map(&h->tm_wy, h->w_y, d_a, lx + hs, GEMM_BM);
  if (bfx || w4) {   // 2-byte rows (bf16, or f16 for W4A16)
    ok &= make_map(&h->tm_uperm.b16, h->u_perm, rows_b, l, GEMM_BROWS);
    ok &= make_map(&h->tm_uperm.b64, h->u_perm, rows_b, l, GEMM_BROWS_BIG);
    ok &= make_map(&h->tm_H.b16, h->H, rows_b, hh, GEMM_BROWS);
    ok &= make_map(&h->tm_H.b64, h->H, rows_b, hh, GEMM_BROWS_BIG);
  }
  // B operand of the y-GEMM: [v | hs], or hs alone (columns [l, l+h_s) of
  // vh, same row pitch) for the standard MoE, whose v is added in the epilogue
  ok &= make_map_strided(&h->tm_vh.b16, h->vh + (l - lx), Tm_b, lx + hs, l + hs, GEMM_BROWS);
  ok &= make_map_strided(&h->tm_vh.b64, h->vh + (l - lx), Tm_b, lx + hs, l + hs,
                         GEMM_BROWS_BIG);
  if (bfx && proj) {
    ok &= make_map(&h->tm_ws1, h->w_x + (N + lx) * d, hs, d, GEMM_BM);
    ok &= make_map_strided(&h->tm_ws2, h->w_y + lx, d_a, hs, lx + hs, GEMM_BM);
    ok &= make_map_strided(&h->tm_hs.b16, h->vh + l, Tm_b, hs, l + hs, GEMM_BROWS);
    ok &= make_map_strided(&h->tm_hs.b64, h->vh + l, Tm_b, hs, l + hs, GEMM_BROWS_BIG);
    ok &= cudaStreamCreateWithFlags(&h->side_st, cudaStreamNonBlocking) == cudaSuccess;
    ok &= cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) == cudaSuccess;
    ok &= cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) == cudaSuccess;
    ok &= set_smem_all<EpiS1>() == cudaSuccess;
    ok &= set_pair_smem<EpiS1>() == cudaSuccess;
  }
  if (bwx) {
    // MN-major operands of the backward GEMMs: 64 x 64 boxes (the same boxes
    // serve K-major token rows); padding rows read as zero
    ok &= cudaMemset(h->dxh, 0, Tm_b * (N + l + hs) * 2) == cudaSuccess;
    ok &= cudaMemset(h->dy_dev, 0, GEMM_BROWS_BIG * d * 2) == cudaSuccess;
    ok &= make_map(&h->tm_wx64, h->w_x, N + lx + hs, d, GEMM_BROWS_BIG);
    ok &= make_map(&h->tm_wy64, h->w_y, d_a, lx + hs, GEMM_BROWS_BIG);
    ok &= make_map(&h->tm_dxh.b16, h->dxh, Tm_b, N + l + hs, GEMM_BROWS);
    ok &= make_map(&h->tm_dxh.b64, h->dxh, Tm_b, N + l + hs, GEMM_BROWS_BIG);
    ok &= set_bw_dgrad_smem<EpiDVH>() == cudaSuccess;
    ok &= set_bw_dgrad_smem<EpiStore>() == cudaSuccess;
    ok &= set_bw_smem<256, true, EpiWRows>() == cudaSuccess;
    ok &= set_bw_smem<256, true, EpiWCols>() == cudaSuccess;
  }
  if (bwd) {
    // the BF16 experts' backward
    ok &= cudaMemset(h->dog, 0, rows_b * l * 2) == cudaSuccess;
    ok &= cudaMemset(h->da, 0, rows_b * hh * 2) == cudaSuccess;
    ok &= make_map(&h->tm_w1_64, h->w1, N * hh, l, GEMM_BROWS_BIG);
    ok &= make_map(&h->tm_w2_64, h->w2, N * l, hh, GEMM_BROWS_BIG);
    ok &= make_map(&h->tm_dog.b16, h->dog, rows_b, l, GEMM_BROWS);
    ok &= make_map(&h->tm_dog.b64, h->dog, rows_b, l, GEMM_BROWS_BIG);
    ok &= make_map(&h->tm_da.b16, h->da, rows_b, hh, GEMM_BROWS);
    ok &= make_map(&h->tm_da.b64, h->da, rows_b, hh, GEMM_BROWS_BIG);
    ok &= set_bw_smem<256, true, EpiWExp>() == cudaSuccess;
  }
  ok &= set_smem_all<EpiX>() == cudaSuccess;
  ok &= set_smem_all<EpiH>() == cudaSuccess;
  ok &= set_smem_all<EpiO>() == cudaSuccess;
  ok &= set_smem_all<EpiY>() == cudaSuccess;
  ok &= set_pair_smem<EpiX>() == cudaSuccess;
  ok &= set_pair_smem<EpiH>() == cudaSuccess;
  ok &= set_pair_smem<EpiO>() == cudaSuccess;
  ok &= set_pair_smem<EpiY>() == cudaSuccess;
  ok &= cudaDeviceSynchronize() == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    free_all(h);
    delete h;
    return LMOE_ERR_CUDA;
  }
  const char* pe = getenv("LMOE_PAIR");
  h->pairs = !(pe && pe[0] == '0');
  *out = h;
  return LMOE_OK;
}

void lmoe_destroy(lmoe_handle* h) {
  if (!h) return;
  DeviceGuard g(h->dev);
  cudaDeviceSynchronize();
  free_all(h);
  delete h;
}

static int overlap_sms(const lmoe_handle* h, int64_t T);

// A dense GEMM of T tokens over F output features and kblocks 64-wide K
// steps: on CTA pairs (256 x 256 tiles) when their tiles fill the GPU; for a
// single token block (decode-sized batches) on pairs with K split into enough
// slices to fill it (each pair loads half the token block that a single CTA
// would, per weight byte), when the partials fit the split-K buffer; else on
// single CTAs (plan_dense).  `ctas` counts pairs for the pair kernel.
struct DenseChoice {
  bool pair;
  int bn, ksplit;
  int ctas;
};
static DenseChoice choose_dense(const lmoe_handle* h, int64_t T, int F, int kblocks) {
  const int fb2 = (F + PAIR_BM - 1) / PAIR_BM;
  const int64_t ptiles = ((T + PAIR_BN - 1) / PAIR_BN) * fb2;
  if (h->pairs && ptiles >= h->sms / 2) return {true, PAIR_BN, 1, h->sms / 2};
  if (h->pairs && T <= PAIR_BN) {
    int64_t ks = (h->sms / 2) / ptiles;
    if (ks > 8) ks = 8;
    if (ks > kblocks / 4) ks = kblocks / 4;
    if (ks >= 2 && ks * T * F <= h->part_floats)
      return {true, PAIR_BN, static_cast<int>(ks), static_cast<int>(ptiles * ks)};
  }
  const int fb = (F + 127) / 128;
  const DensePlan p = plan_dense(T, fb, kblocks, h->sms);
  const int64_t tiles = ((T + p.bn - 1) / p.bn) * fb * p.ksplit;
  return {false, p.bn, p.ksplit, static_cast<int>(tiles < h->sms ? tiles : h->sms)};
}

int lmoe_launches_per_forward(const lmoe_handle* h, int64_t T) {
  if (!h || T < 0 || T > h->cfg.max_tokens) return LMOE_ERR_INVALID_ARG;
  if (T == 0) return 0;
  const lmoe_config& c = h->cfg;
  // a split x-GEMM's reduction replaces the router kernel: same count; the
  // segments take one kernel up to SEG_SMALL_T tokens, else three
  const DenseChoice cy = choose_dense(h, T, c.d, (h->lx + c.shared_hidden) / 64);
  const int seg = (T <= SEG_SMALL_T && c.n_experts <= 1024) ? 1 : 3;
  // an overlapped forward runs the shared expert's two GEMMs apart
  return 7 + seg + (cy.ksplit > 1) + (overlap_sms(h, T) > 0 ? 2 : 0);
}

static int prof_begin(lmoe_handle* h, int kernel, cudaStream_t st) {
  if (!h->prof) return -1;
  if (h->ev_used + 2 > h->ev.size()) return -1;   // pool full: not recorded
  const size_t i = h->ev_used;
  h->ev_used += 2;
  h->ev_kernel[i / 2] = kernel;
  cudaEventRecord(h->ev[i], st);
  return static_cast<int>(i);
}

static void prof_end(lmoe_handle* h, int slot, cudaStream_t st) {
  if (slot >= 0) cudaEventRecord(h->ev[slot + 1], st);
}

#define LMOE_STEP_ON(stream, kidx, call)             \
  do {                                               \
    const int _slot = prof_begin(h, (kidx), stream); \
    const cudaError_t _e = (call);                   \
    prof_end(h, _slot, stream);                      \
    if (_e != cudaSuccess) return LMOE_ERR_CUDA;     \
  } while (0)
#define LMOE_STEP(kidx, call) LMOE_STEP_ON(st, kidx, call)

// SMs for the shared expert on the side stream of an overlapped forward, or
// 0 for a serial one.  The idea: when the grouped GEMMs are bound by HBM
// (below about 256 flops per byte, the ratio of dense BF16 tensor throughput
// to HBM bandwidth on B200) the tensor pipes wait for the experts' weights,
// while the shared expert's dense GEMMs are bound by the tensor pipes, so the
// side stream would get the share of the SMs that makes the two take about
// the same time: (shared flops / 256) against the grouped GEMMs' weight
// bytes.  Measured at Ultra dims it loses (7.1 ms against 5.9 serial): one
// SM streams only ~43 GB/s from HBM, so the grouped GEMMs slow down on fewer
// SMs as much as the overlap saves.  So it is opt-in: LMOE_OVERLAP=-1 uses
// that share, a positive number sets the side stream's SMs, 0 or unset
// keeps the serial forward.
static int overlap_sms(const lmoe_handle* h, int64_t T) {
  const lmoe_config& c = h->cfg;
  if (!h->proj || h->fp4 || h->fp8 || h->w4 || h->ep_dense || h->shard || !h->pairs ||
      !h->side_st)
    return 0;
  int side = 0;
  if (const char* e = getenv("LMOE_OVERLAP")) side = atoi(e);
  if (side == 0) return 0;
  const double rows_per_expert = double(T) * c.top_k / c.n_experts;
  if (side < 0) {
    if (T < 1024 || rows_per_expert > 200.0) return 0;
    const double shared_flops = 4.0 * double(T) * c.d * c.shared_hidden;
    const double weight_bytes = 4.0 * double(c.n_experts) * c.expert_hidden * c.latent;
    side = static_cast<int>(h->sms * (shared_flops / 256.0) / weight_bytes + 0.5);
  }
  side &= ~1;   // CTA pairs
  if (side < 8) side = 8;
  if (side > h->sms / 2) side = h->sms / 2 & ~1;
  return side;
}

// Steps 1-5 of the forward: [W_r; W_dn; W_s1] x (logits, u, shared hidden),
// routing and the per-expert segments.
static int fwd_front(lmoe_handle* h, const void* x, int64_t T, cudaStream_t st, int side = 0) {
  const lmoe_config& c = h->cfg;
  const int64_t d = c.d;
  const int N = c.n_experts, l = c.latent, hs = c.shared_hidden, K = c.top_k;
  const int ldvh = l + hs;
  const int lx = h->lx;   // l, or 0 for the standard MoE
  const unsigned long long lim = h->wait_limit_ns;
  BMaps tm_x;
  if (T < GEMM_BROWS_BIG) {
    // fewer rows than one large TMA box: read x from the padded staging buffer
    if (x != h->x_dev &&
        cudaMemcpyAsync(h->x_dev, x, T * d * 2, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return LMOE_ERR_CUDA;
    if (!make_map(&tm_x.b16, h->x_dev, GEMM_BROWS_BIG, d, GEMM_BROWS) ||
        !make_map(&tm_x.b64, h->x_dev, GEMM_BROWS_BIG, d, GEMM_BROWS_BIG))
      return LMOE_ERR_CUDA;
  } else if (!make_map(&tm_x.b16, x, T, d, GEMM_BROWS) ||
             !make_map(&tm_x.b64, x, T, d, GEMM_BROWS_BIG)) {
    return LMOE_ERR_CUDA;
  }
  h->last_T = T;
  bool routed = false;   // the top-K ran inside the x-GEMM's split-K reduction

  // 1. [W_r; W_dn; W_s1] x: logits, u, shared hidden
  if (side > 0) {
    // overlapped: the side stream computes hs = sqrelu(W_s1 x) and then
    // ys = W_s2 hs on `side` SMs while this stream routes and runs the
    // experts on the others; [W_r; W_dn] x here
    cudaStream_t ss = h->side_st;
    if (cudaEventRecord(h->ev_fork, st) != cudaSuccess ||
        cudaStreamWaitEvent(ss, h->ev_fork, 0) != cudaSuccess)
      return LMOE_ERR_CUDA;
    {
      EpiS1 e1{h->vh, l, ldvh};
      TileSource s1{1, static_cast<int>(T), nullptr, nullptr, (hs + PAIR_BM - 1) / PAIR_BM, 0, hs,
                    static_cast<int>(d / 64), 1, nullptr, 0};
      LMOE_STEP_ON(ss, 24, launch_gemm_pair(h->tm_ws1, tm_x, s1, e1, side / 2, h->err, lim, ss));
      EpiY e2{nullptr, static_cast<int>(d), nullptr, 0, h->ys};
      TileSource s2{1, static_cast<int>(T), nullptr, nullptr,
                    static_cast<int>((d + PAIR_BM - 1) / PAIR_BM), 0, static_cast<int>(d), hs / 64,
                    1, nullptr, 0};
      LMOE_STEP_ON(ss, 25, launch_gemm_pair(h->tm_ws2, h->tm_hs, s2, e2, side / 2, h->err, lim,
                                            ss));
      if (cudaEventRecord(h->ev_join, ss) != cudaSuccess) return LMOE_ERR_CUDA;
    }
    EpiX epi{h->logits, h->u, h->vh, N, lx, l, ldvh, h->uq, h->usf, h->g_u, h->stab, h->uf8, h->r_u8,
             h->u16};
    TileSource s{1, static_cast<int>(T), nullptr, nullptr, (N + lx + PAIR_BM - 1) / PAIR_BM, 0,
                 N + lx, static_cast<int>(d / 64), 1, nullptr, 0};
    LMOE_STEP(0, launch_gemm_pair(h->tm_wx, tm_x, s, epi, (h->sms - side) / 2, h->err, lim, st));
  } else {
    const int F = N + lx + hs;
    const DenseChoice dc = choose_dense(h, T, F, static_cast<int>(d / 64));
    EpiX epi{h->logits, h->u, h->vh, N, lx, l, ldvh, h->uq, h->usf, h->g_u, h->stab, h->uf8, h->r_u8,
             h->u16};
    if (dc.ksplit > 1 && int64_t(dc.ksplit) * T * F > h->part_floats)
      return LMOE_ERR_UNSUPPORTED;   // never: the buffer is sized for every T
    if (dc.pair) {
      TileSource s{1, static_cast<int>(T), nullptr, nullptr, (F + PAIR_BM - 1) / PAIR_BM, 0, F,
                   static_cast<int>(d / 64), dc.ksplit, h->part, dc.ksplit > 1};
      LMOE_STEP(0, launch_gemm_pair(h->tm_wx, tm_x, s, epi, dc.ctas, h->err, lim, st));
    } else {
      TileSource s{1, static_cast<int>(T), nullptr, nullptr, (F + 127) / 128, 0, F,
                   static_cast<int>(d / 64), dc.ksplit, h->part, T <= dc.bn};
      LMOE_STEP(0, launch_gemm_bn(dc.bn, h->tm_wx, tm_x, s, epi, dc.ctas, h->err, lim, st));
    }
    // at split-K sizes the reduction also routes: logits, top-K, weights
    if (dc.ksplit > 1)
      LMOE_STEP(10, launch_reduce_route(h->part, dc.ksplit, static_cast<int>(T), F, N, epi,
                                        h->bias, K, h->logits, h->topk_idx, h->topk_w, st));
    routed = dc.ksplit > 1;
  }
  // 2-5. routing and segments
  const int gbn = grouped_bn(c, T);
  if (!routed)
    LMOE_STEP(1, launch_route(h->logits, h->bias, T, N, K, h->topk_idx, h->topk_w, st));
  if (T <= SEG_SMALL_T && N <= 1024) {
    LMOE_STEP(32, launch_segments_small(h->topk_idx, h->topk_w, T, N, K, gbn, h->counts,
                                        h->offsets, h->perm, h->inv, h->wrow, h->blocks,
                                        h->nblocks, h->rblock, h->err, st));
    return LMOE_OK;
  }
  LMOE_STEP(2, launch_hist(h->topk_idx, T, N, K, h->chunk, h->err, st));
  LMOE_STEP(3, launch_scan(h->chunk, T, N, h->counts, st));
  LMOE_STEP(4, launch_scatter(h->topk_idx, h->topk_w, h->chunk, h->counts, T, N, K, gbn,
                              h->offsets, h->perm, h->inv, h->wrow, h->blocks, h->nblocks,
                              h->rblock, h->err, st));
  return LMOE_OK;
}

// Step 10 of the forward: y = [W_upl | W_s2] [v ; hs] (v already in vh);
// after an overlapped front half, y = W_upl v + ys (the side stream's W_s2 hs).
static int fwd_ygemm(lmoe_handle* h, int64_t T, void* y, cudaStream_t st, bool overlapped = false) {
  const lmoe_config& c = h->cfg;
  const int64_t d = c.d;
  const int l = c.latent, hs = c.shared_hidden;
  const int ldvh = l + hs;
  const int lx = h->lx;
  const unsigned long long lim = h->wait_limit_ns;
  if (overlapped && cudaStreamWaitEvent(st, h->ev_join, 0) != cudaSuccess) return LMOE_ERR_CUDA;
  {
    const int F = static_cast<int>(d);
    const int ky = overlapped ? lx : lx + hs;   // K of the y-GEMM
    const DenseChoice dc = choose_dense(h, T, F, ky / 64);
    if (dc.ksplit > 1 && int64_t(dc.ksplit) * T * d > h->part_floats)
      return LMOE_ERR_UNSUPPORTED;   // never: the buffer is sized for every T
    EpiY epi{static_cast<bf16*>(y), static_cast<int>(d), h->proj ? nullptr : h->vh, ldvh,
             nullptr, overlapped ? h->ys : nullptr};
    if (dc.pair) {
      TileSource s{1, static_cast<int>(T), nullptr, nullptr, (F + PAIR_BM - 1) / PAIR_BM, 0, F,
                   ky / 64, dc.ksplit, h->part, dc.ksplit > 1};
      LMOE_STEP(9, launch_gemm_pair(h->tm_wy, h->tm_vh, s, epi, dc.ctas, h->err, lim, st));
    } else {
      TileSource s{1, static_cast<int>(T), nullptr, nullptr, (F + 127) / 128, 0, F, ky / 64,
                   dc.ksplit, h->part, T <= dc.bn};
      LMOE_STEP(9, launch_gemm_bn(dc.bn, h->tm_wy, h->tm_vh, s, epi, dc.ctas, h->err, lim, st));
    }
    if (dc.ksplit > 1)
      LMOE_STEP(11, launch_reduce(h->part, dc.ksplit, static_cast<int>(T), F, epi, st));
  }
  return LMOE_OK;
}

int lmoe_forward(lmoe_handle* h, const void* x, int64_t T, void* y, void* stream) {
  if (!h || T < 0 || T > h->cfg.max_tokens) return LMOE_ERR_INVALID_ARG;
  if (T == 0) return LMOE_OK;
  if (!x || !y) return LMOE_ERR_INVALID_ARG;
  if (h->shard || h->ep_dense) return LMOE_ERR_UNSUPPORTED;
  const lmoe_config& c = h->cfg;
  const int64_t d = c.d;
  const char* xb = static_cast<const char*>(x);
  const char* yb = static_cast<const char*>(y);
  if (xb < yb + T * d * 2 && yb < xb + T * d * 2) return LMOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 15)
    return LMOE_ERR_INVALID_ARG;
  DeviceGuard g(h->dev);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int l = c.latent, hh = c.expert_hidden, hs = c.shared_hidden, K = c.top_k;
  const int ldvh = l + hs;
  const unsigned long long lim = h->wait_limit_ns;
  const int side = overlap_sms(h, T);   // SMs of the shared expert's side stream, or 0
  const int gsms = h->sms - side;       // SMs of the grouped GEMMs
  int rc = fwd_front(h, x, T, st, side);
  if (rc != LMOE_OK) return rc;
  const int gbn = grouped_bn(c, T);
  if (h->w4) {
    // 6. f16 latent rows into expert order
    LMOE_STEP(5, launch_gather(h->u16, h->perm, T * K, K, l, h->u_perm, st));
    // 7. H = sqrelu(g_W1 * (W1 codes x block scales) u), weights expanded in the GEMM
    {
      TileSource s{0, 0, h->blocks, h->nblocks, hh / 128, hh, hh, l / 64, 1, nullptr,
                   gbn == 32, h->w1sf, nullptr, h->lp / 64};
      EpiH16 epi{reinterpret_cast<__half*>(h->H), h->gw1, hh};
      LMOE_STEP(6, launch_gemm_q<KIND_W4A16>(gbn, h->tm_w1c, h->tm_uperm, s, epi, h->sms,
                                             h->err, lim, st));
    }
    // 8. O = w g_W2 (W2 codes x block scales) H
    {
      TileSource s{0, 0, h->blocks, h->nblocks, l / 128, l, l, hh / 64, 1, nullptr, gbn == 32,
                   h->w2sf, nullptr, h->hp / 64};
      EpiO16 epi{h->O, h->wrow, h->gw2, l};
      LMOE_STEP(7, launch_gemm_q<KIND_W4A16>(gbn, h->tm_w2c, h->tm_H, s, epi, h->sms, h->err,
                                             lim, st));
    }
  } else if (h->fp8) {
    // 6. FP8 latent rows into expert order (rows of l bytes: l/2 bf16 units)
    LMOE_STEP(5, launch_gather(h->uf8, h->perm, T * K, K, l / 2, h->upf8, st));
    // 7. H = E4M3(sqrelu(s_W1 s_u W1q[e] uq) / s_h), kind::f8f6f4
    {
      TileSource s{0, 0, h->blocks, h->nblocks, hh / 128, hh, hh, l / 128, 1, nullptr,
                   gbn == 32};
      EpiH8 epi{h->Hf8, h->sw1, h->g_u, h->r_h8, hh};
      LMOE_STEP(6, launch_gemm_q<KIND_FP8>(gbn, h->tm_w1f8, h->tm_upf8, s, epi, h->sms, h->err,
                                           lim, st));
    }
    // 8. O = w s_W2 s_h W2q[e] Hq
    {
      TileSource s{0, 0, h->blocks, h->nblocks, l / 128, l, l, hh / 128, 1, nullptr, gbn == 32};
      EpiO8 epi{h->O, h->wrow, h->sw2, h->g_h, l};
      LMOE_STEP(7, launch_gemm_q<KIND_FP8>(gbn, h->tm_w2f8, h->tm_Hf8, s, epi, h->sms, h->err,
                                           lim, st));
    }
  } else if (h->fp4) {
    // 6. quantised latent rows (and their scales) into expert order
    LMOE_STEP(5, launch_gather_q(h->uq, h->usf, h->perm, h->rblock, T * K, K, l, h->lp, h->upq,
                                 h->sfbu, st));
    // 7. H = NVFP4(sqrelu(W1[e] u)), block-scaled FP4 MMA
    {
      TileSource s{0, 0, h->blocks, h->nblocks, hh / 128, hh, hh, h->lp / 256, 1, nullptr,
                   gbn == 32, h->w1sf, h->sfbu, h->lp / 64};
      EpiHq epi{h->Hq, h->sfbh, h->gw1, h->g_u, h->g_h, h->hp, h->stab + NVFP4_TAB};
      LMOE_STEP(6, launch_gemm_q<KIND_NVFP4>(gbn, h->tm_w1q, h->tm_upq, s, epi, h->sms, h->err, lim, st));
    }
    // 8. O = w * W2[e] H, block-scaled FP4 MMA
    {
      TileSource s{0, 0, h->blocks, h->nblocks, l / 128, l, l, h->hp / 256, 1, nullptr,
                   gbn == 32, h->w2sf, h->sfbh, h->hp / 64};
      EpiOq epi{h->O, h->wrow, h->gw2, h->g_h, l};
      LMOE_STEP(7, launch_gemm_q<KIND_NVFP4>(gbn, h->tm_w2q, h->tm_Hq, s, epi, h->sms, h->err, lim, st));
    }
  } else {
  // 6. latent rows into expert order
  LMOE_STEP(5, launch_gather(h->proj ? static_cast<const void*>(h->u) : x, h->perm, T * K, K, l,
                             h->u_perm, st));
  // 7. H = sqrelu(W1[e] u)
  {
    EpiH epi{h->H, hh};
    if (h->pairs && gbn == PAIR_BN) {
      TileSource s{0, 0, h->blocks, h->nblocks, (hh + PAIR_BM - 1) / PAIR_BM, hh, hh, l / 64, 1,
                   nullptr, 0};
      LMOE_STEP(6, launch_gemm_pair(h->tm_w1, h->tm_uperm, s, epi, gsms / 2, h->err, lim, st));
    } else {
      TileSource s{0, 0, h->blocks, h->nblocks, (hh + 127) / 128, hh, hh, l / 64, 1, nullptr,
                   gbn == 32};
      LMOE_STEP(6, launch_gemm_bn(gbn, h->tm_w1, h->tm_uperm, s, epi, gsms, h->err, lim, st));
    }
  }
  // 8. O = w * W2[e] H
  {
    EpiO epi{h->O, h->wrow, l};
    if (h->pairs && gbn == PAIR_BN) {
      TileSource s{0, 0, h->blocks, h->nblocks, (l + PAIR_BM - 1) / PAIR_BM, l, l, hh / 64, 1,
                   nullptr, 0};
      LMOE_STEP(7, launch_gemm_pair(h->tm_w2, h->tm_H, s, epi, gsms / 2, h->err, lim, st));
    } else {
      TileSource s{0, 0, h->blocks, h->nblocks, (l + 127) / 128, l, l, hh / 64, 1, nullptr,
                   gbn == 32};
      LMOE_STEP(7, launch_gemm_bn(gbn, h->tm_w2, h->tm_H, s, epi, gsms, h->err, lim, st));
    }
  }
  }
  // 9. v = sum_k O[inv[t][k]]
  LMOE_STEP(8, launch_combine(h->O, h->inv, T, K, l, h->vh, ldvh, st));
  // 10. y = [W_upl | W_s2] [v ; hs], or W_upl v + ys after the side stream
  return fwd_ygemm(h, T, y, st, side > 0);
}

static int experts_bw4(lmoe_handle* h, const void* u, const int32_t* topk_idx,
                       const float* topk_w, const void* dv, int64_t T, uint64_t seed, bf16* du,
                       int ldu, float* dw, float* d_w1, float* d_w2, cudaStream_t st);

int lmoe_backward(lmoe_handle* h, const void* x, const void* dy, int64_t T, void* dx,
                  const lmoe_grads* gr, void* stream) {
  if (!h || T < 0) return LMOE_ERR_INVALID_ARG;
  if (!h->bw && !h->bw4) return LMOE_ERR_UNSUPPORTED;
  if (T == 0) return LMOE_OK;
  if (T != h->last_T || !x || !dy || !dx || !gr || !gr->d_router || !gr->d_dn || !gr->d_w1 ||
      !gr->d_w2 || !gr->d_upl || !gr->d_s1 || !gr->d_s2)
    return LMOE_ERR_INVALID_ARG;
  const lmoe_config& c = h->cfg;
  const int64_t d = c.d;
  const char* xb = static_cast<const char*>(x);
  const char* yb = static_cast<const char*>(dy);
  const char* ob = static_cast<const char*>(dx);
  const int64_t nb = T * d * 2;
  if ((ob < xb + nb && xb < ob + nb) || (ob < yb + nb && yb < ob + nb)) return LMOE_ERR_INVALID_ARG;
  const uintptr_t align = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dy) |
                          reinterpret_cast<uintptr_t>(dx) |
                          reinterpret_cast<uintptr_t>(gr->d_router) |
                          reinterpret_cast<uintptr_t>(gr->d_dn) |
                          reinterpret_cast<uintptr_t>(gr->d_w1) |
                          reinterpret_cast<uintptr_t>(gr->d_w2) |
                          reinterpret_cast<uintptr_t>(gr->d_upl) |
                          reinterpret_cast<uintptr_t>(gr->d_s1) |
                          reinterpret_cast<uintptr_t>(gr->d_s2);
  if (align & 15) return LMOE_ERR_INVALID_ARG;
  DeviceGuard g(h->dev);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int N = c.n_experts, l = c.latent, hh = c.expert_hidden, hs = c.shared_hidden,
            K = c.top_k;
  const int ldvh = l + hs, ldx = N + l + hs;
  const int64_t R = T * K;
  const unsigned long long lim = h->wait_limit_ns;
  // dy and x as 64-row boxes (token rows, or MN-major for the weight
  // gradients); fewer than 64 rows go through the padded staging buffers
  BMaps tm_dy, tm_x;
  const void* dy_src = dy;
  const void* x_src = x;
  int64_t map_rows = T;
  if (T < GEMM_BROWS_BIG) {
    if (cudaMemcpyAsync(h->dy_dev, dy, T * d * 2, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
        (x != h->x_dev &&
         cudaMemcpyAsync(h->x_dev, x, T * d * 2, cudaMemcpyDeviceToDevice, st) != cudaSuccess))
      return LMOE_ERR_CUDA;
    dy_src = h->dy_dev;
    x_src = h->x_dev;
    map_rows = GEMM_BROWS_BIG;
  }
  if (!make_map(&tm_dy.b16, dy_src, map_rows, d, GEMM_BROWS) ||
      !make_map(&tm_dy.b64, dy_src, map_rows, d, GEMM_BROWS_BIG) ||
      !make_map(&tm_x.b64, x_src, map_rows, d, GEMM_BROWS_BIG))
    return LMOE_ERR_CUDA;
  const int dbn = bw_dense_bn(T);
  const int gbn = grouped_bn(c, T);   // the forward's token blocks
  auto grid_of = [&](int64_t tiles) { return static_cast<int>(tiles < h->sms ? tiles : h->sms); };
#define LMOE_BW(kidx, call)                          \
  do {                                               \
    const int _slot = prof_begin(h, 12 + (kidx), st); \
    const cudaError_t _e = (call);                   \
    prof_end(h, _slot, st);                          \
    if (_e != cudaSuccess) {                         \
      cudaGetLastError();                            \
      return LMOE_ERR_CUDA;                          \
    }                                                \
  } while (0)
  // 1. [dv | dhs] = dy [W_upl | W_s2]; dhs_pre = dhs * 2 sqrt(hs)
  {
    const int fb = (l + hs + 127) / 128;
    BwSource s{0, 1, static_cast<int>(T), nullptr, nullptr, 0, static_cast<int>(d / 64), fb,
               l + hs, l + hs};
    EpiDVH epi{h->dv, h->dxh, h->vh, l, ldvh, ldx, N};
    LMOE_BW(0, launch_bw_dgrad(dbn, h->tm_wy64, tm_dy.b16, tm_dy.b64, s, epi,
                            grid_of(((T + dbn - 1) / dbn) * fb), h->err, lim, st));
  }
  if (h->bw4) {
    // 2-6, NVFP4 training recipe: the routed experts' backward (their forward
    // recomputed from the saved u), du into columns [N, N+l) of dxh, dL/dw
    // per (token, slot), dW1 and dW2; then the router through those dL/dw
    const uint64_t seed = h->bw_seed;
    h->bw_seed += 8;
    const int rc = experts_bw4(h, h->u, h->topk_idx, h->topk_w, h->dv, T, seed, h->dxh + N, ldx,
                               h->dwacc, gr->d_w1, gr->d_w2, st);
    if (rc != LMOE_OK) return rc;
    LMOE_BW(5, launch_route_bw(h->logits, h->topk_idx, h->inv, h->wrow, h->dwacc, T, N, K,
                               h->dxh, ldx, true, st));
  } else {
  // 2. do[r] = w_r dv[t(r)] in expert order
  LMOE_BW(1, launch_gather_scaled(h->dv, h->perm, h->wrow, R, K, l, h->dog, st));
  // 3. dg = W2[e]^T do (bf16, into the da buffer)
  {
    BwSource s{0, 0, 0, h->blocks, h->nblocks, l, l / 64, (hh + 127) / 128, hh, hh};
    EpiStore epi{h->da, hh};
    LMOE_BW(2, launch_bw_dgrad(gbn, h->tm_w2_64, h->tm_dog.b16, h->tm_dog.b64, s, epi, h->sms,
                            h->err, lim, st));
  }
  // 3b. da = dg * 2 sqrt(g) in place, dwacc[r] = g . dg (g = the saved H row)
  LMOE_BW(11, launch_dact(h->da, h->H, R, hh, h->dwacc, st));
  // 4. du rows = W1[e]^T da
  {
    BwSource s{0, 0, 0, h->blocks, h->nblocks, hh, hh / 64, (l + 127) / 128, l, l};
    EpiStore epi{h->dup, l};
    LMOE_BW(3, launch_bw_dgrad(gbn, h->tm_w1_64, h->tm_da.b16, h->tm_da.b64, s, epi, h->sms, h->err,
                            lim, st));
  }
  // 5. du[t] = sum_k du rows (slot order) into columns [N, N+l) of dxh
  LMOE_BW(4, launch_combine(h->dup, h->inv, T, K, l, h->dxh + N, ldx, st));
  // 6. router: dz into columns [0, N) of dxh
  LMOE_BW(5, launch_route_bw(h->logits, h->topk_idx, h->inv, h->wrow, h->dwacc, T, N, K, h->dxh,
                             ldx, false, st));
  }
  // 7. dx = [dz | du | dhs_pre] [W_r; W_dn; W_s1]
  {
    const int fb = static_cast<int>((d + 127) / 128);
    BwSource s{0, 1, static_cast<int>(T), nullptr, nullptr, 0, (ldx + 63) / 64, fb,
               static_cast<int>(d), static_cast<int>(d)};
    EpiStore epi{static_cast<bf16*>(dx), static_cast<int>(d)};
    LMOE_BW(6, launch_bw_dgrad(dbn, h->tm_wx64, h->tm_dxh.b16, h->tm_dxh.b64, s, epi,
                            grid_of(((T + dbn - 1) / dbn) * fb), h->err, lim, st));
  }
  // 8. d[W_upl | W_s2] = dy^T [v | hs]  (rows d, columns l + h_s)
  {
    const int fb = (l + hs + 127) / 128, nbk = static_cast<int>((d + 255) / 256);
    BwSource s{1, 0, static_cast<int>(T), nullptr, nullptr, 0, 0, fb, l + hs, l + hs,
               1, nullptr, nbk, static_cast<int>(d), static_cast<int>(d)};
    EpiWCols epi{};
    if (!make_map_f32_out(&epi.m0, gr->d_upl, d, l) || !make_map_f32_out(&epi.m1, gr->d_s2, d, hs))
      return LMOE_ERR_CUDA;
    epi.c1 = l;
    LMOE_BW(7, (launch_bw<256, true>(h->tm_vh.b64, tm_dy.b64, tm_dy.b64, s, epi,
                                  grid_of(int64_t(fb) * nbk), h->err, lim, st)));
  }
  // 9. dW2[e] = do^T g over the expert's rows  ([l][h])
  if (!h->bw4) {
    const int fb = (hh + 127) / 128, nbk = (l + 255) / 256;
    BwSource s{1, 0, 0, nullptr, nullptr, 0, 0, fb, hh, hh, N, h->offsets, nbk, l, l};
    EpiWExp epi{};
    if (!make_map_f32_out(&epi.m, gr->d_w2, int64_t(N) * l, hh)) return LMOE_ERR_CUDA;
    epi.rows_per = l;
    LMOE_BW(8, (launch_bw<256, true>(h->tm_H.b64, h->tm_dog.b64, h->tm_dog.b64, s, epi,
                                  grid_of(int64_t(N) * fb * nbk), h->err, lim, st)));
  }
  // 10. dW1[e] = da^T u over the expert's rows  ([h][l])
  if (!h->bw4) {
    const int fb = (l + 127) / 128, nbk = (hh + 255) / 256;
    BwSource s{1, 0, 0, nullptr, nullptr, 0, 0, fb, l, l, N, h->offsets, nbk, hh, hh};
    EpiWExp epi{};
    if (!make_map_f32_out(&epi.m, gr->d_w1, int64_t(N) * hh, l)) return LMOE_ERR_CUDA;
    epi.rows_per = hh;
    LMOE_BW(9, (launch_bw<256, true>(h->tm_uperm.b64, h->tm_da.b64, h->tm_da.b64, s, epi,
                                  grid_of(int64_t(N) * fb * nbk), h->err, lim, st)));
  }
  // 11. d[W_r; W_dn; W_s1] = dxh^T x  (rows N + l + h_s, columns d)
  {
    const int fb = static_cast<int>((d + 127) / 128), nbk = (ldx + 255) / 256;
    BwSource s{1, 0, static_cast<int>(T), nullptr, nullptr, 0, 0, fb, static_cast<int>(d),
               static_cast<int>(d), 1, nullptr, nbk, ldx, ldx};
    EpiWRows epi{};
    if (!make_map_f32_out(&epi.m0, gr->d_router, N, d) ||
        !make_map_f32_out(&epi.m1, gr->d_dn, l, d) || !make_map_f32_out(&epi.m2, gr->d_s1, hs, d))
      return LMOE_ERR_CUDA;
    epi.r1 = N;
    epi.r2 = N + l;
    LMOE_BW(10, (launch_bw<256, true>(tm_x.b64, h->tm_dxh.b64, h->tm_dxh.b64, s, epi,
                                  grid_of(int64_t(fb) * nbk), h->err, lim, st)));
  }
#undef LMOE_BW
  return LMOE_OK;
}

int lmoe_bias_update(lmoe_handle* h, float rate, void* stream) {
  if (!h || h->last_T <= 0 || !(rate == rate) || rate > 3.0e38f || rate < -3.0e38f)
    return LMOE_ERR_INVALID_ARG;
  DeviceGuard g(h->dev);
  const int64_t total = h->last_T * h->cfg.top_k;
  if (launch_bias_update(h->bias, h->counts, h->cfg.n_experts, total, rate,
                         static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return LMOE_ERR_CUDA;
  }
  return LMOE_OK;
}

int lmoe_sync_status(lmoe_handle* h, void* stream) {
  if (!h) return LMOE_ERR_INVALID_ARG;
  DeviceGuard g(h->dev);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return LMOE_ERR_CUDA;
  int flag = 0;
  if (cudaMemcpy(&flag, h->err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return LMOE_ERR_CUDA;
  if (flag) {
    if (cudaMemset(h->err, 0, 4) != cudaSuccess) return LMOE_ERR_CUDA;
    return (flag & DEVERR_TIMEOUT) ? LMOE_ERR_TIMEOUT : LMOE_ERR_DEVICE;
  }
  return LMOE_OK;
}

// ---------------------------------------------------------------------------
// expert parallelism

int lmoe_forward_dispatch(lmoe_handle* h, const void* x, int64_t T, void* rows_out,
                          int32_t* counts_out, void* stream) {
  if (!h || h->shard || T < 0 || T > h->cfg.max_tokens) return LMOE_ERR_INVALID_ARG;
  if (!h->proj || h->cfg.expert_format != LMOE_FMT_BF16) return LMOE_ERR_UNSUPPORTED;
  if (!counts_out) return LMOE_ERR_INVALID_ARG;
  DeviceGuard g(h->dev);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const lmoe_config& c = h->cfg;
  if (T == 0) {
    h->last_T = 0;
    return cudaMemsetAsync(counts_out, 0, size_t(c.n_experts) * 4, st) == cudaSuccess
               ? LMOE_OK
               : LMOE_ERR_CUDA;
  }
  if (!x || !rows_out ||
      ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(rows_out)) & 15))
    return LMOE_ERR_INVALID_ARG;
  int rc = fwd_front(h, x, T, st);
  if (rc != LMOE_OK) return rc;
  // the latent rows in expert order: the send buffer of the exchange
  LMOE_STEP(5, launch_gather(h->u, h->perm, T * c.top_k, c.top_k, c.latent, rows_out, st));
  if (cudaMemcpyAsync(counts_out, h->counts, size_t(c.n_experts) * 4, cudaMemcpyDeviceToDevice,
                      st) != cudaSuccess)
    return LMOE_ERR_CUDA;
  return LMOE_OK;
}

int lmoe_forward_combine(lmoe_handle* h, const void* rows_in, int64_t T, void* y, void* stream) {
  if (!h || h->shard || T < 0 || T > h->cfg.max_tokens) return LMOE_ERR_INVALID_ARG;
  if (!h->proj || h->cfg.expert_format != LMOE_FMT_BF16) return LMOE_ERR_UNSUPPORTED;
  if (T == 0) return LMOE_OK;
  if (T != h->last_T || !rows_in || !y ||
      ((reinterpret_cast<uintptr_t>(rows_in) | reinterpret_cast<uintptr_t>(y)) & 15))
    return LMOE_ERR_INVALID_ARG;
  DeviceGuard g(h->dev);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const lmoe_config& c = h->cfg;
  // v[t] = sum_k w[t][k] o[inv[t][k]]
  LMOE_STEP(8, launch_combine_w(rows_in, h->inv, h->topk_w, T, c.top_k, c.latent, h->vh,
                                c.latent + c.shared_hidden, st));
  return fwd_ygemm(h, T, y, st);
}

int lmoe_experts_create(const lmoe_config* cfg, int32_t first_expert, int32_t n_local,
                        const void* w1, const void* w2, int64_t max_rows, lmoe_handle** out) {
  if (!out) return LMOE_ERR_INVALID_ARG;
  *out = nullptr;
  int rc = check_cfg(cfg);
  if (rc != LMOE_OK) return rc;
  if (cfg->expert_format != LMOE_FMT_BF16 || (cfg->flags & ~LMOE_FLAG_EP_DENSE))
    return LMOE_ERR_UNSUPPORTED;
  if (!w1 || !w2 || n_local <= 0 || first_expert < 0 || first_expert + n_local > cfg->n_experts ||
      max_rows < 1 || max_rows >= (int64_t(1) << 31) - 65536)
    return LMOE_ERR_INVALID_ARG;
  if (!get_encode()) return LMOE_ERR_CUDA;
  lmoe_handle* h = new (std::nothrow) lmoe_handle();
  if (!h) return LMOE_ERR_OOM;
  h->cfg = *cfg;
  h->cfg.n_experts = n_local;
  h->shard = true;
  h->first_expert = first_expert;
  h->max_rows = max_rows;
  if (cudaGetDevice(&h->dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, h->dev) != cudaSuccess) {
    delete h;
    return LMOE_ERR_CUDA;
  }
  const int64_t n = n_local, l = cfg->latent, hh = cfg->expert_hidden;
  const int64_t rows_b = max_rows < 256 ? 256 : max_rows;
  const int64_t max_blocks = max_rows / 32 + n + 1;
  struct Req {
    void** p;
    size_t bytes;
  } reqs[] = {
      {(void**)&h->w1, size_t(n * hh * l * 2)},
      {(void**)&h->w2, size_t(n * l * hh * 2)},
      {(void**)&h->counts, size_t(n * 4)},
      {(void**)&h->offsets, size_t((n + 1) * 4)},
      {(void**)&h->blocks, size_t(max_blocks * 16)},
      {(void**)&h->nblocks, size_t(4)},
      {(void**)&h->u_perm, size_t(rows_b * l * 2)},
      {(void**)&h->H, size_t(rows_b * hh * 2)},
      {(void**)&h->err, size_t(4)},
  };
  for (auto& r : reqs) {
    if ((rc = alloc_dev(h, r.p, r.bytes)) != LMOE_OK) {
      free_all(h);
      delete h;
      return rc;
    }
  }
  bool ok = cudaMemcpy(h->w1, w1, n * hh * l * 2, cudaMemcpyDeviceToDevice) == cudaSuccess;
  ok &= cudaMemcpy(h->w2, w2, n * l * hh * 2, cudaMemcpyDeviceToDevice) == cudaSuccess;
  ok &= cudaMemset(h->u_perm, 0, rows_b * l * 2) == cudaSuccess;
  ok &= cudaMemset(h->H, 0, rows_b * hh * 2) == cudaSuccess;
  ok &= cudaMemset(h->err, 0, 4) == cudaSuccess;
  ok &= make_map(&h->tm_w1, h->w1, n * hh, l, GEMM_BM);
  ok &= make_map(&h->tm_w2, h->w2, n * l, hh, GEMM_BM);
  ok &= make_map(&h->tm_uperm.b16, h->u_perm, rows_b, l, GEMM_BROWS);
  ok &= make_map(&h->tm_uperm.b64, h->u_perm, rows_b, l, GEMM_BROWS_BIG);
  ok &= make_map(&h->tm_H.b16, h->H, rows_b, hh, GEMM_BROWS);
  ok &= make_map(&h->tm_H.b64, h->H, rows_b, hh, GEMM_BROWS_BIG);
  ok &= set_smem_all<EpiH>() == cudaSuccess;
  ok &= set_smem_all<EpiO>() == cudaSuccess;
  ok &= set_pair_smem<EpiH>() == cudaSuccess;
  ok &= set_pair_smem<EpiO>() == cudaSuccess;
  ok &= cudaDeviceSynchronize() == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    free_all(h);
    delete h;
    return LMOE_ERR_CUDA;
  }
  const char* pe = getenv("LMOE_PAIR");
  h->pairs = !(pe && pe[0] == '0');
  *out = h;
  return LMOE_OK;
}

int lmoe_experts_forward(lmoe_handle* h, const void* rows, const int32_t* counts, int64_t R,
                         void* out, void* stream) {
  if (!h || !h->shard || R < 0 || R > h->max_rows || !counts) return LMOE_ERR_INVALID_ARG;
  if (R > 0 && (!rows || !out ||
                ((reinterpret_cast<uintptr_t>(rows) | reinterpret_cast<uintptr_t>(out)) & 15)))
    return LMOE_ERR_INVALID_ARG;
  const char* rb = static_cast<const char*>(rows);
  const char* ob = static_cast<const char*>(out);
  const int64_t bytes = R * h->cfg.latent * 2;
  if (R > 0 && rb < ob + bytes && ob < rb + bytes) return LMOE_ERR_INVALID_ARG;
  DeviceGuard g(h->dev);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const lmoe_config& c = h->cfg;
  const int n = c.n_experts, l = c.latent, hh = c.expert_hidden;
  const unsigned long long lim = h->wait_limit_ns;
  // counts checked on the device (>= 0, sum R) before any block is built
  LMOE_STEP(2, launch_sanitize_counts(counts, n, R, h->counts, h->err, st));
  if (R == 0) return LMOE_OK;
  const double avg = double(R) / n;
  const int gbn = avg <= 40.0 ? 32 : avg <= 160.0 ? 128 : 256;
  // offsets and token blocks of at most gbn rows per expert from the counts
  LMOE_STEP(4, launch_scatter(nullptr, nullptr, nullptr, h->counts, 0, n, 1, gbn, h->offsets,
                              nullptr, nullptr, nullptr, h->blocks, h->nblocks, nullptr, h->err,
                              st));
  // the B operand: the caller's rows, or the padded staging copy when fewer
  // rows than one TMA box of 256 rows fit
  BMaps tm_rows;
  if (R < 256) {
    if (cudaMemcpyAsync(h->u_perm, rows, bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return LMOE_ERR_CUDA;
    tm_rows = h->tm_uperm;
  } else if (!make_map(&tm_rows.b16, rows, R, l, GEMM_BROWS) ||
             !make_map(&tm_rows.b64, rows, R, l, GEMM_BROWS_BIG)) {
    return LMOE_ERR_CUDA;
  }
  {
    EpiH epi{h->H, hh};
    if (h->pairs && gbn == PAIR_BN) {
      TileSource s{0, 0, h->blocks, h->nblocks, (hh + PAIR_BM - 1) / PAIR_BM, hh, hh, l / 64, 1,
                   nullptr, 0};
      LMOE_STEP(6, launch_gemm_pair(h->tm_w1, tm_rows, s, epi, h->sms / 2, h->err, lim, st));
    } else {
      TileSource s{0, 0, h->blocks, h->nblocks, (hh + 127) / 128, hh, hh, l / 64, 1, nullptr,
                   gbn == 32};
      LMOE_STEP(6, launch_gemm_bn(gbn, h->tm_w1, tm_rows, s, epi, h->sms, h->err, lim, st));
    }
  }
  {
    EpiO epi{static_cast<bf16*>(out), nullptr, l};
    if (h->pairs && gbn == PAIR_BN) {
      TileSource s{0, 0, h->blocks, h->nblocks, (l + PAIR_BM - 1) / PAIR_BM, l, l, hh / 64, 1,
                   nullptr, 0};
      LMOE_STEP(7, launch_gemm_pair(h->tm_w2, h->tm_H, s, epi, h->sms / 2, h->err, lim, st));
    } else {
      TileSource s{0, 0, h->blocks, h->nblocks, (l + 127) / 128, l, l, hh / 64, 1, nullptr,
                   gbn == 32};
      LMOE_STEP(7, launch_gemm_bn(gbn, h->tm_w2, h->tm_H, s, epi, h->sms, h->err, lim, st));
    }
  }
  return LMOE_OK;
}

int lmoe_permute_rows(const void* src, const int32_t* idx, int64_t n, int64_t n_other,
                      int32_t row_bytes, void* dst, int scatter, void* stream) {
  if (n < 0 || n_other < 0 || row_bytes <= 0 || row_bytes % 16) return LMOE_ERR_INVALID_ARG;
  if (n == 0) return LMOE_OK;
  if (!src || !idx || !dst ||
      ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15))
    return LMOE_ERR_INVALID_ARG;
  return launch_permute_rows(src, idx, n, n_other, row_bytes, dst, scatter != 0,
                             static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LMOE_OK
             : LMOE_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// routed experts' forward and backward under the NVFP4 training recipe

// The routed experts' NVFP4 forward and backward on the handle's workspace
// (checked arguments; du rows of pitch ldu elements).
static int experts_bw4(lmoe_handle* h, const void* u, const int32_t* topk_idx,
                       const float* topk_w, const void* dv, int64_t T, uint64_t seed, bf16* du,
                       int ldu, float* dw, float* d_w1, float* d_w2, cudaStream_t st) {
  const lmoe_config& c = h->cfg;
  const int N = c.n_experts, l = c.latent, hh = c.expert_hidden, K = c.top_k;
  const int lp = h->lp, hp = h->hp;
  const int64_t R = T * K;
  const int64_t pitch = h->rp_cap;
  const unsigned long long lim = h->wait_limit_ns;
  h->bw4_T = T;
  if (T == 0) {
    // no rows: every weight gradient is zero
    if (cudaMemsetAsync(d_w1, 0, size_t(N) * hh * l * 4, st) != cudaSuccess ||
        cudaMemsetAsync(d_w2, 0, size_t(N) * l * hh * 4, st) != cudaSuccess)
      return LMOE_ERR_CUDA;
    return LMOE_OK;
  }
  if (cudaMemsetAsync(h->scal, 0, 64, st) != cudaSuccess) return LMOE_ERR_CUDA;
  float* amax = h->scal;        // 0 do, 1 da, 2 do^T, 3 g^T, 4 da^T, 5 u^T
  float* gsc = h->scal + 8;     // their global scales
  const int gbn = grouped_bn(c, T);
  // 1. segments of the given routing
  LMOE_STEP(2, launch_hist(topk_idx, T, N, K, h->chunk, h->err, st));
  LMOE_STEP(3, launch_scan(h->chunk, T, N, h->counts, st));
  LMOE_STEP(4, launch_scatter(topk_idx, topk_w, h->chunk, h->counts, T, N, K, gbn, h->offsets,
                              h->perm, h->inv, h->wrow, h->blocks, h->nblocks, h->rblock, h->err,
                              st));
  // 2. the experts' forward: u -> NVFP4, a = W1q u (kept), g = NVFP4(sqrelu a),
  //    o = W2q g (unweighted)
  LMOE_STEP(5, launch_quant_rows_bf16(u, T, l, h->g_u, h->uq, l / 2, h->usf, st));
  LMOE_STEP(5, launch_gather_q(h->uq, h->usf, h->perm, h->rblock, R, K, l, lp, h->upq, h->sfbu,
                               st));
  {
    TileSource s{0, 0, h->blocks, h->nblocks, hh / 128, hh, hh, lp / 256, 1, nullptr,
                 gbn == 32, h->w1sf, h->sfbu, lp / 64};
    EpiHq epi{h->Hq, h->sfbh, h->gw1, h->g_u, h->g_h, hp, h->stab + NVFP4_TAB, h->a16, hh};
    LMOE_STEP(6, launch_gemm_q<KIND_NVFP4>(gbn, h->tm_w1q, h->tm_upq, s, epi, h->sms, h->err, lim,
                                           st));
  }
  {
    TileSource s{0, 0, h->blocks, h->nblocks, l / 128, l, l, hp / 256, 1, nullptr, gbn == 32,
                 h->w2sf, h->sfbh, hp / 64};
    EpiOq epi{h->O, nullptr, h->gw2, h->g_h, l};
    LMOE_STEP(7, launch_gemm_q<KIND_NVFP4>(gbn, h->tm_w2q, h->tm_Hq, s, epi, h->sms, h->err, lim,
                                           st));
  }
  // 3. dL/dw = o . dv
  LMOE_STEP(26, launch_dw_rows(h->O, h->inv, dv, T, K, l, dw, st));
  // 4. do = w dv rows, stochastically rounded to NVFP4 (1D blocks along l)
  LMOE_STEP(27, launch_rows_scaled(dv, h->perm, h->wrow, R, K, l, h->do32, amax + 0, st));
  LMOE_STEP(27, launch_quant_rows_dev(h->do32, R, l, amax + 0, true, seed + 0, h->doq, lp / 2,
                                      h->doS, gsc + 0, st));
  LMOE_STEP(27, launch_atoms_rblock(h->doS, h->rblock, R, l / 16, lp / 64, h->sfbdo, st));
  // 5. dg = W2q^T Q(do); da = dg 2 max(a, 0) (fp32) and its amax
  {
    TileSource s{0, 0, h->blocks, h->nblocks, hh / 128, hh, hh, lp / 256, 1, nullptr,
                 gbn == 32, h->w2qT_sf, h->sfbdo, lp / 64};
    EpiDA epi{h->da32, h->a16, h->gw2, gsc + 0, hh, amax + 1};
    LMOE_STEP(14, launch_gemm_q<KIND_NVFP4>(gbn, h->tm_w2qT, h->tm_doq, s, epi, h->sms, h->err,
                                            lim, st));
  }
  // 6. da stochastically rounded (1D blocks along h); du rows = W1q^T Q(da)
  LMOE_STEP(28, launch_quant_rows_dev(h->da32, R, hh, amax + 1, true, seed + 1, h->daq, hp / 2,
                                      h->daS, gsc + 1, st));
  LMOE_STEP(28, launch_atoms_rblock(h->daS, h->rblock, R, hh / 16, hp / 64, h->sfbda, st));
  {
    TileSource s{0, 0, h->blocks, h->nblocks, l / 128, l, l, hp / 256, 1, nullptr, gbn == 32,
                 h->w1qT_sf, h->sfbda, hp / 64};
    EpiDU epi{h->O, h->gw1, gsc + 1, l};
    LMOE_STEP(15, launch_gemm_q<KIND_NVFP4>(gbn, h->tm_w1qT, h->tm_daq, s, epi, h->sms, h->err,
                                            lim, st));
  }
  // 7. du = sum of a token's rows
  LMOE_STEP(16, launch_combine(h->O, h->inv, T, K, l, du, ldu, st));
  // 8. weight gradients: per expert, over its rows (the K dimension),
  //    transformed operands padded to 256-row segments
  LMOE_STEP(29, launch_seg_offsets(h->counts, N, h->po16, h->po256, h->kofs, h->grp, st));
  const int64_t kc = pitch / 64;
  TSrc src_do{h->do32, nullptr, nullptr, nullptr, K, 0, 0, 0.f};
  TSrc src_g{h->Hq, nullptr, h->rblock, h->sfbh, K, hp / 2, hp / 64, h->g_h};
  TSrc src_da{h->da32, nullptr, nullptr, nullptr, K, 0, 0, 0.f};
  TSrc src_u{u, h->perm, nullptr, nullptr, K, 0, 0, 0.f};
  // dW2[e] = Q_sr(R(do_e^T)) Q(R(g_e^T))^T: A = g^T (features h), B = do^T (rows l)
  const int32_t *off = h->offsets, *cnt = h->counts, *p16 = h->po16, *p256 = h->po256,
                *grp = h->grp;
  LMOE_STEP(29, launch_tq_amax(2, src_g, off, cnt, p16, p256, grp, N, hh, pitch, seed + 2,
                               amax + 3, st));
  LMOE_STEP(29, launch_tq_amax(0, src_do, off, cnt, p16, p256, grp, N, l, pitch, seed + 2,
                               amax + 2, st));
  LMOE_STEP(29, launch_tq_quant(2, false, src_g, off, cnt, p16, p256, grp, N, hh, pitch, seed + 2,
                                amax + 3, 0, h->tq[1], h->ts[1], h->ta[1], gsc + 3, st));
  LMOE_STEP(29, launch_tq_quant(0, true, src_do, off, cnt, p16, p256, grp, N, l, pitch, seed + 2,
                                amax + 2, seed + 3, h->tq[0], h->ts[0], h->ta[0], gsc + 2, st));
  {
    TileSource s{2, 0, nullptr, nullptr, hh / 128, 0, hh, 0, 1, nullptr, 0, h->ta[1], h->ta[0],
                 static_cast<int>(kc), h->kofs, N, l};
    EpiWq epi{d_w2, l, hh, gsc + 3, gsc + 2, {}};
    if (!make_map_f32_out_sw(&epi.m, d_w2, int64_t(N) * l, hh)) return LMOE_ERR_CUDA;
    LMOE_STEP(20, launch_gemm_q<KIND_NVFP4>(128, h->tm_tA[1], h->tm_tB[0], s, epi, h->sms, h->err,
                                            lim, st));
  }
  // dW1[e] = Q_sr(R(da_e^T)) Q(R(u_e^T))^T: A = u^T (features l), B = da^T (rows h)
  LMOE_STEP(30, launch_tq_amax(1, src_u, off, cnt, p16, p256, grp, N, l, pitch, seed + 4,
                               amax + 5, st));
  LMOE_STEP(30, launch_tq_amax(0, src_da, off, cnt, p16, p256, grp, N, hh, pitch, seed + 4,
                               amax + 4, st));
  LMOE_STEP(30, launch_tq_quant(1, false, src_u, off, cnt, p16, p256, grp, N, l, pitch, seed + 4,
                                amax + 5, 0, h->tq[2], h->ts[2], h->ta[2], gsc + 5, st));
  LMOE_STEP(30, launch_tq_quant(0, true, src_da, off, cnt, p16, p256, grp, N, hh, pitch, seed + 4,
                                amax + 4, seed + 5, h->tq[3], h->ts[3], h->ta[3], gsc + 4, st));
  {
    TileSource s{2, 0, nullptr, nullptr, l / 128, 0, l, 0, 1, nullptr, 0, h->ta[2], h->ta[3],
                 static_cast<int>(kc), h->kofs, N, hh};
    EpiWq epi{d_w1, hh, l, gsc + 5, gsc + 4, {}};
    if (!make_map_f32_out_sw(&epi.m, d_w1, int64_t(N) * hh, l)) return LMOE_ERR_CUDA;
    LMOE_STEP(21, launch_gemm_q<KIND_NVFP4>(128, h->tm_tA[2], h->tm_tB[3], s, epi, h->sms, h->err,
                                            lim, st));
  }
  // experts without rows: zero gradients
  LMOE_STEP(31, launch_zero_empty(h->counts, N, int64_t(l) * hh, d_w2, st));
  LMOE_STEP(31, launch_zero_empty(h->counts, N, int64_t(hh) * l, d_w1, st));
  return LMOE_OK;
}

int lmoe_experts_backward_nvfp4(lmoe_handle* h, const void* u, const int32_t* topk_idx,
                                const float* topk_w, const void* dv, int64_t T, uint64_t seed,
                                void* du, float* dw, float* d_w1, float* d_w2, void* stream) {
  if (!h || h->shard || T < 0 || T > h->cfg.max_tokens) return LMOE_ERR_INVALID_ARG;
  if (!h->bw4) return LMOE_ERR_UNSUPPORTED;
  if (!d_w1 || !d_w2 || (T > 0 && (!u || !topk_idx || !topk_w || !dv || !du || !dw)))
    return LMOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(u) | reinterpret_cast<uintptr_t>(dv) |
       reinterpret_cast<uintptr_t>(du) | reinterpret_cast<uintptr_t>(d_w1) |
       reinterpret_cast<uintptr_t>(d_w2)) & 15)
    return LMOE_ERR_INVALID_ARG;
  DeviceGuard g(h->dev);
  return experts_bw4(h, u, topk_idx, topk_w, dv, T, seed, static_cast<bf16*>(du),
                     h->cfg.latent, dw, d_w1, d_w2, static_cast<cudaStream_t>(stream));
}

int64_t lmoe_nvfp4_bw_columns(const lmoe_handle* h) {
  if (!h) return LMOE_ERR_INVALID_ARG;
  return h->bw4 ? h->rp_cap : LMOE_ERR_UNSUPPORTED;
}

int lmoe_forward_host(lmoe_handle* h, const void* x_host, int64_t T, void* y_host, void* stream) {
  if (!h || T < 0 || T > h->cfg.max_tokens) return LMOE_ERR_INVALID_ARG;
  if (T == 0) return LMOE_OK;
  if (!x_host || !y_host) return LMOE_ERR_INVALID_ARG;
  DeviceGuard g(h->dev);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = size_t(T) * h->cfg.d * 2;
  if (cudaMemcpyAsync(h->x_dev, x_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return LMOE_ERR_CUDA;
  int rc = lmoe_forward(h, h->x_dev, T, h->y_dev, stream);
  if (rc != LMOE_OK) return rc;
  if (cudaMemcpyAsync(y_host, h->y_dev, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return LMOE_ERR_CUDA;
  return lmoe_sync_status(h, stream);
}

int lmoe_get_debug(lmoe_handle* h, int what, void* dst, size_t bytes) {
  if (!h || !dst) return LMOE_ERR_INVALID_ARG;
  if (h->shard) return LMOE_ERR_UNSUPPORTED;
  DeviceGuard g(h->dev);
  const lmoe_config& c = h->cfg;
  const int64_t T = h->last_T, K = c.top_k, N = c.n_experts, l = c.latent,
                hs = c.shared_hidden;
  const void* src = nullptr;
  size_t want = 0;
  bool strided = false;
  size_t col0 = 0, cols = 0;
  switch (what) {
    case LMOE_DBG_TOPK_IDX: src = h->topk_idx; want = T * K * 4; break;
    case LMOE_DBG_TOPK_W: src = h->topk_w; want = T * K * 4; break;
    case LMOE_DBG_COUNTS: src = h->counts; want = N * 4; break;
    case LMOE_DBG_OFFSETS: src = h->offsets; want = (N + 1) * 4; break;
    case LMOE_DBG_PERM: src = h->perm; want = T * K * 4; break;
    case LMOE_DBG_INV: src = h->inv; want = T * K * 4; break;
    case LMOE_DBG_LOGITS: src = h->logits; want = T * N * 4; break;
    case LMOE_DBG_U:
      if (!h->proj) return LMOE_ERR_INVALID_ARG;   // u is x itself
      src = h->u; want = T * l * 2; break;
    case LMOE_DBG_V: strided = true; col0 = 0; cols = l; want = T * l * 2; break;
    case LMOE_DBG_HS: strided = true; col0 = l; cols = hs; want = T * hs * 2; break;
    // quantised expert weights: NVFP4 codes, scale atoms and global scales,
    // or FP8 codes and per-tensor scales (no atoms)
    case LMOE_DBG_W1Q_CODES:
      if (h->fp8) { src = h->w1f8; want = N * c.expert_hidden * l; break; }
      src = h->w1q; want = N * c.expert_hidden * h->lp / 2; break;
    case LMOE_DBG_W1Q_SF: src = h->w1sf; want = (N * c.expert_hidden / 128) * (h->lp / 64) * 512; break;
    case LMOE_DBG_W1Q_G: src = h->fp8 ? h->sw1 : h->gw1; want = N * 4; break;
    case LMOE_DBG_W2Q_CODES:
      if (h->fp8) { src = h->w2f8; want = N * l * c.expert_hidden; break; }
      src = h->w2q; want = N * l * h->hp / 2; break;
    case LMOE_DBG_W2Q_SF: src = h->w2sf; want = (N * l / 128) * (h->hp / 64) * 512; break;
    case LMOE_DBG_BIAS: src = h->bias; want = N * 4; break;
    case LMOE_DBG_W2Q_G: src = h->fp8 ? h->sw2 : h->gw2; want = N * 4; break;
    case LMOE_DBG_DV:
      if (!h->dv) return LMOE_ERR_INVALID_ARG;
      src = h->dv; want = T * l * 2; break;
    case LMOE_DBG_SCALE_TABLES:
      if (!h->fp4) return LMOE_ERR_INVALID_ARG;
      src = h->stab; want = 2 * NVFP4_TAB * 4; break;
    default: break;
  }
  if (what >= LMOE_DBG_BW4_DO_CODES && what <= LMOE_DBG_BW4_DA) {
    // the last lmoe_experts_backward_nvfp4
    if (!h->bw4 || h->bw4_T < 0) return LMOE_ERR_INVALID_ARG;
    const int64_t R = h->bw4_T * K, hh = c.expert_hidden, pc = h->rp_cap;
    switch (what) {
      case LMOE_DBG_BW4_DO_CODES: strided = true; want = R * l / 2; break;
      case LMOE_DBG_BW4_DO_SF: src = h->doS; want = R * l / 16; break;
      case LMOE_DBG_BW4_DOT_CODES: src = h->tq[0]; want = l * pc / 2; break;
      case LMOE_DBG_BW4_DOT_SF: src = h->ts[0]; want = l * pc / 16; break;
      case LMOE_DBG_BW4_UT_CODES: src = h->tq[2]; want = l * pc / 2; break;
      case LMOE_DBG_BW4_UT_SF: src = h->ts[2]; want = l * pc / 16; break;
      case LMOE_DBG_BW4_SCALES: src = h->scal; want = 64; break;
      case LMOE_DBG_BW4_SEG: want = 2 * (N + 1) * 4; break;
      case LMOE_DBG_BW4_DA: src = h->da32; want = R * hh * 4; break;
    }
    if (bytes != want) return LMOE_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return LMOE_ERR_CUDA;
    if (want == 0) return LMOE_OK;
    cudaError_t e;
    if (what == LMOE_DBG_BW4_DO_CODES)
      e = cudaMemcpy2D(dst, l / 2, h->doq, h->lp / 2, l / 2, R, cudaMemcpyDeviceToHost);
    else if (what == LMOE_DBG_BW4_SEG)
      e = cudaMemcpy(dst, h->po16, (N + 1) * 4, cudaMemcpyDeviceToHost) == cudaSuccess
              ? cudaMemcpy(static_cast<char*>(dst) + (N + 1) * 4, h->po256, (N + 1) * 4,
                           cudaMemcpyDeviceToHost)
              : cudaErrorUnknown;
    else
      e = cudaMemcpy(dst, src, want, cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
  }
  if (!src && !strided) return LMOE_ERR_INVALID_ARG;
  if (what >= LMOE_DBG_W1Q_CODES && what <= LMOE_DBG_W2Q_G && !h->fp4 && !h->fp8 && !h->w4)
    return LMOE_ERR_INVALID_ARG;
  if ((what == LMOE_DBG_W1Q_SF || what == LMOE_DBG_W2Q_SF) && !h->fp4 && !h->w4)
    return LMOE_ERR_INVALID_ARG;
  if (bytes != want) return LMOE_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return LMOE_ERR_CUDA;
  if (want == 0) return LMOE_OK;
  cudaError_t e;
  if (strided)
    e = cudaMemcpy2D(dst, cols * 2, h->vh + col0, (l + hs) * 2, cols * 2, T,
                     cudaMemcpyDeviceToHost);
  else
    e = cudaMemcpy(dst, src, want, cudaMemcpyDeviceToHost);
  return e == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

int lmoe_profile_enable(lmoe_handle* h, int on) {
  if (!h) return LMOE_ERR_INVALID_ARG;
  DeviceGuard g(h->dev);
  if (on && h->ev.empty()) {
    const size_t pairs = 4096;
    h->ev.resize(2 * pairs);
    h->ev_kernel.assign(pairs, 0);
    for (auto& e : h->ev)
      if (cudaEventCreate(&e) != cudaSuccess) return LMOE_ERR_CUDA;
  }
  h->prof = on != 0;
  return LMOE_OK;
}

int lmoe_profile_read(lmoe_handle* h, const char** names, double* total_ms, int64_t* launches,
                      int max, int reset) {
  if (!h || max < 0) return LMOE_ERR_INVALID_ARG;
  DeviceGuard g(h->dev);
  if (cudaDeviceSynchronize() != cudaSuccess) return LMOE_ERR_CUDA;
  for (size_t i = 0; i + 1 < h->ev_used; i += 2) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, h->ev[i], h->ev[i + 1]) != cudaSuccess) return LMOE_ERR_CUDA;
    h->prof_ms[h->ev_kernel[i / 2]] += ms;
    h->prof_n[h->ev_kernel[i / 2]] += 1;
  }
  h->ev_used = 0;
  const int n = max < kNumKernels ? max : kNumKernels;
  for (int k = 0; k < n; ++k) {
    if (names) names[k] = kKernelNames[k];
    if (total_ms) total_ms[k] = h->prof_ms[k];
    if (launches) launches[k] = h->prof_n[k];
  }
  if (reset)
    for (int k = 0; k < kNumKernels; ++k) {
      h->prof_ms[k] = 0;
      h->prof_n[k] = 0;
    }
  return n;
}

size_t lmoe_route_workspace_size(int64_t T, int32_t N) {
  if (T < 0 || N <= 0) return 0;
  const int64_t C = (T + 31) / 32;
  const int64_t rows = T * 32;   // K <= 32
  return align256(C * N * 4) + align256(rows * 4) + align256((rows / 32 + N + 1) * 16) +
         align256(4) + align256(4);
}

int lmoe_route(const float* logits, const float* bias, int64_t T, int32_t N, int32_t K,
               int32_t* topk_idx, float* topk_w, int32_t* counts, int32_t* offsets,
               int32_t* perm, int32_t* inv, void* workspace, size_t workspace_bytes,
               void* stream) {
  if (T < 0 || N <= 0 || K <= 0 || K > N) return LMOE_ERR_INVALID_ARG;
  if (N % 32 || N > 1024 || K > 32) return LMOE_ERR_UNSUPPORTED;
  if (T * K >= (int64_t(1) << 31)) return LMOE_ERR_UNSUPPORTED;
  if (!counts || !offsets || (T > 0 && (!logits || !topk_idx || !topk_w || !perm || !inv)))
    return LMOE_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < lmoe_route_workspace_size(T, N) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255))
    return LMOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t C = (T + 31) / 32;
  const int64_t rows = T * 32;
  char* ws = static_cast<char*>(workspace);
  int32_t* chunk = reinterpret_cast<int32_t*>(ws);
  ws += align256(C * N * 4);
  float* wrow = reinterpret_cast<float*>(ws);
  ws += align256(rows * 4);
  int4* blocks = reinterpret_cast<int4*>(ws);
  ws += align256((rows / 32 + N + 1) * 16);
  int32_t* nblocks = reinterpret_cast<int32_t*>(ws);
  ws += align256(4);
  int* err = reinterpret_cast<int*>(ws);
  if (cudaMemsetAsync(err, 0, 4, st) != cudaSuccess) return LMOE_ERR_CUDA;
  if (T == 0) {
    if (cudaMemsetAsync(counts, 0, N * 4, st) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, (N + 1) * 4, st) != cudaSuccess)
      return LMOE_ERR_CUDA;
    return LMOE_OK;
  }
  if (launch_route(logits, bias, T, N, K, topk_idx, topk_w, st) != cudaSuccess) return LMOE_ERR_CUDA;
  if (T <= SEG_SMALL_T)
    return launch_segments_small(topk_idx, topk_w, T, N, K, 256, counts, offsets, perm, inv, wrow,
                                 blocks, nblocks, nullptr, err, st) == cudaSuccess
               ? LMOE_OK
               : LMOE_ERR_CUDA;
  if (launch_hist(topk_idx, T, N, K, chunk, err, st) != cudaSuccess ||
      launch_scan(chunk, T, N, counts, st) != cudaSuccess ||
      launch_scatter(topk_idx, topk_w, chunk, counts, T, N, K, 256, offsets, perm, inv, wrow,
                     blocks, nblocks, nullptr, err, st) != cudaSuccess)
    return LMOE_ERR_CUDA;
  return LMOE_OK;
}

int lmoe_route_status(const void* workspace, int64_t T, int32_t N, void* stream) {
  if (T < 0 || N <= 0 || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return LMOE_ERR_INVALID_ARG;
  const int64_t C = (T + 31) / 32;
  const int64_t rows = T * 32;
  const char* ws = static_cast<const char*>(workspace) + align256(C * N * 4) +
                   align256(rows * 4) + align256((rows / 32 + N + 1) * 16) + align256(4);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return LMOE_ERR_CUDA;
  int flag = 0;
  if (cudaMemcpy(&flag, ws, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return LMOE_ERR_CUDA;
  return flag ? LMOE_ERR_DEVICE : LMOE_OK;
}

int lmoe_nvfp4_quantize(const float* x, int64_t rows, int32_t cols, float g, uint8_t* codes,
                        uint8_t* scales, void* stream) {
  if (rows < 0 || cols <= 0 || cols % 16 || !(g >= 0.0f && g < 3.0e38f))
    return LMOE_ERR_INVALID_ARG;
  if (rows == 0) return LMOE_OK;
  if (!x || !codes || !scales || (reinterpret_cast<uintptr_t>(x) & 15) ||
      (reinterpret_cast<uintptr_t>(codes) & 7))
    return LMOE_ERR_INVALID_ARG;
  return launch_quant_rows(x, rows, cols, g, codes, scales, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? LMOE_OK
             : LMOE_ERR_CUDA;
}

int lmoe_rht16(const float* x, int64_t rows, int32_t cols, uint64_t seed, float* y,
               void* stream) {
  if (rows < 0 || cols <= 0 || cols % 16) return LMOE_ERR_INVALID_ARG;
  if (rows == 0) return LMOE_OK;
  if (!x || !y || ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 15))
    return LMOE_ERR_INVALID_ARG;
  return launch_rht16(x, rows, cols, seed, y, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LMOE_OK
             : LMOE_ERR_CUDA;
}

int lmoe_nvfp4_quantize_sr(const float* x, int64_t rows, int32_t cols, float g, uint64_t seed,
                           uint8_t* codes, uint8_t* scales, void* stream) {
  if (rows < 0 || cols <= 0 || cols % 16 || !(g >= 0.0f && g < 3.0e38f))
    return LMOE_ERR_INVALID_ARG;
  if (rows == 0) return LMOE_OK;
  if (!x || !codes || !scales || (reinterpret_cast<uintptr_t>(x) & 15) ||
      (reinterpret_cast<uintptr_t>(codes) & 7))
    return LMOE_ERR_INVALID_ARG;
  return launch_quant_rows_sr(x, rows, cols, g, seed, codes, scales,
                              static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LMOE_OK
             : LMOE_ERR_CUDA;
}

int lmoe_check_bounded_wait(int64_t limit_ns) {
  if (limit_ns < 1000 || limit_ns > 10000000000ll) return LMOE_ERR_INVALID_ARG;
  int* err = nullptr;
  if (cudaMalloc(&err, 4) != cudaSuccess) return LMOE_ERR_OOM;
  int flag = 0;
  bool ok = cudaMemset(err, 0, 4) == cudaSuccess &&
            launch_wait_probe(err, static_cast<unsigned long long>(limit_ns), 0) == cudaSuccess &&
            cudaDeviceSynchronize() == cudaSuccess &&
            cudaMemcpy(&flag, err, 4, cudaMemcpyDeviceToHost) == cudaSuccess;
  cudaFree(err);
  if (!ok) return LMOE_ERR_CUDA;
  return (flag & DEVERR_TIMEOUT) ? LMOE_ERR_TIMEOUT : LMOE_OK;
}

}  // extern "C"
