// Non-GEMM kernels of the LatentMoE layer backward pass and the aux-loss-free
// bias update.
//
// The layer is that of "NVIDIA Nemotron 3: Efficient and Open Intelligence"
// (section 三 eq.(1), section 五) with the router of "Nemotron-3 Super 精读报告"
// table 6.3 (Sigmoid + Expert Biasing, aux-loss-free balancing with update
// rate 1e-3).  The backward is the exact derivative of the forward; the top-K
// selection is piecewise constant, so the router's gradient flows through the
// renormalised weights w_k = s_k / Z, Z = sum of the selected scores:
//   ds_k = (dw_k - sum_j w_j dw_j) / Z,   dz_k = ds_k s_k (1 - s_k).
#include <cuda_bf16.h>

#include "kernels.h"
#include "launch.cuh"
#include "ptx.cuh"

namespace lmoe {

// ---------------------------------------------------------------------------
// do[r] = w[r] dv[perm[r] / K]: the gradient of the expert output rows, in
// expert order.  One warp per routed row, 8 bf16 per lane-step.
__global__ void __launch_bounds__(256) k_gather_scaled(const uint4* __restrict__ dv,
                                                       const int32_t* __restrict__ perm,
                                                       const float* __restrict__ wrow,
                                                       int64_t rows, int K, int l8,
                                                       uint4* __restrict__ dst) {
  pdl_wait();
  pdl_trigger();
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += nwarps) {
    const int64_t tok = perm[r] / K;
    const float w = wrow[r];
    const uint4* src = dv + tok * l8;
    uint4* out = dst + r * l8;
    for (int i = lane; i < l8; i += 32) {
      uint4 a = src[i];
      __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&a);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(p[j]);
        p[j] = __floats2bfloat162_rn(f.x * w, f.y * w);
      }
      out[i] = a;
    }
  }
}

cudaError_t launch_gather_scaled(const void* dv, const int32_t* perm, const float* wrow,
                                 int64_t rows, int K, int l, void* dst, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  int64_t blocks = (rows + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  return launch_pdl(k_gather_scaled, static_cast<unsigned>(blocks), 256, 0, st,
                    static_cast<const uint4*>(dv), perm, wrow, rows, K, l / 8,
                    static_cast<uint4*>(dst));
}

// ---------------------------------------------------------------------------
// Activation derivative of the experts, one warp per routed row r: with
// dg = W2[e]^T do_r (bf16, in `da`) and g = sqrelu(a) the saved hidden row,
// da = dg * 2 max(a, 0) = dg * 2 sqrt(g) (in place), and
// dwacc[r] = sum_h g[h] dg[h] (lane-strided sums, then a butterfly: a fixed
// order).
__global__ void __launch_bounds__(256) k_dact(uint4* __restrict__ da,
                                              const uint4* __restrict__ H, int64_t rows, int h8,
                                              float* __restrict__ dwacc) {
  pdl_wait();
  pdl_trigger();
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += nwarps) {
    uint4* drow = da + r * h8;
    const uint4* grow = H + r * h8;
    float acc = 0.0f;
    for (int i = lane; i < h8; i += 32) {
      uint4 dv = drow[i];
      const uint4 gv = grow[i];
      __nv_bfloat162* dp = reinterpret_cast<__nv_bfloat162*>(&dv);
      const __nv_bfloat162* gp = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 d = __bfloat1622float2(dp[j]);
        const float2 g = __bfloat1622float2(gp[j]);
        acc = fmaf(g.x, d.x, acc);
        acc = fmaf(g.y, d.y, acc);
        dp[j] = __floats2bfloat162_rn(d.x * (2.0f * sqrtf(g.x)), d.y * (2.0f * sqrtf(g.y)));
      }
      drow[i] = dv;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) dwacc[r] = acc;
  }
}

cudaError_t launch_dact(void* da, const void* H, int64_t rows, int h, float* dwacc,
                        cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  int64_t blocks = (rows + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  return launch_pdl(k_dact, static_cast<unsigned>(blocks), 256, 0, st, static_cast<uint4*>(da),
                    static_cast<const uint4*>(H), rows, h / 8, dwacc);
}

// ---------------------------------------------------------------------------
// Router backward, one warp per token.  dwacc[r] = sum_h g_r[h] dg_r[h] for
// the routed row r (dg_r the gradient of the expert hidden activation under
// the weighted output gradient do_r = w_r dv), so dL/dw_r = dwacc[r] / w_r
// and sum_k w_k dL/dw_k = sum_k dwacc[r_k].
// Writes dz (bf16) into columns [0, N) of the row of dxh: zero except at the
// selected experts.
__global__ void __launch_bounds__(256) k_route_bw(const float* __restrict__ logits,
                                                  const int32_t* __restrict__ topk_idx,
                                                  const int32_t* __restrict__ inv,
                                                  const float* __restrict__ wrow,
                                                  const float* __restrict__ dwacc, int64_t T,
                                                  int N, int K,
                                                  __nv_bfloat16* __restrict__ dxh, int ldx,
                                                  bool direct) {
  pdl_wait();
  pdl_trigger();
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  __nv_bfloat16* row = dxh + t * ldx;
  const __nv_bfloat16 zero = __float2bfloat16_rn(0.0f);
  for (int e = lane; e < N; e += 32) row[e] = zero;
  int e = 0;
  float s = 0.0f, acc = 0.0f, w = 1.0f, dwd = 0.0f;
  if (lane < K) {
    e = topk_idx[t * K + lane];
    const int r = inv[t * K + lane];
    // the score from the same logit and expression as the forward router
    s = 1.0f / (1.0f + expf(-logits[t * N + e]));
    w = wrow[r];
    if (direct) {
      // dL/dw of the slot itself; the weighted sum below takes w dL/dw
      const float dwv = dwacc[t * K + lane];
      acc = w * dwv;
      dwd = dwv;
    } else {
      acc = dwacc[r];
    }
  }
  float Z = 0.0f, m = 0.0f;
  for (int k = 0; k < K; ++k) {   // slot order, as the forward's sum of scores
    Z += __shfl_sync(0xffffffffu, s, k);
    m += __shfl_sync(0xffffffffu, acc, k);
  }
  __syncwarp();
  if (lane < K) {
    // w = 0 only when the selected score underflowed (s = 0); then dz = 0
    // whatever dw is, so 0 stands in for the 0/0 quotient
    const float dw = direct ? dwd : w > 0.0f ? acc / w : 0.0f;
    const float ds = (dw - m) / Z;
    row[e] = __float2bfloat16_rn(ds * s * (1.0f - s));
  }
}

cudaError_t launch_route_bw(const float* logits, const int32_t* topk_idx, const int32_t* inv,
                            const float* wrow, const float* dwacc, int64_t T, int N, int K,
                            void* dxh, int ldx, bool direct, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((T + 7) / 8);
  return launch_pdl(k_route_bw, blocks, 256, 0, st, logits, topk_idx, inv, wrow, dwacc, T, N, K,
                    static_cast<__nv_bfloat16*>(dxh), ldx, direct);
}

// ---------------------------------------------------------------------------
// Aux-loss-free balancing: b_e += rate * sign(total - N c_e), i.e. experts
// above the mean load c = total / N lose `rate`, those below gain it (float32
// arithmetic as the bias is stored).  total = sum of counts (T K).
__global__ void k_bias_update(float* __restrict__ bias, const int32_t* __restrict__ counts,
                              int N, int64_t total, float rate) {
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= N) return;
  const int64_t diff = total - static_cast<int64_t>(N) * counts[e];
  const float sign = diff > 0 ? 1.0f : diff < 0 ? -1.0f : 0.0f;
  bias[e] = __fadd_rn(bias[e], __fmul_rn(rate, sign));
}

cudaError_t launch_bias_update(float* bias, const int32_t* counts, int N, int64_t total, float rate,
                               cudaStream_t st) {
  return launch_pdl(k_bias_update, static_cast<unsigned>((N + 255) / 256), 256, 0, st, bias,
                    counts, N, total, rate);
}

}  // namespace lmoe
