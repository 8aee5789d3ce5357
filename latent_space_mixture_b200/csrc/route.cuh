// Warp-level top-K of the sigmoid router with expert biasing ("Nemotron-3
// Super 精读报告", table 6.3: 路由机制 Sigmoid + Expert Biasing): one warp per
// token, the token's N logits held by its lanes (expert e = lane + 32 i).
// scores s = sigmoid(z), keys s + b; the K largest keys (ties to the lower
// expert id, slots key-descending); weights s_sel / sum(s_sel) from the
// unbiased scores.  Used by the standalone router kernel (k_route) and by the
// split-K reduction of the router GEMM, which computes the logits itself.
#pragma once
#include <cstdint>

namespace lmoe {

// Each candidate is packed into one 64-bit word: the key's bits mapped to an
// unsigned order (high half) and 0xFFFFFFFF - expert (low half), so that the
// largest word is the largest key and, among equal keys, the lowest expert id.
__device__ __forceinline__ uint64_t pack_key(float key, int e) {
  uint32_t b = __float_as_uint(key);
  b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return (static_cast<uint64_t>(b) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(e));
}

// Warp maximum of 64-bit words with two 32-bit reductions: the high halves,
// then the low halves among the lanes holding the high maximum.
__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
  const uint32_t hi = static_cast<uint32_t>(v >> 32);
  const uint32_t mhi = __reduce_max_sync(0xffffffffu, hi);
  const uint32_t lo = hi == mhi ? static_cast<uint32_t>(v) : 0u;
  const uint32_t mlo = __reduce_max_sync(0xffffffffu, lo);
  return (static_cast<uint64_t>(mhi) << 32) | mlo;
}

// compare-exchange for a descending sort network
__device__ __forceinline__ void cas_desc(uint64_t& a, uint64_t& b) {
  const uint64_t hi = a > b ? a : b;
  const uint64_t lo = a > b ? b : a;
  a = hi;
  b = lo;
}

// The selection of one token, all 32 lanes of the warp converged.  zz[i]: the
// logit of expert lane + 32 i (i < npl = N / 32), bb[i] its bias; z_row: the
// token's logits in memory (already written and visible to the warp), from
// which the selected experts' scores are recomputed with the same
// expression.  Lanes k < K write slot k of topk_idx / topk_w (row t).
template <int NPL>
__device__ __forceinline__ void route_select(const float (&zz)[NPL], const float (&bb)[NPL],
                                             int npl, const float* z_row, int K, int lane,
                                             int64_t t, int32_t* __restrict__ topk_idx,
                                             float* __restrict__ topk_w) {
  uint64_t cand[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    cand[i] = 0;   // below every packed key
    if (i < npl) {
      const float sc = 1.0f / (1.0f + expf(-zz[i]));
      cand[i] = pack_key(sc + bb[i], lane + 32 * i);
    }
  }
  // sort the lane's candidates descending (bitonic network on registers)
#pragma unroll
  for (int k = 2; k <= NPL; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        const int p = i ^ j;
        if (p > i) {
          if ((i & k) == 0) cas_desc(cand[i], cand[p]);
          else cas_desc(cand[p], cand[i]);
        }
      }
    }
  }
  // K rounds: the warp maximum of the lanes' heads; the winner shifts its list
  int my_e = 0;
  for (int k = 0; k < K; ++k) {
    const uint64_t win = warp_max_u64(cand[0]);
    if (lane == k) my_e = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(win));
    if (cand[0] == win) {
#pragma unroll
      for (int i = 0; i + 1 < NPL; ++i) cand[i] = cand[i + 1];
      cand[NPL - 1] = 0;
    }
  }
  // weights: the unbiased scores of the selected experts, renormalised
  const float my_s = (lane < K) ? 1.0f / (1.0f + expf(-z_row[my_e])) : 0.0f;
  float sum = 0.0f;
  for (int k = 0; k < K; ++k) sum += __shfl_sync(0xffffffffu, my_s, k);
  if (lane < K) {
    topk_idx[t * K + lane] = my_e;
    topk_w[t * K + lane] = __fdiv_rn(my_s, sum);
  }
}

}  // namespace lmoe
