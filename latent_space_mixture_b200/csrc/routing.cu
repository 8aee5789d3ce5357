// Routing, per-expert segments, row gather and latent combine of the LatentMoE
// forward pass.
//
// Router: sigmoid scores with expert biasing ("Nemotron-3 Super 精读报告",
// table 6.3: 路由机制 Sigmoid + Expert Biasing), top-K per token and weights
// renormalised to sum 1; the gating stays at width d ("NVIDIA Nemotron 3:
// Efficient and Open Intelligence", section 五 架构实现要点).  The bias enters
// the selection only.
//
// Segments: rows ordered by expert, then token (a stable counting sort of the
// routed (token, slot) pairs), built deterministically without atomics on
// global memory: per 32-token chunk a bitmask per expert gives each token's
// rank inside the chunk, a column scan over chunks gives the chunk's base.
#include <atomic>
#include <cfloat>
#include <climits>
#include <cuda_bf16.h>

#include "kernels.h"
#include "launch.cuh"
#include "ptx.cuh"
#include "route.cuh"

namespace lmoe {

// ---------------------------------------------------------------------------
// router: one warp per token, logits read from memory (route.cuh selects)

template <int NPL>   // upper bound of experts per lane (N <= 32 NPL), a power of 2
__global__ void __launch_bounds__(256) k_route(const float* __restrict__ logits,
                                               const float* __restrict__ bias, int64_t T, int N,
                                               int K, int32_t* __restrict__ topk_idx,
                                               float* __restrict__ topk_w) {
  pdl_wait();
  pdl_trigger();
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const float* z = logits + t * N;
  const int npl = N >> 5;   // experts per lane: e = lane + 32 i
  float zz[NPL], bb[NPL];
  // all loads first (independent), then the arithmetic
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    zz[i] = (i < npl) ? z[lane + 32 * i] : 0.0f;
    bb[i] = (i < npl && bias) ? bias[lane + 32 * i] : 0.0f;
  }
  route_select<NPL>(zz, bb, npl, z, K, lane, t, topk_idx, topk_w);
}

cudaError_t launch_route(const float* logits, const float* bias, int64_t T, int N, int K,
                         int32_t* topk_idx, float* topk_w, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((T + 7) / 8);
  if (N <= 32 * 4)
    return launch_pdl(k_route<4>, blocks, 256, 0, st, logits, bias, T, N, K, topk_idx, topk_w);
  if (N <= 32 * 16)
    return launch_pdl(k_route<16>, blocks, 256, 0, st, logits, bias, T, N, K, topk_idx, topk_w);
  return launch_pdl(k_route<32>, blocks, 256, 0, st, logits, bias, T, N, K, topk_idx, topk_w);
}

// ---------------------------------------------------------------------------
// per-chunk expert masks and histograms (chunk = 32 tokens = one warp)

__device__ __forceinline__ void build_chunk_masks(uint32_t* m, const int32_t* __restrict__ idx,
                                                  int64_t c, int64_t T, int N, int K, int lane,
                                                  int* err) {
  for (int e = lane; e < N; e += 32) m[e] = 0u;
  __syncwarp();
  const int64_t t = c * 32 + lane;
  if (t < T) {
    int ek[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) ek[k] = (k < K) ? idx[t * K + k] : 0;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      if (k < K) {
        if (ek[k] < 0 || ek[k] >= N) {
          atomicOr(err, DEVERR_BAD_INDEX);
        } else {
          atomicOr(&m[ek[k]], 1u << lane);
        }
      }
    }
  }
  __syncwarp();
}

__global__ void __launch_bounds__(256) k_hist(const int32_t* __restrict__ idx, int64_t T, int N,
                                              int K, int32_t* __restrict__ chunk_cnt, int* err) {
  extern __shared__ uint32_t hist_masks[];
  pdl_wait();
  pdl_trigger();
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + w;
  const int64_t nchunks = (T + 31) / 32;
  if (c >= nchunks) return;
  uint32_t* m = hist_masks + w * N;
  build_chunk_masks(m, idx, c, T, N, K, lane, err);
  for (int e = lane; e < N; e += 32) chunk_cnt[c * N + e] = __popc(m[e]);
}

cudaError_t launch_hist(const int32_t* topk_idx, int64_t T, int N, int K, int32_t* chunk_cnt,
                        int* err, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  const int64_t nchunks = (T + 31) / 32;
  const unsigned blocks = static_cast<unsigned>((nchunks + 7) / 8);
  return launch_pdl(k_hist, blocks, 256, 8 * N * sizeof(uint32_t), st, topk_idx, T, N, K,
                    chunk_cnt, err);
}

// ---------------------------------------------------------------------------
// exclusive column scan of chunk_cnt over chunks; 32 experts per block

__global__ void __launch_bounds__(1024) k_scan(int32_t* __restrict__ chunk, int64_t C, int N,
                                               int32_t* __restrict__ counts) {
  __shared__ int32_t tile[32][33];
  pdl_wait();
  pdl_trigger();
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int e0 = blockIdx.x * 32;
  int carry = 0;   // running total of expert e0 + ty (held by warp ty)
  for (int64_t g = 0; g < C; g += 32) {
    const int64_t c = g + ty;
    tile[ty][tx] = (c < C) ? chunk[c * N + e0 + tx] : 0;
    __syncthreads();
    // warp ty scans expert column ty over the 32 chunks of this group
    const int v = tile[tx][ty];
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (tx >= off) incl += o;
    }
    tile[tx][ty] = carry + incl - v;
    carry += __shfl_sync(0xffffffffu, incl, 31);
    __syncthreads();
    if (c < C) chunk[c * N + e0 + tx] = tile[ty][tx];
    __syncthreads();
  }
  if (tx == 0) counts[e0 + ty] = carry;
}

cudaError_t launch_scan(int32_t* chunk_cnt, int64_t T, int N, int32_t* counts, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  const int64_t C = (T + 31) / 32;
  return launch_pdl(k_scan, N / 32, dim3(32, 32), 0, st, chunk_cnt, C, N, counts);
}

// ---------------------------------------------------------------------------
// offsets, perm / inv / row weights, and the token-block list

// Exclusive prefix of `v` over the NW x 32 threads of the block (wsum: 2 NW
// ints of shared memory).
template <int NW>
__device__ __forceinline__ int block_excl_scan(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) wsum[w] = incl;
  __syncthreads();
  if (w == 0) {
    int s = (lane < NW) ? wsum[lane] : 0;
    int si = s;
#pragma unroll
    for (int off = 1; off < NW; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, si, off);
      if (lane >= off) si += o;
    }
    if (lane < NW) wsum[NW + lane] = si - s;
    if (lane == NW - 1) *total = si;
  }
  __syncthreads();
  const int r = wsum[NW + w] + incl - v;
  __syncthreads();
  return r;
}

// Expert offsets (exclusive scan of the counts, EPT experts per thread of an
// NW-warp block: N <= 32 NW EPT) and each expert's first token block, into
// shared memory; with `write`, also the offsets, the list of token blocks of
// at most bn rows per expert (in expert order) and its length.
template <int EPT, int NW>
__device__ __forceinline__ void seg_offsets(const int (&cnt)[EPT], int N, int bn, int32_t* off,
                                            int32_t* bbase, bool write, int32_t* offsets,
                                            int4* blocks, int32_t* nblocks, int* wsum,
                                            int* total) {
  const int e0 = threadIdx.x * EPT;
  int sc = 0;
#pragma unroll
  for (int i = 0; i < EPT; ++i) sc += cnt[i];
  int base = block_excl_scan<NW>(sc, wsum, total);
#pragma unroll
  for (int i = 0; i < EPT; ++i) {
    if (e0 + i < N) off[e0 + i] = base;
    base += cnt[i];
  }
  if (threadIdx.x == 0) off[N] = *total;
  __syncthreads();
  int nb[EPT];
  int snb = 0;
#pragma unroll
  for (int i = 0; i < EPT; ++i) {
    nb[i] = (cnt[i] + bn - 1) / bn;
    snb += nb[i];
  }
  int bb = block_excl_scan<NW>(snb, wsum, total);
#pragma unroll
  for (int i = 0; i < EPT; ++i) {
    if (e0 + i < N) bbase[e0 + i] = bb;
    bb += nb[i];
  }
  __syncthreads();
  if (write) {
    for (int e = threadIdx.x; e <= N; e += blockDim.x) offsets[e] = off[e];
#pragma unroll
    for (int i = 0; i < EPT; ++i) {
      const int e = e0 + i;
      for (int j = 0; j < nb[i]; ++j) {
        const int r0 = j * bn;
        blocks[bbase[e] + j] = make_int4(e, off[e] + r0, min(bn, cnt[i] - r0), 0);
      }
    }
    if (threadIdx.x == 0) *nblocks = *total;
  }
}

// Rows of the routed (token, slot) pairs of chunk c (this lane's token): the
// chunk's masks `m` give the rank inside the chunk, base_of(e) the rows of
// expert e in earlier chunks.
template <class BaseOf>
__device__ __forceinline__ void seg_rows(const uint32_t* m, const int32_t* __restrict__ idx,
                                         const float* __restrict__ topk_w, int64_t c, int64_t T,
                                         int N, int K, int bn, const int32_t* off,
                                         const int32_t* bbase, BaseOf base_of,
                                         int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                         float* __restrict__ wrow, int32_t* __restrict__ rblock,
                                         int lane) {
  const int64_t t = c * 32 + lane;
  if (t >= T) return;
  const uint32_t lower = (1u << lane) - 1u;
  int ek[32], base[32];
  float wk[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    ek[k] = (k < K) ? idx[t * K + k] : -1;
    wk[k] = (k < K) ? topk_w[t * K + k] : 0.0f;
  }
#pragma unroll
  for (int k = 0; k < 32; ++k) base[k] = (ek[k] >= 0 && ek[k] < N) ? base_of(ek[k]) : 0;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const int e = ek[k];
    if (k < K && e >= 0 && e < N) {
      const int rank = base[k] + __popc(m[e] & lower);
      const int row = off[e] + rank;
      inv[t * K + k] = row;
      perm[row] = static_cast<int32_t>(t * K + k);
      wrow[row] = wk[k];
      // token block of the row and its index inside the block (bn <= 256)
      if (rblock) rblock[row] = ((bbase[e] + rank / bn) << 8) | (rank % bn);
    }
  }
}

__global__ void __launch_bounds__(256) k_scatter(
    const int32_t* __restrict__ idx, const float* __restrict__ topk_w,
    const int32_t* __restrict__ chunk_base, const int32_t* __restrict__ counts, int64_t T, int N,
    int K, int bn, int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
    int32_t* __restrict__ inv, float* __restrict__ wrow, int4* __restrict__ blocks,
    int32_t* __restrict__ nblocks, int32_t* __restrict__ rblock, int* err) {
  extern __shared__ int32_t sc_smem[];
  int32_t* off = sc_smem;                                    // [N + 1]
  int32_t* bbase = off + N + 1;                              // [N]
  uint32_t* masks = reinterpret_cast<uint32_t*>(bbase + N);  // [8][N]
  __shared__ int wsum[16];
  __shared__ int total;
  pdl_wait();
  pdl_trigger();

  int c4[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) c4[i] = (threadIdx.x * 4 + i < N) ? counts[threadIdx.x * 4 + i] : 0;
  seg_offsets<4, 8>(c4, N, bn, off, bbase, blockIdx.x == 0, offsets, blocks, nblocks, wsum, &total);

  // rows of the routed (token, slot) pairs of this warp's chunk
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * 8 + w;
  const int64_t nchunks = (T + 31) / 32;
  if (c >= nchunks) return;
  uint32_t* m = masks + w * N;
  build_chunk_masks(m, idx, c, T, N, K, lane, err);
  seg_rows(m, idx, topk_w, c, T, N, K, bn, off, bbase,
           [&](int e) { return chunk_base[c * N + e]; }, perm, inv, wrow, rblock, lane);
}

// The whole segment build of at most 256 tokens (8 chunks) in one block of
// 1024 threads, with every global access coalesced: thread i takes the routed
// pairs p = t K + k = i + 1024 j (idx, topk_w and inv in their own order) and
// expert e = i; the pairs, the chunks' expert masks and chunk bases, and the
// row-ordered outputs (perm, rblock) are staged in shared memory and written
// out row by row at the end.  The same rows as k_hist, k_scan and k_scatter in
// turn.  One SM does it all, so the work goes to as many warps as it holds
// (their latencies overlap), and the loops stay rolled: the kernel runs once
// per forward, after the grouped GEMMs of the last one have streamed
// gigabytes through L2, so its code comes from HBM every time.  Shared
// memory: masks and chunk bases [8][N] each, off [N + 1], bbase [N], and four
// [T K] pair / row arrays.
__global__ void __launch_bounds__(1024) k_segments_small(
    const int32_t* __restrict__ idx, const float* __restrict__ topk_w, int64_t T, int N, int K,
    int bn, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv, float* __restrict__ wrow,
    int4* __restrict__ blocks, int32_t* __restrict__ nblocks, int32_t* __restrict__ rblock,
    int* err) {
  extern __shared__ int32_t sc_smem[];
  const int P = static_cast<int>(T) * K;   // routed pairs (<= 256 x 32)
  uint32_t* masks = reinterpret_cast<uint32_t*>(sc_smem);   // [8][N]
  int32_t* cbase = sc_smem + 8 * N;                           // [8][N]
  int32_t* off = cbase + 8 * N;                               // [N + 1]
  int32_t* bbase = off + N + 1;                               // [N]
  int32_t* idx_s = bbase + N;                                 // [P] pairs' experts
  float* w_s = reinterpret_cast<float*>(idx_s + P);           // [P] pairs' weights
  int32_t* perm_s = idx_s + 2 * P;                            // [P] row -> pair
  int32_t* rb_s = idx_s + 3 * P;                              // [P] row -> token block
  __shared__ int wsum[64];
  __shared__ int total;
  pdl_wait();
  pdl_trigger();
  const int nchunks = static_cast<int>((T + 31) / 32);
  // token of pair p: (p + 1/2) / K lies at least 1/(2K) >= 1/64 from an
  // integer, and for p < 2^13 the two roundings below are off by < 1e-3
  const float rK = 1.0f / static_cast<float>(K);
  auto token_of = [rK](int p) { return static_cast<int>((static_cast<float>(p) + 0.5f) * rK); };
#pragma unroll 4
  for (int p = threadIdx.x; p < P; p += 1024) {
    idx_s[p] = idx[p];
    w_s[p] = topk_w[p];
  }
  for (int i = threadIdx.x; i < nchunks * N; i += 1024) masks[i] = 0u;
  __syncthreads();
  // each token's bit in its chunk's mask of every expert it selected
#pragma unroll 1
  for (int p = threadIdx.x; p < P; p += 1024) {
    const int e = idx_s[p], t = token_of(p);
    if (e < 0 || e >= N)
      atomicOr(err, DEVERR_BAD_INDEX);
    else
      atomicOr(&masks[(t >> 5) * N + e], 1u << (t & 31));
  }
  __syncthreads();
  // expert e = threadIdx.x: the rows of earlier chunks (chunk bases), its count
  const int e = threadIdx.x;
  int cnt[1] = {0};
  if (e < N) {
#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
      cbase[c * N + e] = cnt[0];
      cnt[0] += __popc(masks[c * N + e]);
    }
    counts[e] = cnt[0];
  }
  seg_offsets<1, 32>(cnt, N, bn, off, bbase, true, offsets, blocks, nblocks, wsum, &total);
  // each pair's row: expert offset + chunk base + rank inside the chunk
#pragma unroll 1
  for (int p = threadIdx.x; p < P; p += 1024) {
    const int ep = idx_s[p], t = token_of(p);
    if (ep < 0 || ep >= N) continue;
    const int c = t >> 5;
    const int rank = cbase[c * N + ep] + __popc(masks[c * N + ep] & ((1u << (t & 31)) - 1u));
    const int row = off[ep] + rank;
    inv[p] = row;
    perm_s[row] = p;
    rb_s[row] = ((bbase[ep] + rank / bn) << 8) | (rank % bn);
  }
  __syncthreads();
  const int rows = off[N];
#pragma unroll 1
  for (int r = threadIdx.x; r < rows; r += 1024) {
    const int p = perm_s[r];
    perm[r] = p;
    wrow[r] = w_s[p];
    if (rblock) rblock[r] = rb_s[r];
  }
}

cudaError_t launch_scatter(const int32_t* topk_idx, const float* topk_w, const int32_t* chunk_base,
                           const int32_t* counts, int64_t T, int N, int K, int bn,
                           int32_t* offsets, int32_t* perm, int32_t* inv, float* wrow,
                           int4* blocks, int32_t* nblocks, int32_t* rblock, int* err,
                           cudaStream_t st) {
  const int64_t nchunks = (T + 31) / 32;
  const unsigned nblk = static_cast<unsigned>(nchunks > 0 ? (nchunks + 7) / 8 : 1);
  const size_t smem = (2 * N + 1) * sizeof(int32_t) + 8 * N * sizeof(uint32_t);
  return launch_pdl(k_scatter, nblk, 256, smem, st, topk_idx, topk_w, chunk_base, counts, T, N, K,
                    bn, offsets, perm, inv, wrow, blocks, nblocks, rblock, err);
}

cudaError_t launch_segments_small(const int32_t* topk_idx, const float* topk_w, int64_t T, int N,
                                  int K, int bn, int32_t* counts, int32_t* offsets, int32_t* perm,
                                  int32_t* inv, float* wrow, int4* blocks, int32_t* nblocks,
                                  int32_t* rblock, int* err, cudaStream_t st) {
  if (T <= 0 || T > SEG_SMALL_T || N > 1024 || K > 32) return cudaErrorInvalidValue;
  const size_t smem = (18 * N + 1 + 4 * T * K) * sizeof(int32_t);
  // the largest shared memory any call asks for (N = 1024, 256 x 32 pairs:
  // 205 KB), allowed once per device
  constexpr int kMaxSmem = (18 * 1024 + 1 + 4 * SEG_SMALL_T * 32) * sizeof(int32_t);
  static std::atomic<uint64_t> allowed{0};   // bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? uint64_t(1) << dev : 0;
  if (!bit || !(allowed.load() & bit)) {
    e = cudaFuncSetAttribute(k_segments_small, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kMaxSmem);
    if (e != cudaSuccess) return e;
    allowed.fetch_or(bit);
  }
  return launch_pdl(k_segments_small, 1u, 1024, smem, st, topk_idx, topk_w, T, N, K, bn, counts,
                    offsets, perm, inv, wrow, blocks, nblocks, rblock, err);
}

// ---------------------------------------------------------------------------
// gather of latent rows into expert order: u_perm[r] = u[perm[r] / K]

__global__ void __launch_bounds__(256) k_gather(const uint4* __restrict__ u,
                                                const int32_t* __restrict__ perm, int64_t rows,
                                                int K, int l8, uint4* __restrict__ u_perm) {
  pdl_wait();
  pdl_trigger();
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += nwarps) {
    const int64_t tok = perm[r] / K;
    const uint4* src = u + tok * l8;
    uint4* dst = u_perm + r * l8;
    for (int i = lane; i < l8; i += 32) dst[i] = src[i];
  }
}

cudaError_t launch_gather(const void* u, const int32_t* perm, int64_t rows, int K, int l,
                          void* u_perm, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  int64_t blocks = (rows + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  return launch_pdl(k_gather, static_cast<unsigned>(blocks), 256, 0, st,
                    static_cast<const uint4*>(u), perm, rows, K, l / 8, static_cast<uint4*>(u_perm));
}

// ---------------------------------------------------------------------------
// latent combine in token order: v[t] = sum_k O[inv[t][k]], fixed slot order
// (WEIGHTED: sum_k w[t][k] O[inv[t][k]], for rows that come back unweighted
// from an expert-parallel exchange).  One thread per 8 consecutive latent
// elements of one token; the K row indices and the K row loads are issued
// before the (ordered) sum.

template <bool WEIGHTED>
__global__ void __launch_bounds__(256) k_combine(const __nv_bfloat16* __restrict__ O,
                                                 const int32_t* __restrict__ inv,
                                                 const float* __restrict__ wts, int64_t T,
                                                 int K, int l, __nv_bfloat16* __restrict__ vh,
                                                 int ldv) {
  pdl_wait();
  pdl_trigger();
  const int l8 = l >> 3;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t t = g / l8;
  if (t >= T) return;
  const int c = static_cast<int>(g - t * l8) * 8;
  int rows[32];
  float wk[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) rows[k] = (k < K) ? inv[t * K + k] : 0;
#pragma unroll
  for (int k = 0; k < 32; ++k) wk[k] = (WEIGHTED && k < K) ? wts[t * K + k] : 1.0f;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  // eight row loads in flight, then their sums in slot order
#pragma unroll
  for (int k0 = 0; k0 < 32; k0 += 8) {
    if (k0 < K) {
      uint4 raw[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        raw[j] = (k0 + j < K)
                     ? __ldg(reinterpret_cast<const uint4*>(
                           O + static_cast<int64_t>(rows[k0 + j]) * l + c))
                     : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (k0 + j < K) {
          const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw[j]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(p[i]);
            if (WEIGHTED) {
              acc[2 * i] = fmaf(wk[k0 + j], f.x, acc[2 * i]);
              acc[2 * i + 1] = fmaf(wk[k0 + j], f.y, acc[2 * i + 1]);
            } else {
              acc[2 * i] += f.x;
              acc[2 * i + 1] += f.y;
            }
          }
        }
      }
    }
  }
  __nv_bfloat162 outp[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) outp[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
  *reinterpret_cast<uint4*>(vh + t * ldv + c) = *reinterpret_cast<const uint4*>(outp);
}

cudaError_t launch_combine(const void* O, const int32_t* inv, int64_t T, int K, int l, void* vh,
                           int ldv, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  const int64_t blocks = (T * (l / 8) + 255) / 256;
  return launch_pdl(k_combine<false>, static_cast<unsigned>(blocks), 256, 0, st,
                    static_cast<const __nv_bfloat16*>(O), inv, static_cast<const float*>(nullptr),
                    T, K, l, static_cast<__nv_bfloat16*>(vh), ldv);
}

cudaError_t launch_combine_w(const void* O, const int32_t* inv, const float* topk_w, int64_t T,
                             int K, int l, void* vh, int ldv, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  const int64_t blocks = (T * (l / 8) + 255) / 256;
  return launch_pdl(k_combine<true>, static_cast<unsigned>(blocks), 256, 0, st,
                    static_cast<const __nv_bfloat16*>(O), inv, topk_w, T, K, l,
                    static_cast<__nv_bfloat16*>(vh), ldv);
}

// ---------------------------------------------------------------------------
// counts of rows per expert handed in by a caller (an expert-parallel
// receiver): copied when every count is >= 0 and they sum to R, else zeros
// (no rows, no tiles) and DEVERR_BAD_INDEX in *err.  One block of 256 threads.

__global__ void __launch_bounds__(256) k_sanitize_counts(const int32_t* __restrict__ in, int n,
                                                         int64_t R, int32_t* __restrict__ out,
                                                         int* err) {
  __shared__ long long part[256];
  __shared__ int bad;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  long long sum = 0;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int c = in[e];
    if (c < 0) bad = 1;
    sum += c;
  }
  part[threadIdx.x] = sum;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) part[threadIdx.x] += part[threadIdx.x + o];
    __syncthreads();
  }
  const bool ok = !bad && part[0] == R;
  for (int e = threadIdx.x; e < n; e += blockDim.x) out[e] = ok ? in[e] : 0;
  if (!ok && threadIdx.x == 0) atomicOr(err, DEVERR_BAD_INDEX);
}

cudaError_t launch_sanitize_counts(const int32_t* in, int n, int64_t R, int32_t* out, int* err,
                                   cudaStream_t st) {
  return launch_pdl(k_sanitize_counts, 1, 256, 0, st, in, n, R, out, err);
}

// ---------------------------------------------------------------------------
// row permutation of an expert-parallel exchange (one warp per row, 16-byte
// units): gather dst[r] = src[idx[r]], or scatter dst[idx[r]] = src[r].  An
// index outside [0, n_other) -- the row count of the indexed side -- skips
// its row.

template <bool SCATTER>
__global__ void __launch_bounds__(256) k_permute_rows(const uint4* __restrict__ src,
                                                      const int32_t* __restrict__ idx, int64_t n,
                                                      int64_t n_other, int w16,
                                                      uint4* __restrict__ dst) {
  pdl_wait();
  pdl_trigger();
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < n;
       r += nwarps) {
    const int64_t j = idx[r];
    if (j < 0 || j >= n_other) continue;
    const uint4* s = src + (SCATTER ? r : j) * w16;
    uint4* d = dst + (SCATTER ? j : r) * w16;
    for (int i = lane; i < w16; i += 32) d[i] = s[i];
  }
}

cudaError_t launch_permute_rows(const void* src, const int32_t* idx, int64_t n, int64_t n_other,
                                int row_bytes, void* dst, bool scatter, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  int64_t blocks = (n + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  return launch_pdl(scatter ? k_permute_rows<true> : k_permute_rows<false>,
                    static_cast<unsigned>(blocks), 256, 0, st, static_cast<const uint4*>(src), idx,
                    n, n_other, row_bytes / 16, static_cast<uint4*>(dst));
}

// ---------------------------------------------------------------------------
// bounded-wait probe: an mbarrier that nothing arrives on

__global__ void k_wait_probe(int* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, &abort_flag, err, limit_ns);
}

cudaError_t launch_wait_probe(int* err, unsigned long long limit_ns, cudaStream_t st) {
  k_wait_probe<<<1, 32, 0, st>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace lmoe
