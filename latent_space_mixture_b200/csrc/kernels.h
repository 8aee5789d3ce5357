// Launchers of the non-GEMM kernels of the LatentMoE forward pass (host side).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace lmoe {

// Sigmoid router with expert biasing, top-K by key (ties to the lower expert
// id, slots key-descending) and weights renormalised from the unbiased scores.
// One warp per token.  N <= 1024, N % 32 == 0, 1 <= K <= min(N, 32).
cudaError_t launch_route(const float* logits, const float* bias, int64_t T, int N, int K,
                         int32_t* topk_idx, float* topk_w, cudaStream_t st);

// Per-chunk (32 tokens) expert histograms: chunk_cnt[c][e].
cudaError_t launch_hist(const int32_t* topk_idx, int64_t T, int N, int K, int32_t* chunk_cnt,
                        int* err, cudaStream_t st);

// Column scan of chunk_cnt over chunks (in place, exclusive) and counts[e].
cudaError_t launch_scan(int32_t* chunk_cnt, int64_t T, int N, int32_t* counts, cudaStream_t st);

// Offsets (exclusive scan of counts), perm / inv / per-row weights, and the
// list of token blocks (at most `bn` rows, one expert each) for the grouped
// GEMMs: blocks[i] = {expert, first row, rows, 0}, *nblocks = count.
// rblock (optional, may be NULL): per row, (token block << 8) | row in block.
cudaError_t launch_scatter(const int32_t* topk_idx, const float* topk_w, const int32_t* chunk_base,
                           const int32_t* counts, int64_t T, int N, int K, int bn,
                           int32_t* offsets, int32_t* perm, int32_t* inv, float* wrow,
                           int4* blocks, int32_t* nblocks, int32_t* rblock, int* err,
                           cudaStream_t st);

// The three steps above in one block for at most SEG_SMALL_T tokens (N <=
// 1024): counts[e], offsets, perm / inv / row weights, the token-block list
// and rblock, the same values as launch_hist + launch_scan + launch_scatter.
constexpr int SEG_SMALL_T = 256;
cudaError_t launch_segments_small(const int32_t* topk_idx, const float* topk_w, int64_t T, int N,
                                  int K, int bn, int32_t* counts, int32_t* offsets, int32_t* perm,
                                  int32_t* inv, float* wrow, int4* blocks, int32_t* nblocks,
                                  int32_t* rblock, int* err, cudaStream_t st);

// u_perm[r] = u[perm[r] / K] for r < T*K (rows of width l, bf16).
cudaError_t launch_gather(const void* u, const int32_t* perm, int64_t rows, int K, int l,
                          void* u_perm, cudaStream_t st);

// v[t] = sum_k O[inv[t][k]] (fp32, slot order), written as bf16 into the first
// l columns of vh (row pitch ldv).
cudaError_t launch_combine(const void* O, const int32_t* inv, int64_t T, int K, int l, void* vh,
                           int ldv, cudaStream_t st);

// v[t] = sum_k w[t][k] O[inv[t][k]] (fp32, slot order): the combine of rows
// that come back unweighted from an expert-parallel exchange.
cudaError_t launch_combine_w(const void* O, const int32_t* inv, const float* topk_w, int64_t T,
                             int K, int l, void* vh, int ldv, cudaStream_t st);

// Caller-given rows per expert: out = in when every count is >= 0 and they
// sum to R, else zeros and DEVERR_BAD_INDEX in *err.  n <= 1024.
cudaError_t launch_sanitize_counts(const int32_t* in, int n, int64_t R, int32_t* out, int* err,
                                   cudaStream_t st);

// Rows of row_bytes (a multiple of 16): gather dst[r] = src[idx[r]] or
// scatter dst[idx[r]] = src[r] for r < n; indices outside [0, n_other) skip
// their row.
cudaError_t launch_permute_rows(const void* src, const int32_t* idx, int64_t n, int64_t n_other,
                                int row_bytes, void* dst, bool scatter, cudaStream_t st);

// NVFP4 (nvfp4.cu).  Expert weights [E][rows_per][K] bf16 -> codes
// [E*rows_per][Kp/2], scale atoms [E*rows_per/128][Kp/64][512], global scales
// [E]; amax is [E] scratch.  Kp = K rounded up to 256; padding pre-zeroed.
// weight quantiser variants (bit set): 2D 16x16 blocks, MSE-searched scales
constexpr int QUANT_W_2D = 1;
constexpr int QUANT_W_MSE = 2;
cudaError_t launch_quant_weights(const void* w, int E, int rows_per, int K, int Kp, float* amax,
                                 uint8_t* codes, uint8_t* atoms, float* gscale, int variant,
                                 cudaStream_t st);
// FP8 (E4M3) expert weights [E][rows_per][K] bf16 -> codes [E*rows_per][K]
// bytes and per-expert scales [E] (amax / 448); amax is [E] scratch.
cudaError_t launch_quant_w8(const void* w, int E, int rows_per, int K, float* amax, uint8_t* codes,
                            float* scale, cudaStream_t st);
// Scale tables (nvfp4.cuh, NVFP4_TAB floats) of one static global scale g.
cudaError_t launch_scale_tables(float g, float* tab, cudaStream_t st);
// fp32 rows -> codes [rows][cols/2], scales [rows][cols/16] (canonical layout).
cudaError_t launch_quant_rows(const float* x, int64_t rows, int cols, float g, uint8_t* codes,
                              uint8_t* scales, cudaStream_t st);
// Gradient-path pieces of the NVFP4 training recipe: the random Hadamard
// transform (1/4) H16 diag(s) on every 16-element block of fp32 rows, and
// NVFP4 rows with stochastically rounded elements (SplitMix64 counters).
cudaError_t launch_rht16(const float* x, int64_t rows, int cols, uint64_t seed, float* y,
                         cudaStream_t st);
cudaError_t launch_quant_rows_sr(const float* x, int64_t rows, int cols, float g, uint64_t seed,
                                 uint8_t* codes, uint8_t* scales, cudaStream_t st);
// quantised u rows into expert order plus their scales into block atoms.
cudaError_t launch_gather_q(const uint8_t* uq, const uint8_t* usf, const int32_t* perm,
                            const int32_t* rblock, int64_t rows, int K, int l, int lp,
                            uint8_t* u_perm_q, uint8_t* atoms, cudaStream_t st);

// NVFP4 training backward (nvfp4_bw.cu): see that file for the layouts.
cudaError_t launch_quant_rows_bf16(const void* x, int64_t rows, int cols, float g, uint8_t* codes,
                                   int code_pitch, uint8_t* scales, cudaStream_t st);
cudaError_t launch_rows_scaled(const void* dv, const int32_t* perm, const float* wrow, int64_t R,
                               int K, int l, float* out, float* amax, cudaStream_t st);
cudaError_t launch_quant_rows_dev(const float* x, int64_t rows, int cols, const float* amax,
                                  bool sr, uint64_t seed, uint8_t* codes, int code_pitch,
                                  uint8_t* scales, float* g_out, cudaStream_t st);
cudaError_t launch_atoms_rblock(const uint8_t* scales, const int32_t* rblock, int64_t R, int nkb,
                                int kp64, uint8_t* atoms, cudaStream_t st);

cudaError_t launch_dw_rows(const void* O, const int32_t* inv, const void* dv, int64_t T, int K,
                           int l, float* dw, cudaStream_t st);
cudaError_t launch_seg_offsets(const int32_t* counts, int N, int32_t* po16, int32_t* po256,
                               int32_t* kofs, int32_t* grp, cudaStream_t st);
struct TSrc {
  const void* p;           // rows: fp32 [R][F], bf16 token rows [T][F], or NVFP4 codes
  const int32_t* perm;     // bf16 token rows: routed row -> t * K + k
  const int32_t* rblock;   // NVFP4 rows: (token block << 8) | row in block
  const uint8_t* atoms;    // NVFP4 rows: B-operand scale atoms
  int K;
  int code_pitch;          // NVFP4 rows: bytes per row of codes
  int fp64;                // NVFP4 rows: 64-element chunks per row of the atoms
  float g;                 // NVFP4 rows: global scale
};
// transposed, transformed operands of the weight-gradient GEMMs: pass 1 the
// amax, pass 2 codes, canonical scales and scale atoms (nvfp4_bw.cu)
cudaError_t launch_tq_amax(int src_kind, const TSrc& s, const int32_t* offsets,
                           const int32_t* counts, const int32_t* po16, const int32_t* po256,
                           const int32_t* grp, int N, int F, int64_t pitch, uint64_t seed_rht, float* amax,
                           cudaStream_t st);
cudaError_t launch_tq_quant(int src_kind, bool sr, const TSrc& s, const int32_t* offsets,
                            const int32_t* counts, const int32_t* po16, const int32_t* po256,
                            const int32_t* grp, int N, int F, int64_t pitch, uint64_t seed_rht, float* amax,
                            uint64_t seed_sr, uint8_t* codes, uint8_t* scales, uint8_t* atoms,
                            float* g_out, cudaStream_t st);
cudaError_t launch_zero_empty(const int32_t* counts, int N, int64_t per, float* dw,
                              cudaStream_t st);
cudaError_t launch_transpose_w2d(const uint8_t* codes, const uint8_t* atoms, int E, int R, int C,
                                 int Cp, int Rp, uint8_t* tcodes, uint8_t* tatoms,
                                 cudaStream_t st);

// Backward pass (backward.cu).  dst[r] = wrow[r] * dv[perm[r] / K], rows of
// width l (bf16, l % 8 == 0).
cudaError_t launch_gather_scaled(const void* dv, const int32_t* perm, const float* wrow,
                                 int64_t rows, int K, int l, void* dst, cudaStream_t st);

// Expert activation derivative per routed row: da = dg * 2 sqrt(g) in place
// (da holds dg on entry; g = H, both [rows][h] bf16), dwacc[r] = g . dg.
cudaError_t launch_dact(void* da, const void* H, int64_t rows, int h, float* dwacc,
                        cudaStream_t st);

// Router backward: dz of the selected experts (zero elsewhere) into columns
// [0, N) of dxh (bf16, row pitch ldx), from dwacc[r] = sum_h g_r[h] dg_r[h]
// (= w_r dL/dw_r) per routed row, or (direct) from dL/dw per (token, slot).
cudaError_t launch_route_bw(const float* logits, const int32_t* topk_idx, const int32_t* inv,
                            const float* wrow, const float* dwacc, int64_t T, int N, int K,
                            void* dxh, int ldx, bool direct, cudaStream_t st);

// Aux-loss-free bias update: bias[e] += rate * sign(total - N * counts[e]).
cudaError_t launch_bias_update(float* bias, const int32_t* counts, int N, int64_t total, float rate,
                               cudaStream_t st);

// A kernel whose mbarrier wait never completes, bounded by limit_ns: sets
// DEVERR_TIMEOUT in *err and returns.  Used to check the failure path.
cudaError_t launch_wait_probe(int* err, unsigned long long limit_ns, cudaStream_t st);

}  // namespace lmoe
