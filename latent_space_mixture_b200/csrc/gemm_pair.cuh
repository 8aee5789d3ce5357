// The persistent tcgen05 GEMM of gemm_tc.cuh on CTA pairs (clusters of two,
// tcgen05 ... cta_group::2): a tile covers 256 weight rows (128 per CTA) and
// up to BN token rows (BN/2 per CTA), and the MMA of the pair is M = 256.  Per
// SM and k-step the pair moves 16 KB of A and BN/2 x 128 B of B for the same
// MMA work a single CTA does with 16 KB + BN x 128 B, so operand traffic per
// flop drops by a third at BN = 256.
//
// Roles per CTA (192 threads, one CTA per SM):
//   warp 0      TMA producer of this CTA's half: A rows [a_row + 128 r, +128)
//               and B rows [row0 + r n/2, + n/2) (r = rank in the pair, n the
//               tile's MMA N); completion is counted on the even CTA's "full"
//               barrier, which that CTA's producer arms with both halves' bytes;
//   warp 1      TMEM allocation for the pair (both CTAs); in the even CTA the
//               MMA issuer: 4 x tcgen05.mma.cta_group::2 (M256, N, K16) per
//               k-step, commits multicast to both CTAs' "empty" barriers and,
//               per tile, "accumulator full" barriers;
//   warps 2..5  epilogue of this CTA's 128 rows; release the accumulator on
//               the even CTA's barrier (256 arrivals: both CTAs).
// All waits are bounded as in gemm_tc.cuh.
#pragma once
#include "gemm_tc.cuh"

namespace lmoe {

constexpr int PAIR_BM = 256;

// A stage holds KSUB consecutive 64-wide K sub-tiles of both operands (each
// its own 128-byte-swizzled region) and completes on one barrier phase: a
// CTA's TMA stream is limited by a roughly fixed cost per barrier phase
// (~450 clocks: one 16 KB box per phase moves ~36 B/clock, two ~68, three or
// more ~85), so a k-step of 16 KB of weights and a few token rows would be
// bound by it rather than by the MMAs.
template <int BN, int STAGES, int KSUB>
struct PairLayout {
  static constexpr int A_SUB = GEMM_BM * GEMM_ROW_BYTES;
  static constexpr int B_SUB = (BN / 2) * GEMM_ROW_BYTES;
  static constexpr int A_BYTES = KSUB * A_SUB;
  static constexpr int B_BYTES = KSUB * B_SUB;
  static constexpr int STG_BYTES = GEMM_EPI_WARPS * 32 * GEMM_STG_LD * 4;
  static constexpr int BAR_BYTES = (2 * STAGES + 5) * 8;
  static constexpr int SMEM_BYTES =
      1024 + STAGES * (A_BYTES + B_BYTES) + STG_BYTES + BAR_BYTES + 16;
  static constexpr uint32_t TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;
  static_assert(BN % 32 == 0 && BN <= 256, "pair N: two halves of multiples of 16");
  static_assert((TMEM_COLS & (TMEM_COLS - 1)) == 0, "TMEM allocation is a power of 2");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  // one release per stage: the 256-wide MMAs hide the commit, and a paired
  // release would hold a stage of the ring back (measured slower here)
  static constexpr bool PAIRED_RELEASE = false;
};

// tile -> (token block, K slice, 256-row feature block), feature block
// fastest; the CTA of rank r owns weight rows [a_row, a_row + 128).  With
// ksplit > 1 (dense GEMMs of few tokens) each slice writes fp32 partials
// part[slice][row][feature], summed by the split-K reduction kernels.
__device__ __forceinline__ TileInfo pair_tile(const TileSource& s, int BN, int tile, int rank) {
  TileInfo t;
  const int tk = tile / s.FB;
  t.fb = tile - tk * s.FB;
  const int tb = tk / s.ksplit;
  t.tb = tb;
  t.ks = tk - tb * s.ksplit;
  t.kb0 = t.ks * s.kblocks / s.ksplit;
  t.kb1 = (t.ks + 1) * s.kblocks / s.ksplit;
  if (s.dense) {
    t.e = 0;
    t.row0 = tb * BN;
    t.nrows = min(BN, s.T - t.row0);
  } else {
    const int4 b = s.blocks[tb];
    t.e = b.x;
    t.row0 = b.y;
    t.nrows = b.z;
  }
  t.a_row = t.e * s.a_rows_per_expert + t.fb * PAIR_BM + rank * GEMM_BM;
  return t;
}

template <int BN, int STAGES, int KSUB, class Epi>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
k_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmB64, const TileSource src, const Epi epi,
            int* err, unsigned long long limit_ns) {
  using L = PairLayout<BN, STAGES, KSUB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * L::A_BYTES;
  float* stg = reinterpret_cast<float*>(sB + STAGES * L::B_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(stg) + L::STG_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;   // [2]
  uint64_t* tempty = tfull + 2;       // [2], used in the even CTA
  uint64_t* drain = tempty + 2;       // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * GEMM_EPI_WARPS * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmB64);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, L::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // the even CTA's barriers exist before the odd CTA signals them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_tiles = gemm_num_tiles(src, BN);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // whole warp, one elected lane issuing (see k_gemm_tc)
    pdl_wait();
    pdl_trigger();
    const uint64_t pol_a = src.a_stream_once ? policy_evict_first() : policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    long issued = 0;
    bool ok = true;
    for (int tile = pair; ok && tile < num_tiles; tile += npairs) {
      const TileInfo t = pair_tile(src, BN, tile, rank);
      const int n_mma = (t.nrows + 31) & ~31;
      const int half = n_mma / 2;
      const int nbig = half / GEMM_BROWS_BIG;
      const int nsmall = (half - nbig * GEMM_BROWS_BIG) / GEMM_BROWS;
      const int brow0 = t.row0 + rank * half;
      // bytes of one K sub-tile, both CTAs (A halves and B halves)
      const uint32_t tx_sub = 2 * L::A_SUB + n_mma * GEMM_ROW_BYTES;
      for (int kb = t.kb0; kb < t.kb1; kb += KSUB) {
        if (empty_waits_at<L>(stage) &&
            !__all_sync(0xffffffffu, mbar_wait_bounded(&empty[empty_slot<L>(stage)], phase ^ 1,
                                                       abort_flag, err, limit_ns))) {
          ok = false;
          break;
        }
        const uint32_t full_leader = mapa_shared(smem_u32(&full[stage]), 0);
        const int nsub = min(KSUB, t.kb1 - kb);
        if (elect_one()) {
          if (leader) mbar_arrive_expect_tx(&full[stage], nsub * tx_sub);
          for (int q = 0; q < nsub; ++q) {
            const int x = (kb + q) * GEMM_BK;
            tma_load_2d_pair(sA + stage * L::A_BYTES + q * L::A_SUB, &tmA, x, t.a_row,
                             full_leader, pol_a);
            uint8_t* b_dst = sB + stage * L::B_BYTES + q * L::B_SUB;
            for (int j = 0; j < nbig; ++j)
              tma_load_2d_pair(b_dst + j * GEMM_BROWS_BIG * GEMM_ROW_BYTES, &tmB64, x,
                               brow0 + j * GEMM_BROWS_BIG, full_leader, policy_evict_last());
            for (int j = 0; j < nsmall; ++j) {
              const int r = nbig * GEMM_BROWS_BIG + j * GEMM_BROWS;
              tma_load_2d_pair(b_dst + r * GEMM_ROW_BYTES, &tmB, x, brow0 + r, full_leader,
                               policy_evict_last());
            }
          }
        }
        __syncwarp();
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (!ok && lane == 0) {
      // a stage's copies complete on the even CTA's barrier; wait for this
      // CTA's in-flight copies there (bounded) before the CTA exits
      const long first = issued > STAGES ? issued - STAGES : 0;
      for (long i = first; i < issued && leader; ++i) {
        uint64_t* b = &full[i % STAGES];
        const uint32_t par = static_cast<uint32_t>((i / STAGES) & 1);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(b, par) && global_timer_ns() - t0 < limit_ns) {
        }
      }
      if (!leader) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < limit_ns / 4) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    // whole warp, one elected lane issuing (see k_gemm_tc)
    if (leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued_any = false;
      for (int tile = pair; ok && tile < num_tiles; tile += npairs) {
        const TileInfo t = pair_tile(src, BN, tile, 0);
        const int n_mma = (t.nrows + 31) & ~31;
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag,
                                                        err, limit_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        const uint32_t idesc = idesc_bf16(PAIR_BM, n_mma);
        for (int kb = t.kb0; kb < t.kb1; kb += KSUB) {
          if (!__all_sync(0xffffffffu,
                          mbar_wait_bounded(&full[stage], phase, abort_flag, err, limit_ns))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nsub = min(KSUB, t.kb1 - kb);
          if (elect_one()) {
            for (int q = 0; q < nsub; ++q) {
              const uint64_t a0 = sdesc_k_sw128(smem_u32(sA + stage * L::A_BYTES + q * L::A_SUB));
              const uint64_t b0 = sdesc_k_sw128(smem_u32(sB + stage * L::B_BYTES + q * L::B_SUB));
#pragma unroll
              for (int k = 0; k < GEMM_BK / 16; ++k)
                umma_bf16_pair(d_tmem, a0 + 2 * k, b0 + 2 * k, idesc,
                               (kb != t.kb0) || (q != 0) || (k != 0));
            }
            if (empty_commits_at<L>(stage)) umma_commit_pair(&empty[empty_slot<L>(stage)]);
          }
          __syncwarp();
          issued_any = true;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if (elect_one()) umma_commit_pair(&tfull[acc]);
        __syncwarp();
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (!ok && issued_any) {
        if (elect_one()) umma_commit_pair(drain);
        __syncwarp();
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < limit_ns) {
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    float* my = stg + (warp - 2) * 32 * GEMM_STG_LD;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < num_tiles; tile += npairs) {
      const TileInfo t = pair_tile(src, BN, tile, rank);
      int ok = 0;
      if (lane == 0) ok = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, err, limit_ns);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      tc_fence_after();
      const int feat_base = t.fb * PAIR_BM + rank * GEMM_BM + q * 32;
      for (int c0 = 0; c0 < t.nrows; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + c0, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) my[j * GEMM_STG_LD + lane] = __uint_as_float(r[j]);
        __syncwarp();
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int item = lane + 32 * it;
          const int j = item >> 2;
          const int g = item & 3;
          const int feat = feat_base + g * 8;
          const bool valid = c0 + j < t.nrows && feat < src.m_valid;
          const float4* p = reinterpret_cast<const float4*>(my + j * GEMM_STG_LD + g * 8);
          const float4 lo = p[0], hi = p[1];
          const long row = static_cast<long>(t.row0 + c0 + j);
          if (src.ksplit > 1) {
            if (valid) {
              float4* dst = reinterpret_cast<float4*>(
                  src.part + (static_cast<long>(t.ks) * src.T + row) * src.m_valid + feat);
              dst[0] = lo;
              dst[1] = hi;
            }
          } else {
            const float v[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
            epi.store8(t, row, feat, v, valid);
          }
        }
        __syncwarp();
      }
      tc_fence_before();
      mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // the pair's MMAs into this CTA's TMEM are done
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, L::TMEM_COLS);
}

}  // namespace lmoe
