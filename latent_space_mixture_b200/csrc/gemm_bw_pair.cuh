// The expert weight-gradient GEMM of gemm_bw.cuh on CTA pairs (clusters of
// two, tcgen05 ... cta_group::2): dW[e] = B_e^T A_e over the expert's routed
// rows, both operands MN-major.  A pair tile covers 256 output features (the
// A operand's columns; 128 per CTA) and 256 dW rows (the B operand's columns;
// 128 per CTA), and the MMA of the pair is M = 256, N = 256.  Per SM and
// k-step of 64 rows the pair moves 16 KB of A and 16 KB of B for the work a
// single CTA does with 16 KB + 32 KB, so operand traffic from L2 per flop
// drops by a third.
//
// The last k-step of an expert reads rows past its segment (the next
// expert's rows, or stale rows of the buffer).  Instead of clearing them in
// shared memory, which here would have to happen in both CTAs before the even
// CTA's MMAs, both operands' last 64-row blocks come from tail copies
// ([E * 64][F], the segment's last rows, zeros past them; k_wgrad_tails),
// loaded through their own tensor maps.
//
// Roles per CTA (192 threads, one CTA per SM), as k_gemm_pair:
//   warp 0      TMA producer of this CTA's halves (A: 2 boxes of 64 features
//               x 64 rows, B: 2 boxes), completion counted on the even CTA's
//               "full" barrier, which that CTA's producer arms with both
//               halves' bytes;
//   warp 1      TMEM allocation for the pair; in the even CTA the MMA issuer
//               (4 x tcgen05.mma.cta_group::2 M256 N256 K16 per k-step),
//               commits multicast to both CTAs' "empty" and, per tile,
//               "accumulator full" barriers;
//   warps 2..5  epilogue of this CTA's 128 features x 256 dW rows: each
//               32 x 32 chunk stored by TMA (two boxes per warp in flight);
//               release the accumulator on the even CTA's barrier.
// All waits are bounded as in gemm_tc.cuh.
#pragma once
#include "gemm_bw.cuh"

namespace lmoe {

constexpr int WPAIR_STAGES = 6;

struct WPairLayout {
  static constexpr int A_BYTES = 2 * BW_BOX_BYTES;   // 128 features x 64 rows
  static constexpr int B_BYTES = 2 * BW_BOX_BYTES;   // 128 dW rows x 64 rows
  static constexpr int STG_BYTES = GEMM_EPI_WARPS * 2 * BW_TMA_BOX_BYTES;
  static constexpr int BAR_BYTES = (2 * WPAIR_STAGES + 5) * 8;
  static constexpr int SMEM_BYTES =
      1024 + WPAIR_STAGES * (A_BYTES + B_BYTES) + STG_BYTES + BAR_BYTES + 16;
  static constexpr uint32_t TMEM_COLS = 512;   // two accumulators of N = 256
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

// pair tile -> (expert, 256-row dW block, 256-feature block), feature block
// fastest; the CTA of rank r owns features fb*256 + 128 r and dW rows
// nb*256 + 128 r (its halves of A and B)
__device__ __forceinline__ BwTile wpair_tile(const BwSource& s, int tile, int rank) {
  BwTile t;
  const int per = s.NB * s.FB;
  t.e = tile / per;
  const int rem = tile - t.e * per;
  t.nb = rem / s.FB;
  t.fb = rem - t.nb * s.FB;
  const int seg0 = s.offsets[t.e];
  const int cnt = s.offsets[t.e + 1] - seg0;
  t.seg0 = seg0;
  t.kb1 = (cnt + BW_BOX_ROWS - 1) / BW_BOX_ROWS;
  t.k_last = cnt - (t.kb1 - 1) * BW_BOX_ROWS;
  t.row0 = t.nb * 256;
  t.nrows = min(256, s.n_valid - t.row0);
  (void)rank;
  return t;
}

// boxes of 64 columns of a CTA's half (128 columns from col0) that start
// inside a map of `cols` columns
__device__ __forceinline__ int wpair_boxes(int col0, int cols) {
  return col0 >= cols ? 0 : (col0 + 64 < cols ? 2 : 1);
}

template <class Epi>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
k_gemm_wgrad_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmAt, const __grid_constant__ CUtensorMap tmBt,
                  const BwSource src, const __grid_constant__ Epi epi, int* err,
                  unsigned long long limit_ns) {
  using L = WPairLayout;
  constexpr int STAGES = WPAIR_STAGES;
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
    tma_prefetch_desc(&tmAt);
    tma_prefetch_desc(&tmBt);
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
  // every operand may come from the previous kernel
  pdl_wait();
  const int num_tiles = src.groups * src.NB * src.FB;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    long issued = 0;
    bool ok = true;
    for (int tile = pair; ok && tile < num_tiles; tile += npairs) {
      const BwTile t = wpair_tile(src, tile, rank);
      // this CTA's halves and the pair's total bytes per k-step
      const int ax = t.fb * 256 + rank * 128, bx = t.row0 + rank * 128;
      const int na = wpair_boxes(ax, src.a_cols), nbx = wpair_boxes(bx, src.b_cols);
      const int tot = wpair_boxes(t.fb * 256, src.a_cols) + wpair_boxes(t.fb * 256 + 128, src.a_cols) +
                      wpair_boxes(t.row0, src.b_cols) + wpair_boxes(t.row0 + 128, src.b_cols);
      for (int kb = 0; kb < t.kb1; ++kb) {
        if (!__all_sync(0xffffffffu,
                        mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, err, limit_ns))) {
          ok = false;
          break;
        }
        const uint32_t full_leader = mapa_shared(smem_u32(&full[stage]), 0);
        const bool last = kb == t.kb1 - 1;
        // the last block from the tail copies (rows past the segment are zero)
        const CUtensorMap* ma = last ? &tmAt : &tmA;
        const CUtensorMap* mb = last ? &tmBt : &tmB;
        const int ky = last ? t.e * BW_BOX_ROWS : t.seg0 + kb * BW_BOX_ROWS;
        if (elect_one()) {
          if (leader) mbar_arrive_expect_tx(&full[stage], tot * BW_BOX_BYTES);
          uint8_t* a_dst = sA + stage * L::A_BYTES;
          for (int c = 0; c < na; ++c)
            tma_load_2d_pair(a_dst + c * BW_BOX_BYTES, ma, ax + c * 64, ky, full_leader,
                             policy_evict_last());
          uint8_t* b_dst = sB + stage * L::B_BYTES;
          for (int c = 0; c < nbx; ++c)
            tma_load_2d_pair(b_dst + c * BW_BOX_BYTES, mb, bx + c * 64, ky, full_leader,
                             policy_evict_last());
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
    if (leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued_any = false;
      const uint32_t idesc = idesc_bf16(256, 256) | IDESC_A_MN | IDESC_B_MN;   // M over the pair
      for (int tile = pair; ok && tile < num_tiles; tile += npairs) {
        const BwTile t = wpair_tile(src, tile, 0);
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag,
                                                        err, limit_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256;
        for (int kb = 0; kb < t.kb1; ++kb) {
          if (!__all_sync(0xffffffffu,
                          mbar_wait_bounded(&full[stage], phase, abort_flag, err, limit_ns))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const bool last = kb == t.kb1 - 1;
          const int k_end = last ? (t.k_last + 15) & ~15 : BW_BOX_ROWS;   // zeros past k_last
          if (elect_one()) {
            const uint8_t* a_st = sA + stage * L::A_BYTES;
            const uint8_t* b_st = sB + stage * L::B_BYTES;
            for (int k = 0; k < k_end / 16; ++k)
              umma_bf16_pair(d_tmem, sdesc_mn_sw128(smem_u32(a_st + k * 2048), BW_BOX_BYTES),
                             sdesc_mn_sw128(smem_u32(b_st + k * 2048), BW_BOX_BYTES), idesc,
                             (kb != 0) || (k != 0));
            umma_commit_pair(&empty[stage]);
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
    // this CTA's TMEM: lanes = its 128 features, columns = the tile's 256 dW
    // rows; each 32-row chunk of a warp's 32 features goes out as one box
    const int q = warp & 3;
    float* my = stg + (warp - 2) * 2 * (BW_TMA_BOX_BYTES / 4);
    int nbox = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < num_tiles; tile += npairs) {
      const BwTile t = wpair_tile(src, tile, rank);
      int ok = 0;
      if (lane == 0) ok = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, err, limit_ns);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      tc_fence_after();
      const int feat_base = t.fb * 256 + rank * 128 + q * 32;
      if (feat_base < src.m_valid) {
        for (int c0 = 0; c0 < t.nrows; c0 += 32) {
          uint32_t r[32];
          if (t.kb1 > 0) {
            tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * 256 + c0,
                               r);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = 0u;   // no rows: zero gradient
          }
          float* box = my + (nbox & 1) * (BW_TMA_BOX_BYTES / 4);
          // the box stored two chunks ago has been read out of this buffer
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 32; ++j) box[j * 32 + lane] = __uint_as_float(r[j]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const CUtensorMap* map;
            int x, y;
            epi.target(t, static_cast<long>(t.row0 + c0), feat_base, &map, &x, &y);
            tma_store_2d(map, box, x, y);
            bulk_commit_group();
          }
          ++nbox;
        }
      }
      tc_fence_before();
      mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (lane == 0) bulk_wait_group_read<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // the pair's MMAs into this CTA's TMEM are done
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, L::TMEM_COLS);
}

}  // namespace lmoe
