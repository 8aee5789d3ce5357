// Persistent, warp-specialised tcgen05 GEMM for the LatentMoE layer backward
// pass, bf16 operands, fp32 accumulation in TMEM.
//
// Every backward contraction reads one operand along its contiguous (MN)
// dimension: the data gradient of y = x W^T is dx = dy W, which needs W with
// its output-feature dimension as K; the weight gradient dW = dy^T x reduces
// over token rows, which are the slow dimension of both dy and x.  So the A
// operand is always MN-major here, and the B operand is K-major (data
// gradients: token rows, as in the forward) or MN-major (weight gradients).
//
// MN-major tiles are loaded by TMA as boxes of 64 elements (128 bytes) x 64
// K rows with 128-byte swizzle: A (M = 128) is two boxes, an MN-major B
// (N = BN) is BN / 64 boxes.  The tcgen05 shared-memory descriptor of such a
// tile has the byte distance between 64-element chunks as its leading byte
// offset and 1024 bytes between 8-row K groups as its stride byte offset; a
// K = 16 MMA step moves the start address by 16 rows (2048 bytes).
//
// Two kinds of tile lists:
//   dgrad  tiles of (token block, 128-feature block) as the forward grouped
//          and dense GEMMs; K runs over a fixed extent (the output features
//          of the forward weight), per expert for the grouped ones;
//   wgrad  tiles of (group, BN block of output rows of dW, 128-block of its
//          columns); K runs over the group's segment of routed rows (or all
//          T tokens).  The rows of the last K block that lie past the segment
//          (another expert's rows, or stale rows of a padded buffer) are
//          cleared in shared memory by the MMA warp before its MMAs, and the
//          MMAs stop at the next multiple of 16 rows.  A group with no rows
//          writes a zero gradient.
//
// Warp roles as the forward GEMM: warp 0 TMA producer, warp 1 TMEM owner and
// MMA issuer (both converged, one elected lane issues), warps 2..5 epilogue
// through a per-warp transposing smem tile, two TMEM accumulators.  Every
// mbarrier wait is bounded.
#pragma once
#include "gemm_tc.cuh"

namespace lmoe {

constexpr int BW_BOX_ROWS = 64;                    // K rows per MN-major box
constexpr int BW_BOX_BYTES = BW_BOX_ROWS * 128;    // 8 KB: 64 elements x 64 rows

struct BwSource {
  int wgrad;               // 0: dgrad tiles, 1: wgrad tiles
  // dgrad
  int dense;               // 1: tokens [0, T) in blocks of BN; 0: device block list
  int T;                   // dense dgrad: token rows; wgrad without offsets: K rows
  const int4* blocks;      // {expert, first row, rows, 0}
  const int* nblocks;
  int a_k_per_expert;      // dgrad grouped: A map rows (K) per expert
  int kblocks;             // dgrad: K / 64 (rounded up)
  // both
  int FB;                  // 128-wide M blocks (features of the output row)
  int m_valid;             // valid M
  int a_cols;              // columns of the A map (boxes starting past it are skipped)
  // wgrad
  int groups;              // experts, or 1
  const int* offsets;      // [groups + 1] row segments, or nullptr: [0, T)
  int NB;                  // BN-wide blocks of dW rows per group
  int n_valid;             // dW rows per group
  int b_cols;              // columns of the MN-major B map
};

struct BwTile {
  int e, fb, nb, row0, nrows, kb1, k_last, seg0;
};

__device__ __forceinline__ int bw_num_tiles(const BwSource& s, int BN) {
  if (s.wgrad) return s.groups * s.NB * s.FB;
  const int nb = s.dense ? (s.T + BN - 1) / BN : *s.nblocks;
  return nb * s.FB;
}

__device__ __forceinline__ BwTile bw_tile(const BwSource& s, int BN, int tile) {
  BwTile t;
  if (s.wgrad) {
    const int per = s.NB * s.FB;
    t.e = tile / per;
    const int rem = tile - t.e * per;
    t.nb = rem / s.FB;
    t.fb = rem - t.nb * s.FB;
    const int seg0 = s.offsets ? s.offsets[t.e] : 0;
    const int seg1 = s.offsets ? s.offsets[t.e + 1] : s.T;
    const int cnt = seg1 - seg0;
    t.seg0 = seg0;
    t.kb1 = (cnt + BW_BOX_ROWS - 1) / BW_BOX_ROWS;
    t.k_last = cnt - (t.kb1 - 1) * BW_BOX_ROWS;
    t.row0 = t.nb * BN;
    t.nrows = min(BN, s.n_valid - t.row0);
  } else {
    const int tk = tile / s.FB;
    t.fb = tile - tk * s.FB;
    t.nb = tk;
    if (s.dense) {
      t.e = 0;
      t.row0 = tk * BN;
      t.nrows = min(BN, s.T - t.row0);
    } else {
      const int4 b = s.blocks[tk];
      t.e = b.x;
      t.row0 = b.y;
      t.nrows = b.z;
    }
    t.kb1 = s.kblocks;
    t.k_last = BW_BOX_ROWS;
    t.seg0 = t.e * s.a_k_per_expert;
  }
  return t;
}

// fp32 epilogue boxes stored by TMA: 32 features x 32 rows, two per warp
constexpr int BW_TMA_BOX_BYTES = 32 * 32 * 4;

template <int BN, int STAGES, bool B_MN, bool TMA_OUT = false>
struct BwLayout {
  static constexpr int A_BYTES = 2 * BW_BOX_BYTES;          // 128 x 64 bf16
  static constexpr int B_BYTES = BN * GEMM_ROW_BYTES;       // BN x 64 bf16 (either major)
  static constexpr int STG_BYTES = TMA_OUT ? GEMM_EPI_WARPS * 2 * BW_TMA_BOX_BYTES
                                           : GEMM_EPI_WARPS * 32 * GEMM_STG_LD * 4;
  static constexpr int BAR_BYTES = (2 * STAGES + 5) * 8;
  static constexpr int SMEM_BYTES =
      1024 + STAGES * (A_BYTES + B_BYTES) + STG_BYTES + BAR_BYTES + 16;
  static constexpr uint32_t TMEM_COLS =
      2 * BN <= 32 ? 32 : 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N range for M=128");
  static_assert(!B_MN || BN % 64 == 0, "MN-major B: whole 64-element boxes");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

template <int BN, int STAGES, bool B_MN, class Epi>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
k_gemm_bw(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
          const __grid_constant__ CUtensorMap tmB64, const BwSource src,
          const __grid_constant__ Epi epi, int* err, unsigned long long limit_ns) {
  using L = BwLayout<BN, STAGES, B_MN, Epi::kTma>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * L::A_BYTES;
  float* stg = reinterpret_cast<float*>(sB + STAGES * L::B_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(stg) + L::STG_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;   // [2]
  uint64_t* tempty = tfull + 2;       // [2]
  uint64_t* drain = tempty + 2;       // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], GEMM_EPI_WARPS * 32);
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
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // every operand may come from the previous kernel
  pdl_wait();
  const int num_tiles = bw_num_tiles(src, BN);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    long issued = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const BwTile t = bw_tile(src, BN, tile);
      const int ax = t.fb * GEMM_BM;
      const int na = (ax + 64 < src.a_cols) ? 2 : 1;   // A boxes inside the map
      int nbx = 0, nbig = 0, nsmall = 0;
      uint32_t tx = na * BW_BOX_BYTES;
      if constexpr (B_MN) {
        const int left = src.b_cols - t.row0;
        nbx = left >= BN ? BN / 64 : (left + 63) / 64;
        tx += nbx * BW_BOX_BYTES;
      } else {
        nbig = t.nrows / GEMM_BROWS_BIG;
        nsmall = (t.nrows - nbig * GEMM_BROWS_BIG + GEMM_BROWS - 1) / GEMM_BROWS;
        tx += (nbig * GEMM_BROWS_BIG + nsmall * GEMM_BROWS) * GEMM_ROW_BYTES;
      }
      for (int kb = 0; kb < t.kb1; ++kb) {
        if (!__all_sync(0xffffffffu,
                        mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, err, limit_ns))) {
          ok = false;
          break;
        }
        const int ky = t.seg0 + kb * BW_BOX_ROWS;   // K row of the A (and MN-major B) boxes
        if (elect_one()) {
          mbar_arrive_expect_tx(&full[stage], tx);
          uint8_t* a_dst = sA + stage * L::A_BYTES;
          for (int c = 0; c < na; ++c)
            tma_load_2d(a_dst + c * BW_BOX_BYTES, &tmA, ax + c * 64, ky, &full[stage]);
          uint8_t* b_dst = sB + stage * L::B_BYTES;
          if constexpr (B_MN) {
            for (int c = 0; c < nbx; ++c)
              tma_load_2d(b_dst + c * BW_BOX_BYTES, &tmB64, t.row0 + c * 64, ky, &full[stage]);
          } else {
            const int bx = kb * GEMM_BK;
            for (int j = 0; j < nbig; ++j)
              tma_load_2d(b_dst + j * GEMM_BROWS_BIG * GEMM_ROW_BYTES, &tmB64, bx,
                          t.row0 + j * GEMM_BROWS_BIG, &full[stage]);
            for (int j = 0; j < nsmall; ++j) {
              const int r = nbig * GEMM_BROWS_BIG + j * GEMM_BROWS;
              tma_load_2d(b_dst + r * GEMM_ROW_BYTES, &tmB, bx, t.row0 + r, &full[stage]);
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
      // let the copies already issued land before the CTA's smem goes away
      const long first = issued > STAGES ? issued - STAGES : 0;
      for (long i = first; i < issued; ++i) {
        uint64_t* b = &full[i % STAGES];
        const uint32_t par = static_cast<uint32_t>((i / STAGES) & 1);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(b, par) && global_timer_ns() - t0 < limit_ns) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    bool issued_any = false;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const BwTile t = bw_tile(src, BN, tile);
      const int n_mma = B_MN ? BN : (t.nrows + 15) & ~15;
      if (!__all_sync(0xffffffffu,
                      mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, err, limit_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      const uint32_t idesc =
          idesc_bf16(GEMM_BM, n_mma) | IDESC_A_MN | (B_MN ? IDESC_B_MN : 0u);
      for (int kb = 0; kb < t.kb1; ++kb) {
        if (!__all_sync(0xffffffffu,
                        mbar_wait_bounded(&full[stage], phase, abort_flag, err, limit_ns))) {
          ok = false;
          break;
        }
        uint8_t* a_st = sA + stage * L::A_BYTES;
        uint8_t* b_st = sB + stage * L::B_BYTES;
        const bool last = kb == t.kb1 - 1;
        const int k_end = last ? (t.k_last + 15) & ~15 : BW_BOX_ROWS;   // rows the MMAs read
        if (last && t.k_last < k_end) {
          // rows [k_last, k_end) belong to the next segment: clear them in
          // every box (a whole 128-byte row, so the swizzle does not matter)
          const int zr = k_end - t.k_last;
          const int nbox = 2 + (B_MN ? BN / 64 : 0);
          for (int i = lane; i < nbox * zr * 8; i += 32) {
            const int box = i / (zr * 8);
            const int rem = i - box * zr * 8;
            uint8_t* base = box < 2 ? a_st + box * BW_BOX_BYTES : b_st + (box - 2) * BW_BOX_BYTES;
            *reinterpret_cast<uint4*>(base + (t.k_last + (rem >> 3)) * 128 + (rem & 7) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        tc_fence_after();
        if (elect_one()) {
          for (int k = 0; k < k_end / 16; ++k) {
            const uint64_t a_desc = sdesc_mn_sw128(smem_u32(a_st + k * 2048), BW_BOX_BYTES);
            const uint64_t b_desc = B_MN ? sdesc_mn_sw128(smem_u32(b_st + k * 2048), BW_BOX_BYTES)
                                         : sdesc_k_sw128(smem_u32(b_st)) + 2 * k;
            umma_bf16(d_tmem, a_desc, b_desc, idesc, (kb != 0) || (k != 0));
          }
          umma_commit(&empty[stage]);
        }
        __syncwarp();
        issued_any = true;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      if (elect_one()) umma_commit(&tfull[acc]);
      __syncwarp();
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (!ok && issued_any) {
      // wait for the MMAs already issued before the smem goes away
      if (elect_one()) umma_commit(drain);
      __syncwarp();
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < limit_ns) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // An epilogue that reads a second operand per output element (Epi::kAux)
    // gets it through fetch(): the four loads of a 32-row chunk are issued
    // together, one chunk ahead (the first before the accumulator wait), so
    // their latency overlaps the TMEM reads and the stores of the chunk before.
    // An fp32 epilogue with Epi::kTma writes each 32-row chunk as one 32 x 32
    // box through a TMA store (two boxes per warp in flight), so the stores
    // bypass the load/store path.
    const int q = warp & 3;                  // TMEM lane quarter of this warp
    float* my = Epi::kTma ? stg + (warp - 2) * 2 * (BW_TMA_BOX_BYTES / 4)
                          : stg + (warp - 2) * 32 * GEMM_STG_LD;
    int nbox = 0;                            // TMA boxes this warp has issued
    int acc = 0;
    uint32_t acc_phase = 0;
    auto fetch_chunk = [&](const BwTile& t, int c0, uint4 (&aux)[4]) {
      const int fb0 = t.fb * GEMM_BM + q * 32;
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int item = lane + 32 * it;
        const int j = item >> 2;
        const int feat = fb0 + (item & 3) * 8;
        const bool valid = c0 + j < t.nrows && feat < src.m_valid;
        if constexpr (Epi::kAux) aux[it] = epi.fetch(static_cast<long>(t.row0 + c0 + j), feat, valid);
      }
    };
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const BwTile t = bw_tile(src, BN, tile);
      uint4 aux[4] = {};
      if constexpr (Epi::kAux) fetch_chunk(t, 0, aux);
      int ok = 0;
      if (lane == 0) ok = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, err, limit_ns);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      tc_fence_after();
      const int feat_base = t.fb * GEMM_BM + q * 32;
      for (int c0 = 0; c0 < t.nrows; c0 += 32) {
        uint32_t r[32];
        if (t.kb1 > 0) {
          tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + c0, r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = 0u;   // no rows: zero gradient
        }
        if constexpr (Epi::kTma) {
          // rows and features come in whole chunks of 32 (both extents are
          // multiples of 32), so a chunk is either stored or skipped whole
          if (feat_base < src.m_valid) {
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
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) my[j * GEMM_STG_LD + lane] = __uint_as_float(r[j]);
          __syncwarp();
          uint4 nxt[4] = {};
          if constexpr (Epi::kAux)
            if (c0 + 32 < t.nrows) fetch_chunk(t, c0 + 32, nxt);
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            // lanes 4j..4j+3 hold the four 8-feature groups of output row j
            const int item = lane + 32 * it;
            const int j = item >> 2;
            const int g = item & 3;
            const int feat = feat_base + g * 8;
            const bool valid = c0 + j < t.nrows && feat < src.m_valid;
            const float4* p = reinterpret_cast<const float4*>(my + j * GEMM_STG_LD + g * 8);
            const float4 lo = p[0], hi = p[1];
            const float v[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
            if constexpr (Epi::kAux)
              epi.store8(t, static_cast<long>(t.row0 + c0 + j), feat, v, valid, aux[it]);
            else
              epi.store8(t, static_cast<long>(t.row0 + c0 + j), feat, v, valid);
          }
          __syncwarp();
#pragma unroll
          for (int it = 0; it < 4; ++it) aux[it] = nxt[it];
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    // the shared memory of the last boxes stays until the stores have read it
    if constexpr (Epi::kTma)
      if (lane == 0) bulk_wait_group_read<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, L::TMEM_COLS);
}

}  // namespace lmoe
