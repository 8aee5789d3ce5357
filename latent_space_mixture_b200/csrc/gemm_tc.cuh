// Persistent, warp-specialised tcgen05 GEMM used for every contraction of the
// LatentMoE layer forward pass.
//
// Orientation ("swap AB"): the weight matrix W [features][K] is the MMA A
// operand and fills the 128-row M of tcgen05.mma; a block of token rows
// X [tokens][K] is the B operand and sets N per tile at run time (a multiple
// of 16, up to BN).  D = W X^T lands in TMEM with one feature per lane and one
// token per column.  This keeps ragged per-expert token counts cheap: an
// expert with 11 routed rows costs an N=16 MMA, not a 128-row tile.
//
// Warp roles (64 + 32 x epilogue-warp threads, one CTA per SM, persistent
// over a static tile list):
//   warp 0      TMA producer: A tile and B rows (64- and 16-row boxes) per
//               k-step, 128-byte swizzle, completion on a "full" mbarrier;
//               in the NVFP4 variant also the two scale-factor tiles (bulk
//               copies of 2 KB);
//   warp 1      TMEM allocator and MMA issuer: per k-step 4 MMAs of K=16
//               (kind::f16, bf16), K=64 (kind::mxf4nvf4 with 16-element
//               block scales copied into TMEM by tcgen05.cp first) or K=32
//               (kind::f8f6f4, E4M3);
//               tcgen05.commit frees the smem stage, and at the end of a tile
//               marks the accumulator full;
//   warps 2..   epilogue (4 warps, or 8 / 16 where the epilogue outlasts the
//               main loop: GemmEpiWarps): tcgen05.ld 32 columns at a time
//               (warp w reads TMEM lanes 32 (w % 4)..; several warps per lane
//               quarter take alternate 32-column chunks), transpose through a
//               per-warp smem tile, call the epilogue functor on 8 consecutive
//               features of one token row (all lanes call it; `valid` tells
//               which carry data), release the accumulator.
// Two TMEM accumulators (2 x BN columns) let the epilogue of tile i overlap
// the main loop of tile i+1.  Every mbarrier wait is bounded (ptx.cuh).
// The producer and MMA warps run their loops converged and issue the TMA and
// tcgen05 instructions from one elected lane (elect.sync): issued from a lone
// divergent thread, each of these instructions cost several times as long,
// which starved the ring and stretched every small-N MMA.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "nvfp4.cuh"
#include "ptx.cuh"
#include "route.cuh"

namespace lmoe {

constexpr int GEMM_BM = 128;          // MMA M: features per tile
constexpr int GEMM_BK = 64;           // bf16 K elements per stage (128 B per row)
constexpr int GEMM_THREADS = 192;
constexpr int GEMM_EPI_WARPS = 4;
constexpr int GEMM_STG_LD = 36;       // fp32 staging pitch (32 + 4)
constexpr int GEMM_BROWS = 16;        // rows per small B TMA box (ragged tails)
constexpr int GEMM_BROWS_BIG = 64;    // rows per large B TMA box (full row groups)
constexpr int GEMM_ROW_BYTES = 128;   // bytes of one operand row per stage
constexpr int FP4_K_PER_STAGE = 256;  // NVFP4 K elements per stage (128 B per row)
constexpr int FP8_K_PER_STAGE = 128;  // FP8 (E4M3) K elements per stage (128 B per row)
// operand kinds of the GEMM (template parameter KIND)
constexpr int KIND_BF16 = 0;   // kind::f16, bf16 A and B, K = 16 per MMA
constexpr int KIND_NVFP4 = 1;  // kind::mxf4nvf4 block16 with E4M3 block scales, K = 64
constexpr int KIND_FP8 = 2;    // kind::f8f6f4, E4M3 A and B, K = 32
constexpr int KIND_W4A16 = 3;  // NVFP4 weights expanded to f16 in shared memory by
                               // converter warps, f16 B, kind::f16, K = 16
constexpr int W4_CONV_THREADS = 256;          // converter threads: two per weight row
constexpr int W4_KSUB = 2;   // W4A16 stages hold two 64-wide K sub-tiles (one barrier phase)
constexpr int W4_CODE_BYTES = GEMM_BM * 32;   // one k-step of FP4 weight codes
constexpr int FP4_SF_STAGE_BYTES = 4 * SF_ATOM_BYTES;   // 4 chunks of K=64

// Where the tiles of one GEMM come from.
struct TileSource {
  int dense;               // 1: tokens [0, T) in blocks of BN; 0: device block list;
                           // 2: per-group K ranges (weight gradients, below)
  int T;                   // dense: number of token rows
  const int4* blocks;      // list: {expert, first row, rows, 0}
  const int* nblocks;      // list: number of blocks (device scalar)
  int FB;                  // feature blocks of 128 per expert
  int a_rows_per_expert;   // rows of A per expert (0 when dense)
  int m_valid;             // valid features per expert (multiple of 8)
  int kblocks;             // K steps (K/64 bf16, K/256 NVFP4, K/128 FP8)
  int ksplit;              // dense only: K slices (1 = none); each slice writes
  float* part;             //   fp32 partials part[slice][row][feature]
  int a_stream_once;       // 1: each A tile is read by one tile only (L2 evict-first)
  const uint8_t* sfa;      // NVFP4: A scale atoms, [A row / 128][kc][512 B]
  const uint8_t* sfb;      // NVFP4: B scale atoms, [token block][kc][512 B]
  int kc;                  // NVFP4: 64-element chunks per row (4 x kblocks)
  // dense == 2: `groups` groups (experts) share one A matrix (features) and
  // one B matrix of b_rows rows; group g reduces over its own K range, k-steps
  // [kofs[g], kofs[g + 1]) (device array), and writes its own output; a group
  // with an empty range has no tiles (every role skips them)
  const int* kofs = nullptr;
  int groups = 0;
  int b_rows = 0;
};

struct TileInfo {
  int e, fb, row0, nrows, a_row, ks, kb0, kb1, tb;
};

// Features an epilogue takes per call: 8 consecutive features of one token row
// (store8), or 16 for an epilogue that declares kVec = 16 (store16: a whole
// NVFP4 block per lane).
template <class E, class = void>
struct EpiVec {
  static constexpr int value = 8;
};
template <class E>
struct EpiVec<E, std::void_t<decltype(E::kVec)>> {
  static constexpr int value = E::kVec;
};

// Token-major accumulators: an NVFP4 GEMM with 128-row token blocks whose
// epilogue declares kTokMajor swaps the MMA operands (tokens in M, features
// in N; both tiles are 128 K-major rows, so the descriptors and the scale
// atoms only trade places), so that TMEM holds one token row per lane and a
// lane's 32 consecutive features come straight from one tcgen05.ld: the
// epilogue's store32 gets them without the transposing shared-memory tile.
template <class E, class = void>
struct EpiTok {
  static constexpr bool value = false;
};
template <class E>
struct EpiTok<E, std::void_t<decltype(E::kTokMajor)>> {
  static constexpr bool value = E::kTokMajor;
};

__device__ __forceinline__ int gemm_num_tiles(const TileSource& s, int BN) {
  if (s.dense == 2) return s.groups * ((s.b_rows + BN - 1) / BN) * s.FB;
  const int nb = s.dense ? (s.T + BN - 1) / BN : *s.nblocks;
  return nb * s.FB * s.ksplit;
}

// tile -> (token block, K slice, feature block), feature block fastest
__device__ __forceinline__ TileInfo gemm_tile(const TileSource& s, int BN, int tile) {
  TileInfo t;
  const int tk = tile / s.FB;
  t.fb = tile - tk * s.FB;
  if (s.dense == 2) {
    // (group, B row block, feature block), feature block fastest
    const int nbb = (s.b_rows + BN - 1) / BN;
    const int g = tk / nbb;
    const int tb = tk - g * nbb;
    t.tb = tb;
    t.ks = 0;
    t.kb0 = s.kofs[g];
    t.kb1 = s.kofs[g + 1];
    t.e = g;
    t.row0 = tb * BN;
    t.nrows = min(BN, s.b_rows - t.row0);
    t.a_row = t.fb * GEMM_BM;
    return t;
  }
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
  t.a_row = t.e * s.a_rows_per_expert + t.fb * GEMM_BM;
  return t;
}

// epilogue staging of a variant: none (token-major accumulators), the
// transposing tile, or two 32 x 32 fp32 boxes per warp for TMA stores
constexpr int STG_NONE = 0, STG_TRANSPOSE = 1, STG_BOXES = 2;
constexpr int GEMM_BOX_FLOATS = 32 * 32;

template <int BN, int STAGES, int KIND, int EPIW = GEMM_EPI_WARPS, int STG = STG_TRANSPOSE>
struct GemmLayout {
  static constexpr bool FP4 = KIND == KIND_NVFP4;
  static constexpr bool W4 = KIND == KIND_W4A16;
  // 64-wide K sub-tiles per stage: W4A16 moves only 4.5 KB of weights per
  // sub-tile, and a CTA's TMA stream pays a roughly fixed cost per barrier
  // phase, so its stages take two
  static constexpr int KS = W4 ? W4_KSUB : 1;
  static constexpr int A_SUB = GEMM_BM * GEMM_ROW_BYTES;
  static constexpr int B_SUB = BN * GEMM_ROW_BYTES;
  static constexpr int A_BYTES = KS * A_SUB;
  static constexpr int B_BYTES = KS * B_SUB;
  static constexpr int SF_BYTES = FP4 ? 2 * FP4_SF_STAGE_BYTES : 0;
  // W4A16: the stage's FP4 codes (128 rows x 32 B per sub-tile) and A scale atoms
  static constexpr int RAW_BYTES = W4 ? KS * (W4_CODE_BYTES + SF_ATOM_BYTES) : 0;
  // epilogue warps: 4, or several per TMEM lane quarter (each takes every
  // (EPI_WARPS / 4)-th 32-column chunk), chosen per epilogue (GemmEpiWarps)
  static constexpr int EPI_WARPS = EPIW;
  static_assert(EPIW % 4 == 0 && EPIW >= 4 && EPIW <= 16, "epilogue warps per lane quarter");
  static constexpr int THREADS = 64 + 32 * EPI_WARPS + (W4 ? W4_CONV_THREADS : 0);   // + converters
  static constexpr int STG_BYTES = STG == STG_TRANSPOSE ? EPI_WARPS * 32 * GEMM_STG_LD * 4
                                   : STG == STG_BOXES   ? EPI_WARPS * 2 * GEMM_BOX_FLOATS * 4
                                                        : 0;
  static constexpr int BAR_BYTES = (3 * STAGES + 5) * 8;
  static constexpr int SMEM_BYTES = 1024 /*align slack*/ +
                                    STAGES * (A_BYTES + B_BYTES + SF_BYTES + RAW_BYTES) +
                                    STG_BYTES + BAR_BYTES + 16;
  // bytes a stage's TMA and bulk copies bring, besides the B rows
  static constexpr int TX_A = W4 ? RAW_BYTES : A_BYTES + SF_BYTES;
  // TMEM: two accumulators of BN columns, then (NVFP4) 32 scale columns per stage
  static constexpr int SF_COL0 = 2 * BN;
  static constexpr int COLS_USED = 2 * BN + (FP4 ? 32 * STAGES : 0);
  static constexpr uint32_t TMEM_COLS =
      COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64 : COLS_USED <= 128 ? 128
                                                  : COLS_USED <= 256 ? 256 : 512;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N range for M=128");
  static_assert(!FP4 || BN <= 128, "NVFP4 tiles: one scale atom of B rows");
  static_assert(COLS_USED <= 512, "TMEM columns");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  // with an even ring, one tcgen05.commit releases two consecutive stages
  // (every commit costs the tensor pipe a bubble of about 200 clocks)
  static constexpr bool PAIRED_RELEASE = STAGES % 2 == 0 && !W4;
};

// Epilogue warps of a GEMM variant: Epi::kWarps for token blocks of 128 rows
// or more, where the epilogue of a tile can take several times its main loop
// (quantising H to NVFP4 costs ~9x the tile's FP4 MMAs); 4 for the narrow
// decode blocks, whose shared memory goes to the ring.
template <int BN, class Epi>
struct GemmEpiWarps {
  static constexpr int value = BN >= 128 ? Epi::kWarps : GEMM_EPI_WARPS;
};

// Ring depth: `want` stages, or as many as fit in shared memory beside the
// epilogue staging.
template <int BN, int KIND, int EPIW, int STG = STG_TRANSPOSE>
constexpr int gemm_fit_stages(int want) {
  using L2 = GemmLayout<BN, 2, KIND, EPIW, STG>;
  int s = want;
  while (s > 2 && L2::SMEM_BYTES + (s - 2) * (L2::A_BYTES + L2::B_BYTES + L2::SF_BYTES +
                                               L2::RAW_BYTES + 24) > 232448)
    --s;
  return s;
}

// whether variant (BN, Epi, KIND) runs with token-major accumulators
template <int BN, class Epi, int KIND>
struct GemmTok {
  static constexpr bool value = KIND == KIND_NVFP4 && BN == GEMM_BM && EpiTok<Epi>::value;
};

// An fp32 token-major epilogue may declare kTmaBoxes: each warp's 32 x 32
// chunk (rows = TMEM lanes, 32 consecutive features) goes out as one TMA
// store from a 128-byte-swizzled box (a lane writes its row's eight 16-byte
// pieces at positions c ^ (row % 8): no bank conflicts), instead of 32
// lanes each storing to its own row.  The functor gives the chunk's scale
// (scale(t)) and its place (target(t, row, feat, &map, &x, &y)).
template <class E, class = void>
struct EpiBoxes {
  static constexpr bool value = false;
};
template <class E>
struct EpiBoxes<E, std::void_t<decltype(E::kTmaBoxes)>> {
  static constexpr bool value = E::kTmaBoxes;
};

// A token-major epilogue that reads a second operand per element may declare
// kPre32: pre32(t, row, feat, valid, p) loads the 64 bytes of its chunk into
// p before the accumulator wait (so the load overlaps the tile's MMAs), and
// store32 takes them as a sixth argument.
template <class E, class = void>
struct EpiPre {
  static constexpr bool value = false;
};
template <class E>
struct EpiPre<E, std::void_t<decltype(E::kPre32)>> {
  static constexpr bool value = E::kPre32;
};

template <int BN, class Epi, int KIND>
struct GemmStg {
  static constexpr int value = !GemmTok<BN, Epi, KIND>::value ? STG_TRANSPOSE
                               : EpiBoxes<Epi>::value        ? STG_BOXES
                                                             : STG_NONE;
};

// "empty" barrier of ring slot s, and whether the producer waits on it there
template <class L>
__device__ __forceinline__ int empty_slot(int s) { return L::PAIRED_RELEASE ? s >> 1 : s; }
template <class L>
__device__ __forceinline__ bool empty_waits_at(int s) { return !L::PAIRED_RELEASE || !(s & 1); }
template <class L>
__device__ __forceinline__ bool empty_commits_at(int s) { return !L::PAIRED_RELEASE || (s & 1); }

template <int BN, int STAGES, class Epi, int KIND>
__global__ void __launch_bounds__(GemmLayout<BN, STAGES, KIND, GemmEpiWarps<BN, Epi>::value,
                                             GemmStg<BN, Epi, KIND>::value>::THREADS, 1)
k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
          const __grid_constant__ CUtensorMap tmB64, const TileSource src,
          const __grid_constant__ Epi epi, int* err, unsigned long long limit_ns) {
  using L = GemmLayout<BN, STAGES, KIND, GemmEpiWarps<BN, Epi>::value,
                       GemmStg<BN, Epi, KIND>::value>;
  constexpr bool FP4 = KIND == KIND_NVFP4;
  constexpr bool F8 = KIND == KIND_FP8;
  constexpr bool W4 = KIND == KIND_W4A16;
  constexpr bool BYTE_MAPS = FP4 || F8;   // operand maps in bytes (128 per stage row)
  constexpr bool TOK = GemmTok<BN, Epi, KIND>::value;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * L::A_BYTES;
  uint8_t* sSF = sB + STAGES * L::B_BYTES;           // NVFP4: [stage][A 2 KB | B 2 KB]
  uint8_t* sR = sSF + STAGES * L::SF_BYTES;          // W4A16: [stage][codes | atom]
  float* stg = reinterpret_cast<float*>(sR + STAGES * L::RAW_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(stg) + L::STG_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;   // [2]
  uint64_t* tempty = tfull + 2;       // [2]
  uint64_t* drain = tempty + 2;       // [1]
  uint64_t* aready = drain + 1;       // [STAGES] W4A16: the stage's f16 A tile is written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(aready + STAGES);
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
      mbar_init(&tempty[a], L::EPI_WARPS * 32);
    }
    mbar_init(drain, 1);
    if constexpr (W4)
      for (int s = 0; s < STAGES; ++s) mbar_init(&aready[s], W4_CONV_THREADS);
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
  const int num_tiles = gemm_num_tiles(src, BN);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Like the MMA issuer: the whole warp walks the ring (warp-uniform
    // coordinates and addresses), one elected lane issues the copies.  (A lone
    // thread spent about 300 ns issuing one k-step's copies, so the ring ran
    // about one stage ahead of the MMAs instead of STAGES.)
    // weights read once per launch are streamed past L2; weights that
    // several token blocks share are left to the default policy
    const uint64_t pol_a = src.a_stream_once ? policy_evict_first() : policy_evict_last();
    // B operand (and its scales) of one k-step: it depends on the previous
    // kernel; A (weights, and their scales) does not.  Elected lane only.
    auto load_b = [&](int st, const TileInfo& t, int kb) {
      const int nbig = t.nrows / GEMM_BROWS_BIG;
      const int nsmall = (t.nrows - nbig * GEMM_BROWS_BIG + GEMM_BROWS - 1) / GEMM_BROWS;
      for (int q = 0; q < L::KS; ++q) {
        const int bx = BYTE_MAPS ? (kb + q) * GEMM_ROW_BYTES : (kb + q) * GEMM_BK;
        uint8_t* b_dst = sB + st * L::B_BYTES + q * L::B_SUB;
        for (int j = 0; j < nbig; ++j)
          tma_load_2d(b_dst + j * GEMM_BROWS_BIG * GEMM_ROW_BYTES, &tmB64, bx,
                      t.row0 + j * GEMM_BROWS_BIG, &full[st]);
        for (int j = 0; j < nsmall; ++j) {
          const int r = nbig * GEMM_BROWS_BIG + j * GEMM_BROWS;
          tma_load_2d(b_dst + r * GEMM_ROW_BYTES, &tmB, bx, t.row0 + r, &full[st]);
        }
      }
      if constexpr (FP4)
        bulk_load(sSF + st * L::SF_BYTES + FP4_SF_STAGE_BYTES,
                  src.sfb + (static_cast<long>(t.tb) * src.kc + kb * 4) * SF_ATOM_BYTES,
                  FP4_SF_STAGE_BYTES, &full[st]);
    };
    int stage = 0;
    uint32_t phase = 0;
    long issued = 0;
    bool ok = true;
    bool waited = false;   // pdl_wait done; before it only A loads are issued
    int deferred = 0;      // k-steps of the first tile whose B loads wait for it
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const TileInfo t = gemm_tile(src, BN, tile);
      // B rows: 64-row boxes while 64 rows remain, then 16-row boxes
      const int nbig = t.nrows / GEMM_BROWS_BIG;
      const int nsmall = (t.nrows - nbig * GEMM_BROWS_BIG + GEMM_BROWS - 1) / GEMM_BROWS;
      const uint32_t tx =
          L::TX_A + L::KS * (nbig * GEMM_BROWS_BIG + nsmall * GEMM_BROWS) * GEMM_ROW_BYTES;
      for (int kb = t.kb0; kb < t.kb1; kb += L::KS) {
        if (empty_waits_at<L>(stage) &&
            !__all_sync(0xffffffffu, mbar_wait_bounded(&empty[empty_slot<L>(stage)], phase ^ 1,
                                                       abort_flag, err, limit_ns))) {
          ok = false;
          break;
        }
        // x coordinate in elements of the map: bf16 elements or bytes (NVFP4,
        // FP8); W4A16: bytes of FP4 codes, 32 per 64-wide sub-tile
        const int ax = W4 ? kb * 32 : BYTE_MAPS ? kb * GEMM_ROW_BYTES : kb * GEMM_BK;
        if (elect_one()) {
          mbar_arrive_expect_tx(&full[stage], tx);
          if constexpr (W4) {
            uint8_t* raw = sR + stage * L::RAW_BYTES;
            tma_load_2d_hint(raw, &tmA, ax, t.a_row, &full[stage], pol_a);
            // the sub-tiles' scale atoms are consecutive (64-element chunk fastest)
            bulk_load(raw + L::KS * W4_CODE_BYTES,
                      src.sfa + (static_cast<long>(t.a_row / GEMM_BM) * src.kc + kb) * SF_ATOM_BYTES,
                      L::KS * SF_ATOM_BYTES, &full[stage]);
          } else {
            tma_load_2d_hint(sA + stage * L::A_BYTES, &tmA, ax, t.a_row, &full[stage], pol_a);
          }
          if constexpr (FP4)
            bulk_load(sSF + stage * L::SF_BYTES,
                      src.sfa + (static_cast<long>(t.a_row / GEMM_BM) * src.kc + kb * 4) *
                                    SF_ATOM_BYTES,
                      FP4_SF_STAGE_BYTES, &full[stage]);
          if (waited) load_b(stage, t, kb);
        }
        __syncwarp();
        if (!waited && (++deferred == STAGES || kb + L::KS >= t.kb1)) {
          // the first tile's first stages: weights are in flight, now the
          // previous kernel's results
          pdl_wait();
          pdl_trigger();
          waited = true;
          if (elect_one())
            for (int j = 0; j < deferred; ++j) load_b(j, t, t.kb0 + j * L::KS);
          __syncwarp();
        }
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (!waited) {
      pdl_wait();
      pdl_trigger();
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
    // The whole warp walks the ring, so that descriptors and TMEM addresses
    // stay warp-uniform; one elected lane issues the tcgen05 instructions.
    // (Issued from a lone thread, an MMA whose descriptors change every
    // k-step costs the tensor pipe about twice the cycles.)
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    bool issued_any = false;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const TileInfo t = gemm_tile(src, BN, tile);
      if (t.kb0 >= t.kb1) continue;   // an empty K range: no accumulator, no epilogue
      const int n_mma = TOK ? GEMM_BM : (t.nrows + 15) & ~15;
      if (!__all_sync(0xffffffffu,
                      mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, err, limit_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      const uint32_t idesc = FP4  ? idesc_nvf4(GEMM_BM, n_mma)
                             : F8 ? idesc_f8(GEMM_BM, n_mma)
                             : W4 ? idesc_f16(GEMM_BM, n_mma)
                                  : idesc_bf16(GEMM_BM, n_mma);
      for (int kb = t.kb0; kb < t.kb1; kb += L::KS) {
        if (!__all_sync(0xffffffffu,
                        mbar_wait_bounded(&full[stage], phase, abort_flag, err, limit_ns))) {
          ok = false;
          break;
        }
        // W4A16: and the converter warps have written the stage's f16 A tile
        if (W4 && !__all_sync(0xffffffffu, mbar_wait_bounded(&aready[stage], phase, abort_flag,
                                                              err, limit_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t a0 = sdesc_k_sw128(smem_u32(sA + stage * L::A_BYTES));
        const uint64_t b0 = sdesc_k_sw128(smem_u32(sB + stage * L::B_BYTES));
        if (elect_one()) {
          if constexpr (FP4) {
            // scale atoms of this stage into its TMEM slot, then 4 MMAs of K=64
            const uint32_t sf_col = L::SF_COL0 + stage * 32;
            const uint32_t sf_smem = smem_u32(sSF + stage * L::SF_BYTES);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              tmem_cp_32x128b_warpx4(tmem_base + sf_col + 4 * k,
                                     sdesc_sf_atom(sf_smem + k * SF_ATOM_BYTES));
              tmem_cp_32x128b_warpx4(
                  tmem_base + sf_col + 16 + 4 * k,
                  sdesc_sf_atom(sf_smem + FP4_SF_STAGE_BYTES + k * SF_ATOM_BYTES));
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {   // +32 bytes per K=64 step
              if constexpr (TOK)
                umma_nvf4(d_tmem, b0 + 2 * k, a0 + 2 * k, idesc, tmem_base + sf_col + 16 + 4 * k,
                          tmem_base + sf_col + 4 * k, (kb != t.kb0) || (k != 0));
              else
                umma_nvf4(d_tmem, a0 + 2 * k, b0 + 2 * k, idesc, tmem_base + sf_col + 4 * k,
                          tmem_base + sf_col + 16 + 4 * k, (kb != t.kb0) || (k != 0));
            }
          } else if constexpr (F8) {
#pragma unroll
            for (int k = 0; k < 4; ++k)   // +32 bytes per K=32 step
              umma_f8(d_tmem, a0 + 2 * k, b0 + 2 * k, idesc, (kb != t.kb0) || (k != 0));
          } else {
#pragma unroll
            for (int q = 0; q < L::KS; ++q) {
              // sub-tile q: its own 128-byte-swizzled regions (+A_SUB, +B_SUB bytes)
              const uint64_t aq = a0 + ((q * L::A_SUB) >> 4), bq = b0 + ((q * L::B_SUB) >> 4);
#pragma unroll
              for (int k = 0; k < GEMM_BK / 16; ++k)   // +32 bytes per K=16 step
                umma_bf16(d_tmem, aq + 2 * k, bq + 2 * k, idesc,
                          (kb != t.kb0) || (q != 0) || (k != 0));
            }
          }
          if (empty_commits_at<L>(stage)) umma_commit(&empty[empty_slot<L>(stage)]);
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
      if (elect_one()) umma_commit(drain);
      __syncwarp();
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < limit_ns) {
      }
    }
    __syncwarp();
  } else if (warp < 2 + L::EPI_WARPS) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                  // TMEM lane quarter of this warp
    const int ew = warp - 2;                 // epilogue warp index
    const int cstep = 32 * (L::EPI_WARPS / 4);   // column chunks: this warp's, then every cstep
    const int cfirst = 32 * (ew / 4);
    float* my = stg + ew * 32 * GEMM_STG_LD;
    int nbox = 0;   // TMA boxes this warp has stored (kTmaBoxes epilogues)
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const TileInfo t = gemm_tile(src, BN, tile);
      if (t.kb0 >= t.kb1) continue;   // skipped by the MMA warp too
      // token-major: this warp's chunks c = cfirst + i * cstep, i < NCH
      constexpr int NCH = GEMM_BM / (32 * (L::EPI_WARPS / 4));
      [[maybe_unused]] uint4 pre[TOK && EpiPre<Epi>::value ? NCH : 1][4];
      if constexpr (TOK && EpiPre<Epi>::value) {
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          const int feat = t.fb * GEMM_BM + cfirst + i * cstep;
          const bool valid = q * 32 + lane < t.nrows && feat < src.m_valid;
          epi.pre32(t, static_cast<long>(t.row0 + q * 32 + lane), feat, valid, pre[i]);
        }
      }
      // one lane waits, the warp follows: the TMEM loads below are .sync.aligned
      int ok = 0;
      if (lane == 0) ok = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, err, limit_ns);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      tc_fence_after();
      if constexpr (TOK) {
        // lane = token row q*32 + lane of the tile; 32 features per TMEM load
        const int rbase = q * 32;
        if (rbase < t.nrows) {
#pragma unroll
          for (int i = 0; i < NCH; ++i) {
            const int c = cfirst + i * cstep;
            uint32_t r[32];
            tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + c, r);
            tmem_ld_wait();
            const int feat = t.fb * GEMM_BM + c;
            if constexpr (EpiBoxes<Epi>::value) {
              // whole chunks only: rows and features come in multiples of 32
              if (feat < src.m_valid) {
                float* box = stg + (ew * 2 + (nbox & 1)) * GEMM_BOX_FLOATS;
                // the box stored two chunks ago has been read out of this buffer
                if (lane == 0) bulk_wait_group_read<1>();
                __syncwarp();
                const float sc = epi.scale(t);
                float4* row = reinterpret_cast<float4*>(box + lane * 32);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                  row[k ^ (lane & 7)] =
                      make_float4(__uint_as_float(r[4 * k]) * sc, __uint_as_float(r[4 * k + 1]) * sc,
                                  __uint_as_float(r[4 * k + 2]) * sc,
                                  __uint_as_float(r[4 * k + 3]) * sc);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                  const CUtensorMap* map;
                  int x, y;
                  epi.target(t, static_cast<long>(t.row0 + rbase), feat, &map, &x, &y);
                  tma_store_2d(map, box, x, y);
                  bulk_commit_group();
                }
                ++nbox;
              }
            } else {
              const bool valid = rbase + lane < t.nrows && feat < src.m_valid;
              float v[32];
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
              if constexpr (EpiPre<Epi>::value)
                epi.store32(t, static_cast<long>(t.row0 + rbase + lane), feat, v, valid, pre[i]);
              else
                epi.store32(t, static_cast<long>(t.row0 + rbase + lane), feat, v, valid);
            }
          }
        }
      } else {
      const int feat_base = t.fb * GEMM_BM + q * 32;
      for (int c0 = cfirst; c0 < t.nrows; c0 += cstep) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + c0, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) my[j * GEMM_STG_LD + lane] = __uint_as_float(r[j]);
        __syncwarp();
        if constexpr (EpiVec<Epi>::value == 16) {
          // lanes 2j, 2j+1 hold the two 16-feature groups of token row j
#pragma unroll
          for (int it = 0; it < 2; ++it) {
            const int item = lane + 32 * it;
            const int j = item >> 1;
            const int g = item & 1;
            const int feat = feat_base + g * 16;
            const bool valid = c0 + j < t.nrows && feat < src.m_valid;
            const float4* p = reinterpret_cast<const float4*>(my + j * GEMM_STG_LD + g * 16);
            const float4 q0 = p[0], q1 = p[1], q2 = p[2], q3 = p[3];
            const float v[16] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w,
                                 q2.x, q2.y, q2.z, q2.w, q3.x, q3.y, q3.z, q3.w};
            epi.store16(t, static_cast<long>(t.row0 + c0 + j), feat, v, valid);
          }
          __syncwarp();
        } else {
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            // lanes 4j..4j+3 hold the four 8-feature groups of token row j
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
      }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if constexpr (TOK && EpiBoxes<Epi>::value) {
      // the boxes' reads of shared memory end before the CTA does
      if (lane == 0) bulk_wait_group_read<0>();
      __syncwarp();
    }
  }

  if constexpr (W4) {
    if (warp >= 2 + L::EPI_WARPS) {
      // ---------------------------------------------------------- converters
      // One thread per row of the 128-row weight tile and K sub-tile: its 64
      // E2M1 codes times the E4M3 scales of their 16-blocks, as f16 (the
      // product of an E2M1 and an E4M3 value is exact in f16), written in
      // the 128-byte-swizzled K-major layout the MMA reads; the per-expert
      // global scale is applied in the epilogue.
      const int ct = threadIdx.x - (2 + L::EPI_WARPS) * 32;
      const int r = ct >> 1, q = ct & 1;   // row, and K sub-tile of the stage
      static_assert(W4_CONV_THREADS == 128 * W4_KSUB, "a converter thread per row and sub-tile");
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const TileInfo t = gemm_tile(src, BN, tile);
        for (int kb = t.kb0; kb < t.kb1; kb += L::KS) {
          if (!__all_sync(0xffffffffu,
                          mbar_wait_bounded(&full[stage], phase, abort_flag, err, limit_ns))) {
            ok = false;
            break;
          }
          const uint8_t* raw = sR + stage * L::RAW_BYTES;
          // codes: [128 rows][KS x 32 B]; scales: KS atoms after them
          const uint4 c0 = *reinterpret_cast<const uint4*>(raw + r * 32 * L::KS + q * 32);
          const uint4 c1 = *reinterpret_cast<const uint4*>(raw + r * 32 * L::KS + q * 32 + 16);
          const uint32_t sc4 = *reinterpret_cast<const uint32_t*>(
              raw + L::KS * W4_CODE_BYTES + q * SF_ATOM_BYTES + sf_atom_offset(r, 0));
          const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
          uint8_t* dst = sA + stage * L::A_BYTES + q * L::A_SUB + r * GEMM_ROW_BYTES;
#pragma unroll
          for (int blk = 0; blk < 4; ++blk) {   // 16-element blocks of the row
            const uint32_t sb = (sc4 >> (8 * blk)) & 0xFFu;
            const uint32_t s2 = f16x2_from_e4m3x2(sb | (sb << 8));
            uint32_t lo[4], hi[4];
            f16x2_from_e2m1x8(cw[2 * blk], lo);
            f16x2_from_e2m1x8(cw[2 * blk + 1], hi);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              lo[i] = hmul2_f16(lo[i], s2);
              hi[i] = hmul2_f16(hi[i], s2);
            }
            // elements 16 blk .. +15 are 16-byte chunks 2 blk and 2 blk + 1 of the row
            *reinterpret_cast<uint4*>(dst + (((2 * blk) ^ (r & 7)) * 16)) =
                make_uint4(lo[0], lo[1], lo[2], lo[3]);
            *reinterpret_cast<uint4*>(dst + (((2 * blk + 1) ^ (r & 7)) * 16)) =
                make_uint4(hi[0], hi[1], hi[2], hi[3]);
          }
          fence_proxy_async_smem();
          mbar_arrive(&aready[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, L::TMEM_COLS);
}

// Sum of the K-slice partials in slice order (deterministic), then the real
// epilogue: thread per 8 consecutive features of one row.  All threads of a
// warp reach the epilogue call (lanes 2i and 2i+1 hold one 16-feature block).
template <class Epi>
__global__ void __launch_bounds__(256) k_splitk_reduce(const float* __restrict__ part, int ksplit,
                                                       int T, int F, const Epi epi) {
  pdl_wait();
  pdl_trigger();
  const long g = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int f8 = F / 8;
  const long row = g / f8;
  const bool valid = row < T;
  const long r = valid ? row : 0;
  const int feat = valid ? static_cast<int>(g - row * f8) * 8 : 0;
  float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (valid) {
    for (int s = 0; s < ksplit; ++s) {
      const float4* p =
          reinterpret_cast<const float4*>(part + (static_cast<long>(s) * T + r) * F + feat);
      const float4 a = p[0], b = p[1];
      v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
      v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
    }
  }
  TileInfo t{};
  epi.store8(t, r, feat, v, valid);
}

// Split-K reduction of the router GEMM [W_r; W_dn; W_s1] x with the router
// fused into it.  Blocks [0, rblocks) take one token per warp: its N logits,
// the K slices summed in slice order (as k_splitk_reduce), written as fp32
// logits and held in the lanes (expert lane + 32 i) for the warp's top-K,
// scores and renormalised weights (route_select).  The other blocks reduce
// features [N, F) and apply the epilogue, a thread per 8 features of a row.
template <class Epi, int NPL>
__global__ void __launch_bounds__(256) k_splitk_reduce_route(
    const float* __restrict__ part, int ksplit, int T, int F, int N, const Epi epi,
    const float* __restrict__ bias, int K, float* __restrict__ logits,
    int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, int rblocks) {
  pdl_wait();
  pdl_trigger();
  if (static_cast<int>(blockIdx.x) < rblocks) {
    const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    const int npl = N >> 5;
    float zz[NPL], bb[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      zz[i] = 0.0f;
      bb[i] = (i < npl && bias) ? bias[lane + 32 * i] : 0.0f;
    }
    for (int sl = 0; sl < ksplit; ++sl) {
      const float* p = part + (static_cast<int64_t>(sl) * T + t) * F;
#pragma unroll
      for (int i = 0; i < NPL; ++i)
        if (i < npl) zz[i] += p[lane + 32 * i];
    }
    float* zrow = logits + t * N;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (i < npl) zrow[lane + 32 * i] = zz[i];
    __syncwarp();   // the row's logits, written by all lanes, are read back below
    route_select<NPL>(zz, bb, npl, zrow, K, lane, t, topk_idx, topk_w);
    return;
  }
  const long g = static_cast<long>(blockIdx.x - rblocks) * blockDim.x + threadIdx.x;
  const int f8 = (F - N) / 8;
  const long row = g / f8;
  const bool valid = row < T;
  const long r = valid ? row : 0;
  const int feat = N + (valid ? static_cast<int>(g - row * f8) * 8 : 0);
  float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (valid) {
    for (int sl = 0; sl < ksplit; ++sl) {
      const float4* p =
          reinterpret_cast<const float4*>(part + (static_cast<long>(sl) * T + r) * F + feat);
      const float4 a = p[0], b = p[1];
      v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
      v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
    }
  }
  TileInfo ti{};
  epi.store8(ti, r, feat, v, valid);
}

// ---------------------------------------------------------------------------
// epilogue helpers

__device__ __forceinline__ void store8_bf16(__nv_bfloat16* dst, const float* v) {
  __nv_bfloat162 p[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<uint4*>(p);
}

// 8 floats -> 8 f16 (16-byte store), finite: saturating at +-65504
__device__ __forceinline__ void store8_f16(__half* dst, const float* v) {
  __half2 p[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    p[i] = __floats2half2_rn(fminf(fmaxf(v[2 * i], -65504.0f), 65504.0f),
                             fminf(fmaxf(v[2 * i + 1], -65504.0f), 65504.0f));
  *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<uint4*>(p);
}

__device__ __forceinline__ float sqrelu(float a) {
  const float r = fmaxf(a, 0.0f);
  return r * r;
}

// NVFP4 quantisation of 8 features whose 16-block partner is lane ^ 1 (lane
// pairs hold a block's halves; every lane of the warp must call this).
// Returns this lane's 4 code bytes (lower feature in the lower nibble) and
// the block's E4M3 scale code.
__device__ __forceinline__ uint32_t nvfp4_pair(const float* v, float g, uint8_t* sc) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  const float six_g = __fmul_rn(6.0f, g);
  const float sbf = six_g > 0.0f ? __fdiv_rn(amax, six_g) : 0.0f;
  const uint8_t code = e4m3_code(sbf);
  const float denom = __fmul_rn(e4m3_value(code), g);
  const float rcp = denom > 0.0f ? __fdiv_rn(1.0f, denom) : 0.0f;
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w |= e2m1x2(__fmul_rn(v[2 * i], rcp), __fmul_rn(v[2 * i + 1], rcp)) << (8 * i);
  *sc = code;
  return w;
}

// nvfp4_pair with the block scale and its reciprocal from the scale tables of
// the global scale (nvfp4_scale_tab): the same codes, no division.
__device__ __forceinline__ uint32_t nvfp4_pair_tab(const float* v, const float* __restrict__ tab,
                                                   uint8_t* sc) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  float rcp;
  const uint8_t code = nvfp4_scale_tab(amax, tab, &rcp);
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w |= e2m1x2(__fmul_rn(v[2 * i], rcp), __fmul_rn(v[2 * i + 1], rcp)) << (8 * i);
  *sc = code;
  return w;
}

}  // namespace lmoe
