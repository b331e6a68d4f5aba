// Warp-specialised, persistent FP8 block-scaled GEMM for sm_100a.
//
//   D[m,n] = bf16( sum_kb sa[m,kb] * sb[n/128,kb] * sum_{k in block kb} A[m,k] B[n,k] )
//
// (DeepGEMM pages: the juejin.cn Open-Source-Week article, "4 DeepGEMM 架构分析":
// two-level accumulation, warp-specialised TMA / tensor-core / CUDA-core
// overlap, one scheduler for dense and grouped GEMMs with rasterisation; the
// nightvoyager.top report, "UE8M0 int32 packing" and "SF 双 path".)
//
// B200 design.  The per-128-K scale promotion is done by the tensor core
// itself: tcgen05.mma kind::mxf8f6f4 with block scaling multiplies every
// 32-wide K slice by 2^(ea-127) * 2^(eb-127) before accumulating in FP32 in
// tensor memory.  The four K=32 MMAs of a 128-wide block share one scale per
// row (A) and one per column (B), which is exactly the 1x128 / 128x128
// recipe; the scales are powers of two, so the scaling itself is exact.
//
// CTAS = 1: one CTA computes a 128 x BN tile.  CTAS = 2: a cluster of two CTAs
// computes a 256 x BN tile with tcgen05 cta_group::2 MMAs issued by the first
// CTA; each CTA loads its own 128 rows of A and BN/2 rows of B, so every SM
// fetches half of the B tile it would need alone.  No load is multicast.
//
// Roles (one CTA per SM, persistent over output tiles):
//   MMA issuer   TMEM owner (warp 0); in the first CTA of a pair the issuer:
//                tcgen05.cp of the scales, tcgen05.mma, commits of stage
//                releases and finished accumulators (to both CTAs of a pair).
//   producer     TMA loads of A/B K-blocks into a STAGES-deep ring.
//   scale        for every group of 4 K-blocks, the packed UE8M0 words of
//   producer     the tile (or fp32 scales packed here), rearranged into the
//                tensor-memory scale layout (row/column j of a 128-group at
//                lane j%32, column j/32), into a 2- or 4-deep ring of its own,
//                so the load latency of the words never sits on the TMA path.
//   epilogue     eight warps: tcgen05.ld of this CTA's accumulator rows (two
//                warps per TMEM lane quarter, alternate 32-column chunks),
//                BF16 RNE, swizzled staging + TMA store for fully valid 32-row
//                slices, predicated stores for slices with padding/masked rows.
// Warp w runs on sub-partition w % 4, which also fixes the TMEM lane quarter
// it may read.  The issuing threads are sensitive to other warps' instructions
// on their sub-partition, so they share theirs only with a (light) producer
// and two epilogue warps; the scale producers sit on the other two:
//   PIPES = 1: warp 0 issuer, 1 producer, 2 scale producer, 3-10 epilogue.
//   PIPES = 2: warps 0/1 issuers, 2/3 scale producers, 4/5 producers (of
//              pipelines 0/1), 6-13 epilogue.
// Accumulators are double-buffered in TMEM when they fit, so the epilogue of
// tile i overlaps the MMAs of tile i+1.
//
// LAYOUT (dense only): bit 0 set = A stored K x M (MN-major), bit 1 set = B
// stored K x N (MN-major); the pages' NT / NN / TN / TT layouts are LAYOUT
// 0 / 2 / 3 / 1.  An MN-major operand is loaded as 128 x 128 TMA boxes whose
// 128-byte rows run along M (or N) and read by the tensor core through an
// MN-major descriptor: 128-byte swizzle atoms of 8 K-rows, SBO = 1024 B
// between atoms along K, LBO = 16 KB between 128-wide atoms along M/N.
// Each CTA's share of an MN-major B tile is a whole number of 128 columns.
//
// SPLITK (with PIPES = 2): both pipelines work on every tile, pipeline p on
// its half of the K groups, into its own accumulator; the epilogue adds the
// two.  For problems of a few rows (decode) whose K loop is bound by the
// issuing thread, this halves the loop without any workspace.  Without
// SPLITK, two pipelines split the same way only the last tile of a CTA with
// an odd tile count (dense and masked), which would otherwise run alone.
//
// PIPES = 2: every tcgen05 instruction costs its issuing thread
// a fixed ~60-70 cycles, so one thread issuing the 4 MMAs + commit of a
// 128x224x128 K block spends ~300 of the block's 448 tensor-pipe cycles on
// issue alone and, with its waits, cannot keep the pipe busy.  The cost is
// per thread: two threads issuing into two accumulators overlap.  So the CTA
// runs two copies of the load/issue/scale pipeline (warps 0, 4, 2 and 1, 5,
// 3), each with half of the stage ring, its own scale ring and scale slots
// in TMEM, taking alternate tiles of the CTA: tile i goes to pipeline i & 1
// and accumulator i & 1.  The epilogue warps drain the accumulators in tile
// order, as with one pipeline.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace dg {

// Device error word (DG_DEVERR_* bits); one per device, read and cleared by the host.
__device__ int g_dg_error = 0;

enum : int { MODE_DENSE = 0, MODE_CONTIG = 1, MODE_MASKED = 2 };

constexpr int kBK = 128;
// per pipeline an MMA issuer, a producer and a scale producer; eight epilogue warps
template <int PIPES>
constexpr int kThreadsFor = 32 * (8 + 3 * PIPES);
constexpr int kThreads = kThreadsFor<1>;
constexpr int kMaxMaskedGroups = 512;
// Contiguous layout on CTA pairs: the 128-row blocks are paired within each
// expert's run of blocks by a table built on the device, for up to this many
// blocks (M_total <= 131072 rows); the host uses 1-CTA tiles beyond.
constexpr int kMaxContigBlocks = 1024;
constexpr int kMaxSmem = 232448;                  // opt-in shared memory per block on sm_100
// Default limit of every pipeline wait: 2 s, far above any legitimate wait.
// The main-loop waits take theirs from GemmArgs::wait_limit_ns (this value
// unless the host changed it); the waits that drain copies and MMAs in
// flight before a CTA exits always keep this one.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct GemmArgs {
  int rows;           // dense: M; contiguous: M_total; masked: M_max
  int N, K, G;
  int num_m_blocks;   // dense / contiguous, in tiles of 128 * CTAS rows
  int num_n_blocks;
  int raster_m;       // rasterisation group height in M blocks
  int kp;             // words of packed scales along K: ceil(K/128/4)
  int mn4a;           // words of packed A scales along M: align4(rows)
  int nb4;            // words of packed B scales along N: align4(ceil(N / sfb_gran))
  int sfb_gran;       // rows of B per scale: 128 (128x128 blocks) or 1 (1x128 per row)
  const uint32_t* sfa;     // packed UE8M0 words of A, or nullptr when sfa_f32 is given
  const float* sfa_f32;    // A's fp32 power-of-two scales [G][rows][K/128], packed by the scale producer
  int sfa_f32_vec;         // 1: rows of sfa_f32 are 16-byte aligned (K/128 % 4 == 0): one 16-byte load per word
  const uint32_t* sfb;
  const int32_t* m_indices;
  const int32_t* masked_m;
  __nv_bfloat16* d;   // BF16 output (OUT_F32 == false)
  float* d32;         // FP32 output (OUT_F32 == true)
  const float* c;     // optional FP32 addend [rows][N] (OUT_F32 only), nullptr for none
  uint64_t wait_limit_ns;  // limit of each main-loop wait before the CTA gives up
};

template <int BN, int STAGES, int CTAS, int PIPES = 1, int LAYOUT = 0, bool MASKED = true, bool CPAIRS = false,
          int A_ROWS = 128>
struct Layout {
  static_assert(!(LAYOUT & 2) || (BN / CTAS) % 128 == 0, "an MN-major B tile is whole 128-column boxes per CTA");
  static_assert(CTAS == 1 || CTAS == 2, "CTAS is 1 or 2");
  static_assert(PIPES == 1 || (PIPES == 2 && STAGES % 2 == 0), "two pipelines need an even number of stages");
  static constexpr int kStagesPer = STAGES / PIPES;     // stages of each pipeline's ring
  static_assert(BN % 32 == 0 && (BN / CTAS) % 16 == 0 && BN >= 32 && BN <= 256,
                "BN must be a multiple of 32 in [32, 256] with BN/CTAS a multiple of 16");
  static constexpr int kTileM = 128 * CTAS;
  static constexpr int kBRows = BN / CTAS;              // rows of B loaded by each CTA
  static constexpr int kNB128 = (BN + 127) / 128;       // 128-column groups of B scales
  // Rows of A per stage: 128, or 64 for problems of at most 64 rows (A
  // K-major, 1-CTA tiles).  The MMA stays 128 rows tall; with 64-row stages
  // its rows 64-127 read the next 8 KB of shared memory (the next stage, or
  // the first B stage), so those accumulator rows hold garbage that no store
  // writes out (they are rows >= M), and each stage takes a third less room.
  static_assert(A_ROWS == 128 || (A_ROWS == 64 && CTAS == 1 && (LAYOUT & 1) == 0),
                "64-row A stages are built for K-major A on 1-CTA tiles");
  static constexpr int kABytes = A_ROWS * kBK;          // 16 KB (8 KB with 64-row stages)
  static constexpr int kBBytes = kBRows * kBK;
  // Scale words of one K group in shared memory, as tcgen05.cp sources:
  // 128 rows x 32 B (core-matrix layout) holding [SFA | SFB of columns 0-127]
  // for TMEM columns +0..+7 (rows r, r+32, r+64, r+96 identical), then, when
  // BN > 128, 32 rows x 16 B with SFB of columns 128-255 for columns +8..+11.
  static constexpr int kSftMainBytes = 4096;
  static constexpr int kSftBytes = kSftMainBytes + (kNB128 == 2 ? 512 : 0);
  static constexpr int kEpiBuf = 32 * 32 * 2;           // 32 rows x 32 bf16 (or x 16 fp32)
  // TMEM columns: accumulators, then per pipeline two scale slots of 16
  // columns (SFA at +0, SFB at +4).
  static constexpr int kSfSlotCols = 16;
  static constexpr int kAccStride = PIPES == 2 ? (BN + 31) / 32 * 32 : (BN <= 128 ? 128 : 256);
  static constexpr int kNumAcc = (PIPES == 2 || kAccStride + BN + 2 * kSfSlotCols <= 512) ? 2 : 1;
  static constexpr int kSfBaseCol =
      PIPES == 2 ? 2 * kAccStride : (kNumAcc - 1) * kAccStride + ((BN + 15) / 16) * 16;
  static constexpr int kTmemCols = 512;
  // shared-memory offsets (from a 1024-byte aligned base)
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + STAGES * kABytes;
  static constexpr int kOffSft = kOffB + STAGES * kBBytes;
  // the masked layout's per-expert prefix and counts; the contiguous layout's
  // pair table on CTA pairs (count, then first blocks); other modes keep none
  static constexpr int kGroupsBytes =
      MASKED ? (2 * kMaxMaskedGroups + 1) * 4 : (CPAIRS ? (kMaxContigBlocks + 1) * 4 : 0);
  // scale ring depth (per pipeline): 4 groups when shared memory allows, else 2
  static constexpr int kSfRing =
      (kOffSft + PIPES * 4 * kSftBytes + 1023) / 1024 * 1024 + 8 * kEpiBuf + 4096 + kGroupsBytes + 1024 <= kMaxSmem
          ? 4
          : 2;
  static constexpr int kOffEpi = ((kOffSft + PIPES * kSfRing * kSftBytes + 1023) / 1024) * 1024;
  static constexpr int kOffBar = kOffEpi + 8 * kEpiBuf;  // one staging buffer per epilogue warp
  static constexpr int kNumBars = 2 * STAGES + 2 * 2 + 2 + 2 * PIPES * 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // tmem addr, abort flag, 2 peer load counts
  static constexpr int kOffGroups = kOffMisc + 16;          // masked: prefix[G+1], count[G]; contiguous pairs
  static constexpr int kSmemBytes = kOffGroups + kGroupsBytes + 1024;
  static_assert(kSmemBytes <= kMaxSmem, "shared-memory budget exceeded");
  static_assert(kSfBaseCol + PIPES * 2 * kSfSlotCols <= kTmemCols, "TMEM budget exceeded");
};

struct Tile {
  int m_blk, n_blk, g;
  int row0;  // first row of the tile in A / D (per expert for masked)
};

// UE8M0 byte of an fp32 scale: the exponent field of a positive normal power
// of two, 0 for 2^-127 (the fp32 subnormal 0x00400000); anything else is not
// representable and gives byte 0 with `bad` set.
__device__ __forceinline__ uint32_t ue8m0_byte_checked(uint32_t bits, bool& bad) {
  const uint32_t e = (bits >> 23) & 0xFFu;
  if ((bits >> 31) == 0 && e >= 1 && e <= 254 && (bits & 0x7FFFFFu) == 0) return e;
  if (bits != 0x00400000u) bad = true;
  return 0u;
}

// Packed word of K blocks 4kp..4kp+3 of one row of fp32 scales (kbn blocks per row).
__device__ __forceinline__ uint32_t pack_scale_word(const float* row, int kp, int kbn, bool vec) {
  uint32_t word = 0;
  bool bad = false;
  if (vec) {  // 4 | kbn and 16-byte aligned rows: the word's four scales in one load
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(row) + kp);
    word = ue8m0_byte_checked(v.x, bad) | (ue8m0_byte_checked(v.y, bad) << 8) |
           (ue8m0_byte_checked(v.z, bad) << 16) | (ue8m0_byte_checked(v.w, bad) << 24);
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int k = 4 * kp + j;
      if (k < kbn) word |= ue8m0_byte_checked(__float_as_uint(__ldg(row + k)), bad) << (8 * j);
    }
  }
  if (bad) atomicOr(&g_dg_error, 0x1);
  return word;
}

// Bounded wait on an mbarrier phase.  Returns false when the CTA is aborting
// (another role gave up) or this wait exceeded its limit (sets the error word).
// A plain try_wait may keep the thread suspended until the phase completes,
// so every probe here carries a suspend-time hint (kPollNs): the loop looks
// at the clock and the abort flag at least that often.
constexpr uint32_t kPollNs = 1000;
template <bool kCluster>
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                           uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (kCluster ? mbar_try_wait_cluster_hint(bar, parity, kPollNs) : mbar_try_wait_hint(bar, parity, kPollNs))
      return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(&g_dg_error, 0x10);
      return false;
    }
  }
}

// Wait used while draining at exit: ignores the abort flag, still bounded.
__device__ __forceinline__ void wait_phase_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait_hint(bar, parity, kPollNs)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_dg_error, 0x10);
      return;
    }
  }
}

template <int MODE, int CTAS>
__device__ __forceinline__ int total_tiles(const GemmArgs& p, const int* prefix) {
  if (MODE == MODE_MASKED) return prefix[p.G];
  if (MODE == MODE_CONTIG && CTAS == 2) return prefix[0] * p.num_n_blocks;  // pairs from the table
  return p.num_m_blocks * p.num_n_blocks;
}

// Tile order: dense / contiguous use groups of `raster_m` M blocks swept
// column by column, so concurrently running CTAs share A rows and B columns
// in L2; masked runs expert by expert, N block by N block, M blocks fastest.
// Contiguous 2-CTA tiles take their M units from the pair table: pairs of
// consecutive 128-row blocks of one expert's run, a run of odd length ending
// in a block on its own (the pair's second CTA then stores nothing).
template <int MODE, int TILE_M>
__device__ __forceinline__ Tile tile_of(int t, const GemmArgs& p, const int* prefix,
                                        const int* counts) {
  Tile tl;
  if (MODE == MODE_CONTIG && TILE_M == 256) {
    const int pairs = prefix[0];
    const int per_group = p.raster_m * p.num_n_blocks;
    const int grp = t / per_group;
    const int first = grp * p.raster_m;
    const int gsize = min(p.raster_m, pairs - first);
    const int within = t - grp * per_group;
    tl.m_blk = first + within % gsize;
    tl.n_blk = within / gsize;
    tl.g = 0;
    tl.row0 = prefix[1 + tl.m_blk] * 128;
    return tl;
  }
  if (MODE == MODE_MASKED) {
    int g = 0;
    while (prefix[g + 1] <= t) ++g;
    const int local = t - prefix[g];
    const int cnt = (counts[g] + TILE_M - 1) / TILE_M;
    tl.g = g;
    tl.n_blk = local / cnt;
    tl.m_blk = local - tl.n_blk * cnt;
  } else {
    const int per_group = p.raster_m * p.num_n_blocks;
    const int grp = t / per_group;
    const int first_m = grp * p.raster_m;
    const int gsize = min(p.raster_m, p.num_m_blocks - first_m);
    const int within = t - grp * per_group;
    tl.m_blk = first_m + within % gsize;
    tl.n_blk = within / gsize;
    tl.g = 0;
  }
  tl.row0 = tl.m_blk * TILE_M;
  return tl;
}

// N width of the MMAs of a tile.  A ragged last N tile (fewer than BN columns
// of D left) runs narrower MMAs, so the tensor core does not compute columns
// that are never stored.  Only widths that built configurations use already
// are taken: 64 (one CTA) and 128.  An MN-major B tile keeps its width (its
// loads are whole 128-column boxes).
template <int BN, int CTAS, int LAYOUT>
__device__ __forceinline__ int tile_mma_n(int n0, int N) {
  if constexpr ((LAYOUT & 2) != 0) return BN;
  const int rem = N - n0;
  if (rem >= BN) return BN;
  if (CTAS == 1 && BN > 64 && rem <= 64) return 64;
  if (BN > 128 && rem <= 128) return 128;
  return BN;
}

// Expert of a contiguous-layout tile, or -1 when the tile has nothing to
// compute: its (first) block starts with a padding row or an out-of-range index.
template <int CTAS>
__device__ __forceinline__ int contig_expert(const Tile& tl, const GemmArgs& p) {
  const int blk = tl.row0 / 128;
  if (blk >= p.rows / 128) return -1;
  const int e = __ldg(&p.m_indices[blk * 128]);
  if (e < 0 || e >= p.G) return -1;
  return e;
}

template <int BN, int STAGES, int MODE, int CTAS, bool OUT_F32 = false, int PIPES = 1, int LAYOUT = 0,
          bool SPLITK = false, int A_ROWS = 128>
__global__ void __launch_bounds__(kThreadsFor<PIPES>, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_d, const GemmArgs p) {
  using L = Layout<BN, STAGES, CTAS, PIPES, LAYOUT, MODE == MODE_MASKED, MODE == MODE_CONTIG && CTAS == 2, A_ROWS>;
  static_assert(A_ROWS == 128 || MODE != MODE_CONTIG, "64-row A stages hold one tile's rows: dense and masked only");
  static_assert(LAYOUT == 0 || MODE == MODE_DENSE, "MN-major operands are built for the dense GEMM only");
  static_assert(!SPLITK || PIPES == 2, "split-K runs on two pipelines");
  constexpr bool kAmn = (LAYOUT & 1) != 0;
  constexpr bool kBmn = (LAYOUT & 2) != 0;
  constexpr bool kPair = CTAS == 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* tmem_full = bars + 2 * STAGES;
  uint64_t* tmem_empty = bars + 2 * STAGES + 2;
  uint64_t* final_bar = bars + 2 * STAGES + 4;  // one per pipeline
  uint64_t* sf_full = bars + 2 * STAGES + 6;    // [pipeline][ring]
  uint64_t* sf_empty = sf_full + PIPES * L::kSfRing;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  // pairs: loads issued by the second CTA's producers, per pipeline (written into the first CTA)
  uint32_t* peer_loads = reinterpret_cast<uint32_t*>(smem + L::kOffMisc + 8);
  uint32_t prod_it = 0;  // loads issued by this warp's pipeline (producer warps)
  int* prefix = reinterpret_cast<int*>(smem + L::kOffGroups);
  int* counts = prefix + kMaxMaskedGroups + 1;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int num_kb = p.K / kBK;
  const uint32_t rank = kPair ? cluster_cta_rank() : 0;
  const int unit0 = kPair ? static_cast<int>(blockIdx.x / 2) : static_cast<int>(blockIdx.x);
  const int units = kPair ? static_cast<int>(gridDim.x / 2) : static_cast<int>(gridDim.x);
  // role and pipeline of this warp, and the pipeline's share of the rings
  constexpr int kEpi0 = 3 * PIPES;  // first epilogue warp
  const bool is_issuer = warp < PIPES;
  const bool is_producer = PIPES == 2 ? (warp == 4 || warp == 5) : warp == 1;
  const bool is_scale = PIPES == 2 ? (warp == 2 || warp == 3) : warp == 2;
  const int pipe = (PIPES == 2 && warp < kEpi0) ? (warp & 1) : 0;
  const int sbase = pipe * L::kStagesPer;
  const int rbase = pipe * L::kSfRing;
  // With two pipelines and no split-K, the last tile of an odd count is split
  // over both pipelines, so the last round does not run on one issuing
  // thread.  The contiguous layout's tile count depends on device data and
  // keeps plain alternation.
  constexpr bool kTailSplit = PIPES == 2 && !SPLITK && MODE != MODE_CONTIG;

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], CTAS);
      mbar_init(&empty_bar[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tmem_full[i], 1);
      mbar_init(&tmem_empty[i], 8 * CTAS);
      mbar_init(&final_bar[i], 1);
    }
    for (int i = 0; i < PIPES * L::kSfRing; ++i) {
      mbar_init(&sf_full[i], CTAS);
      mbar_init(&sf_empty[i], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
    prefetch_tensormap(&tm_d);
  }
  __syncwarp();
  if (warp == 0) {
    tmem_alloc<CTAS>(tmem_holder, L::kTmemCols);
    tmem_relinquish<CTAS>();
  }
  // Everything above touches no global memory, so it overlaps the previous
  // grid's tail; from here on its results are visible.
  grid_dep_wait();
  grid_dep_launch();
  if (MODE == MODE_MASKED && warp == kEpi0) {
    // counts[g] = clamp(masked_m[g], 0, M_max); prefix = running sum of tiles
    int run = 0;
    for (int base = 0; base < p.G; base += 32) {
      const int g = base + lane;
      int tiles = 0;
      if (g < p.G) {
        int mg = __ldg(&p.masked_m[g]);
        if (mg < 0 || mg > p.rows) {
          if (blockIdx.x == 0) atomicOr(&g_dg_error, 0x4);
          mg = mg < 0 ? 0 : p.rows;
        }
        counts[g] = mg;
        tiles = ((mg + L::kTileM - 1) / L::kTileM) * p.num_n_blocks;
      }
      int incl = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (g < p.G) prefix[g + 1] = run + incl;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) prefix[0] = 0;
  }
  if (MODE == MODE_CONTIG && kPair && warp == kEpi0) {
    // Pair table: block b (128 rows, expert = that of its first row) starts a
    // pair when it lies an even number of blocks into its run of equal
    // experts; blocks with an index outside [0, G) start none.  The experts
    // of all blocks are loaded at once (at most 32 per lane), then scanned.
    const int nb = p.rows / 128;
    int ev[kMaxContigBlocks / 32];
#pragma unroll
    for (int i = 0; i < kMaxContigBlocks / 32; ++i) {
      const int b = 32 * i + lane;
      ev[i] = b < nb ? __ldg(&p.m_indices[b * 128]) : -1;
    }
    int count = 0, run_start = 0, prev_e = -2;
#pragma unroll
    for (int i = 0; i < kMaxContigBlocks / 32; ++i) {
      if (32 * i >= nb) break;
      const int b = 32 * i + lane;
      const int e = ev[i];
      if (b < nb && (e < -1 || e >= p.G) && blockIdx.x == 0) atomicOr(&g_dg_error, 0x2);
      int e_prev = __shfl_up_sync(0xffffffffu, e, 1);
      if (lane == 0) e_prev = prev_e;
      // start of the run holding block b: the last block <= b where the expert changes
      int rs = (b < nb && (b == 0 || e != e_prev)) ? b : -1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, rs, o);
        if (lane >= o) rs = max(rs, v);
      }
      if (rs < 0) rs = run_start;
      const bool starts = b < nb && e >= 0 && e < p.G && ((b - rs) & 1) == 0;
      const uint32_t bal = __ballot_sync(0xffffffffu, starts);
      if (starts) prefix[1 + count + __popc(bal & ((1u << lane) - 1u))] = b;
      count += __popc(bal);
      run_start = __shfl_sync(0xffffffffu, rs, 31);
      prev_e = __shfl_sync(0xffffffffu, e, 31);
    }
    if (lane == 0) prefix[0] = count;
  }
  tc_fence_before();
  if constexpr (kPair) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int ntiles = total_tiles<MODE, CTAS>(p, prefix);
  // Tile i of this CTA (skipped tiles not counted) is either split over both
  // pipelines, each on half of the K groups into its own accumulator, or owned
  // by pipeline tile_pipe(i); every role derives the same plan.
  const int n_mine = ntiles > unit0 ? (ntiles - unit0 + units - 1) / units : 0;
  const int g_half = (p.kp + 1) / 2;
  auto tile_split = [&](uint32_t i) {
    return PIPES == 2 && p.kp >= 2 &&
           (SPLITK || (kTailSplit && (n_mine & 1) != 0 && static_cast<int>(i) == n_mine - 1));
  };
  auto tile_pipe = [&](uint32_t i) { return SPLITK ? 0 : static_cast<int>(i & 1); };
  // Whether this warp's pipeline works on the next tile (li advances), and its K groups [gb, ge).
  auto plan = [&](uint32_t& li, int& gb, int& ge) {
    const uint32_t i = li++;
    gb = 0;
    ge = p.kp;
    if (PIPES == 1) return true;
    if (tile_split(i)) {
      gb = pipe == 0 ? 0 : g_half;
      ge = pipe == 0 ? g_half : p.kp;
      return true;
    }
    return tile_pipe(i) == pipe;
  };

  if (is_producer) {
    // ============================================================ producer
    // Barrier of stage s in the MMA-issuing CTA, as a shared::cluster address.
    const uint32_t full0 = kPair ? mapa_shared(smem_u32(full_bar), 0) : smem_u32(full_bar);
    uint32_t& it = prod_it;
    uint32_t li = 0;
    bool ok = true;
    for (int t = unit0; t < ntiles && ok; t += units) {
      const Tile tl = tile_of<MODE, L::kTileM>(t, p, prefix, counts);
      int grp_a = 0, grp_b = 0;
      if (MODE == MODE_CONTIG) {
        const int e = contig_expert<CTAS>(tl, p);
        if (e < 0) continue;
        grp_b = e;
      } else if (MODE == MODE_MASKED) {
        grp_a = grp_b = tl.g;
      }
      int gb, ge;
      if (!plan(li, gb, ge)) continue;
      const int m_base = tl.row0 + 128 * static_cast<int>(rank);
      const int n0 = tl.n_blk * BN;
      const int kb_hi = min(num_kb, 4 * ge);
      for (int kb = 4 * gb; kb < kb_hi; ++kb, ++it) {
        const int s = sbase + static_cast<int>(it % L::kStagesPer);
        ok = wait_phase<false>(&empty_bar[s], ((it / L::kStagesPer) & 1) ^ 1, abort_flag, p.wait_limit_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (lane == 0) {
          uint8_t* a_dst = smem + L::kOffA + s * L::kABytes;
          uint8_t* b_dst = smem + L::kOffB + s * L::kBBytes;
          // each CTA of a pair holds half of the tile's MMA width of B
          const int b_row = n0 + static_cast<int>(rank) * (tile_mma_n<BN, CTAS, LAYOUT>(n0, p.N) / CTAS);
          // K-major boxes are (K, rows); MN-major boxes are (rows, K), 128 x 128 each
          const int ax = kAmn ? m_base : kb * kBK, ay = kAmn ? kb * kBK : m_base;
          if constexpr (kPair) tma_load_3d_pair(a_dst, &tm_a, full0 + 8 * s, ax, ay, grp_a);
          else tma_load_3d(a_dst, &tm_a, &full_bar[s], ax, ay, grp_a);
          if constexpr (kBmn) {
#pragma unroll
            for (int j = 0; j < L::kBRows / 128; ++j) {
              if constexpr (kPair)
                tma_load_3d_pair(b_dst + j * 128 * kBK, &tm_b, full0 + 8 * s, b_row + 128 * j, kb * kBK, grp_b);
              else
                tma_load_3d(b_dst + j * 128 * kBK, &tm_b, &full_bar[s], b_row + 128 * j, kb * kBK, grp_b);
            }
          } else {
            if constexpr (kPair) tma_load_3d_pair(b_dst, &tm_b, full0 + 8 * s, kb * kBK, b_row, grp_b);
            else tma_load_3d(b_dst, &tm_b, &full_bar[s], kb * kBK, b_row, grp_b);
          }
        }
        if (lane == 0) {
          if constexpr (kPair) mbar_arrive_expect_tx_cluster(full0 + 8 * s, L::kABytes + L::kBBytes);
          else mbar_arrive_expect_tx(&full_bar[s], L::kABytes + L::kBBytes);
        }
      }
    }
    // Drain: every load must land before its CTA exits.  One CTA waits for
    // its last STAGES loads here (an earlier load's stage was consumed before
    // a later load could reuse it).  In a pair every load signals the first
    // CTA's barriers, and after an abort the two CTAs may have issued
    // different counts: the second CTA publishes its count, and the first
    // drains both after the cluster barrier of the teardown.
    if constexpr (!kPair) {
      if (lane == 0) {
        const uint32_t first = it > static_cast<uint32_t>(L::kStagesPer) ? it - L::kStagesPer : 0;
        for (uint32_t i = first; i < it; ++i)
          wait_phase_drain(&full_bar[sbase + i % L::kStagesPer], (i / L::kStagesPer) & 1);
      }
    } else if (rank == 1 && lane == 0) {
      st_shared_cluster_u32(mapa_shared(smem_u32(peer_loads + pipe), 0), it);
    }
    __syncwarp();
  } else if (is_issuer) {
    // ============================================================ MMA issuer
    // A single thread issues.  Each tcgen05 instruction costs the issuing
    // thread ~60 cycles and every other instruction a few more, against 448
    // tensor-pipe cycles per 128x224x128 K block, so the loop is shaped to
    // execute as little as possible per K block: one iteration covers a whole
    // scale group (4 K blocks, unrolled), descriptors and instruction words
    // are precomputed, stage/phase counters are incremental and barrier polls
    // take an inline fast path.
    if ((!kPair || rank == 0) && lane == 0) {
      // LBO only matters for MN-major operands (16 KB between 128-wide boxes);
      // it sits in the low word, SBO (1024 B: 8 rows of 128 B) in the high word
      const uint32_t a_lo0 = static_cast<uint32_t>(
          make_smem_desc(smem_u32(smem + L::kOffA + sbase * L::kABytes), kAmn ? 128 * kBK : 16, 1024, 2));
      const uint32_t b_lo0 = static_cast<uint32_t>(
          make_smem_desc(smem_u32(smem + L::kOffB + sbase * L::kBBytes), kBmn ? 128 * kBK : 16, 1024, 2));
      const uint32_t desc_hi = static_cast<uint32_t>(make_smem_desc(0, 16, 1024, 2) >> 32);
      // start-address step per K = 32 (address field in 16-byte units): K-major,
      // +32 B inside the swizzled 128-byte row; MN-major, +4 atoms of 8 K-rows
      constexpr uint32_t kAStep = kAmn ? 256 : 2, kBStep = kBmn ? 256 : 2;
      constexpr uint32_t kSfIdStep = (1u << 4) | (1u << 29);  // +1 in both scale-factor byte selectors
      const uint32_t full_base = smem_u32(full_bar + sbase);
      const uint32_t empty_base = smem_u32(empty_bar + sbase);
      uint32_t s = 0, phase = 0, own = 0, li = 0, sf_group = 0;
      bool ok = true;
      const uint32_t sft_lo0 = static_cast<uint32_t>(
          make_smem_desc(smem_u32(smem + L::kOffSft + rbase * L::kSftBytes), 128, 256, 0));
      const uint32_t sf_slot0 = tmem_base + L::kSfBaseCol + pipe * 2 * L::kSfSlotCols;
      const uint32_t sft_hi = static_cast<uint32_t>(make_smem_desc(0, 128, 256, 0) >> 32);
      const uint32_t sfx_hi = static_cast<uint32_t>(make_smem_desc(0, 0, 128, 0) >> 32);
      const uint32_t idesc_full = make_idesc_mxf8(L::kTileM, BN, 0, 0, kAmn, kBmn);
      const bool ragged_n = p.N % BN != 0;
      for (int t = unit0; t < ntiles && ok; t += units) {
        // the tile itself is needed only to skip contiguous tiles and to narrow a ragged last N tile
        int n0 = 0;
        if (MODE == MODE_CONTIG || ragged_n) {
          const Tile tl = tile_of<MODE, L::kTileM>(t, p, prefix, counts);
          if (MODE == MODE_CONTIG && contig_expert<CTAS>(tl, p) < 0) continue;
          n0 = tl.n_blk * BN;
        }
        int gb, ge;
        if (!plan(li, gb, ge)) continue;
        const uint32_t idesc_t =
            ragged_n ? make_idesc_mxf8(L::kTileM, tile_mma_n<BN, CTAS, LAYOUT>(n0, p.N), 0, 0, kAmn, kBmn) : idesc_full;
        const int kb_hi = min(num_kb, 4 * ge);
        // one pipeline: alternate accumulators; two: accumulator = pipeline
        const uint32_t acc = PIPES == 2 ? pipe : (L::kNumAcc == 1 ? 0 : (own & 1));
        const uint32_t acc_use = (PIPES == 2 || L::kNumAcc == 1) ? own : (own >> 1);
        ++own;
        if (!mbar_try_wait(&tmem_empty[acc], (acc_use & 1) ^ 1))
          ok = wait_phase<false>(&tmem_empty[acc], (acc_use & 1) ^ 1, abort_flag, p.wait_limit_ns);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * L::kAccStride;
        uint32_t accumulate = 0;
        for (int kb0 = 4 * gb; kb0 < kb_hi && ok; kb0 += 4, ++sf_group) {
          const uint32_t ring = sf_group % L::kSfRing;
          const uint32_t sf_col = sf_slot0 + (sf_group & 1) * L::kSfSlotCols;
          // TMEM scale slot (sf_group & 1) was last read by group sf_group - 2
          if (sf_group >= 2) {
            uint64_t* b = &sf_empty[rbase + (sf_group - 2) % L::kSfRing];
            const uint32_t par = ((sf_group - 2) / L::kSfRing) & 1;
            if (!mbar_try_wait(b, par)) ok = wait_phase<false>(b, par, abort_flag, p.wait_limit_ns);
          }
          // acquire at cluster scope: pairs with the scale producers' release (their
          // shared-memory writes are read by tcgen05.cp)
          if (ok && !(kPair ? mbar_try_wait_cluster(&sf_full[rbase + ring], (sf_group / L::kSfRing) & 1)
                            : mbar_try_wait(&sf_full[rbase + ring], (sf_group / L::kSfRing) & 1)))
            ok = wait_phase<kPair>(&sf_full[rbase + ring], (sf_group / L::kSfRing) & 1, abort_flag, p.wait_limit_ns);
          if (!ok) break;
          tc_fence_after();
          {
            const uint32_t lo = sft_lo0 + ring * (L::kSftBytes >> 4);
            tmem_cp_128x256b<CTAS>(sf_col, (static_cast<uint64_t>(sft_hi) << 32) | lo);
            if constexpr (L::kNB128 == 2)
              tmem_cp_32x128b_warpx4<CTAS>(sf_col + 8, (static_cast<uint64_t>(sfx_hi) << 32) |
                                                           (lo + (L::kSftMainBytes >> 4)));
          }
          const int nk = min(4, kb_hi - kb0);
          uint32_t id = idesc_t;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (j < nk) {
              if (!mbar_try_wait_addr(full_base + 8 * s, phase)) {
                ok = wait_phase<false>(&full_bar[sbase + s], phase, abort_flag, p.wait_limit_ns);
                if (!ok) break;
              }
              const uint64_t a_desc = (static_cast<uint64_t>(desc_hi) << 32) | (a_lo0 + s * (L::kABytes >> 4));
              const uint64_t b_desc = (static_cast<uint64_t>(desc_hi) << 32) | (b_lo0 + s * (L::kBBytes >> 4));
              mma_mxf8f6f4<CTAS>(d_tmem, a_desc, b_desc, id, sf_col, sf_col + 4, accumulate);
              mma_mxf8f6f4<CTAS>(d_tmem, a_desc + kAStep, b_desc + kBStep, id, sf_col, sf_col + 4, 1u);
              mma_mxf8f6f4<CTAS>(d_tmem, a_desc + 2 * kAStep, b_desc + 2 * kBStep, id, sf_col, sf_col + 4, 1u);
              mma_mxf8f6f4<CTAS>(d_tmem, a_desc + 3 * kAStep, b_desc + 3 * kBStep, id, sf_col, sf_col + 4, 1u);
              accumulate = 1;
              if constexpr (kPair) tc_commit_pair_addr(empty_base + 8 * s);
              else tc_commit_addr<1>(empty_base + 8 * s);
              id += kSfIdStep;
              if (++s == L::kStagesPer) {
                s = 0;
                phase ^= 1;
              }
            }
          }
          if (!ok) break;
          if constexpr (kPair) tc_commit_pair(&sf_empty[rbase + ring]);
          else tc_commit<1>(&sf_empty[rbase + ring]);
        }
        if (!ok) break;
        if constexpr (kPair) tc_commit_pair(&tmem_full[acc]);
        else tc_commit<1>(&tmem_full[acc]);
      }
      // Drain: all MMAs / copies issued by this thread complete before TMEM is freed.
      tc_commit<CTAS>(&final_bar[pipe]);
      wait_phase_drain(&final_bar[pipe], 0);
    }
    __syncwarp();
  } else if (is_scale) {
    // ============================================================ scale producer
    const uint32_t sf_full0 = kPair ? mapa_shared(smem_u32(sf_full + rbase), 0) : smem_u32(sf_full + rbase);
    uint32_t group = 0, li = 0;
    bool ok = true;
    for (int t = unit0; t < ntiles && ok; t += units) {
      const Tile tl = tile_of<MODE, L::kTileM>(t, p, prefix, counts);
      int grp_a = 0, grp_b = 0;
      if (MODE == MODE_CONTIG) {
        const int e = contig_expert<CTAS>(tl, p);
        if (e < 0) continue;
        grp_b = e;
      } else if (MODE == MODE_MASKED) {
        grp_a = grp_b = tl.g;
      }
      int gb, ge;
      if (!plan(li, gb, ge)) continue;
      const int m_base = tl.row0 + 128 * static_cast<int>(rank);
      const int n0 = tl.n_blk * BN;
      for (int kp = gb; kp < ge; ++kp, ++group) {
        const uint32_t ring = group % L::kSfRing;
        ok = wait_phase<false>(&sf_empty[rbase + ring], ((group / L::kSfRing) & 1) ^ 1, abort_flag, p.wait_limit_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        // lane r gathers rows / columns r, r+32, r+64, r+96 of each 128-group
        uint32_t wa[4];
        if (p.sfa_f32 != nullptr) {  // fp32 scales: pack this group's word here (the packing step, fused)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int m = m_base + 32 * i + lane;
            wa[i] = m < p.rows ? pack_scale_word(p.sfa_f32 + (static_cast<size_t>(grp_a) * p.rows + m) * num_kb, kp,
                                                 num_kb, p.sfa_f32_vec != 0)
                               : 0u;
          }
        } else {
          const uint32_t* sfa_row = p.sfa + (static_cast<size_t>(grp_a) * p.kp + kp) * p.mn4a;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int m = m_base + 32 * i + lane;
            wa[i] = m < p.mn4a ? __ldg(sfa_row + m) : 0u;
          }
        }
        const uint32_t* sfb_row = p.sfb + (static_cast<size_t>(grp_b) * p.kp + kp) * p.nb4;
        uint32_t wb[L::kNB128][4];
#pragma unroll
        for (int h = 0; h < L::kNB128; ++h)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int j = 128 * h + 32 * c + lane;
            const int nb = p.sfb_gran == 1 ? n0 + j : (n0 + j) >> 7;
            wb[h][c] = (j < BN && nb < p.nb4) ? __ldg(sfb_row + nb) : 0u;
          }
        uint8_t* sft = smem + L::kOffSft + (rbase + ring) * L::kSftBytes;
        const uint4 va = make_uint4(wa[0], wa[1], wa[2], wa[3]);
        const uint4 vb = make_uint4(wb[0][0], wb[0][1], wb[0][2], wb[0][3]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // TMEM lane quarters q hold identical copies
          const int row = lane + 32 * q;
          uint8_t* cm = sft + (row >> 3) * 256 + (row & 7) * 16;
          *reinterpret_cast<uint4*>(cm) = va;         // TMEM columns +0..+3: SFA
          *reinterpret_cast<uint4*>(cm + 128) = vb;   // TMEM columns +4..+7: SFB, columns 0-127
        }
        if constexpr (L::kNB128 == 2)
          *reinterpret_cast<uint4*>(sft + L::kSftMainBytes + lane * 16) =
              make_uint4(wb[1][0], wb[1][1], wb[1][2], wb[1][3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // the words are read by the tensor core on behalf of the MMA-issuing CTA
          if constexpr (kPair) mbar_arrive_cluster(sf_full0 + 8 * ring);
          else mbar_arrive(&sf_full[rbase + ring]);
        }
      }
    }
  } else {
    // ============================================================ epilogue
    // Eight warps: two per TMEM lane quarter (q = warp % 4), the first of
    // each pair taking the even 32-column chunks of the tile, the second the
    // odd ones.  The tcgen05.ld of a warp's next chunk is in flight while the
    // current one is converted and stored.
    const int q = warp % 4;  // TMEM lane quarter this warp may access
    const int epi_idx = warp - kEpi0;
    const int half = epi_idx >> 2;
    uint8_t* buf = smem + L::kOffEpi + epi_idx * L::kEpiBuf;  // staging for one TMA store
    const uint32_t empty0 = kPair ? mapa_shared(smem_u32(tmem_empty), 0) : smem_u32(tmem_empty);
    constexpr int kChunks = BN / 32;
    constexpr int kMaxMine = (kChunks + 1) / 2;
    // a single accumulator (no split tiles: one pipeline) with BF16 output releases it early
    constexpr bool kEarlyRelease = !OUT_F32 && L::kNumAcc == 1 && PIPES == 1;
    const int nmine = half == 0 ? (kChunks + 1) / 2 : kChunks / 2;
    uint32_t local_tile = 0;
    uint32_t uses0 = 0, uses1 = 0;  // tiles that used accumulator 0 / 1 so far (two pipelines)
    for (int t = unit0; t < ntiles; t += units) {
      const Tile tl = tile_of<MODE, L::kTileM>(t, p, prefix, counts);
      int expert = 0, own_e = 0;
      if (MODE == MODE_CONTIG) {
        // expert of this CTA's own 128-row block (a pair's blocks may differ)
        const int own_blk = tl.row0 / 128 + static_cast<int>(rank);
        own_e = own_blk < p.rows / 128 ? __ldg(&p.m_indices[own_blk * 128]) : -1;
        if ((own_e < -1 || own_e >= p.G) && warp == kEpi0 && lane == 0 && tl.n_blk == 0)
          atomicOr(&g_dg_error, 0x2);
        expert = contig_expert<CTAS>(tl, p);
        if (expert < 0) continue;
      }
      // accumulator(s) of this tile and how often each was used before
      uint32_t acc, acc_use;
      bool split = false;
      if constexpr (PIPES == 2) {
        split = tile_split(local_tile);
        acc = split ? 0u : static_cast<uint32_t>(tile_pipe(local_tile));
        acc_use = acc == 0 ? uses0++ : uses1++;
      } else {
        acc = local_tile % L::kNumAcc;
        acc_use = local_tile / L::kNumAcc;
      }
      ++local_tile;
      // FP32 output plus C (dense only): the C values of the warp's chunks are
      // loaded one chunk ahead, the first before the accumulator is ready, so
      // their latency overlaps the MMAs and the previous chunk's stores.
      float4 cbuf[2][8];
      const bool c_rows = OUT_F32 && MODE == MODE_DENSE && p.c != nullptr &&
                          tl.row0 + 128 * static_cast<int>(rank) + 32 * q + lane < p.rows;
      auto load_c = [&](int col0, float4 (&cv)[8]) {
        const float4* cp = reinterpret_cast<const float4*>(
            p.c + static_cast<size_t>(tl.row0 + 128 * static_cast<int>(rank) + 32 * q + lane) * p.N + col0);
#pragma unroll
        for (int i = 0; i < 8; ++i) cv[i] = col0 + 4 * i < p.N ? __ldg(cp + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      };
      if constexpr (OUT_F32) {
        if (c_rows && nmine > 0 && tl.n_blk * BN + 32 * half < p.N) load_c(tl.n_blk * BN + 32 * half, cbuf[0]);
      }
      bool ok = wait_phase<false>(&tmem_full[acc], acc_use & 1, abort_flag, p.wait_limit_ns);
      if (split && ok) ok = wait_phase<false>(&tmem_full[1], uses1++ & 1, abort_flag, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();

      const int row0 = tl.row0 + 128 * static_cast<int>(rank) + 32 * q;  // warp's first row
      const int m_local = row0 + lane;  // row inside A / D (per expert for masked)
      bool valid;
      if (MODE == MODE_DENSE) {
        valid = m_local < p.rows;
      } else if (MODE == MODE_CONTIG) {
        const int idx = m_local < p.rows ? __ldg(&p.m_indices[m_local]) : -1;
        // rows of this CTA's block belong to the tile only when the block's expert is the tile's
        valid = own_e == expert && idx == expert;
        if (own_e == expert && idx != expert && idx != -1 && tl.n_blk == 0 && half == 0)
          atomicOr(&g_dg_error, (idx >= 0 && idx < p.G) ? 0x8 : 0x2);
      } else {
        valid = m_local < counts[tl.g];
      }
      const bool all_valid = __all_sync(0xffffffffu, valid);
      const bool any_valid = __any_sync(0xffffffffu, valid);
      const int n0 = tl.n_blk * BN;
      const int zd = (MODE == MODE_MASKED) ? tl.g : 0;
      const size_t row_g = static_cast<size_t>(zd) * p.rows + m_local;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + acc * L::kAccStride;

      // Converts and stores one 32-column chunk held in rr (lane = row).
      auto store_chunk = [&](uint32_t (&rr)[32], int col0, const float4 (&cv)[8]) {
        if constexpr (OUT_F32) {
          // FP32 output, optionally plus C (prefetched into cv): two 16-column halves of 64 B per row
          if (c_rows) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              if (col0 + 4 * i < p.N) {
                rr[4 * i] = __float_as_uint(__uint_as_float(rr[4 * i]) + cv[i].x);
                rr[4 * i + 1] = __float_as_uint(__uint_as_float(rr[4 * i + 1]) + cv[i].y);
                rr[4 * i + 2] = __float_as_uint(__uint_as_float(rr[4 * i + 2]) + cv[i].z);
                rr[4 * i + 3] = __float_as_uint(__uint_as_float(rr[4 * i + 3]) + cv[i].w);
              }
            }
          }
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int colh = col0 + 16 * hf;
            if (colh >= p.N) break;
            if (all_valid) {
              if (lane == 0) bulk_wait_group_read<0>();  // previous store has read the buffer
              __syncwarp();
              uint8_t* rowp = buf + lane * 64;
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int chunk = i ^ ((lane >> 1) & 3);  // 64-byte swizzle
                *reinterpret_cast<uint4*>(rowp + chunk * 16) = make_uint4(
                    rr[16 * hf + 4 * i], rr[16 * hf + 4 * i + 1], rr[16 * hf + 4 * i + 2], rr[16 * hf + 4 * i + 3]);
              }
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_3d(&tm_d, buf, colh, row0, zd);
                bulk_commit_group();
              }
            } else if (valid) {
              uint4* dst = reinterpret_cast<uint4*>(p.d32 + row_g * p.N + colh);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                if (colh + 4 * i < p.N)
                  dst[i] = make_uint4(rr[16 * hf + 4 * i], rr[16 * hf + 4 * i + 1], rr[16 * hf + 4 * i + 2],
                                      rr[16 * hf + 4 * i + 3]);
            }
          }
        } else {
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(rr[2 * i]), __uint_as_float(rr[2 * i + 1]));
            packed[i] = *reinterpret_cast<uint32_t*>(&h2);
          }
          if (all_valid) {
            if (lane == 0) bulk_wait_group_read<0>();  // previous store has read the buffer
            __syncwarp();
            uint8_t* rowp = buf + lane * 64;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int chunk = i ^ ((lane >> 1) & 3);  // 64-byte swizzle
              *reinterpret_cast<uint4*>(rowp + chunk * 16) =
                  make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&tm_d, buf, col0, row0, zd);
              bulk_commit_group();
            }
          } else if (valid) {
            __nv_bfloat16* dst = p.d + row_g * p.N + col0;
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (col0 + 8 * i < p.N)
                *reinterpret_cast<uint4*>(dst + 8 * i) =
                    make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
        }
      };

      if constexpr (kEarlyRelease) {
        // One accumulator: the next tile's MMAs wait for it, so it is handed
        // back as soon as it has been read.  The warp's chunks go from TMEM
        // to packed BF16 in registers, the accumulator is released, and only
        // then are they staged and stored.
        uint32_t pk[kMaxMine][16];
        if (any_valid) {
#pragma unroll
          for (int i = 0; i < kMaxMine; ++i) {
            const int c = half + 2 * i;
            if (i < nmine && n0 + 32 * c < p.N) {
              uint32_t r[32];
              tmem_ld_32x32b_x32(t_row + 32 * c, r);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
                pk[i][j] = *reinterpret_cast<uint32_t*>(&h2);
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (kPair) mbar_arrive_remote(empty0 + 8 * acc);
          else mbar_arrive(&tmem_empty[acc]);
        }
        if (any_valid) {
#pragma unroll
          for (int i = 0; i < kMaxMine; ++i) {
            const int col0 = n0 + 32 * (half + 2 * i);
            if (i >= nmine || col0 >= p.N) break;
            if (all_valid) {
              if (lane == 0) bulk_wait_group_read<0>();  // previous store has read the buffer
              __syncwarp();
              uint8_t* rowp = buf + lane * 64;
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const int chunk = v ^ ((lane >> 1) & 3);  // 64-byte swizzle
                *reinterpret_cast<uint4*>(rowp + chunk * 16) =
                    make_uint4(pk[i][4 * v], pk[i][4 * v + 1], pk[i][4 * v + 2], pk[i][4 * v + 3]);
              }
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_3d(&tm_d, buf, col0, row0, zd);
                bulk_commit_group();
              }
            } else if (valid) {
              __nv_bfloat16* dst = p.d + row_g * p.N + col0;
#pragma unroll
              for (int v = 0; v < 4; ++v)
                if (col0 + 8 * v < p.N)
                  *reinterpret_cast<uint4*>(dst + 8 * v) =
                      make_uint4(pk[i][4 * v], pk[i][4 * v + 1], pk[i][4 * v + 2], pk[i][4 * v + 3]);
            }
          }
        }
        continue;
      }
      if (any_valid) {
        uint32_t r[2][32];
        if (nmine > 0 && n0 + 32 * half < p.N) tmem_ld_32x32b_x32(t_row + 32 * half, r[0]);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < kMaxMine; ++i) {
          const int c = half + 2 * i;
          const int col0 = n0 + 32 * c;
          if (i >= nmine || col0 >= p.N) break;
          if (i + 1 < nmine && col0 + 64 < p.N) {
            tmem_ld_32x32b_x32(t_row + 32 * (c + 2), r[(i + 1) & 1]);
            if constexpr (OUT_F32) {
              if (c_rows) load_c(col0 + 64, cbuf[(i + 1) & 1]);
            }
          }
          if (split) {
            // a split tile: add the second pipeline's accumulator, 16 columns at a time
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              uint32_t h[16];
              tmem_ld_32x32b_x16(t_row + L::kAccStride + 32 * c + 16 * hh, h);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 16; ++j)
                r[i & 1][16 * hh + j] =
                    __float_as_uint(__uint_as_float(r[i & 1][16 * hh + j]) + __uint_as_float(h[j]));
            }
          }
          store_chunk(r[i & 1], col0, cbuf[i & 1]);
          tmem_wait_ld();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (kPair) mbar_arrive_remote(empty0 + 8 * acc);
        else mbar_arrive(&tmem_empty[acc]);
        if (split) {
          if constexpr (kPair) mbar_arrive_remote(empty0 + 8);
          else mbar_arrive(&tmem_empty[1]);
        }
      }
    }
    // Before the CTA exits its staging buffers must have been read out; the
    // global writes themselves complete with the grid.
    if (lane == 0) bulk_wait_group_read<0>();
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  if constexpr (kPair) {
    cluster_sync();  // both CTAs have stopped issuing; the second CTA's load counts are visible
    if (rank == 0 && is_producer && lane == 0) {
      // Phase j of a stage barrier completes with one arrival per CTA plus
      // the bytes of both loads.  A CTA that gave up before issuing load j
      // never arrives: arrive in its place, then wait for the loads that were
      // issued.  Only the last STAGES phases can be incomplete.
      const uint32_t it1 = *reinterpret_cast<volatile uint32_t*>(peer_loads + pipe);
      const uint32_t hi = prod_it > it1 ? prod_it : it1;
      const uint32_t lo = hi > static_cast<uint32_t>(L::kStagesPer) ? hi - L::kStagesPer : 0;
      for (uint32_t j = lo; j < hi; ++j) {
        uint64_t* b = &full_bar[sbase + j % L::kStagesPer];
        if (j >= prod_it) mbar_arrive(b);
        if (j >= it1) mbar_arrive(b);
        wait_phase_drain(b, (j / L::kStagesPer) & 1);
      }
    }
    __syncwarp();
    cluster_sync();
  } else {
    __syncthreads();
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc<CTAS>(tmem_base, L::kTmemCols);
  }
}

}  // namespace dg
