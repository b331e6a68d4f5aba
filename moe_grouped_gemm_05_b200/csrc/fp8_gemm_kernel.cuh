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
// Roles (one CTA per SM, persistent over output tiles of 128 x BN):
//   warp 0     TMA producer: A/B K-blocks (+ raw packed scale words every 4
//              K-blocks) into a STAGES-deep shared-memory ring.
//   warp 1     TMEM owner and MMA issuer: rearranges the scale words into
//              the tensor-memory scale layout (tcgen05.cp), issues the MMAs,
//              commits stage releases and finished accumulators.
//   warps 2-5  epilogue: tcgen05.ld of the accumulator, BF16 RNE conversion,
//              swizzled staging + TMA store for fully valid 32-row slices,
//              predicated stores for slices holding padding/masked rows.
// Accumulators are double-buffered in TMEM when they fit, so the epilogue of
// tile i overlaps the MMAs of tile i+1.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace dg {

// Device error word (DG_DEVERR_* bits); one per device, read and cleared by the host.
__device__ int g_dg_error = 0;

enum : int { MODE_DENSE = 0, MODE_CONTIG = 1, MODE_MASKED = 2 };

constexpr int kBM = 128;
constexpr int kBK = 128;
constexpr int kThreads = 192;
constexpr int kMaxMaskedGroups = 512;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far above any legitimate wait

struct GemmArgs {
  int rows;           // dense: M; contiguous: M_total; masked: M_max
  int N, K, G;
  int num_m_blocks;   // dense / contiguous
  int num_n_blocks;
  int raster_m;       // rasterisation group height in M blocks
  const int32_t* m_indices;
  const int32_t* masked_m;
  __nv_bfloat16* d;
};

template <int BN, int STAGES>
struct Layout {
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN must be a multiple of 32 in [32, 256]");
  static constexpr int kNB128 = (BN + 127) / 128;        // 128-column groups of B scales
  static constexpr int kABytes = kBM * kBK;              // 16 KB
  static constexpr int kBBytes = BN * kBK;
  static constexpr int kSfaRawBytes = 512;               // 128 words
  static constexpr int kSfbRawBytes = 32;                // 8 words
  static constexpr int kSfRawStride = 640;
  static constexpr int kSftABytes = 512;                 // 32 rows x 16 B
  static constexpr int kSftBBytes = 512 * kNB128;
  static constexpr int kSftSlot = kSftABytes + kSftBBytes;
  static constexpr int kEpiBuf = 32 * 32 * 2;            // 32 rows x 32 bf16
  // TMEM columns: accumulators, then two scale slots of 16 columns (SFA at +0, SFB at +8).
  static constexpr int kSfSlotCols = 16;
  static constexpr int kAccStride = BN <= 128 ? 128 : 256;  // accumulator buffers start on 128-column bounds
  static constexpr int kNumAcc = (kAccStride + BN + 2 * kSfSlotCols <= 512) ? 2 : 1;
  static constexpr int kSfBaseCol = (kNumAcc - 1) * kAccStride + ((BN + 15) / 16) * 16;
  static constexpr int kTmemCols = 512;
  // shared-memory offsets (from a 1024-byte aligned base)
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + STAGES * kABytes;
  static constexpr int kOffSfRaw = kOffB + STAGES * kBBytes;
  static constexpr int kOffSft = kOffSfRaw + STAGES * kSfRawStride;
  static constexpr int kOffEpi = ((kOffSft + 2 * kSftSlot + 1023) / 1024) * 1024;
  static constexpr int kOffBar = kOffEpi + 4 * 2 * kEpiBuf;
  static constexpr int kNumBars = 2 * STAGES + 2 * 2 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // tmem addr, abort flag
  static constexpr int kOffGroups = kOffMisc + 16;          // masked: prefix[G+1], count[G]
  static constexpr int kSmemBytes = kOffGroups + (2 * kMaxMaskedGroups + 1) * 4 + 1024;
};

struct Tile {
  int m_blk, n_blk, g;
};

// Bounded wait on an mbarrier phase.  Returns false when the CTA is aborting
// (another role gave up) or this wait exceeded its limit (sets the error word).
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(&g_dg_error, 0x10);
      return false;
    }
  }
}

// Wait used while draining at exit: ignores the abort flag, still bounded.
__device__ __forceinline__ void wait_phase_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_dg_error, 0x10);
      return;
    }
  }
}

template <int MODE>
__device__ __forceinline__ int total_tiles(const GemmArgs& p, const int* prefix) {
  if (MODE == MODE_MASKED) return prefix[p.G];
  return p.num_m_blocks * p.num_n_blocks;
}

// Tile order: dense / contiguous use groups of `raster_m` M blocks swept
// column by column, so concurrently running CTAs share A rows and B columns
// in L2; masked runs expert by expert, N block by N block, M blocks fastest.
template <int MODE>
__device__ __forceinline__ Tile tile_of(int t, const GemmArgs& p, const int* prefix,
                                        const int* counts) {
  Tile tl;
  if (MODE == MODE_MASKED) {
    int g = 0;
    while (prefix[g + 1] <= t) ++g;
    const int local = t - prefix[g];
    const int cnt = (counts[g] + kBM - 1) / kBM;
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
  return tl;
}

template <int BN, int STAGES, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_sfa,
                    const __grid_constant__ CUtensorMap tm_sfb,
                    const __grid_constant__ CUtensorMap tm_d, const GemmArgs p) {
  using L = Layout<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* tmem_full = bars + 2 * STAGES;
  uint64_t* tmem_empty = bars + 2 * STAGES + 2;
  uint64_t* sf_free = bars + 2 * STAGES + 4;
  uint64_t* final_bar = bars + 2 * STAGES + 6;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  int* prefix = reinterpret_cast<int*>(smem + L::kOffGroups);
  int* counts = prefix + kMaxMaskedGroups + 1;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int num_kb = p.K / kBK;

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tmem_full[i], 1);
      mbar_init(&tmem_empty[i], 4);
      mbar_init(&sf_free[i], 1);
    }
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
    prefetch_tensormap(&tm_sfa);
    prefetch_tensormap(&tm_sfb);
    prefetch_tensormap(&tm_d);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, L::kTmemCols);
    tmem_relinquish();
  }
  if (MODE == MODE_MASKED && warp == 2) {
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
        tiles = ((mg + kBM - 1) / kBM) * p.num_n_blocks;
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int ntiles = total_tiles<MODE>(p, prefix);

  if (warp == 0) {
    // ============================================================ producer
    if (lane == 0) {
      uint32_t it = 0;
      for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
        const Tile tl = tile_of<MODE>(t, p, prefix, counts);
        int grp_a = 0, grp_b = 0;
        if (MODE == MODE_CONTIG) {
          const int e = __ldg(&p.m_indices[tl.m_blk * kBM]);
          if (e < 0 || e >= p.G) continue;
          grp_b = e;
        } else if (MODE == MODE_MASKED) {
          grp_a = grp_b = tl.g;
        }
        const int m0 = tl.m_blk * kBM;
        const int n0 = tl.n_blk * BN;
        const int sfb_x = (n0 / 128) & ~3;
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % STAGES;
          if (!wait_phase(&empty_bar[s], ((it / STAGES) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          const bool with_sf = (kb & 3) == 0;
          mbar_arrive_expect_tx(&full_bar[s], L::kABytes + L::kBBytes +
                                                  (with_sf ? L::kSfaRawBytes + L::kSfbRawBytes : 0));
          tma_load_3d(smem + L::kOffA + s * L::kABytes, &tm_a, &full_bar[s], kb * kBK, m0, grp_a);
          tma_load_3d(smem + L::kOffB + s * L::kBBytes, &tm_b, &full_bar[s], kb * kBK, n0, grp_b);
          if (with_sf) {
            uint8_t* raw = smem + L::kOffSfRaw + s * L::kSfRawStride;
            tma_load_3d(raw, &tm_sfa, &full_bar[s], m0, kb / 4, grp_a);
            tma_load_3d(raw + L::kSfaRawBytes, &tm_sfb, &full_bar[s], sfb_x, kb / 4, grp_b);
          }
        }
        if (!ok) break;
      }
      // Drain: every load issued must have landed before the CTA may exit.
      const uint32_t first = it > static_cast<uint32_t>(STAGES) ? it - STAGES : 0;
      for (uint32_t i = first; i < it; ++i) wait_phase_drain(&full_bar[i % STAGES], (i / STAGES) & 1);
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    uint32_t it = 0, local_tile = 0, sf_group = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      const Tile tl = tile_of<MODE>(t, p, prefix, counts);
      if (MODE == MODE_CONTIG) {
        const int e = __ldg(&p.m_indices[tl.m_blk * kBM]);
        if (e < 0 || e >= p.G) continue;
      }
      const int n0 = tl.n_blk * BN;
      const int sfb_x = (n0 / 128) & ~3;
      const uint32_t acc = local_tile % L::kNumAcc;
      const uint32_t acc_use = local_tile / L::kNumAcc;
      ++local_tile;
      ok = wait_phase(&tmem_empty[acc], (acc_use & 1) ^ 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * L::kAccStride;
      uint32_t slot = 0;
      for (int kb = 0; kb < num_kb; ++kb, ++it) {
        const int s = it % STAGES;
        ok = wait_phase(&full_bar[s], (it / STAGES) & 1, abort_flag);
        if ((kb & 3) == 0 && ok) {
          slot = sf_group & 1;
          const uint32_t use = sf_group >> 1;
          if (use >= 1) ok = wait_phase(&sf_free[slot], (use - 1) & 1, abort_flag);
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        if ((kb & 3) == 0) {
          // Rearrange this tile's scale words for the tensor-memory scale layout:
          // row/column j of a 128-wide group lives at (lane j%32, column j/32).
          const uint32_t* raw = reinterpret_cast<const uint32_t*>(smem + L::kOffSfRaw + s * L::kSfRawStride);
          uint8_t* sft = smem + L::kOffSft + slot * L::kSftSlot;
          uint4 va = make_uint4(raw[lane], raw[32 + lane], raw[64 + lane], raw[96 + lane]);
          *reinterpret_cast<uint4*>(sft + lane * 16) = va;
          const uint32_t* rawb = raw + L::kSfaRawBytes / 4;
#pragma unroll
          for (int h = 0; h < L::kNB128; ++h) {
            uint32_t w[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int j = 128 * h + 32 * c + lane;
              w[c] = (j < BN) ? rawb[(n0 + j) / 128 - sfb_x] : 0u;
            }
            *reinterpret_cast<uint4*>(sft + L::kSftABytes + h * 512 + lane * 16) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const uint32_t sf_col = tmem_base + L::kSfBaseCol + slot * L::kSfSlotCols;
            tmem_cp_32x128b_warpx4(sf_col, make_smem_desc(smem_u32(sft), 0, 128, 0));
#pragma unroll
            for (int h = 0; h < L::kNB128; ++h)
              tmem_cp_32x128b_warpx4(sf_col + 8 + 4 * h,
                                     make_smem_desc(smem_u32(sft + L::kSftABytes + h * 512), 0, 128, 0));
          }
          ++sf_group;
        }
        if (lane == 0) {
          const uint32_t sf_col = tmem_base + L::kSfBaseCol + slot * L::kSfSlotCols;
          const uint32_t idesc = make_idesc_mxf8(kBM, BN, kb & 3, kb & 3);
          const uint64_t a_desc = make_smem_desc(smem_u32(smem + L::kOffA + s * L::kABytes), 16, 1024, 2);
          const uint64_t b_desc = make_smem_desc(smem_u32(smem + L::kOffB + s * L::kBBytes), 16, 1024, 2);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k) {
            // +32 bytes along K inside the 128-byte swizzled row = +2 in the address field
            mma_mxf8f6f4(d_tmem, a_desc + 2 * k, b_desc + 2 * k, idesc, sf_col, sf_col + 8,
                         (kb > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&empty_bar[s]);
          if ((kb & 3) == 3 || kb == num_kb - 1) tc_commit(&sf_free[slot]);
          if (kb == num_kb - 1) tc_commit(&tmem_full[acc]);
        }
        __syncwarp();
      }
    }
    // Drain: all MMAs / copies issued by this thread complete before TMEM is freed.
    if (lane == 0) {
      tc_commit(final_bar);
      wait_phase_drain(final_bar, 0);
    }
    __syncwarp();
  } else {
    // ============================================================ epilogue
    const int q = warp % 4;  // TMEM lane quarter this warp may access
    __nv_bfloat16* epi_base = reinterpret_cast<__nv_bfloat16*>(smem + L::kOffEpi + (warp - 2) * 2 * L::kEpiBuf);
    uint32_t local_tile = 0, store_count = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      const Tile tl = tile_of<MODE>(t, p, prefix, counts);
      int expert = 0;
      if (MODE == MODE_CONTIG) {
        expert = __ldg(&p.m_indices[tl.m_blk * kBM]);
        if (expert < 0 || expert >= p.G) {
          if (expert < -1 || expert >= p.G) {
            if (warp == 2 && lane == 0 && tl.n_blk == 0) atomicOr(&g_dg_error, 0x2);
          }
          continue;
        }
      }
      const uint32_t acc = local_tile % L::kNumAcc;
      const uint32_t acc_use = local_tile / L::kNumAcc;
      ++local_tile;
      bool ok = wait_phase(&tmem_full[acc], acc_use & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();

      const int row_in_tile = 32 * q + lane;
      const int m_local = tl.m_blk * kBM + row_in_tile;  // row inside A / D (per expert for masked)
      bool valid;
      if (MODE == MODE_DENSE) {
        valid = m_local < p.rows;
      } else if (MODE == MODE_CONTIG) {
        const int idx = __ldg(&p.m_indices[m_local]);
        valid = idx == expert;
        if (!valid && idx != -1 && tl.n_blk == 0)
          atomicOr(&g_dg_error, (idx >= 0 && idx < p.G) ? 0x8 : 0x2);
      } else {
        valid = m_local < counts[tl.g];
      }
      const bool all_valid = __all_sync(0xffffffffu, valid);
      const int n0 = tl.n_blk * BN;
      const int zd = (MODE == MODE_MASKED) ? tl.g : 0;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + acc * L::kAccStride;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int col0 = n0 + 32 * c;
        if (col0 >= p.N) break;
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + 32 * c, r);
        tmem_wait_ld();
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
          packed[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        if (all_valid) {
          __nv_bfloat16* buf = epi_base + (store_count & 1) * (L::kEpiBuf / 2);
          ++store_count;
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
          uint8_t* rowp = reinterpret_cast<uint8_t*>(buf) + lane * 64;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int chunk = i ^ ((lane >> 1) & 3);  // 64-byte swizzle
            *reinterpret_cast<uint4*>(rowp + chunk * 16) =
                make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&tm_d, buf, col0, tl.m_blk * kBM + 32 * q, zd);
            bulk_commit_group();
          }
        } else if (valid) {
          const size_t row_g = static_cast<size_t>(zd) * p.rows + m_local;
          __nv_bfloat16* dst = p.d + row_g * p.N + col0;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (col0 + 8 * i < p.N)
              *reinterpret_cast<uint4*>(dst + 8 * i) =
                  make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tmem_empty[acc]);
    }
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace dg
