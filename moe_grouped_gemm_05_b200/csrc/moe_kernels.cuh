// MoE permutation into the contiguous M-grouped layout and the inverse,
// weighted combine (DeepGEMM pages: charles2530.github.io "源码与接入" §七, the
// group_by_expert step before the grouped GEMM and the combine after it;
// juejin.cn §4 "分组 GEMM（连续布局）": expert segments aligned to the M block).
//
// moe_route_kernel   one cluster of 8 CTAs: a stable counting sort of the
//                    routed (token, slot) pairs by expert.  Each warp counts
//                    and later places a run of the slots in slot order; the
//                    CTAs add their counts through distributed shared memory
//                    -> each expert's segment offset (segments in expert
//                    order, each padded to 128 rows), so the layout is
//                    deterministic.  Writes row_of, and m_indices, src_of
//                    and zero scale words for padding rows.
// moe_gather_kernel  full grid, tokens in source order: copies each token's
//                    FP8 codes and packed scale words to the rows of its
//                    routed slots (one read of each token row), and writes
//                    those rows' expert and source token.
// moe_combine_kernel out[t] = bf16(sum_s w[t,s] * D[row_of[t,s]]), FP32 sums.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace dg {

constexpr int kMoeMaxExperts = 1024;
constexpr int kMoeThreads = 1024;

// CTAs of the routing kernel: one cluster, whose CTAs add their counts
// through distributed shared memory.
constexpr int kRouteCluster = 8;
// 32-slot steps of a warp whose ids the routing kernel loads at once.
constexpr int kRouteSteps = 8;
// Dynamic shared memory of the routing kernel for G experts: a [32 warps][G]
// table of counts, then this CTA's slice counts, the expert totals, the
// earlier CTAs' counts and the segment offsets (G words each).
__host__ __device__ constexpr int route_smem_bytes(int G) { return (32 * G + 4 * G) * 4; }

// Lanes of the warp whose key equals this lane's, for keys in [0, 2^nbits).
// Keys of up to 6 bits: match.any; wider: the AND over the key's bits of the
// ballot of the lanes agreeing on that bit (nbits ballots).  In the routing
// kernel's first pass the ballots measured faster with 256 experts (15.0 ->
// 11.8 us) and slower with 8 (2.4 -> 3.7 us).
__device__ __forceinline__ unsigned warp_same_key(int key, int nbits) {
  if (nbits <= 6) return __match_any_sync(0xffffffffu, key);
  unsigned m = 0xffffffffu;
  for (int b = 0; b < nbits; ++b) {
    const bool bit = (key >> b) & 1;
    const unsigned bal = __ballot_sync(0xffffffffu, bit);
    m &= bit ? bal : ~bal;
  }
  return m;
}

// A stable counting sort of the n routed slots by expert, on one cluster of
// kRouteCluster CTAs of 32 warps.  CTA c owns slots [c*slice, (c+1)*slice),
// and warp w of it a run of that range in slot order (whole 32-slot steps).
// 1. every warp counts the slots of its run per expert (lanes with the same
//    expert add once, by their first lane), into its row of the table;
//    unrouted and invalid slots get row_of = -1;
// 2. the CTA turns the table into exclusive prefixes over its warps and its
//    slice counts; the cluster adds every CTA's slice counts through
//    distributed shared memory, giving the expert totals and, per expert,
//    the slots of the CTAs before this one;
// 3. a block scan of the 128-padded totals gives the segment offsets (expert
//    order), and table entry [w][e] becomes the row of warp w's first slot
//    of expert e;
// 4. every warp walks its run again in slot order: a slot's row is its
//    warp's entry plus its rank among the lanes of the step with the same
//    expert, and the first such lane advances the entry; only row_of is
//    written here (coalesced): moe_gather_kernel, on the whole GPU, writes
//    m_indices and src_of of the routed rows from it;
// 5. the padding rows of the segments (one warp per expert, experts split
//    over the CTAs) and the rows past the last segment get index -1 and zero
//    scale words.
__global__ void __launch_bounds__(kMoeThreads) moe_route_kernel(const int32_t* __restrict__ ids, int n,
                                                                int G, int M_cap, int kp, int32_t* __restrict__ m_indices,
                                                                int32_t* __restrict__ row_of,
                                                                int32_t* __restrict__ src_of,
                                                                uint32_t* __restrict__ sfa_perm) {
  extern __shared__ __align__(16) int rsm[];
  int* wtab = rsm;             // [32][G]
  int* ccnt = wtab + 32 * G;   // this CTA's slice counts
  int* tot = ccnt + G;         // expert totals
  int* below = tot + G;        // slots of expert e in the CTAs before this one
  int* seg = below + G;        // segment offsets
  __shared__ int warp_sum[32];
  __shared__ int total_rows_s;
  grid_dep_wait();
  grid_dep_launch();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = static_cast<int>(cluster_cta_rank());
  const int slice = (n + kRouteCluster - 1) / kRouteCluster;
  const int s0 = min(n, c * slice), s1 = min(n, s0 + slice);
  const int per_warp = ((s1 - s0 + 32 * 32 - 1) / (32 * 32)) * 32;  // whole 32-slot steps
  const int w0 = min(s1, s0 + warp * per_warp), w1 = min(s1, w0 + per_warp);
  const unsigned lt = (1u << lane) - 1u;
  const int nbits = 32 - __clz(G);  // keys 0..G (G: unrouted or invalid)
  for (int i = tid; i < 32 * G; i += blockDim.x) wtab[i] = 0;
  __syncthreads();
  // 1. per-warp counts (the ids of kRouteSteps steps are loaded at once; the
  //    first batch's ids and same-expert masks stay in registers for step 4)
  int* row = wtab + warp * G;
  int vs0[kRouteSteps];
  unsigned ms0[kRouteSteps];
  for (int base = w0; base < w1; base += 32 * kRouteSteps) {
    const bool first = base == w0;
    int vs[kRouteSteps];
#pragma unroll
    for (int j = 0; j < kRouteSteps; ++j) {
      const int i = base + 32 * j + lane;
      vs[j] = i < w1 ? __ldg(&ids[i]) : -1;
    }
#pragma unroll
    for (int j = 0; j < kRouteSteps; ++j) {
      const int i = base + 32 * j + lane;
      const int v = vs[j];
      const bool valid = v >= 0 && v < G;
      if (i < w1 && !valid) row_of[i] = -1;
      if (__any_sync(0xffffffffu, i < w1 && v != -1 && !valid) && lane == 0) atomicOr(&g_dg_error, 0x2);
      const unsigned same = warp_same_key(valid ? v : G, nbits);
      if (valid && (same & lt) == 0u) row[v] += __popc(same);
      __syncwarp();
      if (first) {
        vs0[j] = v;
        ms0[j] = same;
      }
    }
  }
  __syncthreads();
  // 2. prefixes over the warps, slice counts, then the cluster's sums
  for (int e = tid; e < G; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int t = wtab[w * G + e];
      wtab[w * G + e] = run;
      run += t;
    }
    ccnt[e] = run;
  }
  cluster_sync();
  for (int e = tid; e < G; e += blockDim.x) {
    const uint32_t a = smem_u32(&ccnt[e]);
    int t = 0, b = 0;
#pragma unroll
    for (int r = 0; r < kRouteCluster; ++r) {
      const int x = static_cast<int>(ld_shared_cluster_u32(mapa_shared(a, r)));
      t += x;
      if (r < c) b += x;
    }
    tot[e] = t;
    below[e] = b;
  }
  cluster_sync();  // every CTA has read every slice count: from here none reads a peer
  // 3. segment offsets: exclusive scan of the padded totals (G <= blockDim)
  {
    const int v = tid < G ? (tot[tid] + 127) & ~127 : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int x = warp_sum[lane];
      int y = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, y, o);
        if (lane >= o) y += u;
      }
      warp_sum[lane] = y - x;
      if (lane == 31) total_rows_s = y;
    }
    __syncthreads();
    if (tid < G) seg[tid] = warp_sum[warp] + incl - v;
    __syncthreads();
  }
  for (int i = tid; i < 32 * G; i += blockDim.x) {
    const int e = i % G;
    wtab[i] += seg[e] + below[e];
  }
  __syncthreads();
  // 4. rows of the routed slots, in slot order
  for (int base = w0; base < w1; base += 32 * kRouteSteps) {
    const bool first = base == w0;
    int vs[kRouteSteps];
#pragma unroll
    for (int j = 0; j < kRouteSteps; ++j) {
      const int i = base + 32 * j + lane;
      vs[j] = first ? vs0[j] : (i < w1 ? __ldg(&ids[i]) : -1);
    }
#pragma unroll
    for (int j = 0; j < kRouteSteps; ++j) {
      const int i = base + 32 * j + lane;
      const int v = vs[j];
      const bool valid = v >= 0 && v < G;
      const unsigned same = first ? ms0[j] : warp_same_key(valid ? v : G, nbits);
      const int pos = valid ? row[v] + __popc(same & lt) : 0;
      __syncwarp();
      if (valid && (same & lt) == 0u) row[v] += __popc(same);
      __syncwarp();
      if (valid) row_of[i] = pos;
    }
  }
  // 5. padding rows of the segments of experts c, c + C, ... (one warp per
  //    expert), and a share of the tail
  for (int e = c + kRouteCluster * warp; e < G; e += kRouteCluster * 32) {
    const int pad0 = seg[e] + tot[e], pad1 = seg[e] + ((tot[e] + 127) & ~127);
    for (int r = pad0 + lane; r < pad1; r += 32) {
      m_indices[r] = -1;
      src_of[r] = -1;
      for (int k = 0; k < kp; ++k) sfa_perm[static_cast<size_t>(k) * M_cap + r] = 0u;
    }
  }
  for (int r = total_rows_s + c * blockDim.x + tid; r < M_cap; r += kRouteCluster * blockDim.x) {
    m_indices[r] = -1;
    src_of[r] = -1;
    for (int k = 0; k < kp; ++k) sfa_perm[static_cast<size_t>(k) * M_cap + r] = 0u;
  }
}

// a_perm[row_of[t][s]] = q[t] (K bytes), sfa_perm[kp][row_of[t][s]] =
// sfa[kp][t], m_indices[row_of[t][s]] = ids[t][s] and src_of[row_of[t][s]] =
// t for every routed slot s of token t: tokens in source order, so
// each token's row is read once however many slots it has.  Each thread takes
// kGatherU 16-byte units per pass (stride apart), loading all of them before
// storing any, so several loads are in flight per thread.  Padding and tail
// rows keep whatever codes they held (their scale words are zeroed by
// moe_route_kernel).
constexpr int kGatherU = 4;
__global__ void __launch_bounds__(256) moe_gather_kernel(const uint8_t* __restrict__ q, const uint32_t* __restrict__ sfa,
                                                        int T, int K, int kp, int topk,
                                                        const int32_t* __restrict__ ids,
                                                        const int32_t* __restrict__ row_of, int M_cap,
                                                        uint8_t* __restrict__ a_perm, uint32_t* __restrict__ sfa_perm,
                                                        int32_t* __restrict__ m_indices, int32_t* __restrict__ src_of) {
  grid_dep_wait();
  grid_dep_launch();
  const int chunks = K / 16;
  const int t4 = (T + 3) & ~3;
  const long long total = static_cast<long long>(T) * chunks;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long u0 = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; u0 < total;
       u0 += kGatherU * stride) {
    int t[kGatherU], ch[kGatherU];
    uint4 v[kGatherU];
    uint32_t w[kGatherU];
#pragma unroll
    for (int j = 0; j < kGatherU; ++j) {
      const long long u = u0 + j * stride;
      t[j] = u < total ? static_cast<int>(u / chunks) : -1;
      ch[j] = u < total ? static_cast<int>(u - static_cast<long long>(t[j]) * chunks) : 0;
      v[j] = t[j] >= 0 ? __ldg(reinterpret_cast<const uint4*>(q + static_cast<size_t>(t[j]) * K) + ch[j])
                       : make_uint4(0, 0, 0, 0);
      w[j] = t[j] >= 0 && ch[j] < kp ? __ldg(&sfa[static_cast<size_t>(ch[j]) * t4 + t[j]]) : 0u;
    }
#pragma unroll
    for (int j = 0; j < kGatherU; ++j) {
      if (t[j] < 0) continue;
      for (int s = 0; s < topk; ++s) {
        const int r = __ldg(&row_of[static_cast<size_t>(t[j]) * topk + s]);
        if (r < 0) continue;
        reinterpret_cast<uint4*>(a_perm + static_cast<size_t>(r) * K)[ch[j]] = v[j];
        if (ch[j] < kp) sfa_perm[static_cast<size_t>(ch[j]) * M_cap + r] = w[j];
        if (ch[j] == 0) {
          m_indices[r] = __ldg(&ids[static_cast<size_t>(t[j]) * topk + s]);
          src_of[r] = t[j];
        }
      }
    }
  }
}

// One thread per (token, 8 output columns).  The slots of the token are
// taken kSlots at a time: first their row indices and weights, then all of
// their 16-byte row loads, then the FP32 sums in slot order, so a thread has
// up to kSlots row loads in flight at once.
template <int kSlots>
__global__ void __launch_bounds__(256) moe_combine_kernel(const __nv_bfloat16* __restrict__ d, const int32_t* __restrict__ row_of,
                                                         const float* __restrict__ w, int T, int topk, int N,
                                                         __nv_bfloat16* __restrict__ out) {
  grid_dep_wait();
  grid_dep_launch();
  const int chunks = N / 8;
  const long long total = static_cast<long long>(T) * chunks;
  for (long long u = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(u / chunks);
    const int ch = static_cast<int>(u - static_cast<long long>(t) * chunks);
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int s0 = 0; s0 < topk; s0 += kSlots) {
      int r[kSlots];
      float ws[kSlots];
#pragma unroll
      for (int q = 0; q < kSlots; ++q) {
        const bool ok = s0 + q < topk;
        const size_t at = static_cast<size_t>(t) * topk + s0 + q;
        r[q] = ok ? __ldg(&row_of[at]) : -1;
        ws[q] = ok && w ? __ldg(&w[at]) : 1.0f;
      }
      uint4 v[kSlots];
#pragma unroll
      for (int q = 0; q < kSlots; ++q)
        v[q] = r[q] >= 0 ? __ldg(reinterpret_cast<const uint4*>(d + static_cast<size_t>(r[q]) * N) + ch)
                         : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int q = 0; q < kSlots; ++q) {
        if (r[q] < 0) continue;
        const uint32_t u32[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = fmaf(ws[q], __uint_as_float(u32[i] << 16), acc[2 * i]);
          acc[2 * i + 1] = fmaf(ws[q], __uint_as_float(u32[i] & 0xFFFF0000u), acc[2 * i + 1]);
        }
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      o[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * N)[ch] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace dg
