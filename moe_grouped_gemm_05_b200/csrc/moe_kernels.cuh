// MoE permutation into the contiguous M-grouped layout and the inverse,
// weighted combine (DeepGEMM pages: charles2530.github.io "源码与接入" §七, the
// group_by_expert step before the grouped GEMM and the combine after it;
// juejin.cn §4 "分组 GEMM（连续布局）": expert segments aligned to the M block).
//
// moe_route_kernel   one CTA per expert, in clusters: the cluster's CTAs
//                    split the histogram of all routing ids and add it up
//                    through distributed shared memory -> each expert's
//                    segment offset (segments in expert order, each padded to
//                    128 rows) -> a stable compaction of the (token, slot)
//                    pairs routed to the CTA's expert (a block scan), so the
//                    layout is deterministic.  Writes m_indices, src_of,
//                    row_of, and zero scale words for padding rows.
// moe_gather_kernel  full grid, tokens in source order: copies each token's
//                    FP8 codes and packed scale words to the rows of its
//                    routed slots (one read of each token row).
// moe_combine_kernel out[t] = bf16(sum_s w[t,s] * D[row_of[t,s]]), FP32 sums.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace dg {

constexpr int kMoeMaxExperts = 1024;
constexpr int kMoeThreads = 1024;
// Routed slots up to which the routing kernel stages all ids in shared memory (192 KB).
constexpr int kMoeStagedIds = 48 * 1024;

// CTAs per cluster of the routing kernel: the cluster's CTAs split the
// histogram of the ids and add their slices through distributed shared memory.
constexpr int kRouteCluster = 8;

// One CTA per expert (the grid is G rounded up to whole clusters).
// kStaged: every CTA first copies the n ids into dynamic shared memory
// (n <= kMoeStagedIds), so it reads them from global memory once.
// 1. CTA r of a cluster counts the ids of slice r (1/kRouteCluster of them)
//    for every expert, and marks that slice's unrouted slots;
// 2. the cluster adds the slice counts through distributed shared memory,
//    and every CTA derives the segment offsets (expert order, 128-aligned);
// 3. CTA e compacts the slots routed to expert e, in slot order (16 slots a
//    thread per chunk, a block scan orders the threads), and pads its segment.
template <bool kStaged>
__global__ void __launch_bounds__(kMoeThreads) moe_route_kernel(const int32_t* __restrict__ ids, int n, int topk,
                                                                int G, int M_cap, int kp, int32_t* __restrict__ m_indices,
                                                                int32_t* __restrict__ row_of,
                                                                int32_t* __restrict__ src_of,
                                                                uint32_t* __restrict__ sfa_perm) {
  __shared__ int cnt[kMoeMaxExperts];  // this CTA's slice counts
  __shared__ int tot[kMoeMaxExperts];  // the whole histogram
  __shared__ int warp_tot[2][32];      // double-buffered by chunk parity: one barrier pair per chunk
  __shared__ int chunk_off[2];
  __shared__ int seg_off, total_rows;
  extern __shared__ __align__(16) int32_t ids_s[];  // kStaged: ids[0, n)
  grid_dep_wait();
  grid_dep_launch();
  const int e = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = blockDim.x >> 5;
  const int crank = static_cast<int>(cluster_cta_rank());
  for (int i = tid; i < G; i += blockDim.x) cnt[i] = 0;
  if constexpr (kStaged) {
    // 8 independent loads in flight per thread, then their stores
    for (int base = 0; base < n; base += 8 * kMoeThreads) {
      int r[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = base + j * kMoeThreads + tid;
        r[j] = i < n ? __ldg(&ids[i]) : 0;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = base + j * kMoeThreads + tid;
        if (i < n) ids_s[i] = r[j];
      }
    }
  }
  auto id_at = [&](int i) -> int {
    if constexpr (kStaged) return ids_s[i];
    else return __ldg(&ids[i]);
  };
  __syncthreads();
  // 1. this CTA's slice: counts (lanes holding the same id add once per warp),
  //    unrouted and out-of-range slots
  const int slice = (n + kRouteCluster - 1) / kRouteCluster;
  const int s0 = min(n, crank * slice), s1 = min(n, s0 + slice);
  for (int base = s0; base < s1; base += blockDim.x) {
    const int i = base + tid;
    const int v = i < s1 ? id_at(i) : -1;
    if (i < s1 && (v < 0 || v >= G)) row_of[i] = -1;
    if (__any_sync(0xffffffffu, i < s1 && !(v >= -1 && v < G)) && lane == 0) atomicOr(&g_dg_error, 0x2);
    const unsigned same = __match_any_sync(0xffffffffu, v);
    if (v >= 0 && v < G && lane == __ffs(same) - 1) atomicAdd(&cnt[v], __popc(same));
  }
  cluster_sync();
  // 2. the histogram: the sum of the cluster's slice counts
  for (int g = tid; g < G; g += blockDim.x) {
    const uint32_t a = smem_u32(&cnt[g]);
    int t = 0;
#pragma unroll
    for (int c = 0; c < kRouteCluster; ++c) t += static_cast<int>(ld_shared_cluster_u32(mapa_shared(a, c)));
    tot[g] = t;
  }
  cluster_sync();  // every CTA has read every slice: from here none reads a peer
  if (tid == 0) {
    int off = 0, all = 0;
    for (int g = 0; g < G; ++g) {
      const int padded = (tot[g] + 127) & ~127;
      if (g < e) off += padded;
      all += padded;
    }
    seg_off = off;
    total_rows = all;
    chunk_off[0] = 0;
  }
  __syncthreads();
  if (e >= G) return;  // a CTA that only completes the last cluster
  // 3. stable compaction of the slots routed to expert e
  int par = 0;
  for (int base = 0; base < n; base += 16 * kMoeThreads, par ^= 1) {
    const int i0 = base + 16 * tid;
    unsigned flags = 0;
    if (kStaged && i0 + 15 < n) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int4 v4 = reinterpret_cast<const int4*>(ids_s + i0)[q];  // i0 is a multiple of 16: aligned
        flags |= (static_cast<unsigned>(v4.x == e) | (static_cast<unsigned>(v4.y == e) << 1) |
                  (static_cast<unsigned>(v4.z == e) << 2) | (static_cast<unsigned>(v4.w == e) << 3))
                 << (4 * q);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int i = i0 + j;
        flags |= static_cast<unsigned>(i < n && id_at(i) == e) << j;
      }
    }
    const int c = __popc(flags);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) warp_tot[par][warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int v = lane < nw ? warp_tot[par][lane] : 0;
      int x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += u;
      }
      if (lane < nw) warp_tot[par][lane] = x - v;  // exclusive prefix of the warps
      if (lane == 31) chunk_off[par ^ 1] = chunk_off[par] + x;
    }
    __syncthreads();
    int pos = seg_off + chunk_off[par] + warp_tot[par][warp] + incl - c;
    while (flags != 0u) {
      const int i = i0 + __ffs(flags) - 1;
      flags &= flags - 1u;
      m_indices[pos] = e;
      src_of[pos] = i / topk;
      row_of[i] = pos;
      ++pos;
    }
  }
  // padding rows of this segment (scale words 0); CTA 0 also marks the tail past the last segment
  const int c = tot[e];
  const int pad0 = seg_off + c, pad1 = seg_off + ((c + 127) & ~127);
  for (int r = pad0 + tid; r < pad1; r += blockDim.x) {
    m_indices[r] = -1;
    src_of[r] = -1;
  }
  for (int u = tid; u < (pad1 - pad0) * kp; u += blockDim.x)
    sfa_perm[static_cast<size_t>(u / (pad1 - pad0)) * M_cap + pad0 + u % (pad1 - pad0)] = 0u;
  if (e == 0) {
    for (int r = total_rows + tid; r < M_cap; r += blockDim.x) {
      m_indices[r] = -1;
      src_of[r] = -1;
    }
    const int tail = M_cap - total_rows;
    for (long long u = tid; u < static_cast<long long>(tail) * kp; u += blockDim.x)
      sfa_perm[static_cast<size_t>(u / tail) * M_cap + total_rows + u % tail] = 0u;
  }
}

// a_perm[row_of[t][s]] = q[t] (K bytes) and sfa_perm[kp][row_of[t][s]] =
// sfa[kp][t] for every routed slot s of token t: tokens in source order, so
// each token's row is read once however many slots it has.  Padding and tail
// rows keep whatever codes they held (their scale words are zeroed by
// moe_route_kernel).
__global__ void __launch_bounds__(256) moe_gather_kernel(const uint8_t* __restrict__ q, const uint32_t* __restrict__ sfa,
                                                        int T, int K, int kp, int topk,
                                                        const int32_t* __restrict__ row_of, int M_cap,
                                                        uint8_t* __restrict__ a_perm, uint32_t* __restrict__ sfa_perm) {
  grid_dep_wait();
  grid_dep_launch();
  const int chunks = K / 16;
  const int t4 = (T + 3) & ~3;
  const long long total = static_cast<long long>(T) * chunks;
  for (long long u = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(u / chunks);
    const int ch = static_cast<int>(u - static_cast<long long>(t) * chunks);
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(q + static_cast<size_t>(t) * K) + ch);
    const uint32_t w = ch < kp ? __ldg(&sfa[static_cast<size_t>(ch) * t4 + t]) : 0u;
    for (int s = 0; s < topk; ++s) {
      const int r = __ldg(&row_of[static_cast<size_t>(t) * topk + s]);
      if (r < 0) continue;
      reinterpret_cast<uint4*>(a_perm + static_cast<size_t>(r) * K)[ch] = v;
      if (ch < kp) sfa_perm[static_cast<size_t>(ch) * M_cap + r] = w;
    }
  }
}

// One thread per (token, 8 output columns).
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
    for (int s = 0; s < topk; ++s) {
      const int r = __ldg(&row_of[t * topk + s]);
      if (r < 0) continue;
      const float ws = w ? __ldg(&w[t * topk + s]) : 1.0f;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(d + static_cast<size_t>(r) * N) + ch);
      const uint32_t u32[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(ws, __uint_as_float(u32[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = fmaf(ws, __uint_as_float(u32[i] & 0xFFFF0000u), acc[2 * i + 1]);
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
