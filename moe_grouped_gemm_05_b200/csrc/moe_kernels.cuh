// MoE permutation into the contiguous M-grouped layout and the inverse,
// weighted combine (DeepGEMM pages: charles2530.github.io "源码与接入" §七, the
// group_by_expert step before the grouped GEMM and the combine after it;
// juejin.cn §4 "分组 GEMM（连续布局）": expert segments aligned to the M block).
//
// moe_route_kernel   one CTA per expert: histogram of all routing ids in
//                    shared memory -> this expert's segment offset (segments
//                    in expert order, each padded to 128 rows) -> a stable
//                    compaction of the (token, slot) pairs routed to it
//                    (warp ballots + a block scan), so the layout is
//                    deterministic.  Writes m_indices, src_of and row_of.
// moe_gather_kernel  full grid: copies each routed row's FP8 codes and its
//                    packed scale words to its destination row.
// moe_combine_kernel out[t] = bf16(sum_s w[t,s] * D[row_of[t,s]]), FP32 sums.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace dg {

constexpr int kMoeMaxExperts = 1024;
constexpr int kMoeThreads = 1024;

__global__ void __launch_bounds__(kMoeThreads) moe_route_kernel(const int32_t* __restrict__ ids, int n, int topk,
                                                                int G, int M_cap, int32_t* __restrict__ m_indices,
                                                                int32_t* __restrict__ row_of,
                                                                int32_t* __restrict__ src_of) {
  __shared__ int cnt[kMoeMaxExperts];
  __shared__ int warp_tot[32];
  __shared__ int seg_off, total_rows, running;
  grid_dep_wait();
  grid_dep_launch();
  const int e = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < G; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  for (int i = tid; i < n; i += blockDim.x) {
    const int v = __ldg(&ids[i]);
    if (v >= 0 && v < G) atomicAdd(&cnt[v], 1);
    else if (v != -1 && e == 0) atomicOr(&g_dg_error, 0x2);
  }
  __syncthreads();
  if (tid == 0) {
    int off = 0, tot = 0;
    for (int g = 0; g < G; ++g) {
      const int padded = (cnt[g] + 127) & ~127;
      if (g < e) off += padded;
      tot += padded;
    }
    seg_off = off;
    total_rows = tot;
    running = 0;
  }
  __syncthreads();
  // stable compaction of the slots routed to expert e
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + tid;
    const bool flag = i < n && __ldg(&ids[i]) == e;
    const unsigned ballot = __ballot_sync(0xffffffffu, flag);
    if (lane == 0) warp_tot[warp] = __popc(ballot);
    __syncthreads();
    if (warp == 0) {
      const int nw = blockDim.x >> 5;
      int v = lane < nw ? warp_tot[lane] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (lane < nw) warp_tot[lane] = incl - v;  // exclusive
    }
    __syncthreads();
    if (flag) {
      const int pos = seg_off + running + warp_tot[warp] + __popc(ballot & ((1u << lane) - 1u));
      m_indices[pos] = e;
      src_of[pos] = i / topk;
      row_of[i] = pos;
    }
    __syncthreads();
    if (tid == blockDim.x - 1) running += warp_tot[warp] + __popc(ballot);
    __syncthreads();
  }
  // padding rows of this segment; CTA 0 also marks the tail and the unrouted slots
  const int c = cnt[e];
  const int padded = (c + 127) & ~127;
  for (int r = seg_off + c + tid; r < seg_off + padded; r += blockDim.x) {
    m_indices[r] = -1;
    src_of[r] = -1;
  }
  if (e == 0) {
    for (int r = total_rows + tid; r < M_cap; r += blockDim.x) {
      m_indices[r] = -1;
      src_of[r] = -1;
    }
    for (int i = tid; i < n; i += blockDim.x) {
      const int v = __ldg(&ids[i]);
      if (v < 0 || v >= G) row_of[i] = -1;
    }
  }
}

// a_perm[r] = q[src_of[r]] (K bytes) and sfa_perm[kp][r] = sfa[kp][src_of[r]];
// padding rows get scale words 0 and keep whatever codes they held.
__global__ void __launch_bounds__(256) moe_gather_kernel(const uint8_t* __restrict__ q, const uint32_t* __restrict__ sfa,
                                                        int T, int K, int kp, const int32_t* __restrict__ src_of,
                                                        int M_cap, uint8_t* __restrict__ a_perm,
                                                        uint32_t* __restrict__ sfa_perm) {
  grid_dep_wait();
  grid_dep_launch();
  const int chunks = K / 16;
  const int t4 = (T + 3) & ~3;
  const long long total = static_cast<long long>(M_cap) * chunks;
  for (long long u = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(u / chunks);
    const int ch = static_cast<int>(u - static_cast<long long>(r) * chunks);
    const int t = __ldg(&src_of[r]);
    if (t >= 0)
      reinterpret_cast<uint4*>(a_perm + static_cast<size_t>(r) * K)[ch] =
          __ldg(reinterpret_cast<const uint4*>(q + static_cast<size_t>(t) * K) + ch);
    if (ch < kp) sfa_perm[static_cast<size_t>(ch) * M_cap + r] = t >= 0 ? __ldg(&sfa[static_cast<size_t>(ch) * t4 + t]) : 0u;
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
