// Host side of libdg.so: argument validation, tensor maps, the tile
// heuristic, kernel launches, the UE8M0 scale-packing kernel and the
// device error word.  See include/dg.h for the contract of each entry point.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "dg.h"
#include "fp8_gemm_kernel.cuh"
#include "quant_kernel.cuh"
#include "moe_kernels.cuh"

namespace dg {

// ------------------------------------------------------------------ errors

static thread_local char t_last_error[512] = "";

static int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
  return code;
}

#define DG_CUDA_TRY(expr)                                                               \
  do {                                                                                  \
    cudaError_t e_ = (expr);                                                            \
    if (e_ != cudaSuccess)                                                              \
      return fail(DG_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(e_));         \
  } while (0)

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// ------------------------------------------------------------------ device info

static std::atomic<int> g_num_sms_override{0};
// Share of the GPU's tensor cores (SMs) a call may occupy, in percent.
static std::atomic<int> g_tc_util{100};

// SMs a call plans and launches for: the device's, capped by dg_set_num_sms
// and by the dg_set_tc_util share (at least one CTA pair).
static int usable_sms(int device_sms) {
  const int o = g_num_sms_override.load(std::memory_order_relaxed);
  int g = o > 0 ? std::min(o, device_sms) : device_sms;
  const int u = g_tc_util.load(std::memory_order_relaxed);
  if (u < 100) g = std::max(2, g * u / 100);
  return g;
}
// Programmatic dependent launch of every kernel (on by default): a kernel may
// start its set-up while the previous grid of the stream finishes, and waits
// (griddepcontrol.wait) before its first global-memory access.
static std::atomic<int> g_pdl{1};
// Limit of every main-loop pipeline wait inside the GEMM kernels, in ns.
static std::atomic<uint64_t> g_wait_limit_ns{kWaitLimitNs};

// Environment defaults of the run-time knobs, read once when the library is
// loaded: DG_NUM_SMS (as dg_set_num_sms), DG_TC_UTIL (as dg_set_tc_util, a
// percent) and DG_PDL (as dg_set_pdl, 0 or 1).  A value that is not an
// integer in the knob's range is ignored.  Calls of the setters override them.
static int env_int(const char* name, long lo, long hi, int fallback) {
  const char* v = std::getenv(name);
  if (v == nullptr || *v == '\0') return fallback;
  char* end = nullptr;
  const long x = std::strtol(v, &end, 10);
  if (*end != '\0' || x < lo || x > hi) return fallback;
  return static_cast<int>(x);
}
static const bool g_env_applied = [] {
  g_num_sms_override.store(env_int("DG_NUM_SMS", 0, 1 << 20, 0));
  g_tc_util.store(env_int("DG_TC_UTIL", 1, 100, 100));
  g_pdl.store(env_int("DG_PDL", 0, 1, 1));
  return true;
}();

// One launch attribute set: programmatic stream serialisation when enabled,
// plus a cluster of `cluster` CTAs along x when cluster > 1.
struct LaunchAttrs {
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  explicit LaunchAttrs(int cluster) {
    if (g_pdl.load(std::memory_order_relaxed)) {
      attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[n].val.programmaticStreamSerializationAllowed = 1;
      ++n;
    }
    if (cluster > 1) {
      attr[n].id = cudaLaunchAttributeClusterDimension;
      attr[n].val.clusterDim.x = cluster;
      attr[n].val.clusterDim.y = 1;
      attr[n].val.clusterDim.z = 1;
      ++n;
    }
  }
};

// cudaLaunchKernelEx of a kernel with the PDL attribute (and clusters of `cluster` CTAs).
template <typename... Params, typename... Args>
static cudaError_t launch_plain_smem(void (*kernel)(Params...), long long blocks, int threads, size_t smem,
                                     cudaStream_t st, int cluster, Args&&... args) {
  LaunchAttrs la(cluster);
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(static_cast<unsigned>(blocks));
  lc.blockDim = dim3(threads);
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  lc.attrs = la.attr;
  lc.numAttrs = la.n;
  return cudaLaunchKernelEx(&lc, kernel, std::forward<Args>(args)...);
}
template <typename... Params, typename... Args>
static cudaError_t launch_plain(void (*kernel)(Params...), long long blocks, int threads, cudaStream_t st,
                                Args&&... args) {
  return launch_plain_smem(kernel, blocks, threads, 0, st, 1, std::forward<Args>(args)...);
}
static thread_local int t_force_bn = 0;

struct DeviceInfo {
  int sms = 0;
  int major = 0, minor = 0;
  int max_smem = 0;
};

static int device_info(DeviceInfo* out) {
  int dev = 0;
  DG_CUDA_TRY(cudaGetDevice(&dev));
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool have[64] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= 64) return fail(DG_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  if (!have[dev]) {
    DeviceInfo d;
    DG_CUDA_TRY(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    DG_CUDA_TRY(cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev));
    DG_CUDA_TRY(cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev));
    DG_CUDA_TRY(cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
    cache[dev] = d;
    have[dev] = true;
  }
  *out = cache[dev];
  if (out->major != 10 || out->minor != 0)
    return fail(DG_ERR_UNSUPPORTED, "sm_%d%d device: this library is built for sm_100a only",
                out->major, out->minor);
  return DG_OK;
}

// ------------------------------------------------------------------ tensor maps

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D tiled map: dims {d0 (contiguous), d1, d2}, byte strides of d1 and d2, box {b0, b1, 1}.
static int make_map(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t d0,
                    uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t b0,
                    uint32_t b1, CUtensorMapSwizzle swz, const char* what) {
  auto fn = encode_fn();
  if (!fn) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1, stride2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, type, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(DG_ERR_CUDA, "tensor map for %s rejected (CUresult %d; dims %llu x %llu x %llu)", what,
                static_cast<int>(r), (unsigned long long)d0, (unsigned long long)d1,
                (unsigned long long)d2);
  return DG_OK;
}

// ------------------------------------------------------------------ configurations

using KernelFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, GemmArgs);

struct Config {
  int bn = 0;
  int stages = 0;
  int ctas = 1;
  int smem = 0;
  int num_acc = 1;
  int pipes = 1;  // load/MMA pipelines per CTA (alternate tiles)
  int layout = 0; // bit 0: A MN-major, bit 1: B MN-major
  bool splitk = false;  // both pipelines on every tile, each on half of K
  int a_rows = 128;     // rows of A per stage and TMA box: 128, or 64 for problems of at most 64 rows
  int threads = kThreads;
  KernelFn fn = nullptr;
};

template <int BN, int STAGES, int MODE, int CTAS, bool OUT_F32 = false, int PIPES = 1, int LAYOUT = 0,
          bool SPLITK = false, int A_ROWS = 128>
static Config make_config() {
  Config c;
  c.bn = BN;
  c.stages = STAGES;
  c.ctas = CTAS;
  using L = Layout<BN, STAGES, CTAS, PIPES, LAYOUT, MODE == MODE_MASKED, MODE == MODE_CONTIG && CTAS == 2, A_ROWS>;
  c.smem = L::kSmemBytes;
  c.num_acc = L::kNumAcc;
  c.pipes = PIPES;
  c.layout = LAYOUT;
  c.splitk = SPLITK;
  c.a_rows = A_ROWS;
  c.threads = kThreadsFor<PIPES>;
  c.fn = reinterpret_cast<KernelFn>(&fp8_gemm_kernel<BN, STAGES, MODE, CTAS, OUT_F32, PIPES, LAYOUT, SPLITK, A_ROWS>);
  return c;
}

// Built configurations.  A 2-CTA tile spans 256 rows, which the contiguous
// layout (128-row expert alignment) cannot guarantee to be one expert; its
// 2-CTA tiles pair 128-row blocks within each expert's run of blocks (a table
// the kernel builds from m_indices), an odd run ending in a half-empty pair.
// Host-side id of the dense kernels with FP32 output (optionally + C).
constexpr int MODE_DENSE_F32 = 3;
// Host-side ids of the dense kernels with MN-major operands: MODE_DENSE_MN + LAYOUT - 1
// (LAYOUT 1: A MN-major (TT), 2: B MN-major (NN), 3: both (TN)).
constexpr int MODE_DENSE_MN = 4;

template <int MODE>
static const Config* config_table(int* count) {
  if constexpr (MODE == MODE_DENSE_F32) {
    static const Config table[] = {
        make_config<128, 6, MODE_DENSE, 1, true>(), make_config<224, 4, MODE_DENSE, 1, true>(),
        make_config<256, 4, MODE_DENSE, 1, true>(),
    };
    *count = static_cast<int>(sizeof(table) / sizeof(table[0]));
    return table;
  } else if constexpr (MODE == MODE_DENSE_MN) {
    static const Config table[] = {
        make_config<128, 6, MODE_DENSE, 1, false, 1, 1>(), make_config<224, 4, MODE_DENSE, 1, false, 1, 1>(),
        make_config<224, 6, MODE_DENSE, 2, false, 2, 1>(),
    };
    *count = static_cast<int>(sizeof(table) / sizeof(table[0]));
    return table;
  } else if constexpr (MODE == MODE_DENSE_MN + 1 || MODE == MODE_DENSE_MN + 2) {
    // an MN-major B tile is whole 128-column boxes per CTA: 128 or 256 wide, 256 on a pair
    constexpr int LAYOUT = MODE - MODE_DENSE_MN + 1;
    static const Config table[] = {
        make_config<128, 6, MODE_DENSE, 1, false, 1, LAYOUT>(), make_config<256, 4, MODE_DENSE, 1, false, 1, LAYOUT>(),
        make_config<256, 6, MODE_DENSE, 2, false, 1, LAYOUT>(),
    };
    *count = static_cast<int>(sizeof(table) / sizeof(table[0]));
    return table;
  } else if constexpr (MODE == MODE_CONTIG) {
    static const Config table[] = {
        make_config<128, 6, MODE, 1>(), make_config<224, 4, MODE, 1>(), make_config<256, 4, MODE, 1>(),
        make_config<224, 6, MODE, 2, false, 2>(),
    };
    *count = static_cast<int>(sizeof(table) / sizeof(table[0]));
    return table;
  } else {
    static const Config table[] = {
        make_config<128, 6, MODE, 1>(), make_config<224, 4, MODE, 1>(), make_config<256, 4, MODE, 1>(),
        make_config<128, 6, MODE, 2>(), make_config<224, 6, MODE, 2>(), make_config<256, 6, MODE, 2>(),
        make_config<224, 6, MODE, 2, false, 2>(), make_config<128, 6, MODE, 2, false, 2>(),
        make_config<64, 8, MODE, 1>(),
        // decode: split-K tiles with 64-row A stages (problems of at most 64 rows per group) come
        // first, so that they win ties and forced lookups where they fit
        make_config<64, (MODE == MODE_DENSE ? 12 : 10), MODE, 1, false, 2, 0, true, 64>(),
        make_config<64, (MODE == MODE_DENSE ? 8 : 6), MODE, 1, false, 2, 0, true>(),
        make_config<128, 4, MODE, 1, false, 2, 0, true>(),
    };
    *count = static_cast<int>(sizeof(table) / sizeof(table[0]));
    return table;
  }
}

// Whether configuration c can run a problem whose groups hold a_extent rows of A.
static bool a_rows_fit(const Config& c, long long a_extent) { return c.a_rows == 128 || a_extent <= c.a_rows; }

// First built configuration with this tile width, CTA count (0: any) and
// number of pipelines (0: any) that fits groups of a_extent rows of A (-1: any size).
template <int MODE>
static const Config* find_config(int bn, int ctas, int pipes = 0, long long a_extent = -1) {
  int n = 0;
  const Config* t = config_table<MODE>(&n);
  for (int i = 0; i < n; ++i)
    if (t[i].bn == bn && (ctas == 0 || t[i].ctas == ctas) && (pipes == 0 || t[i].pipes == pipes) &&
        (a_extent < 0 || a_rows_fit(t[i], a_extent)))
      return &t[i];
  return nullptr;
}

static thread_local int t_force_ctas = 0;
static thread_local int t_force_pipes = 0;

// Heuristic: a cost model fitted to measurements on B200.  A configuration
// spends, per tile of a CTA (or CTA pair), kb_ns per 128-wide K block plus
// tile_ns for the rest (first loads, epilogue drain, tile switch); a problem
// costs (tiles / units) such tiles, at least one, so both the K depth and the
// N tile count enter.  Problems that stream more bytes than that time can
// carry are bound by HBM instead: max(compute, bytes / kHbmBytesPerNs).
// The constants were fitted to CUDA-event timings of every built
// configuration, back to back under the 1 kW power cap, on dense
// 4096x7168x2048 (K = 2048) and 8192^3 (K = 8192), and checked against the
// contiguous 8 x (4096 x 7168) workload (within 3 %) and the masked and
// 64-row decode workloads (the model's pick is the fastest measured).
// Every tcgen05 instruction costs the thread that issues it ~60 cycles, so
// narrow tiles pay more per FLOP (kb_ns of a 128-wide tile is not half that
// of a 256-wide one); 2-CTA tiles halve the B bytes an SM loads; two
// pipelines per CTA hide one issuing thread's overhead behind the other's.
struct CostParams {
  int bn, ctas, pipes;
  bool splitk;
  double kb_ns, tile_ns;
};
// The contiguous layout's tiles run slower per K block than dense ones when
// the experts' weights exceed L2 (8 x 4096 x 7168 bytes here), most of all
// the 1-CTA 224-wide tile, which loads twice the B bytes of a 2-CTA tile per
// SM; its kb_ns are fitted on that workload (interleaved runs), tile_ns kept.
// The 256-wide tile has one accumulator, which its epilogue releases as soon
// as it has been read; the 2-CTA tiles pair blocks within each expert's run.
static const CostParams kCostContig[] = {
    {128, 1, 1, false, 363, 757}, {224, 1, 1, false, 531, 1345}, {256, 1, 1, false, 522, 2250},
    {224, 2, 2, false, 405, 2023},
};
static const CostParams kCost[] = {
    {128, 1, 1, false, 360, 757},  {224, 1, 1, false, 453, 1345}, {256, 1, 1, false, 514, 2566},
    {128, 2, 1, false, 366, 1095}, {224, 2, 1, false, 442, 1865}, {256, 2, 1, false, 482, 3280},
    {224, 2, 2, false, 408, 2023}, {128, 2, 2, false, 286, 1186}, {64, 1, 1, false, 313, 577},
    {64, 1, 2, true, 387, 959},    {128, 1, 2, true, 680, 1288},
};
// Sustained HBM read+write rate of a streaming GEMM (the masked workload's measured 5.4 TB/s), bytes per ns.
constexpr double kHbmBytesPerNs = 5400.0;

template <int MODE>
static const CostParams* cost_params(const Config& c) {
  if (MODE == MODE_CONTIG)
    for (const CostParams& k : kCostContig)
      if (k.bn == c.bn && k.ctas == c.ctas && k.pipes == c.pipes && k.splitk == c.splitk) return &k;
  const CostParams* best = nullptr;
  for (const CostParams& k : kCost) {
    if (k.bn == c.bn && k.ctas == c.ctas && k.pipes == c.pipes && k.splitk == c.splitk) return &k;
    if (k.bn == c.bn && k.ctas == c.ctas && !best) best = &k;  // layouts / FP32 output: same tile shape
  }
  return best;
}

// Estimated time (ns) of configuration c.  rows_est: rows of the problem
// (masked: the expected valid rows); groups: experts (contiguous, masked).
template <int MODE>
static double config_cost(const Config& c, long long rows_est, int N, int K, int sms, int groups) {
  const CostParams* k = cost_params<MODE>(c);
  if (!k) return 1e300;
  const long long tile_m = 128LL * c.ctas;
  long long m_tiles;
  if (MODE == MODE_MASKED) {
    const long long per = std::max<long long>(1, rows_est / std::max(1, groups));
    m_tiles = static_cast<long long>(groups) * ((per + tile_m - 1) / tile_m);
  } else {
    m_tiles = (rows_est + tile_m - 1) / tile_m;
    // pairs within each expert's run of blocks: about one half-empty pair per two experts
    if (MODE == MODE_CONTIG && c.ctas == 2) m_tiles += (groups + 1) / 2;
  }
  // the last N tile runs a narrower MMA when it is ragged (64 or 128 columns)
  const int full = N / c.bn, rem = N - full * c.bn;
  double n_tiles = full;
  if (rem > 0) {
    const int nt = (c.ctas == 1 && c.bn > 64 && rem <= 64) ? 64 : ((c.bn > 128 && rem <= 128) ? 128 : c.bn);
    n_tiles += static_cast<double>(nt) / c.bn;
  }
  const double units = std::max(1, sms / c.ctas);
  const double waves = std::max(1.0, static_cast<double>(m_tiles) * n_tiles / units);
  const double kb = (K / 128) * (c.splitk ? 0.5 : 1.0);
  const double compute = waves * (kb * k->kb_ns + k->tile_ns);
  const double experts = MODE == MODE_DENSE ? 1.0 : groups;
  const double bytes = static_cast<double>(rows_est) * (K + 2.0 * N) + experts * static_cast<double>(N) * K;
  const double memory = bytes / kHbmBytesPerNs;
  // the smaller term is not fully hidden behind the larger one (first loads,
  // last epilogue): a tenth of it breaks ties between HBM-bound configurations
  return std::max(compute, memory) + 0.1 * std::min(compute, memory);
}

// a_extent: rows of A per group (dense and contiguous: the rows; masked: M_max), -1 for rows_est.
template <int MODE>
static const Config* choose_config(long long rows_est, int N, int K, int sms, int groups = 1,
                                   long long a_extent = -1) {
  if (a_extent < 0) a_extent = rows_est;
  // A forced tile applies to the entry points that have it built; the others
  // keep the heuristic (each layout and output type builds its own set).
  if (t_force_bn) {
    const Config* f = find_config<MODE>(t_force_bn, t_force_ctas, t_force_pipes, a_extent);
    if (f && !(MODE == MODE_CONTIG && f->ctas == 2 && rows_est / 128 > kMaxContigBlocks)) return f;
  }
  int n = 0;
  const Config* t = config_table<MODE>(&n);
  const Config* best = nullptr;
  double best_cost = 1e300;
  for (int i = 0; i < n; ++i) {
    const Config& c = t[i];
    if (!a_rows_fit(c, a_extent)) continue;
    // split-K tiles keep no second accumulator for overlap; they need at least two groups of 4 K blocks
    if (c.splitk && K <= 4 * 128) continue;
    // contiguous CTA pairs: the device-built pair table holds kMaxContigBlocks blocks
    if (MODE == MODE_CONTIG && c.ctas == 2 && rows_est / 128 > kMaxContigBlocks) continue;
    const double cost = config_cost<MODE == MODE_CONTIG || MODE == MODE_MASKED ? MODE : MODE_DENSE>(
        c, rows_est, N, K, sms, groups);
    if (cost < best_cost * 0.999) {
      best_cost = cost;
      best = &c;
    }
  }
  return best;
}

static int raster_group(int num_m_blocks) { return std::min(num_m_blocks, 16); }

// Clusters of two CTAs must sit in one GPC, so fewer than sms/2 pairs may be
// resident at once; a persistent grid larger than that would run a second
// wave.  Queried once per configuration and device.
static int max_active_pairs(const Config* cfg, int sms) {
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, int> cache;  // (device, kernel) -> pairs
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return sms / 2;
  const auto key = std::make_pair(dev, reinterpret_cast<const void*>(cfg->fn));
  std::lock_guard<std::mutex> lock(mu);
  if (cache.find(key) == cache.end()) {
    if (cudaFuncSetAttribute(reinterpret_cast<const void*>(cfg->fn), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             cfg->smem) != cudaSuccess)
      return sms / 2;
    cudaLaunchConfig_t lc = {};
    cudaLaunchAttribute attr[1];
    lc.gridDim = dim3(sms / 2 * 2);
    lc.blockDim = dim3(cfg->threads);
    lc.dynamicSmemBytes = cfg->smem;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(cfg->fn), &lc) != cudaSuccess || n <= 0)
      n = sms / 2;
    cache[key] = std::min(n, sms / 2);
  }
  return cache[key];
}

template <int MODE>
static int launch(const Config* cfg, int grid, const CUtensorMap* maps, GemmArgs args,
                  cudaStream_t stream) {
  args.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  // The shared-memory opt-in is a per-device function attribute: set it once
  // per (device, configuration).
  constexpr int kMaxDevices = 64, kMaxConfigs = 32;
  static std::mutex mu;
  static bool attr_done[kMaxDevices][kMaxConfigs] = {};
  int n = 0;
  const Config* t = config_table<MODE>(&n);
  const int idx = static_cast<int>(cfg - t);
  int dev = 0;
  DG_CUDA_TRY(cudaGetDevice(&dev));
  if (idx < 0 || idx >= n || idx >= kMaxConfigs || dev < 0 || dev >= kMaxDevices)
    return fail(DG_ERR_UNSUPPORTED, "configuration %d / device %d outside the launch table", idx, dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!attr_done[dev][idx]) {
      DG_CUDA_TRY(cudaFuncSetAttribute(reinterpret_cast<const void*>(cfg->fn),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, cfg->smem));
      attr_done[dev][idx] = true;
    }
  }
  LaunchAttrs la(cfg->ctas);
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(cfg->threads);
  lc.dynamicSmemBytes = cfg->smem;
  lc.stream = stream;
  lc.attrs = la.attr;
  lc.numAttrs = la.n;
  DG_CUDA_TRY(cudaLaunchKernelEx(&lc, cfg->fn, maps[0], maps[1], maps[2], args));
  return DG_OK;
}

// Builds the tensor maps of one call.
//   A : [GA][rowsA][K] bytes    box 128 x 128 (K x rows; 128 x 64 with 64-row stages), 128-byte swizzle
//       ([GA][K][rowsA] when MN-major: box 128 x 128 (rows x K))
//   B : [GB][N][K] bytes        box 128 x BN/CTAS,         128-byte swizzle
//       ([GB][K][N] when MN-major: box 128 x 128 (N x K), BN/CTAS/128 boxes per stage)
//   D : [GD][rowsD][N] bf16     box 32 x 32,               64-byte swizzle
static int build_maps(CUtensorMap* maps, const Config* cfg, const void* a, const void* b, void* d,
                      int rowsA, int GA, int N, int K, int GB, int rowsD, int GD, bool d_f32 = false) {
  int r;
  if (cfg->layout & 1) {  // A stored [GA][K][rowsA]: 128 rows x 128 K per box
    if ((r = make_map(&maps[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, a, rowsA, K, GA, rowsA,
                      static_cast<uint64_t>(rowsA) * K, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B, "A")))
      return r;
  } else if ((r = make_map(&maps[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, a, K, rowsA, GA, K,
                           static_cast<uint64_t>(rowsA) * K, 128, cfg->a_rows, CU_TENSOR_MAP_SWIZZLE_128B, "A"))) {
    return r;
  }
  if (cfg->layout & 2) {  // B stored [GB][K][N]: 128 columns x 128 K per box
    if ((r = make_map(&maps[1], CU_TENSOR_MAP_DATA_TYPE_UINT8, b, N, K, GB, N, static_cast<uint64_t>(N) * K, 128,
                      128, CU_TENSOR_MAP_SWIZZLE_128B, "B")))
      return r;
  } else if ((r = make_map(&maps[1], CU_TENSOR_MAP_DATA_TYPE_UINT8, b, K, N, GB, K, static_cast<uint64_t>(N) * K,
                           128, cfg->bn / cfg->ctas, CU_TENSOR_MAP_SWIZZLE_128B, "B"))) {
    return r;
  }
  if (d_f32) {  // 16 FP32 columns (64 B) per box row
    if ((r = make_map(&maps[2], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, d, N, rowsD, GD, static_cast<uint64_t>(N) * 4,
                      static_cast<uint64_t>(rowsD) * N * 4, 16, 32, CU_TENSOR_MAP_SWIZZLE_64B, "D")))
      return r;
  } else if ((r = make_map(&maps[2], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d, N, rowsD, GD,
                           static_cast<uint64_t>(N) * 2, static_cast<uint64_t>(rowsD) * N * 2, 32, 32,
                           CU_TENSOR_MAP_SWIZZLE_64B, "D")))
    return r;
  return DG_OK;
}

// Tensor maps depend only on pointers, shapes and the tile configuration, so
// repeated calls (weights, rotating activation buffers, graph replays on the
// host side) reuse them: a small per-thread direct-mapped cache keyed by all
// inputs of build_maps.
struct MapKey {
  const void* a;
  const void* b;
  const void* d;
  const void* cfg;
  int rowsA, GA, N, K, GB, rowsD, GD, dev;
  bool operator==(const MapKey& o) const { return std::memcmp(this, &o, sizeof(MapKey)) == 0; }
};

struct MapEntry {
  bool valid = false;
  MapKey key;
  CUtensorMap maps[3];
};

static int build_maps_cached(CUtensorMap* maps, const Config* cfg, const void* a, const void* b, void* d,
                             int rowsA, int GA, int N, int K, int GB, int rowsD, int GD, bool d_f32 = false) {
  constexpr int kSlots = 64;
  static thread_local MapEntry cache[kSlots];
  MapKey key;
  std::memset(&key, 0, sizeof(key));
  key.a = a;
  key.b = b;
  key.d = d;
  key.cfg = cfg;
  key.rowsA = rowsA;
  key.GA = GA;
  key.N = N;
  key.K = K;
  key.GB = GB;
  key.rowsD = rowsD;
  key.GD = GD;
  if (cudaGetDevice(&key.dev) != cudaSuccess) key.dev = -1;
  uint64_t h = 1469598103934665603ull;
  const unsigned char* kb = reinterpret_cast<const unsigned char*>(&key);
  for (size_t i = 0; i < sizeof(key); ++i) h = (h ^ kb[i]) * 1099511628211ull;
  MapEntry& e = cache[h % kSlots];
  if (e.valid && e.key == key) {
    std::memcpy(maps, e.maps, sizeof(e.maps));
    return DG_OK;
  }
  int r = build_maps(maps, cfg, a, b, d, rowsA, GA, N, K, GB, rowsD, GD, d_f32);
  if (r) return r;
  e.valid = true;
  e.key = key;
  std::memcpy(e.maps, maps, sizeof(e.maps));
  return DG_OK;
}

// sfa is either packed UE8M0 words or, with sfa_fp32, the fp32 scales [G][rowsA][K/128] that the
// kernel's scale producer packs on the fly.
static void fill_scale_args(GemmArgs* args, const void* sfa, const int32_t* sfb, int rowsA, int N, int K,
                            int sfb_gran = 128, bool sfa_fp32 = false) {
  args->kp = (K / 128 + 3) / 4;
  args->mn4a = (rowsA + 3) / 4 * 4;
  args->sfb_gran = sfb_gran;
  args->nb4 = ((N + sfb_gran - 1) / sfb_gran + 3) / 4 * 4;
  args->sfa = sfa_fp32 ? nullptr : static_cast<const uint32_t*>(sfa);
  args->sfa_f32 = sfa_fp32 ? static_cast<const float*>(sfa) : nullptr;
  args->sfa_f32_vec = sfa_fp32 && (K / 128) % 4 == 0 && aligned16(sfa);
  args->sfb = reinterpret_cast<const uint32_t*>(sfb);
}

static int check_common(const void* a, const void* sfa, const void* b, const int32_t* sfb,
                        void* d, int N, int K, bool sfa_fp32 = false) {
  if (!a || !sfa || !b || !sfb || !d) return fail(DG_ERR_NULL, "a, sfa, b, sfb and d must be non-NULL");
  if (!aligned16(a) || !aligned16(b) || !aligned16(d) || !aligned16(sfb))
    return fail(DG_ERR_ALIGN, "a, b, sfb and d must be 16-byte aligned");
  if (sfa_fp32 ? (reinterpret_cast<uintptr_t>(sfa) & 3) != 0 : !aligned16(sfa))
    return fail(DG_ERR_ALIGN, sfa_fp32 ? "fp32 sfa must be 4-byte aligned" : "sfa must be 16-byte aligned");
  if (K <= 0 || K % 128 != 0) return fail(DG_ERR_SHAPE, "K=%d must be a positive multiple of 128", K);
  if (N <= 0 || N % 16 != 0) return fail(DG_ERR_SHAPE, "N=%d must be a positive multiple of 16", N);
  return DG_OK;
}

// Persistent grid: one CTA per SM (co-resident pairs for 2-CTA tiles), never
// more units than tiles.
static int grid_size(int sms, long long tiles, const Config* cfg) {
  const int g = usable_sms(sms);
  long long units = g / cfg->ctas;
  if (cfg->ctas == 2) units = std::min<long long>(units, max_active_pairs(cfg, sms));
  if (tiles < units) units = std::max<long long>(tiles, 1);
  return static_cast<int>(units * cfg->ctas);
}

// ------------------------------------------------------------------ pack kernel

__global__ void pack_sf_ue8m0_kernel(const float* __restrict__ sf, uint32_t* __restrict__ out,
                                     int batch, int mn, int kb, int kp, int mn4) {
  grid_dep_wait();
  grid_dep_launch();
  const long long total = static_cast<long long>(batch) * kp * mn4;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(i % mn4);
    const long long rest = i / mn4;
    const int p = static_cast<int>(rest % kp);
    const int bt = static_cast<int>(rest / kp);
    uint32_t word = 0;
    bool bad = false;
    if (m < mn) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = 4 * p + j;
        if (k >= kb) break;
        word |= ue8m0_byte_checked(__float_as_uint(sf[(static_cast<long long>(bt) * mn + m) * kb + k]), bad) << (8 * j);
      }
    }
    out[i] = word;
    if (bad) atomicOr(&g_dg_error, DG_DEVERR_BAD_SCALE);
  }
}

// The error word as last taken by take_error_kernel (one per device).
__device__ int g_dg_error_taken = 0;

// Reads and clears the error word in one atomic step, ordered after the
// stream's earlier work; bits set meanwhile by kernels on other streams stay
// in the word for the next read.
__global__ void take_error_kernel() { g_dg_error_taken = atomicExch(&g_dg_error, 0); }

}  // namespace dg

using namespace dg;

// ==================================================================== C ABI

template <int HMODE>
static int gemm_dense(const void* a, const void* sfa, const void* b, const int32_t* sfb, void* d, int M,
                      int N, int K, void* stream, bool sfa_fp32 = false) {
  int r = check_common(a, sfa, b, sfb, d, N, K, sfa_fp32);
  if (r) return r;
  if (M < 0) return fail(DG_ERR_SHAPE, "M=%d must be >= 0", M);
  if (M == 0) return DG_OK;
  if (HMODE == MODE_DENSE_MN || HMODE == MODE_DENSE_MN + 2) {
    if (M % 16 != 0) return fail(DG_ERR_SHAPE, "M=%d must be a multiple of 16 when A is stored K x M", M);
  }
  DeviceInfo di;
  if ((r = device_info(&di))) return r;
  const Config* cfg = choose_config<HMODE>(M, N, K, usable_sms(di.sms));
  if (!cfg) return fail(DG_ERR_UNSUPPORTED, "no built configuration");
  CUtensorMap maps[3];
  if ((r = build_maps_cached(maps, cfg, a, b, d, M, 1, N, K, 1, M, 1))) return r;
  GemmArgs args = {};
  args.rows = M;
  args.N = N;
  args.K = K;
  args.G = 1;
  args.num_m_blocks = (M + 128 * cfg->ctas - 1) / (128 * cfg->ctas);
  args.num_n_blocks = (N + cfg->bn - 1) / cfg->bn;
  args.raster_m = raster_group(args.num_m_blocks);
  args.d = static_cast<__nv_bfloat16*>(d);
  fill_scale_args(&args, sfa, sfb, M, N, K, 128, sfa_fp32);
  const long long tiles = static_cast<long long>(args.num_m_blocks) * args.num_n_blocks;
  return launch<HMODE>(cfg, grid_size(di.sms, tiles, cfg), maps, args, static_cast<cudaStream_t>(stream));
}

extern "C" {

int dg_get_mk_alignment_for_contiguous_layout(void) { return 128; }

int64_t dg_packed_sf_words(int mn, int kb) {
  if (mn < 0 || kb < 0) return -1;
  return static_cast<int64_t>((kb + 3) / 4) * ((static_cast<int64_t>(mn) + 3) / 4 * 4);
}

const char* dg_get_last_error(void) { return t_last_error; }

int dg_set_num_sms(int n) {
  return g_num_sms_override.exchange(n > 0 ? n : 0);
}

int dg_set_pdl(int enable) { return g_pdl.exchange(enable ? 1 : 0); }

int dg_set_tc_util(int percent) {
  if (percent < 1 || percent > 100) return fail(DG_ERR_SHAPE, "percent=%d must be in [1, 100]", percent);
  return g_tc_util.exchange(percent);
}

int dg_get_num_sms(void) {
  DeviceInfo di;
  const int o = g_num_sms_override.load(std::memory_order_relaxed);
  if (device_info(&di) != DG_OK) return o;
  return o > 0 ? std::min(o, di.sms) : di.sms;
}

int dg_set_config(int block_n, int ctas, int pipes) {
  if (block_n == 0) {
    t_force_bn = 0;
    t_force_ctas = 0;
    t_force_pipes = 0;
    return DG_OK;
  }
  if (ctas < 0 || ctas > 2) return fail(DG_ERR_UNSUPPORTED, "ctas=%d must be 0, 1 or 2", ctas);
  if (pipes < 0 || pipes > 2) return fail(DG_ERR_UNSUPPORTED, "pipes=%d must be 0, 1 or 2", pipes);
  if (!find_config<MODE_DENSE>(block_n, ctas, pipes) && !find_config<MODE_CONTIG>(block_n, ctas, pipes) &&
      !find_config<MODE_MASKED>(block_n, ctas, pipes) && !find_config<MODE_DENSE_F32>(block_n, ctas, pipes) &&
      !find_config<MODE_DENSE_MN>(block_n, ctas, pipes) && !find_config<MODE_DENSE_MN + 1>(block_n, ctas, pipes) &&
      !find_config<MODE_DENSE_MN + 2>(block_n, ctas, pipes))
    return fail(DG_ERR_UNSUPPORTED, "block_n=%d with ctas=%d, pipes=%d is not built", block_n, ctas, pipes);
  t_force_bn = block_n;
  t_force_ctas = ctas;
  t_force_pipes = pipes;
  return DG_OK;
}

int dg_describe_config(int kind, int M, int N, int K, int num_groups, char* buf, int buflen) {
  if (!buf || buflen <= 0) return fail(DG_ERR_NULL, "buf must be non-NULL");
  DeviceInfo di;
  int sms = 148;
  if (device_info(&di) == DG_OK) sms = di.sms;
  const int device_sms = sms;
  sms = usable_sms(sms);
  if (N <= 0 || K <= 0) return fail(DG_ERR_SHAPE, "N and K must be positive");
  const Config* c = nullptr;
  long long tiles = 0;
  if (kind == 2) {
    const long long est = std::max<long long>(1, static_cast<long long>(num_groups) * M / 2);
    c = choose_config<MODE_MASKED>(est, N, K, sms, num_groups, M);
    if (c) tiles = static_cast<long long>(num_groups) * ((M + 128 * c->ctas - 1) / (128 * c->ctas)) * ((N + c->bn - 1) / c->bn);
  } else {
    c = kind == 1 ? choose_config<MODE_CONTIG>(M, N, K, sms, num_groups) : choose_config<MODE_DENSE>(M, N, K, sms);
    if (c) tiles = static_cast<long long>((M + 128 * c->ctas - 1) / (128 * c->ctas)) * ((N + c->bn - 1) / c->bn);
  }
  if (!c) return fail(DG_ERR_UNSUPPORTED, "no configuration");
  snprintf(buf, buflen, "%dx%dx%d%s%s%s%s/%d", 128 * c->ctas, c->bn, c->stages, c->ctas == 2 ? "(2cta)" : "",
           c->pipes == 2 ? "(2pipe)" : "", c->splitk ? "(splitk)" : "", c->a_rows == 64 ? "(a64)" : "",
           grid_size(device_sms, tiles, c));
  return DG_OK;
}

int dg_get_device_error(void* stream, int* err) {
  if (!err) return fail(DG_ERR_NULL, "err must be non-NULL");
  // one reader at a time per process: the taken copy is a single word per device
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  auto st = static_cast<cudaStream_t>(stream);
  // a plain launch (no programmatic serialisation): it starts after the stream's earlier kernels end
  take_error_kernel<<<1, 1, 0, st>>>();
  DG_CUDA_TRY(cudaGetLastError());
  int v = 0;
  DG_CUDA_TRY(cudaMemcpyFromSymbolAsync(&v, g_dg_error_taken, sizeof(int), 0, cudaMemcpyDeviceToHost, st));
  DG_CUDA_TRY(cudaStreamSynchronize(st));
  *err = v;
  return DG_OK;
}

uint64_t dg_set_wait_limit_ns(uint64_t ns) { return g_wait_limit_ns.exchange(ns); }

int dg_pack_sf_ue8m0(const float* sf, int32_t* packed, int batch, int mn, int kb, void* stream) {
  if (!sf || !packed) return fail(DG_ERR_NULL, "sf and packed must be non-NULL");
  if (batch < 0 || mn < 0 || kb < 0) return fail(DG_ERR_SHAPE, "negative size");
  if (!aligned16(packed)) return fail(DG_ERR_ALIGN, "packed must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(sf) & 3) != 0) return fail(DG_ERR_ALIGN, "sf must be 4-byte aligned");
  const int kp = (kb + 3) / 4;
  const int mn4 = (mn + 3) / 4 * 4;
  const long long total = static_cast<long long>(batch) * kp * mn4;
  if (total == 0) return DG_OK;
  DeviceInfo di;
  int r = device_info(&di);
  if (r) return r;
  const int threads = 256;
  const long long blocks = std::min<long long>((total + threads - 1) / threads, 8LL * di.sms);
  DG_CUDA_TRY(launch_plain(pack_sf_ue8m0_kernel, blocks, threads, static_cast<cudaStream_t>(stream), sf,
                           reinterpret_cast<uint32_t*>(packed), batch, mn, kb, kp, mn4));
  return DG_OK;
}

int dg_quantize_fp8_1x128(const void* x, int x_dtype, void* q, int32_t* sf, int batch, int M, int K,
                          void* stream) {
  if (!x || !q || !sf) return fail(DG_ERR_NULL, "x, q and sf must be non-NULL");
  if (x_dtype != 0 && x_dtype != 1) return fail(DG_ERR_UNSUPPORTED, "x_dtype=%d (0: bf16, 1: fp32)", x_dtype);
  if (!aligned16(x) || !aligned16(q) || !aligned16(sf)) return fail(DG_ERR_ALIGN, "x, q and sf must be 16-byte aligned");
  if (K <= 0 || K % 128 != 0) return fail(DG_ERR_SHAPE, "K=%d must be a positive multiple of 128", K);
  if (M < 0 || batch < 0) return fail(DG_ERR_SHAPE, "negative size");
  const int kp = (K / 128 + 3) / 4;
  const int mn4 = (M + 3) / 4 * 4;
  const long long units = static_cast<long long>(batch) * mn4 * kp;
  if (units == 0) return DG_OK;
  DeviceInfo di;
  int r = device_info(&di);
  if (r) return r;
  const int threads = 256;
  const long long blocks = std::min<long long>((units + 7) / 8, 32LL * di.sms);
  auto st = static_cast<cudaStream_t>(stream);
  if (x_dtype == 0)
    DG_CUDA_TRY(launch_plain(quantize_1x128_kernel<__nv_bfloat16>, blocks, threads, st,
                             static_cast<const __nv_bfloat16*>(x), static_cast<uint8_t*>(q),
                             reinterpret_cast<uint32_t*>(sf), batch, M, K, kp, mn4));
  else
    DG_CUDA_TRY(launch_plain(quantize_1x128_kernel<float>, blocks, threads, st, static_cast<const float*>(x),
                             static_cast<uint8_t*>(q), reinterpret_cast<uint32_t*>(sf), batch, M, K, kp, mn4));
  return DG_OK;
}

int dg_moe_permute_capacity(int T, int topk, int num_experts) {
  if (T < 0 || topk <= 0 || num_experts <= 0) return fail(DG_ERR_SHAPE, "bad sizes");
  const long long rows = static_cast<long long>(T) * topk + 127LL * num_experts;
  const long long cap = (rows + 127) / 128 * 128;
  if (cap > 0x7FFFFFFFLL) return fail(DG_ERR_SHAPE, "capacity overflows int");
  return static_cast<int>(cap);
}

int dg_moe_permute(const int32_t* topk_ids, int T, int topk, int num_experts, const void* q, const int32_t* sfa, int K,
                   void* a_perm, int32_t* sfa_perm, int32_t* m_indices, int32_t* row_of, int32_t* src_of, int M_cap,
                   void* stream) {
  if (!a_perm || !sfa_perm || !m_indices || !src_of || (T != 0 && (!topk_ids || !q || !sfa || !row_of)))
    return fail(DG_ERR_NULL, "every pointer must be non-NULL (topk_ids, q, sfa and row_of may be NULL when T = 0)");
  if (!aligned16(q) || !aligned16(a_perm) || !aligned16(sfa) || !aligned16(sfa_perm))
    return fail(DG_ERR_ALIGN, "q, sfa, a_perm and sfa_perm must be 16-byte aligned");
  if (T < 0 || topk <= 0 || num_experts <= 0 || num_experts > kMoeMaxExperts)
    return fail(DG_ERR_SHAPE, "T=%d topk=%d num_experts=%d (at most %d experts)", T, topk, num_experts, kMoeMaxExperts);
  if (K <= 0 || K % 128 != 0) return fail(DG_ERR_SHAPE, "K=%d must be a positive multiple of 128", K);
  const int cap = dg_moe_permute_capacity(T, topk, num_experts);
  if (cap < 0) return cap;
  if (M_cap < cap || M_cap % 128 != 0)
    return fail(DG_ERR_SHAPE, "M_cap=%d must be a multiple of 128 and >= %d (dg_moe_permute_capacity)", M_cap, cap);
  const long long n = static_cast<long long>(T) * topk;
  if (n > 0x7FFFFFFFLL) return fail(DG_ERR_SHAPE, "too many routed slots");
  DeviceInfo di;
  int r = device_info(&di);
  if (r) return r;
  auto st = static_cast<cudaStream_t>(stream);
  const int kp = (K / 128 + 3) / 4;
  // the routing kernel: one cluster; its table needs more than 48 KB of shared memory beyond 320 experts
  {
    static std::mutex mu;
    static bool attr_done[64] = {};
    int dev = 0;
    DG_CUDA_TRY(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return fail(DG_ERR_UNSUPPORTED, "device %d outside the launch table", dev);
    if (!attr_done[dev]) {
      DG_CUDA_TRY(cudaFuncSetAttribute(reinterpret_cast<const void*>(&moe_route_kernel),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, route_smem_bytes(kMoeMaxExperts)));
      attr_done[dev] = true;
    }
  }
  DG_CUDA_TRY(launch_plain_smem(moe_route_kernel, kRouteCluster, kMoeThreads,
                                static_cast<size_t>(route_smem_bytes(num_experts)), st, kRouteCluster, topk_ids,
                                static_cast<int>(n), num_experts, M_cap, kp, m_indices, row_of, src_of,
                                reinterpret_cast<uint32_t*>(sfa_perm)));
  const long long work = static_cast<long long>(T) * (K / 16);
  if (work == 0) return DG_OK;
  const long long blocks =
      std::max<long long>(1, std::min<long long>((work + 256 * kGatherU - 1) / (256 * kGatherU), 8LL * di.sms));
  DG_CUDA_TRY(launch_plain(moe_gather_kernel, blocks, 256, st, static_cast<const uint8_t*>(q),
                           reinterpret_cast<const uint32_t*>(sfa), T, K, kp, topk, topk_ids,
                           static_cast<const int32_t*>(row_of), M_cap, static_cast<uint8_t*>(a_perm),
                           reinterpret_cast<uint32_t*>(sfa_perm), m_indices, src_of));
  return DG_OK;
}

int dg_moe_unpermute_combine(const void* d_perm, const int32_t* row_of, const float* weights, int T, int topk, int N,
                             void* out, void* stream) {
  if (!d_perm || !row_of || !out) return fail(DG_ERR_NULL, "d_perm, row_of and out must be non-NULL");
  if (!aligned16(d_perm) || !aligned16(out)) return fail(DG_ERR_ALIGN, "d_perm and out must be 16-byte aligned");
  if (T < 0 || topk <= 0 || N <= 0 || N % 16 != 0) return fail(DG_ERR_SHAPE, "T=%d topk=%d N=%d", T, topk, N);
  const long long work = static_cast<long long>(T) * (N / 8);
  if (work == 0) return DG_OK;
  DeviceInfo di;
  int r = device_info(&di);
  if (r) return r;
  // slots per pass: one at a time up to top-4, else 8 (passes of 8 beyond top-8); measured
  // fastest on top-2 and top-4 (N = 4096) and on top-8 (N = 7168) respectively
  const int slots = topk <= 4 ? 1 : 8;
  const long long blocks = std::max<long long>(1, std::min<long long>((work + 255) / 256, 16LL * di.sms));
  auto st = static_cast<cudaStream_t>(stream);
  auto dp = static_cast<const __nv_bfloat16*>(d_perm);
  auto op = static_cast<__nv_bfloat16*>(out);
  if (slots == 1) DG_CUDA_TRY(launch_plain(moe_combine_kernel<1>, blocks, 256, st, dp, row_of, weights, T, topk, N, op));
  else DG_CUDA_TRY(launch_plain(moe_combine_kernel<8>, blocks, 256, st, dp, row_of, weights, T, topk, N, op));
  return DG_OK;
}

int dg_fp8_gemm_nt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d,
                   int M, int N, int K, void* stream) {
  return gemm_dense<MODE_DENSE>(a, sfa, b, sfb, d, M, N, K, stream);
}

int dg_fp8_gemm_nt_fp32sfa(const void* a, const float* sfa, const void* b, const int32_t* sfb, void* d,
                           int M, int N, int K, void* stream) {
  return gemm_dense<MODE_DENSE>(a, sfa, b, sfb, d, M, N, K, stream, true);
}

int dg_fp8_gemm_nn(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d,
                   int M, int N, int K, void* stream) {
  return gemm_dense<MODE_DENSE_MN + 1>(a, sfa, b, sfb, d, M, N, K, stream);
}

int dg_fp8_gemm_tn(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d,
                   int M, int N, int K, void* stream) {
  return gemm_dense<MODE_DENSE_MN + 2>(a, sfa, b, sfb, d, M, N, K, stream);
}

int dg_fp8_gemm_tt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d,
                   int M, int N, int K, void* stream) {
  return gemm_dense<MODE_DENSE_MN>(a, sfa, b, sfb, d, M, N, K, stream);
}

int dg_fp8_gemm_nt_ex(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, const float* c,
                      void* d, int M, int N, int K, int sfb_gran_n, int d_is_fp32, void* stream) {
  int r = check_common(a, sfa, b, sfb, d, N, K);
  if (r) return r;
  if (sfb_gran_n != 1 && sfb_gran_n != 128)
    return fail(DG_ERR_UNSUPPORTED, "sfb_gran_n=%d must be 1 (per-row B scales) or 128 (128x128 blocks)", sfb_gran_n);
  if (d_is_fp32 != 0 && d_is_fp32 != 1) return fail(DG_ERR_UNSUPPORTED, "d_is_fp32=%d must be 0 or 1", d_is_fp32);
  if (c && !d_is_fp32) return fail(DG_ERR_UNSUPPORTED, "accumulating into c needs an FP32 d");
  if (c && !aligned16(c)) return fail(DG_ERR_ALIGN, "c must be 16-byte aligned");
  if (M < 0) return fail(DG_ERR_SHAPE, "M=%d must be >= 0", M);
  if (M == 0) return DG_OK;
  DeviceInfo di;
  if ((r = device_info(&di))) return r;
  const Config* cfg = d_is_fp32 ? choose_config<MODE_DENSE_F32>(M, N, K, usable_sms(di.sms)) : choose_config<MODE_DENSE>(M, N, K, usable_sms(di.sms));
  if (!cfg && d_is_fp32) cfg = find_config<MODE_DENSE_F32>(224, 1);  // forced 2-CTA configs have no FP32 form
  if (!cfg) return fail(DG_ERR_UNSUPPORTED, "no built configuration");
  CUtensorMap maps[3];
  if ((r = build_maps_cached(maps, cfg, a, b, d, M, 1, N, K, 1, M, 1, d_is_fp32 != 0))) return r;
  GemmArgs args = {};
  args.rows = M;
  args.N = N;
  args.K = K;
  args.G = 1;
  args.num_m_blocks = (M + 128 * cfg->ctas - 1) / (128 * cfg->ctas);
  args.num_n_blocks = (N + cfg->bn - 1) / cfg->bn;
  args.raster_m = raster_group(args.num_m_blocks);
  if (d_is_fp32) args.d32 = static_cast<float*>(d);
  else args.d = static_cast<__nv_bfloat16*>(d);
  args.c = c;
  fill_scale_args(&args, sfa, sfb, M, N, K, sfb_gran_n);
  const long long tiles = static_cast<long long>(args.num_m_blocks) * args.num_n_blocks;
  if (d_is_fp32)
    return launch<MODE_DENSE_F32>(cfg, grid_size(di.sms, tiles, cfg), maps, args, static_cast<cudaStream_t>(stream));
  return launch<MODE_DENSE>(cfg, grid_size(di.sms, tiles, cfg), maps, args, static_cast<cudaStream_t>(stream));
}

static int contiguous_impl(const void* a, const void* sfa, const void* b, const int32_t* sfb, void* d,
                           const int32_t* m_indices, int M_total, int N, int K, int num_groups, void* stream,
                           bool sfa_fp32) {
  int r = check_common(a, sfa, b, sfb, d, N, K, sfa_fp32);
  if (r) return r;
  if (!m_indices) return fail(DG_ERR_NULL, "m_indices must be non-NULL");
  if (num_groups <= 0) return fail(DG_ERR_SHAPE, "num_groups=%d must be positive", num_groups);
  if (M_total < 0 || M_total % 128 != 0)
    return fail(DG_ERR_SHAPE, "M_total=%d must be a non-negative multiple of %d", M_total, 128);
  if (M_total == 0) return DG_OK;
  DeviceInfo di;
  if ((r = device_info(&di))) return r;
  const Config* cfg = choose_config<MODE_CONTIG>(M_total, N, K, usable_sms(di.sms), num_groups);
  if (!cfg) return fail(DG_ERR_UNSUPPORTED, "no built configuration");
  CUtensorMap maps[3];
  if ((r = build_maps_cached(maps, cfg, a, b, d, M_total, 1, N, K, num_groups, M_total, 1))) return r;
  GemmArgs args = {};
  args.rows = M_total;
  args.N = N;
  args.K = K;
  args.G = num_groups;
  // 128-row blocks (1-CTA tiles) or an estimate of the pairs (2-CTA tiles: the kernel pairs blocks itself)
  args.num_m_blocks = (M_total + 128 * cfg->ctas - 1) / (128 * cfg->ctas);
  args.num_n_blocks = (N + cfg->bn - 1) / cfg->bn;
  args.raster_m = raster_group(args.num_m_blocks);
  args.m_indices = m_indices;
  args.d = static_cast<__nv_bfloat16*>(d);
  fill_scale_args(&args, sfa, sfb, M_total, N, K, 128, sfa_fp32);
  const long long tiles = static_cast<long long>(args.num_m_blocks) * args.num_n_blocks;
  return launch<MODE_CONTIG>(cfg, grid_size(di.sms, tiles, cfg), maps, args,
                             static_cast<cudaStream_t>(stream));
}

int dg_m_grouped_fp8_gemm_nt_contiguous(const void* a, const int32_t* sfa, const void* b,
                                        const int32_t* sfb, void* d, const int32_t* m_indices,
                                        int M_total, int N, int K, int num_groups, void* stream) {
  return contiguous_impl(a, sfa, b, sfb, d, m_indices, M_total, N, K, num_groups, stream, false);
}

int dg_m_grouped_fp8_gemm_nt_contiguous_fp32sfa(const void* a, const float* sfa, const void* b,
                                                const int32_t* sfb, void* d, const int32_t* m_indices,
                                                int M_total, int N, int K, int num_groups, void* stream) {
  return contiguous_impl(a, sfa, b, sfb, d, m_indices, M_total, N, K, num_groups, stream, true);
}

static int masked_impl(const void* a, const void* sfa, const void* b, const int32_t* sfb, void* d,
                       const int32_t* masked_m, int num_groups, int M_max, int N, int K, void* stream,
                       bool sfa_fp32) {
  int r = check_common(a, sfa, b, sfb, d, N, K, sfa_fp32);
  if (r) return r;
  if (!masked_m) return fail(DG_ERR_NULL, "masked_m must be non-NULL");
  if (num_groups <= 0 || num_groups > kMaxMaskedGroups)
    return fail(DG_ERR_SHAPE, "num_groups=%d must be in [1, %d]", num_groups, kMaxMaskedGroups);
  if (M_max < 0) return fail(DG_ERR_SHAPE, "M_max=%d must be >= 0", M_max);
  if (M_max == 0) return DG_OK;
  DeviceInfo di;
  if ((r = device_info(&di))) return r;
  // the device decides the real tile count; the heuristic assumes half-full experts
  const long long rows_est = std::max<long long>(1, static_cast<long long>(num_groups) * M_max / 2);
  const Config* cfg = choose_config<MODE_MASKED>(rows_est, N, K, usable_sms(di.sms), num_groups, M_max);
  if (!cfg) return fail(DG_ERR_UNSUPPORTED, "no built configuration");
  CUtensorMap maps[3];
  if ((r = build_maps_cached(maps, cfg, a, b, d, M_max, num_groups, N, K, num_groups, M_max, num_groups)))
    return r;
  GemmArgs args = {};
  args.rows = M_max;
  args.N = N;
  args.K = K;
  args.G = num_groups;
  args.num_m_blocks = (M_max + 128 * cfg->ctas - 1) / (128 * cfg->ctas);
  args.num_n_blocks = (N + cfg->bn - 1) / cfg->bn;
  args.raster_m = 1;
  args.masked_m = masked_m;
  args.d = static_cast<__nv_bfloat16*>(d);
  fill_scale_args(&args, sfa, sfb, M_max, N, K, 128, sfa_fp32);
  const long long max_tiles = static_cast<long long>(num_groups) * args.num_m_blocks * args.num_n_blocks;
  return launch<MODE_MASKED>(cfg, grid_size(di.sms, max_tiles, cfg), maps, args,
                             static_cast<cudaStream_t>(stream));
}

int dg_m_grouped_fp8_gemm_nt_masked(const void* a, const int32_t* sfa, const void* b,
                                    const int32_t* sfb, void* d, const int32_t* masked_m,
                                    int num_groups, int M_max, int N, int K, void* stream) {
  return masked_impl(a, sfa, b, sfb, d, masked_m, num_groups, M_max, N, K, stream, false);
}

int dg_m_grouped_fp8_gemm_nt_masked_fp32sfa(const void* a, const float* sfa, const void* b,
                                            const int32_t* sfb, void* d, const int32_t* masked_m,
                                            int num_groups, int M_max, int N, int K, void* stream) {
  return masked_impl(a, sfa, b, sfb, d, masked_m, num_groups, M_max, N, K, stream, true);
}

}  // extern "C"
