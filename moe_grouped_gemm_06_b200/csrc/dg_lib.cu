// dg_lib.cu -- host side of the C ABI declared in include/dg.h: argument
// validation, the tile/split heuristic, TMA descriptor encoding, split-K
// workspaces and kernel launches.  All device code lives in the included
// headers so that this file is the library's single translation unit.
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include "../../include/dg.h"
#include "dg_gemm.cuh"
#include "dg_prep.cuh"
#include "dg_probe.cuh"

namespace {

std::atomic<uint64_t> g_launches{0};
int g_num_sms_override = 0;
std::atomic<int> g_pdl{1};  // programmatic dependent launch on (dg_set_pdl)

// Launches a kernel on `s`, as a programmatic dependent of the previous work
// on the stream when PDL is enabled.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster,
                   Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (g_pdl.load()) {
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
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

unsigned long long timeout_ns() {
  static unsigned long long v = [] {
    const char* e = std::getenv("DG_TIMEOUT_MS");
    long long ms = e ? std::atoll(e) : 4000;
    if (ms <= 0) ms = 4000;
    return (unsigned long long)ms * 1000000ull;
  }();
  return v;
}

bool log_enabled() {
  static bool v = [] {
    const char* e = std::getenv("DG_LOG");
    return e && e[0] == '1';
  }();
  return v;
}

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms;
}

int num_sms() {
  if (g_num_sms_override > 0) return g_num_sms_override;
  return device_sms();
}

// ------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 3-D map: dims {d0 (innermost, elements), d1, d2}, strides in bytes of dims 1, 2.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
              uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------ heuristic

struct Plan {
  int bn = 128;
  long long dp_tiles = 0; // tiles computed whole (all tiles when sk_tiles = 0)
  int sk_tiles = 0;       // stream-K tiles after them (dense only)
  int max_seg = 0;        // workspace slots per stream-K tile
  int sk_split = 0;       // > 0: each stream-K tile cut into this many K-slices
  long long sk_iters = 0;
  int split = 0;          // > 0: every tile cut into this many K-slices on a cluster of as many CTAs
  int grid = 0;
  double cost = 0;        // estimated microseconds
  size_t ws_bytes() const { return (size_t)sk_tiles * max_seg * dg::kBM * bn * sizeof(float); }
};

long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }

// Per-tile time of each instantiated block width on B200, fitted to measured
// dense sweeps (M = 4096, K from 512 to 16384; microseconds at the SM clock
// under load):
//   tile = max(K-blocks x per_kb + per_tile, epilogue)
// With two or three accumulator buffers the epilogue of one tile overlaps the
// main loop of the next, so a tile costs the slower of the two; at 256
// columns the two buffers share 64 columns, so a tile's MMAs wait for the
// first quarter of the previous tile's epilogue, and the rest of the
// epilogue's cost per tile is inside per_tile (3.1 us: forced 256-wide runs
// of 4096 x 7168 x 16384 and 4096 x 32768 x 512).  Widths 160
// and 224 re-base their scale words on the MMA-issuing thread, which costs
// more than they gain; they are available through dg_set_tile_config but
// never chosen automatically.
// FP4 B (per_kb_fp4) is staged from half the bytes, which helps wide tiles,
// but every K-block needs its own scale-factor copy into TMEM ahead of its
// MMAs (1x32 scales), which costs narrow tiles.
// BF16 (per_kb_bf16, per 64-element K-block) runs a 192-wide MMA at the
// rate of its width, where e4m3 pays nearly the 256-wide cost for it.
struct WidthCost {
  int bn;
  double per_kb, per_tile, epilogue;
  bool automatic;
  double per_kb_fp4, per_kb_bf16;
};
constexpr WidthCost kWidthCosts[] = {
    {64, 0.19, 1.5, 1.6, true, 0.21, 0.13},      {128, 0.2305, 1.9, 2.94, true, 0.264, 0.213},
    {160, 0.32, 2.4, 3.6, false, 0.33, 0.26},    {192, 0.368, 1.6, 3.97, true, 0.345, 0.284},
    {224, 0.45, 3.0, 4.6, false, 0.36, 0.33},    {256, 0.4236, 3.1, 0.0, true, 0.343, 0.357},
};

// Tile-configuration override (dg_set_tile_config; initial values from the
// environment variables DG_BLOCK_N and DG_SCHEDULE): one block width, and/or
// one schedule: whole tiles (1), tail cut into per-tile K-slices (2),
// stream-K tail (3), or every tile split over a cluster of S = schedule - 2
// CTAs (4 .. 10: S = 2 .. 8).
int env_int(const char* name) {
  const char* e = std::getenv(name);
  return e ? std::atoi(e) : 0;
}
std::atomic<int> g_force_bn{env_int("DG_BLOCK_N")};
std::atomic<int> g_force_schedule{(env_int("DG_SCHEDULE") >= 1 && env_int("DG_SCHEDULE") <= 10) ? env_int("DG_SCHEDULE")
                                                                                              : 0};

int forced_block_n() {
  const int b = g_force_bn.load();
  for (const WidthCost& wc : kWidthCosts)
    if (wc.bn == b) return b;
  return 0;
}

double tile_time(const WidthCost& wc, int kb) { return std::max(kb * wc.per_kb + wc.per_tile, wc.epilogue); }

// Stream-K split of the last sk_tiles tiles over G CTAs: exact slots per
// tile (CTAs whose shares meet the tile), 0 when some share would be empty.
int sk_max_segments(int sk_tiles, int kb, int G) {
  const long long iters = (long long)sk_tiles * kb;
  if (sk_tiles <= 0 || iters < G) return 0;
  int mx = 0;
  for (int j = 0; j < sk_tiles; ++j) {
    const long long x0 = (long long)j * kb;
    mx = std::max(mx, dg::sk_cta_of(x0 + kb - 1, G, iters) - dg::sk_cta_of(x0, G, iters) + 1);
  }
  return mx;
}

// Chooses the block width and the schedule minimising the estimated time
// (microseconds; constants measured on B200):
//   whole tiles:  ceil(tiles / SMs) x tile time
//   tail split:   q full waves of whole tiles (q = the number of full waves,
//                 or one less), then the remaining r tiles shared over the
//                 SMs, either each cut into s = SMs / r equal K-slices (one
//                 piece per CTA), or as stream-K (even shares of all their
//                 K-iterations, pieces crossing tiles; at one accumulator
//                 buffer a CTA's pieces run one after the other); plus the
//                 fix-up kernel (7.5 us for slices, 9.5 us for stream-K, of
//                 launch, partial writes and reads, + the partial bytes at
//                 ~5 TB/s) and, after full waves, the HBM reads of the shared
//                 tiles' A and B rows (pieces of different K ranges do not
//                 reuse each other's tiles in L2).
// Every plan is at least the time to move the unique bytes of A, B, C and D
// through HBM (~5.5 TB/s), and at small M (at most two 128-row blocks, where
// B streams from HBM in 128-byte rows) at least the time to stream B at
// ~4 TB/s and the time one SM needs to stream its share (~63 GB/s per SM);
// among plans at the floor the one with the least estimated SM time wins.  Sharing is offered for the dense layout only
// (allow_sk) and only within ws_cap bytes of workspace (0: no cap).  Ties
// keep whole tiles.
// MN-major B (mn_b) is staged in 128-wide column blocks: widths 128 and 256.
int split_capacity(int bn, bool fp4, int cluster);

// only_bn: plan this block width alone (the promotion kernels are 128 wide).
// allow_split: the dense NT kernels may cut every tile over a cluster (below).
Plan plan_gemm(long long m_blocks, int n, int k, int sms, bool allow_sk, size_t ws_cap = 0, bool fp4 = false,
               bool bf16 = false, bool mn_b = false, int only_bn = 0, bool allow_split = false) {
  Plan best;
  best.cost = 1e300;
  const int kb = k / 128;
  const int sched = g_force_schedule.load();
  const double rows = (double)m_blocks * dg::kBM;
  const bool streams_b = m_blocks <= 2;
  const double hbm_floor = std::max((rows * k + (double)n * k + 4.0 * rows * n) / 5.5e6,
                                    streams_b ? (double)n * k / 4.0e6 : 0.0);
  for (const WidthCost& base : kWidthCosts) {
    WidthCost wc = base;
    if (fp4) wc.per_kb = wc.per_kb_fp4;
    if (bf16) wc.per_kb = wc.per_kb_bf16;
    const int bn = wc.bn;
    if (only_bn != 0) {
      if (bn != only_bn) continue;
    } else if (forced_block_n() ? bn != forced_block_n() : !wc.automatic) {
      continue;
    }
    if (mn_b && bn % 128 != 0) continue;
    // 64-wide tiles double the CTAs of a dense problem of at most two
    // m-blocks; elsewhere (and for the grouped layouts) they only add A reads
    if (bn == 64 && !forced_block_n() && !(streams_b && allow_sk)) continue;
    const long long tiles = m_blocks * ceil_div(n, bn);
    auto consider = [&](const Plan& p) {
      if (p.cost < best.cost * (1 - 1e-9)) best = p;
    };
    // time for one CTA to stream kbs K-blocks of B from HBM (small M only)
    auto stream_b = [&](long long kbs) { return streams_b ? (double)kbs * bn * 128.0 / 6.3e4 : 0.0; };
    Plan dp;
    dp.bn = bn;
    dp.dp_tiles = tiles;
    dp.grid = (int)std::max<long long>(1, std::min<long long>(tiles, sms));
    const long long waves = ceil_div(tiles, sms);
    // at the floor, the plan with less work on the SMs wins (5% of it counts)
    auto floored = [&](double t) { return std::max(t, hbm_floor) + 0.05 * t; };
    dp.cost = floored(std::max((double)waves * tile_time(wc, kb), waves * stream_b(kb))) * (sched >= 2 ? 1e6 : 1.0);
    consider(dp);
    // (c) every tile's K-blocks cut into S slices computed by the S CTAs of a
    // cluster, their sums added through distributed shared memory: no
    // workspace and no fix-up kernel, for problems with few tiles.  The cost
    // of the sum is the DSMEM reads of one band (kBM / S rows of S slices).
    if (allow_split && (bn == 128 || bn == 256) && (sched == 0 || sched >= 4)) {
      for (int sp = 2; sp <= 8; ++sp) {
        if ((sched >= 4 && sp != sched - 2) || kb < sp) continue;
        const int cap = split_capacity(bn, fp4, sp);  // clusters the GPU holds at once
        if (cap <= 0) continue;
        const long long kbs = ceil_div(kb, sp);
        const double piece = std::max(kbs * wc.per_kb + wc.per_tile, stream_b(kbs));
        const double reduce = 0.8 + 512.0 * bn / 1.2e5;
        Plan pc;
        pc.bn = bn;
        pc.dp_tiles = tiles;
        pc.split = sp;
        pc.grid = (int)(tiles * sp);
        pc.cost = floored((double)ceil_div(tiles, cap) * (piece + reduce));
        consider(pc);
      }
    }
    if (!allow_sk || sched == 1 || sched >= 4) continue;
    const long long full_waves = tiles / sms;
    for (long long q = full_waves; q >= std::max(0LL, full_waves - 1); --q) {
      const long long sk = tiles - q * sms;
      // (the fix-up kernel indexes a shared tile's elements with 32-bit ints)
      if (sk <= 0 || sk > 4 * (long long)sms || sk * dg::kBM * (bn / 4) >= (1LL << 31)) continue;
      const double shared_reads = q > 0 ? (double)sk * (dg::kBM + bn) * k / 6e6 : 0.0;
      Plan p;
      p.bn = bn;
      p.dp_tiles = q * sms;
      p.sk_tiles = (int)sk;
      // (a) each remaining tile cut into s K-slices
      const long long s_split = std::min<long long>(sms / sk, kb);
      if (s_split >= 2 && sched != 3) {
        Plan ps = p;
        ps.sk_split = (int)s_split;
        ps.max_seg = (int)s_split;
        ps.grid = (int)(q > 0 ? sms : sk * s_split);
        const long long kbs = ceil_div(kb, s_split);
        const double piece = std::max(tile_time(wc, (int)kbs), stream_b(kbs)) + shared_reads;
        const double fixup = 7.5 + (double)sk * s_split * dg::kBM * bn * 4.0 / 5e6;
        ps.cost = floored((double)q * tile_time(wc, kb) + piece + fixup);
        if (ws_cap == 0 || ps.ws_bytes() <= ws_cap) consider(ps);
      }
      // (b) stream-K over all SMs
      if (sched == 2) continue;
      const long long iters = sk * kb;
      const int G = (int)std::min<long long>(sms, iters);
      if (G < 2 || (q > 0 && G != sms)) continue;
      const int max_seg = sk_max_segments((int)sk, kb, G);
      if (max_seg == 0 || max_seg > 64) continue;
      p.max_seg = max_seg;
      p.sk_iters = iters;
      p.grid = G;
      if (ws_cap != 0 && p.ws_bytes() > ws_cap) continue;
      const long long share = ceil_div(iters, G);
      const long long pieces = std::min<long long>(share, ceil_div(share, kb) + 1);
      const double compute = (wc.epilogue > 0.0)
                                 ? std::max(share * wc.per_kb + pieces * wc.per_tile, pieces * wc.epilogue)
                                 : share * wc.per_kb + pieces * wc.per_tile;
      const double piece = std::max(compute, stream_b(share)) + shared_reads;
      const double fixup = 9.5 + (double)(sk + G) * dg::kBM * bn * 4.0 / 5e6;
      p.cost = floored((double)q * tile_time(wc, kb) + piece + fixup);
      consider(p);
    }
  }
  return best;
}

// ------------------------------------------------------------ workspaces

struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};
std::mutex g_ws_mutex;
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;

// Stream-K partial sums of this (device, stream), allocated stream-ordered on
// first use and grown on demand.
float* workspace(size_t bytes, cudaStream_t s) {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(g_ws_mutex);
  Workspace& w = g_ws[{dev, s}];
  if (w.bytes < bytes) {
    if (w.ptr) cudaFreeAsync(w.ptr, s);
    w.ptr = nullptr;
    w.bytes = 0;
    if (cudaMallocAsync(&w.ptr, bytes, s) != cudaSuccess) return nullptr;
    w.bytes = bytes;
  }
  return static_cast<float*>(w.ptr);
}

// ------------------------------------------------------------ launches

// The tensor maps of one call: A (128-row and 32-row boxes), B, D, and C in
// D's boxes (for L2 prefetches of the next tile's C; a copy of D's map when
// there is no C).
struct Maps {
  CUtensorMap a, a32, b, d, c;
};

template <int BN, bool FP4, int LAYOUT, int EPI = dg::kEpiPlain, bool BF16 = false, int MAJ = dg::kMajorK>
dg_status launch_gemm(const Maps& mp,
                      const dg::GemmArgs& args, int grid, cudaStream_t s, int cluster = 1) {
  using C = dg::Cfg<BN, FP4, BF16, (LAYOUT == dg::kMasked || LAYOUT == dg::kKGrouped), EPI == dg::kEpiPromote>;
  auto kern = dg::gemm_kernel<BN, FP4, LAYOUT, EPI, BF16, MAJ>;
  static std::atomic<uint64_t> attr_set_mask{0};  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_set_mask.load() & bit)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
      return DG_ERR_CUDA;
    attr_set_mask.fetch_or(bit);
  }
  if (launch(kern, dim3(grid), dim3(dg::block_threads<BN, BF16>()), C::kSmemBytes, s, cluster, mp.a, mp.a32, mp.b, mp.d,
             mp.c, args) !=
      cudaSuccess)
    return DG_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return DG_OK;
}

// Clusters of `cluster` CTAs of the split kernel (block width bn) that the
// current device can hold at once (cudaOccupancyMaxActiveClusters), cached
// per device; 0 when the query fails.
template <int BN, bool FP4>
int split_capacity_of(int cluster) {
  using C = dg::Cfg<BN, FP4, false, false>;
  auto kern = dg::gemm_kernel<BN, FP4, dg::kDenseSplit>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cluster);
  cfg.blockDim = dim3(dg::block_threads<BN, false>());
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = cluster;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

int split_capacity(int bn, bool fp4, int cluster) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const auto key = std::make_tuple(dev, bn, (int)fp4, cluster);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int n = 0;
  if (bn == 128) n = fp4 ? split_capacity_of<128, true>(cluster) : split_capacity_of<128, false>(cluster);
  if (bn == 256) n = fp4 ? split_capacity_of<256, true>(cluster) : split_capacity_of<256, false>(cluster);
  cache[key] = n;
  return n;
}

template <bool FP4>
dg_status dispatch_split(int bn, int split, const Maps& mp, const dg::GemmArgs& args, int grid, cudaStream_t s) {
  switch (bn) {
    case 128: return launch_gemm<128, FP4, dg::kDenseSplit>(mp, args, grid, s, split);
    case 256: return launch_gemm<256, FP4, dg::kDenseSplit>(mp, args, grid, s, split);
    default: return DG_ERR_UNSUPPORTED;
  }
}

template <bool FP4, int LAYOUT, int EPI = dg::kEpiPlain, bool BF16 = false, int MAJ = dg::kMajorK>
dg_status dispatch(int bn, const Maps& mp, const dg::GemmArgs& args, int grid, cudaStream_t s) {
  if constexpr (MAJ != dg::kMajorK) {
    // MN-major operands: FP8, plain epilogue, 128-wide column blocks
    static_assert(!FP4 && !BF16 && EPI == dg::kEpiPlain, "MN-major: FP8, plain epilogue");
    switch (bn) {
      case 128: return launch_gemm<128, false, LAYOUT, EPI, false, MAJ>(mp, args, grid, s);
      case 256: return launch_gemm<256, false, LAYOUT, EPI, false, MAJ>(mp, args, grid, s);
      default: return DG_ERR_UNSUPPORTED;
    }
  } else if constexpr (LAYOUT == dg::kKGrouped) {
    return DG_ERR_UNSUPPORTED;  // (k-grouped is MN-major only)
  } else if constexpr (BF16) {
    // bf16: dense tiles of the widths the heuristic picks
    switch (bn) {
      case 64: return launch_gemm<64, false, LAYOUT, EPI, true>(mp, args, grid, s);
      case 128: return launch_gemm<128, false, LAYOUT, EPI, true>(mp, args, grid, s);
      case 192: return launch_gemm<192, false, LAYOUT, EPI, true>(mp, args, grid, s);
      case 256: return launch_gemm<256, false, LAYOUT, EPI, true>(mp, args, grid, s);
      default: return DG_ERR_UNSUPPORTED;
    }
  } else if constexpr (EPI == dg::kEpiPromote) {
    // per-K-block promotion: e4m3 A and B, 128-wide tiles
    static_assert(!FP4 && LAYOUT == dg::kDense, "promotion: dense e4m3");
    if (bn != 128) return DG_ERR_UNSUPPORTED;
    return launch_gemm<128, false, LAYOUT, EPI>(mp, args, grid, s);
  } else if constexpr (EPI == dg::kEpiSwiGlu) {
    // SwiGLU tiles hold whole (64 gate, 64 up) row blocks: widths 128, 256
    switch (bn) {
      case 128: return launch_gemm<128, FP4, LAYOUT, EPI>(mp, args, grid, s);
      case 256: return launch_gemm<256, FP4, LAYOUT, EPI>(mp, args, grid, s);
      default: return DG_ERR_UNSUPPORTED;
    }
  } else {
    switch (bn) {
      case 64: return launch_gemm<64, FP4, LAYOUT>(mp, args, grid, s);
      case 128: return launch_gemm<128, FP4, LAYOUT>(mp, args, grid, s);
      case 160: return launch_gemm<160, FP4, LAYOUT>(mp, args, grid, s);
      case 192: return launch_gemm<192, FP4, LAYOUT>(mp, args, grid, s);
      case 224: return launch_gemm<224, FP4, LAYOUT>(mp, args, grid, s);
      case 256: return launch_gemm<256, FP4, LAYOUT>(mp, args, grid, s);
      default: return DG_ERR_UNSUPPORTED;
    }
  }
}

struct Problem {
  const void* a;
  const int32_t* sfa;
  const void* b;
  const int32_t* sfb;
  const void* c;
  void* d;
  const int32_t* m_indices;
  const int32_t* masked_m;
  int rows;        // dense m, contiguous m_total, masked max_m
  int n, k;
  int groups;      // 1 for dense
  int expected_m;  // masked hint
  const int32_t* ks = nullptr;  // k-grouped: K of each group (device)
};

// mean K of a k-grouped call's groups (the planner's K), at least one block
int k_plan_mn(const Problem& p) { return std::max(128, (int)(p.k / p.groups) / 128 * 128); }

// fixed_ws / fixed_ws_bytes: when given, stream-K partials go to this
// caller-provided device buffer instead of the per-stream workspace, and the
// planner only considers plans that fit in fixed_ws_bytes (whole tiles
// always do).
// The plan a call of this layout and operand kind runs (block width, schedule,
// grid), as run_gemm launches it; dg_query_config reports it.
Plan select_plan(const Problem& p, int layout, bool fp4, bool bf16, bool mn, bool swiglu, int sms,
                 size_t ws_cap, bool promote = false) {
  // a bf16 stage covers 64 K-elements in the time an e4m3 stage covers 128:
  // the planner sees bf16 as an e4m3 problem of twice the K
  const int k_plan = bf16 ? 2 * p.k : p.k;
  const long long m_blocks = ceil_div(p.rows, dg::kBM);
  Plan plan;
  if (layout == dg::kMasked) {
    const int em = p.expected_m > 0 ? std::min(p.expected_m, p.rows) : p.rows;
    plan = plan_gemm((long long)p.groups * ceil_div(em, dg::kBM), p.n, p.k, sms, false);
    if (swiglu && plan.bn != 128 && plan.bn != 256 && !forced_block_n())
      plan.bn = plan.bn > 192 ? 256 : 128;  // SwiGLU tiles hold whole gate/up block pairs
    plan.grid = (int)std::min<long long>((long long)p.groups * m_blocks * ceil_div(p.n, plan.bn), sms);
  } else if (layout == dg::kKGrouped) {
    // every group has the same tiles; planned at the mean K of a group
    plan = plan_gemm((long long)p.groups * m_blocks, p.n, k_plan_mn(p), sms, false, 0, false, false, true);
  } else {
    // MN-major operands run in 128- and 256-wide tiles only
    plan = plan_gemm(m_blocks, p.n, k_plan, sms, layout == dg::kDense, ws_cap, fp4, bf16, mn, promote ? 128 : 0,
                     layout == dg::kDense && !promote && !bf16 && !mn);
  }
  return plan;
}

// Work units (tiles) of a plan, as the kernel counts them (masked: at the
// maximum of max_m rows per group).
long long plan_units(const Problem& p, const Plan& plan, int layout) {
  const long long nb = ceil_div(p.n, plan.bn), mb = ceil_div(p.rows, dg::kBM);
  if (layout == dg::kDense) return mb * nb;
  return (long long)(layout == dg::kContig ? 1 : p.groups) * mb * nb;
}

// fixed_ws / fixed_ws_bytes: when given, stream-K partials go to this
// caller-provided device buffer instead of the per-stream workspace, and the
// planner only considers plans that fit in fixed_ws_bytes (whole tiles
// always do).
template <bool FP4, int LAYOUT, int EPI = dg::kEpiPlain, bool BF16 = false, int MAJ = dg::kMajorK>
dg_status run_gemm(const Problem& p, cudaStream_t s, float* fixed_ws = nullptr, size_t fixed_ws_bytes = 0) {
  constexpr bool kAMn = (MAJ & dg::kAMajorMN) != 0;
  constexpr bool kBMn = (MAJ & dg::kBMajorMN) != 0;
  const int sms = num_sms();
  if (sms <= 0) return DG_ERR_CUDA;
  const long long m_blocks = ceil_div(p.rows, dg::kBM);
  const Plan plan = select_plan(p, LAYOUT, FP4, BF16, MAJ != dg::kMajorK, EPI == dg::kEpiSwiGlu, sms,
                                fixed_ws != nullptr ? fixed_ws_bytes : 0, EPI == dg::kEpiPromote);
  if (plan.grid <= 0) return DG_ERR_UNSUPPORTED;  // (a forced width this layout cannot use)

  dg::GemmArgs args{};
  args.sfa = p.sfa;
  args.sfb = p.sfb;
  args.c = static_cast<const uint16_t*>(p.c);
  args.d = static_cast<uint16_t*>(p.d);
  args.ws = nullptr;
  args.m_indices = p.m_indices;
  args.masked_m = p.masked_m;
  args.ks = p.ks;
  args.rows = p.rows;
  args.n = p.n;
  args.d_cols = (EPI == dg::kEpiSwiGlu) ? p.n / 2 : p.n;
  args.k = p.k;
  args.num_groups = p.groups;
  args.num_m_blocks = (int)m_blocks;
  args.num_n_blocks = (int)ceil_div(p.n, plan.bn);
  args.kb_total = p.k / (BF16 ? 64 : 128);
  args.dp_tiles = (int)plan.dp_tiles;
  args.sk_tiles = plan.sk_tiles;
  args.max_seg = plan.max_seg;
  args.sk_split = plan.sk_split;
  args.sk_iters = plan.sk_iters;
  args.sfa_chunks = (int)ceil_div(p.rows, 128);
  args.sfb_chunks = (int)ceil_div(p.n, 128);
  args.sfa_q = (int)ceil_div(p.k / 128, 4);
  args.sfb_q = FP4 ? p.k / 128 : args.sfa_q;
  args.sfa_group_words = (long long)args.sfa_q * args.sfa_chunks * 128;
  // L2 prefetch of C a unit ahead, where the register prefetch is off (four
  // 32-column chunks per epilogue warp) and a K loop of at most 16 K-blocks
  // cannot hide C's HBM latency (measured: 4096 x 32768 x 512 140 -> 125 us;
  // at K >= 7168 the prefetched lines only compete with A and B in L2, ~1%)
  args.c_prefetch = (p.c != nullptr && p.k <= 2048) ? 1 : 0;
  args.sfb_group_words = (long long)args.sfb_q * args.sfb_chunks * 128;
  // tiles with fewer than 128 valid rows of A exist only for an M tail or in
  // the masked layout; elsewhere the producer skips the trimming arithmetic
  args.a_trim = (!kAMn && (LAYOUT == dg::kMasked || p.rows % dg::kBM != 0)) ? 1 : 0;
  args.raster = 8;
  args.band_div.init((uint32_t)(args.raster * args.num_n_blocks));
  args.group_div.init((uint32_t)(args.num_m_blocks * args.num_n_blocks));
  args.timeout_ns = timeout_ns();
  args.sfa_words = args.sfa_group_words * ((LAYOUT == dg::kMasked) ? p.groups : 1);
  args.sfb_words = args.sfb_group_words * ((LAYOUT == dg::kDense || LAYOUT == dg::kKGrouped) ? 1 : p.groups);

  if (plan.sk_tiles > 0) {
    const size_t need = plan.ws_bytes();
    if (fixed_ws != nullptr) {
      if (need > fixed_ws_bytes) return DG_ERR_SCRATCH_LIMIT;
      args.ws = fixed_ws;
    } else {
      args.ws = workspace(need, s);
      if (!args.ws) return DG_ERR_CUDA;
    }
  }

  const int ga = (LAYOUT == dg::kMasked) ? p.groups : 1;
  const int gb = (LAYOUT == dg::kDense || LAYOUT == dg::kKGrouped) ? 1 : p.groups;
  const int gd = (LAYOUT == dg::kMasked || LAYOUT == dg::kKGrouped) ? p.groups : 1;
  const uint64_t k_ext = (uint64_t)std::max(p.k, 128);  // K rows of MN-major maps
  // ta32: the same A in boxes of 32 rows, for tiles with fewer valid rows
  Maps mp;
  CUtensorMap &ta = mp.a, &ta32 = mp.a32, &tb = mp.b, &td = mp.d;
  bool ok;
  if (BF16) {
    ok = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.a, p.k, p.rows, ga, (uint64_t)p.k * 2,
                  (uint64_t)p.rows * p.k * 2, 64, dg::kBM, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&ta32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.a, p.k, p.rows, ga, (uint64_t)p.k * 2,
                        (uint64_t)p.rows * p.k * 2, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.b, p.k, p.n, gb, (uint64_t)p.k * 2,
                        (uint64_t)p.n * p.k * 2, 64, plan.bn, CU_TENSOR_MAP_SWIZZLE_128B);
  } else if (kAMn) {
    // A stored [K][rows]: boxes of 128 rows of A (contiguous) x 128 K rows
    // (K = 0, all groups empty: a map of one box that no load reads)
    ok = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.a, p.rows, k_ext, ga, (uint64_t)p.rows,
                  (uint64_t)p.rows * k_ext, dg::kBM, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    ta32 = ta;  // (not used: MN-major tiles are never trimmed)
  } else {
    ok = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.a, p.k, p.rows, ga, (uint64_t)p.k, (uint64_t)p.rows * p.k,
                  128, dg::kBM, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&ta32, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.a, p.k, p.rows, ga, (uint64_t)p.k,
                        (uint64_t)p.rows * p.k, 128, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (BF16) {
  } else if (kBMn)
    // B stored [K][n]: boxes of 128 columns x 128 K rows
    ok = ok && make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.b, p.n, k_ext, gb, (uint64_t)p.n, (uint64_t)p.n * k_ext,
                        128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  else if (FP4)
    ok = ok && make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, p.b, p.k, p.n, gb, (uint64_t)p.k / 2,
                        (uint64_t)p.n * p.k / 2, 128, plan.bn, CU_TENSOR_MAP_SWIZZLE_128B);
  else
    ok = ok && make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.b, p.k, p.n, gb, (uint64_t)p.k, (uint64_t)p.n * p.k,
                        128, plan.bn, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&td, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.d, args.d_cols, p.rows, gd, (uint64_t)args.d_cols * 2,
                      (uint64_t)p.rows * args.d_cols * 2, dg::kEpiCols, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  // C [gd][rows][n] in the same boxes (read only by L2 prefetches)
  if (p.c != nullptr)
    ok = ok && make_map(&mp.c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.c, p.n, p.rows, gd, (uint64_t)p.n * 2,
                        (uint64_t)p.rows * p.n * 2, dg::kEpiCols, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  else
    mp.c = td;
  if (!ok) return DG_ERR_CUDA;

  if (log_enabled())
    std::fprintf(stderr,
                 "[dg] layout=%d fp4=%d rows=%d n=%d k=%d groups=%d -> block_n=%d dp_tiles=%lld sk_tiles=%d "
                 "split=%d max_seg=%d cluster_split=%d grid=%d est=%.1fus\n",
                 LAYOUT, (int)FP4, p.rows, p.n, p.k, p.groups, plan.bn, plan.dp_tiles, plan.sk_tiles, plan.sk_split,
                 plan.max_seg, plan.split, plan.grid, plan.cost);

  dg_status st;
  if constexpr (LAYOUT == dg::kDense && EPI == dg::kEpiPlain && !BF16 && MAJ == dg::kMajorK) {
    if (plan.split > 0) {
      args.split = plan.split;
      return dispatch_split<FP4>(plan.bn, plan.split, mp, args, plan.grid, s);
    }
  }
  st = dispatch<FP4, LAYOUT, EPI, BF16, MAJ>(plan.bn, mp, args, plan.grid, s);
  if (st != DG_OK || plan.sk_tiles == 0) return st;

  dg::SkReduceArgs r{};
  r.ws = args.ws;
  r.c = args.c;
  r.d = args.d;
  r.rows = p.rows;
  r.n = p.n;
  r.bn = plan.bn;
  r.kb_total = args.kb_total;
  r.dp_tiles = args.dp_tiles;
  r.sk_tiles = plan.sk_tiles;
  r.max_seg = plan.max_seg;
  r.sk_split = plan.sk_split;
  r.ctas = plan.grid;
  r.sk_iters = plan.sk_iters;
  r.raster = args.raster;
  r.num_m_blocks = args.num_m_blocks;
  r.num_n_blocks = args.num_n_blocks;
  const long long items = (long long)plan.sk_tiles * dg::kBM * (plan.bn / 4);
  const int threads = 256;
  const int blocks = (int)std::min<long long>(ceil_div(items, threads), (long long)sms * 8);
  if (launch(dg::sk_reduce_kernel, dim3(blocks), dim3(threads), 0, s, 1, r) != cudaSuccess) return DG_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return DG_OK;
}

template <int KIND, int BN>
dg_status launch_probe(int kblocks, int grid, cudaStream_t s) {
  auto kern = dg::mma_peak_kernel<KIND, BN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dg::kProbeSmem) != cudaSuccess)
    return DG_ERR_CUDA;
  kern<<<grid, dg::kProbeThreads, dg::kProbeSmem, s>>>(kblocks, timeout_ns());
  if (cudaGetLastError() != cudaSuccess) return DG_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return DG_OK;
}

dg_status check_common(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, const void* c,
                       const void* d, int n, int k) {
  if (!a || !sfa || !b || !sfb || !d) return DG_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(sfa) || !aligned16(b) || !aligned16(sfb) || !aligned16(d)) return DG_ERR_INVALID_ARG;
  if (c && !aligned16(c)) return DG_ERR_INVALID_ARG;
  if (n <= 0 || n % 8 != 0 || k <= 0 || k % 128 != 0) return DG_ERR_INVALID_ARG;
  return DG_OK;
}

}  // namespace

extern "C" {

dg_status dg_fp8_gemm_nt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, const void* c, void* d,
                         int m, int n, int k, void* stream) {
  if (m < 0) return DG_ERR_INVALID_ARG;
  dg_status st = check_common(a, sfa, b, sfb, c, d, n, k);
  if (st != DG_OK) return st;
  if (m == 0) return DG_OK;
  Problem p{a, sfa, b, sfb, c, d, nullptr, nullptr, m, n, k, 1, 0};
  return run_gemm<false, dg::kDense>(p, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ---------------------------------------------------------------- no-alloc
//
// Scratch of dg_fp8_gemm_nt_noalloc: one fixed array per device, part of
// this library's device image.  It is committed on a device when the module
// is loaded there (with CUDA's lazy module loading, at the first kernel
// launch or symbol lookup of this library on that device) and held until the
// process exits.  All calls on a device share it.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
}  // namespace
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

namespace {
// Device address of g_noalloc_scratch, cached per device together with the
// context it was looked up in: after a device reset (or any other change of
// the current context) the module is loaded anew and the array may move, so
// a context that differs from the cached one triggers a new lookup.
struct NoAllocAddr {
  std::atomic<void*> ctx{nullptr};
  std::atomic<float*> addr{nullptr};
};
NoAllocAddr g_noalloc_addr[64];
std::mutex g_noalloc_mutex;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CUcontext current_context() {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (CtxGetCurrentFn) nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  CUcontext ctx = nullptr;
  if (fn == nullptr || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}

// Host code holds only a stand-in symbol for the array, so its device address
// is looked up with the device current (cudaGetSymbolAddress allocates
// nothing); the lock is taken only for a lookup, not on the cached path.
dg_status noalloc_scratch(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DG_ERR_CUDA;
  NoAllocAddr& e = g_noalloc_addr[dev];
  void* ctx = current_context();
  if (ctx != nullptr && e.ctx.load(std::memory_order_acquire) == ctx) {
    *out = e.addr.load(std::memory_order_relaxed);
    return DG_OK;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return DG_ERR_CUDA;
  e.addr.store(static_cast<float*>(p), std::memory_order_relaxed);
  e.ctx.store(current_context(), std::memory_order_release);  // (the lookup made the primary context current)
  *out = static_cast<float*>(p);
  return DG_OK;
}

void forget_noalloc_addresses() {
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  for (NoAllocAddr& e : g_noalloc_addr) {
    e.ctx.store(nullptr, std::memory_order_release);
    e.addr.store(nullptr, std::memory_order_relaxed);
  }
}
}  // namespace

extern "C" {

dg_status dg_fp8_gemm_nt_noalloc(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                 const void* c, void* d, int m, int n, int k, void* stream) {
  if (m < 0) return DG_ERR_INVALID_ARG;
  dg_status st = check_common(a, sfa, b, sfb, c, d, n, k);
  if (st != DG_OK) return st;
  if (m == 0) return DG_OK;
  float* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != DG_OK) return st;
  Problem p{a, sfa, b, sfb, c, d, nullptr, nullptr, m, n, k, 1, 0};
  return run_gemm<false, dg::kDense>(p, static_cast<cudaStream_t>(stream), scratch, kNoAllocScratchBytes);
}

size_t dg_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

dg_status dg_fp8_gemm_nt_promoted(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                  const void* c, void* d, int m, int n, int k, void* stream) {
  if (m < 0) return DG_ERR_INVALID_ARG;
  dg_status st = check_common(a, sfa, b, sfb, c, d, n, k);
  if (st != DG_OK) return st;
  if (m == 0) return DG_OK;
  Problem p{a, sfa, b, sfb, c, d, nullptr, nullptr, m, n, k, 1, 0};
  return run_gemm<false, dg::kDense, dg::kEpiPromote>(p, static_cast<cudaStream_t>(stream));
}

dg_status dg_bf16_gemm_nt(const void* a, const void* b, const void* c, void* d, int m, int n, int k, void* stream) {
  if (m < 0 || !a || !b || !d || !aligned16(a) || !aligned16(b) || !aligned16(d) || (c && !aligned16(c)))
    return DG_ERR_INVALID_ARG;
  if (n <= 0 || n % 8 != 0 || k <= 0 || k % 64 != 0) return DG_ERR_INVALID_ARG;
  if (m == 0) return DG_OK;
  Problem p{a, nullptr, b, nullptr, c, d, nullptr, nullptr, m, n, k, 1, 0};
  return run_gemm<false, dg::kDense, dg::kEpiPlain, true>(p, static_cast<cudaStream_t>(stream));
}

// Dense FP8 GEMM with A and / or B stored with K as the row index.
static dg_status dense_layout_impl(bool a_mn, bool b_mn, const void* a, const int32_t* sfa, const void* b,
                                   const int32_t* sfb, const void* c, void* d, int m, int n, int k, void* stream) {
  if (m < 0) return DG_ERR_INVALID_ARG;
  dg_status st = check_common(a, sfa, b, sfb, c, d, n, k);
  if (st != DG_OK) return st;
  // the rows of an MN-major operand are m or n bytes: 16-byte TMA row stride
  if ((a_mn && m % 16 != 0) || (b_mn && n % 16 != 0)) return DG_ERR_INVALID_ARG;
  if (m == 0) return DG_OK;
  Problem p{a, sfa, b, sfb, c, d, nullptr, nullptr, m, n, k, 1, 0};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (a_mn && b_mn) return run_gemm<false, dg::kDense, dg::kEpiPlain, false, dg::kAMajorMN | dg::kBMajorMN>(p, s);
  if (a_mn) return run_gemm<false, dg::kDense, dg::kEpiPlain, false, dg::kAMajorMN>(p, s);
  return run_gemm<false, dg::kDense, dg::kEpiPlain, false, dg::kBMajorMN>(p, s);
}

dg_status dg_fp8_gemm_nn(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, const void* c, void* d,
                         int m, int n, int k, void* stream) {
  return dense_layout_impl(false, true, a, sfa, b, sfb, c, d, m, n, k, stream);
}

dg_status dg_fp8_gemm_tn(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, const void* c, void* d,
                         int m, int n, int k, void* stream) {
  return dense_layout_impl(true, true, a, sfa, b, sfb, c, d, m, n, k, stream);
}

dg_status dg_fp8_gemm_tt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, const void* c, void* d,
                         int m, int n, int k, void* stream) {
  return dense_layout_impl(true, false, a, sfa, b, sfb, c, d, m, n, k, stream);
}

dg_status dg_fp8_fp4_gemm_nt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, const void* c,
                             void* d, int m, int n, int k, void* stream) {
  if (m < 0) return DG_ERR_INVALID_ARG;
  dg_status st = check_common(a, sfa, b, sfb, c, d, n, k);
  if (st != DG_OK) return st;
  if (m == 0) return DG_OK;
  Problem p{a, sfa, b, sfb, c, d, nullptr, nullptr, m, n, k, 1, 0};
  return run_gemm<true, dg::kDense>(p, static_cast<cudaStream_t>(stream));
}

static dg_status contiguous_impl(bool fp4, const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                 const void* c, void* d, const int32_t* m_indices, int m_total, int n, int k,
                                 int num_groups, void* stream) {
  if (m_total < 0 || m_total % 128 != 0 || num_groups <= 0 || !m_indices) return DG_ERR_INVALID_ARG;
  dg_status st = check_common(a, sfa, b, sfb, c, d, n, k);
  if (st != DG_OK) return st;
  if (c == d && c != nullptr) return DG_ERR_INVALID_ARG;
  if (m_total == 0) return DG_OK;
  Problem p{a, sfa, b, sfb, c, d, m_indices, nullptr, m_total, n, k, num_groups, 0};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return fp4 ? run_gemm<true, dg::kContig>(p, s) : run_gemm<false, dg::kContig>(p, s);
}

dg_status dg_m_grouped_fp8_gemm_nt_contiguous(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                              const void* c, void* d, const int32_t* m_indices, int m_total, int n,
                                              int k, int num_groups, void* stream) {
  return contiguous_impl(false, a, sfa, b, sfb, c, d, m_indices, m_total, n, k, num_groups, stream);
}

dg_status dg_m_grouped_fp8_fp4_gemm_nt_contiguous(const void* a, const int32_t* sfa, const void* b,
                                                  const int32_t* sfb, const void* c, void* d,
                                                  const int32_t* m_indices, int m_total, int n, int k,
                                                  int num_groups, void* stream) {
  return contiguous_impl(true, a, sfa, b, sfb, c, d, m_indices, m_total, n, k, num_groups, stream);
}

dg_status dg_m_grouped_fp8_gemm_nn_contiguous(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                              const void* c, void* d, const int32_t* m_indices, int m_total, int n,
                                              int k, int num_groups, void* stream) {
  if (m_total < 0 || m_total % 128 != 0 || num_groups <= 0 || !m_indices) return DG_ERR_INVALID_ARG;
  dg_status st = check_common(a, sfa, b, sfb, c, d, n, k);
  if (st != DG_OK) return st;
  if (n % 16 != 0) return DG_ERR_INVALID_ARG;  // B's K rows are n bytes: 16-byte TMA row stride
  if (c == d && c != nullptr) return DG_ERR_INVALID_ARG;
  if (m_total == 0) return DG_OK;
  Problem p{a, sfa, b, sfb, c, d, m_indices, nullptr, m_total, n, k, num_groups, 0};
  return run_gemm<false, dg::kContig, dg::kEpiPlain, false, dg::kBMajorMN>(p, static_cast<cudaStream_t>(stream));
}

dg_status dg_k_grouped_fp8_gemm_tn_contiguous(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                              const void* c, void* d, const int32_t* ks, int num_groups, int m,
                                              int n, int k_total, void* stream) {
  if (!a || !sfa || !b || !sfb || !d || !ks) return DG_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(sfa) || !aligned16(b) || !aligned16(sfb) || !aligned16(d) || !aligned16(ks))
    return DG_ERR_INVALID_ARG;
  if (c && !aligned16(c)) return DG_ERR_INVALID_ARG;
  if (num_groups <= 0 || num_groups > dg::kMaxMaskedGroups) return DG_ERR_INVALID_ARG;
  // A's and B's K rows are m and n bytes (16-byte TMA row stride)
  if (m <= 0 || m % 16 != 0 || n <= 0 || n % 16 != 0) return DG_ERR_INVALID_ARG;
  if (k_total < 0 || k_total % 128 != 0) return DG_ERR_INVALID_ARG;
  Problem p{a, sfa, b, sfb, c, d, nullptr, nullptr, m, n, k_total, num_groups, 0, ks};
  return run_gemm<false, dg::kKGrouped, dg::kEpiPlain, false, dg::kAMajorMN | dg::kBMajorMN>(
      p, static_cast<cudaStream_t>(stream));
}

static dg_status masked_impl(bool fp4, bool swiglu, const void* a, const int32_t* sfa, const void* b,
                             const int32_t* sfb, void* d, const int32_t* masked_m, int num_groups, int max_m, int n,
                             int k, int expected_m, void* stream) {
  if (num_groups <= 0 || num_groups > dg::kMaxMaskedGroups || max_m <= 0 || !masked_m || expected_m < 0)
    return DG_ERR_INVALID_ARG;
  if (swiglu && n % (2 * dg::kSwiGluBlock) != 0) return DG_ERR_INVALID_ARG;
  dg_status st = check_common(a, sfa, b, sfb, nullptr, d, n, k);
  if (st != DG_OK) return st;
  Problem p{a, sfa, b, sfb, nullptr, d, nullptr, masked_m, max_m, n, k, num_groups, expected_m};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (swiglu)
    return fp4 ? run_gemm<true, dg::kMasked, dg::kEpiSwiGlu>(p, s) : run_gemm<false, dg::kMasked, dg::kEpiSwiGlu>(p, s);
  return fp4 ? run_gemm<true, dg::kMasked>(p, s) : run_gemm<false, dg::kMasked>(p, s);
}

dg_status dg_m_grouped_fp8_gemm_nt_masked(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                          void* d, const int32_t* masked_m, int num_groups, int max_m, int n, int k,
                                          int expected_m, void* stream) {
  return masked_impl(false, false, a, sfa, b, sfb, d, masked_m, num_groups, max_m, n, k, expected_m, stream);
}

dg_status dg_m_grouped_fp8_fp4_gemm_nt_masked(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                              void* d, const int32_t* masked_m, int num_groups, int max_m, int n,
                                              int k, int expected_m, void* stream) {
  return masked_impl(true, false, a, sfa, b, sfb, d, masked_m, num_groups, max_m, n, k, expected_m, stream);
}

dg_status dg_m_grouped_fp8_gemm_nt_masked_swiglu(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                                 void* d, const int32_t* masked_m, int num_groups, int max_m, int n,
                                                 int k, int expected_m, void* stream) {
  return masked_impl(false, true, a, sfa, b, sfb, d, masked_m, num_groups, max_m, n, k, expected_m, stream);
}

dg_status dg_m_grouped_fp8_fp4_gemm_nt_masked_swiglu(const void* a, const int32_t* sfa, const void* b,
                                                     const int32_t* sfb, void* d, const int32_t* masked_m,
                                                     int num_groups, int max_m, int n, int k, int expected_m,
                                                     void* stream) {
  return masked_impl(true, true, a, sfa, b, sfb, d, masked_m, num_groups, max_m, n, k, expected_m, stream);
}

dg_status dg_quantize_fp8(const float* x, int rows, int cols, int block_rows, uint8_t* q, uint8_t* sf,
                          void* stream) {
  if (!x || !q || !sf || rows < 0 || cols <= 0 || cols % 128 != 0) return DG_ERR_INVALID_ARG;
  if (block_rows != 1 && block_rows != 128) return DG_ERR_INVALID_ARG;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(q) & 3u)) return DG_ERR_INVALID_ARG;
  if (rows == 0) return DG_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = std::max(1, device_sms());
  if (block_rows == 1) {
    const long long warps = (long long)rows * (cols / 128);
    const int blocks = (int)std::min<long long>(ceil_div(warps * 32, 256), (long long)sms * 16);
    dg::quant_fp8_1x128_kernel<<<blocks, 256, 0, s>>>(x, rows, cols, q, sf);
  } else {
    const long long nblk = ceil_div(rows, 128) * (cols / 128);
    const int blocks = (int)std::min<long long>(nblk, (long long)sms * 8);
    dg::quant_fp8_128x128_kernel<<<blocks, 256, 0, s>>>(x, rows, cols, q, sf);
  }
  if (cudaGetLastError() != cudaSuccess) return DG_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return DG_OK;
}

dg_status dg_quantize_fp4(const float* x, int rows, int cols, uint8_t* q, uint8_t* sf, void* stream) {
  if (!x || !q || !sf || rows < 0 || cols <= 0 || cols % 32 != 0) return DG_ERR_INVALID_ARG;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(q) & 3u)) return DG_ERR_INVALID_ARG;
  if (rows == 0) return DG_OK;
  const int sms = std::max(1, device_sms());
  const long long thr = (long long)rows * (cols / 32) * 4;
  const int blocks = (int)std::min<long long>(ceil_div(thr, 256), (long long)sms * 16);
  dg::quant_fp4_1x32_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, rows, cols, q, sf);
  if (cudaGetLastError() != cudaSuccess) return DG_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return DG_OK;
}

int64_t dg_packed_sf_words(int rows, int num_sf_cols) {
  if (rows <= 0 || num_sf_cols <= 0) return 0;
  return (int64_t)ceil_div(num_sf_cols, 4) * ceil_div(rows, 128) * 128;
}

dg_status dg_pack_sf(const uint8_t* sf, int rows, int num_sf_cols, int row_div, int32_t* packed, void* stream) {
  if (!sf || !packed || rows <= 0 || num_sf_cols <= 0 || row_div <= 0) return DG_ERR_INVALID_ARG;
  const long long total = dg_packed_sf_words(rows, num_sf_cols);
  const int sms = std::max(1, device_sms());
  const int blocks = (int)std::min<long long>(ceil_div(total, 256), (long long)sms * 16);
  dg::pack_sf_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(sf, rows, num_sf_cols, row_div, packed);
  if (cudaGetLastError() != cudaSuccess) return DG_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return DG_OK;
}

int dg_get_num_sms(void) { return num_sms(); }

dg_status dg_set_num_sms(int n) {
  if (n < 0) return DG_ERR_INVALID_ARG;
  g_num_sms_override = n;
  return DG_OK;
}

int dg_get_mk_alignment_for_contiguous_layout(void) { return dg::kBM; }

dg_status dg_set_pdl(int enable) {
  g_pdl.store(enable ? 1 : 0);
  return DG_OK;
}

int dg_get_pdl(void) { return g_pdl.load(); }

dg_status dg_set_tile_config(int block_n, int schedule) {
  if (block_n != 0) {
    bool known = false;
    for (const WidthCost& wc : kWidthCosts) known = known || (wc.bn == block_n);
    if (!known) return DG_ERR_INVALID_ARG;
  }
  if (schedule < 0 || schedule > 10) return DG_ERR_INVALID_ARG;
  g_force_bn.store(block_n);
  g_force_schedule.store(schedule);
  return DG_OK;
}

dg_status dg_get_last_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DG_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, dg::g_error_word, sizeof(int)) != cudaSuccess) return DG_ERR_CUDA;
  if (v != 0) {
    int zero = 0;
    if (cudaMemcpyToSymbol(dg::g_error_word, &zero, sizeof(int)) != cudaSuccess) return DG_ERR_CUDA;
  }
  return static_cast<dg_status>(v);
}

dg_status dg_debug_starved_wait(unsigned int limit_us, void* stream) {
  dg::starved_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((unsigned long long)limit_us * 1000ull);
  if (cudaGetLastError() != cudaSuccess) return DG_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return DG_OK;
}

const char* dg_status_string(int status) {
  switch (status) {
    case DG_OK: return "DG_OK";
    case DG_ERR_INVALID_ARG: return "DG_ERR_INVALID_ARG";
    case DG_ERR_UNSUPPORTED: return "DG_ERR_UNSUPPORTED";
    case DG_ERR_CUDA: return "DG_ERR_CUDA";
    case DG_ERR_TIMEOUT: return "DG_ERR_TIMEOUT";
    case DG_ERR_BAD_METADATA: return "DG_ERR_BAD_METADATA";
    case DG_ERR_SCRATCH_LIMIT: return "DG_ERR_SCRATCH_LIMIT";
    default: return "DG_ERR_UNKNOWN";
  }
}

uint64_t dg_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

dg_status dg_query_dense_config(int m, int n, int k, int64_t workspace_cap, int* block_n, int* dp_tiles,
                                int* sk_tiles, int* sk_split, int* max_segments, int* grid,
                                int64_t* workspace_bytes) {
  if (m <= 0 || n <= 0 || k <= 0 || k % 128 != 0 || workspace_cap < 0) return DG_ERR_INVALID_ARG;
  const int sms = num_sms();
  if (sms <= 0) return DG_ERR_CUDA;
  Plan p = plan_gemm(ceil_div(m, dg::kBM), n, k, sms, true, (size_t)workspace_cap, false, false, false, 0, true);
  if (block_n) *block_n = p.bn;
  if (dp_tiles) *dp_tiles = (int)p.dp_tiles;
  if (sk_tiles) *sk_tiles = p.sk_tiles;
  if (sk_split) *sk_split = p.sk_split;
  if (max_segments) *max_segments = p.max_seg;
  if (grid) *grid = p.grid;
  if (workspace_bytes) *workspace_bytes = (int64_t)p.ws_bytes();
  return DG_OK;
}

int dg_debug_cluster_capacity(int block_n, int fp4, int cluster) {
  if ((block_n != 128 && block_n != 256) || cluster < 2 || cluster > 8) return -1;
  return split_capacity(block_n, fp4 != 0, cluster);
}

int dg_query_dense_cluster_split(int m, int n, int k, int64_t workspace_cap) {
  if (m <= 0 || n <= 0 || k <= 0 || k % 128 != 0 || workspace_cap < 0) return -1;
  const int sms = num_sms();
  if (sms <= 0) return -1;
  return plan_gemm(ceil_div(m, dg::kBM), n, k, sms, true, (size_t)workspace_cap, false, false, false, 0, true).split;
}

dg_status dg_query_config(int layout, int fp4, int swiglu, int rows, int n, int k, int num_groups, int expected_m,
                          int* block_n, int* grid, int64_t* units) {
  if (layout < DG_LAYOUT_DENSE || layout > DG_LAYOUT_MASKED || rows <= 0 || n <= 0 || k <= 0 || k % 128 != 0 ||
      num_groups <= 0 || expected_m < 0 || (swiglu && layout != DG_LAYOUT_MASKED))
    return DG_ERR_INVALID_ARG;
  const int sms = num_sms();
  if (sms <= 0) return DG_ERR_CUDA;
  const int lay = layout == DG_LAYOUT_DENSE ? dg::kDense : (layout == DG_LAYOUT_CONTIGUOUS ? dg::kContig : dg::kMasked);
  Problem p{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, rows, n, k,
            lay == dg::kDense ? 1 : num_groups, expected_m};
  const Plan plan = select_plan(p, lay, fp4 != 0, false, false, swiglu != 0, sms, 0);
  if (block_n) *block_n = plan.bn;
  if (grid) *grid = plan.grid;
  if (units) *units = plan_units(p, plan, lay);
  return DG_OK;
}

dg_status dg_probe_mma_peak(int kind, int block_n, int kblocks, void* stream) {
  const bool narrow = (block_n == 32 || block_n == 64 || block_n == 192);
  if (kind < DG_PROBE_FP8_SCALED || kind > DG_PROBE_BF16 || (block_n != 128 && block_n != 256 && !narrow) ||
      (narrow && kind != DG_PROBE_FP8_SCALED) || kblocks <= 0 || kblocks > (1 << 22))
    return DG_ERR_INVALID_ARG;
  const int grid = device_sms();
  if (grid <= 0) return DG_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (kind == DG_PROBE_FP8_SCALED) {
    switch (block_n) {
      case 32: return launch_probe<dg::kProbeScaled, 32>(kblocks, grid, s);
      case 64: return launch_probe<dg::kProbeScaled, 64>(kblocks, grid, s);
      case 128: return launch_probe<dg::kProbeScaled, 128>(kblocks, grid, s);
      case 192: return launch_probe<dg::kProbeScaled, 192>(kblocks, grid, s);
      default: return launch_probe<dg::kProbeScaled, 256>(kblocks, grid, s);
    }
  }
  if (kind == DG_PROBE_FP8_PLAIN)
    return block_n == 128 ? launch_probe<dg::kProbePlain, 128>(kblocks, grid, s)
                          : launch_probe<dg::kProbePlain, 256>(kblocks, grid, s);
  return block_n == 128 ? launch_probe<dg::kProbeBf16, 128>(kblocks, grid, s)
                        : launch_probe<dg::kProbeBf16, 256>(kblocks, grid, s);
}

uint32_t dg_debug_fastdiv(uint32_t d, uint32_t n) {
  if (d == 0 || n >= (1u << 31)) return 0xFFFFFFFFu;
  dg::FastDiv f;
  f.init(d);
  return f.div(n);
}

int64_t dg_num_tiles(int m, int n, int block_m, int block_n) {
  if (m <= 0 || n <= 0 || block_m <= 0 || block_n <= 0) return 0;
  return ceil_div(m, block_m) * ceil_div(n, block_n);
}

void dg_shutdown(void) {
  forget_noalloc_addresses();
  std::lock_guard<std::mutex> lock(g_ws_mutex);
  int prev = 0;
  cudaGetDevice(&prev);
  for (auto& kv : g_ws) {
    if (kv.second.ptr) {
      cudaSetDevice(kv.first.first);
      cudaStreamSynchronize(kv.first.second);
      cudaFree(kv.second.ptr);
    }
  }
  g_ws.clear();
  cudaSetDevice(prev);
}

}  // extern "C"
