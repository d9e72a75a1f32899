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
#include <utility>

#include "../../include/dg.h"
#include "dg_gemm.cuh"
#include "dg_prep.cuh"

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

constexpr int kBlockNs[] = {128, 192, 256};  // multiples of 64 (see Cfg in dg_gemm.cuh)

struct Plan {
  int bn = 128;
  int ctas = 1;  // 2: a cluster of two CTAs computes 256-row tiles
  int splits = 1;
  int kb_per_split = 1;
  long long units = 0;
  int grid = 0;
};

long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }

// Estimated critical path (per SM) in units of "B rows x K-blocks" streamed
// through the tensor core: waves x (BN x K-blocks per unit + a per-unit
// overhead of 4 K-blocks), with a 3% surcharge per extra split-K slice for
// the partial-sum round trip.  Minimised over the instantiated block sizes;
// ties keep fewer slices, then the larger block.
// Tile-configuration override (dg_set_tile_config; initial values from the
// environment variables DG_BLOCK_N and DG_CTAS): restricts the heuristic's
// search to one block width and/or to single CTAs (1) or CTA pairs (2).
int env_int(const char* name) {
  const char* e = std::getenv(name);
  return e ? std::atoi(e) : 0;
}
std::atomic<int> g_force_bn{env_int("DG_BLOCK_N")};
std::atomic<int> g_force_ctas{env_int("DG_CTAS") == 1 ? 1 : 0};

int forced_ctas() {
  const int c = g_force_ctas.load();
  return (c == 1 || c == 2) ? c : 0;
}

int forced_block_n() {
  const int b = g_force_bn.load();
  for (int bn : kBlockNs)
    if (bn == b) return b;
  return 0;
}

// CTA pairs (dense only, allow_pair) are costed per cluster: half the SMs,
// tiles of 256 rows, no split-K, and 0.85x the per-unit time for staging half
// of B per SM.
Plan plan_gemm(long long m_blocks, int n, int k, int sms, bool allow_split, bool allow_pair = false) {
  Plan best;
  double best_cost = 1e300;
  const int kb = k / 128;
  if (allow_pair && m_blocks >= 2 && forced_ctas() != 1) {
    for (int bn : kBlockNs) {
      if (bn < 192 || (forced_block_n() && bn != forced_block_n())) continue;
      const long long units = ((m_blocks + 1) / 2) * ceil_div(n, bn);
      const double waves = (double)ceil_div(units, sms / 2);
      const double cost = waves * (double)bn * (kb + 4) * 0.85;
      if (cost < best_cost * (1 - 1e-9)) {
        best_cost = cost;
        best.bn = bn;
        best.ctas = 2;
        best.splits = 1;
        best.kb_per_split = kb;
        best.units = units;
      }
    }
  }
  for (int bn : kBlockNs) {
    if (forced_ctas() == 2 && best.ctas == 2) break;
    if (forced_block_n() && bn != forced_block_n()) continue;
    const long long tiles = m_blocks * ceil_div(n, bn);
    const int max_s = allow_split ? std::max(1, std::min(dg::kMaxSplits, kb / 2)) : 1;
    for (int s = 1; s <= max_s; ++s) {
      const int kbps = (int)ceil_div(kb, s);
      const int s_eff = (int)ceil_div(kb, kbps);
      if (s_eff != s) continue;
      const long long units = tiles * s;
      const double waves = (double)ceil_div(units, sms);
      const double cost = waves * (double)bn * (kbps + 4) * (1.0 + 0.03 * (s - 1));
      if (cost < best_cost * (1 - 1e-9)) {
        best_cost = cost;
        best.bn = bn;
        best.ctas = 1;
        best.splits = s;
        best.kb_per_split = kbps;
        best.units = units;
      }
    }
  }
  if (best.ctas == 2)
    best.grid = 2 * (int)std::max<long long>(1, std::min<long long>(best.units, sms / 2));
  else
    best.grid = (int)std::max<long long>(1, std::min<long long>(best.units, sms));
  return best;
}

// ------------------------------------------------------------ workspaces

struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};
std::mutex g_ws_mutex;
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;

// Split-K FP32 partials of this (device, stream), allocated stream-ordered on
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

template <int BN, bool FP4, int LAYOUT, int CTAS>
dg_status launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td, const CUtensorMap& tsfa,
                      const CUtensorMap& tsfb, const dg::GemmArgs& args, int grid, cudaStream_t s) {
  using C = dg::Cfg<BN, FP4, CTAS>;
  auto kern = dg::gemm_kernel<BN, FP4, LAYOUT, CTAS>;
  static std::atomic<uint64_t> attr_set_mask{0};  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_set_mask.load() & bit)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
      return DG_ERR_CUDA;
    attr_set_mask.fetch_or(bit);
  }
  if (launch(kern, dim3(grid), dim3(dg::kThreads), C::kSmemBytes, s, CTAS, ta, tb, td, tsfa, tsfb, args) !=
      cudaSuccess)
    return DG_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return DG_OK;
}

template <bool FP4, int LAYOUT>
dg_status dispatch(int bn, int ctas, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td,
                   const CUtensorMap& tsfa, const CUtensorMap& tsfb, const dg::GemmArgs& args, int grid,
                   cudaStream_t s) {
  // CTA-pair (cta_group::2) kernels are not launched: on B200 they stopped
  // with "illegal instruction" and the cause is not yet known.
  if (ctas != 1) return DG_ERR_UNSUPPORTED;
  switch (bn) {
    case 128: return launch_gemm<128, FP4, LAYOUT, 1>(ta, tb, td, tsfa, tsfb, args, grid, s);
    case 192: return launch_gemm<192, FP4, LAYOUT, 1>(ta, tb, td, tsfa, tsfb, args, grid, s);
    case 256: return launch_gemm<256, FP4, LAYOUT, 1>(ta, tb, td, tsfa, tsfb, args, grid, s);
    default: return DG_ERR_UNSUPPORTED;
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
};

// fixed_ws / fixed_ws_bytes: when given, split-K partials go to this caller-
// provided device buffer instead of the per-stream workspace, and a plan that
// needs more than fixed_ws_bytes is rejected with DG_ERR_SCRATCH_LIMIT.
template <bool FP4, int LAYOUT>
dg_status run_gemm(const Problem& p, cudaStream_t s, float* fixed_ws = nullptr, size_t fixed_ws_bytes = 0) {
  const int sms = num_sms();
  if (sms <= 0) return DG_ERR_CUDA;
  const long long m_blocks = ceil_div(p.rows, dg::kBM);
  Plan plan;
  if (LAYOUT == dg::kMasked) {
    const int em = p.expected_m > 0 ? std::min(p.expected_m, p.rows) : p.rows;
    plan = plan_gemm((long long)p.groups * ceil_div(em, dg::kBM), p.n, p.k, sms, false);
    plan.grid = (int)std::min<long long>((long long)p.groups * m_blocks * ceil_div(p.n, plan.bn), sms);
  } else {
    const bool allow_split = (LAYOUT == dg::kDense) && p.rows <= 1024;
    plan = plan_gemm(m_blocks, p.n, p.k, sms, allow_split, /*allow_pair=*/false);
  }

  dg::GemmArgs args{};
  args.sfa = p.sfa;
  args.sfb = p.sfb;
  args.c = static_cast<const uint16_t*>(p.c);
  args.d = static_cast<uint16_t*>(p.d);
  args.ws = nullptr;
  args.m_indices = p.m_indices;
  args.masked_m = p.masked_m;
  args.rows = p.rows;
  args.n = p.n;
  args.k = p.k;
  args.num_groups = p.groups;
  args.num_m_blocks = (int)(plan.ctas == 2 ? ceil_div(p.rows, 2 * dg::kBM) : m_blocks);
  args.num_n_blocks = (int)ceil_div(p.n, plan.bn);
  args.kb_total = p.k / 128;
  args.splits = plan.splits;
  args.kb_per_split = plan.kb_per_split;
  args.sfa_chunks = (int)ceil_div(p.rows, 128);
  args.sfb_chunks = (int)ceil_div(p.n, 128);
  args.sfa_q = (int)ceil_div(p.k / 128, 4);
  args.sfb_q = FP4 ? p.k / 128 : args.sfa_q;
  args.sfa_group_words = (long long)args.sfa_q * args.sfa_chunks * 128;
  args.sfb_group_words = (long long)args.sfb_q * args.sfb_chunks * 128;
  args.raster = 8;
  args.timeout_ns = timeout_ns();
  args.sfa_words = args.sfa_group_words * ((LAYOUT == dg::kMasked) ? p.groups : 1);
  args.sfb_words = args.sfb_group_words * ((LAYOUT == dg::kDense) ? 1 : p.groups);

  if (plan.splits > 1) {
    const size_t need = (size_t)plan.splits * p.rows * p.n * sizeof(float);
    if (fixed_ws != nullptr) {
      if (need > fixed_ws_bytes) return DG_ERR_SCRATCH_LIMIT;
      args.ws = fixed_ws;
    } else {
      args.ws = workspace(need, s);
      if (!args.ws) return DG_ERR_CUDA;
    }
  }

  const int ga = (LAYOUT == dg::kMasked) ? p.groups : 1;
  const int gb = (LAYOUT == dg::kDense) ? 1 : p.groups;
  CUtensorMap ta, tb, td;
  bool ok = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.a, p.k, p.rows, ga, (uint64_t)p.k,
                     (uint64_t)p.rows * p.k, 128, dg::kBM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (FP4)
    ok = ok && make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, p.b, p.k, p.n, gb, (uint64_t)p.k / 2,
                        (uint64_t)p.n * p.k / 2, 128, plan.bn / plan.ctas, CU_TENSOR_MAP_SWIZZLE_128B);
  else
    ok = ok && make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.b, p.k, p.n, gb, (uint64_t)p.k, (uint64_t)p.n * p.k,
                        128, plan.bn / plan.ctas, CU_TENSOR_MAP_SWIZZLE_128B);
  // packed scale words as rows of 128 words (one 128-row chunk per row): the
  // CTA-pair kernel loads them with tiled copies that can complete on the
  // leader's barrier; single-CTA kernels use plain bulk copies instead
  CUtensorMap tsfa = ta, tsfb = ta;
  if (plan.ctas == 2) {
    const uint64_t rows_a = (uint64_t)args.sfa_q * args.sfa_chunks;
    const uint64_t rows_b = (uint64_t)args.sfb_q * args.sfb_chunks;
    ok = ok && make_map(&tsfa, CU_TENSOR_MAP_DATA_TYPE_INT32, p.sfa, 128, rows_a, 1, 512, rows_a * 512, 128, 1,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
    ok = ok && make_map(&tsfb, CU_TENSOR_MAP_DATA_TYPE_INT32, p.sfb, 128, rows_b, 1, 512, rows_b * 512, 128, 1,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  ok = ok && make_map(&td, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.d, p.n, p.rows, ga, (uint64_t)p.n * 2,
                      (uint64_t)p.rows * p.n * 2, dg::kEpiCols, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  if (!ok) return DG_ERR_CUDA;

  if (log_enabled())
    std::fprintf(stderr,
                 "[dg] layout=%d fp4=%d rows=%d n=%d k=%d groups=%d -> block_n=%d ctas=%d splits=%d units=%lld grid=%d\n",
                 LAYOUT, (int)FP4, p.rows, p.n, p.k, p.groups, plan.bn, plan.ctas, plan.splits, plan.units, plan.grid);

  dg_status st = dispatch<FP4, LAYOUT>(plan.bn, plan.ctas, ta, tb, td, tsfa, tsfb, args, plan.grid, s);
  if (st != DG_OK || plan.splits == 1) return st;

  const long long units = (long long)p.rows * (p.n / 4);
  const int threads = 256;
  const int blocks = (int)std::min<long long>(ceil_div(units, threads), (long long)sms * 8);
  if (launch(dg::splitk_reduce_kernel, dim3(blocks), dim3(threads), 0, s, 1, (const float*)args.ws, args.c, args.d,
             p.rows, p.n, plan.splits) != cudaSuccess)
    return DG_ERR_CUDA;
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
// this library's device image, so it exists on every GPU that loads the
// library until the process exits.  All calls on a device share it.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
}  // namespace
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

namespace {
std::mutex g_noalloc_mutex;
float* g_noalloc_addr[64] = {};

// Device address of g_noalloc_scratch on the current device.  Host code
// only holds a stand-in symbol for the array, so the address is looked up
// once per device, with that device current, and cached.
dg_status noalloc_scratch(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DG_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return DG_ERR_CUDA;
    g_noalloc_addr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_addr[dev];
  return DG_OK;
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

dg_status dg_m_grouped_fp8_gemm_nt_masked(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                          void* d, const int32_t* masked_m, int num_groups, int max_m, int n, int k,
                                          int expected_m, void* stream) {
  if (num_groups <= 0 || num_groups > dg::kMaxMaskedGroups || max_m <= 0 || !masked_m || expected_m < 0)
    return DG_ERR_INVALID_ARG;
  dg_status st = check_common(a, sfa, b, sfb, nullptr, d, n, k);
  if (st != DG_OK) return st;
  Problem p{a, sfa, b, sfb, nullptr, d, nullptr, masked_m, max_m, n, k, num_groups, expected_m};
  return run_gemm<false, dg::kMasked>(p, static_cast<cudaStream_t>(stream));
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

dg_status dg_set_tile_config(int block_n, int ctas) {
  if (block_n != 0) {
    bool known = false;
    for (int bn : kBlockNs) known = known || (bn == block_n);
    if (!known) return DG_ERR_INVALID_ARG;
  }
  if (ctas != 0 && ctas != 1 && ctas != 2) return DG_ERR_INVALID_ARG;
  if (ctas == 2) return DG_ERR_UNSUPPORTED;  // CTA pairs are not launched (see dispatch)
  g_force_bn.store(block_n);
  g_force_ctas.store(ctas);
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

dg_status dg_query_dense_config(int m, int n, int k, int* block_n, int* splits, int* units, int* grid, int* ctas) {
  if (m <= 0 || n <= 0 || k <= 0 || k % 128 != 0) return DG_ERR_INVALID_ARG;
  const int sms = num_sms();
  if (sms <= 0) return DG_ERR_CUDA;
  Plan p = plan_gemm(ceil_div(m, dg::kBM), n, k, sms, m <= 1024, /*allow_pair=*/false);
  if (block_n) *block_n = p.bn;
  if (splits) *splits = p.splits;
  if (units) *units = (int)p.units;
  if (grid) *grid = p.grid;
  if (ctas) *ctas = p.ctas;
  return DG_OK;
}

int64_t dg_num_tiles(int m, int n, int block_m, int block_n) {
  if (m <= 0 || n <= 0 || block_m <= 0 || block_n <= 0) return 0;
  return ceil_div(m, block_m) * ceil_div(n, block_n);
}

void dg_shutdown(void) {
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
