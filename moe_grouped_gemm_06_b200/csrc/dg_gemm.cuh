// dg_gemm.cuh -- the persistent, warp-specialised, block-scaled GEMM for sm_100a.
//
//   D = C + A * B^T   (A: M x K e4m3, B: N x K e4m3 or e2m1, K-major, or
//                      either stored with K as the row index (MN-major);
//                      C, D: bf16 row-major; FP32 accumulation in TMEM)
//
// with DeepSeek-V3 fine-grained scaling: one UE8M0 scale per 1x128 row-group
// of A and per 128x128 block of B (FP4 B: per 1x32 row-group).  Sources:
// "DeepSeek 开源第三弹 ... DeepGEMM" (app.myzaker.com), sections "DeepGEMM"
// (fine-grained scaling), "优化技术" (persistent warp specialisation, TMA
// loads/stores, unified block scheduler with L2 rasterisation, unaligned
// block sizes); "DeepGEMM：统一高性能张量核心 GEMM 计算库编译与使用指南"
// (zhouruolin.cn), section 五 (D = C + A @ B, NT layout and on SM100 also TN,
// NN and TT, packed UE8M0 scales, M-grouped contiguous and masked layouts,
// the K-grouped weight-gradient layout); "DeepSeek 发布 DeepGEMM 重大更新"
// (linlog.top), section "FP4 精度支持" (FP8 x FP4).
//
// Roles (320 threads, one CTA per SM, persistent over work units):
//   warp 0      TMA producer: A/B tiles (128-byte swizzle) and packed scale
//               words into a STAGES-deep shared-memory ring.
//   warp 1      allocates TMEM; one lane issues tcgen05.cp (scales -> TMEM)
//               and tcgen05.mma.kind::mxf8f6f4.block_scale into a
//               double-buffered FP32 accumulator.
//   warps 2..9  epilogue, two warps per TMEM sub-partition (one column half
//               each): C prefetched into registers, tcgen05.ld -> (+C) ->
//               bf16 -> swizzled smem -> TMA store; rows past a masked
//               group's count are never written.  Stream-K pieces go to
//               FP32 workspace slots, summed by sk_reduce_kernel.
//
// The scales are applied inside the MMA: the UE8M0 code of a 1x128 group is
// used for each of the four K=32 steps of its 128-wide block (the instruction
// descriptor's scale-factor id selects the byte of the packed word), which
// replaces the Hopper design's CUDA-core promotion of every K-block.
#pragma once
#include <cuda_bf16.h>
#include "dg_ptx.cuh"

namespace dg {

constexpr int kBM = 128;           // rows of A per tile (= TMEM lanes)
constexpr int kBK = 128;           // K per pipeline stage (= one scale block)
constexpr int kEpiWarps = 8;        // 4 TMEM sub-partitions x kEpiParts column parts
constexpr int kEpiParts = kEpiWarps / 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;  // warp 0 TMA, warp 1 MMA, the rest epilogue
// Blocks of tiles whose width is not a multiple of 64 carry one more warp
// (index 2 + kEpiWarps), which re-bases their B scale words (Cfg::kRebase).
template <int BN, bool BF16>
__host__ __device__ constexpr int block_threads() {
  return kThreads + ((BN % 64 != 0 && !BF16) ? 32 : 0);
}
constexpr int kEpiCols = 32;       // columns per epilogue store box
constexpr int kTmemCols = 512;
constexpr int kMaxMaskedGroups = 1024;

// kKGrouped: the weight-gradient layout, grouped along K -- group g owns the
// K rows [K_0 + ... + K_(g-1), ... + K_g) of A and B and its own D[g].
// kDenseSplit: the dense layout with every tile's K-blocks cut into `split`
// (2 to 8) slices computed by the CTAs of one thread-block cluster, whose FP32
// partial sums are added through distributed shared memory (no workspace, no
// second kernel); for problems with too few tiles to fill the SMs.
enum : int { kDense = 0, kContig = 1, kMasked = 2, kKGrouped = 3, kDenseSplit = 4 };

// Operand majorness (template parameter MAJ): which of A and B are stored
// MN-major (M or N contiguous, K rows) instead of K-major.
enum : int { kMajorK = 0, kAMajorMN = 1, kBMajorMN = 2 };

// Epilogues: D = bf16(acc + C), or SwiGLU on B rows interleaved in blocks of
// kSwiGluBlock (gate rows, then the matching up rows): act = bf16(silu(gate)
// * up), half as many columns as the GEMM.  kEpiPromote: D = bf16(acc + C)
// where the scales are not applied by the MMA: each 128-deep K-block is
// summed unscaled by a plain kind::f8f6f4 MMA into a TMEM buffer of its own,
// and the epilogue warps "promote" it -- multiply by sa * sb and add into
// FP32 registers -- the two-level accumulation of the pages' Hopper design
// ("DeepSeek 开源第三弹 ... DeepGEMM" (app.myzaker.com), sections "DeepGEMM"
// and "持久化线程束专用化"), kept as the measured alternative to the
// block-scaled MMA.
enum : int { kEpiPlain = 0, kEpiSwiGlu = 1, kEpiPromote = 2 };
constexpr int kSwiGluBlock = 64;

// Unsigned division by a run-time divisor d >= 1 fixed per launch, as one
// multiply-high, an add and a shift (Granlund and Montgomery, "Division by
// invariant integers using multiplication", 1994): with s = ceil(log2 d) and
// m = floor(2^32 (2^s - d) / d) + 1, n / d = (mulhi(n, m) + n) >> s for every
// n < 2^31.
struct FastDiv {
  uint32_t d, mul, shift;
  __host__ __device__ void init(uint32_t dd) {
    d = dd;
    shift = 0;
    while ((1ull << shift) < d) ++shift;
    mul = (uint32_t)(((1ull << 32) * ((1ull << shift) - d)) / d + 1);
  }
  __host__ __device__ __forceinline__ uint32_t div(uint32_t n) const {
#ifdef __CUDA_ARCH__
    const uint32_t t = __umulhi(n, mul);
#else
    const uint32_t t = (uint32_t)(((uint64_t)n * mul) >> 32);
#endif
    return (t + n) >> shift;
  }
};

struct GemmArgs {
  const int32_t* sfa;        // packed scale words of A
  const int32_t* sfb;        // packed scale words of B
  const uint16_t* c;         // bf16 bits [rows][n] or nullptr
  uint16_t* d;               // bf16 bits (predicated-store path)
  float* ws;                 // stream-K partials [sk_tiles][max_seg][kBM][BN] (FP32)
  const int32_t* m_indices;  // contiguous: group of each row (-1 = padding)
  const int32_t* masked_m;   // masked: valid rows per group
  const int32_t* ks;         // k-grouped: K of each group (multiples of 128)
  int rows;                  // dense: M; contiguous: M_total; masked: max_m
  int n, k;
  int d_cols;                // columns of D: n, or n / 2 for SwiGLU
  int num_groups;
  int num_m_blocks;          // per group for masked
  int num_n_blocks;
  int kb_total;              // k / 128
  // dense schedule: the first dp_tiles tiles (raster order) are computed
  // whole, round robin over the CTAs; the K-iterations of the sk_tiles tiles
  // after them are shared out:
  //   sk_split = s > 0: tile j's K-blocks cut into s equal slices, slice t on
  //                     CTA j*s + t (one piece per CTA, slot t);
  //   sk_split = 0:     stream-K: sk_iters = sk_tiles x kb_total iterations,
  //                     CTA c taking [c sk_iters / G, (c + 1) sk_iters / G),
  //                     slot = CTA - first CTA of the tile.
  // A tile's pieces land in its max_seg workspace slots.
  int dp_tiles, sk_tiles, max_seg, sk_split;
  long long sk_iters;
  int split;                           // kDenseSplit: CTAs (K-slices) per tile = cluster size
  int a_trim;                          // some tiles have fewer than kBM valid rows of A (M tail, masked)
  int sfa_chunks, sfb_chunks;          // ceil(rows/128), ceil(n/128)
  long long sfa_group_words, sfb_group_words;
  int sfa_q, sfb_q;                    // packed groups along K
  int c_prefetch;                      // L2 prefetch of the next unit's C (short K, wide tiles)
  int raster;                          // m-blocks per raster band
  FastDiv band_div;                    // division by raster * num_n_blocks (tiles per band)
  FastDiv group_div;                   // k-grouped: division by num_m_blocks * num_n_blocks
  unsigned long long timeout_ns;
  long long sfa_words, sfb_words;      // total packed words (self-check bounds)
};

// BF16 = true: A and B bf16 (kind::f16, no scales); a stage then holds 64
// K-elements, the same 128-byte rows as 128 e4m3 elements, so the staging,
// descriptors and schedules are shared with the FP8 kernels.
// PREFIX = true (masked and k-grouped layouts): shared memory also holds the
// per-group prefix of tile counts or K-blocks; the other layouts give those
// bytes to the stage ring.
// PROMO = true (kEpiPromote): no scale words are staged (the epilogue reads
// them from global memory) and TMEM holds only per-K-block partial sums.
// OVL = true (256-wide tiles, plain epilogue): two accumulators that share 64
// columns, at columns 0 and 192, instead of a single one: 512 TMEM columns
// hold two whole 256-column accumulators only without the scale factors, so
// the second one overlaps the first and the next tile's MMAs wait only until
// the epilogue has drained the shared columns (it drains them first).
template <int BN, bool FP4, bool BF16 = false, bool PREFIX = true, bool PROMO = false, bool OVL = false>
struct Cfg {
  static_assert(!(BF16 && FP4), "bf16 A and B");
  static_assert(!PROMO || (!FP4 && !BF16 && BN == 128), "promotion: e4m3 A and B, 128-wide tiles");
  static_assert(!OVL || (BN == 256 && !PROMO), "overlapping accumulators: 256-wide tiles");
  static constexpr int kKPerStage = BF16 ? 64 : kBK;  // K-elements per stage
  // The scale-factor operand of the MMA is addressed in TMEM columns of 32
  // rows (a 128-row chunk spans 4 columns), and that address must be even: a
  // tile starting 32 or 96 rows into a chunk (odd column) faults with a
  // misaligned-address error.  Tiles of a width that is not a multiple of 64
  // therefore have their B scale words re-based in shared memory (kRebase) so
  // that the MMA reads them from column offset 0.
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "BN");
  static constexpr int kMaxOffRows = (BN % 128 == 0) ? 0 : (BN % 64 == 0 ? 64 : 96);
  static constexpr int kSfbChunks = (kMaxOffRows + BN + 127) / 128;  // 128-row scale chunks a tile can touch
  static constexpr bool kRebase = (BN % 64 != 0);
  static constexpr int kSfrChunks = (BN + 127) / 128;                // re-based chunks (tile rows only)
  static constexpr bool kRebaseWarp = kRebase && !BF16 && !PROMO;   // see block_threads()
  static constexpr int kSfrBytes = kRebaseWarp ? kSfrChunks * 512 : 0;
  // FP32 accumulator buffers in TMEM: three of 128 columns (BN = 128), two at
  // columns 0 and 256 (BN = 192), one (BN = 256); scale factors after them.
  // Promotion: four 128-column buffers of K-block partial sums, no scales.
  static constexpr int kAccBufs = PROMO ? 4 : (OVL ? 2 : ((BN <= 128) ? 3 : (BN <= 240 ? 2 : 1)));
  static constexpr int kABytes = kBM * kBK;                  // 16 KB
  static constexpr int kBBytes = BN * kBK;                   // smem bytes (FP4 lands padded to 1 B/elt)
  static constexpr int kBTxBytes = FP4 ? kBBytes / 2 : kBBytes;  // bytes the TMA copy reports (packed)
  static constexpr int kSfaBytes = (BF16 || PROMO) ? 0 : 512;
  static constexpr int kSfbBytes = (BF16 || PROMO) ? 0 : kSfbChunks * 512;
  static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes + kSfrBytes;
  static constexpr int kEpiBytes = kEpiWarps * 32 * 64;        // one 32 x 64 B staging box per epilogue warp
  static constexpr int kMaskBytes = PREFIX ? ((kMaxMaskedGroups + 1) * 4 + 15) / 16 * 16 : 0;
  static constexpr int kBarBytes = 256;
  static constexpr int kBudget = 232448 - 1024;              // 227 KB minus alignment slack
  static constexpr int kStagesRaw = (kBudget - kEpiBytes - kMaskBytes - kBarBytes) / kStageBytes;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static_assert(kStages >= 2, "stages");
  // barriers: full, empty (and re-based, kRebaseWarp) per stage; 4 + 4 + 2 + 1
  // accumulator ones; the TMEM address and the abort flag
  static_assert(((kRebaseWarp ? 3 : 2) * kStages + 12) * 8 <= kBarBytes, "barrier bytes");
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kEpiBytes + kMaskBytes + kBarBytes;
  static constexpr uint32_t kColAcc = 0;
  static constexpr uint32_t kAccStride = OVL ? 192 : ((BN <= 128) ? 128 : 256);
  static constexpr uint32_t kColSfa = (kAccBufs - 1) * kAccStride + BN;  // even, 4-column aligned
  static constexpr uint32_t kColSfb = kColSfa + 4;
  static_assert(PROMO ? kAccBufs * kAccStride <= kTmemCols : kColSfb + 4 * kSfbChunks <= kTmemCols, "TMEM columns");
  // Instruction descriptor of kind::mxf8f6f4 with block scaling: A = E4M3,
  // B = E4M3 (0) or E2M1 (5), both K-major, UE8M0 scales, M = 128, N = BN.
  static constexpr uint32_t kIdescScaled = (0u << 7) | ((FP4 ? 5u : 0u) << 10) | ((uint32_t)(BN >> 3) << 17) |
                                           (1u << 23) | ((uint32_t)(kBM >> 4) << 24);
  // kind::f16: FP32 accumulator (bits 4-5 = 1), A and B bf16 (formats 1),
  // both K-major, N >> 3, M >> 4
  static constexpr uint32_t kIdescBf16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                         ((uint32_t)(kBM >> 4) << 24);
  // kind::f8f6f4 (promotion): FP32 accumulator, A and B E4M3, K-major
  static constexpr uint32_t kIdescPlain = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
  static constexpr uint32_t kIdesc = BF16 ? kIdescBf16 : (PROMO ? kIdescPlain : kIdescScaled);
};

template <bool B>
struct BoolC {
  static constexpr bool value = B;
};

struct Unit {
  int g, mb, nb;
  int kb0, kb1;   // K-blocks of this unit
  int slot;       // stream-K workspace slot, -1: the whole tile (result to D)
  int sk;         // stream-K tile index (slot >= 0)
  bool valid;
};

// Stream-K bookkeeping (host and device): the CTA whose share of the G-way
// even split of `iters` iterations contains iteration x, and the first
// iteration of CTA c.  Valid for iters >= G (every share non-empty).
__host__ __device__ __forceinline__ int sk_cta_of(long long x, int G, long long iters) {
  return (int)(((x + 1) * G - 1) / iters);
}
__host__ __device__ __forceinline__ long long sk_begin(int c, int G, long long iters) {
  return (long long)c * iters / G;
}

// (m-block, n-block) of tile tl in raster order: bands of `raster` m-blocks,
// m fastest inside a band, so that the CTAs running at the same time share
// the A rows and B columns of one band.
__host__ __device__ __forceinline__ void raster_tile(int tl, int raster, int num_m_blocks, int num_n_blocks,
                                                     int& mb, int& nb) {
  const int band_tiles = raster * num_n_blocks;
  const int band = tl / band_tiles;
  const int rem = tl - band * band_tiles;
  const int band_rows = min(raster, num_m_blocks - band * raster);
  mb = band * raster + rem % band_rows;
  nb = rem / band_rows;
}

// raster_tile with the band division precomputed (FastDiv) and the usual
// band height of 8 m-blocks done with a shift and a mask.
__device__ __forceinline__ void raster_tile_fast(int tl, const GemmArgs& a, int& mb, int& nb) {
  const int band = (int)a.band_div.div((uint32_t)tl);
  const int rem = tl - band * (int)a.band_div.d;
  const int band_rows = min(a.raster, a.num_m_blocks - band * a.raster);
  if (band_rows == 8) {
    mb = band * 8 + (rem & 7);
    nb = rem >> 3;
  } else {
    mb = band * a.raster + rem % band_rows;
    nb = rem / band_rows;
  }
}

// Work units of one CTA, in the order all three roles walk them.
// Dense: the whole tiles t = cta, cta + G, ... below dp_tiles, then this
// CTA's stream-K share cut at tile boundaries.  Contiguous: every tile of the
// raster order round robin (a tile's group from its first row).  Masked:
// group by group, n-blocks, m-blocks fastest (m-blocks of a group share its B
// tiles).  K-grouped: group by group, raster order inside a group; a unit's
// K-blocks are its group's (global K-block indices, from s_prefix).
template <int LAYOUT>
struct WorkIter {
  int t, step, cta;
  long long x, x_end;  // stream-K iterations of this CTA still to walk

  __device__ __forceinline__ WorkIter(const GemmArgs& a, int cta_, int G) : t(cta_), step(G), cta(cta_) {
    x = x_end = 0;
    if (LAYOUT == kDenseSplit) x_end = 1;  // one unit: this CTA's slice of its tile
    if (LAYOUT == kDense && a.sk_tiles > 0) {
      if (a.sk_split > 0) {
        x_end = (cta_ < a.sk_tiles * a.sk_split) ? 1 : 0;  // one piece
      } else {
        x = sk_begin(cta_, G, a.sk_iters);
        x_end = sk_begin(cta_ + 1, G, a.sk_iters);
      }
    }
  }

  __device__ __forceinline__ bool next(const GemmArgs& a, const int* s_prefix, int num_units, Unit& u) {
    u.valid = true;
    u.g = 0;
    u.slot = -1;
    u.sk = 0;
    u.kb0 = 0;
    u.kb1 = a.kb_total;
    if (LAYOUT == kDenseSplit) {
      if (x >= x_end) return false;
      const int r = cta % a.split;  // = the CTA's rank in its cluster
      raster_tile_fast(cta / a.split, a, u.mb, u.nb);
      u.kb0 = (int)((long long)r * a.kb_total / a.split);
      u.kb1 = (int)((long long)(r + 1) * a.kb_total / a.split);
      x = x_end;
      return true;
    }
    if (t < num_units) {
      if (LAYOUT == kMasked) {
        // the group whose tile range holds t: s_prefix[g] <= t < s_prefix[g + 1]
        int g = 0, hi = a.num_groups;
        while (hi - g > 1) {
          const int mid = (g + hi) >> 1;
          if (s_prefix[mid] <= t)
            g = mid;
          else
            hi = mid;
        }
        const int local = t - s_prefix[g];
        const int valid_rows = min(max(__ldg(a.masked_m + g), 0), a.rows);
        const int mcount = (valid_rows + kBM - 1) / kBM;
        u.g = g;
        u.nb = local / mcount;
        u.mb = local % mcount;
      } else if (LAYOUT == kKGrouped) {
        const int g = (int)a.group_div.div((uint32_t)t);
        raster_tile_fast(t - g * (int)a.group_div.d, a, u.mb, u.nb);
        u.g = g;
        u.kb0 = s_prefix[g];
        u.kb1 = s_prefix[g + 1];
      } else {
        raster_tile_fast(t, a, u.mb, u.nb);
        if (LAYOUT == kContig) {
          const int g = __ldg(a.m_indices + (long long)u.mb * kBM);  // 1-CTA tiles only
          u.g = g;
          u.valid = (g >= 0 && g < a.num_groups);
        }
      }
      t += step;
      return true;
    }
    if (LAYOUT != kDense || x >= x_end) return false;
    const int kbt = a.kb_total;
    if (a.sk_split > 0) {
      const int j = cta / a.sk_split;
      const int t = cta - j * a.sk_split;
      u.sk = j;
      u.slot = t;
      u.kb0 = (int)((long long)t * kbt / a.sk_split);
      u.kb1 = (int)((long long)(t + 1) * kbt / a.sk_split);
      raster_tile_fast(a.dp_tiles + j, a, u.mb, u.nb);
      x = x_end;
      return true;
    }
    const int j = (int)(x / kbt);
    u.sk = j;
    u.kb0 = (int)(x - (long long)j * kbt);
    const long long left = x_end - x;
    u.kb1 = (left < (long long)(kbt - u.kb0)) ? u.kb0 + (int)left : kbt;
    u.slot = cta - sk_cta_of((long long)j * kbt, step, a.sk_iters);
    raster_tile_fast(a.dp_tiles + j, a, u.mb, u.nb);
    x += u.kb1 - u.kb0;
    return true;
  }
};

// MAJ != kMajorK: A and/or B staged MN-major (NN, TN, TT layouts): each 128-wide
// M or N block of a stage is one TMA box of 128 elements x 128 K rows, and
// the MMA reads it through an MN-major descriptor (plain FP8 tiles of width
// 128 or 256 only).
template <int BN, bool FP4, int LAYOUT, int EPI = kEpiPlain, bool BF16 = false, int MAJ = kMajorK>
__global__ void __launch_bounds__(block_threads<BN, BF16>(), 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a32,
                const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_d,
                const __grid_constant__ CUtensorMap tm_c, const GemmArgs args) {
  static_assert(EPI == kEpiPlain || BN % (2 * kSwiGluBlock) == 0, "SwiGLU tiles hold whole block pairs");
  constexpr bool kPromo = (EPI == kEpiPromote);
  constexpr bool kOvl = (BN == 256 && EPI == kEpiPlain);
  using C = Cfg<BN, FP4, BF16, (LAYOUT == kMasked || LAYOUT == kKGrouped), kPromo, kOvl>;
  static_assert(!BF16 || EPI == kEpiPlain, "bf16: plain epilogue");
  static_assert(!kPromo || (LAYOUT == kDense && MAJ == kMajorK), "promotion: dense NT");
  constexpr bool kAMn = (MAJ & kAMajorMN) != 0;
  constexpr bool kBMn = (MAJ & kBMajorMN) != 0;
  static_assert(MAJ == kMajorK || (!FP4 && !BF16 && EPI == kEpiPlain && BN % 128 == 0),
                "MN-major operands: FP8, plain epilogue, 128-wide column blocks");
  static_assert(LAYOUT != kKGrouped || MAJ == (kAMajorMN | kBMajorMN), "k-grouped: A and B MN-major");
  // D and C of the masked and k-grouped layouts are [groups][rows][n]
  constexpr bool kGroupRows = (LAYOUT == kMasked || LAYOUT == kKGrouped);
  // split tiles: row pitch (floats) of a slice's partial sums in shared memory
  // (4 floats of padding put the rows of a warp's float4 stores in distinct banks)
  constexpr int kSplitPitch = BN + 4;
  static_assert(LAYOUT != kDenseSplit || kBM * kSplitPitch * 4 <= C::kStages * C::kStageBytes,
                "a split tile's partial sums fit in the stage ring");
  static_assert(LAYOUT != kDenseSplit || (EPI == kEpiPlain && MAJ == kMajorK), "split tiles: dense NT, plain");
  constexpr int S = C::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_a = smem;
  uint8_t* s_b = s_a + S * C::kABytes;
  uint8_t* s_sfa = s_b + S * C::kBBytes;
  uint8_t* s_sfb = s_sfa + S * C::kSfaBytes;
  uint8_t* s_sfr = s_sfb + S * C::kSfbBytes;   // re-based B scale words (kRebase only)
  uint8_t* s_epi = s_sfr + S * C::kSfrBytes;
  int* s_prefix = reinterpret_cast<int*>(s_epi + C::kEpiBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(s_prefix) + C::kMaskBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;       // [4]: accumulator buffer b holds a result
  uint64_t* tempty = bars + 2 * S + 4;  // [4]: the epilogue has read buffer b
  uint64_t* tovl = bars + 2 * S + 8;    // [2]: the epilogue has read the columns buffer b shares (kOvl)
  uint64_t* drain = bars + 2 * S + 10;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * S + 11);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  uint64_t* rb = bars + 2 * S + 12;     // [S]: the re-base warp is done with the stage (kRebaseWarp)
  constexpr int kBlockThreads = block_threads<BN, BF16>();
  static_assert(kBlockThreads == kThreads + (C::kRebaseWarp ? 32 : 0), "re-base warp");

  const int warp = threadIdx.x / 32;
  const uint32_t lane = lane_id();
  const GemmArgs& a = args;
  const int cta_id = blockIdx.x, num_ctas = gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 4; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps);
    }
    for (int b = 0; b < 2; ++b) mbar_init(&tovl[b], kEpiWarps / 2);  // the warps of one column half
    if constexpr (C::kRebaseWarp)
      for (int s = 0; s < S; ++s) mbar_init(&rb[s], 1);
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    if constexpr (!kAMn) prefetch_tmap(&tm_a32);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_d);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  // Prologue above touches no global memory; with programmatic dependent
  // launch it overlaps the previous kernel's tail.  Everything below may
  // read inputs the previous kernel wrote.
  pdl_wait();
  pdl_launch_dependents();
  int num_units;
  if (LAYOUT == kMasked) {
    // tiles per group, read from device memory (so the call stays
    // graph-capturable), then an exclusive prefix over the groups
    for (int g = threadIdx.x; g < a.num_groups; g += kBlockThreads) {
      int mm = __ldg(a.masked_m + g);
      if (mm < 0 || mm > a.rows) record_error(-5 /* DG_ERR_BAD_METADATA */);
      mm = min(max(mm, 0), a.rows);
      s_prefix[g + 1] = ((mm + kBM - 1) / kBM) * a.num_n_blocks;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      s_prefix[0] = 0;
      for (int g = 0; g < a.num_groups; ++g) s_prefix[g + 1] += s_prefix[g];
    }
  }
  if (LAYOUT == kKGrouped) {
    // K-blocks per group, read from device memory, then an exclusive prefix
    // (the first K-block of each group); K of a group must be a non-negative
    // multiple of 128 and the groups must fit in the K rows of A and B
    for (int g = threadIdx.x; g < a.num_groups; g += kBlockThreads) {
      int kk = __ldg(a.ks + g);
      if (kk < 0 || kk % kBK != 0) {
        record_error(-5 /* DG_ERR_BAD_METADATA */);
        kk = 0;
      }
      s_prefix[g + 1] = kk / kBK;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      s_prefix[0] = 0;
      for (int g = 0; g < a.num_groups; ++g) {
        int next = s_prefix[g] + s_prefix[g + 1];
        if (next > a.kb_total) {
          record_error(-5 /* DG_ERR_BAD_METADATA */);
          next = a.kb_total;
        }
        s_prefix[g + 1] = next;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  if (LAYOUT == kMasked)
    num_units = s_prefix[a.num_groups];
  else if (LAYOUT == kDense)
    num_units = a.dp_tiles;
  else if (LAYOUT == kKGrouped)
    num_units = a.num_groups * a.num_m_blocks * a.num_n_blocks;
  else
    num_units = a.num_m_blocks * a.num_n_blocks;

  const uint64_t limit = a.timeout_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t filled_phase[8];
      uint32_t filled_mask = 0;
      bool ok = true;
      WorkIter<LAYOUT> it(a, cta_id, num_ctas);
      Unit u;
      while (ok && it.next(a, s_prefix, num_units, u)) {
        if (LAYOUT == kContig && !u.valid) {
          if (u.g >= a.num_groups) record_error(-5);
          continue;
        }
        const int kb0 = u.kb0;
        const int kb1 = u.kb1;
        const int n0 = u.nb * BN;
        const int c0 = n0 / 128;
        const int c1 = (min(n0 + BN, a.n) - 1) / 128;
        const int nchunks = c1 - c0 + 1;
        const int a_row = u.mb * kBM;
        const int a_grp = (LAYOUT == kMasked) ? u.g : 0;
        const int b_grp = (LAYOUT == kDense || LAYOUT == kKGrouped) ? 0 : u.g;
        // MN-major B: the 128-wide column blocks of the tile that hold
        // columns below n (a block wholly past n is not loaded; the MMA
        // columns it feeds are never stored)
        const int b_blocks = kBMn ? min(BN / 128, (a.n - n0 + 127) / 128) : 1;
        // K-major A: a tile with fewer than 128 valid rows (an M tail, the
        // last block of a masked group) loads only the 32-row boxes that hold
        // them; the MMA's remaining rows read stale shared memory and feed
        // accumulator rows that are never stored
        int a_boxes = 4;
        if (!kAMn && a.a_trim) {
          int lim = a.rows;
          if (LAYOUT == kMasked) lim = min(max(__ldg(a.masked_m + u.g), 0), a.rows);
          a_boxes = max(1, min(4, (lim - a_row + 31) / 32));
        }
        const uint32_t a_bytes = (a_boxes == 4) ? (uint32_t)C::kABytes : (uint32_t)a_boxes * (32 * 128);
        const int32_t* sfa_g = a.sfa + (LAYOUT == kMasked ? (long long)u.g * a.sfa_group_words : 0);
        const int32_t* sfb_g = a.sfb + (long long)b_grp * a.sfb_group_words;
        // the K-loop in two versions, so that the untrimmed one (every full
        // tile) carries no per-K-block branch on the box count
        auto k_loop = [&](auto trim_c) {
          constexpr bool kTrim = decltype(trim_c)::value;
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!dg_wait(&empty[stage], phase ^ 1, s_abort, limit)) {
              ok = false;
              break;
            }
            const bool new_sfa = !BF16 && !kPromo && (((kb & 3) == 0) || kb == kb0);
            const bool new_sfb = !BF16 && !kPromo && (FP4 || new_sfa);
            uint32_t bytes = (kTrim ? a_bytes : (uint32_t)C::kABytes) +
                             (kBMn ? (uint32_t)b_blocks * (kBK * 128) : (uint32_t)C::kBTxBytes);
            if (new_sfa) bytes += C::kSfaBytes;
            if (new_sfb) bytes += 512u * nchunks;
            DG_CHECK(((smem_u32(s_a + stage * C::kABytes) | smem_u32(s_b + stage * C::kBBytes)) & 1023) == 0 &&
                         u.mb < a.num_m_blocks && u.nb < a.num_n_blocks && kb < a.kb_total,
                     6);
            mbar_arrive_expect_tx(&full[stage], bytes);
            if constexpr (kAMn) {
              tma_load_3d(s_a + stage * C::kABytes, &tm_a, &full[stage], a_row, kb * kBK, a_grp);
            } else if constexpr (!kTrim) {
              tma_load_3d(s_a + stage * C::kABytes, &tm_a, &full[stage], kb * C::kKPerStage, a_row, a_grp);
            } else {
              // 32-row boxes land 4 KB apart, at 1024-byte-aligned addresses,
              // so the 128-byte swizzle places their rows where one 128-row
              // box would
              for (int i = 0; i < a_boxes; ++i)
                tma_load_3d(s_a + stage * C::kABytes + i * (32 * 128), &tm_a32, &full[stage], kb * C::kKPerStage,
                            a_row + 32 * i, a_grp);
            }
            if constexpr (kBMn) {
              for (int cb = 0; cb < b_blocks; ++cb)
                tma_load_3d(s_b + stage * C::kBBytes + cb * (kBK * 128), &tm_b, &full[stage], n0 + 128 * cb, kb * kBK,
                            b_grp);
            } else {
              tma_load_3d(s_b + stage * C::kBBytes, &tm_b, &full[stage], kb * C::kKPerStage, n0, b_grp);
            }
            if (new_sfa) {
              const int32_t* src = sfa_g + ((long long)(kb >> 2) * a.sfa_chunks + u.mb) * 128;
              if (DG_CHECK(src >= a.sfa && src + 128 <= a.sfa + a.sfa_words &&
                               ((reinterpret_cast<uintptr_t>(src) | smem_u32(s_sfa + stage * C::kSfaBytes)) & 15) == 0,
                           4))
                bulk_load(s_sfa + stage * C::kSfaBytes, src, C::kSfaBytes, &full[stage]);
            }
            if (new_sfb) {
              const int q = FP4 ? kb : (kb >> 2);
              const int32_t* src = sfb_g + ((long long)q * a.sfb_chunks + c0) * 128;
              if (DG_CHECK(src >= a.sfb && src + 128 * nchunks <= a.sfb + a.sfb_words && nchunks >= 1 &&
                               nchunks <= C::kSfbChunks &&
                               ((reinterpret_cast<uintptr_t>(src) | smem_u32(s_sfb + stage * C::kSfbBytes)) & 15) == 0,
                           5))
                bulk_load(s_sfb + stage * C::kSfbBytes, src, 512u * nchunks, &full[stage]);
            }
            filled_phase[stage] = phase;
            filled_mask |= 1u << stage;
            if (++stage == S) {
              stage = 0;
              phase ^= 1;
            }
          }
        };
        if (a_boxes == 4)
          k_loop(BoolC<false>{});
        else
          k_loop(BoolC<true>{});
      }
      if (!ok) {
        // never leave copies in flight into shared memory: wait (bounded) for
        // the last fill of every stage
        for (int s = 0; s < S; ++s)
          if (filled_mask & (1u << s)) {
            uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(&full[s], filled_phase[s]) && global_timer_ns() - t0 < limit) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // One lane waits on the barriers and issues every tcgen05 operation (a
    // warp-wide loop with per-K-block warp synchronisation measured 1.8x
    // slower).  Where the re-base warp exists it also waits for that warp's
    // hand-over of each stage.
    if (kPromo && lane == 0) {
      // promotion: every K-block's four unscaled MMAs go to the next of the
      // rotating partial-sum buffers, which the epilogue scales and frees
      int stage = 0;
      uint32_t phase = 0;
      uint32_t kcount = 0;
      bool ok = true;
      WorkIter<LAYOUT> it(a, cta_id, num_ctas);
      Unit u;
      while (ok && it.next(a, s_prefix, num_units, u)) {
        for (int kb = u.kb0; kb < u.kb1; ++kb, ++kcount) {
          const int buf = (int)(kcount % C::kAccBufs);
          const uint32_t use = kcount / C::kAccBufs;
          if (!dg_wait(&tempty[buf], (use & 1) ^ 1, s_abort, limit) || !dg_wait(&full[stage], phase, s_abort, limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_t = tmem_base + C::kColAcc + buf * C::kAccStride;
          const uint64_t adesc = sdesc_k_sw128(s_a + stage * C::kABytes);
          const uint64_t bdesc = sdesc_k_sw128(s_b + stage * C::kBBytes);
#pragma unroll
          for (int ks = 0; ks < kBK / 32; ++ks)
            tc_mma_f8f6f4(d_t, adesc + (uint64_t)(2 * ks), bdesc + (uint64_t)(2 * ks), C::kIdesc, ks > 0 ? 1u : 0u);
          tc_commit(&empty[stage]);
          tc_commit(&tfull[buf]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      tc_commit(drain);
      uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < limit) {
      }
    } else if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      const uint32_t sfa_t = tmem_base + C::kColSfa;
      WorkIter<LAYOUT> it(a, cta_id, num_ctas);
      Unit u;
      while (ok && it.next(a, s_prefix, num_units, u)) {
        if (LAYOUT == kContig && !u.valid) continue;
        // a k-grouped tile of an empty group takes no accumulator: its
        // epilogue writes C (or zeros) alone
        if (LAYOUT == kKGrouped && u.kb0 == u.kb1) continue;
        const int kb0 = u.kb0;
        const int kb1 = u.kb1;
        const int n0 = u.nb * BN;
        const int nchunks = (min(n0 + BN, a.n) - 1) / 128 - n0 / 128 + 1;
        const int off = (n0 % 128) / 32;  // 32-row groups into the first scale chunk
        const bool rebase = C::kRebase && (off & 1);
        const uint32_t sfb_t = tmem_base + C::kColSfb + (uint32_t)(rebase ? 0 : off);
        const int buf = local % C::kAccBufs;
        const uint32_t use = (uint32_t)(local / C::kAccBufs);
        if (!dg_wait(&tempty[buf], (use & 1) ^ 1, s_abort, limit)) {
          ok = false;
          break;
        }
        // overlapping accumulators: the previous tile's epilogue must also have
        // read the 64 columns its buffer shares with this one
        if (kOvl && local > 0 && !dg_wait(&tovl[(local - 1) & 1], (uint32_t)((local - 1) >> 1) & 1u, s_abort, limit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_t = tmem_base + C::kColAcc + buf * C::kAccStride;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!dg_wait(&full[stage], phase, s_abort, limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if constexpr (BF16) {
            // 4 x (M=128, N=BN, K=16) per stage, 32 bytes of each row apart
            const uint64_t adesc = sdesc_k_sw128(s_a + stage * C::kABytes);
            const uint64_t bdesc = sdesc_k_sw128(s_b + stage * C::kBBytes);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              tc_mma_f16(d_t, adesc + (uint64_t)(ks * 2), bdesc + (uint64_t)(ks * 2), C::kIdesc,
                         (kb > kb0 || ks > 0) ? 1u : 0u);
            tc_commit(&empty[stage]);
            if (++stage == S) {
              stage = 0;
              phase ^= 1;
            }
            continue;
          }
          const bool new_sfa = ((kb & 3) == 0) || kb == kb0;
          const bool new_sfb = FP4 || new_sfa;
          const uint8_t* sfb_src = s_sfb + stage * C::kSfbBytes;
          const uint8_t* sfb_reb = s_sfr + stage * C::kSfrBytes;
          if constexpr (C::kRebaseWarp) {
            if (!dg_wait(&rb[stage], phase, s_abort, limit)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if (new_sfa) tc_cp_32x128b_x4(sfa_t, sdesc_sf_32x16(s_sfa + stage * C::kSfaBytes));
          if (new_sfb) {
            const int ncp = rebase ? C::kSfrChunks : nchunks;
            for (int ch = 0; ch < ncp; ++ch) {
              tc_cp_32x128b_x4(tmem_base + C::kColSfb + 4 * ch,
                               sdesc_sf_32x16((rebase ? sfb_reb : sfb_src) + ch * 512));
            }
          }
          // K-major: a K-step of 32 e4m3 is 32 bytes along the swizzled rows
          // (+2 in the 16-byte address field); MN-major: 32 rows of 128 bytes
          // (+256).  Bits 15 / 16 of the instruction descriptor mark A / B
          // as MN-major.
          const uint64_t adesc = kAMn ? sdesc_mn_sw128(s_a + stage * C::kABytes, 0)
                                      : sdesc_k_sw128(s_a + stage * C::kABytes);
          const uint64_t bdesc = kBMn ? sdesc_mn_sw128(s_b + stage * C::kBBytes, kBK * 128)
                                      : sdesc_k_sw128(s_b + stage * C::kBBytes);
          constexpr uint64_t kAStep = kAMn ? 256 : 2, kBStep = kBMn ? 256 : 2;
          constexpr uint32_t kMajBits = (kAMn ? 1u << 15 : 0u) | (kBMn ? 1u << 16 : 0u);
          const uint32_t ida = (uint32_t)(kb & 3);
#pragma unroll
          for (int ks = 0; ks < kBK / 32; ++ks) {
            const uint32_t idb = FP4 ? (uint32_t)ks : ida;
            const uint32_t idesc = C::kIdesc | kMajBits | (ida << 29) | (idb << 4);
            tc_mma_mxf8f6f4(d_t, adesc + kAStep * ks, bdesc + kBStep * ks, idesc, sfa_t | (ida << 30),
                            sfb_t | (idb << 30), (kb > kb0 || ks > 0) ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(&tfull[buf]);
        ++local;
      }
      // all tcgen05 work of this thread complete before TMEM is released
      tc_commit(drain);
      uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < limit) {
      }
    }
  } else if (C::kRebaseWarp && warp == 2 + kEpiWarps) {
    // ------------------------------------------------------------ scale re-base
    // A tile that starts an odd number of 32-row groups into its first 128-row
    // scale chunk reads its B scale words from a re-based copy (the MMA's
    // scale-factor address must be an even TMEM column): word w of line l of
    // re-based chunk v is word (off + w) % 4 of line l of loaded chunk
    // v + (off + w) / 4 (chunks past the loaded range only feed rows outside
    // the tile).  Lane l builds line l.  The warp walks every K-block of the
    // MMA lane's sequence, waiting on each stage's fill in order (so no
    // barrier phase is skipped) and handing the stage on through rb[], which
    // the MMA lane waits on before it copies the scales: the re-base runs
    // while the MMA lane is still working on earlier stages.
    if constexpr (C::kRebaseWarp) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      WorkIter<LAYOUT> it(a, cta_id, num_ctas);
      Unit u;
      while (ok && it.next(a, s_prefix, num_units, u)) {
        if (LAYOUT == kContig && !u.valid) continue;
        if (LAYOUT == kKGrouped && u.kb0 == u.kb1) continue;
        const int off = ((u.nb * BN) % 128) / 32;
        const bool rebase = (off & 1) != 0;
        for (int kb = u.kb0; kb < u.kb1; ++kb) {
          // every lane waits (a lane's own acquire of the fill), and the warp
          // leaves together if any lane gave up
          const bool got = dg_wait(&full[stage], phase, s_abort, limit);
          if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
          }
          const bool new_sfb = FP4 || ((kb & 3) == 0) || kb == u.kb0;
          if (rebase && new_sfb) {
            const uint8_t* src = s_sfb + stage * C::kSfbBytes + lane * 16;
            uint8_t* dst = s_sfr + stage * C::kSfrBytes + lane * 16;
            uint4 ld[C::kSfbChunks];
#pragma unroll
            for (int c = 0; c < C::kSfbChunks; ++c) ld[c] = *reinterpret_cast<const uint4*>(src + c * 512);
#pragma unroll
            for (int v = 0; v < C::kSfrChunks; ++v) {
              uint32_t w4[4];
#pragma unroll
              for (int w = 0; w < 4; ++w) {
                const int j = off + w;
                const uint4 q4 = ld[min(v + (j >> 2), C::kSfbChunks - 1)];
                const int e = j & 3;
                w4[w] = e == 0 ? q4.x : (e == 1 ? q4.y : (e == 2 ? q4.z : q4.w));
              }
              *reinterpret_cast<uint4*>(dst + v * 512) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            fence_proxy_async_smem();  // the copy is read by tcgen05.cp (async proxy)
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&rb[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Two warps per TMEM sub-partition: warp w reads lanes 32*(w%4).. and the
    // column half (w-2)/4 of the tile.  All C loads of a tile are issued into
    // registers before waiting for its accumulator, so they overlap the MMAs.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;             // column part of this warp (0 .. kEpiParts - 1)
    constexpr int kNch = BN / kEpiCols;           // 32-column chunks of the tile
    constexpr int kChunks = (kNch + kEpiParts - 1) / kEpiParts;  // chunks per part (the last may have fewer)
    constexpr int kCols = kChunks * kEpiCols;     // columns between parts
    const int nch_w = max(0, min(kChunks, kNch - half * kChunks));  // chunks of this warp
    uint8_t* stg = s_epi + (warp - 2) * (32 * 64);
    int local = 0;
    // C of one unit for this warp's 32 rows x kCols columns, loaded
    // coalesced: in load i the four lanes 4r..4r+3 read the four 16-byte
    // pieces of row 8i + r of each 32-column chunk, so one warp load covers 8
    // rows x 64 contiguous bytes (zeros where there is no C or no row).
    // dst[j][i] is piece (lane & 3) of row 8i + (lane >> 2) of chunk j;
    // stage_c() hands each lane its own row through the staging box.
    auto load_c_rows = [&](uint4 (&dst)[kChunks][4], const Unit& uu, bool want) {
#pragma unroll
      for (int j = 0; j < kChunks; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[j][i] = make_uint4(0u, 0u, 0u, 0u);
      if (!want) return;
      const int rr0 = uu.mb * kBM + q * 32;
      int lim = a.rows;
      if (LAYOUT == kMasked) lim = min(max(__ldg(a.masked_m + uu.g), 0), a.rows);
      const int cw = uu.nb * BN + half * kCols;
      const int seg = (int)(lane & 3);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int rrow = rr0 + 8 * i + (int)(lane >> 2);
        const long long rg = kGroupRows ? (long long)uu.g * a.rows + rrow : rrow;
        if (rrow < lim &&
            DG_CHECK(((reinterpret_cast<uintptr_t>(a.c + rg * a.n + cw) & 15) == 0) && rrow < a.rows && rg >= 0, 1)) {
          const uint4* src = reinterpret_cast<const uint4*>(a.c + rg * a.n + cw) + seg;
#pragma unroll
          for (int j = 0; j < kChunks; ++j)
            if (j < nch_w && cw + j * kEpiCols + 8 * seg < a.n) dst[j][i] = __ldg(src + j * 4);
        }
      }
    };
    // C of chunk j (as loaded by load_c_rows) into the staging box, in the
    // swizzled layout the D store uses; each lane then reads its own row's
    // pieces back while converting, and the bf16 result overwrites them
    auto stage_c = [&](const uint4 (&cj)[4]) {
      if (lane == 0) bulk_wait_group_read<0>();  // the previous TMA store has read the box
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int rw = 8 * i + (int)(lane >> 2);
        const int pos = (int)(lane & 3) ^ ((rw >> 1) & 3);
        *reinterpret_cast<uint4*>(stg + rw * 64 + pos * 16) = cj[i];
      }
      __syncwarp();
    };
    // bf16 result of one 32-column chunk of the 32 rows r0 .. r0 + 31 (vr of
    // them valid, below `lim`; group g of a grouped D) -> D
    auto store_rows = [&](int col0, const uint32_t (&packed)[kEpiCols / 2], int r0, int vr, int g, int lim) {
      const int row = r0 + (int)lane;
      const long long grow = kGroupRows ? (long long)g * a.rows + row : row;
      if (vr == 32) {
        // full 32-row box: swizzled staging (64-byte rows) + TMA store
        // 64-byte swizzle: the pattern XORs address bits 7-8 into 4-5, so the
        // staging box needs 512-byte alignment
        DG_CHECK((smem_u32(stg) & 511) == 0 && stg >= s_epi && stg + 2048 <= s_epi + C::kEpiBytes &&
                     (col0 % 8) == 0 && r0 + 32 <= lim,
                 7);
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int pos = ch ^ ((lane >> 1) & 3);
          *reinterpret_cast<uint4*>(stg + lane * 64 + pos * 16) =
              make_uint4(packed[4 * ch], packed[4 * ch + 1], packed[4 * ch + 2], packed[4 * ch + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tm_d, stg, col0, r0, kGroupRows ? g : 0);
          bulk_commit_group();
        }
      } else if ((int)lane < vr &&
                 DG_CHECK((reinterpret_cast<uintptr_t>(a.d + grow * a.d_cols + col0) & 15) == 0 && row < lim, 2)) {
        // partial box (M tail or masked group tail): predicated row stores
        uint4* dst = reinterpret_cast<uint4*>(a.d + grow * a.d_cols + col0);
#pragma unroll
        for (int v = 0; v < kEpiCols / 8; ++v)
          if (col0 + 8 * v < a.d_cols)
            dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
      }
    };
    // D = bf16(acc + C) of one 32-column chunk: C (when given) comes from the
    // staging box, where stage_c put it; the result overwrites it in place
    auto add_c_pack = [&](const float (&acc)[kEpiCols], bool with_c, uint32_t (&packed)[kEpiCols / 2]) {
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 c4 = with_c ? *reinterpret_cast<const uint4*>(stg + lane * 64 + ((v ^ ((lane >> 1) & 3)) * 16))
                                : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t cw[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int i = 4 * v + h;
          __nv_bfloat162 bv = __floats2bfloat162_rn(acc[2 * i] + __uint_as_float(cw[h] << 16),
                                                    acc[2 * i + 1] + __uint_as_float(cw[h] & 0xFFFF0000u));
          packed[i] = *reinterpret_cast<uint32_t*>(&bv);
        }
      }
    };
    // one unit of look-ahead for C where registers allow
    constexpr bool kPrefetchC = (kChunks <= 3);
    uint4 cnext[kChunks][4];
    bool have_next_c = false;  // cnext holds C of the next unit this warp drains
    (void)cnext;
    auto release_acc = [&](int b) { mbar_arrive(&tempty[b]); };
    // the iterator runs one unit ahead, so each unit is decoded once and the
    // next unit (un) is known for the C prefetch
    if constexpr (kPromo) {
      // ---- promotion: for every K-block, read this warp's 32 rows x kCols
      // columns of unscaled partial sums from TMEM, hand the buffer back to
      // the MMA issuer, and add the partial times sa * sb into FP32
      // registers (sa: the row's 1x128 code, sb: the 128x128 block's code);
      // after the unit's last K-block, D = bf16(acc + C) as in the plain
      // epilogue (or the FP32 sums to a workspace slot for a shared tile)
      WorkIter<LAYOUT> it(a, cta_id, num_ctas);
      Unit u;
      uint32_t kcount = 0;
      bool ok = true;
      while (ok && it.next(a, s_prefix, num_units, u)) {
        const int r0 = u.mb * kBM + q * 32;
        const int vr = min(32, a.rows - r0);
        const int colw = u.nb * BN + half * kCols;
        const bool load_c = a.c != nullptr && u.slot < 0;
        uint4 creg[kChunks][4];
        load_c_rows(creg, u, load_c);
        float acc[kChunks][kEpiCols];
#pragma unroll
        for (int j = 0; j < kChunks; ++j)
#pragma unroll
          for (int i = 0; i < kEpiCols; ++i) acc[j][i] = 0.f;
        // this row's packed A word and the B block's word (the same for all
        // rows of a 128-row block) of K-block group g4; the next group's
        // words are loaded one group ahead
        const int32_t* sfa_row = a.sfa + (long long)u.mb * 128 + lane * 4 + q;
        const int32_t* sfb_blk = a.sfb + (long long)(colw / 128) * 128;
        auto load_scales = [&](int g4, uint32_t& sa, uint32_t& sb) {
          sa = (uint32_t)__ldg(sfa_row + (long long)g4 * a.sfa_chunks * 128);
          sb = colw < a.n ? (uint32_t)__ldg(sfb_blk + (long long)g4 * a.sfb_chunks * 128) : 0x7F7F7F7Fu;
        };
        uint32_t sa_w, sb_w, sa_n = 0, sb_n = 0;
        load_scales(u.kb0 >> 2, sa_w, sb_w);
        if (((u.kb0 >> 2) + 1) * 4 < u.kb1) load_scales((u.kb0 >> 2) + 1, sa_n, sb_n);
        for (int kb = u.kb0; kb < u.kb1; ++kb, ++kcount) {
          if (kb > u.kb0 && (kb & 3) == 0) {
            sa_w = sa_n;
            sb_w = sb_n;
            if (kb + 4 < u.kb1) load_scales((kb >> 2) + 1, sa_n, sb_n);
          }
          const int buf = (int)(kcount % C::kAccBufs);
          const uint32_t use = kcount / C::kAccBufs;
          int okw = 1;
          if (lane == 0) okw = dg_wait(&tfull[buf], use & 1, s_abort, limit) ? 1 : 0;
          okw = __shfl_sync(0xffffffffu, okw, 0);
          if (!okw) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + C::kColAcc + buf * C::kAccStride +
                                 (uint32_t)(half * kCols);
          const int sh = 8 * (kb & 3);
          const float scale = ue8m0_to_float((sa_w >> sh) & 0xFFu) * ue8m0_to_float((sb_w >> sh) & 0xFFu);
          // both chunks' loads in flight at once, one wait, then the buffer
          // goes back to the MMA issuer before the FMAs
          uint32_t part[kChunks][kEpiCols];
#pragma unroll
          for (int j = 0; j < kChunks; ++j) tc_ld_32x32b_x32(t_row + j * kEpiCols, part[j]);
#pragma unroll
          for (int j = 0; j < kChunks; ++j) tc_wait_ld_regs(part[j]);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
#pragma unroll
          for (int j = 0; j < kChunks; ++j)
#pragma unroll
            for (int i = 0; i < kEpiCols; ++i) acc[j][i] = fmaf(scale, __uint_as_float(part[j][i]), acc[j][i]);
        }
        if (!ok) break;
        if (u.slot >= 0) {
          // a piece of a shared tile: FP32 sums to its workspace slot
          float* tile_ws = a.ws + ((long long)u.sk * a.max_seg + u.slot) * (kBM * BN);
#pragma unroll
          for (int j = 0; j < kChunks; ++j) {
            const int col0 = colw + j * kEpiCols;
            float* dst_row = tile_ws + (q * 32 + (int)lane) * BN + (col0 - u.nb * BN);
            if (j < nch_w && (int)lane < vr && col0 < a.n &&
                DG_CHECK(a.ws != nullptr && u.sk < a.sk_tiles && u.slot < a.max_seg &&
                             (reinterpret_cast<uintptr_t>(dst_row) & 15) == 0,
                         3)) {
#pragma unroll
              for (int v = 0; v < kEpiCols / 4; ++v)
                if (col0 + 4 * v < a.n)
                  reinterpret_cast<float4*>(dst_row)[v] =
                      make_float4(acc[j][4 * v], acc[j][4 * v + 1], acc[j][4 * v + 2], acc[j][4 * v + 3]);
            }
          }
          continue;
        }
#pragma unroll
        for (int j = 0; j < kChunks; ++j) {
          const int col0 = colw + j * kEpiCols;
          if (j < nch_w && vr > 0 && col0 < a.n) {
            if (load_c) stage_c(creg[j]);
            uint32_t packed[kEpiCols / 2];
            add_c_pack(acc[j], load_c, packed);
            store_rows(col0, packed, r0, vr, 0, a.rows);
          }
        }
      }
    } else {
    WorkIter<LAYOUT> it(a, cta_id, num_ctas);
    Unit u, un;
    bool has_un = it.next(a, s_prefix, num_units, un);
    while (has_un) {
      u = un;
      has_un = it.next(a, s_prefix, num_units, un);
      if constexpr (!kPrefetchC && EPI == kEpiPlain && LAYOUT != kDenseSplit) {
        // no register room for the next unit's C here (four chunks a warp):
        // where a unit's K loop is too short to hide C's HBM latency, bring
        // this warp's part of the next unit's C into L2 a whole unit ahead
        if (lane == 0 && a.c_prefetch && a.c != nullptr && has_un && un.valid && un.slot < 0) {
          const int rn = un.mb * kBM + q * 32;
          const int cn = un.nb * BN + half * kCols;
#pragma unroll
          for (int j = 0; j < kChunks; ++j)
            if (j < nch_w && cn + j * kEpiCols < a.n) tma_prefetch_3d(&tm_c, cn + j * kEpiCols, rn, kGroupRows ? un.g : 0);
        }
      }
      if (LAYOUT == kContig && !u.valid) continue;
      const int buf = local % C::kAccBufs;
      const uint32_t use = (uint32_t)(local / C::kAccBufs);
      const int r0 = u.mb * kBM + q * 32;  // first row of this warp (in the group if masked)
      int limit_rows = a.rows;
      if (LAYOUT == kMasked) limit_rows = min(max(__ldg(a.masked_m + u.g), 0), a.rows);
      const int vr = min(32, limit_rows - r0);
      const int row = r0 + (int)lane;
      const long long grow = kGroupRows ? (long long)u.g * a.rows + row : row;
      (void)grow;
      // k-grouped tile of an empty group: no accumulator, D = C (or 0)
      const bool empty_k = (LAYOUT == kKGrouped) && u.kb0 == u.kb1;
      const int colw = u.nb * BN + half * kCols;  // first column of this warp

      uint4 creg[kChunks][4];
      // (a split tile adds C when its slices are summed, after the loop)
      const bool load_c = a.c != nullptr && u.slot < 0 && LAYOUT != kDenseSplit;
      if constexpr (kPrefetchC) {
        if (have_next_c) {
          // C of this unit was loaded while the previous unit was stored
#pragma unroll
          for (int j = 0; j < kChunks; ++j)
#pragma unroll
            for (int v = 0; v < 4; ++v) creg[j][v] = cnext[j][v];
        } else {
          load_c_rows(creg, u, load_c);
        }
        // issue the loads of the next unit's C now, so that they arrive while
        // this unit is drained and stored
        have_next_c = false;
        if (a.c != nullptr && has_un && un.valid && un.slot < 0) {
          load_c_rows(cnext, un, true);
          have_next_c = true;
        }
      } else {
        load_c_rows(creg, u, load_c);
      }
      if constexpr (LAYOUT == kContig) {
        // The contiguous layout's precondition, checked once per m-block (on
        // its first n-block) while the MMAs run: every row of a 128-row
        // block carries the block's group (from its first row) or -1, and
        // padding rows (-1) only follow the valid rows.  A block that mixes
        // groups, or has a valid row after a padding row, is reported.
        if (u.nb == 0 && half == 0) {
          const int v = __ldg(a.m_indices + row);
          const int next = (lane == 31 && q < 3) ? __ldg(a.m_indices + row + 1) : v;
          const uint32_t pad = __ballot_sync(0xffffffffu, v == -1);
          const uint32_t valid_rows = ~pad;  // must be lanes 0 .. j-1 only
          const bool mixed = (v != u.g && v != -1) || (v == -1 && next != -1);
          if (__any_sync(0xffffffffu, mixed) || (valid_rows & (valid_rows + 1u)) != 0u) {
            if (lane == 0) record_error(-5 /* DG_ERR_BAD_METADATA */);
          }
        }
      }

      int ok = 1;
      if (lane == 0 && !empty_k) ok = dg_wait(&tfull[buf], use & 1, s_abort, limit) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + C::kColAcc + buf * C::kAccStride +
                             (uint32_t)(half * kCols);

      // bf16 result of one 32-column chunk of this warp's rows -> D
      auto store_chunk = [&](int col0, const uint32_t (&packed)[kEpiCols / 2]) {
        store_rows(col0, packed, r0, vr, u.g, limit_rows);
      };

      if constexpr (LAYOUT == kDenseSplit) {
        // ---- this CTA's K-slice of a split tile: its FP32 sums go to this
        // CTA's shared memory (the stage ring, idle once the last MMA has
        // completed), [kBM][BN + 4] floats; they are summed after the loop
        float* part = reinterpret_cast<float*>(smem) + (q * 32 + (int)lane) * kSplitPitch + half * kCols;
#pragma unroll
        for (int j = 0; j < kChunks; ++j) {
          if (j < nch_w) {
            uint32_t acc[kEpiCols];
            tc_ld_32x32b_x32(t_row + j * kEpiCols, acc);
            tc_wait_ld_regs(acc);
#pragma unroll
            for (int v = 0; v < kEpiCols / 4; ++v)
              *reinterpret_cast<float4*>(part + j * kEpiCols + 4 * v) =
                  make_float4(__uint_as_float(acc[4 * v]), __uint_as_float(acc[4 * v + 1]),
                              __uint_as_float(acc[4 * v + 2]), __uint_as_float(acc[4 * v + 3]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (kOvl && half == (buf == 0 ? 1 : 0)) mbar_arrive(&tovl[buf]);
          release_acc(buf);
        }
        ++local;
        continue;
      }

      if (u.slot >= 0) {
        // ---- stream-K piece: FP32 partial sums of kb0..kb1 into the tile's
        // workspace slot; sk_reduce_kernel adds the slots in K order (+C)
        // and writes D
        float* tile_ws = a.ws + ((long long)u.sk * a.max_seg + u.slot) * (kBM * BN);
#pragma unroll
        for (int j = 0; j < kChunks; ++j) {
          const int col0 = colw + j * kEpiCols;
          if (j < nch_w && vr > 0 && col0 < a.n) {
            uint32_t acc[kEpiCols];
            tc_ld_32x32b_x32(t_row + j * kEpiCols, acc);
            tc_wait_ld_regs(acc);
            float* dst_row = tile_ws + (q * 32 + (int)lane) * BN + (col0 - u.nb * BN);
            if ((int)lane < vr &&
                DG_CHECK(a.ws != nullptr && u.sk < a.sk_tiles && u.slot < a.max_seg && row < a.rows &&
                             (reinterpret_cast<uintptr_t>(dst_row) & 15) == 0,
                         3)) {
              float4* dst = reinterpret_cast<float4*>(dst_row);
#pragma unroll
              for (int v = 0; v < kEpiCols / 4; ++v)
                if (col0 + 4 * v < a.n)
                  dst[v] = make_float4(__uint_as_float(acc[4 * v]), __uint_as_float(acc[4 * v + 1]),
                                       __uint_as_float(acc[4 * v + 2]), __uint_as_float(acc[4 * v + 3]));
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (kOvl && half == (buf == 0 ? 1 : 0)) mbar_arrive(&tovl[buf]);
          release_acc(buf);
        }
        ++local;
        continue;
      }

      if constexpr (EPI == kEpiSwiGlu) {
        // ---- SwiGLU: the tile's BN columns are BN / 128 pairs of 64 gate and
        // 64 up columns; its BN / 2 output columns are cut into 32-column
        // chunks, the first half of them for warp half 0.  Output chunk c
        // reads gate chunk 4 (c / 2) + c % 2 and up chunk 4 (c / 2) + 2 + c % 2.
        constexpr int kOutCh = BN / (2 * kEpiCols);
        constexpr int kOutPer = (kOutCh + kEpiParts - 1) / kEpiParts;
        const uint32_t t_tile = tmem_base + ((uint32_t)(q * 32) << 16) + C::kColAcc + buf * C::kAccStride;
#pragma unroll
        for (int e = 0; e < kOutPer; ++e) {
          const int c = half * kOutPer + e;
          const int col0 = u.nb * (BN / 2) + c * kEpiCols;
          if (c < kOutCh && vr > 0 && col0 < a.d_cols) {
            const int gch = 4 * (c >> 1) + (c & 1);
            uint32_t g[kEpiCols], up[kEpiCols];
            DG_CHECK(((t_tile & 0xFFFF) + (gch + 2) * kEpiCols + kEpiCols <= (uint32_t)kTmemCols), 8);
            tc_ld_32x32b_x32(t_tile + gch * kEpiCols, g);
            tc_ld_32x32b_x32(t_tile + (gch + 2) * kEpiCols, up);
            tc_wait_ld_regs(g);
            tc_wait_ld_regs(up);
            uint32_t packed[kEpiCols / 2];
#pragma unroll
            for (int i = 0; i < kEpiCols / 2; ++i) {
              const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
              const float s0 = g0 / (1.0f + __expf(-g0)), s1 = g1 / (1.0f + __expf(-g1));
              __nv_bfloat162 bv =
                  __floats2bfloat162_rn(s0 * __uint_as_float(up[2 * i]), s1 * __uint_as_float(up[2 * i + 1]));
              packed[i] = *reinterpret_cast<uint32_t*>(&bv);
            }
            store_chunk(col0, packed);
          }
        }
      } else {
        // one 32-column chunk j of this warp's columns: TMEM -> +C -> bf16 -> D
        auto plain_chunk = [&](int j) {
          const int col0 = colw + j * kEpiCols;
          if (j < nch_w && vr > 0 && col0 < a.n) {
            uint32_t acc[kEpiCols];
            DG_CHECK(((t_row & 0xFFFF) + j * kEpiCols + kEpiCols <= (uint32_t)kTmemCols) &&
                         ((t_row >> 16) & 0xFFFF) == (uint32_t)(q * 32) + (tmem_base >> 16) && (warp & 3) == q,
                     8);
            if (!empty_k) {
              tc_ld_32x32b_x32(t_row + j * kEpiCols, acc);
            } else {
#pragma unroll
              for (int i = 0; i < kEpiCols; ++i) acc[i] = 0u;
            }
            if (load_c) stage_c(creg[j]);
            if (!empty_k) tc_wait_ld_regs(acc);
            uint32_t packed[kEpiCols / 2];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint4 c4 = load_c ? *reinterpret_cast<const uint4*>(stg + lane * 64 + ((v ^ ((lane >> 1) & 3)) * 16))
                                      : make_uint4(0u, 0u, 0u, 0u);
              const uint32_t cw[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const int i = 4 * v + h;
                __nv_bfloat162 bv = __floats2bfloat162_rn(__uint_as_float(acc[2 * i]) + __uint_as_float(cw[h] << 16),
                                                          __uint_as_float(acc[2 * i + 1]) +
                                                              __uint_as_float(cw[h] & 0xFFFF0000u));
                packed[i] = *reinterpret_cast<uint32_t*>(&bv);
              }
            }
            store_chunk(col0, packed);
          }
        };
        if constexpr (kOvl) {
          // the 64 columns this buffer shares with the other one are drained
          // first and reported (tovl), so the next tile's MMAs can start:
          // buffer 0 shares tile columns 192..255 (chunks 2, 3 of column
          // half 1), buffer 1 tile columns 0..63 (chunks 0, 1 of half 0)
          static_assert(kChunks == 4, "256-wide tiles: four chunks per warp");
          const bool owner = (half == (buf == 0 ? 1 : 0));
          auto shared_drained = [&]() {
            if (empty_k) return;  // (a tile of an empty group took no accumulator)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tovl[buf]);
          };
          if (owner && buf == 0) {
            plain_chunk(2);
            plain_chunk(3);
            shared_drained();
            plain_chunk(0);
            plain_chunk(1);
          } else {
            plain_chunk(0);
            plain_chunk(1);
            if (owner) shared_drained();
            plain_chunk(2);
            plain_chunk(3);
          }
        } else {
#pragma unroll
          for (int j = 0; j < kChunks; ++j) plain_chunk(j);
        }
      }  // plain epilogue
      if (empty_k) continue;  // (no accumulator taken)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) release_acc(buf);
      ++local;
    }
    }  // (kPromo)
    if constexpr (LAYOUT == kDenseSplit) {
      // ---- the slices of this CTA's tile lie in the shared memory of the
      // cluster's CTAs (slice r in CTA r).  Once every CTA has written its
      // own, CTA r sums rows [r kBM / S, (r + 1) kBM / S) of the tile (integer
      // division: any S from 2 to 8) over the slices in slice (= K) order,
      // adds C and writes D; the second cluster barrier keeps every CTA's
      // slice alive until the others have read it.
      cluster_sync_all();
      const int splits = a.split;
      const uint32_t rank = cluster_ctarank();
      int mb, nb;
      raster_tile_fast((int)blockIdx.x / splits, a, mb, nb);
      const int lr0 = (int)rank * kBM / splits;  // this CTA's rows [lr0, lr1) of the tile
      const int band = ((int)rank + 1) * kBM / splits - lr0;
      constexpr int kQ = BN / 4;  // float4 columns of a tile row
      const float* part = reinterpret_cast<const float*>(smem);
      for (int it = (int)threadIdx.x - 64; it < band * kQ; it += 32 * kEpiWarps) {
        const int lr = lr0 + it / kQ;
        const int c4 = it % kQ;
        const int row = mb * kBM + lr, col = nb * BN + 4 * c4;
        if (row >= a.rows || col >= a.n) continue;
        uint2 cw = make_uint2(0u, 0u);
        if (a.c != nullptr) cw = __ldg(reinterpret_cast<const uint2*>(a.c + (long long)row * a.n + col));
        const float* src = part + lr * kSplitPitch + 4 * c4;
        float4 v[8];
#pragma unroll
        for (int r = 0; r < 8; ++r)
          if (r < splits) v[r] = ld_shared_cluster_f4(mapa_shared(src, (uint32_t)r));
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < 8; ++r)
          if (r < splits) {
            acc.x += v[r].x;
            acc.y += v[r].y;
            acc.z += v[r].z;
            acc.w += v[r].w;
          }
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x + __uint_as_float(cw.x << 16),
                                                  acc.y + __uint_as_float(cw.x & 0xFFFF0000u));
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z + __uint_as_float(cw.y << 16),
                                                  acc.w + __uint_as_float(cw.y & 0xFFFF0000u));
        *reinterpret_cast<uint2*>(a.d + (long long)row * a.n + col) =
            make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
      }
      cluster_sync_all();
    }
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  if constexpr (LAYOUT == kDenseSplit) {
    // the producer and MMA warps take part in the epilogue's two cluster
    // barriers (every thread of the cluster arrives at each)
    if (warp < 2) {
      __syncwarp();
      cluster_sync_all();
      cluster_sync_all();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Stream-K fix-up: for every stream-K tile, D = bf16(sum of its workspace
// slots in slot (= K) order + C), so the result does not depend on timing.
// One thread per 4 columns of a tile row; the slots are loaded 8 at a time
// before they are added.
struct SkReduceArgs {
  const float* ws;
  const uint16_t* c;
  uint16_t* d;
  int rows, n, bn;
  int kb_total, dp_tiles, sk_tiles, max_seg, sk_split, ctas;
  long long sk_iters;
  int raster, num_m_blocks, num_n_blocks;
};

__global__ void __launch_bounds__(256) sk_reduce_kernel(const SkReduceArgs r) {
  pdl_wait();
  const int q4 = r.bn / 4;
  const int per_tile = kBM * q4;
  const int items = r.sk_tiles * per_tile;  // < 2^31: at most 4 x 148 tiles of 128 x 256
  const long long slot4 = (long long)kBM * r.bn / 4;  // float4s between slots
  for (int it = blockIdx.x * blockDim.x + threadIdx.x; it < items; it += gridDim.x * blockDim.x) {
    const int j = it / per_tile;
    const int rem = it - j * per_tile;
    const int lr = rem / q4;
    const int lc = (rem - lr * q4) * 4;
    int mb, nb;
    raster_tile(r.dp_tiles + j, r.raster, r.num_m_blocks, r.num_n_blocks, mb, nb);
    const int row = mb * kBM + lr;
    const int col = nb * r.bn + lc;
    if (row >= r.rows || col >= r.n) continue;
    // C first, so its load overlaps the slots'
    uint2 cw = make_uint2(0u, 0u);
    if (r.c != nullptr) cw = __ldg(reinterpret_cast<const uint2*>(r.c + (long long)row * r.n + col));
    int nseg = r.sk_split;
    if (nseg == 0) {
      const long long x0 = (long long)j * r.kb_total;
      nseg = sk_cta_of(x0 + r.kb_total - 1, r.ctas, r.sk_iters) - sk_cta_of(x0, r.ctas, r.sk_iters) + 1;
    }
    const float4* p = reinterpret_cast<const float4*>(r.ws + ((long long)j * r.max_seg * kBM + lr) * r.bn + lc);
    float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
    for (int s0 = 0; s0 < nseg; s0 += 8) {
      float4 part[8];
#pragma unroll
      for (int s = 0; s < 8; ++s)
        part[s] = (s0 + s < nseg) ? __ldcg(p + (s0 + s) * slot4) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        acc0 += part[s].x;
        acc1 += part[s].y;
        acc2 += part[s].z;
        acc3 += part[s].w;
      }
    }
    acc0 += __uint_as_float(cw.x << 16);
    acc1 += __uint_as_float(cw.x & 0xFFFF0000u);
    acc2 += __uint_as_float(cw.y << 16);
    acc3 += __uint_as_float(cw.y & 0xFFFF0000u);
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc0, acc1), hi = __floats2bfloat162_rn(acc2, acc3);
    *reinterpret_cast<uint2*>(r.d + (long long)row * r.n + col) =
        make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
  }
}

}  // namespace dg
