/*
 * dg.h -- C ABI of the B200 (sm_100a) fine-grained-scaled low-precision GEMM
 * library:  D = C + A * B^T.
 *
 * Problem statement (sources are cited by page title and section):
 *   - "DeepGEMM：统一高性能张量核心 GEMM 计算库编译与使用指南" (zhouruolin.cn),
 *     section 五 "使用方法": the naming convention D = C + A @ B with the NT
 *     layout (A [M,K] not transposed, B [N,K] transposed, both K-major); SM100
 *     takes packed UE8M0 scale factors; grouping only along M with N and K
 *     shared (contiguous layout for prefill / training forward, masked layout
 *     for decoding); utilities set_num_sms / get_num_sms and
 *     get_mk_alignment_for_contiguous_layout.
 *   - "DeepSeek 开源第三弹 ... DeepGEMM" (app.myzaker.com), section "DeepGEMM":
 *     FP8 with the fine-grained scaling of DeepSeek-V3 -- one scale per 1x128
 *     row-group of A, one per 128x128 block of B; FP32 accumulation.
 *   - "DeepSeek 发布 DeepGEMM 重大更新" (linlog.top), section "FP4 精度支持":
 *     FP8 x FP4 GEMM, FP4 weights with UE8M0 scales packed 4 per int32.
 *   - "DeepGEMM：FP8 GEMM 与 Mega-MoE" (charles2530.github.io), sections
 *     "难点解释" (the scale layout is part of the interface) and "四、在 MoE
 *     Serving 里的位置" (masked layout is CUDA-Graph friendly).
 *
 * Data types.  "e4m3": OCP FP8 E4M3FN codes, one byte each.  "e2m1": OCP FP4
 * E2M1 codes packed two per byte along K, low nibble = even k.  "ue8m0": one
 * byte e meaning 2^(e-127).  "bf16": bfloat16 bit patterns.  Accumulation is
 * FP32; D is C + A*B^T rounded once to bf16 (round to nearest even).
 *
 * Packed scale layout ("sf words").  Scale codes of a matrix with R rows and
 * G scale columns along K are packed into int32 words, 4 codes per word:
 *     words[Q][ceil(R/128)][128],  Q = ceil(G/4);
 *     the word of (row r, word-group q) is words[q][r/128][(r%32)*4 + (r%128)/32]
 *     and its byte j (little endian) is the code of scale column 4q+j;
 *     unused bytes hold 127.
 * dg_pack_sf() produces it; dg_packed_sf_words() gives its length.  For e4m3
 * operands the scale columns are the K/128 blocks (B's 128x128 block scales
 * are expanded to one copy per row by dg_pack_sf with row_div = 128); for the
 * e2m1 operand they are the K/32 groups.  Grouped operands store one packed
 * block per group, back to back.
 *
 * Pointers.  Every matrix / scale / index pointer is a DEVICE pointer owned
 * by the caller, 16-byte aligned, and may not alias an output (except C == D
 * for in-place accumulation in the dense calls).  `stream` is a cudaStream_t
 * (NULL = the legacy default stream).  Every call is asynchronous and
 * stream-ordered; none synchronises the host, except dg_get_last_error.
 *
 * Errors.  Argument checks happen on the host before anything is launched
 * and return DG_ERR_INVALID_ARG (nothing is written).  A launch failure
 * returns DG_ERR_CUDA.  Conditions only the device can see (a wait that ran
 * past its time limit, group metadata out of range) are recorded in a
 * device-side error word and reported later by dg_get_last_error().
 *
 * Scratch memory.  When the host heuristic shares the K-iterations of some
 * tiles out over several CTAs of a launch (per-tile K-slices or stream-K,
 * mostly the last partial wave of tiles), the dense calls keep their FP32
 * partial sums in a workspace per (device, stream), allocated stream-ordered
 * on first use and grown on demand; dg_shutdown() releases it.  A dense plan
 * that splits every tile over a thread-block cluster (small M) sums the
 * partials in the cluster's shared memory and needs none.  No other call
 * allocates device memory.
 */
#ifndef DG_H_
#define DG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = -1,   /* rejected on the host, nothing launched        */
  DG_ERR_UNSUPPORTED = -2,   /* valid but not implemented (e.g. no sm_100a)   */
  DG_ERR_CUDA = -3,          /* a CUDA runtime call or launch failed          */
  DG_ERR_TIMEOUT = -4,       /* a device wait ran past its limit (reported by
                                dg_get_last_error)                            */
  DG_ERR_BAD_METADATA = -5,  /* masked_m outside [0, max_m] or m_indices >=
                                num_groups, seen on the device                */
  DG_ERR_SCRATCH_LIMIT = -6  /* reserved: a plan needing more scratch than
                                the fixed no-alloc array (not returned by this
                                version, whose no-alloc planner keeps within
                                the array)                                    */
} dg_status;

/* ---------------------------------------------------------------- GEMMs */

/* Dense NT FP8 GEMM: D[M,N] = C + A * B^T.
 *   a    e4m3 [m][k] row-major          sfa  sf words of A: R = m, G = k/128
 *   b    e4m3 [n][k] row-major          sfb  sf words of B: R = n, G = k/128
 *                                            (128x128 block codes expanded per row)
 *   c    bf16 [m][n] or NULL (C = 0); may equal d
 *   d    bf16 [m][n]
 * Requires m >= 0, n > 0 and n % 8 == 0, k > 0 and k % 128 == 0.  m == 0 is a
 * no-op.  Source: zhouruolin.cn guide, section 五, "非分组 FP8 GEMM". */
dg_status dg_fp8_gemm_nt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                         const void* c, void* d, int m, int n, int k, void* stream);

/* Dense NT FP8 GEMM with the scales applied by per-K-block promotion instead
 * of inside the MMA: the same operands, layouts, result definition,
 * requirements and errors as dg_fp8_gemm_nt.  Each 128-deep K-block of a
 * 128 x 128 tile is summed unscaled by kind::f8f6f4 MMAs into a TMEM buffer
 * of its own (four rotate); epilogue warps read it, multiply by
 * sa[m, kb] * sb[n/128, kb] and add into FP32 registers, then D = bf16(acc +
 * C).  This is the two-level accumulation of the pages' Hopper design
 * ("DeepSeek 开源第三弹 ... DeepGEMM" (app.myzaker.com), sections "DeepGEMM"
 * and "持久化线程束专用化"), built on sm_100a as the measured alternative to
 * dg_fp8_gemm_nt's block-scaled MMA.  Tiles are always 128 wide; shared
 * tiles use the per-stream workspace as dg_fp8_gemm_nt does. */
dg_status dg_fp8_gemm_nt_promoted(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                  const void* c, void* d, int m, int n, int k, void* stream);

/* Dense FP8 GEMM in the other three storage layouts (the guide, section 五:
 * SM100 takes all of NT, TN, NN and TT).  The first letter names A's storage,
 * the second B's, relative to D = A * B with A [m][k] and B [k][n]:
 *   dg_fp8_gemm_nn   a e4m3 [m][k] (k contiguous), b e4m3 [k][n] (n contiguous)
 *   dg_fp8_gemm_tn   a e4m3 [k][m] (m contiguous), b e4m3 [k][n]
 *   dg_fp8_gemm_tt   a e4m3 [k][m],                b e4m3 [n][k] (as the NT call)
 * The scales do not depend on the storage: sfa as for dg_fp8_gemm_nt (R = m,
 * one code per row of D and 128-block of K), sfb as for dg_fp8_gemm_nt (the
 * 128x128 block codes of B, block (n/128, k/128), expanded per n).  c, d, the
 * result, the requirements and the errors are those of dg_fp8_gemm_nt, plus
 * m % 16 == 0 when A is stored [k][m] and n % 16 == 0 when B is stored [k][n]
 * (those rows are m or n bytes).  Operands stored with k as the row index are
 * staged MN-major and the tiles are 128 or 256 columns wide. */
dg_status dg_fp8_gemm_nn(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                         const void* c, void* d, int m, int n, int k, void* stream);
dg_status dg_fp8_gemm_tn(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                         const void* c, void* d, int m, int n, int k, void* stream);
dg_status dg_fp8_gemm_tt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                         const void* c, void* d, int m, int n, int k, void* stream);

/* M-grouped contiguous FP8 GEMM (MoE prefill / training forward): the rows of
 * all groups are concatenated along M, each group padded to a multiple of
 * dg_get_mk_alignment_for_contiguous_layout() (= 128) rows.
 *   a          e4m3 [m_total][k]           sfa  sf words, R = m_total, G = k/128
 *   b          e4m3 [num_groups][n][k]     sfb  num_groups blocks of sf words, R = n
 *   c          bf16 [m_total][n] or NULL
 *   d          bf16 [m_total][n]
 *   m_indices  int32 [m_total] on the device: group of each row, or -1 for a
 *              padding row.  All rows of one 128-row block belong to one group
 *              or are padding; a block whose first row is padding is skipped.
 * D rows of padding rows are unspecified.  Requires m_total % 128 == 0.
 * Source: zhouruolin.cn guide, section 五, m_grouped_fp8_gemm_nt_contiguous. */
dg_status dg_m_grouped_fp8_gemm_nt_contiguous(const void* a, const int32_t* sfa, const void* b,
                                              const int32_t* sfb, const void* c, void* d,
                                              const int32_t* m_indices, int m_total, int n, int k,
                                              int num_groups, void* stream);

/* M-grouped contiguous FP8 GEMM with B not transposed (NN): as
 * dg_m_grouped_fp8_gemm_nt_contiguous, D = C + A * B[g] per row, but
 *   b    e4m3 [num_groups][k][n] row-major (n contiguous: "MN-major")
 *   sfb  num_groups blocks of sf words, R = n, G = k/128: the 128x128 block
 *        codes of B[g] (block (k/128, n/128)) expanded per column n, exactly
 *        as for the NT call's B
 * Requires n % 16 == 0 as well (the rows of B are n bytes).  Other
 * arguments, rules and errors as dg_m_grouped_fp8_gemm_nt_contiguous.
 * Source: zhouruolin.cn guide, section 五 (SM100 takes all of the NT, TN, NN
 * and TT layouts; m_grouped_fp8_gemm_{nt, nn}_contiguous for the training
 * forward / prefill). */
dg_status dg_m_grouped_fp8_gemm_nn_contiguous(const void* a, const int32_t* sfa, const void* b,
                                              const int32_t* sfb, const void* c, void* d,
                                              const int32_t* m_indices, int m_total, int n, int k,
                                              int num_groups, void* stream);

/* K-grouped FP8 GEMM, TN layout (MoE weight gradient): the K axis (tokens)
 * is cut into num_groups consecutive ranges, group g owning the ks[g] rows
 * starting at k_g = ks[0] + ... + ks[g-1], and for every group
 *   D[g] = C[g] + A_g^T * B_g,   A_g = a[k_g .. k_g + ks[g]),  B_g likewise,
 * i.e. d[g][i][j] = c[g][i][j] + sum_k a[k][i] * b[k][j] with the scales below.
 *   a    e4m3 [k_total][m] row-major (m contiguous)
 *   sfa  sf words, R = m, G = k_total/128: one UE8M0 code per (column i of a,
 *        128-row block of K) -- A quantised 1x128 along K
 *   b    e4m3 [k_total][n] row-major (n contiguous)
 *   sfb  sf words, R = n, G = k_total/128: one code per (column j, 128-row
 *        block of K) -- B quantised 1x128 along K as well (no 128x128 blocks)
 *   c    bf16 [num_groups][m][n] or NULL (C = 0); may equal d
 *   d    bf16 [num_groups][m][n]; a group with ks[g] == 0 gets D[g] = C[g] (0)
 *   ks   int32 [num_groups] on the device: rows of K per group, each a
 *        multiple of 128 (so no 128-row scale block spans two groups), read
 *        inside the kernel (graph-capturable); their sum may not exceed k_total
 * Requires 1 <= num_groups <= 1024, m > 0 and m % 16 == 0, n > 0 and
 * n % 16 == 0, k_total >= 0 and k_total % 128 == 0.  A ks value that is
 * negative or not a multiple of 128 counts as 0 and a sum beyond k_total is
 * cut at k_total, both reported as DG_ERR_BAD_METADATA by dg_get_last_error.
 * Source: zhouruolin.cn guide, section 五 (k_grouped_fp8_gemm_tn_contiguous,
 * weight backward grouped along K; SM100 takes the TN layout). */
dg_status dg_k_grouped_fp8_gemm_tn_contiguous(const void* a, const int32_t* sfa, const void* b,
                                              const int32_t* sfb, const void* c, void* d,
                                              const int32_t* ks, int num_groups, int m, int n, int k_total,
                                              void* stream);

/* M-grouped masked FP8 GEMM (MoE decode): group g uses rows [0, masked_m[g])
 * of its [max_m][k] slab of A.
 *   a         e4m3 [num_groups][max_m][k]  sfa  num_groups blocks of sf words, R = max_m
 *   b         e4m3 [num_groups][n][k]      sfb  num_groups blocks of sf words, R = n
 *   d         bf16 [num_groups][max_m][n]; rows m >= masked_m[g] are never written
 *   masked_m  int32 [num_groups] on the device (read inside the kernel, so the
 *             call can be captured in a CUDA graph and replayed with new counts)
 *   expected_m host-side hint of the typical masked_m (heuristic only; may be 0)
 * Requires 1 <= num_groups <= 1024, max_m > 0.  masked_m values outside
 * [0, max_m] are clamped and reported as DG_ERR_BAD_METADATA.
 * Source: zhouruolin.cn guide, section 五, m_grouped_fp8_gemm_nt_masked. */
dg_status dg_m_grouped_fp8_gemm_nt_masked(const void* a, const int32_t* sfa, const void* b,
                                          const int32_t* sfb, void* d, const int32_t* masked_m,
                                          int num_groups, int max_m, int n, int k, int expected_m,
                                          void* stream);

/* M-grouped masked FP8 x FP4 GEMM: as dg_m_grouped_fp8_gemm_nt_masked with
 * B in e2m1 like dg_fp8_fp4_gemm_nt:
 *   b    e2m1 [num_groups][n][k/2] (two per byte, low nibble = even k)
 *   sfb  num_groups blocks of sf words, R = n, G = k/32 (one UE8M0 per 1x32)
 * Source: linlog.top, "FP4 精度支持" (FP8 x FP4 GEMM); masked layout as above. */
dg_status dg_m_grouped_fp8_fp4_gemm_nt_masked(const void* a, const int32_t* sfa, const void* b,
                                              const int32_t* sfb, void* d, const int32_t* masked_m,
                                              int num_groups, int max_m, int n, int k, int expected_m,
                                              void* stream);

/* Masked GEMM with SwiGLU fused into the epilogue (the linear1 -> SwiGLU step
 * of a MoE expert: the pages' "linear1 -> SwiGLU -> linear2", charles2530.github.io
 * "DeepGEMM：FP8 GEMM 与 Mega-MoE" and the Mega MoE section of the linlog.top page).
 * B holds the gate and up projections with their rows interleaved in blocks
 * of 64: B rows [128j, 128j + 64) are gate rows 64j.., rows [128j + 64,
 * 128j + 128) the matching up rows.  With G = A * B^T in FP32 (n columns),
 *   d[g][m][64j + i] = bf16( silu(G[m][128j + i]) * G[m][128j + 64 + i] ),
 *   silu(x) = x / (1 + exp(-x)),   i < 64,
 * so d is bf16 [num_groups][max_m][n/2].  Requires n % 128 == 0; no C.  The
 * _fp4_ form takes B as in dg_m_grouped_fp8_fp4_gemm_nt_masked.  Other
 * arguments, metadata rules and errors as dg_m_grouped_fp8_gemm_nt_masked. */
dg_status dg_m_grouped_fp8_gemm_nt_masked_swiglu(const void* a, const int32_t* sfa, const void* b,
                                                 const int32_t* sfb, void* d, const int32_t* masked_m,
                                                 int num_groups, int max_m, int n, int k, int expected_m,
                                                 void* stream);
dg_status dg_m_grouped_fp8_fp4_gemm_nt_masked_swiglu(const void* a, const int32_t* sfa, const void* b,
                                                     const int32_t* sfb, void* d, const int32_t* masked_m,
                                                     int num_groups, int max_m, int n, int k, int expected_m,
                                                     void* stream);

/* Dense NT FP8 GEMM that allocates no memory.  The pages have no counterpart
 * of this call; it exists for callers that cannot allocate device memory at
 * call time -- for example code running under another framework's memory
 * manager, a serving loop whose memory is fixed up front, or a library whose
 * own rule forbids cudaMalloc/cudaFree on the hot path (they can synchronise
 * the device and they fail when memory is exhausted).
 *
 * Arguments, results and errors are those of dg_fp8_gemm_nt.  Stream-K
 * partial sums go to one fixed device array of dg_noalloc_scratch_bytes() =
 * 32 MiB that is part of this library's device image: every GPU that loads
 * the library holds it until the process exits.  The heuristic only picks
 * plans whose partials fit in it (whole tiles need none), so the plan -- and
 * the rounding of the result -- can differ from dg_fp8_gemm_nt's for
 * problems whose best stream-K split needs more; dg_query_dense_config with
 * that cap shows the plan.  Nothing in the array has to start at zero: every
 * partial that is read is first written by the same call.
 *
 * All calls on a device share the array and it keeps the last call's
 * contents, so two calls whose kernels overlap on the GPU (different streams,
 * or different host threads without ordering) race and give wrong results;
 * order them on one stream.
 *
 * When the 32 MiB are committed: with CUDA's lazy module loading (the default
 * since CUDA 12.2) the array is allocated on a device when this library's
 * module is first loaded there -- at its first kernel launch or symbol lookup
 * on that device, which may be this call.  That load can fail for lack of
 * memory (DG_ERR_CUDA) if the caller has already claimed the device's memory,
 * so make one warm-up call per device before fixing the memory budget, or set
 * CUDA_MODULE_LOADING=EAGER.
 *
 * The first call on each device (and in each new context of it) looks up the
 * array's device address (cudaGetSymbolAddress) with that device current and
 * caches it per device and context; make that first call before any stream
 * capture.  After a device reset the next call looks the address up again;
 * dg_shutdown() also forgets the cached addresses. */
dg_status dg_fp8_gemm_nt_noalloc(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                 const void* c, void* d, int m, int n, int k, void* stream);

/* Size in bytes of the fixed scratch array used by dg_fp8_gemm_nt_noalloc. */
size_t dg_noalloc_scratch_bytes(void);

/* Dense NT BF16 GEMM on the same persistent kernel: D[M,N] = C + A * B^T
 * with bf16 A [m][k], B [n][k] (row-major, K contiguous), FP32 accumulation
 * in TMEM (tcgen05 kind::f16), bf16 D; c bf16 [m][n] or NULL, may equal d.
 * No scale factors.  Requires m >= 0, n > 0 and n % 8 == 0, k > 0 and
 * k % 64 == 0; 16-byte aligned pointers.  The pages list BF16 GEMM among
 * the library's kernels ("DeepGEMM：统一高性能张量核心 GEMM 计算库编译与使用
 * 指南" (zhouruolin.cn), introduction; "DeepGEMM：FP8 GEMM 与 Mega-MoE"
 * (charles2530.github.io), section 一). */
dg_status dg_bf16_gemm_nt(const void* a, const void* b, const void* c, void* d, int m, int n, int k, void* stream);

/* FP8 x FP4 dense NT GEMM: as dg_fp8_gemm_nt but
 *   b    e2m1 [n][k/2] (two codes per byte, low nibble = even k)
 *   sfb  sf words of B: R = n, G = k/32 (one UE8M0 code per 1x32 group)
 * Source: linlog.top update, section "FP4 精度支持". */
dg_status dg_fp8_fp4_gemm_nt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                             const void* c, void* d, int m, int n, int k, void* stream);

/* FP8 x FP4 M-grouped contiguous GEMM: as the FP8 contiguous call with B in
 * e2m1 [num_groups][n][k/2] and per-group sf words R = n, G = k/32. */
dg_status dg_m_grouped_fp8_fp4_gemm_nt_contiguous(const void* a, const int32_t* sfa, const void* b,
                                                  const int32_t* sfb, const void* c, void* d,
                                                  const int32_t* m_indices, int m_total, int n, int k,
                                                  int num_groups, void* stream);

/* ------------------------------------------------------ input preparation */

/* Quantise FP32 x [rows][cols] to e4m3 with one UE8M0 scale per
 * block_rows x 128 block (block_rows = 1: activations, 1x128; block_rows =
 * 128: weights, 128x128).  scale = 2^i, i = min{ i : 448 * 2^i >= amax }
 * (amax = 0 gives i = 0), q = e4m3(x / scale) rounded to nearest even.
 *   q   e4m3 [rows][cols]
 *   sf  ue8m0 [ceil(rows/block_rows)][cols/128]
 * Requires cols % 128 == 0. */
dg_status dg_quantize_fp8(const float* x, int rows, int cols, int block_rows, uint8_t* q, uint8_t* sf,
                          void* stream);

/* Quantise FP32 x [rows][cols] to e2m1 with one UE8M0 scale per 1x32 group
 * (qmax = 6).  q: e2m1 [rows][cols/2]; sf: ue8m0 [rows][cols/32].
 * Requires cols % 32 == 0. */
dg_status dg_quantize_fp4(const float* x, int rows, int cols, uint8_t* q, uint8_t* sf, void* stream);

/* Pack UE8M0 codes sf [ceil(rows/row_div)][num_sf_cols] into sf words (layout
 * above) for a matrix of `rows` rows; row r reads code row r/row_div
 * (row_div = 1 per-row scales, 128 for 128x128 block scales).
 * packed has dg_packed_sf_words(rows, num_sf_cols) int32 entries. */
dg_status dg_pack_sf(const uint8_t* sf, int rows, int num_sf_cols, int row_div, int32_t* packed,
                     void* stream);

/* Number of int32 words of the packed layout: ceil(cols/4) * ceil(rows/128) * 128. */
int64_t dg_packed_sf_words(int rows, int num_sf_cols);

/* --------------------------------------------------------------- utilities */

/* Number of SMs the GEMM kernels use (default: all SMs of the current
 * device).  dg_set_num_sms(0) restores the default. */
int dg_get_num_sms(void);
dg_status dg_set_num_sms(int num_sms);

/* Programmatic dependent launch (default on): every kernel of this library
 * is launched as a programmatic dependent of the preceding work on its
 * stream, so its launch and prologue (barrier set-up, TMEM allocation,
 * descriptor prefetch) overlap the previous kernel's tail; it touches no
 * global memory before that work has completed.  dg_set_pdl(0) launches
 * plainly.  Source: "DeepGEMM：统一高性能张量核心 GEMM 计算库编译与使用指南"
 * (zhouruolin.cn), section "工具函数" (set_pdl), and "DeepSeek 发布 DeepGEMM
 * 重大更新" (linlog.top), section "其他更新" (PDL). */
dg_status dg_set_pdl(int enable);
int dg_get_pdl(void);

/* Restricts the tile heuristic (all later calls, all threads): block_n in
 * {64, 128, 160, 192, 224, 256} (0 = the heuristic's choice among 128, 192,
 * 256; the others are only used when forced) and schedule 0 (heuristic), 1
 * (whole tiles only), 2 (the last tiles cut into per-tile K-slices, one per
 * CTA) or 3 (stream-K: the last tiles' K-iterations shared evenly over the
 * grid), or 4 to 10 (every tile's K-blocks cut into S = schedule - 2 slices,
 * 2 to 8, computed by the CTAs of one thread-block cluster and summed through
 * distributed shared memory; 128- and 256-wide dense NT tiles); 2 to 10 apply
 * to the dense calls whenever such a split exists.
 * Anything else returns DG_ERR_INVALID_ARG and changes nothing.  Meant for
 * tuning and tests.  The environment variables DG_BLOCK_N and DG_SCHEDULE set
 * the initial values. */
dg_status dg_set_tile_config(int block_n, int schedule);

/* Row alignment of groups in the contiguous layout: 128. */
int dg_get_mk_alignment_for_contiguous_layout(void);

/* Synchronises `stream`, then returns and clears the first device-side error
 * recorded on the current device (DG_OK if none). */
dg_status dg_get_last_error(void* stream);

/* Test hook: launches a kernel whose single wait can never be satisfied and
 * must give up after limit_us microseconds; dg_get_last_error() then reports
 * DG_ERR_TIMEOUT.  Faults nothing and leaves the context usable. */
dg_status dg_debug_starved_wait(unsigned int limit_us, void* stream);

/* Test hook: n / d computed the way the kernels divide by per-launch
 * constants (multiply-high, add, shift); d >= 1 and n < 2^31, else
 * 0xFFFFFFFF. */
uint32_t dg_debug_fastdiv(uint32_t d, uint32_t n);

/* Human-readable name of a status code (static string). */
const char* dg_status_string(int status);

/* Kernels this library has launched in this process (all devices). */
uint64_t dg_launch_count(void);

/* Plan the dense heuristic picks for (m, n, k) with at most workspace_cap
 * bytes of workspace (0: no cap, the plan of dg_fp8_gemm_nt;
 * dg_noalloc_scratch_bytes(): the plan of dg_fp8_gemm_nt_noalloc): block_n,
 * tiles computed whole (dp_tiles), tiles after them whose K-blocks are
 * shared over several CTAs (sk_tiles, 0 = none), how: sk_split > 0 = each
 * cut into that many equal K-slices, 0 = stream-K (even shares of all their
 * K-blocks over the grid), workspace slots per shared tile, grid size in CTAs
 * and workspace bytes.  Any output pointer may be NULL.  DG_ERR_INVALID_ARG
 * for m, n <= 0, k not a positive multiple of 128 or a negative cap. */
dg_status dg_query_dense_config(int m, int n, int k, int64_t workspace_cap, int* block_n, int* dp_tiles,
                                int* sk_tiles, int* sk_split, int* max_segments, int* grid,
                                int64_t* workspace_bytes);

/* Cluster split of the dense plan for (m, n, k) with at most workspace_cap
 * bytes of workspace: S > 0 when every output tile's K-blocks are cut into S
 * slices computed by the S CTAs of one thread-block cluster, whose FP32
 * partial sums are added through distributed shared memory inside the same
 * kernel (no workspace, no second kernel; the plan dg_query_dense_config then
 * reports as dp_tiles = the tiles, sk_tiles = 0, grid = tiles x S); 0 when the
 * plan is another one; -1 for invalid sizes. */
int dg_query_dense_cluster_split(int m, int n, int k, int64_t workspace_cap);

/* Clusters of `cluster` CTAs (2 .. 8) of the split kernel with block width
 * block_n (128 or 256; fp4 nonzero: e2m1 B) that the current device holds at
 * once (cudaOccupancyMaxActiveClusters); the planner's capacity for cluster
 * splits.  -1 for other arguments, 0 when the query fails. */
int dg_debug_cluster_capacity(int block_n, int fp4, int cluster);

/* Layouts named by dg_query_config. */
enum { DG_LAYOUT_DENSE = 0, DG_LAYOUT_CONTIGUOUS = 1, DG_LAYOUT_MASKED = 2 };

/* Plan of an NT call of the given layout as the library would launch it on
 * the current device: block width (block_n), grid size in CTAs and the work
 * units (output tiles) the persistent grid walks (masked: counted at max_m
 * rows per group; the kernel walks only the tiles of the valid rows).
 *   layout     DG_LAYOUT_DENSE / _CONTIGUOUS / _MASKED
 *   fp4        nonzero: e2m1 B (the *_fp8_fp4_* calls)
 *   swiglu     nonzero: the masked *_swiglu calls (masked layout only)
 *   rows       dense m, contiguous m_total, masked max_m
 *   num_groups 1 for dense; expected_m the masked hint (0 = none)
 * Any output pointer may be NULL.  Nothing is launched.  DG_ERR_INVALID_ARG
 * for an unknown layout, non-positive sizes, k not a multiple of 128 or
 * swiglu outside the masked layout. */
dg_status dg_query_config(int layout, int fp4, int swiglu, int rows, int n, int k, int num_groups, int expected_m,
                          int* block_n, int* grid, int64_t* units);

/* Tensor-core throughput probe: one CTA per SM issues kblocks x 4
 * tcgen05 MMAs of M = 128, N = block_n (128 or 256; block-scaled e4m3 also 32, 64 or 192), K = 32 (bf16: 16) from
 * operand tiles held in shared memory, with no global-memory traffic, into a
 * TMEM accumulator.  Kinds:
 *   DG_PROBE_FP8_SCALED  kind::mxf8f6f4.block_scale, e4m3, UE8M0 scales (the
 *                        instruction of the GEMM kernels)
 *   DG_PROBE_FP8_PLAIN   kind::f8f6f4, e4m3, no scales (the per-K-block
 *                        promotion variant's instruction)
 *   DG_PROBE_BF16        kind::f16, bf16 operands
 * One launch performs SMs x kblocks x 4 x 2 x 128 x block_n x 32 FLOPs (bf16:
 * x 16); time it with events on `stream` to get the pipe's peak rate, the
 * denominator beside the nominal dense FP8 peak of the B200 (4.5 PFLOP/s).
 * Asynchronous.  DG_ERR_INVALID_ARG for an unknown kind, another width or
 * kblocks outside [1, 2^22]. */
enum { DG_PROBE_FP8_SCALED = 0, DG_PROBE_FP8_PLAIN = 1, DG_PROBE_BF16 = 2 };
dg_status dg_probe_mma_peak(int kind, int block_n, int kblocks, void* stream);

/* Output tiles of an m x n problem cut into block_m x block_n tiles (the
 * count the heuristic balances against the SM count; "DeepSeek 开源第三弹 ...
 * DeepGEMM" (app.myzaker.com), section "非对齐块大小"). */
int64_t dg_num_tiles(int m, int n, int block_m, int block_n);

/* Releases the stream-K workspaces of all devices (synchronises each) and
 * forgets the cached scratch addresses of dg_fp8_gemm_nt_noalloc.  Call it
 * before resetting a device this library has used. */
void dg_shutdown(void);

#ifdef __cplusplus
}
#endif

#endif /* DG_H_ */
