/*
 * dg_oracle.c -- CPU oracle for the fine-grained-scaled GEMM D = C + A * B^T.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this file: only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline use it.  It shares no code, header, table or constant with the CUDA
 * library under moe_grouped_gemm_06_b200/.
 *
 * Everything is computed the slow, plain way:
 *   - every 8-bit / 4-bit code is decoded through a table built from the bit
 *     fields of the format (no casts, no hardware conversions);
 *   - dot products are accumulated in double precision in the natural order
 *     (row, K-block, k), with the two scale factors applied per K-block;
 *   - quantisation finds the nearest code by searching the ascending table of
 *     non-negative codes, ties going to the code with an even mantissa.
 *
 * Sources (page title, section):
 *   [P4] "DeepSeek 开源第三弹 ... DeepGEMM" (app.myzaker.com), section "DeepGEMM":
 *        FP8 GEMM with the fine-grained scaling of DeepSeek-V3 -- one scale per
 *        1x128 row-group of the activations, one per 128x128 block of weights.
 *   [P5] "DeepGEMM：统一高性能张量核心 GEMM 计算库编译与使用指南" (zhouruolin.cn),
 *        section 五 "使用方法": naming convention D = C + A @ B with NT layout
 *        (A not transposed, B transposed); SM100 scale factors are packed UE8M0;
 *        grouping is only along M (N, K shared), contiguous layout for
 *        prefill, masked layout for decoding.
 *   [P1] "DeepSeek 发布 DeepGEMM 重大更新" (linlog.top), section "FP4 精度支持":
 *        FP8 x FP4 GEMM, FP4 weights with UE8M0 scale factors, 4 per int32.
 *   [P5] also: SM100 takes every one of the NT, TN, NN and TT layouts; the
 *        contiguous grouped GEMM comes as nt and nn; the weight backward is
 *        k_grouped_fp8_gemm_tn_contiguous, grouped along K.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - FP8 means OCP E4M3FN: bias 7, no infinities, S.1111.111 is NaN, max 448.
 *   - UE8M0 code e means 2^(e-127); code 255 is NaN.
 *   - FP4 means OCP E2M1: values +-{0,.5,1,1.5,2,3,4,6}.
 *   - scale exponent i = min{ i : qmax * 2^i >= amax } (= ceil(log2(amax/qmax))),
 *     clamped to [-127, 127]; amax == 0 gives i = 0 (code 127).
 *   - FP4 codes are packed two per byte along K, low nibble = even k.
 *   - packed scale layout: see or_pack_sf below.
 *   - NN: B is stored [K][N] (B[k][n] is the element the NT layout stores at
 *     [n][k]); its 128x128 block scales keep the NT indexing (n/128, k/128).
 *   - K-grouped TN: group g owns the K rows [k_g, k_g + ks[g]) of A [K][M] and
 *     B [K][N] and writes D[g] = C[g] + A_g^T B_g ([M][N]); both operands
 *     carry one scale per (column, 128-row block of K), the ks[g] being
 *     multiples of 128; an empty group gives D[g] = C[g].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Format tables, built from the bit fields.                                 */
/* ------------------------------------------------------------------------ */

static double E4M3[256];
static double E2M1[16];
static double UE8M0[256];
static int tables_ready = 0;

/* E4M3: sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0.
 * Exponent field 0 is subnormal: m * 2^-9.  S.1111.111 is NaN. */
static double e4m3_from_bits(int code) {
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.
 * Exponent field 0 is subnormal: m * 0.5. */
static double e2m1_from_bits(int code) {
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v;
    if (e == 0) v = 0.5 * m;
    else v = ldexp(1.0 + m / 2.0, e - 1);
    return s ? -v : v;
}

static void build_tables(void) {
    if (tables_ready) return;
    for (int c = 0; c < 256; ++c) E4M3[c] = e4m3_from_bits(c);
    for (int c = 0; c < 16; ++c) E2M1[c] = e2m1_from_bits(c);
    for (int c = 0; c < 256; ++c) UE8M0[c] = (c == 255) ? NAN : ldexp(1.0, c - 127);
    tables_ready = 1;
}

void or_tables(double* e4m3, double* e2m1, double* ue8m0) {
    build_tables();
    if (e4m3) memcpy(e4m3, E4M3, sizeof(E4M3));
    if (e2m1) memcpy(e2m1, E2M1, sizeof(E2M1));
    if (ue8m0) memcpy(ue8m0, UE8M0, sizeof(UE8M0));
}

int or_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static double bf16_bits_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* Quantisation (the input recipe: per-group amax -> power-of-two scale ->    */
/* round-to-nearest-even into the code set).                                  */
/* ------------------------------------------------------------------------ */

/* Nearest code among the ascending non-negative values tab[0..top];
 * ties go to the even code (mantissa LSB = code LSB).  |v| >= tab[top]
 * saturates to top. */
static int nearest_code(const double* tab, int top, double a) {
    if (!(a < tab[top])) return top;
    int lo = 0, hi = top;                 /* largest c with tab[c] <= a */
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (tab[mid] <= a) lo = mid; else hi = mid - 1;
    }
    double dlo = a - tab[lo], dhi = tab[lo + 1] - a;
    if (dhi < dlo) return lo + 1;
    if (dhi == dlo && ((lo + 1) & 1) == 0) return lo + 1;
    return lo;
}

static uint8_t encode_e4m3(double v) {
    if (isnan(v)) return 0x7F;
    int s = signbit(v) ? 0x80 : 0;
    return (uint8_t)(s | nearest_code(E4M3, 0x7E, fabs(v)));
}

static uint8_t encode_e2m1(double v) {
    int s = signbit(v) ? 0x8 : 0;
    return (uint8_t)(s | nearest_code(E2M1, 7, fabs(v)));
}

/* i = min{ i : qmax * 2^i >= amax }, clamped to [-127, 127]; amax == 0 -> 0. */
static int scale_exponent(double amax, double qmax) {
    if (!(amax > 0)) return 0;
    int i = (int)ceil(log2(amax / qmax));
    while (i > -127 && ldexp(qmax, i - 1) >= amax) --i;
    while (i < 127 && ldexp(qmax, i) < amax) ++i;
    if (i < -127) i = -127;
    if (i > 127) i = 127;
    return i;
}

void or_scale_exponents_probe(const double* amax, int64_t n, double qmax, int32_t* out) {
    for (int64_t j = 0; j < n; ++j) out[j] = scale_exponent(amax[j], qmax);
}

void or_encode_e4m3(const double* v, int64_t n, uint8_t* out) {
    build_tables();
    for (int64_t j = 0; j < n; ++j) out[j] = encode_e4m3(v[j]);
}

void or_encode_e2m1(const double* v, int64_t n, uint8_t* out) {
    build_tables();
    for (int64_t j = 0; j < n; ++j) out[j] = encode_e2m1(v[j]);
}

/* FP8 E4M3 quantisation of x[rows][cols] in blocks of gr rows x gc columns.
 * q[rows][cols] receives the codes, e[ceil(rows/gr)][cols/gc] the UE8M0 codes.
 * gr = 1, gc = 128 gives the activation (1x128) recipe; gr = gc = 128 the
 * weight (128x128) recipe.  cols must be a multiple of gc. */
void or_quantize_fp8(const float* x, int64_t rows, int64_t cols, int gr, int gc,
                     uint8_t* q, uint8_t* e) {
    build_tables();
    int64_t nbr = (rows + gr - 1) / gr, nbc = cols / gc;
#pragma omp parallel for schedule(dynamic)
    for (int64_t br = 0; br < nbr; ++br) {
        for (int64_t bc = 0; bc < nbc; ++bc) {
            int64_t r0 = br * gr, r1 = r0 + gr < rows ? r0 + gr : rows;
            double amax = 0;
            for (int64_t r = r0; r < r1; ++r)
                for (int64_t c = bc * gc; c < (bc + 1) * gc; ++c) {
                    double a = fabs((double)x[r * cols + c]);
                    if (a > amax) amax = a;
                }
            int i = scale_exponent(amax, 448.0);
            e[br * nbc + bc] = (uint8_t)(i + 127);
            for (int64_t r = r0; r < r1; ++r)
                for (int64_t c = bc * gc; c < (bc + 1) * gc; ++c)
                    q[r * cols + c] = encode_e4m3(ldexp((double)x[r * cols + c], -i));
        }
    }
}

/* FP4 E2M1 quantisation of x[rows][cols] in 1 x gc groups (gc = 32).
 * q[rows][cols/2] packs two codes per byte, low nibble = even column;
 * e[rows][cols/gc] receives the UE8M0 codes. */
void or_quantize_fp4(const float* x, int64_t rows, int64_t cols, int gc,
                     uint8_t* q, uint8_t* e) {
    build_tables();
    int64_t nbc = cols / gc;
#pragma omp parallel for schedule(dynamic)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t bc = 0; bc < nbc; ++bc) {
            double amax = 0;
            for (int64_t c = bc * gc; c < (bc + 1) * gc; ++c) {
                double a = fabs((double)x[r * cols + c]);
                if (a > amax) amax = a;
            }
            int i = scale_exponent(amax, 6.0);
            e[r * nbc + bc] = (uint8_t)(i + 127);
            for (int64_t c = bc * gc; c < (bc + 1) * gc; c += 2) {
                uint8_t lo = encode_e2m1(ldexp((double)x[r * cols + c], -i));
                uint8_t hi = encode_e2m1(ldexp((double)x[r * cols + c + 1], -i));
                q[r * (cols / 2) + c / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Scale packing: 4 UE8M0 codes per int32.                                   */
/* ------------------------------------------------------------------------ */

/* Packed layout (our reading of "4 UE8M0 per int32, TMA-aligned"):
 *   out is int32[Q][Cr][128] with Q = ceil(ng/4) groups of 4 scale columns and
 *   Cr = ceil(rows/128) chunks of 128 rows.  The word for (row r, group q) sits
 *   at ((q*Cr + r/128)*128 + (r%32)*4 + (r%128)/32); its byte j (little
 *   endian) is the scale of column 4q+j.  Bytes with no scale (4q+j >= ng, or
 *   r >= rows) hold 127 (= 1.0).
 * e is uint8[rows_of_e][ng]; row r of the output takes row (r / row_div) of e,
 * so row_div = 1 packs per-row scales and row_div = 128 expands 128x128 block
 * scales to one copy per row. */
void or_pack_sf(const uint8_t* e, int64_t rows, int64_t ng, int row_div, int32_t* out) {
    int64_t Q = (ng + 3) / 4, Cr = (rows + 127) / 128;
    for (int64_t q = 0; q < Q; ++q)
        for (int64_t r = 0; r < Cr * 128; ++r) {
            uint32_t w = 0;
            for (int j = 0; j < 4; ++j) {
                uint32_t byte = 127;
                if (r < rows && 4 * q + j < ng) byte = e[(r / row_div) * ng + 4 * q + j];
                w |= byte << (8 * j);
            }
            int64_t idx = (q * Cr + r / 128) * 128 + (r % 32) * 4 + (r % 128) / 32;
            out[idx] = (int32_t)w;
        }
}

/* ------------------------------------------------------------------------ */
/* The contraction.                                                          */
/* ------------------------------------------------------------------------ */

/* One operand of the product: codes plus the scale lookup.  Element (r, k)
 * of an fp8 operand is codes[r * row_stride + k * k_stride] (K-major storage
 * [rows][K]: row_stride = K, k_stride = 1; MN-major storage [K][rows]:
 * row_stride = 1, k_stride = rows).  An fp4 operand is always K-major with
 * two codes per byte. */
typedef struct {
    const uint8_t* codes;
    int64_t row_stride, k_stride;
    const uint8_t* sf;      /* UE8M0 codes, [ceil(rows/sf_rows)][sf_cols] */
    int64_t sf_cols;        /* scale columns per scale row (K / sf_k) */
    int fp4;                /* 1: E2M1 packed two per byte, low nibble = even k */
    int sf_rows;            /* rows sharing one scale (1 or 128) */
    int sf_k;               /* K elements sharing one scale (128 or 32) */
} operand_t;

static double elem(const operand_t* o, int64_t r, int64_t k) {
    if (o->fp4) {
        uint8_t byte = o->codes[r * o->row_stride + k / 2];
        return E2M1[(k & 1) ? (byte >> 4) : (byte & 15)];
    }
    return E4M3[o->codes[r * o->row_stride + k * o->k_stride]];
}

static double scale(const operand_t* o, int64_t r, int64_t k) {
    return UE8M0[o->sf[(r / o->sf_rows) * o->sf_cols + k / o->sf_k]];
}

/* sum over k in [k_begin, k_end) of s_a(m,k) s_b(n,k) a(m,k) b(n,k),
 * evaluated block by block: the K axis is cut at every scale boundary of
 * either operand (k_begin is one), each piece is summed unscaled and then
 * multiplied by the two scales of that piece. */
static double dot_range(const operand_t* A, int64_t m, const operand_t* B, int64_t n, int64_t k_begin,
                        int64_t k_end) {
    int64_t step = A->sf_k < B->sf_k ? A->sf_k : B->sf_k;
    double acc = 0;
    if (!A->fp4 && !B->fp4 && A->k_stride == 1 && B->k_stride == 1) {
        /* both rows contiguous along K: the same sums, read as two byte rows */
        const uint8_t* ra = A->codes + m * A->row_stride;
        const uint8_t* rb = B->codes + n * B->row_stride;
        for (int64_t k0 = k_begin; k0 < k_end; k0 += step) {
            double part = 0;
            for (int64_t k = k0; k < k0 + step; ++k) part += E4M3[ra[k]] * E4M3[rb[k]];
            acc += scale(A, m, k0) * scale(B, n, k0) * part;
        }
        return acc;
    }
    for (int64_t k0 = k_begin; k0 < k_end; k0 += step) {
        double part = 0;
        for (int64_t k = k0; k < k0 + step; ++k) part += elem(A, m, k) * elem(B, n, k);
        acc += scale(A, m, k0) * scale(B, n, k0) * part;
    }
    return acc;
}

static double dot(const operand_t* A, int64_t m, const operand_t* B, int64_t n, int64_t K) {
    return dot_range(A, m, B, n, 0, K);
}

/* The NT operands: A [M][K] with 1x128 scales, B [N][K] with 128x128 block
 * scales (fp8) or [N][K/2] with 1x32 scales (fp4). */
static void make_ops(operand_t* A, operand_t* B, const uint8_t* a, const uint8_t* sfa,
                     const uint8_t* b, const uint8_t* sfb, int b_fp4, int64_t K) {
    A->codes = a; A->row_stride = K; A->k_stride = 1;
    A->sf = sfa; A->sf_cols = K / 128; A->fp4 = 0; A->sf_rows = 1; A->sf_k = 128;
    B->codes = b; B->fp4 = b_fp4;
    B->row_stride = b_fp4 ? K / 2 : K; B->k_stride = 1;
    B->sf = sfb;
    B->sf_rows = b_fp4 ? 1 : 128;
    B->sf_k = b_fp4 ? 32 : 128;
    B->sf_cols = K / B->sf_k;
}

/* Dense NT: out[m][n] = C[m][n] + sum_k ...  for all m < M, n < N.
 *   a: e4m3 [M][K], sfa: UE8M0 [M][K/128]
 *   b: e4m3 [N][K] with sfb [ceil(N/128)][K/128]   (b_fp4 = 0), or
 *      e2m1 [N][K/2] with sfb [N][K/32]            (b_fp4 = 1)
 *   c: bf16 bits [M][N] or NULL (C = 0).  out: double [M][N]. */
void or_gemm(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb,
             int b_fp4, const uint16_t* c, int64_t M, int64_t N, int64_t K, double* out) {
    build_tables();
    operand_t A, B;
    make_ops(&A, &B, a, sfa, b, sfb, b_fp4, K);
#pragma omp parallel for schedule(dynamic)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double base = c ? bf16_bits_to_double(c[m * N + n]) : 0.0;
            out[m * N + n] = base + dot(&A, m, &B, n, K);
        }
}

/* The same definition evaluated only at the listed (m, n) points. */
void or_gemm_points(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb,
                    int b_fp4, const uint16_t* c, int64_t M, int64_t N, int64_t K,
                    const int64_t* pm, const int64_t* pn, int64_t npts, double* out) {
    build_tables();
    (void)M;
    operand_t A, B;
    make_ops(&A, &B, a, sfa, b, sfb, b_fp4, K);
#pragma omp parallel for schedule(dynamic)
    for (int64_t t = 0; t < npts; ++t) {
        int64_t m = pm[t], n = pn[t];
        double base = c ? bf16_bits_to_double(c[m * N + n]) : 0.0;
        out[t] = base + dot(&A, m, &B, n, K);
    }
}

/* Size in bytes of one group's B codes and B scale codes. */
static void b_group_sizes(int b_fp4, int64_t N, int64_t K, int64_t* codes, int64_t* sfs) {
    *codes = b_fp4 ? N * (K / 2) : N * K;
    *sfs = b_fp4 ? N * (K / 32) : ((N + 127) / 128) * (K / 128);
}

/* M-grouped contiguous: row m of A belongs to group g = m_indices[m] (or is
 * padding when g < 0).  B holds num_groups weight matrices back to back.
 * out[m][n] is written only for rows with g >= 0; padding rows are left as
 * they were.  Rows with g >= num_groups are invalid and also left alone. */
void or_gemm_contiguous(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                        const uint8_t* sfb, int b_fp4, const uint16_t* c,
                        const int32_t* m_indices, int64_t M, int64_t N, int64_t K,
                        int64_t num_groups, double* out) {
    build_tables();
    int64_t bc, bs;
    b_group_sizes(b_fp4, N, K, &bc, &bs);
#pragma omp parallel for schedule(dynamic)
    for (int64_t m = 0; m < M; ++m) {
        int64_t g = m_indices[m];
        if (g < 0 || g >= num_groups) continue;
        operand_t A, B;
        make_ops(&A, &B, a, sfa, b + g * bc, sfb + g * bs, b_fp4, K);
        for (int64_t n = 0; n < N; ++n) {
            double base = c ? bf16_bits_to_double(c[m * N + n]) : 0.0;
            out[m * N + n] = base + dot(&A, m, &B, n, K);
        }
    }
}

/* M-grouped masked: A is [G][max_m][K]; in group g only rows m < masked_m[g]
 * count.  out is [G][max_m][N]; rows m >= masked_m[g] are left untouched.
 * masked_m[g] is clipped to [0, max_m]. */
void or_gemm_masked(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                    const uint8_t* sfb, int b_fp4, const int32_t* masked_m,
                    int64_t G, int64_t max_m, int64_t N, int64_t K, double* out) {
    build_tables();
    int64_t bc, bs;
    b_group_sizes(b_fp4, N, K, &bc, &bs);
#pragma omp parallel for schedule(dynamic) collapse(2)
    for (int64_t g = 0; g < G; ++g)
        for (int64_t m = 0; m < max_m; ++m) {
            int64_t valid = masked_m[g] < 0 ? 0 : (masked_m[g] > max_m ? max_m : masked_m[g]);
            if (m >= valid) continue;
            operand_t A, B;
            make_ops(&A, &B, a + g * max_m * K, sfa + g * max_m * (K / 128),
                     b + g * bc, sfb + g * bs, b_fp4, K);
            for (int64_t n = 0; n < N; ++n)
                out[(g * max_m + m) * N + n] = dot(&A, m, &B, n, K);
        }
}

/* M-grouped contiguous with B not transposed (NN): as or_gemm_contiguous,
 * but group g's weights are stored [K][N] (b + g*K*N, element (n, k) at
 * [k][n]); the 128x128 block scales sfb + g*ceil(N/128)*(K/128) keep the
 * [n/128][k/128] indexing of the NT call. */
void or_gemm_nn_contiguous(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                           const uint8_t* sfb, const uint16_t* c, const int32_t* m_indices,
                           int64_t M, int64_t N, int64_t K, int64_t num_groups, double* out) {
    build_tables();
    const int64_t bs = ((N + 127) / 128) * (K / 128);
#pragma omp parallel for schedule(dynamic)
    for (int64_t m = 0; m < M; ++m) {
        int64_t g = m_indices[m];
        if (g < 0 || g >= num_groups) continue;
        operand_t A, B;
        make_ops(&A, &B, a, sfa, b + g * K * N, sfb + g * bs, 0, K);
        B.row_stride = 1;          /* (n, k) at [k][n] */
        B.k_stride = N;
        for (int64_t n = 0; n < N; ++n) {
            double base = c ? bf16_bits_to_double(c[m * N + n]) : 0.0;
            out[m * N + n] = base + dot(&A, m, &B, n, K);
        }
    }
}

/* K-grouped TN: a is [Kt][M], b is [Kt][N] (Kt = sum of ks); sfa is
 * [M][Kt/128] and sfb [N][Kt/128] (one code per column and 128-row block of
 * K).  out[g][i][j] = C[g][i][j] + sum over group g's K rows of
 * a[k][i] b[k][j] scaled per block; ks[g] are multiples of 128. */
void or_gemm_k_grouped_tn(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                          const uint8_t* sfb, const uint16_t* c, const int32_t* ks,
                          int64_t G, int64_t M, int64_t N, int64_t Kt, double* out) {
    build_tables();
    operand_t A, B;
    A.codes = a; A.row_stride = 1; A.k_stride = M;
    A.sf = sfa; A.sf_cols = Kt / 128; A.fp4 = 0; A.sf_rows = 1; A.sf_k = 128;
    B.codes = b; B.row_stride = 1; B.k_stride = N;
    B.sf = sfb; B.sf_cols = Kt / 128; B.fp4 = 0; B.sf_rows = 1; B.sf_k = 128;
    int64_t k0 = 0;
    for (int64_t g = 0; g < G; ++g) {
        const int64_t k1 = k0 + ks[g];
#pragma omp parallel for schedule(dynamic)
        for (int64_t i = 0; i < M; ++i)
            for (int64_t j = 0; j < N; ++j) {
                const int64_t o = (g * M + i) * N + j;
                double base = c ? bf16_bits_to_double(c[o]) : 0.0;
                out[o] = base + dot_range(&A, i, &B, j, k0, k1);
            }
        k0 = k1;
    }
}

/* or_gemm_k_grouped_tn at the points (pg[t], pi[t], pj[t]) only. */
void or_gemm_k_grouped_tn_points(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                                 const uint8_t* sfb, const uint16_t* c, const int32_t* ks,
                                 int64_t G, int64_t M, int64_t N, int64_t Kt,
                                 const int64_t* pg, const int64_t* pi, const int64_t* pj,
                                 int64_t npts, double* out) {
    build_tables();
    operand_t A, B;
    A.codes = a; A.row_stride = 1; A.k_stride = M;
    A.sf = sfa; A.sf_cols = Kt / 128; A.fp4 = 0; A.sf_rows = 1; A.sf_k = 128;
    B.codes = b; B.row_stride = 1; B.k_stride = N;
    B.sf = sfb; B.sf_cols = Kt / 128; B.fp4 = 0; B.sf_rows = 1; B.sf_k = 128;
#pragma omp parallel for schedule(dynamic)
    for (int64_t t = 0; t < npts; ++t) {
        const int64_t g = pg[t], i = pi[t], j = pj[t];
        int64_t k0 = 0;
        for (int64_t h = 0; h < g; ++h) k0 += ks[h];
        const int64_t o = (g * M + i) * N + j;
        double base = c ? bf16_bits_to_double(c[o]) : 0.0;
        out[t] = base + dot_range(&A, i, &B, j, k0, k0 + ks[g]);
    }
}

/* Dense FP8 GEMM in any of the four storage layouts of A and B (NT, NN, TN,
 * TT): a_mn = 1 stores A as [K][M] (else [M][K]); b_mn = 1 stores B as [K][N]
 * (else [N][K]).  The scales do not depend on the storage: sfa [M][K/128]
 * (1x128 along K), sfb [ceil(N/128)][K/128] (128x128 blocks).  out[m][n] =
 * C[m][n] + sum_k ..., as or_gemm. */
void or_gemm_layout(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb,
                    const uint16_t* c, int a_mn, int b_mn, int64_t M, int64_t N, int64_t K, double* out) {
    build_tables();
    operand_t A, B;
    make_ops(&A, &B, a, sfa, b, sfb, 0, K);
    if (a_mn) { A.row_stride = 1; A.k_stride = M; }
    if (b_mn) { B.row_stride = 1; B.k_stride = N; }
#pragma omp parallel for schedule(dynamic)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double base = c ? bf16_bits_to_double(c[m * N + n]) : 0.0;
            out[m * N + n] = base + dot(&A, m, &B, n, K);
        }
}
