// dg_prep.cuh -- input preparation kernels: fine-grained quantisation of FP32
// data to E4M3 (1x128 or 128x128 groups) or E2M1 (1x32 groups) with UE8M0
// power-of-two scales, and packing of UE8M0 codes 4 per int32 into the layout
// the GEMM kernel copies straight into tensor memory.
//
// Sources: "DeepSeek 开源第三弹 ... DeepGEMM" (app.myzaker.com), section
// "DeepGEMM" (DeepSeek-V3 fine-grained scaling); "DeepSeek 发布 DeepGEMM 重大更新"
// (linlog.top), section "FP4 精度支持" (UE8M0 scale factors packed 4 per
// int32); "DeepGEMM：FP8 GEMM 与 Mega-MoE" (charles2530.github.io), section
// "难点解释：为什么 scale layout 也是接口" (the scale layout is part of the
// interface and must suit TMA).
#pragma once
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include "dg_ptx.cuh"

namespace dg {

// Least i with qmax * 2^i >= amax (amax > 0, finite), clamped to [-127, 127].
// qmax = 448 = 1.75 * 2^8 for E4M3 and 6 = 1.5 * 2^2 for E2M1.  Writing
// amax = 1.m * 2^e: qmax * 2^i >= amax  <=>  i >= e - emax + [1.m > 1.qmax].
__device__ __forceinline__ int scale_exp(float amax, int qmax_exp, uint32_t qmax_mant) {
  if (!(amax > 0.f)) return 0;
  int bias = 0;
  if (amax < 1e-30f) {  // lift subnormals into the normal range exactly
    amax *= 18446744073709551616.0f;  // 2^64
    bias = 64;
  }
  const uint32_t u = __float_as_uint(amax);
  const int e = (int)((u >> 23) & 0xFF) - 127 - bias;
  const uint32_t m = u & 0x7FFFFFu;
  int i = e - qmax_exp + (m > qmax_mant ? 1 : 0);
  return min(max(i, -127), 127);
}

// Exact 2^-i as a float for i in [-127, 126].
__device__ __forceinline__ float pow2_neg(int i) {
  return __uint_as_float((uint32_t)(127 - i) << 23);
}

constexpr int kE4M3MaxExp = 8;
constexpr uint32_t kE4M3MaxMant = 0x600000u;  // 448 = 1.75 * 2^8
constexpr int kE2M1MaxExp = 2;
constexpr uint32_t kE2M1MaxMant = 0x400000u;  // 6 = 1.5 * 2^2

// 1x128 groups: one warp per (row, group); each lane owns 4 consecutive values.
__global__ void quant_fp8_1x128_kernel(const float* __restrict__ x, long long rows, int cols,
                                       uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  const int groups = cols / 128;
  const long long nwarps = rows * groups;
  const int lane = threadIdx.x & 31;
  for (long long w = (blockIdx.x * (long long)blockDim.x + threadIdx.x) / 32; w < nwarps;
       w += (long long)gridDim.x * blockDim.x / 32) {
    const long long r = w / groups;
    const int g = (int)(w - r * groups);
    const long long off = r * cols + g * 128 + lane * 4;
    const float4 v = __ldg(reinterpret_cast<const float4*>(x + off));
    float amax = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int i = scale_exp(amax, kE4M3MaxExp, kE4M3MaxMant);
    const float s = pow2_neg(i);
    const uint32_t b0 = __nv_cvt_float_to_fp8(v.x * s, __NV_SATFINITE, __NV_E4M3);
    const uint32_t b1 = __nv_cvt_float_to_fp8(v.y * s, __NV_SATFINITE, __NV_E4M3);
    const uint32_t b2 = __nv_cvt_float_to_fp8(v.z * s, __NV_SATFINITE, __NV_E4M3);
    const uint32_t b3 = __nv_cvt_float_to_fp8(v.w * s, __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<uint32_t*>(q + off) = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
    if (lane == 0) sf[r * groups + g] = (uint8_t)(i + 127);
  }
}

// 128x128 blocks: one CTA (256 threads) per block.
__global__ void quant_fp8_128x128_kernel(const float* __restrict__ x, long long rows, int cols,
                                         uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  __shared__ float red[8];
  const int groups = cols / 128;
  const long long rblocks = (rows + 127) / 128;
  for (long long blk = blockIdx.x; blk < rblocks * groups; blk += gridDim.x) {
    const long long br = blk / groups;
    const int bc = (int)(blk - br * groups);
    float amax = 0.f;
    for (int u = threadIdx.x; u < 128 * 32; u += blockDim.x) {
      const long long r = br * 128 + u / 32;
      if (r < rows) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(x + r * cols + bc * 128 + (u % 32) * 4));
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = amax;
    __syncthreads();
    amax = red[0];
    for (int k = 1; k < (int)(blockDim.x / 32); ++k) amax = fmaxf(amax, red[k]);
    __syncthreads();
    const int i = scale_exp(amax, kE4M3MaxExp, kE4M3MaxMant);
    const float s = pow2_neg(i);
    for (int u = threadIdx.x; u < 128 * 32; u += blockDim.x) {
      const long long r = br * 128 + u / 32;
      if (r < rows) {
        const long long off = r * cols + bc * 128 + (u % 32) * 4;
        const float4 v = __ldg(reinterpret_cast<const float4*>(x + off));
        const uint32_t b0 = __nv_cvt_float_to_fp8(v.x * s, __NV_SATFINITE, __NV_E4M3);
        const uint32_t b1 = __nv_cvt_float_to_fp8(v.y * s, __NV_SATFINITE, __NV_E4M3);
        const uint32_t b2 = __nv_cvt_float_to_fp8(v.z * s, __NV_SATFINITE, __NV_E4M3);
        const uint32_t b3 = __nv_cvt_float_to_fp8(v.w * s, __NV_SATFINITE, __NV_E4M3);
        *reinterpret_cast<uint32_t*>(q + off) = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
      }
    }
    if (threadIdx.x == 0) sf[br * groups + bc] = (uint8_t)(i + 127);
  }
}

// 1x32 groups to E2M1, two codes per byte (low nibble = even column); four
// threads per group, eight values per thread.
__global__ void quant_fp4_1x32_kernel(const float* __restrict__ x, long long rows, int cols,
                                      uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  const int groups = cols / 32;
  const long long nthr = rows * groups * 4;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < nthr;
       t += (long long)gridDim.x * blockDim.x) {
    const long long gidx = t / 4;
    const int sub = (int)(t & 3);
    const long long r = gidx / groups;
    const int g = (int)(gidx - r * groups);
    const long long off = r * cols + g * 32 + sub * 8;
    const float4 v0 = __ldg(reinterpret_cast<const float4*>(x + off));
    const float4 v1 = __ldg(reinterpret_cast<const float4*>(x + off + 4));
    float amax = fmaxf(fmaxf(fmaxf(fabsf(v0.x), fabsf(v0.y)), fmaxf(fabsf(v0.z), fabsf(v0.w))),
                       fmaxf(fmaxf(fabsf(v1.x), fabsf(v1.y)), fmaxf(fabsf(v1.z), fabsf(v1.w))));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int i = scale_exp(amax, kE2M1MaxExp, kE2M1MaxMant);
    const float s = pow2_neg(i);
    const uint32_t p0 = __nv_cvt_float2_to_fp4x2(make_float2(v0.x * s, v0.y * s), __NV_E2M1, cudaRoundNearest);
    const uint32_t p1 = __nv_cvt_float2_to_fp4x2(make_float2(v0.z * s, v0.w * s), __NV_E2M1, cudaRoundNearest);
    const uint32_t p2 = __nv_cvt_float2_to_fp4x2(make_float2(v1.x * s, v1.y * s), __NV_E2M1, cudaRoundNearest);
    const uint32_t p3 = __nv_cvt_float2_to_fp4x2(make_float2(v1.z * s, v1.w * s), __NV_E2M1, cudaRoundNearest);
    *reinterpret_cast<uint32_t*>(q + off / 2) = p0 | (p1 << 8) | (p2 << 16) | (p3 << 24);
    if (sub == 0) sf[r * groups + g] = (uint8_t)(i + 127);
  }
}

// Packed scale words: out[Q][Cr][128] int32, Q = ceil(ng/4), Cr = ceil(rows/128).
// The word of (row r, group q) sits at index (r%32)*4 + (r%128)/32 inside
// chunk (q, r/128) -- 32 lines of 16 bytes, line l holding rows l, l+32,
// l+64, l+96 -- which is the 32x128b source shape the MMA warp copies into
// tensor memory unchanged.  Byte j of the word is scale column 4q+j; empty
// bytes hold 127 (= 1.0).  Row r reads row r/row_div of `sf` (row_div = 128
// expands 128x128 block scales to one copy per row).
__global__ void pack_sf_kernel(const uint8_t* __restrict__ sf, long long rows, int ng, int row_div,
                               int32_t* __restrict__ out) {
  const int Q = (ng + 3) / 4;
  const long long Cr = (rows + 127) / 128;
  const long long total = (long long)Q * Cr * 128;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int w = (int)(idx & 127);
    const long long qc = idx >> 7;
    const long long chunk = qc % Cr;
    const int qg = (int)(qc / Cr);
    const long long r = chunk * 128 + (w & 3) * 32 + (w >> 2);
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t byte = 127;
      const int col = 4 * qg + j;
      if (r < rows && col < ng) byte = __ldg(sf + (r / row_div) * ng + col);
      word |= byte << (8 * j);
    }
    out[idx] = (int32_t)word;
  }
}

// Test-only: one thread waits on an mbarrier that nothing ever arrives at,
// through the same bounded wait as the GEMM; it must give up after `limit_ns`
// and record DG_ERR_TIMEOUT.
__global__ void starved_wait_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) dg_wait(&bar, 0, &abort_flag, limit_ns);
}

}  // namespace dg
