// dg_probe.cuh -- tensor-core throughput probe for sm_100a.
//
// One CTA per SM issues back-to-back tcgen05 MMAs from operand tiles that
// stay in shared memory (no global-memory traffic inside the loop), so the
// CUDA-event time of a launch measures the tensor pipe alone.  Used to put a
// measured denominator beside the nominal dense FP8 peak (4.5 PFLOP/s per
// B200) when reporting how close the GEMM kernels come to the tensor roofline.
//
// Kinds:
//   kProbeScaled  kind::mxf8f6f4.block_scale, e4m3 x e4m3, UE8M0 scales
//                 (the instruction the GEMM kernels issue)
//   kProbePlain   kind::f8f6f4, e4m3 x e4m3, no scales (the instruction of
//                 the per-K-block promotion variant)
//   kProbeBf16    kind::f16 with bf16 operands (comparable with cuBLAS bf16)
// Each K-block is 4 MMAs of M = 128, N = BN, K = 32 (bf16: K = 16, so a bf16
// K-block is 4 x 16 deep and counts half the FLOPs of an e4m3 one).
#pragma once
#include "dg_ptx.cuh"

namespace dg {

enum : int { kProbeScaled = 0, kProbePlain = 1, kProbeBf16 = 2 };

// Instruction descriptor of kind::f8f6f4: FP32 accumulator (bits 4-5 = 1),
// A and B e4m3 (formats 0), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_f8f6f4(int m, int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

constexpr int kProbeThreads = 128;
constexpr int kProbeSmem = 1024 + 128 * 128 + 256 * 128 + 1024 + 64;

template <int KIND, int BN>
__global__ void __launch_bounds__(kProbeThreads, 1) mma_peak_kernel(int kblocks, unsigned long long timeout_ns) {
  extern __shared__ __align__(1024) uint8_t probe_smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(probe_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_a = smem;                  // 128 rows x 128 bytes
  uint8_t* s_b = s_a + 128 * 128;       // 256 rows x 128 bytes
  uint8_t* s_sf = s_b + 256 * 128;      // 2 x 512 bytes of scale words
  uint64_t* bar = reinterpret_cast<uint64_t*>(s_sf + 1024);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  const int warp = threadIdx.x / 32;

  // operands: e4m3 1.0 (0x38) or bf16 1.0 (0x3F80) everywhere; scale code 127
  const uint32_t fill = (KIND == kProbeBf16) ? 0x3F803F80u : 0x38383838u;
  for (int i = threadIdx.x; i < (128 * 128 + 256 * 128) / 4; i += kProbeThreads)
    reinterpret_cast<uint32_t*>(s_a)[i] = fill;
  for (int i = threadIdx.x; i < 1024 / 4; i += kProbeThreads) reinterpret_cast<uint32_t*>(s_sf)[i] = 0x7F7F7F7Fu;
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  if (threadIdx.x == 0) {
    const uint32_t d_t = tmem;                // BN accumulator columns at 0
    const uint32_t sfa_t = tmem + 256;        // 4 columns
    const uint32_t sfb_t = tmem + 260;        // 8 columns (two 128-row chunks)
    if (KIND == kProbeScaled) {
      tc_cp_32x128b_x4(sfa_t, sdesc_sf_32x16(s_sf));
      tc_cp_32x128b_x4(sfb_t, sdesc_sf_32x16(s_sf + 512));
      tc_cp_32x128b_x4(sfb_t + 4, sdesc_sf_32x16(s_sf + 512));
    }
    const uint64_t adesc = sdesc_k_sw128(s_a);
    const uint64_t bdesc = sdesc_k_sw128(s_b);
    constexpr uint32_t kIdScaled = (0u << 7) | (0u << 10) | ((uint32_t)(BN >> 3) << 17) | (1u << 23) | (8u << 24);
    constexpr uint32_t kIdBf16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | (8u << 24);
    for (int kb = 0; kb < kblocks; ++kb) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint32_t acc = (kb > 0 || ks > 0) ? 1u : 0u;
        if constexpr (KIND == kProbeScaled)
          tc_mma_mxf8f6f4(d_t, adesc + 2 * ks, bdesc + 2 * ks, kIdScaled, sfa_t, sfb_t, acc);
        else if constexpr (KIND == kProbePlain)
          tc_mma_f8f6f4(d_t, adesc + 2 * ks, bdesc + 2 * ks, idesc_f8f6f4(128, BN), acc);
        else
          tc_mma_f16(d_t, adesc + 2 * ks, bdesc + 2 * ks, kIdBf16, acc);
      }
    }
    tc_commit(bar);
    if (!dg_wait(bar, 0, s_abort, timeout_ns)) {
      // the MMAs are still in flight: wait (bounded) before TMEM is freed
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(bar, 0) && global_timer_ns() - t0 < timeout_ns) {
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace dg
