// Tensor-core rate probe: how many dense FLOPs per second this GPU's tcgen05
// pipe delivers for the three MMA forms the attention kernel issues, so that
// its roofline can be stated against measured rates as well as nominal ones.
//
//   kind 0: kind::mxf4nvf4.block_scale.scale_vec::4X, A and B in shared memory,
//           128 x N x 64 per instruction (the FP4 Q K^T product);
//   kind 1: kind::f8f6f4 e4m3, A in tensor memory, B in shared memory,
//           128 x N x 32 per instruction (the FP8 P V product);
//   kind 2: kind::f16 BF16, A and B in shared memory, 128 x N x 16 per
//           instruction (the BF16 Q K^T product).
//
// One CTA per SM; one thread issues `iters` K=128 steps into one FP32
// accumulator in tensor memory and waits (bounded) for their completion.  The
// operands are fixed pseudo-random bytes without NaN codes; their values do
// not change the tensor pipe's rate.
#include "dev.cuh"
#include "kernels.h"

namespace thrift {
namespace probe {

constexpr int kThreads = 128;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ uint32_t g_probe_error;

template <int KIND, int N>
struct ProbeLayout {
  // A: 128 rows x 128 K-elements; B: N rows x 128 K-elements
  static constexpr int ROW_A = KIND == 0 ? 64 : (KIND == 1 ? 128 : 256);  // bytes per 128 elements
  static constexpr int A_BYTES = 128 * ROW_A;
  static constexpr int B_BYTES = N * ROW_A;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = A_BYTES;
  static constexpr int OFF_SF = OFF_B + B_BYTES;          // 2 x 512 (A) + 2 x 512 (B) scale bytes
  static constexpr int OFF_BAR = OFF_SF + 4096;
  static constexpr int BYTES = OFF_BAR + 64;
};

__device__ __forceinline__ uint32_t mix(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7feb352dU;
  x ^= x >> 15;
  x *= 0x846ca68bU;
  x ^= x >> 16;
  return x;
}

template <int KIND, int N>
__global__ void __launch_bounds__(kThreads, 1) mma_probe_kernel(int iters, unsigned long long* cycles) {
  using L = ProbeLayout<KIND, N>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  __shared__ uint32_t tmem_holder;
  const int tid = threadIdx.x, warp = tid >> 5;
  // operands: FP4 any nibble; e4m3 bytes masked to 0x3F|sign (no NaN); bf16 small normal values
  uint32_t* w = reinterpret_cast<uint32_t*>(smem);
  for (int i = tid; i < (L::OFF_SF) / 4; i += kThreads) {
    const uint32_t r = mix(i * 2654435761u + blockIdx.x);
    uint32_t val = r;
    if (KIND == 1) val = r & 0xBFBFBFBFu;
    if (KIND == 2) val = (r & 0x807F807Fu) | 0x3E003E00u;
    w[i] = val;
  }
  for (int i = tid; i < 4096 / 4; i += kThreads) w[L::OFF_SF / 4 + i] = 0x38383838u;  // scale 1.0
  const uint32_t bar = sb + L::OFF_BAR;
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_holder;
  if (KIND == 1) {
    // A operand (P) in tensor memory columns [256, 256 + 32): e4m3 bytes, four per column
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    uint32_t r[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) r[c] = mix(tid * 64 + c) & 0x3F3F3F3Fu;
    tmem_st32(tmem + lane_base + 256, r);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) {
    const uint32_t d = tmem;  // accumulator columns [0, N)
    if (KIND == 0) {
      tmem_cp_32x128b_x4(tmem + 384, smem_desc(sb + L::OFF_SF, 16, 128, SWZ_NONE));
      tmem_cp_32x128b_x4(tmem + 388, smem_desc(sb + L::OFF_SF + 512, 16, 128, SWZ_NONE));
      tmem_cp_32x128b_x4(tmem + 392, smem_desc(sb + L::OFF_SF + 1024, 16, 128, SWZ_NONE));
      tmem_cp_32x128b_x4(tmem + 396, smem_desc(sb + L::OFF_SF + 1536, 16, 128, SWZ_NONE));
    }
    const unsigned long long c0 = clock64();
    for (int it = 0; it < iters; ++it) {
      if (KIND == 0) {
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
          mma_nvfp4_ss(d, smem_desc(sb + L::OFF_A + kb * 32, 16, 512, SWZ_64B),
                       smem_desc(sb + L::OFF_B + kb * 32, 16, 512, SWZ_64B), idesc_nvfp4(N), tmem + 384 + 4 * kb,
                       tmem + 392 + 4 * kb, (it > 0 || kb > 0) ? 1u : 0u);
      } else if (KIND == 1) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_e4m3_ts(d, tmem + 256 + 8 * k, smem_desc(sb + L::OFF_B + k * 32, 16, 1024, SWZ_128B), idesc_e4m3(N),
                      (it > 0 || k > 0) ? 1u : 0u);
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off_a = (k >> 2) * (128 * 128) + (k & 3) * 32;
          const uint32_t off_b = (k >> 2) * (N * 128) + (k & 3) * 32;
          mma_bf16_ss(d, smem_desc(sb + L::OFF_A + off_a, 16, 1024, SWZ_128B),
                      smem_desc(sb + L::OFF_B + off_b, 16, 1024, SWZ_128B), idesc_bf16(N), (it > 0 || k > 0) ? 1u : 0u);
        }
      }
    }
    tc_commit(bar);
    volatile int never = 0;
    if (!mbar_wait(bar, 0, &never, kWaitLimitNs)) atomicOr(&g_probe_error, 1u);
    const unsigned long long c1 = clock64();
    cycles[blockIdx.x] = c1 - c0;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int KIND, int N>
static int run(int iters, int ctas, float* ms, unsigned long long* cycles_dev, cudaStream_t st) {
  using L = ProbeLayout<KIND, N>;
  auto kern = mma_probe_kernel<KIND, N>;
  // at least 116 KB of shared memory: one CTA (and its 512 TMEM columns) per SM
  const int dyn = (L::BYTES + 1024 > 116 * 1024) ? L::BYTES + 1024 : 116 * 1024;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn) != cudaSuccess)
    return THRIFT_ERR_CUDA;
  cudaEvent_t e0, e1;
  if (cudaEventCreate(&e0) != cudaSuccess) return THRIFT_ERR_CUDA;
  if (cudaEventCreate(&e1) != cudaSuccess) {
    cudaEventDestroy(e0);
    return THRIFT_ERR_CUDA;
  }
  cudaEventRecord(e0, st);
  kern<<<ctas, kThreads, dyn, st>>>(iters, cycles_dev);
  count_launches(1);
  cudaEventRecord(e1, st);
  cudaError_t err = cudaEventSynchronize(e1);
  if (err == cudaSuccess) err = cudaEventElapsedTime(ms, e0, e1);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  if (err != cudaSuccess || cudaGetLastError() != cudaSuccess) return THRIFT_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpyFromSymbol(&word, g_probe_error, sizeof(word)) != cudaSuccess) return THRIFT_ERR_CUDA;
  if (word != 0) {
    const uint32_t zero = 0;
    cudaMemcpyToSymbol(g_probe_error, &zero, sizeof(zero));
    return THRIFT_ERR_TIMEOUT;
  }
  return THRIFT_OK;
}

}  // namespace probe

int launch_mma_probe(int kind, int n, int iters, int ctas, float* ms, unsigned long long* cycles_dev,
                     cudaStream_t st) {
  using namespace probe;
  if (kind == 0 && n == 128) return run<0, 128>(iters, ctas, ms, cycles_dev, st);
  if (kind == 1 && n == 128) return run<1, 128>(iters, ctas, ms, cycles_dev, st);
  if (kind == 1 && n == 256) return run<1, 256>(iters, ctas, ms, cycles_dev, st);
  if (kind == 2 && n == 128) return run<2, 128>(iters, ctas, ms, cycles_dev, st);
  if (kind == 2 && n == 256) return run<2, 256>(iters, ctas, ms, cycles_dev, st);
  return THRIFT_ERR_UNSUPPORTED;
}

}  // namespace thrift
