// Stage 1: choose the query-key tile pairs that run in BF16.
//
// ThriftAttention: Selective Mixed Precision for Long-Context FP4 Attention
// (abstract, first stage): a cheap heuristic selects a few important
// query-key block pairs for high precision.  HyQuant: Hybrid-Precision
// Quantization for LLM Attention (abstract): sink ("vertical line") tokens
// and the local window stay in full precision.  This library's rule: mean
// pooled 128-row tiles, score = pooled q . pooled k, forced sink tile 0 and
// diagonal tile i, the rest of the per-row budget by top-k.
//
// Bit-exactness with the CPU statement of the rule comes from fixed FP32
// operation order: pooled sums in ascending rows, dot products in ascending
// channels with separately rounded multiplies and adds, and an exact
// radix selection with (score desc, index asc) tie-breaking.
#include "dev.cuh"
#include "kernels.h"

namespace thrift {

// Pooled column means.  grid (T, B*Hq + B*Hkv); thread = 2 channels.
// Q means -> qp[bh][t][c]; K means -> kpT[bh][c][t] (channel-major, so the
// score kernel reads them coalesced).
template <int D>
__global__ void __launch_bounds__(D / 2) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                      const __nv_bfloat16* __restrict__ k, int BHq, int N, int T,
                                                      float* __restrict__ qp, float* __restrict__ kpT) {
  const int t = blockIdx.x, y = blockIdx.y;
  const bool isq = y < BHq;
  const int bh = isq ? y : y - BHq;
  const __nv_bfloat16* x = isq ? q : k;
  const int c = threadIdx.x * 2;
  const int r0 = t * 128;
  const int cnt = min(128, N - r0);
  const uint32_t* p = reinterpret_cast<const uint32_t*>(x + ((long long)bh * N + r0) * D + c);
  float s0 = 0.0f, s1 = 0.0f;
#pragma unroll 8
  for (int r = 0; r < cnt; ++r) {
    const uint32_t w = __ldg(p + (long long)r * (D / 2));
    s0 = __fadd_rn(s0, __uint_as_float(w << 16));
    s1 = __fadd_rn(s1, __uint_as_float(w & 0xFFFF0000u));
  }
  const float fc = (float)cnt;
  const float m0 = __fdiv_rn(s0, fc), m1 = __fdiv_rn(s1, fc);
  if (isq) {
    float* o = qp + ((long long)bh * T + t) * D + c;
    o[0] = m0;
    o[1] = m1;
  } else {
    kpT[((long long)bh * D + c) * T + t] = m0;
    kpT[((long long)bh * D + c + 1) * T + t] = m1;
  }
}

// IEEE float -> uint key whose unsigned order is the float order; -0 == +0.
// Every finite float maps to a key >= 1, so 0 marks "not a candidate".
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.0f) f = 0.0f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int NT>
__device__ __forceinline__ int block_sum(int v, int* red) {
  v = __reduce_add_sync(0xffffffffu, v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  int s = 0;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) s += red[i];
  return s;
}

// Scores + selection for one (b, hq, query tile i).  grid (T, B*Hq), 256 threads.
// Dynamic shared memory: T keys (uint32) + T selection bytes.
template <int D>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ qp, const float* __restrict__ kpT,
                                                   int Hq, int Hkv, int T, int W, int causal, int budget_bp,
                                                   int budget_tiles, uint32_t* __restrict__ mask,
                                                   int32_t* __restrict__ counts) {
  constexpr int NT = 256;
  extern __shared__ uint32_t dyn[];
  uint32_t* key = dyn;
  uint8_t* sel = reinterpret_cast<uint8_t*>(dyn + T);
  __shared__ float qs[D];
  __shared__ int red[NT / 32];
  __shared__ int eq_base;
  const int i = blockIdx.x, bhq = blockIdx.y;
  const int b = bhq / Hq, h = bhq % Hq;
  const int bhk = b * Hkv + h / (Hq / Hkv);
  for (int c = threadIdx.x; c < D; c += NT) qs[c] = qp[((long long)bhq * T + i) * D + c];
  __syncthreads();

  const int n_i = causal ? i + 1 : T;
  const int nf = (i == 0) ? 1 : 2;  // forced {0, i}, both always candidates
  int k_i;
  if (budget_tiles > 0) k_i = min(n_i, max(nf, budget_tiles));
  else if (budget_bp <= 0) k_i = 0;
  else if (budget_bp >= 10000) k_i = n_i;
  else k_i = min(n_i, max(nf, (int)(((long long)budget_bp * n_i + 9999) / 10000)));
  const int kprime = k_i > 0 ? k_i - nf : 0;

  const float* kcol = kpT + (long long)bhk * D * T;
  for (int j = threadIdx.x; j < T; j += NT) {
    uint32_t kk = 0;
    const bool forced = (j == 0 || j == i);
    if (j < n_i && !forced && kprime > 0) {
      float acc = 0.0f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) acc = __fadd_rn(acc, __fmul_rn(qs[c], __ldg(kcol + (long long)c * T + j)));
      kk = order_key(acc);
    }
    key[j] = kk;
    sel[j] = (k_i > 0 && forced && j < n_i) ? 1 : 0;
  }
  __syncthreads();

  if (kprime > 0) {
    // tau = the kprime-th largest key among candidates (bitwise search).
    uint32_t tau = 0;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = tau | (1u << bit);
      int cnt = 0;
      for (int j = threadIdx.x; j < T; j += NT) cnt += (key[j] >= cand) ? 1 : 0;
      if (block_sum<NT>(cnt, red) >= kprime) tau = cand;
    }
    int gt = 0;
    for (int j = threadIdx.x; j < T; j += NT) gt += (key[j] > tau) ? 1 : 0;
    const int n_gt = block_sum<NT>(gt, red);
    const int need_eq = kprime - n_gt;  // >= 1
    if (threadIdx.x == 0) eq_base = 0;
    __syncthreads();
    // keys > tau all selected; keys == tau selected in ascending index order.
    for (int j0 = 0; j0 < T; j0 += NT) {
      const int j = j0 + threadIdx.x;
      const bool eq = (j < T) && key[j] == tau;
      const uint32_t bal = __ballot_sync(0xffffffffu, eq);
      const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
      __syncthreads();
      if (lane == 0) red[w] = __popc(bal);
      __syncthreads();
      int before = eq_base;
      for (int q = 0; q < w; ++q) before += red[q];
      before += __popc(bal & ((1u << lane) - 1u));
      if (j < T) {
        if (key[j] > tau) sel[j] = 1;
        else if (eq && before < need_eq) sel[j] = 1;
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        int s = 0;
        for (int q = 0; q < NT / 32; ++q) s += red[q];
        eq_base += s;
      }
      __syncthreads();
    }
  }
  __syncthreads();
  // pack the bitmask: one warp per 32-tile word
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int pc = 0;
  for (int wd = warp; wd < W; wd += NT / 32) {
    const int j = wd * 32 + lane;
    const bool bit = (j < T) && sel[j];
    const uint32_t word = __ballot_sync(0xffffffffu, bit);
    if (lane == 0) mask[((long long)bhq * T + i) * W + wd] = word;
    pc += (lane == 0) ? __popc(word) : 0;
  }
  const int total = block_sum<NT>(pc, red);
  if (counts != nullptr && threadIdx.x == 0) counts[(long long)bhq * T + i] = total;
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t s) {
  const int D = a.d, T = (a.N + 127) / 128, W = (T + 31) / 32;
  const int BHq = a.B * a.Hq, BHk = a.B * a.Hkv;
  float* qp = a.pool_ws;
  float* kpT = qp + (size_t)BHq * T * D;
  dim3 gp(T, BHq + BHk);
  const size_t dyn = (size_t)T * 5 + 16;
  if (D == 128) {
    pool_kernel<128><<<gp, 64, 0, s>>>(a.q, a.k, BHq, a.N, T, qp, kpT);
    if (dyn > 48 * 1024) cudaFuncSetAttribute(topk_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    topk_kernel<128><<<dim3(T, BHq), 256, dyn, s>>>(qp, kpT, a.Hq, a.Hkv, T, W, a.causal, a.budget_bp,
                                                    a.budget_tiles, a.mask, a.counts);
  } else {
    pool_kernel<64><<<gp, 32, 0, s>>>(a.q, a.k, BHq, a.N, T, qp, kpT);
    if (dyn > 48 * 1024) cudaFuncSetAttribute(topk_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    topk_kernel<64><<<dim3(T, BHq), 256, dyn, s>>>(qp, kpT, a.Hq, a.Hkv, T, W, a.causal, a.budget_bp,
                                                   a.budget_tiles, a.mask, a.counts);
  }
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace thrift
