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

// The kprime-th largest of the nonzero keys key(j), j in [0, jend), found by one warp
// with a 4-pass radix select (8-bit digits, a 256-bin histogram in shared memory):
// returns tau = that key and need_eq = how many keys equal to tau are among the
// kprime largest (>= 1).  kprime <= 0 gives tau = 0xFFFFFFFF, need_eq = 0.
template <typename KeyFn>
__device__ __forceinline__ void radix_kth(KeyFn key, int jend, int kprime, uint32_t* hist, int lane, uint32_t& tau,
                                          int& need_eq) {
  tau = 0xFFFFFFFFu;
  need_eq = 0;
  if (kprime <= 0) return;
  uint32_t prefix = 0, pmask = 0;
  int remaining = kprime;  // keys still to take among those matching the prefix
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
#pragma unroll
    for (int q = 0; q < 8; ++q) hist[lane * 8 + q] = 0u;
    __syncwarp();
    for (int j = lane; j < jend; j += 32) {
      const uint32_t k = key(j);
      if (k != 0u && (k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
    }
    __syncwarp();
    // lane l owns digits [8l, 8l+8); counts above each lane's range by a suffix scan
    uint32_t hv[8];
    uint32_t lsum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      hv[q] = hist[lane * 8 + q];
      lsum += hv[q];
    }
    uint32_t above = lsum;  // inclusive suffix sum over lanes >= this one
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_down_sync(0xffffffffu, above, o);
      if (lane + o < 32) above += t;
    }
    const uint32_t above_excl = above - lsum;  // keys in higher lanes' digits
    // the lane whose range holds the remaining-th largest key
    const bool mine = above_excl < (uint32_t)remaining && above >= (uint32_t)remaining;
    int digit = 0, rem_new = 0;
    if (mine) {
      uint32_t cum = above_excl;
#pragma unroll
      for (int q = 7; q >= 0; --q) {
        if (cum + hv[q] >= (uint32_t)remaining) {
          digit = lane * 8 + q;
          rem_new = remaining - (int)cum;
          break;
        }
        cum += hv[q];
      }
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, mine);
    const int src = __ffs(bal) - 1;
    digit = __shfl_sync(0xffffffffu, digit, src);
    rem_new = __shfl_sync(0xffffffffu, rem_new, src);
    prefix |= (uint32_t)digit << shift;
    pmask |= 0xFFu << shift;
    remaining = rem_new;
    __syncwarp();
  }
  tau = prefix;
  need_eq = remaining;
}

// Scores + selection for R consecutive query tiles of one (b, hq).
// grid (ceil(T / R), B*Hq), 32*R threads: R warps.
// Scores: thread t takes the key tiles j = t, t + 32R, ... and accumulates the R
// rows' dot products together, so each pooled key column is read once per CTA.
// Selection: warp r takes query tile i0 + r.
//  VERT = false (score mode): the kprime largest candidate scores (ties by index
//    ascending); when `votes` is not null, every tile taken besides the forced
//    ones adds one vote to its column, votes[b, hq, j].
//  VERT = true (vertical-line mode): the candidates ranked by (votes desc,
//    score desc, index asc), votes from a score-mode pass: first the vote count
//    of the kprime-th candidate, then the scores among the candidates with that
//    count.
// Dynamic shared memory: R * T keys (uint32).
template <int D, int R, bool VERT>
__global__ void __launch_bounds__(32 * R) topk_kernel(const float* __restrict__ qp, const float* __restrict__ kpT,
                                                      int Hq, int Hkv, int T, int W, int causal, int budget_bp,
                                                      int budget_tiles, uint32_t* __restrict__ mask,
                                                      int32_t* __restrict__ counts, int32_t* __restrict__ votes) {
  constexpr int NT = 32 * R;
  extern __shared__ uint32_t keys[];  // [R][T]
  __shared__ float qs[R][D];
  __shared__ uint32_t hist[R][256];
  const int i0 = blockIdx.x * R, bhq = blockIdx.y;
  const int b = bhq / Hq, h = bhq % Hq;
  const int bhk = b * Hkv + h / (Hq / Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int x = threadIdx.x; x < R * D; x += NT) {
    const int r = x / D, c = x % D;
    qs[r][c] = (i0 + r < T) ? qp[((long long)bhq * T + i0 + r) * D + c] : 0.0f;
  }
  __syncthreads();

  // per-row budget: forced {0, i} count toward k_i
  auto budget = [&](int i, int& n_i, int& nf, int& k_i) {
    n_i = causal ? i + 1 : T;
    nf = (i == 0) ? 1 : 2;
    if (budget_tiles > 0) k_i = min(n_i, max(nf, budget_tiles));
    else if (budget_bp <= 0) k_i = 0;
    else if (budget_bp >= 10000) k_i = n_i;
    else k_i = min(n_i, max(nf, (int)(((long long)budget_bp * n_i + 9999) / 10000)));
  };

  // scores in FP32, channels in ascending order, separately rounded multiply and add
  const float* kcol = kpT + (long long)bhk * D * T;
  const int jmax = causal ? min(T, i0 + R) : T;  // no row of this CTA looks past it
  for (int j = threadIdx.x; j < jmax; j += NT) {
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.0f;
#pragma unroll 16
    for (int c = 0; c < D; ++c) {
      const float kv = __ldg(kcol + (long long)c * T + j);
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] = __fadd_rn(acc[r], __fmul_rn(qs[r][c], kv));
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = i0 + r;
      uint32_t kk = 0;  // 0: not a candidate
      if (i < T) {
        int n_i, nf, k_i;
        budget(i, n_i, nf, k_i);
        if (j < n_i && j != 0 && j != i && k_i > nf) kk = order_key(acc[r]);
      }
      keys[r * T + j] = kk;
    }
  }
  __syncthreads();

  const int i = i0 + warp;
  if (i >= T) return;
  int n_i, nf, k_i;
  budget(i, n_i, nf, k_i);
  const int kprime = k_i > 0 ? k_i - nf : 0;
  const uint32_t* key = keys + warp * T;
  const int jend = causal ? n_i : T;  // keys past the causal limit were never written
  const int32_t* vrow = VERT ? votes + (long long)bhq * T : nullptr;
  // VERT: key1(j) = votes + 1 for candidates (0 otherwise), key2(j) = the score key of the
  // candidates whose key1 is the threshold v1
  uint32_t v1 = 0xFFFFFFFFu;
  int need_v = 0;
  if (VERT) {
    radix_kth([&](int j) -> uint32_t { return key[j] != 0u ? (uint32_t)__ldg(vrow + j) + 1u : 0u; }, jend, kprime,
              hist[warp], lane, v1, need_v);
  }
  auto key2 = [&](int j) -> uint32_t {
    if (j >= jend) return 0u;
    const uint32_t k = key[j];
    if (!VERT) return k;
    return (k != 0u && (uint32_t)__ldg(vrow + j) + 1u == v1) ? k : 0u;
  };
  uint32_t tau;
  int need_eq;
  radix_kth(key2, jend, VERT ? need_v : kprime, hist[warp], lane, tau, need_eq);
  // bit j set: forced tile; VERT: more votes than v1 - 1; then key above tau, or one of
  // the first need_eq keys equal to tau in ascending tile order
  int eq_seen = 0, total = 0;
  for (int wd = 0; wd < W; ++wd) {
    const int j = wd * 32 + lane;
    const uint32_t k = key2(j);
    const bool eq = k != 0u && k == tau;
    const uint32_t beq = __ballot_sync(0xffffffffu, eq);
    const int before = eq_seen + __popc(beq & ((1u << lane) - 1u));
    const bool forced = k_i > 0 && j < n_i && (j == 0 || j == i);
    bool pick = (k != 0u && k > tau) || (eq && before < need_eq);
    if (VERT && j < jend && key[j] != 0u && (uint32_t)__ldg(vrow + j) + 1u > v1) pick = true;
    const bool bit = forced || (pick && kprime > 0);
    const uint32_t word = __ballot_sync(0xffffffffu, bit);
    if (lane == 0) mask[((long long)bhq * T + i) * W + wd] = word;
    if (!VERT && votes != nullptr && bit && !forced) atomicAdd(votes + (long long)bhq * T + j, 1);
    eq_seen += __popc(beq);
    total += __popc(word);
  }
  if (counts != nullptr && lane == 0) counts[(long long)bhq * T + i] = total;
}

template <int D>
static void launch_select_d(const SelectArgs& a, int T, int W, float* qp, float* kpT, cudaStream_t s) {
  const int BHq = a.B * a.Hq, BHk = a.B * a.Hkv;
  constexpr int R = 8;
  const size_t dyn = (size_t)R * T * 4;
  const dim3 gp(T, BHq + BHk), gt((T + R - 1) / R, BHq);
  pool_kernel<D><<<gp, D / 2, 0, s>>>(a.q, a.k, BHq, a.N, T, qp, kpT);
  if (dyn > 48 * 1024) cudaFuncSetAttribute(topk_kernel<D, R, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
  topk_kernel<D, R, false><<<gt, 32 * R, dyn, s>>>(qp, kpT, a.Hq, a.Hkv, T, W, a.causal, a.budget_bp, a.budget_tiles,
                                                   a.mask, a.counts, a.votes);
  count_launches(2);
  if (a.vertical) {
    if (dyn > 48 * 1024) cudaFuncSetAttribute(topk_kernel<D, R, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    topk_kernel<D, R, true><<<gt, 32 * R, dyn, s>>>(qp, kpT, a.Hq, a.Hkv, T, W, a.causal, a.budget_bp, a.budget_tiles,
                                                    a.mask, a.counts, a.votes);
    count_launches(1);
  }
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t s) {
  const int T = (a.N + 127) / 128, W = (T + 31) / 32;
  const int BHq = a.B * a.Hq;
  float* qp = a.pool_ws;
  float* kpT = qp + (size_t)BHq * T * a.d;
  if (a.vertical) {
    cudaError_t err = cudaMemsetAsync(a.votes, 0, sizeof(int32_t) * (size_t)BHq * T, s);
    if (err != cudaSuccess) return err;
  }
  if (a.d == 128) launch_select_d<128>(a, T, W, qp, kpT, s);
  else launch_select_d<64>(a, T, W, qp, kpT, s);
  return cudaGetLastError();
}

}  // namespace thrift
