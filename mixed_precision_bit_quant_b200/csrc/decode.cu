// One decode step against a mixed-precision KV cache.
//
// HyQuant: Hybrid-Precision Quantization for LLM Attention (abstract, decode
// stage): the KV cache is compressed with the prefill operator's principle --
// sink ("vertical-line") tokens and the local window stay in high precision,
// the rest is low-bit -- and the dequantisation is fused into the attention.
// This library's reading: every cached token is quantised on its own (the
// cache grows a token at a time), K as MXFP4 and V as MXFP8 (e4m3), one e8m0
// scale per 32 channels of the token; tokens [0, 128) and [L - 128, L) are read
// from the BF16 cache; the query stays BF16; exact softmax over all L tokens in
// FP32, the two products on the tensor cores with exact operands (the step reads
// each cached byte once: HBM-bound).
//
// Kernels:
//   decode_quantize_kernel  per-token MX quantisation of cache rows [t0, t1)
//   decode_partial_kernel   one CTA per (b, kv head, chunk of 256 tokens), all G
//                           query heads of the group: logits S = K Q^T and
//                           O = P V on the tensor cores (mma.sync, TF32 operands:
//                           the e2m1, e4m3 and BF16 values are exact in TF32,
//                           P enters as two TF32 terms), dequantisation in
//                           registers, chunk max / exp sum per head; writes the
//                           chunk's softmax state (max, sum, unnormalised O)
//   decode_merge_kernel     combines the chunks' states per query head.
#include "dev.cuh"
#include "kernels.h"

namespace thrift {
namespace dec {

constexpr int kChunk = 256;    // cache tokens per CTA
constexpr int kThreads = 256;  // 8 warps
constexpr int kSink = 128, kWindow = 128;

__device__ __forceinline__ int mx_exp(float amax, int emax) {
  const uint32_t bits = __float_as_uint(amax);
  if (bits == 0u) return -127;
  const int ef = (int)(bits >> 23);
  const int fl = ef > 0 ? ef - 127 : (31 - __clz((int)bits)) - 149;  // floor(log2 amax), subnormals too
  const int e = fl - emax;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// One thread = one 32-channel block of one token of K and of V (rows are [b][hkv][t]).
template <int D>
__global__ void __launch_bounds__(256) decode_quantize_kernel(const __nv_bfloat16* __restrict__ k,
                                                              const __nv_bfloat16* __restrict__ v, int BHk, int L,
                                                              int t0, int t1, uint8_t* __restrict__ kc,
                                                              uint8_t* __restrict__ ksc, uint8_t* __restrict__ vc,
                                                              uint8_t* __restrict__ vsc) {
  constexpr int NB = D / 32;
  const long long nt = t1 - t0;
  const long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= (long long)BHk * nt * NB) return;
  const int blk = (int)(item % NB);
  const long long rr = item / NB;
  const long long row = (rr / nt) * L + t0 + rr % nt;
  const uint4* ks = reinterpret_cast<const uint4*>(k + row * D + blk * 32);
  const uint4* vs = reinterpret_cast<const uint4*>(v + row * D + blk * 32);
  float fk[32], fv[32], ak = 0.0f, av = 0.0f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 a = __ldg(ks + q), b = __ldg(vs + q);
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      fk[8 * q + 2 * e] = __uint_as_float(wa[e] << 16);
      fk[8 * q + 2 * e + 1] = __uint_as_float(wa[e] & 0xFFFF0000u);
      fv[8 * q + 2 * e] = __uint_as_float(wb[e] << 16);
      fv[8 * q + 2 * e + 1] = __uint_as_float(wb[e] & 0xFFFF0000u);
    }
  }
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    ak = fmaxf(ak, fabsf(fk[e]));
    av = fmaxf(av, fabsf(fv[e]));
  }
  // e = floor(log2 amax) - emax (2 for e2m1, 8 for e4m3); 2^-e is a normal FP32
  // power of two because a BF16 block maximum gives e <= 125
  const int ek = mx_exp(ak, 2), ev = mx_exp(av, 8);
  const float mk = __uint_as_float((uint32_t)(127 - ek) << 23), mv = __uint_as_float((uint32_t)(127 - ev) << 23);
  uint32_t wk[4], wv[8];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t x = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      x |= cvt_e2m1x2(__fmul_rn(fk[8 * w + 2 * e], mk), __fmul_rn(fk[8 * w + 2 * e + 1], mk)) << (8 * e);
    wk[w] = x;
  }
#pragma unroll
  for (int w = 0; w < 8; ++w)
    wv[w] = cvt_e4m3x2(__fmul_rn(fv[4 * w], mv), __fmul_rn(fv[4 * w + 1], mv)) |
            (cvt_e4m3x2(__fmul_rn(fv[4 * w + 2], mv), __fmul_rn(fv[4 * w + 3], mv)) << 16);
  *reinterpret_cast<uint4*>(kc + row * (D / 2) + blk * 16) = make_uint4(wk[0], wk[1], wk[2], wk[3]);
  uint4* dv = reinterpret_cast<uint4*>(vc + row * D + blk * 32);
  dv[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
  dv[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
  ksc[row * NB + blk] = (uint8_t)(ek + 127);
  vsc[row * NB + blk] = (uint8_t)(ev + 127);
}

// Two e2m1 codes (one byte, element 2t in the low nibble) -> two floats, exact: the
// hardware conversion to f16x2, then f16 -> f32.
__device__ __forceinline__ float2 e2m1x2_to_float2(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tmov.b16 {t, _}, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(r) : "h"((unsigned short)byte));
  return __half22float2(*reinterpret_cast<const __half2*>(&r));
}
// Two e4m3 codes (low byte first) -> two floats, exact.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\tmov.b16 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(r) : "h"((unsigned short)two));
  return __half22float2(*reinterpret_cast<const __half2*>(&r));
}
// e8m0 code -> 2^(code - 127), exact (code 0 gives the subnormal 2^-127).
__device__ __forceinline__ float e8m0_value(uint32_t code) {
  return code > 0u ? __uint_as_float(code << 23) : __uint_as_float(0x00400000u);
}

struct DecParams {
  const __nv_bfloat16 *q, *k, *v;
  const uint8_t *kc, *ksc, *vc, *vsc;
  float* ws;
  int Hq, Hkv, L, nchunk;
  float scale;
};

constexpr int kPS = kChunk + 4;  // row stride of the probabilities in shared memory (spreads banks)

// Shared memory of one CTA for a group of G query heads, in floats: the chunk's staged e2m1
// K codes and e4m3 V codes, the group's query rows, the chunk's
// logits / probabilities, the per-head maximum and sum, and every warp's partial P.V --
// which reuses the K codes' space once the logits are done, when it fits there (G <= 4).
__host__ __device__ constexpr int osum_floats(int D, int G) { return (kThreads / 32) * G * D; }
__host__ __device__ constexpr int kstage_floats(int D) { return kChunk * (D / 2) / 4; }
__host__ __device__ constexpr int vstage_floats(int D) { return kChunk * D / 4; }
__host__ __device__ constexpr bool osum_in_kstage(int D, int G) { return osum_floats(D, G) <= kstage_floats(D); }
// The logits' FP16 query fragments of every lane, built once per CTA: [32 lanes][NT][NB][4]
// f16x2 words (NT = 8-head tiles, NB = 32-channel blocks), then one exponent per head (16
// words, keeping what follows 8-byte aligned).
__host__ __device__ constexpr int qfrag_words(int D, int G) { return 32 * ((G + 7) / 8) * (D / 32) * 4 + 16; }
__host__ __device__ constexpr int partial_smem_floats(int D, int G) {
  return kstage_floats(D) + vstage_floats(D) + qfrag_words(D, G) + G * kPS + 2 * G +
         (osum_in_kstage(D, G) ? 0 : osum_floats(D, G)) + 4 /* mbarrier */;
}

__device__ uint32_t g_decode_error_word;
constexpr uint64_t kStageWaitNs = 2000000000ull;  // 2 s: far above any legitimate copy

// D[16x8] += A[16x8] B[8x8]: TF32 operands (the top 19 bits of FP32 registers), FP32
// accumulation.  Fragments: a0 (row g, col t), a1 (row g+8, col t), a2 (row g, col t+4),
// a3 (row g+8, col t+4); b0 (row t, col g), b1 (row t+4, col g); d0 (row g, col 2t),
// d1 (row g, col 2t+1), d2 (row g+8, col 2t), d3 (row g+8, col 2t+1); g = lane / 4,
// t = lane % 4.
__device__ __forceinline__ void mma_tf32(float (&d)[4], float a0, float a1, float a2, float a3, float b0, float b1) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(__float_as_uint(a0)), "r"(__float_as_uint(a1)), "r"(__float_as_uint(a2)), "r"(__float_as_uint(a3)),
        "r"(__float_as_uint(b0)), "r"(__float_as_uint(b1)));
}

// Channels 32c + 8t .. 32c + 8t + 7 of cache row `row` of K, as FP32: the BF16 row for a
// high-precision token, else the e2m1 codes (bytes 16c + 4t .. +3 of the row) unscaled.
template <int D>
__device__ __forceinline__ void load_k8(const DecParams& p, long long row, bool valid, bool high, int c, int t,
                                        float (&a)[8]) {
  if (!valid) {
#pragma unroll
    for (int m = 0; m < 8; ++m) a[m] = 0.0f;
  } else if (high) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p.k + row * D + 32 * c + 8 * t));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      a[2 * e] = __uint_as_float(w[e] << 16);
      a[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
  } else {
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(p.kc + row * (D / 2) + 16 * c + 4 * t));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 x = e2m1x2_to_float2((w >> (8 * j)) & 0xFFu);
      a[2 * j] = x.x;
      a[2 * j + 1] = x.y;
    }
  }
}

// Channels 32c + 4g .. 32c + 4g + 3 of cache row `row` of V, as FP32: the BF16 row for a
// high-precision token, else the e4m3 codes unscaled.
template <int D>
__device__ __forceinline__ void load_v4(const DecParams& p, long long row, bool valid, bool high, int c, int g,
                                        float (&x)[4]) {
  if (!valid) {
#pragma unroll
    for (int m = 0; m < 4; ++m) x[m] = 0.0f;
  } else if (high) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p.v + row * D + 32 * c + 4 * g));
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xFFFF0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xFFFF0000u);
  } else {
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(p.vc + row * D + 32 * c + 4 * g));
    const float2 lo = e4m3x2_to_float2(w & 0xFFFFu), hi = e4m3x2_to_float2(w >> 16);
    x[0] = lo.x;
    x[1] = lo.y;
    x[2] = hi.x;
    x[3] = hi.y;
  }
}

// The e8m0 scale codes of one cache row (one byte per 32-channel block, block 0 lowest).
template <int D>
__device__ __forceinline__ uint32_t load_scales(const uint8_t* sc, long long row) {
  constexpr int NB = D / 32;
  if (NB == 4) return __ldg(reinterpret_cast<const uint32_t*>(sc + row * 4));
  return (uint32_t)__ldg(reinterpret_cast<const uint16_t*>(sc + row * 2));
}

// D[16x8] += A[16x16] B[16x8]: FP16 operands, FP32 accumulation.  Fragments (two FP16
// per register, the lower k in the low half): a0 (row g, k 2t..2t+1), a1 (row g+8,
// k 2t..2t+1), a2 (row g, k 2t+8..2t+9), a3 (row g+8, k 2t+8..2t+9); b0 (k 2t..2t+1,
// col g), b1 (k 2t+8..2t+9, col g); d as for mma_tf32.
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two e2m1 codes (one byte, element 2t in the low nibble) -> f16x2, exact.
__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tmov.b16 {t, _}, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(r) : "h"((unsigned short)byte));
  return r;
}

// FP32 -> two TF32 terms whose sum carries it to ~21 bits: hi keeps the top 11
// significant bits, lo = x - hi (exact in FP32) is rounded by the tensor core.
__device__ __forceinline__ void split_tf32(float x, float& hi, float& lo) {
  hi = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
  lo = x - hi;
}

// Four CTAs per SM for groups of up to 4 heads (64 registers a thread), two above: with
// the chunk's codes staged by bulk copies, more resident CTAs keep more of the cache in
// flight.
template <int D, int G>
__global__ void __launch_bounds__(kThreads, G <= 4 ? 4 : 2) decode_partial_kernel(const DecParams p) {
  constexpr int NB = D / 32;         // 32-channel scale blocks per row
  constexpr int NT = (G + 7) / 8;    // 8-head column tiles of the products
  const int chunk = blockIdx.x, bk = blockIdx.y, b = bk / p.Hkv, hk = bk % p.Hkv;
  const int t0 = chunk * kChunk, nt = min(p.L, t0 + kChunk) - t0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  extern __shared__ __align__(16) float dsm[];
  uint8_t* kcs = reinterpret_cast<uint8_t*>(dsm);                 // [kChunk][D/2] staged K codes
  uint8_t* vcs = kcs + kChunk * (D / 2);                           // [kChunk][D] staged V codes
  uint32_t* qfrag = reinterpret_cast<uint32_t*>(dsm + kstage_floats(D) + vstage_floats(D));  // [32][NT][NB][4]
  int* qexp = reinterpret_cast<int*>(qfrag + 32 * NT * NB * 4);   // [G] per-head exponent e
  float* ps = dsm + kstage_floats(D) + vstage_floats(D) + qfrag_words(D, G);  // [G][kPS]
  float* red = ps + G * kPS;                                       // [G][2]
  float* osum = osum_in_kstage(D, G) ? dsm : red + 2 * G;          // [8 warps][G][D]
  uint64_t* stage_bar = reinterpret_cast<uint64_t*>(red + 2 * G + (osum_in_kstage(D, G) ? 0 : osum_floats(D, G)));
  const long long row0 = (long long)bk * p.L + t0;  // cache row of the chunk's first token
  // A whole chunk's codes are contiguous in the cache: one bulk copy each for K and V,
  // issued first so that the CTA's bytes are all in flight while it sets up.
  const bool staged = (nt == kChunk);
  const uint32_t bar = smem_u32(stage_bar);
  if (staged && threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_expect_tx(bar, kChunk * (D / 2) + kChunk * D);
    bulk_load(smem_u32(kcs), p.kc + row0 * (D / 2), kChunk * (D / 2), bar);
    bulk_load(smem_u32(vcs), p.vc + row0 * D, kChunk * D, bar);
  }
  // The group's query: each head's largest |q| (as FP32 bits, which order like the
  // values), then every lane's FP16 fragments of the logits' products, built once here:
  // word (l, n, c, m) = q[8n + l/4][32c + 8(l%4) + 2m .. +1] * 2^-e, e per head (below).
  const __nv_bfloat16* qg = p.q + ((long long)b * p.Hq + hk * G) * D;
  if (threadIdx.x < G) qexp[threadIdx.x] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < G * D; i += kThreads) {  // a warp's 32 elements are one head's
    uint32_t m = __float_as_uint(fabsf(__bfloat162float(qg[i])));
    m = __reduce_max_sync(0xffffffffu, m);
    if (lane == 0) atomicMax(qexp + i / D, (int)m);
  }
  __syncthreads();
  if (threadIdx.x < G) {
    // e = floor(log2 amax) - 14 puts the head's largest component in [2^14, 2^15)
    const int ex = (int)((((uint32_t)qexp[threadIdx.x]) >> 23) & 0xFFu) - 127;
    qexp[threadIdx.x] = max(-110, min(110, ex - 14));
  }
  __syncthreads();
  for (int wi = threadIdx.x; wi < 32 * NT * NB * 4; wi += kThreads) {
    const int m = wi & 3, c = (wi >> 2) % NB, n = (wi >> 2) / NB % NT, l = wi / (4 * NB * NT);
    const int h = 8 * n + (l >> 2), ch = 32 * c + 8 * (l & 3) + 2 * m;
    uint32_t w = 0u;
    if (h < G) {
      const float down = pow2f(-qexp[h]);
      const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162*>(qg + h * D + ch);
      const __half2 h2 = __floats2half2_rn(__low2float(q2) * down, __high2float(q2) * down);
      w = *reinterpret_cast<const uint32_t*>(&h2);
    }
    qfrag[wi] = w;
  }
  __syncthreads();
  auto high = [&](int tt) -> bool {
    const int t = t0 + tt;
    return t < kSink || t >= p.L - kWindow;
  };

  // A warp whose 32 tokens are all quantised, in a staged chunk, takes the fast path: its
  // codes come from the staged copy and its scale words (lane l: token 32w + l) from one
  // load per lane, passed between lanes by shuffles.  Warps that meet the sink, the window
  // or a partial last chunk load per element from global memory as they go.
  const int wt0 = 32 * warp;
  const bool fast = staged && (t0 + wt0 >= kSink) && (t0 + wt0 + 32 <= p.L - kWindow);
  uint32_t ksw = 0u, vsw = 0u;
  if (fast) {
    ksw = load_scales<D>(p.ksc, row0 + wt0 + lane);
    vsw = load_scales<D>(p.vsc, row0 + wt0 + lane);
  }
  if (staged) {
    // every thread sees the copy complete (bounded: on a timeout the error word is set and
    // the CTA waits once more, again bounded, for its own copies before it returns)
    volatile int no_abort = 0;
    const bool landed = mbar_wait(bar, 0, &no_abort, kStageWaitNs);
    if (!__syncthreads_and(landed)) {
      if (threadIdx.x == 0) {
        atomicOr(&g_decode_error_word, 1u);
        mbar_wait(bar, 0, &no_abort, kStageWaitNs);
      }
      __syncthreads();
      return;
    }
  }

  // ---- logits S = K Q^T on the tensor cores.  Warp w takes the chunk's tokens
  // [32w, 32w + 32) as two 16-row tiles; the 8 columns are query heads.  Each 32-channel
  // block's product is scaled by its row's e8m0 scale (a power of two: exact) before it
  // joins the row's sum.
  //   Fast warps: mma.sync m16n8k16 FP16.  The e2m1 codes are exact in FP16 (one
  // hardware e2m1x2 -> f16x2 conversion per byte), and the query enters as FP16 after a
  // per-head power-of-two scaling 2^-e (e = floor(log2 amax) - 14) that puts its largest
  // component in [2^14, 2^15); components more than 2^28 below it fall into FP16
  // subnormals and lose bits; the logits are scaled back by 2^e.  Within block c, MMA 0 pairs
  // k = 2t, 2t+1 with channels 32c + 8t, +1 and k = 2t+8, 2t+9 with 32c + 8t + 2, +3;
  // MMA 1 the next four channels, so that a thread's codes of a row are one 32-bit word.
  //   Other warps (sink, window, partial chunk): mma.sync m16n8k8 TF32, exact for the
  // BF16 rows and query; step j pairs k = t with channel 32c + 8t + 2j and k = t + 4
  // with the next channel.
  if (fast) {
    uint32_t qh[NT][NB][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int c = 0; c < NB; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(qfrag + ((lane * NT + n) * NB + c) * 4);
        qh[n][c][0] = u.x;
        qh[n][c][1] = u.y;
        qh[n][c][2] = u.z;
        qh[n][c][3] = u.w;
      }
#pragma unroll
    for (int tile = 0; tile < 2; ++tile) {
      const int r_lo = wt0 + 16 * tile + g, r_hi = r_lo + 8;
      const uint32_t ks_lo = __shfl_sync(0xffffffffu, ksw, 16 * tile + g);
      const uint32_t ks_hi = __shfl_sync(0xffffffffu, ksw, 16 * tile + g + 8);
      float s[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[n][e] = 0.0f;
#pragma unroll
      for (int c = 0; c < NB; ++c) {
        const uint32_t kw_lo = *reinterpret_cast<const uint32_t*>(kcs + r_lo * (D / 2) + 16 * c + 4 * tq);
        const uint32_t kw_hi = *reinterpret_cast<const uint32_t*>(kcs + r_hi * (D / 2) + 16 * c + 4 * tq);
        uint32_t al[4], ah[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          al[j] = e2m1x2_to_h2((kw_lo >> (8 * j)) & 0xFFu);
          ah[j] = e2m1x2_to_h2((kw_hi >> (8 * j)) & 0xFFu);
        }
        const float sc_lo = e8m0_value((ks_lo >> (8 * c)) & 0xFFu), sc_hi = e8m0_value((ks_hi >> (8 * c)) & 0xFFu);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          float cb[4] = {0.0f, 0.0f, 0.0f, 0.0f};
          mma_f16(cb, al[0], ah[0], al[1], ah[1], qh[n][c][0], qh[n][c][1]);
          mma_f16(cb, al[2], ah[2], al[3], ah[3], qh[n][c][2], qh[n][c][3]);
          s[n][0] = fmaf(cb[0], sc_lo, s[n][0]);
          s[n][1] = fmaf(cb[1], sc_lo, s[n][1]);
          s[n][2] = fmaf(cb[2], sc_hi, s[n][2]);
          s[n][3] = fmaf(cb[3], sc_hi, s[n][3]);
        }
      }
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = 8 * n + 2 * tq + e;
          const float up = (h < G ? pow2f(qexp[h]) : 0.0f) * p.scale;
          if (h < G) {
            ps[h * kPS + r_lo] = s[n][e] * up;
            ps[h * kPS + r_hi] = s[n][2 + e] * up;
          }
        }
    }
  } else {
    float bq[NT][NB][8];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int c = 0; c < NB; ++c)
#pragma unroll
        for (int m = 0; m < 8; ++m)
          bq[n][c][m] = (8 * n + g < G) ? __bfloat162float(qg[(8 * n + g) * D + 32 * c + 8 * tq + m]) : 0.0f;
#pragma unroll
    for (int tile = 0; tile < 2; ++tile) {
      const int r_lo = wt0 + 16 * tile + g, r_hi = r_lo + 8;
      const bool v_lo = r_lo < nt, v_hi = r_hi < nt;
      const bool h_lo = v_lo && high(r_lo), h_hi = v_hi && high(r_hi);
      const uint32_t ks_lo = (v_lo && !h_lo) ? load_scales<D>(p.ksc, row0 + r_lo) : 0x7F7F7F7Fu;
      const uint32_t ks_hi = (v_hi && !h_hi) ? load_scales<D>(p.ksc, row0 + r_hi) : 0x7F7F7F7Fu;
      float s[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[n][e] = 0.0f;
#pragma unroll
      for (int c = 0; c < NB; ++c) {
        float a_lo[8], a_hi[8];
        load_k8<D>(p, row0 + r_lo, v_lo, h_lo, c, tq, a_lo);
        load_k8<D>(p, row0 + r_hi, v_hi, h_hi, c, tq, a_hi);
        const float sc_lo = e8m0_value((ks_lo >> (8 * c)) & 0xFFu), sc_hi = e8m0_value((ks_hi >> (8 * c)) & 0xFFu);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          float cb[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_tf32(cb, a_lo[2 * j], a_hi[2 * j], a_lo[2 * j + 1], a_hi[2 * j + 1], bq[n][c][2 * j],
                     bq[n][c][2 * j + 1]);
          s[n][0] = fmaf(cb[0], sc_lo, s[n][0]);
          s[n][1] = fmaf(cb[1], sc_lo, s[n][1]);
          s[n][2] = fmaf(cb[2], sc_hi, s[n][2]);
          s[n][3] = fmaf(cb[3], sc_hi, s[n][3]);
        }
      }
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = 8 * n + 2 * tq + e;
          if (h < G) {
            if (v_lo) ps[h * kPS + r_lo] = s[n][e] * p.scale;
            if (v_hi) ps[h * kPS + r_hi] = s[n][2 + e] * p.scale;
          }
        }
    }
  }
  __syncthreads();
  // ---- chunk maximum and exponential sum per head (one warp per head)
  for (int h = warp; h < G; h += kThreads / 32) {
    float m = -INFINITY;
    for (int i = lane; i < nt; i += 32) m = fmaxf(m, ps[h * kPS + i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float l = 0.0f;
    for (int i = lane; i < nt; i += 32) {
      const float e = __expf(ps[h * kPS + i] - m);
      ps[h * kPS + i] = e;
      l += e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) {
      red[2 * h] = m;
      red[2 * h + 1] = l;
    }
  }
  __syncthreads();
  // ---- P.V on the tensor cores: O^T[channel][head] += V^T[channel][token] P^T[token][head]
  // over the warp's 32 tokens, 8 per step (k = t: token base + t, k = t + 4: token
  // base + t + 4).  Tile (c, u) of block c: row g is channel 32c + 4g + 2u and row g+8 the
  // next, so that a thread's channels of a token are four consecutive bytes.  V's e8m0
  // scale (per token and block) goes into P (exact powers of two), and P enters as two
  // TF32 terms.
  float acc[NT][NB][2][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int c = 0; c < NB; ++c)
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[n][c][u][e] = 0.0f;
#pragma unroll
  for (int step = 0; step < 4; ++step) {
    const int ta = wt0 + 8 * step + tq, tb = ta + 4;
    const bool va = ta < nt, vb = tb < nt;
    const bool ha = va && high(ta), hb = vb && high(tb);
    uint32_t vs_a = 0x7F7F7F7Fu, vs_b = 0x7F7F7F7Fu;
    if (fast) {
      vs_a = __shfl_sync(0xffffffffu, vsw, 8 * step + tq);
      vs_b = __shfl_sync(0xffffffffu, vsw, 8 * step + tq + 4);
    } else {
      if (va && !ha) vs_a = load_scales<D>(p.vsc, row0 + ta);
      if (vb && !hb) vs_b = load_scales<D>(p.vsc, row0 + tb);
    }
    float pa[NT], pb[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int h = 8 * n + g;
      pa[n] = (h < G && va) ? ps[h * kPS + ta] : 0.0f;
      pb[n] = (h < G && vb) ? ps[h * kPS + tb] : 0.0f;
    }
#pragma unroll
    for (int c = 0; c < NB; ++c) {
      float xa[4], xb[4];
      if (fast) {
        const uint32_t wa = *reinterpret_cast<const uint32_t*>(vcs + ta * D + 32 * c + 4 * g);
        const uint32_t wb = *reinterpret_cast<const uint32_t*>(vcs + tb * D + 32 * c + 4 * g);
        const float2 a0 = e4m3x2_to_float2(wa & 0xFFFFu), a1 = e4m3x2_to_float2(wa >> 16);
        const float2 b0 = e4m3x2_to_float2(wb & 0xFFFFu), b1 = e4m3x2_to_float2(wb >> 16);
        xa[0] = a0.x; xa[1] = a0.y; xa[2] = a1.x; xa[3] = a1.y;
        xb[0] = b0.x; xb[1] = b0.y; xb[2] = b1.x; xb[3] = b1.y;
      } else {
        load_v4<D>(p, row0 + ta, va, ha, c, g, xa);
        load_v4<D>(p, row0 + tb, vb, hb, c, g, xb);
      }
      const float sa = e8m0_value((vs_a >> (8 * c)) & 0xFFu), sb = e8m0_value((vs_b >> (8 * c)) & 0xFFu);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        float pa_hi, pa_lo, pb_hi, pb_lo;
        split_tf32(pa[n] * sa, pa_hi, pa_lo);
        split_tf32(pb[n] * sb, pb_hi, pb_lo);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          mma_tf32(acc[n][c][u], xa[2 * u], xa[2 * u + 1], xb[2 * u], xb[2 * u + 1], pa_hi, pb_hi);
          mma_tf32(acc[n][c][u], xa[2 * u], xa[2 * u + 1], xb[2 * u], xb[2 * u + 1], pa_lo, pb_lo);
        }
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int c = 0; c < NB; ++c)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int h = 8 * n + 2 * tq, ch = 32 * c + 4 * g + 2 * u;
        if (h < G) {
          osum[(warp * G + h) * D + ch] = acc[n][c][u][0];
          osum[(warp * G + h) * D + ch + 1] = acc[n][c][u][2];
        }
        if (h + 1 < G) {
          osum[(warp * G + h + 1) * D + ch] = acc[n][c][u][1];
          osum[(warp * G + h + 1) * D + ch + 1] = acc[n][c][u][3];
        }
      }
  __syncthreads();
  // ---- chunk state: [max, sum, O[0..D)] per head
  float* st = p.ws + ((long long)bk * p.nchunk + chunk) * G * (2 + D);
  for (int i = threadIdx.x; i < G * D; i += kThreads) {
    const int h = i / D, c = i % D;
    float o = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) o += osum[(w * G + h) * D + c];
    st[h * (2 + D) + 2 + c] = o;
  }
  if (threadIdx.x < G) {
    st[threadIdx.x * (2 + D)] = red[2 * threadIdx.x];
    st[threadIdx.x * (2 + D) + 1] = red[2 * threadIdx.x + 1];
  }
}

// Merge the chunks' softmax states of one (b, hq): grid B*Hq, D threads.
template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(const float* __restrict__ ws, int Hq, int Hkv, int nchunk,
                                                         __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
  const int bh = blockIdx.x, b = bh / Hq, h = bh % Hq, G = Hq / Hkv, hk = h / G, g = h % G;
  const long long base = (long long)(b * Hkv + hk) * nchunk;
  float m = -INFINITY;
  for (int c = 0; c < nchunk; ++c) m = fmaxf(m, ws[((base + c) * G + g) * (2 + D)]);
  float l = 0.0f, acc = 0.0f;
  for (int c = 0; c < nchunk; ++c) {
    const float* st = ws + ((base + c) * G + g) * (2 + D);
    const float f = __expf(st[0] - m);
    l += st[1] * f;
    acc += st[2 + threadIdx.x] * f;
  }
  o[(long long)bh * D + threadIdx.x] = __float2bfloat16(acc / l);
  if (lse != nullptr && threadIdx.x == 0) lse[bh] = m + logf(l);
}


}  // namespace dec

// Chunks of 256 tokens per (b, kv head): one CTA each.
int decode_nchunk(int B, int Hkv, int L) {
  (void)B;
  (void)Hkv;
  return (L + dec::kChunk - 1) / dec::kChunk;
}

// Bit 0: a decode step's CTA gave up waiting for its staged cache bytes.
cudaError_t read_and_clear_decode_error(uint32_t* word) {
  uint32_t w = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&w, dec::g_decode_error_word, sizeof(w));
  if (e == cudaSuccess && w != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(dec::g_decode_error_word, &zero, sizeof(zero));
  }
  *word = w;
  return e;
}

cudaError_t launch_decode_quantize(const DecodeArgs& a, int t0, int t1, cudaStream_t s) {
  const int BHk = a.B * a.Hkv;
  const long long items = (long long)BHk * (t1 - t0) * (a.d / 32);
  const unsigned grid = (unsigned)((items + 255) / 256);
  if (a.d == 128)
    dec::decode_quantize_kernel<128><<<grid, 256, 0, s>>>(a.k, a.v, BHk, a.L, t0, t1, a.kc, a.ksc, a.vc, a.vsc);
  else
    dec::decode_quantize_kernel<64><<<grid, 256, 0, s>>>(a.k, a.v, BHk, a.L, t0, t1, a.kc, a.ksc, a.vc, a.vsc);
  count_launches(1);
  return cudaGetLastError();
}

template <int D, int G>
static cudaError_t launch_partial(const dec::DecParams& p, dim3 grid, cudaStream_t s) {
  const int sm = (int)sizeof(float) * dec::partial_smem_floats(D, G);
  auto kern = dec::decode_partial_kernel<D, G>;
  if (sm > 48 * 1024 && cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) != cudaSuccess)
    return cudaErrorInvalidValue;
  kern<<<grid, dec::kThreads, sm, s>>>(p);
  return cudaSuccess;
}

template <int D>
static cudaError_t launch_partial_d(const dec::DecParams& p, int G, dim3 grid, cudaStream_t s) {
  switch (G) {
    case 1: return launch_partial<D, 1>(p, grid, s);
    case 2: return launch_partial<D, 2>(p, grid, s);
    case 4: return launch_partial<D, 4>(p, grid, s);
    case 8: return launch_partial<D, 8>(p, grid, s);
    case 16: return launch_partial<D, 16>(p, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

bool decode_group_supported(int G) { return G == 1 || G == 2 || G == 4 || G == 8 || G == 16; }

cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t s) {
  dec::DecParams p;
  p.q = a.q; p.k = a.k; p.v = a.v;
  p.kc = a.kc; p.ksc = a.ksc; p.vc = a.vc; p.vsc = a.vsc;
  p.ws = a.ws;
  p.Hq = a.Hq; p.Hkv = a.Hkv; p.L = a.L;
  p.nchunk = decode_nchunk(a.B, a.Hkv, a.L);
  p.scale = a.softmax_scale > 0.0f ? a.softmax_scale : 1.0f / sqrtf((float)a.d);
  const dim3 grid(p.nchunk, a.B * a.Hkv);
  const int G = a.Hq / a.Hkv;
  cudaError_t err = a.d == 128 ? launch_partial_d<128>(p, G, grid, s) : launch_partial_d<64>(p, G, grid, s);
  if (err != cudaSuccess) return err;
  if (a.d == 128)
    dec::decode_merge_kernel<128><<<a.B * a.Hq, 128, 0, s>>>(a.ws, a.Hq, a.Hkv, p.nchunk, a.o, a.lse);
  else
    dec::decode_merge_kernel<64><<<a.B * a.Hq, 64, 0, s>>>(a.ws, a.Hq, a.Hkv, p.nchunk, a.o, a.lse);
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace thrift
