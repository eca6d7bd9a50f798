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
// FP32 on CUDA cores (the step reads each cached byte once: HBM-bound).
//
// Kernels:
//   decode_quantize_kernel  per-token MX quantisation of cache rows [t0, t1)
//   decode_partial_kernel   one CTA per (b, kv head, chunk of 256 tokens), all G
//                           query heads of the group: logits (one lane per token),
//                           chunk max / exp sum per head, P.V (one lane per four
//                           channels, one warp per token stream); writes the
//                           chunk's softmax state (max, sum, unnormalised O)
//   decode_merge_kernel     combines the chunks' states per query head.
#include "dev.cuh"
#include "kernels.h"

namespace thrift {
namespace dec {

constexpr int kChunk = 256;    // cache tokens per CTA
constexpr int kThreads = 256;  // 8 warps
constexpr int kMaxG = 16;      // query heads per kv head
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

// e2m1 code (4 bits) -> float, exact: 0, 0.5 and (1 + (i & 1) / 2) * 2^((i >> 1) - 1) for i >= 2.
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t i = c & 7u;
  const float m = i < 2u ? 0.5f * (float)i : __uint_as_float(((126u + (i >> 1)) << 23) | ((i & 1u) << 22));
  return (c & 8u) ? -m : m;
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

template <int D>
__global__ void __launch_bounds__(kThreads) decode_partial_kernel(const DecParams p) {
  constexpr int CPL = D / 32;  // channels per lane in the P.V phase
  const int G = p.Hq / p.Hkv;
  const int chunk = blockIdx.x, bk = blockIdx.y, b = bk / p.Hkv, hk = bk % p.Hkv;
  const int t0 = chunk * kChunk, t1 = min(p.L, t0 + kChunk), nt = t1 - t0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  extern __shared__ float dsm[];
  float* qs = dsm;                        // [kMaxG][D]
  float* ps = qs + kMaxG * D;             // [kMaxG][kChunk]
  float* red = ps + kMaxG * kChunk;       // [kMaxG][2]
  float* osum = red + 2 * kMaxG;          // [8 warps][kMaxG][D]
  for (int i = threadIdx.x; i < G * D; i += kThreads)
    qs[i] = __bfloat162float(p.q[((long long)b * p.Hq + hk * G + i / D) * D + i % D]);
  __syncthreads();
  const long long row0 = (long long)bk * p.L;
  // ---- logits: one lane per token, all G heads, channels ascending
  for (int tt = threadIdx.x; tt < nt; tt += kThreads) {
    const int t = t0 + tt;
    const long long row = row0 + t;
    float s[kMaxG];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) s[h] = 0.0f;
    const bool hp = t < kSink || t >= p.L - kWindow;
    if (hp) {
      const uint4* kr = reinterpret_cast<const uint4*>(p.k + row * D);
#pragma unroll 2
      for (int c8 = 0; c8 < D / 8; ++c8) {
        const uint4 u = __ldg(kr + c8);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = __uint_as_float(w[e] << 16), x1 = __uint_as_float(w[e] & 0xFFFF0000u);
          const int c = 8 * c8 + 2 * e;
#pragma unroll
          for (int h = 0; h < kMaxG; ++h)
            if (h < G) s[h] = fmaf(qs[h * D + c + 1], x1, fmaf(qs[h * D + c], x0, s[h]));
        }
      }
    } else {
      const uint4* kr = reinterpret_cast<const uint4*>(p.kc + row * (D / 2));
#pragma unroll 1
      for (int c32 = 0; c32 < D / 32; ++c32) {
        const float sc = e8m0_value(__ldg(p.ksc + row * (D / 32) + c32));
        const uint4 u = __ldg(kr + c32);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
#pragma unroll
          for (int n = 0; n < 8; ++n) {
            const int c = 32 * c32 + 8 * e + n;
            const float x = e2m1_value(w[e] >> (4 * n)) * sc;
#pragma unroll
            for (int h = 0; h < kMaxG; ++h)
              if (h < G) s[h] = fmaf(qs[h * D + c], x, s[h]);
          }
        }
      }
    }
#pragma unroll
    for (int h = 0; h < kMaxG; ++h)
      if (h < G) ps[h * kChunk + tt] = s[h] * p.scale;
  }
  __syncthreads();
  // ---- chunk maximum and exponential sum per head (one warp per head)
  for (int h = warp; h < G; h += kThreads / 32) {
    float m = -INFINITY;
    for (int i = lane; i < nt; i += 32) m = fmaxf(m, ps[h * kChunk + i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float l = 0.0f;
    for (int i = lane; i < nt; i += 32) {
      const float e = __expf(ps[h * kChunk + i] - m);
      ps[h * kChunk + i] = e;
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
  // ---- P.V: warp w takes tokens t0 + w, t0 + w + 8, ...; lane owns CPL consecutive channels
  float acc[kMaxG][CPL];
#pragma unroll
  for (int h = 0; h < kMaxG; ++h)
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[h][c] = 0.0f;
  const int c0 = lane * CPL;
  for (int tt = warp; tt < nt; tt += kThreads / 32) {
    const int t = t0 + tt;
    const long long row = row0 + t;
    float x[CPL];
    if (t < kSink || t >= p.L - kWindow) {
      const __nv_bfloat16* vr = p.v + row * D + c0;
#pragma unroll
      for (int c = 0; c < CPL; ++c) x[c] = __bfloat162float(vr[c]);
    } else {
      const float sc = e8m0_value(__ldg(p.vsc + row * (D / 32) + c0 / 32));
      uint32_t bytes;
      if (CPL == 4) bytes = __ldg(reinterpret_cast<const uint32_t*>(p.vc + row * D + c0));
      else bytes = __ldg(reinterpret_cast<const uint16_t*>(p.vc + row * D + c0));
#pragma unroll
      for (int c = 0; c < CPL; ++c) x[c] = e4m3_mag_value((bytes >> (8 * c)) & 0x7Fu) * sc * (((bytes >> (8 * c)) & 0x80u) ? -1.0f : 1.0f);
    }
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
      if (h < G) {
        const float pw = ps[h * kChunk + tt];
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[h][c] = fmaf(pw, x[c], acc[h][c]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < kMaxG; ++h)
    if (h < G)
#pragma unroll
      for (int c = 0; c < CPL; ++c) osum[(warp * kMaxG + h) * D + c0 + c] = acc[h][c];
  __syncthreads();
  // ---- chunk state: [max, sum, O[0..D)] per head
  float* st = p.ws + ((long long)bk * p.nchunk + chunk) * G * (2 + D);
  for (int i = threadIdx.x; i < G * D; i += kThreads) {
    const int h = i / D, c = i % D;
    float o = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) o += osum[(w * kMaxG + h) * D + c];
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

constexpr size_t partial_smem(int D) {
  return sizeof(float) * ((size_t)kMaxG * D + (size_t)kMaxG * kChunk + 2 * kMaxG + (size_t)(kThreads / 32) * kMaxG * D);
}

}  // namespace dec

int decode_nchunk(int L) { return (L + dec::kChunk - 1) / dec::kChunk; }
int decode_max_group() { return dec::kMaxG; }

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

cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t s) {
  dec::DecParams p;
  p.q = a.q; p.k = a.k; p.v = a.v;
  p.kc = a.kc; p.ksc = a.ksc; p.vc = a.vc; p.vsc = a.vsc;
  p.ws = a.ws;
  p.Hq = a.Hq; p.Hkv = a.Hkv; p.L = a.L;
  p.nchunk = decode_nchunk(a.L);
  p.scale = a.softmax_scale > 0.0f ? a.softmax_scale : 1.0f / sqrtf((float)a.d);
  const dim3 grid(p.nchunk, a.B * a.Hkv);
  if (a.d == 128) {
    const size_t sm = dec::partial_smem(128);
    if (cudaFuncSetAttribute(dec::decode_partial_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) !=
        cudaSuccess)
      return cudaErrorInvalidValue;
    dec::decode_partial_kernel<128><<<grid, dec::kThreads, sm, s>>>(p);
    dec::decode_merge_kernel<128><<<a.B * a.Hq, 128, 0, s>>>(a.ws, a.Hq, a.Hkv, p.nchunk, a.o, a.lse);
  } else {
    const size_t sm = dec::partial_smem(64);
    if (cudaFuncSetAttribute(dec::decode_partial_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) !=
        cudaSuccess)
      return cudaErrorInvalidValue;
    dec::decode_partial_kernel<64><<<grid, dec::kThreads, sm, s>>>(p);
    dec::decode_merge_kernel<64><<<a.B * a.Hq, 64, 0, s>>>(a.ws, a.Hq, a.Hkv, p.nchunk, a.o, a.lse);
  }
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace thrift
