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
//                           chunk max / exp sum per head, P.V (one lane per d/32
//                           channels, one warp per token stream, four tokens'
//                           rows loaded together); writes the
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

// Shared memory of one CTA for a group of G query heads (floats).
__host__ __device__ constexpr int partial_smem_floats(int D, int G) {
  return G * D + G * kChunk + 2 * G + (kThreads / 32) * G * D;
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads) decode_partial_kernel(const DecParams p) {
  constexpr int CPL = D / 32;  // channels per lane in the P.V phase
  constexpr int NB = D / 32;   // 32-channel scale blocks per row
  const int chunk = blockIdx.x, bk = blockIdx.y, b = bk / p.Hkv, hk = bk % p.Hkv;
  const int t0 = chunk * kChunk, t1 = min(p.L, t0 + kChunk), nt = t1 - t0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  extern __shared__ float dsm[];
  float* qs = dsm;                 // [G][D]
  float* ps = qs + G * D;          // [G][kChunk]
  float* red = ps + G * kChunk;    // [G][2]
  float* osum = red + 2 * G;       // [8 warps][G][D]
  for (int i = threadIdx.x; i < G * D; i += kThreads)
    qs[i] = __bfloat162float(p.q[((long long)b * p.Hq + hk * G + i / D) * D + i % D]);
  __syncthreads();
  const long long row0 = (long long)bk * p.L;
  // ---- logits: one thread per token, all G heads, channels ascending; the whole
  // row is loaded before it is used, so each thread has its row's bytes in flight
  for (int tt = threadIdx.x; tt < nt; tt += kThreads) {
    const int t = t0 + tt;
    const long long row = row0 + t;
    float s[G];
#pragma unroll
    for (int h = 0; h < G; ++h) s[h] = 0.0f;
    if (t < kSink || t >= p.L - kWindow) {
      const uint4* kr = reinterpret_cast<const uint4*>(p.k + row * D);
      uint4 u[D / 8];
#pragma unroll
      for (int c8 = 0; c8 < D / 8; ++c8) u[c8] = __ldg(kr + c8);
#pragma unroll
      for (int c8 = 0; c8 < D / 8; ++c8) {
        const uint32_t w[4] = {u[c8].x, u[c8].y, u[c8].z, u[c8].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = __uint_as_float(w[e] << 16), x1 = __uint_as_float(w[e] & 0xFFFF0000u);
          const int c = 8 * c8 + 2 * e;
#pragma unroll
          for (int h = 0; h < G; ++h) s[h] = fmaf(qs[h * D + c + 1], x1, fmaf(qs[h * D + c], x0, s[h]));
        }
      }
    } else {
      const uint4* kr = reinterpret_cast<const uint4*>(p.kc + row * (D / 2));
      uint4 u[NB];
      uint32_t scw[NB];
#pragma unroll
      for (int c32 = 0; c32 < NB; ++c32) {
        u[c32] = __ldg(kr + c32);
        scw[c32] = __ldg(p.ksc + row * NB + c32);
      }
#pragma unroll
      for (int c32 = 0; c32 < NB; ++c32) {
        const float sc = e8m0_value(scw[c32]);
        const uint32_t w[4] = {u[c32].x, u[c32].y, u[c32].z, u[c32].w};
        float blk[G];
#pragma unroll
        for (int h = 0; h < G; ++h) blk[h] = 0.0f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
#pragma unroll
          for (int n = 0; n < 4; ++n) {
            const float2 x = e2m1x2_to_float2((w[e] >> (8 * n)) & 0xFFu);
            const int c = 32 * c32 + 8 * e + 2 * n;
#pragma unroll
            for (int h = 0; h < G; ++h) blk[h] = fmaf(qs[h * D + c + 1], x.y, fmaf(qs[h * D + c], x.x, blk[h]));
          }
        }
        // the block's scale is a power of two: scaling the block's partial sum is exact
#pragma unroll
        for (int h = 0; h < G; ++h) s[h] = fmaf(blk[h], sc, s[h]);
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) ps[h * kChunk + tt] = s[h] * p.scale;
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
  // ---- P.V: warp w takes tokens t0 + w, t0 + w + 8, ... four at a time (their rows
  // loaded together); lane owns CPL consecutive channels
  float acc[G][CPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[h][c] = 0.0f;
  const int c0 = lane * CPL;
  constexpr int U = 4;
  for (int tb = warp; tb < nt; tb += U * (kThreads / 32)) {
    // raw row bytes of U tokens first: BF16 rows 2*CPL bytes (w0: channels c0, c0+1;
    // w1: c0+2, c0+3), FP8 rows CPL bytes (w0)
    uint32_t w0[U], w1[U];
    float sc[U];
    bool hp[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int tt = tb + u * (kThreads / 32);
      const int t = t0 + tt;
      const long long row = row0 + t;
      hp[u] = t < kSink || t >= p.L - kWindow;
      w0[u] = 0u;
      w1[u] = 0u;
      sc[u] = 0.0f;
      if (tt < nt) {
        if (hp[u]) {
          if (CPL == 4) {
            const uint2 x = __ldg(reinterpret_cast<const uint2*>(p.v + row * D + c0));
            w0[u] = x.x;
            w1[u] = x.y;
          } else {
            w0[u] = __ldg(reinterpret_cast<const uint32_t*>(p.v + row * D + c0));
          }
        } else {
          w0[u] = CPL == 4 ? __ldg(reinterpret_cast<const uint32_t*>(p.vc + row * D + c0))
                           : (uint32_t)__ldg(reinterpret_cast<const uint16_t*>(p.vc + row * D + c0));
          sc[u] = e8m0_value(__ldg(p.vsc + row * NB + c0 / 32));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int tt = tb + u * (kThreads / 32);
      if (tt >= nt) break;
      float x[CPL];
      if (hp[u]) {
        x[0] = __uint_as_float(w0[u] << 16);
        x[1] = __uint_as_float(w0[u] & 0xFFFF0000u);
        if (CPL == 4) {
          x[2 % CPL] = __uint_as_float(w1[u] << 16);
          x[3 % CPL] = __uint_as_float(w1[u] & 0xFFFF0000u);
        }
      } else {
        const float2 a = e4m3x2_to_float2(w0[u] & 0xFFFFu);
        x[0] = a.x * sc[u];
        x[1] = a.y * sc[u];
        if (CPL == 4) {
          const float2 bq = e4m3x2_to_float2(w0[u] >> 16);
          x[2 % CPL] = bq.x * sc[u];
          x[3 % CPL] = bq.y * sc[u];
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float pw = ps[h * kChunk + tt];
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[h][c] = fmaf(pw, x[c], acc[h][c]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int c = 0; c < CPL; ++c) osum[(warp * G + h) * D + c0 + c] = acc[h][c];
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

// The decode kernels wait on nothing, so they never set an error; the word exists so
// that thrift_device_status reads the same interface for every kernel of the library.
cudaError_t read_and_clear_decode_error(uint32_t* word) {
  *word = 0;
  return cudaSuccess;
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
