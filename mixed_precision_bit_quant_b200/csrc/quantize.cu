// Stage 0: NVFP4 quantisation of Q and K, per-channel FP8 quantisation of V.
//
// ThriftAttention: Selective Mixed Precision for Long-Context FP4 Attention
// (abstract) computes most attention blocks in 4-bit with block-scaled
// quantisation on Blackwell; the NVFP4 recipe (16-element e4m3 scales, one
// FP32 tensor scale per head) and the power-of-two per-channel FP8 scale of V
// are this library's fixed reading of that statement.
//
// All kernels are HBM-bound: 16-byte loads, warp-level max reductions, one
// atomic per warp for the amax passes.
#include <mutex>

#include "dev.cuh"
#include "kernels.h"

namespace thrift {

// ---------------------------------------------------------------------------
// amax of |x| per head (Q, K).  x: [BH][N*d] bf16.  amax: [BH] float bits.
// grid (chunks, BH), each thread reads 8 bf16 (16 bytes) per step.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) amax_head_kernel(const __nv_bfloat16* __restrict__ x,
                                                        long long per_head, uint32_t* __restrict__ amax) {
  const int bh = blockIdx.y;
  const uint4* p = reinterpret_cast<const uint4*>(x + (long long)bh * per_head);
  const long long nvec = per_head / 8;
  const long long stride = (long long)gridDim.x * blockDim.x;
  uint32_t m = 0;
  // |bf16| as float bits: clear the sign, shift into the high half
  auto fold = [&](const uint4& u) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) m = max(m, max((w[t] & 0x7FFFu) << 16, w[t] & 0x7FFF0000u));
  };
  long long v = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  // four independent 16-byte loads in flight per thread
  for (; v + 3 * stride < nvec; v += 4 * stride) {
    const uint4 u0 = __ldg(p + v), u1 = __ldg(p + v + stride), u2 = __ldg(p + v + 2 * stride),
                u3 = __ldg(p + v + 3 * stride);
    fold(u0);
    fold(u1);
    fold(u2);
    fold(u3);
  }
  for (; v < nvec; v += stride) fold(__ldg(p + v));
  m = __reduce_max_sync(0xffffffffu, m);
  if ((threadIdx.x & 31) == 0 && m != 0) atomicMax(amax + bh, m);
}

// ---------------------------------------------------------------------------
// amax of |v| per (head, channel).  v: [BH][N][D] bf16.  amax: [BH][D].
// Thread t covers channels 8*(t % (D/8)) .. +8 of rows t / (D/8) + k*RPB.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) amax_chan_kernel(const __nv_bfloat16* __restrict__ v, int N,
                                                        int rows_per_block, uint32_t* __restrict__ amax) {
  constexpr int G = D / 8;             // 16-byte groups per row
  constexpr int RS = 256 / G;          // rows per step
  __shared__ uint32_t red[RS][D];
  const int bh = blockIdx.y;
  const int g = threadIdx.x % G, rr = threadIdx.x / G;
  const int r0 = blockIdx.x * rows_per_block;
  const int r1 = min(N, r0 + rows_per_block);
  uint32_t m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const __nv_bfloat16* base = v + (long long)bh * N * D + g * 8;
  auto fold = [&](const uint4& u) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      m[2 * t] = max(m[2 * t], (w[t] & 0x7FFFu) << 16);
      m[2 * t + 1] = max(m[2 * t + 1], w[t] & 0x7FFF0000u);
    }
  };
  int r = r0 + rr;
  // four independent 16-byte loads in flight per thread
  for (; r + 3 * RS < r1; r += 4 * RS) {
    const uint4 u0 = __ldg(reinterpret_cast<const uint4*>(base + (long long)r * D));
    const uint4 u1 = __ldg(reinterpret_cast<const uint4*>(base + (long long)(r + RS) * D));
    const uint4 u2 = __ldg(reinterpret_cast<const uint4*>(base + (long long)(r + 2 * RS) * D));
    const uint4 u3 = __ldg(reinterpret_cast<const uint4*>(base + (long long)(r + 3 * RS) * D));
    fold(u0);
    fold(u1);
    fold(u2);
    fold(u3);
  }
  for (; r < r1; r += RS) fold(__ldg(reinterpret_cast<const uint4*>(base + (long long)r * D)));
#pragma unroll
  for (int t = 0; t < 8; ++t) red[rr][g * 8 + t] = m[t];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    uint32_t mm = 0;
    for (int s = 0; s < RS; ++s) mm = max(mm, red[s][c]);
    if (mm != 0) atomicMax(amax + (long long)bh * D + c, mm);
  }
}

// ---------------------------------------------------------------------------
// NVFP4 pack of Q or K.  One thread = 64 consecutive elements (4 scale blocks)
// of one row, rows 0 .. 128*T-1 (rows >= N only clear their tensor-core scales).
// A code is the e2m1 rounding of the correctly rounded quotient x / (s * g),
// taken two at a time by the hardware conversion to e2m1x2: round to nearest
// with ties to the even code, saturating at +-6, the sign kept for values that
// round to zero -- the rounding rule of the format as this library reads it.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) nvfp4_pack_kernel(
    const __nv_bfloat16* __restrict__ x, int BH, int N, int T, const uint32_t* __restrict__ amax_bits,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, uint8_t* __restrict__ sf_mma,
    float* __restrict__ gs) {
  constexpr int KB = D / 64;  // 64-element groups per row
  const long long rows_pad = (long long)T * 128;
  const long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= (long long)BH * rows_pad * KB) return;
  const int kb = (int)(item % KB);
  const long long rowg = item / KB;
  const int bh = (int)(rowg / rows_pad);
  const int row = (int)(rowg % rows_pad);
  const float amax = __uint_as_float(amax_bits[bh]);
  const float g = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
  if (row == 0 && kb == 0) gs[bh] = g;
  const int t = row >> 7, rr = row & 127;
  uint32_t* mma_word = reinterpret_cast<uint32_t*>(
      sf_mma + ((long long)(bh * T + t) * KB + kb) * 512 + (rr & 31) * 16 + (rr >> 5) * 4);
  if (row >= N) {
    *mma_word = 0u;
    return;
  }
  const float six_g = __fmul_rn(6.0f, g);
  const uint4* src = reinterpret_cast<const uint4*>(x + ((long long)bh * N + row) * D + kb * 64);
  uint32_t sfw = 0;
  uint32_t out[8];
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    uint4 u0 = __ldg(src + 2 * b), u1 = __ldg(src + 2 * b + 1);
    uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
    float f[16];
    float am = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      f[2 * e] = __uint_as_float(w[e] << 16);
      f[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
      am = fmaxf(am, fmaxf(fabsf(f[2 * e]), fabsf(f[2 * e + 1])));
    }
    const uint32_t s = e4m3_mag_code(__fdiv_rn(am, six_g));
    const float sd = e4m3_mag_value(s);
    const float den = __fmul_rn(sd, g);
    uint32_t lo = 0, hi = 0;
    if (sd > 0.0f) {
      // The code of the correctly rounded quotient x / den, without a division per
      // element: q = x * fl(1/den) is within 1.5 ulps of it, so q (1 - 2^-20) and
      // q (1 + 2^-20) bracket it, and the e2m1 rounding (monotone) of the two ends
      // decides the code when they agree.  Pairs whose ends disagree (a quotient at a
      // rounding threshold) take the correctly rounded division.  A divisor below
      // 2^-100 (reciprocal near overflow) takes the division for the whole block.
      const bool recip_ok = den >= 7.888609052210118e-31f;  // 2^-100
      const float rcp = __frcp_rn(den);
      const uint64_t r2 = f2pack(rcp, rcp);
      const uint64_t dn2 = f2pack(0.99999904632568359375f, 0.99999904632568359375f);  // 1 - 2^-20
      const uint64_t up2 = f2pack(1.00000095367431640625f, 1.00000095367431640625f);  // 1 + 2^-20
      uint32_t code[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float fa = f[2 * e], fb = f[2 * e + 1];
        const uint64_t q2 = fmul2(f2pack(fa, fb), r2);
        float la, lb, ha, hb;
        f2unpack(fmul2(q2, dn2), la, lb);
        f2unpack(fmul2(q2, up2), ha, hb);
        uint32_t c = cvt_e2m1x2(la, lb);
        if (!recip_ok || c != cvt_e2m1x2(ha, hb)) c = cvt_e2m1x2(__fdiv_rn(fa, den), __fdiv_rn(fb, den));
        code[e] = c;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        lo |= code[e] << (8 * e);
        hi |= code[4 + e] << (8 * e);
      }
    }
    out[2 * b] = lo;
    out[2 * b + 1] = hi;
    sfw |= s << (8 * b);
  }
  uint4* dst = reinterpret_cast<uint4*>(codes + ((long long)bh * N + row) * (D / 2) + kb * 32);
  dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
  dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  *reinterpret_cast<uint32_t*>(sf + ((long long)bh * N + row) * (D / 16) + kb * 4) = sfw;
  *mma_word = sfw;
}

// ---------------------------------------------------------------------------
// FP8 V: per-channel exponent, e4m3 codes and BF16 copy, both
// transposed to [BH][D][Np].  grid (T, BH); a 128-key tile per block.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) fp8_v_pack_kernel(
    const __nv_bfloat16* __restrict__ v, int N, int T, const uint32_t* __restrict__ amax_bits,
    uint8_t* __restrict__ v_fp8t, __nv_bfloat16* __restrict__ v_st, int8_t* __restrict__ v_exp) {
  constexpr int LD = D + 2;  // padded row (bf16) to spread banks on column reads
  __shared__ __nv_bfloat16 tile[128][LD];
  __shared__ float inv_scale[D];
  const int t = blockIdx.x, bh = blockIdx.y;
  const long long Np = (long long)T * 128;
  const int n0 = t * 128;
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    const float am = __uint_as_float(amax_bits[(long long)bh * D + c]);
    int e = 0;
    if (am > 0.0f) {
      // am = m * 2^E with m in [0.5, 1); 448 = 0.875 * 2^9
      int E;
      const float m = frexpf(am, &E);
      e = (m <= 0.875f) ? E - 9 : E - 8;
    }
    inv_scale[c] = pow2f(-e);
    if (t == 0) v_exp[(long long)bh * D + c] = (int8_t)e;
  }
  // stage the tile (rows >= N as zeros)
  constexpr int G = D / 8;
  for (int it = threadIdx.x; it < 128 * G; it += blockDim.x) {
    const int r = it / G, g = it % G;
    uint4 u = make_uint4(0, 0, 0, 0);
    if (n0 + r < N) u = __ldg(reinterpret_cast<const uint4*>(v + ((long long)bh * N + n0 + r) * D + g * 8));
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t* dst = reinterpret_cast<uint32_t*>(&tile[r][g * 8]);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = w[q];
  }
  __syncthreads();
  // each item: channel c, 16 consecutive keys
  for (int it = threadIdx.x; it < D * 8; it += blockDim.x) {
    const int c = it >> 3, seg = it & 7;
    const float sc = inv_scale[c];
    uint32_t codes[4] = {0, 0, 0, 0};
    uint32_t bf[8];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float x = __bfloat162float(tile[seg * 16 + k][c]);
      const float y = __fmul_rn(x, sc);  // exact (a power of two) unless far in the subnormals
      codes[k >> 2] |= e4m3_code(y) << (8 * (k & 3));
      // the BF16 copy: exact for every y >= 2^-126 (8 significant bits); BF16 subnormals
      // round to nearest, ties to even
      const uint32_t yb = __bfloat16_as_ushort(__float2bfloat16_rn(y));
      if (k & 1) bf[k >> 1] |= yb << 16; else bf[k >> 1] = yb;
    }
    const long long off = ((long long)bh * D + c) * Np + n0 + seg * 16;
    *reinterpret_cast<uint4*>(v_fp8t + off) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
    uint4* d2 = reinterpret_cast<uint4*>(v_st + off);
    d2[0] = make_uint4(bf[0], bf[1], bf[2], bf[3]);
    d2[1] = make_uint4(bf[4], bf[5], bf[6], bf[7]);
  }
}

// ---------------------------------------------------------------------------
// MXFP4 pack of Q or K: the microscaling variant of the low path (the
// attention-quantization topic page lists MXFP4 beside NVFP4; the format is
// the OCP microscaling one).  One e8m0 power-of-two scale per 32 consecutive
// elements along d, no tensor scale (gs = 1).  Scale exponent e =
// floor(log2 amax_block) - 2 (2 is the exponent of e2m1's largest value 6),
// clamped to [-127, 127], -127 for an all-zero block; codes are the e2m1
// rounding (nearest, ties to the even code, saturating, sign kept) of
// x * 2^-e, an exact scaling.  One thread = 64 consecutive elements (two
// blocks) of one row, rows 0 .. 128*T-1 (rows >= N only clear their
// tensor-core scales).
// Outputs: codes [BH][N][D/2]; sf [BH][N][D/32] e8m0 codes, row-major;
// sf_mma [BH][T][D/64][512]: per 64 elements of d one 512-byte chunk in the
// tensor core's scale order, word 16*(r%32) + 4*(r/32) of row r holding the
// two block scales of that K=64 step in bytes 0 and 1 (bytes 2, 3 zero).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int mx_scale_exp(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  if (bits == 0u) return -127;
  const int ef = (int)(bits >> 23);
  const int fl = ef > 0 ? ef - 127 : (31 - __clz((int)bits)) - 149;  // floor(log2 amax), subnormals too
  const int e = fl - 2;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

template <int D>
__global__ void __launch_bounds__(256) mxfp4_pack_kernel(
    const __nv_bfloat16* __restrict__ x, int BH, int N, int T, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ sf, uint8_t* __restrict__ sf_mma, float* __restrict__ gs) {
  constexpr int KB = D / 64;  // 64-element groups per row
  const long long rows_pad = (long long)T * 128;
  const long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= (long long)BH * rows_pad * KB) return;
  const int kb = (int)(item % KB);
  const long long rowg = item / KB;
  const int bh = (int)(rowg / rows_pad);
  const int row = (int)(rowg % rows_pad);
  if (row == 0 && kb == 0) gs[bh] = 1.0f;
  const int t = row >> 7, rr = row & 127;
  uint32_t* mma_word = reinterpret_cast<uint32_t*>(
      sf_mma + ((long long)(bh * T + t) * KB + kb) * 512 + (rr & 31) * 16 + (rr >> 5) * 4);
  if (row >= N) {
    *mma_word = 0u;
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(x + ((long long)bh * N + row) * D + kb * 64);
  uint32_t out[8];
  uint32_t sb[2];
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    float f[32];
    float am = 0.0f;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 u = __ldg(src + 4 * b + v);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        f[8 * v + 2 * e] = __uint_as_float(w[e] << 16);
        f[8 * v + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
#pragma unroll
    for (int e = 0; e < 32; ++e) am = fmaxf(am, fabsf(f[e]));
    const int ex = mx_scale_exp(am);
    // 2^-ex: a normal FP32 power of two, since a BF16 block maximum gives ex <= 125
    const float mul = __uint_as_float((uint32_t)(127 - ex) << 23);
#pragma unroll
    for (int w4 = 0; w4 < 4; ++w4) {
      uint32_t word = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        word |= cvt_e2m1x2(__fmul_rn(f[8 * w4 + 2 * e], mul), __fmul_rn(f[8 * w4 + 2 * e + 1], mul)) << (8 * e);
      out[4 * b + w4] = word;
    }
    sb[b] = (uint32_t)(ex + 127);
  }
  uint4* dst = reinterpret_cast<uint4*>(codes + ((long long)bh * N + row) * (D / 2) + kb * 32);
  dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
  dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  const uint32_t pair = sb[0] | (sb[1] << 8);
  *reinterpret_cast<uint16_t*>(sf + ((long long)bh * N + row) * (D / 32) + kb * 2) = (uint16_t)pair;
  *mma_word = pair;
}

// ---------------------------------------------------------------------------
// Host launchers.
// ---------------------------------------------------------------------------
static int grid_chunks(long long work, int per_block, int cap) {
  long long c = (work + per_block - 1) / per_block;
  return (int)(c < 1 ? 1 : (c > cap ? cap : c));
}

cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t s) {
  const int D = a.d, T = (a.N + 127) / 128;
  const int BHq = a.B * a.Hq, BHk = a.B * a.Hkv;
  cudaError_t err = cudaMemsetAsync(a.amax_ws, 0, sizeof(uint32_t) * (size_t)(BHq + BHk + BHk * D), s);
  if (err != cudaSuccess) return err;
  uint32_t* amax_q = a.amax_ws;
  uint32_t* amax_k = amax_q + BHq;
  uint32_t* amax_v = amax_k + BHk;
  const long long per_head = (long long)a.N * D;
  {
    dim3 gq(grid_chunks(per_head / 8, 256 * 8, 256), BHq);
    amax_head_kernel<<<gq, 256, 0, s>>>(a.q, per_head, amax_q);
    dim3 gk(grid_chunks(per_head / 8, 256 * 8, 256), BHk);
    amax_head_kernel<<<gk, 256, 0, s>>>(a.k, per_head, amax_k);
    const int rpb = 512;
    dim3 gv((a.N + rpb - 1) / rpb, BHk);
    if (D == 128) amax_chan_kernel<128><<<gv, 256, 0, s>>>(a.v, a.N, rpb, amax_v);
    else amax_chan_kernel<64><<<gv, 256, 0, s>>>(a.v, a.N, rpb, amax_v);
    count_launches(3);
  }
  {
    const int KB = D / 64;
    const long long itq = (long long)BHq * T * 128 * KB, itk = (long long)BHk * T * 128 * KB;
    if (D == 128) {
      nvfp4_pack_kernel<128><<<(unsigned)((itq + 255) / 256), 256, 0, s>>>(a.q, BHq, a.N, T, amax_q, a.out.q_fp4,
                                                                          a.out.q_sf, a.out.q_sf_mma, a.out.q_gs);
      nvfp4_pack_kernel<128><<<(unsigned)((itk + 255) / 256), 256, 0, s>>>(a.k, BHk, a.N, T, amax_k, a.out.k_fp4,
                                                                          a.out.k_sf, a.out.k_sf_mma, a.out.k_gs);
      fp8_v_pack_kernel<128><<<dim3(T, BHk), 256, 0, s>>>(a.v, a.N, T, amax_v, a.out.v_fp8t,
                                                          reinterpret_cast<__nv_bfloat16*>(a.out.v_st), a.out.v_exp);
    } else {
      nvfp4_pack_kernel<64><<<(unsigned)((itq + 255) / 256), 256, 0, s>>>(a.q, BHq, a.N, T, amax_q, a.out.q_fp4,
                                                                         a.out.q_sf, a.out.q_sf_mma, a.out.q_gs);
      nvfp4_pack_kernel<64><<<(unsigned)((itk + 255) / 256), 256, 0, s>>>(a.k, BHk, a.N, T, amax_k, a.out.k_fp4,
                                                                         a.out.k_sf, a.out.k_sf_mma, a.out.k_gs);
      fp8_v_pack_kernel<64><<<dim3(T, BHk), 256, 0, s>>>(a.v, a.N, T, amax_v, a.out.v_fp8t,
                                                         reinterpret_cast<__nv_bfloat16*>(a.out.v_st), a.out.v_exp);
    }
    count_launches(3);
  }
  return cudaGetLastError();
}


// MXFP4 Q and K (mxfp4_pack_kernel), V as in launch_quantize (per-channel FP8).
// Workspace: the per-channel amax of V, B*Hkv*d words.
cudaError_t launch_quantize_mx(const QuantArgs& a, cudaStream_t s) {
  const int D = a.d, T = (a.N + 127) / 128;
  const int BHq = a.B * a.Hq, BHk = a.B * a.Hkv;
  uint32_t* amax_v = a.amax_ws;
  cudaError_t err = cudaMemsetAsync(amax_v, 0, sizeof(uint32_t) * (size_t)BHk * D, s);
  if (err != cudaSuccess) return err;
  const int rpb = 512;
  const dim3 gv((a.N + rpb - 1) / rpb, BHk);
  const int KB = D / 64;
  const long long itq = (long long)BHq * T * 128 * KB, itk = (long long)BHk * T * 128 * KB;
  if (D == 128) {
    amax_chan_kernel<128><<<gv, 256, 0, s>>>(a.v, a.N, rpb, amax_v);
    mxfp4_pack_kernel<128><<<(unsigned)((itq + 255) / 256), 256, 0, s>>>(a.q, BHq, a.N, T, a.out.q_fp4, a.out.q_sf,
                                                                        a.out.q_sf_mma, a.out.q_gs);
    mxfp4_pack_kernel<128><<<(unsigned)((itk + 255) / 256), 256, 0, s>>>(a.k, BHk, a.N, T, a.out.k_fp4, a.out.k_sf,
                                                                        a.out.k_sf_mma, a.out.k_gs);
    fp8_v_pack_kernel<128><<<dim3(T, BHk), 256, 0, s>>>(a.v, a.N, T, amax_v, a.out.v_fp8t,
                                                        reinterpret_cast<__nv_bfloat16*>(a.out.v_st), a.out.v_exp);
  } else {
    amax_chan_kernel<64><<<gv, 256, 0, s>>>(a.v, a.N, rpb, amax_v);
    mxfp4_pack_kernel<64><<<(unsigned)((itq + 255) / 256), 256, 0, s>>>(a.q, BHq, a.N, T, a.out.q_fp4, a.out.q_sf,
                                                                       a.out.q_sf_mma, a.out.q_gs);
    mxfp4_pack_kernel<64><<<(unsigned)((itk + 255) / 256), 256, 0, s>>>(a.k, BHk, a.N, T, a.out.k_fp4, a.out.k_sf,
                                                                       a.out.k_sf_mma, a.out.k_gs);
    fp8_v_pack_kernel<64><<<dim3(T, BHk), 256, 0, s>>>(a.v, a.N, T, amax_v, a.out.v_fp8t,
                                                       reinterpret_cast<__nv_bfloat16*>(a.out.v_st), a.out.v_exp);
  }
  count_launches(4);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Workspace-free quantisation.  Some callers cannot hand the library a device
// workspace: code that runs where device allocation is not allowed or not
// possible (for example inside a host callback or a custom allocator hook, in
// a process whose memory pool is owned by someone else, or in a C host program
// that only holds the input and output buffers).  For them the amax
// accumulators live in a fixed array in this library's device memory.
//
// The array holds kNoAllocWords 32-bit words (256 KB) on every GPU that loads
// the library, for the life of the process.  All calls share it: each call
// clears the words it uses before use, and calls whose work overlaps on the
// GPU (different streams, or different host threads on one device) race on it.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocWords = 65536;
static __device__ __align__(256) uint32_t g_noalloc_amax[kNoAllocWords];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
uint32_t* g_noalloc_ptr[kMaxDevices] = {};
}  // namespace

size_t noalloc_scratch_words() { return kNoAllocWords; }

// Host code must not pass `g_noalloc_amax` itself to a kernel: on the host that
// name is only a stand-in for the device array.  The device address is looked
// up once per device, with that device current, on the first call made on it,
// and kept: it is not looked up again after a reset of the device's context.
cudaError_t launch_quantize_noalloc(QuantArgs a, cudaStream_t s) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  uint32_t* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
      void* p = nullptr;
      err = cudaGetSymbolAddress(&p, g_noalloc_amax);
      if (err != cudaSuccess) return err;
      g_noalloc_ptr[dev] = static_cast<uint32_t*>(p);
    }
    ptr = g_noalloc_ptr[dev];
  }
  a.amax_ws = ptr;  // launch_quantize clears the words it uses before the amax passes
  return launch_quantize(a, s);
}

}  // namespace thrift
