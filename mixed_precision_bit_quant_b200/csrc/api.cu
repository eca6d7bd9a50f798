// C ABI of libthrift: argument validation, sizes and dispatch to the kernels.
#include <atomic>
#include <cmath>

#include "kernels.h"

namespace thrift {

static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

static bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 0 = ok, otherwise a thrift_status.
static int check_shape(const thrift_shape* s) {
  if (s == nullptr) return THRIFT_ERR_INVALID;
  if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->N < 1) return THRIFT_ERR_INVALID;
  if (s->Hq % s->Hkv != 0) return THRIFT_ERR_INVALID;
  if (s->causal != 0 && s->causal != 1) return THRIFT_ERR_INVALID;
  if (!(s->softmax_scale >= 0.0f) || std::isinf(s->softmax_scale)) return THRIFT_ERR_INVALID;
  if (s->d != 64 && s->d != 128) return THRIFT_ERR_UNSUPPORTED;
  const long long T = (s->N + 127) / 128;
  if (T > 4096) return THRIFT_ERR_UNSUPPORTED;                           // mask row fits the kernel's buffer
  if ((long long)s->B * s->Hq * T > 0x7FFFFFFFLL) return THRIFT_ERR_UNSUPPORTED;  // grid size
  if ((long long)s->B * (s->Hq + s->Hkv) > 65535) return THRIFT_ERR_UNSUPPORTED;   // grid.y of the per-head kernels
  return 0;
}

static size_t field_bytes(const thrift_shape* s, int f) {
  const size_t B = s->B, Hq = s->Hq, Hk = s->Hkv, N = s->N, d = s->d;
  const size_t T = (N + 127) / 128, Np = T * 128;
  switch (f) {
    case THRIFT_Q_FP4: return B * Hq * N * d / 2;
    case THRIFT_Q_SF: return B * Hq * N * d / 16;
    case THRIFT_Q_SF_MMA: return B * Hq * T * (d / 64) * 512;
    case THRIFT_Q_GS: return B * Hq * sizeof(float);
    case THRIFT_K_FP4: return B * Hk * N * d / 2;
    case THRIFT_K_SF: return B * Hk * N * d / 16;
    case THRIFT_K_SF_MMA: return B * Hk * T * (d / 64) * 512;
    case THRIFT_K_GS: return B * Hk * sizeof(float);
    case THRIFT_V_FP8T: return B * Hk * d * Np;
    case THRIFT_V_ST: return B * Hk * d * Np * 2;
    case THRIFT_V_EXP: return B * Hk * d;
    default: return 0;
  }
}

static int check_quant(const thrift_quant* q) {
  if (q == nullptr) return THRIFT_ERR_INVALID;
  const void* ptrs[] = {q->q_fp4, q->q_sf, q->q_sf_mma, q->q_gs, q->k_fp4, q->k_sf,
                        q->k_sf_mma, q->k_gs, q->v_fp8t, q->v_st, q->v_exp};
  for (const void* p : ptrs)
    if (!aligned16(p)) return THRIFT_ERR_INVALID;
  return 0;
}

}  // namespace thrift

using namespace thrift;

extern "C" {

size_t thrift_quant_bytes(const thrift_shape* shape, int field) {
  if (check_shape(shape) != 0) return 0;
  return field_bytes(shape, field);
}

size_t thrift_workspace_bytes(const thrift_shape* s, int op) {
  if (check_shape(s) != 0) return 0;
  const size_t T = ((size_t)s->N + 127) / 128;
  switch (op) {
    case THRIFT_OP_QUANTIZE:
      return sizeof(uint32_t) * ((size_t)s->B * s->Hq + (size_t)s->B * s->Hkv + (size_t)s->B * s->Hkv * s->d);
    case THRIFT_OP_SELECT:
      return sizeof(float) * T * (size_t)s->d * ((size_t)s->B * s->Hq + (size_t)s->B * s->Hkv);
    case THRIFT_OP_ATTN:
      return 0;
    case THRIFT_OP_QUANTIZE_MX:
      return sizeof(uint32_t) * (size_t)s->B * s->Hkv * s->d;
    case THRIFT_OP_SELECT_VERTICAL:
      return sizeof(float) * T * (size_t)s->d * ((size_t)s->B * s->Hq + (size_t)s->B * s->Hkv) +
             sizeof(int32_t) * T * (size_t)s->B * s->Hq;
    default:
      return 0;
  }
}

thrift_status thrift_quantize(const thrift_shape* shape, const void* q, const void* k, const void* v,
                              const thrift_quant* out, void* ws, size_t ws_bytes, void* stream) {
  int e = check_shape(shape);
  if (e) return (thrift_status)e;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(ws)) return THRIFT_ERR_INVALID;
  if ((e = check_quant(out))) return (thrift_status)e;
  if (ws_bytes < thrift_workspace_bytes(shape, THRIFT_OP_QUANTIZE)) return THRIFT_ERR_INVALID;
  QuantArgs a;
  a.B = shape->B; a.Hq = shape->Hq; a.Hkv = shape->Hkv; a.N = shape->N; a.d = shape->d;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.out = *out;
  a.amax_ws = static_cast<uint32_t*>(ws);
  return launch_quantize(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

thrift_status thrift_quantize_mx(const thrift_shape* shape, const void* q, const void* k, const void* v,
                                 const thrift_quant* out, void* ws, size_t ws_bytes, void* stream) {
  int e = check_shape(shape);
  if (e) return (thrift_status)e;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(ws)) return THRIFT_ERR_INVALID;
  if ((e = check_quant(out))) return (thrift_status)e;
  if (ws_bytes < thrift_workspace_bytes(shape, THRIFT_OP_QUANTIZE_MX)) return THRIFT_ERR_INVALID;
  QuantArgs a;
  a.B = shape->B; a.Hq = shape->Hq; a.Hkv = shape->Hkv; a.N = shape->N; a.d = shape->d;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.out = *out;
  a.amax_ws = static_cast<uint32_t*>(ws);
  return launch_quantize_mx(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

thrift_status thrift_quantize_noalloc(const thrift_shape* shape, const void* q, const void* k, const void* v,
                                      const thrift_quant* out, void* stream) {
  int e = check_shape(shape);
  if (e) return (thrift_status)e;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return THRIFT_ERR_INVALID;
  if ((e = check_quant(out))) return (thrift_status)e;
  const size_t words = thrift_workspace_bytes(shape, THRIFT_OP_QUANTIZE) / sizeof(uint32_t);
  if (words > noalloc_scratch_words()) return THRIFT_ERR_UNSUPPORTED;
  QuantArgs a;
  a.B = shape->B; a.Hq = shape->Hq; a.Hkv = shape->Hkv; a.N = shape->N; a.d = shape->d;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.out = *out;
  a.amax_ws = nullptr;
  return launch_quantize_noalloc(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

static thrift_status select_common(const thrift_shape* shape, const void* q, const void* k, int32_t budget_bp,
                                   int32_t budget_tiles, uint32_t* mask, int32_t* counts, void* ws, size_t ws_bytes,
                                   void* stream, int vertical) {
  int e = check_shape(shape);
  if (e) return (thrift_status)e;
  if (!aligned16(q) || !aligned16(k) || !aligned16(ws) || mask == nullptr) return THRIFT_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(mask) & 3u) != 0) return THRIFT_ERR_INVALID;
  if (counts != nullptr && (reinterpret_cast<uintptr_t>(counts) & 3u) != 0) return THRIFT_ERR_INVALID;
  if (budget_bp < 0 || budget_tiles < 0) return THRIFT_ERR_INVALID;
  if (ws_bytes < thrift_workspace_bytes(shape, vertical ? THRIFT_OP_SELECT_VERTICAL : THRIFT_OP_SELECT))
    return THRIFT_ERR_INVALID;
  SelectArgs a;
  a.B = shape->B; a.Hq = shape->Hq; a.Hkv = shape->Hkv; a.N = shape->N; a.d = shape->d;
  a.causal = shape->causal;
  a.budget_bp = budget_bp;
  a.budget_tiles = budget_tiles;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.mask = mask;
  a.counts = counts;
  a.pool_ws = static_cast<float*>(ws);
  a.vertical = vertical;
  a.votes = nullptr;
  if (vertical) {
    const size_t T = ((size_t)shape->N + 127) / 128;
    a.votes = reinterpret_cast<int32_t*>(a.pool_ws + T * (size_t)shape->d *
                                                         ((size_t)shape->B * shape->Hq + (size_t)shape->B * shape->Hkv));
  }
  return launch_select(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

thrift_status thrift_select(const thrift_shape* shape, const void* q, const void* k, int32_t budget_bp,
                            int32_t budget_tiles, uint32_t* mask, int32_t* counts, void* ws, size_t ws_bytes,
                            void* stream) {
  return select_common(shape, q, k, budget_bp, budget_tiles, mask, counts, ws, ws_bytes, stream, 0);
}

thrift_status thrift_select_vertical(const thrift_shape* shape, const void* q, const void* k, int32_t budget_bp,
                                     int32_t budget_tiles, uint32_t* mask, int32_t* counts, void* ws,
                                     size_t ws_bytes, void* stream) {
  return select_common(shape, q, k, budget_bp, budget_tiles, mask, counts, ws, ws_bytes, stream, 1);
}

static thrift_status attn_common(const thrift_shape* shape, const thrift_quant* quant, const void* q, const void* k,
                                 const uint32_t* mask, void* o, float* lse, void* stream, int mx) {
  int e = check_shape(shape);
  if (e) return (thrift_status)e;
  if ((e = check_quant(quant))) return (thrift_status)e;
  if (!aligned16(q) || !aligned16(k) || !aligned16(o) || !aligned16(mask)) return THRIFT_ERR_INVALID;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return THRIFT_ERR_INVALID;
  AttnArgs a;
  a.B = shape->B; a.Hq = shape->Hq; a.Hkv = shape->Hkv; a.N = shape->N; a.d = shape->d;
  a.causal = shape->causal;
  a.softmax_scale = shape->softmax_scale;
  a.quant = quant;
  a.q = q;
  a.k = k;
  a.mask = mask;
  a.o = o;
  a.lse = lse;
  a.mx = mx;
  return (thrift_status)launch_attn(a, static_cast<cudaStream_t>(stream));
}

thrift_status thrift_attn_fwd(const thrift_shape* shape, const thrift_quant* quant, const void* q, const void* k,
                              const uint32_t* mask, void* o, float* lse, void* ws, size_t ws_bytes, void* stream) {
  (void)ws;
  (void)ws_bytes;
  return attn_common(shape, quant, q, k, mask, o, lse, stream, 0);
}

thrift_status thrift_attn_fwd_mx(const thrift_shape* shape, const thrift_quant* quant, const void* q, const void* k,
                                 const uint32_t* mask, void* o, float* lse, void* stream) {
  return attn_common(shape, quant, q, k, mask, o, lse, stream, 1);
}

static int check_decode_shape(const thrift_decode_shape* s) {
  if (s == nullptr) return THRIFT_ERR_INVALID;
  if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->L < 1 || s->Hq % s->Hkv != 0) return THRIFT_ERR_INVALID;
  if (!(s->softmax_scale >= 0.0f) || std::isinf(s->softmax_scale)) return THRIFT_ERR_INVALID;
  if (s->d != 64 && s->d != 128) return THRIFT_ERR_UNSUPPORTED;
  if (!decode_group_supported(s->Hq / s->Hkv)) return THRIFT_ERR_UNSUPPORTED;
  if ((long long)s->B * s->Hkv > 65535 || (long long)s->B * s->Hq > 0x7FFFFFFFLL) return THRIFT_ERR_UNSUPPORTED;
  return 0;
}

size_t thrift_decode_cache_bytes(const thrift_decode_shape* s, int field) {
  if (check_decode_shape(s) != 0) return 0;
  const size_t rows = (size_t)s->B * s->Hkv * s->L;
  switch (field) {
    case THRIFT_DEC_KC: return rows * s->d / 2;
    case THRIFT_DEC_KSC: return rows * s->d / 32;
    case THRIFT_DEC_VC: return rows * s->d;
    case THRIFT_DEC_VSC: return rows * s->d / 32;
    default: return 0;
  }
}

size_t thrift_decode_workspace_bytes(const thrift_decode_shape* s) {
  if (check_decode_shape(s) != 0) return 0;
  return sizeof(float) * (size_t)s->B * s->Hq * decode_nchunk(s->B, s->Hkv, s->L) * (2 + (size_t)s->d);
}

static bool decode_cache_ok(const thrift_decode_cache* c) {
  return c != nullptr && aligned16(c->kc) && aligned16(c->ksc) && aligned16(c->vc) && aligned16(c->vsc);
}

static DecodeArgs decode_args(const thrift_decode_shape* s, const void* k, const void* v, const thrift_decode_cache* c) {
  DecodeArgs a;
  a.B = s->B; a.Hq = s->Hq; a.Hkv = s->Hkv; a.L = s->L; a.d = s->d;
  a.softmax_scale = s->softmax_scale;
  a.q = nullptr;
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.kc = c->kc; a.ksc = c->ksc; a.vc = c->vc; a.vsc = c->vsc;
  a.o = nullptr;
  a.lse = nullptr;
  a.ws = nullptr;
  return a;
}

thrift_status thrift_decode_quantize_cache(const thrift_decode_shape* shape, const void* k, const void* v,
                                           const thrift_decode_cache* cache, int32_t t_begin, int32_t t_end,
                                           void* stream) {
  int e = check_decode_shape(shape);
  if (e) return (thrift_status)e;
  if (!aligned16(k) || !aligned16(v) || !decode_cache_ok(cache)) return THRIFT_ERR_INVALID;
  if (t_begin < 0 || t_end > shape->L || t_begin > t_end) return THRIFT_ERR_INVALID;
  if (t_begin == t_end) return THRIFT_OK;
  const DecodeArgs a = decode_args(shape, k, v, cache);
  return launch_decode_quantize(a, t_begin, t_end, static_cast<cudaStream_t>(stream)) == cudaSuccess ? THRIFT_OK
                                                                                                     : THRIFT_ERR_CUDA;
}

thrift_status thrift_decode_step(const thrift_decode_shape* shape, const void* q, const void* k, const void* v,
                                 const thrift_decode_cache* cache, void* o, float* lse, void* ws, size_t ws_bytes,
                                 void* stream) {
  int e = check_decode_shape(shape);
  if (e) return (thrift_status)e;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(ws) || !decode_cache_ok(cache))
    return THRIFT_ERR_INVALID;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return THRIFT_ERR_INVALID;
  if (ws_bytes < thrift_decode_workspace_bytes(shape)) return THRIFT_ERR_INVALID;
  DecodeArgs a = decode_args(shape, k, v, cache);
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.ws = static_cast<float*>(ws);
  return launch_decode_step(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

thrift_status thrift_device_status(void* stream, uint32_t* detail) {
  uint32_t w = 0, wd = 0;
  if (read_and_clear_device_error(static_cast<cudaStream_t>(stream), &w) != cudaSuccess) return THRIFT_ERR_CUDA;
  if (read_and_clear_decode_error(&wd) != cudaSuccess) return THRIFT_ERR_CUDA;
  w |= wd << 8;
  if (detail != nullptr) *detail = w;
  return w != 0 ? THRIFT_ERR_TIMEOUT : THRIFT_OK;
}

thrift_status thrift_debug_withhold_v_load(int32_t tile) {
  set_withhold_v(tile);
  return THRIFT_OK;
}

const char* thrift_status_string(thrift_status s) {
  switch (s) {
    case THRIFT_OK: return "THRIFT_OK";
    case THRIFT_ERR_INVALID: return "THRIFT_ERR_INVALID";
    case THRIFT_ERR_UNSUPPORTED: return "THRIFT_ERR_UNSUPPORTED";
    case THRIFT_ERR_CUDA: return "THRIFT_ERR_CUDA";
    case THRIFT_ERR_TIMEOUT: return "THRIFT_ERR_TIMEOUT";
    default: return "THRIFT_ERR_UNKNOWN";
  }
}

thrift_status thrift_probe_mma(int32_t kind, int32_t n, int32_t iters, int32_t ctas, float* ms,
                              unsigned long long* cycles, void* stream) {
  if (ms == nullptr || cycles == nullptr || iters < 1 || iters > (1 << 22) || ctas < 1 || ctas > 65535)
    return THRIFT_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(cycles) & 7u) != 0) return THRIFT_ERR_INVALID;
  return (thrift_status)launch_mma_probe(kind, n, iters, ctas, ms, cycles, static_cast<cudaStream_t>(stream));
}

uint64_t thrift_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* thrift_version(void) { return "libthrift 0.1 (sm_100a)"; }

}  // extern "C"
