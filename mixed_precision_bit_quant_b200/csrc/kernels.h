// Internal launch interface between the C ABI layer and the kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/thrift.h"

namespace thrift {

void count_launches(int n);

struct QuantArgs {
  int B, Hq, Hkv, N, d;
  const __nv_bfloat16 *q, *k, *v;
  thrift_quant out;
  uint32_t* amax_ws;  // [B*Hq + B*Hkv + B*Hkv*d]
};
cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t s);
// MXFP4 Q and K, per-channel FP8 V; amax_ws: [B*Hkv*d].
cudaError_t launch_quantize_mx(const QuantArgs& a, cudaStream_t s);
// Same as launch_quantize, with the amax scratch in the library's static device array.
cudaError_t launch_quantize_noalloc(QuantArgs a, cudaStream_t s);
size_t noalloc_scratch_words();

struct SelectArgs {
  int B, Hq, Hkv, N, d, causal;
  int budget_bp, budget_tiles;
  const __nv_bfloat16 *q, *k;
  uint32_t* mask;
  int32_t* counts;
  float* pool_ws;  // [B*Hq*T*d + B*Hkv*T*d]
  int vertical;     // 0: score mode; 1: vertical-line mode (votes from a score-mode pass)
  int32_t* votes;   // [B*Hq*T] column votes (vertical mode; null in score mode)
};
cudaError_t launch_select(const SelectArgs& a, cudaStream_t s);

struct AttnArgs {
  int B, Hq, Hkv, N, d, causal;
  float softmax_scale;
  const thrift_quant* quant;
  const void *q, *k;
  const uint32_t* mask;
  void* o;
  float* lse;
  int mx;  // 1: the FP4 operands are MXFP4 (e8m0 scales per 32), 0: NVFP4
};
// Returns a thrift_status.
int launch_attn(const AttnArgs& a, cudaStream_t s);

struct DecodeArgs {
  int B, Hq, Hkv, L, d;
  float softmax_scale;
  const __nv_bfloat16 *q, *k, *v;
  uint8_t *kc, *ksc, *vc, *vsc;
  __nv_bfloat16* o;
  float* lse;
  float* ws;  // [B*Hq][nchunk][2 + d] chunk softmax states
};
int decode_nchunk(int B, int Hkv, int L);  // splits per (b, kv head)
bool decode_group_supported(int G);  // query heads per kv head: 1, 2, 4, 8 or 16
cudaError_t launch_decode_quantize(const DecodeArgs& a, int t0, int t1, cudaStream_t s);
cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t s);
// reads and clears the decode kernels' device error word (1: a chunk copy's wait gave up)
cudaError_t read_and_clear_decode_error(uint32_t* word);

cudaError_t read_and_clear_device_error(cudaStream_t s, uint32_t* word);

// Tensor-core rate probe (returns a thrift_status); cycles_dev: [ctas] per-CTA clock counts.
int launch_mma_probe(int kind, int n, int iters, int ctas, float* ms, unsigned long long* cycles_dev,
                     cudaStream_t st);
void set_withhold_v(int tile);  // watchdog test hook (-1: off)

}  // namespace thrift
