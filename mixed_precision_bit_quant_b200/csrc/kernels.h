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
};
// Returns a thrift_status.
int launch_attn(const AttnArgs& a, cudaStream_t s);

cudaError_t read_and_clear_device_error(cudaStream_t s, uint32_t* word);
void set_withhold_v(int tile);  // watchdog test hook (-1: off)

}  // namespace thrift
