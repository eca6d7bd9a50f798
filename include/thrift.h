/*
 * thrift.h -- C ABI of libthrift: mixed FP4/BF16 attention forward (prefill)
 * for NVIDIA B200 (sm_100a).
 *
 * The method.  ThriftAttention: Selective Mixed Precision for Long-Context
 * FP4 Attention (abstract) runs attention in two stages: a cheap heuristic
 * picks a few important query-key block pairs for high precision, then the
 * selected blocks are computed in high precision and all others in 4-bit,
 * both merged by online softmax into one output.  HyQuant: Hybrid-Precision
 * Quantization for LLM Attention (abstract) keeps sink ("vertical line")
 * tokens and the local window in full precision.  Here the high precision
 * is BF16 (the inputs' own type), the low precision is NVFP4 for Q and K
 * and FP8 e4m3 for V and for the probabilities, tiles are 128 x 128.
 *
 * Three calls make one forward pass, in this order, on one stream:
 *   thrift_quantize  -> NVFP4 Q, K and FP8 V            (stage 0: operands)
 *   thrift_select    -> bitmask of BF16 tile pairs       (stage 1)
 *   thrift_attn_fwd  -> O (and optionally LSE)           (stage 2)
 *
 * Conventions for every call:
 *  - All tensor arguments are DEVICE pointers, allocated and owned by the
 *    caller; the library allocates no device memory.  Inputs are BF16,
 *    contiguous, head-major: q[B][Hq][N][d], k and v [B][Hkv][N][d].
 *    Every pointer must be 16-byte aligned.
 *  - Query head h reads key/value head h / (Hq / Hkv).
 *  - All work is enqueued on `stream` (a cudaStream_t, 0 = legacy default);
 *    no call synchronises.  Host-side argument errors are returned before
 *    anything is enqueued.  No exception crosses this interface.
 *  - T = ceil(N / 128) tiles, W = ceil(T / 32) mask words per query tile,
 *    Np = 128 * T (N padded to whole tiles).
 *  - Inputs must be finite; non-finite values give undefined results.
 *  - Supported: d in {64, 128}; Hq % Hkv == 0; 1 <= N; causal in {0, 1}.
 *    Limits: N <= 524288 (T <= 4096: one query tile's mask row is held in
 *    shared memory), B * Hq * T < 2^31 and B * (Hq + Hkv) <= 65535 (grid
 *    dimensions); larger shapes return THRIFT_ERR_UNSUPPORTED.
 */
#ifndef THRIFT_H
#define THRIFT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define THRIFT_API __attribute__((visibility("default")))
#else
#define THRIFT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  THRIFT_OK = 0,
  THRIFT_ERR_INVALID = 1,      /* bad argument (null / misaligned pointer, bad size) */
  THRIFT_ERR_UNSUPPORTED = 2,  /* valid but not supported (e.g. d not in {64,128}) */
  THRIFT_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  THRIFT_ERR_TIMEOUT = 4       /* a kernel's bounded wait gave up (device watchdog) */
} thrift_status;

/* Problem shape.  softmax_scale == 0 selects 1/sqrt(d). */
typedef struct {
  int32_t B, Hq, Hkv, N, d;
  int32_t causal;
  float softmax_scale;
} thrift_shape;

/*
 * Quantised operands written by thrift_quantize and read by thrift_attn_fwd.
 * Device pointers, caller-owned; sizes from thrift_quant_bytes().
 *
 * NVFP4 (Q and K): per (batch, head) tensor scale g = amax / 2688 (1 for an
 * all-zero head); per 16 consecutive elements along d an e4m3 scale
 * s = e4m3(amax_blk / (6 g)); element code e2m1(x / (dec(s) g)); all
 * arithmetic in FP32 with correctly rounded operations, round-to-nearest-even,
 * saturating; a block whose scale decodes to 0 gets zero codes.
 *
 * FP8 V: per (batch, kv head, channel c) the smallest integer e_c with
 * amax_c <= 448 * 2^e_c (0 for a zero channel); v_code = e4m3(v * 2^-e_c)
 * and the BF16 copy v * 2^-e_c (exact; values that fall into the BF16
 * subnormals round to nearest even), both stored transposed (channel-major)
 * and zero-padded to Np keys.
 */
typedef struct {
  uint8_t *q_fp4;     /* [B][Hq][N][d/2]   e2m1 codes, element 2t in the low nibble */
  uint8_t *q_sf;      /* [B][Hq][N][d/16]  e4m3 block scales, row-major             */
  uint8_t *q_sf_mma;  /* [B][Hq][T][d/64][512] the same scales in tensor-core order:
                         byte r0*16 + r1*4 + k of chunk kb holds the scale of row
                         128 t + 32 r1 + r0, block 4 kb + k; rows >= N hold 0     */
  float   *q_gs;      /* [B][Hq]           tensor scales g                          */
  uint8_t *k_fp4;     /* [B][Hkv][N][d/2]                                           */
  uint8_t *k_sf;      /* [B][Hkv][N][d/16]                                          */
  uint8_t *k_sf_mma;  /* [B][Hkv][T][d/64][512]                                     */
  float   *k_gs;      /* [B][Hkv]                                                   */
  uint8_t *v_fp8t;    /* [B][Hkv][d][Np]   e4m3 codes of v * 2^-e_c, transposed      */
  uint16_t *v_st;     /* [B][Hkv][d][Np]   bf16 v * 2^-e_c, transposed               */
  int8_t  *v_exp;     /* [B][Hkv][d]       e_c                                       */
} thrift_quant;

/* Field indices for thrift_quant_bytes, in struct order. */
enum {
  THRIFT_Q_FP4 = 0, THRIFT_Q_SF, THRIFT_Q_SF_MMA, THRIFT_Q_GS,
  THRIFT_K_FP4, THRIFT_K_SF, THRIFT_K_SF_MMA, THRIFT_K_GS,
  THRIFT_V_FP8T, THRIFT_V_ST, THRIFT_V_EXP, THRIFT_QUANT_NFIELDS
};

/* Operation indices for thrift_workspace_bytes. */
enum {
  THRIFT_OP_QUANTIZE = 0, THRIFT_OP_SELECT = 1, THRIFT_OP_ATTN = 2, THRIFT_OP_SELECT_VERTICAL = 3,
  THRIFT_OP_QUANTIZE_MX = 4
};

/* Bytes of one thrift_quant field for `shape` (0 for a bad shape or index). */
THRIFT_API size_t thrift_quant_bytes(const thrift_shape *shape, int field);

/* Bytes of device workspace an operation needs (0 = none; the pointer may be NULL). */
THRIFT_API size_t thrift_workspace_bytes(const thrift_shape *shape, int op);

/*
 * Stage 0: quantise Q, K to NVFP4 and V to FP8 (see thrift_quant).
 * q, k, v: BF16 device inputs.  out: every field must be non-NULL.
 * ws: device workspace of thrift_workspace_bytes(shape, THRIFT_OP_QUANTIZE)
 * bytes (per-head and per-channel amax accumulators, cleared by this call).
 */
THRIFT_API thrift_status thrift_quantize(const thrift_shape *shape, const void *q, const void *k,
                              const void *v, const thrift_quant *out, void *ws,
                              size_t ws_bytes, void *stream);

/*
 * Stage 0, microscaling variant: Q and K in MXFP4 instead of NVFP4.  The
 * attention-quantization topic page lists MXFP4 beside NVFP4 (and a
 * diagonal-tiled mixed-precision MXFP method); the format is the OCP
 * microscaling one: per 32 consecutive elements along d one e8m0 scale
 * 2^e, e = floor(log2 amax_block) - 2 clamped to [-127, 127] (-127 for an
 * all-zero block), codes e2m1(x * 2^-e) rounded to nearest, ties to the even
 * code, saturating at +-6, sign kept; no tensor scale.  V is quantised exactly
 * as by thrift_quantize (per-channel FP8).  Field use (buffers sized by
 * thrift_quant_bytes, as for NVFP4):
 *   q_fp4 / k_fp4   [B][H][N][d/2] e2m1 codes, element 2t in the low nibble;
 *   q_sf / k_sf     [B][H][N][d/32] e8m0 codes (the first half of the buffer);
 *   q_sf_mma / k_sf_mma [B][H][T][d/64][512]: per 64 elements of d a chunk whose
 *                   word 16*(r%32) + 4*(r/32) holds row r's two block scales of
 *                   that step in bytes 0 and 1 (bytes 2 and 3 zero; rows >= N 0);
 *   q_gs / k_gs     1.0f.
 * ws: thrift_workspace_bytes(shape, THRIFT_OP_QUANTIZE_MX) bytes (V's per-channel
 * amax, cleared by this call).  Read these operands with thrift_attn_fwd_mx.
 */
THRIFT_API thrift_status thrift_quantize_mx(const thrift_shape *shape, const void *q, const void *k,
                                            const void *v, const thrift_quant *out, void *ws,
                                            size_t ws_bytes, void *stream);

/*
 * thrift_quantize without a workspace argument.  The pages have no
 * counterpart of this call; it exists for callers that cannot allocate device
 * memory, e.g. a C host program that owns only its input and output buffers,
 * code running in a host callback or allocator hook where allocating is not
 * allowed, or a process whose device memory pool belongs to another component.
 *
 * Results are identical to thrift_quantize.  The per-head and per-channel amax
 * accumulators live in a fixed array inside the library: 65536 32-bit words
 * (256 KB) of device memory on every GPU that loads the library, held until the
 * process exits.  A shape needing more than that, i.e. with
 * B*Hq + B*Hkv + B*Hkv*d > 65536, is rejected with THRIFT_ERR_UNSUPPORTED.
 * Nothing is allocated or freed by this call.
 *
 * The first call on a device looks up the array's device address with that
 * device current (a one-time set-up per device); make that first call before
 * any stream capture.  The address found then is kept for the life of the
 * process: it does not survive cudaDeviceReset or any other teardown of the
 * device's primary context, after which this call must not be used in that
 * process.  All calls share the array and each clears the words it
 * uses before it uses them, so calls whose work can overlap on the GPU (other
 * streams, other host threads on the same device) race on it and must be
 * serialised by the caller.
 */
THRIFT_API thrift_status thrift_quantize_noalloc(const thrift_shape *shape, const void *q,
                                                const void *k, const void *v,
                                                const thrift_quant *out, void *stream);

/*
 * Stage 1: the BF16 tile-pair bitmask.
 * For every (b, hq, query tile i): pooled means qp_i, kp_j (FP32 column sums
 * over the tile's valid rows in ascending order, divided by the row count);
 * score(i,j) = sum over c ascending of FP32 products qp_i[c] * kp_j[c] with
 * FP32 additions (no fused multiply-add); candidates j in {0..i} (causal) or
 * {0..T-1}; the sink tile 0 and the diagonal tile i are forced; the budget
 * k_i is min(n_i, max(|forced|, budget_tiles)) when budget_tiles > 0, else
 * 0 for budget_bp == 0, n_i for budget_bp >= 10000, and
 * min(n_i, max(|forced|, ceil(budget_bp * n_i / 10000))) otherwise; the
 * forced tiles plus the best remaining candidates by (score descending,
 * index ascending) fill it.
 * mask: [B][Hq][T][W] uint32, bit j%32 of word j/32 = pair (i, j) in BF16.
 * counts: [B][Hq][T] int32 popcounts, or NULL.
 * ws: thrift_workspace_bytes(shape, THRIFT_OP_SELECT) bytes (pooled means).
 */
THRIFT_API thrift_status thrift_select(const thrift_shape *shape, const void *q, const void *k,
                            int32_t budget_bp, int32_t budget_tiles, uint32_t *mask,
                            int32_t *counts, void *ws, size_t ws_bytes, void *stream);

/*
 * Stage 1, vertical-line mode.  HyQuant: Hybrid-Precision Quantization for
 * LLM Attention (abstract) keeps "vertical-line" keys -- the ones many queries
 * attend to -- and the local window in high precision, chosen by a light
 * attention-pattern signal the page does not define.  This library's signal,
 * at tile level and in integers: every query tile of a (b, hq) votes for the
 * tiles thrift_select would add to its forced ones; a key tile's vote count is
 * its column importance; each query tile then keeps its forced tiles (sink 0,
 * diagonal i) and fills the same budget k_i with the remaining candidates
 * ranked by (votes descending, score descending, index ascending).
 * Same arguments, layouts and budget rule as thrift_select; ws must hold
 * thrift_workspace_bytes(shape, THRIFT_OP_SELECT_VERTICAL) bytes (pooled
 * means, then the int32 votes [B][Hq][T], cleared by this call).
 */
THRIFT_API thrift_status thrift_select_vertical(const thrift_shape *shape, const void *q, const void *k,
                                                int32_t budget_bp, int32_t budget_tiles, uint32_t *mask,
                                                int32_t *counts, void *ws, size_t ws_bytes, void *stream);

/*
 * Stage 2: the fused mixed-precision attention forward.
 * For each (b, hq, query tile i) and key tiles j ascending: BF16 pairs use
 * S = Q K^T * scale on the BF16 inputs; FP4 pairs use the block-scaled NVFP4
 * product times g_q g_k * scale; causal / ragged entries are -inf; the
 * running maximum is exact; p = exp(S - m) in FP32; l accumulates uncast p;
 * P is cast to e4m3 (FP4 pairs, with FP8 V) or BF16 (BF16 pairs, with the
 * BF16 V copy) after scaling by 2^8, and both products accumulate into one
 * FP32 output, which is finally scaled by 2^(e_c - 8) / l.
 * q, k: the BF16 inputs (read on BF16 pairs).  mask from thrift_select.
 * o: [B][Hq][N][d] BF16 output.  lse: [B][Hq][N] FP32 natural-log
 * log-sum-exp of the scaled logits, or NULL.
 * ws: may be NULL (thrift_workspace_bytes(..., THRIFT_OP_ATTN) == 0).
 */
THRIFT_API thrift_status thrift_attn_fwd(const thrift_shape *shape, const thrift_quant *quant,
                              const void *q, const void *k, const uint32_t *mask,
                              void *o, float *lse, void *ws, size_t ws_bytes, void *stream);

/*
 * Stage 2 on MXFP4 operands (written by thrift_quantize_mx): the FP4 tile
 * pairs run kind::mxf4 block-scaled tensor-core products (e8m0 scales per 32
 * elements); everything else -- BF16 pairs, the online softmax, the e4m3 cast
 * of P, the FP8 P.V product, masking, GQA, outputs -- is that of
 * thrift_attn_fwd.  Same arguments except the workspace (none).
 */
THRIFT_API thrift_status thrift_attn_fwd_mx(const thrift_shape *shape, const thrift_quant *quant,
                                            const void *q, const void *k, const uint32_t *mask,
                                            void *o, float *lse, void *stream);

/* ------------------------------------------------------------------------
 * Decode: one step of one new query token per sequence against a
 * mixed-precision KV cache.  HyQuant: Hybrid-Precision Quantization for LLM
 * Attention (abstract, decode stage) compresses the KV cache with the prefill
 * operator's principle -- sink ("vertical-line") tokens and the local window
 * in high precision, the rest low-bit -- and fuses the dequantisation into the
 * attention.  This library's reading: every cached token is quantised on its
 * own, as it is appended -- K as MXFP4, V as MXFP8 (e4m3), one e8m0 scale
 * 2^e per 32 channels, e = floor(log2 amax) - emax (2 for e2m1, 8 for e4m3),
 * clamped to [-127, 127], -127 for a zero block, elements rounded to nearest
 * with ties to the even code and saturated, sign kept; tokens [0, 128) (the
 * sink tile) and [L - 128, L) (the local window) are read from the BF16 cache,
 * every other token from its quantised form; the query stays BF16; logits
 * q . k * scale, exact softmax over all L tokens in FP32.  Both products run on
 * the tensor cores.  Logits: FP16 operands for quantised tokens (the e2m1
 * codes are exact; the query is scaled per head by a power of two that puts
 * its largest component in [2^14, 2^15), so components more than 2^28 below it
 * lose bits to FP16 subnormals)
 * and TF32 for the BF16 rows; P.V: TF32, the e4m3 codes exact and P (times V's
 * power-of-two block scale) as the sum of two TF32 terms, about 21 bits.
 * ------------------------------------------------------------------------ */
typedef struct {
  int32_t B, Hq, Hkv, L, d; /* L: cached tokens (>= 1); d in {64, 128}; Hq / Hkv in {1, 2, 4, 8, 16} */
  float softmax_scale;      /* 0 selects 1/sqrt(d) */
} thrift_decode_shape;

/* The quantised cache (device pointers, caller-owned, sizes from thrift_decode_cache_bytes). */
typedef struct {
  uint8_t *kc;   /* [B][Hkv][L][d/2]  e2m1 codes of K, channel 2t in the low nibble */
  uint8_t *ksc;  /* [B][Hkv][L][d/32] e8m0 scale codes of K                        */
  uint8_t *vc;   /* [B][Hkv][L][d]    e4m3 codes of V                              */
  uint8_t *vsc;  /* [B][Hkv][L][d/32] e8m0 scale codes of V                        */
} thrift_decode_cache;

enum { THRIFT_DEC_KC = 0, THRIFT_DEC_KSC, THRIFT_DEC_VC, THRIFT_DEC_VSC, THRIFT_DEC_NFIELDS };

/* Bytes of one thrift_decode_cache field (0 for a bad shape or index). */
THRIFT_API size_t thrift_decode_cache_bytes(const thrift_decode_shape *shape, int field);

/* Bytes of device workspace thrift_decode_step needs (the per-chunk softmax states). */
THRIFT_API size_t thrift_decode_workspace_bytes(const thrift_decode_shape *shape);

/*
 * Quantise cache tokens [t_begin, t_end) of every (b, kv head) into `cache`
 * (appending a token t is the call with [t, t + 1)).  k, v: the BF16 cache
 * [B][Hkv][L][d], device.  0 <= t_begin <= t_end <= L, else
 * THRIFT_ERR_INVALID; an empty range enqueues nothing.
 */
THRIFT_API thrift_status thrift_decode_quantize_cache(const thrift_decode_shape *shape, const void *k,
                                                      const void *v, const thrift_decode_cache *cache,
                                                      int32_t t_begin, int32_t t_end, void *stream);

/*
 * One decode step.  q: [B][Hq][d] BF16; k, v: the BF16 cache (only the sink
 * and window rows are read); cache: its quantised form (every token outside
 * the sink and the window must have been quantised); o: [B][Hq][d] BF16;
 * lse: [B][Hq] FP32 natural-log log-sum-exp, or NULL; ws:
 * thrift_decode_workspace_bytes(shape) bytes.  Query head h reads kv head
 * h / (Hq / Hkv).  Every pointer 16-byte aligned (lse: 4).
 */
THRIFT_API thrift_status thrift_decode_step(const thrift_decode_shape *shape, const void *q, const void *k,
                                            const void *v, const thrift_decode_cache *cache, void *o,
                                            float *lse, void *ws, size_t ws_bytes, void *stream);

/*
 * Synchronises `stream`, then reads and clears the library's device error
 * words.  Returns THRIFT_ERR_TIMEOUT if a kernel's bounded wait gave up since
 * the last call (the kernel then returned early and its outputs are
 * undefined); *detail (if non-NULL) receives the raw error word: bits 0-2
 * from thrift_attn_fwd (1 producer, 2 tensor-core issuer, 4 softmax), bit 8
 * from thrift_decode_step (a CTA's wait for its bulk-copied cache codes); the
 * other kernels wait on nothing and set no bit.
 */
THRIFT_API thrift_status thrift_device_status(void *stream, uint32_t *detail);

/*
 * Test hook for the device watchdog.  After thrift_debug_withhold_v_load(t)
 * with t >= 0, every later thrift_attn_fwd launch of this process skips the
 * copy of key tile t's V operand in each work tile that reaches key tile t, so
 * the product P_t V_t waits for data that never arrives.  That bounded wait
 * gives up after 2 s; the work tile raises the abort flag, every role of it
 * returns, its outputs are left undefined, and the next thrift_device_status
 * reports THRIFT_ERR_TIMEOUT.  The CUDA context stays usable.  t < 0 turns the
 * hook off (the default).  Process-wide; set it only while no launch is being
 * issued from another thread.  Always returns THRIFT_OK.
 */
THRIFT_API thrift_status thrift_debug_withhold_v_load(int32_t tile);

/*
 * Measurement utility (not part of the method): the dense rate of the three
 * tensor-core instruction forms the attention kernel issues, for stating its
 * roofline against measured rates.  kind 0: block-scaled NVFP4 (e2m1 x e2m1,
 * e4m3 scales per 16), both operands in shared memory, 128 x n x 64 per
 * instruction; kind 1: e4m3 x e4m3 with A in tensor memory, 128 x n x 32;
 * kind 2: BF16 x BF16 from shared memory, 128 x n x 16.  n: 128 (kinds 0-2)
 * or 256 (kinds 1, 2).  `ctas` CTAs (one per SM when ctas <= SM count) each
 * issue `iters` steps of K = 128 into one FP32 accumulator:
 * 2 * 128 * n * 128 * iters * ctas FLOPs.  Synchronises `stream`; *ms gets the
 * CUDA-event time of the launch; cycles: DEVICE buffer of `ctas` uint64
 * (8-byte aligned) receiving each CTA's clock-cycle count.  1 <= iters <= 2^22,
 * 1 <= ctas <= 65535, else THRIFT_ERR_INVALID; other kind / n pairs
 * THRIFT_ERR_UNSUPPORTED; a wait longer than 2 s THRIFT_ERR_TIMEOUT.
 */
THRIFT_API thrift_status thrift_probe_mma(int32_t kind, int32_t n, int32_t iters, int32_t ctas, float *ms,
                                          unsigned long long *cycles, void *stream);

/* Human-readable name of a status code (static storage). */
THRIFT_API const char *thrift_status_string(thrift_status status);

/* Number of kernels this library has launched since load (all devices). */
THRIFT_API uint64_t thrift_launch_count(void);

/* Library version string. */
THRIFT_API const char *thrift_version(void);

#ifdef __cplusplus
}
#endif

#endif /* THRIFT_H */
