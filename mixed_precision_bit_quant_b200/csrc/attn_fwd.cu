// Stage 2: fused mixed FP4 / BF16 attention forward on tcgen05 tensor cores.
//
// ThriftAttention: Selective Mixed Precision for Long-Context FP4 Attention
// (abstract, second stage): the selected query-key blocks are computed in
// high precision and the rest in FP4, both merged by online softmax into a
// single output.  HyQuant: Hybrid-Precision Quantization for LLM Attention
// (abstract): one hybrid-precision attention operator for prefill.
//
// One CTA computes one 128-row query tile (b, hq, i) against the key tiles
// j = 0 .. (causal ? i : T-1) in ascending order.  512 threads, 16 warps:
//   warps 0-11 softmax groups 0, 1, 2 (four warps each); group g takes the tiles
//              j = g, g+3, ...  One thread owns one query row (= TMEM lane) of its
//              tiles: read S from TMEM once, mask edge tiles, row max, take the
//              exact running maximum m_{j-1} from the group of tile j-1 (shared
//              memory + mbarrier), exp2, partial row sums, P (e4m3 or bf16) into
//              TMEM, O rescaled in TMEM when a row's maximum grows.  Three groups
//              put three softmax warps on each SM sub-partition, so one group's
//              exponentials run while the others load S, reduce maxima or wait.
//   warps 12/14 TMA producers: warp 12 loads Q (NVFP4 + scales + BF16) once and
//              per key tile NVFP4 K + scales or BF16 K; warp 14 loads e4m3 V^T or
//              BF16 V^T, per mask bit.
//   warp 13    TMEM allocator and QK^T issuer (one thread): FP4 pair
//              S = Q4 K4^T kind::mxf4nvf4 (block scales in TMEM), BF16 pair
//              S = Q K^T kind::f16, into S buffer j % 2 as soon as S_{j-2} was read.
//   warp 15    P.V issuer (one thread): O += P8 V8 kind::f8f6f4 or O += P16 Vs
//              kind::f16, P read from TMEM; each product's completion is committed
//              to a ring of mbarriers that the softmax groups wait on before
//              they reuse a P region or rescale O.
//   Warps 12-15 form the last warpgroup, whose registers the softmax warps take
//   over with setmaxnreg.
// The exponentials of a 32-column chunk form one branch-free block that makes
// both P encodings (e4m3 and bf16); one copy of this block serves FP4 and BF16
// tiles alike, which keeps the loop small enough for the instruction cache.
// TMEM columns: S double buffer [0,256), O [256,256+D), three 32-column e4m3 P
// regions [256+D, 352+D) (region j % 3 belongs to group j % 3; BF16 tiles keep P
// in their S buffer), block scales after.
#include <cuda.h>
#include <stdlib.h>

#include <atomic>

#include "dev.cuh"
#include "kernels.h"

namespace thrift {

__device__ uint32_t g_attn_error_word;
// Test hook for the device watchdog (thrift_debug_withhold_v_load): a key tile
// whose V load the producer skips, so the P.V issuer's bounded wait runs out.
static std::atomic<int> g_withhold_v{-1};

void set_withhold_v(int tile) { g_withhold_v.store(tile < 0 ? -1 : tile, std::memory_order_relaxed); }

namespace attn {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait: far above any legitimate wait
constexpr int kGroups = 3;                          // softmax groups of four warps
constexpr int kThreads = 128 * kGroups + 128;       // + 4 producer / issuer warps
constexpr int kSoftmaxRegs = 152, kOtherRegs = 56;  // 3*128*152 + 128*56 = 512*128 (the launch budget)
static_assert(kGroups * 128 * kSoftmaxRegs + 128 * kOtherRegs <= 65536, "register split exceeds the launch budget");
constexpr int kPRing = 8;                           // P_FULL barriers per group
constexpr int kMaxW = 128;                          // mask words per query tile (T <= 4096)
// Operand rings: FP4 tiles use NLO slots of K (e2m1 + scales) and of V^T (e4m3);
// BF16 tiles use NHI slots of bf16 K and V^T.  Producer and MMA issuer walk the
// tiles in order and count FP4 and BF16 tiles separately to find slot and phase.
constexpr int NLO = 4, NHI = 1;
enum Bar : int {
  Q_FULL = 0,
  KL_FULL = 1, KL_EMPTY = KL_FULL + NLO, VL_FULL = KL_EMPTY + NLO, VL_EMPTY = VL_FULL + NLO,
  KH_FULL = VL_EMPTY + NLO, KH_EMPTY = KH_FULL + NHI, VH_FULL = KH_EMPTY + NHI, VH_EMPTY = VH_FULL + NHI,
  // P_FULL is a ring of kPRing barriers per softmax group, indexed by the group's
  // tile count: a group reuses a slot 3 * kPRing tiles later, so it must not run that
  // far ahead of the P.V issuer.  It cannot: to start tile j it needed m_{j-1}, so
  // tile j-2 had started and tile j-5 (same group) had finished; an FP4 tile j-5
  // waited for P_{j-8} V_{j-8}, a BF16 tile j-5 made S_{j-3} wait for P_{j-5} V_{j-5}.
  // Either way the issuer is past tile j-8 when tile j's P arrives.
  // PVC is the ring of P.V completion barriers (see pv_wait).
  // S_FULL is indexed by tile % 4 (three groups share the two S buffers: a group may
  // wait for its next tile while the buffer still has the phase of the tile before)
  S_FULL = VH_EMPTY + NHI, S_FREE = S_FULL + 4, P_FULL = S_FREE + 2, PVC = P_FULL + kPRing * kGroups,
  QK_DRAIN = PVC + 8, PV_DRAIN = QK_DRAIN + 1,
  MX = PV_DRAIN + 1,  // running-max hand-off [group][quarter]
  NBAR = MX + 4 * kGroups
};

__host__ __device__ constexpr int al(int x, int a) { return (x + a - 1) / a * a; }

// Ring slot and use count of the n-th FP4 (NLO slots) or BF16 (NHI slots) tile, with
// constant divisors in each branch.
__device__ __forceinline__ void ring_pos(bool hi, int n, int& slot, int& use) {
  if (hi) {
    slot = n % NHI;
    use = n / NHI;
  } else {
    slot = n % NLO;
    use = n / NLO;
  }
}

template <int D>
struct Layout {
  static constexpr int QFP4 = 128 * D / 2;    // packed e2m1 Q tile
  static constexpr int QBF = 128 * D * 2;      // bf16 Q tile (D/64 boxes of 128 x 64)
  static constexpr int SF = (D / 64) * 512;    // block scales of one tile, tensor-core order
  static constexpr int KLO = 128 * D / 2;     // e2m1 K tile
  static constexpr int VLO = D * 128;         // e4m3 V^T tile
  static constexpr int KHI = 128 * D * 2;     // bf16 K tile (D/64 boxes of 128 x 64)
  static constexpr int VHI = D * 128 * 2;     // bf16 V^T tile (2 boxes of D x 64)
  static constexpr int OFF_QFP4 = 0;
  static constexpr int OFF_QBF = al(OFF_QFP4 + QFP4, 1024);
  static constexpr int OFF_KL = OFF_QBF + QBF;         // NLO slots
  static constexpr int OFF_VL = OFF_KL + NLO * KLO;    // NLO slots
  static constexpr int OFF_KH = OFF_VL + NLO * VLO;    // NHI slots
  static constexpr int OFF_VH = OFF_KH + NHI * KHI;    // NHI slots
  static constexpr int OFF_QSF = OFF_VH + NHI * VHI;
  static constexpr int OFF_KSF = OFF_QSF + SF;         // NLO slots
  static constexpr int OFF_BAR = al(OFF_KSF + NLO * SF, 64);
  static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;  // tmem holder, abort flag, completed-P.V count
  static constexpr int OFF_MASK = al(OFF_MISC + 16, 16);
  static constexpr int OFF_VSC = OFF_MASK + 4 * kMaxW;  // per-channel output scales
  static constexpr int OFF_XCH = OFF_VSC + 4 * D;       // running maxima [groups][128 rows]
  static constexpr int OFF_FIN = OFF_XCH + 4 * 128 * kGroups;  // final partial sums [groups][128], maxima after
  static constexpr int BYTES = OFF_FIN + 4 * 256 * kGroups;
  // request at least 116 KB so that one CTA (and its 512 TMEM columns) owns an SM
  static constexpr int DYN = (BYTES + 1024 > 116 * 1024) ? BYTES + 1024 : 116 * 1024;
  // TMEM columns
  // FP4 tiles write P (e4m3, 32 columns) into P region j % 3; BF16 tiles write P
  // (bf16, 64 columns) over the leading columns of their own S buffer.
  static constexpr uint32_t S_COL0 = 0, O_COL = 256, P_COL = 256 + D, SFA_COL = P_COL + 96,
                            SFB_COL0 = SFA_COL + 8;
};

struct Params {
  const uint8_t* q_sf_mma;
  const uint8_t* k_sf_mma;
  const float* q_gs;
  const float* k_gs;
  const int8_t* v_exp;
  const uint32_t* mask;
  __nv_bfloat16* o;
  float* lse;
  int B, Hq, Hkv, N, T, W, causal;
  float scale_log2;  // softmax scale * log2(e)
  int withhold_v;    // test hook: key tile whose V load is never issued (-1: none)
};

__device__ __forceinline__ void raise_error(volatile int* abort, uint32_t code) {
  *abort = 1;
  atomicOr(&g_attn_error_word, code);
}

template <int D, bool MXFP4>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_qfp4, const __grid_constant__ CUtensorMap tm_kfp4,
                    const __grid_constant__ CUtensorMap tm_qbf, const __grid_constant__ CUtensorMap tm_kbf,
                    const __grid_constant__ CUtensorMap tm_vfp8, const __grid_constant__ CUtensorMap tm_vbf,
                    const Params p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // longest rows first for causal problems
  const int BHq = p.B * p.Hq;
  const int lin = blockIdx.x;
  const int i = p.causal ? (p.T - 1 - lin / BHq) : (lin / BHq);
  const int bhq = lin % BHq;
  const int b = bhq / p.Hq, h = bhq % p.Hq;
  const int bhk = b * p.Hkv + h / (p.Hq / p.Hkv);
  const int nj = p.causal ? i + 1 : p.T;

  auto BAR = [&](int k) -> uint32_t { return sb + L::OFF_BAR + 8 * k; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  uint32_t* mrow = reinterpret_cast<uint32_t*>(smem + L::OFF_MASK);
  float* vsc = reinterpret_cast<float*>(smem + L::OFF_VSC);

  if (warp == 0) {
    // the lanes of warp 0 initialise the barriers (Q_FULL is the K producer's, below)
    for (int k = lane; k < NBAR; k += 32) {
      const bool by_group = (k >= S_FREE && k < S_FREE + 2) || (k >= P_FULL && k < P_FULL + kPRing * kGroups);
      if (k != Q_FULL) mbar_init(BAR(k), by_group ? 4 : 1);  // softmax barriers: one arrival per warp of the group
    }
    if (lane == 0) {
      *abort = 0;
      *reinterpret_cast<volatile uint32_t*>(smem + L::OFF_MISC + 8) = 0u;
    }
    fence_mbar_init();
  } else if (warp == 4 * kGroups && lane == 0) {
    // Q is loaded before the CTA-wide setup completes: its latency overlaps the rest
    mbar_init(BAR(Q_FULL), 1);
    fence_mbar_init();
    mbar_expect_tx(BAR(Q_FULL), L::QFP4 + L::QBF + L::SF);
    tma_load_3d(sb + L::OFF_QFP4, &tm_qfp4, 0, i * 128, bhq, BAR(Q_FULL));
    tma_load_3d(sb + L::OFF_QBF, &tm_qbf, 0, i * 128, bhq, BAR(Q_FULL));
    if (D == 128) tma_load_3d(sb + L::OFF_QBF + 16384, &tm_qbf, 64, i * 128, bhq, BAR(Q_FULL));
    bulk_load(sb + L::OFF_QSF, p.q_sf_mma + ((size_t)bhq * p.T + i) * L::SF, L::SF, BAR(Q_FULL));
  }
  if (warp == 4 * kGroups + 1) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  for (int w = tid; w < p.W; w += kThreads) mrow[w] = p.mask[((size_t)bhq * p.T + i) * p.W + w];
  for (int c = tid; c < D; c += kThreads) vsc[c] = pow2f((int)p.v_exp[(size_t)bhk * D + c]);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  auto is_hi = [&](int j) -> bool { return (mrow[j >> 5] >> (j & 31)) & 1u; };
  volatile int never = 0;
  // P_t V_t completion: tcgen05.commit to PVC[t % 8] (products complete in issue order).  A
  // waiter for tile t cannot see the barrier two phases ahead: P_{t+8} exists only after
  // m_{t+7}, i.e. after tile t+7 started, so tiles t+1 (O rescale) and t+3 (P region) had
  // finished and the QK^T issuer had passed S_{t+2}: every wait for P_t V_t came first.
  auto pv_wait = [&](int t) -> bool { return mbar_wait(BAR(PVC + (t & 7)), (t >> 3) & 1, abort, kWaitLimitNs); };
  int issued_lo = 0, issued_hi = 0;                 // loads a producer issued (drained on abort)

  if (warp >= 4 * kGroups) {
    regs_dec<kOtherRegs>();
    if ((warp == 4 * kGroups || warp == 4 * kGroups + 2) && lane == 0) {
      // ---------------------------------------------------------- producers
      // warp 12 loads Q once and the K tiles, warp 14 the V tiles: K loads run
      // ahead of the softmax, bounded only by the QK^T that frees their stage.
      const bool kside = (warp == 4 * kGroups);
      if (kside) {
        prefetch_tmap(&tm_kfp4); prefetch_tmap(&tm_kbf);
      } else {
        prefetch_tmap(&tm_vfp8); prefetch_tmap(&tm_vbf);
      }
      int nlo = 0, nhi = 0;
      for (int j = 0; j < nj; ++j) {
        const bool hi = is_hi(j);
        int slot, use;
        ring_pos(hi, hi ? nhi : nlo, slot, use);
        const int FULL = kside ? (hi ? KH_FULL : KL_FULL) : (hi ? VH_FULL : VL_FULL);
        const int EMPTY = kside ? (hi ? KH_EMPTY : KL_EMPTY) : (hi ? VH_EMPTY : VL_EMPTY);
        if (use > 0 && !mbar_wait(BAR(EMPTY + slot), (use - 1) & 1, abort, kWaitLimitNs)) {
          raise_error(abort, 1u);
          break;
        }
        const uint32_t full = BAR(FULL + slot);
        if (kside) {
          if (hi) {
            const uint32_t kb = sb + L::OFF_KH + slot * L::KHI;
            mbar_expect_tx(full, L::KHI);
            tma_load_3d(kb, &tm_kbf, 0, j * 128, bhk, full);
            if (D == 128) tma_load_3d(kb + 16384, &tm_kbf, 64, j * 128, bhk, full);
          } else {
            mbar_expect_tx(full, L::KLO + L::SF);
            tma_load_3d(sb + L::OFF_KL + slot * L::KLO, &tm_kfp4, 0, j * 128, bhk, full);
            bulk_load(sb + L::OFF_KSF + slot * L::SF, p.k_sf_mma + ((size_t)bhk * p.T + j) * L::SF, L::SF, full);
          }
        } else if (j != p.withhold_v) {
          if (hi) {
            const uint32_t vb = sb + L::OFF_VH + slot * L::VHI;
            mbar_expect_tx(full, L::VHI);
            tma_load_3d(vb, &tm_vbf, j * 128, 0, bhk, full);
            tma_load_3d(vb + D * 128, &tm_vbf, j * 128 + 64, 0, bhk, full);
          } else {
            mbar_expect_tx(full, L::VLO);
            tma_load_3d(sb + L::OFF_VL + slot * L::VLO, &tm_vfp8, j * 128, 0, bhk, full);
          }
        }
        if (hi) ++nhi; else ++nlo;
      }
      issued_lo = nlo;
      issued_hi = nhi;
    } else if (warp == 4 * kGroups + 1 && lane == 0) {
      // ---------------------------------------------------------- QK^T issuer
      constexpr int KB = D / 64;
      constexpr uint32_t fp4_row = D / 2;
      constexpr uint32_t fp4_swz = (D == 128) ? SWZ_64B : SWZ_32B;
      bool ok = mbar_wait(BAR(Q_FULL), 0, abort, kWaitLimitNs);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
          tmem_cp_32x128b_x4(tmem + L::SFA_COL + 4 * kb, smem_desc(sb + L::OFF_QSF + kb * 512, 16, 128, SWZ_NONE));
      }
      int n_lo = 0, n_hi = 0;
      uint32_t mw = 0;
      for (int j = 0; ok && j < nj; ++j) {
        if ((j & 31) == 0) mw = mrow[j >> 5];
        const bool hi = (mw >> (j & 31)) & 1u;
        const int s = j & 1;
        // S buffer s is free once the softmax group has read S_{j-2} and, when tile j-2 was
        // BF16 (its P lives in that buffer), once P_{j-2} V_{j-2} has completed
        if (j >= 2) {
          if (!mbar_wait(BAR(S_FREE + s), ((j - 2) >> 1) & 1, abort, kWaitLimitNs)) { ok = false; break; }
          if (((j - 2) >> 5) == (j >> 5) ? ((mw >> ((j - 2) & 31)) & 1u) : is_hi(j - 2)) {
            if (!pv_wait(j - 2)) { ok = false; break; }
          }
        }
        int slot, use;
        ring_pos(hi, hi ? n_hi : n_lo, slot, use);
        if (!mbar_wait(BAR((hi ? KH_FULL : KL_FULL) + slot), use & 1, abort, kWaitLimitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_s = tmem + L::S_COL0 + 128 * s;
        if (hi) {
          const uint32_t kb_addr = sb + L::OFF_KH + slot * L::KHI;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
            mma_bf16_ss(d_s, smem_desc(sb + L::OFF_QBF + off, 16, 1024, SWZ_128B),
                        smem_desc(kb_addr + off, 16, 1024, SWZ_128B), idesc_bf16(128), k > 0);
          }
          tc_commit(BAR(KH_EMPTY + slot));
          ++n_hi;
        } else {
          const uint32_t kb_addr = sb + L::OFF_KL + slot * L::KLO;
          const uint32_t sfb = tmem + L::SFB_COL0 + 8 * s;
#pragma unroll
          for (int kb = 0; kb < KB; ++kb)
            tmem_cp_32x128b_x4(sfb + 4 * kb, smem_desc(sb + L::OFF_KSF + slot * L::SF + kb * 512, 16, 128, SWZ_NONE));
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const uint64_t ad = smem_desc(sb + L::OFF_QFP4 + kb * 32, 16, 8 * fp4_row, fp4_swz);
            const uint64_t bd = smem_desc(kb_addr + kb * 32, 16, 8 * fp4_row, fp4_swz);
            if constexpr (MXFP4)
              mma_mxfp4_ss(d_s, ad, bd, idesc_mxfp4(128), tmem + L::SFA_COL + 4 * kb, sfb + 4 * kb, kb > 0);
            else
              mma_nvfp4_ss(d_s, ad, bd, idesc_nvfp4(128), tmem + L::SFA_COL + 4 * kb, sfb + 4 * kb, kb > 0);
          }
          tc_commit(BAR(KL_EMPTY + slot));
          ++n_lo;
        }
        tc_commit(BAR(S_FULL + (j & 3)));
      }
      if (!ok) raise_error(abort, 2u);
      // every tcgen05 op issued above completes before TMEM is released
      tc_commit(BAR(QK_DRAIN));
      mbar_wait(BAR(QK_DRAIN), 0, &never, kWaitLimitNs);
    } else if (warp == 4 * kGroups + 3 && lane == 0) {
      // ---------------------------------------------------------- P.V issuer
      // Issues P_t V_t in order, waits for its completion and publishes the count of
      // completed products, which the softmax groups and the epilogue wait on.
      bool ok = true;
      int n_lo = 0, n_hi = 0;
      uint32_t mw = 0;
      for (int t = 0; t < nj; ++t) {
        if ((t & 31) == 0) mw = mrow[t >> 5];
        const bool hi = (mw >> (t & 31)) & 1u;
        const int s = t & 1, g = t % kGroups, u = t / kGroups;
        int slot, use;
        ring_pos(hi, hi ? n_hi : n_lo, slot, use);
        if (!mbar_wait(BAR(P_FULL + kPRing * g + (u % kPRing)), (u / kPRing) & 1, abort, kWaitLimitNs) ||
            !mbar_wait(BAR((hi ? VH_FULL : VL_FULL) + slot), use & 1, abort, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_o = tmem + L::O_COL;
        if (hi) {
          const uint32_t vb = sb + L::OFF_VH + slot * L::VHI;
          const uint32_t a_p = tmem + L::S_COL0 + 128 * s;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_bf16_ts(d_o, a_p + 8 * k, smem_desc(vb + (k >> 2) * (D * 128) + (k & 3) * 32, 16, 1024, SWZ_128B),
                        idesc_bf16(D), (t > 0 || k > 0) ? 1u : 0u);
          tc_commit(BAR(VH_EMPTY + slot));
          ++n_hi;
        } else {
          const uint32_t vb = sb + L::OFF_VL + slot * L::VLO;
          const uint32_t a_p = tmem + L::P_COL + 32 * (t % 3);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_e4m3_ts(d_o, a_p + 8 * k, smem_desc(vb + k * 32, 16, 1024, SWZ_128B), idesc_e4m3(D),
                        (t > 0 || k > 0) ? 1u : 0u);
          tc_commit(BAR(VL_EMPTY + slot));
          ++n_lo;
        }
        tc_commit(BAR(PVC + (t & 7)));
      }
      if (!ok) raise_error(abort, 2u);
      tc_commit(BAR(PV_DRAIN));
      mbar_wait(BAR(PV_DRAIN), 0, &never, kWaitLimitNs);
    }
  } else {
    regs_inc<kSoftmaxRegs>();
    // ------------------------------------------------------------ softmax
    // Three groups of four warps: group wg takes the key tiles j = wg, wg+3, ... (S
    // buffer j % 2) and each thread owns one query row (= TMEM lane).  The exact
    // running maximum is the only sequential state across tiles: group wg writes
    // m_j per row to shared memory and signals the group of tile j+1 (mbarrier) as
    // soon as it is known, so one group's exponentials overlap the other groups'
    // loads, maxima, stores and O rescales.  Each group keeps its own partial row
    // sum relative to the maximum of its own last tile; all are combined at the end.
    const int q4 = warp & 3, wg = warp >> 2;
    const int r = q4 * 32 + lane;  // query row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const int row_g = i * 128 + r;
    float* mbuf = reinterpret_cast<float*>(smem + L::OFF_XCH);  // [groups][128 rows] running max
    const int wprev = (wg + kGroups - 1) % kGroups;  // the group of tile j-1
    const uint32_t mx_out = BAR(MX + wg * 4 + q4), mx_in = BAR(MX + wprev * 4 + q4);
    const float sc_hi = p.scale_log2;
    const float sc_lo = p.scale_log2 * (p.q_gs[bhq] * p.k_gs[bhk]);
    const uint32_t p_base = tmem + lane_base + L::P_COL;
    float l = 0.0f, m_ref = -INFINITY;
    bool ok = true;
    uint32_t mw = 0;
    for (int j = wg; j < nj; j += kGroups) {
      const int u = j / kGroups;  // this group's tile count
      const int sbuf = j & 1;     // S buffer of tile j
      mw = mrow[j >> 5];
      const bool hi = (mw >> (j & 31)) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(BAR(S_FULL + (j & 3)), (j >> 2) & 1, abort, kWaitLimitNs))) {
        raise_error(abort, 4u);
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[128];
      const uint32_t s_addr = tmem + lane_base + L::S_COL0 + 128 * sbuf;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(s_addr + 32 * c4, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c4]));
      tmem_ld_wait();
      // S is in registers: its TMEM buffer may take S_{j+2}
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(S_FREE + sbuf));
      if ((p.causal && j == i) || ((j + 1) * 128 > p.N)) {  // warp-uniform: only edge tiles mask
        const int lim = min(p.causal ? row_g + 1 : p.N, p.N) - j * 128;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= lim) v[c] = __float_as_uint(-INFINITY);
      }
      // row max of the raw logits: a tree of three-input maxima
      float mloc;
      {
        float t1[43];
#pragma unroll
        for (int c = 0; c < 42; ++c)
          t1[c] = fmax3(__uint_as_float(v[3 * c]), __uint_as_float(v[3 * c + 1]), __uint_as_float(v[3 * c + 2]));
        t1[42] = fmaxf(__uint_as_float(v[126]), __uint_as_float(v[127]));
        float t2[15];
#pragma unroll
        for (int c = 0; c < 14; ++c) t2[c] = fmax3(t1[3 * c], t1[3 * c + 1], t1[3 * c + 2]);
        t2[14] = t1[42];
        float t3[5];
#pragma unroll
        for (int c = 0; c < 5; ++c) t3[c] = fmax3(t2[3 * c], t2[3 * c + 1], t2[3 * c + 2]);
        mloc = fmaxf(fmax3(t3[0], t3[1], t3[2]), fmaxf(t3[3], t3[4]));
      }
      const float sc = hi ? sc_hi : sc_lo;
      float m_prev = -INFINITY;
      if (j > 0) {
        // m_{j-1} from the warp of the same quarter in the group of tile j-1
        if (!__all_sync(0xffffffffu, mbar_wait(mx_in, ((j - 1) / kGroups) & 1, abort, kWaitLimitNs))) {
          raise_error(abort, 4u);
          ok = false;
          break;
        }
        m_prev = mbuf[wprev * 128 + r];
      }
      const float m_new = fmaxf(m_prev, mloc * sc);
      mbuf[wg * 128 + r] = m_new;
      __syncwarp();
      if (j + 1 < nj && lane == 0) mbar_arrive(mx_out);
      const float alpha = (m_prev == -INFINITY) ? 0.0f : ex2_approx(m_prev - m_new);  // O rescale
      const float beta = (m_ref == -INFINITY) ? 0.0f : ex2_approx(m_ref - m_new);     // own partial sum
      const uint64_t sc2 = f2pack(sc, sc);
      const uint64_t nb2 = f2pack(8.0f - m_new, 8.0f - m_new);  // p * 2^8 = 2^(s*sc - m_new + 8)
      uint64_t acc[4] = {0, 0, 0, 0};
      if (!hi && j >= 3) {
        // P region j % 3 (this group's own) was last read by P_{j-3} V_{j-3}, issued a
        // whole round of tiles ago: wait until it completed
        if (!__all_sync(0xffffffffu, pv_wait(j - 3))) {
          raise_error(abort, 4u);
          ok = false;
          break;
        }
        tc_fence_after();
      }
      // per chunk of 32 columns: exponentials in place (v[c] becomes p * 2^8 in FP32),
      // then P in the tile's own precision only
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
#pragma unroll
        for (int t = 16 * ch; t < 16 * ch + 16; ++t) {
          const uint64_t y2 = ffma2(f2pack(__uint_as_float(v[2 * t]), __uint_as_float(v[2 * t + 1])), sc2, nb2);
          float a0, a1;
          f2unpack(y2, a0, a1);
          const uint64_t e2 = f2pack(ex2_approx(a0), ex2_approx(a1));
          acc[t & 3] = fadd2(acc[t & 3], e2);
          float e0, e1;
          f2unpack(e2, e0, e1);
          v[2 * t] = __float_as_uint(e0);
          v[2 * t + 1] = __float_as_uint(e1);
        }
        if (hi) {
          // BF16 P overwrites the leading 64 columns of this tile's own S buffer (already read)
          uint32_t pb[16];
#pragma unroll
          for (int t = 0; t < 16; ++t)
            pb[t] = cvt_bf16x2(__uint_as_float(v[32 * ch + 2 * t]), __uint_as_float(v[32 * ch + 2 * t + 1]));
          tmem_st16(s_addr + 16 * ch, pb);
        } else {
          uint32_t pe[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int c = 32 * ch + 4 * t;
            pe[t] = __byte_perm(cvt_e4m3x2(__uint_as_float(v[c]), __uint_as_float(v[c + 1])),
                                cvt_e4m3x2(__uint_as_float(v[c + 2]), __uint_as_float(v[c + 3])), 0x5410);
          }
          tmem_st8(p_base + 32 * (j % 3) + 8 * ch, pe);
        }
      }
      float r0, r1, r2, r3, r4, r5, r6, r7;
      f2unpack(acc[0], r0, r1);
      f2unpack(acc[1], r2, r3);
      f2unpack(acc[2], r4, r5);
      f2unpack(acc[3], r6, r7);
      l = l * beta + (((r0 + r1) + (r2 + r3)) + ((r4 + r5) + (r6 + r7)));
      m_ref = m_new;
      // rescale O when any row of the warp has a new maximum (alpha == 1 is a no-op)
      if (__any_sync(0xffffffffu, (j > 0) && (alpha != 1.0f))) {
        if (!__all_sync(0xffffffffu, pv_wait(j - 1))) {
          raise_error(abort, 4u);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t al2 = f2pack(alpha, alpha);
        // the whole O row in one TMEM round trip: v (P is stored) holds it
        const uint32_t o_addr = tmem + lane_base + L::O_COL;
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) tmem_ld32(o_addr + 32 * c4, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c4]));
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < D; c += 2) {
          float a0, a1;
          f2unpack(fmul2(f2pack(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), al2), a0, a1);
          v[c] = __float_as_uint(a0);
          v[c + 1] = __float_as_uint(a1);
        }
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) tmem_st32(o_addr + 32 * c4, *reinterpret_cast<const uint32_t(*)[32]>(&v[32 * c4]));
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(P_FULL + kPRing * wg + (u % kPRing)));
    }
    // ---------------------------------------------------------- epilogue
    // combine the groups' partial row sums; groups 0 and 1 write D/2 columns each
    ok = ok && __all_sync(0xffffffffu, pv_wait(nj - 1));
    float* xl = reinterpret_cast<float*>(smem + L::OFF_FIN);  // sums [groups][128], maxima [groups][128]
    xl[wg * 128 + r] = l;
    xl[128 * kGroups + wg * 128 + r] = m_ref;
    named_bar_sync(1 + q4, 32 * kGroups);
    if (ok) {
      tc_fence_after();
      float m_fin = -INFINITY;
#pragma unroll
      for (int g = 0; g < kGroups; ++g) m_fin = fmaxf(m_fin, xl[128 * kGroups + g * 128 + r]);
      float lt = 0.0f;
#pragma unroll
      for (int g = 0; g < kGroups; ++g) {
        const float mg = xl[128 * kGroups + g * 128 + r];
        if (mg != -INFINITY) lt += xl[g * 128 + r] * ex2_approx(mg - m_fin);
      }
      const float inv_l = 1.0f / lt;
      if (wg < 2) {
        __nv_bfloat16* orow = p.o + ((size_t)bhq * p.N + row_g) * D + (D / 2) * wg;
#pragma unroll
        for (int c4 = 0; c4 < D / 64; ++c4) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_base + L::O_COL + (D / 2) * wg + 32 * c4, ov);
          tmem_ld_wait();
          uint32_t packed[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const int cc = (D / 2) * wg + c4 * 32 + c;
            const float a0 = __uint_as_float(ov[c]) * (vsc[cc] * inv_l);
            const float a1 = __uint_as_float(ov[c + 1]) * (vsc[cc + 1] * inv_l);
            packed[c >> 1] = cvt_bf16x2(a0, a1);
          }
          if (row_g < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c4 * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
          }
        }
      }
      if (wg == 0 && p.lse != nullptr && row_g < p.N)
        p.lse[(size_t)bhq * p.N + row_g] = (m_fin - 8.0f) * 0.69314718055994531f + logf(lt);
    } else {
      raise_error(abort, 4u);
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 4 * kGroups + 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if ((warp == 4 * kGroups || warp == 4 * kGroups + 2) && lane == 0 && *abort) {
    // every role has returned and the abort flag is final: let the copies this
    // producer issued land before the CTA's shared memory goes away (a copy that
    // was never issued times out here after a quarter of the wait limit)
    const bool kside = (warp == 4 * kGroups);
    if (kside) mbar_wait(BAR(Q_FULL), 0, &never, kWaitLimitNs / 4);
    for (int k = 0; k < NLO && k < issued_lo; ++k) {
      const int n = issued_lo - 1 - k, slot = n % NLO;
      mbar_wait(BAR((kside ? KL_FULL : VL_FULL) + slot), (n / NLO) & 1, &never, kWaitLimitNs / 4);
    }
    for (int k = 0; k < NHI && k < issued_hi; ++k) {
      const int n = issued_hi - 1 - k, slot = n % NHI;
      mbar_wait(BAR((kside ? KH_FULL : VH_FULL) + slot), (n / NHI) & 1, &never, kWaitLimitNs / 4);
    }
  }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch.
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

static bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
                     uint64_t d2, uint64_t s1_bytes, uint64_t s2_bytes, uint32_t b0, uint32_t b1,
                     CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1_bytes, s2_bytes};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool MXFP4>
static int launch_d(const AttnArgs& a, cudaStream_t st) {
  using L = Layout<D>;
  const int T = (a.N + 127) / 128, W = (T + 31) / 32;
  const uint64_t N = (uint64_t)a.N, Np = (uint64_t)T * 128;
  const uint64_t BHq = (uint64_t)a.B * a.Hq, BHk = (uint64_t)a.B * a.Hkv;
  const thrift_quant& qz = *a.quant;
  CUtensorMap m_qfp4, m_kfp4, m_qbf, m_kbf, m_vfp8, m_vbf;
  const CUtensorMapSwizzle fp4_swz = (D == 128) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  bool ok = true;
  ok &= make_map(&m_qfp4, CU_TENSOR_MAP_DATA_TYPE_UINT8, qz.q_fp4, D / 2, N, BHq, D / 2, N * D / 2, D / 2, 128, fp4_swz);
  ok &= make_map(&m_kfp4, CU_TENSOR_MAP_DATA_TYPE_UINT8, qz.k_fp4, D / 2, N, BHk, D / 2, N * D / 2, D / 2, 128, fp4_swz);
  ok &= make_map(&m_qbf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.q, D, N, BHq, D * 2, N * D * 2, 64, 128,
                 CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&m_kbf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.k, D, N, BHk, D * 2, N * D * 2, 64, 128,
                 CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&m_vfp8, CU_TENSOR_MAP_DATA_TYPE_UINT8, qz.v_fp8t, Np, D, BHk, Np, Np * D, 128, D,
                 CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&m_vbf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, qz.v_st, Np, D, BHk, Np * 2, Np * D * 2, 64, D,
                 CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return THRIFT_ERR_CUDA;
  Params p;
  p.q_sf_mma = qz.q_sf_mma;
  p.k_sf_mma = qz.k_sf_mma;
  p.q_gs = qz.q_gs;
  p.k_gs = qz.k_gs;
  p.v_exp = qz.v_exp;
  p.mask = a.mask;
  p.o = reinterpret_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse;
  p.B = a.B; p.Hq = a.Hq; p.Hkv = a.Hkv; p.N = a.N; p.T = T; p.W = W; p.causal = a.causal;
  const float scale = a.softmax_scale > 0.0f ? a.softmax_scale : 1.0f / sqrtf((float)D);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.withhold_v = g_withhold_v.load(std::memory_order_relaxed);
  auto kern = attn_fwd_kernel<D, MXFP4>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::DYN) != cudaSuccess)
    return THRIFT_ERR_CUDA;
  const unsigned grid = (unsigned)(BHq * (uint64_t)T);
  kern<<<grid, kThreads, L::DYN, st>>>(m_qfp4, m_kfp4, m_qbf, m_kbf, m_vfp8, m_vbf, p);
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

}  // namespace attn

int launch_attn(const AttnArgs& a, cudaStream_t s) {
  if (a.mx) return a.d == 128 ? attn::launch_d<128, true>(a, s) : attn::launch_d<64, true>(a, s);
  return a.d == 128 ? attn::launch_d<128, false>(a, s) : attn::launch_d<64, false>(a, s);
}

cudaError_t read_and_clear_device_error(cudaStream_t s, uint32_t* word) {
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  uint32_t w = 0;
  e = cudaMemcpyFromSymbol(&w, g_attn_error_word, sizeof(w));
  if (e != cudaSuccess) return e;
  if (w != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_attn_error_word, &zero, sizeof(zero));
  }
  *word = w;
  return e;
}

}  // namespace thrift
