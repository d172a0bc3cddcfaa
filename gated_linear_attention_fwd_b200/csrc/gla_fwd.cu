// gla_fwd.cu -- chunkwise Gated Linear Attention forward on sm_100a.
//
// What is computed (DiG slides, GLA eq. (5)-(8)): for every (batch, head)
// sequence, in scan order t,
//     alpha_t = exp(inv_tau * logsigmoid(z_t)),  S_t = diag(alpha_t) S_{t-1} + k_t^T v_t,
//     o_t = q_t S_t,
// evaluated chunkwise (slides "計算効率の分析", paper "Efficiency Analysis": the
// sequence is cut into chunks that fit on-chip).  For a chunk of C tokens with
// in-chunk inclusive log-decay cumsum b_t and a reference r = b at the chunk's
// middle token,
//     qbar_t = q_t * e^{b_t - r},  kbar_s = k_s * e^{r - b_s},  khat_s = k_s * e^{Gamma - b_s}
//     P = (qbar kbar^T) masked to s <= t               (tensor core, C x C)
//     O = qbar (diag(e^r) S_in) + P V                   (tensor core)
//     S_out = diag(e^Gamma) S_in + khat^T V             (tensor core + fp32 carry)
// which equals the recurrence in exact arithmetic.  The reference point at the
// chunk middle halves the exponent range the factorisation needs; a chunk whose
// |b - r| exceeds 80 in some channel is flagged (DIG_ERR_GATE_RANGE).
//
// Work decomposition: one CTA per (sequence, segment of consecutive chunks).
// With more than one segment per sequence the CTA first sweeps its chunks to
// form the segment's (summed decay, state) record, publishes it, combines the
// records of the earlier segments (they are all resident: cooperative launch),
// and then sweeps again producing outputs.  The second sweep re-reads k, v, z;
// those re-reads are meant to hit L2.
//
// Data movement: each of the 256 threads owns one token row (t = tid % 128)
// and one half of the channels; it gathers its row directly from the
// grid-ordered tensors at pi(t) (the SREM scan order is fused into the load, no
// permuted copy exists), converts to fp32, applies the gate factors and writes
// the operands in the tensor core's canonical K-major layout.  Accumulators
// live in TMEM; token row t is TMEM lane t.
//
// Operand precision: the gated operands (qbar, kbar, khat, P, the state) are not
// representable in bf16, so each is stored as a sum of bf16 terms (hi + lo, or
// hi + mid + lo for fp32 inputs) and every product is issued as the pairs of
// terms whose combined order matters (kind::f16 MMAs, fp32 accumulation).  Two
// terms carry ~16 significant bits (relative error ~2^-17 per product), far
// below the bf16-input tolerance; three terms reach fp32 accuracy.  Raw bf16
// inputs (v) are exact in one term.
#include <type_traits>

#include "gla.h"
#include "gla_common.cuh"

namespace dig {

template <int C_, int NTG_, int NTV_, int DK_, int DV_>
struct FwdCfg {
  static constexpr int C = C_, NTG = NTG_, NTV = NTV_, DK = DK_, DV = DV_;
  static constexpr int DKP = cround(DK, 16), DVP = cround(DV, 16);
  // per-thread channel halves (multiples of 4 so rows stay 8/16-byte aligned)
  static constexpr int DK0 = cround((DK + 1) / 2, 4), DK1 = DK - DK0;
  static constexpr int DV0 = cround((DV + 1) / 2, 8), DV1 = DV - DV0;
  static constexpr int DKH = cmax(DK0, DK1), DVH = cmax(DV0, DV1);
  // K-major bf16 strides (bytes).  Buffers whose K dimension is the token axis
  // are written column-wise (one token per thread): LBO = 144 spreads a warp's
  // column writes over all banks.  Row buffers pad SBO by 64 bytes so that the
  // four 8-row groups a warp writes fall on alternating bank halves.
  static constexpr int LBO_T = 144, SBO_T = (C / 8) * LBO_T;
  static constexpr int SBO_K = DKP * 16 + 64;  // rows of DKP values
  static constexpr int SBO_P = C * 16 + 64;    // rows of C values
  static constexpr int VT_SZ = (DVP / 8) * SBO_T;
  static constexpr int KHT_SZ = (DKP / 8) * SBO_T;
  static constexpr int AQ_SZ = (C / 8) * SBO_K;
  static constexpr int BK_SZ = (C / 8) * SBO_K;
  static constexpr int SPT_SZ = (DVP / 8) * SBO_K;
  static constexpr int P_SZ = (C / 8) * SBO_P;
  static constexpr int OFF_VT = 0;
  static constexpr int OFF_AQ = OFF_VT + NTV * VT_SZ;
  static constexpr int OFF_BK = OFF_AQ + NTG * AQ_SZ;
  static constexpr int OFF_KHT = OFF_BK + NTG * BK_SZ;
  static constexpr int OFF_SPT = OFF_KHT + NTG * KHT_SZ;
  static constexpr int OFF_P = OFF_AQ;  // P reuses the first-stage operand space
  static constexpr int END_DATA = OFF_SPT + NTG * SPT_SZ;
  // M = 128 MMAs read 16 row groups of an A operand even when fewer rows are
  // real; those reads must stay inside the allocation (their rows are ignored).
  static constexpr int END_VT = OFF_VT + (NTV - 1) * VT_SZ + 16 * SBO_T;
  static constexpr int END_AQ = OFF_AQ + (NTG - 1) * AQ_SZ + 16 * SBO_K;
  static constexpr int END_P = OFF_P + (NTG - 1) * P_SZ + 16 * SBO_P;
  static constexpr int SMEM = cmax(cmax(END_DATA, END_VT), cmax(END_AQ, END_P));
  // TMEM columns
  static constexpr int TM_P = 0, TM_O = C, TM_DS = C + DVP;
  static constexpr int TM_COLS = pow2ceil(C + DVP + DKP);
  static_assert(TM_COLS <= 512, "TMEM budget");
  static_assert(SMEM <= 200 * 1024, "shared-memory budget");
  static_assert(DK % 4 == 0 && DV % 4 == 0 && DK1 > 0 && DV1 > 0, "head dims");
  static_assert(C == 64 || C == 128, "chunk");
};

struct FwdSmem {
  float wtot[8][32];  // per-warp totals of the log2 decay, per channel of the warp's half
  float red[256];     // epilogue row sums of squares
  uint64_t bar;       // MMA completion barrier
  uint32_t tmem;      // TMEM base address
  int range_bad;
};

// The per-thread program.
template <int C, int DK, int DV, typename TIN, typename TOUT, int H>
__device__ __forceinline__ void fwd_thread(const GlaArgs& a, uint8_t* smem, FwdSmem& sh) {
  constexpr int NTG = std::is_same<TIN, float>::value ? 3 : 2;
  constexpr int NTV = std::is_same<TIN, float>::value ? 3 : 1;
  using Cfg = FwdCfg<C, NTG, NTV, DK, DV>;
  constexpr int DKP = Cfg::DKP, DVP = Cfg::DVP;
  constexpr int KO = H ? Cfg::DK0 : 0, KN = H ? Cfg::DK1 : Cfg::DK0;
  constexpr int VO = H ? Cfg::DV0 : 0, VN = H ? Cfg::DV1 : Cfg::DV0;
  static_assert(KN <= 32 && KN % 4 == 0 && VN % 4 == 0, "channel split");
  using RT = typename Raw4<TIN>::type;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = tid & 127, wq = warp & 3;
  const int nseq = a.B * a.H;
  const int bh = blockIdx.x % nseq, seg = blockIdx.x / nseq;
  const int b = bh / a.H, h = bh % a.H;
  const int hz = a.gate_heads == 1 ? 0 : h;
  const int c_begin = (int)((long long)seg * a.nchunks / a.nseg);
  const int c_end = (int)((long long)(seg + 1) * a.nchunks / a.nseg);
  const bool tok = t < C;
  const bool state_thr = t < DV;
  const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
  const uint32_t tmem = sh.tmem;
  const uint32_t sbase = smem_u32(smem);
  uint32_t phase = 0;
  bool timed_out = false;

  float S[KN];     // state S[KO + i][t]
  float Gacc[KN];  // summed log2 decay of this segment (first sweep)
#pragma unroll
  for (int i = 0; i < KN; ++i) S[i] = 0.f, Gacc[i] = 0.f;

  // prefetched rows of the next chunk
  RT rq[KN / 4], rk[KN / 4], rvv[VN / 4];
  float4 rz[KN / 4];
  bool valid = false;
  long long grow = 0;
  auto fetch = [&](int n, bool with_q) {
    const int p = n * C + t;
    valid = tok && n < c_end && p < a.L;
    grow = valid ? (long long)b * a.L + scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode) : 0;
    const size_t rk_off = ((size_t)grow * a.H + h) * DK + KO;
    const RT* kp = reinterpret_cast<const RT*>(reinterpret_cast<const TIN*>(a.k) + rk_off);
    const RT* qp = reinterpret_cast<const RT*>(reinterpret_cast<const TIN*>(a.q) + rk_off);
    const RT* vp = reinterpret_cast<const RT*>(reinterpret_cast<const TIN*>(a.v) + ((size_t)grow * a.H + h) * DV + VO);
    const float4* zp = reinterpret_cast<const float4*>(a.z + ((size_t)grow * a.gate_heads + hz) * DK + KO);
#pragma unroll
    for (int g = 0; g < KN / 4; ++g) {
      rk[g] = valid ? __ldg(kp + g) : zero4<RT>();
      rq[g] = (valid && with_q) ? __ldg(qp + g) : zero4<RT>();
      rz[g] = valid ? __ldg(zp + g) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int g = 0; g < VN / 4; ++g) rvv[g] = valid ? __ldg(vp + g) : zero4<RT>();
  };

  // base descriptors of every operand (term 0, K-step 0)
  const uint64_t dAQ = sdesc(sbase + Cfg::OFF_AQ, 128, Cfg::SBO_K);
  const uint64_t dBK = sdesc(sbase + Cfg::OFF_BK, 128, Cfg::SBO_K);
  const uint64_t dSPT = sdesc(sbase + Cfg::OFF_SPT, 128, Cfg::SBO_K);
  const uint64_t dVT = sdesc(sbase + Cfg::OFF_VT, Cfg::LBO_T, Cfg::SBO_T);
  const uint64_t dKHT = sdesc(sbase + Cfg::OFF_KHT, Cfg::LBO_T, Cfg::SBO_T);
  const uint64_t dP = sdesc(sbase + Cfg::OFF_P, 128, Cfg::SBO_P);
  auto wait_mma = [&]() {
    if (!mbar_wait(&sh.bar, phase, kSpinLimitNs)) timed_out = true;
    phase ^= 1u;
    tc_fence_after();
  };

  // One chunk.  OUT = false: state sweep only (segment record); OUT = true: outputs.
  auto chunk = [&](auto out_tag, int n, int next_n, bool next_out) {
    constexpr bool OUT = decltype(out_tag)::value;
    const bool my_valid = valid;
    const long long my_row = grow;
    // gate: base-2 log decay and its inclusive cumsum over the chunk's tokens
    float b2[KN];
#pragma unroll
    for (int g = 0; g < KN / 4; ++g) {
      float zz[4];
      unpack4(rz[g], zz);
#pragma unroll
      for (int u = 0; u < 4; ++u) b2[4 * g + u] = my_valid ? log2_decay(zz[u], a.inv_tau) : 0.f;
    }
#pragma unroll
    for (int i = 0; i < KN; ++i) {
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, b2[i], off);
        if (lane >= off) b2[i] += y;
      }
    }
    if (lane == 31) {
#pragma unroll
      for (int i = 0; i < KN; ++i) sh.wtot[warp][i] = b2[i];
    }
    __syncthreads();
    float r2[KN], g2[KN];
    constexpr int REFW = C / 64;  // warps before the reference token C/2 - 1
#pragma unroll
    for (int i = 0; i < KN; ++i) {
      float pre = 0.f, tot = 0.f, ref = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float w = sh.wtot[H * 4 + u][i];
        pre += (u < wq) ? w : 0.f;
        ref += (u < REFW) ? w : 0.f;
        tot += w;
      }
      b2[i] += pre;
      r2[i] = ref;
      g2[i] = tot;
    }
    // operands
    bool bad = false;
    if (tok) {
      float kv[KN], qv[KN];
#pragma unroll
      for (int g = 0; g < KN / 4; ++g) {
        unpack4(rk[g], kv + 4 * g);
        unpack4(rq[g], qv + 4 * g);
      }
#pragma unroll
      for (int i = 0; i < KN; ++i) {
        const float d = b2[i] - r2[i];
        bad |= fabsf(d) > 115.f;  // |b - r| > 80 in natural-log units
        st_op<NTG>(smem + Cfg::OFF_KHT, Cfg::KHT_SZ, kmaj16(KO + i, t, Cfg::LBO_T, Cfg::SBO_T),
                   kv[i] * exp2f(g2[i] - b2[i]));
        if (OUT) {
          qv[i] *= exp2f(d);
          kv[i] *= exp2f(-d);
        }
      }
#pragma unroll
      for (int g = 0; g < VN / 4; ++g) {
        float vv[4];
        unpack4(rvv[g], vv);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          st_op<NTV>(smem + Cfg::OFF_VT, Cfg::VT_SZ, kmaj16(VO + 4 * g + u, t, Cfg::LBO_T, Cfg::SBO_T), vv[u]);
      }
      if (OUT) {
#pragma unroll
        for (int g = 0; g < KN / 4; ++g) {
          const uint32_t off = kmaj16(t, KO + 4 * g, 128, Cfg::SBO_K);
          st_op4<NTG>(smem + Cfg::OFF_AQ, Cfg::AQ_SZ, off, qv[4 * g], qv[4 * g + 1], qv[4 * g + 2], qv[4 * g + 3]);
          st_op4<NTG>(smem + Cfg::OFF_BK, Cfg::BK_SZ, off, kv[4 * g], kv[4 * g + 1], kv[4 * g + 2], kv[4 * g + 3]);
        }
        if (H == 1) {
#pragma unroll
          for (int c = DK; c < DKP; c += 4) {
            const uint32_t off = kmaj16(t, c, 128, Cfg::SBO_K);
            st_op4<NTG>(smem + Cfg::OFF_AQ, Cfg::AQ_SZ, off, 0.f, 0.f, 0.f, 0.f);
            st_op4<NTG>(smem + Cfg::OFF_BK, Cfg::BK_SZ, off, 0.f, 0.f, 0.f, 0.f);
          }
        }
      }
    }
    if (OUT && state_thr) {
      // B operand of O += qbar S': row j = t of S'^T, S' = diag(2^{r2}) S_in
#pragma unroll
      for (int g = 0; g < KN / 4; ++g) {
        float e[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) e[u] = exp2f(r2[4 * g + u]) * S[4 * g + u];
        st_op4<NTG>(smem + Cfg::OFF_SPT, Cfg::SPT_SZ, kmaj16(t, KO + 4 * g, 128, Cfg::SBO_K), e[0], e[1], e[2], e[3]);
      }
      if (H == 1) {
#pragma unroll
        for (int c = DK; c < DKP; c += 4)
          st_op4<NTG>(smem + Cfg::OFF_SPT, Cfg::SPT_SZ, kmaj16(t, c, 128, Cfg::SBO_K), 0.f, 0.f, 0.f, 0.f);
      }
    }
    if (bad) sh.range_bad = 1;
    // the next chunk's rows are fetched while this chunk's MMAs run
    fetch(next_n, next_out);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      if (OUT) {
        mma_issue<NTG, NTG, DKP / 16>(tmem + Cfg::TM_P, dAQ, Cfg::AQ_SZ, 256, dBK, Cfg::BK_SZ, 256,
                                      idesc_bf16(128, C), false);
        mma_issue<NTG, NTG, DKP / 16>(tmem + Cfg::TM_O, dAQ, Cfg::AQ_SZ, 256, dSPT, Cfg::SPT_SZ, 256,
                                      idesc_bf16(128, DVP), false);
      }
      mma_issue<NTV, NTG, C / 16>(tmem + Cfg::TM_DS, dVT, Cfg::VT_SZ, 2 * Cfg::LBO_T, dKHT, Cfg::KHT_SZ,
                                  2 * Cfg::LBO_T, idesc_bf16(128, DKP), false);
      mma_commit(&sh.bar);
    }
    wait_mma();
    // state carry: S <- diag(2^{g2}) S + khat^T V   (TMEM lane j holds row j of (khat^T V)^T)
    {
      float ds[cround(KN, 8)];
#pragma unroll
      for (int c = 0; c < cround(KN, 8); c += 8) tmem_ld8(tmem + lane_base + Cfg::TM_DS + KO + c, ds + c);
      tmem_ld_wait();
      if (state_thr) {
#pragma unroll
        for (int i = 0; i < KN; ++i) S[i] = exp2f(g2[i]) * S[i] + ds[i];
      }
      if (!OUT) {
#pragma unroll
        for (int i = 0; i < KN; ++i) Gacc[i] += g2[i];
      }
    }
    if (OUT) {
      // P row t: keep s <= t, store as the A operand of P V
#pragma unroll
      for (int cb = 0; cb < C / 2; cb += 16) {
        float pv[16];
        tmem_ld16(tmem + lane_base + Cfg::TM_P + H * (C / 2) + cb, pv);
        tmem_ld_wait();
        if (tok) {
          const int s0 = H * (C / 2) + cb;
#pragma unroll
          for (int u = 0; u < 16; u += 4) {
            float x[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) x[w] = (s0 + u + w <= t) ? pv[u + w] : 0.f;
            st_op4<NTG>(smem + Cfg::OFF_P, Cfg::P_SZ, kmaj16(t, s0 + u, 128, Cfg::SBO_P), x[0], x[1], x[2], x[3]);
          }
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (tid == 0) {
        mma_issue<NTG, NTV, C / 16>(tmem + Cfg::TM_O, dP, Cfg::P_SZ, 256, dVT, Cfg::VT_SZ, 2 * Cfg::LBO_T,
                                    idesc_bf16(128, DVP), true);
        mma_commit(&sh.bar);
      }
      wait_mma();
      float ov[cround(VN, 8)];
#pragma unroll
      for (int c = 0; c < cround(VN, 8); c += 8) tmem_ld8(tmem + lane_base + Cfg::TM_O + VO + c, ov + c);
      tmem_ld_wait();
      const size_t ro = ((size_t)my_row * a.H + h) * DV + VO;
      if (my_valid) store_row<VN>(reinterpret_cast<TOUT*>(a.o) + ro, ov);
      if (a.y != nullptr && a.r != nullptr) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < VN; ++i) ss += ov[i] * ov[i];
        sh.red[tid] = my_valid ? ss : 0.f;
        __syncthreads();
        const float inv = rsqrtf((sh.red[t] + sh.red[t + 128]) / (float)DV + a.eps);
        if (my_valid) {
          float rr[VN], yv[VN];
          load_row<VN>(reinterpret_cast<const TIN*>(a.r) + ro, rr);
#pragma unroll
          for (int i = 0; i < VN; ++i) {
            const float gmm = a.gamma != nullptr ? __ldg(a.gamma + VO + i) : 1.f;
            const float sw = rr[i] / (1.f + exp2f(-rr[i] * kLog2e));
            yv[i] = sw * ov[i] * inv * gmm;
          }
          store_row<VN>(reinterpret_cast<TOUT*>(a.y) + ro, yv);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  };

  // ---------------------------------------------------------------- sweep 1
  const int rec = bh * a.nseg + seg;
  if (a.nseg > 1) {
    fetch(c_begin, false);
    for (int n = c_begin; n < c_end; ++n) {
      const bool last = n + 1 == c_end;
      chunk(std::false_type{}, n, last ? c_begin : n + 1, last);
    }
    if (state_thr) {
      float* dst = a.seg_S + ((size_t)rec * DV + t) * DK + KO;
#pragma unroll
      for (int i = 0; i < KN; ++i) dst[i] = S[i];
    }
    if (t == 0) {
#pragma unroll
      for (int i = 0; i < KN; ++i) a.seg_gam[(size_t)rec * DKP + KO + i] = Gacc[i];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) st_release(a.flags + rec, 1u);
    // combine the records of all earlier segments of this sequence
#pragma unroll
    for (int i = 0; i < KN; ++i) S[i] = 0.f;
    if (seg > 0) {
      if (tid == 0) {
        for (int s2 = 0; s2 < seg; ++s2)
          if (!wait_flag(a.flags + bh * a.nseg + s2, 1u, kSpinLimitNs)) timed_out = true;
      }
      __syncthreads();
      if (state_thr) {
        for (int s2 = 0; s2 < seg; ++s2) {
          const size_t r2 = (size_t)bh * a.nseg + s2;
          const float* src = a.seg_S + (r2 * DV + t) * DK + KO;
#pragma unroll
          for (int i = 0; i < KN; ++i) S[i] = exp2f(__ldcg(a.seg_gam + r2 * DKP + KO + i)) * S[i] + __ldcg(src + i);
        }
      }
    }
  } else {
    fetch(c_begin, true);
  }
  // ---------------------------------------------------------------- sweep 2
  for (int n = c_begin; n < c_end; ++n) chunk(std::true_type{}, n, n + 1, true);

  if (timed_out) set_status(a.status, DIG_ERR_DEVICE_TIMEOUT);
}

template <int C, int DK, int DV, typename TIN, typename TOUT>
__global__ void __launch_bounds__(256, 1) gla_fwd_kernel(const GlaArgs a) {
  constexpr int NTG = std::is_same<TIN, float>::value ? 3 : 2;
  constexpr int NTV = std::is_same<TIN, float>::value ? 3 : 1;
  using Cfg = FwdCfg<C, NTG, NTV, DK, DV>;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ FwdSmem sh;
  const int tid = threadIdx.x, warp = tid >> 5;
  if (warp == 0) {
    tmem_alloc(&sh.tmem, Cfg::TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&sh.bar, 1);
    fence_mbar_init();
    sh.range_bad = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid < 128) fwd_thread<C, DK, DV, TIN, TOUT, 0>(a, smem, sh);
  else fwd_thread<C, DK, DV, TIN, TOUT, 1>(a, smem, sh);
  // teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(sh.tmem, Cfg::TM_COLS);
  if (tid == 0 && sh.range_bad) set_status(a.status, DIG_ERR_GATE_RANGE);
  if (a.nseg > 1 && tid == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(a.done, 1u);
    if (prev == gridDim.x - 1) {  // every CTA is past its flag reads: reset for the next call
      const int n = a.B * a.H * a.nseg;
      for (int i = 0; i < n; ++i) a.flags[i] = 0u;
      *a.done = 0u;
      __threadfence();
    }
  }
}

// ------------------------------------------------------------------ launch
template <int C, int DK, int DV, typename TIN>
using FwdCfgOf = FwdCfg<C, std::is_same<TIN, float>::value ? 3 : 2, std::is_same<TIN, float>::value ? 3 : 1, DK, DV>;

template <int C, int DK, int DV, typename TIN, typename TOUT>
static cudaError_t launch_one(const GlaArgs& a, int grid, bool coop, cudaStream_t s) {
  using Cfg = FwdCfgOf<C, DK, DV, TIN>;
  auto kern = gla_fwd_kernel<C, DK, DV, TIN, TOUT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e != cudaSuccess) return e;
  if (coop) {
    GlaArgs copy = a;
    void* args[] = {&copy};
    return cudaLaunchCooperativeKernel((const void*)kern, dim3(grid), dim3(256), args, Cfg::SMEM, s);
  }
  kern<<<grid, 256, Cfg::SMEM, s>>>(a);
  return cudaGetLastError();
}

template <int C, int DK, int DV, typename TIN, typename TOUT>
static int occupancy_one() {
  using Cfg = FwdCfgOf<C, DK, DV, TIN>;
  auto kern = gla_fwd_kernel<C, DK, DV, TIN, TOUT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM) != cudaSuccess) return 0;
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, 256, Cfg::SMEM) != cudaSuccess) return 0;
  return nb;
}

template <int DK, int DV>
static cudaError_t dispatch_types(const GlaVariant& v, const GlaArgs& a, int grid, bool coop, cudaStream_t s,
                                  int* occ) {
  using bf = __nv_bfloat16;
  if (v.tin == DIG_BF16) {
    if (v.tout == DIG_BF16) return occ ? (*occ = occupancy_one<128, DK, DV, bf, bf>(), cudaSuccess)
                                       : launch_one<128, DK, DV, bf, bf>(a, grid, coop, s);
    return occ ? (*occ = occupancy_one<128, DK, DV, bf, float>(), cudaSuccess)
               : launch_one<128, DK, DV, bf, float>(a, grid, coop, s);
  }
  if (v.tout == DIG_BF16) return occ ? (*occ = occupancy_one<64, DK, DV, float, bf>(), cudaSuccess)
                                     : launch_one<64, DK, DV, float, bf>(a, grid, coop, s);
  return occ ? (*occ = occupancy_one<64, DK, DV, float, float>(), cudaSuccess)
             : launch_one<64, DK, DV, float, float>(a, grid, coop, s);
}

static cudaError_t dispatch(const GlaVariant& v, const GlaArgs& a, int grid, bool coop, cudaStream_t s, int* occ) {
  if (v.dk == 32 && v.dv == 64) return dispatch_types<32, 64>(v, a, grid, coop, s, occ);
  if (v.dk == 36 && v.dv == 72) return dispatch_types<36, 72>(v, a, grid, coop, s, occ);
  if (v.dk == 64 && v.dv == 64) return dispatch_types<64, 64>(v, a, grid, coop, s, occ);
  return cudaErrorInvalidValue;
}

bool gla_variant_built(int dk, int dv) {
  return (dk == 32 && dv == 64) || (dk == 36 && dv == 72) || (dk == 64 && dv == 64);
}

cudaError_t launch_gla_fwd(const GlaVariant& v, const GlaArgs& a, int grid, bool coop, cudaStream_t s) {
  return dispatch(v, a, grid, coop, s, nullptr);
}

int gla_fwd_blocks_per_sm(const GlaVariant& v) {
  int occ = 0;
  if (dispatch(v, GlaArgs{}, 0, false, nullptr, &occ) != cudaSuccess) return 0;
  return occ;
}

}  // namespace dig
