// gla_bwd.cu -- chunkwise Gated Linear Attention backward on sm_100a.
//
// Gradients of sum(o * dO) for the forward in gla_fwd.cu (DiG slides, GLA eq.
// (5)-(8)).  Per sequence in scan order, with dS_t = dLoss/dS_t:
//     dq_t = dO_t S_t^T,  dk_t = v_t dS_t^T,  dv_t = k_t dS_t,
//     dlog(alpha_t) = sum_{t' >= t} (q_t' * dq_t' - k_t' * dk_t')     (reverse cumsum)
// Chunkwise, with the same chunk quantities as the forward (b = in-chunk
// inclusive log decay, r = b at the chunk middle, Gamma = chunk total):
//     qbar = q e^{b-r}, kbar = k e^{r-b}, khat = k e^{Gamma-b},
//     P = (qbar kbar^T) masked s <= t,  Dp = (dO V^T) masked s <= t,
//     S' = diag(e^r) S_in,  dH' = diag(e^{Gamma-r}) dH_out   (dH_out: gradient of the
//     state leaving the chunk, from later tokens)
//     dq = [dO S'^T + Dp kbar] * e^{b-r}
//     dk = [Dp^T qbar + V dH'^T] * e^{r-b}
//     dv =  P^T dO + khat dH_out
//     dH_in = diag(e^Gamma) dH_out + diag(e^r) qbar^T dO
// All products run on the tensor core (kind::f16, split-term bf16 operands as in
// the forward; M = 128 MMAs over 64-token chunks, the rows past the chunk are
// ignored).
//
// Decomposition: one CTA per (sequence, segment of chunks), all CTAs resident
// (cooperative launch).  Pass A sweeps the segment forward, storing the
// in-segment state entering each chunk (workspace) and accumulating the
// segment's state-gradient record sum_t diag(e^{decay from segment start to t})
// q_t^T dO_t on the tensor core; the segment publishes (decay, state, gradient)
// records, and every CTA folds the records of the earlier segments (state
// entering) and of the later segments (gradient leaving).  Pass B sweeps the
// chunks backward.  The reverse cumsum of dlog(alpha) starts at the segment end
// from rowsum(dH_out * S_out), which equals the sum of the later tokens' terms.
#include "gla.h"
#include "gla_common.cuh"

namespace dig {

template <int C_, int NTG_, int NTV_, int DK_, int DV_>
struct BwdCfg {
  static constexpr int C = C_, NTG = NTG_, NTV = NTV_, DK = DK_, DV = DV_;
  static constexpr int DKP = cround(DK, 16), DVP = cround(DV, 16);
  static constexpr int DK0 = cround((DK + 1) / 2, 4), DK1 = DK - DK0;
  static constexpr int DV0 = cround((DV + 1) / 2, 8), DV1 = DV - DV0;
  static constexpr int KNMAX = cmax(DK0, DK1), VNMAX = cmax(DV0, DV1);
  // K-major bf16 strides.  "T" buffers have the token axis as K and are written
  // one column (token) per thread; "J" buffers have the value axis as K and are
  // written one column (value row j) per state thread.
  static constexpr int LBO_T = 144, SBO_T = (C / 8) * LBO_T;
  static constexpr int SBO_J = (DVP / 8) * 144;
  static constexpr int SBO_RK = DKP * 16 + 64;  // rows of DKP values
  static constexpr int SBO_RV = DVP * 16 + 64;  // rows of DVP values
  static constexpr int SBO_RC = C * 16 + 64;    // rows of C values
  // one-copy sizes
  static constexpr int AQ_SZ = (C / 8) * SBO_RK, BK_SZ = AQ_SZ, KH_SZ = AQ_SZ;
  static constexpr int DO_SZ = (C / 8) * SBO_RV, VR_SZ = DO_SZ;
  static constexpr int QT_SZ = (DKP / 8) * SBO_T, KT_SZ = QT_SZ, DOT_SZ = (DVP / 8) * SBO_T;
  static constexpr int SP_SZ = (DKP / 8) * SBO_J, DHP_SZ = SP_SZ;
  static constexpr int DHT_SZ = (DVP / 8) * SBO_RK;
  static constexpr int DP_SZ = (C / 8) * SBO_RC;
  static constexpr int PT_SZ = (C / 8) * SBO_T, DPT_SZ = PT_SZ;
  // pass B layout: first-batch-only operands (AQ, BK) share space with the
  // second-batch operands (DP, DPT, PT); everything else follows.
  static constexpr int R1 = NTG * (AQ_SZ + BK_SZ);
  static constexpr int R3 = NTG * (DP_SZ + DPT_SZ + PT_SZ);
  static constexpr int OFF_AQ = 0, OFF_BK = OFF_AQ + NTG * AQ_SZ;
  static constexpr int OFF_DP = 0, OFF_DPT = OFF_DP + NTG * DP_SZ, OFF_PT = OFF_DPT + NTG * DPT_SZ;
  static constexpr int R2 = cmax(R1, R3);
  static constexpr int OFF_DO = R2;
  static constexpr int OFF_VR = OFF_DO + NTV * DO_SZ;
  static constexpr int OFF_KH = OFF_VR + NTV * VR_SZ;
  static constexpr int OFF_DOT = OFF_KH + NTG * KH_SZ;
  static constexpr int OFF_QT = OFF_DOT + NTV * DOT_SZ;
  static constexpr int OFF_KT = OFF_QT + NTG * QT_SZ;
  static constexpr int OFF_SP = OFF_KT + NTG * KT_SZ;
  static constexpr int OFF_DHP = OFF_SP + NTG * SP_SZ;
  static constexpr int OFF_DHT = OFF_DHP + NTG * DHP_SZ;
  static constexpr int END_B = OFF_DHT + NTG * DHT_SZ;
  // pass A layout (a separate phase; overlaps pass B's space)
  static constexpr int VT_SZ = (DVP / 8) * SBO_T, KHT_SZ = (DKP / 8) * SBO_T;
  static constexpr int OFF_VT = 0, OFF_KHT = OFF_VT + NTV * VT_SZ, OFF_QTT = OFF_KHT + NTG * KHT_SZ;
  static constexpr int OFF_ADOT = OFF_QTT + NTG * KHT_SZ;
  static constexpr int END_A = OFF_ADOT + NTV * DOT_SZ;
  // M = 128 reads of A operands run 16 row groups past each copy's start
  static constexpr int W_AQ = OFF_AQ + (NTG - 1) * AQ_SZ + 16 * SBO_RK;
  static constexpr int W_DO = OFF_DO + (NTV - 1) * DO_SZ + 16 * SBO_RV;
  static constexpr int W_VR = OFF_VR + (NTV - 1) * VR_SZ + 16 * SBO_RV;
  static constexpr int W_KH = OFF_KH + (NTG - 1) * KH_SZ + 16 * SBO_RK;
  static constexpr int W_DOT = OFF_DOT + (NTV - 1) * DOT_SZ + 16 * SBO_T;
  static constexpr int W_DP = OFF_DP + (NTG - 1) * DP_SZ + 16 * SBO_RC;
  static constexpr int W_DPT = OFF_DPT + (NTG - 1) * DPT_SZ + 16 * SBO_T;
  static constexpr int W_PT = OFF_PT + (NTG - 1) * PT_SZ + 16 * SBO_T;
  static constexpr int W_VT = OFF_VT + (NTV - 1) * VT_SZ + 16 * SBO_T;
  static constexpr int W_ADOT = OFF_ADOT + (NTV - 1) * DOT_SZ + 16 * SBO_T;
  static constexpr int SMEM =
      cmax(cmax(cmax(END_B, END_A), cmax(W_AQ, W_DO)),
           cmax(cmax(cmax(W_VR, W_KH), cmax(W_DOT, W_DP)), cmax(cmax(W_DPT, W_PT), cmax(W_VT, W_ADOT))));
  // TMEM columns
  static constexpr int TM_P = 0, TM_DPA = C, TM_DQ = 2 * C, TM_DK = TM_DQ + DKP, TM_DV = TM_DK + DKP,
                       TM_DH = TM_DV + DVP;
  static constexpr int TM_COLS = pow2ceil(TM_DH + DKP);
  static_assert(TM_COLS <= 512, "TMEM budget");
  static_assert(SMEM <= 210 * 1024, "shared-memory budget");
  static_assert(DK % 4 == 0 && DV % 4 == 0 && DK1 > 0 && DV1 > 0, "head dims");
  static_assert(C == 32 || C == 64, "chunk");
};

struct BwdSmem {
  float wtot[8][32];   // per-warp totals (log decay, then dlog(alpha) partial sums)
  float cinit[2][32];  // rowsum(dH_out * S_out) per channel, per half
  float ref[2][32];    // reference log decay r of the current chunk
  uint64_t bar;
  uint32_t tmem;
  int range_bad;
};

template <int C, int DK, int DV, typename TIN, typename TOUT, int H>
__device__ __forceinline__ void bwd_thread(const GlaArgs& a, uint8_t* smem, BwdSmem& sh) {
  constexpr int NTG = std::is_same<TIN, float>::value ? 3 : 2;
  constexpr int NTV = std::is_same<TIN, float>::value ? 3 : 1;
  using Cfg = BwdCfg<C, NTG, NTV, DK, DV>;
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
  const bool jpad_thr = t >= DV && t < DVP;  // writes the zero K-padding of the J buffers
  const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
  const uint32_t tmem = sh.tmem;
  const uint32_t sbase = smem_u32(smem);
  uint32_t phase = 0;
  bool timed_out = false;

  // ------------------------------------------------------------ descriptors
  const uint64_t dAQ = sdesc(sbase + Cfg::OFF_AQ, 128, Cfg::SBO_RK);
  const uint64_t dBK = sdesc(sbase + Cfg::OFF_BK, 128, Cfg::SBO_RK);
  const uint64_t dKH = sdesc(sbase + Cfg::OFF_KH, 128, Cfg::SBO_RK);
  const uint64_t dDO = sdesc(sbase + Cfg::OFF_DO, 128, Cfg::SBO_RV);
  const uint64_t dVR = sdesc(sbase + Cfg::OFF_VR, 128, Cfg::SBO_RV);
  const uint64_t dDOT = sdesc(sbase + Cfg::OFF_DOT, Cfg::LBO_T, Cfg::SBO_T);
  const uint64_t dQT = sdesc(sbase + Cfg::OFF_QT, Cfg::LBO_T, Cfg::SBO_T);
  const uint64_t dKT = sdesc(sbase + Cfg::OFF_KT, Cfg::LBO_T, Cfg::SBO_T);
  const uint64_t dSP = sdesc(sbase + Cfg::OFF_SP, 144, Cfg::SBO_J);
  const uint64_t dDHP = sdesc(sbase + Cfg::OFF_DHP, 144, Cfg::SBO_J);
  const uint64_t dDHT = sdesc(sbase + Cfg::OFF_DHT, 128, Cfg::SBO_RK);
  const uint64_t dDP = sdesc(sbase + Cfg::OFF_DP, 128, Cfg::SBO_RC);
  const uint64_t dDPT = sdesc(sbase + Cfg::OFF_DPT, Cfg::LBO_T, Cfg::SBO_T);
  const uint64_t dPT = sdesc(sbase + Cfg::OFF_PT, Cfg::LBO_T, Cfg::SBO_T);
  const uint64_t dVT = sdesc(sbase + Cfg::OFF_VT, Cfg::LBO_T, Cfg::SBO_T);
  const uint64_t dKHT = sdesc(sbase + Cfg::OFF_KHT, Cfg::LBO_T, Cfg::SBO_T);
  const uint64_t dQTT = sdesc(sbase + Cfg::OFF_QTT, Cfg::LBO_T, Cfg::SBO_T);
  const uint64_t dADOT = sdesc(sbase + Cfg::OFF_ADOT, Cfg::LBO_T, Cfg::SBO_T);
  constexpr uint32_t KS_R = 256, KS_T = 2 * Cfg::LBO_T, KS_J = 288;  // bytes per K-step

  auto wait_mma = [&]() {
    if (!mbar_wait(&sh.bar, phase, kSpinLimitNs)) timed_out = true;
    phase ^= 1u;
    tc_fence_after();
  };
  auto sync_mma = [&]() {  // make this thread's smem operand writes visible, then barrier
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  };

  // ------------------------------------------------------------ prefetch
  RT rq[KN / 4], rk[KN / 4], rvv[VN / 4], rdo[VN / 4];
  float4 rz[KN / 4];
  bool valid = false;
  long long grow = 0;
  auto fetch = [&](int n) {
    const int p = n * C + t;
    valid = tok && n >= c_begin && n < c_end && p < a.L;
    grow = valid ? (long long)b * a.L + scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode) : 0;
    const size_t ok = ((size_t)grow * a.H + h) * DK + KO, ov = ((size_t)grow * a.H + h) * DV + VO;
    const RT* kp = reinterpret_cast<const RT*>(reinterpret_cast<const TIN*>(a.k) + ok);
    const RT* qp = reinterpret_cast<const RT*>(reinterpret_cast<const TIN*>(a.q) + ok);
    const RT* vp = reinterpret_cast<const RT*>(reinterpret_cast<const TIN*>(a.v) + ov);
    const RT* dp = reinterpret_cast<const RT*>(reinterpret_cast<const TIN*>(a.dO) + ov);
    const float4* zp = reinterpret_cast<const float4*>(a.z + ((size_t)grow * a.gate_heads + hz) * DK + KO);
#pragma unroll
    for (int g = 0; g < KN / 4; ++g) {
      rk[g] = valid ? __ldg(kp + g) : zero4<RT>();
      rq[g] = valid ? __ldg(qp + g) : zero4<RT>();
      rz[g] = valid ? __ldg(zp + g) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int g = 0; g < VN / 4; ++g) {
      rvv[g] = valid ? __ldg(vp + g) : zero4<RT>();
      rdo[g] = valid ? __ldg(dp + g) : zero4<RT>();
    }
  };

  // gate of the fetched chunk: b2 (in-chunk inclusive base-2 log decay), r2, g2
  auto gate = [&](float* b2, float* r2, float* g2) {
#pragma unroll
    for (int g = 0; g < KN / 4; ++g) {
      float zz[4];
      unpack4(rz[g], zz);
#pragma unroll
      for (int u = 0; u < 4; ++u) b2[4 * g + u] = valid ? log2_decay(zz[u], a.inv_tau) : 0.f;
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
#pragma unroll
    for (int i = 0; i < KN; ++i) {
      float pre = 0.f, tot = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float w = sh.wtot[H * 4 + u][i];
        pre += (u < wq) ? w : 0.f;
        tot += w;
      }
      b2[i] += pre;
      g2[i] = tot;
    }
    // reference r = inclusive decay at token C/2 - 1, broadcast through shared memory
    if (t == C / 2 - 1) {
#pragma unroll
      for (int i = 0; i < KN; ++i) sh.ref[H][i] = b2[i];
    }
    __syncthreads();  // also separates these wtot reads from the next writes
#pragma unroll
    for (int i = 0; i < KN; ++i) r2[i] = sh.ref[H][i];
  };

  // ------------------------------------------------------------ pass A
  float S[KN];     // in-segment state S[KO+i][t] (state threads)
  float Bacc[KN];  // log2 decay from the segment start to the current chunk start
#pragma unroll
  for (int i = 0; i < KN; ++i) S[i] = 0.f, Bacc[i] = 0.f;
  fetch(c_begin);
  for (int n = c_begin; n < c_end; ++n) {
    float b2[KN], r2[KN], g2[KN];
    gate(b2, r2, g2);
    if (tok) {
      float kv[KN], qv[KN];
#pragma unroll
      for (int g = 0; g < KN / 4; ++g) {
        unpack4(rk[g], kv + 4 * g);
        unpack4(rq[g], qv + 4 * g);
      }
#pragma unroll
      for (int i = 0; i < KN; ++i) {
        const uint32_t off = kmaj16(KO + i, t, Cfg::LBO_T, Cfg::SBO_T);
        st_op<NTG>(smem + Cfg::OFF_KHT, Cfg::KHT_SZ, off, kv[i] * exp2f(g2[i] - b2[i]));
        st_op<NTG>(smem + Cfg::OFF_QTT, Cfg::KHT_SZ, off, qv[i] * exp2f(Bacc[i] + b2[i]));
      }
#pragma unroll
      for (int g = 0; g < VN / 4; ++g) {
        float vv[4], dd[4];
        unpack4(rvv[g], vv);
        unpack4(rdo[g], dd);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t off = kmaj16(VO + 4 * g + u, t, Cfg::LBO_T, Cfg::SBO_T);
          st_op<NTV>(smem + Cfg::OFF_VT, Cfg::VT_SZ, off, vv[u]);
          st_op<NTV>(smem + Cfg::OFF_ADOT, Cfg::DOT_SZ, off, dd[u]);
        }
      }
    }
    if (state_thr) {  // state entering chunk n, relative to the segment start
      float* dst = a.chunk_S + (((size_t)bh * a.nchunks + n) * DV + t) * DK + KO;
#pragma unroll
      for (int i = 0; i < KN; ++i) dst[i] = S[i];
    }
    if (t == 0) {
#pragma unroll
      for (int i = 0; i < KN; ++i) a.chunk_B[((size_t)bh * a.nchunks + n) * DKP + KO + i] = Bacc[i];
    }
    fetch(n + 1);
    sync_mma();
    if (tid == 0) {
      mma_issue<NTV, NTG, C / 16>(tmem + Cfg::TM_DQ, dVT, Cfg::VT_SZ, KS_T, dKHT, Cfg::KHT_SZ, KS_T,
                                  idesc_bf16(128, DKP), false);
      mma_issue<NTV, NTG, C / 16>(tmem + Cfg::TM_DH, dADOT, Cfg::DOT_SZ, KS_T, dQTT, Cfg::KHT_SZ, KS_T,
                                  idesc_bf16(128, DKP), n > c_begin);
      mma_commit(&sh.bar);
    }
    wait_mma();
    {
      float ds[cround(KN, 8)];
#pragma unroll
      for (int c = 0; c < cround(KN, 8); c += 8) tmem_ld8(tmem + lane_base + Cfg::TM_DQ + KO + c, ds + c);
      tmem_ld_wait();
      if (state_thr) {
#pragma unroll
        for (int i = 0; i < KN; ++i) S[i] = exp2f(g2[i]) * S[i] + ds[i];
      }
#pragma unroll
      for (int i = 0; i < KN; ++i) Bacc[i] += g2[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  // publish the segment records: decay, state, state gradient at the segment start
  const int rec = bh * a.nseg + seg;
  {
    float dh[cround(KN, 8)];
#pragma unroll
    for (int c = 0; c < cround(KN, 8); c += 8) tmem_ld8(tmem + lane_base + Cfg::TM_DH + KO + c, dh + c);
    tmem_ld_wait();
    if (a.nseg > 1) {
      if (state_thr) {
        float* ds = a.seg_S + ((size_t)rec * DV + t) * DK + KO;
        float* dhp = a.seg_H + ((size_t)rec * DV + t) * DK + KO;
#pragma unroll
        for (int i = 0; i < KN; ++i) {
          ds[i] = S[i];
          dhp[i] = dh[i];
        }
      }
      if (t == 0) {
#pragma unroll
        for (int i = 0; i < KN; ++i) a.seg_gam[(size_t)rec * DKP + KO + i] = Bacc[i];
      }
    }
  }
  float Sin[KN], dH[KN];  // state entering the segment; state gradient leaving it
#pragma unroll
  for (int i = 0; i < KN; ++i) Sin[i] = 0.f, dH[i] = 0.f;
  if (a.nseg > 1) {
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      st_release(a.flags + rec, 1u);
      for (int s2 = 0; s2 < a.nseg; ++s2)
        if (s2 != seg && !wait_flag(a.flags + bh * a.nseg + s2, 1u, kSpinLimitNs)) timed_out = true;
    }
    __syncthreads();
    if (state_thr) {
      for (int s2 = 0; s2 < seg; ++s2) {  // forward fold: state entering this segment
        const size_t r2 = (size_t)bh * a.nseg + s2;
        const float* src = a.seg_S + (r2 * DV + t) * DK + KO;
#pragma unroll
        for (int i = 0; i < KN; ++i) Sin[i] = exp2f(__ldcg(a.seg_gam + r2 * DKP + KO + i)) * Sin[i] + __ldcg(src + i);
      }
      for (int s2 = a.nseg - 1; s2 > seg; --s2) {  // backward fold: gradient leaving this segment
        const size_t r2 = (size_t)bh * a.nseg + s2;
        const float* src = a.seg_H + (r2 * DV + t) * DK + KO;
#pragma unroll
        for (int i = 0; i < KN; ++i) dH[i] = __ldcg(src + i) + exp2f(__ldcg(a.seg_gam + r2 * DKP + KO + i)) * dH[i];
      }
    }
  }
  // dlog(alpha) of the token after the segment = rowsum(dH_out * S_out)
  if (tid < 64) sh.cinit[tid >> 5][tid & 31] = 0.f;
  __syncthreads();
  {
#pragma unroll
    for (int i = 0; i < KN; ++i) {
      float pr = state_thr ? dH[i] * (exp2f(Bacc[i]) * Sin[i] + S[i]) : 0.f;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) pr += __shfl_xor_sync(0xffffffffu, pr, off);
      if (lane == 0 && wq * 32 < DV) atomicAdd(&sh.cinit[H][i], pr);
    }
  }
  __syncthreads();
  float carry[KN];
#pragma unroll
  for (int i = 0; i < KN; ++i) carry[i] = sh.cinit[H][i];

  // ------------------------------------------------------------ pass B
  fetch(c_end - 1);
  for (int n = c_end - 1; n >= c_begin; --n) {
    const bool my_valid = valid;
    const long long my_row = grow;
    float b2[KN], r2[KN], g2[KN];
    gate(b2, r2, g2);
    float qv[KN], kv[KN];
#pragma unroll
    for (int g = 0; g < KN / 4; ++g) {
      unpack4(rq[g], qv + 4 * g);
      unpack4(rk[g], kv + 4 * g);
    }
    if (tok) {
      // token rows: qbar, kbar, khat (row and column forms), dO and v
#pragma unroll
      for (int g = 0; g < KN / 4; ++g) {
        float qb[4], kb[4], kh[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = 4 * g + u;
          const float d = b2[i] - r2[i];
          if (fabsf(d) > 115.f) sh.range_bad = 1;
          qb[u] = qv[i] * exp2f(d);
          kb[u] = kv[i] * exp2f(-d);
          kh[u] = kv[i] * exp2f(g2[i] - b2[i]);
          const uint32_t offc = kmaj16(KO + i, t, Cfg::LBO_T, Cfg::SBO_T);
          st_op<NTG>(smem + Cfg::OFF_QT, Cfg::QT_SZ, offc, qb[u]);
          st_op<NTG>(smem + Cfg::OFF_KT, Cfg::KT_SZ, offc, kb[u]);
        }
        const uint32_t off = kmaj16(t, KO + 4 * g, 128, Cfg::SBO_RK);
        st_op4<NTG>(smem + Cfg::OFF_AQ, Cfg::AQ_SZ, off, qb[0], qb[1], qb[2], qb[3]);
        st_op4<NTG>(smem + Cfg::OFF_BK, Cfg::BK_SZ, off, kb[0], kb[1], kb[2], kb[3]);
        st_op4<NTG>(smem + Cfg::OFF_KH, Cfg::KH_SZ, off, kh[0], kh[1], kh[2], kh[3]);
      }
#pragma unroll
      for (int g = 0; g < VN / 4; ++g) {
        float vv[4], dd[4];
        unpack4(rvv[g], vv);
        unpack4(rdo[g], dd);
        const uint32_t off = kmaj16(t, VO + 4 * g, 128, Cfg::SBO_RV);
        st_op4<NTV>(smem + Cfg::OFF_VR, Cfg::VR_SZ, off, vv[0], vv[1], vv[2], vv[3]);
        st_op4<NTV>(smem + Cfg::OFF_DO, Cfg::DO_SZ, off, dd[0], dd[1], dd[2], dd[3]);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          st_op<NTV>(smem + Cfg::OFF_DOT, Cfg::DOT_SZ, kmaj16(VO + 4 * g + u, t, Cfg::LBO_T, Cfg::SBO_T), dd[u]);
      }
      if (H == 1) {  // zero K-padding of the row buffers
#pragma unroll
        for (int c = DK; c < DKP; c += 4) {
          const uint32_t off = kmaj16(t, c, 128, Cfg::SBO_RK);
          st_op4<NTG>(smem + Cfg::OFF_AQ, Cfg::AQ_SZ, off, 0.f, 0.f, 0.f, 0.f);
          st_op4<NTG>(smem + Cfg::OFF_BK, Cfg::BK_SZ, off, 0.f, 0.f, 0.f, 0.f);
          st_op4<NTG>(smem + Cfg::OFF_KH, Cfg::KH_SZ, off, 0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int c = DV; c < DVP; c += 4) {
          const uint32_t off = kmaj16(t, c, 128, Cfg::SBO_RV);
          st_op4<NTV>(smem + Cfg::OFF_VR, Cfg::VR_SZ, off, 0.f, 0.f, 0.f, 0.f);
          st_op4<NTV>(smem + Cfg::OFF_DO, Cfg::DO_SZ, off, 0.f, 0.f, 0.f, 0.f);
        }
      }
    }
    if (state_thr) {
      // S_{n-1} = in-segment state + decayed state entering the segment
      float Sn[KN];
      const float* src = a.chunk_S + (((size_t)bh * a.nchunks + n) * DV + t) * DK + KO;
#pragma unroll
      for (int i = 0; i < KN; ++i)
        Sn[i] = __ldcg(src + i) + exp2f(__ldcg(a.chunk_B + ((size_t)bh * a.nchunks + n) * DKP + KO + i)) * Sin[i];
#pragma unroll
      for (int i = 0; i < KN; ++i) {
        const uint32_t offj = kmaj16(KO + i, t, 144, Cfg::SBO_J);
        st_op<NTG>(smem + Cfg::OFF_SP, Cfg::SP_SZ, offj, exp2f(r2[i]) * Sn[i]);
        st_op<NTG>(smem + Cfg::OFF_DHP, Cfg::DHP_SZ, offj, exp2f(g2[i] - r2[i]) * dH[i]);
      }
#pragma unroll
      for (int g = 0; g < KN / 4; ++g)
        st_op4<NTG>(smem + Cfg::OFF_DHT, Cfg::DHT_SZ, kmaj16(t, KO + 4 * g, 128, Cfg::SBO_RK), dH[4 * g],
                    dH[4 * g + 1], dH[4 * g + 2], dH[4 * g + 3]);
      if (H == 1) {
#pragma unroll
        for (int c = DK; c < DKP; c += 4)
          st_op4<NTG>(smem + Cfg::OFF_DHT, Cfg::DHT_SZ, kmaj16(t, c, 128, Cfg::SBO_RK), 0.f, 0.f, 0.f, 0.f);
      }
    } else if (jpad_thr) {  // zero K-padding (value rows DV..DVP-1) of S' and dH'
#pragma unroll
      for (int i = 0; i < KN; ++i) {
        const uint32_t offj = kmaj16(KO + i, t, 144, Cfg::SBO_J);
        st_op<NTG>(smem + Cfg::OFF_SP, Cfg::SP_SZ, offj, 0.f);
        st_op<NTG>(smem + Cfg::OFF_DHP, Cfg::DHP_SZ, offj, 0.f);
      }
    }
    fetch(n - 1);
    sync_mma();
    if (tid == 0) {
      mma_issue<NTG, NTG, DKP / 16>(tmem + Cfg::TM_P, dAQ, Cfg::AQ_SZ, KS_R, dBK, Cfg::BK_SZ, KS_R,
                                    idesc_bf16(128, C), false);
      mma_issue<NTV, NTV, DVP / 16>(tmem + Cfg::TM_DPA, dDO, Cfg::DO_SZ, KS_R, dVR, Cfg::VR_SZ, KS_R,
                                    idesc_bf16(128, C), false);
      mma_issue<NTV, NTG, DVP / 16>(tmem + Cfg::TM_DQ, dDO, Cfg::DO_SZ, KS_R, dSP, Cfg::SP_SZ, KS_J,
                                    idesc_bf16(128, DKP), false);
      mma_issue<NTV, NTG, DVP / 16>(tmem + Cfg::TM_DK, dVR, Cfg::VR_SZ, KS_R, dDHP, Cfg::DHP_SZ, KS_J,
                                    idesc_bf16(128, DKP), false);
      mma_issue<NTG, NTG, DKP / 16>(tmem + Cfg::TM_DV, dKH, Cfg::KH_SZ, KS_R, dDHT, Cfg::DHT_SZ, KS_R,
                                    idesc_bf16(128, DVP), false);
      mma_issue<NTV, NTG, C / 16>(tmem + Cfg::TM_DH, dDOT, Cfg::DOT_SZ, KS_T, dQT, Cfg::QT_SZ, KS_T,
                                  idesc_bf16(128, DKP), false);
      mma_commit(&sh.bar);
    }
    wait_mma();
    // masked P and Dp -> second-batch operands (Dp row form and transposed, P transposed)
#pragma unroll
    for (int cb = 0; cb < C / 2; cb += 16) {
      float pv[16], dv16[16];
      tmem_ld16(tmem + lane_base + Cfg::TM_P + H * (C / 2) + cb, pv);
      tmem_ld16(tmem + lane_base + Cfg::TM_DPA + H * (C / 2) + cb, dv16);
      tmem_ld_wait();
      if (tok) {
        const int s0 = H * (C / 2) + cb;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const bool keep = s0 + u <= t;
          pv[u] = keep ? pv[u] : 0.f;
          dv16[u] = keep ? dv16[u] : 0.f;
          const uint32_t offc = kmaj16(s0 + u, t, Cfg::LBO_T, Cfg::SBO_T);
          st_op<NTG>(smem + Cfg::OFF_PT, Cfg::PT_SZ, offc, pv[u]);
          st_op<NTG>(smem + Cfg::OFF_DPT, Cfg::DPT_SZ, offc, dv16[u]);
        }
#pragma unroll
        for (int u = 0; u < 16; u += 4)
          st_op4<NTG>(smem + Cfg::OFF_DP, Cfg::DP_SZ, kmaj16(t, s0 + u, 128, Cfg::SBO_RC), dv16[u], dv16[u + 1],
                      dv16[u + 2], dv16[u + 3]);
      }
    }
    sync_mma();
    if (tid == 0) {
      mma_issue<NTG, NTG, C / 16>(tmem + Cfg::TM_DQ, dDP, Cfg::DP_SZ, KS_R, dKT, Cfg::KT_SZ, KS_T,
                                  idesc_bf16(128, DKP), true);
      mma_issue<NTG, NTG, C / 16>(tmem + Cfg::TM_DK, dDPT, Cfg::DPT_SZ, KS_T, dQT, Cfg::QT_SZ, KS_T,
                                  idesc_bf16(128, DKP), true);
      mma_issue<NTG, NTV, C / 16>(tmem + Cfg::TM_DV, dPT, Cfg::PT_SZ, KS_T, dDOT, Cfg::DOT_SZ, KS_T,
                                  idesc_bf16(128, DVP), true);
      mma_commit(&sh.bar);
    }
    wait_mma();
    // epilogue: dq, dk, dv; dlog(alpha) terms; state-gradient carry
    float gq[cround(KN, 8)], gk[cround(KN, 8)], gv[cround(VN, 8)], gh[cround(KN, 8)];
#pragma unroll
    for (int c = 0; c < cround(KN, 8); c += 8) {
      tmem_ld8(tmem + lane_base + Cfg::TM_DQ + KO + c, gq + c);
      tmem_ld8(tmem + lane_base + Cfg::TM_DK + KO + c, gk + c);
      tmem_ld8(tmem + lane_base + Cfg::TM_DH + KO + c, gh + c);
    }
#pragma unroll
    for (int c = 0; c < cround(VN, 8); c += 8) tmem_ld8(tmem + lane_base + Cfg::TM_DV + VO + c, gv + c);
    tmem_ld_wait();
    float gl[KN];
#pragma unroll
    for (int i = 0; i < KN; ++i) {
      const float d = b2[i] - r2[i];
      gq[i] *= exp2f(d);
      gk[i] *= exp2f(-d);
      gl[i] = my_valid ? qv[i] * gq[i] - kv[i] * gk[i] : 0.f;
    }
    if (my_valid) {
      const size_t ok = ((size_t)my_row * a.H + h) * DK + KO, ov = ((size_t)my_row * a.H + h) * DV + VO;
      store_row<KN>(reinterpret_cast<TOUT*>(a.dq) + ok, gq);
      store_row<KN>(reinterpret_cast<TOUT*>(a.dk) + ok, gk);
      store_row<VN>(reinterpret_cast<TOUT*>(a.dv) + ov, gv);
    }
    if (state_thr) {
#pragma unroll
      for (int i = 0; i < KN; ++i) dH[i] = exp2f(g2[i]) * dH[i] + exp2f(r2[i]) * gh[i];
    }
    // reverse inclusive cumsum of q*dq - k*dk over the chunk, plus the carry
#pragma unroll
    for (int i = 0; i < KN; ++i) {
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_down_sync(0xffffffffu, gl[i], off);
        if (lane + off < 32) gl[i] += y;
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int i = 0; i < KN; ++i) sh.wtot[warp][i] = gl[i];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < KN; ++i) {
      float post = 0.f, tot = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float w = sh.wtot[H * 4 + u][i];
        post += (u > wq) ? w : 0.f;
        tot += w;
      }
      gl[i] += post + carry[i];
      carry[i] += tot;
    }
    if (my_valid) {
      float* dst = a.dla + ((size_t)my_row * a.gate_heads + hz) * DK + KO;
      if (a.gate_heads == 1) {
#pragma unroll
        for (int i = 0; i < KN; ++i) atomicAdd(dst + i, gl[i]);
      } else {
        store_row<KN>(dst, gl);
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (timed_out) set_status(a.status, DIG_ERR_DEVICE_TIMEOUT);
}

template <int C, int DK, int DV, typename TIN, typename TOUT>
__global__ void __launch_bounds__(256, 1) gla_bwd_kernel(const GlaArgs a) {
  constexpr int NTG = std::is_same<TIN, float>::value ? 3 : 2;
  constexpr int NTV = std::is_same<TIN, float>::value ? 3 : 1;
  using Cfg = BwdCfg<C, NTG, NTV, DK, DV>;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ BwdSmem sh;
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
  if (tid < 128) bwd_thread<C, DK, DV, TIN, TOUT, 0>(a, smem, sh);
  else bwd_thread<C, DK, DV, TIN, TOUT, 1>(a, smem, sh);
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
template <int C, int DK, int DV, typename TIN, typename TOUT>
static cudaError_t bwd_launch_one(const GlaArgs& a, int grid, bool coop, cudaStream_t s, int* occ) {
  using Cfg = BwdCfg<C, std::is_same<TIN, float>::value ? 3 : 2, std::is_same<TIN, float>::value ? 3 : 1, DK, DV>;
  auto kern = gla_bwd_kernel<C, DK, DV, TIN, TOUT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e != cudaSuccess) return e;
  if (occ) return cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, kern, 256, Cfg::SMEM);
  if (coop) {
    GlaArgs copy = a;
    void* args[] = {&copy};
    return cudaLaunchCooperativeKernel((const void*)kern, dim3(grid), dim3(256), args, Cfg::SMEM, s);
  }
  kern<<<grid, 256, Cfg::SMEM, s>>>(a);
  return cudaGetLastError();
}

template <int DK, int DV>
static cudaError_t bwd_dispatch_types(const GlaVariant& v, const GlaArgs& a, int grid, bool coop, cudaStream_t s,
                                      int* occ) {
  using bf = __nv_bfloat16;
  if (v.tin == DIG_BF16) {
    if (v.tout == DIG_BF16) return bwd_launch_one<64, DK, DV, bf, bf>(a, grid, coop, s, occ);
    return bwd_launch_one<64, DK, DV, bf, float>(a, grid, coop, s, occ);
  }
  if (v.tout == DIG_BF16) return bwd_launch_one<32, DK, DV, float, bf>(a, grid, coop, s, occ);
  return bwd_launch_one<32, DK, DV, float, float>(a, grid, coop, s, occ);
}

static cudaError_t bwd_dispatch(const GlaVariant& v, const GlaArgs& a, int grid, bool coop, cudaStream_t s, int* occ) {
  if (v.dk == 32 && v.dv == 64) return bwd_dispatch_types<32, 64>(v, a, grid, coop, s, occ);
  if (v.dk == 36 && v.dv == 72) return bwd_dispatch_types<36, 72>(v, a, grid, coop, s, occ);
  if (v.dk == 64 && v.dv == 64) return bwd_dispatch_types<64, 64>(v, a, grid, coop, s, occ);
  return cudaErrorInvalidValue;
}

cudaError_t launch_gla_bwd(const GlaVariant& v, const GlaArgs& a, int grid, bool coop, cudaStream_t s) {
  return bwd_dispatch(v, a, grid, coop, s, nullptr);
}

int gla_bwd_blocks_per_sm(const GlaVariant& v) {
  int occ = 0;
  if (bwd_dispatch(v, GlaArgs{}, 0, false, nullptr, &occ) != cudaSuccess) return 0;
  return occ;
}

}  // namespace dig
