// gla_fwd.cu -- chunkwise Gated Linear Attention forward on sm_100a.
//
// What is computed (DiG slides, GLA eq. (5)-(8)): for every (batch, head)
// sequence, in scan order t,
//     alpha_t = exp(inv_tau * logsigmoid(z_t)),  S_t = diag(alpha_t) S_{t-1} + k_t^T v_t,
//     o_t = q_t S_t,
// evaluated chunkwise (slides "計算効率の分析", paper "Efficiency Analysis": the
// sequence is cut into chunks that fit on-chip).  For a chunk of C tokens with
// in-chunk inclusive log-decay cumsum b_t, reference r = b at the chunk's
// middle token and chunk decay Gamma (factors from gla_gate.cu),
//     qbar_t = q_t * e^{b_t - r},  kbar_s = k_s * e^{r - b_s},  khat_s = kbar_s * e^{Gamma - r}
//     P = (qbar kbar^T) masked to s <= t               (tensor core, C x C)
//     O = qbar (diag(e^r) S_in) + P V                   (tensor core)
//     S_out = diag(e^Gamma) S_in + khat^T V             (tensor core + fp32 carry)
// which equals the recurrence in exact arithmetic.
//
// Work decomposition: one CTA per (sequence, segment of consecutive chunks),
// all CTAs resident (cooperative launch).  With more than one segment per
// sequence, sweep 1 runs the segment's chunks last-to-first and accumulates the
// segment's state record sum_n diag(e^{decay after chunn n}) khat_n^T V_n in
// TMEM (no per-chunk read-back), publishes it, and folds the records of the
// earlier segments into the state entering the segment.  Sweep 2 produces the
// outputs, software-pipelined: while the tensor core runs P V of chunk n and the
// first products of chunk n+1, the threads build chunk n+1's operands and store
// chunk n's outputs (V and O are double-buffered).
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
  // Every operand is stored as token rows (bf16, K-major over its channels,
  // LBO = 128 between 8-channel groups) and read either K-major or, for the
  // products that contract over tokens, MN-major.  Row strides are padded by 64
  // bytes (when it fits) so the four 8-row groups a warp writes alternate bank
  // halves.
  static constexpr int PADK = DKP >= 64 ? 0 : 64, PADC = C >= 128 && DKP >= 64 ? 0 : 64;
  static constexpr int SBO_K = DKP * 16 + PADK;  // rows of DKP values (q, k, khat, S')
  static constexpr int SBO_V = DVP * 16 + 64;    // rows of DVP values (v)
  static constexpr int SBO_P = C * 16 + PADC;    // rows of C values (P)
  static constexpr int VR_SZ = (C / 8) * SBO_V;
  static constexpr int AQ_SZ = (C / 8) * SBO_K;
  static constexpr int SPT_SZ = (DVP / 8) * SBO_K;
  static constexpr int P_SZ = (C / 8) * SBO_P;
  static constexpr int OFF_VR0 = 0;
  static constexpr int OFF_VR1 = NTV * VR_SZ;
  static constexpr int OFF_P = 2 * NTV * VR_SZ;
  static constexpr int OFF_AQ = OFF_P + NTG * P_SZ;
  static constexpr int OFF_BK = OFF_AQ + NTG * AQ_SZ;
  static constexpr int OFF_KH = OFF_BK + NTG * AQ_SZ;
  static constexpr int OFF_SPT = OFF_KH + NTG * AQ_SZ;
  static constexpr int END_DATA = OFF_SPT + NTG * SPT_SZ;
  // M = 128 reads of A operands cover 128 rows (K-major) or 16 MN groups
  // (MN-major) even where fewer are real; they must stay inside the allocation.
  static constexpr int END_VR = OFF_VR1 + (NTV - 1) * VR_SZ + (C / 8 - 1) * SBO_V + 16 * 128;
  static constexpr int END_AQ = OFF_AQ + (NTG - 1) * AQ_SZ + 16 * SBO_K;
  static constexpr int END_P = OFF_P + (NTG - 1) * P_SZ + 16 * SBO_P;
  static constexpr int SMEM = cmax(cmax(END_DATA, END_VR), cmax(END_AQ, END_P));
  // TMEM columns: P, two O accumulators, the chunk state update
  static constexpr int TM_P = 0, TM_O0 = C, TM_O1 = C + DVP, TM_DS = C + 2 * DVP;
  static constexpr int TM_COLS = pow2ceil(C + 2 * DVP + DKP);
  static_assert(TM_COLS <= 512, "TMEM budget");
  static_assert(SMEM <= 225 * 1024, "shared-memory budget");  // + ~4 KB static stays under 227 KB
  static_assert(DK % 4 == 0 && DV % 4 == 0 && DK1 > 0 && DV1 > 0, "head dims");
  static_assert(C == 64 || C == 128, "chunk");
};

struct FwdSmem {
  float ch[2][4][64];  // chunk constants 2^r, 2^(Gamma-r), 2^Gamma, Gamma (double-buffered)
  float red[256];      // epilogue row sums of squares
  uint64_t bar_a;      // first products of a chunk (P, qbar S', khat^T V)
  uint64_t bar_b;      // P V of a chunk
  uint64_t bar_s[2];   // sweep 1: the state-record products of the two operand stages
  uint32_t tmem;
};

constexpr int kFwdThreads = 256;

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
  using WK = RowWriter<NTG, KO, KN>;          // q/k-like rows, this half's channels
  using WV = RowWriter<NTV, VO, VN>;          // v rows
  using WP = RowWriter<NTG, DK, DKP - DK>;    // zero K-padding of q/k-like rows (half 1)

  const int tid = threadIdx.x, warp = tid >> 5;
  const int t = tid & 127, wq = warp & 3;
  const int nseq = a.B * a.H;
  const int bh = blockIdx.x % nseq, seg = blockIdx.x / nseq;
  const int b = bh / a.H, h = bh % a.H;
  const int hz = a.gate_heads == 1 ? 0 : h;
  const int bz = b * a.gate_heads + hz;
  const int c_begin = (int)((long long)seg * a.nchunks / a.nseg);
  const int c_end = (int)((long long)(seg + 1) * a.nchunks / a.nseg);
  const bool tok = t < C;
  const bool state_thr = t < DV;
  const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
  const uint32_t tmem = sh.tmem;
  const uint32_t sbase = smem_u32(smem);
  uint32_t ph_a = 0, ph_b = 0, ph_s0 = 0, ph_s1 = 0;
  bool timed_out = false;
  auto sync_mma = [&]() {  // publish this thread's operand writes to the tensor core, then barrier
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  };

  // K-major descriptors (LBO 128, SBO row stride) and MN-major ones for the
  // token-contracting products (LBO row stride, SBO 128)
  const uint64_t dVRm0 = sdesc(sbase + Cfg::OFF_VR0, Cfg::SBO_V, 128);
  const uint64_t dVRm1 = sdesc(sbase + Cfg::OFF_VR1, Cfg::SBO_V, 128);
  const uint64_t dP = sdesc(sbase + Cfg::OFF_P, 128, Cfg::SBO_P);
  const uint64_t dAQ = sdesc(sbase + Cfg::OFF_AQ, 128, Cfg::SBO_K);
  const uint64_t dBK = sdesc(sbase + Cfg::OFF_BK, 128, Cfg::SBO_K);
  const uint64_t dKHm = sdesc(sbase + Cfg::OFF_KH, Cfg::SBO_K, 128);
  const uint64_t dAQm = sdesc(sbase + Cfg::OFF_AQ, Cfg::SBO_K, 128);  // second khat stage of sweep 1
  const uint64_t dSPT = sdesc(sbase + Cfg::OFF_SPT, 128, Cfg::SBO_K);
  // this thread's row addresses
  const uint32_t rowK_AQ = row_addr(sbase + Cfg::OFF_AQ, t, Cfg::SBO_K);
  const uint32_t rowK_BK = row_addr(sbase + Cfg::OFF_BK, t, Cfg::SBO_K);
  const uint32_t rowK_KH = row_addr(sbase + Cfg::OFF_KH, t, Cfg::SBO_K);
  const uint32_t rowV0 = row_addr(sbase + Cfg::OFF_VR0, t, Cfg::SBO_V);
  const uint32_t rowV1 = row_addr(sbase + Cfg::OFF_VR1, t, Cfg::SBO_V);
  const uint32_t rowSPT = row_addr(sbase + Cfg::OFF_SPT, t, Cfg::SBO_K);
  const uint32_t rowP = row_addr(sbase + Cfg::OFF_P, t, Cfg::SBO_P);

  auto wait_bar = [&](uint64_t* bar, uint32_t& ph) {
    if (!mbar_wait(bar, ph, kSpinLimitNs)) timed_out = true;
    ph ^= 1u;
    tc_fence_after();
  };
  // chunk constants -> shared stage (asynchronous; completed by cp_async_wait_all)
  auto load_ch = [&](int n, int stage) {
    if (n >= c_begin && n < c_end && tid < DK) {
      const int arr = tid / (DK / 4), g = tid % (DK / 4);
      cp_async16(&sh.ch[stage][arr][4 * g], a.gCH + (((size_t)bz * a.nchunks + n) * 4 + arr) * DK + 4 * g);
    }
  };

  // prefetched rows of the next chunk (registers)
  RT rq[KN / 4], rk[KN / 4], rvv[VN / 4];
  float4 req[KN / 4];
  bool valid = false;
  long long grow = 0;
  auto fetch = [&](int n, bool with_q) {
    const int p = n * C + t;
    valid = tok && n >= c_begin && n < c_end && p < a.L;
    grow = valid ? (long long)b * a.L + scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode) : 0;
    const size_t rk_off = ((size_t)grow * a.H + h) * DK + KO;
    const RT* kp = reinterpret_cast<const RT*>(reinterpret_cast<const TIN*>(a.k) + rk_off);
    const RT* qp = reinterpret_cast<const RT*>(reinterpret_cast<const TIN*>(a.q) + rk_off);
    const RT* vp = reinterpret_cast<const RT*>(reinterpret_cast<const TIN*>(a.v) + ((size_t)grow * a.H + h) * DV + VO);
    const float4* ep = reinterpret_cast<const float4*>(a.gEQ + ((size_t)bz * a.L + (valid ? p : 0)) * DK + KO);
#pragma unroll
    for (int g = 0; g < KN / 4; ++g) {
      rk[g] = valid ? __ldg(kp + g) : zero4<RT>();
      rq[g] = (valid && with_q) ? __ldg(qp + g) : zero4<RT>();
      req[g] = valid ? __ldcg(ep + g) : make_float4(1.f, 1.f, 1.f, 1.f);
    }
#pragma unroll
    for (int g = 0; g < VN / 4; ++g) rvv[g] = valid ? __ldg(vp + g) : zero4<RT>();
  };

  float S[KN];  // state S[KO + i][t] (state threads)
#pragma unroll
  for (int i = 0; i < KN; ++i) S[i] = 0.f;

  // ---------------------------------------------------------------- sweep 1
  const int rec = bh * a.nseg + seg;
  if (a.nseg > 1) {
    float Gsuf[KN];  // log2 decay of the segment's chunks after the current one
#pragma unroll
    for (int i = 0; i < KN; ++i) Gsuf[i] = 0.f;
    fetch(c_end - 1, false);
    load_ch(c_end - 1, (c_end - 1) & 1);
    cp_async_wait_all();
    __syncthreads();
    for (int n = c_end - 1; n >= c_begin; --n) {
      const int st = n & 1;
      // stage st was last read by the products of chunk n + 2
      if (n + 2 <= c_end - 1) {
        if (st) wait_bar(&sh.bar_s[1], ph_s1);
        else wait_bar(&sh.bar_s[0], ph_s0);
      }
      if (tok) {
        float kv[KN], ev[KN];
#pragma unroll
        for (int g = 0; g < KN / 4; ++g) {
          unpack4(rk[g], kv + 4 * g);
          unpack4(req[g], ev + 4 * g);
        }
#pragma unroll
        for (int i = 0; i < KN; ++i)  // khat scaled by the decay of the later chunks of the segment
          kv[i] *= __fdividef(1.f, ev[i]) * sh.ch[st][1][KO + i] * exp2f(Gsuf[i]);
        WK::run(st ? row_addr(sbase + Cfg::OFF_AQ, t, Cfg::SBO_K) : rowK_KH, Cfg::AQ_SZ, kv);
        float vv[VN];
#pragma unroll
        for (int g = 0; g < VN / 4; ++g) unpack4(rvv[g], vv + 4 * g);
        WV::run(st ? rowV1 : rowV0, Cfg::VR_SZ, vv);
      }
#pragma unroll
      for (int i = 0; i < KN; ++i) Gsuf[i] += sh.ch[st][3][KO + i];
      fetch(n - 1, false);
      load_ch(n - 1, st ^ 1);
      cp_async_wait_all();
      sync_mma();
      if (tid == 0) {
        mma_issue<NTV, NTG, C / 16>(tmem + Cfg::TM_DS, st ? dVRm1 : dVRm0, Cfg::VR_SZ, 2 * Cfg::SBO_V,
                                    st ? dAQm : dKHm, Cfg::AQ_SZ, 2 * Cfg::SBO_K, idesc_bf16(128, DKP, true, true),
                                    n != c_end - 1);
        mma_commit(&sh.bar_s[st]);
      }
    }
    // the last two chunks' products
    {
      const int nlast = c_begin, nprev = c_begin + 1;
      if (nprev <= c_end - 1) {
        if (nprev & 1) wait_bar(&sh.bar_s[1], ph_s1);
        else wait_bar(&sh.bar_s[0], ph_s0);
      }
      if (nlast & 1) wait_bar(&sh.bar_s[1], ph_s1);
      else wait_bar(&sh.bar_s[0], ph_s0);
    }
    {
      float ds[cround(KN, 8)];
#pragma unroll
      for (int c = 0; c < cround(KN, 8); c += 8) tmem_ld8(tmem + lane_base + Cfg::TM_DS + KO + c, ds + c);
      tmem_ld_wait();
      if (state_thr) {
        float* dst = a.seg_S + ((size_t)rec * DV + t) * DK + KO;
#pragma unroll
        for (int i = 0; i < KN; ++i) dst[i] = ds[i];
      }
      if (t == 0) {
#pragma unroll
        for (int i = 0; i < KN; ++i) a.seg_gam[(size_t)rec * DKP + KO + i] = Gsuf[i];
      }
    }
    __threadfence();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) st_release(a.flags + rec, 1u);
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
  }

  // ---------------------------------------------------------------- sweep 2
  // P keeps its never-written (fully masked) blocks zero from here on
  for (int i = tid; i < NTG * Cfg::P_SZ / 16; i += 256)
    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(sbase + Cfg::OFF_P + 16u * i), "r"(0u) : "memory");
  fetch(c_begin, true);
  load_ch(c_begin, c_begin & 1);
  cp_async_wait_all();
  __syncthreads();
  bool e_valid = false;  // epilogue bookkeeping of the chunk whose P V is in flight
  long long e_row = 0;
  RT rr_raw[VN / 4];
  const bool with_y = a.y != nullptr && a.r != nullptr;

  auto epilogue = [&](int n_prev) {
    const int st = n_prev & 1;
    float ov[cround(VN, 8)];
#pragma unroll
    for (int c = 0; c < cround(VN, 8); c += 8)
      tmem_ld8(tmem + lane_base + (st ? Cfg::TM_O1 : Cfg::TM_O0) + VO + c, ov + c);
    tmem_ld_wait();
    const size_t ro = ((size_t)e_row * a.H + h) * DV + VO;
    if (e_valid) store_row<VN>(reinterpret_cast<TOUT*>(a.o) + ro, ov);
    if (with_y) {
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < VN; ++i) ss += ov[i] * ov[i];
      sh.red[tid] = e_valid ? ss : 0.f;
      __syncthreads();
      const float inv = rsqrtf((sh.red[t] + sh.red[t + 128]) / (float)DV + a.eps);
      __syncthreads();  // red is rewritten by the next epilogue
      if (e_valid) {
        float rr[VN], yv[VN];
#pragma unroll
        for (int g = 0; g < VN / 4; ++g) unpack4(rr_raw[g], rr + 4 * g);
#pragma unroll
        for (int i = 0; i < VN; ++i) {
          const float gmm = a.gamma != nullptr ? __ldg(a.gamma + VO + i) : 1.f;
          const float sw = rr[i] / (1.f + exp2f(-rr[i] * kLog2e));
          yv[i] = sw * ov[i] * inv * gmm;
        }
        store_row<VN>(reinterpret_cast<TOUT*>(a.y) + ro, yv);
      }
    }
  };

  for (int n = c_begin; n < c_end; ++n) {
    const int st = n & 1;
    const bool my_valid = valid;
    const long long my_row = grow;
    // ---- A: operands of chunk n
    if (tok) {
      float qv[KN], kv[KN], ev[KN], kh[KN];
#pragma unroll
      for (int g = 0; g < KN / 4; ++g) {
        unpack4(rq[g], qv + 4 * g);
        unpack4(rk[g], kv + 4 * g);
        unpack4(req[g], ev + 4 * g);
      }
#pragma unroll
      for (int i = 0; i < KN; ++i) {
        qv[i] *= ev[i];
        kv[i] *= __fdividef(1.f, ev[i]);
        kh[i] = kv[i] * sh.ch[st][1][KO + i];
      }
      WK::run(rowK_AQ, Cfg::AQ_SZ, qv);
      WK::run(rowK_BK, Cfg::AQ_SZ, kv);
      WK::run(rowK_KH, Cfg::AQ_SZ, kh);
      if (H == 1) {
        const float zz[16] = {};
        WP::run(rowK_AQ, Cfg::AQ_SZ, zz);
        WP::run(rowK_BK, Cfg::AQ_SZ, zz);
      }
      float vv[VN];
#pragma unroll
      for (int g = 0; g < VN / 4; ++g) unpack4(rvv[g], vv + 4 * g);
      WV::run(st ? rowV1 : rowV0, Cfg::VR_SZ, vv);
    }
    if (state_thr) {
      // B operand of O += qbar S': row j = t of S'^T, S' = diag(2^r) S_in
      float e[KN];
#pragma unroll
      for (int i = 0; i < KN; ++i) e[i] = sh.ch[st][0][KO + i] * S[i];
      WK::run(rowSPT, Cfg::SPT_SZ, e);
      if (H == 1) {
        const float zz[16] = {};
        WP::run(rowSPT, Cfg::SPT_SZ, zz);
      }
    }
    float eg[KN];
#pragma unroll
    for (int i = 0; i < KN; ++i) eg[i] = sh.ch[st][2][KO + i];
    fetch(n + 1, true);
    load_ch(n + 1, st ^ 1);
    sync_mma();
    if (tid == 0) {
      mma_issue<NTG, NTG, DKP / 16>(tmem + Cfg::TM_P, dAQ, Cfg::AQ_SZ, 256, dBK, Cfg::AQ_SZ, 256, idesc_bf16(128, C),
                                    false);
      mma_issue<NTG, NTG, DKP / 16>(tmem + (st ? Cfg::TM_O1 : Cfg::TM_O0), dAQ, Cfg::AQ_SZ, 256, dSPT, Cfg::SPT_SZ,
                                    256, idesc_bf16(128, DVP), false);
      mma_issue<NTV, NTG, C / 16>(tmem + Cfg::TM_DS, st ? dVRm1 : dVRm0, Cfg::VR_SZ, 2 * Cfg::SBO_V, dKHm, Cfg::AQ_SZ,
                                  2 * Cfg::SBO_K, idesc_bf16(128, DKP, true, true), false);
      mma_commit(&sh.bar_a);
    }
    // ---- B: outputs of chunk n - 1 (its P V has been issued)
    if (n > c_begin) {
      wait_bar(&sh.bar_b, ph_b);
      epilogue(n - 1);
    }
    // ---- C: state carry, P of chunk n, issue P V
    wait_bar(&sh.bar_a, ph_a);
    {
      float ds[cround(KN, 8)];
#pragma unroll
      for (int c = 0; c < cround(KN, 8); c += 8) tmem_ld8(tmem + lane_base + Cfg::TM_DS + KO + c, ds + c);
      tmem_ld_wait();
      if (state_thr) {
#pragma unroll
        for (int i = 0; i < KN; ++i) S[i] = eg[i] * S[i] + ds[i];
      }
    }
#pragma unroll
    for (int cb = 0; cb < C / 2; cb += 16) {
      const int s0 = H * (C / 2) + cb;
      if (s0 > 32 * wq + 31) continue;  // the whole warp's rows are masked: block stays zero
      float pv[16];
      tmem_ld16(tmem + lane_base + Cfg::TM_P + s0, pv);
      tmem_ld_wait();
      if (tok) {
#pragma unroll
        for (int u = 0; u < 16; ++u) pv[u] = (s0 + u <= t) ? pv[u] : 0.f;
        sts_op8<NTG>(rowP + (s0 / 8) * 128, Cfg::P_SZ, pv);
        sts_op8<NTG>(rowP + (s0 / 8 + 1) * 128, Cfg::P_SZ, pv + 8);
      }
    }
    if (with_y && my_valid) {
      const RT* rp = reinterpret_cast<const RT*>(reinterpret_cast<const TIN*>(a.r) + ((size_t)my_row * a.H + h) * DV + VO);
#pragma unroll
      for (int g = 0; g < VN / 4; ++g) rr_raw[g] = __ldg(rp + g);
    }
    cp_async_wait_all();  // chunk n+1's constants (issued with the row fetch)
    sync_mma();
    if (tid == 0) {
      mma_issue<NTG, NTV, C / 16>(tmem + (st ? Cfg::TM_O1 : Cfg::TM_O0), dP, Cfg::P_SZ, 256, st ? dVRm1 : dVRm0,
                                  Cfg::VR_SZ, 2 * Cfg::SBO_V, idesc_bf16(128, DVP, false, true), true);
      mma_commit(&sh.bar_b);
    }
    e_valid = my_valid;
    e_row = my_row;
  }
  if (c_end > c_begin) {
    wait_bar(&sh.bar_b, ph_b);
    epilogue(c_end - 1);
  }
  if (timed_out) set_status(a.status, DIG_ERR_DEVICE_TIMEOUT);
}


template <int C, int DK, int DV, typename TIN, typename TOUT>
__global__ void __launch_bounds__(kFwdThreads, 1) gla_fwd_kernel(const GlaArgs a) {
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
    mbar_init(&sh.bar_a, 1);
    mbar_init(&sh.bar_b, 1);
    mbar_init(&sh.bar_s[0], 1);
    mbar_init(&sh.bar_s[1], 1);
    fence_mbar_init();
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
    return cudaLaunchCooperativeKernel((const void*)kern, dim3(grid), dim3(kFwdThreads), args, Cfg::SMEM, s);
  }
  kern<<<grid, kFwdThreads, Cfg::SMEM, s>>>(a);
  return cudaGetLastError();
}

template <int C, int DK, int DV, typename TIN, typename TOUT>
static int occupancy_one() {
  using Cfg = FwdCfgOf<C, DK, DV, TIN>;
  auto kern = gla_fwd_kernel<C, DK, DV, TIN, TOUT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM) != cudaSuccess) return 0;
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kFwdThreads, Cfg::SMEM) != cudaSuccess) return 0;
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
