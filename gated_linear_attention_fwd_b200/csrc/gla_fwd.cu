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
// tf32 operands in the tensor core's canonical K-major layout.  Accumulators
// live in TMEM; token row t is TMEM lane t.
#include <type_traits>

#include "dig_common.cuh"
#include "gla.h"
#include "sm100.cuh"

namespace dig {

__host__ __device__ constexpr int cround(int x, int m) { return (x + m - 1) / m * m; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }
__host__ __device__ constexpr int pow2ceil(int x) {
  int p = 32;
  while (p < x) p <<= 1;
  return p;
}

template <int C_, int SPLIT_, int DK_, int DV_>
struct FwdCfg {
  static constexpr int C = C_, SPLIT = SPLIT_, DK = DK_, DV = DV_;
  static constexpr int DKP = cround(DK, 16), DVP = cround(DV, 16);
  // per-thread channel halves (multiples of 4 so rows stay 8/16-byte aligned)
  static constexpr int DK0 = cround((DK + 1) / 2, 4), DK1 = DK - DK0;
  static constexpr int DV0 = cround((DV + 1) / 2, 8), DV1 = DV - DV0;
  static constexpr int DKH = cmax(DK0, DK1), DVH = cmax(DV0, DV1);
  // K-major strides (bytes).  Buffers whose K dimension is the token axis are
  // written column-wise (one token per thread): LBO = 144 spreads a warp's 32
  // column writes over all banks.
  static constexpr int LBO_T = 144, SBO_T = (C / 4) * LBO_T;
  static constexpr int SBO_K = (DKP / 4) * 128;  // rows of DKP values
  static constexpr int SBO_P = (C / 4) * 128;    // rows of C values
  static constexpr int VT_SZ = (DVP / 8) * SBO_T;
  static constexpr int KHT_SZ = (DKP / 8) * SBO_T;
  static constexpr int AQ_SZ = (C / 8) * SBO_K;
  static constexpr int BK_SZ = (C / 8) * SBO_K;
  static constexpr int SPT_SZ = (DVP / 8) * SBO_K;
  static constexpr int P_SZ = (C / 8) * SBO_P;
  static constexpr int OFF_VT = 0;
  static constexpr int OFF_AQ = OFF_VT + SPLIT * VT_SZ;
  static constexpr int OFF_BK = OFF_AQ + SPLIT * AQ_SZ;
  static constexpr int OFF_KHT = OFF_BK + SPLIT * BK_SZ;
  static constexpr int OFF_SPT = OFF_KHT + SPLIT * KHT_SZ;
  static constexpr int OFF_P = OFF_AQ;  // P reuses the first-stage operand space
  static constexpr int END_DATA = OFF_SPT + SPLIT * SPT_SZ;
  // M = 128 MMAs read 16 row groups of an A operand even when fewer rows are
  // real; those reads must stay inside the allocation (their rows are ignored).
  static constexpr int END_VT = OFF_VT + (SPLIT - 1) * VT_SZ + 16 * SBO_T;
  static constexpr int END_AQ = OFF_AQ + (SPLIT - 1) * AQ_SZ + 16 * SBO_K;
  static constexpr int END_P = OFF_P + (SPLIT - 1) * P_SZ + 16 * SBO_P;
  static constexpr int SMEM = cmax(cmax(END_DATA, END_VT), cmax(END_AQ, END_P));
  // TMEM columns
  static constexpr int TM_P = 0, TM_O = C, TM_DS = C + DVP;
  static constexpr int TM_COLS = pow2ceil(C + DVP + DKP);
  static_assert(TM_COLS <= 512, "TMEM budget");
  static_assert(SMEM <= 200 * 1024, "shared-memory budget");
  static_assert(DK % 4 == 0 && DV % 4 == 0 && DK1 > 0 && DV1 > 0, "head dims");
  static_assert(C == 64 || C == 128, "chunk");
};

// Store one operand value (tf32, plus its tf32 remainder when SPLIT == 2).
template <int SPLIT>
__device__ __forceinline__ void st_op(uint8_t* base, int copy_bytes, uint32_t off, float x) {
  const float hi = to_tf32(x);
  *reinterpret_cast<float*>(base + off) = hi;
  if constexpr (SPLIT == 2) *reinterpret_cast<float*>(base + copy_bytes + off) = to_tf32(x - hi);
}
template <int SPLIT>
__device__ __forceinline__ void st_op4(uint8_t* base, int copy_bytes, uint32_t off, float x0, float x1, float x2,
                                       float x3) {
  const float4 hi = make_float4(to_tf32(x0), to_tf32(x1), to_tf32(x2), to_tf32(x3));
  *reinterpret_cast<float4*>(base + off) = hi;
  if constexpr (SPLIT == 2)
    *reinterpret_cast<float4*>(base + copy_bytes + off) =
        make_float4(to_tf32(x0 - hi.x), to_tf32(x1 - hi.y), to_tf32(x2 - hi.z), to_tf32(x3 - hi.w));
}

// Predicated load of `cnt` (multiple of 4, <= MAXN) consecutive elements.
template <int MAXN, typename T>
__device__ __forceinline__ void load_part(const T* p, float* out, int cnt) {
#pragma unroll
  for (int g = 0; g < MAXN / 4; ++g)
    if (4 * g < cnt) load_row<4>(p + 4 * g, out + 4 * g);
}

// Loads `n8` x 8 consecutive TMEM columns of this warp's 32 lanes (warp-collective).
template <int MAXN>
__device__ __forceinline__ void tmem_row(uint32_t taddr, float* v, int cnt) {
#pragma unroll
  for (int c = 0; c < MAXN; c += 16) {
    if (c + 16 <= cround(cnt, 8)) {
      tmem_ld16(taddr + c, v + c);
    } else if (c + 8 <= cround(cnt, 8)) {
      tmem_ld8(taddr + c, v + c);
    }
  }
  tmem_ld_wait();
}

template <int C, int SPLIT, int DK, int DV, typename TIN, typename TOUT>
__global__ void __launch_bounds__(256, 1) gla_fwd_kernel(const GlaArgs a) {
  using Cfg = FwdCfg<C, SPLIT, DK, DV>;
  constexpr int DKH = Cfg::DKH, DVH = Cfg::DVH, DKP = Cfg::DKP, DVP = Cfg::DVP;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ float s_wtot[8][DKH];
  __shared__ float s_red[256];
  __shared__ uint64_t s_bar;
  __shared__ uint32_t s_tmem;
  __shared__ int s_range_bad;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = tid & 127, half = tid >> 7, wq = warp & 3;
  const int nseq = a.B * a.H;
  const int bh = blockIdx.x % nseq, seg = blockIdx.x / nseq;
  const int b = bh / a.H, h = bh % a.H;
  const int hz = a.gate_heads == 1 ? 0 : h;
  const int c_begin = (int)((long long)seg * a.nchunks / a.nseg);
  const int c_end = (int)((long long)(seg + 1) * a.nchunks / a.nseg);
  const int kofs = half ? Cfg::DK0 : 0, kcnt = half ? Cfg::DK1 : Cfg::DK0;
  const int vofs = half ? Cfg::DV0 : 0, vcnt = half ? Cfg::DV1 : Cfg::DV0;
  const bool tok = t < C;       // this thread owns a token row of the chunk
  const bool state_thr = t < DV;  // this thread owns state row j = t (its channel half)
  const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;

  if (warp == 0) {
    tmem_alloc(&s_tmem, Cfg::TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&s_bar, 1);
    fence_mbar_init();
    s_range_bad = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t sbase = smem_u32(smem);
  uint32_t phase = 0;
  bool timed_out = false;

  float S[DKH];    // state S[kofs + i][t] (fp32 carry)
  float Gacc[DKH]; // summed log decay of this CTA's segment (first sweep)
#pragma unroll
  for (int i = 0; i < DKH; ++i) S[i] = 0.f, Gacc[i] = 0.f;

  auto mma_prod = [&](uint32_t dcol, uint32_t offA, uint32_t szA, uint32_t lboA, uint32_t sboA, uint32_t offB,
                      uint32_t szB, uint32_t lboB, uint32_t sboB, int ksteps, uint32_t idesc, bool acc) {
    constexpr int nterm = SPLIT == 1 ? 1 : 3;
#pragma unroll 1
    for (int term = 0; term < nterm; ++term) {
      const uint32_t oa = offA + (term == 2 ? szA : 0u);  // terms: hi*hi, hi*lo, lo*hi
      const uint32_t ob = offB + (term == 1 ? szB : 0u);
#pragma unroll 1
      for (int s = 0; s < ksteps; ++s)
        mma_tf32(tmem + dcol, sdesc(sbase + oa + 2u * s * lboA, lboA, sboA), sdesc(sbase + ob + 2u * s * lboB, lboB, sboB),
                 idesc, (acc || term > 0 || s > 0) ? 1u : 0u);
    }
  };
  auto wait_mma = [&]() {
    if (!mbar_wait(&s_bar, phase, kSpinLimitNs)) timed_out = true;
    phase ^= 1u;
    tc_fence_after();
  };

  auto chunk = [&](auto out_tag, int n) {
    constexpr bool OUT = decltype(out_tag)::value;
    const int p = n * C + t;
    const bool valid = tok && p < a.L;
    long long grow = 0;
    if (valid) grow = (long long)b * a.L + scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode);
    float qv[DKH], kv[DKH], av[DKH], vv[DVH];
#pragma unroll
    for (int i = 0; i < DKH; ++i) qv[i] = 0.f, kv[i] = 0.f, av[i] = 0.f;
#pragma unroll
    for (int i = 0; i < DVH; ++i) vv[i] = 0.f;
    if (valid) {
      const size_t rk = ((size_t)grow * a.H + h) * DK + kofs;
      load_part<DKH>(reinterpret_cast<const TIN*>(a.k) + rk, kv, kcnt);
      if (OUT) load_part<DKH>(reinterpret_cast<const TIN*>(a.q) + rk, qv, kcnt);
      load_part<DVH>(reinterpret_cast<const TIN*>(a.v) + ((size_t)grow * a.H + h) * DV + vofs, vv, vcnt);
      load_part<DKH>(a.z + ((size_t)grow * a.gate_heads + hz) * DK + kofs, av, kcnt);
#pragma unroll
      for (int i = 0; i < DKH; ++i)
        if (i < kcnt) av[i] = a.inv_tau * log_sigmoid(av[i]);
    }
    // inclusive cumsum of the log decay over the chunk's tokens (per channel)
#pragma unroll
    for (int i = 0; i < DKH; ++i) {
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, av[i], off);
        if (lane >= off) av[i] += y;
      }
    }
    if (lane == 31) {
#pragma unroll
      for (int i = 0; i < DKH; ++i) s_wtot[warp][i] = av[i];
    }
    __syncthreads();
    float rv[DKH], gv[DKH];
    constexpr int REFW = C / 64;  // warps before the reference token (C/2 - 1)
#pragma unroll
    for (int i = 0; i < DKH; ++i) {
      float pre = 0.f, tot = 0.f, ref = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float w = s_wtot[half * 4 + u][i];
        if (u < wq) pre += w;
        if (u < REFW) ref += w;
        tot += w;
      }
      av[i] += pre;  // b_t
      rv[i] = ref;   // r
      gv[i] = tot;   // Gamma
    }
    // operands
    bool bad = false;
    if (tok) {
#pragma unroll
      for (int i = 0; i < DKH; ++i) {
        if (i < kcnt) {
          const float d = av[i] - rv[i];
          bad |= fabsf(d) > 80.f;
          const float ek = expf(-d);
          st_op<SPLIT>(smem + Cfg::OFF_KHT, Cfg::KHT_SZ, kmajor_off(kofs + i, t, Cfg::LBO_T, Cfg::SBO_T),
                       kv[i] * ek * expf(gv[i] - rv[i]));
          if (OUT) {
            qv[i] *= expf(d);
            kv[i] *= ek;
          }
        }
      }
#pragma unroll
      for (int j = 0; j < DVH; ++j)
        if (j < vcnt) st_op<SPLIT>(smem + Cfg::OFF_VT, Cfg::VT_SZ, kmajor_off(vofs + j, t, Cfg::LBO_T, Cfg::SBO_T), vv[j]);
      if (OUT) {
#pragma unroll
        for (int g = 0; g < DKH / 4; ++g) {
          if (4 * g < kcnt) {
            const uint32_t off = kmajor_off(t, kofs + 4 * g, 128, Cfg::SBO_K);
            st_op4<SPLIT>(smem + Cfg::OFF_AQ, Cfg::AQ_SZ, off, qv[4 * g], qv[4 * g + 1], qv[4 * g + 2], qv[4 * g + 3]);
            st_op4<SPLIT>(smem + Cfg::OFF_BK, Cfg::BK_SZ, off, kv[4 * g], kv[4 * g + 1], kv[4 * g + 2], kv[4 * g + 3]);
          }
        }
        if (half == 1) {
#pragma unroll
          for (int c = DK; c < DKP; c += 4) {
            const uint32_t off = kmajor_off(t, c, 128, Cfg::SBO_K);
            st_op4<SPLIT>(smem + Cfg::OFF_AQ, Cfg::AQ_SZ, off, 0.f, 0.f, 0.f, 0.f);
            st_op4<SPLIT>(smem + Cfg::OFF_BK, Cfg::BK_SZ, off, 0.f, 0.f, 0.f, 0.f);
          }
        }
      }
    }
    if (OUT && state_thr) {
      // B operand of O += qbar * S': row j = t of S'^T, S' = diag(e^r) S_in
#pragma unroll
      for (int g = 0; g < DKH / 4; ++g) {
        if (4 * g < kcnt) {
          float e[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) e[u] = expf(rv[4 * g + u]) * S[4 * g + u];
          st_op4<SPLIT>(smem + Cfg::OFF_SPT, Cfg::SPT_SZ, kmajor_off(t, kofs + 4 * g, 128, Cfg::SBO_K), e[0], e[1], e[2],
                        e[3]);
        }
      }
      if (half == 1) {
#pragma unroll
        for (int c = DK; c < DKP; c += 4)
          st_op4<SPLIT>(smem + Cfg::OFF_SPT, Cfg::SPT_SZ, kmajor_off(t, c, 128, Cfg::SBO_K), 0.f, 0.f, 0.f, 0.f);
      }
    }
    if (bad) s_range_bad = 1;
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      if (OUT) {
        mma_prod(Cfg::TM_P, Cfg::OFF_AQ, Cfg::AQ_SZ, 128, Cfg::SBO_K, Cfg::OFF_BK, Cfg::BK_SZ, 128, Cfg::SBO_K, DKP / 8,
                 idesc_tf32(128, C, false, false), false);
        mma_prod(Cfg::TM_O, Cfg::OFF_AQ, Cfg::AQ_SZ, 128, Cfg::SBO_K, Cfg::OFF_SPT, Cfg::SPT_SZ, 128, Cfg::SBO_K, DKP / 8,
                 idesc_tf32(128, DVP, false, false), false);
      }
      mma_prod(Cfg::TM_DS, Cfg::OFF_VT, Cfg::VT_SZ, Cfg::LBO_T, Cfg::SBO_T, Cfg::OFF_KHT, Cfg::KHT_SZ, Cfg::LBO_T,
               Cfg::SBO_T, C / 8, idesc_tf32(128, DKP, false, false), false);
      mma_commit(&s_bar);
    }
    wait_mma();
    // state carry: S <- diag(e^Gamma) S + khat^T V   (TMEM lane j holds row j of (khat^T V)^T)
    {
      float ds[cround(DKH, 16)];
      tmem_row<cround(DKH, 16)>(tmem + lane_base + Cfg::TM_DS + kofs, ds, kcnt);
      if (state_thr) {
#pragma unroll
        for (int i = 0; i < DKH; ++i)
          if (i < kcnt) S[i] = expf(gv[i]) * S[i] + ds[i];
      }
      if (!OUT) {
#pragma unroll
        for (int i = 0; i < DKH; ++i) Gacc[i] += gv[i];
      }
    }
    if (OUT) {
      // P row t: mask s <= t, store as the A operand of P V
#pragma unroll
      for (int cb = 0; cb < C / 2; cb += 16) {
        float pv[16];
        tmem_ld16(tmem + lane_base + Cfg::TM_P + half * (C / 2) + cb, pv);
        tmem_ld_wait();
        if (tok) {
          const int s0 = half * (C / 2) + cb;
#pragma unroll
          for (int u = 0; u < 16; u += 4) {
            float x[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) x[w] = (s0 + u + w <= t) ? pv[u + w] : 0.f;
            st_op4<SPLIT>(smem + Cfg::OFF_P, Cfg::P_SZ, kmajor_off(t, s0 + u, 128, Cfg::SBO_P), x[0], x[1], x[2], x[3]);
          }
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (tid == 0) {
        mma_prod(Cfg::TM_O, Cfg::OFF_P, Cfg::P_SZ, 128, Cfg::SBO_P, Cfg::OFF_VT, Cfg::VT_SZ, Cfg::LBO_T, Cfg::SBO_T, C / 8,
                 idesc_tf32(128, DVP, false, false), true);
        mma_commit(&s_bar);
      }
      wait_mma();
      float ov[cround(DVH, 16)];
      tmem_row<cround(DVH, 16)>(tmem + lane_base + Cfg::TM_O + vofs, ov, vcnt);
      const size_t ro = ((size_t)grow * a.H + h) * DV + vofs;
      if (valid) {
        TOUT* op = reinterpret_cast<TOUT*>(a.o) + ro;
        if (half == 0) store_row<Cfg::DV0>(op, ov);
        else store_row<Cfg::DV1>(op, ov);
      }
      if (a.y != nullptr && a.r != nullptr) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < DVH; ++i)
          if (i < vcnt) ss += ov[i] * ov[i];
        s_red[tid] = valid ? ss : 0.f;
        __syncthreads();
        const float inv = rsqrtf((s_red[t] + s_red[t + 128]) / (float)DV + a.eps);
        if (valid) {
          float rr[DVH], yv[DVH];
          load_part<DVH>(reinterpret_cast<const TIN*>(a.r) + ro, rr, vcnt);
#pragma unroll
          for (int i = 0; i < DVH; ++i) {
            const float gmm = (a.gamma != nullptr && i < vcnt) ? __ldg(a.gamma + vofs + i) : 1.f;
            const float sw = rr[i] / (1.f + expf(-rr[i]));
            yv[i] = sw * ov[i] * inv * gmm;
          }
          TOUT* yp = reinterpret_cast<TOUT*>(a.y) + ro;
          if (half == 0) store_row<Cfg::DV0>(yp, yv);
          else store_row<Cfg::DV1>(yp, yv);
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
    for (int n = c_begin; n < c_end; ++n) chunk(std::false_type{}, n);
    if (state_thr) {
      float* dst = a.seg_S + ((size_t)rec * DV + t) * DK + kofs;
#pragma unroll
      for (int i = 0; i < DKH; ++i)
        if (i < kcnt) dst[i] = S[i];
    }
    if (t == 0) {
#pragma unroll
      for (int i = 0; i < DKH; ++i)
        if (i < kcnt) a.seg_gam[(size_t)rec * DKP + kofs + i] = Gacc[i];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) st_release(a.flags + rec, 1u);
    // combine the records of all earlier segments of this sequence
    if (seg > 0) {
      if (tid == 0) {
        for (int s2 = 0; s2 < seg; ++s2)
          if (!wait_flag(a.flags + bh * a.nseg + s2, 1u, kSpinLimitNs)) timed_out = true;
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < DKH; ++i) S[i] = 0.f;
      if (state_thr) {
        for (int s2 = 0; s2 < seg; ++s2) {
          const size_t r2 = (size_t)bh * a.nseg + s2;
          const float* src = a.seg_S + (r2 * DV + t) * DK + kofs;
#pragma unroll
          for (int i = 0; i < DKH; ++i)
            if (i < kcnt) S[i] = expf(__ldcg(a.seg_gam + r2 * DKP + kofs + i)) * S[i] + __ldcg(src + i);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < DKH; ++i) S[i] = 0.f;
    }
  }
  // ---------------------------------------------------------------- sweep 2
  for (int n = c_begin; n < c_end; ++n) chunk(std::true_type{}, n);

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, Cfg::TM_COLS);
  if (timed_out) set_status(a.status, DIG_ERR_DEVICE_TIMEOUT);
  if (tid == 0 && s_range_bad) set_status(a.status, DIG_ERR_GATE_RANGE);
  if (a.nseg > 1 && tid == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(a.done, 1u);
    if (prev == gridDim.x - 1) {  // every CTA is past its flag reads: reset for the next call
      for (int i = 0; i < nseq * a.nseg; ++i) a.flags[i] = 0u;
      *a.done = 0u;
      __threadfence();
    }
  }
}

// ------------------------------------------------------------------ launch
template <int C, int SPLIT, int DK, int DV, typename TIN, typename TOUT>
static cudaError_t launch_one(const GlaArgs& a, int grid, bool coop, cudaStream_t s) {
  using Cfg = FwdCfg<C, SPLIT, DK, DV>;
  auto kern = gla_fwd_kernel<C, SPLIT, DK, DV, TIN, TOUT>;
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

template <int C, int SPLIT, int DK, int DV, typename TIN, typename TOUT>
static int occupancy_one() {
  using Cfg = FwdCfg<C, SPLIT, DK, DV>;
  auto kern = gla_fwd_kernel<C, SPLIT, DK, DV, TIN, TOUT>;
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
    if (v.tout == DIG_BF16) return occ ? (*occ = occupancy_one<128, 1, DK, DV, bf, bf>(), cudaSuccess)
                                       : launch_one<128, 1, DK, DV, bf, bf>(a, grid, coop, s);
    return occ ? (*occ = occupancy_one<128, 1, DK, DV, bf, float>(), cudaSuccess)
               : launch_one<128, 1, DK, DV, bf, float>(a, grid, coop, s);
  }
  if (v.tout == DIG_BF16) return occ ? (*occ = occupancy_one<64, 2, DK, DV, float, bf>(), cudaSuccess)
                                     : launch_one<64, 2, DK, DV, float, bf>(a, grid, coop, s);
  return occ ? (*occ = occupancy_one<64, 2, DK, DV, float, float>(), cudaSuccess)
             : launch_one<64, 2, DK, DV, float, float>(a, grid, coop, s);
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
