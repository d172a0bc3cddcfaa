// gla_fwd_tma.cu -- the GLA forward's per-chunk outputs (o, and the fused
// Swish(r) * RMSNorm(o) epilogue y) with tile copies by the tensor memory
// accelerator.
//
// Same chunk algebra as gla_chunk_out_kernel (gla_fwd.cu; DiG slides, GLA eq.
// (6)-(8), the output gate eq. (9)-(10)): per (sequence, chunk) unit with entry
// state S_n,
//     qbar = q 2^(b-r),  kbar = k 2^(r-b),  S' = diag(2^r) S_n
//     [P | O] = qbar [kbar ; S'^T]^T,   P masked to s <= t,   O += P V
//     y = Swish(r) * O / sqrt(mean(O^2) + eps) * gamma
// with the operands as two bf16 terms each (the precision of the exact path).
// What differs is the data path: q, k, v, r arrive as whole tiles by TMA (one
// box for the row scan orders, 16-row column segments for the column orders;
// the scan permutation is the box coordinates), the gate factors and the entry
// state by TMA / bulk copies, o and y leave by TMA tile stores.  Each input
// slot is refilled for the next unit as soon as this unit has consumed it (q, k
// after the first product, v after the second, the state after the operands
// are formed), so those loads run under this unit's work.  Only bf16 inputs with
// d_k = 32, d_v = 64 and 128-token chunks that tile the sequence (and, for the
// column orders, 16-row column segments) take this kernel.
#include "gla_strong.cuh"
#include "tma_tiles.cuh"

namespace dig {

struct OutMaps {
  CUtensorMap q, k, v, r;  // inputs (bf16)
  CUtensorMap eq;          // gate factors 2^(b - r), [B * gate_heads * L][d_k] fp32 (scan order)
  CUtensorMap o, y;        // outputs (bf16 or fp32)
};

template <typename TOUT>
struct TmaOutCfg {
  static constexpr int C = 128, DK = 32, DV = 64, NB = C + DV;
  static constexpr int RBK = 64, RBV = 128;
  static constexpr int OFF_QH = 0, OFF_QL = 8192;       // qbar terms, [C][DK] bf16, 64-byte swizzle (q lands in hi)
  static constexpr int OFF_BH = 16384, OFF_BL = 28672;  // [kbar ; S'^T] terms, [C + DV][DK] (k lands in hi)
  static constexpr int OFF_V = 40960;                   // v, [C][DV] bf16, 128-byte swizzle
  static constexpr int OFF_R = 57344;                   // r, then y (bf16 outputs) in place
  static constexpr int OFF_EQ = 73728;                  // gate factors [C][DK] fp32, 128-byte swizzle; then o staging
  static constexpr int OFF_S = 90112;                   // raw entry state [DV][DK] fp32
  static constexpr int END = 98304;
  static constexpr int SMEM = END + 1024;
  static constexpr int TM_P = 0, TM_O = 128, TM_COLS = 256;
  static constexpr bool F32OUT = std::is_same<TOUT, float>::value;
  // fp32 staging (channels 0-31 / 32-63 of o and y), over slots free by then
  static constexpr int OFF_OLO = OFF_EQ, OFF_OHI = OFF_QH, OFF_YLO = OFF_BH, OFF_YHI = OFF_V;
  static constexpr uint32_t QK_BYTES = 2 * C * RBK, V_BYTES = C * RBV, R_BYTES = C * RBV, EQ_BYTES = C * DK * 4;
  static constexpr uint32_t S_BYTES = DV * DK * 4, GCH_BYTES = DK * 4;
};

struct TmaOutSmem {
  alignas(16) float gch[32];  // 2^r of the unit's chunk
  float gamma[64];
  float red[256];             // row sums of squares of the two channel halves
  uint64_t bar_qk, bar_s, bar_eq, bar_v, bar_r, bar_g0, bar_g1;
  uint32_t tmem;
  int abort;
};

// Masks P (TMEM lane = row; keep column <= row, or >= row when `upper`) and
// rewrites it in place as two bf16 terms: K-step k (16 columns) becomes its hi
// term at 16 k .. 16 k + 7 and its lo term at 16 k + 8 .. 16 k + 15.
__device__ __forceinline__ void mask_to_bf16x2(uint32_t tmem, uint32_t region, bool upper) {
  const int tid = threadIdx.x, t = tid & 127, wq = t >> 5, half = tid >> 7;
  const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
    const int s0 = half * 64 + 32 * kk;
    const bool zero_block = upper ? (s0 < 32 * wq) : (s0 > 32 * wq);  // warp-uniform
    float pv[32];
    if (!zero_block) {
      tmem_ld32(tmem + lane_base + region + s0, pv);
      tmem_ld_wait();
      if (s0 == 32 * wq) {
#pragma unroll
        for (int e = 0; e < 32; ++e) pv[e] = (upper ? (s0 + e >= t) : (s0 + e <= t)) ? pv[e] : 0.f;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) pv[e] = 0.f;
    }
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {  // the block's two K-steps
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float x0 = pv[16 * ks + 2 * e], x1 = pv[16 * ks + 2 * e + 1];
        const __nv_bfloat162 hi = __floats2bfloat162_rn(x0, x1);
        const __nv_bfloat162 lo = __floats2bfloat162_rn(x0 - __low2float(hi), x1 - __high2float(hi));
        pk[e] = *reinterpret_cast<const uint32_t*>(&hi);
        pk[8 + e] = *reinterpret_cast<const uint32_t*>(&lo);
      }
      tmem_st16(tmem + lane_base + region + s0 + 16 * ks, pk);
    }
  }
}

// hi and lo bf16 terms of 8 values, packed (hi: x, lo: y of the result).
__device__ __forceinline__ void split8(const float* v, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v[2 * w], v[2 * w + 1]);
    const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * w] - __low2float(a), v[2 * w + 1] - __high2float(a));
    h[w] = *reinterpret_cast<const uint32_t*>(&a);
    l[w] = *reinterpret_cast<const uint32_t*>(&b);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

template <typename TOUT>
__global__ void __launch_bounds__(256, 2) gla_out_tma_kernel(const __grid_constant__ OutMaps mp, const GlaArgs a) {
  using TC = TmaOutCfg<TOUT>;
  constexpr int C = TC::C, DK = TC::DK, DV = TC::DV;
  extern __shared__ uint8_t smem_raw[];
  __shared__ TmaOutSmem sh;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t sb = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int nunits = a.B * a.H * a.nchunks;
  const uint64_t spin = a.spin_ns ? a.spin_ns : kSpinLimitNs;
  const bool with_y = a.y != nullptr && a.r != nullptr;
  if (warp == 0) {
    tmem_alloc(&sh.tmem, TC::TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&sh.bar_qk, 1);
    mbar_init(&sh.bar_s, 1);
    mbar_init(&sh.bar_eq, 1);
    mbar_init(&sh.bar_v, 1);
    mbar_init(&sh.bar_r, 1);
    mbar_init(&sh.bar_g0, 1);
    mbar_init(&sh.bar_g1, 1);
    sh.abort = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem;
  const int t = tid & 127, wq = t >> 5, half = tid >> 7;
  const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
  bool timed_out = false;
  auto wait_bar = [&](uint64_t* bar, uint32_t parity) {
    if (!mbar_wait(bar, parity, spin)) {
      timed_out = true;
      sh.abort = 1;
    }
  };
  // thread 0's loads in flight (barrier and phase), and the last product group: drained before exit
  uint64_t* const lbar[5] = {&sh.bar_qk, &sh.bar_s, &sh.bar_eq, &sh.bar_v, &sh.bar_r};
  bool pend[5] = {false, false, false, false, false};
  uint32_t pph[5] = {0, 0, 0, 0, 0};
  int last_g = -1;
  uint32_t last_ph = 0;
  bool last_done = true;
  enum { QK = 0, ST = 1, EQ = 2, VV = 3, RR = 4 };
  auto issue = [&](int which, const TileUnit& T, int u, uint32_t phase) {
    pend[which] = true;
    pph[which] = phase;
    switch (which) {
      case QK:
        mbar_arrive_expect_tx(&sh.bar_qk, TC::QK_BYTES);
        tile_load<C>(sb + TC::OFF_QH, mp.q, T.h * DK, T, a, TC::RBK, &sh.bar_qk);
        tile_load<C>(sb + TC::OFF_BH, mp.k, T.h * DK, T, a, TC::RBK, &sh.bar_qk);
        break;
      case ST:
        mbar_arrive_expect_tx(&sh.bar_s, TC::S_BYTES + TC::GCH_BYTES);
        bulk_copy_g2s(sb + TC::OFF_S, a.dsn + (size_t)u * DV * DK, TC::S_BYTES, &sh.bar_s);
        bulk_copy_g2s(smem_u32(sh.gch), a.gCH + ((size_t)T.bz * a.nchunks + T.n) * 4 * DK, TC::GCH_BYTES, &sh.bar_s);
        break;
      case EQ:
        mbar_arrive_expect_tx(&sh.bar_eq, TC::EQ_BYTES);
        tma_load_2d(sb + TC::OFF_EQ, mp.eq, 0, T.bz * a.L + T.n * C, &sh.bar_eq);
        break;
      case VV:
        mbar_arrive_expect_tx(&sh.bar_v, TC::V_BYTES);
        tile_load<C>(sb + TC::OFF_V, mp.v, T.h * DV, T, a, TC::RBV, &sh.bar_v);
        break;
      default:
        mbar_arrive_expect_tx(&sh.bar_r, TC::R_BYTES);
        tile_load<C>(sb + TC::OFF_R, mp.r, T.h * DV, T, a, TC::RBV, &sh.bar_r);
        break;
    }
  };
  auto waited = [&](int which) {
    if (tid == 0 && !timed_out) pend[which] = false;
  };

  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  if (tid < DV) sh.gamma[tid] = a.gamma != nullptr ? a.gamma[tid] : 1.f;
  if (tid == 0 && (int)blockIdx.x < nunits) {
    const TileUnit T0(a, blockIdx.x, C);
    issue(QK, T0, blockIdx.x, 0);
    issue(ST, T0, blockIdx.x, 0);
    issue(EQ, T0, blockIdx.x, 0);
    issue(VV, T0, blockIdx.x, 0);
    if (with_y) issue(RR, T0, blockIdx.x, 0);
  }
  __syncthreads();  // gamma

  int it = 0;
  bool any_strong = false;  // uniform: a unit of this CTA has a chunk flagged by the gate kernel (strong gate)
  for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++it) {
    const uint32_t ph = it & 1;
    const TileUnit T(a, u, C);
    const bool skip = strong::flagged(a, T.bz, T.n);  // its o and y come after the loop
    const int un = u + gridDim.x;
    const bool has_next = un < nunits;
    auto can_issue = [&]() { return tid == 0 && !timed_out && !sh.abort; };

    // ---- 1. operands: qbar, kbar and S'^T rows as hi / lo bf16 terms
    wait_bar(&sh.bar_qk, ph);
    waited(QK);
    wait_bar(&sh.bar_s, ph);
    waited(ST);
    wait_bar(&sh.bar_eq, ph);
    waited(EQ);
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int k = tid + 256 * m;  // 16-byte chunk of the q / k tiles
      const int i = k >> 2, c = (k & 3) ^ ((i >> 1) & 3);
      const int ti = T.rev ? C - 1 - i : i;
      const float4 e0 = lds128f(sb + TC::OFF_EQ + swz_off<128>(ti, 2 * c));
      const float4 e1 = lds128f(sb + TC::OFF_EQ + swz_off<128>(ti, 2 * c + 1));
      const float e[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
      const uint4 qr = lds128(sb + TC::OFF_QH + 16u * k), kr = lds128(sb + TC::OFF_BH + 16u * k);
      const uint32_t qw[4] = {qr.x, qr.y, qr.z, qr.w}, kw[4] = {kr.x, kr.y, kr.z, kr.w};
      float qv[8], kv[8];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        qv[2 * w] = bf_lo(qw[w]) * e[2 * w];
        qv[2 * w + 1] = bf_hi(qw[w]) * e[2 * w + 1];
        kv[2 * w] = bf_lo(kw[w]) * __frcp_rn(e[2 * w]);
        kv[2 * w + 1] = bf_hi(kw[w]) * __frcp_rn(e[2 * w + 1]);
      }
      uint4 hi, lo;
      split8(qv, hi, lo);
      sts128(sb + TC::OFF_QH + 16u * k, hi);
      sts128(sb + TC::OFF_QL + 16u * k, lo);
      split8(kv, hi, lo);
      sts128(sb + TC::OFF_BH + 16u * k, hi);
      sts128(sb + TC::OFF_BL + 16u * k, lo);
    }
    {  // S'^T rows: value channel j, key channels 8 cc .. 8 cc + 7, after the C kbar rows
      const int j = tid >> 2, cc = tid & 3;
      const uint32_t src = sb + TC::OFF_S + (uint32_t)(j * DK + 8 * cc) * 4u;
      const float4 s0 = lds128f(src), s1 = lds128f(src + 16);
      const float4 r0 = *reinterpret_cast<const float4*>(&sh.gch[8 * cc]);
      const float4 r1 = *reinterpret_cast<const float4*>(&sh.gch[8 * cc + 4]);
      const float sv[8] = {s0.x * r0.x, s0.y * r0.y, s0.z * r0.z, s0.w * r0.w,
                           s1.x * r1.x, s1.y * r1.y, s1.z * r1.z, s1.w * r1.w};
      uint4 hi, lo;
      split8(sv, hi, lo);
      sts128(sb + TC::OFF_BH + swz_off<64>(C + j, cc), hi);
      sts128(sb + TC::OFF_BL + swz_off<64>(C + j, cc), lo);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (can_issue() && has_next) issue(ST, TileUnit(a, un, C), un, ph ^ 1u);  // the state slot is free

    // ---- 2. [P | O] = qbar [kbar ; S'^T]^T  (term pairs hi.hi, hi.lo, lo.hi)
    if (can_issue()) {
      const uint32_t A[2] = {sb + TC::OFF_QH, sb + TC::OFF_QL}, Bo[2] = {sb + TC::OFF_BH, sb + TC::OFF_BL};
      bool first = true;
#pragma unroll
      for (int ia = 0; ia < 2; ++ia)
#pragma unroll
        for (int jb = 0; jb < 2; ++jb) {
          if (ia + jb > 1) continue;
#pragma unroll
          for (int s = 0; s < DK / 16; ++s) {
            mma_bf16(tmem + TC::TM_P, sdesc_sw<64>(A[ia] + 32 * s), sdesc_sw<64>(Bo[jb] + 32 * s),
                     idesc_bf16(128, TC::NB), first ? 0u : 1u);
            first = false;
          }
        }
      mma_commit(&sh.bar_g0);
      last_g = 0;
      last_ph = ph;
      last_done = false;
    }
    wait_bar(&sh.bar_g0, ph);
    if (tid == 0 && last_g == 0 && !timed_out) last_done = true;
    tc_fence_after();
    if constexpr (!TC::F32OUT) {  // the qbar and [kbar ; S'] slots are free: the next unit's q, k
      if (can_issue() && has_next) issue(QK, TileUnit(a, un, C), un, ph ^ 1u);
    }

    // ---- 3. P masked to s <= t (scan order), as bf16 terms in TMEM
    mask_to_bf16x2(tmem, TC::TM_P, T.rev);
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- 4. O += P V  (once the v tile has landed)
    wait_bar(&sh.bar_v, ph);
    waited(VV);
    if (can_issue()) {
#pragma unroll
      for (int s = 0; s < C / 16; ++s)
#pragma unroll
        for (int ia = 0; ia < 2; ++ia)
          mma_bf16_ts(tmem + TC::TM_O, tmem + TC::TM_P + 16 * s + 8 * ia, sdesc_sw<128>(sb + TC::OFF_V + 2048 * s),
                      idesc_bf16(128, DV, false, true), 1);
      mma_commit(&sh.bar_g1);
      last_g = 1;
      last_ph = ph;
      last_done = false;
    }
    wait_bar(&sh.bar_g1, ph);
    if (tid == 0 && last_g == 1 && !timed_out) last_done = true;
    tc_fence_after();
    if constexpr (!TC::F32OUT) {  // the v slot is free
      if (can_issue() && has_next) issue(VV, TileUnit(a, un, C), un, ph ^ 1u);
    }

    // ---- 5. epilogue: o rows of this thread's token and channel half; y = Swish(r) o / rms(o) gamma
    float ov[32];
    tmem_ld32(tmem + lane_base + TC::TM_O + 32 * half, ov);
    tmem_ld_wait();
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) ss = fmaf(ov[e], ov[e], ss);
    sh.red[tid] = ss;
    if (with_y) {
      wait_bar(&sh.bar_r, ph);
      waited(RR);
    }
    tc_fence_before();
    __syncthreads();  // row sums; every TMEM read of O done
    float yv[32];
    if (with_y) {
      const float inv = rsqrtf((sh.red[t] + sh.red[t + 128]) / (float)DV + a.eps);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const uint4 rr = lds128(sb + TC::OFF_R + swz_off<128>(t, 4 * half + m));
        const uint32_t rw[4] = {rr.x, rr.y, rr.z, rr.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int c = 8 * m + 2 * w;
          const float ra = bf_lo(rw[w]), rb = bf_hi(rw[w]);
          const float swa = __fdividef(ra, 1.f + ex2(-ra * kLog2e)), swb = __fdividef(rb, 1.f + ex2(-rb * kLog2e));
          yv[c] = swa * ov[c] * inv * sh.gamma[32 * half + c];
          yv[c + 1] = swb * ov[c + 1] * inv * sh.gamma[32 * half + c + 1];
        }
      }
    }
    if constexpr (!TC::F32OUT) {
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        sts128(sb + TC::OFF_EQ + swz_off<128>(t, 4 * half + m),
               make_uint4(pack_bf16x2(ov[8 * m], ov[8 * m + 1]), pack_bf16x2(ov[8 * m + 2], ov[8 * m + 3]),
                          pack_bf16x2(ov[8 * m + 4], ov[8 * m + 5]), pack_bf16x2(ov[8 * m + 6], ov[8 * m + 7])));
        if (with_y)  // over this thread's own r values
          sts128(sb + TC::OFF_R + swz_off<128>(t, 4 * half + m),
                 make_uint4(pack_bf16x2(yv[8 * m], yv[8 * m + 1]), pack_bf16x2(yv[8 * m + 2], yv[8 * m + 3]),
                            pack_bf16x2(yv[8 * m + 4], yv[8 * m + 5]), pack_bf16x2(yv[8 * m + 6], yv[8 * m + 7])));
      }
    } else {
      const uint32_t od = sb + (half ? TC::OFF_OHI : TC::OFF_OLO), yd = sb + (half ? TC::OFF_YHI : TC::OFF_YLO);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        sts128(od + swz_off<128>(t, m), make_uint4(__float_as_uint(ov[4 * m]), __float_as_uint(ov[4 * m + 1]),
                                                   __float_as_uint(ov[4 * m + 2]), __float_as_uint(ov[4 * m + 3])));
        if (with_y)
          sts128(yd + swz_off<128>(t, m), make_uint4(__float_as_uint(yv[4 * m]), __float_as_uint(yv[4 * m + 1]),
                                                     __float_as_uint(yv[4 * m + 2]), __float_as_uint(yv[4 * m + 3])));
      }
    }
    fence_async_smem();  // staging writes precede the TMA stores that read them
    __syncthreads();

    // ---- 6. stores (thread 0), then the slots the stores read are refilled
    if (tid == 0) {
      if (!timed_out && !sh.abort && !skip) {
        if constexpr (!TC::F32OUT) {
          tile_store<C>(mp.o, T.h * DV, T, a, sb + TC::OFF_EQ, TC::RBV);
          if (with_y) tile_store<C>(mp.y, T.h * DV, T, a, sb + TC::OFF_R, TC::RBV);
        } else {
          tile_store<C>(mp.o, T.h * DV, T, a, sb + TC::OFF_OLO, 128);
          tile_store<C>(mp.o, T.h * DV + 32, T, a, sb + TC::OFF_OHI, 128);
          if (with_y) {
            tile_store<C>(mp.y, T.h * DV, T, a, sb + TC::OFF_YLO, 128);
            tile_store<C>(mp.y, T.h * DV + 32, T, a, sb + TC::OFF_YHI, 128);
          }
        }
        bulk_commit();
      }
      if (has_next && !timed_out && !sh.abort) {
        bulk_wait_read_all();
        const TileUnit Tn(a, un, C);
        issue(EQ, Tn, un, ph ^ 1u);
        if (with_y) issue(RR, Tn, un, ph ^ 1u);
        if constexpr (TC::F32OUT) {
          issue(QK, Tn, un, ph ^ 1u);
          issue(VV, Tn, un, ph ^ 1u);
        }
      }
    }
    any_strong |= skip;
    if (sh.abort) break;  // uniform: read after the barrier above
  }

  // ---- drain: no copy or product outlives the CTA (each wait bounded by the normal limit)
  if (timed_out) set_status(a.status, DIG_ERR_DEVICE_TIMEOUT);
  if (tid == 0) {
    bulk_wait_all();
    for (int i = 0; i < 5; ++i)
      if (pend[i]) mbar_wait(lbar[i], pph[i], kSpinLimitNs);
    if (last_g >= 0 && !last_done) mbar_wait(last_g == 0 ? &sh.bar_g0 : &sh.bar_g1, last_ph, kSpinLimitNs);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TC::TM_COLS);
  // this CTA's units of flagged chunks, exactly in fp32, over the drained operand slots
  static_assert(TC::SMEM - 1024 >= strong::Cfg<C, DK, DV>::SMEM_OUT, "shared memory of the strong-gate phase");
  if (any_strong && !__syncthreads_or(timed_out || sh.abort))
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      const TileUnit T(a, u, C);
      if (strong::flagged(a, T.bz, T.n))
        strong::out_unit<C, DK, DV, __nv_bfloat16, TOUT>(a, u, smem_raw + (sb - smem_u32(smem_raw)));
    }
}

// ------------------------------------------------------------------ launch
// The row scan orders only: a column-order tile takes eight 16-row segment copies
// per tensor (q, k, v, r in, o, y out), whose issue by one thread lengthens every
// unit's chain beyond what the exact kernel's row-piece gathers cost (at DiG-S/2
// 1792^2 with the epilogue: 83 vs 74 us for the whole forward).
bool gla_out_tma_eligible(const GlaArgs& a, int dk, int dv, int tin, int chunk) {
  if (tin != DIG_BF16 || dk != 32 || dv != 64 || chunk != 128 || a.L % 128 != 0) return false;
  if (a.mode & 2) return false;
  return tmap_available();
}

cudaError_t launch_out_tma(const GlaArgs& a, int tout, cudaStream_t s, bool* launched) {
  *launched = false;
  constexpr int C = 128, DK = 32, DV = 64;
  const bool f32 = tout == DIG_F32;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, fp = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  OutMaps mp;
  memset(&mp, 0, sizeof(mp));
  const bool with_y = a.y != nullptr && a.r != nullptr;
  bool ok = encode_tile_map(&mp.q, a.q, bf, 2, a.H * DK, DK, 64, a, C) &&
            encode_tile_map(&mp.k, a.k, bf, 2, a.H * DK, DK, 64, a, C) &&
            encode_tile_map(&mp.v, a.v, bf, 2, a.H * DV, DV, 128, a, C) &&
            encode_tile_map(&mp.o, a.o, f32 ? fp : bf, f32 ? 4 : 2, a.H * DV, f32 ? 32 : DV, 128, a, C) &&
            tmap_rows(&mp.eq, a.gEQ, fp, 4, DK, (uint64_t)a.B * a.gate_heads * a.L, DK, C, 128);
  if (ok && with_y)
    ok = encode_tile_map(&mp.r, a.r, bf, 2, a.H * DV, DV, 128, a, C) &&
         encode_tile_map(&mp.y, a.y, f32 ? fp : bf, f32 ? 4 : 2, a.H * DV, f32 ? 32 : DV, 128, a, C);
  if (!ok) return cudaSuccess;  // not encodable: the caller runs the exact kernel
  const long long units = (long long)a.B * a.H * a.nchunks;
  cudaError_t e;
  if (f32) {
    auto k = gla_out_tma_kernel<float>;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, TmaOutCfg<float>::SMEM)) !=
        cudaSuccess)
      return e;
    e = launch_pdl(k, persistent_grid(2, units), 256, TmaOutCfg<float>::SMEM, s, mp, a);
  } else {
    auto k = gla_out_tma_kernel<__nv_bfloat16>;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  TmaOutCfg<__nv_bfloat16>::SMEM)) != cudaSuccess)
      return e;
    e = launch_pdl(k, persistent_grid(2, units), 256, TmaOutCfg<__nv_bfloat16>::SMEM, s, mp, a);
  }
  if (e == cudaSuccess) *launched = true;
  return e;
}

}  // namespace dig
