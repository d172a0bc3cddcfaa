// gla_bwd_tma.cu -- the GLA backward's per-chunk gradients (dq, dk, dv, d log alpha)
// with tile copies by the tensor memory accelerator and single-term fp16
// tensor-core operands.
//
// Same chunk algebra as gla_chunk_grad_kernel (gla_bwd.cu; DiG slides, GLA eq.
// (5)-(8) and their chain rule): per (sequence, chunk) unit, with qbar =
// q 2^(b-r), kbar = k 2^(r-b), S' = diag(2^r) S_n, Gt = diag(2^(Gamma-r)) G_n,
//     P^T = mask(kbar qbar^T),  dP^T = mask(V dO^T),  dP = mask(dO V^T)
//     dv = P^T dO + kbar Gt,  dkbar = dP^T qbar + V Gt^T,  dqbar = dP kbar + dO S'^T
//     dq = dqbar 2^(b-r),  dk = dkbar 2^(r-b)
//     d log alpha_t = sum_{u >= t in chunk} (qbar dqbar - kbar dkbar)_u + rowsum(S_{n+1} o G_n).
// What differs is the data path and the operand precision:
//   * q, k, v, dO arrive as whole tiles by TMA (one box per tensor for the row
//     scan orders, eight 16-row column segments for the column orders; the scan
//     permutation is the box coordinates, no reordered copy exists), already in
//     the 64- / 128-byte swizzled layout the tensor core reads; the gate factors,
//     chunk constants and states by TMA / bulk copies as well.
//   * Operands are converted in place to single fp16 terms (11 significant bits);
//     the masked C x C products are fp16 in TMEM.  Each product is one MMA group
//     instead of the bf16 term pairs.
//   * dq, dk, dv leave by TMA tile stores from swizzled staging, d log alpha by a
//     TMA tile add-reduction (heads sharing a gate add into one tensor).
//   * Loads of the next unit are in flight while this unit computes.
// A unit whose values leave fp16's comfortable range (a gate factor outside
// 2^+-8, an operand or masked product of magnitude 2^15 or more) is not stored;
// it is appended to a list that the exact kernel (two bf16 terms per operand)
// then processes.  Only bf16 inputs with d_k = 32, d_v = 64 and 128-token chunks
// that tile the sequence (and, for the column orders, 16-row column segments)
// take this kernel; everything else runs the exact kernel directly.
#include "gla_chunk.cuh"
#include "tma.cuh"
#include "gla_strong.cuh"
#include "tma_tiles.cuh"
#include "tmap.h"

namespace dig {

struct GradMaps {
  CUtensorMap q, k, v, dO;  // inputs (bf16)
  CUtensorMap eq;           // gate factors 2^(b - r), [B * gate_heads * L][d_k] fp32 (scan order)
  CUtensorMap dq, dk, dv;   // outputs (bf16 or fp32)
  CUtensorMap dla;          // d log alpha [B * L][gate_heads * d_k] fp32
};

template <typename TOUT>
struct TmaGradCfg {
  static constexpr int C = 128, DK = 32, DV = 64;
  static constexpr int RBK = 64, RBV = 128;  // bytes of a q / k row and of a v / dO row (2-byte values)
  static constexpr int OFF_Q = 0, OFF_K = 8192, OFF_V = 16384, OFF_DO = 32768;
  static constexpr int OFF_SP = 49152, OFF_GT = 53248;  // fp16 [DV][DK], 64-byte swizzle
  static constexpr int OFF_EQ = 57344;                  // fp32 [C][DK], 128-byte swizzle
  static constexpr int OFF_ST = 73728;                  // raw fp32 S_n [DV][DK], then G_n
  static constexpr int OFF_DLA = 90112;                 // raw S_{n+1} [DV][DK]
  // bf16 outputs ("decoupled"): once the key gradients are formed, the d log alpha
  // rows go over the raw states, dq and dk over the gate factors and dv over
  // S_{n+1}, so the operand tiles are free at once and the next unit's q, k, v,
  // dO are requested then; the small loads (gate factors, states) follow the
  // stores.  fp32 outputs (twice the staging) stage over the operand tiles and
  // request the next unit after the stores have been read.
  static constexpr bool DEC = !std::is_same<TOUT, float>::value;
  static constexpr int OFF_X = DEC ? OFF_ST : OFF_DLA;   // d log alpha rows, fp32 [C][DK], 128-byte swizzle
  static constexpr int OFF_SDQ = DEC ? OFF_EQ : 0, OFF_SDK = DEC ? OFF_EQ + 8192 : 16384;
  static constexpr int OFF_SDV = DEC ? OFF_DLA : 32768;
  static constexpr int END = 106496;
  static constexpr int SMEM = END + 1024;               // the base is aligned up to 1024 bytes
  static constexpr int TM_R = 0, TM_DQ = 128, TM_DK = 160, TM_DV = 192, TM_COLS = 256;
  static constexpr bool F32OUT = std::is_same<TOUT, float>::value;
  static constexpr uint32_t IN_BYTES = 2 * C * RBK + 2 * C * RBV;  // q, k, v, dO
  static constexpr uint32_t EQ_BYTES = C * DK * 4;
  static constexpr uint32_t SB = DV * DK * 4;                     // one state block
  static constexpr uint32_t GCH_BYTES = 2 * DK * 4;
};

struct TmaGradSmem {
  alignas(16) float gch[64];  // 2^r (d_k values), then 2^(Gamma - r)
  float red[8][32];           // partial sums of the boundary term
  float bnd[32];              // rowsum(S_{n+1} o G_n)
  float segtot[8][32];        // d log alpha segment totals
  uint64_t bar_ld;            // q, k, v, dO and gate factors of a unit
  uint64_t bar_st;            // S_n, G_n, S_{n+1} and the chunk constants of a unit
  uint64_t bar[6];            // the six product groups of a unit
  uint32_t tmem;
  int abort;                  // a wait gave up: stop after this unit
};

// Masks one C x C product in TMEM (lane = row r; keep column c >= r when
// `upper`, else c <= r) and rewrites it in place as fp16 pairs: the 32-column
// block s0 = 64 half + 32 kk becomes the 16 columns at 64 half + 16 kk, i.e.
// K-step j (16 columns) ends up at acol(j), the A-operand layout.  Tracks
// |value| in `amax`.
__device__ __forceinline__ void mask_to_f16(uint32_t tmem, uint32_t region, bool upper, uint32_t& amax) {
  const int tid = threadIdx.x, t = tid & 127, wq = t >> 5, half = tid >> 7;
  const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
    const int s0 = half * 64 + 32 * kk;  // 32-aligned: the block is this warp's diagonal block or off it
    const bool zero_block = upper ? (s0 < 32 * wq) : (s0 > 32 * wq);  // warp-uniform
    float pv[32];
    if (!zero_block) {
      tmem_ld32(tmem + lane_base + region + s0, pv);
      tmem_ld_wait();
      if (s0 == 32 * wq) {  // the diagonal block
#pragma unroll
        for (int e = 0; e < 32; ++e) pv[e] = (upper ? (s0 + e >= t) : (s0 + e <= t)) ? pv[e] : 0.f;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) pv[e] = 0.f;
    }
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      pk[e] = pack_f16x2(pv[2 * e], pv[2 * e + 1]);
      amax = absmax_f16x2(amax, pk[e]);
    }
    tmem_st16(tmem + lane_base + region + half * 64 + 16 * kk, pk);
  }
}
// TMEM column of K-step j (16 tokens) of a converted C x C product.
__device__ __forceinline__ uint32_t acol(int j) { return (uint32_t)((j >> 2) * 64 + (j & 3) * 8); }

template <typename TOUT>
__global__ void __launch_bounds__(256, 2) gla_grad_tma_kernel(const __grid_constant__ GradMaps mp, const GlaArgs a) {
  using TC = TmaGradCfg<TOUT>;
  constexpr int C = TC::C, DK = TC::DK, DV = TC::DV;
  extern __shared__ uint8_t smem_raw[];
  __shared__ TmaGradSmem sh;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t sb = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int nunits = a.B * a.H * a.nchunks;
  const uint64_t spin = a.spin_ns ? a.spin_ns : kSpinLimitNs;
  if (warp == 0) {
    tmem_alloc(&sh.tmem, TC::TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&sh.bar_ld, 1);
    mbar_init(&sh.bar_st, 1);
    for (int i = 0; i < 6; ++i) mbar_init(&sh.bar[i], 1);
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
  // Thread 0's record of the asynchronous work in flight, drained before exit:
  // per load barrier 0 = nothing pending, 1 = bytes expected but not yet
  // arrived, 2 = arrived (the phase completes when the bytes land); and the
  // last committed product group.
  int ld_state = 0, st_state = 0;
  uint32_t ld_ph = 0, st_ph = 0;
  int last_bar = -1;
  uint32_t last_ph = 0;
  bool last_done = true;

  // ---- thread 0: TMA issue
  // The last request of a barrier phase arrives on it (the phase completes once
  // that arrival and all requested bytes are in); earlier ones only add bytes.
  auto expect = [&](uint64_t* bar, uint32_t bytes, bool arrive) {
    if (arrive) mbar_arrive_expect_tx(bar, bytes);
    else mbar_expect_tx(bar, bytes);
  };
  auto issue_tiles = [&](const TileUnit& T, uint32_t phase, bool arrive) {  // q, k, v, dO
    ld_state = arrive ? 2 : 1;
    ld_ph = phase;
    expect(&sh.bar_ld, TC::IN_BYTES, arrive);
    if (!T.col) {
      tma_load_2d(sb + TC::OFF_Q, mp.q, T.h * DK, T.y, &sh.bar_ld);
      tma_load_2d(sb + TC::OFF_K, mp.k, T.h * DK, T.y, &sh.bar_ld);
      tma_load_2d(sb + TC::OFF_V, mp.v, T.h * DV, T.y, &sh.bar_ld);
      tma_load_2d(sb + TC::OFF_DO, mp.dO, T.h * DV, T.y, &sh.bar_ld);
    } else {
      for (int j = 0; j < C / 16; ++j) {
        int row, cl;
        T.seg(a, j, row, cl);
        tma_load_4d(sb + TC::OFF_Q + j * 16 * TC::RBK, mp.q, T.h * DK, row, cl, T.b, &sh.bar_ld);
        tma_load_4d(sb + TC::OFF_K + j * 16 * TC::RBK, mp.k, T.h * DK, row, cl, T.b, &sh.bar_ld);
        tma_load_4d(sb + TC::OFF_V + j * 16 * TC::RBV, mp.v, T.h * DV, row, cl, T.b, &sh.bar_ld);
        tma_load_4d(sb + TC::OFF_DO + j * 16 * TC::RBV, mp.dO, T.h * DV, row, cl, T.b, &sh.bar_ld);
      }
    }
  };
  auto issue_eq = [&](const TileUnit& T, uint32_t phase, bool arrive) {  // gate factors (scan order)
    ld_state = arrive ? 2 : 1;
    ld_ph = phase;
    expect(&sh.bar_ld, TC::EQ_BYTES, arrive);
    tma_load_2d(sb + TC::OFF_EQ, mp.eq, 0, T.bz * a.L + T.n * C, &sh.bar_ld);
  };
  auto issue_states = [&](int u, const TileUnit& T, uint32_t phase, bool arrive) {  // S_n, G_n, chunk constants
    st_state = arrive ? 2 : 1;
    st_ph = phase;
    expect(&sh.bar_st, 2 * TC::SB + TC::GCH_BYTES, arrive);
    bulk_copy_g2s(sb + TC::OFF_ST, a.dsn + (size_t)u * DV * DK, TC::SB, &sh.bar_st);
    bulk_copy_g2s(sb + TC::OFF_ST + TC::SB, a.dhn + (size_t)u * DV * DK, TC::SB, &sh.bar_st);
    bulk_copy_g2s(smem_u32(sh.gch), a.gCH + ((size_t)T.bz * a.nchunks + T.n) * 4 * DK, TC::GCH_BYTES, &sh.bar_st);
  };
  auto issue_next_state = [&](int u, const TileUnit& T, uint32_t phase) {  // S_{n+1}; completes the phase
    const bool has_next_chunk = T.n + 1 < a.nchunks;  // G of the last chunk is zero: no boundary term
    st_state = 2;
    st_ph = phase;
    mbar_arrive_expect_tx(&sh.bar_st, has_next_chunk ? TC::SB : 0u);
    if (has_next_chunk) bulk_copy_g2s(sb + TC::OFF_DLA, a.dsn + (size_t)(u + 1) * DV * DK, TC::SB, &sh.bar_st);
  };

  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  if (tid == 0 && (int)blockIdx.x < nunits) {
    const TileUnit T0(a, blockIdx.x, C);
    issue_tiles(T0, 0, false);
    issue_eq(T0, 0, true);
    issue_states(blockIdx.x, T0, 0, false);
    issue_next_state(blockIdx.x, T0, 0);
  }

  int it = 0;
  for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++it) {
    const uint32_t ph = it & 1;
    const TileUnit T(a, u, C);
    const int un = u + gridDim.x;
    const bool has_next = un < nunits;
    const bool has_next_chunk = T.n + 1 < a.nchunks;
    uint32_t amax = 0;  // running |value| of this thread's fp16 operands and products
    bool out_of_range = false;
    const bool strong_unit = strong::flagged(a, T.bz, T.n);

    // ---- 1. states: the boundary term and the S', Gt operands
    wait_bar(&sh.bar_st, ph);
    if (tid == 0 && !timed_out) st_state = 0;
    {
      const int c = tid & 31, g = tid >> 5;
      float part = 0.f;
      if (has_next_chunk) {
        const float* S1 = reinterpret_cast<const float*>(smem_raw + (sb - smem_u32(smem_raw)) + TC::OFF_DLA);
        const float* G = reinterpret_cast<const float*>(smem_raw + (sb - smem_u32(smem_raw)) + TC::OFF_ST + TC::SB);
#pragma unroll
        for (int j = 0; j < 8; ++j) part = fmaf(S1[(8 * g + j) * DK + c], G[(8 * g + j) * DK + c], part);
      }
      sh.red[g][c] = part;
      // S' = 2^r S_n and Gt = 2^(Gamma - r) G_n rows (value channel j, key channels 8 cc .. 8 cc + 7)
      const int j = tid >> 2, cc = tid & 3;
      const uint32_t src = sb + TC::OFF_ST + (uint32_t)(j * DK + 8 * cc) * 4u;
      const float4 s0 = lds128f(src), s1 = lds128f(src + 16);
      const float4 g0 = lds128f(src + TC::SB), g1 = lds128f(src + TC::SB + 16);
      const float4 r0 = *reinterpret_cast<const float4*>(&sh.gch[8 * cc]);
      const float4 r1 = *reinterpret_cast<const float4*>(&sh.gch[8 * cc + 4]);
      const float4 e0 = *reinterpret_cast<const float4*>(&sh.gch[DK + 8 * cc]);
      const float4 e1 = *reinterpret_cast<const float4*>(&sh.gch[DK + 8 * cc + 4]);
      uint4 sp, gt;
      sp.x = pack_f16x2(s0.x * r0.x, s0.y * r0.y);
      sp.y = pack_f16x2(s0.z * r0.z, s0.w * r0.w);
      sp.z = pack_f16x2(s1.x * r1.x, s1.y * r1.y);
      sp.w = pack_f16x2(s1.z * r1.z, s1.w * r1.w);
      gt.x = pack_f16x2(g0.x * e0.x, g0.y * e0.y);
      gt.y = pack_f16x2(g0.z * e0.z, g0.w * e0.w);
      gt.z = pack_f16x2(g1.x * e1.x, g1.y * e1.y);
      gt.w = pack_f16x2(g1.z * e1.z, g1.w * e1.w);
      amax = absmax_f16x2(absmax_f16x2(absmax_f16x2(absmax_f16x2(amax, sp.x), sp.y), sp.z), sp.w);
      amax = absmax_f16x2(absmax_f16x2(absmax_f16x2(absmax_f16x2(amax, gt.x), gt.y), gt.z), gt.w);
      sts128(sb + TC::OFF_SP + swz_off<64>(j, cc), sp);
      sts128(sb + TC::OFF_GT + swz_off<64>(j, cc), gt);
    }
    fence_async_smem();  // the raw state reads precede the next unit's copies into the same slots
    __syncthreads();
    if (tid < 32) {
      float s = 0.f;
#pragma unroll
      for (int g = 0; g < 8; ++g) s += sh.red[g][tid];
      sh.bnd[tid] = s;
    }
    if constexpr (!TC::DEC) {  // the raw-state slot is free: the next unit's S_n, G_n
      if (tid == 0 && has_next && !timed_out && !sh.abort) issue_states(un, TileUnit(a, un, C), ph ^ 1u, false);
    }

    // ---- 2. inputs, converted in place to fp16 operands: qbar = q EQ, kbar = k / EQ, v, dO
    wait_bar(&sh.bar_ld, ph);
    if (tid == 0 && !timed_out) ld_state = 0;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int k = tid + 256 * m;  // 16-byte chunk of the q / k tiles
      const int i = k >> 2, c = (k & 3) ^ ((i >> 1) & 3);
      const int ti = T.rev ? C - 1 - i : i;
      const float4 e0 = lds128f(sb + TC::OFF_EQ + swz_off<128>(ti, 2 * c));
      const float4 e1 = lds128f(sb + TC::OFF_EQ + swz_off<128>(ti, 2 * c + 1));
      const float e[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
      const uint4 qr = lds128(sb + TC::OFF_Q + 16u * k), kr = lds128(sb + TC::OFF_K + 16u * k);
      const uint32_t qw[4] = {qr.x, qr.y, qr.z, qr.w}, kw[4] = {kr.x, kr.y, kr.z, kr.w};
      uint32_t qo[4], ko[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float ea = e[2 * w], eb = e[2 * w + 1];
        out_of_range |= !(ea >= 0.00390625f && ea <= 256.f && eb >= 0.00390625f && eb <= 256.f);
        qo[w] = pack_f16x2(bf_lo(qw[w]) * ea, bf_hi(qw[w]) * eb);
        ko[w] = pack_f16x2(bf_lo(kw[w]) * __frcp_rn(ea), bf_hi(kw[w]) * __frcp_rn(eb));
        amax = absmax_f16x2(absmax_f16x2(amax, qo[w]), ko[w]);
      }
      sts128(sb + TC::OFF_Q + 16u * k, make_uint4(qo[0], qo[1], qo[2], qo[3]));
      sts128(sb + TC::OFF_K + 16u * k, make_uint4(ko[0], ko[1], ko[2], ko[3]));
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const uint32_t off = 16u * (uint32_t)(tid + 256 * m);
      const uint4 vr = lds128(sb + TC::OFF_V + off), dr = lds128(sb + TC::OFF_DO + off);
      uint4 vo, dd;
      vo.x = pack_f16x2(bf_lo(vr.x), bf_hi(vr.x));
      vo.y = pack_f16x2(bf_lo(vr.y), bf_hi(vr.y));
      vo.z = pack_f16x2(bf_lo(vr.z), bf_hi(vr.z));
      vo.w = pack_f16x2(bf_lo(vr.w), bf_hi(vr.w));
      dd.x = pack_f16x2(bf_lo(dr.x), bf_hi(dr.x));
      dd.y = pack_f16x2(bf_lo(dr.y), bf_hi(dr.y));
      dd.z = pack_f16x2(bf_lo(dr.z), bf_hi(dr.z));
      dd.w = pack_f16x2(bf_lo(dr.w), bf_hi(dr.w));
      amax = absmax_f16x2(absmax_f16x2(absmax_f16x2(absmax_f16x2(amax, vo.x), vo.y), vo.z), vo.w);
      amax = absmax_f16x2(absmax_f16x2(absmax_f16x2(absmax_f16x2(amax, dd.x), dd.y), dd.z), dd.w);
      sts128(sb + TC::OFF_V + off, vo);
      sts128(sb + TC::OFF_DO + off, dd);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- 3. products (thread 0 issues; single fp16 terms)
    const uint32_t sQ = sb + TC::OFF_Q, sK = sb + TC::OFF_K, sV = sb + TC::OFF_V, sD = sb + TC::OFF_DO;
    const uint32_t sS = sb + TC::OFF_SP, sG = sb + TC::OFF_GT;
    auto can_issue = [&]() { return tid == 0 && !timed_out && !sh.abort; };
    auto commit = [&](int i) {
      mma_commit(&sh.bar[i]);
      last_bar = i;
      last_ph = ph;
      last_done = false;
    };
    auto wait_group = [&](int i) {  // every thread waits for product group i
      wait_bar(&sh.bar[i], ph);
      if (tid == 0 && last_bar == i && !timed_out) last_done = true;
      tc_fence_after();
    };
    if (can_issue()) {
#pragma unroll
      for (int s = 0; s < DK / 16; ++s)  // P^T[s][t] = kbar qbar^T
        mma_bf16(tmem + TC::TM_R, sdesc_sw<64>(sK + 32 * s), sdesc_sw<64>(sQ + 32 * s), idesc_f16(128, C), s > 0);
#pragma unroll
      for (int s = 0; s < DV / 16; ++s) {  // dqbar = dO S'^T, dkbar = V Gt^T
        mma_bf16(tmem + TC::TM_DQ, sdesc_sw<128>(sD + 32 * s), sdesc_sw<64>(sS + 1024 * s),
                 idesc_f16(128, DK, false, true), s > 0);
        mma_bf16(tmem + TC::TM_DK, sdesc_sw<128>(sV + 32 * s), sdesc_sw<64>(sG + 1024 * s),
                 idesc_f16(128, DK, false, true), s > 0);
      }
#pragma unroll
      for (int s = 0; s < DK / 16; ++s)  // dv = kbar Gt
        mma_bf16(tmem + TC::TM_DV, sdesc_sw<64>(sK + 32 * s), sdesc_sw<64>(sG + 32 * s), idesc_f16(128, DV), s > 0);
      commit(0);
    }
    auto publish_tmem = [&]() {
      tmem_st_wait();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
    };
    wait_group(0);
    mask_to_f16(tmem, TC::TM_R, !T.rev, amax);  // P^T: keep scan(s) <= scan(t)
    publish_tmem();
    if (can_issue()) {
#pragma unroll
      for (int s = 0; s < C / 16; ++s)  // dv += P^T dO
        mma_bf16_ts(tmem + TC::TM_DV, tmem + TC::TM_R + acol(s), sdesc_sw<128>(sD + 2048 * s),
                    idesc_f16(128, DV, false, true), 1);
      commit(1);
      wait_group(1);  // P^T has been read: dP^T takes its columns
      if (can_issue()) {
#pragma unroll
        for (int s = 0; s < DV / 16; ++s)  // dP^T[s][t] = V dO^T
          mma_bf16(tmem + TC::TM_R, sdesc_sw<128>(sV + 32 * s), sdesc_sw<128>(sD + 32 * s), idesc_f16(128, C), s > 0);
        commit(2);
      }
    }
    wait_group(2);
    mask_to_f16(tmem, TC::TM_R, !T.rev, amax);
    publish_tmem();
    if (can_issue()) {
#pragma unroll
      for (int s = 0; s < C / 16; ++s)  // dkbar += dP^T qbar
        mma_bf16_ts(tmem + TC::TM_DK, tmem + TC::TM_R + acol(s), sdesc_sw<64>(sQ + 1024 * s),
                    idesc_f16(128, DK, false, true), 1);
      commit(3);
      wait_group(3);  // dP^T has been read: dP takes its columns
      if (can_issue()) {
#pragma unroll
        for (int s = 0; s < DV / 16; ++s)  // dP[t][s] = dO V^T
          mma_bf16(tmem + TC::TM_R, sdesc_sw<128>(sD + 32 * s), sdesc_sw<128>(sV + 32 * s), idesc_f16(128, C), s > 0);
        commit(4);
      }
    }
    wait_group(4);
    mask_to_f16(tmem, TC::TM_R, T.rev, amax);  // dP[t][s]: keep scan(s) <= scan(t)
    publish_tmem();
    if (can_issue()) {
#pragma unroll
      for (int s = 0; s < C / 16; ++s)  // dqbar += dP kbar
        mma_bf16_ts(tmem + TC::TM_DQ, tmem + TC::TM_R + acol(s), sdesc_sw<64>(sK + 1024 * s),
                    idesc_f16(128, DK, false, true), 1);
      commit(5);
    }
    wait_group(5);

    // ---- 4. key gradients of this thread's token (TMEM lane t) and channel half; d log alpha terms
    float dq[16], dk[16], x[16];
    {
      const int ti = T.rev ? C - 1 - t : t;
      float dqb[16], dkb[16];
      tmem_ld8(tmem + lane_base + TC::TM_DQ + 16 * half, dqb);
      tmem_ld8(tmem + lane_base + TC::TM_DQ + 16 * half + 8, dqb + 8);
      tmem_ld8(tmem + lane_base + TC::TM_DK + 16 * half, dkb);
      tmem_ld8(tmem + lane_base + TC::TM_DK + 16 * half + 8, dkb + 8);
      float4 ef[4];
      uint4 qv[2], kv[2];
#pragma unroll
      for (int m = 0; m < 4; ++m) ef[m] = lds128f(sb + TC::OFF_EQ + swz_off<128>(ti, 4 * half + m));
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        qv[m] = lds128(sQ + swz_off<64>(t, 2 * half + m));
        kv[m] = lds128(sK + swz_off<64>(t, 2 * half + m));
      }
      tmem_ld_wait();
      const float e[16] = {ef[0].x, ef[0].y, ef[0].z, ef[0].w, ef[1].x, ef[1].y, ef[1].z, ef[1].w,
                           ef[2].x, ef[2].y, ef[2].z, ef[2].w, ef[3].x, ef[3].y, ef[3].z, ef[3].w};
      const uint32_t qw[8] = {qv[0].x, qv[0].y, qv[0].z, qv[0].w, qv[1].x, qv[1].y, qv[1].z, qv[1].w};
      const uint32_t kw[8] = {kv[0].x, kv[0].y, kv[0].z, kv[0].w, kv[1].x, kv[1].y, kv[1].z, kv[1].w};
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float qa = h_lo(qw[w]), qb2 = h_hi(qw[w]), ka = h_lo(kw[w]), kb2 = h_hi(kw[w]);
        const int c = 2 * w;
        dq[c] = dqb[c] * e[c];
        dq[c + 1] = dqb[c + 1] * e[c + 1];
        dk[c] = dkb[c] * __frcp_rn(e[c]);
        dk[c + 1] = dkb[c + 1] * __frcp_rn(e[c + 1]);
        x[c] = qa * dqb[c] - ka * dkb[c];
        x[c + 1] = qb2 * dqb[c + 1] - kb2 * dkb[c + 1];
      }
    }
    fence_async_smem();  // the gate-factor and operand reads precede the copies into those slots
    tc_fence_before();
    __syncthreads();  // qbar, kbar and gate factors read; every product complete
    if constexpr (TC::DEC) {  // the operand tiles are free: the next unit's q, k, v, dO
      if (tid == 0 && has_next && !timed_out && !sh.abort) issue_tiles(TileUnit(a, un, C), ph ^ 1u, false);
    }
#pragma unroll
    for (int m = 0; m < 4; ++m)
      sts128(sb + TC::OFF_X + swz_off<128>(t, 4 * half + m),
             make_uint4(__float_as_uint(x[4 * m]), __float_as_uint(x[4 * m + 1]), __float_as_uint(x[4 * m + 2]),
                        __float_as_uint(x[4 * m + 3])));

    // ---- 5. outputs to staging over the operand tiles (swizzled like the store boxes)
    {
      float dv[32];
#pragma unroll
      for (int c = 0; c < 32; c += 8) tmem_ld8(tmem + lane_base + TC::TM_DV + 32 * half + c, dv + c);
      tmem_ld_wait();
      if constexpr (!TC::F32OUT) {
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          sts128(sb + TC::OFF_SDQ + swz_off<64>(t, 2 * half + m),
                 make_uint4(pack_bf16x2(dq[8 * m], dq[8 * m + 1]), pack_bf16x2(dq[8 * m + 2], dq[8 * m + 3]),
                            pack_bf16x2(dq[8 * m + 4], dq[8 * m + 5]), pack_bf16x2(dq[8 * m + 6], dq[8 * m + 7])));
          sts128(sb + TC::OFF_SDK + swz_off<64>(t, 2 * half + m),
                 make_uint4(pack_bf16x2(dk[8 * m], dk[8 * m + 1]), pack_bf16x2(dk[8 * m + 2], dk[8 * m + 3]),
                            pack_bf16x2(dk[8 * m + 4], dk[8 * m + 5]), pack_bf16x2(dk[8 * m + 6], dk[8 * m + 7])));
        }
#pragma unroll
        for (int m = 0; m < 4; ++m)
          sts128(sb + TC::OFF_SDV + swz_off<128>(t, 4 * half + m),
                 make_uint4(pack_bf16x2(dv[8 * m], dv[8 * m + 1]), pack_bf16x2(dv[8 * m + 2], dv[8 * m + 3]),
                            pack_bf16x2(dv[8 * m + 4], dv[8 * m + 5]), pack_bf16x2(dv[8 * m + 6], dv[8 * m + 7])));
      } else {
        // fp32: dq [0, 16K), dk [16K, 32K), dv channels 0-31 [32K, 48K), 32-63 over the gate factors
        const uint32_t dvdst = half ? sb + TC::OFF_EQ : sb + 32768u;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          sts128(sb + swz_off<128>(t, 4 * half + m),
                 make_uint4(__float_as_uint(dq[4 * m]), __float_as_uint(dq[4 * m + 1]), __float_as_uint(dq[4 * m + 2]),
                            __float_as_uint(dq[4 * m + 3])));
          sts128(sb + 16384u + swz_off<128>(t, 4 * half + m),
                 make_uint4(__float_as_uint(dk[4 * m]), __float_as_uint(dk[4 * m + 1]), __float_as_uint(dk[4 * m + 2]),
                            __float_as_uint(dk[4 * m + 3])));
        }
#pragma unroll
        for (int m = 0; m < 8; ++m)
          sts128(dvdst + swz_off<128>(t, m),
                 make_uint4(__float_as_uint(dv[4 * m]), __float_as_uint(dv[4 * m + 1]), __float_as_uint(dv[4 * m + 2]),
                            __float_as_uint(dv[4 * m + 3])));
      }
    }

    // ---- 6. d log alpha: cumsum over the chunk in scan order (tile order reversed when `rev`)
    {
      const int c = tid & 31, sg = tid >> 5;  // channel, 16-row segment
      const uint32_t cbase = sb + TC::OFF_X + (uint32_t)(c & 3) * 4u;
      float xv[16];
      __syncthreads();  // every x row written
#pragma unroll
      for (int e = 0; e < 16; ++e)
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(xv[e]) : "r"(cbase + swz_off<128>(16 * sg + e, c >> 2)));
      // scan order runs down the rows (suffix sums) or, reversed, up them (prefix sums)
      if (T.rev) {
#pragma unroll
        for (int e = 1; e < 16; ++e) xv[e] += xv[e - 1];
        sh.segtot[sg][c] = xv[15];
      } else {
#pragma unroll
        for (int e = 14; e >= 0; --e) xv[e] += xv[e + 1];
        sh.segtot[sg][c] = xv[0];
      }
      __syncthreads();
      float post = sh.bnd[c];
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        if (T.rev ? s2 < sg : s2 > sg) post += sh.segtot[s2][c];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(cbase + swz_off<128>(16 * sg + e, c >> 2)), "f"(xv[e] + post)
                     : "memory");
    }
    fence_async_smem();  // staging writes precede the TMA stores that read them
    // a chunk flagged by the gate kernel (strong gate) goes to the exact kernel too
    const int bad = __syncthreads_or(out_of_range || f16x2_too_large(amax) || strong_unit);

    // ---- 7. stores (thread 0), then the next unit's tiles into the freed slots
    if (tid == 0) {
      if (bad) {
        const uint32_t slot = atomicAdd(a.flist, 1u);  // the exact kernel computes this unit
        a.flist[1 + slot] = (uint32_t)u;
      } else if (!sh.abort) {
        if (!T.col) {
          if constexpr (!TC::F32OUT) {
            tma_store_2d(mp.dq, T.h * DK, T.y, sb + TC::OFF_SDQ);
            tma_store_2d(mp.dk, T.h * DK, T.y, sb + TC::OFF_SDK);
            tma_store_2d(mp.dv, T.h * DV, T.y, sb + TC::OFF_SDV);
          } else {
            tma_store_2d(mp.dq, T.h * DK, T.y, sb);
            tma_store_2d(mp.dk, T.h * DK, T.y, sb + 16384u);
            tma_store_2d(mp.dv, T.h * DV, T.y, sb + 32768u);
            tma_store_2d(mp.dv, T.h * DV + 32, T.y, sb + TC::OFF_EQ);
          }
          if (a.gate_heads == 1) tma_reduce_add_2d(mp.dla, T.hz * DK, T.y, sb + TC::OFF_X);
          else tma_store_2d(mp.dla, T.hz * DK, T.y, sb + TC::OFF_X);
        } else {
          for (int j = 0; j < C / 16; ++j) {
            int row, cl;
            T.seg(a, j, row, cl);
            if constexpr (!TC::F32OUT) {
              tma_store_4d(mp.dq, T.h * DK, row, cl, T.b, sb + TC::OFF_SDQ + j * 16 * TC::RBK);
              tma_store_4d(mp.dk, T.h * DK, row, cl, T.b, sb + TC::OFF_SDK + j * 16 * TC::RBK);
              tma_store_4d(mp.dv, T.h * DV, row, cl, T.b, sb + TC::OFF_SDV + j * 16 * TC::RBV);
            } else {
              tma_store_4d(mp.dq, T.h * DK, row, cl, T.b, sb + j * 2048);
              tma_store_4d(mp.dk, T.h * DK, row, cl, T.b, sb + 16384u + j * 2048);
              tma_store_4d(mp.dv, T.h * DV, row, cl, T.b, sb + 32768u + j * 2048);
              tma_store_4d(mp.dv, T.h * DV + 32, row, cl, T.b, sb + TC::OFF_EQ + j * 2048);
            }
            if (a.gate_heads == 1) tma_reduce_add_4d(mp.dla, T.hz * DK, row, cl, T.b, sb + TC::OFF_X + j * 2048);
            else tma_store_4d(mp.dla, T.hz * DK, row, cl, T.b, sb + TC::OFF_X + j * 2048);
          }
        }
        bulk_commit();
      }
      if (has_next && !timed_out && !sh.abort) {
        bulk_wait_read_all();  // the staging has been read
        const TileUnit Tn(a, un, C);
        if constexpr (TC::DEC) {  // the q, k, v, dO tiles are already on their way
          issue_eq(Tn, ph ^ 1u, true);
          issue_states(un, Tn, ph ^ 1u, false);
        } else {
          issue_tiles(Tn, ph ^ 1u, false);
          issue_eq(Tn, ph ^ 1u, true);
        }
        issue_next_state(un, Tn, ph ^ 1u);
      }
    }
    if (sh.abort) break;  // uniform: read after the barrier above
  }

  // ---- drain: no copy, reduction or product may outlive the CTA.  After a
  // wait gave up, nothing new was issued; here the copies already issued land,
  // the stores finish and the last product group completes (each wait bounded
  // by the normal limit) before TMEM is released.
  if (timed_out) set_status(a.status, DIG_ERR_DEVICE_TIMEOUT);
  if (tid == 0) {
    bulk_wait_all();
    if (ld_state == 1) mbar_arrive(&sh.bar_ld);  // complete the phase once its bytes land
    if (ld_state) mbar_wait(&sh.bar_ld, ld_ph, kSpinLimitNs);
    if (st_state == 1) mbar_arrive(&sh.bar_st);
    if (st_state) mbar_wait(&sh.bar_st, st_ph, kSpinLimitNs);
    if (last_bar >= 0 && !last_done) mbar_wait(&sh.bar[last_bar], last_ph, kSpinLimitNs);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TC::TM_COLS);
}

// ------------------------------------------------------------------ launch
namespace {

bool encode_maps(GradMaps& mp, const GlaArgs& a, bool f32out) {
  const int BL = a.B * a.L, gh = a.gate_heads;
  constexpr int DK = 32, DV = 64, C = 128;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const CUtensorMapDataType ot = f32out ? f32 : bf;
  const int oe = f32out ? 4 : 2;
  const int okb = f32out ? 128 : 64;   // swizzle span of a dq / dk box row
  const int ovb = 128;                 // dv box rows: 64 bf16 or 32 fp32
  const uint32_t ov_box = f32out ? 32 : 64;
  const bool col = (a.mode & 2) != 0;
  const uint32_t rows = col ? 16 : C;
  auto tile = [&](CUtensorMap* m, const void* p, CUtensorMapDataType dt, int esize, int row_elems, uint32_t box,
                  int rb) {
    return col ? tmap_cols(m, p, dt, esize, row_elems, a.Hg, a.Wg, a.B, box, rows, rb)
               : tmap_rows(m, p, dt, esize, row_elems, BL, box, rows, rb);
  };
  bool ok = tile(&mp.q, a.q, bf, 2, a.H * DK, DK, 64) && tile(&mp.k, a.k, bf, 2, a.H * DK, DK, 64) &&
            tile(&mp.v, a.v, bf, 2, a.H * DV, DV, 128) && tile(&mp.dO, a.dO, bf, 2, a.H * DV, DV, 128) &&
            tile(&mp.dq, a.dq, ot, oe, a.H * DK, DK, okb) && tile(&mp.dk, a.dk, ot, oe, a.H * DK, DK, okb) &&
            tile(&mp.dv, a.dv, ot, oe, a.H * DV, ov_box, ovb) && tile(&mp.dla, a.dla, f32, 4, gh * DK, DK, 128);
  ok = ok && tmap_rows(&mp.eq, a.gEQ, f32, 4, DK, (uint64_t)a.B * gh * a.L, DK, C, 128);
  return ok;
}

}  // namespace

bool gla_grad_tma_eligible(const GlaArgs& a, int dk, int dv, int tin, int chunk) {
  if (tin != DIG_BF16 || dk != 32 || dv != 64 || chunk != 128 || a.L % 128 != 0) return false;
  if ((a.mode & 2) && a.Hg % 16 != 0) return false;
  return tmap_available();
}

// Launches the TMA kernel; units it cannot take are listed in a.flist for the exact kernel.
cudaError_t launch_grad_tma(const GlaArgs& a, int tout, cudaStream_t s, bool* launched) {
  *launched = false;
  GradMaps mp;
  if (!encode_maps(mp, a, tout == DIG_F32)) return cudaSuccess;  // not encodable: the caller runs the exact kernel
  const long long units = (long long)a.B * a.H * a.nchunks;
  cudaError_t e;
  if (tout == DIG_F32) {
    auto k = gla_grad_tma_kernel<float>;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, TmaGradCfg<float>::SMEM)) !=
        cudaSuccess)
      return e;
    e = launch_pdl(k, persistent_grid(2, units), 256, TmaGradCfg<float>::SMEM, s, mp, a);
  } else {
    auto k = gla_grad_tma_kernel<__nv_bfloat16>;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  TmaGradCfg<__nv_bfloat16>::SMEM)) != cudaSuccess)
      return e;
    e = launch_pdl(k, persistent_grid(2, units), 256, TmaGradCfg<__nv_bfloat16>::SMEM, s, mp, a);
  }
  if (e == cudaSuccess) *launched = true;
  return e;
}

}  // namespace dig
