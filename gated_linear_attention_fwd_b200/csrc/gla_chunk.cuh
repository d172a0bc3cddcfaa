// gla_chunk.cuh -- pieces shared by the chunk-parallel GLA kernels (forward
// and backward): operand layouts, the unit decomposition, row loads, the gate
// kernel (per gate head and chunk: the cumsum of the log decays as gate
// factors) and the chunk-state kernel (per-chunk state contribution, and for
// the backward the per-chunk state-gradient contribution).
//
// A unit is one chunk of C consecutive scan positions of one (batch, head)
// sequence.  Units are independent: kernels loop over them persistently and
// never wait on one another.
#pragma once
#include <type_traits>

#include "gla.h"
#include "gla_common.cuh"

namespace dig {

// Bound of the kernels' waits: the call's test bound when one was set, else the default.
__device__ __forceinline__ uint64_t spin_limit(const GlaArgs& a) { return a.spin_ns ? a.spin_ns : kSpinLimitNs; }

template <int C_, int DK_, int DV_, typename TIN>
struct ChunkCfg {
  static constexpr int C = C_, DK = DK_, DV = DV_;
  static constexpr int NTG = std::is_same<TIN, float>::value ? 3 : 2;  // terms of gated operands
  static constexpr int NTV = std::is_same<TIN, float>::value ? 3 : 1;  // terms of raw v / dO
  static constexpr int DKP = cround(DK, 16), DVP = cround(DV, 16);
  // per-thread channel halves for TMEM row reads (multiples of 4 so rows stay 16-byte aligned)
  static constexpr int DK0 = cround((DK + 1) / 2, 4), DK1 = DK - DK0;
  static constexpr int DV0 = cround((DV + 1) / 2, 8), DV1 = DV - DV0;
  // Operands are token rows (bf16, K-major over channels: 8-row x 16-byte core
  // matrices, LBO = 128 between 8-channel groups, SBO = row-group stride), read
  // K-major or, for products that contract over tokens, MN-major.
  static constexpr int SBO_K = DKP * 16;            // rows of DKP values (q, k, khat, S', dH')
  static constexpr int SBO_V = DVP * 16;            // rows of DVP values (v, dO)
  static constexpr int AQ_SZ = (C / 8) * SBO_K;     // one term, C rows
  static constexpr int VR_SZ = (C / 8) * SBO_V;     // one term, C rows
  static constexpr int SPT_SZ = (DVP / 8) * SBO_K;  // one term, DVP rows
  // an M = 128 read of C-row operands covers 128 rows (K-major) or, read
  // MN-major as v^T / dO^T, 16 channel groups of every token group
  static constexpr int AQ_READ = (NTG - 1) * AQ_SZ + 16 * SBO_K;
  static constexpr int VR_READ = cmax((NTV - 1) * VR_SZ + (C / 8 - 1) * SBO_V + 16 * 128,
                                      (NTV - 1) * VR_SZ + 16 * SBO_V);
  // ---- row pieces of the coalesced loads and stores (see piece_of)
  static constexpr int PSK = DK % 8 == 0 ? 8 : 4;  // channels per piece of q / k rows
  static constexpr int NGK = DK / PSK;
  static constexpr int NPK = cdiv(C * NGK, 256);    // pieces per thread
  static constexpr int NGZ = DK / 4;                // gate logits / factors: 4 fp32 channels per piece
  static constexpr int NPZ = cdiv(C * NGZ, 256);
  static constexpr int NGS = DK / 4;                // state rows (fp32)
  static constexpr int NPS = cdiv(DV * NGS, 256);
  static constexpr int NGV = DV / 8;                // v / dO / r / o / y / dv rows: 8 channels per piece
  static constexpr int NPV = cdiv(C * NGV, 256);
  static constexpr int NPAD = (DKP - DK) / 4;       // zero pieces of the key-channel padding, per row
  static constexpr int NPADV = (DVP - DV) / 8;      // zero pieces of the value-channel padding, per row
  static_assert(DK % 4 == 0 && DV % 8 == 0 && DK1 > 0 && DV1 > 0 && DK <= 64 && DV <= 128, "head dims");
  static_assert(C == 32 || C == 64 || C == 128, "chunk");
};

// Layout of the chunk-state kernel (BWD adds q 2^b and dO operands).
template <int C, int DK, int DV, typename TIN, bool BWD>
struct StateCfg {
  using K = ChunkCfg<C, DK, DV, TIN>;
  static constexpr int OFF_KH = 0;
  static constexpr int OFF_QB = OFF_KH + K::NTG * K::AQ_SZ;  // BWD: q 2^b
  static constexpr int OFF_VR = OFF_QB + (BWD ? K::NTG * K::AQ_SZ : 0);
  static constexpr int OFF_DO = OFF_VR + K::NTV * K::VR_SZ;  // BWD: dO
  static constexpr int END_ROWS = OFF_DO + (BWD ? K::NTV * K::VR_SZ : 0);
  static constexpr int SDP = DK + 4;                // row pitch of the dS / dH staging rows
  static constexpr int OFF_SD = cround(END_ROWS, 16);
  // the M = 128 reads of v^T / dO^T may run past their rows into the next
  // buffers (those lanes are unused); they only have to stay inside the allocation
  static constexpr int SMEM = cmax(cmax(OFF_SD + (BWD ? 2 : 1) * DV * SDP * 4, OFF_VR + K::VR_READ),
                                   BWD ? OFF_DO + K::VR_READ : 0);
  static constexpr int TM_DH = K::DKP;              // BWD: dH columns after dS
  static constexpr int TM_COLS = pow2ceil((BWD ? 2 : 1) * K::DKP);
  // resident CTAs per SM: by shared memory, and by registers (the forward kernel
  // with d_k > 32 holds more row pieces than three CTAs' registers allow)
  static constexpr int MINB = BWD ? 2 : (DK <= 32 ? 3 : 2);
  static constexpr int PER_SM = cmax(1, SMEM <= 72 * 1024 ? cmin(3, MINB) : SMEM <= 110 * 1024 ? cmin(2, MINB) : 1);
  static_assert(SMEM <= 225 * 1024, "shared-memory budget");
};

struct StateSmem {
  long long rows[2][128];  // grid tokens of the units whose loads are in flight (by unit parity)
  uint64_t bar;
  uint32_t tmem;
  int mma_pend;            // thread 0: products committed and not yet seen complete (drained before exit)
  uint32_t mma_ph;
};

// Unit u -> (sequence bh, chunk n); units of one sequence are consecutive.
struct Unit {
  int bh, n, b, h, bz;
  __device__ Unit(const GlaArgs& a, int u) {
    bh = u / a.nchunks;
    n = u - bh * a.nchunks;
    b = bh / a.H;
    h = bh - b * a.H;
    bz = b * a.gate_heads + (a.gate_heads == 1 ? 0 : h);
  }
};

// Grid token of token t of a unit, b * L + pi(n C + t), or -1 past the chunk or
// the sequence end; its row in the [B, L, H, *] tensors is that times H plus h.
// Kernels fill a unit's 128 entries into shared memory once (one thread per
// token) instead of mapping the scan position of every row piece.
__device__ __forceinline__ long long unit_grow(const GlaArgs& a, const Unit& U, int C, int t) {
  const int p = U.n * C + t;
  if (t >= C || p >= a.L) return -1;
  return (long long)U.b * a.L + scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode);
}
__device__ __forceinline__ void fill_rows(const GlaArgs& a, int u, int C, long long* grows) {
  if ((int)threadIdx.x < 128) grows[threadIdx.x] = unit_grow(a, Unit(a, u), C, threadIdx.x);
}
// Row of the unit's token in a [B, L, H, *] tensor (0 for an invalid token, which is never dereferenced).
__device__ __forceinline__ size_t tok_row(long long grow, const GlaArgs& a, int h) {
  return grow >= 0 ? (size_t)grow * a.H + h : 0;
}

// Rows of a [B, L, H, DV] tensor (v or dO) for a unit's chunk, its grid tokens
// from a table (see unit_grow), into a K-major operand buffer at `vr` (token
// rows of DVP channels).  bf16 values are copied unchanged (one exact term) by
// asynchronous 16-byte copies, zero-filled past the sequence end (complete after
// cp_async_wait_all); fp32 values are split into three bf16 terms.  Channels
// DV..DVP are zeroed (they are a contracted dimension in some products).
// NTH threads of the CTA share the pieces.
// With a value gate (VS != VS_NONE, fp32 inputs only) each row is scaled on the
// way by its token's value-gate factor EQb = 2^(e - rho) of the unit's chunk
// (gate row bz, chunk n): v / EQb (VS_VBAR), v 2^(Gb - rho) / EQb = v 2^(Gb - e)
// (VS_VHAT), dO EQb (VS_DOBAR) or dO EQb 2^rho = dO 2^e (VS_DOE).
enum { VS_NONE = 0, VS_VBAR = 1, VS_VHAT = 2, VS_DOBAR = 3, VS_DOE = 4 };
template <int C, int DK, int DV, typename TIN, int NTH = 256, int VS = VS_NONE>
__device__ __forceinline__ void load_v_rows_t(const GlaArgs& a, int h, const long long* rows, const void* src,
                                              uint32_t vr, int bz = 0, int n = 0) {
  using Cfg = ChunkCfg<C, DK, DV, TIN>;
  constexpr int NPV = cdiv(C * Cfg::NGV, NTH);
  const int tid = threadIdx.x;
  static_assert(VS == VS_NONE || std::is_same<TIN, float>::value, "value-gate scaling on the fp32 path only");
  if constexpr (std::is_same<TIN, __nv_bfloat16>::value) {
#pragma unroll
    for (int j = 0; j < NPV; ++j) {
      const int i = tid + NTH * j;
      int t, g;
      piece_of<Cfg::NGV>(i, t, g);
      if (i < C * Cfg::NGV) {
        const long long gr = rows[t];
        cp_async16_zfill(row_addr(vr, t, Cfg::SBO_V) + 128u * g,
                         reinterpret_cast<const TIN*>(src) + tok_row(gr, a, h) * DV + 8 * g, gr >= 0);
      }
    }
  } else {
    Piece<TIN, 8> pv[NPV];
#pragma unroll
    for (int j = 0; j < NPV; ++j) {
      const int i = tid + NTH * j;
      int t, g;
      piece_of<Cfg::NGV>(i, t, g);
      const long long gr = i < C * Cfg::NGV ? rows[t] : -1;
      pv[j].load(reinterpret_cast<const TIN*>(src) + tok_row(gr, a, h) * DV + 8 * g, gr >= 0);
    }
#pragma unroll
    for (int j = 0; j < NPV; ++j) {
      const int i = tid + NTH * j;
      int t, g;
      piece_of<Cfg::NGV>(i, t, g);
      if (i < C * Cfg::NGV) {
        float x[8];
        pv[j].unpack(x);
        if constexpr (VS != VS_NONE) {
          if (rows[t] >= 0) {
            const float* eq = a.gEQb + ((size_t)bz * a.L + (size_t)n * C + t) * DV + 8 * g;
            const float* ch = a.gCHb + ((size_t)bz * a.nchunks + n) * 4 * DV + 8 * g;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float f = __ldg(eq + e);
              if constexpr (VS == VS_VBAR) x[e] = __fdiv_rn(x[e], f);
              if constexpr (VS == VS_VHAT) x[e] = __fdiv_rn(x[e] * __ldg(ch + DV + e), f);
              if constexpr (VS == VS_DOBAR) x[e] *= f;
              if constexpr (VS == VS_DOE) x[e] *= f * __ldg(ch + e);
            }
          }
        }
        st_piece<Cfg::NTV, 8>(vr, t, Cfg::SBO_V, 8 * g, Cfg::VR_SZ, x);
      }
    }
  }
  if constexpr (Cfg::NPADV > 0) {
    const float zz[8] = {};
    for (int i = tid; i < C * Cfg::NPADV; i += NTH)
      st_piece<Cfg::NTV, 8>(vr, i / Cfg::NPADV, Cfg::SBO_V, DV + 8 * (i % Cfg::NPADV), Cfg::VR_SZ, zz);
  }
}

// ============================================================== chunk state
// Rows of a dS / dH accumulator (TMEM lane j = value channel j, columns `col0`
// + key channels) of this thread's channel half -> staging rows.
template <int C, int DK, int DV, typename TIN, int H>
__device__ __forceinline__ void stage_rows_dk(uint32_t tmem, int col0, float* sd, int pitch) {
  using Cfg = ChunkCfg<C, DK, DV, TIN>;
  constexpr int KO = H ? Cfg::DK0 : 0, KN = H ? Cfg::DK1 : Cfg::DK0;
  const int t = threadIdx.x & 127, wq = t >> 5;
  if (32 * wq >= DV) return;  // warp-uniform: these lanes hold no value channel
  float ds[cround(KN, 8)];
#pragma unroll
  for (int c = 0; c < cround(KN, 8); c += 8)
    tmem_ld8(tmem + (static_cast<uint32_t>(32 * wq) << 16) + col0 + KO + c, ds + c);
  tmem_ld_wait();
  if (t < DV) {
#pragma unroll
    for (int g = 0; g < KN / 4; ++g)
      *reinterpret_cast<float4*>(sd + t * pitch + KO + 4 * g) =
          make_float4(ds[4 * g], ds[4 * g + 1], ds[4 * g + 2], ds[4 * g + 3]);
  }
}

// ============================================================== gate
// Per (gate head, chunk): the inclusive cumsum b of the base-2 log decays over
// the chunk's tokens, per key channel, stored as the factors EQ = 2^(b - r)
// (r = b at the chunk's middle token) and the chunk constants {2^r,
// 2^(Gamma - r), 2^Gamma, Gamma}.  Computed once; every head that shares the
// gate reads them.  Tokens past the sequence end do not decay.  A chunk with a
// factor outside 2^+-115 is flagged in a.sflag and gets neutral factors (EQ = 1,
// constants {1, 0, 2^Gamma, Gamma}: the chunk kernels then form finite values
// there, the scans the right decay), and gla_strong.cu recomputes it exactly;
// without a flag array it sets DIG_ERR_GATE_RANGE.
template <int C, int DK>
__global__ void __launch_bounds__(256) gla_gate_kernel(const GlaArgs a) {
  constexpr int GP = DK + 4;     // row pitch (floats) of the cumsum buffer
  constexpr int NSG = 256 / DK;  // token segments of the cumsum
  constexpr int SEGL = cdiv(C, NSG);
  constexpr int NG = DK / 4;     // 4-channel groups of a token row
  static_assert(NSG >= 1 && NSG <= 8 && DK % 4 == 0, "cumsum segments");
  __shared__ __align__(16) float G[C * GP];
  __shared__ float segtot[8][DK];
  __shared__ float gam[DK];
  __shared__ long long grows[C];
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  const int tid = threadIdx.x;
  const int nunits = a.B * a.gate_heads * a.nchunks;
  bool bad = false;
  for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
    const int bz = u / a.nchunks, n = u - bz * a.nchunks;
    const int b = bz / a.gate_heads, hz = bz - b * a.gate_heads;
    if (tid < C) {
      const int p = n * C + tid;
      grows[tid] = p < a.L ? (long long)b * a.L + scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode) : -1;
    }
    __syncthreads();
    // ---- base-2 log decays of the chunk's tokens (consecutive threads: consecutive channel groups of a token)
    for (int i = tid; i < C * NG; i += 256) {
      const int t = i / NG, g = i - t * NG;
      const long long gr = grows[t];
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);  // padding tokens (and an absent gate) do not decay
      if (gr >= 0 && a.z != nullptr) {
        const float4 zz = __ldg(reinterpret_cast<const float4*>(a.z + ((size_t)gr * a.gate_heads + hz) * DK) + g);
        x = make_float4(log2_decay(zz.x, a.inv_tau), log2_decay(zz.y, a.inv_tau), log2_decay(zz.z, a.inv_tau),
                        log2_decay(zz.w, a.inv_tau));
      }
      *reinterpret_cast<float4*>(G + t * GP + 4 * g) = x;
    }
    __syncthreads();
    // ---- inclusive cumsum over the tokens, per key channel: token segments, then their prefixes
    const int sc = tid % DK, sg = tid / DK;
    const int t0 = sg * SEGL, t1 = min(C, t0 + SEGL);
    if (sg < NSG) {
      float acc = 0.f;
      for (int t = t0; t < t1; ++t) {
        acc += G[t * GP + sc];
        G[t * GP + sc] = acc;
      }
      segtot[sg][sc] = acc;
    }
    __syncthreads();
    if (sg < NSG) {
      float pre = 0.f, tot = 0.f;
      for (int s2 = 0; s2 < NSG; ++s2) {
        const float x = segtot[s2][sc];
        pre += s2 < sg ? x : 0.f;
        tot += x;
      }
      if (sg > 0)
        for (int t = t0; t < t1; ++t) G[t * GP + sc] += pre;
      if (sg == 0) gam[sc] = tot;
    }
    __syncthreads();
    // ---- gate factors and chunk constants
    const float* Gr = G + (C / 2 - 1) * GP;  // b at the reference token
    bool out_of_range = false;
    for (int i = tid; i < C * NG; i += 256) {
      const int t = i / NG, g = i - t * NG;
      const int p = n * C + t;
      if (p < a.L) {
        const float4 bt = *reinterpret_cast<const float4*>(G + t * GP + 4 * g);
        const float4 rr = *reinterpret_cast<const float4*>(Gr + 4 * g);
        const float d0 = bt.x - rr.x, d1 = bt.y - rr.y, d2 = bt.z - rr.z, d3 = bt.w - rr.w;
        out_of_range |= !(fmaxf(fmaxf(fabsf(d0), fabsf(d1)), fmaxf(fabsf(d2), fabsf(d3))) <= 115.f);
        *reinterpret_cast<float4*>(a.gEQ + ((size_t)bz * a.L + p) * DK + 4 * g) =
            make_float4(ex2(d0), ex2(d1), ex2(d2), ex2(d3));
      }
    }
    const float r = tid < DK ? Gr[tid] : 0.f, gm = tid < DK ? gam[tid] : 0.f;
    // uniform: the chunk leaves the range; after this barrier the cumsum buffer,
    // token table and segment totals may be rewritten by the next unit
    const bool strong = __syncthreads_or(out_of_range) != 0;
    if (strong && a.sflag == nullptr) bad = true;
    if (strong && a.sflag != nullptr) {  // this thread's factors of the chunk become neutral
      for (int i = tid; i < C * NG; i += 256) {
        const int t = i / NG, g = i - t * NG;
        const int p = n * C + t;
        if (p < a.L)
          *reinterpret_cast<float4*>(a.gEQ + ((size_t)bz * a.L + p) * DK + 4 * g) = make_float4(1.f, 1.f, 1.f, 1.f);
      }
    }
    if (tid < DK) {
      float* ch = a.gCH + ((size_t)bz * a.nchunks + n) * 4 * DK + tid;
      const bool neutral = strong && a.sflag != nullptr;
      ch[0 * DK] = neutral ? 1.f : exp2f(r);
      ch[1 * DK] = neutral ? 0.f : exp2f(gm - r);
      ch[2 * DK] = exp2f(gm);
      ch[3 * DK] = gm;
    }
    if (tid == 0 && a.sflag != nullptr) a.sflag[u] = strong ? 1 : 0;
  }
  if (bad) set_status(a.status, DIG_ERR_GATE_RANGE);
}

// ============================================================== chunk state
// Per unit: the chunk's state contribution dS = khat^T v with khat =
// k 2^(Gamma - b) = k 2^(Gamma - r) / EQ (value-major rows, to `dsn`), from the
// gate kernel's factors.  With BWD it also forms the chunk's state-gradient
// contribution dH = (q 2^b)^T dO, q 2^b = q EQ 2^r (to `dhn`), which the reverse
// scan turns into the gradient of every chunk's exit state.
// With EXT (value gate, fp32 inputs) v is scaled to v 2^(Gb - e) and dO to dO 2^e
// on load, so that dS and dH carry the value-side decays too.
template <int C, int DK, int DV, typename TIN, bool BWD, bool EXT = false>
__global__ void __launch_bounds__(256, StateCfg<C, DK, DV, TIN, BWD>::MINB) gla_chunk_state_kernel(const GlaArgs a) {
  using Cfg = ChunkCfg<C, DK, DV, TIN>;
  using SC = StateCfg<C, DK, DV, TIN, BWD>;
  constexpr int NTG = Cfg::NTG, NTV = Cfg::NTV, DKP = Cfg::DKP, PSK = Cfg::PSK;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ StateSmem sh;
  const int tid = threadIdx.x, warp = tid >> 5;
  if (warp == 0) {
    tmem_alloc(&sh.tmem, SC::TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&sh.bar, 1);
    fence_mbar_init();
  }
  if ((int)blockIdx.x < a.B * a.H * a.nchunks) fill_rows(a, blockIdx.x, C, sh.rows[0]);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  const uint32_t tmem = sh.tmem;
  const uint32_t sbase = smem_u32(smem);
  float* SD = reinterpret_cast<float*>(smem + SC::OFF_SD);  // [DV][SDP] dS staging, then dH
  const uint64_t dVRm = sdesc(sbase + SC::OFF_VR, Cfg::SBO_V, 128);
  const uint64_t dKHm = sdesc(sbase + SC::OFF_KH, Cfg::SBO_K, 128);
  const uint64_t dDOm = sdesc(sbase + SC::OFF_DO, Cfg::SBO_V, 128);
  const uint64_t dQBm = sdesc(sbase + SC::OFF_QB, Cfg::SBO_K, 128);
  const int nunits = a.B * a.H * a.nchunks;
  uint32_t ph = 0;
  bool timed_out = false;   // a wait of this thread gave up: the CTA stops after this unit
  if (tid == 0) sh.mma_pend = 0;

  // Row pieces of a unit, loaded one unit ahead: gate factors EQ = 2^(b - r),
  // the chunk constants and k (and q) are issued once the current unit's
  // operands are written, v (and dO) once its products have completed.
  // all of a thread's pieces share one channel group when the groups divide 32
  // (piece_of), and then one load of the chunk constants serves them all
  constexpr int NPC = 32 % Cfg::NGK == 0 ? 1 : Cfg::NPK;
  Piece<float, PSK> pe[Cfg::NPK], pc[NPC], pc0[BWD ? NPC : 1];
  Piece<TIN, PSK> pk[Cfg::NPK], pq[BWD ? Cfg::NPK : 1];
  auto issue_rows = [&](int u, const long long* rows) {
    const Unit U(a, u);
#pragma unroll
    for (int j = 0; j < Cfg::NPK; ++j) {
      const int i = tid + 256 * j;
      int t, g;
      piece_of<Cfg::NGK>(i, t, g);
      const long long gr = i < C * Cfg::NGK ? rows[t] : -1;
      const bool valid = gr >= 0;
      const size_t off = tok_row(gr, a, U.h) * DK + g * PSK;
      pk[j].load(reinterpret_cast<const TIN*>(a.k) + off, valid);
      if constexpr (BWD) pq[j].load(reinterpret_cast<const TIN*>(a.q) + off, valid);
      pe[j].load(a.gEQ + ((size_t)U.bz * a.L + (valid ? U.n * C + t : 0)) * DK + g * PSK, valid);
      if (j < NPC) {
        const float* ch = a.gCH + ((size_t)U.bz * a.nchunks + U.n) * 4 * DK + g * PSK;
        pc[j].load(ch + DK, i < C * Cfg::NGK);  // 2^(Gamma - r)
        if constexpr (BWD) pc0[j].load(ch, i < C * Cfg::NGK);  // 2^r
      }
    }
  };
  auto issue_vd = [&](int u, const long long* rows) {
    const Unit U(a, u);
    load_v_rows_t<C, DK, DV, TIN, 256, EXT ? VS_VHAT : VS_NONE>(a, U.h, rows, a.v, sbase + SC::OFF_VR, U.bz, U.n);
    if constexpr (BWD)
      load_v_rows_t<C, DK, DV, TIN, 256, EXT ? VS_DOE : VS_NONE>(a, U.h, rows, a.dO, sbase + SC::OFF_DO, U.bz, U.n);
  };
  if ((int)blockIdx.x < nunits) {
    issue_rows(blockIdx.x, sh.rows[0]);
    issue_vd(blockIdx.x, sh.rows[0]);
  }

  int it = 0;
  for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++it) {
    const Unit U(a, u);
    const int un = u + gridDim.x;
    const bool has_next = un < nunits;
    long long* rows_next = sh.rows[(it + 1) & 1];
    if (has_next) fill_rows(a, un, C, rows_next);  // read after the barrier before this unit's products
    // ---- khat = k 2^(Gamma - b) = k 2^(Gamma - r) / EQ   (BWD: and q 2^b = q EQ 2^r)
#pragma unroll
    for (int j = 0; j < Cfg::NPK; ++j) {
      const int i = tid + 256 * j;
      int t, g;
      piece_of<Cfg::NGK>(i, t, g);
      if (i < C * Cfg::NGK) {
        const bool valid = U.n * C + t < a.L;  // padding tokens hold zeros
        float kv[PSK], ev[PSK], cv[PSK];
        pk[j].unpack(kv);
        pe[j].unpack(ev);
        pc[NPC == 1 ? 0 : j].unpack(cv);
#pragma unroll
        for (int e = 0; e < PSK; ++e) kv[e] *= valid ? __fdividef(cv[e], ev[e]) : 0.f;
        st_piece<NTG, PSK>(sbase + SC::OFF_KH, t, Cfg::SBO_K, g * PSK, Cfg::AQ_SZ, kv);
        if constexpr (BWD) {
          float qv[PSK], c0[PSK];
          pq[j].unpack(qv);
          pc0[NPC == 1 ? 0 : j].unpack(c0);
#pragma unroll
          for (int e = 0; e < PSK; ++e) qv[e] *= valid ? ev[e] * c0[e] : 0.f;
          st_piece<NTG, PSK>(sbase + SC::OFF_QB, t, Cfg::SBO_K, g * PSK, Cfg::AQ_SZ, qv);
        }
      }
    }
    if constexpr (Cfg::NPAD > 0) {
      const float zz[4] = {0.f, 0.f, 0.f, 0.f};
      for (int i = tid; i < C * Cfg::NPAD; i += 256) {
        st_piece<NTG, 4>(sbase + SC::OFF_KH, i / Cfg::NPAD, Cfg::SBO_K, DK + 4 * (i % Cfg::NPAD), Cfg::AQ_SZ, zz);
        if constexpr (BWD)
          st_piece<NTG, 4>(sbase + SC::OFF_QB, i / Cfg::NPAD, Cfg::SBO_K, DK + 4 * (i % Cfg::NPAD), Cfg::AQ_SZ, zz);
      }
    }
    cp_async_wait_all();
    // ---- dS = v^T khat, dH = dO^T (q 2^b)  (M = value channels, N = key channels, K = tokens)
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // this unit's row pieces are consumed, and the next unit's row table (filled
    // at the top of this iteration) is visible after the barrier above
    if (has_next) issue_rows(un, rows_next);
    if (tid == 0) {
      mma_issue<NTV, NTG, C / 16>(tmem, dVRm, Cfg::VR_SZ, 2 * Cfg::SBO_V, dKHm, Cfg::AQ_SZ, 2 * Cfg::SBO_K,
                                  idesc_bf16(128, DKP, true, true), false);
      if constexpr (BWD)
        mma_issue<NTV, NTG, C / 16>(tmem + SC::TM_DH, dDOm, Cfg::VR_SZ, 2 * Cfg::SBO_V, dQBm, Cfg::AQ_SZ,
                                    2 * Cfg::SBO_K, idesc_bf16(128, DKP, true, true), false);
      mma_commit(&sh.bar);
      sh.mma_pend = 1;
      sh.mma_ph = ph;
    }
    if (!mbar_wait(&sh.bar, ph, spin_limit(a))) timed_out = true;
    else if (tid == 0) sh.mma_pend = 0;
    ph ^= 1u;
    tc_fence_after();
    if (has_next && !timed_out) issue_vd(un, rows_next);  // v (and dO) of this unit are consumed
    if (tid < 128) stage_rows_dk<C, DK, DV, TIN, 0>(tmem, 0, SD, SC::SDP);
    else stage_rows_dk<C, DK, DV, TIN, 1>(tmem, 0, SD, SC::SDP);
    if constexpr (BWD) {
      if (tid < 128) stage_rows_dk<C, DK, DV, TIN, 0>(tmem, SC::TM_DH, SD + DV * SC::SDP, SC::SDP);
      else stage_rows_dk<C, DK, DV, TIN, 1>(tmem, SC::TM_DH, SD + DV * SC::SDP, SC::SDP);
    }
    tc_fence_before();
    __syncthreads();
    // ---- coalesced copies of dS (and dH): DV x DK, contiguous per unit
    {
      float4* dst = reinterpret_cast<float4*>(a.dsn + (size_t)u * DV * DK);
      for (int i = tid; i < DV * DK / 4; i += 256) {
        const int row = i / (DK / 4), c4 = i - row * (DK / 4);
        __stcg(dst + i, *reinterpret_cast<const float4*>(SD + row * SC::SDP + 4 * c4));
      }
      if constexpr (BWD) {
        float4* dh = reinterpret_cast<float4*>(a.dhn + (size_t)u * DV * DK);
        for (int i = tid; i < DV * DK / 4; i += 256) {
          const int row = i / (DK / 4), c4 = i - row * (DK / 4);
          __stcg(dh + i, *reinterpret_cast<const float4*>(SD + (DV + row) * SC::SDP + 4 * c4));
        }
      }
    }
    // operands, staging and the cumsum buffer are reused by the next unit; after a
    // wait gave up anywhere in the CTA, no further unit starts
    if (__syncthreads_or(timed_out)) break;
  }
  // ---- drain: this thread's row copies, and the last products, complete before exit
  if (timed_out) set_status(a.status, DIG_ERR_DEVICE_TIMEOUT);
  cp_async_wait_all();
  if (tid == 0 && sh.mma_pend) mbar_wait(&sh.bar, sh.mma_ph, kSpinLimitNs);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, SC::TM_COLS);
}

// Issues D (+)= A * B with A's NA terms in TMEM (term i of K-step s at column
// a_tm + i * 8 + s * a_kstep) and B's NB terms in shared memory.
template <int NA, int NB, int KSTEPS>
__device__ __forceinline__ void mma_issue_ts(uint32_t dtm, uint32_t a_tm, uint32_t a_kstep, uint64_t b0,
                                             uint32_t b_term, uint32_t b_kstep, uint32_t idesc, bool accumulate) {
  constexpr int ORD = NA > NB ? NA : NB;
  bool first = !accumulate;
#pragma unroll
  for (int i = 0; i < NA; ++i) {
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      if (i + j >= ORD) continue;
#pragma unroll
      for (int s = 0; s < KSTEPS; ++s) {
        mma_bf16_ts(dtm, a_tm + i * 8 + s * a_kstep, b0 + (uint64_t)((j * b_term + s * b_kstep) >> 4), idesc,
                    first ? 0u : 1u);
        first = false;
      }
    }
  }
}

// O rows (TMEM lane t = token t) of this thread's channel half -> staging and
// the row's partial sum of squares.
int num_sms();
// Persistent grid: `per_sm` CTAs per SM (the residency each kernel is sized
// for), never more than there are units.  Units are independent, so CTAs that
// do not fit at once simply start later.
inline int persistent_grid(int per_sm, long long units) {
  const long long slots = (long long)per_sm * num_sms();
  return (int)(units < slots ? units : slots);
}

// Per-chunk dS (bwd = false, from k and v into `dsn`) or dH (bwd = true, from q
// and dO into `dhn`) by the tile-copy kernel (gla_state_tma.cu), for bf16 inputs
// with d_k = 32, d_v = 64 and 128-token chunks that tile the sequence.
// `launched` stays false when the tensor maps cannot be encoded.
bool gla_reduce_tma_eligible(const GlaArgs& a, int dk, int dv, int tin, int chunk);
cudaError_t launch_reduce_tma(const GlaArgs& a, bool bwd, cudaStream_t s, bool* launched);

// The value gate's factors: the gate kernel over the value channels, from zb
// into gEQb / gCHb.
template <int C, int DV>
cudaError_t launch_value_gate(const GlaArgs& a, cudaStream_t s) {
  GlaArgs g = a;
  g.z = a.zb;
  g.gEQ = a.gEQb;
  g.gCH = a.gCHb;
  g.sflag = nullptr;  // a value-gate chunk out of range is reported, not recomputed
  const long long gunits = (long long)a.B * a.gate_heads * a.nchunks;
  return launch_pdl(gla_gate_kernel<C, DV>, dim3(persistent_grid(4, gunits)), dim3(256), 0, s, g);
}

// Gate kernel(s), then chunk-state kernel (which reads the gate factors).
template <int C, int DK, int DV, typename TIN, bool BWD, bool EXT = false>
cudaError_t launch_chunk_state(const GlaArgs& a, cudaStream_t s) {
  using SC = StateCfg<C, DK, DV, TIN, BWD>;
  const long long units = (long long)a.B * a.H * a.nchunks;
  if (units <= 0) return cudaSuccess;
  const long long gunits = (long long)a.B * a.gate_heads * a.nchunks;
  cudaError_t e = launch_pdl(gla_gate_kernel<C, DK>, dim3(persistent_grid(4, gunits)), dim3(256), 0, s, a);
  if (e != cudaSuccess) return e;
  if constexpr (EXT) {
    if ((e = launch_value_gate<C, DV>(a, s)) != cudaSuccess) return e;
  }
  if (!EXT && std::is_same<TIN, __nv_bfloat16>::value && gla_reduce_tma_eligible(a, DK, DV, DIG_BF16, C)) {
    bool launched = false;
    if ((e = launch_reduce_tma(a, false, s, &launched)) != cudaSuccess) return e;
    if (launched && BWD && (e = launch_reduce_tma(a, true, s, &launched)) != cudaSuccess) return e;
    if (launched) return cudaSuccess;
  }
  auto k1 = gla_chunk_state_kernel<C, DK, DV, TIN, BWD, EXT>;
  if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, SC::SMEM)) != cudaSuccess) return e;
  return launch_pdl(k1, persistent_grid(SC::PER_SM, units), 256, SC::SMEM, s, a);
}

// Optional ends of the scans (per buffer): the carry entering the first step
// (NULL: zero) and the carry after the last step, written in the caller's
// [B*H][DK][DV] layout (fin) and in the state layout [B*H][DV][DK] (fin_rows).
struct ScanEnds {
  const float* seed[2];
  float* fin[2];
  float* fin_rows[2];
};
// Scan of per-chunk contributions X_n (DV x DK fp32 each, per sequence) into
// the state entering every chunk: Y_0 = 0 (or the seed), Y_{n+1} =
// diag(2^Gamma_n) Y_n diag(2^Gb_n) + X_n (Gb = 0 without a value gate; reverse:
// the same recurrence from the last chunk down, giving the gradient leaving
// every chunk).  In place in buf0 and, when not null, buf1 (one launch).
cudaError_t launch_state_scan(const GlaArgs& a, float* buf0, bool rev0, float* buf1, bool rev1, int dk, int dv,
                              cudaStream_t s, uint32_t* zero_word = nullptr, const ScanEnds* ends = nullptr);

}  // namespace dig
