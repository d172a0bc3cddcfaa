// gla_fwd.cu -- chunkwise Gated Linear Attention forward on sm_100a.
//
// What is computed (DiG slides, GLA eq. (5)-(8)): for every (batch, head)
// sequence, in scan order t,
//     alpha_t = exp(inv_tau * logsigmoid(z_t)),  S_t = diag(alpha_t) S_{t-1} + k_t^T v_t,
//     o_t = q_t S_t,
// evaluated chunkwise (slides "計算効率の分析", paper "Efficiency Analysis": the
// sequence is cut into chunks that fit on-chip).  For a chunk n of C tokens
// with entry state S_n, in-chunk inclusive base-2 log-decay cumsum b_t,
// reference r = b at the chunk's middle token and chunk decay Gamma = b_last:
//     qbar_t = q_t 2^(b_t - r),  kbar_s = k_s 2^(r - b_s),  khat_s = k_s 2^(Gamma - b_s)
//     P = (qbar kbar^T) masked to s <= t                          (tensor core, C x C)
//     O = qbar S'_n + P V,   S'_n = diag(2^r) S_n                  (tensor core)
//     S_{n+1} = diag(2^Gamma) S_n + khat^T V
// which equals the recurrence in exact arithmetic.
//
// Three kernels, each over independent (sequence, chunk) units:
//   1. gla_chunk_state_kernel: the gate of the chunk (cumsum over its tokens),
//      written once per gate head as per-token factors 2^(b - r) and per-chunk
//      constants; and the chunk's state contribution dS_n = khat^T V.
//   2. gla_state_scan_kernel: S_{n+1} = diag(2^Gamma_n) S_n + dS_n over the
//      chunks, an associative scan (sixteen chunk ranges per state element,
//      then a carry fold), overwriting dS_n with the entry state S_n.
//   3. gla_chunk_out_kernel: the outputs of every chunk from its entry state,
//      and the fused Swish(r) * RMSNorm(o) epilogue.
// No unit waits on another, so several CTAs share an SM and hide each other's
// memory latency; there is no inter-CTA signalling.
//
// Data movement: rows are gathered directly from the grid-ordered tensors at
// pi(t) (the SREM scan order is fused into the loads and stores; no permuted
// copy exists).  Loads, operand stores and output stores go by row pieces of
// 16 bytes spread so that a warp touches eight rows (coalesced global access,
// conflict-free shared memory); v is copied straight into its operand rows with
// asynchronous copies.  Operands are written in the tensor core's canonical
// K-major layout; accumulators live in TMEM (token row t is TMEM lane t) and are
// read back by row, then transposed through shared memory for the stores.
//
// Operand precision: the gated operands (qbar, kbar, khat, P, the state) are not
// representable in bf16, so each is stored as a sum of bf16 terms (hi + lo, or
// hi + mid + lo for fp32 inputs) and every product is issued as the pairs of
// terms whose combined order matters (kind::f16 MMAs, fp32 accumulation).  Two
// terms carry ~16 significant bits (relative error ~2^-17 per product), far
// below the bf16-input tolerance; three terms reach fp32 accuracy.  Raw bf16
// inputs (v) are exact in one term.  The masked P is converted to its terms in
// place in TMEM and read from there as the A operand of P V.
#include <type_traits>

#include "gla.h"
#include "gla_common.cuh"

namespace dig {

template <int C_, int DK_, int DV_, typename TIN>
struct ChunkCfg {
  static constexpr int C = C_, DK = DK_, DV = DV_;
  static constexpr int NTG = std::is_same<TIN, float>::value ? 3 : 2;  // terms of gated operands
  static constexpr int NTV = std::is_same<TIN, float>::value ? 3 : 1;  // terms of v
  static constexpr int DKP = cround(DK, 16), DVP = cround(DV, 16);
  // per-thread channel halves (multiples of 4 so rows stay 8/16-byte aligned)
  static constexpr int DK0 = cround((DK + 1) / 2, 4), DK1 = DK - DK0;
  static constexpr int DV0 = cround((DV + 1) / 2, 8), DV1 = DV - DV0;
  // Operands are token rows (bf16, K-major over channels, LBO = 128 between
  // 8-channel groups), read K-major or, for products that contract over
  // tokens, MN-major.  Row strides are padded by 64 bytes (when it fits) so the
  // four 8-row groups a warp writes alternate bank halves.
  static constexpr int PADK = DKP >= 64 ? 0 : 64;
  static constexpr int SBO_K = DKP * 16 + PADK;     // rows of DKP values (q, k, khat, S')
  static constexpr int SBO_V = DVP * 16 + 64;       // rows of DVP values (v)
  static constexpr int AQ_SZ = (C / 8) * SBO_K;     // one term, C rows
  static constexpr int VR_SZ = (C / 8) * SBO_V;     // one term, C rows
  static constexpr int SPT_SZ = (DVP / 8) * SBO_K;  // one term, DVP rows
  // ---- row pieces of the coalesced loads and stores (see piece_of)
  static constexpr int PSK = DK % 8 == 0 ? 8 : 4;  // channels per piece of q / k / khat rows
  static constexpr int NGK = DK / PSK;
  static constexpr int NPK = cdiv(C * NGK, 256);    // pieces per thread
  static constexpr int NGZ = DK / 4;                // gate logits / factors: 4 fp32 channels per piece
  static constexpr int NPZ = cdiv(C * NGZ, 256);
  static constexpr int NGS = DK / 4;                // state rows (fp32)
  static constexpr int NPS = cdiv(DV * NGS, 256);
  static constexpr int NGV = DV / 8;                // v / r / o / y rows: 8 channels per piece
  static constexpr int NPV = cdiv(C * NGV, 256);
  static constexpr int NPAD = (DKP - DK) / 4;       // zero pieces of the K padding, per row
  // ---- state kernel: khat, v, the token cumsum of the gate
  static constexpr int S_OFF_KH = 0;
  static constexpr int S_OFF_VR = NTG * AQ_SZ;
  // the M = 128 read of v^T (MN-major) covers 16 channel groups of every token group
  static constexpr int S_END_VR =
      cmax(S_OFF_VR + NTV * VR_SZ, S_OFF_VR + (NTV - 1) * VR_SZ + (C / 8 - 1) * SBO_V + 16 * 128);
  static constexpr int GP = DK + 4;                 // row pitch (floats) of the cumsum buffer
  static constexpr int S_OFF_G = cround(S_END_VR, 16);
  static constexpr int S_SMEM = S_OFF_G + C * GP * 4;
  static constexpr int SDP = DK + 4;                // row pitch of the dS staging rows (over khat)
  static_assert(DV * SDP * 4 <= NTG * AQ_SZ, "dS staging fits over khat");
  static constexpr int NSG = 256 / DK;              // token segments of the cumsum
  static constexpr int SEGL = cdiv(C, NSG);
  static constexpr int S_TM_COLS = pow2ceil(DKP);
  // ---- output kernel: qbar, kbar, S'^T, v
  static constexpr int O_OFF_AQ = 0;
  static constexpr int O_OFF_BK = NTG * AQ_SZ;
  static constexpr int O_OFF_SPT = 2 * NTG * AQ_SZ;
  static constexpr int O_OFF_VR = O_OFF_SPT + NTG * SPT_SZ;
  static constexpr int OP = DV + 4;                 // row pitch of the output staging (over the operands)
  // the M = 128 read of qbar covers 128 rows even where C = 64
  static constexpr int O_SMEM = cmax(cmax(O_OFF_VR + NTV * VR_SZ, O_OFF_AQ + (NTG - 1) * AQ_SZ + 16 * SBO_K),
                                     C * OP * 4);
  // TMEM columns: P (fp32), P as bf16 terms (8 columns per term and K-step,
  // the terms of K-step k at TM_PT + k * PT_STRIDE; in place over P when two
  // terms fit), O
  static constexpr int TM_P = 0;
  static constexpr int TM_PT = NTG == 2 ? 0 : C;
  static constexpr int PT_STRIDE = NTG * 8;
  static constexpr int TM_O = NTG == 2 ? C : C + NTG * C / 2;
  static constexpr int O_TM_COLS = pow2ceil(TM_O + DVP);
  static_assert(O_TM_COLS <= 256, "two output CTAs per SM share the 512 TMEM columns");
  static_assert(O_SMEM <= 110 * 1024, "two output CTAs per SM share shared memory");
  static constexpr int S_PER_SM = S_SMEM <= 72 * 1024 ? 3 : 2;  // state CTAs per SM
  static_assert(S_SMEM <= 110 * 1024, "two state CTAs per SM share shared memory");
  static_assert(DK % 4 == 0 && DV % 8 == 0 && DK1 > 0 && DV1 > 0, "head dims");
  static_assert(NSG <= 8 && DK <= 64, "cumsum segments");
  static_assert(C == 64 || C == 128, "chunk");
};

struct StateSmem {
  float segtot[8][64];  // cumsum totals of the token segments
  float gam[64];        // chunk decay Gamma (log2)
  uint64_t bar;
  uint32_t tmem;
};

struct OutSmem {
  float red[256];  // epilogue row sums of squares
  uint64_t bar_a;  // P, qbar S'
  uint64_t bar_b;  // P V
  uint32_t tmem;
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

// v rows of the unit's chunk into a K-major operand buffer at `vr` (token rows
// of DVP channels).  bf16 values are copied unchanged (one exact term) by
// asynchronous 16-byte copies, zero-filled past the sequence end (complete
// after cp_async_wait_all); fp32 values are split into three bf16 terms.
template <int C, int DK, int DV, typename TIN>
__device__ __forceinline__ void load_v_rows(const GlaArgs& a, const Unit& U, uint32_t vr) {
  using Cfg = ChunkCfg<C, DK, DV, TIN>;
  const int tid = threadIdx.x;
  if constexpr (std::is_same<TIN, __nv_bfloat16>::value) {
#pragma unroll
    for (int j = 0; j < Cfg::NPV; ++j) {
      const int i = tid + 256 * j;
      int t, g;
      piece_of<Cfg::NGV>(i, t, g);
      if (i < C * Cfg::NGV) {
        const int p = U.n * C + t;
        const bool valid = p < a.L;
        const long long grow = valid ? (long long)U.b * a.L + scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode) : 0;
        cp_async16_zfill(row_addr(vr, t, Cfg::SBO_V) + 128u * g,
                         reinterpret_cast<const TIN*>(a.v) + ((size_t)grow * a.H + U.h) * DV + 8 * g, valid);
      }
    }
  } else {
    Piece<TIN, 8> pv[Cfg::NPV];
#pragma unroll
    for (int j = 0; j < Cfg::NPV; ++j) {
      const int i = tid + 256 * j;
      int t, g;
      piece_of<Cfg::NGV>(i, t, g);
      const int p = U.n * C + t;
      const bool valid = i < C * Cfg::NGV && p < a.L;
      const long long grow = valid ? (long long)U.b * a.L + scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode) : 0;
      pv[j].load(reinterpret_cast<const TIN*>(a.v) + ((size_t)grow * a.H + U.h) * DV + 8 * g, valid);
    }
#pragma unroll
    for (int j = 0; j < Cfg::NPV; ++j) {
      const int i = tid + 256 * j;
      int t, g;
      piece_of<Cfg::NGV>(i, t, g);
      if (i < C * Cfg::NGV) {
        float x[8];
        pv[j].unpack(x);
        st_piece<Cfg::NTV, 8>(vr, t, Cfg::SBO_V, 8 * g, Cfg::VR_SZ, x);
      }
    }
  }
}

// ============================================================== 1. chunk state
// dS rows (TMEM lane j = value channel j) of this thread's channel half -> staging.
template <int C, int DK, int DV, typename TIN, int H>
__device__ __forceinline__ void stage_ds(uint32_t tmem, float* sd) {
  using Cfg = ChunkCfg<C, DK, DV, TIN>;
  constexpr int KO = H ? Cfg::DK0 : 0, KN = H ? Cfg::DK1 : Cfg::DK0;
  const int t = threadIdx.x & 127, wq = t >> 5;
  if (32 * wq >= DV) return;  // warp-uniform: these lanes hold no value channel
  float ds[cround(KN, 8)];
#pragma unroll
  for (int c = 0; c < cround(KN, 8); c += 8) tmem_ld8(tmem + (static_cast<uint32_t>(32 * wq) << 16) + KO + c, ds + c);
  tmem_ld_wait();
  if (t < DV) {
#pragma unroll
    for (int g = 0; g < KN / 4; ++g)
      *reinterpret_cast<float4*>(sd + t * Cfg::SDP + KO + 4 * g) =
          make_float4(ds[4 * g], ds[4 * g + 1], ds[4 * g + 2], ds[4 * g + 3]);
  }
}

template <int C, int DK, int DV, typename TIN>
__global__ void __launch_bounds__(256, 3) gla_chunk_state_kernel(const GlaArgs a) {
  using Cfg = ChunkCfg<C, DK, DV, TIN>;
  constexpr int NTG = Cfg::NTG, NTV = Cfg::NTV, DKP = Cfg::DKP, PSK = Cfg::PSK;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ StateSmem sh;
  const int tid = threadIdx.x, warp = tid >> 5;
  if (warp == 0) {
    tmem_alloc(&sh.tmem, Cfg::S_TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&sh.bar, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem;
  const uint32_t sbase = smem_u32(smem);
  float* G = reinterpret_cast<float*>(smem + Cfg::S_OFF_G);  // [C][GP] cumsum of log2 decays
  float* SD = reinterpret_cast<float*>(smem);                // [DV][SDP] dS staging (over khat)
  const uint64_t dVRm = sdesc(sbase + Cfg::S_OFF_VR, Cfg::SBO_V, 128);
  const uint64_t dKHm = sdesc(sbase + Cfg::S_OFF_KH, Cfg::SBO_K, 128);
  const int nunits = a.B * a.H * a.nchunks;
  uint32_t ph = 0;
  bool timed_out = false, bad = false;

  for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
    const Unit U(a, u);
    const bool writer = a.gate_heads != 1 || U.h == 0;  // one unit per gate head stores the factors
    const int hz = U.bz - U.b * a.gate_heads;
    // ---- loads: gate logits, k pieces; v straight into its operand rows
    Piece<float, 4> pz[Cfg::NPZ];
    Piece<TIN, PSK> pk[Cfg::NPK];
#pragma unroll
    for (int j = 0; j < Cfg::NPZ; ++j) {
      const int i = tid + 256 * j;
      int t, g;
      piece_of<Cfg::NGZ>(i, t, g);
      const int p = U.n * C + t;
      const bool valid = i < C * Cfg::NGZ && p < a.L;
      const long long grow = valid ? (long long)U.b * a.L + scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode) : 0;
      pz[j].load(a.z + ((size_t)grow * a.gate_heads + hz) * DK + 4 * g, valid);
    }
#pragma unroll
    for (int j = 0; j < Cfg::NPK; ++j) {
      const int i = tid + 256 * j;
      int t, g;
      piece_of<Cfg::NGK>(i, t, g);
      const int p = U.n * C + t;
      const bool valid = i < C * Cfg::NGK && p < a.L;
      const long long grow = valid ? (long long)U.b * a.L + scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode) : 0;
      pk[j].load(reinterpret_cast<const TIN*>(a.k) + ((size_t)grow * a.H + U.h) * DK + g * PSK, valid);
    }
    load_v_rows<C, DK, DV, TIN>(a, U, sbase + Cfg::S_OFF_VR);
    // ---- inclusive cumsum over the chunk's tokens, per key channel (shared memory)
#pragma unroll
    for (int j = 0; j < Cfg::NPZ; ++j) {
      const int i = tid + 256 * j;
      int t, g;
      piece_of<Cfg::NGZ>(i, t, g);
      if (i < C * Cfg::NGZ) {
        const int p = U.n * C + t;
        float zz[4];
        pz[j].unpack(zz);
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);  // padding tokens do not decay
        if (p < a.L)
          x = make_float4(log2_decay(zz[0], a.inv_tau), log2_decay(zz[1], a.inv_tau), log2_decay(zz[2], a.inv_tau),
                          log2_decay(zz[3], a.inv_tau));
        *reinterpret_cast<float4*>(G + t * Cfg::GP + 4 * g) = x;
      }
    }
    __syncthreads();
    const int sc = tid % DK, sg = tid / DK;
    const int t0 = sg * Cfg::SEGL, t1 = min(C, t0 + Cfg::SEGL);
    if (sg < Cfg::NSG) {
      float acc = 0.f;
      for (int t = t0; t < t1; ++t) {
        acc += G[t * Cfg::GP + sc];
        G[t * Cfg::GP + sc] = acc;
      }
      sh.segtot[sg][sc] = acc;
    }
    __syncthreads();
    if (sg < Cfg::NSG) {
      float pre = 0.f, tot = 0.f;
      for (int s2 = 0; s2 < Cfg::NSG; ++s2) {
        const float x = sh.segtot[s2][sc];
        pre += s2 < sg ? x : 0.f;
        tot += x;
      }
      if (sg > 0)
        for (int t = t0; t < t1; ++t) G[t * Cfg::GP + sc] += pre;
      if (sg == 0) sh.gam[sc] = tot;
    }
    __syncthreads();
    const float* Gr = G + (C / 2 - 1) * Cfg::GP;  // b at the reference token
    // ---- gate factors (one writer per gate head)
#pragma unroll
    for (int j = 0; j < Cfg::NPZ; ++j) {
      const int i = tid + 256 * j;
      int t, g;
      piece_of<Cfg::NGZ>(i, t, g);
      const int p = U.n * C + t;
      if (i < C * Cfg::NGZ && p < a.L) {
        const float4 bt = *reinterpret_cast<const float4*>(G + t * Cfg::GP + 4 * g);
        const float4 rr = *reinterpret_cast<const float4*>(Gr + 4 * g);
        const float d0 = bt.x - rr.x, d1 = bt.y - rr.y, d2 = bt.z - rr.z, d3 = bt.w - rr.w;
        bad |= fmaxf(fmaxf(fabsf(d0), fabsf(d1)), fmaxf(fabsf(d2), fabsf(d3))) > 115.f;
        if (writer)
          *reinterpret_cast<float4*>(a.gEQ + ((size_t)U.bz * a.L + p) * DK + 4 * g) =
              make_float4(exp2f(d0), exp2f(d1), exp2f(d2), exp2f(d3));
      }
    }
    if (writer && tid < DK) {
      float* ch = a.gCH + ((size_t)U.bz * a.nchunks + U.n) * 4 * DK + tid;
      const float r = Gr[tid], gm = sh.gam[tid];
      ch[0 * DK] = exp2f(r);
      ch[1 * DK] = exp2f(gm - r);
      ch[2 * DK] = exp2f(gm);
      ch[3 * DK] = gm;
    }
    // ---- khat = k * 2^(Gamma - b)
#pragma unroll
    for (int j = 0; j < Cfg::NPK; ++j) {
      const int i = tid + 256 * j;
      int t, g;
      piece_of<Cfg::NGK>(i, t, g);
      if (i < C * Cfg::NGK) {
        float kv[PSK];
        pk[j].unpack(kv);
#pragma unroll
        for (int e = 0; e < PSK; ++e) kv[e] *= exp2f(sh.gam[g * PSK + e] - G[t * Cfg::GP + g * PSK + e]);
        st_piece<NTG, PSK>(sbase + Cfg::S_OFF_KH, t, Cfg::SBO_K, g * PSK, Cfg::AQ_SZ, kv);
      }
    }
    if constexpr (Cfg::NPAD > 0) {
      const float zz[4] = {0.f, 0.f, 0.f, 0.f};
      for (int i = tid; i < C * Cfg::NPAD; i += 256)
        st_piece<NTG, 4>(sbase + Cfg::S_OFF_KH, i / Cfg::NPAD, Cfg::SBO_K, DK + 4 * (i % Cfg::NPAD), Cfg::AQ_SZ, zz);
    }
    cp_async_wait_all();
    // ---- dS = v^T khat (M = value channels, N = key channels, K = tokens)
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      mma_issue<NTV, NTG, C / 16>(tmem, dVRm, Cfg::VR_SZ, 2 * Cfg::SBO_V, dKHm, Cfg::AQ_SZ, 2 * Cfg::SBO_K,
                                  idesc_bf16(128, DKP, true, true), false);
      mma_commit(&sh.bar);
    }
    if (!mbar_wait(&sh.bar, ph, kSpinLimitNs)) timed_out = true;
    ph ^= 1u;
    tc_fence_after();
    if (tid < 128) stage_ds<C, DK, DV, TIN, 0>(tmem, SD);
    else stage_ds<C, DK, DV, TIN, 1>(tmem, SD);
    tc_fence_before();
    __syncthreads();
    // ---- coalesced copy of dS (DV x DK, contiguous per unit)
    float4* dst = reinterpret_cast<float4*>(a.dsn + (size_t)u * DV * DK);
    for (int i = tid; i < DV * DK / 4; i += 256) {
      const int row = i / (DK / 4), c4 = i - row * (DK / 4);
      __stcg(dst + i, *reinterpret_cast<const float4*>(SD + row * Cfg::SDP + 4 * c4));
    }
    __syncthreads();  // operands, staging and the cumsum buffer are reused by the next unit
  }
  if (bad) set_status(a.status, DIG_ERR_GATE_RANGE);
  if (timed_out) set_status(a.status, DIG_ERR_DEVICE_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, Cfg::S_TM_COLS);
}

// ============================================================== 2. state scan
// One block covers 128 state elements (32 quads of 4) of one sequence; warp w
// of 16 owns chunks [w*per, (w+1)*per) of them, loaded eight chunks at a time.
// Pass 1 folds each range into (decay product A, partial state s); the carry
// entering range w is the fold of ranges 0..w-1; pass 2 rewrites dS_n with the
// state entering chunk n.
constexpr int kScanRanges = 16;
__global__ void __launch_bounds__(32 * kScanRanges) gla_state_scan_kernel(const GlaArgs a, int dk, int dv) {
  __shared__ float4 sA[kScanRanges][32], sS[kScanRanges][32];
  const int nq = dv * dk / 4;
  const int nblk = (nq + 31) / 32;
  const int bh = blockIdx.x / nblk, blk = blockIdx.x - bh * nblk;
  const int lanei = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int quad = blk * 32 + lanei;
  const bool act = quad < nq;
  const int c0 = (quad * 4) % dk;  // the quad's four key channels (dk % 4 == 0)
  const int b = bh / a.H, h = bh - b * a.H;
  const int bz = b * a.gate_heads + (a.gate_heads == 1 ? 0 : h);
  const int nch = a.nchunks;
  const int per = (nch + kScanRanges - 1) / kScanRanges;
  const int n0 = min(nch, w * per), n1 = min(nch, n0 + per);
  float4* st = reinterpret_cast<float4*>(a.dsn + (size_t)bh * nch * dv * dk) + quad;
  const size_t st_stride = (size_t)nq;
  const float* dec = a.gCH + ((size_t)bz * nch * 4 + 2) * dk + c0;  // 2^Gamma of chunk n at dec + n * 4 * dk
  auto fma4 = [](float4 g, float4 s, float4 d) {
    return make_float4(fmaf(g.x, s.x, d.x), fmaf(g.y, s.y, d.y), fmaf(g.z, s.z, d.z), fmaf(g.w, s.w, d.w));
  };
  float4 A = make_float4(1.f, 1.f, 1.f, 1.f), s = make_float4(0.f, 0.f, 0.f, 0.f);
  if (act) {
    for (int w0 = n0; w0 < n1; w0 += 8) {
      float4 g[8], d[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (w0 + e < n1) {
          g[e] = __ldg(reinterpret_cast<const float4*>(dec + (size_t)(w0 + e) * 4 * dk));
          d[e] = __ldcg(st + (w0 + e) * st_stride);
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (w0 + e < n1) {
          s = fma4(g[e], s, d[e]);
          A = make_float4(g[e].x * A.x, g[e].y * A.y, g[e].z * A.z, g[e].w * A.w);
        }
      }
    }
  }
  sA[w][lanei] = A;
  sS[w][lanei] = s;
  __syncthreads();
  if (!act) return;
  float4 S = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int m = 0; m < w; ++m) S = fma4(sA[m][lanei], S, sS[m][lanei]);
  for (int w0 = n0; w0 < n1; w0 += 8) {
    float4 g[8], d[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (w0 + e < n1) {
        g[e] = __ldg(reinterpret_cast<const float4*>(dec + (size_t)(w0 + e) * 4 * dk));
        d[e] = __ldcg(st + (w0 + e) * st_stride);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (w0 + e < n1) {
        __stcg(st + (w0 + e) * st_stride, S);
        S = fma4(g[e], S, d[e]);
      }
    }
  }
}

// ============================================================== 3. outputs
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
template <int C, int DK, int DV, typename TIN, int H>
__device__ __forceinline__ void stage_o(uint32_t tmem, float* stage, float* red) {
  using Cfg = ChunkCfg<C, DK, DV, TIN>;
  constexpr int VO = H ? Cfg::DV0 : 0, VN = H ? Cfg::DV1 : Cfg::DV0;
  const int tid = threadIdx.x, t = tid & 127, wq = t >> 5;
  float ov[cround(VN, 8)];
#pragma unroll
  for (int c = 0; c < cround(VN, 8); c += 8)
    tmem_ld8(tmem + (static_cast<uint32_t>(32 * wq) << 16) + Cfg::TM_O + VO + c, ov + c);
  tmem_ld_wait();
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < VN; ++i) ss += ov[i] * ov[i];
  red[tid] = ss;
  if (t < C) {
#pragma unroll
    for (int g = 0; g < VN / 4; ++g)
      *reinterpret_cast<float4*>(stage + t * Cfg::OP + VO + 4 * g) =
          make_float4(ov[4 * g], ov[4 * g + 1], ov[4 * g + 2], ov[4 * g + 3]);
  }
}

template <int C, int DK, int DV, typename TIN, typename TOUT>
__global__ void __launch_bounds__(256, 2) gla_chunk_out_kernel(const GlaArgs a) {
  using Cfg = ChunkCfg<C, DK, DV, TIN>;
  constexpr int NTG = Cfg::NTG, NTV = Cfg::NTV, DKP = Cfg::DKP, DVP = Cfg::DVP, PSK = Cfg::PSK;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ OutSmem sh;
  const int tid = threadIdx.x, warp = tid >> 5;
  if (warp == 0) {
    tmem_alloc(&sh.tmem, Cfg::O_TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&sh.bar_a, 1);
    mbar_init(&sh.bar_b, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int t = tid & 127, wq = (tid >> 5) & 3, half = tid >> 7;
  const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
  const uint32_t tmem = sh.tmem;
  const uint32_t sbase = smem_u32(smem);
  float* stage = reinterpret_cast<float*>(smem);  // [C][OP] output rows, over the operands
  const uint64_t dAQ = sdesc(sbase + Cfg::O_OFF_AQ, 128, Cfg::SBO_K);
  const uint64_t dBK = sdesc(sbase + Cfg::O_OFF_BK, 128, Cfg::SBO_K);
  const uint64_t dSPT = sdesc(sbase + Cfg::O_OFF_SPT, 128, Cfg::SBO_K);
  const uint64_t dVRm = sdesc(sbase + Cfg::O_OFF_VR, Cfg::SBO_V, 128);
  const int nunits = a.B * a.H * a.nchunks;
  const bool with_y = a.y != nullptr && a.r != nullptr;
  uint32_t ph = 0;
  bool timed_out = false;

  for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
    const Unit U(a, u);
    // ---- loads: q, k and gate-factor pieces, the entry-state rows; v straight into its operand rows
    Piece<TIN, PSK> pq[Cfg::NPK], pk[Cfg::NPK];
    Piece<float, PSK> pe[Cfg::NPK];
#pragma unroll
    for (int j = 0; j < Cfg::NPK; ++j) {
      const int i = tid + 256 * j;
      int tt, g;
      piece_of<Cfg::NGK>(i, tt, g);
      const int p = U.n * C + tt;
      const bool valid = i < C * Cfg::NGK && p < a.L;
      const long long grow = valid ? (long long)U.b * a.L + scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode) : 0;
      const size_t off = ((size_t)grow * a.H + U.h) * DK + g * PSK;
      pq[j].load(reinterpret_cast<const TIN*>(a.q) + off, valid);
      pk[j].load(reinterpret_cast<const TIN*>(a.k) + off, valid);
      pe[j].load(a.gEQ + ((size_t)U.bz * a.L + (valid ? p : 0)) * DK + g * PSK, valid);
    }
    Piece<float, 4> ps[Cfg::NPS], pc[Cfg::NPS];
#pragma unroll
    for (int j = 0; j < Cfg::NPS; ++j) {
      const int i = tid + 256 * j;
      int jr, g;
      piece_of<Cfg::NGS>(i, jr, g);
      const bool in = i < DV * Cfg::NGS;
      ps[j].load_cg(a.dsn + ((size_t)u * DV + (in ? jr : 0)) * DK + 4 * g, in);
      pc[j].load(a.gCH + ((size_t)U.bz * a.nchunks + U.n) * 4 * DK + 4 * g, in);
    }
    load_v_rows<C, DK, DV, TIN>(a, U, sbase + Cfg::O_OFF_VR);
    // ---- operands: qbar = q 2^(b-r), kbar = k 2^(r-b); S'^T rows = (2^r S_n)[:, j]
#pragma unroll
    for (int j = 0; j < Cfg::NPK; ++j) {
      const int i = tid + 256 * j;
      int tt, g;
      piece_of<Cfg::NGK>(i, tt, g);
      if (i < C * Cfg::NGK) {
        const bool valid = U.n * C + tt < a.L;
        float qv[PSK], kv[PSK], ev[PSK];
        pq[j].unpack(qv);
        pk[j].unpack(kv);
        pe[j].unpack(ev);
#pragma unroll
        for (int e = 0; e < PSK; ++e) {
          const float f = valid ? ev[e] : 1.f;
          qv[e] *= f;
          kv[e] *= __fdividef(1.f, f);
        }
        st_piece<NTG, PSK>(sbase + Cfg::O_OFF_AQ, tt, Cfg::SBO_K, g * PSK, Cfg::AQ_SZ, qv);
        st_piece<NTG, PSK>(sbase + Cfg::O_OFF_BK, tt, Cfg::SBO_K, g * PSK, Cfg::AQ_SZ, kv);
      }
    }
#pragma unroll
    for (int j = 0; j < Cfg::NPS; ++j) {
      const int i = tid + 256 * j;
      int jr, g;
      piece_of<Cfg::NGS>(i, jr, g);
      if (i < DV * Cfg::NGS) {
        float sv[4], cv[4];
        ps[j].unpack(sv);
        pc[j].unpack(cv);
#pragma unroll
        for (int e = 0; e < 4; ++e) sv[e] *= cv[e];
        st_piece<NTG, 4>(sbase + Cfg::O_OFF_SPT, jr, Cfg::SBO_K, 4 * g, Cfg::SPT_SZ, sv);
      }
    }
    if constexpr (Cfg::NPAD > 0) {  // zero K padding (the output staging of the previous unit overwrote it)
      const float zz[4] = {0.f, 0.f, 0.f, 0.f};
      for (int i = tid; i < C * Cfg::NPAD; i += 256) {
        const int row = i / Cfg::NPAD, c = DK + 4 * (i % Cfg::NPAD);
        st_piece<NTG, 4>(sbase + Cfg::O_OFF_AQ, row, Cfg::SBO_K, c, Cfg::AQ_SZ, zz);
        st_piece<NTG, 4>(sbase + Cfg::O_OFF_BK, row, Cfg::SBO_K, c, Cfg::AQ_SZ, zz);
        if (row < DV) st_piece<NTG, 4>(sbase + Cfg::O_OFF_SPT, row, Cfg::SBO_K, c, Cfg::SPT_SZ, zz);
      }
    }
    cp_async_wait_all();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      mma_issue<NTG, NTG, DKP / 16>(tmem + Cfg::TM_P, dAQ, Cfg::AQ_SZ, 256, dBK, Cfg::AQ_SZ, 256, idesc_bf16(128, C),
                                    false);
      mma_issue<NTG, NTG, DKP / 16>(tmem + Cfg::TM_O, dAQ, Cfg::AQ_SZ, 256, dSPT, Cfg::SPT_SZ, 256,
                                    idesc_bf16(128, DVP), false);
      mma_commit(&sh.bar_a);
    }
    if (!mbar_wait(&sh.bar_a, ph, kSpinLimitNs)) timed_out = true;
    tc_fence_after();
    // ---- mask P (s <= t) and store it as bf16 terms in TMEM, one K-step of 16 at a time
    if (32 * wq < C) {  // warp-uniform: lanes that are token rows
#pragma unroll
      for (int kk = 0; kk < C / 32; ++kk) {
        const int s0 = half * (C / 2) + 16 * kk;
        float pv[16];
        if (s0 <= 32 * wq + 31) {
          tmem_ld16(tmem + lane_base + Cfg::TM_P + s0, pv);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) pv[e] = (s0 + e <= t) ? pv[e] : 0.f;
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) pv[e] = 0.f;  // the whole warp's rows precede this block
        }
#pragma unroll
        for (int i = 0; i < NTG; ++i) {
          uint32_t pk8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const __nv_bfloat162 hb = __floats2bfloat162_rn(pv[2 * e], pv[2 * e + 1]);
            pk8[e] = *reinterpret_cast<const uint32_t*>(&hb);
            pv[2 * e] -= __low2float(hb);
            pv[2 * e + 1] -= __high2float(hb);
          }
          tmem_st8(tmem + lane_base + Cfg::TM_PT + (s0 / 16) * Cfg::PT_STRIDE + 8 * i, pk8);
        }
      }
      tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      mma_issue_ts<NTG, NTV, C / 16>(tmem + Cfg::TM_O, tmem + Cfg::TM_PT, Cfg::PT_STRIDE, dVRm, Cfg::VR_SZ,
                                     2 * Cfg::SBO_V, idesc_bf16(128, DVP, false, true), true);
      mma_commit(&sh.bar_b);
    }
    // ---- epilogue inputs while P V runs
    Piece<TIN, 8> pr[Cfg::NPV];
    if (with_y) {
#pragma unroll
      for (int j = 0; j < Cfg::NPV; ++j) {
        const int i = tid + 256 * j;
        int tt, g;
        piece_of<Cfg::NGV>(i, tt, g);
        const int p = U.n * C + tt;
        const bool valid = i < C * Cfg::NGV && p < a.L;
        const long long grow = valid ? (long long)U.b * a.L + scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode) : 0;
        pr[j].load(reinterpret_cast<const TIN*>(a.r) + ((size_t)grow * a.H + U.h) * DV + 8 * g, valid);
      }
    }
    if (!mbar_wait(&sh.bar_b, ph, kSpinLimitNs)) timed_out = true;
    ph ^= 1u;
    tc_fence_after();
    if (tid < 128) stage_o<C, DK, DV, TIN, 0>(tmem, stage, sh.red);
    else stage_o<C, DK, DV, TIN, 1>(tmem, stage, sh.red);
    tc_fence_before();
    __syncthreads();
    // ---- o and y rows, 8 channels per piece
#pragma unroll
    for (int j = 0; j < Cfg::NPV; ++j) {
      const int i = tid + 256 * j;
      int tt, g;
      piece_of<Cfg::NGV>(i, tt, g);
      const int p = U.n * C + tt;
      if (i < C * Cfg::NGV && p < a.L) {
        const long long grow = (long long)U.b * a.L + scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode);
        const size_t off = ((size_t)grow * a.H + U.h) * DV + 8 * g;
        float ov[8];
        const float4 o0 = *reinterpret_cast<const float4*>(stage + tt * Cfg::OP + 8 * g);
        const float4 o1 = *reinterpret_cast<const float4*>(stage + tt * Cfg::OP + 8 * g + 4);
        ov[0] = o0.x; ov[1] = o0.y; ov[2] = o0.z; ov[3] = o0.w;
        ov[4] = o1.x; ov[5] = o1.y; ov[6] = o1.z; ov[7] = o1.w;
        st_global8(reinterpret_cast<TOUT*>(a.o) + off, ov);
        if (with_y) {
          const float inv = rsqrtf((sh.red[tt] + sh.red[tt + 128]) / (float)DV + a.eps);
          float rv[8], yv[8];
          pr[j].unpack(rv);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float gmm = a.gamma != nullptr ? __ldg(a.gamma + 8 * g + e) : 1.f;
            const float sw = rv[e] / (1.f + exp2f(-rv[e] * kLog2e));
            yv[e] = sw * ov[e] * inv * gmm;
          }
          st_global8(reinterpret_cast<TOUT*>(a.y) + off, yv);
        }
      }
    }
    __syncthreads();  // staging and row sums are rewritten by the next unit
  }
  if (timed_out) set_status(a.status, DIG_ERR_DEVICE_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, Cfg::O_TM_COLS);
}

// ------------------------------------------------------------------ launch
namespace {

int g_sms_cache[64];
int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (g_sms_cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sms_cache[dev] = n;
  }
  return g_sms_cache[dev];
}

// Persistent grid: `per_sm` CTAs per SM (the residency each kernel is sized
// for), never more than there are units.  Units are independent, so CTAs
// that do not fit at once simply start later.
int persistent_grid(int per_sm, long long units) {
  const long long slots = (long long)per_sm * num_sms();
  return (int)(units < slots ? units : slots);
}

template <int C, int DK, int DV, typename TIN, typename TOUT>
cudaError_t launch_typed(const GlaArgs& a, cudaStream_t s) {
  using Cfg = ChunkCfg<C, DK, DV, TIN>;
  const long long units = (long long)a.B * a.H * a.nchunks;
  if (units <= 0) return cudaSuccess;
  auto k1 = gla_chunk_state_kernel<C, DK, DV, TIN>;
  auto k3 = gla_chunk_out_kernel<C, DK, DV, TIN, TOUT>;
  cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::S_SMEM);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::O_SMEM);
  if (e != cudaSuccess) return e;
  k1<<<persistent_grid(Cfg::S_PER_SM, units), 256, Cfg::S_SMEM, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int nq = DV * DK / 4;
  const long long scan_blocks = (long long)a.B * a.H * ((nq + 31) / 32);
  if (scan_blocks > 2147483647LL) return cudaErrorInvalidValue;
  gla_state_scan_kernel<<<(unsigned)scan_blocks, 32 * kScanRanges, 0, s>>>(a, DK, DV);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k3<<<persistent_grid(2, units), 256, Cfg::O_SMEM, s>>>(a);
  return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t dispatch_types(const GlaVariant& v, const GlaArgs& a, cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (v.tin == DIG_BF16) {
    if (v.tout == DIG_BF16) return launch_typed<128, DK, DV, bf, bf>(a, s);
    return launch_typed<128, DK, DV, bf, float>(a, s);
  }
  if (v.tout == DIG_BF16) return launch_typed<64, DK, DV, float, bf>(a, s);
  return launch_typed<64, DK, DV, float, float>(a, s);
}

}  // namespace

bool gla_variant_built(int dk, int dv) {
  return (dk == 32 && dv == 64) || (dk == 36 && dv == 72) || (dk == 64 && dv == 64);
}

cudaError_t launch_gla_fwd(const GlaVariant& v, const GlaArgs& a, cudaStream_t s) {
  if (v.dk == 32 && v.dv == 64) return dispatch_types<32, 64>(v, a, s);
  if (v.dk == 36 && v.dv == 72) return dispatch_types<36, 72>(v, a, s);
  if (v.dk == 64 && v.dv == 64) return dispatch_types<64, 64>(v, a, s);
  return cudaErrorInvalidValue;
}

}  // namespace dig
