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
// Four kernels, each over independent units (the first three are shared with
// the backward, gla_chunk.cuh):
//   1. gla_gate_kernel: per (gate head, chunk), the gate of the chunk (cumsum
//      over its tokens) as per-token factors 2^(b - r) and per-chunk constants.
//   2. gla_chunk_state_kernel: per (sequence, chunk), the chunk's state
//      contribution dS_n = khat^T V.
//   3. gla_state_scan_kernel: S_{n+1} = diag(2^Gamma_n) S_n + dS_n over the
//      chunks, an associative scan (sixteen chunk ranges per state element,
//      then a carry fold), overwriting dS_n with the entry state S_n.
//   4. gla_chunk_out_kernel: per (sequence, chunk), the outputs from the
//      chunk's entry state, and the fused Swish(r) * RMSNorm(o) epilogue.
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
#include "gla_chunk.cuh"
#include "gla_strong.cuh"

namespace dig {


// Layout of the chunk-output kernel.  P = qbar kbar^T and O = qbar S' share
// their A operand, so kbar rows and S'^T rows are one B operand (N = C + DVP,
// per term: C kbar rows then DVP S'^T rows) and one product fills the
// adjacent P and O columns of TMEM.
template <int C, int DK, int DV, typename TIN>
struct OutCfg {
  using K = ChunkCfg<C, DK, DV, TIN>;
  static constexpr int NB = C + K::DVP;                       // rows of the combined B operand
  static constexpr int BS_SZ = (NB / 8) * K::SBO_K;           // one term of it
  static constexpr int OFF_AQ = 0;                            // qbar
  static constexpr int OFF_BS = K::NTG * K::AQ_SZ;            // kbar rows, then S'^T rows
  static constexpr int OFF_VR = OFF_BS + K::NTG * BS_SZ;
  static constexpr int OP = DV + 4;                           // row pitch of the output staging (over the operands)
  static constexpr int SMEM = cmax(cmax(OFF_VR + K::NTV * K::VR_SZ, OFF_AQ + K::AQ_READ), C * OP * 4);
  // TMEM columns: P (fp32) and O side by side, P as bf16 terms (8 columns per
  // term and K-step, the terms of K-step k at TM_PT + k * PT_STRIDE; in place
  // over P when two terms fit)
  static constexpr int TM_P = 0, TM_O = C;
  static constexpr int TM_PT = K::NTG == 2 ? 0 : C + K::DVP;
  static constexpr int PT_STRIDE = K::NTG * 8;
  static constexpr int TM_COLS = pow2ceil(K::NTG == 2 ? C + K::DVP : C + K::DVP + K::NTG * C / 2);
  static_assert(NB <= 256 && NB % 16 == 0, "one M = 128 product");
  static_assert(TM_COLS <= 256, "two output CTAs per SM share the 512 TMEM columns");
  static_assert(SMEM <= 110 * 1024, "two output CTAs per SM share shared memory");
  static_assert(C * OP * 4 <= OFF_VR, "the output staging leaves v's rows alone (v is prefetched during the epilogue)");
};

struct OutSmem {
  long long rows[2][128];  // grid tokens of the current and the next unit (by unit parity)
  float red[256];  // epilogue row sums of squares
  uint64_t bar_a;  // P, qbar S'
  uint64_t bar_b;  // P V
  uint32_t tmem;
  int mma_pend;    // thread 0: product group (0: P / qbar S', 1: P V) not yet seen complete, -1: none
  uint32_t mma_ph;
};

// ============================================================== 2. state scan
// A block covers 64 state elements (16 quads of 4) of one sequence: lane l of
// warp w owns quad l % 16 and chunk range 2w + l / 16 of 16, i.e. chunks
// [range*per, (range+1)*per) in scan direction.  Pass 1 folds each range into
// (decay product A, partial state s); the carry entering a range is the fold
// of the ranges before it; pass 2 rewrites X_n with the value entering chunk n.
// Ranges of up to kScanWindow chunks keep their chunks in registers between
// the passes (two memory round trips in all); longer ones stream in windows.
// blockIdx.y selects one of two buffers (the backward scans its states forward
// and its state gradients in reverse in one launch); `reverse` runs the chunks
// from the last to the first.  With a value gate the decay of element (j, c) is
// 2^Gamma[c] 2^Gb[j].  The carry entering the first step is zero or a given
// seed (S_0, or the gradient of the final state), and the carry after the last
// step (the final state, or the gradient of S_0) can be written out.
constexpr int kScanRanges = 16, kScanQuads = 16, kScanWindow = 8;
struct ScanJob {
  float* buf[2];
  int reverse[2];
  uint32_t* zero_word;  // set to 0 by the scan (the count of the backward's unit list), or NULL
  ScanEnds ends;
};
// One thread's share of the scan of a sequence with a chunk flagged by the gate
// kernel (strong gate): both passes again, each flagged chunk contributing the
// block formed from its tokens (strong::state_quad) instead of the stored one.
// Every thread of the CTA calls it (it holds a barrier).  The value-gated entry
// points never flag a chunk, so it writes no scan ends and applies no value decay.
struct ScanRange {
  float4* st;
  size_t st_stride;
  int reverse, bh, bz, c0, jrow, n0, n1, rg, lq;
  bool act;
  float4 seed4;
  int dk, dv;
};
__device__ __noinline__ void scan_exact(const GlaArgs a, const ScanRange r, float4 (*sA)[kScanQuads],
                                        float4 (*sS)[kScanQuads]) {
  const int nch = a.nchunks;
  const int* flags = a.sflag + (size_t)r.bz * nch;
  const float* dec = a.gCH + ((size_t)r.bz * nch * 4 + 2) * r.dk + r.c0;  // 2^Gamma of chunk n at dec + n * 4 * dk
  auto at = [&](int m) { return r.reverse ? nch - 1 - m : m; };
  auto decay = [&](int n) { return __ldg(reinterpret_cast<const float4*>(dec + (size_t)n * 4 * r.dk)); };
  auto contrib = [&](int n) {
    return __ldcg(flags + n) != 0 ? strong::state_quad(a, r.reverse != 0, r.bh, n, r.c0, r.jrow, r.dk, r.dv)
                                  : __ldcg(r.st + n * r.st_stride);
  };
  auto fma4 = [](float4 g, float4 s, float4 d) {
    return make_float4(fmaf(g.x, s.x, d.x), fmaf(g.y, s.y, d.y), fmaf(g.z, s.z, d.z), fmaf(g.w, s.w, d.w));
  };
  float4 A = make_float4(1.f, 1.f, 1.f, 1.f), s = make_float4(0.f, 0.f, 0.f, 0.f);
  if (r.act) {
    for (int m = r.n0; m < r.n1; ++m) {
      const float4 g = decay(at(m));
      s = fma4(g, s, contrib(at(m)));
      A = make_float4(g.x * A.x, g.y * A.y, g.z * A.z, g.w * A.w);
    }
  }
  sA[r.rg][r.lq] = A;  // only this thread wrote or read its entry since the last barrier
  sS[r.rg][r.lq] = s;
  __syncthreads();
  if (!r.act) return;
  float4 S = r.seed4;
  for (int m = 0; m < r.rg; ++m) S = fma4(sA[m][r.lq], S, sS[m][r.lq]);
  for (int m = r.n0; m < r.n1; ++m) {
    const float4 dd = contrib(at(m));  // read before the entering state takes its place
    __stcg(r.st + at(m) * r.st_stride, S);
    S = fma4(decay(at(m)), S, dd);
  }
}

__global__ void __launch_bounds__(kScanRanges * kScanQuads, 2) gla_state_scan_kernel(const GlaArgs a, ScanJob job,
                                                                                     int dk, int dv) {
  __shared__ float4 sA[kScanRanges][kScanQuads], sS[kScanRanges][kScanQuads];
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  if (job.zero_word != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *job.zero_word = 0u;
  float* buf = blockIdx.y ? job.buf[1] : job.buf[0];
  const int reverse = blockIdx.y ? job.reverse[1] : job.reverse[0];
  const int nq = dv * dk / 4;
  const int nblk = (nq + kScanQuads - 1) / kScanQuads;
  const int bh = blockIdx.x / nblk, blk = blockIdx.x - bh * nblk;
  const int lq = threadIdx.x & (kScanQuads - 1), rg = threadIdx.x / kScanQuads;
  const int quad = blk * kScanQuads + lq;
  const bool act = quad < nq;
  const int c0 = (quad * 4) % dk;  // the quad's four key channels (dk % 4 == 0)
  const int b = bh / a.H, h = bh - b * a.H;
  const int bz = b * a.gate_heads + (a.gate_heads == 1 ? 0 : h);
  const int nch = a.nchunks;
  const int per = (nch + kScanRanges - 1) / kScanRanges;
  const int n0 = min(nch, rg * per), n1 = min(nch, n0 + per);
  float4* st = reinterpret_cast<float4*>(buf + (size_t)bh * nch * dv * dk) + quad;
  const size_t st_stride = (size_t)nq;
  const float* dec = a.gCH + ((size_t)bz * nch * 4 + 2) * dk + c0;  // 2^Gamma of chunk n at dec + n * 4 * dk
  const int jrow = (quad * 4) / dk;                                   // the quad's value channel
  const float* decb = a.gCHb ? a.gCHb + ((size_t)bz * nch * 4 + 2) * dv + jrow : nullptr;  // 2^Gb[j]
  auto at = [&](int n) { return reverse ? nch - 1 - n : n; };         // physical chunk of scan step n
  auto fma4 = [](float4 g, float4 s, float4 d) {
    return make_float4(fmaf(g.x, s.x, d.x), fmaf(g.y, s.y, d.y), fmaf(g.z, s.z, d.z), fmaf(g.w, s.w, d.w));
  };
  auto mul4 = [](float4 g, float4 x) { return make_float4(g.x * x.x, g.y * x.y, g.z * x.z, g.w * x.w); };
  auto decay = [&](int n) {  // the element decay of physical chunk n
    float4 g = __ldg(reinterpret_cast<const float4*>(dec + (size_t)n * 4 * dk));
    if (decb != nullptr) {
      const float gb = __ldg(decb + (size_t)n * 4 * dv);
      g = make_float4(g.x * gb, g.y * gb, g.z * gb, g.w * gb);
    }
    return g;
  };
  const int side = blockIdx.y;
  const float* seed = job.ends.seed[side];
  float4 seed4 = make_float4(0.f, 0.f, 0.f, 0.f);
  if (seed != nullptr && act) {  // [B*H][DK][DV]: element (j, c) at c * dv + j
    const float* sp = seed + (size_t)bh * dk * dv + (size_t)c0 * dv + jrow;
    seed4 = make_float4(__ldg(sp), __ldg(sp + dv), __ldg(sp + 2 * dv), __ldg(sp + 3 * dv));
  }
  // Chunks of this sequence flagged by the gate kernel (strong gates) send the
  // whole CTA down the exact path below; each thread reads the flags of its range
  // with its first pass's loads, and the CTA looks at them at the barrier after it.
  const int* flags = a.sflag != nullptr ? a.sflag + (size_t)bz * nch : nullptr;
  int flagged_seq = 0;
  float4 A = make_float4(1.f, 1.f, 1.f, 1.f), s = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 d[kScanWindow];
  const bool resident = per <= kScanWindow;  // uniform: one window holds the whole range
  if (act) {
    for (int w0 = n0; w0 < n1; w0 += kScanWindow) {
      float4 g[kScanWindow];
      int fl[kScanWindow];
#pragma unroll
      for (int e = 0; e < kScanWindow; ++e) {
        fl[e] = 0;
        if (w0 + e < n1) {
          g[e] = decay(at(w0 + e));
          d[e] = __ldcg(st + at(w0 + e) * st_stride);
          if (flags != nullptr) fl[e] = __ldcg(flags + at(w0 + e));
        }
      }
#pragma unroll
      for (int e = 0; e < kScanWindow; ++e) {
        if (w0 + e < n1) {
          s = fma4(g[e], s, d[e]);
          A = mul4(g[e], A);
          flagged_seq |= fl[e];  // next to the block's use: the loads have landed by now
        }
      }
    }
  }
  sA[rg][lq] = A;
  sS[rg][lq] = s;
  if (__syncthreads_or(flagged_seq != 0)) {  // rare: both passes again, exactly (strong gates)
    const ScanRange r{st, st_stride, reverse, bh, bz, c0, jrow, n0, n1, rg, lq, act, seed4, dk, dv};
    scan_exact(a, r, sA, sS);
    return;
  }
  if (!act) return;
  if (rg == 0 && (job.ends.fin[side] != nullptr || job.ends.fin_rows[side] != nullptr)) {
    float4 F = seed4;  // the carry after the last step: every range folded onto the seed
    for (int m = 0; m < kScanRanges; ++m) F = fma4(sA[m][lq], F, sS[m][lq]);
    if (job.ends.fin_rows[side] != nullptr)
      reinterpret_cast<float4*>(job.ends.fin_rows[side] + (size_t)bh * dk * dv)[quad] = F;
    if (job.ends.fin[side] != nullptr) {
      float* fp = job.ends.fin[side] + (size_t)bh * dk * dv + (size_t)c0 * dv + jrow;
      fp[0] = F.x;
      fp[dv] = F.y;
      fp[2 * dv] = F.z;
      fp[3 * dv] = F.w;
    }
  }
  float4 S = seed4;
  for (int m = 0; m < rg; ++m) S = fma4(sA[m][lq], S, sS[m][lq]);
  if (resident) {  // the range's contributions are still in registers; its decays are reread (L1)
#pragma unroll
    for (int e = 0; e < kScanWindow; ++e) {
      if (n0 + e < n1) {
        __stcg(st + at(n0 + e) * st_stride, S);
        S = fma4(decay(at(n0 + e)), S, d[e]);
      }
    }
    return;
  }
  for (int w0 = n0; w0 < n1; w0 += kScanWindow) {
    float4 g[kScanWindow];
#pragma unroll
    for (int e = 0; e < kScanWindow; ++e) {
      if (w0 + e < n1) {
        g[e] = decay(at(w0 + e));
        d[e] = __ldcg(st + at(w0 + e) * st_stride);
      }
    }
#pragma unroll
    for (int e = 0; e < kScanWindow; ++e) {
      if (w0 + e < n1) {
        __stcg(st + at(w0 + e) * st_stride, S);
        S = fma4(g[e], S, d[e]);
      }
    }
  }
}

// ============================================================== 3. outputs
// O rows (TMEM lane t = token t) of this thread's channel half -> staging and
// the row's partial sum of squares.  With a value gate (`eqb`: the unit's rows
// of 2^(e - rho), NULL otherwise) the product P vbar + qbar S'^T is rescaled to
// o = EQb (P vbar + qbar S'^T) first; `nvalid` tokens of the chunk are real.
template <int C, int DK, int DV, typename TIN, int H>
__device__ __forceinline__ void stage_o(uint32_t tmem, float* stage, float* red, const float* eqb = nullptr,
                                        int nvalid = 0) {
  using Cfg = ChunkCfg<C, DK, DV, TIN>;
  using OC = OutCfg<C, DK, DV, TIN>;
  constexpr int VO = H ? Cfg::DV0 : 0, VN = H ? Cfg::DV1 : Cfg::DV0;
  const int tid = threadIdx.x, t = tid & 127, wq = t >> 5;
  float ov[cround(VN, 8)];
#pragma unroll
  for (int c = 0; c < cround(VN, 8); c += 8)
    tmem_ld8(tmem + (static_cast<uint32_t>(32 * wq) << 16) + OC::TM_O + VO + c, ov + c);
  tmem_ld_wait();
  if (eqb != nullptr && t < nvalid) {
#pragma unroll
    for (int i = 0; i < VN; ++i) ov[i] *= __ldg(eqb + (size_t)t * DV + VO + i);
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < VN; ++i) ss += ov[i] * ov[i];
  red[tid] = ss;
  if (t < C) {
#pragma unroll
    for (int g = 0; g < VN / 4; ++g)
      *reinterpret_cast<float4*>(stage + t * OC::OP + VO + 4 * g) =
          make_float4(ov[4 * g], ov[4 * g + 1], ov[4 * g + 2], ov[4 * g + 3]);
  }
}

// With EXT (value gate, fp32 inputs): v is loaded as vbar = v / EQb, the S'^T
// rows carry 2^rho of their value channel, and the output is rescaled by EQb.
template <int C, int DK, int DV, typename TIN, typename TOUT, bool EXT = false>
__global__ void __launch_bounds__(256, 2) gla_chunk_out_kernel(const GlaArgs a) {
  using Cfg = ChunkCfg<C, DK, DV, TIN>;
  using OC = OutCfg<C, DK, DV, TIN>;
  constexpr int NTG = Cfg::NTG, NTV = Cfg::NTV, DKP = Cfg::DKP, DVP = Cfg::DVP, PSK = Cfg::PSK;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ OutSmem sh;
  const int tid = threadIdx.x, warp = tid >> 5;
  if (warp == 0) {
    tmem_alloc(&sh.tmem, OC::TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&sh.bar_a, 1);
    mbar_init(&sh.bar_b, 1);
    fence_mbar_init();
  }
  if ((int)blockIdx.x < a.B * a.H * a.nchunks) fill_rows(a, blockIdx.x, C, sh.rows[0]);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int t = tid & 127, wq = (tid >> 5) & 3, half = tid >> 7;
  const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
  const uint32_t tmem = sh.tmem;
  const uint32_t sbase = smem_u32(smem);
  float* stage = reinterpret_cast<float*>(smem);  // [C][OP] output rows, over the operands
  const uint64_t dAQ = sdesc(sbase + OC::OFF_AQ, 128, Cfg::SBO_K);
  const uint64_t dBS = sdesc(sbase + OC::OFF_BS, 128, Cfg::SBO_K);
  const uint32_t sSPT = sbase + OC::OFF_BS + (C / 8) * Cfg::SBO_K;  // S'^T rows inside the combined operand
  const uint64_t dVRm = sdesc(sbase + OC::OFF_VR, Cfg::SBO_V, 128);
  const int nunits = a.B * a.H * a.nchunks;
  const bool with_y = a.y != nullptr && a.r != nullptr;
  uint32_t ph = 0;
  bool timed_out = false;  // a wait of this thread gave up: the CTA stops after this unit
  if (tid == 0) sh.mma_pend = -1;

  // Row pieces of a unit, loaded one unit ahead: q, k, gate factors, entry-state
  // rows and 2^r are issued as soon as the current unit's operands are written,
  // v once its P V has completed, r once its epilogue is done.
  Piece<TIN, PSK> pq[Cfg::NPK], pk[Cfg::NPK];
  Piece<float, PSK> pe[Cfg::NPK];
  Piece<float, 4> ps[Cfg::NPS], pc[Cfg::NPS];
  Piece<TIN, 8> pr[Cfg::NPV];
  auto issue_rows = [&](int u, const long long* rows) {
    const Unit U(a, u);
#pragma unroll
    for (int j = 0; j < Cfg::NPK; ++j) {
      const int i = tid + 256 * j;
      int tt, g;
      piece_of<Cfg::NGK>(i, tt, g);
      const long long gr = i < C * Cfg::NGK ? rows[tt] : -1;
      const bool valid = gr >= 0;
      const size_t off = tok_row(gr, a, U.h) * DK + g * PSK;
      pq[j].load(reinterpret_cast<const TIN*>(a.q) + off, valid);
      pk[j].load(reinterpret_cast<const TIN*>(a.k) + off, valid);
      pe[j].load(a.gEQ + ((size_t)U.bz * a.L + (valid ? U.n * C + tt : 0)) * DK + g * PSK, valid);
    }
#pragma unroll
    for (int j = 0; j < Cfg::NPS; ++j) {
      const int i = tid + 256 * j;
      int jr, g;
      piece_of<Cfg::NGS>(i, jr, g);
      pc[j].load(a.gCH + ((size_t)U.bz * a.nchunks + U.n) * 4 * DK + 4 * g, i < DV * Cfg::NGS);
    }
  };
  auto issue_s = [&](int u) {  // entry-state rows (written by the scan before this kernel)
#pragma unroll
    for (int j = 0; j < Cfg::NPS; ++j) {
      const int i = tid + 256 * j;
      int jr, g;
      piece_of<Cfg::NGS>(i, jr, g);
      const bool in = i < DV * Cfg::NGS;
      ps[j].load_cg(a.dsn + ((size_t)u * DV + (in ? jr : 0)) * DK + 4 * g, in);
    }
  };
  auto issue_r = [&](int h, const long long* rows) {
    if (!with_y) return;
#pragma unroll
    for (int j = 0; j < Cfg::NPV; ++j) {
      const int i = tid + 256 * j;
      int tt, g;
      piece_of<Cfg::NGV>(i, tt, g);
      const long long gr = i < C * Cfg::NGV ? rows[tt] : -1;
      pr[j].load(reinterpret_cast<const TIN*>(a.r) + tok_row(gr, a, h) * DV + 8 * g, gr >= 0);
    }
  };
  // Loading one unit ahead holds two units' pieces in registers; with 8-byte
  // pieces (d_k not a multiple of 8) that spills, so those variants load per unit.
  constexpr bool kAhead = PSK == 8;
  // The kernel before this one is the state scan, which writes only the chunk
  // states; everything older has completed.  So the first unit's other rows are
  // requested before the wait for that scan.
  constexpr int VSV = EXT ? VS_VBAR : VS_NONE;
  if (kAhead && (int)blockIdx.x < nunits) {
    const Unit U0(a, blockIdx.x);
    issue_rows(blockIdx.x, sh.rows[0]);
    load_v_rows_t<C, DK, DV, TIN, 256, VSV>(a, U0.h, sh.rows[0], a.v, sbase + OC::OFF_VR, U0.bz, U0.n);
    issue_r(U0.h, sh.rows[0]);
  }
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  if (kAhead && (int)blockIdx.x < nunits) issue_s(blockIdx.x);

  int it = 0;
  bool any_strong = false;  // uniform: a unit of this CTA has a flagged chunk
  for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++it) {
    const Unit U(a, u);
    const bool skip = !EXT && strong::flagged(a, U.bz, U.n);  // strong gate: o and y come after the loop
    any_strong |= skip;
    const int un = u + gridDim.x;
    const bool has_next = kAhead && un < nunits;
    const long long* rows = sh.rows[it & 1];
    long long* rows_next = sh.rows[(it + 1) & 1];
    if (!kAhead) {
      if (it > 0) {  // the first unit's rows were filled before the first barrier
        fill_rows(a, u, C, sh.rows[it & 1]);
        __syncthreads();
      }
      issue_rows(u, rows);
      issue_s(u);
      load_v_rows_t<C, DK, DV, TIN, 256, VSV>(a, U.h, rows, a.v, sbase + OC::OFF_VR, U.bz, U.n);
    }
    if (has_next) fill_rows(a, un, C, rows_next);  // visible after the next barrier
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
        st_piece<NTG, PSK>(sbase + OC::OFF_AQ, tt, Cfg::SBO_K, g * PSK, Cfg::AQ_SZ, qv);
        st_piece<NTG, PSK>(sbase + OC::OFF_BS, tt, Cfg::SBO_K, g * PSK, OC::BS_SZ, kv);
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
        // value-gate reference of the row's value channel (1 without a value gate)
        const float rb = EXT ? __ldg(a.gCHb + ((size_t)U.bz * a.nchunks + U.n) * 4 * DV + jr) : 1.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) sv[e] *= cv[e] * rb;
        st_piece<NTG, 4>(sSPT, jr, Cfg::SBO_K, 4 * g, OC::BS_SZ, sv);
      }
    }
    if constexpr (Cfg::NPAD > 0) {  // zero K padding (the output staging of the previous unit overwrote it)
      // of the C token rows of qbar and kbar and of the DV rows of S'^T (more than C when d_v > C)
      const float zz[4] = {0.f, 0.f, 0.f, 0.f};
      constexpr int NR = C > DV ? C : DV;
      for (int i = tid; i < NR * Cfg::NPAD; i += 256) {
        const int row = i / Cfg::NPAD, c = DK + 4 * (i % Cfg::NPAD);
        if (row < C) {
          st_piece<NTG, 4>(sbase + OC::OFF_AQ, row, Cfg::SBO_K, c, Cfg::AQ_SZ, zz);
          st_piece<NTG, 4>(sbase + OC::OFF_BS, row, Cfg::SBO_K, c, OC::BS_SZ, zz);
        }
        if (row < DV) st_piece<NTG, 4>(sSPT, row, Cfg::SBO_K, c, OC::BS_SZ, zz);
      }
    }
    cp_async_wait_all();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      mma_issue<NTG, NTG, DKP / 16>(tmem + OC::TM_P, dAQ, Cfg::AQ_SZ, 256, dBS, OC::BS_SZ, 256,
                                    idesc_bf16(128, OC::NB), false);  // [P | O] = qbar [kbar | S'^T]^T
      mma_commit(&sh.bar_a);
      sh.mma_pend = 0;
      sh.mma_ph = ph;
    }
    if (has_next) {  // this unit's row pieces are consumed
      issue_rows(un, rows_next);
      issue_s(un);
    }
    if (!mbar_wait(&sh.bar_a, ph, spin_limit(a))) timed_out = true;
    else if (tid == 0) sh.mma_pend = -1;
    tc_fence_after();
    // ---- mask P (s <= t) and store it as bf16 terms in TMEM, one K-step of 16 at a time
    if (32 * wq < C) {  // warp-uniform: lanes that are token rows
#pragma unroll
      for (int kk = 0; kk < C / 32; ++kk) {
        const int s0 = half * (C / 2) + 16 * kk;
        float pv[16];
        if (s0 <= 32 * wq + 31) {
          tmem_ld16(tmem + lane_base + OC::TM_P + s0, pv);
          tmem_ld_wait();
          if (s0 + 15 > 32 * wq) {  // warp-uniform: the block crosses this warp's diagonal
#pragma unroll
            for (int e = 0; e < 16; ++e) pv[e] = (s0 + e <= t) ? pv[e] : 0.f;
          }
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
          tmem_st8(tmem + lane_base + OC::TM_PT + (s0 / 16) * OC::PT_STRIDE + 8 * i, pk8);
        }
      }
      tmem_st_wait();
    }
    tc_fence_before();
    const bool stop = __syncthreads_or(timed_out);  // a wait gave up: no further products
    tc_fence_after();
    if (tid == 0 && !stop) {
      mma_issue_ts<NTG, NTV, C / 16>(tmem + OC::TM_O, tmem + OC::TM_PT, OC::PT_STRIDE, dVRm, Cfg::VR_SZ,
                                     2 * Cfg::SBO_V, idesc_bf16(128, DVP, false, true), true);
      mma_commit(&sh.bar_b);
      sh.mma_pend = 1;
      sh.mma_ph = ph;
    }
    if (!stop) {
      if (!mbar_wait(&sh.bar_b, ph, spin_limit(a))) timed_out = true;
      else if (tid == 0) sh.mma_pend = -1;
    }
    ph ^= 1u;
    tc_fence_after();
    const Unit Un(a, has_next ? un : u);
    const int hn = Un.h;
    if (has_next && !stop)  // v of this unit is consumed
      load_v_rows_t<C, DK, DV, TIN, 256, VSV>(a, hn, rows_next, a.v, sbase + OC::OFF_VR, Un.bz, Un.n);
    if (!kAhead) issue_r(U.h, rows);
    const float* eqb = EXT ? a.gEQb + ((size_t)U.bz * a.L + (size_t)U.n * C) * DV : nullptr;
    const int nvalid = min(C, a.L - U.n * C);
    if (tid < 128) stage_o<C, DK, DV, TIN, 0>(tmem, stage, sh.red, eqb, nvalid);
    else stage_o<C, DK, DV, TIN, 1>(tmem, stage, sh.red, eqb, nvalid);
    tc_fence_before();
    __syncthreads();
    // ---- o and y rows, 8 channels per piece
#pragma unroll
    for (int j = 0; j < Cfg::NPV; ++j) {
      const int i = tid + 256 * j;
      int tt, g;
      piece_of<Cfg::NGV>(i, tt, g);
      const long long gr = i < C * Cfg::NGV ? rows[tt] : -1;
      if (gr >= 0 && !skip) {
        const size_t off = tok_row(gr, a, U.h) * DV + 8 * g;
        float ov[8];
        const float4 o0 = *reinterpret_cast<const float4*>(stage + tt * OC::OP + 8 * g);
        const float4 o1 = *reinterpret_cast<const float4*>(stage + tt * OC::OP + 8 * g + 4);
        ov[0] = o0.x; ov[1] = o0.y; ov[2] = o0.z; ov[3] = o0.w;
        ov[4] = o1.x; ov[5] = o1.y; ov[6] = o1.z; ov[7] = o1.w;
        st_global8(reinterpret_cast<TOUT*>(a.o) + off, ov);
        if (with_y) {
          const float inv = rsqrtf((sh.red[tt] + sh.red[tt + 128]) / (float)DV + a.eps);
          float rv[8], yv[8], gm[8];
          pr[j].unpack(rv);
          if (a.gamma != nullptr) {
            const float4 g0 = __ldg(reinterpret_cast<const float4*>(a.gamma + 8 * g));
            const float4 g1 = __ldg(reinterpret_cast<const float4*>(a.gamma + 8 * g) + 1);
            gm[0] = g0.x; gm[1] = g0.y; gm[2] = g0.z; gm[3] = g0.w;
            gm[4] = g1.x; gm[5] = g1.y; gm[6] = g1.z; gm[7] = g1.w;
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) gm[e] = 1.f;
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float sw = __fdividef(rv[e], 1.f + ex2(-rv[e] * kLog2e));  // Swish(r) = r sigmoid(r)
            yv[e] = sw * ov[e] * inv * gm[e];
          }
          st_global8(reinterpret_cast<TOUT*>(a.y) + off, yv);
        }
      }
    }
    if (has_next) issue_r(hn, rows_next);
    // staging and row sums are rewritten by the next unit; after a wait gave up
    // anywhere in the CTA, no further unit starts
    if (__syncthreads_or(timed_out)) break;
  }
  // ---- drain: this thread's row copies, and the last products, complete before exit
  if (timed_out) set_status(a.status, DIG_ERR_DEVICE_TIMEOUT);
  cp_async_wait_all();
  if (tid == 0 && sh.mma_pend >= 0) mbar_wait(sh.mma_pend ? &sh.bar_b : &sh.bar_a, sh.mma_ph, kSpinLimitNs);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, OC::TM_COLS);
  if constexpr (!EXT) {  // this CTA's units of chunks flagged by the gate kernel (strong gates), exactly in fp32
    static_assert(OC::SMEM >= strong::Cfg<C, DK, DV>::SMEM_OUT, "shared memory of the strong-gate phase");
    if (any_strong && !__syncthreads_or(timed_out))
      for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
        const Unit U(a, u);
        if (strong::flagged(a, U.bz, U.n)) strong::out_unit<C, DK, DV, TIN, TOUT>(a, u, smem);
      }
  }
}

// ------------------------------------------------------------------ launch
// ------------------------------------------------------------------ launch
namespace {
int g_sms_cache[64];
}  // namespace

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

cudaError_t launch_state_scan(const GlaArgs& a, float* buf0, bool rev0, float* buf1, bool rev1, int dk, int dv,
                              cudaStream_t s, uint32_t* zero_word, const ScanEnds* ends) {
  const int nq = dv * dk / 4;
  const long long blocks = (long long)a.B * a.H * ((nq + kScanQuads - 1) / kScanQuads);
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 2147483647LL) return cudaErrorInvalidValue;
  ScanJob job{{buf0, buf1}, {rev0 ? 1 : 0, rev1 ? 1 : 0}, zero_word, ends ? *ends : ScanEnds{}};
  return launch_pdl(gla_state_scan_kernel, dim3((unsigned)blocks, buf1 ? 2u : 1u), kScanRanges * kScanQuads, 0, s, a,
                    job, dk, dv);
}

bool gla_out_tma_eligible(const GlaArgs& a, int dk, int dv, int tin, int chunk);  // gla_fwd_tma.cu
cudaError_t launch_out_tma(const GlaArgs& a, int tout, cudaStream_t s, bool* launched);

namespace {

template <int C, int DK, int DV, typename TIN, typename TOUT, bool EXT = false>
cudaError_t launch_typed(const GlaArgs& a, cudaStream_t s, const ScanEnds* ends = nullptr) {
  using OC = OutCfg<C, DK, DV, TIN>;
  const long long units = (long long)a.B * a.H * a.nchunks;
  if (units <= 0) return cudaSuccess;
  cudaError_t e = launch_chunk_state<C, DK, DV, TIN, false, EXT>(a, s);
  if (e != cudaSuccess) return e;
  if ((e = launch_state_scan(a, a.dsn, false, nullptr, false, DK, DV, s, nullptr, ends)) != cudaSuccess) return e;
  if (!EXT && std::is_same<TIN, __nv_bfloat16>::value && gla_out_tma_eligible(a, DK, DV, DIG_BF16, C)) {
    bool launched = false;
    if ((e = launch_out_tma(a, std::is_same<TOUT, float>::value ? DIG_F32 : DIG_BF16, s, &launched)) != cudaSuccess)
      return e;
    if (launched) return cudaGetLastError();
  }
  auto k3 = gla_chunk_out_kernel<C, DK, DV, TIN, TOUT, EXT>;
  if ((e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, OC::SMEM)) != cudaSuccess) return e;
  if ((e = launch_pdl(k3, persistent_grid(2, units), 256, OC::SMEM, s, a)) != cudaSuccess) return e;
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

template <int DK, int DV>
cudaError_t dispatch_ext(const GlaVariant& v, const GlaArgs& a, const ScanEnds& ends, cudaStream_t s) {
  if (v.tout == DIG_BF16) return launch_typed<64, DK, DV, float, __nv_bfloat16, true>(a, s, &ends);
  return launch_typed<64, DK, DV, float, float, true>(a, s, &ends);
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

cudaError_t launch_gla_fwd_ext(const GlaVariant& v, const GlaArgs& a, const ScanEnds& ends, cudaStream_t s) {
  if (v.tin != DIG_F32 || v.chunk != 64) return cudaErrorInvalidValue;
  if (v.dk == 32 && v.dv == 64) return dispatch_ext<32, 64>(v, a, ends, s);
  if (v.dk == 36 && v.dv == 72) return dispatch_ext<36, 72>(v, a, ends, s);
  if (v.dk == 64 && v.dv == 64) return dispatch_ext<64, 64>(v, a, ends, s);
  return cudaErrorInvalidValue;
}

}  // namespace dig
