// gla_bwd.cu -- chunkwise Gated Linear Attention backward on sm_100a.
//
// Gradients of sum(o * dO) for the forward of gla_fwd.cu (DiG slides, GLA eq.
// (5)-(8)).  With the chunk quantities of the forward (entry state S_n, token
// cumsum b, reference r, chunk decay Gamma; qbar = q 2^(b-r), kbar = k 2^(r-b),
// S' = diag(2^r) S_n) and G_n, the gradient of the state leaving chunk n
// (G_{N-1} = 0, G_{n-1} = diag(2^Gamma_n) G_n + dH_n, dH_n = (q 2^b)^T dO):
//     dP  = mask(dO V^T)                       (s <= t)
//     P^T = mask(kbar qbar^T)                  (t >= s)
//     dqbar = dP kbar + dO S'^T                -> dq = dqbar 2^(b-r)
//     dkbar = dP^T qbar + V Gt^T               -> dk = dkbar 2^(r-b)
//     dv    = P^T dO + kbar Gt                 Gt = diag(2^(Gamma-r)) G_n
//     dlog alpha_t = sum_{u >= t in chunk} (qbar dqbar - kbar dkbar)_u + rowsum(S_{n+1} o G_n)
// The last term is the sum of the later chunks' (q dq - k dk) terms: scaling
// the state leaving the chunk by e^delta is the same as shifting every later
// log-decay cumsum by delta (natural-log units throughout).
//
// Kernels: the forward's gate kernel and its chunk-state kernel in backward mode
// (dS_n and dH_n per chunk), the state scan forward over dS (entry states S_n) and in reverse over
// dH (exit gradients G_n), then gla_chunk_grad_kernel over independent
// (sequence, chunk) units.  P^T, dP^T and dP are formed by separate tensor-core
// products so none needs a transpose.  They take turns in one TMEM region: each
// is masked and converted to two bf16 terms in place, then read as the A operand
// of its gradient product before the next one overwrites the region.  With the
// three gradient accumulators this is 256 TMEM columns, so two CTAs share an SM.
#include "gla_chunk.cuh"
#include "gla_strong.cuh"

namespace dig {

// Backward chunk length: 128 tokens when one C x C region and the three
// gradient accumulators fit 256 TMEM columns (two CTAs per SM) and the operands
// fit shared memory (bf16 inputs), else 64.
__host__ __device__ constexpr int bwd_chunk_len(int dk, int dv, bool f32) {
  return !f32 && 128 + 2 * cround(dk, 16) + cround(dv, 16) <= 256 ? 128 : 64;
}

template <int C, int DK, int DV, typename TIN, typename TOUT>
struct BwdCfg {
  using K = ChunkCfg<C, DK, DV, TIN>;
  static constexpr int NTG = K::NTG, NTV = K::NTV;
  static constexpr int NTP = 2;  // terms of the masked P-type matrices
  // shared memory: v and dO rows first (the next unit's copies land there while
  // this unit finishes), then qbar, kbar (token rows), S', Gt (value-channel rows)
  static constexpr int OFF_V = 0;
  static constexpr int OFF_DO = OFF_V + NTV * K::VR_SZ;
  static constexpr int OFF_Q = OFF_DO + NTV * K::VR_SZ;
  static constexpr int OFF_K = OFF_Q + NTG * K::AQ_SZ;
  static constexpr int OFF_SP = OFF_K + NTG * K::AQ_SZ;
  static constexpr int OFF_GT = OFF_SP + NTG * K::SPT_SZ;
  static constexpr int END_OPS = OFF_GT + NTG * K::SPT_SZ;
  // gate factors EQ of the chunk's tokens (fp32 rows), overwritten in place by
  // the tokens' d log alpha terms
  static constexpr int EP = DK + 4;
  static constexpr int OFF_EQ = cround(END_OPS, 16);
  static constexpr int END_EQ = OFF_EQ + C * EP * 4;
  // staging of the gradient rows in the output type, over qbar .. Gt once the
  // last product is done; rows an odd number of 16-byte units apart (no bank
  // conflicts between 8 consecutive rows)
  static constexpr int KSB = 16 * (cdiv(DK * (int)sizeof(TOUT), 16) | 1);
  static constexpr int VSB = 16 * (cdiv(DV * (int)sizeof(TOUT), 16) | 1);
  static constexpr int OFF_SQ = OFF_Q, OFF_SK = OFF_SQ + C * KSB;
  // dv beside dq and dk when all three fit, else alone in a second pass
  static constexpr bool ONE_PASS = OFF_SK + C * KSB + C * VSB <= END_OPS;
  static constexpr int OFF_SV = ONE_PASS ? OFF_SK + C * KSB : OFF_Q;
  // M = 128 reads of C-row A operands (v, dO, kbar) may run past their rows
  // into the next buffers (those lanes are unused) but stay inside the allocation
  static constexpr int V_READ = (NTV - 1) * K::VR_SZ + 16 * K::SBO_V;
  static constexpr int SMEM = cmax(cmax(END_EQ, OFF_K + K::AQ_READ), OFF_DO + V_READ);
  static constexpr int PER_SM = SMEM <= 110 * 1024 ? 2 : 1;
  // TMEM: one C x C region (P^T, then dP^T, then dP), dqbar, dkbar, dv
  static constexpr int PT_STRIDE = NTP * 8;
  static constexpr int TM_R = 0;
  static constexpr int TM_DQ = C, TM_DK = TM_DQ + K::DKP, TM_DV = TM_DK + K::DKP;
  static constexpr int TM_COLS = 256;
  static constexpr int NSG = 256 / DK;  // token segments of the d log alpha reverse cumsum
  static constexpr int SEGL = cdiv(C, NSG);
  static_assert(OFF_SK + C * KSB <= END_OPS && OFF_SV + C * VSB <= END_OPS, "staging");
  // the unit's state blocks (DV x DK fp32) land by bulk copy in the S', Gt and
  // qbar slots and are converted in place
  static_assert(DV * DK * 4 <= NTG * K::SPT_SZ && DV * DK * 4 <= NTG * K::AQ_SZ && (DV * DK * 4) % 16 == 0,
                "state landing");
  static_assert(TM_DV + K::DVP <= TM_COLS, "TMEM budget");
  static_assert(SMEM <= 225 * 1024, "shared-memory budget");
  static_assert(C == bwd_chunk_len(DK, DV, std::is_same<TIN, float>::value), "chunk length");
};

struct GradSmem {
  long long rows[2][128];  // grid tokens of the current and the next unit (by unit parity)
  alignas(16) float gch[128];  // the unit's chunk constants: 2^r (d_k values), then 2^(Gamma - r) (bulk copy)
  float segtot[8][64];  // reverse-cumsum totals of the token segments
  float bnd[2][64];     // rowsum(S_{n+1} o G_n), double-buffered by unit parity
  uint64_t bar[6];      // completion of the six product groups of a unit
  uint64_t sbar;        // completion of the unit's bulk copies (states and chunk constants)
  uint32_t tmem;
  // thread 0's record of asynchronous work not yet seen complete, drained before exit
  int mma_pend;         // the product group whose commit is outstanding (-1: none)
  uint32_t mma_ph;
  int st_pend;          // state copies requested and not yet seen landed
  uint32_t st_ph;
};

// Masks one C x C product in TMEM (lane = row r; keep column c >= r when
// `upper`, else c <= r) and rewrites it as two bf16 terms in place, one K-step
// of 16 columns at a time.  This thread covers the columns of its half.  (One
// wait per 16-column load measured faster than waiting once for all of them.)
template <int C, int PT_STRIDE>
__device__ __forceinline__ void mask_to_terms(uint32_t tmem, uint32_t region, bool upper) {
  const int tid = threadIdx.x, t = tid & 127, wq = t >> 5, half = tid >> 7;
  if (32 * wq >= C) return;  // warp-uniform: lanes past the chunk
  const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
#pragma unroll
  for (int kk = 0; kk < C / 32; ++kk) {
    const int s0 = half * (C / 2) + 16 * kk;
    const bool zero_block = upper ? (s0 + 15 < 32 * wq) : (s0 > 32 * wq + 31);  // warp-uniform
    float pv[16];
    if (!zero_block) {
      tmem_ld16(tmem + lane_base + region + s0, pv);
      tmem_ld_wait();
      // warp-uniform: only a block that crosses this warp's diagonal needs the mask
      const bool full = upper ? (s0 >= 32 * wq + 31) : (s0 + 15 <= 32 * wq);
      if (!full) {
#pragma unroll
        for (int e = 0; e < 16; ++e) pv[e] = (upper ? (s0 + e >= t) : (s0 + e <= t)) ? pv[e] : 0.f;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) pv[e] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      uint32_t pk8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const __nv_bfloat162 hb = __floats2bfloat162_rn(pv[2 * e], pv[2 * e + 1]);
        pk8[e] = *reinterpret_cast<const uint32_t*>(&hb);
        pv[2 * e] -= __low2float(hb);
        pv[2 * e + 1] -= __high2float(hb);
      }
      tmem_st8(tmem + lane_base + region + (s0 / 16) * PT_STRIDE + 8 * i, pk8);
    }
  }
}

// Sum of the NT bf16 terms of four consecutive K values of one operand row.
template <int NT>
__device__ __forceinline__ void ld_terms4(uint32_t saddr, uint32_t copy_bytes, float* x) {
  x[0] = x[1] = x[2] = x[3] = 0.f;
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    uint32_t w0, w1;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(saddr + i * copy_bytes));
    x[0] += __uint_as_float(w0 << 16);
    x[1] += __uint_as_float(w0 & 0xFFFF0000u);
    x[2] += __uint_as_float(w1 << 16);
    x[3] += __uint_as_float(w1 & 0xFFFF0000u);
  }
}

// Four values in the output type to shared memory (8 bytes bf16, 16 bytes fp32).
__device__ __forceinline__ void st_out4(__nv_bfloat16* p, const float* v) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}
__device__ __forceinline__ void st_out4(float* p, const float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
// BYTES (8, 16 or 32) from shared staging to global memory.
template <int BYTES>
__device__ __forceinline__ void copy_piece(void* dst, const void* src) {
  if constexpr (BYTES == 8) {
    *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(src);
  } else {
#pragma unroll
    for (int i = 0; i < BYTES / 16; ++i) reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(src)[i];
  }
}

// Key gradients of this thread's token (TMEM lane t) and channel half:
// dq = dqbar EQ and dk = dkbar / EQ into registers, and the token's d log alpha
// terms x = qbar dqbar - kbar dkbar (qbar, kbar from their operand terms)
// written over its EQ values.
template <int C, int DK, int DV, typename TIN, typename TOUT, int H>
__device__ __forceinline__ void key_grads(uint32_t tmem, uint32_t sbase, float* eqx, float* dq, float* dk) {
  using K = ChunkCfg<C, DK, DV, TIN>;
  using BC = BwdCfg<C, DK, DV, TIN, TOUT>;
  constexpr int KO = H ? K::DK0 : 0, KN = H ? K::DK1 : K::DK0, NL = cround(KN, 8);
  const int t = threadIdx.x & 127, wq = t >> 5;
  if (32 * wq >= C) return;  // warp-uniform: lanes past the chunk
  const uint32_t lt = tmem + (static_cast<uint32_t>(32 * wq) << 16);
  float* row = eqx + t * BC::EP + KO;
#pragma unroll
  for (int c8 = 0; c8 < NL; c8 += 8) {
    float dqb[8], dkb[8];
    tmem_ld8(lt + BC::TM_DQ + KO + c8, dqb);
    tmem_ld8(lt + BC::TM_DK + KO + c8, dkb);
    tmem_ld_wait();
#pragma unroll
    for (int c4 = 0; c4 < 8 && c8 + c4 < KN; c4 += 4) {
      const int c = c8 + c4;
      const float4 f4 = *reinterpret_cast<const float4*>(row + c);
      const float f[4] = {f4.x, f4.y, f4.z, f4.w};
      float qb[4], kb[4], x[4];
      ld_terms4<BC::NTG>(sbase + BC::OFF_Q + kmaj16(t, KO + c, 128, K::SBO_K), K::AQ_SZ, qb);
      ld_terms4<BC::NTG>(sbase + BC::OFF_K + kmaj16(t, KO + c, 128, K::SBO_K), K::AQ_SZ, kb);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        dq[c + e] = dqb[c4 + e] * f[e];
        dk[c + e] = dkb[c4 + e] * __fdividef(1.f, f[e]);
        x[e] = qb[e] * dqb[c4 + e] - kb[e] * dkb[c4 + e];
      }
      *reinterpret_cast<float4*>(row + c) = make_float4(x[0], x[1], x[2], x[3]);
    }
  }
}

// dq and dk of this thread's token and channel half -> staging rows.
template <int C, int DK, int DV, typename TIN, typename TOUT, int H>
__device__ __forceinline__ void stage_key_grads(uint8_t* smem, const float* dq, const float* dk) {
  using K = ChunkCfg<C, DK, DV, TIN>;
  using BC = BwdCfg<C, DK, DV, TIN, TOUT>;
  constexpr int KO = H ? K::DK0 : 0, KN = H ? K::DK1 : K::DK0;
  const int t = threadIdx.x & 127;
  if (t >= C) return;
  TOUT* sq = reinterpret_cast<TOUT*>(smem + BC::OFF_SQ + t * BC::KSB) + KO;
  TOUT* sk = reinterpret_cast<TOUT*>(smem + BC::OFF_SK + t * BC::KSB) + KO;
#pragma unroll
  for (int c = 0; c < KN; c += 4) {
    st_out4(sq + c, dq + c);
    st_out4(sk + c, dk + c);
  }
}

// dv of this thread's token (TMEM lane t) and channel half -> staging row.  With
// a value gate (`eqb`: the unit's rows of 2^(e - rho)) the product is the
// gradient of vbar = v / EQb and is rescaled to dv = dvbar / EQb.
template <int C, int DK, int DV, typename TIN, typename TOUT, int H>
__device__ __forceinline__ void stage_dv(uint32_t tmem, uint8_t* smem, const float* eqb = nullptr, int nvalid = 0) {
  using K = ChunkCfg<C, DK, DV, TIN>;
  using BC = BwdCfg<C, DK, DV, TIN, TOUT>;
  constexpr int VO = H ? K::DV0 : 0, VN = H ? K::DV1 : K::DV0;
  const int t = threadIdx.x & 127, wq = t >> 5;
  if (32 * wq >= C) return;  // warp-uniform
  const uint32_t lt = tmem + (static_cast<uint32_t>(32 * wq) << 16) + BC::TM_DV + VO;
  float v[VN];
#pragma unroll
  for (int c = 0; c < VN; c += 8) tmem_ld8(lt + c, v + c);
  tmem_ld_wait();
  if (eqb != nullptr && t < nvalid) {
#pragma unroll
    for (int i = 0; i < VN; ++i) v[i] = __fdiv_rn(v[i], __ldg(eqb + (size_t)t * DV + VO + i));
  }
  TOUT* sv = reinterpret_cast<TOUT*>(smem + BC::OFF_SV + t * BC::VSB) + VO;
#pragma unroll
  for (int c = 0; c < VN; c += 4) st_out4(sv + c, v + c);
}

// With EXT (value gate and state input / output, fp32 inputs): v and dO are
// loaded as vbar = v / EQb and dObar = dO EQb, S' and Gt carry the value-side
// references 2^rho and 2^(Gb - rho) of their rows, dv is rescaled by 1 / EQb, and
// the last chunk's boundary term uses the final state (its G is the gradient of
// the final state, zero when none is given).
template <int C, int DK, int DV, typename TIN, typename TOUT, bool EXT = false>
__global__ void __launch_bounds__(256, 2) gla_chunk_grad_kernel(const GlaArgs a) {
  using K = ChunkCfg<C, DK, DV, TIN>;
  using BC = BwdCfg<C, DK, DV, TIN, TOUT>;
  constexpr int NTG = BC::NTG, NTV = BC::NTV, NTP = BC::NTP, DKP = K::DKP, DVP = K::DVP, PSK = K::PSK;
  constexpr int KL = cround(K::DK0, 8);  // key-gradient registers of a channel half
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ GradSmem sh;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int nunits = a.B * a.H * a.nchunks;
  if (a.flist != nullptr) {  // unit-list mode: CTAs beyond the list end before taking any resource
    griddep_wait();
    if ((int)blockIdx.x >= (int)__ldcg(a.flist)) return;
  }
  if (warp == 0) {
    tmem_alloc(&sh.tmem, BC::TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < 6; ++i) mbar_init(&sh.bar[i], 1);
    mbar_init(&sh.sbar, 1);
    sh.mma_pend = -1;
    sh.st_pend = 0;
    fence_mbar_init();
  }
  if (tid < 128) sh.bnd[tid >> 6][tid & 63] = 0.f;
  // With a unit list (the units the fp16 gradient kernel left), only those units
  // are processed; the list is written by that kernel, so it is read after the wait.
  const bool listed = a.flist != nullptr;
  if (!listed && (int)blockIdx.x < nunits) fill_rows(a, blockIdx.x, C, sh.rows[0]);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem;
  const uint32_t sbase = smem_u32(smem);
  const uint64_t dQk = sdesc(sbase + BC::OFF_Q, 128, K::SBO_K), dQm = sdesc(sbase + BC::OFF_Q, K::SBO_K, 128);
  const uint64_t dKk = sdesc(sbase + BC::OFF_K, 128, K::SBO_K), dKm = sdesc(sbase + BC::OFF_K, K::SBO_K, 128);
  const uint64_t dVk = sdesc(sbase + BC::OFF_V, 128, K::SBO_V);
  const uint64_t dDOk = sdesc(sbase + BC::OFF_DO, 128, K::SBO_V), dDOm = sdesc(sbase + BC::OFF_DO, K::SBO_V, 128);
  const uint64_t dSPm = sdesc(sbase + BC::OFF_SP, K::SBO_K, 128);
  const uint64_t dGTm = sdesc(sbase + BC::OFF_GT, K::SBO_K, 128), dGTk = sdesc(sbase + BC::OFF_GT, 128, K::SBO_K);
  float* EQ = reinterpret_cast<float*>(smem + BC::OFF_EQ);  // EQ rows, then the d log alpha terms
  uint32_t ph = 0;
  int it = 0;
  bool timed_out = false;  // a wait of this thread gave up: nothing further is issued
  bool stop = false;       // some wait of the CTA gave up (uniform, from the last barrier)
  auto commit = [&](int i) {
    mma_commit(&sh.bar[i]);
    sh.mma_pend = i;
    sh.mma_ph = ph;
  };
  auto wait_group = [&](int i) {  // one thread: product group i of this unit is complete
    if (!mbar_wait(&sh.bar[i], ph, spin_limit(a))) timed_out = true;
    else if (tid == 0 && sh.mma_pend == i) sh.mma_pend = -1;
  };
  auto wait_all = [&](int i) {  // every thread: product group i of this unit is complete
    if (!stop) wait_group(i);
    tc_fence_after();
  };
  auto publish = [&]() {  // this thread's TMEM / shared writes, then a CTA barrier
    fence_async_smem();
    tc_fence_before();
    stop = __syncthreads_or(timed_out);
    tc_fence_after();
  };

  // Row pieces of a unit (q, k, EQ).  With 128-token chunks (where they fit 40
  // registers) they are loaded one unit ahead: issued while the previous unit's
  // d log alpha is formed, consumed as the unit's operands.  Otherwise
  // (64-token chunks, whose wider rows leave no room) they are loaded when the
  // unit starts.
  constexpr int RQ = K::NPK * (2 * PSK * (int)sizeof(TIN) / 4 + PSK);
  constexpr bool PRE = C == 128 && RQ <= 40;
  Piece<TIN, PSK> pq[K::NPK], pk[K::NPK];
  Piece<float, PSK> pe[K::NPK];
  auto issue_qk = [&](int u, const long long* rows) {
    const Unit U(a, u);
#pragma unroll
    for (int j = 0; j < K::NPK; ++j) {
      const int i = tid + 256 * j;
      int tt, g;
      piece_of<K::NGK>(i, tt, g);
      const long long gr = i < C * K::NGK ? rows[tt] : -1;
      const bool valid = gr >= 0;
      const size_t off = tok_row(gr, a, U.h) * DK + g * PSK;
      pq[j].load(reinterpret_cast<const TIN*>(a.q) + off, valid);
      pk[j].load(reinterpret_cast<const TIN*>(a.k) + off, valid);
      pe[j].load(a.gEQ + ((size_t)U.bz * a.L + (valid ? U.n * C + tt : 0)) * DK + g * PSK, valid);
    }
  };
  // The unit's contiguous blocks by bulk copy (one thread; they bypass the
  // load/store path): S_n into the S' slot, G_n into the Gt slot, S_{n+1} (not
  // for the last chunk) into the qbar slot, and the chunk constants.  Issued for
  // the next unit once this unit's gradient rows have left the staging over
  // those slots, so they land while this unit's d log alpha is formed.
  constexpr uint32_t SB = DV * DK * 4;
  auto issue_states = [&](int u) {
    const Unit U(a, u);
    const bool has_next_chunk = U.n + 1 < a.nchunks;  // G of the last chunk is zero without EXT
    const bool has_bnd = has_next_chunk || EXT;
    const float* s_next = has_next_chunk ? a.dsn + (size_t)(u + 1) * DV * DK : a.sfin + (size_t)U.bh * DV * DK;
    sh.st_pend = 1;
    sh.st_ph = ph;
    mbar_arrive_expect_tx(&sh.sbar, 2 * SB + (has_bnd ? SB : 0u) + 2 * DK * 4);
    bulk_copy_g2s(sbase + BC::OFF_SP, a.dsn + (size_t)u * DV * DK, SB, &sh.sbar);
    bulk_copy_g2s(sbase + BC::OFF_GT, a.dhn + (size_t)u * DV * DK, SB, &sh.sbar);
    if (has_bnd) bulk_copy_g2s(sbase + BC::OFF_Q, s_next, SB, &sh.sbar);
    bulk_copy_g2s(smem_u32(sh.gch), a.gCH + ((size_t)U.bz * a.nchunks + U.n) * 4 * DK, 2 * DK * 4, &sh.sbar);
  };
  // The kernel before this one is the state scan, which writes only the chunk
  // states and state gradients; everything older has completed.  So the first
  // unit's other rows are requested before the wait for that scan.
  constexpr int VSV = EXT ? VS_VBAR : VS_NONE, VSD = EXT ? VS_DOBAR : VS_NONE;
  auto first_rows = [&](int u0) {
    const Unit U0(a, u0);
    if constexpr (PRE) issue_qk(u0, sh.rows[0]);
    load_v_rows_t<C, DK, DV, TIN, 256, VSV>(a, U0.h, sh.rows[0], a.v, sbase + BC::OFF_V, U0.bz, U0.n);
    load_v_rows_t<C, DK, DV, TIN, 256, VSD>(a, U0.h, sh.rows[0], a.dO, sbase + BC::OFF_DO, U0.bz, U0.n);
  };
  if (!listed && (int)blockIdx.x < nunits) first_rows(blockIdx.x);
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  const int count = listed ? (int)__ldcg(a.flist) : nunits;
  auto unit_at = [&](int kx) { return listed ? (int)__ldcg(a.flist + 1 + kx) : kx; };
  if (listed && (int)blockIdx.x < count) {
    fill_rows(a, unit_at(blockIdx.x), C, sh.rows[0]);
    __syncthreads();
    first_rows(unit_at(blockIdx.x));
  }
  if (tid == 0 && (int)blockIdx.x < count) issue_states(unit_at(blockIdx.x));

  bool any_strong = false;  // uniform: a unit of this CTA has a flagged chunk
  for (int kx = blockIdx.x; kx < count; kx += gridDim.x, ++it) {
    const int u = unit_at(kx);
    const Unit U(a, u);
    const int hz = U.bz - U.b * a.gate_heads;
    const bool skip = !EXT && strong::flagged(a, U.bz, U.n);  // strong gate: its gradients come after the loop
    any_strong |= skip;
    const bool has_next = kx + (int)gridDim.x < count;
    const int un = has_next ? unit_at(kx + gridDim.x) : 0;
    float* bnd = sh.bnd[it & 1];
    const long long* rows = sh.rows[it & 1];  // this unit's grid tokens
    long long* rows_next = sh.rows[(it + 1) & 1];
    if (has_next) fill_rows(a, un, C, rows_next);  // read after the operand barrier
    // ---- the state blocks, read in place: S' and Gt rows (to registers) and the boundary term
    const bool has_next_chunk = U.n + 1 < a.nchunks;
    const bool has_bnd = has_next_chunk || EXT;
    if (!mbar_wait(&sh.sbar, ph, spin_limit(a))) timed_out = true;
    else if (tid == 0) sh.st_pend = 0;
    float spv[K::NPS][4], gtv[K::NPS][4];
#pragma unroll
    for (int j = 0; j < K::NPS; ++j) {
      const int i = tid + 256 * j;
      int jr, g;
      piece_of<K::NGS>(i, jr, g);
      const bool in = i < DV * K::NGS;
      const int off = (in ? jr * DK : 0) + 4 * g;
      const float4 sv = *reinterpret_cast<const float4*>(smem + BC::OFF_SP + 4 * off);
      const float4 gv = *reinterpret_cast<const float4*>(smem + BC::OFF_GT + 4 * off);
      const float4 nv = has_bnd ? *reinterpret_cast<const float4*>(smem + BC::OFF_Q + 4 * off)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
      float4 c0 = *reinterpret_cast<const float4*>(&sh.gch[4 * g]);
      float4 c1 = *reinterpret_cast<const float4*>(&sh.gch[DK + 4 * g]);
      if constexpr (EXT) {  // the row's value-side references: 2^rho (S'), 2^(Gb - rho) (Gt)
        const float* chb = a.gCHb + ((size_t)U.bz * a.nchunks + U.n) * 4 * DV + (in ? jr : 0);
        const float rb = __ldg(chb), gb = __ldg(chb + DV);
        c0 = make_float4(c0.x * rb, c0.y * rb, c0.z * rb, c0.w * rb);
        c1 = make_float4(c1.x * gb, c1.y * gb, c1.z * gb, c1.w * gb);
      }
      spv[j][0] = sv.x * c0.x;  // S' = 2^r S_n (2^rho with a value gate)
      spv[j][1] = sv.y * c0.y;
      spv[j][2] = sv.z * c0.z;
      spv[j][3] = sv.w * c0.w;
      gtv[j][0] = gv.x * c1.x;  // Gt = 2^(Gamma - r) G_n (2^(Gb - rho))
      gtv[j][1] = gv.y * c1.y;
      gtv[j][2] = gv.z * c1.z;
      gtv[j][3] = gv.w * c1.w;
      float bp[4] = {in ? nv.x * gv.x : 0.f, in ? nv.y * gv.y : 0.f, in ? nv.z * gv.z : 0.f, in ? nv.w * gv.w : 0.f};
      // sum over the 8 rows of this lane group (lanes i..i+7 share the channel group)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        bp[e] += __shfl_xor_sync(0xffffffffu, bp[e], 1);
        bp[e] += __shfl_xor_sync(0xffffffffu, bp[e], 2);
        bp[e] += __shfl_xor_sync(0xffffffffu, bp[e], 4);
      }
      if (in && (i & 7) == 0) {
#pragma unroll
        for (int e = 0; e < 4; ++e) atomicAdd(&bnd[4 * g + e], bp[e]);
      }
    }
    __syncthreads();  // every state row read: the slots take the operands
    // ---- operands: S' and Gt rows; qbar, kbar rows and EQ (from the q / k pieces)
#pragma unroll
    for (int j = 0; j < K::NPS; ++j) {
      const int i = tid + 256 * j;
      int jr, g;
      piece_of<K::NGS>(i, jr, g);
      if (i < DV * K::NGS) {
        st_piece<NTG, 4>(sbase + BC::OFF_SP, jr, K::SBO_K, 4 * g, K::SPT_SZ, spv[j]);
        st_piece<NTG, 4>(sbase + BC::OFF_GT, jr, K::SBO_K, 4 * g, K::SPT_SZ, gtv[j]);
      }
    }
    if constexpr (!PRE) issue_qk(u, rows);
#pragma unroll
    for (int j = 0; j < K::NPK; ++j) {
      const int i = tid + 256 * j;
      int tt, g;
      piece_of<K::NGK>(i, tt, g);
      if (i < C * K::NGK) {
        const bool valid = U.n * C + tt < a.L;
        float qv[PSK], kv[PSK], ev[PSK];
        pq[j].unpack(qv);
        pk[j].unpack(kv);
        pe[j].unpack(ev);
#pragma unroll
        for (int e = 0; e < PSK; ++e) {
          ev[e] = valid ? ev[e] : 1.f;
          qv[e] *= ev[e];
          kv[e] *= __fdividef(1.f, ev[e]);
        }
        st_piece<NTG, PSK>(sbase + BC::OFF_Q, tt, K::SBO_K, g * PSK, K::AQ_SZ, qv);
        st_piece<NTG, PSK>(sbase + BC::OFF_K, tt, K::SBO_K, g * PSK, K::AQ_SZ, kv);
#pragma unroll
        for (int e = 0; e < PSK; e += 4)
          *reinterpret_cast<float4*>(EQ + tt * BC::EP + g * PSK + e) =
              make_float4(ev[e], ev[e + 1], ev[e + 2], ev[e + 3]);
      }
    }
    {  // zero padding: key channels DK..DKP of every row; value rows DV..DVP of S' and Gt
      const float zz[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (K::NPAD > 0) {
        for (int i = tid; i < C * K::NPAD; i += 256) {
          const int row = i / K::NPAD, c = DK + 4 * (i % K::NPAD);
          st_piece<NTG, 4>(sbase + BC::OFF_Q, row, K::SBO_K, c, K::AQ_SZ, zz);
          st_piece<NTG, 4>(sbase + BC::OFF_K, row, K::SBO_K, c, K::AQ_SZ, zz);
        }
        for (int i = tid; i < DV * K::NPAD; i += 256) {
          const int row = i / K::NPAD, c = DK + 4 * (i % K::NPAD);
          st_piece<NTG, 4>(sbase + BC::OFF_SP, row, K::SBO_K, c, K::SPT_SZ, zz);
          st_piece<NTG, 4>(sbase + BC::OFF_GT, row, K::SBO_K, c, K::SPT_SZ, zz);
        }
      }
      if constexpr (DVP > DV) {
        for (int i = tid; i < (DVP - DV) * (DKP / 4); i += 256) {
          const int row = DV + i / (DKP / 4), c = 4 * (i % (DKP / 4));
          st_piece<NTG, 4>(sbase + BC::OFF_SP, row, K::SBO_K, c, K::SPT_SZ, zz);
          st_piece<NTG, 4>(sbase + BC::OFF_GT, row, K::SBO_K, c, K::SPT_SZ, zz);
        }
      }
    }
    cp_async_wait_all();
    publish();
    // ---- P^T and the three inter-chunk terms
    if (tid == 0 && !stop) {
      mma_issue<NTG, NTG, DKP / 16>(tmem + BC::TM_R, dKk, K::AQ_SZ, 256, dQk, K::AQ_SZ, 256, idesc_bf16(128, C),
                                    false);  // P^T[s][t]
      mma_issue<NTV, NTG, DVP / 16>(tmem + BC::TM_DQ, dDOk, K::VR_SZ, 256, dSPm, K::SPT_SZ, 2 * K::SBO_K,
                                    idesc_bf16(128, DKP, false, true), false);  // dO S'^T
      mma_issue<NTV, NTG, DVP / 16>(tmem + BC::TM_DK, dVk, K::VR_SZ, 256, dGTm, K::SPT_SZ, 2 * K::SBO_K,
                                    idesc_bf16(128, DKP, false, true), false);  // V Gt^T
      mma_issue<NTG, NTG, DKP / 16>(tmem + BC::TM_DV, dKk, K::AQ_SZ, 256, dGTk, K::SPT_SZ, 256, idesc_bf16(128, DVP),
                                    false);  // kbar Gt
      commit(0);
    }
    wait_all(0);
    mask_to_terms<C, BC::PT_STRIDE>(tmem, BC::TM_R, true);
    tmem_st_wait();
    publish();
    // ---- dv += P^T dO; then dP^T into the region once that product has read it
    if (tid == 0 && !stop) {
      mma_issue_ts<NTP, NTV, C / 16>(tmem + BC::TM_DV, tmem + BC::TM_R, BC::PT_STRIDE, dDOm, K::VR_SZ, 2 * K::SBO_V,
                                     idesc_bf16(128, DVP, false, true), true);
      commit(1);
      wait_group(1);
      tc_fence_after();
      if (!timed_out) {
        mma_issue<NTV, NTV, DVP / 16>(tmem + BC::TM_R, dVk, K::VR_SZ, 256, dDOk, K::VR_SZ, 256, idesc_bf16(128, C),
                                      false);  // dP^T[s][t]
        commit(2);
      }
    }
    wait_all(2);
    mask_to_terms<C, BC::PT_STRIDE>(tmem, BC::TM_R, true);
    tmem_st_wait();
    publish();
    // ---- dkbar += dP^T qbar; then dP
    if (tid == 0 && !stop) {
      mma_issue_ts<NTP, NTG, C / 16>(tmem + BC::TM_DK, tmem + BC::TM_R, BC::PT_STRIDE, dQm, K::AQ_SZ, 2 * K::SBO_K,
                                     idesc_bf16(128, DKP, false, true), true);
      commit(3);
      wait_group(3);
      tc_fence_after();
      if (!timed_out) {
        mma_issue<NTV, NTV, DVP / 16>(tmem + BC::TM_R, dDOk, K::VR_SZ, 256, dVk, K::VR_SZ, 256, idesc_bf16(128, C),
                                      false);  // dP[t][s]
        commit(4);
      }
    }
    wait_all(4);
    // v and dO are no longer read: the next unit's rows start to arrive now
    if (has_next && !timed_out && !stop) {
      const Unit Un(a, un);
      load_v_rows_t<C, DK, DV, TIN, 256, VSV>(a, Un.h, rows_next, a.v, sbase + BC::OFF_V, Un.bz, Un.n);
      load_v_rows_t<C, DK, DV, TIN, 256, VSD>(a, Un.h, rows_next, a.dO, sbase + BC::OFF_DO, Un.bz, Un.n);
    }
    mask_to_terms<C, BC::PT_STRIDE>(tmem, BC::TM_R, false);
    tmem_st_wait();
    publish();
    // ---- dqbar += dP kbar
    if (tid == 0 && !stop) {
      mma_issue_ts<NTP, NTG, C / 16>(tmem + BC::TM_DQ, tmem + BC::TM_R, BC::PT_STRIDE, dKm, K::AQ_SZ, 2 * K::SBO_K,
                                     idesc_bf16(128, DKP, false, true), true);
      commit(5);
    }
    wait_all(5);
    ph ^= 1u;
    // ---- dq, dk and the tokens' d log alpha terms from TMEM, the operands and EQ
    const float* eqb = EXT ? a.gEQb + ((size_t)U.bz * a.L + (size_t)U.n * C) * DV : nullptr;
    const int nvalid = min(C, a.L - U.n * C);
    float dq[KL], dk[KL];
    if (tid < 128) key_grads<C, DK, DV, TIN, TOUT, 0>(tmem, sbase, EQ, dq, dk);
    else key_grads<C, DK, DV, TIN, TOUT, 1>(tmem, sbase, EQ, dq, dk);
    tc_fence_before();
    __syncthreads();  // qbar, kbar read: their rows become staging
    if (tid < 128) stage_key_grads<C, DK, DV, TIN, TOUT, 0>(smem, dq, dk);
    else stage_key_grads<C, DK, DV, TIN, TOUT, 1>(smem, dq, dk);
    if constexpr (BC::ONE_PASS) {
      if (tid < 128) stage_dv<C, DK, DV, TIN, TOUT, 0>(tmem, smem, eqb, nvalid);
      else stage_dv<C, DK, DV, TIN, TOUT, 1>(tmem, smem, eqb, nvalid);
    }
    tc_fence_before();
    __syncthreads();
    // ---- the next unit's q, k and EQ pieces start to arrive; dq, dk (and dv) rows as coalesced pieces
    if (PRE && has_next) issue_qk(un, rows_next);
    constexpr int KPB = PSK * (int)sizeof(TOUT), VPB = 8 * (int)sizeof(TOUT);
#pragma unroll
    for (int j = 0; j < K::NPK; ++j) {
      const int i = tid + 256 * j;
      int tt, g;
      piece_of<K::NGK>(i, tt, g);
      const long long gr = i < C * K::NGK ? rows[tt] : -1;
      if (gr >= 0 && !skip) {
        const size_t off = tok_row(gr, a, U.h) * DK + g * PSK;
        copy_piece<KPB>(reinterpret_cast<TOUT*>(a.dq) + off, smem + BC::OFF_SQ + tt * BC::KSB + g * KPB);
        copy_piece<KPB>(reinterpret_cast<TOUT*>(a.dk) + off, smem + BC::OFF_SK + tt * BC::KSB + g * KPB);
      }
    }
    auto store_dv = [&]() {
#pragma unroll
      for (int j = 0; j < K::NPV; ++j) {
        const int i = tid + 256 * j;
        int tt, g;
        piece_of<K::NGV>(i, tt, g);
        const long long gr = i < C * K::NGV ? rows[tt] : -1;
        if (gr >= 0 && !skip)
          copy_piece<VPB>(reinterpret_cast<TOUT*>(a.dv) + tok_row(gr, a, U.h) * DV + 8 * g,
                          smem + BC::OFF_SV + tt * BC::VSB + g * VPB);
      }
    };
    if constexpr (BC::ONE_PASS) {
      store_dv();
    } else {
      __syncthreads();  // dq / dk staging read: dv takes its place
      if (tid < 128) stage_dv<C, DK, DV, TIN, TOUT, 0>(tmem, smem, eqb, nvalid);
      else stage_dv<C, DK, DV, TIN, TOUT, 1>(tmem, smem, eqb, nvalid);
      __syncthreads();
      store_dv();
    }
    // ---- d log alpha: reverse cumsum over the chunk's tokens + the boundary term
    const int sc = tid % DK, sg = tid / DK;
    const int t0 = sg * BC::SEGL, t1 = min(C, t0 + BC::SEGL);
    if (sg < BC::NSG) {
      float acc = 0.f;
      for (int t = t1 - 1; t >= t0; --t) {
        acc += EQ[t * BC::EP + sc];
        EQ[t * BC::EP + sc] = acc;
      }
      sh.segtot[sg][sc] = acc;
    }
    if (tid < 64) sh.bnd[(it + 1) & 1][tid] = 0.f;  // the next unit's accumulator
    fence_async_smem();  // the staging reads precede the next unit's bulk copies into the same slots
    stop = __syncthreads_or(timed_out);
    if (tid == 0 && has_next && !stop) issue_states(un);  // they land while d log alpha is finished
    if (sg < BC::NSG) {
      float post = bnd[sc];
      for (int s2 = sg + 1; s2 < BC::NSG; ++s2) post += sh.segtot[s2][sc];
      for (int t = t0; t < t1; ++t) {
        const long long gr = rows[t];
        if (gr >= 0 && !skip) {
          float* dst = a.dla + ((size_t)gr * a.gate_heads + hz) * DK + sc;
          const float val = EQ[t * BC::EP + sc] + post;
          if (a.gate_heads == 1) atomicAdd(dst, val);
          else *dst = val;
        }
      }
    }
    // staging, EQ rows and segment totals are reused by the next unit; after a
    // wait gave up anywhere in the CTA, no further unit starts
    if (__syncthreads_or(timed_out)) break;
  }
  // ---- drain: this thread's row copies, the state copies and the last products
  // complete before TMEM is released and the CTA exits
  if (timed_out) set_status(a.status, DIG_ERR_DEVICE_TIMEOUT);
  cp_async_wait_all();
  if (tid == 0) {
    if (sh.st_pend) mbar_wait(&sh.sbar, sh.st_ph, kSpinLimitNs);
    if (sh.mma_pend >= 0) mbar_wait(&sh.bar[sh.mma_pend], sh.mma_ph, kSpinLimitNs);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, BC::TM_COLS);
  if constexpr (!EXT) {  // this CTA's units of chunks flagged by the gate kernel (strong gates), exactly in fp32
    static_assert(BC::SMEM >= strong::Cfg<C, DK, DV>::SMEM_GRAD, "shared memory of the strong-gate phase");
    if (any_strong && !__syncthreads_or(timed_out))
      for (int kx = blockIdx.x; kx < count; kx += gridDim.x) {
        const int u = unit_at(kx);
        const Unit U(a, u);
        if (strong::flagged(a, U.bz, U.n)) strong::grad_unit<C, DK, DV, TIN, TOUT>(a, u, smem);
      }
  }
}

// ============================================================== dH from saved records
// Per unit, when the forward's gate factors and states are reused: the chunk's
// state-gradient contribution dH = (q 2^b)^T dO with q 2^b = q * EQ * 2^r (no
// gate cumsum, no dS), rows stored value-major to `dhn`.
template <int C, int DK, int DV, typename TIN>
struct DhCfg {
  using K = ChunkCfg<C, DK, DV, TIN>;
  static constexpr int OFF_QB = 0;
  static constexpr int OFF_DO = K::NTG * K::AQ_SZ;
  static constexpr int SDP = DK + 4;
  static constexpr int OFF_SD = cround(OFF_DO + K::NTV * K::VR_SZ, 16);
  static constexpr int SMEM = cmax(OFF_SD + DV * SDP * 4, OFF_DO + K::VR_READ);
  static constexpr int TM_COLS = pow2ceil(K::DKP);
  static constexpr int PER_SM = SMEM <= 72 * 1024 ? 3 : SMEM <= 110 * 1024 ? 2 : 1;
  static_assert(SMEM <= 225 * 1024, "shared-memory budget");
};

template <int C, int DK, int DV, typename TIN>
__global__ void __launch_bounds__(256, 3) gla_chunk_dh_kernel(const GlaArgs a) {
  using K = ChunkCfg<C, DK, DV, TIN>;
  using DC = DhCfg<C, DK, DV, TIN>;
  constexpr int NTG = K::NTG, NTV = K::NTV, DKP = K::DKP, PSK = K::PSK;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ StateSmem sh;
  const int tid = threadIdx.x, warp = tid >> 5;
  if (warp == 0) {
    tmem_alloc(&sh.tmem, DC::TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&sh.bar, 1);
    fence_mbar_init();
  }
  const int nunits = a.B * a.H * a.nchunks;
  if ((int)blockIdx.x < nunits) fill_rows(a, blockIdx.x, C, sh.rows[0]);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  const uint32_t tmem = sh.tmem;
  const uint32_t sbase = smem_u32(smem);
  float* SD = reinterpret_cast<float*>(smem + DC::OFF_SD);
  const uint64_t dDOm = sdesc(sbase + DC::OFF_DO, K::SBO_V, 128);
  const uint64_t dQBm = sdesc(sbase + DC::OFF_QB, K::SBO_K, 128);
  uint32_t ph = 0;
  bool timed_out = false;  // a wait of this thread gave up: the CTA stops after this unit
  if (tid == 0) sh.mma_pend = 0;
  Piece<TIN, PSK> pq[K::NPK];
  Piece<float, PSK> pe[K::NPK];
  Piece<float, 4> pc[K::NPK * PSK / 4];  // 2^r of the piece's channels
  auto issue_rows = [&](int u, const long long* rows) {
    const Unit U(a, u);
#pragma unroll
    for (int j = 0; j < K::NPK; ++j) {
      const int i = tid + 256 * j;
      int tt, g;
      piece_of<K::NGK>(i, tt, g);
      const long long gr = i < C * K::NGK ? rows[tt] : -1;
      const bool valid = gr >= 0;
      pq[j].load(reinterpret_cast<const TIN*>(a.q) + tok_row(gr, a, U.h) * DK + g * PSK, valid);
      pe[j].load(a.gEQ + ((size_t)U.bz * a.L + (valid ? U.n * C + tt : 0)) * DK + g * PSK, valid);
      const float* ch = a.gCH + ((size_t)U.bz * a.nchunks + U.n) * 4 * DK + g * PSK;
#pragma unroll
      for (int e = 0; e < PSK / 4; ++e) pc[j * (PSK / 4) + e].load(ch + 4 * e, i < C * K::NGK);
    }
  };
  if ((int)blockIdx.x < nunits) {
    issue_rows(blockIdx.x, sh.rows[0]);
    load_v_rows_t<C, DK, DV, TIN>(a, Unit(a, blockIdx.x).h, sh.rows[0], a.dO, sbase + DC::OFF_DO);
  }
  int it = 0;
  for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++it) {
    const int un = u + gridDim.x;
    const bool has_next = un < nunits;
    long long* rows_next = sh.rows[(it + 1) & 1];
    if (has_next) fill_rows(a, un, C, rows_next);  // read after the next barrier
    // ---- q 2^b = q * EQ * 2^r as operand rows
#pragma unroll
    for (int j = 0; j < K::NPK; ++j) {
      const int i = tid + 256 * j;
      int tt, g;
      piece_of<K::NGK>(i, tt, g);
      if (i < C * K::NGK) {
        float qv[PSK], ev[PSK], cv[PSK];
        pq[j].unpack(qv);
        pe[j].unpack(ev);
#pragma unroll
        for (int e = 0; e < PSK / 4; ++e) pc[j * (PSK / 4) + e].unpack(cv + 4 * e);
#pragma unroll
        for (int e = 0; e < PSK; ++e) qv[e] *= ev[e] * cv[e];
        st_piece<NTG, PSK>(sbase + DC::OFF_QB, tt, K::SBO_K, g * PSK, K::AQ_SZ, qv);
      }
    }
    if constexpr (K::NPAD > 0) {
      const float zz[4] = {0.f, 0.f, 0.f, 0.f};
      for (int i = tid; i < C * K::NPAD; i += 256)
        st_piece<NTG, 4>(sbase + DC::OFF_QB, i / K::NPAD, K::SBO_K, DK + 4 * (i % K::NPAD), K::AQ_SZ, zz);
    }
    cp_async_wait_all();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (has_next) issue_rows(un, rows_next);  // this unit's row pieces are consumed
    if (tid == 0) {
      mma_issue<NTV, NTG, C / 16>(tmem, dDOm, K::VR_SZ, 2 * K::SBO_V, dQBm, K::AQ_SZ, 2 * K::SBO_K,
                                  idesc_bf16(128, DKP, true, true), false);
      mma_commit(&sh.bar);
      sh.mma_pend = 1;
      sh.mma_ph = ph;
    }
    if (!mbar_wait(&sh.bar, ph, spin_limit(a))) timed_out = true;
    else if (tid == 0) sh.mma_pend = 0;
    ph ^= 1u;
    tc_fence_after();
    if (has_next && !timed_out)
      load_v_rows_t<C, DK, DV, TIN>(a, Unit(a, un).h, rows_next, a.dO, sbase + DC::OFF_DO);
    if (tid < 128) stage_rows_dk<C, DK, DV, TIN, 0>(tmem, 0, SD, DC::SDP);
    else stage_rows_dk<C, DK, DV, TIN, 1>(tmem, 0, SD, DC::SDP);
    tc_fence_before();
    __syncthreads();
    float4* dst = reinterpret_cast<float4*>(a.dhn + (size_t)u * DV * DK);
    for (int i = tid; i < DV * DK / 4; i += 256) {
      const int row = i / (DK / 4), c4 = i - row * (DK / 4);
      __stcg(dst + i, *reinterpret_cast<const float4*>(SD + row * DC::SDP + 4 * c4));
    }
    // staging and operands are reused by the next unit; after a wait gave up
    // anywhere in the CTA, no further unit starts
    if (__syncthreads_or(timed_out)) break;
  }
  // ---- drain: this thread's row copies, and the last products, complete before exit
  if (timed_out) set_status(a.status, DIG_ERR_DEVICE_TIMEOUT);
  cp_async_wait_all();
  if (tid == 0 && sh.mma_pend) mbar_wait(&sh.bar, sh.mma_ph, kSpinLimitNs);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, DC::TM_COLS);
}

// ------------------------------------------------------------------ launch
bool gla_grad_tma_eligible(const GlaArgs& a, int dk, int dv, int tin, int chunk);  // gla_bwd_tma.cu
cudaError_t launch_grad_tma(const GlaArgs& a, int tout, cudaStream_t s, bool* launched);

namespace {

template <int DK, int DV, typename TIN, typename TOUT>
cudaError_t launch_typed(const GlaArgs& a, bool saved, cudaStream_t s) {
  constexpr int C = bwd_chunk_len(DK, DV, std::is_same<TIN, float>::value);
  using BC = BwdCfg<C, DK, DV, TIN, TOUT>;
  const long long units = (long long)a.B * a.H * a.nchunks;
  if (units <= 0) return cudaSuccess;
  cudaError_t e;
  // bf16 inputs of the shapes the fp16 / TMA gradient kernel covers go through it;
  // the scan just before it clears the list of units it hands back.
  const bool tma = std::is_same<TIN, __nv_bfloat16>::value && a.flist != nullptr &&
                   gla_grad_tma_eligible(a, DK, DV, DIG_BF16, C);
  uint32_t* zero_word = tma ? a.flist : nullptr;
  if (saved) {  // gate factors and entry states come from the forward: only dH and its reverse scan
    bool reduced = false;
    if (std::is_same<TIN, __nv_bfloat16>::value && gla_reduce_tma_eligible(a, DK, DV, DIG_BF16, C))
      if ((e = launch_reduce_tma(a, true, s, &reduced)) != cudaSuccess) return e;
    if (!reduced) {
      using DC = DhCfg<C, DK, DV, TIN>;
      auto kd = gla_chunk_dh_kernel<C, DK, DV, TIN>;
      if ((e = cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize, DC::SMEM)) != cudaSuccess)
        return e;
      if ((e = launch_pdl(kd, persistent_grid(DC::PER_SM, units), 256, DC::SMEM, s, a)) != cudaSuccess) return e;
    }
    if ((e = launch_state_scan(a, a.dhn, true, nullptr, false, DK, DV, s, zero_word)) != cudaSuccess) return e;
  } else {
    if ((e = launch_chunk_state<C, DK, DV, TIN, true>(a, s)) != cudaSuccess) return e;
    if ((e = launch_state_scan(a, a.dsn, false, a.dhn, true, DK, DV, s, zero_word)) != cudaSuccess) return e;
  }
  GlaArgs b = a;
  b.flist = nullptr;
  if (tma) {
    bool launched = false;
    if ((e = launch_grad_tma(a, std::is_same<TOUT, float>::value ? DIG_F32 : DIG_BF16, s, &launched)) != cudaSuccess)
      return e;
    if (launched) b.flist = a.flist;  // the exact kernel takes only the units handed back
  }
  auto k = gla_chunk_grad_kernel<C, DK, DV, TIN, TOUT>;
  if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, BC::SMEM)) != cudaSuccess) return e;
  return launch_pdl(k, persistent_grid(BC::PER_SM, units), 256, BC::SMEM, s, b);
}

// Value gate and state input / output (fp32 inputs, exact kernels): gates, dS and
// dH, the forward scan seeded with S_0 (its final carry, the final state, kept
// for the last chunk's boundary term) and the reverse scan seeded with the final
// state's gradient (its final carry is the gradient of S_0), then the gradients.
template <int DK, int DV, typename TOUT>
cudaError_t launch_typed_ext(const GlaArgs& a, const ScanEnds& ends, cudaStream_t s) {
  constexpr int C = bwd_chunk_len(DK, DV, true);
  using BC = BwdCfg<C, DK, DV, float, TOUT>;
  const long long units = (long long)a.B * a.H * a.nchunks;
  if (units <= 0) return cudaSuccess;
  cudaError_t e;
  if ((e = launch_chunk_state<C, DK, DV, float, true, true>(a, s)) != cudaSuccess) return e;
  if ((e = launch_state_scan(a, a.dsn, false, a.dhn, true, DK, DV, s, nullptr, &ends)) != cudaSuccess) return e;
  GlaArgs b = a;
  b.flist = nullptr;
  auto k = gla_chunk_grad_kernel<C, DK, DV, float, TOUT, true>;
  if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, BC::SMEM)) != cudaSuccess) return e;
  return launch_pdl(k, persistent_grid(BC::PER_SM, units), 256, BC::SMEM, s, b);
}

template <int DK, int DV>
cudaError_t dispatch_types(const GlaVariant& v, const GlaArgs& a, bool saved, cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (v.tin == DIG_BF16) {
    if (v.tout == DIG_BF16) return launch_typed<DK, DV, bf, bf>(a, saved, s);
    return launch_typed<DK, DV, bf, float>(a, saved, s);
  }
  if (v.tout == DIG_BF16) return launch_typed<DK, DV, float, bf>(a, saved, s);
  return launch_typed<DK, DV, float, float>(a, saved, s);
}

}  // namespace

int gla_bwd_chunk(int dk, int dv, int dtype) { return bwd_chunk_len(dk, dv, dtype != DIG_BF16); }

cudaError_t launch_gla_bwd(const GlaVariant& v, const GlaArgs& a, bool saved, cudaStream_t s) {
  if (v.dk == 32 && v.dv == 64) return dispatch_types<32, 64>(v, a, saved, s);
  if (v.dk == 36 && v.dv == 72) return dispatch_types<36, 72>(v, a, saved, s);
  if (v.dk == 64 && v.dv == 64) return dispatch_types<64, 64>(v, a, saved, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_gla_bwd_ext(const GlaVariant& v, const GlaArgs& a, const ScanEnds& ends, cudaStream_t s) {
  if (v.tin != DIG_F32 || v.chunk != bwd_chunk_len(v.dk, v.dv, true)) return cudaErrorInvalidValue;
  const bool bf = v.tout == DIG_BF16;
  if (v.dk == 32 && v.dv == 64)
    return bf ? launch_typed_ext<32, 64, __nv_bfloat16>(a, ends, s) : launch_typed_ext<32, 64, float>(a, ends, s);
  if (v.dk == 36 && v.dv == 72)
    return bf ? launch_typed_ext<36, 72, __nv_bfloat16>(a, ends, s) : launch_typed_ext<36, 72, float>(a, ends, s);
  if (v.dk == 64 && v.dv == 64)
    return bf ? launch_typed_ext<64, 64, __nv_bfloat16>(a, ends, s) : launch_typed_ext<64, 64, float>(a, ends, s);
  return cudaErrorInvalidValue;
}

}  // namespace dig
