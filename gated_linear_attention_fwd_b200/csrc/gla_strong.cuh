// gla_strong.cuh -- chunks whose key gate decays too fast for the chunk
// factorisation (the chunkwise form of GLA eq. (5)-(8), DiG slides "GLA の導入";
// DiG "Efficiency Analysis").
//
// The chunk kernels split each pairwise decay 2^(b_t - b_s) (b the base-2 log
// cumsum of the gate over the chunk) into q 2^(b_t - r) times k 2^(r - b_s)
// about the chunk's middle token r.  A chunk whose base-2 log decay over half a
// chunk exceeds 115 in some key channel would overflow those factors in fp32.
// The gate kernel flags such a chunk (GlaArgs::sflag) and gives it neutral
// factors, so that the chunk kernels form finite values there and the scans the
// right chunk decay 2^Gamma.  The code below computes every result of a flagged
// chunk exactly in fp32, forming each decay as a product of per-token gates
// alpha_t <= 1 or as 2 to a partial sum of log decays (<= 0), so that nothing
// overflows for any finite gate logit.  It runs inside kernels that are
// launched anyway, so that ordinary gates pay one flag load per chunk:
//   * the state scan forms a flagged chunk's contribution itself (state_quad):
//     dS = sum_t diag(2^(Gamma - b_t)) k_t v_t^T (forward) or
//     dH = sum_t diag(2^(b_t)) q_t dO_t^T (reverse), instead of reading the block;
//   * the output kernels skip a flagged chunk's stores and, after their loop,
//     form (out_unit) o_t = S_t^T q_t with S_t = diag(alpha_t) S_{t-1} + k_t v_t^T
//     from the state entering the chunk, and y = Swish(r) o / rms(o) gamma;
//   * the fp16 gradient kernel hands a flagged chunk to the exact gradient
//     kernel, which skips its stores and, after its loop, forms (grad_unit), with
//     R_t the gradient of S_t (R_last = G + q dO^T at the chunk's last token,
//     R_{t-1} = diag(alpha_t) R_t + q_{t-1} dO_{t-1}^T, G the gradient of the state
//     leaving the chunk), dq_t = S_t dO_t (forward sweep), dk_t = R_t v_t and
//     dv_t = R_t^T k_t (reverse sweeps), and the head's share of
//     d log alpha_t = sum_{u >= t} (q_u dq_u - k_u dk_u) + rowsum(S_{n+1} o G).
// A kernel reaches those functions only when one of its own units was flagged,
// with all 256 threads and its dynamic shared memory.  The sweeps go token by
// token: a thread holds a slice of the d_k x d_v state in registers, and partial
// sums are reduced across the 2-8 consecutive lanes that share a row (key
// channel) or a column (value channel) of it.  Inputs are staged in shared memory
// 32 tokens at a time, as fp32.
#pragma once
#include <cuda_bf16.h>

#include "dig_common.cuh"
#include "gla.h"
#include "gla_common.cuh"

namespace dig {
namespace strong {

__host__ __device__ constexpr int p2floor(int x) {
  int p = 1;
  while (2 * p <= x) p *= 2;
  return p;
}

template <int C, int DK, int DV>
struct Cfg {
  static constexpr int TB = 32;                  // tokens staged at a time
  static constexpr int TPJ = p2floor(256 / DV);  // lanes per value channel (column sweeps)
  static constexpr int NCJ = cdiv(DK, TPJ);      // key channels per lane there
  static constexpr int TPC = p2floor(256 / DK);  // lanes per key channel (row sweeps)
  static constexpr int NJC = cdiv(DV, TPC);      // value channels per lane there
  // shared memory (fp32 unless noted): A [C][DK], qs, ks [TB][DK], vs, ds [TB][DV], rows [C] (int64),
  // bnd [DK], and for the gradients X [C][DK]
  static constexpr int OFF_Q = C * DK * 4;
  static constexpr int OFF_K = OFF_Q + TB * DK * 4;
  static constexpr int OFF_V = OFF_K + TB * DK * 4;
  static constexpr int OFF_D = OFF_V + TB * DV * 4;
  static constexpr int OFF_ROWS = OFF_D + TB * DV * 4;
  static constexpr int OFF_BND = OFF_ROWS + C * 8;
  static constexpr int OFF_X = OFF_BND + cround(DK, 4) * 4;
  static constexpr int SMEM_OUT = OFF_X;                  // bytes the output phase needs
  static constexpr int SMEM_GRAD = OFF_X + C * DK * 4;    // bytes the gradient phase needs
  static_assert(TPJ >= 2 && TPJ <= 32 && TPC >= 2 && TPC <= 32, "lane groups inside a warp");
  static_assert(NCJ <= 32 && NJC <= 32, "register slices");
};

__device__ __forceinline__ bool flagged(const GlaArgs& a, int bz, int n) {
  return a.sflag != nullptr && __ldcg(a.sflag + (size_t)bz * a.nchunks + n) != 0;
}

__device__ __forceinline__ float ld_in(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld_in(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_out(float* p, float x) { *p = x; }
__device__ __forceinline__ void st_out(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

template <int W>
__device__ __forceinline__ float group_sum(float x) {  // over W consecutive lanes (W a power of 2)
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Stages rows t0 .. t0 + tb - 1 of the chunk (grid tokens in `rows`) of a
// [B, L, H, D] tensor as fp32 into dst [TB][D].
template <int D, typename TIN>
__device__ __forceinline__ void stage_rows(float* dst, const TIN* src, const long long* rows, int t0, int tb, int H,
                                           int h) {
  for (int i = threadIdx.x; i < tb * D; i += 256) {
    const int t = i / D, c = i - t * D;
    dst[i] = ld_in(src + ((size_t)rows[t0 + t] * H + h) * D + c);
  }
}

// The grid tokens of the chunk of unit u = (sequence b * H + h, chunk n) (rows)
// and its gates alpha ([C][DK] into A); returns the number of tokens in the
// chunk.  Begins with a barrier (the caller's shared memory is free after it)
// and ends with one.
template <int C, int DK>
__device__ __forceinline__ int prep_unit(const GlaArgs& a, int u, float* A, long long* rows, int& b, int& h, int& hz,
                                         int& n) {
  const int tid = threadIdx.x;
  const int bh = u / a.nchunks;
  n = u - bh * a.nchunks;
  b = bh / a.H;
  h = bh - b * a.H;
  hz = a.gate_heads == 1 ? 0 : h;
  const int nvalid = min(C, a.L - n * C);
  __syncthreads();
  for (int t = tid; t < C; t += 256)
    rows[t] = t < nvalid ? (long long)b * a.L + scan_to_grid(n * C + t, a.L, a.Hg, a.Wg, a.mode) : 0;
  __syncthreads();
  for (int i = tid; i < C * DK; i += 256) {
    const int t = i / DK, c = i - t * DK;
    A[i] = t < nvalid ? exp2f(log2_decay(__ldg(a.z + ((size_t)rows[t] * a.gate_heads + hz) * DK + c), a.inv_tau))
                      : 1.f;
  }
  __syncthreads();
  return nvalid;
}

// ------------------------------------------------------------------ outputs
// o (and y) of unit u (sequence x chunk) of a flagged chunk.  Needs
// Cfg::SMEM_OUT bytes of shared memory at `smem` (16-byte aligned) and 256 threads.
template <int C, int DK, int DV, typename TIN, typename TOUT>
__device__ __noinline__ void out_unit(const GlaArgs a, int u, uint8_t* smem) {
  using SC = Cfg<C, DK, DV>;
  constexpr int TB = SC::TB, TPJ = SC::TPJ, NCJ = SC::NCJ;
  float* A = reinterpret_cast<float*>(smem);  // alpha [C][DK]
  float* qs = reinterpret_cast<float*>(smem + SC::OFF_Q);
  float* ks = reinterpret_cast<float*>(smem + SC::OFF_K);
  float* vs = reinterpret_cast<float*>(smem + SC::OFF_V);
  float* os = reinterpret_cast<float*>(smem + SC::OFF_D);  // o rows of the block
  long long* rows = reinterpret_cast<long long*>(smem + SC::OFF_ROWS);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool with_y = a.y != nullptr && a.r != nullptr;
  const TIN* q = static_cast<const TIN*>(a.q);
  const TIN* k = static_cast<const TIN*>(a.k);
  const TIN* v = static_cast<const TIN*>(a.v);
  const int j = min(tid / TPJ, DV - 1), part = tid % TPJ;
  const bool act = tid / TPJ < DV;
  int b, h, hz, n;
  const int nvalid = prep_unit<C, DK>(a, u, A, rows, b, h, hz, n);
  const float* S0 = a.dsn + (size_t)u * DV * DK;  // the state entering the chunk, [DV][DK]
  float S[NCJ];
#pragma unroll
  for (int i = 0; i < NCJ; ++i) {
    const int c = part + TPJ * i;
    S[i] = c < DK ? __ldcg(S0 + j * DK + c) : 0.f;
  }
  for (int t0 = 0; t0 < nvalid; t0 += TB) {
    const int tb = min(TB, nvalid - t0);
    __syncthreads();  // the previous block's rows are written out
    stage_rows<DK>(qs, q, rows, t0, tb, a.H, h);
    stage_rows<DK>(ks, k, rows, t0, tb, a.H, h);
    stage_rows<DV>(vs, v, rows, t0, tb, a.H, h);
    __syncthreads();
    for (int t = 0; t < tb; ++t) {
      const float* al = A + (t0 + t) * DK;
      const float vj = vs[t * DV + j];
      float po = 0.f;
#pragma unroll
      for (int i = 0; i < NCJ; ++i) {
        const int c = part + TPJ * i;
        if (c < DK) {
          S[i] = fmaf(al[c], S[i], ks[t * DK + c] * vj);
          po = fmaf(qs[t * DK + c], S[i], po);
        }
      }
      po = group_sum<TPJ>(po);
      if (part == 0 && act) os[t * DV + j] = po;
    }
    __syncthreads();
    for (int t = warp; t < tb; t += 8) {  // one warp per token row
      const size_t row = ((size_t)rows[t0 + t] * a.H + h) * DV;
      float ss = 0.f;
      for (int jj = lane; jj < DV; jj += 32) ss = fmaf(os[t * DV + jj], os[t * DV + jj], ss);
      ss = group_sum<32>(ss);
      const float inv = rsqrtf(ss / (float)DV + a.eps);
      for (int jj = lane; jj < DV; jj += 32) {
        const float ov = os[t * DV + jj];
        st_out(static_cast<TOUT*>(a.o) + row + jj, ov);
        if (with_y) {
          const float rv = ld_in(static_cast<const TIN*>(a.r) + row + jj);
          const float gm = a.gamma != nullptr ? __ldg(a.gamma + jj) : 1.f;
          const float sw = rv / (1.f + expf(-rv));  // Swish(r) = r sigmoid(r)
          st_out(static_cast<TOUT*>(a.y) + row + jj, sw * ov * inv * gm);
        }
      }
    }
  }
}

// ------------------------------------------------------------------ gradients
// dq, dk, dv of unit u (sequence x chunk) of a flagged chunk, and the head's
// share of d log alpha: added to d log alpha when heads share the gate (the
// chunk kernels leave those rows alone, so they hold the other heads' shares
// or zero), stored otherwise.  Needs Cfg::SMEM_GRAD bytes of shared memory at
// `smem` (16-byte aligned) and 256 threads.
template <int C, int DK, int DV, typename TIN, typename TOUT>
__device__ __noinline__ void grad_unit(const GlaArgs a, int u, uint8_t* smem) {
  using SC = Cfg<C, DK, DV>;
  constexpr int TB = SC::TB, TPJ = SC::TPJ, NCJ = SC::NCJ, TPC = SC::TPC, NJC = SC::NJC;
  float* A = reinterpret_cast<float*>(smem);                // alpha [C][DK]
  float* X = reinterpret_cast<float*>(smem + SC::OFF_X);    // d log alpha terms [C][DK]
  float* qs = reinterpret_cast<float*>(smem + SC::OFF_Q);
  float* ks = reinterpret_cast<float*>(smem + SC::OFF_K);
  float* vs = reinterpret_cast<float*>(smem + SC::OFF_V);
  float* ds = reinterpret_cast<float*>(smem + SC::OFF_D);
  long long* rows = reinterpret_cast<long long*>(smem + SC::OFF_ROWS);
  float* bnd = reinterpret_cast<float*>(smem + SC::OFF_BND);  // rowsum(S_{n+1} o G)
  const int tid = threadIdx.x;
  const TIN* q = static_cast<const TIN*>(a.q);
  const TIN* k = static_cast<const TIN*>(a.k);
  const TIN* v = static_cast<const TIN*>(a.v);
  const TIN* dO = static_cast<const TIN*>(a.dO);
  const int c = min(tid / TPC, DK - 1), pc = tid % TPC;  // row sweeps: key channel c
  const bool actc = tid / TPC < DK;
  const int j = min(tid / TPJ, DV - 1), pj = tid % TPJ;  // column sweep: value channel j
  const bool actj = tid / TPJ < DV;
  int b, h, hz, n;
  const int nvalid = prep_unit<C, DK>(a, u, A, rows, b, h, hz, n);
  for (int i = tid; i < C * DK; i += 256) X[i] = 0.f;
  if (tid < DK) bnd[tid] = 0.f;
  const int nblk = (nvalid + TB - 1) / TB;
  const size_t blk = (size_t)u * DV * DK;
  const float* Sn = a.dsn + blk;   // the state entering the chunk (forward scan)
  const float* G = a.dhn + blk;    // the gradient of the state leaving it (reverse scan)
  const float* Sn1 = n + 1 < a.nchunks ? a.dsn + blk + (size_t)DV * DK : nullptr;  // the state leaving it
  auto stage_all = [&](int t0, int tb) {
    __syncthreads();  // the previous block is consumed (and X, bnd cleared)
    stage_rows<DK>(qs, q, rows, t0, tb, a.H, h);
    stage_rows<DK>(ks, k, rows, t0, tb, a.H, h);
    stage_rows<DV>(vs, v, rows, t0, tb, a.H, h);
    stage_rows<DV>(ds, dO, rows, t0, tb, a.H, h);
    __syncthreads();
  };
  // -- forward sweep (rows): dq_t = S_t dO_t
  {
    float S[NJC];
#pragma unroll
    for (int i = 0; i < NJC; ++i) {
      const int jj = pc + TPC * i;
      S[i] = jj < DV ? __ldcg(Sn + jj * DK + c) : 0.f;
    }
    for (int bi = 0; bi < nblk; ++bi) {
      const int t0 = bi * TB, tb = min(TB, nvalid - t0);
      stage_all(t0, tb);
      for (int t = 0; t < tb; ++t) {
        const float al = A[(t0 + t) * DK + c], kc = ks[t * DK + c];
        float pd = 0.f;
#pragma unroll
        for (int i = 0; i < NJC; ++i) {
          const int jj = pc + TPC * i;
          if (jj < DV) {
            S[i] = fmaf(al, S[i], kc * vs[t * DV + jj]);
            pd = fmaf(S[i], ds[t * DV + jj], pd);
          }
        }
        pd = group_sum<TPC>(pd);
        if (pc == 0 && actc) {
          st_out(static_cast<TOUT*>(a.dq) + ((size_t)rows[t0 + t] * a.H + h) * DK + c, pd);
          X[(t0 + t) * DK + c] += qs[t * DK + c] * pd;
        }
      }
    }
  }
  // -- reverse sweep (rows): dk_t = R_t v_t; the boundary term rowsum(S_{n+1} o G)
  {
    float R[NJC];
    float pb = 0.f;
#pragma unroll
    for (int i = 0; i < NJC; ++i) {
      const int jj = pc + TPC * i;
      R[i] = jj < DV ? __ldcg(G + jj * DK + c) : 0.f;
      if (Sn1 != nullptr && jj < DV) pb = fmaf(R[i], __ldcg(Sn1 + jj * DK + c), pb);
    }
    pb = group_sum<TPC>(pb);
    if (pc == 0 && actc) bnd[c] = pb;
    for (int bi = nblk - 1; bi >= 0; --bi) {
      const int t0 = bi * TB, tb = min(TB, nvalid - t0);
      stage_all(t0, tb);
      for (int t = tb - 1; t >= 0; --t) {
        const float qc = qs[t * DK + c], al = A[(t0 + t) * DK + c];
        float pk = 0.f;
#pragma unroll
        for (int i = 0; i < NJC; ++i) {
          const int jj = pc + TPC * i;
          if (jj < DV) {
            R[i] = fmaf(qc, ds[t * DV + jj], R[i]);
            pk = fmaf(R[i], vs[t * DV + jj], pk);
            R[i] *= al;
          }
        }
        pk = group_sum<TPC>(pk);
        if (pc == 0 && actc) {
          st_out(static_cast<TOUT*>(a.dk) + ((size_t)rows[t0 + t] * a.H + h) * DK + c, pk);
          X[(t0 + t) * DK + c] -= ks[t * DK + c] * pk;
        }
      }
    }
  }
  // -- reverse sweep (columns): dv_t = R_t^T k_t
  {
    float R[NCJ];
#pragma unroll
    for (int i = 0; i < NCJ; ++i) {
      const int cc = pj + TPJ * i;
      R[i] = cc < DK ? __ldcg(G + j * DK + cc) : 0.f;
    }
    for (int bi = nblk - 1; bi >= 0; --bi) {
      const int t0 = bi * TB, tb = min(TB, nvalid - t0);
      stage_all(t0, tb);
      for (int t = tb - 1; t >= 0; --t) {
        const float* al = A + (t0 + t) * DK;
        const float dj = ds[t * DV + j];
        float pv = 0.f;
#pragma unroll
        for (int i = 0; i < NCJ; ++i) {
          const int cc = pj + TPJ * i;
          if (cc < DK) {
            R[i] = fmaf(qs[t * DK + cc], dj, R[i]);
            pv = fmaf(R[i], ks[t * DK + cc], pv);
            R[i] *= al[cc];
          }
        }
        pv = group_sum<TPJ>(pv);
        if (pj == 0 && actj) st_out(static_cast<TOUT*>(a.dv) + ((size_t)rows[t0 + t] * a.H + h) * DV + j, pv);
      }
    }
  }
  __syncthreads();  // the terms are in X and bnd
  if (tid < DK) {   // d log alpha: reverse cumsum over the chunk + the boundary term
    float acc = 0.f;
    for (int t = nvalid - 1; t >= 0; --t) {
      acc += X[t * DK + tid];
      float* dst = a.dla + ((size_t)rows[t] * a.gate_heads + hz) * DK + tid;
      if (a.gate_heads == 1) atomicAdd(dst, acc + bnd[tid]);
      else *dst = acc + bnd[tid];
    }
  }
}

// ------------------------------------------------------------------ scan
// Four state elements (key channels c0 .. c0 + 3, value channel j; dk % 4 == 0)
// of a flagged chunk's contribution to the scan of sequence bh: dS (dh false,
// the forward scan) or dH (dh true, the reverse scan), summed token by token.
static __device__ __noinline__ float4 state_quad(const GlaArgs& a, bool dh, int bh, int n, int c0, int j, int dk, int dv) {
  const int b = bh / a.H, h = bh - b * a.H;
  const int hz = a.gate_heads == 1 ? 0 : h;
  const int nvalid = min(a.chunk, a.L - n * a.chunk);
  const void* kin = dh ? a.q : a.k;
  const void* vin = dh ? a.dO : a.v;
  float acc[4] = {0.f, 0.f, 0.f, 0.f}, e[4] = {0.f, 0.f, 0.f, 0.f};  // running log2 decays
  for (int s = 0; s < nvalid; ++s) {
    const int t = dh ? s : nvalid - 1 - s;  // dH: inclusive prefix decays; dS: exclusive suffix decays
    const long long gr = (long long)b * a.L + scan_to_grid(n * a.chunk + t, a.L, a.Hg, a.Wg, a.mode);
    const size_t kr = ((size_t)gr * a.H + h) * dk + c0, vr = ((size_t)gr * a.H + h) * dv + j;
    float kv[4], vj;
    if (a.in_bf16) {
      const __nv_bfloat16* kp = static_cast<const __nv_bfloat16*>(kin) + kr;
      for (int i = 0; i < 4; ++i) kv[i] = __bfloat162float(kp[i]);
      vj = __bfloat162float(static_cast<const __nv_bfloat16*>(vin)[vr]);
    } else {
      const float4 k4 = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(kin) + kr));
      kv[0] = k4.x; kv[1] = k4.y; kv[2] = k4.z; kv[3] = k4.w;
      vj = __ldg(static_cast<const float*>(vin) + vr);
    }
    const float4 z4 = __ldg(reinterpret_cast<const float4*>(a.z + ((size_t)gr * a.gate_heads + hz) * dk + c0));
    const float l[4] = {log2_decay(z4.x, a.inv_tau), log2_decay(z4.y, a.inv_tau), log2_decay(z4.z, a.inv_tau),
                        log2_decay(z4.w, a.inv_tau)};
    for (int i = 0; i < 4; ++i) {
      if (dh) e[i] += l[i];
      acc[i] = fmaf(exp2f(e[i]) * kv[i], vj, acc[i]);
      if (!dh) e[i] += l[i];
    }
  }
  return make_float4(acc[0], acc[1], acc[2], acc[3]);
}

}  // namespace strong
}  // namespace dig
