// gla_state_tma.cu -- per-chunk state contributions with tile copies by the
// tensor memory accelerator and two units in flight per CTA.
//
// Two reductions over a chunk's tokens (DiG slides, GLA eq. (6)-(7) and the
// chain rule of eq. (8)):
//   forward:   dS_n = V^T khat,            khat = k 2^(Gamma - b) = k 2^(Gamma - r) / EQ
//   backward:  dH_n = dO^T (q 2^b),        q 2^b = q EQ 2^r
// (EQ = 2^(b - r) from the gate kernel, r the chunk's reference, Gamma its total
// decay), each a [d_v][d_k] fp32 block per (sequence, chunk), the input of the
// state scans.  The same arithmetic as gla_chunk_state_kernel /
// gla_chunk_dh_kernel (the gated operand as two bf16 terms, the raw v / dO as
// one); what differs is the data path: k (or q), v (or dO) and the gate factors
// arrive as whole tiles by TMA into one of two stages, so the next unit's tiles
// land while this unit is converted and multiplied, and the block leaves by a
// TMA tile store.  Only bf16 inputs with d_k = 32, d_v = 64, 128-token chunks
// that tile the sequence and the row scan orders take this kernel (the kernel
// itself also reads the column orders' tiles as 16-row segments).
#include "tma_tiles.cuh"

namespace dig {

struct ReduceMaps {
  CUtensorMap x;    // k (forward) or q (backward), bf16
  CUtensorMap y;    // v (forward) or dO (backward), bf16
  CUtensorMap eq;   // gate factors [B * gate_heads * L][d_k] fp32 (scan order)
  CUtensorMap out;  // [units * d_v][d_k] fp32 blocks
};

struct TmaReduceCfg {
  static constexpr int C = 128, DK = 32, DV = 64;
  static constexpr int RBX = 64, RBY = 128;
  // one stage: x tile (hi term in place), its lo term, y tile, gate factors
  static constexpr int S_XH = 0, S_XL = 8192, S_Y = 16384, S_EQ = 32768, STAGE = 49152;
  static constexpr int OFF_OUT = 2 * STAGE;         // [d_v][d_k] fp32, 128-byte swizzle
  static constexpr int END = OFF_OUT + DV * DK * 4;  // 106496
  static constexpr int SMEM = END + 1024;
  static constexpr int TM_COLS = 128;                // per stage: the hi and lo terms' products, 32 columns each
  static constexpr uint32_t IN_BYTES = C * RBX + C * RBY + C * DK * 4, GCH_BYTES = 2 * DK * 4;
};

struct TmaReduceSmem {
  alignas(16) float gch[2][64];  // per stage: 2^r (d_k values), then 2^(Gamma - r)
  uint64_t full[2];              // a stage's tiles have landed
  uint64_t mma[2];               // a stage's product is complete
  uint32_t tmem;
  int abort;
};

template <bool BWD>
__global__ void __launch_bounds__(256, 2) gla_reduce_tma_kernel(const __grid_constant__ ReduceMaps mp,
                                                                const GlaArgs a) {
  using TC = TmaReduceCfg;
  constexpr int C = TC::C, DK = TC::DK, DV = TC::DV;
  extern __shared__ uint8_t smem_raw[];
  __shared__ TmaReduceSmem sh;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t sb = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int nunits = a.B * a.H * a.nchunks;
  const uint64_t spin = a.spin_ns ? a.spin_ns : kSpinLimitNs;
  if (warp == 0) {
    tmem_alloc(&sh.tmem, TC::TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.mma[i], 1);
    }
    sh.abort = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem;
  bool timed_out = false;
  auto wait_bar = [&](uint64_t* bar, uint32_t parity) {
    if (!mbar_wait(bar, parity, spin)) {
      timed_out = true;
      sh.abort = 1;
    }
  };
  // thread 0's record of work in flight, drained before exit: bit s of `pend`
  // (copies into stage s) and of `pend >> 2` (stage s's product), with their
  // phases in the same bits of `pph`
  uint32_t pend = 0, pph = 0;
  bool stored = false;
  auto mark = [&](int bit, uint32_t phase) {
    pend |= 1u << bit;
    pph = (pph & ~(1u << bit)) | (phase << bit);
  };

  auto issue = [&](int u, int s, uint32_t phase) {
    const TileUnit T(a, u, C);
    mark(s, phase);
    const uint32_t st = sb + s * TC::STAGE;
    mbar_arrive_expect_tx(&sh.full[s], TC::IN_BYTES + TC::GCH_BYTES);
    tile_load<C>(st + TC::S_XH, mp.x, T.h * DK, T, a, TC::RBX, &sh.full[s]);
    tile_load<C>(st + TC::S_Y, mp.y, T.h * DV, T, a, TC::RBY, &sh.full[s]);
    tma_load_2d(st + TC::S_EQ, mp.eq, 0, T.bz * a.L + T.n * C, &sh.full[s]);
    bulk_copy_g2s(smem_u32(sh.gch[s]), a.gCH + ((size_t)T.bz * a.nchunks + T.n) * 4 * DK, TC::GCH_BYTES,
                  &sh.full[s]);
  };

  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  if (tid == 0) {
    if ((int)blockIdx.x < nunits) issue(blockIdx.x, 0, 0);
    if ((int)(blockIdx.x + gridDim.x) < nunits) issue(blockIdx.x + gridDim.x, 1, 0);
  }

  int it = 0;
  for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++it) {
    const int s = it & 1;
    const uint32_t ph = (it >> 1) & 1;
    const uint32_t st = sb + s * TC::STAGE;
    const TileUnit T(a, u, C);
    wait_bar(&sh.full[s], ph);
    if (tid == 0 && !timed_out) pend &= ~(1u << s);
    // ---- the gated operand as two bf16 terms, in place: forward khat = k 2^(Gamma - r) / EQ,
    //      backward q 2^b = q EQ 2^r
    const float* gc = sh.gch[s] + (BWD ? 0 : DK);
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int k = tid + 256 * m;  // 16-byte chunk of the x tile
      const int i = k >> 2, c = (k & 3) ^ ((i >> 1) & 3);
      const int ti = T.rev ? C - 1 - i : i;
      const float4 e0 = lds128f(st + TC::S_EQ + swz_off<128>(ti, 2 * c));
      const float4 e1 = lds128f(st + TC::S_EQ + swz_off<128>(ti, 2 * c + 1));
      const float4 g0 = *reinterpret_cast<const float4*>(gc + 8 * c);
      const float4 g1 = *reinterpret_cast<const float4*>(gc + 8 * c + 4);
      const float e[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
      const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      const uint4 xr = lds128(st + TC::S_XH + 16u * k);
      const uint32_t xw[4] = {xr.x, xr.y, xr.z, xr.w};
      float xv[8];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float f0 = BWD ? e[2 * w] * g[2 * w] : __fdividef(g[2 * w], e[2 * w]);
        const float f1 = BWD ? e[2 * w + 1] * g[2 * w + 1] : __fdividef(g[2 * w + 1], e[2 * w + 1]);
        xv[2 * w] = bf_lo(xw[w]) * f0;
        xv[2 * w + 1] = bf_hi(xw[w]) * f1;
      }
      uint32_t h[4], l[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const __nv_bfloat162 hi = __floats2bfloat162_rn(xv[2 * w], xv[2 * w + 1]);
        const __nv_bfloat162 lo = __floats2bfloat162_rn(xv[2 * w] - __low2float(hi), xv[2 * w + 1] - __high2float(hi));
        h[w] = *reinterpret_cast<const uint32_t*>(&hi);
        l[w] = *reinterpret_cast<const uint32_t*>(&lo);
      }
      sts128(st + TC::S_XH + 16u * k, make_uint4(h[0], h[1], h[2], h[3]));
      sts128(st + TC::S_XL + 16u * k, make_uint4(l[0], l[1], l[2], l[3]));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- D[j][c'] = sum_t Y[t][j] X'[t][c']: A = the y tile read MN-major (M = value
    //      channels, 64 of 128 rows used), B = the hi and lo terms side by side (N = 2 d_k:
    //      two 32-channel MN atoms 8 KB apart), K = tokens; the two halves are added on
    //      the way out.  One N = 64 product per K-step instead of two N = 32 ones: the
    //      tensor core takes about as long per instruction at either width.
    if (tid == 0 && !timed_out && !sh.abort) {
      const uint32_t dtm = tmem + 64u * s;
      uint64_t bdesc = sdesc_sw<64>(st + TC::S_XH);
      bdesc &= ~(static_cast<uint64_t>(0x3FFF) << 16);  // leading byte offset: the lo term's atom
      bdesc |= static_cast<uint64_t>(((TC::S_XL - TC::S_XH) >> 4) & 0x3FFF) << 16;
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks)
        mma_bf16(dtm, sdesc_sw<128>(st + TC::S_Y + 2048 * ks), bdesc + (uint64_t)((1024 * ks) >> 4),
                 idesc_bf16(128, 2 * DK, true, true), ks ? 1u : 0u);
      mma_commit(&sh.mma[s]);
      mark(2 + s, ph);
    }
    wait_bar(&sh.mma[s], ph);
    tc_fence_after();
    if (tid == 0 && !timed_out) pend &= ~(4u << s);
    // the stage's tiles are consumed: the unit two ahead lands there
    if (tid == 0 && !timed_out && !sh.abort && u + 2 * (int)gridDim.x < nunits) issue(u + 2 * gridDim.x, s, ph ^ 1u);
    // ---- the block: TMEM lane j (value channel j < d_v) -> staging row j -> one tile store
    if (tid == 0 && stored) bulk_wait_read_all();  // the previous block has left the staging
    __syncthreads();
    if (warp < 2) {  // lanes 0 .. 63
      float d[32], dl[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 64u * s, d);
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 64u * s + 32u, dl);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) d[i] += dl[i];
      const int j = tid;
#pragma unroll
      for (int m = 0; m < 8; ++m)
        sts128(sb + TC::OFF_OUT + swz_off<128>(j, m),
               make_uint4(__float_as_uint(d[4 * m]), __float_as_uint(d[4 * m + 1]), __float_as_uint(d[4 * m + 2]),
                          __float_as_uint(d[4 * m + 3])));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && !timed_out && !sh.abort) {
      tma_store_2d(mp.out, 0, u * DV, sb + TC::OFF_OUT);
      bulk_commit();
      stored = true;
    }
    if (sh.abort) break;
  }

  // ---- drain: no copy, store or product outlives the CTA
  if (timed_out) set_status(a.status, DIG_ERR_DEVICE_TIMEOUT);
  if (tid == 0) {
    bulk_wait_all();
    for (int s = 0; s < 2; ++s) {
      if (pend >> s & 1u) mbar_wait(&sh.full[s], pph >> s & 1u, kSpinLimitNs);
      if (pend >> (2 + s) & 1u) mbar_wait(&sh.mma[s], pph >> (2 + s) & 1u, kSpinLimitNs);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TC::TM_COLS);
}

// ------------------------------------------------------------------ launch
// The row scan orders only: in the column orders the tile arrives as eight 16-row
// segment copies per tensor, and the row-piece kernels were faster there (same box,
// DiG-S/2 1792^2: forward 82 vs 85 us, backward 111.6 vs 112.6 us), while this kernel
// wins in the row orders (forward 73.5 vs 76.7 us, backward 98.3 vs 100.3 us).
bool gla_reduce_tma_eligible(const GlaArgs& a, int dk, int dv, int tin, int chunk) {
  if (tin != DIG_BF16 || dk != 32 || dv != 64 || chunk != 128 || a.L % 128 != 0) return false;
  if (a.mode & 2) return false;
  return tmap_available();
}

// The forward's dS blocks (bwd = false: from k and v into a.dsn) or the
// backward's dH blocks (bwd = true: from q and dO into a.dhn).
cudaError_t launch_reduce_tma(const GlaArgs& a, bool bwd, cudaStream_t s, bool* launched) {
  *launched = false;
  constexpr int C = 128, DK = 32, DV = 64;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, fp = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  ReduceMaps mp;
  memset(&mp, 0, sizeof(mp));
  const long long units = (long long)a.B * a.H * a.nchunks;
  if (units * DV > 2147483647LL) return cudaSuccess;  // block rows beyond a tensor-map coordinate
  bool ok = encode_tile_map(&mp.x, bwd ? a.q : a.k, bf, 2, a.H * DK, DK, 64, a, C) &&
            encode_tile_map(&mp.y, bwd ? a.dO : a.v, bf, 2, a.H * DV, DV, 128, a, C) &&
            tmap_rows(&mp.eq, a.gEQ, fp, 4, DK, (uint64_t)a.B * a.gate_heads * a.L, DK, C, 128) &&
            tmap_rows(&mp.out, bwd ? a.dhn : a.dsn, fp, 4, DK, (uint64_t)units * DV, DK, DV, 128);
  if (!ok) return cudaSuccess;
  cudaError_t e;
  auto k = bwd ? gla_reduce_tma_kernel<true> : gla_reduce_tma_kernel<false>;
  if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, TmaReduceCfg::SMEM)) != cudaSuccess)
    return e;
  e = launch_pdl(k, persistent_grid(2, units), 256, TmaReduceCfg::SMEM, s, mp, a);
  if (e == cudaSuccess) *launched = true;
  return e;
}

}  // namespace dig
