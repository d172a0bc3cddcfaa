// gla.h -- host/device parameter blocks and launcher declarations of the GLA
// kernels (internal to libdig.so).
#pragma once
#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace dig {

struct GlaArgs {
  // inputs (grid order)
  const void* q;
  const void* k;
  const void* v;
  const float* z;
  const void* dO;      // backward only
  const void* r;       // forward epilogue (optional)
  const float* gamma;  // forward epilogue (optional)
  // outputs
  void* o;
  void* y;
  void* dq;
  void* dk;
  void* dv;
  float* dla;
  // shape
  int B, H, L, Hg, Wg, mode, gate_heads;
  float inv_tau, eps;
  int nchunks;  // chunks per sequence
  // workspace
  uint32_t* status;  // device status word (DIG_OK or the first condition found)
  float* gEQ;        // [B * gate_heads][L (scan order)][DK]   2^(b - r)
  float* gCH;        // [B * gate_heads][nchunks][4][DK]       2^r, 2^(Gamma-r), 2^Gamma, Gamma
  float* dsn;        // [nseq][nchunks][DV][DK]  chunk state contribution, then the state entering the chunk
  float* dhn;        // backward: [nseq][nchunks][DV][DK] chunk state-gradient contribution, then the
                     // gradient of the state leaving the chunk
  uint32_t* flist;   // backward: [0] count, [1..] units the fp16 gradient kernel left to the exact one
                     // (the exact kernel then processes only those; NULL: every unit)
  unsigned long long spin_ns;  // bound of a device wait in ns (0: the default of two seconds)
  // value gate and state input / output (the extended entry points; all NULL otherwise)
  const float* zb;   // value-gate logits [B, L, gate_heads, DV] (grid order)
  float* gEQb;       // [B * gate_heads][L (scan order)][DV]   2^(e - rho), e the value-gate cumsum
  float* gCHb;       // [B * gate_heads][nchunks][4][DV]       2^rho, 2^(Gb - rho), 2^Gb, Gb
  float* sfin;       // [nseq][DV][DK] the state after the last chunk (written by the forward scan)
  // chunks whose key gate decays too fast for the chunk factorisation
  int* sflag;        // [B * gate_heads][nchunks] 1 where such a chunk was found (written by the gate
                     // kernel; those chunks are recomputed exactly, gla_strong.cuh); NULL: such a
                     // chunk sets DIG_ERR_GATE_RANGE instead
  int chunk;         // tokens per chunk of this call
  int in_bf16;       // q, k, v, dO are bf16 (else fp32)
};

// Kernel-variant selection: chunk length, split count, head dims, types.
struct GlaVariant {
  int chunk;      // tokens per chunk
  int split;      // bf16 terms of a gated operand (2 for bf16 inputs, 3 for fp32)
  int dk, dv;
  int tin, tout;  // DIG_F32 / DIG_BF16
};

// Workspace layout (bytes from the workspace start): a 256-byte header holding
// the status word, the gate factors, the per-chunk states and, for the
// backward, the per-chunk state gradients.
struct WsLayout {
  size_t gEQ, gCH, dsn, dhn, flist, sflag, total;
};
WsLayout ws_layout(int B, int H, int gate_heads, int L, int nchunks, int dk, int dv, bool backward);

// Launch helpers; return cudaSuccess or the launch error.  The forward enqueues
// its four kernels (gate factors, chunk states, state scan, outputs); the
// backward its four (gate factors, chunk states and state gradients, the
// forward and reverse scans, gradients), or with `saved` (gEQ, gCH and dsn from
// the forward) only the state gradients, their reverse scan and the gradients.
cudaError_t launch_gla_fwd(const GlaVariant& var, const GlaArgs& a, cudaStream_t s);
cudaError_t launch_gla_bwd(const GlaVariant& var, const GlaArgs& a, bool saved, cudaStream_t s);
bool gla_variant_built(int dk, int dv);
int gla_bwd_chunk(int dk, int dv, int dtype);  // tokens per chunk of the backward

cudaError_t launch_srem(const void* x, const float* w, const float* bias, void* y, int B, int Hg, int Wg, int C,
                        int mode, int tin, int tout, cudaStream_t s);

}  // namespace dig
