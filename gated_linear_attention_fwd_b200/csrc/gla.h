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
  // decomposition
  int nchunks;  // chunks per sequence
  int nseg;     // segments (CTAs) per sequence
  // workspace
  uint32_t* status;
  uint32_t* done;
  uint32_t* flags;   // [nseq * nseg]         forward segment records ready
  uint32_t* flags2;  // [nseq * nseg]         backward segment records ready
  float* seg_gam;    // [nseq * nseg][DKP]    summed log decay of the segment
  float* seg_S;      // [nseq * nseg][DV][DK] segment state (forward scan record)
  float* seg_H;      // [nseq * nseg][DV][DK] segment state gradient (backward scan record)
  float* chunk_S;    // [nseq * nchunks][DV][DK] in-segment state entering each chunk (backward)
  float* chunk_B;    // [nseq * nchunks][DKP] in-segment log decay before each chunk (backward)
  // forward: gate factors shared by the heads, and the chunk states
  float* gEQ;        // [B * gate_heads][L (scan order)][DK]   2^(b - r)
  float* gCH;        // [B * gate_heads][nchunks][4][DK]       2^r, 2^(Gamma-r), 2^Gamma, Gamma
  float* dsn;        // [nseq][nchunks][DV][DK]  chunk state contribution, then the state entering the chunk
};

// Kernel-variant selection: chunk length, split count, head dims, types.
struct GlaVariant {
  int chunk;   // tokens per chunk
  int split;   // 1: tf32 operands, 2: hi+lo tf32 (three products)
  int dk, dv;
  int tin, tout;  // DIG_F32 / DIG_BF16
};

// Workspace layout for a given decomposition (bytes from the workspace start).
struct WsLayout {
  size_t flags, flags2, seg_gam, seg_S, seg_H, chunk_S, chunk_B, gEQ, gCH, dsn, total;
};
// Forward (backward = false): gate factors and chunk states.  Backward: the
// segment records of its two sweeps.
WsLayout ws_layout(int B, int H, int gate_heads, int L, int nseg, int nchunks, int dk, int dv, bool backward);

// Launch helpers; return cudaSuccess or the launch error.  The forward enqueues
// its three kernels (chunk states, state scan, outputs).  For the backward,
// `coop` requests a cooperative launch (all CTAs co-resident; needed when
// nseg > 1).
cudaError_t launch_gla_fwd(const GlaVariant& var, const GlaArgs& a, cudaStream_t s);
cudaError_t launch_gla_bwd(const GlaVariant& var, const GlaArgs& a, int grid, bool coop, cudaStream_t s);
// Resident CTAs per SM of the backward kernel (0 if the variant is not built).
int gla_bwd_blocks_per_sm(const GlaVariant& var);
bool gla_variant_built(int dk, int dv);

cudaError_t launch_srem(const void* x, const float* w, const float* bias, void* y, int B, int Hg, int Wg, int C,
                        int mode, int tin, int tout, cudaStream_t s);

}  // namespace dig
