// dig_ext_api.cu -- the extended GLA entry points of the C ABI (include/dig.h):
// value gate beta and state input / output (DiG slides, "Gated Linear Attention
// Transformer (GLA) の導入", eq. (5): G_t = alpha_t^T beta_t, S_t = G_t (*)
// S_{t-1} + k_t^T v_t, o_t = q_t S_t, from a given S_0 and returning S_L).
// These run the fp32 exact kernels (64-token chunks) in their value-gate form;
// bf16 inputs are widened to fp32 in the workspace first (exactly).
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "../../include/dig.h"
#include "dig_common.cuh"
#include "gla.h"
#include "gla_chunk.cuh"

namespace dig {

void set_last_error(const char* msg);  // dig_api.cu
unsigned long long spin_limit_ns();    // dig_api.cu
dig_status check_common(int B, int H, int L, int d_k, int d_v, int grid_h, int grid_w, int scan_mode, int dtype,
                        int out_dtype, int gate_heads);  // dig_api.cu
cudaError_t launch_gla_fwd_ext(const GlaVariant& v, const GlaArgs& a, const ScanEnds& ends, cudaStream_t s);
cudaError_t launch_gla_bwd_ext(const GlaVariant& v, const GlaArgs& a, const ScanEnds& ends, cudaStream_t s);
cudaError_t launch_widen_bf16(const void* src, float* dst, long long n, cudaStream_t s);
cudaError_t launch_dlogbeta(const GlaArgs& a, int dk, int dv, int tout, const void* o, float* dlb, cudaStream_t s);

namespace {

constexpr int kExtChunk = 64;

dig_status efail(dig_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  set_last_error(buf);
  return st;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// The standard layout of the pass (64-token chunks), then the value gate's
// factors, the final state in the state layout, and fp32 copies of the bf16
// inputs.
struct ExtLayout {
  WsLayout base;
  size_t gEQb, gCHb, sfin, q32, k32, v32, x32, total;  // x32: r (forward) or dO (backward)
};

ExtLayout ext_layout(int B, int H, int gate_heads, int L, int dk, int dv, int dtype, bool backward) {
  const int nchunks = (L + kExtChunk - 1) / kExtChunk;
  ExtLayout e{};
  e.base = ws_layout(B, H, gate_heads, L, nchunks, dk, dv, backward);
  size_t off = e.base.total;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = up256(off + bytes);
    return at;
  };
  const size_t nbz = (size_t)B * gate_heads, nseq = (size_t)B * H, tok = (size_t)B * L * H;
  e.gEQb = take(nbz * (size_t)L * dv * 4);
  e.gCHb = take(nbz * (size_t)nchunks * 4 * dv * 4);
  e.sfin = take(nseq * (size_t)dk * dv * 4);
  const bool widen = dtype == DIG_BF16;
  e.q32 = take(widen ? tok * dk * 4 : 0);
  e.k32 = take(widen ? tok * dk * 4 : 0);
  e.v32 = take(widen ? tok * dv * 4 : 0);
  e.x32 = take(widen ? tok * dv * 4 : 0);
  e.total = off;
  return e;
}

// Common checks and the argument block (inputs widened when bf16).
dig_status ext_setup(const void* q, const void* k, const void* v, const float* z, const float* zb, int gate_heads,
                     float inv_tau, const void* x /* r or dO */, int B, int H, int L, int d_k, int d_v, int grid_h,
                     int grid_w, int scan_mode, int dtype, int out_dtype, void* workspace, size_t workspace_bytes,
                     bool backward, cudaStream_t s, GlaArgs* a, bool* empty) {
  *empty = false;
  dig_status st = check_common(B, H, L, d_k, d_v, grid_h, grid_w, scan_mode, dtype, out_dtype, gate_heads);
  if (st != DIG_OK) return st;
  if (d_v != 64 && d_v != 72) return efail(DIG_ERR_UNSUPPORTED, "the value gate is built for d_v = 64 or 72");
  if (!workspace) return efail(DIG_ERR_INVALID_ARGUMENT, "workspace is NULL");
  if (!al16(workspace)) return efail(DIG_ERR_MISALIGNED, "workspace not 16-byte aligned");
  if (B == 0 || L == 0) {
    *empty = true;
    return DIG_OK;
  }
  if (!q || !k || !v || !z) return efail(DIG_ERR_INVALID_ARGUMENT, "q, k, v and z must be non-NULL");
  if (!al16(q) || !al16(k) || !al16(v) || !al16(z) || !al16(zb) || !al16(x))
    return efail(DIG_ERR_MISALIGNED, "a tensor pointer is not 16-byte aligned");
  const ExtLayout lay = ext_layout(B, H, gate_heads, L, d_k, d_v, dtype, backward);
  if (workspace_bytes < lay.total)
    return efail(DIG_ERR_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, needs %zu", workspace_bytes, lay.total);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  *a = GlaArgs{};
  a->q = q; a->k = k; a->v = v; a->z = z; a->zb = zb;
  a->B = B; a->H = H; a->L = L; a->Hg = grid_h; a->Wg = grid_w; a->mode = scan_mode; a->gate_heads = gate_heads;
  a->inv_tau = inv_tau;
  a->nchunks = (L + kExtChunk - 1) / kExtChunk;
  a->chunk = kExtChunk;
  a->in_bf16 = 0;  // the kernels read fp32 copies of bf16 inputs
  a->status = reinterpret_cast<uint32_t*>(ws);
  a->gEQ = reinterpret_cast<float*>(ws + lay.base.gEQ);
  a->gCH = reinterpret_cast<float*>(ws + lay.base.gCH);
  a->dsn = reinterpret_cast<float*>(ws + lay.base.dsn);
  a->dhn = backward ? reinterpret_cast<float*>(ws + lay.base.dhn) : nullptr;
  a->gEQb = reinterpret_cast<float*>(ws + lay.gEQb);
  a->gCHb = reinterpret_cast<float*>(ws + lay.gCHb);
  a->sfin = reinterpret_cast<float*>(ws + lay.sfin);
  a->spin_ns = spin_limit_ns();
  if (dtype == DIG_BF16) {  // the fp32 kernels read exact fp32 copies
    const long long tok = (long long)B * L * H;
    float* q32 = reinterpret_cast<float*>(ws + lay.q32);
    float* k32 = reinterpret_cast<float*>(ws + lay.k32);
    float* v32 = reinterpret_cast<float*>(ws + lay.v32);
    float* x32 = reinterpret_cast<float*>(ws + lay.x32);
    cudaError_t e = launch_widen_bf16(q, q32, tok * d_k, s);
    if (e == cudaSuccess) e = launch_widen_bf16(k, k32, tok * d_k, s);
    if (e == cudaSuccess) e = launch_widen_bf16(v, v32, tok * d_v, s);
    if (e == cudaSuccess && x) e = launch_widen_bf16(x, x32, tok * d_v, s);
    if (e != cudaSuccess) return efail(DIG_ERR_CUDA, "input widening: %s", cudaGetErrorString(e));
    a->q = q32; a->k = k32; a->v = v32;
    if (x) {
      if (backward) a->dO = x32;
      else a->r = x32;
    }
  } else if (x) {
    if (backward) a->dO = x;
    else a->r = x;
  }
  return DIG_OK;
}

}  // namespace
}  // namespace dig

using namespace dig;

extern "C" {

size_t dig_gla_ext_workspace_bytes(int B, int H, int gate_heads, int L, int d_k, int d_v, int dtype, int pass) {
  if (B < 0 || H <= 0 || L < 0 || (pass != 0 && pass != 1) || (dtype != DIG_F32 && dtype != DIG_BF16)) return 0;
  if (gate_heads != 1 && gate_heads != H) return 0;
  if (!gla_variant_built(d_k, d_v) || (d_v != 64 && d_v != 72)) return 0;
  return ext_layout(B > 0 ? B : 1, H, gate_heads, L, d_k, d_v, dtype, pass == 1).total;
}

dig_status dig_gla_fwd_ext(const void* q, const void* k, const void* v, const float* z, const float* zb,
                           int gate_heads, float inv_tau, const float* S0, void* o, const void* r,
                           const float* gamma, float eps, void* y, float* S_final, int B, int H, int L, int d_k,
                           int d_v, int grid_h, int grid_w, int scan_mode, int dtype, int out_dtype, void* workspace,
                           size_t workspace_bytes, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!al16(S0) || !al16(o) || !al16(gamma) || !al16(y) || !al16(S_final))
    return efail(DIG_ERR_MISALIGNED, "a tensor pointer is not 16-byte aligned");
  if (B > 0 && L > 0 && !o) return efail(DIG_ERR_INVALID_ARGUMENT, "o must be non-NULL");
  GlaArgs a;
  bool empty = false;
  const bool with_y = r != nullptr && y != nullptr;
  dig_status st = ext_setup(q, k, v, z, zb, gate_heads, inv_tau, with_y ? r : nullptr, B, H, L, d_k, d_v, grid_h,
                            grid_w, scan_mode, dtype, out_dtype, workspace, workspace_bytes, false, s, &a, &empty);
  if (st != DIG_OK) return st;
  if (empty) {  // an empty sequence leaves the state as it was
    if (S_final && B > 0) {
      const size_t bytes = (size_t)B * H * d_k * d_v * sizeof(float);
      const cudaError_t e = S0 ? cudaMemcpyAsync(S_final, S0, bytes, cudaMemcpyDeviceToDevice, s)
                               : cudaMemsetAsync(S_final, 0, bytes, s);
      if (e != cudaSuccess) return efail(DIG_ERR_CUDA, "final state: %s", cudaGetErrorString(e));
    }
    return DIG_OK;
  }
  a.o = o;
  a.y = with_y ? y : nullptr;
  if (!with_y) a.r = nullptr;
  a.gamma = gamma;
  a.eps = eps;
  ScanEnds ends{};
  ends.seed[0] = S0;
  ends.fin[0] = S_final;
  ends.fin_rows[0] = a.sfin;
  GlaVariant var{kExtChunk, 3, d_k, d_v, DIG_F32, out_dtype};
  const cudaError_t e = launch_gla_fwd_ext(var, a, ends, s);
  if (e != cudaSuccess) return efail(DIG_ERR_CUDA, "gla_fwd_ext launch: %s", cudaGetErrorString(e));
  return DIG_OK;
}

dig_status dig_gla_bwd_ext(const void* q, const void* k, const void* v, const float* z, const float* zb,
                           int gate_heads, float inv_tau, const float* S0, const void* o, const void* dO,
                           const float* dS_final, void* dq, void* dk, void* dv, float* dlog_alpha, float* dlog_beta,
                           float* dS0, int B, int H, int L, int d_k, int d_v, int grid_h, int grid_w, int scan_mode,
                           int dtype, int out_dtype, void* workspace, size_t workspace_bytes, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!al16(S0) || !al16(o) || !al16(dS_final) || !al16(dq) || !al16(dk) || !al16(dv) || !al16(dlog_alpha) ||
      !al16(dlog_beta) || !al16(dS0))
    return efail(DIG_ERR_MISALIGNED, "a tensor pointer is not 16-byte aligned");
  if (dlog_beta && !zb) return efail(DIG_ERR_INVALID_ARGUMENT, "dlog_beta needs the value-gate logits zb");
  if (dlog_beta && !o) return efail(DIG_ERR_INVALID_ARGUMENT, "dlog_beta needs the forward output o");
  if (B > 0 && L > 0 && (!dO || !dq || !dk || !dv || !dlog_alpha))
    return efail(DIG_ERR_INVALID_ARGUMENT, "dO, dq, dk, dv and dlog_alpha must be non-NULL");
  GlaArgs a;
  bool empty = false;
  dig_status st = ext_setup(q, k, v, z, zb, gate_heads, inv_tau, dO, B, H, L, d_k, d_v, grid_h, grid_w, scan_mode,
                            dtype, out_dtype, workspace, workspace_bytes, true, s, &a, &empty);
  if (st != DIG_OK) return st;
  if (empty) {  // the gradient passes through an empty sequence unchanged
    if (dS0 && B > 0) {
      const size_t bytes = (size_t)B * H * d_k * d_v * sizeof(float);
      const cudaError_t e = dS_final ? cudaMemcpyAsync(dS0, dS_final, bytes, cudaMemcpyDeviceToDevice, s)
                                     : cudaMemsetAsync(dS0, 0, bytes, s);
      if (e != cudaSuccess) return efail(DIG_ERR_CUDA, "initial-state gradient: %s", cudaGetErrorString(e));
    }
    return DIG_OK;
  }
  a.dq = dq; a.dk = dk; a.dv = dv; a.dla = dlog_alpha;
  if (gate_heads == 1) {  // heads add their contributions into dlog_alpha
    const cudaError_t e = cudaMemsetAsync(dlog_alpha, 0, (size_t)B * L * d_k * sizeof(float), s);
    if (e != cudaSuccess) return efail(DIG_ERR_CUDA, "dlog_alpha clear: %s", cudaGetErrorString(e));
  }
  ScanEnds ends{};
  ends.seed[0] = S0;
  ends.fin_rows[0] = a.sfin;
  ends.seed[1] = dS_final;
  ends.fin[1] = dS0;
  GlaVariant var{kExtChunk, 3, d_k, d_v, DIG_F32, out_dtype};
  cudaError_t e = launch_gla_bwd_ext(var, a, ends, s);
  if (e == cudaSuccess && dlog_beta) e = launch_dlogbeta(a, d_k, d_v, out_dtype, o, dlog_beta, s);
  if (e != cudaSuccess) return efail(DIG_ERR_CUDA, "gla_bwd_ext launch: %s", cudaGetErrorString(e));
  return DIG_OK;
}

}  // extern "C"
