// dig_api.cu -- the C ABI of libdig.so (include/dig.h): argument validation,
// work decomposition, workspace layout, launches.  No allocation and no
// synchronisation (except dig_read_status).  The library keeps no device state
// of its own, with one exception: the 16 MiB scratch array of
// dig_gla_fwd_noalloc (dig_noalloc.cu), held per device until the process exits.
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "../../include/dig.h"
#include "dig_common.cuh"
#include "bwd_ops.h"
#include "gate_proj.h"
#include "gla.h"

namespace dig {

static thread_local char g_last_error[512] = "";

static dig_status fail(dig_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Lets other entry points of the library report a message through dig_last_error.
void set_last_error(const char* msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }

WsLayout ws_layout(int B, int H, int gate_heads, int L, int nchunks, int dk, int dv, bool backward) {
  const size_t nseq = (size_t)B * H;
  const size_t nbz = (size_t)B * gate_heads;
  WsLayout w{};
  size_t off = sizeof(WsHeader);
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  w.gEQ = take(nbz * (size_t)L * dk * 4);
  w.gCH = take(nbz * (size_t)nchunks * 4 * dk * 4);
  w.dsn = take(nseq * (size_t)nchunks * dk * dv * 4);
  w.dhn = take(backward ? nseq * (size_t)nchunks * dk * dv * 4 : 0);
  w.flist = take(backward ? (1 + nseq * (size_t)nchunks) * 4 : 0);
  w.sflag = take(nbz * (size_t)nchunks * 4);
  w.total = off;
  return w;
}

namespace {

// Tokens per chunk: forward 128 (bf16 inputs) / 64 (fp32); backward by head dims.
int chunk_len(int dtype, bool backward, int dk, int dv) {
  if (backward) return gla_bwd_chunk(dk, dv, dtype);
  return dtype == DIG_BF16 ? 128 : 64;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

// Bound of the kernels' device waits: DIG_DEVICE_WAIT_LIMIT_NS in the environment
// (a test hook that makes a wait run out on purpose), else the two-second default.
unsigned long long spin_limit_ns() {
  const char* e = getenv("DIG_DEVICE_WAIT_LIMIT_NS");
  if (!e || !*e) return 0;
  const unsigned long long v = strtoull(e, nullptr, 10);
  return v;
}

dig_status check_common(int B, int H, int L, int d_k, int d_v, int grid_h, int grid_w, int scan_mode, int dtype,
                        int out_dtype, int gate_heads) {
  if (B < 0 || H <= 0 || L < 0 || grid_h < 0 || grid_w < 0)
    return fail(DIG_ERR_INVALID_ARGUMENT, "negative or zero size (B=%d H=%d L=%d grid=%dx%d)", B, H, L, grid_h, grid_w);
  if ((long long)grid_h * grid_w != L)
    return fail(DIG_ERR_INVALID_ARGUMENT, "L=%d is not grid_h*grid_w=%d*%d", L, grid_h, grid_w);
  if (scan_mode < 0 || scan_mode > 3) return fail(DIG_ERR_INVALID_ARGUMENT, "scan_mode %d not in 0..3", scan_mode);
  if ((dtype != DIG_F32 && dtype != DIG_BF16) || (out_dtype != DIG_F32 && out_dtype != DIG_BF16))
    return fail(DIG_ERR_INVALID_ARGUMENT, "dtype %d / out_dtype %d not DIG_F32 or DIG_BF16", dtype, out_dtype);
  if (gate_heads != 1 && gate_heads != H)
    return fail(DIG_ERR_INVALID_ARGUMENT, "gate_heads=%d must be 1 or H=%d", gate_heads, H);
  if (d_k <= 0 || d_v <= 0) return fail(DIG_ERR_INVALID_ARGUMENT, "head dims must be positive");
  if (!gla_variant_built(d_k, d_v))
    return fail(DIG_ERR_UNSUPPORTED, "(d_k, d_v) = (%d, %d) is not built (supported: (32,64), (36,72), (64,64))", d_k,
                d_v);
  if ((long long)B * L * H * (d_k > d_v ? d_k : d_v) >= (1ll << 40))
    return fail(DIG_ERR_INVALID_ARGUMENT, "tensor too large");
  return DIG_OK;
}

}  // namespace dig

using namespace dig;

extern "C" {

int dig_gla_supported(int d_k, int d_v) { return gla_variant_built(d_k, d_v) ? 1 : 0; }

size_t dig_gla_workspace_bytes(int B, int H, int gate_heads, int L, int d_k, int d_v, int pass) {
  if (B < 0 || H <= 0 || L < 0 || d_k <= 0 || d_v <= 0 || (pass != 0 && pass != 1)) return 0;
  if (gate_heads != 1 && gate_heads != H) return 0;
  if (!gla_variant_built(d_k, d_v)) return 0;
  // sized for the largest chunk count of either input type
  const int C = pass == 1 ? gla_bwd_chunk(d_k, d_v, DIG_F32) : 64;
  const int nchunks = (L + C - 1) / C;
  return ws_layout(B > 0 ? B : 1, H, gate_heads, L, nchunks, d_k, d_v, pass == 1).total;
}

}  // extern "C"

namespace dig {
// Every synchronous check of dig_gla_fwd (also run by dig_gla_fwd_noalloc before
// it enqueues anything).  DIG_OK with *nothing_to_do set means an empty problem.
dig_status gla_fwd_check(const void* q, const void* k, const void* v, const float* z, int gate_heads, void* o,
                         const void* r, const float* gamma, void* y, int B, int H, int L, int d_k, int d_v,
                         int grid_h, int grid_w, int scan_mode, int dtype, int out_dtype, const void* workspace,
                         size_t workspace_bytes, bool* nothing_to_do) {
  *nothing_to_do = false;
  dig_status st = check_common(B, H, L, d_k, d_v, grid_h, grid_w, scan_mode, dtype, out_dtype, gate_heads);
  if (st != DIG_OK) return st;
  if (!workspace) return fail(DIG_ERR_INVALID_ARGUMENT, "workspace is NULL");
  if (!aligned16(workspace)) return fail(DIG_ERR_MISALIGNED, "workspace not 16-byte aligned");
  if (B == 0 || L == 0) {
    *nothing_to_do = true;
    return DIG_OK;
  }
  if (!q || !k || !v || !z || !o) return fail(DIG_ERR_INVALID_ARGUMENT, "q, k, v, z and o must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(z) || !aligned16(o) || !aligned16(r) ||
      !aligned16(gamma) || !aligned16(y))
    return fail(DIG_ERR_MISALIGNED, "a tensor pointer is not 16-byte aligned");
  const int C = chunk_len(dtype, false, d_k, d_v);
  const WsLayout lay = ws_layout(B, H, gate_heads, L, (L + C - 1) / C, d_k, d_v, false);
  if (workspace_bytes < lay.total)
    return fail(DIG_ERR_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, needs %zu", workspace_bytes, lay.total);
  return DIG_OK;
}
}  // namespace dig

extern "C" {

dig_status dig_gla_fwd(const void* q, const void* k, const void* v, const float* z, int gate_heads, float inv_tau,
                       void* o, const void* r, const float* gamma, float eps, void* y, int B, int H, int L, int d_k,
                       int d_v, int grid_h, int grid_w, int scan_mode, int dtype, int out_dtype, void* workspace,
                       size_t workspace_bytes, void* stream) {
  bool empty = false;
  const dig_status st = gla_fwd_check(q, k, v, z, gate_heads, o, r, gamma, y, B, H, L, d_k, d_v, grid_h, grid_w,
                                      scan_mode, dtype, out_dtype, workspace, workspace_bytes, &empty);
  if (st != DIG_OK || empty) return st;
  const int C = chunk_len(dtype, false, d_k, d_v);
  const int nchunks = (L + C - 1) / C;
  const WsLayout lay = ws_layout(B, H, gate_heads, L, nchunks, d_k, d_v, false);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  GlaArgs a{};
  a.q = q; a.k = k; a.v = v; a.z = z; a.r = r; a.gamma = gamma; a.o = o; a.y = y;
  a.B = B; a.H = H; a.L = L; a.Hg = grid_h; a.Wg = grid_w; a.mode = scan_mode; a.gate_heads = gate_heads;
  a.inv_tau = inv_tau; a.eps = eps;
  a.nchunks = nchunks;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.gEQ = reinterpret_cast<float*>(ws + lay.gEQ);
  a.gCH = reinterpret_cast<float*>(ws + lay.gCH);
  a.dsn = reinterpret_cast<float*>(ws + lay.dsn);
  a.sflag = reinterpret_cast<int*>(ws + lay.sflag);
  a.chunk = C;
  a.in_bf16 = dtype == DIG_BF16;
  a.spin_ns = spin_limit_ns();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  GlaVariant var{C, dtype == DIG_BF16 ? 2 : 3, d_k, d_v, dtype, out_dtype};
  const cudaError_t e = launch_gla_fwd(var, a, s);
  if (e != cudaSuccess) return fail(DIG_ERR_CUDA, "gla_fwd launch: %s", cudaGetErrorString(e));
  return DIG_OK;
}

static dig_status gla_bwd_impl(const void* q, const void* k, const void* v, const float* z, int gate_heads,
                               float inv_tau, const void* dO, void* dq, void* dk, void* dv, float* dlog_alpha, int B,
                               int H, int L, int d_k, int d_v, int grid_h, int grid_w, int scan_mode, int dtype,
                               int out_dtype, const void* fwd_workspace, size_t fwd_workspace_bytes, void* workspace,
                               size_t workspace_bytes, void* stream) {
  dig_status st = check_common(B, H, L, d_k, d_v, grid_h, grid_w, scan_mode, dtype, out_dtype, gate_heads);
  if (st != DIG_OK) return st;
  if (!workspace) return fail(DIG_ERR_INVALID_ARGUMENT, "workspace is NULL");
  if (!aligned16(workspace) || !aligned16(fwd_workspace)) return fail(DIG_ERR_MISALIGNED, "workspace not 16-byte aligned");
  if (B == 0 || L == 0) return DIG_OK;
  if (!q || !k || !v || !z || !dO || !dq || !dk || !dv || !dlog_alpha)
    return fail(DIG_ERR_INVALID_ARGUMENT, "all tensor pointers of the backward must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(z) || !aligned16(dO) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(dlog_alpha))
    return fail(DIG_ERR_MISALIGNED, "a tensor pointer is not 16-byte aligned");
  const int C = chunk_len(dtype, true, d_k, d_v);
  const int nchunks = (L + C - 1) / C;
  const WsLayout lay = ws_layout(B, H, gate_heads, L, nchunks, d_k, d_v, true);
  if (workspace_bytes < lay.total)
    return fail(DIG_ERR_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, needs %zu", workspace_bytes, lay.total);
  // The forward's records are usable when both passes cut the sequence into the same chunks.
  const bool saved = fwd_workspace != nullptr && chunk_len(dtype, false, d_k, d_v) == C;
  const WsLayout flay = ws_layout(B, H, gate_heads, L, nchunks, d_k, d_v, false);
  if (saved && fwd_workspace_bytes < flay.total)
    return fail(DIG_ERR_WORKSPACE_TOO_SMALL, "forward workspace has %zu bytes, needs %zu", fwd_workspace_bytes,
                flay.total);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* fws = static_cast<uint8_t*>(const_cast<void*>(fwd_workspace));  // only read
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (gate_heads == 1) {
    // heads add their contributions into dlog_alpha
    const cudaError_t e = cudaMemsetAsync(dlog_alpha, 0, (size_t)B * L * d_k * sizeof(float), s);
    if (e != cudaSuccess) return fail(DIG_ERR_CUDA, "dlog_alpha clear: %s", cudaGetErrorString(e));
  }
  GlaArgs a{};
  a.q = q; a.k = k; a.v = v; a.z = z; a.dO = dO; a.dq = dq; a.dk = dk; a.dv = dv; a.dla = dlog_alpha;
  a.B = B; a.H = H; a.L = L; a.Hg = grid_h; a.Wg = grid_w; a.mode = scan_mode; a.gate_heads = gate_heads;
  a.inv_tau = inv_tau;
  a.nchunks = nchunks;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.gEQ = reinterpret_cast<float*>((saved ? fws + flay.gEQ : ws + lay.gEQ));
  a.gCH = reinterpret_cast<float*>((saved ? fws + flay.gCH : ws + lay.gCH));
  a.dsn = reinterpret_cast<float*>((saved ? fws + flay.dsn : ws + lay.dsn));
  a.dhn = reinterpret_cast<float*>(ws + lay.dhn);
  a.flist = reinterpret_cast<uint32_t*>(ws + lay.flist);
  a.sflag = reinterpret_cast<int*>((saved ? fws + flay.sflag : ws + lay.sflag));
  a.chunk = C;
  a.in_bf16 = dtype == DIG_BF16;
  a.spin_ns = spin_limit_ns();
  GlaVariant var{C, dtype == DIG_BF16 ? 2 : 3, d_k, d_v, dtype, out_dtype};
  const cudaError_t e = launch_gla_bwd(var, a, saved, s);
  if (e != cudaSuccess) return fail(DIG_ERR_CUDA, "gla_bwd launch: %s", cudaGetErrorString(e));
  return DIG_OK;
}

dig_status dig_gla_bwd(const void* q, const void* k, const void* v, const float* z, int gate_heads, float inv_tau,
                       const void* dO, void* dq, void* dk, void* dv, float* dlog_alpha, int B, int H, int L, int d_k,
                       int d_v, int grid_h, int grid_w, int scan_mode, int dtype, int out_dtype, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return gla_bwd_impl(q, k, v, z, gate_heads, inv_tau, dO, dq, dk, dv, dlog_alpha, B, H, L, d_k, d_v, grid_h, grid_w,
                      scan_mode, dtype, out_dtype, nullptr, 0, workspace, workspace_bytes, stream);
}

dig_status dig_gla_bwd_saved(const void* q, const void* k, const void* v, const float* z, int gate_heads,
                             float inv_tau, const void* dO, void* dq, void* dk, void* dv, float* dlog_alpha, int B,
                             int H, int L, int d_k, int d_v, int grid_h, int grid_w, int scan_mode, int dtype,
                             int out_dtype, const void* fwd_workspace, size_t fwd_workspace_bytes, void* workspace,
                             size_t workspace_bytes, void* stream) {
  if (!fwd_workspace) return fail(DIG_ERR_INVALID_ARGUMENT, "fwd_workspace is NULL");
  return gla_bwd_impl(q, k, v, z, gate_heads, inv_tau, dO, dq, dk, dv, dlog_alpha, B, H, L, d_k, d_v, grid_h, grid_w,
                      scan_mode, dtype, out_dtype, fwd_workspace, fwd_workspace_bytes, workspace, workspace_bytes,
                      stream);
}

dig_status dig_srem_reorient_dwconv(const void* x, const float* w, const float* bias, void* y, int B, int grid_h,
                                    int grid_w, int C, int scan_mode, int dtype, int out_dtype, void* stream) {
  if (B < 0 || grid_h < 0 || grid_w < 0 || C <= 0)
    return fail(DIG_ERR_INVALID_ARGUMENT, "bad size (B=%d grid=%dx%d C=%d)", B, grid_h, grid_w, C);
  if (scan_mode < 0 || scan_mode > 3) return fail(DIG_ERR_INVALID_ARGUMENT, "scan_mode %d not in 0..3", scan_mode);
  if ((dtype != DIG_F32 && dtype != DIG_BF16) || (out_dtype != DIG_F32 && out_dtype != DIG_BF16))
    return fail(DIG_ERR_INVALID_ARGUMENT, "dtype %d / out_dtype %d not DIG_F32 or DIG_BF16", dtype, out_dtype);
  if ((long long)B * grid_h * grid_w * C >= (1ll << 40)) return fail(DIG_ERR_INVALID_ARGUMENT, "tensor too large");
  if (B == 0 || grid_h == 0 || grid_w == 0) return DIG_OK;
  if (!x || !w || !y) return fail(DIG_ERR_INVALID_ARGUMENT, "x, w and y must be non-NULL");
  if (!aligned16(x) || !aligned16(y) || !aligned16(w) || !aligned16(bias))
    return fail(DIG_ERR_MISALIGNED, "a tensor pointer is not 16-byte aligned");
  const cudaError_t e =
      launch_srem(x, w, bias, y, B, grid_h, grid_w, C, scan_mode, dtype, out_dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(DIG_ERR_CUDA, "srem launch: %s", cudaGetErrorString(e));
  return DIG_OK;
}

dig_status dig_srem_reorient_dwconv_bwd(const void* x, const float* w, const void* dY, void* dx, float* dw,
                                        float* dbias, int B, int grid_h, int grid_w, int C, int scan_mode, int dtype,
                                        int out_dtype, void* stream) {
  if (B < 0 || grid_h < 0 || grid_w < 0 || C <= 0)
    return fail(DIG_ERR_INVALID_ARGUMENT, "bad size (B=%d grid=%dx%d C=%d)", B, grid_h, grid_w, C);
  if (scan_mode < 0 || scan_mode > 3) return fail(DIG_ERR_INVALID_ARGUMENT, "scan_mode %d not in 0..3", scan_mode);
  if ((dtype != DIG_F32 && dtype != DIG_BF16) || (out_dtype != DIG_F32 && out_dtype != DIG_BF16))
    return fail(DIG_ERR_INVALID_ARGUMENT, "dtype %d / out_dtype %d not DIG_F32 or DIG_BF16", dtype, out_dtype);
  if ((long long)B * grid_h * grid_w * C >= (1ll << 40)) return fail(DIG_ERR_INVALID_ARGUMENT, "tensor too large");
  if ((long long)grid_h * grid_w >= (1ll << 31)) return fail(DIG_ERR_INVALID_ARGUMENT, "grid too large");
  if (!w) return fail(DIG_ERR_INVALID_ARGUMENT, "w must be non-NULL");
  if (!aligned16(x) || !aligned16(w) || !aligned16(dY) || !aligned16(dx) || !aligned16(dw) || !aligned16(dbias))
    return fail(DIG_ERR_MISALIGNED, "a tensor pointer is not 16-byte aligned");
  if (B == 0 || grid_h == 0 || grid_w == 0) {  // no pixels: the parameter gradients are zero
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = dw ? cudaMemsetAsync(dw, 0, (size_t)C * 9 * sizeof(float), s) : cudaSuccess;
    if (e == cudaSuccess && dbias) e = cudaMemsetAsync(dbias, 0, (size_t)C * sizeof(float), s);
    if (e != cudaSuccess) return fail(DIG_ERR_CUDA, "memset: %s", cudaGetErrorString(e));
    return DIG_OK;
  }
  if (!dY || !dx) return fail(DIG_ERR_INVALID_ARGUMENT, "dY and dx must be non-NULL");
  if ((dw || dbias) && !x) return fail(DIG_ERR_INVALID_ARGUMENT, "x must be non-NULL when dw or dbias is wanted");
  const cudaError_t e = launch_srem_bwd(x, w, dY, dx, dw, dbias, B, grid_h, grid_w, C, scan_mode, dtype, out_dtype,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(DIG_ERR_CUDA, "srem backward launch: %s", cudaGetErrorString(e));
  return DIG_OK;
}

dig_status dig_epilogue_bwd(const void* o, const void* r, const float* gamma, float eps, const void* dY, void* d_o,
                            void* d_r, float* d_gamma, long long rows, int d_v, int dtype, int out_dtype,
                            void* stream) {
  if (rows < 0 || d_v <= 0) return fail(DIG_ERR_INVALID_ARGUMENT, "bad size (rows=%lld d_v=%d)", rows, d_v);
  if (d_v > 8192) return fail(DIG_ERR_UNSUPPORTED, "d_v=%d above 8192", d_v);
  if (!(eps >= 0.f)) return fail(DIG_ERR_INVALID_ARGUMENT, "eps must be >= 0");
  if ((dtype != DIG_F32 && dtype != DIG_BF16) || (out_dtype != DIG_F32 && out_dtype != DIG_BF16))
    return fail(DIG_ERR_INVALID_ARGUMENT, "dtype %d / out_dtype %d not DIG_F32 or DIG_BF16", dtype, out_dtype);
  if (rows >= (1ll << 40) / d_v) return fail(DIG_ERR_INVALID_ARGUMENT, "tensor too large");
  if (rows > 0 && (!o || !r || !dY || !d_o || !d_r))
    return fail(DIG_ERR_INVALID_ARGUMENT, "o, r, dY, d_o and d_r must be non-NULL");
  if (!aligned16(o) || !aligned16(r) || !aligned16(dY) || !aligned16(d_o) || !aligned16(d_r) ||
      !aligned16(gamma) || !aligned16(d_gamma))
    return fail(DIG_ERR_MISALIGNED, "a tensor pointer is not 16-byte aligned");
  const cudaError_t e = launch_epilogue_bwd(o, r, gamma, eps, dY, d_o, d_r, d_gamma, rows, d_v, dtype, out_dtype,
                                            static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(DIG_ERR_CUDA, "epilogue backward launch: %s", cudaGetErrorString(e));
  return DIG_OK;
}

static dig_status check_gate_shape(long long rows, int D, int R, int d_k, bool backward) {
  if (rows < 0 || D <= 0 || R <= 0 || d_k <= 0)
    return fail(DIG_ERR_INVALID_ARGUMENT, "bad size (rows=%lld D=%d R=%d d_k=%d)", rows, D, R, d_k);
  if (D % 8 != 0 || R > 32 || d_k > 128)
    return fail(DIG_ERR_UNSUPPORTED, "gate projection built for D %% 8 == 0, R <= 32, d_k <= 128 (D=%d R=%d d_k=%d)",
                D, R, d_k);
  if (gate_proj_smem_bytes(D, R, d_k, backward) > 227u * 1024u)
    return fail(DIG_ERR_UNSUPPORTED, "gate projection weights do not fit shared memory (D=%d R=%d d_k=%d)", D, R,
                d_k);
  if (rows >= (1ll << 40) / D) return fail(DIG_ERR_INVALID_ARGUMENT, "tensor too large");
  return DIG_OK;
}

dig_status dig_gate_proj_fwd(const void* x, const float* W1, const float* W2, const float* b, float* z, float* u,
                             long long rows, int D, int R, int d_k, int dtype, void* stream) {
  const dig_status st = check_gate_shape(rows, D, R, d_k, false);
  if (st != DIG_OK) return st;
  if (dtype != DIG_F32 && dtype != DIG_BF16) return fail(DIG_ERR_INVALID_ARGUMENT, "dtype %d not DIG_F32 or DIG_BF16", dtype);
  if (rows > 0 && (!x || !W1 || !W2 || !z)) return fail(DIG_ERR_INVALID_ARGUMENT, "x, W1, W2 and z must be non-NULL");
  if (!aligned16(x) || !aligned16(W1) || !aligned16(W2) || !aligned16(b) || !aligned16(z) || !aligned16(u))
    return fail(DIG_ERR_MISALIGNED, "a tensor pointer is not 16-byte aligned");
  const cudaError_t e = launch_gate_proj_fwd(x, W1, W2, b, z, u, rows, D, R, d_k, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(DIG_ERR_CUDA, "gate projection launch: %s", cudaGetErrorString(e));
  return DIG_OK;
}

dig_status dig_gate_proj_bwd(const void* x, const float* W1, const float* W2, const float* u, const float* z,
                             const float* dlog_alpha, float inv_tau, void* dx, float* dW1, float* dW2, float* db,
                             long long rows, int D, int R, int d_k, int dtype, int out_dtype, void* stream) {
  const dig_status st = check_gate_shape(rows, D, R, d_k, true);
  if (st != DIG_OK) return st;
  if ((dtype != DIG_F32 && dtype != DIG_BF16) || (out_dtype != DIG_F32 && out_dtype != DIG_BF16))
    return fail(DIG_ERR_INVALID_ARGUMENT, "dtype %d / out_dtype %d not DIG_F32 or DIG_BF16", dtype, out_dtype);
  if (!(inv_tau > 0.f && inv_tau < 1e30f)) return fail(DIG_ERR_INVALID_ARGUMENT, "inv_tau must be positive and finite");
  if (!dW1 || !dW2) return fail(DIG_ERR_INVALID_ARGUMENT, "dW1 and dW2 must be non-NULL");
  if (rows > 0 && (!x || !W1 || !W2 || !u || !z || !dlog_alpha || !dx))
    return fail(DIG_ERR_INVALID_ARGUMENT, "x, W1, W2, u, z, dlog_alpha and dx must be non-NULL");
  if (!aligned16(x) || !aligned16(W1) || !aligned16(W2) || !aligned16(u) || !aligned16(z) || !aligned16(dlog_alpha) ||
      !aligned16(dx) || !aligned16(dW1) || !aligned16(dW2) || !aligned16(db))
    return fail(DIG_ERR_MISALIGNED, "a tensor pointer is not 16-byte aligned");
  const cudaError_t e = launch_gate_proj_bwd(x, W1, W2, u, z, dlog_alpha, inv_tau, dx, dW1, dW2, db, rows, D, R, d_k,
                                             dtype, out_dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(DIG_ERR_CUDA, "gate projection backward launch: %s", cudaGetErrorString(e));
  return DIG_OK;
}

dig_status dig_read_status(void* workspace, void* stream) {
  if (!workspace) return fail(DIG_ERR_INVALID_ARGUMENT, "workspace is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t host = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&host, workspace, sizeof(host), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && host != 0) e = cudaMemset(workspace, 0, sizeof(uint32_t));
  if (e != cudaSuccess) return fail(DIG_ERR_CUDA, "read status: %s", cudaGetErrorString(e));
  return static_cast<dig_status>(host);
}

const char* dig_status_string(dig_status s) {
  switch (s) {
    case DIG_OK: return "ok";
    case DIG_ERR_INVALID_ARGUMENT: return "invalid argument";
    case DIG_ERR_UNSUPPORTED: return "unsupported configuration";
    case DIG_ERR_MISALIGNED: return "misaligned pointer";
    case DIG_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case DIG_ERR_CUDA: return "CUDA error";
    case DIG_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case DIG_ERR_GATE_RANGE: return "gate decay outside the chunked factorisation's range";
    default: return "unknown status";
  }
}

const char* dig_last_error(void) { return g_last_error; }

}  // extern "C"
