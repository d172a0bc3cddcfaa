// gate_proj_tc.cu -- the gate logits' low-rank projection on the tensor cores
// (DiG slides, "Gated Linear Attention Transformer (GLA) の導入", eq. (5): the
// key gate is sigmoid of a low-rank projection D -> R -> d_k of the block input):
//
//   u = x W1   [rows, R],   z = u W2 + b   [rows, d_k]
//
// About 2 D R multiply-adds per token against 2 D bytes of x: 16 per byte at
// R = 16, beyond what the FP32 pipes deliver at HBM speed, so x W1 is a tcgen05
// product: per tile of 128 token rows, A = the x tile (bf16, K-major, tiles of
// 64 channels by TMA with the 128-byte swizzle), B = W1^T as two bf16 terms
// (hi + lo, so the product keeps fp32-level accuracy), M = 128, N = 16, into one
// of two TMEM accumulators.  One thread streams the x blocks through a ring of
// eight stages and issues the products; four warps read u back (lane = row),
// form z = u W2 + b from W2 in shared memory and store u and z.  bf16 x, R <= 16,
// D a multiple of 64 (up to 1152) and d_k <= 64 take this kernel.
#include "tma.cuh"
#include "tma_tiles.cuh"
#include "tmap.h"

namespace dig {

namespace {

constexpr int kBM = 128, kKB = 64, kNS = 8;  // rows per tile, channels per x block, ring stages
constexpr uint32_t kXB = kBM * kKB * 2;       // bytes of one x block (16 KB)
constexpr int kMaxD = 1152;

struct GpSmem {
  uint64_t full[kNS], empty[kNS], acc_full[2], acc_empty[2], wbar;
  uint32_t tmem;
  int abort;
};

// Stages of the x ring: eight, six when D > 768 (the W1 terms then need the room).
__host__ __device__ inline int ring_stages(int D) { return D > 768 ? 6 : kNS; }

// Dynamic shared memory: the x ring (whose last stages first receive W1 and W2 as
// fp32 by bulk copy), W1^T terms (D / 64 blocks of 16 rows x 128 bytes per term), W2 [16][d_k]
// and b [d_k] (fp32), and the output staging (z [128][d_k], u [128][R] fp32).
struct GpLayout {
  uint32_t ring, w1, w2, bias, zst, ust, total;
  __host__ __device__ GpLayout(int D, int dk) {
    ring = 0;
    w1 = (uint32_t)ring_stages(D) * kXB;
    w2 = w1 + 2u * (uint32_t)(D / kKB) * 2048u;
    bias = w2 + 16u * dk * 4u;
    zst = (bias + (uint32_t)dk * 4u + 15u) & ~15u;
    ust = zst + (uint32_t)kBM * dk * 4u;
    total = ust + (uint32_t)kBM * 16u * 4u;
  }
};

// OR of a predicate over the 128 threads of the four epilogue warps (named barrier 1).
__device__ __forceinline__ bool epi_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

template <int DK>
__global__ void __launch_bounds__(256, 1) gate_proj_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                                                              const float* __restrict__ W1,
                                                              const float* __restrict__ W2,
                                                              const float* __restrict__ b, float* __restrict__ z,
                                                              float* __restrict__ u, long long rows, int D, int R,
                                                              uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ GpSmem sh;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t sb = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sb - smem_u32(smem_raw));
  const GpLayout lay(D, DK);
  const int nkb = D / kKB;
  const long long ntiles = (rows + kBM - 1) / kBM;
  const int mytiles = blockIdx.x < ntiles ? (int)((ntiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;
  const int total = mytiles * nkb;  // x blocks this CTA consumes
  if (warp == 0) {
    tmem_alloc(&sh.tmem, 32);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.acc_full[i], 1);
      mbar_init(&sh.acc_empty[i], 128);
    }
    mbar_init(&sh.wbar, 1);
    sh.abort = 0;
    fence_mbar_init();
  }
  // every thread waits on these barriers (the weights' one first): they must be
  // initialised before any thread reaches a wait
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  const int ns = ring_stages(D);
  // ---- W1 and W2 (fp32) into the ring's last stages by two bulk copies (the first x
  // blocks go into the other stages at once), then W1^T as two bf16 terms (row n = output
  // r, K-major, 128-byte swizzle), W2 and b into their places
  const uint32_t w1_bytes = (uint32_t)D * R * 4u, w2_off = (w1_bytes + 15u) & ~15u;
  const int nraw = (int)((w2_off + (uint32_t)R * DK * 4u + kXB - 1) / kXB);  // stages the raw weights take
  const uint32_t raw = lay.ring + (uint32_t)(ns - nraw) * kXB;
  if (tid == 0) {
    mbar_arrive_expect_tx(&sh.wbar, w1_bytes + (uint32_t)R * DK * 4u);
    bulk_copy_g2s(sb + raw, W1, w1_bytes, &sh.wbar);
    bulk_copy_g2s(sb + raw + w2_off, W2, (uint32_t)R * DK * 4u, &sh.wbar);
  }
  auto tile_row = [&](int g) { return (int)((blockIdx.x + (long long)(g / nkb) * gridDim.x) * kBM); };
  auto load = [&](int g) {
    const int s = g % ns;
    mbar_arrive_expect_tx(&sh.full[s], kXB);
    tma_load_2d(sb + lay.ring + s * kXB, xmap, (g % nkb) * kKB, tile_row(g), &sh.full[s]);
  };
  int issued = 0;  // thread 0: blocks requested
  if (tid == 0)
    for (; issued < total && issued < ns - nraw; ++issued) load(issued);
  float* sW2 = reinterpret_cast<float*>(sgen + lay.w2);
  float* sB = reinterpret_cast<float*>(sgen + lay.bias);
  const float bv = (tid < DK && b != nullptr) ? __ldg(b + tid) : 0.f;
  const bool w_ok = mbar_wait(&sh.wbar, 0, kSpinLimitNs);
  const float* rawW1 = reinterpret_cast<const float*>(sgen + raw);
  const float* rawW2 = reinterpret_cast<const float*>(sgen + raw + w2_off);
  for (int i = tid; i < 16 * D; i += 256) {  // element (k, n), i = 16 k + n
    const int k = i >> 4, n = i & 15;
    const float w = (n < R && w_ok) ? rawW1[k * R + n] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
    const uint32_t off = (uint32_t)(k / kKB) * 2048u + swz_off<128>(n, (k % kKB) / 8) + (k % 8) * 2;
    *reinterpret_cast<__nv_bfloat16*>(sgen + lay.w1 + off) = hi;
    *reinterpret_cast<__nv_bfloat16*>(sgen + lay.w1 + (uint32_t)nkb * 2048u + off) = lo;
  }
  for (int i = tid; i < 16 * DK; i += 256) sW2[i] = (i / DK < R && w_ok) ? rawW2[i] : 0.f;
  if (tid < DK) sB[tid] = bv;
  if (!w_ok) {
    sh.abort = 1;
    if (status != nullptr) set_status(status, DIG_ERR_DEVICE_TIMEOUT);
  }
  // every thread's reads of the raw weights precede the x copies into the ring
  fence_async_smem();
  __syncthreads();
  if (tid == 0 && !sh.abort)  // the raw weights are read: their stages take x blocks too
    for (; issued < total && issued < ns; ++issued) load(issued);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem;
  const uint64_t spin = kSpinLimitNs;

  if (warp == 0) {
    // ---------------- one thread: x blocks through the ring, products into the accumulators
    if (tid == 0) {
      int committed = -1;  // the last block whose products were committed
      bool stop = false;
      for (int g = 0; g < total && !stop && !sh.abort; ++g) {
        const int s = g % ns, i = g / nkb, kb = g % nkb, ac = i & 1;
        if (!mbar_wait(&sh.full[s], (g / ns) & 1, spin)) { stop = true; break; }
        if (kb == 0 && i >= 2 && !mbar_wait(&sh.acc_empty[ac], ((i >> 1) - 1) & 1, spin)) { stop = true; break; }
        tc_fence_after();
        const uint32_t xs = sb + lay.ring + s * kXB;
#pragma unroll
        for (int ks = 0; ks < kKB / 16; ++ks)
#pragma unroll
          for (int tt = 0; tt < 2; ++tt)
            mma_bf16(tmem + 16u * ac, sdesc_sw<128>(xs + 32 * ks),
                     sdesc_sw<128>(sb + lay.w1 + (uint32_t)(tt * nkb + kb) * 2048u + 32 * ks),
                     idesc_bf16(kBM, 16), (kb | ks | tt) ? 1u : 0u);
        mma_commit(&sh.empty[s]);
        if (kb == nkb - 1) mma_commit(&sh.acc_full[ac]);
        committed = g;
        // the block before this one has been read: its stage takes the block ns - 1 ahead
        if (g >= 1 && issued < total) {
          const int gp = g - 1;
          if (!mbar_wait(&sh.empty[gp % ns], (gp / ns) & 1, spin)) { stop = true; break; }
          load(issued++);
        }
      }
      if (stop) sh.abort = 1;
      // drain: every requested block has landed and the last products completed
      for (int g = (committed < 0 ? 0 : committed + 1); g < issued; ++g)
        mbar_wait(&sh.full[g % ns], (g / ns) & 1, kSpinLimitNs);
      if (committed >= 0) mbar_wait(&sh.empty[committed % ns], (committed / ns) & 1, kSpinLimitNs);
      if (stop && status != nullptr) set_status(status, DIG_ERR_DEVICE_TIMEOUT);
    }
  } else if (warp >= 4) {
    // ---------------- four warps: u from TMEM (lane = tile row), z = u W2 + b, stores
    const int lr = tid - 128;  // TMEM lane = row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp - 4)) << 16;
    for (int i = 0; i < mytiles; ++i) {
      const int ac = i & 1;
      const bool ok = mbar_wait(&sh.acc_full[ac], (i >> 1) & 1, spin);
      if (epi_any(!ok || sh.abort)) {  // uniform over the four warps (they share barrier 1)
        sh.abort = 1;
        if (status != nullptr) set_status(status, DIG_ERR_DEVICE_TIMEOUT);
        break;
      }
      tc_fence_after();
      float uv[16];
      tmem_ld16(tmem + lane_base + 16u * ac, uv);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&sh.acc_empty[ac]);
      // z = u W2 + b of this row, then the tile's u and z rows (contiguous in global
      // memory) leave through shared memory as coalesced 16-byte stores
      float* zs = reinterpret_cast<float*>(sgen + lay.zst);
      float* us = reinterpret_cast<float*>(sgen + lay.ust);
      named_bar(1, 128);  // the previous tile's staged rows have been stored
#pragma unroll
      for (int r = 0; r < 16; ++r)
        if (r < R) us[lr * R + r] = uv[r];
#pragma unroll
      for (int c0 = 0; c0 < DK; c0 += 4) {
        float acc[4] = {sB[c0], sB[c0 + 1], sB[c0 + 2], sB[c0 + 3]};
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const float4 w4 = *reinterpret_cast<const float4*>(sW2 + r * DK + c0);
          acc[0] = fmaf(uv[r], w4.x, acc[0]);
          acc[1] = fmaf(uv[r], w4.y, acc[1]);
          acc[2] = fmaf(uv[r], w4.z, acc[2]);
          acc[3] = fmaf(uv[r], w4.w, acc[3]);
        }
        *reinterpret_cast<float4*>(zs + lr * DK + c0) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      }
      named_bar(1, 128);
      const long long row0 = (blockIdx.x + (long long)i * gridDim.x) * kBM;
      const int nrow = (int)(rows - row0 < kBM ? rows - row0 : kBM);
      const int zq = nrow * DK / 4, uq = nrow * R;  // float4s of z; floats of u
      float4* zg = reinterpret_cast<float4*>(z + row0 * DK);
      for (int q = lr; q < zq; q += 128) zg[q] = reinterpret_cast<const float4*>(zs)[q];
      if (u != nullptr) {
        float* ug = u + row0 * R;
        for (int q = lr; q < uq; q += 128) ug[q] = us[q];
      }
    }
  }
  if (tid == 0 && !w_ok) mbar_wait(&sh.wbar, 0, kSpinLimitNs);  // the weights' copies have landed
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 32);
}

template <int DK>
cudaError_t launch_dk(const CUtensorMap& m, const float* W1, const float* W2, const float* b, float* z, float* u,
                      long long rows, int D, int R, uint32_t* status, cudaStream_t s) {
  auto k = gate_proj_tc_kernel<DK>;
  const uint32_t smem = GpLayout(D, DK).total + 1024;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long ntiles = (rows + kBM - 1) / kBM;
  const int grid = (int)(ntiles < num_sms() ? ntiles : num_sms());
  return launch_pdl(k, dim3(grid), dim3(256), smem, s, m, W1, W2, b, z, u, rows, D, R, status);
}

}  // namespace

bool gate_proj_tc_eligible(long long rows, int D, int R, int dk, int tin) {
  return tin == DIG_BF16 && rows > 0 && rows <= 0x7FFFFFFFLL && R >= 1 && R <= 16 && D % kKB == 0 && D <= kMaxD &&
         (dk == 32 || dk == 36 || dk == 64) && tmap_available();
}

// `launched` stays false when the tensor map cannot be encoded (the caller runs
// the CUDA-core kernel).  `status`: a device word that receives
// DIG_ERR_DEVICE_TIMEOUT if a wait gives up, or NULL.
cudaError_t launch_gate_proj_tc(const void* x, const float* W1, const float* W2, const float* b, float* z, float* u,
                                long long rows, int D, int R, int dk, uint32_t* status, cudaStream_t s,
                                bool* launched) {
  *launched = false;
  CUtensorMap m;
  memset(&m, 0, sizeof(m));
  if (!tmap_rows(&m, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, (uint64_t)rows, kKB, kBM, 128)) return cudaSuccess;
  cudaError_t e;
  if (dk == 32) e = launch_dk<32>(m, W1, W2, b, z, u, rows, D, R, status, s);
  else if (dk == 36) e = launch_dk<36>(m, W1, W2, b, z, u, rows, D, R, status, s);
  else e = launch_dk<64>(m, W1, W2, b, z, u, rows, D, R, status, s);
  if (e == cudaSuccess) *launched = true;
  return e;
}

}  // namespace dig
