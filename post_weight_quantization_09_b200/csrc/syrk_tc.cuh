// Proxy Hessian on the 5th-generation tensor cores: H_acc (+)= X^T X for
// bf16 activations X (N tokens x n channels, row-major), fp32 accumulation
// (QuIP, adaptive-rounding section: H is the second moment of the
// calibration inputs).
//
// Only the lower triangle is needed, so the grid enumerates the 256 x 256
// output tiles (ti, tj) with ti >= tj.  Per CTA (one per SM, 256 threads):
//  * warp 0 / lane 0 streams K-slabs of 64 tokens with TMA: the A slab is
//    channels [256 ti, +256) and the B slab channels [256 tj, +256), each as
//    four 64-channel x 64-token boxes with the 128-byte swizzle.  In X's
//    row-major layout both operands are MN-major (channels contiguous), so
//    no transpose pass is needed; on diagonal tiles A and B are the same slab
//    and are loaded once.
//  * warp 1 / lane 0 issues tcgen05.mma kind::f16 (M = 128, N = 256, K = 16),
//    two per K-step (tile rows 0..127 and 128..255), accumulating in TMEM
//    columns [0, 256) and [256, 512).
//  * 3-stage smem ring (64 KB per stage) with full / empty mbarriers; the
//    MMA thread frees a stage with tcgen05.commit.
//  * The tensor core's fp32 accumulation drops low bits (about one ulp of
//    the running sum per MMA step), so the token range is cut into chunks of
//    2048: each chunk starts a fresh TMEM accumulator, and warps 4..7 add the
//    chunk's sums into H in fp32 (the first chunk stores, later chunks add by
//    vector reductions issued by the same thread to the same addresses, so
//    the order, and the result, are fixed) while the producer already loads
//    the next chunk.  Warp w reads TMEM lanes 32 (w - 4) of both accumulators.
// Every mbarrier wait is bounded (common.cuh); on a timeout the CTA records
// QUIP_ERR_TIMEOUT, skips the stores, waits for its own MMAs and frees TMEM.
#pragma once

#include "common.cuh"

namespace quip {
namespace syrk {

constexpr int BT = 256;                       // output tile (square)
constexpr int BK = 64;                        // tokens per K-step
constexpr int STAGES = 3;
constexpr int BOX_BYTES = 64 * BK * 2;        // 64 channels x 64 tokens bf16 = 8 KB
constexpr int SLAB_BYTES = 4 * BOX_BYTES;     // 256 channels = 32 KB
constexpr int STAGE_BYTES = 2 * SLAB_BYTES;   // A + B = 64 KB
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t IDESC = make_idesc_bf16(128, 256, /*a_mn=*/1, /*b_mn=*/1);

constexpr int KCHUNK = 2048 / BK;              // K-steps per accumulation chunk

struct Shared {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull;          // chunk accumulated (MMA -> epilogue)
  uint64_t tempty;         // chunk drained (epilogue -> MMA)
  uint32_t tmem_base;
  int abort;
};

// Tile index -> (ti, tj), ti >= tj, row-major over the lower triangle.
__device__ __forceinline__ void tri_decode(int x, int& ti, int& tj) {
  int i = (int)((sqrtf(8.f * (float)x + 1.f) - 1.f) * 0.5f);
  while ((i + 1) * (i + 2) / 2 <= x) ++i;
  while (i * (i + 1) / 2 > x) --i;
  ti = i;
  tj = x - i * (i + 1) / 2;
}

__global__ void __launch_bounds__(256, 1)
    k_syrk_tc(const __grid_constant__ CUtensorMap tmX, float* __restrict__ H, int n, int N,
              int accumulate) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Shared* sh = reinterpret_cast<Shared*>(smem + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int ti, tj;
  tri_decode(blockIdx.x, ti, tj);
  const bool diag = (ti == tj);
  const int i0 = ti * BT, j0 = tj * BT;
  const int nkb = (N + BK - 1) / BK;
  const int nch = (nkb + KCHUNK - 1) / KCHUNK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], 1);
    }
    mbar_init(&sh->tfull, 1);
    mbar_init(&sh->tempty, 4);                  // one arrival per epilogue warp
    sh->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&sh->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    tma_prefetch_desc(&tmX);
    const uint32_t bytes = diag ? SLAB_BYTES : STAGE_BYTES;
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % STAGES;
      const uint32_t par = (uint32_t)((kb / STAGES) & 1);
      if (!mbar_wait(&sh->empty[s], par ^ 1u)) {
        sh->abort = 1;
        break;
      }
      uint8_t* a = smem + s * STAGE_BYTES;
      uint8_t* b = a + SLAB_BYTES;
      mbar_arrive_expect_tx(&sh->full[s], bytes);
      for (int c = 0; c < 4; ++c) tma_load_2d(a + c * BOX_BYTES, &tmX, &sh->full[s], i0 + 64 * c, kb * BK);
      if (!diag)
        for (int c = 0; c < 4; ++c) tma_load_2d(b + c * BOX_BYTES, &tmX, &sh->full[s], j0 + 64 * c, kb * BK);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    for (int kb = 0; kb < nkb; ++kb) {
      const int kc = kb % KCHUNK, ch = kb / KCHUNK;
      if (kc == 0 && ch > 0) {                   // wait until chunk ch - 1 is drained
        if (!mbar_wait(&sh->tempty, (uint32_t)((ch - 1) & 1))) {
          sh->abort = 1;
          break;
        }
        tc_fence_after();
      }
      const int s = kb % STAGES;
      const uint32_t par = (uint32_t)((kb / STAGES) & 1);
      if (!mbar_wait(&sh->full[s], par)) {
        sh->abort = 1;
        break;
      }
      tc_fence_after();
      const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
      const uint32_t b_addr = diag ? a_addr : a_addr + SLAB_BYTES;
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        // MN-major SW128: LBO = stride between 64-channel boxes, SBO = 8 token rows
        const uint64_t bdesc = make_sw128_desc(b_addr + kk * 2048, BOX_BYTES, 1024);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint64_t adesc =
              make_sw128_desc(a_addr + h * 2 * BOX_BYTES + kk * 2048, BOX_BYTES, 1024);
          tc_mma_f16(tmem + h * 256, adesc, bdesc, IDESC, (kc | kk) != 0);
        }
      }
      tc_commit(&sh->empty[s]);
      if (kc == KCHUNK - 1 || kb == nkb - 1) tc_commit(&sh->tfull);
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: H (+)= chunk sums, lower triangle only
    const int quarter = warp - 4;
    for (int ch = 0; ch < nch; ++ch) {
      bool ok = mbar_wait(&sh->tfull, (uint32_t)(ch & 1));
      ok = __all_sync(0xffffffffu, ok) && !sh->abort;
      if (!ok) break;
      tc_fence_after();
      const bool add = accumulate || ch > 0;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int row = i0 + h * 128 + quarter * 32 + lane;
        const uint32_t tb = tmem + ((uint32_t)(quarter * 32) << 16) + h * 256;
        float* hrow = H + (int64_t)(row < n ? row : 0) * n;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          float v[32];
          tmem_ld32(tb + c * 32, v);
          const int jc = j0 + c * 32;
          if (row < n && jc <= row) {
            if (jc + 32 <= n && (n & 3) == 0) {
              float4* dst = reinterpret_cast<float4*>(hrow + jc);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 f = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                if (add) atomicAdd(dst + q, f);
                else dst[q] = f;
              }
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (jc + e < n) {
                  if (add) atomicAdd(hrow + jc + e, v[e]);
                  else hrow[jc + e] = v[e];
                }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->tempty);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace syrk
}  // namespace quip
