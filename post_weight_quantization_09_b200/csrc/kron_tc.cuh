// Kronecker-factor products of the incoherence transform on the tcgen05
// tensor cores (QuIP, Introduction and "Incoherence processing": the random
// orthogonal matrix is a Kronecker product A (x) B of two small random
// orthogonal factors).  Applied to the columns of an R x c matrix X
// (R = p q, the m side of W), (A (x) B) X is two batched products:
//
//   T_a' = B X_a'   for each slab X_a' = X[a' q : a' q + q, :]      (q x q) (q x c)
//   Y    = A T      with T viewed as p x (q c)                      (p x p) (p x q c)
//
// (transposed factors for the inverse).  Both have the same form,
//
//   Y[z] = F X[z],   F: M x K (the factor),  X[z]: K x N (a slab of the data),
//
// with the data in its natural row-major layout, i.e. MN-major for the
// tensor core.  fp32 accuracy comes from bf16 pieces: the factor is carried
// as three pieces f = f0 + f1 + f2 (x0 = bf16(x), x1 = bf16(x - x0), ...),
// the data as three pieces, or as one when it is bf16 already (the layer's
// weights); the terms f_i x_j with i + j <= 2 are formed, smallest first
// (bf16 x bf16 products are exact in the fp32 accumulator).
//
// Tile 128 (M) x 256 (N), K in 64-row blocks (the factor's columns past K
// arrive as zeros from TMA, so rows of the data past the slab contribute
// nothing); per (K block, term) one stage of a 4-deep TMA ring holds the
// factor piece (128 x 64, K-major, 128-byte swizzle) and the data piece
// (64 x 256 as four 64-column boxes, MN-major, 128-byte swizzle), consumed
// by four M=128 N=256 K=16 tcgen05.mma.  Persistent CTAs walk the tiles
// (slab, N tile, M tile); two TMEM accumulators (2 x 256 columns) let the
// epilogue of one tile overlap the next tile's products.  The epilogue
// (warps 4..7, one output row per thread) stores fp32 or the three bf16
// pieces of the result (the next product's data operand).
// Every mbarrier wait is bounded (common.cuh); on a timeout the CTA records
// QUIP_ERR_TIMEOUT and stops.
#pragma once

#include "common.cuh"

namespace quip {
namespace kron {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;              // 16 KB: factor piece tile
constexpr int BOX_BYTES = 64 * BK * 2;            // 8 KB: 64 data columns x 64 rows
constexpr int B_BYTES = 4 * BOX_BYTES;            // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr uint32_t IDESC = make_idesc_bf16(BM, BN, /*a_mn=*/0, /*b_mn=*/1);

enum { OUT_F32 = 0, OUT_PIECES = 1 };

struct Params {
  int M, K, N;               // per slab: output rows (factor rows), contraction, columns
  int slabs;
  int f_piece_rows;          // row offset between factor pieces in the factor map
  int x_pieces;              // 1 or 3
  int64_t x_piece_rows;      // row offset between data pieces in the data map
  int64_t x_slab_rows;       // row offset between slabs in the data map
  float* Y;                  // OUT_F32: Y[z][m][n] at Y + (z * y_slab_rows + m) * ldy + n
  __nv_bfloat16* Yp;         // OUT_PIECES: piece f at Yp + f * y_piece_elems + (same offset)
  int64_t ldy, y_slab_rows, y_piece_elems;
  int tiles_m, tiles_n;
};

struct Shared {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];       // accumulator b complete (MMA -> epilogue)
  uint64_t tempty[2];      // accumulator b drained (epilogue -> MMA)
  uint32_t tmem_base;
  int abort;
};

// Terms (factor piece, data piece), smallest first: three-piece data
// (2,0) (1,1) (0,2) (1,0) (0,1) (0,0); one-piece data (2,0) (1,0) (0,0).
__device__ __forceinline__ void term(int xp, int t, int& pf, int& px) {
  if (xp == 3) {
    pf = (int)((0x001012u >> (4 * t)) & 0xFu);
    px = (int)((0x010210u >> (4 * t)) & 0xFu);
  } else {
    pf = 2 - t;
    px = 0;
  }
}

__device__ __forceinline__ void tile_of(const Params& p, int t, int& z, int& m0, int& n0) {
  const int tm = t % p.tiles_m;
  const int rest = t / p.tiles_m;
  const int tn = rest % p.tiles_n;
  z = rest / p.tiles_n;
  m0 = tm * BM;
  n0 = tn * BN;
}

__global__ void __launch_bounds__(256, 1)
    k_kron_tc(const __grid_constant__ CUtensorMap tmF, const __grid_constant__ CUtensorMap tmX,
              Params p, int mode) {
  extern __shared__ uint8_t smem_raw[];
  pdl_wait_then_release();
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Shared* sh = reinterpret_cast<Shared*>(smem + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = p.tiles_m * p.tiles_n * p.slabs;
  const int nkb = (p.K + BK - 1) / BK;
  const int nterm = p.x_pieces == 3 ? 6 : 3;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh->tfull[b], 1);
      mbar_init(&sh->tempty[b], 4);                // one arrival per epilogue warp
    }
    sh->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&sh->tmem_base, 2 * BN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    tma_prefetch_desc(&tmF);
    tma_prefetch_desc(&tmX);
    int it = 0;
    for (int t = blockIdx.x; t < ntiles && !sh->abort; t += gridDim.x) {
      int z, m0, n0;
      tile_of(p, t, z, m0, n0);
      for (int kb = 0; kb < nkb && !sh->abort; ++kb) {
        for (int tt = 0; tt < nterm; ++tt, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&sh->empty[s], (uint32_t)(((it / STAGES) & 1) ^ 1))) {
            sh->abort = 1;
            break;
          }
          int pf, px;
          term(p.x_pieces, tt, pf, px);
          uint8_t* a = smem + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&sh->full[s], STAGE_BYTES);
          tma_load_2d(a, &tmF, &sh->full[s], kb * BK, pf * p.f_piece_rows + m0);
          const int64_t xr = px * p.x_piece_rows + z * p.x_slab_rows + (int64_t)kb * BK;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tma_load_2d(a + A_BYTES + c * BOX_BYTES, &tmX, &sh->full[s], n0 + 64 * c, (int)xr);
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    int it = 0, lt = 0;                              // lt: this CTA's tile counter
    for (int t = blockIdx.x; t < ntiles && !sh->abort; t += gridDim.x, ++lt) {
      const int b = lt & 1;
      if (!mbar_wait(&sh->tempty[b], (uint32_t)(((lt >> 1) & 1) ^ 1))) {
        sh->abort = 1;
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(b * BN);
      bool first = true;
      for (int kb = 0; kb < nkb && !sh->abort; ++kb) {
        for (int tt = 0; tt < nterm; ++tt, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&sh->full[s], (uint32_t)((it / STAGES) & 1))) {
            sh->abort = 1;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // A: K-major, 8-row groups 1024 B apart, K advances 32 B per 16;
            // B: MN-major, 64-column boxes 8 KB apart (LBO), 8 rows 1024 B (SBO),
            // K advances 16 rows = 2048 B
            const uint64_t adesc = make_sw128_desc(a_addr + k * 32, 16, 1024);
            const uint64_t bdesc = make_sw128_desc(b_addr + k * 2048, BOX_BYTES, 1024);
            tc_mma_f16(acc, adesc, bdesc, IDESC, first ? 0u : 1u);
            first = false;
          }
          tc_commit(&sh->empty[s]);
        }
      }
      tc_commit(&sh->tfull[b]);
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: one output row per thread
    const int quarter = warp - 4;
    int lt = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
      const int b = lt & 1;
      bool ok = mbar_wait(&sh->tfull[b], (uint32_t)((lt >> 1) & 1));
      ok = __all_sync(0xffffffffu, ok) && !sh->abort;
      if (!ok) break;
      tc_fence_after();
      int z, m0, n0;
      tile_of(p, t, z, m0, n0);
      const int m = m0 + quarter * 32 + lane;
      const bool live = m < p.M;
      const int64_t off = ((int64_t)z * p.y_slab_rows + (live ? m : 0)) * p.ldy;
      const uint32_t tb = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(tb + c * 32, v);
        const int nc = n0 + c * 32;
        if (!live || nc >= p.N) continue;
        const bool full32 = nc + 32 <= p.N;
        if (mode == OUT_F32) {
          float* y = p.Y + off + nc;
          if (full32) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              reinterpret_cast<float4*>(y)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (nc + e < p.N) y[e] = v[e];
          }
        } else {
          // three bf16 pieces, packed two per 32-bit word as they are formed
          uint32_t w[3][16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            uint32_t h[3][2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const __nv_bfloat16 h0 = __float2bfloat16_rn(v[e + u]);
              const float r1 = v[e + u] - __bfloat162float(h0);
              const __nv_bfloat16 h1 = __float2bfloat16_rn(r1);
              const __nv_bfloat16 h2 = __float2bfloat16_rn(r1 - __bfloat162float(h1));
              h[0][u] = __bfloat16_as_ushort(h0);
              h[1][u] = __bfloat16_as_ushort(h1);
              h[2][u] = __bfloat16_as_ushort(h2);
            }
#pragma unroll
            for (int f = 0; f < 3; ++f) w[f][e / 2] = h[f][0] | (h[f][1] << 16);
          }
#pragma unroll
          for (int f = 0; f < 3; ++f) {
            __nv_bfloat16* y = p.Yp + f * p.y_piece_elems + off + nc;
            if (full32) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                reinterpret_cast<uint4*>(y)[q] = make_uint4(w[f][4 * q], w[f][4 * q + 1], w[f][4 * q + 2], w[f][4 * q + 3]);
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (nc + e < p.N)
                  y[e] = __ushort_as_bfloat16((unsigned short)((w[f][e / 2] >> (16 * (e & 1))) & 0xFFFFu));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->tempty[b]);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * BN);
  }
}

}  // namespace kron

// Three bf16 pieces of a d x d fp32 factor F, or of its transpose:
// out[f][i][j] = piece_f(trans ? F[j][i] : F[i][j]), row stride ld (>= d; the
// padding columns are never read: the tensor maps end at column d), piece
// stride d * ld.
__global__ void k_split_factor(const float* __restrict__ F, int d, int trans, int ld,
                               __nv_bfloat16* __restrict__ out) {
  const int64_t n = (int64_t)d * d, pn = (int64_t)d * ld;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(e / d), j = (int)(e % d);
    const float x = trans ? F[(int64_t)j * d + i] : F[e];
    const __nv_bfloat16 h0 = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(h0);
    const __nv_bfloat16 h1 = __float2bfloat16_rn(r1);
    const int64_t o = (int64_t)i * ld + j;
    out[o] = h0;
    out[pn + o] = h1;
    out[2 * pn + o] = __float2bfloat16_rn(r1 - __bfloat162float(h1));
  }
}

// Three bf16 pieces of an fp32 matrix (rows x cols, row stride ld) into
// out[f][r][c] (row stride cols, piece stride rows * cols); four elements
// per thread (cols % 4 == 0, 16-byte aligned rows).
__global__ void k_split_rows3(const float* __restrict__ in, int64_t ld, int64_t rows, int64_t cols,
                              __nv_bfloat16* __restrict__ out) {
  const int64_t total4 = rows * cols / 4, pn = rows * cols;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total4;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = (4 * e) / cols, c = (4 * e) % cols;
    const float4 v = *reinterpret_cast<const float4*>(in + r * ld + c);
    const float x[4] = {v.x, v.y, v.z, v.w};
    __nv_bfloat16 pc[3][4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_bfloat16 h0 = __float2bfloat16_rn(x[k]);
      const float r1 = x[k] - __bfloat162float(h0);
      const __nv_bfloat16 h1 = __float2bfloat16_rn(r1);
      pc[0][k] = h0;
      pc[1][k] = h1;
      pc[2][k] = __float2bfloat16_rn(r1 - __bfloat162float(h1));
    }
#pragma unroll
    for (int f = 0; f < 3; ++f)
      *reinterpret_cast<uint2*>(out + f * pn + r * cols + c) = *reinterpret_cast<const uint2*>(pc[f]);
  }
}

}  // namespace quip
