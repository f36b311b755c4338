// Kronecker-factor products of the incoherence transform on the tcgen05
// tensor cores (QuIP, Introduction and "Incoherence processing": the random
// orthogonal matrix is a Kronecker product A (x) B of two small random
// orthogonal factors).  Applied to the columns of an R x c matrix X
// (R = p q, the m side of W), (A (x) B) X is two batched products:
//
//   T_a' = B X_a'   for each slab X_a' = X[a' q : a' q + q, :]      (q x q) (q x c)
//   Y    = A T      with T viewed as p x (q c)                      (p x p) (p x q c)
//
// (transposed factors for the inverse).  Both have the form
//
//   Y[z] = F X[z],   F: d x d (the factor),  X[z]: d x N (a slab of the data),
//
// computed as its transpose Y[z]^T = X[z]^T F^T on the tensor core: a tile
// is 128 data columns (the MMA's M, the data's rows of 128 columns being
// MN-major for it) against the whole factor (the MMA's N = d rounded up to
// 16, at most 256; K-major), so the data is read once and the factor is not
// padded to 128 rows.  fp32 accuracy comes from bf16 pieces: the factor is
// carried as three pieces f = f0 + f1 + f2 (x0 = bf16(x), x1 = bf16(x - x0),
// ...), the data as three pieces, or as one when it is bf16 already (the
// layer's weights); the terms f_i x_j with i + j <= 2 are formed, smallest
// first (bf16 x bf16 products are exact in the fp32 accumulator).
//
// K runs in 64-row blocks (the factor's columns past d arrive as zeros from
// TMA, so rows of the data past the slab contribute nothing).  Every piece
// is loaded once per K block: the three factor pieces (NF x 64 each, 128-byte
// swizzle) into one of two F slots, the data pieces (64 rows x 128 columns
// each, as two 64-column boxes, 128-byte swizzle) into a ring; each term is
// four M=128 N=NF K=16 tcgen05.mma.  Persistent CTAs walk the tiles (slab,
// column tile); two TMEM accumulators (2 x NF columns) let the epilogue of
// one tile overlap the next tile's products.  The epilogue (warps 4..7) has
// one data column per thread and writes, for each output row, 32
// consecutive columns per warp (full 128-byte lines): fp32, or the three
// bf16 pieces of the result (the next product's data operand).
// Every mbarrier wait is bounded (common.cuh); on a timeout the CTA records
// QUIP_ERR_TIMEOUT and stops.
#pragma once

#include "common.cuh"

namespace quip {
namespace kron {

constexpr int BM = 128, BK = 64;                  // data columns per tile, K block
constexpr int D_BOX = 64 * BK * 2;                // 8 KB: 64 data columns x 64 rows
constexpr int D_BYTES = 2 * D_BOX;                // 16 KB: a data piece tile
constexpr int F_SLOTS = 2;
constexpr int MAX_D_SLOTS = 8;
constexpr int SMEM_LIMIT = 227 * 1024;
__host__ __device__ constexpr int f_piece_bytes(int nf) { return nf * BK * 2; }
__host__ __device__ constexpr int f_slot_bytes(int nf) { return 3 * f_piece_bytes(nf); }
__host__ __device__ constexpr int d_slots(int nf) {
  return (SMEM_LIMIT - 1024 - 256 - F_SLOTS * f_slot_bytes(nf)) / D_BYTES > MAX_D_SLOTS
             ? MAX_D_SLOTS
             : (SMEM_LIMIT - 1024 - 256 - F_SLOTS * f_slot_bytes(nf)) / D_BYTES;
}
__host__ __device__ constexpr int smem_bytes(int nf) {
  return F_SLOTS * f_slot_bytes(nf) + d_slots(nf) * D_BYTES + 1024 + 256;
}

enum { OUT_F32 = 0, OUT_PIECES = 1 };

struct Params {
  int d;                     // factor size: output rows per slab and contraction length
  int nf;                    // MMA N: d rounded up to 16 (<= 256)
  int N;                     // data columns per slab
  int slabs;
  int f_piece_rows;          // row offset between factor pieces in the factor map
  int x_pieces;              // 1 or 3
  int64_t x_piece_rows;      // row offset between data pieces in the data map
  int64_t x_slab_rows;       // row offset between slabs in the data map
  float* Y;                  // OUT_F32: Y[z][a][n] at Y + (z * y_slab_rows + a) * ldy + n
  __nv_bfloat16* Yp;         // OUT_PIECES: piece f at Yp + f * y_piece_elems + (same offset)
  int64_t ldy, y_slab_rows, y_piece_elems;
  int tiles_m;               // column tiles per slab
};

struct Shared {
  uint64_t full_f[F_SLOTS];
  uint64_t empty_f[F_SLOTS];
  uint64_t full_d[MAX_D_SLOTS];
  uint64_t empty_d[MAX_D_SLOTS];
  uint64_t tfull[2];       // accumulator b complete (MMA -> epilogue)
  uint64_t tempty[2];      // accumulator b drained (epilogue -> MMA)
  uint32_t tmem_base;
  int abort;
};

__global__ void __launch_bounds__(256, 1)
    k_kron_tc(const __grid_constant__ CUtensorMap tmF, const __grid_constant__ CUtensorMap tmX,
              Params p, int mode) {
  extern __shared__ uint8_t smem_raw[];
  pdl_wait_then_release();
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int FSB = f_slot_bytes(p.nf), FPB = f_piece_bytes(p.nf), NDS = d_slots(p.nf);
  uint8_t* sf = smem;                                // F slots (three factor pieces each)
  uint8_t* sd = smem + F_SLOTS * FSB;                // data ring (one piece each)
  Shared* sh = reinterpret_cast<Shared*>(sd + NDS * D_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = p.tiles_m * p.slabs;
  const int nkb = (p.d + BK - 1) / BK;
  // M = 128, N = nf, A (data) MN-major, B (factor) K-major
  const uint32_t idesc = make_idesc_bf16(BM, p.nf, /*a_mn=*/1, /*b_mn=*/0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < F_SLOTS; ++i) {
      mbar_init(&sh->full_f[i], 1);
      mbar_init(&sh->empty_f[i], 1);
    }
    for (int i = 0; i < NDS; ++i) {
      mbar_init(&sh->full_d[i], 1);
      mbar_init(&sh->empty_d[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh->tfull[b], 1);
      mbar_init(&sh->tempty[b], 4);                // one arrival per epilogue warp
    }
    sh->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&sh->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  // Per K block: the three factor pieces into an F slot, then the data
  // pieces, the last first, each into the ring; the terms that need a data
  // piece run once it has landed: piece 2 with factor piece 0, piece 1 with
  // 1 and 0, piece 0 with 2, 1 and 0 (a one-piece data operand has only
  // piece 0), so the small terms come first.
  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    tma_prefetch_desc(&tmF);
    tma_prefetch_desc(&tmX);
    int kf = 0, kd = 0;
    for (int t = blockIdx.x; t < ntiles && !sh->abort; t += gridDim.x) {
      const int z = t / p.tiles_m, m0 = (t % p.tiles_m) * BM;
      for (int k = 0; k < nkb && !sh->abort; ++k, ++kf) {
        const int s = kf % F_SLOTS;
        if (!mbar_wait(&sh->empty_f[s], (uint32_t)(((kf / F_SLOTS) & 1) ^ 1))) {
          sh->abort = 1;
          break;
        }
        mbar_arrive_expect_tx(&sh->full_f[s], (uint32_t)FSB);
#pragma unroll
        for (int pf = 0; pf < 3; ++pf)
          tma_load_2d(sf + s * FSB + pf * FPB, &tmF, &sh->full_f[s], k * BK, pf * p.f_piece_rows);
        for (int px = p.x_pieces - 1; px >= 0; --px, ++kd) {
          const int r = kd % NDS;
          if (!mbar_wait(&sh->empty_d[r], (uint32_t)(((kd / NDS) & 1) ^ 1))) {
            sh->abort = 1;
            break;
          }
          mbar_arrive_expect_tx(&sh->full_d[r], D_BYTES);
          const int64_t xr = px * p.x_piece_rows + z * p.x_slab_rows + (int64_t)k * BK;
#pragma unroll
          for (int c = 0; c < 2; ++c)
            tma_load_2d(sd + r * D_BYTES + c * D_BOX, &tmX, &sh->full_d[r], m0 + 64 * c, (int)xr);
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    int kf = 0, kd = 0, lt = 0;                      // lt: this CTA's tile counter
    for (int t = blockIdx.x; t < ntiles && !sh->abort; t += gridDim.x, ++lt) {
      const int b = lt & 1;
      if (!mbar_wait(&sh->tempty[b], (uint32_t)(((lt >> 1) & 1) ^ 1))) {
        sh->abort = 1;
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(b * 256);
      bool first = true;
      for (int k = 0; k < nkb && !sh->abort; ++k, ++kf) {
        const int s = kf % F_SLOTS;
        if (!mbar_wait(&sh->full_f[s], (uint32_t)((kf / F_SLOTS) & 1))) {
          sh->abort = 1;
          break;
        }
        const uint32_t f_base = smem_u32(sf + s * FSB);
        for (int px = p.x_pieces - 1; px >= 0; --px, ++kd) {
          const int r = kd % NDS;
          if (!mbar_wait(&sh->full_d[r], (uint32_t)((kd / NDS) & 1))) {
            sh->abort = 1;
            break;
          }
          tc_fence_after();
          const uint32_t d_addr = smem_u32(sd + r * D_BYTES);
          for (int pf = 2 - px; pf >= 0; --pf) {
            const uint32_t f_addr = f_base + pf * FPB;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              // A (data): MN-major, the two 64-column boxes 8 KB apart (LBO),
              // 8 rows 1024 B (SBO), K advances 16 rows = 2048 B;
              // B (factor): K-major, 8-row groups 1024 B apart, K advances 32 B per 16
              const uint64_t adesc = make_sw128_desc(d_addr + kk * 2048, D_BOX, 1024);
              const uint64_t bdesc = make_sw128_desc(f_addr + kk * 32, 16, 1024);
              tc_mma_f16(acc, adesc, bdesc, idesc, first ? 0u : 1u);
              first = false;
            }
          }
          tc_commit(&sh->empty_d[r]);
        }
        tc_commit(&sh->empty_f[s]);
      }
      tc_commit(&sh->tfull[b]);
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: one data column per thread, output rows a
    const int quarter = warp - 4;
    int lt = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
      const int b = lt & 1;
      bool ok = mbar_wait(&sh->tfull[b], (uint32_t)((lt >> 1) & 1));
      ok = __all_sync(0xffffffffu, ok) && !sh->abort;
      if (!ok) break;
      tc_fence_after();
      const int z = t / p.tiles_m, m0 = (t % p.tiles_m) * BM;
      const int col = m0 + quarter * 32 + lane;
      const bool live = col < p.N;
      const int64_t base = (int64_t)z * p.y_slab_rows * p.ldy + (live ? col : 0);
      const uint32_t tb = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * 256);
#pragma unroll 1
      for (int a0 = 0; a0 < p.nf; a0 += 32) {
        float v[32];
        if (a0 + 32 <= p.nf) {
          tmem_ld32(tb + a0, v);
        } else {                                     // nf % 32 == 16: the last 16 columns
          float h[16];
          tmem_ld16(tb + a0, h);
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = h[e], v[16 + e] = 0.f;
        }
        if (!live) continue;
        if (mode == OUT_F32) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (a0 + e < p.d) p.Y[base + (int64_t)(a0 + e) * p.ldy] = v[e];
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if (a0 + e < p.d) {
              const __nv_bfloat16 h0 = __float2bfloat16_rn(v[e]);
              const float r1 = v[e] - __bfloat162float(h0);
              const __nv_bfloat16 h1 = __float2bfloat16_rn(r1);
              const int64_t o = base + (int64_t)(a0 + e) * p.ldy;
              p.Yp[o] = h0;
              p.Yp[p.y_piece_elems + o] = h1;
              p.Yp[2 * p.y_piece_elems + o] = __float2bfloat16_rn(r1 - __bfloat162float(h1));
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
    tmem_dealloc(tmem, 512);
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
