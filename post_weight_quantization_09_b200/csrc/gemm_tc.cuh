// fp32-accurate GEMM on the tcgen05 tensor cores from operands split into
// three bf16 pieces:  x = x0 + x1 + x2 (x0 = bf16(x), x1 = bf16(x - x0),
// x2 = bf16(x - x0 - x1)), so x is carried to ~24 significant bits.  The
// product sum_k a_k b_k is formed from the six piece products whose order is
// at most 2 (x_i y_j, i + j <= 2); the three dropped ones are below 2^-27
// relative.  bf16 x bf16 products are exact in the fp32 accumulator.
//
//   C[i][j] += alpha * sum_t sum_k A_pa(t)[i][k] * B_pb(t)[j][k]
//
// Both operands K-major (row-major [rows][K] bf16, piece p at row offset
// p * piece_rows), loaded by TMA as 64-wide K boxes with the 128-byte swizzle.
// Tile 128 x TN (TN = 256, or 128 / 64 for narrow outputs), one M=128 N=TN
// K=16 tcgen05.mma per 16 k.  Every piece is loaded once per 64-wide K block:
// the three A pieces together into one of two A slots (48 KB), the B pieces
// one at a time into a ring of B slots, B2 first; the terms that need a B
// piece run as soon as it lands: (0,2), then (1,1) (0,1), then (2,0) (1,0)
// (0,0), so within a K block the small terms come first.
// The tensor core's fp32 accumulation drops low bits (about one ulp of the
// running sum per MMA), so K is cut into chunks of KCP = 512 per piece, each
// accumulated in a fresh TMEM buffer.  With more than one chunk per tile the
// epilogue folds each chunk into an fp32 running sum kept in a second TMEM
// buffer (round-to-nearest adds) and adds the tile's sum to C once, at its
// last chunk; with one chunk per tile the two TMEM buffers take alternate
// tiles, so the next tile's products overlap this tile's epilogue.
// Bounded mbarrier waits as in the SYRK.
#pragma once

#include "common.cuh"

namespace quip {
namespace sgemm {

// Tile N width BN: 256, or 128 / 64 for narrow outputs (more tiles, more CTAs).
constexpr int BM = 128, BN = 256, BK = 64;
constexpr int A_PIECE_BYTES = BM * BK * 2;        // 16 KB
constexpr int A_BYTES = 3 * A_PIECE_BYTES;        // one A slot: the three pieces
constexpr int A_SLOTS = 2;
template <int TN> __host__ __device__ constexpr int b_bytes() { return TN * BK * 2; }
template <int TN> __host__ __device__ constexpr int b_slots() { return TN == 256 ? 4 : 8; }
template <int TN> __host__ __device__ constexpr int smem_bytes() {
  return A_SLOTS * A_BYTES + b_slots<TN>() * b_bytes<TN>() + 1024 + 256;
}
constexpr int SMEM_BYTES = smem_bytes<BN>();

struct Params {
  float* C;
  int64_t ldc;
  int M, N;                // output extent
  int K;                   // K per piece (multiple of 64)
  int a_piece_rows, b_piece_rows;   // row offset between pieces in the maps
  int a_row0, b_row0;      // first row of the operand views in the maps
  int a_k0, b_k0;          // first K column of the operand views
  float alpha;
  int upper_only;          // 1: skip tiles with no element i <= j (C square views)
  int tiles_n;             // number of tile columns
};

constexpr int KCP = 512;                           // K per piece per accumulation chunk

struct Shared {
  uint64_t full_a[A_SLOTS];
  uint64_t empty_a[A_SLOTS];
  uint64_t full_b[8];
  uint64_t empty_b[8];
  uint64_t tfull[2];       // accumulator buffer complete (MMA -> epilogue)
  uint64_t tempty[2];      // accumulator buffer drained (epilogue -> MMA)
  uint32_t tmem_base;
  int abort;
};

// Tile t of the grid (row-major over tiles_m x tiles_n); false if skipped.
template <int TN>
__device__ __forceinline__ bool tile_coords(const Params& p, int t, int& i0, int& j0) {
  const int ti = t / p.tiles_n, tj = t % p.tiles_n;
  i0 = ti * BM;
  j0 = tj * TN;
  return !(p.upper_only && i0 > j0 + TN - 1);
}

// Persistent: CTA b handles tiles b, b + gridDim.x, ...  Warp 0 lane 0: TMA
// producer; warp 1 lane 0: MMA issuer; warps 4..7: epilogue (warp w reads
// TMEM lanes 32 (w - 4)..; one output row per thread, TN columns).
// Accumulator buffers: with one chunk per tile (K <= KCP) buffer (local tile
// index & 1); otherwise buffer 0 takes every chunk and buffer 1 holds the
// running sum.
template <int TN>
__global__ void __launch_bounds__(256, 1)
    k_gemm_split_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    Params p, int ntiles) {
  constexpr int B_BYTES = b_bytes<TN>();
  constexpr int NB = b_slots<TN>();
  constexpr uint32_t IDESC = make_idesc_bf16(BM, TN, 0, 0);
  constexpr uint32_t TCOLS = 2 * TN;
  extern __shared__ uint8_t smem_raw[];
  pdl_wait_then_release();
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sa = smem;                                // A slots
  uint8_t* sb = smem + A_SLOTS * A_BYTES;            // B slots
  Shared* sh = reinterpret_cast<Shared*>(sb + NB * B_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunk = (p.K + KCP - 1) / KCP;
  const bool single = nchunk == 1;
  constexpr int nbp = 3;                            // B pieces

  if (threadIdx.x == 0) {
    for (int s = 0; s < A_SLOTS; ++s) {
      mbar_init(&sh->full_a[s], 1);
      mbar_init(&sh->empty_a[s], 1);
    }
    for (int s = 0; s < NB; ++s) {
      mbar_init(&sh->full_b[s], 1);
      mbar_init(&sh->empty_b[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh->tfull[b], 1);
      mbar_init(&sh->tempty[b], 4);                 // one arrival per epilogue warp
    }
    sh->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&sh->tmem_base, TCOLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    int ka = 0, kb = 0;                             // A-slot and B-slot counters
    for (int t = blockIdx.x; t < ntiles && !sh->abort; t += gridDim.x) {
      int i0, j0;
      if (!tile_coords<TN>(p, t, i0, j0)) continue;
      for (int k = 0; k < p.K && !sh->abort; k += BK, ++ka) {
        const int s = ka % A_SLOTS;
        if (!mbar_wait(&sh->empty_a[s], (uint32_t)(((ka / A_SLOTS) & 1) ^ 1))) {
          sh->abort = 1;
          break;
        }
        mbar_arrive_expect_tx(&sh->full_a[s], A_BYTES);
#pragma unroll
        for (int pa = 0; pa < 3; ++pa)
          tma_load_2d(sa + s * A_BYTES + pa * A_PIECE_BYTES, &tmA, &sh->full_a[s], p.a_k0 + k,
                      pa * p.a_piece_rows + p.a_row0 + i0);
        for (int pb = nbp - 1; pb >= 0; --pb, ++kb) {
          const int r = kb % NB;
          if (!mbar_wait(&sh->empty_b[r], (uint32_t)(((kb / NB) & 1) ^ 1))) {
            sh->abort = 1;
            break;
          }
          mbar_arrive_expect_tx(&sh->full_b[r], B_BYTES);
          tma_load_2d(sb + r * B_BYTES, &tmB, &sh->full_b[r], p.b_k0 + k, pb * p.b_piece_rows + p.b_row0 + j0);
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    int ka = 0, kb = 0, gc = 0, lt = 0;             // gc: chunks, lt: tiles of this CTA
    for (int t = blockIdx.x; t < ntiles && !sh->abort; t += gridDim.x) {
      int i0, j0;
      if (!tile_coords<TN>(p, t, i0, j0)) continue;
      for (int c = 0; c < nchunk && !sh->abort; ++c, ++gc) {
        // single chunk: buffer lt & 1, its use count lt >> 1; else buffer 0, use count gc
        const int buf = single ? (lt & 1) : 0;
        const int use = single ? (lt >> 1) : gc;
        if (!mbar_wait(&sh->tempty[buf], (uint32_t)((use & 1) ^ 1))) {
          sh->abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(buf * TN);
        const int kc0 = c * KCP, kc1 = min(p.K, kc0 + KCP);
        bool first = true;
        for (int k = kc0; k < kc1 && !sh->abort; k += BK, ++ka) {
          const int s = ka % A_SLOTS;
          if (!mbar_wait(&sh->full_a[s], (uint32_t)((ka / A_SLOTS) & 1))) {
            sh->abort = 1;
            break;
          }
          const uint32_t a_base = smem_u32(sa + s * A_BYTES);
          for (int pb = nbp - 1; pb >= 0; --pb, ++kb) {
            const int r = kb % NB;
            if (!mbar_wait(&sh->full_b[r], (uint32_t)((kb / NB) & 1))) {
              sh->abort = 1;
              break;
            }
            tc_fence_after();
            const uint32_t b_addr = smem_u32(sb + r * B_BYTES);
            // the A pieces pa with pa + pb <= 2, larger pa (smaller term) first
            for (int pa = 2 - pb; pa >= 0; --pa) {
              const uint32_t a_addr = a_base + pa * A_PIECE_BYTES;
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk) {
                // K-major SW128: 8-row groups 1024 B apart; K advances 32 B per 16 elements
                const uint64_t adesc = make_sw128_desc(a_addr + kk * 32, 16, 1024);
                const uint64_t bdesc = make_sw128_desc(b_addr + kk * 32, 16, 1024);
                tc_mma_f16(acc, adesc, bdesc, IDESC, first ? 0u : 1u);
                first = false;
              }
            }
            tc_commit(&sh->empty_b[r]);
          }
          tc_commit(&sh->empty_a[s]);
        }
        tc_commit(&sh->tfull[buf]);
      }
      ++lt;
    }
  } else if (warp >= 4) {
    const int quarter = warp - 4;
    int gc = 0, lt = 0;
    bool stop = false;
    for (int t = blockIdx.x; t < ntiles && !stop; t += gridDim.x) {
      int i0, j0;
      if (!tile_coords<TN>(p, t, i0, j0)) continue;
      const int row = i0 + quarter * 32 + lane;
      const bool rok = row < p.M;
      float* crow = p.C + (int64_t)(rok ? row : 0) * p.ldc;
      const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
      const bool vec = (p.ldc & 3) == 0;
      for (int c = 0; c < nchunk; ++c, ++gc) {
        const int buf = single ? (lt & 1) : 0;
        const int use = single ? (lt >> 1) : gc;
        bool ok = mbar_wait(&sh->tfull[buf], (uint32_t)(use & 1));
        ok = __all_sync(0xffffffffu, ok) && !sh->abort;
        if (!ok) {
          stop = true;
          break;
        }
        tc_fence_after();
        const bool first = c == 0, last = c == nchunk - 1;
        const uint32_t tb = tmem + lanes + (uint32_t)(buf * TN);
#pragma unroll 1
        for (int c8 = 0; c8 < TN / 32; ++c8) {
          float v[32];
          tmem_ld32(tb + c8 * 32, v);
          if (!single) {
            if (!first) {
              float su[32];
              tmem_ld32(tmem + lanes + TN + c8 * 32, su);
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] += su[e];
            }
            if (!last) {
              tmem_st32(tmem + lanes + TN + c8 * 32, v);
              continue;
            }
          }
          // C += alpha * sum through fire-and-forget vector reductions in L2
          const int jc = j0 + c8 * 32;
          if (rok && jc < p.N) {
            if (vec && jc + 32 <= p.N) {
              float4* dst = reinterpret_cast<float4*>(crow + jc);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                atomicAdd(dst + q, make_float4(p.alpha * v[4 * q], p.alpha * v[4 * q + 1],
                                               p.alpha * v[4 * q + 2], p.alpha * v[4 * q + 3]));
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (jc + e < p.N) atomicAdd(crow + jc + e, p.alpha * v[e]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->tempty[buf]);
      }
      ++lt;
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TCOLS);
  }
}

}  // namespace sgemm

// fp32 -> three bf16 pieces, row-major copy: out[p][i][k] for p = 0..2.
// Rows `rows`, K `cols` of the source (row stride lds); output row stride
// ldo, piece stride piece_elems.
// out[p][j][i] = piece_p(U[i][j]) for i < j (strict upper), 0 otherwise:
// the transposed, split copy of the LDL factor that LDLQ's trailing GEMM
// reads as its K-major B operand; outf[j][i] = U[i][j] (same zeros), the
// fp32 transposed copy the LDLQ block kernel reads.  32 x 32 tiles through
// shared memory; source tiles below the diagonal are not read (all their
// outputs are zero); each thread writes two adjacent outputs.  n even.
__global__ void __launch_bounds__(256) k_split_upper_transposed(const float* __restrict__ U,
                                                                int64_t ldu, int64_t n,
                                                                __nv_bfloat16* __restrict__ out,
                                                                float* __restrict__ outf) {
  __shared__ float t[32][33];
  const int64_t bi = blockIdx.y, bj = blockIdx.x;   // source tile (rows bi, cols bj)
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const bool below = bi > bj;
  if (!below) {
    for (int r = ty; r < 32; r += 8) {
      const int64_t i = bi * 32 + r, j = bj * 32 + tx;
      t[r][tx] = (i < n && j < n && i < j) ? U[i * ldu + j] : 0.f;
    }
  }
  __syncthreads();
  const int64_t pn = n * n;
  const int i2 = 2 * (tx & 15);
  for (int rr = 2 * ty + (tx >> 4); rr < 32; rr += 16) {
    const int64_t j = bj * 32 + rr, i = bi * 32 + i2;   // out row j, columns i, i + 1
    if (j >= n || i >= n) continue;
    const float a = below ? 0.f : t[i2][rr], b = below ? 0.f : t[i2 + 1][rr];
    __nv_bfloat16 pa[3], pb[3];
    split3(a, pa[0], pa[1], pa[2]);
    split3(b, pb[0], pb[1], pb[2]);
#pragma unroll
    for (int p = 0; p < 3; ++p) {
      __nv_bfloat162 v;
      v.x = pa[p], v.y = pb[p];
      *reinterpret_cast<__nv_bfloat162*>(out + p * pn + j * n + i) = v;
    }
    *reinterpret_cast<float2*>(outf + j * n + i) = make_float2(a, b);
  }
}

}  // namespace quip
