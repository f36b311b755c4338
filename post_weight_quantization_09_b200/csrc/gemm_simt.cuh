// Strided, batched fp32 FFMA GEMM on the CUDA cores:
//   C_b[i][j] = alpha * sum_k A_b[i][k] * B_b[k][j] + beta * C_b[i][j]
// with arbitrary element strides for every operand (so transposes are free).
// Used where the contraction is small or must stay in fp32: the Kronecker
// factors of the incoherence transform and the fp32-input Hessian.  With
// Acc = double the products and sums are taken in fp64 (inputs converted on
// the way into shared memory, the result rounded to fp32 once): the Hessian's
// Kronecker transform uses it, because an fp32 sum over a Haar factor's row
// carries an error proportional to the largest entries of H into every entry
// of the transformed H, including its small-eigenvalue directions.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace quip {

struct GemmArgs {
  int64_t M, N, K;
  float alpha, beta;              // beta == 0: C is not read
  const void* A;
  int64_t sam, sak, sab;          // A[b][i][k] = A[b*sab + i*sam + k*sak]
  const void* B;
  int64_t sbk, sbn, sbb;          // B[b][k][j] = B[b*sbb + k*sbk + j*sbn]
  float* C;
  int64_t scm, scn, scb;          // C[b][i][j]
  int tri;                        // 0 all tiles, 1 tiles with ti >= tj, 2 ti <= tj
};

constexpr int SG_BM = 64, SG_BN = 64, SG_BK = 16;

// 256 threads; each computes a 4 x 4 block of the 64 x 64 tile.
template <typename Acc, typename T>
__device__ __forceinline__ Acc to_acc(T x) {
  if constexpr (std::is_same<T, double>::value) return (Acc)x;
  else return (Acc)to_f32<T>(x);
}

template <typename TA, typename TB, typename Acc = float>
__global__ void __launch_bounds__(256) k_gemm_simt(GemmArgs g) {
  const int64_t ti = blockIdx.y, tj = blockIdx.x, b = blockIdx.z;
  if (g.tri == 1 && ti < tj) return;
  if (g.tri == 2 && ti > tj) return;
  __shared__ Acc sA[SG_BK][SG_BM + 4];
  __shared__ Acc sB[SG_BK][SG_BN + 4];
  const TA* A = reinterpret_cast<const TA*>(g.A) + b * g.sab;
  const TB* B = reinterpret_cast<const TB*>(g.B) + b * g.sbb;
  float* C = g.C + b * g.scb;
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int64_t i0 = ti * SG_BM, j0 = tj * SG_BN;
  Acc acc[4][4] = {};
  for (int64_t k0 = 0; k0 < g.K; k0 += SG_BK) {
    // A tile 64 x 16 and B tile 16 x 64: 1024 elements each, 4 per thread.
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int idx = tid + e * 256;
      {  // A: consecutive threads walk k first when A is k-contiguous
        const int kk = (g.sak == 1) ? (idx % SG_BK) : (idx / SG_BM);
        const int ii = (g.sak == 1) ? (idx / SG_BK) : (idx % SG_BM);
        const int64_t gi = i0 + ii, gk = k0 + kk;
        sA[kk][ii] = (gi < g.M && gk < g.K) ? to_acc<Acc, TA>(A[gi * g.sam + gk * g.sak]) : Acc(0);
      }
      {
        const int jj = (g.sbn == 1) ? (idx % SG_BN) : (idx / SG_BK);
        const int kk = (g.sbn == 1) ? (idx / SG_BN) : (idx % SG_BK);
        const int64_t gj = j0 + jj, gk = k0 + kk;
        sB[kk][jj] = (gj < g.N && gk < g.K) ? to_acc<Acc, TB>(B[gk * g.sbk + gj * g.sbn]) : Acc(0);
      }
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SG_BK; ++kk) {
      Acc a[4], bb[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = sA[kk][ty + 16 * r];
#pragma unroll
      for (int c = 0; c < 4; ++c) bb[c] = sB[kk][tx + 16 * c];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fma(a[r], bb[c], acc[r][c]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t gi = i0 + ty + 16 * r;
    if (gi >= g.M) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int64_t gj = j0 + tx + 16 * c;
      if (gj >= g.N) continue;
      float* p = C + gi * g.scm + gj * g.scn;
      const float v = (float)((Acc)g.alpha * acc[r][c]);
      *p = (g.beta == 0.f) ? v : fmaf(g.beta, *p, v);
    }
  }
}

// fp64-accumulating GEMM with a larger register tile, for the products that
// need fp64 sums (the n-side Kronecker factors): 128 x 128 output tile per
// CTA of 256 threads, each thread 8 x 8 outputs as four 4 x 4 quadrants
// (rows 4 ty + {0..3} and 64 + 4 ty + {0..3}, columns likewise with tx), so
// a thread reads 16 doubles from shared memory per 64 FMAs and a warp's
// reads are two 16-byte words per lane without bank conflicts.  K in slabs
// of 8, the next slab loaded into registers while the current one is
// used.  Inputs of any type are converted to fp64 on the way into shared
// memory; the result is rounded to fp32 once.  Same GemmArgs as k_gemm_simt
// (tri must be 0).
constexpr int G64_BM = 128, G64_BN = 128, G64_BK = 8;

template <typename TA, typename TB>
__global__ void __launch_bounds__(256) k_gemm64(GemmArgs g) {
  __shared__ __align__(16) double sA[2][G64_BK][G64_BM];
  __shared__ __align__(16) double sB[2][G64_BK][G64_BN];
  const int64_t ti = blockIdx.y, tj = blockIdx.x, b = blockIdx.z;
  const TA* A = reinterpret_cast<const TA*>(g.A) + b * g.sab;
  const TB* B = reinterpret_cast<const TB*>(g.B) + b * g.sbb;
  float* C = g.C + b * g.scb;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t i0 = ti * G64_BM, j0 = tj * G64_BN;
  // staging: 128 x 8 elements of A and 8 x 128 of B per slab, 4 each per thread
  double ra[4], rb[4];
  auto load = [&](int64_t k0) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int idx = tid + e * 256;
      {
        const int kk = (g.sak == 1) ? (idx % G64_BK) : (idx / G64_BM);
        const int ii = (g.sak == 1) ? (idx / G64_BK) : (idx % G64_BM);
        const int64_t gi = i0 + ii, gk = k0 + kk;
        ra[e] = (gi < g.M && gk < g.K) ? to_acc<double, TA>(A[gi * g.sam + gk * g.sak]) : 0.0;
      }
      {
        const int jj = (g.sbn == 1) ? (idx % G64_BN) : (idx / G64_BK);
        const int kk = (g.sbn == 1) ? (idx / G64_BN) : (idx % G64_BK);
        const int64_t gj = j0 + jj, gk = k0 + kk;
        rb[e] = (gj < g.N && gk < g.K) ? to_acc<double, TB>(B[gk * g.sbk + gj * g.sbn]) : 0.0;
      }
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int idx = tid + e * 256;
      {
        const int kk = (g.sak == 1) ? (idx % G64_BK) : (idx / G64_BM);
        const int ii = (g.sak == 1) ? (idx / G64_BK) : (idx % G64_BM);
        sA[buf][kk][ii] = ra[e];
      }
      {
        const int jj = (g.sbn == 1) ? (idx % G64_BN) : (idx / G64_BK);
        const int kk = (g.sbn == 1) ? (idx / G64_BN) : (idx % G64_BK);
        sB[buf][kk][jj] = rb[e];
      }
    }
  };
  double acc[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[r][c] = 0.0;
  load(0);
  store(0);
  __syncthreads();
  int buf = 0;
  for (int64_t k0 = 0; k0 < g.K; k0 += G64_BK) {
    const bool more = k0 + G64_BK < g.K;
    if (more) load(k0 + G64_BK);
#pragma unroll
    for (int kk = 0; kk < G64_BK; ++kk) {
      double a[8], bv[8];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const double2 a0 = *reinterpret_cast<const double2*>(&sA[buf][kk][64 * h + 4 * ty]);
        const double2 a1 = *reinterpret_cast<const double2*>(&sA[buf][kk][64 * h + 4 * ty + 2]);
        a[4 * h] = a0.x, a[4 * h + 1] = a0.y, a[4 * h + 2] = a1.x, a[4 * h + 3] = a1.y;
        const double2 b0 = *reinterpret_cast<const double2*>(&sB[buf][kk][64 * h + 4 * tx]);
        const double2 b1 = *reinterpret_cast<const double2*>(&sB[buf][kk][64 * h + 4 * tx + 2]);
        bv[4 * h] = b0.x, bv[4 * h + 1] = b0.y, bv[4 * h + 2] = b1.x, bv[4 * h + 3] = b1.y;
      }
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = fma(a[r], bv[c], acc[r][c]);
    }
    if (more) {
      store(buf ^ 1);
      __syncthreads();
      buf ^= 1;
    }
  }
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int64_t gi = i0 + 64 * (r >> 2) + 4 * ty + (r & 3);
    if (gi >= g.M) continue;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int64_t gj = j0 + 64 * (c >> 2) + 4 * tx + (c & 3);
      if (gj >= g.N) continue;
      float* p = C + gi * g.scm + gj * g.scn;
      const float v = (float)(g.alpha * acc[r][c]);
      *p = (g.beta == 0.f) ? v : fmaf(g.beta, *p, v);
    }
  }
}

template <typename TA, typename TB, typename Acc = float>
inline cudaError_t gemm_simt(const GemmArgs& g, int64_t batch, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || batch <= 0) return cudaSuccess;
  if constexpr (std::is_same<Acc, double>::value) {
    if (g.tri == 0) {
      dim3 grid((unsigned)((g.N + G64_BN - 1) / G64_BN), (unsigned)((g.M + G64_BM - 1) / G64_BM),
                (unsigned)batch);
      LaunchScope ls("k_gemm64", st);
      k_gemm64<TA, TB><<<grid, 256, 0, st>>>(g);
      return cudaGetLastError();
    }
  }
  dim3 grid((unsigned)((g.N + SG_BN - 1) / SG_BN), (unsigned)((g.M + SG_BM - 1) / SG_BM),
            (unsigned)batch);
  {
    LaunchScope ls("k_gemm_simt", st);
    k_gemm_simt<TA, TB, Acc><<<grid, 256, 0, st>>>(g);
  }
  return cudaGetLastError();
}

}  // namespace quip
