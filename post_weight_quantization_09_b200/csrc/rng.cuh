// Random orthogonal transforms drawn on the device.
//
// QuIP ("QuIP: 2-Bit Quantization of Large Language Models With Guarantees"),
// Introduction and incoherence-processing section: U, V random orthogonal,
// as a Kronecker product of two small random orthogonal matrices.
// QuIP# (arXiv 2402.04396), abstract: randomized Hadamard transform, i.e.
// H_d diag(s) with random signs s.
//
// Randomness: counter-based SplitMix64 (Steele, Lea & Flood, "Fast splittable
// pseudorandom number generators", OOPSLA 2014): output k >= 1 of the
// sequence seeded with `seed` is mix(seed + k * 0x9E3779B97F4A7C15); stream t,
// element i uses k = t * 2^40 + i + 1.
#pragma once

#include "common.cuh"

namespace quip {

__host__ __device__ __forceinline__ uint64_t splitmix64(uint64_t seed, uint32_t stream,
                                                        uint64_t idx) {
  const uint64_t k = ((uint64_t)stream << 40) + idx + 1ull;
  uint64_t z = seed + k * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// s_i = -1 when the top bit of draw i is set, +1 otherwise.
__global__ void k_random_signs(float* s, int64_t n, uint64_t seed, uint32_t stream) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    s[i] = (splitmix64(seed, stream, (uint64_t)i) >> 63) ? -1.0f : 1.0f;
  }
}

// Random permutation of n coordinates: key_i = draw i of `stream`; pi sorts
// the keys in increasing order ((P x)_r = x_{pi[r]}).  The draws are
// distinct (the SplitMix64 finaliser is a bijection), so the rank of key i,
// #{j : key_j < key_i}, is pi^-1[i].
__global__ void k_perm_keys(uint64_t* keys, int64_t n, uint64_t seed, uint32_t stream) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    keys[i] = splitmix64(seed, stream, (uint64_t)i);
}

// rank by counting (n <= 65536: n^2 comparisons, keys staged through shared
// memory in tiles): iperm[i] = rank of key i, perm[rank] = i.
constexpr int PERM_TILE = 2048;
__global__ void __launch_bounds__(256) k_perm_rank(const uint64_t* __restrict__ keys, int64_t n,
                                                   int32_t* __restrict__ perm,
                                                   int32_t* __restrict__ iperm) {
  __shared__ uint64_t tile[PERM_TILE];
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const uint64_t ki = i < n ? keys[i] : 0ull;
  int32_t rank = 0;
  for (int64_t j0 = 0; j0 < n; j0 += PERM_TILE) {
    const int len = (int)min((int64_t)PERM_TILE, n - j0);
    __syncthreads();
    for (int t = threadIdx.x; t < len; t += blockDim.x) tile[t] = keys[j0 + t];
    __syncthreads();
#pragma unroll 8
    for (int t = 0; t < len; ++t) rank += tile[t] < ki ? 1 : 0;
  }
  if (i < n) {
    iperm[i] = rank;
    perm[rank] = (int32_t)i;
  }
}

// p x p Gaussian matrix, row-major element e from draws 2e, 2e+1:
// u = ((draw >> 11) + 1) 2^-53 in (0, 1], g = sqrt(-2 ln u1) cos(2 pi u2).
__global__ void k_gaussian(double* G, int64_t count, uint64_t seed, uint32_t stream) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < count;
       e += (int64_t)gridDim.x * blockDim.x) {
    const double u1 = ((double)(splitmix64(seed, stream, 2 * (uint64_t)e) >> 11) + 1.0) *
                      1.1102230246251565e-16;
    const double u2 = ((double)(splitmix64(seed, stream, 2 * (uint64_t)e + 1) >> 11) + 1.0) *
                      1.1102230246251565e-16;
    G[e] = sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
  }
}

// Q of G = QR with diag(R) > 0 (the Haar-distributed orthogonal factor), by
// classical Gram-Schmidt with one re-orthogonalisation pass (CGS2) in fp64.
// One CTA of 256 threads; p <= 256.  Qc: p x p fp64 workspace (column j of Q
// stored contiguously at Qc + j*p).  Q: p x p fp32 output, row-major; Q64
// the same in fp64.
__global__ void __launch_bounds__(256) k_haar_cgs2(const double* __restrict__ G,
                                                    double* __restrict__ Qc,
                                                    float* __restrict__ Q,
                                                    double* __restrict__ Q64, int p) {
  __shared__ double v[256];
  __shared__ double r[256];
  __shared__ double red[8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int j = 0; j < p; ++j) {
    if (tid < p) v[tid] = G[(int64_t)tid * p + j];
    __syncthreads();
    for (int pass = 0; pass < 2; ++pass) {
      // r_i = <q_i, v> for i < j: one warp per column i, lanes over rows.
      for (int i = warp; i < j; i += 8) {
        double s = 0.0;
        for (int row = lane; row < p; row += 32) s += Qc[(int64_t)i * p + row] * v[row];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) r[i] = s;
      }
      __syncthreads();
      // v <- v - Q[:, :j] r
      if (tid < p) {
        double s = 0.0;
        for (int i = 0; i < j; ++i) s += Qc[(int64_t)i * p + tid] * r[i];
        v[tid] -= s;
      }
      __syncthreads();
    }
    double sq = (tid < p) ? v[tid] * v[tid] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) red[warp] = sq;
    __syncthreads();
    double nrm2 = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) nrm2 += red[w];
    const double inv = 1.0 / sqrt(nrm2);
    if (tid < p) Qc[(int64_t)j * p + tid] = v[tid] * inv;
    __syncthreads();
  }
  for (int64_t e = tid; e < (int64_t)p * p; e += blockDim.x) {
    const int row = (int)(e / p), col = (int)(e % p);
    const double x = Qc[(int64_t)col * p + row];
    Q[e] = (float)x;
    Q64[e] = x;
  }
}

// ---------------------------------------------------------------- Haar factor by Cholesky-QR2
// Q of G = QR with diag(R) > 0 also equals Y R2^-1 with Y = G R1^-1, R1 the
// upper Cholesky factor of G^T G and R2 that of Y^T Y (Cholesky-QR applied
// twice): both factors have a positive diagonal, so R = R2 R1 does too and
// Q is the same unique factor as any other QR with that sign convention,
// up to rounding.  In fp64 one pass leaves Y orthogonal to about
// cond(G)^2 u; the second pass brings it to u.  Square Gaussian factors up to
// 224 x 224 (cond(G) of order p) are far inside that range.

// Offset of (i, j), i <= j, in the column-major packed upper triangle
// (column j holds rows 0 .. j).
__host__ __device__ __forceinline__ int64_t packed_col(int64_t i, int64_t j) { return j * (j + 1) / 2 + i; }

// Cp = Y^T Y (p x p, fp64), the upper triangle, packed by columns.  One
// 32 x 32 output tile per CTA (tiles below the diagonal exit at once), 256
// threads with four outputs each; 32-row slabs of both column blocks of Y
// through shared memory; each sum runs over the rows in order.
__global__ void __launch_bounds__(256) k_gram64(const double* __restrict__ Y,
                                                double* __restrict__ Cp, int p) {
  const int bi = blockIdx.y, bj = blockIdx.x;
  if (bi > bj) return;
  __shared__ double a[32][33], b[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int i0 = 32 * bi, j0 = 32 * bj;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int r0 = 0; r0 < p; r0 += 32) {
    for (int rr = ty; rr < 32; rr += 8) {
      const int r = r0 + rr;
      a[rr][tx] = (r < p && i0 + tx < p) ? Y[(int64_t)r * p + i0 + tx] : 0.0;
      b[rr][tx] = (r < p && j0 + tx < p) ? Y[(int64_t)r * p + j0 + tx] : 0.0;
    }
    __syncthreads();
#pragma unroll 8
    for (int rr = 0; rr < 32; ++rr) {
      const double bv = b[rr][tx];
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] = fma(a[rr][ty + 8 * u], bv, acc[u]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ty + 8 * u, j = j0 + tx;
    if (i < p && j < p && j >= i) Cp[packed_col(i, j)] = acc[u];
  }
}

constexpr int HAAR_CHOL_MAX = 224;          // packed factor + two rows fit in shared memory
constexpr int HAAR_CHOL_T = HAAR_CHOL_MAX / 32;
__host__ __device__ constexpr size_t chol_solve_smem(int p) {
  return ((size_t)p * (p + 1) / 2 + 2 * (size_t)p) * sizeof(double);
}

__device__ __forceinline__ double warp_allsum64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Offset of (i, j), i <= j, in the row-major packed upper triangle (row i
// holds columns i .. p - 1).
__host__ __device__ __forceinline__ int64_t packed_row(int64_t i, int64_t j, int64_t p) {
  return i * p - i * (i - 1) / 2 + (j - i);
}

constexpr int HAAR_CHOL_PARTS = 4;          // threads summing one entry of a row of R

// R: the upper Cholesky factor of C (C = R^T R; Cp packed by columns,
// fp64), written packed by columns to Rp (Rp may alias Cp).  One CTA of 1024
// threads, p <= HAAR_CHOL_MAX.  Cp is copied to shared memory packed by rows
// and factored in place, left-looking, one row of R per step:
// R[k, j] = (C[k, j] - sum_{i<k} R[i, k] R[i, j]) / R[k, k],
// R[k, k] = sqrt(C[k, k] - sum_{i<k} R[i, k]^2).  Thread (part, jj) forms the
// part of the sum for column j = k + jj over i = part, part + 4, ... (a
// warp reads 32 consecutive entries of a row of R and broadcasts R[i, k]);
// the four parts meet in shared memory.  A pivot that is not positive and
// finite is recorded as QUIP_ERR_NONFINITE (and Rp is left as it is).
// Dynamic smem: chol_solve_smem(p) (the packed factor and 2 p doubles) plus
// HAAR_CHOL_PARTS x 256 doubles.
__host__ __device__ constexpr size_t chol64_smem(int p) {
  return chol_solve_smem(p) + (size_t)HAAR_CHOL_PARTS * 256 * sizeof(double) + 256 * sizeof(int);
}
__global__ void __launch_bounds__(1024, 1) k_chol64(const double* Cp, double* Rp, int p) {
  extern __shared__ double chs[];
  double* R = chs;                                   // packed by rows, p (p + 1) / 2
  double* part_s = R + (int64_t)p * (p + 1) / 2 + 2 * p;   // [HAAR_CHOL_PARTS][256]
  int* rb = reinterpret_cast<int*>(part_s + HAAR_CHOL_PARTS * 256);   // R[i][j] = R[rb[i] + j]
  const int tid = threadIdx.x, part = tid >> 8, jj = tid & 255;
  for (int i = tid; i < p; i += blockDim.x) rb[i] = (int)(packed_row(i, i, p) - i);
  for (int j = tid; j < p; j += blockDim.x)
    for (int i = 0; i <= j; ++i) R[packed_row(i, j, p)] = Cp[packed_col(i, j)];
  __syncthreads();
  bool ok = true;
  for (int k = 0; k < p; ++k) {
    const int j = k + jj;
    // row k is rewritten below, after the barrier: read its diagonal first
    const double ckk = R[rb[k] + k];
    double s = 0.0;
    if (j < p)
      for (int i = part; i < k; i += HAAR_CHOL_PARTS) {
        const double* ri = R + rb[i];
        s = fma(ri[k], ri[j], s);
      }
    part_s[part * 256 + jj] = s;
    __syncthreads();
    const double d = ckk - ((part_s[0] + part_s[256]) + (part_s[512] + part_s[768]));
    ok = ok && d > 0.0 && d < INFINITY;
    if (part == 0 && j < p) {
      const double rkk = sqrt(d);
      const double v = R[rb[k] + j] - ((part_s[jj] + part_s[256 + jj]) + (part_s[512 + jj] + part_s[768 + jj]));
      R[rb[k] + j] = (jj == 0) ? rkk : v / rkk;
    }
    __syncthreads();
  }
  if (!ok) {
    if (tid == 0) record_status(QUIP_ERR_NONFINITE);
    return;
  }
  for (int j = tid; j < p; j += blockDim.x)
    for (int i = 0; i <= j; ++i) Rp[packed_col(i, j)] = R[packed_row(i, j, p)];
}

constexpr int HAAR_SOLVE_ROWS = 8;          // rows of X per CTA (one warp each)

// X = Y R^-1, one warp per row of X (HAAR_SOLVE_ROWS rows per CTA), R (packed
// by columns) copied to each CTA's shared memory: for k = 0 .. p - 1,
// X[r, k] = (Y[r, k] - sum_{i<k} X[r, i] R[i, k]) / R[k, k], lane l keeping
// X[r, i] and Y[r, i] for i = l, l + 32, ... in registers.  X must not alias
// Y or Rp.  out32, when not NULL, gets X rounded to fp32 (row-major).
// p <= HAAR_CHOL_MAX.  Dynamic smem: p (p + 1) / 2 doubles.
__global__ void __launch_bounds__(32 * HAAR_SOLVE_ROWS) k_trsm_rows64(const double* __restrict__ Rp,
                                                                    const double* __restrict__ Y,
                                                                    double* __restrict__ X,
                                                                    float* __restrict__ out32, int p) {
  extern __shared__ double chs[];
  double* R = chs;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t np = (int64_t)p * (p + 1) / 2;
  for (int64_t e = tid; e < np; e += blockDim.x) R[e] = Rp[e];
  __syncthreads();
  const int r = blockIdx.x * HAAR_SOLVE_ROWS + warp;
  if (r >= p) return;
  double yv[HAAR_CHOL_T], xv[HAAR_CHOL_T];
#pragma unroll
  for (int t = 0; t < HAAR_CHOL_T; ++t) {
    const int i = lane + 32 * t;
    yv[t] = i < p ? Y[(int64_t)r * p + i] : 0.0;
    xv[t] = 0.0;
  }
#pragma unroll
  for (int kq = 0; kq < HAAR_CHOL_T; ++kq) {
    for (int kl = 0; kl < 32; ++kl) {
      const int k = 32 * kq + kl;
      if (k >= p) break;
      double s = 0.0;
#pragma unroll
      for (int t = 0; t <= kq; ++t) {
        const int i = lane + 32 * t;
        if (i < k) s = fma(xv[t], R[packed_col(i, k)], s);
      }
      s = warp_allsum64(s);
      if (lane == kl) xv[kq] = (yv[kq] - s) / R[packed_col(k, k)];
    }
  }
#pragma unroll
  for (int t = 0; t < HAAR_CHOL_T; ++t) {
    const int i = lane + 32 * t;
    if (i < p) {
      X[(int64_t)r * p + i] = xv[t];
      if (out32) out32[(int64_t)r * p + i] = (float)xv[t];
    }
  }
}

}  // namespace quip
