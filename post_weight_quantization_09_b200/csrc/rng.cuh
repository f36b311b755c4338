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

}  // namespace quip
