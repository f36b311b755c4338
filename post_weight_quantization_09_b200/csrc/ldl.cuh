// LDL factorisation H = (I + Ů) D (I + Ů)^T, Ů strictly upper triangular:
// the factorisation whose Ů is LDLQ's linear feedback (QuIP, adaptive-
// rounding section; the display of the factorisation was lost from the page,
// the form is the one LDLQ's column order requires: column k is corrected by
// columns j < k only).
//
// Computed as H = R R^T with R upper triangular ("backward" Cholesky), then
// D_k = R_kk^2 and Ů_jk = R_jk / R_kk.  Blocked right-looking from the
// bottom-right, panel width PB:
//   for p = P-1 .. 0 (columns [p*PB, (p+1)*PB)):
//     R_pp        = backward Cholesky of the updated diagonal block  (1 CTA)
//     R[:p, p]    = H[:p, p] R_pp^-T                      (row-parallel solve)
//     H[:p, :p]  -= R[:p, p] R[:p, p]^T   (upper triangle; trailing update)
// Everything in place in the upper triangle of H (row-major, stride n).
#pragma once

#include "common.cuh"

namespace quip {

constexpr int LDL_PB = 64;

// Backward Cholesky of the PB x PB diagonal block at (c0, c0), upper part:
// for k = PB-1 .. 0: r = sqrt(A_kk); A_ik /= r (i < k); A_ij -= A_ik A_jk
// (i <= j < k).  Valid size `w` <= PB (the last block may be partial).
__global__ void __launch_bounds__(256) k_ldl_diag(float* H, int64_t n, int64_t c0, int w) {
  __shared__ float A[LDL_PB][LDL_PB + 1];
  __shared__ int bad;
  const int tid = threadIdx.x;
  if (tid == 0) bad = 0;
  for (int e = tid; e < LDL_PB * LDL_PB; e += 256) {
    const int i = e / LDL_PB, j = e % LDL_PB;
    A[i][j] = (i < w && j < w && j >= i) ? H[(c0 + i) * n + c0 + j] : 0.f;
  }
  __syncthreads();
  for (int k = w - 1; k >= 0; --k) {
    const float d = A[k][k];
    if (!(d > 0.f) || !isfinite(d)) {   // uniform: every thread reads the same value
      if (tid == 0) bad = 1;
      break;
    }
    const float r = sqrtf(d);
    __syncthreads();
    if (tid < k) A[tid][k] /= r;
    if (tid == 0) A[k][k] = r;
    __syncthreads();
    // A[i][j] -= A[i][k] * A[j][k] for i <= j < k
    for (int e = tid; e < k * k; e += 256) {
      const int i = e / k, j = e % k;
      if (i <= j) A[i][j] -= A[i][k] * A[j][k];
    }
    __syncthreads();
  }
  __syncthreads();
  if (bad && tid == 0) record_status(QUIP_ERR_NOT_PD);
  for (int e = tid; e < w * w; e += 256) {
    const int i = e / w, j = e % w;
    if (j >= i) H[(c0 + i) * n + c0 + j] = A[i][j];
  }
}

// R[i, c0:c0+w] = H[i, c0:c0+w] R_pp^-T for rows i < c0: back substitution
// r_k = (h_k - sum_{j>k} R_kj r_j) / R_kk, k = w-1 .. 0.  64 rows per CTA
// (one thread each), the row tile staged through shared memory so the
// global reads and writes are coalesced.
__global__ void __launch_bounds__(64) k_ldl_trsm(float* H, int64_t n, int64_t c0, int w) {
  __shared__ float R[LDL_PB][LDL_PB + 1];
  __shared__ float X[64][LDL_PB + 1];
  const int tid = threadIdx.x;
  const int64_t r0 = (int64_t)blockIdx.x * 64;
  for (int e = tid; e < LDL_PB * LDL_PB; e += 64) {
    const int i = e / LDL_PB, j = e % LDL_PB;
    R[i][j] = (i < w && j < w && j >= i) ? H[(c0 + i) * n + c0 + j] : 0.f;
  }
  for (int e = tid; e < 64 * LDL_PB; e += 64) {
    const int i = e / LDL_PB, j = e % LDL_PB;
    const int64_t gi = r0 + i;
    X[i][j] = (gi < c0 && j < w) ? H[gi * n + c0 + j] : 0.f;
  }
  __syncthreads();
  for (int k = w - 1; k >= 0; --k) {
    float s = X[tid][k];
    for (int j = k + 1; j < w; ++j) s -= R[k][j] * X[tid][j];
    X[tid][k] = s / R[k][k];
  }
  __syncthreads();
  for (int e = tid; e < 64 * LDL_PB; e += 64) {
    const int i = e / LDL_PB, j = e % LDL_PB;
    const int64_t gi = r0 + i;
    if (gi < c0 && j < w) H[gi * n + c0 + j] = X[i][j];
  }
}

}  // namespace quip
