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
// The trailing update is split in two (look-ahead): the columns of panel
// p - 1 first, on the critical path, then the rest on a second stream, where
// it overlaps the next panel's diagonal factor and row solve.
// Everything in place in the upper triangle of H (row-major, stride n).
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace quip {

constexpr int LDL_PB = 128;
constexpr int LDL_LD = LDL_PB + 1;     // padded shared-memory row

// ---------------------------------------------------------------- warp-level 32 x 32 blocks

// Backward Cholesky and inverse of a 32 x 32 block in one sweep, one warp,
// everything in registers: lane i keeps row i of A (a[]) and column i of
// X = R^-1 (x[]).  Step k (31 .. 0): the pivot comes from lane k by shuffle;
// 1 / sqrt(A_kk) is one rsqrt (a few ulp, far inside the fp32 factorisation
// error); lane i forms R[i][k]; row k of R is read from lane k by shuffles to
// form x_kj = (delta_kj - sum_{m>k} R_km x_mj) / R_kk; the leading block is
// updated with the new column, the entry the next pivot needs first.
// S: block (upper triangle read, R written back); Xo: X (32 x 32, full).
// Returns false (warp-uniform) if a pivot is not positive.
__device__ __forceinline__ bool warp_chol_inv32(float* S, int lds, float* Xo, int ldx) {
  const int lane = threadIdx.x & 31;
  float a[32], x[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    a[j] = (j >= lane) ? S[lane * lds + j] : S[j * lds + lane];
    x[j] = 0.f;
  }
  bool ok = true;
#pragma unroll
  for (int k = 31; k >= 0; --k) {
    const float d = __shfl_sync(0xffffffffu, a[k], k);
    ok = ok && (d > 0.f) && isfinite(d);
    const float ir = rsqrtf(d);
    const float l = (lane == k) ? d * ir : a[k] * ir;
    a[k] = l;
#pragma unroll
    for (int j = k - 1; j >= 0; --j) a[j] = fmaf(-l, __shfl_sync(0xffffffffu, l, j), a[j]);
    float s0 = (lane == k) ? 1.f : 0.f, s1 = 0.f;
#pragma unroll
    for (int m = k + 1; m < 32; m += 2) {
      s0 = fmaf(-__shfl_sync(0xffffffffu, a[m], k), x[m], s0);
      if (m + 1 < 32) s1 = fmaf(-__shfl_sync(0xffffffffu, a[m + 1], k), x[m + 1], s1);
    }
    x[k] = (lane >= k) ? (s0 + s1) * ir : 0.f;
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    if (j >= lane) S[lane * lds + j] = a[j];
    Xo[j * ldx + lane] = x[j];
  }
  __syncwarp();
  return ok;
}

// Factor the panel's 128 x 128 diagonal block held in shared memory A
// (rows of LDL_LD floats, upper triangle valid, identity-padded past w) as
// 4 x 4 blocks of 32, by the whole CTA (256 threads).  For J = 3 .. 0:
//   warp 0:  A_JJ = R_JJ R_JJ^T and X_JJ = R_JJ^-1 (warp_chol_inv32);
//   all:     R_IJ = A_IJ X_JJ^T for the rows above (I < J);
//   all:     the next diagonal block A_{J-1,J-1} -= R_{J-1,J} R_{J-1,J}^T;
//   warps 1-7 (while warp 0 factors block J-1): the rest of
//            A[0:32J, 0:32J] -= R[0:32J, J] R[0:32J, J]^T (upper part).
// On return A's upper triangle holds R and X[J] (32 x 33 each) the inverses.
// Returns false if a pivot was not positive.
__device__ bool ldl_factor_diag(float* A, float* X, float* rb, float* rk, int* bad) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  (void)rk;
  if (tid == 0) *bad = 0;
  __syncthreads();
  for (int J = 3; J >= 0; --J) {
    float* XJ = X + J * 32 * 33;
    if (warp == 0) {
      const bool ok = warp_chol_inv32(A + (32 * J) * LDL_LD + 32 * J, LDL_LD, XJ, 33);
      if (!ok && lane == 0) *bad = 1;
    }
    __syncthreads();                              // also orders the rest-update of J + 1
    if (J == 0) break;
    const int rows = 32 * J;
    {
      float out[3][4];
      const int k0 = tid & 7, ib = tid >> 3;
#pragma unroll
      for (int rg = 0; rg < 3; ++rg) {
        const int i = ib + 32 * rg;
#pragma unroll
        for (int c = 0; c < 4; ++c) out[rg][c] = 0.f;
        if (i < rows) {
          const float* ar = A + i * LDL_LD + 32 * J;
#pragma unroll 8
          for (int t = 0; t < 32; ++t) {
            const float av = ar[t];
#pragma unroll
            for (int c = 0; c < 4; ++c) out[rg][c] = fmaf(av, XJ[(k0 + 8 * c) * 33 + t], out[rg][c]);
          }
        }
      }
      __syncthreads();
#pragma unroll
      for (int rg = 0; rg < 3; ++rg) {
        const int i = ib + 32 * rg;
        if (i < rows)
#pragma unroll
          for (int c = 0; c < 4; ++c) A[i * LDL_LD + 32 * J + k0 + 8 * c] = out[rg][c];
      }
      __syncthreads();
    }
    {
      const int i = 32 * (J - 1) + (tid >> 3);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int k = 32 * (J - 1) + (tid & 7) + 8 * c;
        if (k < i) continue;
        const float* ri = A + i * LDL_LD + 32 * J;
        const float* rr = A + k * LDL_LD + 32 * J;
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int t = 0; t < 32; t += 2) {
          s0 = fmaf(ri[t], rr[t], s0);
          s1 = fmaf(ri[t + 1], rr[t + 1], s1);
        }
        A[i * LDL_LD + k] -= s0 + s1;
      }
    }
    __syncthreads();
    if (warp > 0) {
      const int nr = 32 * (J - 1);
      const int t0 = tid - 32, nt = 224;
      for (int e = t0; e < nr * rows; e += nt) {
        const int i = e / rows, k = e % rows;
        if (k < i) continue;
        const float* ri = A + i * LDL_LD + 32 * J;
        const float* rr = A + k * LDL_LD + 32 * J;
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
        for (int t = 0; t < 32; t += 4) {
          s0 = fmaf(ri[t], rr[t], s0);
          s1 = fmaf(ri[t + 1], rr[t + 1], s1);
          s2 = fmaf(ri[t + 2], rr[t + 2], s2);
          s3 = fmaf(ri[t + 3], rr[t + 3], s3);
        }
        A[i * LDL_LD + k] -= (s0 + s1) + (s2 + s3);
      }
    }
  }
  __syncthreads();
  return *bad == 0;
}

// Diagonal block of one panel, columns [c0, c0 + w), w <= 128, by one CTA:
// load the updated block (identity-padded past w), factor it
// (ldl_factor_diag), write R_pp to Rd (128 x 128, upper triangle valid) and
// the inverses X_JJ of its 32 x 32 diagonal blocks to Xw (4 x 32 x 33).
// R_pp goes to the workspace, not into H: H's own diagonal blocks are copied
// in by k_ldl_scatter_diag after the last panel.
// Dynamic smem: 128 x 129 + 4 x 32 x 33 floats.
__global__ void __launch_bounds__(256) k_ldl_diag(const float* __restrict__ H, int64_t n,
                                                  int64_t c0, int w, float* __restrict__ Rd,
                                                  float* __restrict__ Xw) {
  extern __shared__ __align__(16) float sm[];
  float* R = sm;                                  // 128 x LDL_LD
  float* X = R + LDL_PB * LDL_LD;                 // 4 x 32 x 33
  __shared__ __align__(16) float rb[32];
  __shared__ float rk[32];
  __shared__ int bad;
  const int tid = threadIdx.x;
#pragma unroll 4
  for (int e = tid; e < LDL_PB * 32; e += 256) {
    const int i = e >> 5, j4 = (e & 31) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < w && j4 < w) v = *reinterpret_cast<const float4*>(H + (c0 + i) * n + c0 + j4);
    float* d = R + i * LDL_LD + j4;
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = j4 + c;
      d[c] = (i < w && j < w) ? (j >= i ? vv[c] : 0.f) : (i == j ? 1.f : 0.f);
    }
  }
  __syncthreads();
  const bool ok = ldl_factor_diag(R, X, rb, rk, &bad);
  if (!ok && tid == 0) record_status(QUIP_ERR_NOT_PD);
#pragma unroll 4
  for (int e = tid; e < LDL_PB * LDL_PB; e += 256) Rd[e] = R[(e >> 7) * LDL_LD + (e & 127)];
  for (int e = tid; e < 4 * 32 * 33; e += 256) Xw[e] = X[e];
}

// Rows [64 b, 64 b + 64) of R12 = H12 R_pp^-T for one panel (H12 = H[:c0,
// c0:c0+w]), from the panel's R_pp (Rd) and X_JJ (Xw), by block back
// substitution over the four 32-column blocks (J = 3 .. 0):
//   t_J = h_J - sum_{K > J} r_K R_JK^T,   r_J = t_J X_JJ^T,
// with a 2 x 4 register tile per thread (rows 2 ty, 2 ty + 1; columns tx + 8 c).
// R12 goes back into H's columns [c0, c0 + w) and, as three bf16 pieces,
// into Rs[q][i][k] (piece stride n * 128, row stride 128; columns >= w zero).
// Grid: ceil(c0 / 64) CTAs of 256 threads.
// Dynamic smem: 96 x 129 (the rows of R_pp that hold blocks R_JK, J < K)
// + 64 x 129 (row tile) + 4 x 32 x 33 floats.
constexpr int LDL_RROWS = 96;
__global__ void __launch_bounds__(256) k_ldl_rows(float* __restrict__ H, int64_t n, int64_t c0,
                                                  int w, const float* __restrict__ Rd,
                                                  const float* __restrict__ Xw,
                                                  __nv_bfloat16* __restrict__ Rs) {
  extern __shared__ __align__(16) float sm[];
  float* R = sm;                                  // 96 x LDL_LD
  float* T = R + LDL_RROWS * LDL_LD;              // 64 x LDL_LD
  float* X = T + 64 * LDL_LD;                     // 4 x 32 x 33
  const int tid = threadIdx.x;
  const int64_t r0 = (int64_t)blockIdx.x * 64;
#pragma unroll 4
  for (int e = tid; e < LDL_RROWS * 32; e += 256) {
    const int i = e >> 5, j4 = (e & 31) * 4;
    const float4 v = *reinterpret_cast<const float4*>(Rd + i * LDL_PB + j4);
    float* d = R + i * LDL_LD + j4;
    d[0] = v.x, d[1] = v.y, d[2] = v.z, d[3] = v.w;
  }
  for (int e = tid; e < 4 * 32 * 33; e += 256) X[e] = Xw[e];
#pragma unroll 4
  for (int e = tid; e < 64 * 32; e += 256) {
    const int i = e >> 5, j4 = (e & 31) * 4;
    const int64_t gi = r0 + i;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (gi < c0 && j4 < w) v = *reinterpret_cast<const float4*>(H + gi * n + c0 + j4);
    float* d = T + i * LDL_LD + j4;
    d[0] = (j4 < w) ? v.x : 0.f;
    d[1] = (j4 + 1 < w) ? v.y : 0.f;
    d[2] = (j4 + 2 < w) ? v.z : 0.f;
    d[3] = (j4 + 3 < w) ? v.w : 0.f;
  }
  __syncthreads();
  const int ty = tid >> 3, tx = tid & 7;
  const int i0 = 2 * ty;
  for (int J = 3; J >= 0; --J) {
    float acc[2][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = T[(i0 + a) * LDL_LD + 32 * J + tx + 8 * c];
    for (int K = J + 1; K < 4; ++K) {
#pragma unroll 8
      for (int t = 0; t < 32; ++t) {
        const float h0 = T[i0 * LDL_LD + 32 * K + t], h1 = T[(i0 + 1) * LDL_LD + 32 * K + t];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float rv = R[(32 * J + tx + 8 * c) * LDL_LD + 32 * K + t];
          acc[0][c] = fmaf(-h0, rv, acc[0][c]);
          acc[1][c] = fmaf(-h1, rv, acc[1][c]);
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) T[(i0 + a) * LDL_LD + 32 * J + tx + 8 * c] = acc[a][c];
    __syncthreads();
    const float* XJ = X + J * 32 * 33;
    float out[2][4] = {};
#pragma unroll 8
    for (int t = 0; t < 32; ++t) {
      const float h0 = T[i0 * LDL_LD + 32 * J + t], h1 = T[(i0 + 1) * LDL_LD + 32 * J + t];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float xv = XJ[(tx + 8 * c) * 33 + t];
        out[0][c] = fmaf(h0, xv, out[0][c]);
        out[1][c] = fmaf(h1, xv, out[1][c]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) T[(i0 + a) * LDL_LD + 32 * J + tx + 8 * c] = out[a][c];
    __syncthreads();
  }
  const int64_t pstride = n * LDL_PB;
  for (int e = tid; e < 64 * LDL_PB; e += 256) {
    const int ii = e >> 7, k = e & 127;
    const int64_t gi = r0 + ii;
    if (gi >= c0) continue;
    const float v = (k < w) ? T[ii * LDL_LD + k] : 0.f;
    if (k < w) H[gi * n + c0 + k] = v;
    __nv_bfloat16 p0, p1, p2;
    split3(v, p0, p1, p2);
    Rs[gi * LDL_PB + k] = p0;
    Rs[pstride + gi * LDL_PB + k] = p1;
    Rs[2 * pstride + gi * LDL_PB + k] = p2;
  }
}

// Copy every panel's diagonal factor block from Rd[p] (128 x 128) into H's
// upper triangle: block p covers rows / columns [128 p, 128 p + w).
__global__ void k_ldl_scatter_diag(float* __restrict__ H, int64_t n, const float* __restrict__ Rd) {
  const int64_t p = blockIdx.x;
  const int64_t c0 = p * LDL_PB;
  const int w = (int)((n - c0) < LDL_PB ? (n - c0) : LDL_PB);
  const float* src = Rd + p * LDL_PB * LDL_PB;
  for (int e = threadIdx.x; e < LDL_PB * LDL_PB; e += blockDim.x) {
    const int i = e >> 7, j = e & 127;
    if (i < w && j < w && j >= i) H[(c0 + i) * n + c0 + j] = src[e];
  }
}

}  // namespace quip
