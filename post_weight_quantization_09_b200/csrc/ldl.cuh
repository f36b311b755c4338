// LDL factorisation H = (I + Ů) D (I + Ů)^T, Ů strictly upper triangular:
// the factorisation whose Ů is LDLQ's linear feedback (QuIP, adaptive-
// rounding section; the display of the factorisation was lost from the page,
// the form is the one LDLQ's column order requires: column k is corrected by
// columns j < k only).
//
// Computed as H = R R^T with R upper triangular ("backward" Cholesky), then
// D_k = R_kk^2 and Ů_jk = R_jk / R_kk.  Blocked right-looking from the
// bottom-right in panels of PB = 128 columns; panel p covers columns
// [c0, c0 + w), c0 = 128 p, and R12(p) = R[:c0, panel p]:
//
//   k_ldl_factor(p)  R_pp = backward Cholesky of the updated diagonal block,
//                    with the inverses X_J of its four 32 x 32 diagonal
//                    blocks, the block's Ů and D, and the 128 "next" rows
//                    Nx = R12(p)[c0-128 : c0] (4 CTAs, each factors the block
//                    redundantly and solves 32 of those rows);
//   k_ldl_rows(p)    R12(p) = H[:c0, panel p] R_pp^-T (32 rows per block;
//                    the rows of Nx are taken from there), its Ů and bf16
//                    pieces, and the look-ahead product L(p) = R12(p) Nx^T,
//                    i.e. panel p's update of panel p - 1, into a side buffer;
//   bulk(p)          H[:c0-128, :c0-128] -= R12 R12^T (upper tiles; tensor-
//                    core split GEMM on a second stream, quip_api.cu).
//
// Panel p - 1 is read as H - L(p): every element of a column panel receives
// its updates in panel order (the bulk updates in stream order, then L(p)),
// as in the unblocked factorisation, so the result does not depend on how
// the two streams interleave.  The bulk update of panel p + 1 overlaps the
// factor and row kernels of panel p.
// Everything in place in the upper triangle of H (row-major, stride n).
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace quip {

constexpr int LDL_PB = 128;
constexpr int LDL_LDA = 132;    // smem row stride of 128-wide tiles (16-B rows)
constexpr int LDL_LDX = 36;     // smem row stride of 32-wide tiles (16-B rows)
constexpr int LDL_FT = 512;     // threads of k_ldl_factor
constexpr int LDL_NX = 128;     // next rows solved by k_ldl_factor (32 per CTA)
constexpr int LDL_FCTAS = LDL_NX / 32;
constexpr int LDL_RT = 256;     // threads of k_ldl_rows
constexpr int LDL_RR = 32;      // rows per k_ldl_rows block
constexpr int LDL_HT = 384;     // helper threads of k_ldl_factor (warps w % 4 != 0)

// ---------------------------------------------------------------- helpers

// acc[a][b] += sum_{t < len} P[a * ps + t] * Q[b * qs + t]; len % 4 == 0,
// every row 16-byte aligned.  Sums run in t order.
template <int NA, int NB>
__device__ __forceinline__ void dot_rows(float (&acc)[NA][NB], const float* P, int ps,
                                         const float* Q, int qs, int len) {
#pragma unroll 2
  for (int t = 0; t < len; t += 4) {
    float4 pv[NA], qv[NB];
#pragma unroll
    for (int a = 0; a < NA; ++a) pv[a] = *reinterpret_cast<const float4*>(P + a * ps + t);
#pragma unroll
    for (int b = 0; b < NB; ++b) qv[b] = *reinterpret_cast<const float4*>(Q + b * qs + t);
#pragma unroll
    for (int a = 0; a < NA; ++a)
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        acc[a][b] = fmaf(pv[a].x, qv[b].x, acc[a][b]);
        acc[a][b] = fmaf(pv[a].y, qv[b].y, acc[a][b]);
        acc[a][b] = fmaf(pv[a].z, qv[b].z, acc[a][b]);
        acc[a][b] = fmaf(pv[a].w, qv[b].w, acc[a][b]);
      }
  }
}

__device__ __forceinline__ void helpers_sync() {      // the helper warps of k_ldl_factor
  asm volatile("bar.sync 1, %0;" ::"n"(LDL_HT) : "memory");
}

// Backward Cholesky of a 32 x 32 block S (upper triangle read, row stride
// lds, 16-byte rows) and the inverse of its factor, by one warp.  Lane i
// keeps row i of the block in registers (only j >= i is ever used).  Step k
// (31 .. 0): the pivot comes by shuffle from lane k, which formed it from its
// own previous column entry (so the chain from pivot to pivot is one
// shuffle, one rsqrtf, one multiply and one fma); lane i forms
// R[i][k] = l_i and updates its entry of the next column with R[k-1][k]
// from a second shuffle, then publishes l_i in a double-buffered shared
// column (broadcast 16-byte loads) whose other entries, j < k - 1, it
// applies in step k - 1 while that step's rsqrtf is in flight (warps issue
// in order: the updates no longer hold up the next pivot).  1 / R_kk is the rsqrtf of the pivot.  Then X = R^-1 column by
// column (lane j: column j), right-looking back substitution over the
// columns of R, read as broadcast rows of a transposed copy.
// scratch: 32 x LDL_LDX + 64 floats.  On return S's upper triangle holds R
// (its lower triangle zero) and X (row stride ldx, lower part zero) holds
// R^-1.  Returns false (warp-uniform) if a pivot was not positive and finite.
__device__ __forceinline__ bool warp_chol_inv32(float* S, int lds, float* X, int ldx,
                                                float* scratch) {
  const int lane = threadIdx.x & 31;
  float a[32];
  float* col = scratch + 32 * LDL_LDX;            // 2 x 32
  float* rin = col + 64;                          // 32: 1 / R_kk (kept in shared memory, not registers)
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 v = *reinterpret_cast<const float4*>(S + lane * lds + 4 * q);
    a[4 * q + 0] = (4 * q + 0 >= lane) ? v.x : 0.f;
    a[4 * q + 1] = (4 * q + 1 >= lane) ? v.y : 0.f;
    a[4 * q + 2] = (4 * q + 2 >= lane) ? v.z : 0.f;
    a[4 * q + 3] = (4 * q + 3 >= lane) ? v.w : 0.f;
  }
  bool ok = true;
  float self = a[31];
  float v[32];                                    // the previous step's column, from shared memory
  float lp = 0.f;                                 // the previous step's l_i
#pragma unroll
  for (int k = 31; k >= 0; --k) {
    const float piv = __shfl_sync(0xffffffffu, self, k);
    ok = ok && (piv > 0.f) && (piv < INFINITY);
    const float r = rsqrtf(piv);
    // step k + 1's updates of the columns j < k, issued while rsqrtf is in
    // flight (each entry still takes its updates in step order)
    if (k < 31) {
#pragma unroll
      for (int j = 0; j < k; ++j) a[j] = fmaf(-lp, v[j], a[j]);
    }
    if (lane == 0) rin[k] = r;
    const float l = (lane == k) ? piv * r : a[k] * r;
    a[k] = l;
    if (k > 0) {
      // the next column at once, with one shuffle (R[k-1][k] from lane k - 1):
      // the next pivot (lane k - 1) and the next column wait for no
      // shared-memory round trip
      const float lk1 = __shfl_sync(0xffffffffu, l, k - 1);
      a[k - 1] = fmaf(-l, lk1, a[k - 1]);
      self = a[k - 1];                     // lane k - 1: its next pivot
      // the older columns through the shared column, applied in the next step
      float* cb = col + (k & 1) * 32;
      cb[lane] = l;
      __syncwarp();
#pragma unroll
      for (int j4 = 0; j4 < k - 1; j4 += 4) {
        const float4 c = *reinterpret_cast<const float4*>(cb + j4);
        v[j4] = c.x, v[j4 + 1] = c.y, v[j4 + 2] = c.z, v[j4 + 3] = c.w;
      }
      lp = l;
    }
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 v = make_float4(4 * q + 0 >= lane ? a[4 * q + 0] : 0.f, 4 * q + 1 >= lane ? a[4 * q + 1] : 0.f,
                                 4 * q + 2 >= lane ? a[4 * q + 2] : 0.f, 4 * q + 3 >= lane ? a[4 * q + 3] : 0.f);
    *reinterpret_cast<float4*>(S + lane * lds + 4 * q) = v;
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) scratch[j * LDL_LDX + lane] = (j >= lane) ? a[j] : 0.f;   // row j = column j of R
  __syncwarp();                                   // also publishes rin
  float x[32];
#pragma unroll
  for (int m = 0; m < 32; ++m) x[m] = (m == lane) ? 1.f : 0.f;
#pragma unroll
  for (int k = 31; k >= 0; --k) {
    x[k] *= rin[k];                               // broadcast read
    const float* rc = scratch + k * LDL_LDX;
#pragma unroll
    for (int m4 = 0; m4 < k; m4 += 4) {
      const float4 v = *reinterpret_cast<const float4*>(rc + m4);
      if (m4 + 0 < k) x[m4 + 0] = fmaf(-v.x, x[k], x[m4 + 0]);
      if (m4 + 1 < k) x[m4 + 1] = fmaf(-v.y, x[k], x[m4 + 1]);
      if (m4 + 2 < k) x[m4 + 2] = fmaf(-v.z, x[k], x[m4 + 2]);
      if (m4 + 3 < k) x[m4 + 3] = fmaf(-v.w, x[k], x[m4 + 3]);
    }
  }
#pragma unroll
  for (int m = 0; m < 32; ++m) X[m * ldx + lane] = x[m];
  __syncwarp();
  return ok;
}

// ---------------------------------------------------------------- block steps on shared tiles
// Tiles are row-major 128-wide (stride LDL_LDA) or 32-wide (stride
// LDL_LDX).  Each step maps tasks of 2 x 2 outputs onto threads
// [t0, t0 + nt): rows (ti, ti + h) and columns (tk, tk + 16), consecutive
// threads on consecutive columns (conflict-free 16-byte loads).

// R_IJ = A_IJ X_J^T for rows [i0, i0 + nr) of column block J, in place
// (nr even, <= 2 * 16 * 2 tasks per thread: nr * 8 <= 2 nt).  `bar` syncs the
// participating threads between the reads and the writes.
template <typename Bar>
__device__ __forceinline__ void blk_trsm(float* A, const float* XJ, int J, int i0, int nr, int t,
                                         int nt, Bar bar) {
  const int h = nr / 2, ntask = h * 16;
  float out[2][2][2];
  int tasks[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int e = t + u * nt;
    tasks[u] = e;
    if (e < ntask) {
      const int ti = e >> 4, tk = e & 15;
      float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      dot_rows<2, 2>(acc, A + (i0 + ti) * LDL_LDA + 32 * J, h * LDL_LDA, XJ + tk * LDL_LDX,
                     16 * LDL_LDX, 32);
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b) out[u][a][b] = acc[a][b];
    }
  }
  bar();
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int e = tasks[u];
    if (e < ntask) {
      const int ti = e >> 4, tk = e & 15;
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b) A[(i0 + ti + a * h) * LDL_LDA + 32 * J + tk + 16 * b] = out[u][a][b];
    }
  }
  bar();
}

// A[i][j] -= sum_t R[i][32J + t] R[j][32J + t] (R = A's column block J) for
// the upper elements (j >= i) of rows [i0, i0 + nr) x columns [j0, j0 + nc)
// (nr, nc even).  Tasks: rows (ti, ti + nr/2), columns (tj, tj + nc/2).
__device__ __forceinline__ void blk_update(float* A, int J, int i0, int nr, int j0, int nc, int t,
                                           int nt) {
  const int hr = nr / 2, hc = nc / 2, ntask = hr * hc;
  for (int e = t; e < ntask; e += nt) {
    const int ti = e / hc, tj = e % hc;
    const int ia = i0 + ti, ja = j0 + tj;
    if (ia > ja + hc) continue;                       // all four below the diagonal
    float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    dot_rows<2, 2>(acc, A + ia * LDL_LDA + 32 * J, hr * LDL_LDA, A + ja * LDL_LDA + 32 * J,
                   hc * LDL_LDA, 32);
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const int i = ia + a * hr, j = ja + b * hc;
        if (j >= i) A[i * LDL_LDA + j] -= acc[a][b];
      }
  }
}

// One column block J of the back substitution R12 = T R_pp^-T for an
// NR-row tile T (stride LDL_LDA; columns of blocks K > J already solved):
//   T[:, J] -= sum_{K > J} T[:, K] R_JK^T,   T[:, J] = T[:, J] X_J^T.
// Rp: rows of R_pp (stride LDL_LDA), XJ: X_J (stride LDL_LDX).
// NR * 8 tasks of 2 x 2: rows (ti, ti + NR/2), columns (tk, tk + 16); at
// most two per thread.
template <int NR, typename Bar>
__device__ __forceinline__ void blk_solve(float* T, const float* Rp, const float* XJ, int J,
                                          int t, int nt, Bar bar) {
  constexpr int NTASK = NR * 8, HR = NR / 2;
  float out[2][2][2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int e = t + u * nt;
    if (e < NTASK && J < 3) {
      const int ti = e >> 4, tk = e & 15;
      float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      const int c1 = 32 * (J + 1);
      dot_rows<2, 2>(acc, T + ti * LDL_LDA + c1, HR * LDL_LDA, Rp + (32 * J + tk) * LDL_LDA + c1,
                     16 * LDL_LDA, LDL_PB - c1);
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b) T[(ti + HR * a) * LDL_LDA + 32 * J + tk + 16 * b] -= acc[a][b];
    }
  }
  bar();
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int e = t + u * nt;
    if (e < NTASK) {
      const int ti = e >> 4, tk = e & 15;
      float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      dot_rows<2, 2>(acc, T + ti * LDL_LDA + 32 * J, HR * LDL_LDA, XJ + tk * LDL_LDX,
                     16 * LDL_LDX, 32);
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b) out[u][a][b] = acc[a][b];
    }
  }
  bar();
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int e = t + u * nt;
    if (e < NTASK) {
      const int ti = e >> 4, tk = e & 15;
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b) T[(ti + HR * a) * LDL_LDA + 32 * J + tk + 16 * b] = out[u][a][b];
    }
  }
  bar();
}

// ---------------------------------------------------------------- kernels

// One thread waits for the CTA's tile copies (bounded; after a timeout it
// waits once more for the copies still in flight) and tells the CTA.
__device__ __forceinline__ bool tiles_arrived(uint64_t* bar, int* flag) {
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(bar, 0);
    if (!ok) mbar_wait(bar, 0);
    *flag = ok ? 1 : 0;
  }
  __syncthreads();
  return *flag != 0;
}

__device__ __forceinline__ float* align128(uint8_t* p) {
  return reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(p) + 127) & ~uintptr_t(127));
}


// Factor of panel p, columns [c0, c0 + w), w <= 128.  Every CTA loads the
// updated diagonal block (H - Lin, identity-padded past w) and factors it
// (the same deterministic computation in each), as 4 x 4 blocks of 32:
//   for J = 3 .. 0:
//     warp 0:      R_JJ, X_J = R_JJ^-1                         (warp_chol_inv32)
//     all:         R_{J-1,J} = A_{J-1,J} X_J^T;  A_{J-1,J-1} -= R_{J-1,J} R_{J-1,J}^T
//     helpers (warps w % 4 != 0), while warp 0 factors block J - 1: the other rows of block
//                  column J (R_IJ, I < J - 1), the rest of the trailing
//                  update, and column block J of this CTA's 32 next rows
//                  (blk_solve).
// CTA c (when c0 > 0) solves next rows c0 - 128 + 32 c .. + 31 of R12(p)
// into Nx (128 x 128, row i = global row c0 - 128 + i).  The CTAs split the
// stores of R_pp (Rd, 128 x 128, upper; lower zero) and X_J (Xw, 4 x 32 x
// 32); CTA 0 writes D (Dv[c0 + k] = R_kk^2); the CTAs split the block's rows
// for its Ů in H.  Lin: the look-ahead buffer of panel p + 1 (rows
// [0, c0 + 128) x 128), or NULL.
// Dynamic smem: (128 + 32) x LDL_LDA + 5 x 32 x LDL_LDX + 96 floats.
__global__ void __launch_bounds__(LDL_FT, 1)
    k_ldl_factor(float* __restrict__ H, int64_t n, int64_t c0, int w, const float* __restrict__ Lin,
                 float* __restrict__ Rd, float* __restrict__ Xw, float* __restrict__ Nx,
                 float* __restrict__ Dv) {
  extern __shared__ __align__(16) float sm[];
  pdl_wait_then_release();
  float* A = sm;                                     // 128 x LDL_LDA
  float* T = A + LDL_PB * LDL_LDA;                   // 32 x LDL_LDA (next rows)
  float* X = T + 32 * LDL_LDA;                       // 4 x 32 x LDL_LDX
  float* scr = X + 4 * 32 * LDL_LDX;                 // 32 x LDL_LDX + 96
  __shared__ int bad;
  const int tid = threadIdx.x, warp = tid >> 5;
  const bool has_next = c0 > 0;
  if (tid == 0) bad = 0;
#pragma unroll
  for (int e = tid; e < LDL_PB * 32; e += LDL_FT) {
    const int i = e >> 5, j4 = (e & 31) * 4;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (i < w && j4 < w) {
      const float4 h = *reinterpret_cast<const float4*>(H + (c0 + i) * n + c0 + j4);
      v[0] = h.x, v[1] = h.y, v[2] = h.z, v[3] = h.w;
      if (Lin) {
        const float4 l = *reinterpret_cast<const float4*>(Lin + (c0 + i) * LDL_PB + j4);
        v[0] -= l.x, v[1] -= l.y, v[2] -= l.z, v[3] -= l.w;
      }
    }
    float o[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = j4 + c;
      o[c] = (i < w && j < w) ? (j >= i ? v[c] : 0.f) : (i == j ? 1.f : 0.f);
    }
    *reinterpret_cast<float4*>(A + i * LDL_LDA + j4) = make_float4(o[0], o[1], o[2], o[3]);
  }
  if (has_next) {
    const int64_t g0 = c0 - LDL_PB + 32 * (int64_t)blockIdx.x;
#pragma unroll
    for (int e = tid; e < 32 * 32; e += LDL_FT) {
      const int i = e >> 5, j4 = (e & 31) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j4 < w) {
        v = *reinterpret_cast<const float4*>(H + (g0 + i) * n + c0 + j4);
        if (Lin) {
          const float4 l = *reinterpret_cast<const float4*>(Lin + (g0 + i) * LDL_PB + j4);
          v.x -= l.x, v.y -= l.y, v.z -= l.z, v.w -= l.w;
        }
      }
      *reinterpret_cast<float4*>(T + i * LDL_LDA + j4) = v;   // w % 4 == 0
    }
  }
  __syncthreads();

  auto all_sync = [] { __syncthreads(); };
  for (int J = 3; J >= 0; --J) {
    if (warp == 0) {
      const bool ok = warp_chol_inv32(A + 32 * J * LDL_LDA + 32 * J, LDL_LDA, X + J * 32 * LDL_LDX,
                                      LDL_LDX, scr);
      if (!ok && (tid & 31) == 0) bad = 1;
    } else if (J < 3 && (warp & 3)) {
      // deferred work of block column JJ = J + 1, on the warps that do not
      // share warp 0's scheduler (warp w runs on sub-partition w % 4)
      const int JJ = J + 1, th = (warp - 1 - (warp >> 2)) * 32 + (tid & 31), nth = LDL_HT;
      if (JJ >= 2) {
        blk_trsm(A, X + JJ * 32 * LDL_LDX, JJ, 0, 32 * (JJ - 1), th, nth, helpers_sync);
        blk_update(A, JJ, 0, 32 * (JJ - 1), 0, 32 * JJ, th, nth);
      }
      if (has_next) blk_solve<32>(T, A, X + JJ * 32 * LDL_LDX, JJ, th, nth, helpers_sync);
    }
    __syncthreads();
    if (J == 0) break;
    blk_trsm(A, X + J * 32 * LDL_LDX, J, 32 * (J - 1), 32, tid, LDL_FT, all_sync);
    blk_update(A, J, 32 * (J - 1), 32, 32 * (J - 1), 32, tid, LDL_FT);
    __syncthreads();
  }
  if (has_next) blk_solve<32>(T, A, X, 0, tid, LDL_FT, all_sync);

  {
    // R_pp, X_J and D: every CTA holds the same factor, so the CTAs split
    // the stores (CTA c: rows / blocks c, c + gridDim.x, ... of four)
    if (blockIdx.x == 0 && tid == 0 && bad) record_status(QUIP_ERR_NOT_PD);
    const int nc = gridDim.x;
    for (int e = tid + LDL_FT * blockIdx.x; e < LDL_PB * 32; e += LDL_FT * nc) {
      const int i = e >> 5, j4 = (e & 31) * 4;
      const float4 v = *reinterpret_cast<const float4*>(A + i * LDL_LDA + j4);
      *reinterpret_cast<float4*>(Rd + i * LDL_PB + j4) =
          make_float4(j4 >= i ? v.x : 0.f, j4 + 1 >= i ? v.y : 0.f, j4 + 2 >= i ? v.z : 0.f,
                      j4 + 3 >= i ? v.w : 0.f);
    }
    for (int e = tid + LDL_FT * blockIdx.x; e < 4 * 32 * 32; e += LDL_FT * nc)
      Xw[e] = X[(e >> 10) * 32 * LDL_LDX + ((e >> 5) & 31) * LDL_LDX + (e & 31)];
    if (blockIdx.x == 0)
      for (int k = tid; k < w; k += LDL_FT) {
        const float r = A[k * LDL_LDA + k];
        Dv[c0 + k] = r * r;
      }
  }
  {
    // this CTA's share of the block's Ů
    const int rows = LDL_PB / gridDim.x, i0 = rows * blockIdx.x;
    for (int e = tid; e < rows * LDL_PB; e += LDL_FT) {
      const int i = i0 + (e >> 7), j = e & 127;
      if (i < j && j < w) H[(c0 + i) * n + c0 + j] = A[i * LDL_LDA + j] / A[j * LDL_LDA + j];
    }
  }
  if (has_next) {
    for (int e = tid; e < 32 * 32; e += LDL_FT) {
      const int i = e >> 5, j4 = (e & 31) * 4;
      *reinterpret_cast<float4*>(Nx + (32 * blockIdx.x + i) * LDL_PB + j4) =
          *reinterpret_cast<const float4*>(T + i * LDL_LDA + j4);
    }
  }
}

// Tiles come in by TMA from fp32 2-D maps without swizzle whose boxes are
// LDL_LDA (or LDL_LDX) columns wide, so that they land with the padded smem
// row stride; rows and columns past a tensor's extent arrive as zeros.

// Row blocks r0 = row0 + 32 b .. + 31 (b = blockIdx.x, blockIdx.x +
// gridDim.x, ... < nblk) of panel p:
//   R12 = (H - Lin)[rows, panel p] R_pp^-T by block back substitution with
//         R_pp (Rd) and X_J (Xw); rows in [c0 - 128, c0) are taken from Nx;
//   Ů:    H[r, c0 + k] = R12[r][k] / R_kk          (k < w)
//   Rs:   R12 as three bf16 pieces Rs[q][r][k]     (piece stride n * 128; zero for k >= w)
//   Lout[r][j] = sum_k R12[r][k] Nx[j][k]          (panel p's update of panel p - 1)
// 256 threads; Lout's product: warp v columns [16 v, 16 v + 16), lane
// (rg, cg) rows rg + 8 a and columns 16 v + cg + 4 b.  R_pp, X_J and Nx are
// loaded once per CTA; the row tiles of each block on the mbarrier's next
// phase.
// Maps: mH32 / mL32 as for k_ldl_factor; mR: Rd (128 x 128, 128-row box);
// mX: Xw as 128 x 32 (box LDL_LDX wide); mN32 / mN128: Nx (32 / 128-row
// boxes).
// Dynamic smem: 128 + (2 x 32 + 2 x 128) x LDL_LDA x 4 + 128 x LDL_LDX x 4 bytes.
__global__ void __launch_bounds__(LDL_RT, 1)
    k_ldl_rows(const __grid_constant__ CUtensorMap mH32, const __grid_constant__ CUtensorMap mL32,
               const __grid_constant__ CUtensorMap mR, const __grid_constant__ CUtensorMap mX,
               const __grid_constant__ CUtensorMap mN32, const __grid_constant__ CUtensorMap mN128,
               float* __restrict__ H, int64_t n, int64_t c0, int w, int lin0, int64_t row0,
               int nblk, __nv_bfloat16* __restrict__ Rs, float* __restrict__ Lout) {
  extern __shared__ __align__(16) uint8_t ldl_smem_raw[];
  pdl_wait_then_release();
  float* T = align128(ldl_smem_raw);                 // LDL_RR x LDL_LDA: H - Lin, then R12
  float* Lt = T + LDL_RR * LDL_LDA;                  // LDL_RR x LDL_LDA: Lin rows, then Lout
  float* Rp = Lt + LDL_RR * LDL_LDA;                 // 128 x LDL_LDA: R_pp
  float* N = Rp + LDL_PB * LDL_LDA;                  // 128 x LDL_LDA: Nx
  float* X = N + LDL_PB * LDL_LDA;                   // 4 x 32 x LDL_LDX
  __shared__ float rkk[LDL_PB];
  __shared__ int ld_ok;
  __shared__ __align__(8) uint64_t ld_bar;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(&ld_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto all_sync = [] { __syncthreads(); };
  const int64_t pstride = n * LDL_PB;
  constexpr int RA = LDL_RR / 8;
  const int rg = lane & 7, cg = lane >> 3, cw = 16 * warp;
  int it = 0;
  for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x, ++it) {
    const int64_t r0 = row0 + (int64_t)blk * LDL_RR;
    const bool from_nx = r0 >= c0 - LDL_NX, lin = lin0 >= 0 && !from_nx;
    if (tid == 0) {
      constexpr uint32_t B128 = LDL_PB * LDL_LDA * 4, B32 = LDL_RR * LDL_LDA * 4,
                         BX = LDL_PB * LDL_LDX * 4;
      mbar_arrive_expect_tx(&ld_bar, B32 * (lin ? 2u : 1u) + (it == 0 ? 2u * B128 + BX : 0u));
      if (from_nx) {
        tma_load_2d(T, &mN32, &ld_bar, 0, (int)(r0 - c0 + LDL_NX));
      } else {
        tma_load_2d(T, &mH32, &ld_bar, (int)c0, (int)r0);
        if (lin) tma_load_2d(Lt, &mL32, &ld_bar, 0, lin0 + (int)r0);
      }
      if (it == 0) {
        tma_load_2d(X, &mX, &ld_bar, 0, 0);
        tma_load_2d(Rp, &mR, &ld_bar, 0, 0);
        tma_load_2d(N, &mN128, &ld_bar, 0, 0);
      }
      const bool ok = mbar_wait(&ld_bar, (uint32_t)(it & 1));
      if (!ok) mbar_wait(&ld_bar, (uint32_t)(it & 1));   // copies in flight: bounded again
      ld_ok = ok ? 1 : 0;
    }
    __syncthreads();
    if (!ld_ok) return;
    if (!from_nx) {
      // T = H - Lin on columns < w, zero past w
      for (int e = tid; e < LDL_RR * 32; e += LDL_RT) {
        const int i = e >> 5, j4 = (e & 31) * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j4 < w) {
          v = *reinterpret_cast<const float4*>(T + i * LDL_LDA + j4);
          if (lin) {
            const float4 l = *reinterpret_cast<const float4*>(Lt + i * LDL_LDA + j4);
            v.x -= l.x, v.y -= l.y, v.z -= l.z, v.w -= l.w;
          }
        }
        *reinterpret_cast<float4*>(T + i * LDL_LDA + j4) = v;
      }
    }
    if (it == 0 && tid < LDL_PB) rkk[tid] = Rp[tid * LDL_LDA + tid];
    __syncthreads();
    if (!from_nx)
      for (int J = 3; J >= 0; --J) blk_solve<LDL_RR>(T, Rp, X + J * 32 * LDL_LDX, J, tid, LDL_RT, all_sync);

    // Ů and the bf16 pieces, 4 columns per task
    for (int e = tid; e < LDL_RR * 32; e += LDL_RT) {
      const int i = e >> 5, k4 = (e & 31) * 4;
      const int64_t g = r0 + i;
      const float4 v = *reinterpret_cast<const float4*>(T + i * LDL_LDA + k4);
      if (k4 < w)
        *reinterpret_cast<float4*>(H + g * n + c0 + k4) =
            make_float4(v.x / rkk[k4], v.y / rkk[k4 + 1], v.z / rkk[k4 + 2], v.w / rkk[k4 + 3]);
      __nv_bfloat16 pc[3][4];
      split3(v.x, pc[0][0], pc[1][0], pc[2][0]);
      split3(v.y, pc[0][1], pc[1][1], pc[2][1]);
      split3(v.z, pc[0][2], pc[1][2], pc[2][2]);
      split3(v.w, pc[0][3], pc[1][3], pc[2][3]);
#pragma unroll
      for (int q = 0; q < 3; ++q)
        *reinterpret_cast<uint2*>(Rs + q * pstride + g * LDL_PB + k4) =
            *reinterpret_cast<const uint2*>(pc[q]);
    }

    // Lout = R12 Nx^T, staged in Lt for row-contiguous stores
    float acc[RA][4];
#pragma unroll
    for (int a = 0; a < RA; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
    dot_rows<RA, 4>(acc, T + rg * LDL_LDA, 8 * LDL_LDA, N + (cw + cg) * LDL_LDA, 4 * LDL_LDA, LDL_PB);
#pragma unroll
    for (int a = 0; a < RA; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) Lt[(rg + 8 * a) * LDL_LDA + cw + cg + 4 * b] = acc[a][b];
    __syncthreads();
    for (int e = tid; e < LDL_RR * 32; e += LDL_RT) {
      const int i = e >> 5, j4 = (e & 31) * 4;
      *reinterpret_cast<float4*>(Lout + (r0 + i) * LDL_PB + j4) =
          *reinterpret_cast<const float4*>(Lt + i * LDL_LDA + j4);
    }
    fence_proxy_async_smem();                         // T and Lt free for the next block's copies
    __syncthreads();
  }
}

}  // namespace quip
