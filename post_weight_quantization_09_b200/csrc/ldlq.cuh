// LDLQ adaptive rounding (QuIP, adaptive-rounding section: LDLQ rounds
// column k of the incoherent weights after adding the linear feedback
// (W - W^) Ů_k of the columns already rounded; "Methods.": LDLQ = OPTQ),
// on a per-row b-bit min/max grid.
//
// Blocked over BLK columns: inside a block every column's error is fed back
// to the block's later columns at once (k_ldlq_chunk8); across blocks the
// feedback sum is split recursively (see quip_ldlq_quantize): the errors of
// a left half of the columns reach the right half in one tensor-core GEMM,
// A[:, right] += Err[:, left] * Ů[left, right].  The accumulator A starts as
// W~ and collects the feedback of all earlier columns.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace quip {

// Per row: lo = min, s = (max - min) / qmax (s = 1 for a constant row).
// One warp per row.
__global__ void __launch_bounds__(256) k_row_grid(const float* __restrict__ Wt, int64_t m,
                                                  int64_t n, int qmax, float* lo, float* sc) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= m) return;
  const float* w = Wt + row * n;
  float mn = INFINITY, mx = -INFINITY;
  bool fin = true;
  if ((n & 3) == 0) {
    for (int64_t j = 4 * lane; j < n; j += 128) {
      const float4 v = *reinterpret_cast<const float4*>(w + j);
      mn = fminf(mn, fminf(fminf(v.x, v.y), fminf(v.z, v.w)));
      mx = fmaxf(mx, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
      fin &= isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w);
    }
  } else {
    for (int64_t j = lane; j < n; j += 32) {
      mn = fminf(mn, w[j]);
      mx = fmaxf(mx, w[j]);
      fin &= isfinite(w[j]);
    }
  }
  mn = warp_min(mn);
  mx = warp_max(mx);
  fin = __all_sync(0xffffffffu, fin);
  if (lane == 0) {
    if (!fin) record_status(QUIP_ERR_NONFINITE);
    lo[row] = mn;
    sc[row] = (mx > mn) ? (mx - mn) / (float)qmax : 1.0f;
  }
}

// Block step: 8 threads per row (16 rows per CTA); thread q owns
// the 16 contiguous columns j = 16 q + t of a 128-column block (BLK / 8 in
// general) in registers.  Columns are taken in 8 chunks of 16, chunk c owned
// by thread c: inside a chunk the step is unrolled, so the rounded column is
// the compile-time register a[t]; the error is broadcast by one shuffle from
// the owner and every thread adds err * Ů[k][16 q + t] to all its registers
// (Ů[k][j] = 0 for j <= k), reading the Ů row slice with four 16-byte loads
// from a padded, conflict-free layout Us[k][q][t] (row stride NT + 4).
// Errors go out as three bf16 pieces Es[p][row][k0 + j] (row stride lde,
// piece stride m * lde).
template <int BLK>
__global__ void __launch_bounds__(128) k_ldlq_chunk8(const float* __restrict__ Wt,
                                                     const float* __restrict__ A, int64_t m,
                                                     int64_t n, int64_t k0,
                                                     const float* __restrict__ U, int64_t ldu,
                                                     const float* __restrict__ lo,
                                                     const float* __restrict__ sc, float qmax,
                                                     uint8_t* __restrict__ codes,
                                                     __nv_bfloat16* __restrict__ Es, int64_t lde) {
  constexpr int NT = BLK / 8;                   // columns per thread
  constexpr int QS = NT + 4;                    // padded per-thread stride in Us
  constexpr int KS = 8 * QS;                    // Us row stride
  constexpr int RPC = 16;
  constexpr int LDT = BLK + 4;
  constexpr int V4 = BLK / 4;
  extern __shared__ __align__(16) float smem[];
  float* Us = smem;                             // [k][q][t], BLK x KS
  float* tile = Us + BLK * KS;                  // RPC x LDT staging
  uint8_t* ctile = reinterpret_cast<uint8_t*>(tile + RPC * LDT);
  const int tid = threadIdx.x, lane = tid & 31, q = tid & 7, rl = tid >> 3;
  const int64_t r0 = (int64_t)blockIdx.x * RPC;

  // Ů block (strict upper part), 16-byte loads and stores
#pragma unroll 8
  for (int e = tid; e < BLK * V4; e += 128) {
    const int k = e / V4, j4 = (e % V4) * 4;
    float4 u = *reinterpret_cast<const float4*>(U + (k0 + k) * ldu + k0 + j4);
    u.x = (j4 > k) ? u.x : 0.f;
    u.y = (j4 + 1 > k) ? u.y : 0.f;
    u.z = (j4 + 2 > k) ? u.z : 0.f;
    u.w = (j4 + 3 > k) ? u.w : 0.f;
    *reinterpret_cast<float4*>(Us + k * KS + (j4 / NT) * QS + (j4 % NT)) = u;
  }
  float a[NT], w[NT];
#pragma unroll 4
  for (int e = tid; e < RPC * V4; e += 128) {
    const int r = e / V4, j4 = (e % V4) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < m) v = *reinterpret_cast<const float4*>(A + (r0 + r) * n + k0 + j4);
    *reinterpret_cast<float4*>(tile + r * LDT + j4) = v;
  }
  __syncthreads();
#pragma unroll
  for (int t = 0; t < NT; ++t) a[t] = tile[rl * LDT + NT * q + t];
  __syncthreads();
#pragma unroll 4
  for (int e = tid; e < RPC * V4; e += 128) {
    const int r = e / V4, j4 = (e % V4) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < m) v = *reinterpret_cast<const float4*>(Wt + (r0 + r) * n + k0 + j4);
    *reinterpret_cast<float4*>(tile + r * LDT + j4) = v;
  }
  __syncthreads();
#pragma unroll
  for (int t = 0; t < NT; ++t) w[t] = tile[rl * LDT + NT * q + t];
  __syncthreads();

  const int64_t row = r0 + rl;
  const float l = (row < m) ? lo[row] : 0.f;
  const float s = (row < m) ? sc[row] : 1.f;
  const float inv = 1.0f / s;
  const int base = lane & ~7;
#pragma unroll 1
  for (int c = 0; c < 8; ++c) {                  // chunk c: columns NT c .. NT c + NT - 1
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int k = NT * c + t;
      const float z = (a[t] - l) * inv;
      const float cq = fminf(fmaxf(rintf(z), 0.f), qmax);
      const float err_own = w[t] - fmaf(s, cq, l);
      const float err = __shfl_sync(0xffffffffu, err_own, base | c);
      if (q == c) {
        tile[rl * LDT + k] = err;
        ctile[rl * BLK + k] = (uint8_t)cq;
      }
      const float4* ur = reinterpret_cast<const float4*>(Us + k * KS + q * QS);
#pragma unroll
      for (int v = 0; v < NT / 4; ++v) {
        const float4 u = ur[v];
        a[4 * v] = fmaf(err, u.x, a[4 * v]);
        a[4 * v + 1] = fmaf(err, u.y, a[4 * v + 1]);
        a[4 * v + 2] = fmaf(err, u.z, a[4 * v + 2]);
        a[4 * v + 3] = fmaf(err, u.w, a[4 * v + 3]);
      }
    }
  }
  __syncthreads();
  const int64_t pst = m * lde;
  for (int e = tid; e < RPC * BLK; e += 128) {
    const int r = e / BLK, j = e % BLK;
    if (r0 + r < m) {
      __nv_bfloat16 p0, p1, p2;
      split3(tile[r * LDT + j], p0, p1, p2);
      const int64_t o = (r0 + r) * lde + k0 + j;
      Es[o] = p0;
      Es[pst + o] = p1;
      Es[2 * pst + o] = p2;
      codes[(r0 + r) * n + k0 + j] = ctile[r * BLK + j];
    }
  }
}

// W~^[i][j] = lo[i] + s[i] * codes[i][j]
__global__ void k_dequant(const uint8_t* __restrict__ codes, const float* __restrict__ lo,
                          const float* __restrict__ sc, int64_t m, int64_t n, float* out) {
  const int64_t total = m * n;
  for (int64_t e = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) * 4; e < total;
       e += (int64_t)gridDim.x * blockDim.x * 4) {
    if (e + 3 < total && (n & 3) == 0) {
      const int64_t i = e / n;
      const uchar4 c = *reinterpret_cast<const uchar4*>(codes + e);
      const float l = lo[i], s = sc[i];
      float4 v;
      v.x = fmaf(s, (float)c.x, l), v.y = fmaf(s, (float)c.y, l);
      v.z = fmaf(s, (float)c.z, l), v.w = fmaf(s, (float)c.w, l);
      *reinterpret_cast<float4*>(out + e) = v;
    } else {
      for (int64_t f = e; f < e + 4 && f < total; ++f) {
        const int64_t i = f / n;
        out[f] = fmaf(sc[i], (float)codes[f], lo[i]);
      }
    }
  }
}

}  // namespace quip
