// LDLQ adaptive rounding (QuIP, adaptive-rounding section: LDLQ rounds
// column k of the incoherent weights after adding the linear feedback
// (W - W^) Ů_k of the columns already rounded; "Methods.": LDLQ = OPTQ),
// on a per-row b-bit min/max grid.
//
// Blocked over BLK columns ("lazy batch"): inside a block every column's
// error is fed back to the block's later columns at once (k_ldlq_block);
// when the block ends the trailing columns receive Err_blk * Ů[blk, rest]
// in one GEMM.  The accumulator A starts as W~ and collects the feedback of
// all earlier blocks.
#pragma once

#include "common.cuh"

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

// One block of BLK columns [k0, k0+BLK) for 32 rows per CTA, 4 threads per
// row; thread qd of a row owns columns j = 4t + qd (t < BLK/4) in registers.
// Column k: its owner rounds a_k, computes err = W~_k - (lo + s c_k), the
// error is broadcast inside the row's quad, and every thread adds
// err * Ů[k][j] to its later columns (Ů[k][j] = 0 for j <= k).
// Writes codes[:, k0:k0+BLK] and E = W~ - W^ for the block (m x BLK).
template <int BLK>
__global__ void __launch_bounds__(128) k_ldlq_block(const float* __restrict__ Wt,
                                                    const float* __restrict__ A, int64_t m,
                                                    int64_t n, int64_t k0,
                                                    const float* __restrict__ U, int64_t ldu,
                                                    const float* __restrict__ lo,
                                                    const float* __restrict__ sc, float qmax,
                                                    uint8_t* __restrict__ codes,
                                                    float* __restrict__ E) {
  constexpr int NT = BLK / 4;
  constexpr int LDT = BLK + 4;                  // padded staging row
  extern __shared__ __align__(16) float smem[];
  float* Uq = smem;                             // [k][qd][t], BLK*BLK floats
  float* tile = Uq + BLK * BLK;                 // 32 x LDT staging
  uint8_t* ctile = reinterpret_cast<uint8_t*>(tile + 32 * LDT);   // 32 x BLK codes
  const int tid = threadIdx.x, lane = tid & 31, qd = tid & 3, rl = tid >> 2;
  const int64_t r0 = (int64_t)blockIdx.x * 32;

  for (int e = tid; e < BLK * BLK; e += 128) {
    const int k = e / BLK, j = e % BLK;
    const float u = (j > k) ? U[(k0 + k) * ldu + k0 + j] : 0.f;
    Uq[k * BLK + (j & 3) * NT + (j >> 2)] = u;
  }
  float a[NT], w[NT];
  // stage A then W~ rows through shared memory (coalesced global reads)
  for (int e = tid; e < 32 * BLK; e += 128) {
    const int r = e / BLK, j = e % BLK;
    tile[r * LDT + j] = (r0 + r < m) ? A[(r0 + r) * n + k0 + j] : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int t = 0; t < NT; ++t) a[t] = tile[rl * LDT + 4 * t + qd];
  __syncthreads();
  for (int e = tid; e < 32 * BLK; e += 128) {
    const int r = e / BLK, j = e % BLK;
    tile[r * LDT + j] = (r0 + r < m) ? Wt[(r0 + r) * n + k0 + j] : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int t = 0; t < NT; ++t) w[t] = tile[rl * LDT + 4 * t + qd];
  __syncthreads();

  const int64_t row = r0 + rl;
  const float l = (row < m) ? lo[row] : 0.f;
  const float s = (row < m) ? sc[row] : 1.f;
  const float inv = 1.0f / s;
  const int base = lane & ~3;
#pragma unroll
  for (int k = 0; k < BLK; ++k) {
    const int own = k & 3, slot = k >> 2;
    const float z = (a[slot] - l) * inv;
    const float c = fminf(fmaxf(rintf(z), 0.f), qmax);
    const float err_own = w[slot] - fmaf(s, c, l);
    const float err = __shfl_sync(0xffffffffu, err_own, base | own);
    if (qd == own) {
      tile[rl * LDT + k] = err;
      ctile[rl * BLK + k] = (uint8_t)c;
    }
    const float* urow = Uq + k * BLK + qd * NT;
#pragma unroll
    for (int t = slot; t < NT; ++t) a[t] = fmaf(err, urow[t], a[t]);
  }
  __syncthreads();
  for (int e = tid; e < 32 * BLK; e += 128) {
    const int r = e / BLK, j = e % BLK;
    if (r0 + r < m) {
      E[(r0 + r) * BLK + j] = tile[r * LDT + j];
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
