// Proxy Hessian finalisation (QuIP, adaptive-rounding section: H is the
// second moment of the calibration inputs; Experiments, "Methods.": damping
// H <- H + alpha * mean(diag(H)) * I).
//
// The accumulation itself (sum_t x_t x_t^T) is the tensor-core SYRK in
// syrk_tc.cuh for bf16 activations, or the FFMA GEMM for fp32 activations.
#pragma once

#include "common.cuh"

namespace quip {

// One CTA: diag <- diag / N + damp * trace / (N * n).  Reading and writing
// only the diagonal in one CTA keeps the trace free of races and scratch.
__global__ void __launch_bounds__(1024) k_finalize_diag(float* H, int64_t n, double inv_N,
                                                        double damp) {
  __shared__ double red[32];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s += (double)H[i * n + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  double tr = 0.0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tr += red[w];
  const double mu = damp * tr * inv_N / (double)n;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
    const float d = (float)((double)H[i * n + i] * inv_N + mu);
    H[i * n + i] = d;
    if (!isfinite(d)) record_status(QUIP_ERR_NONFINITE);
  }
}

// Strict lower triangle -> scaled by 1/N and mirrored into the upper one.
// 32 x 32 tiles (bi >= bj), staged through shared memory so both the read
// and the transposed write are coalesced.
__global__ void __launch_bounds__(256) k_mirror_scale(float* H, int64_t n, float inv_N) {
  const int64_t bi = blockIdx.y, bj = blockIdx.x;
  if (bi < bj) return;
  __shared__ float t[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r = ty; r < 32; r += 8) {
    const int64_t i = bi * 32 + r, j = bj * 32 + tx;
    float v = 0.f;
    if (i < n && j < n && i > j) {
      v = H[i * n + j] * inv_N;
      H[i * n + j] = v;
    }
    t[r][tx] = v;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int64_t i = bj * 32 + r, j = bi * 32 + tx;   // upper element (i < j)
    if (i < n && j < n && j > i) H[i * n + j] = t[tx][r];
  }
}

}  // namespace quip
