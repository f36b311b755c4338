// The quantized layer times full-precision vectors, for inference (QuIP,
// Experiments, "Throughput Comparison.": a quantized-matrix full-precision-
// vector product, with the incoherence processing applied around it):
//   y = W^ x = U^T (W~^ (V x)),   W~^[i][j] = lo_i + s_i c_ij,
// so the product in the incoherent domain is
//   z_i = lo_i sum_j x'_j + s_i sum_j c_ij x'_j,   x' = V x,
// and y = U^T z.  This file holds the packing of the codes, the product
// with the two transforms in the same launch (k_qlinear: Hadamard or
// identity sides), a Kronecker side on a few vectors (k_kron_vec), and the
// bare product (k_qmatvec) that the library's row transforms and gathers
// surround when a side permutes.
//
// Packed layout (see quip.h): code j of row i sits in word j mod Wd of the
// row at bit (j div Wd) * slot, Wd a multiple of 4.  A lane that loads the
// 16-byte group of words 4q..4q+3 thus holds, for each slot t, the codes of
// the four consecutive columns Wd t + 4q .. + 3, and reads their x' as one
// float4: consecutive lanes read consecutive float4s.
#pragma once

#include <utility>

#include "common.cuh"

namespace quip {

// One thread per packed word: word w of row i collects codes w + Wd t.
template <int SLOT>
__global__ void __launch_bounds__(256) k_pack_codes(const uint8_t* __restrict__ codes, int64_t m,
                                                    int64_t n, int64_t Wd, uint32_t* __restrict__ packed,
                                                    int64_t ldp) {
  constexpr int PER = 32 / SLOT;
  constexpr uint32_t MASK = (1u << SLOT) - 1u;
  const int64_t total = m * Wd;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / Wd, w = e % Wd;
    const uint8_t* c = codes + i * n;
    uint32_t v = 0;
#pragma unroll
    for (int t = 0; t < PER; ++t) {
      const int64_t j = w + Wd * t;
      if (j < n) v |= ((uint32_t)c[j] & MASK) << (t * SLOT);
    }
    packed[i * ldp + w] = v;
  }
}

// Rows per warp task for a chunk of BC vectors: x' is read once per slot
// and feeds R rows, so more rows per warp cut the x' traffic (BC x 4 bytes
// per code / R) while fewer keep more warps in flight.
template <int BC>
__host__ __device__ constexpr int qmv_rows() { return BC >= 4 ? 4 : BC; }

// A code c of a SLOT-bit slot as an fp32 value, two integer operations:
// for SLOT <= 4 the float 1 + c 2^-SLOT (c moved to the top mantissa bits
// of 1.0), so sum_j f_j x_j = S + 2^-SLOT sum_j c_j x_j; for SLOT = 8 the
// float 2^23 + c, minus 2^23 (exact).  qmv_code_sum turns the accumulated
// sum back into sum_j c_j x_j given S = sum_j x_j over the same columns.
template <int SLOT, int T>
__device__ __forceinline__ float qmv_code(uint32_t w) {
  constexpr uint32_t MASK = (1u << SLOT) - 1u;
  if constexpr (SLOT == 8) {
    return __uint_as_float(0x4B000000u | ((w >> (T * SLOT)) & MASK)) - 8388608.f;
  } else {
    constexpr int SH = (23 - SLOT) - T * SLOT;         // code bits -> mantissa bits 23-SLOT .. 22
    const uint32_t v = SH >= 0 ? (w << (SH >= 0 ? SH : 0)) : (w >> (SH < 0 ? -SH : 0));
    return __uint_as_float((v & (MASK << (23 - SLOT))) | 0x3F800000u);
  }
}
template <int SLOT>
__device__ __forceinline__ float qmv_code_sum(float acc, float S) {
  if constexpr (SLOT == 8) return acc;
  else return (acc - S) * (float)(1 << SLOT);
}

// acc[r][b] += sum over one 16-byte word group of R rows (words 4q..4q+3,
// every slot) of the decoded codes times x'; xload(b, j) returns the float4
// of vector b at columns j..j+3.  Slots past column n are skipped (n % 4 ==
// 0: whole groups).
template <int SLOT, int BC, int R, int T, typename XLoad>
__device__ __forceinline__ void qmv_slot(const uint4 (&w)[R], int Wd, int j0, int nslot, XLoad xload,
                                         float (&acc)[R][BC]) {
  if (T < nslot) {
    const int j = j0 + Wd * T;
    float c[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      c[r][0] = qmv_code<SLOT, T>(w[r].x);
      c[r][1] = qmv_code<SLOT, T>(w[r].y);
      c[r][2] = qmv_code<SLOT, T>(w[r].z);
      c[r][3] = qmv_code<SLOT, T>(w[r].w);
    }
#pragma unroll
    for (int b = 0; b < BC; ++b) {
      const float4 xv = xload(b, j);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        acc[r][b] = fmaf(c[r][0], xv.x, acc[r][b]);
        acc[r][b] = fmaf(c[r][1], xv.y, acc[r][b]);
        acc[r][b] = fmaf(c[r][2], xv.z, acc[r][b]);
        acc[r][b] = fmaf(c[r][3], xv.w, acc[r][b]);
      }
    }
  }
}
template <int SLOT, int BC, int R, typename XLoad, int... Ts>
__device__ __forceinline__ void qmv_slots(const uint4 (&w)[R], int Wd, int j0, int nslot, XLoad xload,
                                          float (&acc)[R][BC], std::integer_sequence<int, Ts...>) {
  (qmv_slot<SLOT, BC, R, Ts>(w, Wd, j0, nslot, xload, acc), ...);
}
// One 16-byte word group q of R rows: every slot whose columns Wd t + 4q ..
// + 3 lie below n (n % 4 == 0: whole groups).
template <int SLOT, int BC, int R, typename XLoad>
__device__ __forceinline__ void qmv_group(const uint4 (&w)[R], int Wd, int q, int n, XLoad xload,
                                          float (&acc)[R][BC]) {
  const int j0 = 4 * q;
  const int nslot = (n - j0 + Wd - 1) / Wd;            // slots t with j0 + Wd t < n
  qmv_slots<SLOT, BC, R>(w, Wd, j0, nslot, xload, acc, std::make_integer_sequence<int, 32 / SLOT>{});
}

// One warp task: rows r0 .. r0 + R - 1 (past m: zero words), all groups.
template <int SLOT, int BC, int R, typename XLoad>
__device__ __forceinline__ void qmv_task(const uint32_t* __restrict__ packed, int64_t ldp, int64_t Wd,
                                         int64_t m, int64_t n, int64_t r0, int lane, XLoad xload,
                                         float (&acc)[R][BC]) {
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int b = 0; b < BC; ++b) acc[r][b] = 0.f;
  const int nq = (int)(Wd / 4);
  const uint4* rows[R];
#pragma unroll
  for (int r = 0; r < R; ++r)
    rows[r] = reinterpret_cast<const uint4*>(packed + (r0 + r < m ? r0 + r : r0) * ldp);
  for (int q = lane; q < nq; q += 32) {
    uint4 w[R];
#pragma unroll
    for (int r = 0; r < R; ++r) w[r] = (r0 + r < m) ? __ldg(rows[r] + q) : make_uint4(0u, 0u, 0u, 0u);
    qmv_group<SLOT, BC, R>(w, (int)Wd, q, (int)n, xload, acc);
  }
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int b = 0; b < BC; ++b)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[r][b] += __shfl_xor_sync(0xffffffffu, acc[r][b], o);
}

// z[b][i] = lo_i S_b + s_i sum_j c_ij x'[b][j] for nb <= BC vectors (S_b =
// sum_j x'[b][j]; x' rows of n fp32, n % 4 == 0, 16-byte aligned, read
// through L1).  Warp tasks of qmv_rows<BC>() rows, grid-stride.  Each warp
// sums x' on its first task; the other tasks reuse it.
constexpr int QMV_WARPS = 8;
template <int SLOT, int BC>
__global__ void __launch_bounds__(QMV_WARPS * 32) k_qmatvec(const uint32_t* __restrict__ packed,
                                                            int64_t ldp, int64_t Wd,
                                                            const float* __restrict__ lo,
                                                            const float* __restrict__ sc, int64_t m,
                                                            int64_t n, const float* __restrict__ xs,
                                                            int64_t ldx, int nb, float* __restrict__ z,
                                                            int64_t ldz) {
  constexpr int R = qmv_rows<BC>();
  const int lane = threadIdx.x & 31;
  const int64_t ntask = (m + R - 1) / R;
  float S[BC];
  bool first = true;
  auto xload = [=](int b, int j) {
    return b < nb ? __ldg(reinterpret_cast<const float4*>(xs + b * ldx + j)) : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  for (int64_t task = (int64_t)blockIdx.x * QMV_WARPS + (threadIdx.x >> 5); task < ntask;
       task += (int64_t)gridDim.x * QMV_WARPS) {
    if (first) {
      // S_b over this lane's columns, then across the warp
#pragma unroll
      for (int b = 0; b < BC; ++b) {
        float v = 0.f;
        for (int64_t j = 4 * lane; j < n; j += 128) {
          const float4 xv = xload(b, j);
          v += (xv.x + xv.y) + (xv.z + xv.w);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        S[b] = v;
      }
      first = false;
    }
    const int64_t r0 = task * R;
    float acc[R][BC];
    qmv_task<SLOT, BC, R>(packed, ldp, Wd, m, n, r0, lane, xload, acc);
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int64_t row = r0 + r;
        if (row < m) {
          const float l = lo[row], s = sc[row];
#pragma unroll
          for (int b = 0; b < BC; ++b)
            if (b < nb) z[b * ldz + row] = fmaf(s, qmv_code_sum<SLOT>(acc[r][b], S[b]), l * S[b]);
        }
      }
    }
  }
}

// In-place Walsh-Hadamard transform (Sylvester order, unnormalised) of nvec
// vectors of length d = 2^L in shared memory, v[b * ld + i]; the whole CTA
// takes part.  Passes of up to four butterfly stages: in the pass over
// stages g0 .. g0 + r - 1 a thread loads the 2^r elements base + k 2^g0 of a
// chunk into registers, runs the r stages there and stores them back; one
// barrier per pass.
__device__ __forceinline__ void smem_fwht(float* v, int d, int nvec, int ld) {
  const int L = 31 - __clz(d);
  for (int g0 = 0; g0 < L; g0 += 4) {
    const int r = min(4, L - g0);
    const int cnt = 1 << r, h0 = 1 << g0, nchunk = d >> r;
    for (int e = threadIdx.x; e < nvec * nchunk; e += blockDim.x) {
      const int b = e / nchunk, c = e - b * nchunk;
      const int base = ((c >> g0) << (g0 + r)) | (c & (h0 - 1));
      float* p = v + b * ld + base;
      float a[16];
      if (g0 == 0 && cnt == 16) {
        // 16 consecutive elements: four 16-byte loads (ld % 4 == 0)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 f = reinterpret_cast<const float4*>(p)[k];
          a[4 * k] = f.x, a[4 * k + 1] = f.y, a[4 * k + 2] = f.z, a[4 * k + 3] = f.w;
        }
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) a[k] = k < cnt ? p[k * h0] : 0.f;
      }
#pragma unroll
      for (int st = 1; st < 16; st <<= 1) {
        if (st < cnt) {
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if ((k & st) == 0) {
              const float x0 = a[k], x1 = a[k + st];
              a[k] = x0 + x1;
              a[k + st] = x0 - x1;
            }
        }
      }
      if (g0 == 0 && cnt == 16) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          reinterpret_cast<float4*>(p)[k] = make_float4(a[4 * k], a[4 * k + 1], a[4 * k + 2], a[4 * k + 3]);
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k)
          if (k < cnt) p[k * h0] = a[k];
      }
    }
    __syncthreads();
  }
}

// One launch per product for layers whose two sides are randomized Hadamard
// (or identity) without permutation:
//   prologue (every CTA): x' = H_n (s_n . x) for the chunk's vectors, in
//     shared memory (the 1 / sqrt(n) is applied to z at the end), and
//     S_b = sum x';
//   body: z = lo S + s (codes x'), warp tasks as in k_qmatvec with x' from
//     shared memory, written to the workspace z (B x m);
//   epilogue: each CTA publishes its rows (fence, then a ticket from an
//     atomic counter); the CTA that draws the last ticket reads all of z and
//     writes y = s_m . (H_m z) / sqrt(m) (U^T z), then resets the counter.
// Nothing waits on another CTA: the last CTA is the one that finds every
// other CTA done.  vs / us = the sides' signs (NULL: identity side),
// vscale / uscale = their 1 / sqrt(d) (1 for an identity side).
// Warps per CTA: 32 for one or two vectors (registers allow it), else 8.
template <int BC>
__host__ __device__ constexpr int ql_warps() { return BC <= 2 ? 32 : 8; }
template <int SLOT, int BC, typename TX>
__global__ void __launch_bounds__(ql_warps<BC>() * 32) k_qlinear(const uint32_t* __restrict__ packed,
                                                            int64_t ldp, int64_t Wd,
                                                            const float* __restrict__ lo,
                                                            const float* __restrict__ sc, int m, int n,
                                                            const TX* __restrict__ x, int64_t ldx, int nb,
                                                            const float* __restrict__ vs, float vscale,
                                                            const float* __restrict__ us, float uscale,
                                                            float* __restrict__ z,
                                                            unsigned* __restrict__ counter,
                                                            float* __restrict__ y, int64_t ldy) {
  constexpr int R = qmv_rows<BC>();
  constexpr int QL_WARPS = ql_warps<BC>();
  extern __shared__ __align__(16) float qlv[];         // [BC][ld]
  __shared__ float qls[QL_WARPS][BC];
  __shared__ float qlS[BC];
  __shared__ unsigned ql_last;
  const int ld = (max(n, m) + 3) & ~3;                  // 16-byte aligned vector rows
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // ---- prologue: x' = H (s . x) per vector
#pragma unroll
  for (int b = 0; b < BC; ++b)
    for (int j = tid; j < n; j += blockDim.x) {
      float v = 0.f;
      if (b < nb) {
        v = to_f32(x[b * ldx + j]);
        if (vs) v *= vs[j];
      }
      qlv[b * ld + j] = v;
    }
  __syncthreads();
  if (vs) smem_fwht(qlv, n, BC, ld);
  float part[BC];
#pragma unroll
  for (int b = 0; b < BC; ++b) part[b] = 0.f;
  for (int j = tid; j < n; j += blockDim.x)
#pragma unroll
    for (int b = 0; b < BC; ++b) part[b] += qlv[b * ld + j];
#pragma unroll
  for (int b = 0; b < BC; ++b) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part[b] += __shfl_xor_sync(0xffffffffu, part[b], o);
    if (lane == 0) qls[warp][b] = part[b];
  }
  __syncthreads();
  if (tid < BC) {
    float v = 0.f;
    for (int w = 0; w < QL_WARPS; ++w) v += qls[w][tid];
    qlS[tid] = v;
  }
  __syncthreads();
  // ---- body
  auto xload = [=](int b, int j) { return *reinterpret_cast<const float4*>(qlv + b * ld + j); };
  const int64_t ntask = (m + R - 1) / R;
  for (int64_t task = (int64_t)blockIdx.x * QL_WARPS + warp; task < ntask;
       task += (int64_t)gridDim.x * QL_WARPS) {
    const int64_t r0 = task * R;
    float acc[R][BC];
    qmv_task<SLOT, BC, R>(packed, ldp, Wd, m, n, r0, lane, xload, acc);
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int64_t row = r0 + r;
        if (row < m) {
          const float l = lo[row], s = sc[row];
#pragma unroll
          for (int b = 0; b < BC; ++b)
            if (b < nb)
              z[b * (int64_t)m + row] = vscale * fmaf(s, qmv_code_sum<SLOT>(acc[r][b], qlS[b]), l * qlS[b]);
        }
      }
    }
  }
  // ---- epilogue: the last CTA to finish applies U^T
  __threadfence();
  __syncthreads();
  if (tid == 0) ql_last = (atomicAdd(counter, 1u) == gridDim.x - 1) ? 1u : 0u;
  __syncthreads();
  if (!ql_last) return;
  __threadfence();
#pragma unroll
  for (int b = 0; b < BC; ++b)
    for (int i = tid; i < m; i += blockDim.x) qlv[b * ld + i] = b < nb ? __ldcg(z + b * (int64_t)m + i) : 0.f;
  __syncthreads();
  if (us) smem_fwht(qlv, m, BC, ld);
  for (int b = 0; b < nb; ++b)
    for (int i = tid; i < m; i += blockDim.x) {
      float v = qlv[b * ld + i] * uscale;
      if (us) v *= us[i];
      y[b * ldy + i] = v;
    }
  if (tid == 0) *counter = 0u;
}

// Kronecker side applied to a few vectors: y_b = (A (x) B) x_b (forward) or
// (A (x) B)^T x_b (inverse), x_b read as the p x q matrix X (x[a q + c]):
// forward Y = A X B^T, inverse Y = A^T X B.  One CTA of 256 threads per
// (output row a, vector b): u = sum_a' A[a][a'] X[a'] (A[a'][a] inverse),
// then Y[a][c] = sum_c' u[c'] B[c][c'] forward (a warp per output c, lanes
// along the row of B), or sum_c' u[c'] B[c'][c] inverse (a thread per c,
// coalesced down the columns).  p, q <= 1024.
__global__ void __launch_bounds__(256) k_kron_vec(const float* __restrict__ A, const float* __restrict__ Bm,
                                                  int p, int q, int inverse, const float* __restrict__ x,
                                                  int64_t ldx, float* __restrict__ y, int64_t ldy) {
  __shared__ float u[1024];
  const int a = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* xb = x + b * ldx;
  for (int c = tid; c < q; c += blockDim.x) {
    float v0 = 0.f, v1 = 0.f;
    int a2 = 0;
    for (; a2 + 1 < p; a2 += 2) {
      const float w0 = inverse ? A[a2 * p + a] : A[a * p + a2];
      const float w1 = inverse ? A[(a2 + 1) * p + a] : A[a * p + a2 + 1];
      v0 = fmaf(w0, xb[a2 * q + c], v0);
      v1 = fmaf(w1, xb[(a2 + 1) * q + c], v1);
    }
    if (a2 < p) v0 = fmaf(inverse ? A[a2 * p + a] : A[a * p + a2], xb[a2 * q + c], v0);
    u[c] = v0 + v1;
  }
  __syncthreads();
  float* yb = y + b * ldy + (int64_t)a * q;
  if (inverse) {
    for (int c = tid; c < q; c += blockDim.x) {
      float v = 0.f;
      for (int c2 = 0; c2 < q; ++c2) v = fmaf(u[c2], Bm[c2 * q + c], v);
      yb[c] = v;
    }
  } else {
    for (int c = warp; c < q; c += blockDim.x / 32) {
      float v = 0.f;
      for (int c2 = lane; c2 < q; c2 += 32) v = fmaf(u[c2], Bm[c * q + c2], v);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) yb[c] = v;
    }
  }
}

}  // namespace quip
