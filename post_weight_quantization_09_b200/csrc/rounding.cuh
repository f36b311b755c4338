// The rounding methods beside LDLQ (QuIP, Experiments, "Methods."):
// nearest rounding; LDLQ-RG's quantisation order, the columns by decreasing
// diag(H); and the greedy updates of the proxy tr((W^ - W) H (W^ - W)^T)
// that "Greedy" performs alone and LDLQ-RG after LDLQ.
//
// A greedy pass visits the columns k = 0..n-1 and sets column k, per row, to
// the grid point nearest
//   t_k = W_k - sum_{j != k} (W^_j - W_j) H_jk / H_kk,
// the minimiser of the proxy over that column with the others held.  With
// E = W^old - W (the codes at the start of the pass) and d_j the change of
// column j during the pass, t_k = W^old_k - (E H)_k / H_kk
//                                  - sum_{j < k} d_j H_jk / H_kk.
// That is LDLQ's recursion with
//   accumulator start  T = W^old - (E H) D^-1          (one full GEMM),
//   "weights"          W^old  (so the error of column j is -d_j),
//   feedback factor    U'_jk = H_jk / H_kk for j < k,
// so a pass runs on the LDLQ machinery: the block kernel inside 128-column
// blocks, tensor-core GEMMs across them (see quip_greedy_refine).
#pragma once

#include "common.cuh"
#include "ldlq.cuh"

namespace quip {

// codes[i][j] = clamp(rint((W[i][j] - lo_i) / s_i), 0, qmax) with the fp32
// steps of the LDLQ block kernel's rounding (multiply by 1 / s, clamp, then
// add and subtract 1.5 * 2^23: round half to even).  Rows i = blockIdx.y,
// + gridDim.y, ...; with vec (n % 4 == 0, W 16-byte and codes 4-byte
// aligned) each thread rounds 4-element groups, else single elements.
constexpr int NR_THREADS = 256;
__device__ __forceinline__ uint32_t round_code(float w, float l, float inv, float qmax) {
  const float zr = fminf(fmaxf((w - l) * inv, 0.f), qmax) + 12582912.0f;
  return __float_as_uint(zr) & 0xffu;
}
__global__ void __launch_bounds__(NR_THREADS) k_nearest(const float* __restrict__ W,
                                                        const float* __restrict__ lo,
                                                        const float* __restrict__ sc, int64_t m,
                                                        int64_t n, int vec, float qmax,
                                                        uint8_t* __restrict__ codes) {
  for (int64_t i = blockIdx.y; i < m; i += gridDim.y) {
    const float l = lo[i], inv = 1.0f / sc[i];
    const float* w = W + i * n;
    uint8_t* c = codes + i * n;
    if (vec) {
      for (int64_t j = 4 * ((int64_t)blockIdx.x * NR_THREADS + threadIdx.x); j < n;
           j += 4 * (int64_t)gridDim.x * NR_THREADS) {
        const float4 v = *reinterpret_cast<const float4*>(w + j);
        *reinterpret_cast<uint32_t*>(c + j) =
            round_code(v.x, l, inv, qmax) | (round_code(v.y, l, inv, qmax) << 8) |
            (round_code(v.z, l, inv, qmax) << 16) | (round_code(v.w, l, inv, qmax) << 24);
      }
    } else {
      for (int64_t j = (int64_t)blockIdx.x * NR_THREADS + threadIdx.x; j < n;
           j += (int64_t)gridDim.x * NR_THREADS)
        c[j] = (uint8_t)round_code(w[j], l, inv, qmax);
    }
  }
}

// LDLQ-RG's order: perm[r] = the column with the r-th largest H_kk (equal
// values by increasing index), iperm[perm[r]] = r.  Rank by counting, as
// k_perm_rank: key(k) = (descending bits of H_kk) << 32 | k, all distinct;
// -0 is read as +0.  n <= 65536.
__device__ __forceinline__ uint64_t diag_key(const float* H, int64_t ldh, int64_t k) {
  float d = H[k * ldh + k];
  if (d == 0.f) d = 0.f;
  const uint32_t u = __float_as_uint(d);
  const uint32_t asc = (u & 0x80000000u) ? ~u : (u | 0x80000000u);   // increasing with d
  return ((uint64_t)(~asc) << 32) | (uint64_t)k;
}
__global__ void __launch_bounds__(256) k_diag_rank(const float* __restrict__ H, int64_t ldh,
                                                   int64_t n, int32_t* __restrict__ perm,
                                                   int32_t* __restrict__ iperm) {
  __shared__ uint64_t tile[PERM_TILE];
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const uint64_t ki = i < n ? diag_key(H, ldh, i) : 0ull;
  int32_t rank = 0;
  for (int64_t j0 = 0; j0 < n; j0 += PERM_TILE) {
    const int len = (int)min((int64_t)PERM_TILE, n - j0);
    __syncthreads();
    for (int t = threadIdx.x; t < len; t += blockDim.x) tile[t] = diag_key(H, ldh, j0 + t);
    __syncthreads();
#pragma unroll 8
    for (int t = 0; t < len; ++t) rank += tile[t] < ki ? 1 : 0;
  }
  if (i < n) {
    if (iperm) iperm[i] = rank;
    perm[rank] = (int32_t)i;
  }
}

// out[r][c] = in[rp[r]][cp[c]] for any element type T (a NULL index list is
// the identity).  An index outside [0, rows) / [0, cols) records
// QUIP_ERR_ARG and writes zero.  Rows by blockIdx.y (grid-stride).
template <typename T>
__global__ void __launch_bounds__(256) k_permute(const T* __restrict__ in, int64_t ldin,
                                                 T* __restrict__ out, int64_t ldout, int64_t rows,
                                                 int64_t cols, const int32_t* __restrict__ rp,
                                                 const int32_t* __restrict__ cp) {
  for (int64_t r = blockIdx.y; r < rows; r += gridDim.y) {
    const int64_t sr = rp ? (int64_t)rp[r] : r;
    T* dst = out + r * ldout;
    const bool rok = sr >= 0 && sr < rows;
    if (!rok && threadIdx.x == 0 && blockIdx.x == 0) record_status(QUIP_ERR_ARG);
    const T* src = in + (rok ? sr : 0) * ldin;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < cols;
         c += (int64_t)gridDim.x * blockDim.x) {
      const int64_t sc = cp ? (int64_t)cp[c] : c;
      const bool ok = rok && sc >= 0 && sc < cols;
      if (!ok && rok) record_status(QUIP_ERR_ARG);
      dst[c] = ok ? src[sc] : T(0);
    }
  }
}

// The same gather with the source row staged in shared memory: the row is
// read once with coalesced (16-byte when aligned) loads, the column gather
// reads shared memory, and the output row is written coalesced.  One row
// at a time per CTA, rows grid-stride; dynamic shared memory
// cols * sizeof(TIn) rounded up to 16 bytes.  TOut may differ from TIn
// (bf16 in, fp32 out); otherwise the bits are copied.
template <typename TOut, typename TIn>
__device__ __forceinline__ TOut gather_cvt(TIn v) { return (TOut)v; }
template <>
__device__ __forceinline__ float gather_cvt<float, __nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <typename TIn, typename TOut>
__global__ void __launch_bounds__(256) k_permute_staged(const TIn* __restrict__ in, int64_t ldin,
                                                        TOut* __restrict__ out, int64_t ldout,
                                                        int64_t rows, int64_t cols, int vec,
                                                        const int32_t* __restrict__ rp,
                                                        const int32_t* __restrict__ cp) {
  extern __shared__ __align__(16) uint8_t pst_raw[];
  TIn* row = reinterpret_cast<TIn*>(pst_raw);
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const int64_t sr = rp ? (int64_t)rp[r] : r;
    const bool rok = sr >= 0 && sr < rows;
    if (!rok && threadIdx.x == 0) record_status(QUIP_ERR_ARG);
    const TIn* src = in + (rok ? sr : 0) * ldin;
    if (rok) {
      if (vec) {
        const int64_t nv = cols * (int64_t)sizeof(TIn) / 16;
        for (int64_t v = threadIdx.x; v < nv; v += blockDim.x)
          reinterpret_cast<uint4*>(row)[v] = reinterpret_cast<const uint4*>(src)[v];
      } else {
        for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) row[c] = src[c];
      }
    }
    __syncthreads();
    TOut* dst = out + r * ldout;
    for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) {
      const int64_t sc = cp ? (int64_t)cp[c] : c;
      const bool ok = rok && sc >= 0 && sc < cols;
      if (!ok && rok) record_status(QUIP_ERR_ARG);
      dst[c] = ok ? gather_cvt<TOut>(row[sc]) : TOut(0);
    }
    __syncthreads();
  }
}
constexpr int64_t PERMUTE_STAGE_MAX = 96 * 1024;   // bytes of a staged row

// Greedy factors from the upper triangle of a symmetric H (h(j, k) =
// H[min(j,k)][max(j,k)]), n x n, n % 32 == 0:
//   UTf[j][k] = h(j, k) / h(j, j)   (fp32; its three bf16 pieces in UTs,
//                                    piece p at rows p n)
//   Ur[j][k]  = h(j, k) / h(k, k)   (fp32)
// UTf is U'^T (the block kernel's transposed factor and, in pieces, the B
// operand of the GEMMs: its row k scaled by 1 / H_kk gives (E H D^-1)_k);
// Ur is U' itself (the band next to the diagonal).  One 32 x 32 tile per
// CTA, read coalesced from H's upper triangle (transposed in shared memory
// below the diagonal).
__global__ void __launch_bounds__(256) k_greedy_factors(const float* __restrict__ H, int64_t ldh,
                                                        int64_t n, float* __restrict__ UTf,
                                                        __nv_bfloat16* __restrict__ UTs,
                                                        float* __restrict__ Ur) {
  __shared__ float t[32][33];
  __shared__ float dr[32], dc[32];
  const int64_t R = blockIdx.y, C = blockIdx.x;
  const int64_t sr0 = 32 * min(R, C), sc0 = 32 * max(R, C);   // source tile, upper triangle
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int a = ty; a < 32; a += 8) t[a][tx] = H[(sr0 + a) * ldh + sc0 + tx];
  if (threadIdx.x < 32) dr[tx] = H[(32 * R + tx) * ldh + 32 * R + tx];
  else if (threadIdx.x < 64) dc[tx] = H[(32 * C + tx) * ldh + 32 * C + tx];
  __syncthreads();
  const int64_t pst = n * n;
  for (int i = ty; i < 32; i += 8) {
    const int j = tx;
    // h(32 R + i, 32 C + j)
    const float h = R < C ? t[i][j] : R > C ? t[j][i] : (i <= j ? t[i][j] : t[j][i]);
    const int64_t e = (32 * R + i) * n + 32 * C + j;
    const float u = h / dr[i];
    UTf[e] = u;
    Ur[e] = h / dc[j];
    const __nv_bfloat16 p0 = __float2bfloat16_rn(u);
    const float r1 = u - __bfloat162float(p0);
    const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
    UTs[e] = p0;
    UTs[pst + e] = p1;
    UTs[2 * pst + e] = __float2bfloat16_rn(r1 - __bfloat162float(p1));
  }
}

// Start of a greedy pass: W^old = lo + s codes (What), the accumulator's
// start A = W^old (the GEMM then subtracts (E H) D^-1), and the three bf16
// pieces of E = W^old - W (Es, piece p at rows p m).  4-element groups;
// n % 4 == 0.  Rows i = blockIdx.y, + gridDim.y, ...
__global__ void __launch_bounds__(256) k_greedy_start(const uint8_t* __restrict__ codes,
                                                      const float* __restrict__ lo,
                                                      const float* __restrict__ sc,
                                                      const float* __restrict__ W, int64_t m,
                                                      int64_t n, float* __restrict__ What,
                                                      float* __restrict__ A,
                                                      __nv_bfloat16* __restrict__ Es) {
  const int64_t pst = m * n;
  for (int64_t i = blockIdx.y; i < m; i += gridDim.y) {
    const float l = lo[i], s = sc[i];
    for (int64_t j = 4 * ((int64_t)blockIdx.x * 256 + threadIdx.x); j < n;
         j += 4 * (int64_t)gridDim.x * 256) {
      const int64_t e = i * n + j;
      const uint32_t cw = *reinterpret_cast<const uint32_t*>(codes + e);
      const float4 w = *reinterpret_cast<const float4*>(W + e);
      const float4 h = make_float4(fmaf(s, (float)(cw & 0xffu), l), fmaf(s, (float)((cw >> 8) & 0xffu), l),
                                   fmaf(s, (float)((cw >> 16) & 0xffu), l), fmaf(s, (float)(cw >> 24), l));
      *reinterpret_cast<float4*>(What + e) = h;
      *reinterpret_cast<float4*>(A + e) = h;
      uint32_t a0, a1, a2, b0, b1, b2;
      split3x2(h.x - w.x, h.y - w.y, a0, a1, a2);
      split3x2(h.z - w.z, h.w - w.w, b0, b1, b2);
      *reinterpret_cast<uint2*>(Es + e) = make_uint2(a0, b0);
      *reinterpret_cast<uint2*>(Es + pst + e) = make_uint2(a1, b1);
      *reinterpret_cast<uint2*>(Es + 2 * pst + e) = make_uint2(a2, b2);
    }
  }
}

}  // namespace quip
