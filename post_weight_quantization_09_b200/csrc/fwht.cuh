// Randomized Hadamard transform (QuIP#, arXiv 2402.04396, abstract; QuIP,
// incoherence-processing section): y = H_d diag(s) x / sqrt(d) with the
// Sylvester H_d (H_1 = [1], H_2k = [[H_k, H_k], [H_k, -H_k]]).
//
// Two kernels, both HBM-bound (d log d add/sub per vector, one read and one
// write of every element):
//  * k_fwht_rows: transforms each contiguous row of a matrix.  A row of
//    d = 2^L values is held by d/16 threads, 16 values each: the low 4 index
//    bits are done in registers, the next 5 with warp shuffles, the rest
//    (L > 9) after one transposition through shared memory, again in
//    registers.  Loads and stores are 16-byte vectors / full 128-byte lines.
//  * k_fwht_cols: mixes groups of g = 2^G rows (16 <= g <= 256) at a row
//    stride, 32 columns per CTA; H_R = H_a (x) H_b lets a column transform of
//    length R = a*b run as two such passes (inner rows then strided rows).
//  * d = 4096 (rows) and R = 4096 (columns) have dedicated one-pass kernels,
//    k_fwht_row4096 and k_fwht_col4096 (radix 16 in registers, shared-memory
//    transpositions in between).
// Optional sign vectors: pre (applied to the input index), post (applied to
// the output index), and a per-row sign for the orthogonal direction.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace quip {

__device__ __forceinline__ void load16(const float* p, float (&v)[16]) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 f = q[i];
    v[4 * i] = f.x, v[4 * i + 1] = f.y, v[4 * i + 2] = f.z, v[4 * i + 3] = f.w;
  }
}
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float (&v)[16]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint4 u = q[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[8 * i + 2 * k] = __uint_as_float(w[k] << 16);
      v[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
}

// Butterflies over register index bits given by h = 1, 2, 4, ... < (1 << nbits).
template <int NB, int N>
__device__ __forceinline__ void reg_fwht(float (&v)[N]) {
#pragma unroll
  for (int h = 1; h < (1 << NB); h <<= 1) {
#pragma unroll
    for (int r = 0; r < N; ++r) {
      if ((r & h) == 0) {
        const float a = v[r], b = v[r + h];
        v[r] = a + b;
        v[r + h] = a - b;
      }
    }
  }
}

// Padded shared-memory index (one pad word per 32) for the row kernel.
__device__ __forceinline__ int pidx(int i) { return i + (i >> 5); }

// rows x d matrix, d = 2^LOGN, 16 <= d <= 8192.  CTA = max(256, d/16)
// threads; each group of d/16 threads owns one row.  In place allowed
// (in == out with equal strides).
template <int LOGN, typename TIn>
__global__ void __launch_bounds__((1 << LOGN) / 16 > 256 ? (1 << LOGN) / 16 : 256)
    k_fwht_rows(const TIn* in, int64_t ldin, float* out, int64_t ldout, int64_t rows,
                const float* __restrict__ pre, const float* __restrict__ post,
                const float* __restrict__ row_sign, float scale) {
  constexpr int D = 1 << LOGN;
  constexpr int T = D / 16;                           // threads per row
  constexpr int NT = T > 256 ? T : 256;               // threads per CTA
  constexpr int RPC = NT / T;                         // rows per CTA
  constexpr int LB = (LOGN - 4) < 5 ? (LOGN - 4) : 5; // lane-bit stages
  constexpr int W = LOGN > 9 ? LOGN - 9 : 0;          // stages after transpose
  extern __shared__ float smem[];
  const int t = threadIdx.x % T;
  const int rl = threadIdx.x / T;
  const int64_t row = (int64_t)blockIdx.x * RPC + rl;
  const bool active = row < rows;
  float v[16];
  if (active) {
    load16(in + row * ldin + 16 * t, v);
    if (pre) {
#pragma unroll
      for (int r = 0; r < 16; ++r) v[r] *= pre[16 * t + r];
    }
  } else {
#pragma unroll
    for (int r = 0; r < 16; ++r) v[r] = 0.f;
  }
  reg_fwht<4>(v);
#pragma unroll
  for (int b = 0; b < LB; ++b) {
    const int mask = 1 << b;
    const bool upper = (t & mask) != 0;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const float o = __shfl_xor_sync(0xffffffffu, v[r], mask);
      v[r] = upper ? (o - v[r]) : (v[r] + o);
    }
  }
  const float rs = (row_sign && active) ? row_sign[row] * scale : scale;
  if constexpr (W == 0) {
    if (active) {
      float* o = out + row * ldout + 16 * t;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float4 f;
        f.x = v[4 * q] * rs, f.y = v[4 * q + 1] * rs, f.z = v[4 * q + 2] * rs, f.w = v[4 * q + 3] * rs;
        if (post) {
          f.x *= post[16 * t + 4 * q], f.y *= post[16 * t + 4 * q + 1];
          f.z *= post[16 * t + 4 * q + 2], f.w *= post[16 * t + 4 * q + 3];
        }
        reinterpret_cast<float4*>(o)[q] = f;
      }
    }
  } else {
    // D >= 1024: RPC = NT / T rows per CTA, each with its own padded slice.
    float* sr = smem + rl * (D + D / 32);
#pragma unroll
    for (int r = 0; r < 16; ++r) sr[pidx(16 * t + r)] = v[r];
    __syncthreads();
    constexpr int NH = 1 << W;        // values of the high bits
    constexpr int NK = 16 / NH;       // low-part values per thread
#pragma unroll
    for (int k = 0; k < NK; ++k)
#pragma unroll
      for (int h = 0; h < NH; ++h) v[k * NH + h] = sr[pidx(t + k * T + (h << 9))];
    // butterflies over h (register bits 0..W-1 inside each k group)
#pragma unroll
    for (int hb = 1; hb < NH; hb <<= 1) {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        if ((e & hb) == 0) {
          const float a = v[e], b = v[e + hb];
          v[e] = a + b;
          v[e + hb] = a - b;
        }
      }
    }
    if (active) {
      float* o = out + row * ldout;
#pragma unroll
      for (int k = 0; k < NK; ++k)
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          const int idx = t + k * T + (h << 9);
          float x = v[k * NH + h] * rs;
          if (post) x *= post[idx];
          o[idx] = x;
        }
    }
  }
}

// d < 16: one thread per row, everything in registers.
template <typename TIn>
__global__ void k_fwht_rows_small(const TIn* in, int64_t ldin, float* out, int64_t ldout,
                                  int64_t rows, int d, const float* pre, const float* post,
                                  const float* row_sign, float scale) {
  const int64_t row = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (row >= rows) return;
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i)
    v[i] = (i < d) ? to_f32<TIn>(in[row * ldin + i]) * (pre ? pre[i] : 1.f) : 0.f;
  for (int h = 1; h < d; h <<= 1)
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (i < d && (i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
  const float rs = row_sign ? row_sign[row] * scale : scale;
  for (int i = 0; i < d; ++i) out[row * ldout + i] = v[i] * rs * (post ? post[i] : 1.f);
}

// Column pass: for every base row b0 (u in [0, R/g): b0 = (u / gs) * g * gs + u % gs)
// and every column c, transform the g values A[b0 + k*gs][c], k < g = 2^LOGG.
// pre / post are indexed by the global row; scale multiplies the output.
// CTA: 32 columns x (g/16) warps; thread (lane c, warp q) first holds
// k = q + (g/16) r (high 4 bits in registers), then k = 16 q + r.
template <int LOGG>
__global__ void __launch_bounds__(32 * ((1 << LOGG) / 16))
    k_fwht_cols(float* A, int64_t ld, int64_t ncols, int64_t gs, const float* __restrict__ pre,
                const float* __restrict__ post, float scale) {
  constexpr int G = 1 << LOGG;
  constexpr int NW = G / 16;
  constexpr int LOW = LOGG - 4;   // bits handled after the transposition
  __shared__ float s[G][32];
  const int c = threadIdx.x & 31, q = threadIdx.x >> 5;
  const int64_t col = (int64_t)blockIdx.x * 32 + c;
  const int64_t u = blockIdx.y;
  const int64_t b0 = (u / gs) * (int64_t)G * gs + (u % gs);
  const bool cok = col < ncols;
  float v[16];
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const int k = q + NW * r;
    const int64_t grow = b0 + (int64_t)k * gs;
    float x = cok ? A[grow * ld + col] : 0.f;
    if (pre) x *= pre[grow];
    v[r] = x;
  }
  reg_fwht<4>(v);     // high 4 bits of k
#pragma unroll
  for (int r = 0; r < 16; ++r) s[q + NW * r][c] = v[r];
  __syncthreads();
#pragma unroll
  for (int r = 0; r < 16; ++r) v[r] = s[16 * q + r][c];
  if constexpr (LOW > 0) reg_fwht<LOW>(v);
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const int k = 16 * q + r;
    const int64_t grow = b0 + (int64_t)k * gs;
    float x = v[r] * scale;
    if (post) x *= post[grow];
    if (cok) A[grow * ld + col] = x;
  }
}

// ---------------------------------------------------------------- 4096-point transforms
// Radix-16 in three register stages (index bits 0-3, 4-7, 8-11) with two
// transpositions through shared memory between them; the shared index of
// element k is k + k/16 (one pad word per 16), which makes every stage's
// accesses conflict-free.

__device__ __forceinline__ int pad16(int k) { return k + (k >> 4); }

// Row sources and sinks of the two one-row-per-CTA kernels below.  A source
// is fp32, bf16, or b-bit codes (uint8) dequantised on the way in as
// lo[row] + s[row] * code (the product and sum of the dequantisation kernel,
// one fused multiply-add).  The sink (row stride ld) is
//   ROW_F32     fp32 values y into out;
//   ROW_PIECES  the three bf16 pieces of every y (split3) into outp, piece
//               stride pst: the split the Kronecker kernel's inputs take;
//   ROW_GRID    y into out and out2 (W~ and the start of LDLQ's
//               accumulator), and the row's b-bit min / max grid lo[row] =
//               min y, sc[row] = (max y - min y) / qmax (1 for a constant
//               row), with QUIP_ERR_NONFINITE recorded for a non-finite y:
//               the values of the row-grid kernel, taken while the row is
//               still in registers.
struct RowDequant {
  const float* lo;
  const float* s;
};
enum { ROW_F32 = 0, ROW_PIECES = 1, ROW_GRID = 2 };
struct RowSink {
  float* out;
  float* out2;
  __nv_bfloat16* outp;
  int64_t ld, pst;
  float* lo;
  float* sc;
  float qmax;
};

// Row grid of ROW_GRID from each thread's min / max / finiteness (the whole
// CTA, NT threads, holds the row).  red: 3 * NT / 32 floats of shared memory.
template <int NT>
__device__ __forceinline__ void row_grid_store(float mn, float mx, bool fin, const RowSink& sk, int64_t row,
                                               float* red) {
  constexpr int NW = NT / 32;
  mn = warp_min(mn);
  mx = warp_max(mx);
  fin = __all_sync(0xffffffffu, fin);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();                                   // red may alias smem the transform used
  if (l == 0) red[w] = mn, red[NW + w] = mx, red[2 * NW + w] = fin ? 1.f : 0.f;
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = red[0], b = red[NW];
    bool f = red[2 * NW] != 0.f;
    for (int i = 1; i < NW; ++i) a = fminf(a, red[i]), b = fmaxf(b, red[NW + i]), f = f && red[2 * NW + i] != 0.f;
    if (!f) record_status(QUIP_ERR_NONFINITE);
    sk.lo[row] = a;
    sk.sc[row] = (b > a) ? (b - a) / sk.qmax : 1.0f;
  }
}

__device__ __forceinline__ void load16(const uint8_t* p, float (&v)[16]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int b = 0; b < 4; ++b) v[4 * k + b] = (float)((w[k] >> (8 * b)) & 0xffu);
}

template <typename TIn, int N>
__device__ __forceinline__ void dequant_in(const RowDequant& dq, int64_t row, float (&v)[N]) {
  if constexpr (std::is_same<TIn, uint8_t>::value) {
    const float l = dq.lo[row], sc = dq.s[row];
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = fmaf(sc, v[i], l);
  }
}

// One row of 4096 per CTA (256 threads).  Thread t: stage A on elements
// 16 t + j (16-byte loads), stage B on 256 (t / 16) + 16 j + t % 16, stage C
// on 256 j + t, stored straight from registers (coalesced across threads).
template <typename TIn, int SINK>
__global__ void __launch_bounds__(256)
    k_fwht_row4096(const TIn* __restrict__ in, int64_t ldin, RowDequant dq, RowSink sk,
                   const float* __restrict__ pre, const float* __restrict__ post,
                   const float* __restrict__ row_sign, float scale) {
  __shared__ float sr[4096 + 256];
  const int t = threadIdx.x;
  const int64_t row = blockIdx.x;
  float v[16];
  load16(in + row * ldin + 16 * t, v);
  dequant_in<TIn>(dq, row, v);
  if (pre) {
    const float4* pp = reinterpret_cast<const float4*>(pre + 16 * t);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f = pp[q];
      v[4 * q] *= f.x, v[4 * q + 1] *= f.y, v[4 * q + 2] *= f.z, v[4 * q + 3] *= f.w;
    }
  }
  reg_fwht<4>(v);
#pragma unroll
  for (int j = 0; j < 16; ++j) sr[pad16(16 * t + j)] = v[j];
  __syncthreads();
  const int hi = t >> 4, lo = t & 15;
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = sr[pad16(256 * hi + 16 * j + lo)];
  reg_fwht<4>(v);
#pragma unroll
  for (int j = 0; j < 16; ++j) sr[pad16(256 * hi + 16 * j + lo)] = v[j];
  __syncthreads();
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = sr[pad16(256 * j + t)];
  reg_fwht<4>(v);
  const float rs = row_sign ? row_sign[row] * scale : scale;
  float mn = INFINITY, mx = -INFINITY;
  bool fin = true;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int k = 256 * j + t;
    const float y = v[j] * rs * (post ? post[k] : 1.f);
    if constexpr (SINK == ROW_PIECES) {
      __nv_bfloat16* o = sk.outp + row * sk.ld + k;
      split3(y, o[0], o[sk.pst], o[2 * sk.pst]);
    } else {
      sk.out[row * sk.ld + k] = y;
    }
    if constexpr (SINK == ROW_GRID) {
      sk.out2[row * sk.ld + k] = y;
      mn = fminf(mn, y), mx = fmaxf(mx, y), fin = fin && isfinite(y);
    }
  }
  if constexpr (SINK == ROW_GRID) row_grid_store<256>(mn, mx, fin, sk, row, sr);
}

// ---------------------------------------------------------------- 8192-point rows
// Radix 32 x 16 x 16 ... as 32 x 32 x 8: index bits 0-4, 5-9 and 10-12 in
// registers, 32 values per thread, two transpositions through shared memory
// between them.  Shared index of element k: k + 4 (k / 32) (four pad words
// per 32), so a thread's 32 consecutive elements start 16-byte aligned (the
// first write is four-wide) and every other access of a warp covers 32
// consecutive elements: conflict-free throughout, and no shuffles.
__device__ __forceinline__ int pad32x4(int k) { return k + 4 * (k >> 5); }

__device__ __forceinline__ void load32(const float* p, float (&v)[32]) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 f = q[i];
    v[4 * i] = f.x, v[4 * i + 1] = f.y, v[4 * i + 2] = f.z, v[4 * i + 3] = f.w;
  }
}
__device__ __forceinline__ void load32(const __nv_bfloat16* p, float (&v)[32]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = q[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[8 * i + 2 * k] = __uint_as_float(w[k] << 16);
      v[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ void load32(const uint8_t* p, float (&v)[32]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint4 u = q[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int b = 0; b < 4; ++b) v[16 * i + 4 * k + b] = (float)((w[k] >> (8 * b)) & 0xffu);
  }
}

// One row of 8192 per CTA (256 threads).  Thread t (warp w, lane l): stage A
// on elements 32 t + r (r = bits 0-4); stage B on l + 32 r + 1024 w (bits
// 5-9); stage C on 4 t + j + 1024 r (j < 4, r < 8: bits 10-12), read from
// shared memory and stored four consecutive values at a time (16-byte
// accesses; a warp's store covers 512 contiguous bytes).
template <typename TIn, int SINK>
__global__ void __launch_bounds__(256, 4)
    k_fwht_row8192(const TIn* __restrict__ in, int64_t ldin, RowDequant dq, RowSink sk,
                   const float* __restrict__ pre, const float* __restrict__ post,
                   const float* __restrict__ row_sign, float scale) {
  __shared__ __align__(16) float sr[8192 + 1024];
  const int t = threadIdx.x, w = t >> 5, l = t & 31;
  const int64_t row = blockIdx.x;
  float v[32];
  load32(in + row * ldin + 32 * t, v);
  dequant_in<TIn>(dq, row, v);
  if (pre) {
    const float4* pp = reinterpret_cast<const float4*>(pre + 32 * t);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 f = pp[q];
      v[4 * q] *= f.x, v[4 * q + 1] *= f.y, v[4 * q + 2] *= f.z, v[4 * q + 3] *= f.w;
    }
  }
  reg_fwht<5>(v);
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<float4*>(sr + pad32x4(32 * t) + 4 * q) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  __syncthreads();
#pragma unroll
  for (int r = 0; r < 32; ++r) v[r] = sr[pad32x4(l + 32 * r + 1024 * w)];
  reg_fwht<5>(v);
#pragma unroll
  for (int r = 0; r < 32; ++r) sr[pad32x4(l + 32 * r + 1024 * w)] = v[r];
  __syncthreads();
  // stage C: register index 4 r + j holds element 4 t + j + 1024 r
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const float4 f = *reinterpret_cast<const float4*>(sr + pad32x4(4 * t + 1024 * r));
    v[4 * r] = f.x, v[4 * r + 1] = f.y, v[4 * r + 2] = f.z, v[4 * r + 3] = f.w;
  }
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if ((r & h) == 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float a = v[4 * r + j], b = v[4 * (r + h) + j];
          v[4 * r + j] = a + b;
          v[4 * (r + h) + j] = a - b;
        }
      }
    }
  }
  const float rs = row_sign ? row_sign[row] * scale : scale;
  float mn = INFINITY, mx = -INFINITY;
  bool fin = true;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int k = 4 * t + 1024 * r;
    float y[4];
    if (post) {
      const float4 f = *reinterpret_cast<const float4*>(post + k);
      y[0] = v[4 * r] * rs * f.x, y[1] = v[4 * r + 1] * rs * f.y;
      y[2] = v[4 * r + 2] * rs * f.z, y[3] = v[4 * r + 3] * rs * f.w;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) y[j] = v[4 * r + j] * rs;
    }
    if constexpr (SINK == ROW_PIECES) {
      __nv_bfloat16 pc[3][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) split3(y[j], pc[0][j], pc[1][j], pc[2][j]);
      __nv_bfloat16* o = sk.outp + row * sk.ld + k;
#pragma unroll
      for (int f = 0; f < 3; ++f) *reinterpret_cast<uint2*>(o + f * sk.pst) = *reinterpret_cast<const uint2*>(pc[f]);
    } else {
      *reinterpret_cast<float4*>(sk.out + row * sk.ld + k) = make_float4(y[0], y[1], y[2], y[3]);
    }
    if constexpr (SINK == ROW_GRID) {
      *reinterpret_cast<float4*>(sk.out2 + row * sk.ld + k) = make_float4(y[0], y[1], y[2], y[3]);
#pragma unroll
      for (int j = 0; j < 4; ++j) mn = fminf(mn, y[j]), mx = fmaxf(mx, y[j]), fin = fin && isfinite(y[j]);
    }
  }
  if constexpr (SINK == ROW_GRID) row_grid_store<256>(mn, mx, fin, sk, row, sr);
}

// 4096-point column transform of 8 columns per CTA (1024 threads), in place.
// Thread unit u (two per thread) handles column c = u % 8: stage A on rows
// 16 o + j (o = u / 8; loaded straight from global memory), stage B on rows
// 256 (u / 128) + 16 j + (u / 8) % 16, stage C on rows 256 j + u / 8 (stored
// straight to global memory).  Shared index of (row k, column c):
// pad16(k) 8 + c, conflict-free.  pre / post are indexed by the row; scale
// multiplies the output.  Dynamic smem: (4096 + 256) x 8 floats.
constexpr int FWHT_C4K_NC = 8, FWHT_C4K_THREADS = 1024;
__global__ void __launch_bounds__(FWHT_C4K_THREADS, 1)
    k_fwht_col4096(float* A, int64_t ld, int64_t ncols, const float* __restrict__ pre,
                   const float* __restrict__ post, float scale) {
  constexpr int NC = FWHT_C4K_NC, NTH = FWHT_C4K_THREADS;
  extern __shared__ float sc[];
  const int tid = threadIdx.x;
  const int64_t c0 = (int64_t)blockIdx.x * NC;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int u = tid + NTH * h, c = u % NC, o = u / NC;
    const bool cok = c0 + c < ncols;
    float v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int k = 16 * o + j;
      float x = cok ? A[k * ld + c0 + c] : 0.f;
      if (pre) x *= pre[k];
      v[j] = x;
    }
    reg_fwht<4>(v);
#pragma unroll
    for (int j = 0; j < 16; ++j) sc[pad16(16 * o + j) * NC + c] = v[j];
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int u = tid + NTH * h, c = u % NC, lo = (u / NC) & 15, hi = u / (16 * NC);
    float v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = sc[pad16(256 * hi + 16 * j + lo) * NC + c];
    reg_fwht<4>(v);
#pragma unroll
    for (int j = 0; j < 16; ++j) sc[pad16(256 * hi + 16 * j + lo) * NC + c] = v[j];
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int u = tid + NTH * h, c = u % NC, low = u / NC;
    const bool cok = c0 + c < ncols;
    float v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = sc[pad16(256 * j + low) * NC + c];
    reg_fwht<4>(v);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int k = 256 * j + low;
      float x = v[j] * scale;
      if (post) x *= post[k];
      if (cok) A[k * ld + c0 + c] = x;
    }
  }
}

// R < 16 rows: one thread per column.
__global__ void k_fwht_cols_small(float* A, int64_t ld, int64_t ncols, int R,
                                  const float* pre, const float* post, float scale) {
  const int64_t col = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (col >= ncols) return;
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = (i < R) ? A[i * ld + col] * (pre ? pre[i] : 1.f) : 0.f;
  for (int h = 1; h < R; h <<= 1)
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (i < R && (i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
  for (int i = 0; i < R; ++i) A[i * ld + col] = v[i] * scale * (post ? post[i] : 1.f);
}

}  // namespace quip
