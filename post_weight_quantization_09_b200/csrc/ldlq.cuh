// LDLQ adaptive rounding (QuIP, adaptive-rounding section: LDLQ rounds
// column k of the incoherent weights after adding the linear feedback
// (W - W^) Ů_k of the columns already rounded; "Methods.": LDLQ = OPTQ),
// on a per-row b-bit min/max grid.
//
// Blocked over 128 columns: inside a block every column's error is fed back
// to the block's later columns (k_ldlq_tc); across blocks the
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

// Block step over the w columns [k0, k0 + w) (w = 128, or 64 for a last,
// partial block) for 128 rows per CTA.  Row warps 0-3 (thread = row = TMEM
// lane; column j of the block = TMEM column j, holding the row's accumulated
// value) and helper warps 4-7 (helper thread h serves row h).  Columns are
// taken in groups of 16; for group g the row thread
//   1. waits for the MMAs of group g - 2, loads the group's 16 values from
//      TMEM (tcgen05.ld) and adds the previous group's feedback `carry`;
//   2. rounds column by column, feeding each error to the group's later
//      columns (fp32 fma; Ů from a shared fp32 band);
//   3. forms, along the way, the group's feedback to the next group
//      (`carry`, fp32) and hands the 16 errors and codes to its helper
//      through shared memory.
// The helper writes the errors' three bf16 pieces into a shared A operand
// (128-byte swizzled, K-major) and then the codes and pieces to global
// memory; once all 128 rows are there, warp 8 issues the group's feedback
// to every column from two groups on as six tcgen05.mma kind::f16
// (M = 128, N = w - 16 (g + 2), K = 16; the three-piece product terms of
// order <= 2, as in the split GEMM) accumulating in TMEM.  The B operand is
// the block of the split transposed factor (Ů^T pieces), loaded once by TMA.
// Named barriers pass the two double-buffered hand-off slots between the
// warp groups; MMA completion is signalled on two alternating mbarriers.
// Every mbarrier wait is bounded; on a timeout the CTA records
// QUIP_ERR_TIMEOUT and stops issuing MMAs.
constexpr int LQT_TILE = 128 * 64 * 2;                 // one SW128 operand tile, bytes
constexpr int LQT_B_OFF = 0;                           // 2 K-halves x 3 pieces (Ů^T)
constexpr int LQT_A_OFF = 6 * LQT_TILE;                // 3 pieces (errors)
constexpr int LQT_BAND_OFF = 9 * LQT_TILE;             // 128 x 32 fp32
constexpr int LQT_E_OFF = LQT_BAND_OFF + 128 * 32 * 4; // 2 slots x 128 rows x (16 fp32 + 16 codes)
constexpr int LQT_E_ROW = 16 * 4 + 16;
constexpr int LQT_BAR_OFF = LQT_E_OFF + 2 * 128 * LQT_E_ROW;
constexpr int LQT_SMEM = LQT_BAR_OFF + 64 + 1024;      // + room to align the base to 1 KB

struct LqtShared {
  uint64_t tma_bar;
  uint64_t mma_bar[2];
  uint32_t tmem_base;
  int fail;
};

// Named barriers (id 0 is __syncthreads): FULL + slot (rows -> helpers),
// EMPTY + slot (helpers -> rows), AREADY + slot (helpers -> MMA warp).
constexpr int LQT_FULL = 1, LQT_EMPTY = 3, LQT_AREADY = 5;
constexpr int LQT_THREADS = 288;                       // 4 row, 4 helper, 1 MMA warp

// Three bf16 pieces of two values at once (the same pieces as split3 on each):
// returns the packed bf16 pairs (low half = a) of piece 0, 1, 2.
__device__ __forceinline__ void split3x2(float a, float b, uint32_t& q0, uint32_t& q1,
                                         uint32_t& q2) {
  const __nv_bfloat162 p0 = __floats2bfloat162_rn(a, b);
  const float2 f0 = __bfloat1622float2(p0);
  const float a1 = a - f0.x, b1 = b - f0.y;
  const __nv_bfloat162 p1 = __floats2bfloat162_rn(a1, b1);
  const float2 f1 = __bfloat1622float2(p1);
  const __nv_bfloat162 p2 = __floats2bfloat162_rn(a1 - f1.x, b1 - f1.y);
  q0 = *reinterpret_cast<const uint32_t*>(&p0);
  q1 = *reinterpret_cast<const uint32_t*>(&p1);
  q2 = *reinterpret_cast<const uint32_t*>(&p2);
}
__device__ __forceinline__ void nb_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void nb_arrive(int id, int count) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__global__ void __launch_bounds__(LQT_THREADS, 1)
    k_ldlq_tc(const __grid_constant__ CUtensorMap tmU, const float* __restrict__ Wt,
              const float* __restrict__ A, int64_t m, int64_t n, int64_t k0, int w,
              const float* __restrict__ U, int64_t ldu, const float* __restrict__ lo,
              const float* __restrict__ sc, float qmax, uint8_t* __restrict__ codes,
              __nv_bfloat16* __restrict__ Es, int64_t lde) {
  extern __shared__ uint8_t smem_raw[];
  pdl_wait_then_release();
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  LqtShared* sh = reinterpret_cast<LqtShared*>(smem + LQT_BAR_OFF);
  float* band = reinterpret_cast<float*>(smem + LQT_BAND_OFF);
  const int tid = threadIdx.x, warp = tid >> 5;
  const bool helper = warp >= 4 && warp < 8;
  const bool mma_warp = warp == 8;
  const int r = tid & 127;                              // row within the CTA
  const int64_t row = (int64_t)blockIdx.x * 128 + r;
  const bool valid = row < m;
  const int nh = (w + 63) / 64;                         // K halves of the Ů^T block
  const int ngroups = w / 16;

  if (tid == 0) {
    mbar_init(&sh->tma_bar, 1);
    mbar_init(&sh->mma_bar[0], 1);
    mbar_init(&sh->mma_bar[1], 1);
    sh->fail = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&sh->tmem_base, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const uint32_t lanes = (uint32_t)((warp & 3) * 32) << 16;
  if (tid == 256) {
    // Ů^T pieces: map rows p n + j (j in [k0, k0 + 128)), columns k in [k0 + 64 h, + 64)
    tma_prefetch_desc(&tmU);
    mbar_arrive_expect_tx(&sh->tma_bar, (uint32_t)(3 * nh * LQT_TILE));
    for (int h = 0; h < nh; ++h)
      for (int p = 0; p < 3; ++p)
        tma_load_2d(smem + LQT_B_OFF + (h * 3 + p) * LQT_TILE, &tmU, &sh->tma_bar,
                    (int)(k0 + 64 * h), (int)(p * n + k0));
  }
  if (helper) {
    // fp32 band of Ů: row k, columns [16 (k / 16), + 32) (the own and the next group)
    const int h = tid - 128;
#pragma unroll 32
    for (int e = h; e < 128 * 32; e += 128) {
      const int k = e >> 5, jj = e & 31, j = 16 * (k >> 4) + jj;
      band[e] = (k < w && j < w && j > k) ? U[(k0 + k) * ldu + k0 + j] : 0.f;
    }
  } else if (!mma_warp) {
    // the row's accumulated values into TMEM columns [0, w)
    for (int c64 = 0; c64 < w / 64; ++c64) {
      float v[2][32];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
        if (valid) f = *reinterpret_cast<const float4*>(A + row * n + k0 + 64 * c64 + 4 * q);
        v[q >> 3][4 * (q & 7)] = f.x, v[q >> 3][4 * (q & 7) + 1] = f.y;
        v[q >> 3][4 * (q & 7) + 2] = f.z, v[q >> 3][4 * (q & 7) + 3] = f.w;
      }
      tmem_st32(tmem + lanes + 64 * c64, v[0]);
      tmem_st32(tmem + lanes + 64 * c64 + 32, v[1]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (!helper && !mma_warp) {
    // ------------------------------------------------------------ row warps
    const float l = valid ? lo[row] : 0.f;
    const float s = valid ? sc[row] : 1.f;
    const float inv = 1.0f / s;
    float carry[16], wv[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) carry[t] = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
      if (valid) f = *reinterpret_cast<const float4*>(Wt + row * n + k0 + 4 * q);
      wv[4 * q] = f.x, wv[4 * q + 1] = f.y, wv[4 * q + 2] = f.z, wv[4 * q + 3] = f.w;
    }
#pragma unroll 1
    for (int g = 0; g < ngroups; ++g) {
      const int slot = g & 1;
      // columns of this group have every MMA update once group g - 2's are
      // done (groups < ngroups - 2 issue MMAs, so g - 2 did)
      if (g >= 2) {
        if (!mbar_wait(&sh->mma_bar[slot], (uint32_t)(((g - 2) >> 1) & 1))) sh->fail = 1;
        tc_fence_after();
      }
      float cur[16];
      tmem_ld16(tmem + lanes + 16 * g, cur);
#pragma unroll
      for (int t = 0; t < 16; ++t) cur[t] += carry[t];
      float wn[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
        if (valid && g + 1 < ngroups)
          f = *reinterpret_cast<const float4*>(Wt + row * n + k0 + 16 * (g + 1) + 4 * q);
        wn[4 * q] = f.x, wn[4 * q + 1] = f.y, wn[4 * q + 2] = f.z, wn[4 * q + 3] = f.w;
      }
      float e[16];
      uint32_t cw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int j = 0; j < 16; ++j) carry[j] = 0.f;
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const float z = (cur[t] - l) * inv;
        const float cq = fminf(fmaxf(rintf(z), 0.f), qmax);
        const float err = wv[t] - fmaf(s, cq, l);
        e[t] = err;
        cw[t >> 2] |= (uint32_t)cq << (8 * (t & 3));
        // band row 16 g + t: this group's later columns, then the next group's
        const float* ur = band + (16 * g + t) * 32;
#pragma unroll
        for (int q4 = ((t + 1) >> 2) << 2; q4 < 16; q4 += 4) {
          const float4 u = *reinterpret_cast<const float4*>(ur + q4);
          if (q4 + 0 > t) cur[q4 + 0] = fmaf(err, u.x, cur[q4 + 0]);
          if (q4 + 1 > t) cur[q4 + 1] = fmaf(err, u.y, cur[q4 + 1]);
          if (q4 + 2 > t) cur[q4 + 2] = fmaf(err, u.z, cur[q4 + 2]);
          if (q4 + 3 > t) cur[q4 + 3] = fmaf(err, u.w, cur[q4 + 3]);
        }
#pragma unroll
        for (int q4 = 0; q4 < 16; q4 += 4) {
          const float4 u = *reinterpret_cast<const float4*>(ur + 16 + q4);
          carry[q4 + 0] = fmaf(err, u.x, carry[q4 + 0]);
          carry[q4 + 1] = fmaf(err, u.y, carry[q4 + 1]);
          carry[q4 + 2] = fmaf(err, u.z, carry[q4 + 2]);
          carry[q4 + 3] = fmaf(err, u.w, carry[q4 + 3]);
        }
      }
      // hand the errors and codes to the helper (slot free once it read group g - 2)
      if (g >= 2) nb_sync(LQT_EMPTY + slot, 256);
      uint8_t* er = smem + LQT_E_OFF + (slot * 128 + r) * LQT_E_ROW;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        reinterpret_cast<float4*>(er)[q] = make_float4(e[4 * q], e[4 * q + 1], e[4 * q + 2], e[4 * q + 3]);
      *reinterpret_cast<uint4*>(er + 64) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      nb_arrive(LQT_FULL + slot, 256);
#pragma unroll
      for (int t = 0; t < 16; ++t) wv[t] = wn[t];
    }
  } else if (helper) {
    // ------------------------------------------------------------ helper warps
    const int64_t pst = m * lde;
#pragma unroll 1
    for (int g = 0; g < ngroups; ++g) {
      const int slot = g & 1;
      nb_sync(LQT_FULL + slot, 256);
      const uint8_t* er = smem + LQT_E_OFF + (slot * 128 + r) * LQT_E_ROW;
      float e[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 f = reinterpret_cast<const float4*>(er)[q];
        e[4 * q] = f.x, e[4 * q + 1] = f.y, e[4 * q + 2] = f.z, e[4 * q + 3] = f.w;
      }
      const uint4 cw = *reinterpret_cast<const uint4*>(er + 64);
      if (g + 2 < ngroups) nb_arrive(LQT_EMPTY + slot, 256);
      uint32_t pk[3][8];
#pragma unroll
      for (int t = 0; t < 16; t += 2)
        split3x2(e[t], e[t + 1], pk[0][t >> 1], pk[1][t >> 1], pk[2][t >> 1]);
      const int nN = w - 16 * (g + 2);
      if (nN > 0) {
        // K-slice sl = g % 4 of the A operand: 16-byte chunks 2 sl, 2 sl + 1
        // of row r, at the 128-byte swizzle position chunk ^ (r % 8).  Group
        // g - 4 used this slice; its MMAs finished before group g - 2's,
        // which the row warps waited for before handing over group g.
        const int sl = g & 3;
        uint8_t* rowp = smem + LQT_A_OFF + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int p = 0; p < 3; ++p) {
          uint8_t* tile = rowp + p * LQT_TILE;
          *reinterpret_cast<uint4*>(tile + (((2 * sl) ^ (r & 7)) << 4)) =
              make_uint4(pk[p][0], pk[p][1], pk[p][2], pk[p][3]);
          *reinterpret_cast<uint4*>(tile + (((2 * sl + 1) ^ (r & 7)) << 4)) =
              make_uint4(pk[p][4], pk[p][5], pk[p][6], pk[p][7]);
        }
        fence_proxy_async_smem();
        nb_arrive(LQT_AREADY + slot, 160);
      }
      if (valid) {
        *reinterpret_cast<uint4*>(codes + row * n + k0 + 16 * g) = cw;
#pragma unroll
        for (int p = 0; p < 3; ++p) {
          uint4* dst = reinterpret_cast<uint4*>(Es + p * pst + row * lde + k0 + 16 * g);
          dst[0] = make_uint4(pk[p][0], pk[p][1], pk[p][2], pk[p][3]);
          dst[1] = make_uint4(pk[p][4], pk[p][5], pk[p][6], pk[p][7]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ MMA warp
    bool tma_done = false;
    // descriptor bases; a K-slice and a row offset add (bytes >> 4) to the
    // start-address field (all shared addresses here are below 256 KB)
    uint64_t adesc0[3], bdesc0[2][3];
#pragma unroll
    for (int p = 0; p < 3; ++p) {
      adesc0[p] = make_sw128_desc(smem_u32(smem + LQT_A_OFF + p * LQT_TILE), 16, 1024);
      bdesc0[0][p] = make_sw128_desc(smem_u32(smem + LQT_B_OFF + p * LQT_TILE), 16, 1024);
      bdesc0[1][p] = make_sw128_desc(smem_u32(smem + LQT_B_OFF + (3 + p) * LQT_TILE), 16, 1024);
    }
#pragma unroll 1
    for (int g = 0; g + 2 < ngroups; ++g) {
      const int slot = g & 1, sl = g & 3, nN = w - 16 * (g + 2);
      nb_sync(LQT_AREADY + slot, 160);
      if ((tid & 31) == 0) {
        if (!tma_done && !sh->fail) {
          if (!mbar_wait(&sh->tma_bar, 0)) sh->fail = 1;
          tma_done = true;
        }
        if (!sh->fail) {
          tc_fence_after();
          const uint32_t idesc = make_idesc_bf16(128, nN, 0, 0);
          const int h = g >> 2;
          const uint64_t aoff = (uint64_t)((sl * 32) >> 4);
          const uint64_t boff = (uint64_t)((sl * 32 + 16 * (g + 2) * 128) >> 4);
          const uint32_t dcol = tmem + 16 * (g + 2);
          const uint64_t b0 = (h ? bdesc0[1][0] : bdesc0[0][0]) + boff;
          const uint64_t b1 = (h ? bdesc0[1][1] : bdesc0[0][1]) + boff;
          const uint64_t b2 = (h ? bdesc0[1][2] : bdesc0[0][2]) + boff;
          // (2,0) (1,1) (0,2) (1,0) (0,1) (0,0): smallest terms first
          tc_mma_f16(dcol, adesc0[2] + aoff, b0, idesc, 1u);
          tc_mma_f16(dcol, adesc0[1] + aoff, b1, idesc, 1u);
          tc_mma_f16(dcol, adesc0[0] + aoff, b2, idesc, 1u);
          tc_mma_f16(dcol, adesc0[1] + aoff, b0, idesc, 1u);
          tc_mma_f16(dcol, adesc0[0] + aoff, b1, idesc, 1u);
          tc_mma_f16(dcol, adesc0[0] + aoff, b0, idesc, 1u);
        }
        // always signal, so the row warps' bounded waits see the phase
        tc_commit(&sh->mma_bar[slot]);
      }
      __syncwarp();
    }
    // every MMA done before TMEM is freed: the last group that issued any
    const int last = ngroups - 3;
    if ((tid & 31) == 0 && last >= 0) {
      if (!mbar_wait(&sh->mma_bar[last & 1], (uint32_t)((last >> 1) & 1))) sh->fail = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && sh->fail) record_status(QUIP_ERR_TIMEOUT);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
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
