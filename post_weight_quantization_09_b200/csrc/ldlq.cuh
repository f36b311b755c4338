// LDLQ adaptive rounding (QuIP, adaptive-rounding section: LDLQ rounds
// column k of the incoherent weights after adding the linear feedback
// (W - W^) Ů_k of the columns already rounded; "Methods.": LDLQ = OPTQ),
// on a per-row b-bit min/max grid.
//
// Blocked over 128 columns: inside a block every column's error is fed back
// to the block's later columns (k_ldlq_block); across blocks the
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
#pragma unroll 8
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

// Block step over the w columns [k0, k0 + w) (w = 128, or 64 for a last,
// partial block) for 32 rows per sub-group, on the FP32 pipes: one warp
// rounds (lane r = row r), the other three apply the feedback that can wait.  Global
// memory is touched only by the copies in and the stores out: TMA brings
// the rows' W~ and accumulated values of the block (wt, acc; row r at stride LQB_S:
// 16-byte accesses of a warp are conflict-free), the transposed Ů block
// (UT[j][k] = Ů[k0 + k][k0 + j], zero for k >= j) and the band of Ů next to
// the diagonal (band[k][jj] = Ů[k0 + k][k0 + 16 (k / 16) + jj], as eight
// 16 x 32 boxes; entries with j <= k or j >= w are zeroed after the copy).
// Columns are taken in groups of 16.  For group g, the rounding warp
//   1. waits until the helpers have applied group g - 2's feedback, then
//      takes cur = the group's accumulated values + carry (the previous
//      group's feedback, in registers);
//   2. rounds column by column, feeding each error to the group's later
//      columns and into the group's feedback to the next group (carry);
//   3. hands the 16 errors and codes to the helpers (shared slot g % 2).
// The helpers write the codes and the errors' three bf16 pieces (the
// trailing GEMMs' A operand) of each group to global memory as the group is
// handed over (helper 0, lane r: row r; 16-byte stores spread over the
// block instead of one burst at its end) and add group g's feedback to the columns from
// two groups on, acc[r][j] += sum_t e_t Ů[16 g + t][j] (each thread: four
// rows and every twelfth 4-column chunk, so one broadcast 16-byte load of a
// UT row serves 16 fmas; the chunks' accumulated values stay in registers and
// are stored to the shared tile once, after their last feedback, two groups
// before the rounding warp reads them), while the rounding warp takes group
// g + 1.  Named
// barriers pass the hand-off slots: READY + slot (rounding warp -> helpers,
// every group) and DONE + slot (helpers -> rounding warp, only for groups
// it will wait on).
// Rounding: clamp to [0, qmax] first, then add and subtract 1.5 * 2^23,
// which rounds half to even exactly like rintf on that range (and leaves
// the integer, the code, in the low mantissa bits).
// Maps: tmA over the accumulator and tmW over W~ (m x n fp32, LQB_S x 32 boxes), tmUT over
// the transposed factor (n x n fp32, LQB_S x 128 boxes), tmU over the
// factor Ů (the LDL's output, row stride ldu; 32 x 16 boxes).
constexpr int LQB_ROWS = 32;                           // rows per sub-group
constexpr int LQB_THREADS = 128;                       // per sub-group: one warp rounds, three help
constexpr int LQB_S = 132;                             // smem row stride of acc and UT
constexpr int LQB_ES = 20;                             // smem row stride of the slots: 16 errors, 4 code words
constexpr int LQB_ACC = LQB_ROWS * LQB_S * 4;          // bytes of the acc tile
constexpr int LQB_UT = 128 * LQB_S * 4;                // bytes of the UT tile
constexpr int LQB_BAND = 128 * 32 * 4;                 // bytes of the band
constexpr int LQB_E = 2 * LQB_ROWS * LQB_ES * 4;       // bytes of the two error slots (+ codes)
// Shared memory of a CTA of SUB sub-groups: per sub-group acc, wt and the
// slots; UT and the band once.
__host__ __device__ constexpr int lqb_smem(int sub) {
  return 128 + LQB_UT + LQB_BAND + sub * (2 * LQB_ACC + LQB_E);
}
constexpr int LQB_SMEM = lqb_smem(1);
constexpr int LQB_READY = 1, LQB_DONE = 3;             // named barrier ids (+ slot, + 4 x sub-group)

// SUB sub-groups of 32 rows per CTA (SUB x 128 threads): each sub-group is
// the 32-row unit described above, with its own rounding warp, helpers,
// slots and named barriers; the sub-groups share the UT and band tiles.
template <int SUB>
__global__ void __launch_bounds__(SUB * LQB_THREADS, 1)
    k_ldlq_block(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmUT,
                 const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmW,
                 int64_t m, int64_t n, int64_t k0, int w, const float* __restrict__ lo,
                 const float* __restrict__ sc, float qmax, uint8_t* __restrict__ codes,
                 __nv_bfloat16* __restrict__ Es, int64_t lde) {
  constexpr int CROWS = SUB * LQB_ROWS;                // rows per CTA
  constexpr int CTHREADS = SUB * LQB_THREADS;
  extern __shared__ __align__(16) uint8_t lqb_raw[];
  float* UT = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(lqb_raw) + 127) & ~uintptr_t(127));
  float* band = UT + 128 * LQB_S;
  float* acc0 = band + 128 * 32;                       // [CROWS][LQB_S]: accumulated values
  float* wt0 = acc0 + CROWS * LQB_S;                   // [CROWS][LQB_S]: the rows' W~ of the block
  float* eslot0 = wt0 + CROWS * LQB_S;                 // [SUB][2][32][LQB_ES]
  __shared__ __align__(8) uint64_t bar;
  __shared__ int ok_s;
  const int tid = threadIdx.x, sg = tid / LQB_THREADS, warp = (tid % LQB_THREADS) >> 5, r = tid & 31;
  // the rounding warp of sub-group sg is its warp sg % 4: CTA warp 4 sg + sg,
  // so the rounding warps sit on different SM sub-partitions (warp % 4) and
  // do not share an issue slot
  const int rw = sg & 3;
  const int srow = sg * LQB_ROWS + r;                  // this thread's row within the CTA
  const int64_t row = (int64_t)blockIdx.x * CROWS + srow;
  const bool valid = row < m;
  float* acc = acc0 + sg * LQB_ROWS * LQB_S;           // this sub-group's tiles
  float* wt = wt0 + sg * LQB_ROWS * LQB_S;
  float* eslot = eslot0 + sg * 2 * LQB_ROWS * LQB_ES;
  const int bar_ready = LQB_READY + 4 * sg, bar_done = LQB_DONE + 4 * sg;
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // W~, the transposed factor and the band come from kernels that finished
  // before the one just ahead of this launch (a programmatic dependent launch
  // starts only once its predecessor has passed its own wait): their copies
  // start before the wait; the accumulated values, which that predecessor
  // (a trailing GEMM) writes, after it
  if (tid == 0) {
    mbar_arrive_expect_tx(&bar, (uint32_t)(SUB * 2 * LQB_ACC + LQB_UT + LQB_BAND));
    for (int u = 0; u < SUB; ++u)
      tma_load_2d(wt0 + u * LQB_ROWS * LQB_S, &tmW, &bar, (int)k0, (int)(blockIdx.x * CROWS + u * LQB_ROWS));
    tma_load_2d(UT, &tmUT, &bar, (int)k0, (int)k0);
    for (int i = 0; i < 8; ++i)
      tma_load_2d(band + 16 * 32 * i, &tmU, &bar, (int)(k0 + 16 * i), (int)(k0 + 16 * i));
  }
  pdl_wait_then_release();
  if (tid == 0) {
    for (int u = 0; u < SUB; ++u)
      tma_load_2d(acc0 + u * LQB_ROWS * LQB_S, &tmA, &bar, (int)k0, (int)(blockIdx.x * CROWS + u * LQB_ROWS));
    const bool ok = mbar_wait(&bar, 0);
    if (!ok) mbar_wait(&bar, 0);                       // copies in flight: bounded again
    ok_s = ok ? 1 : 0;
  }
  __syncthreads();
  if (!ok_s) return;
  // band: keep Ů[k][j] for k < j < w only
#pragma unroll 4
  for (int e = tid; e < 128 * 32; e += CTHREADS) {
    const int k = e >> 5, j = 16 * (k >> 4) + (e & 31);
    if (j <= k || j >= w) band[e] = 0.f;
  }
  __syncthreads();
  const int ngroups = w / 16;

  if (warp != rw) {
    // ------------------------------------------------------------ helpers
    // thread (h, lane): rows lane % 8 + 8 i (i < 4) and the 4-column chunks
    // c with c % 12 == 4 h + lane / 8 (every Ů^T load serves four rows);
    // helper warp 0 also stores row `lane`'s codes and error pieces.
    const int h = warp < rw ? warp : warp - 1, rb = r & 7, cls = 4 * h + (r >> 3);
    // this thread's chunks that take feedback (c >= 8, c < w / 4): at most two,
    // cls + 12 k; their accumulated values stay in registers for the block
    int cc[2];
    bool has[2];
    cc[0] = cls >= 8 ? cls : cls + 12;
    cc[1] = cc[0] + 12;
    float a[2][4][4];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      has[k] = 4 * cc[k] < w;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float4 a4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (has[k]) a4 = *reinterpret_cast<const float4*>(acc + (rb + 8 * i) * LQB_S + 4 * cc[k]);
        a[k][i][0] = a4.x, a[k][i][1] = a4.y, a[k][i][2] = a4.z, a[k][i][3] = a4.w;
      }
    }
#pragma unroll 1
    for (int g = 0; g < ngroups; ++g) {
      const int slot = g & 1;
      nb_sync(bar_ready + slot, LQB_THREADS);
      const float* eb = eslot + slot * LQB_ROWS * LQB_ES;
      if (h == 0) {
        // row r's codes and error pieces of the group straight to global
        // memory: 16-byte stores spread over the block's groups
        const float* es = eb + r * LQB_ES;
        float e[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 v = *reinterpret_cast<const float4*>(es + 4 * q);
          e[4 * q] = v.x, e[4 * q + 1] = v.y, e[4 * q + 2] = v.z, e[4 * q + 3] = v.w;
        }
        uint32_t pk[3][8];
#pragma unroll
        for (int t = 0; t < 16; t += 2)
          split3x2(e[t], e[t + 1], pk[0][t >> 1], pk[1][t >> 1], pk[2][t >> 1]);
        if (valid) {
          *reinterpret_cast<uint4*>(codes + row * n + k0 + 16 * g) = *reinterpret_cast<const uint4*>(es + 16);
          const int64_t pst = m * lde;
#pragma unroll
          for (int p = 0; p < 3; ++p) {
            uint4* dst = reinterpret_cast<uint4*>(Es + p * pst + row * lde + k0 + 16 * g);
            dst[0] = make_uint4(pk[p][0], pk[p][1], pk[p][2], pk[p][3]);
            dst[1] = make_uint4(pk[p][4], pk[p][5], pk[p][6], pk[p][7]);
          }
        }
      }
      // group g's feedback into this thread's chunks from two groups on
      const int c0 = 4 * (g + 2);
      if ((has[0] && cc[0] >= c0) || (has[1] && cc[1] >= c0)) {
        float e[4][16];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 v = *reinterpret_cast<const float4*>(eb + (rb + 8 * i) * LQB_ES + 4 * q);
            e[i][4 * q] = v.x, e[i][4 * q + 1] = v.y, e[i][4 * q + 2] = v.z, e[i][4 * q + 3] = v.w;
          }
        const float* ug = UT + 16 * g;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          if (!has[k] || cc[k] < c0) continue;
          const int j = 4 * cc[k];
#pragma unroll
          for (int t4 = 0; t4 < 16; t4 += 4) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 u = *reinterpret_cast<const float4*>(ug + (j + q) * LQB_S + t4);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                a[k][i][q] = fmaf(e[i][t4 + 0], u.x, a[k][i][q]);
                a[k][i][q] = fmaf(e[i][t4 + 1], u.y, a[k][i][q]);
                a[k][i][q] = fmaf(e[i][t4 + 2], u.z, a[k][i][q]);
                a[k][i][q] = fmaf(e[i][t4 + 3], u.w, a[k][i][q]);
              }
            }
          }
        }
      }
      // chunks the rounding warp takes two groups on have all their feedback:
      // back to the shared tile (the only shared-memory traffic of acc)
#pragma unroll
      for (int k = 0; k < 2; ++k)
        if (has[k] && (cc[k] >> 2) == g + 2)
#pragma unroll
          for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4*>(acc + (rb + 8 * i) * LQB_S + 4 * cc[k]) =
                make_float4(a[k][i][0], a[k][i][1], a[k][i][2], a[k][i][3]);
      if (g + 2 < ngroups) nb_arrive(bar_done + slot, LQB_THREADS);
    }
  } else {

  // ------------------------------------------------------------ the rounding warp
  const float l = valid ? lo[row] : 0.f;
  const float s = valid ? sc[row] : 1.f;
  const float inv = 1.0f / s;
  constexpr float kRound = 12582912.0f;                // 1.5 * 2^23
  const float* myacc = acc + r * LQB_S;
  const float* mywt = wt + r * LQB_S;
  float carry[16], wv[16];
#pragma unroll
  for (int t = 0; t < 16; ++t) carry[t] = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 f = *reinterpret_cast<const float4*>(mywt + 4 * q);
    wv[4 * q] = f.x, wv[4 * q + 1] = f.y, wv[4 * q + 2] = f.z, wv[4 * q + 3] = f.w;
  }
#pragma unroll 1
  for (int g = 0; g < ngroups; ++g) {
    const int slot = g & 1;
    // group g - 2's feedback is in acc, and its slot is free again
    if (g >= 2) nb_sync(bar_done + slot, LQB_THREADS);
    float cur[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 a = *reinterpret_cast<const float4*>(myacc + 16 * g + 4 * q);
      cur[4 * q + 0] = a.x + carry[4 * q + 0];
      cur[4 * q + 1] = a.y + carry[4 * q + 1];
      cur[4 * q + 2] = a.z + carry[4 * q + 2];
      cur[4 * q + 3] = a.w + carry[4 * q + 3];
    }
    // carry now collects this group's feedback to the next group, one column
    // at a time as the errors appear (the terms of every element summed in
    // column order), in the issue slots the rounding chain leaves free
#pragma unroll
    for (int j = 0; j < 16; ++j) carry[j] = 0.f;
    float wn[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f = *reinterpret_cast<const float4*>(mywt + 16 * ((g + 1) & 7) + 4 * q);
      wn[4 * q] = f.x, wn[4 * q + 1] = f.y, wn[4 * q + 2] = f.z, wn[4 * q + 3] = f.w;
    }
    float e[16];
    uint32_t cw[4] = {0u, 0u, 0u, 0u};
    // the group's super-diagonal Ů[t][t + 1] in registers: the rounding chain
    // (column t's error into column t + 1) never waits for shared memory
    float sd[15];
#pragma unroll
    for (int t = 0; t < 15; ++t) sd[t] = band[(16 * g + t) * 32 + t + 1];
    // Software-pipelined: column t's error reaches column t + 1 at once (the
    // super-diagonal), and the group's later columns one step later, after
    // column t + 1 has been rounded, from a band row loaded a step ahead.
    float bprev[16], eprev = 0.f;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      float bcur[16];
      const float* ur = band + (16 * g + t) * 32;      // band row 16 g + t
#pragma unroll
      for (int q4 = ((t + 2) >> 2) << 2; q4 < 16; q4 += 4) {
        const float4 u = *reinterpret_cast<const float4*>(ur + q4);
        bcur[q4] = u.x, bcur[q4 + 1] = u.y, bcur[q4 + 2] = u.z, bcur[q4 + 3] = u.w;
      }
      const float z = (cur[t] - l) * inv;
      const float zr = fminf(fmaxf(z, 0.f), qmax) + kRound;
      const float cq = zr - kRound;
      const float err = wv[t] - fmaf(s, cq, l);
      e[t] = err;
      if (t < 15) cur[t + 1] = fmaf(err, sd[t], cur[t + 1]);
#pragma unroll
      for (int q4 = 0; q4 < 16; q4 += 4) {
        const float4 u = *reinterpret_cast<const float4*>(ur + 16 + q4);
        carry[q4 + 0] = fmaf(err, u.x, carry[q4 + 0]);
        carry[q4 + 1] = fmaf(err, u.y, carry[q4 + 1]);
        carry[q4 + 2] = fmaf(err, u.z, carry[q4 + 2]);
        carry[q4 + 3] = fmaf(err, u.w, carry[q4 + 3]);
      }
      cw[t >> 2] |= (__float_as_uint(zr) & 0xffu) << (8 * (t & 3));
      // column t - 1's error into columns t + 1 ..
#pragma unroll
      for (int j = t + 1; j < 16; ++j)
        if (t >= 1) cur[j] = fmaf(eprev, bprev[j], cur[j]);
      eprev = err;
#pragma unroll
      for (int j = t + 2; j < 16; ++j) bprev[j] = bcur[j];
    }
    // hand the errors and codes to the helpers
    float* es = eslot + (slot * LQB_ROWS + r) * LQB_ES;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      *reinterpret_cast<float4*>(es + 4 * q) = make_float4(e[4 * q], e[4 * q + 1], e[4 * q + 2], e[4 * q + 3]);
    *reinterpret_cast<uint4*>(es + 16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    nb_arrive(bar_ready + slot, LQB_THREADS);
#pragma unroll
    for (int t = 0; t < 16; ++t) wv[t] = wn[t];
  }
  }
}

// W~^[i][j] = lo[i] + s[i] * codes[i][j].  Rows i = blockIdx.y, + gridDim.y,
// ...; with vec (n % 4 == 0, both arrays 16-byte aligned) thread t of CTA x
// expands the 4-code groups 4 (1024 x + 256 q + t), q < 4 (coalesced 4-byte
// loads and 16-byte stores across the CTA), else one code at a time.
constexpr int DQ_THREADS = 256;
__global__ void __launch_bounds__(DQ_THREADS) k_dequant(const uint8_t* __restrict__ codes,
                                                        const float* __restrict__ lo,
                                                        const float* __restrict__ sc, int64_t m,
                                                        int64_t n, int vec, float* __restrict__ out) {
  for (int64_t i = blockIdx.y; i < m; i += gridDim.y) {
    const float l = lo[i], s = sc[i];
    const uint8_t* c = codes + i * n;
    float* o = out + i * n;
    if (vec) {
      for (int64_t j0 = 4 * (int64_t)blockIdx.x * 4 * DQ_THREADS; j0 < n;
           j0 += 16 * (int64_t)gridDim.x * DQ_THREADS) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int64_t j = j0 + 4 * (q * DQ_THREADS + threadIdx.x);
          if (j < n) {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(c + j);
            *reinterpret_cast<float4*>(o + j) =
                make_float4(fmaf(s, (float)(w & 0xffu), l), fmaf(s, (float)((w >> 8) & 0xffu), l),
                            fmaf(s, (float)((w >> 16) & 0xffu), l), fmaf(s, (float)(w >> 24), l));
          }
        }
      }
    } else {
      for (int64_t j = (int64_t)blockIdx.x * DQ_THREADS + threadIdx.x; j < n;
           j += (int64_t)gridDim.x * DQ_THREADS)
        o[j] = fmaf(s, (float)c[j], l);
    }
  }
}

}  // namespace quip
