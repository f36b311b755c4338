// libquip: the C ABI declared in include/quip.h, built as one translation
// unit for sm_100a.  Host code here checks arguments, lays out workspace and
// enqueues the kernels of the *.cuh files on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "fwht.cuh"
#include "gemm_simt.cuh"
#include "hessian.cuh"
#include "ldl.cuh"
#include "ldlq.cuh"
#include "rng.cuh"
#include "rounding.cuh"
#include "qmatvec.cuh"
#include "syrk_tc.cuh"
#include "gemm_tc.cuh"
#include "kron_tc.cuh"

using namespace quip;

namespace {

#define QCHECK(expr)                                 \
  do {                                               \
    cudaError_t e_ = (expr);                         \
    if (e_ != cudaSuccess) return QUIP_ERR_CUDA;     \
  } while (0)

struct SideData {
  int kind = QUIP_T_IDENTITY;
  int64_t dim = 0, p = 0, q = 0;
  float* signs = nullptr;   // HADAMARD
  float* A = nullptr;       // KRONECKER p x p
  float* B = nullptr;       // KRONECKER q x q
  double* A64 = nullptr;    // KRONECKER: the same factors in fp64 (Hessian transform)
  double* B64 = nullptr;
  double* G = nullptr;      // KRONECKER: Gaussian draw scratch, max(p,q)^2
  double* Qc = nullptr;     // KRONECKER: QR scratch, max(p,q)^2
  // KRONECKER: three bf16 pieces of A, A^T, B, B^T for the tensor-core
  // products, each 3 x d x ld_piece(d) (rows padded to 16 bytes)
  __nv_bfloat16* fpc = nullptr;
  bool permute = false;     // S = T P, (P x)_r = x_{perm[r]}
  int32_t* perm = nullptr;  // pi (dim)
  int32_t* iperm = nullptr; // pi^-1 (dim)
  uint64_t* keys = nullptr; // permutation draws (dim)
};

// Row stride (elements) of a d x d factor's bf16 pieces: rows padded to 16
// bytes, as TMA requires.
static int64_t factor_ld(int64_t d) { return (d + 7) / 8 * 8; }
static int64_t factor_pieces_elems(int64_t p, int64_t q) {
  return 6 * (p * factor_ld(p) + q * factor_ld(q));
}
// Pieces of factor v: 0 = A, 1 = A^T, 2 = B, 3 = B^T (each 3 x d x factor_ld(d)).
static __nv_bfloat16* factor_pieces(const SideData& sd, int v) {
  const int64_t a = 3 * sd.p * factor_ld(sd.p), b = 3 * sd.q * factor_ld(sd.q);
  switch (v) {
    case 0: return sd.fpc;
    case 1: return sd.fpc + a;
    case 2: return sd.fpc + 2 * a;
    default: return sd.fpc + 2 * a + b;
  }
}


inline bool is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }
inline int ilog2(int64_t x) {
  int l = 0;
  while ((int64_t(1) << l) < x) ++l;
  return l;
}
inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline size_t round256(size_t b) { return (b + 255) & ~size_t(255); }

// ---------------------------------------------------------------- TMA descriptors

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor map with 64 x 64 boxes and the 128-byte swizzle.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 2-D map without swizzle (boxes may be wider than the tensor: the
// columns past it arrive as zeros).
bool make_tmap_f32_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                      uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A second stream per device for the LDL bulk updates, with a fork event and
// a ring of join events, created on first use and kept for the process.
constexpr int kJoinRing = 4;
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr;
  cudaEvent_t join[kJoinRing] = {};
};
cudaError_t side_stream(SideStream& out) {
  static std::mutex mu;
  static SideStream per_dev[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  SideStream& ss = per_dev[dev];
  if (!ss.s) {
    SideStream t;
    if ((e = cudaStreamCreateWithFlags(&t.s, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&t.fork, cudaEventDisableTiming)) != cudaSuccess) return e;
    for (int i = 0; i < kJoinRing; ++i)
      if ((e = cudaEventCreateWithFlags(&t.join[i], cudaEventDisableTiming)) != cudaSuccess) return e;
    ss = t;
  }
  out = ss;
  return cudaSuccess;
}

// A per-device stream of the highest priority for the Hessian path of the
// whole-layer call (H, H~, the LDL: a latency-bound chain that should get
// SMs first), created on first use and kept for the process.
cudaError_t hpath_stream(cudaStream_t* out) {
  static std::mutex mu;
  static cudaStream_t streams[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev]) {
    int least = 0, greatest = 0;
    if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) != cudaSuccess) return e;
    e = cudaStreamCreateWithPriority(&streams[dev], cudaStreamNonBlocking, greatest);
    if (e != cudaSuccess) return e;
  }
  *out = streams[dev];
  return cudaSuccess;
}

// Launch with programmatic stream serialization (the kernel starts with
// pdl_wait_then_release, so it may be scheduled while its predecessor on
// the stream finishes).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

int num_sms() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

// C (+)= alpha * (3-piece A) (3-piece B)^T on the tensor cores; see gemm_tc.cuh.
// max_ctas > 0 caps the persistent grid (leaves SMs to a concurrent stream).
// tb64, when given, is B's map with 64-row boxes: outputs too narrow to fill
// the GPU with 256-wide tiles then use 64-wide ones.
template <int TN>
cudaError_t split_gemm_tn(const CUtensorMap& ta, const CUtensorMap& tb, sgemm::Params p,
                          cudaStream_t st, const char* name, int max_ctas) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(sgemm::k_gemm_split_tc<TN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         sgemm::smem_bytes<TN>());
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int tm = (p.M + sgemm::BM - 1) / sgemm::BM, tn = (p.N + TN - 1) / TN;
  p.tiles_n = tn;
  int valid = 0;                      // tiles that survive the upper-only filter
  for (int ti = 0; ti < tm; ++ti)
    for (int tj = 0; tj < tn; ++tj)
      if (!(p.upper_only && ti * sgemm::BM > tj * TN + TN - 1)) ++valid;
  const int cap = max_ctas > 0 ? std::min(max_ctas, num_sms()) : num_sms();
  const int grid = std::max(1, std::min(valid, cap));
  LaunchScope ls(name, st);
  return launch_pdl(sgemm::k_gemm_split_tc<TN>, dim3(grid), dim3(256), (size_t)sgemm::smem_bytes<TN>(),
                    st, ta, tb, p, tm * tn);
}

cudaError_t split_gemm(const CUtensorMap& ta, const CUtensorMap& tb, sgemm::Params p,
                       cudaStream_t st, const char* name, int max_ctas = 0,
                       const CUtensorMap* tb64 = nullptr, const CUtensorMap* tb128 = nullptr) {
  if (p.M <= 0 || p.N <= 0) return cudaSuccess;
  if (p.upper_only || (!tb64 && !tb128))
    return split_gemm_tn<sgemm::BN>(ta, tb, p, st, name, max_ctas);
  // Tile width by a cost model: waves of tiles x tile width (a tile's time
  // grows with its width at a fixed K); narrower tiles move more operand
  // bytes per product from L2 (an A slot per K block serves TN columns), so
  // 128-wide tiles count 1.25 times and 64-wide ones double (their MMAs are
  // also bound by the A operand's shared-memory reads).  Ties go to the
  // wider tile.
  const int cap = max_ctas > 0 ? std::min(max_ctas, num_sms()) : num_sms();
  const int64_t tm = (p.M + sgemm::BM - 1) / sgemm::BM;
  auto cost = [&](int tn) {
    const int64_t tiles = tm * ((p.N + tn - 1) / tn);
    return ((tiles + cap - 1) / cap) * tn * (tn == 64 ? 8 : tn == 128 ? 5 : 4);
  };
  int best = sgemm::BN;
  if (tb128 && cost(128) < cost(best)) best = 128;
  if (tb64 && cost(64) < cost(best)) best = 64;
  if (best == 128) return split_gemm_tn<128>(ta, *tb128, p, st, name, max_ctas);
  if (best == 64) return split_gemm_tn<64>(ta, *tb64, p, st, name, max_ctas);
  return split_gemm_tn<sgemm::BN>(ta, tb, p, st, name, max_ctas);
}

// ---------------------------------------------------------------- Hadamard plans

inline RowSink f32_sink(float* out, int64_t ld) {
  RowSink k{};
  k.out = out, k.ld = ld;
  return k;
}

template <typename TIn>
cudaError_t fwht_rows(const TIn* in, int64_t ldin, float* out, int64_t ldout, int64_t rows,
                      int64_t d, const float* pre, const float* post, const float* row_sign,
                      float scale, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const int L = ilog2(d);
  if (L < 4) {
    LaunchScope ls("k_fwht_rows", st);
    k_fwht_rows_small<TIn><<<(unsigned)((rows + 127) / 128), 128, 0, st>>>(
        in, ldin, out, ldout, rows, (int)d, pre, post, row_sign, scale);
    return cudaGetLastError();
  }
  if (L == 12) {
    LaunchScope ls("k_fwht_rows", st);
    k_fwht_row4096<TIn, ROW_F32><<<(unsigned)rows, 256, 0, st>>>(in, ldin, RowDequant{}, f32_sink(out, ldout),
                                                                  pre, post, row_sign, scale);
    return cudaGetLastError();
  }
  if (L == 13) {
    LaunchScope ls("k_fwht_rows", st);
    k_fwht_row8192<TIn, ROW_F32><<<(unsigned)rows, 256, 0, st>>>(in, ldin, RowDequant{}, f32_sink(out, ldout),
                                                                  pre, post, row_sign, scale);
    return cudaGetLastError();
  }
  const int T = (int)(d / 16);
  const int NT = T > 256 ? T : 256;
  const int RPC = NT / T;
  const size_t smem = (L > 9) ? (size_t)RPC * (d + d / 32) * sizeof(float) : 0;
  const unsigned grid = (unsigned)((rows + RPC - 1) / RPC);
#define QUIP_ROWS_CASE(LL)                                                                    \
  case LL:                                                                                    \
    {                                                                                         \
      LaunchScope ls("k_fwht_rows", st);                                                      \
      k_fwht_rows<LL, TIn><<<grid, NT, smem, st>>>(in, ldin, out, ldout, rows, pre, post,     \
                                                   row_sign, scale);                          \
    }                                                                                         \
    break;
  switch (L) {
    QUIP_ROWS_CASE(4)
    QUIP_ROWS_CASE(5)
    QUIP_ROWS_CASE(6)
    QUIP_ROWS_CASE(7)
    QUIP_ROWS_CASE(8)
    QUIP_ROWS_CASE(9)
    QUIP_ROWS_CASE(10)
    QUIP_ROWS_CASE(11)
    QUIP_ROWS_CASE(12)
    QUIP_ROWS_CASE(13)
    default:
      return cudaErrorInvalidValue;
  }
#undef QUIP_ROWS_CASE
  return cudaGetLastError();
}

cudaError_t fwht_cols_pass(float* A, int64_t ld, int64_t ncols, int64_t R, int LG, int64_t gs,
                           const float* pre, const float* post, float scale, cudaStream_t st) {
  dim3 grid((unsigned)((ncols + 31) / 32), (unsigned)(R >> LG));
  const int threads = 32 * ((1 << LG) / 16);
#define QUIP_COLS_CASE(LL)                                                                 \
  case LL:                                                                                 \
    {                                                                                      \
      LaunchScope ls("k_fwht_cols", st);                                                   \
      k_fwht_cols<LL><<<grid, threads, 0, st>>>(A, ld, ncols, gs, pre, post, scale);       \
    }                                                                                      \
    break;
  switch (LG) {
    QUIP_COLS_CASE(4)
    QUIP_COLS_CASE(5)
    QUIP_COLS_CASE(6)
    QUIP_COLS_CASE(7)
    QUIP_COLS_CASE(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef QUIP_COLS_CASE
  return cudaGetLastError();
}

// Column Hadamard of an R x ncols matrix (R = 2^L): H_R = H_outer (x) H_inner,
// the inner factor on consecutive rows.  pre-sign on the first pass,
// post-sign and the 1/sqrt(R) scale on the last.
cudaError_t fwht_cols(float* A, int64_t ld, int64_t ncols, int64_t R, const float* pre,
                      const float* post, cudaStream_t st) {
  const int L = ilog2(R);
  const float scale = (float)(1.0 / std::sqrt((double)R));
  if (L < 4) {
    LaunchScope ls("k_fwht_cols", st);
    k_fwht_cols_small<<<(unsigned)((ncols + 127) / 128), 128, 0, st>>>(A, ld, ncols, (int)R,
                                                                        pre, post, scale);
    return cudaGetLastError();
  }
  if (L <= 8) return fwht_cols_pass(A, ld, ncols, R, L, 1, pre, post, scale, st);
  if (L == 12) {
    constexpr int kSmem = (4096 + 256) * FWHT_C4K_NC * (int)sizeof(float);
    static bool attr = false;
    if (!attr) {
      cudaError_t e = cudaFuncSetAttribute(k_fwht_col4096, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
      if (e != cudaSuccess) return e;
      attr = true;
    }
    const int64_t ntiles = (ncols + FWHT_C4K_NC - 1) / FWHT_C4K_NC;
    LaunchScope ls("k_fwht_cols", st);
    k_fwht_col4096<<<(unsigned)ntiles, FWHT_C4K_THREADS, kSmem, st>>>(A, ld, ncols,
                                                                                       pre, post, scale);
    return cudaGetLastError();
  }
  const int Li = (L + 1) / 2, Lo = L - Li;
  cudaError_t e = fwht_cols_pass(A, ld, ncols, R, Li, 1, pre, nullptr, 1.0f, st);
  if (e != cudaSuccess) return e;
  return fwht_cols_pass(A, ld, ncols, R, Lo, int64_t(1) << Li, nullptr, post, scale, st);
}

// ---------------------------------------------------------------- Kronecker plans

// Rows: dst[i, :] = vec(A' Xr_i B'^T) for each row Xr_i (p x q view) of src,
// with A' = A or A^T, B' = B or B^T (transpose = inverse transform).
// Acc = double: fp64 factors and fp64 sums (the Hessian's transform).
template <typename Acc>
struct KronFactors {
  using F = typename std::conditional<std::is_same<Acc, double>::value, double, float>::type;
  static const F* A(const SideData& sd) {
    if constexpr (std::is_same<Acc, double>::value) return sd.A64;
    else return sd.A;
  }
  static const F* B(const SideData& sd) {
    if constexpr (std::is_same<Acc, double>::value) return sd.B64;
    else return sd.B;
  }
};

template <typename TIn, typename Acc = float>
cudaError_t kron_rows(const TIn* src, int64_t ldsrc, float* dst, int64_t rows,
                      const SideData& sd, bool transpose, float* tmp, cudaStream_t st) {
  using KF = KronFactors<Acc>;
  using F = typename KF::F;
  const int64_t p = sd.p, q = sd.q, n = p * q;
  GemmArgs g{};
  // tmp_i = Xr_i B'^T : M = p, N = q, K = q, batched over rows
  g.M = p, g.N = q, g.K = q, g.alpha = 1.f, g.beta = 0.f, g.tri = 0;
  g.A = src, g.sam = q, g.sak = 1, g.sab = ldsrc;
  g.B = KF::B(sd);
  if (!transpose) g.sbk = 1, g.sbn = q;   // B'^T[k][j] = B[j][k]
  else g.sbk = q, g.sbn = 1;              // (B^T)^T = B
  g.sbb = 0;
  g.C = tmp, g.scm = q, g.scn = 1, g.scb = n;
  int64_t batches = rows;
  if (ldsrc == n) {
    // contiguous rows: the p x q views of all rows stack into one (rows p) x q
    // matrix, one GEMM instead of `rows` small ones
    g.M = rows * p, g.sab = 0, g.scb = 0;
    batches = 1;
  }
  cudaError_t e = gemm_simt<TIn, F, Acc>(g, batches, st);
  if (e != cudaSuccess) return e;
  // dst_i = A' tmp_i : M = p, N = q, K = p
  GemmArgs h{};
  h.M = p, h.N = q, h.K = p, h.alpha = 1.f, h.beta = 0.f, h.tri = 0;
  h.A = KF::A(sd);
  if (!transpose) h.sam = p, h.sak = 1;
  else h.sam = 1, h.sak = p;
  h.sab = 0;
  h.B = tmp, h.sbk = q, h.sbn = 1, h.sbb = n;
  h.C = dst, h.scm = q, h.scn = 1, h.scb = n;
  return gemm_simt<F, float, Acc>(h, rows, st);
}

// Columns: X (R x ncols, R = p q) <- (A' (x) B') X, through tmp.
template <typename Acc = float>
cudaError_t kron_cols(float* X, int64_t ncols, const SideData& sd, bool transpose, float* tmp,
                      cudaStream_t st) {
  using KF = KronFactors<Acc>;
  using F = typename KF::F;
  const int64_t p = sd.p, q = sd.q;
  GemmArgs g{};
  // tmp[a'] = B' X[a'] : batch p, M = q, N = ncols, K = q
  g.M = q, g.N = ncols, g.K = q, g.alpha = 1.f, g.beta = 0.f, g.tri = 0;
  g.A = KF::B(sd);
  if (!transpose) g.sam = q, g.sak = 1;
  else g.sam = 1, g.sak = q;
  g.sab = 0;
  g.B = X, g.sbk = ncols, g.sbn = 1, g.sbb = q * ncols;
  g.C = tmp, g.scm = ncols, g.scn = 1, g.scb = q * ncols;
  cudaError_t e = gemm_simt<F, float, Acc>(g, p, st);
  if (e != cudaSuccess) return e;
  // X = A' tmp (tmp as p x (q ncols))
  GemmArgs h{};
  h.M = p, h.N = q * ncols, h.K = p, h.alpha = 1.f, h.beta = 0.f, h.tri = 0;
  h.A = KF::A(sd);
  if (!transpose) h.sam = p, h.sak = 1;
  else h.sam = 1, h.sak = p;
  h.B = tmp, h.sbk = q * ncols, h.sbn = 1;
  h.C = X, h.scm = q * ncols, h.scn = 1;
  return gemm_simt<F, float, Acc>(h, 1, st);
}

// ---------------------------------------------------------------- Kronecker on the tensor cores

// One batched factor product Y[z] = F X[z] (kron_tc.cuh).
cudaError_t kron_tc_launch(const CUtensorMap& tf, const CUtensorMap& tx, kron::Params kp, int mode,
                           cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kron::k_kron_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kron::SMEM_LIMIT);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  kp.tiles_m = (kp.N + kron::BM - 1) / kron::BM;
  const int64_t tiles = (int64_t)kp.tiles_m * kp.slabs;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, num_sms()));
  LaunchScope ls("k_kron_tc", st);
  return launch_pdl(kron::k_kron_tc, dim3(grid), dim3(256), (size_t)kron::smem_bytes(kp.nf), st, tf, tx, kp, mode);
}

// Whether the m-side (column) Kronecker transform of an R x c matrix runs on
// the tensor cores: TMA needs 16-byte row strides (c % 8 == 0), the products
// index tiles with 32-bit coordinates.
bool kron_cols_tc_ok(const SideData& sd, int64_t c) {
  return sd.kind == QUIP_T_KRONECKER && c >= 8 && (c % 8) == 0 && sd.p * sd.q * 3 < ((int64_t)1 << 31) &&
         sd.q * c < ((int64_t)1 << 31);
}

// Workspace of kron_cols_tc: two sets of three bf16 pieces of the R x c data.
size_t kron_cols_tc_bytes(int64_t R, int64_t c) { return 2 * round256((size_t)3 * R * c * 2); }

// dst (R x c fp32, row stride c) = (A' (x) B') src on the tensor cores, with
// A' = A, B' = B (forward) or A^T, B^T (inverse).  src: bf16 (one piece) or
// fp32 (split into three pieces first), row stride ld.  dst may alias an
// fp32 src.  ws: kron_cols_tc_bytes(R, c).
// The two products of kron_cols_tc from data already in xp bf16 pieces
// (xp = 1: bf16 data; xp = 3: the three pieces of fp32 data), piece f of row
// r at xsrc + (f R + r) xld.  Stage 1 writes its pieces to the second half
// of ws, so xsrc may be the first half.
cudaError_t kron_cols_tc_x(const SideData& sd, bool transpose, const __nv_bfloat16* xsrc, int xp, int64_t xld,
                           float* dst, int64_t c, void* ws, cudaStream_t st) {
  const int64_t p = sd.p, q = sd.q, R = p * q;
  __nv_bfloat16* P2 = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(ws) + round256((size_t)3 * R * c * 2));
  // stage 1: T_a' = B' X_a' for the p slabs of q rows, into P2 as pieces
  CUtensorMap mf, mx;
  const int nfq = (int)((q + 15) / 16 * 16), nfp = (int)((p + 15) / 16 * 16);
  const __nv_bfloat16* fb = factor_pieces(sd, transpose ? 3 : 2);
  if (!make_tmap_bf16_2d(&mf, fb, (uint64_t)q, 3 * (uint64_t)q, (uint64_t)factor_ld(q) * 2, 64, (uint32_t)nfq) ||
      !make_tmap_bf16_2d(&mx, xsrc, (uint64_t)c, (uint64_t)(xp * R), (uint64_t)xld * 2, 64, 64))
    return cudaErrorInvalidValue;
  kron::Params kp{};
  kp.d = (int)q, kp.nf = nfq, kp.N = (int)c, kp.slabs = (int)p;
  kp.f_piece_rows = (int)q, kp.x_pieces = xp, kp.x_piece_rows = R, kp.x_slab_rows = q;
  kp.Yp = P2, kp.ldy = c, kp.y_slab_rows = q, kp.y_piece_elems = R * c;
  cudaError_t e = kron_tc_launch(mf, mx, kp, kron::OUT_PIECES, st);
  if (e != cudaSuccess) return e;
  // stage 2: Y = A' T with T as p x (q c), into dst (fp32)
  const __nv_bfloat16* fa = factor_pieces(sd, transpose ? 1 : 0);
  if (!make_tmap_bf16_2d(&mf, fa, (uint64_t)p, 3 * (uint64_t)p, (uint64_t)factor_ld(p) * 2, 64, (uint32_t)nfp) ||
      !make_tmap_bf16_2d(&mx, P2, (uint64_t)(q * c), 3 * (uint64_t)p, (uint64_t)(q * c) * 2, 64, 64))
    return cudaErrorInvalidValue;
  kron::Params k2{};
  k2.d = (int)p, k2.nf = nfp, k2.N = (int)(q * c), k2.slabs = 1;
  k2.f_piece_rows = (int)p, k2.x_pieces = 3, k2.x_piece_rows = p, k2.x_slab_rows = 0;
  k2.Y = dst, k2.ldy = q * c, k2.y_slab_rows = 0;
  return kron_tc_launch(mf, mx, k2, kron::OUT_F32, st);
}

template <typename TIn>
cudaError_t kron_cols_tc(const SideData& sd, bool transpose, const TIn* src, int64_t ld, float* dst,
                         int64_t c, void* ws, cudaStream_t st) {
  if constexpr (std::is_same<TIn, __nv_bfloat16>::value) {
    return kron_cols_tc_x(sd, transpose, src, 1, ld, dst, c, ws, st);
  } else {
    const int64_t R = sd.p * sd.q;
    __nv_bfloat16* P1 = static_cast<__nv_bfloat16*>(ws);
    const int64_t total4 = R * c / 4;
    const unsigned g = (unsigned)std::min<int64_t>((total4 + 255) / 256, 148 * 16);
    {
      LaunchScope ls("k_split_rows3", st);
      k_split_rows3<<<g, 256, 0, st>>>(src, ld, R, c, P1);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return kron_cols_tc_x(sd, transpose, P1, 3, c, dst, c, ws, st);
  }
}

__global__ void k_convert_rows_bf16(const __nv_bfloat16* in, int64_t ld, float* out, int64_t m,
                                    int64_t n) {
  const int64_t total = m * n;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x)
    out[e] = __bfloat162float(in[(e / n) * ld + e % n]);
}
__global__ void k_copy_rows_f32(const float* in, int64_t ld, float* out, int64_t m, int64_t n) {
  const int64_t total = m * n;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x)
    out[e] = in[(e / n) * ld + e % n];
}

// n-side (row) transform of an m x n source into dst (row stride n).
// wide: a Kronecker side takes fp64 factors and sums (the forward transform of
// W: the rounding decisions of LDLQ are sensitive to the error of W~ itself,
// and an fp32 sum over a factor row carries ~sqrt(q) u of it).
template <typename TIn>
cudaError_t side_rows(const SideData& sd, bool inverse, const TIn* src, int64_t ldsrc, float* dst,
                      int64_t rows, float* tmp, cudaStream_t st, bool wide = false) {
  const int64_t n = sd.dim;
  if (sd.kind == QUIP_T_HADAMARD) {
    const float scale = (float)(1.0 / std::sqrt((double)n));
    // forward: y = H (s . x) / sqrt(n); inverse: x = s . (H y) / sqrt(n)
    return fwht_rows<TIn>(src, ldsrc, dst, n, rows, n, inverse ? nullptr : sd.signs,
                          inverse ? sd.signs : nullptr, nullptr, scale, st);
  }
  if (sd.kind == QUIP_T_KRONECKER)
    return wide ? kron_rows<TIn, double>(src, ldsrc, dst, rows, sd, inverse, tmp, st)
                : kron_rows<TIn>(src, ldsrc, dst, rows, sd, inverse, tmp, st);
  // identity
  const unsigned grid = (unsigned)std::min<int64_t>((rows * n + 255) / 256, 65535 * 8);
  if constexpr (std::is_same<TIn, float>::value) {
    if ((const void*)src == (const void*)dst && ldsrc == n) return cudaSuccess;
    LaunchScope ls("k_copy_rows", st);
    k_copy_rows_f32<<<grid, 256, 0, st>>>(src, ldsrc, dst, rows, n);
  } else {
    LaunchScope ls("k_copy_rows", st);
    k_convert_rows_bf16<<<grid, 256, 0, st>>>(src, ldsrc, dst, rows, n);
  }
  return cudaGetLastError();
}

// m-side (column) transform in place on X (R x ncols, row stride ncols).
cudaError_t side_cols(const SideData& sd, bool inverse, float* X, int64_t ncols, float* tmp,
                      cudaStream_t st) {
  if (sd.kind == QUIP_T_HADAMARD)
    return fwht_cols(X, ncols, ncols, sd.dim, inverse ? nullptr : sd.signs,
                     inverse ? sd.signs : nullptr, st);
  if (sd.kind == QUIP_T_KRONECKER) return kron_cols(X, ncols, sd, inverse, tmp, st);
  return cudaSuccess;
}

// out[r][c] = in[rp[r]][cp[c]] (a NULL permutation is the identity), fp32
// out; rows by blockIdx.y (grid-stride), four output columns per thread.
template <typename TIn>
__global__ void __launch_bounds__(256) k_gather2d(const TIn* __restrict__ in, int64_t ldin,
                                                  float* __restrict__ out, int64_t ldout,
                                                  int64_t rows, int64_t cols,
                                                  const int32_t* __restrict__ rp,
                                                  const int32_t* __restrict__ cp) {
  for (int64_t r = blockIdx.y; r < rows; r += gridDim.y) {
    const TIn* src = in + (rp ? (int64_t)rp[r] : r) * ldin;
    float* dst = out + r * ldout;
    for (int64_t c = 4 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x); c < cols;
         c += 4 * (int64_t)gridDim.x * blockDim.x) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (c + k < cols) dst[c + k] = to_f32(src[cp ? (int64_t)cp[c + k] : c + k]);
    }
  }
}

// Row gather with the source row staged in shared memory (k_permute_staged),
// for rows of at most PERMUTE_STAGE_MAX bytes.
template <typename TIn, typename TOut>
cudaError_t permute_staged(const TIn* in, int64_t ldin, TOut* out, int64_t ldout, int64_t rows,
                           int64_t cols, const int32_t* rp, const int32_t* cp, cudaStream_t st,
                           const char* name) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_permute_staged<TIn, TOut>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)PERMUTE_STAGE_MAX);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int64_t row_bytes = cols * (int64_t)sizeof(TIn);
  const size_t smem = (size_t)((row_bytes + 15) / 16 * 16);
  const int vec = (row_bytes % 16 == 0) && ((ldin * (int64_t)sizeof(TIn)) % 16 == 0) &&
                  (reinterpret_cast<uintptr_t>(in) & 15) == 0;
  const unsigned grid = (unsigned)std::min<int64_t>(rows, (int64_t)num_sms() * 8);
  LaunchScope ls(name, st);
  k_permute_staged<TIn, TOut><<<grid, 256, smem, st>>>(in, ldin, out, ldout, rows, cols, vec, rp, cp);
  return cudaGetLastError();
}

template <typename TIn>
cudaError_t gather2d(const TIn* in, int64_t ldin, float* out, int64_t ldout, int64_t rows,
                     int64_t cols, const int32_t* rp, const int32_t* cp, cudaStream_t st) {
  if (cols * (int64_t)sizeof(TIn) <= PERMUTE_STAGE_MAX)
    return permute_staged<TIn, float>(in, ldin, out, ldout, rows, cols, rp, cp, st, "k_gather2d");
  const unsigned gx = (unsigned)std::min<int64_t>((cols + 1023) / 1024, 64);
  const unsigned gy = (unsigned)std::min<int64_t>(rows, 65535);
  LaunchScope ls("k_gather2d", st);
  k_gather2d<TIn><<<dim3(gx, gy), 256, 0, st>>>(in, ldin, out, ldout, rows, cols, rp, cp);
  return cudaGetLastError();
}

}  // namespace

struct quip_transform {
  int device = 0;
  int64_t m = 0, n = 0;
  SideData side[2];
};

// ============================================================================
extern "C" {

const char* quip_status_string(int s) {
  switch (s) {
    case QUIP_OK: return "ok";
    case QUIP_ERR_ARG: return "invalid argument";
    case QUIP_ERR_SHAPE: return "invalid or unsupported shape";
    case QUIP_ERR_UNSUPPORTED: return "unsupported";
    case QUIP_ERR_NOT_PD: return "matrix not positive definite (LDL pivot <= 0)";
    case QUIP_ERR_NONFINITE: return "non-finite value";
    case QUIP_ERR_CUDA: return "CUDA error";
    case QUIP_ERR_TIMEOUT: return "device-side wait timed out";
    case QUIP_ERR_WORKSPACE: return "workspace too small or misaligned";
    default: return "unknown status";
  }
}

const char* quip_version(void) { return "quip-b200 0.1.0 sm_100a"; }

uint64_t quip_kernel_launches(void) { return g_launch_count.load(); }

static quip_status check_side(int kind_flags, int64_t dim, int64_t p, int64_t q) {
  if (kind_flags & ~(0xFF | QUIP_T_PERMUTE)) return QUIP_ERR_ARG;
  const int kind = kind_flags & 0xFF;
  if (dim <= 0) return QUIP_ERR_SHAPE;
  if ((kind_flags & QUIP_T_PERMUTE) && dim > 65536) return QUIP_ERR_SHAPE;
  if (kind == QUIP_T_IDENTITY) return QUIP_OK;
  if (kind == QUIP_T_HADAMARD) return (is_pow2(dim) && dim >= 2 && dim <= 8192) ? QUIP_OK : QUIP_ERR_SHAPE;
  if (kind == QUIP_T_KRONECKER)
    return (p >= 1 && q >= 1 && p <= 256 && q <= 256 && p * q == dim) ? QUIP_OK : QUIP_ERR_SHAPE;
  return QUIP_ERR_ARG;
}

static quip_status alloc_side(SideData& sd, int kind_flags, int64_t dim, int64_t p, int64_t q) {
  const int kind = kind_flags & 0xFF;
  sd.kind = kind, sd.dim = dim, sd.p = p, sd.q = q;
  sd.permute = (kind_flags & QUIP_T_PERMUTE) != 0;
  if (sd.permute) {
    QCHECK(cudaMalloc(&sd.perm, dim * sizeof(int32_t)));
    QCHECK(cudaMalloc(&sd.iperm, dim * sizeof(int32_t)));
    QCHECK(cudaMalloc(&sd.keys, dim * sizeof(uint64_t)));
  }
  if (kind == QUIP_T_HADAMARD) {
    QCHECK(cudaMalloc(&sd.signs, dim * sizeof(float)));
  } else if (kind == QUIP_T_KRONECKER) {
    const int64_t mx = std::max(p, q);
    QCHECK(cudaMalloc(&sd.A, p * p * sizeof(float)));
    QCHECK(cudaMalloc(&sd.B, q * q * sizeof(float)));
    QCHECK(cudaMalloc(&sd.A64, p * p * sizeof(double)));
    QCHECK(cudaMalloc(&sd.B64, q * q * sizeof(double)));
    QCHECK(cudaMalloc(&sd.G, mx * mx * sizeof(double)));
    QCHECK(cudaMalloc(&sd.Qc, mx * mx * sizeof(double)));
    QCHECK(cudaMalloc(&sd.fpc, factor_pieces_elems(p, q) * sizeof(__nv_bfloat16)));
  }
  return QUIP_OK;
}

// Draw one side's random data from `seed` into its existing buffers.
static quip_status draw_side(const SideData& sd, uint64_t seed, int which, cudaStream_t st) {
  if (sd.permute) {
    const unsigned g = (unsigned)((sd.dim + 255) / 256);
    {
      LaunchScope ls("k_perm_keys", st);
      k_perm_keys<<<g, 256, 0, st>>>(sd.keys, sd.dim, seed, which == 0 ? 6u : 7u);
    }
    LaunchScope ls("k_perm_rank", st);
    k_perm_rank<<<g, 256, 0, st>>>(sd.keys, sd.dim, sd.perm, sd.iperm);
  }
  if (sd.kind == QUIP_T_HADAMARD) {
    LaunchScope ls("k_random_signs", st);
    k_random_signs<<<(unsigned)((sd.dim + 255) / 256), 256, 0, st>>>(sd.signs, sd.dim, seed,
                                                                      which == 0 ? 0u : 1u);
  } else if (sd.kind == QUIP_T_KRONECKER) {
    const uint32_t sa = which == 0 ? 2u : 4u, sb = which == 0 ? 3u : 5u;
    for (int f = 0; f < 2; ++f) {
      const int64_t d = f == 0 ? sd.p : sd.q;
      {
        LaunchScope ls("k_gaussian", st);
        k_gaussian<<<(unsigned)((d * d + 255) / 256), 256, 0, st>>>(sd.G, d * d, seed, f == 0 ? sa : sb);
      }
      float* Q = f == 0 ? sd.A : sd.B;
      double* Q64 = f == 0 ? sd.A64 : sd.B64;
      if (d > HAAR_CHOL_MAX) {
        LaunchScope ls("k_haar_cgs2", st);
        k_haar_cgs2<<<1, 256, 0, st>>>(sd.G, sd.Qc, Q, Q64, (int)d);
        continue;
      }
      // Cholesky-QR2 (rng.cuh).  Pass 1: C1 = G^T G packed into Qc, R1 in
      // place, Y = G R1^-1 into Q64 (free until the end).  Pass 2: C2 = Y^T Y
      // into Qc, R2 in place, Q = Y R2^-1 into G (free by then) and, rounded,
      // into Q; then G is copied to Q64.
      static bool attr = false;
      if (!attr) {
        QCHECK(cudaFuncSetAttribute(k_chol64, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)chol64_smem(HAAR_CHOL_MAX)));
        QCHECK(cudaFuncSetAttribute(k_trsm_rows64, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)chol_solve_smem(HAAR_CHOL_MAX)));
        attr = true;
      }
      const unsigned t = (unsigned)((d + 31) / 32);
      const size_t smem = chol64_smem((int)d);
      const size_t smem_t = (size_t)d * (d + 1) / 2 * sizeof(double);
      const unsigned rows = (unsigned)((d + HAAR_SOLVE_ROWS - 1) / HAAR_SOLVE_ROWS);
      // pass 1: C1 = G^T G (Qc, packed), R1 in place, Y = G R1^-1 into Q64
      {
        LaunchScope ls("k_gram64", st);
        k_gram64<<<dim3(t, t), 256, 0, st>>>(sd.G, sd.Qc, (int)d);
      }
      {
        LaunchScope ls("k_chol64", st);
        k_chol64<<<1, 1024, smem, st>>>(sd.Qc, sd.Qc, (int)d);
      }
      {
        LaunchScope ls("k_trsm_rows64", st);
        k_trsm_rows64<<<rows, 32 * HAAR_SOLVE_ROWS, smem_t, st>>>(sd.Qc, sd.G, Q64, nullptr, (int)d);
      }
      // pass 2: C2 = Y^T Y (Qc), R2 in place, Q = Y R2^-1 into G, then to Q64 / Q
      {
        LaunchScope ls("k_gram64", st);
        k_gram64<<<dim3(t, t), 256, 0, st>>>(Q64, sd.Qc, (int)d);
      }
      {
        LaunchScope ls("k_chol64", st);
        k_chol64<<<1, 1024, smem, st>>>(sd.Qc, sd.Qc, (int)d);
      }
      {
        LaunchScope ls("k_trsm_rows64", st);
        k_trsm_rows64<<<rows, 32 * HAAR_SOLVE_ROWS, smem_t, st>>>(sd.Qc, Q64, sd.G, Q, (int)d);
      }
      QCHECK(cudaMemcpyAsync(Q64, sd.G, (size_t)d * d * sizeof(double), cudaMemcpyDeviceToDevice, st));
    }
    // bf16 pieces of A, A^T, B, B^T for the tensor-core products
    for (int v = 0; v < 4; ++v) {
      const int64_t d = v < 2 ? sd.p : sd.q;
      LaunchScope ls("k_split_factor", st);
      k_split_factor<<<(unsigned)((d * d + 255) / 256), 256, 0, st>>>(
          v < 2 ? sd.A : sd.B, (int)d, (int)(v & 1), (int)factor_ld(d), factor_pieces(sd, v));
    }
  }
  QCHECK(cudaGetLastError());
  return QUIP_OK;
}

quip_status quip_transform_create(uint64_t seed, int64_t m, int64_t n, int m_kind, int64_t m_p,
                                  int64_t m_q, int n_kind, int64_t n_p, int64_t n_q, void* stream,
                                  quip_transform** out) {
  if (!out) return QUIP_ERR_ARG;
  *out = nullptr;
  quip_status s;
  if ((s = check_side(m_kind, m, m_p, m_q)) != QUIP_OK) return s;
  if ((s = check_side(n_kind, n, n_p, n_q)) != QUIP_OK) return s;
  quip_transform* tf = new quip_transform();
  cudaGetDevice(&tf->device);
  tf->m = m, tf->n = n;
  if ((s = alloc_side(tf->side[0], m_kind, m, m_p, m_q)) != QUIP_OK ||
      (s = alloc_side(tf->side[1], n_kind, n, n_p, n_q)) != QUIP_OK ||
      (s = quip_transform_draw(tf, seed, stream)) != QUIP_OK) {
    quip_transform_destroy(tf);
    return s;
  }
  *out = tf;
  return QUIP_OK;
}

quip_status quip_transform_draw(quip_transform* tf, uint64_t seed, void* stream) {
  if (!tf) return QUIP_ERR_ARG;
  quip_status s;
  if ((s = draw_side(tf->side[0], seed, 0, S(stream))) != QUIP_OK) return s;
  return draw_side(tf->side[1], seed, 1, S(stream));
}

quip_status quip_transform_destroy(quip_transform* tf) {
  if (!tf) return QUIP_OK;
  cudaDeviceSynchronize();
  for (auto& sd : tf->side) {
    cudaFree(sd.signs);
    cudaFree(sd.A);
    cudaFree(sd.B);
    cudaFree(sd.A64);
    cudaFree(sd.B64);
    cudaFree(sd.G);
    cudaFree(sd.Qc);
    cudaFree(sd.fpc);
    cudaFree(sd.perm);
    cudaFree(sd.iperm);
    cudaFree(sd.keys);
  }
  delete tf;
  return QUIP_OK;
}

quip_status quip_transform_info(const quip_transform* tf, int side, int* kind, int64_t* p,
                                int64_t* q, const float** signs, const float** A,
                                const float** B) {
  if (!tf || side < 0 || side > 1) return QUIP_ERR_ARG;
  const SideData& sd = tf->side[side];
  if (kind) *kind = sd.kind;
  if (p) *p = sd.p;
  if (q) *q = sd.q;
  if (signs) *signs = sd.signs;
  if (A) *A = sd.A;
  if (B) *B = sd.B;
  return QUIP_OK;
}

quip_status quip_transform_permutation(const quip_transform* tf, int side, const int32_t** perm) {
  if (!tf || side < 0 || side > 1 || !perm) return QUIP_ERR_ARG;
  *perm = tf->side[side].perm;
  return QUIP_OK;
}

quip_status quip_hessian_accumulate(const void* X, int dtype, int64_t N, int64_t n, int64_t ldx,
                                    float* H_acc, int accumulate, void* stream) {
  if (!H_acc || (!X && N > 0)) return QUIP_ERR_ARG;
  if (dtype != QUIP_F32 && dtype != QUIP_BF16) return QUIP_ERR_ARG;
  if (n <= 0 || N < 0 || ldx < n || n > (int64_t)1 << 16 || N > ((int64_t)1 << 31) - 64)
    return QUIP_ERR_SHAPE;
  cudaStream_t st = S(stream);
  if (N == 0) {
    if (!accumulate) QCHECK(cudaMemsetAsync(H_acc, 0, n * n * sizeof(float), st));
    return QUIP_OK;
  }
  const bool tma_ok = dtype == QUIP_BF16 && n >= 64 && (ldx % 8) == 0 &&
                      (reinterpret_cast<uintptr_t>(X) % 16) == 0;
  if (tma_ok) {
    CUtensorMap map;
    if (!make_tmap_bf16_2d(&map, X, (uint64_t)n, (uint64_t)N, (uint64_t)ldx * 2, 64, 64))
      return QUIP_ERR_CUDA;
    static bool attr = false;
    if (!attr) {
      QCHECK(cudaFuncSetAttribute(syrk::k_syrk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  syrk::SMEM_BYTES));
      attr = true;
    }
    const int T = (int)((n + syrk::BT - 1) / syrk::BT);
    {
      LaunchScope ls("k_syrk_tc", st);
      syrk::k_syrk_tc<<<T * (T + 1) / 2, 256, syrk::SMEM_BYTES, st>>>(map, H_acc, (int)n, (int)N,
                                                                       accumulate ? 1 : 0);
    }
    QCHECK(cudaGetLastError());
    return QUIP_OK;
  }
  GemmArgs g{};
  g.M = n, g.N = n, g.K = N, g.alpha = 1.f, g.beta = accumulate ? 1.f : 0.f, g.tri = 1;
  g.A = X, g.sam = 1, g.sak = ldx;        // A[i][t] = X[t][i]
  g.B = X, g.sbk = ldx, g.sbn = 1;        // B[t][j] = X[t][j]
  g.C = H_acc, g.scm = n, g.scn = 1;
  if (dtype == QUIP_BF16) QCHECK((gemm_simt<__nv_bfloat16, __nv_bfloat16>(g, 1, st)));
  else QCHECK((gemm_simt<float, float>(g, 1, st)));
  return QUIP_OK;
}

quip_status quip_hessian_finalize(float* H, int64_t n, int64_t N_total, float damp, void* stream) {
  if (!H) return QUIP_ERR_ARG;
  if (n <= 0 || N_total < 1) return QUIP_ERR_SHAPE;
  if (!(damp >= 0.f) || !std::isfinite(damp)) return QUIP_ERR_ARG;
  cudaStream_t st = S(stream);
  {
    LaunchScope ls("k_finalize_diag", st);
    k_finalize_diag<<<1, 1024, 0, st>>>(H, n, 1.0 / (double)N_total, (double)damp);
  }
  const unsigned T = (unsigned)((n + 31) / 32);
  {
    LaunchScope ls("k_mirror_scale", st);
    k_mirror_scale<<<dim3(T, T), 256, 0, st>>>(H, n, (float)(1.0 / (double)N_total));
  }
  QCHECK(cudaGetLastError());
  return QUIP_OK;
}

static int64_t ldl_panels(int64_t n) { return (n + LDL_PB - 1) / LDL_PB; }
// LDL workspace: the current panel's R_pp (128 x 128 fp32), X_J blocks
// (4 x 32 x 32 fp32) and next rows (128 x 128 fp32); two look-ahead buffers
// (n x 128 fp32) and two panels' R12 as three bf16 pieces (3 x n x 128).
static size_t ldl_ws_bytes(int64_t n) {
  return 2 * round256((size_t)LDL_PB * LDL_PB * 4) + round256((size_t)4 * 32 * 32 * 4) +
         round256((size_t)2 * n * LDL_PB * 4) + round256((size_t)6 * n * LDL_PB * 2);
}
// LDLQ workspace: accumulator A (m x n fp32), the error of every column as
// three bf16 pieces (3 x m x n), the split transposed factor (3 x n x n
// bf16) and the transposed factor (n x n fp32).
static size_t ldlq_ws_bytes(int64_t m, int64_t n, int64_t block) {
  (void)block;
  return round256((size_t)m * n * 4) + round256((size_t)3 * m * n * 2) +
         round256((size_t)3 * n * n * 2) + round256((size_t)n * n * 4);
}

// Greedy workspace: the LDLQ run's buffers (accumulator, error pieces, the
// transposed factor in pieces and in fp32) plus the factor U' (n x n fp32)
// and the pass's starting W^ (m x n fp32).
static size_t greedy_ws_bytes(int64_t m, int64_t n) {
  return ldlq_ws_bytes(m, n, 128) + round256((size_t)n * n * 4) + round256((size_t)m * n * 4);
}

// Quantized product: the transformed vectors x' (B x n), the products z
// (B x m) and the Kronecker temporaries of the row transforms (B x max(m, n)),
// all fp32.
static size_t qmatvec_ws_bytes(int64_t m, int64_t n, int64_t B) {
  return round256((size_t)B * n * 4) + round256((size_t)B * m * 4) +
         round256((size_t)B * std::max(m, n) * 4) + 256;
}

// Slot width of a code in a packed word and the words of a packed row.
static int code_slot(int bits) { return (bits == 1 || bits == 2 || bits == 4 || bits == 8) ? bits : (bits < 4 ? 4 : 8); }
static int64_t packed_row_words(int64_t n, int bits) {
  const int64_t per = 32 / code_slot(bits);
  return ((n + per - 1) / per + 3) / 4 * 4;
}

// Transform workspace: Kronecker temporaries, then the permutation scratch
// (the forward pass gathers H into it, the inverse gathers W^).
static size_t transform_kron_bytes(const quip_transform* tf, int op) {
  const SideData &U = tf->side[0], &V = tf->side[1];
  const bool u_tc = kron_cols_tc_ok(U, tf->n);
  size_t b = 0;
  if (V.kind == QUIP_T_KRONECKER || (U.kind == QUIP_T_KRONECKER && !u_tc)) {
    // CUDA-core temporaries: one m x n (and, forward, n x n) fp32 matrix
    size_t e = (size_t)tf->m * tf->n;
    if (op == QUIP_OP_INCOHERENCE_FORWARD) e = std::max(e, (size_t)tf->n * tf->n);
    b = round256(e * sizeof(float));
  }
  if (u_tc) b = std::max(b, kron_cols_tc_bytes(tf->m, tf->n));   // tensor-core pieces
  return b;
}
static size_t transform_perm_bytes(const quip_transform* tf, int op) {
  if (op == QUIP_OP_INCOHERENCE_FORWARD)
    return tf->side[1].permute ? round256((size_t)tf->n * tf->n * sizeof(float)) : 0;
  return (tf->side[0].permute || tf->side[1].permute) ? round256((size_t)tf->m * tf->n * sizeof(float))
                                                      : 0;
}

quip_status quip_workspace_size(int op, const quip_transform* tf, int64_t m, int64_t n,
                                int64_t block, size_t* bytes) {
  if (!bytes) return QUIP_ERR_ARG;
  *bytes = 0;
  switch (op) {
    case QUIP_OP_INCOHERENCE_FORWARD:
    case QUIP_OP_INCOHERENCE_INVERSE: {
      if (!tf) return QUIP_ERR_ARG;
      *bytes = transform_kron_bytes(tf, op) + transform_perm_bytes(tf, op);
      return QUIP_OK;
    }
    case QUIP_OP_LDL:
      if (n <= 0) return QUIP_ERR_SHAPE;
      *bytes = ldl_ws_bytes(n);
      return QUIP_OK;
    case QUIP_OP_LDLQ:
      if (m <= 0 || n <= 0 || block <= 0) return QUIP_ERR_SHAPE;
      *bytes = ldlq_ws_bytes(m, n, block);
      return QUIP_OK;
    case QUIP_OP_GREEDY:
      if (m <= 0 || n <= 0) return QUIP_ERR_SHAPE;
      *bytes = greedy_ws_bytes(m, n);
      return QUIP_OK;
    case QUIP_OP_QMATVEC:
      if (!tf) return QUIP_ERR_ARG;
      if (block <= 0) return QUIP_ERR_SHAPE;
      *bytes = qmatvec_ws_bytes(tf->m, tf->n, block);
      return QUIP_OK;
    default:
      return QUIP_ERR_ARG;
  }
}

static quip_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return QUIP_OK;
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255)) return QUIP_ERR_WORKSPACE;
  return QUIP_OK;
}

quip_status quip_incoherence_forward(const quip_transform* tf, const void* W, int w_dtype,
                                     int64_t ldw, float* W_t, float* H, void* ws, size_t ws_bytes,
                                     void* stream) {
  if (!tf || (!W && !H) || (W && !W_t)) return QUIP_ERR_ARG;
  const int64_t m = tf->m, n = tf->n;
  const SideData &U = tf->side[0], &V = tf->side[1];
  if (W) {
    if (w_dtype != QUIP_F32 && w_dtype != QUIP_BF16) return QUIP_ERR_ARG;
    if (ldw < n) return QUIP_ERR_SHAPE;
    if (V.kind == QUIP_T_HADAMARD && n >= 16) {   // vector loads and stores in the row kernels
      const size_t esz = w_dtype == QUIP_BF16 ? 2 : 4;
      if ((reinterpret_cast<uintptr_t>(W) % 16) || ((ldw * esz) % 16) || (reinterpret_cast<uintptr_t>(W_t) % 16))
        return QUIP_ERR_ARG;
    }
  }
  if (H && V.kind == QUIP_T_HADAMARD && n >= 16 && (reinterpret_cast<uintptr_t>(H) % 16)) return QUIP_ERR_ARG;
  size_t need = 0;
  quip_status s = quip_workspace_size(QUIP_OP_INCOHERENCE_FORWARD, tf, m, n, 0, &need);
  if (s != QUIP_OK) return s;
  if ((s = check_ws(ws, ws_bytes, need)) != QUIP_OK) return s;
  cudaStream_t st = S(stream);
  float* tmp = static_cast<float*>(ws);
  float* pscr = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                         transform_kron_bytes(tf, QUIP_OP_INCOHERENCE_FORWARD));
  const bool u_tc = kron_cols_tc_ok(U, n);
  if (W) {
    const int32_t* rp = U.permute ? U.perm : nullptr;
    const int32_t* cp = V.permute ? V.perm : nullptr;
    if (u_tc && !rp && !cp && w_dtype == QUIP_BF16 && (ldw % 8) == 0) {
      // bf16 W is its own single piece: the m-side Kronecker factors first,
      // straight from W (three products per term pair), then the n side in place
      QCHECK(kron_cols_tc<__nv_bfloat16>(U, false, static_cast<const __nv_bfloat16*>(W), ldw, W_t, n, ws, st));
      QCHECK(side_rows<float>(V, false, W_t, n, W_t, m, tmp, st, true));
    } else if (rp || cp) {
      // W_t = P_m W P_n^T (W_t[r][c] = W[pi_m[r]][pi_n[c]]), then the structured factors in place
      if (w_dtype == QUIP_BF16)
        QCHECK(gather2d<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(W), ldw, W_t, n, m, n, rp, cp, st));
      else
        QCHECK(gather2d<float>(static_cast<const float*>(W), ldw, W_t, n, m, n, rp, cp, st));
      QCHECK(side_rows<float>(V, false, W_t, n, W_t, m, tmp, st, true));
    } else if (w_dtype == QUIP_BF16) {
      QCHECK(side_rows<__nv_bfloat16>(V, false, static_cast<const __nv_bfloat16*>(W), ldw, W_t, m, tmp, st, true));
    } else {
      QCHECK(side_rows<float>(V, false, static_cast<const float*>(W), ldw, W_t, m, tmp, st, true));
    }
    if (!(u_tc && !rp && !cp && w_dtype == QUIP_BF16 && (ldw % 8) == 0)) {
      if (u_tc) QCHECK(kron_cols_tc<float>(U, false, W_t, n, W_t, n, ws, st));
      else QCHECK(side_cols(U, false, W_t, n, tmp, st));
    }
  }
  if (H && V.permute) {
    // P_n H P_n^T, through the scratch
    QCHECK(gather2d<float>(H, n, pscr, n, n, n, V.perm, V.perm, st));
    QCHECK(cudaMemcpyAsync(H, pscr, (size_t)n * n * sizeof(float), cudaMemcpyDeviceToDevice, st));
  }
  if (H) {
    if (V.kind == QUIP_T_KRONECKER) {                           // fp64 sums, see gemm_simt.cuh
      QCHECK((kron_rows<float, double>(H, n, H, n, V, false, tmp, st)));   // H V^T
      QCHECK((kron_cols<double>(H, n, V, false, tmp, st)));                // V (H V^T)
    } else {
      QCHECK(side_rows<float>(V, false, H, n, H, n, tmp, st));   // H V^T
      QCHECK(side_cols(V, false, H, n, tmp, st));                // V (H V^T)
    }
  }
  return QUIP_OK;
}

quip_status quip_incoherence_inverse(const quip_transform* tf, const float* W_hat_t, float* W_hat,
                                     void* ws, size_t ws_bytes, void* stream) {
  if (!tf || !W_hat_t || !W_hat) return QUIP_ERR_ARG;
  const int64_t m = tf->m, n = tf->n;
  if (tf->side[1].kind == QUIP_T_HADAMARD && n >= 16 &&
      ((reinterpret_cast<uintptr_t>(W_hat_t) % 16) || (reinterpret_cast<uintptr_t>(W_hat) % 16)))
    return QUIP_ERR_ARG;                               // vector loads and stores in the row kernels
  size_t need = 0;
  quip_status s = quip_workspace_size(QUIP_OP_INCOHERENCE_INVERSE, tf, m, n, 0, &need);
  if (s != QUIP_OK) return s;
  if ((s = check_ws(ws, ws_bytes, need)) != QUIP_OK) return s;
  cudaStream_t st = S(stream);
  float* tmp = static_cast<float*>(ws);
  QCHECK(side_rows<float>(tf->side[1], true, W_hat_t, n, W_hat, m, tmp, st));
  if (kron_cols_tc_ok(tf->side[0], n)) QCHECK(kron_cols_tc<float>(tf->side[0], true, W_hat, n, W_hat, n, ws, st));
  else QCHECK(side_cols(tf->side[0], true, W_hat, n, tmp, st));
  const SideData &U = tf->side[0], &V = tf->side[1];
  if (U.permute || V.permute) {
    // W^ = P_m^T (T_m^T W~^ T_n) P_n: W^[r][c] = M[pi_m^-1[r]][pi_n^-1[c]], through the scratch
    float* pscr = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                           transform_kron_bytes(tf, QUIP_OP_INCOHERENCE_INVERSE));
    QCHECK(gather2d<float>(W_hat, n, pscr, n, m, n, U.permute ? U.iperm : nullptr,
                           V.permute ? V.iperm : nullptr, st));
    QCHECK(cudaMemcpyAsync(W_hat, pscr, (size_t)m * n * sizeof(float), cudaMemcpyDeviceToDevice, st));
  }
  return QUIP_OK;
}

quip_status quip_ldl(float* H_t, float* D, int64_t n, void* ws, size_t ws_bytes, void* stream) {
  if (!H_t || !D) return QUIP_ERR_ARG;
  if (n <= 0 || n > ((int64_t)1 << 16)) return QUIP_ERR_SHAPE;
  if ((n & 3) || (reinterpret_cast<uintptr_t>(H_t) & 15)) return QUIP_ERR_SHAPE;
  quip_status s = check_ws(ws, ws_bytes, ldl_ws_bytes(n));
  if (s != QUIP_OK) return s;
  cudaStream_t st = S(stream);
  const int64_t P = ldl_panels(n);
  char* w8 = static_cast<char*>(ws);
  float* Rd = reinterpret_cast<float*>(w8);
  w8 += round256((size_t)LDL_PB * LDL_PB * 4);
  float* Nx = reinterpret_cast<float*>(w8);
  w8 += round256((size_t)LDL_PB * LDL_PB * 4);
  float* Xw = reinterpret_cast<float*>(w8);
  w8 += round256((size_t)4 * 32 * 32 * 4);
  float* Lb = reinterpret_cast<float*>(w8);
  w8 += round256((size_t)2 * n * LDL_PB * 4);
  __nv_bfloat16* Rs = reinterpret_cast<__nv_bfloat16*>(w8);
  const size_t smem_f = ((size_t)(LDL_PB + 32) * LDL_LDA + 5 * 32 * LDL_LDX + 96) * sizeof(float);
  const size_t smem_r =
      128 + ((size_t)(2 * LDL_RR + 2 * LDL_PB) * LDL_LDA + LDL_PB * LDL_LDX) * sizeof(float);
  static bool attr = false;
  if (!attr) {
    QCHECK(cudaFuncSetAttribute(k_ldl_factor, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_f));
    QCHECK(cudaFuncSetAttribute(k_ldl_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_r));
    attr = true;
  }
  // fp32 tiles for the row kernel, landing with the padded smem row stride
  CUtensorMap mH32, mL32, mR, mX, mN32, mN128;
  if (!make_tmap_f32_2d(&mH32, H_t, n, n, n * 4, LDL_LDA, LDL_RR) ||
      !make_tmap_f32_2d(&mL32, Lb, LDL_PB, 2 * n, LDL_PB * 4, LDL_LDA, LDL_RR) ||
      !make_tmap_f32_2d(&mR, Rd, LDL_PB, LDL_PB, LDL_PB * 4, LDL_LDA, LDL_PB) ||
      !make_tmap_f32_2d(&mX, Xw, 32, LDL_PB, 32 * 4, LDL_LDX, LDL_PB) ||
      !make_tmap_f32_2d(&mN32, Nx, LDL_PB, LDL_PB, LDL_PB * 4, LDL_LDA, LDL_RR) ||
      !make_tmap_f32_2d(&mN128, Nx, LDL_PB, LDL_PB, LDL_PB * 4, LDL_LDA, LDL_PB))
    return QUIP_ERR_CUDA;
  // Rs holds two panels' R12 (buffer p & 1), pieces at rows (3 buf + q) n.
  CUtensorMap ta, tb;
  SideStream side;
  if (P > 2) {
    if (!make_tmap_bf16_2d(&ta, Rs, LDL_PB, 6 * (uint64_t)n, LDL_PB * 2, 64, sgemm::BM) ||
        !make_tmap_bf16_2d(&tb, Rs, LDL_PB, 6 * (uint64_t)n, LDL_PB * 2, 64, sgemm::BN))
      return QUIP_ERR_CUDA;
    QCHECK(side_stream(side));
  }
  const float* Lin = nullptr;
  int lin0 = -1;                 // Lin's first row in mL32
  for (int64_t p = P - 1; p >= 0; --p) {
    const int64_t c0 = p * LDL_PB;
    const int w = (int)std::min<int64_t>(LDL_PB, n - c0);
    const int buf = (int)(p & 1);
    // panel p has had every update except panel p + 1's once the bulk update
    // of panel p + 2 is done (panel p + 1's arrives through Lin)
    if (p + 2 <= P - 1) QCHECK(cudaStreamWaitEvent(st, side.join[(p + 2) % kJoinRing], 0));
    {
      LaunchScope ls("k_ldl_factor", st);
      QCHECK(launch_pdl(k_ldl_factor, dim3(c0 > 0 ? LDL_FCTAS : 1), dim3(LDL_FT), smem_f, st, H_t, n,
                        c0, w, Lin, Rd, Xw, Nx, D));
    }
    if (c0 == 0) break;
    float* Lout = Lb + (size_t)buf * n * LDL_PB;
    {
      const int nblk = (int)(c0 / LDL_RR);
      LaunchScope ls("k_ldl_rows", st);
      QCHECK(launch_pdl(k_ldl_rows, dim3((unsigned)nblk), dim3(LDL_RT), smem_r, st, mH32, mL32, mR, mX,
                        mN32, mN128, H_t, n, c0, w, lin0, (int64_t)0, nblk,
                        Rs + (size_t)buf * 3 * n * LDL_PB, Lout));
    }
    if (c0 > LDL_PB) {
      // H[:c0-128, :c0-128] -= R12 R12^T on the upper tiles, on the side
      // stream; the SMs that the next panel's factor and row kernels need
      // stay free.
      QCHECK(cudaEventRecord(side.fork, st));
      QCHECK(cudaStreamWaitEvent(side.s, side.fork, 0));
      sgemm::Params gp{};
      gp.C = H_t, gp.ldc = n, gp.M = (int)(c0 - LDL_PB), gp.N = (int)(c0 - LDL_PB), gp.K = LDL_PB;
      gp.a_piece_rows = (int)n, gp.b_piece_rows = (int)n;
      gp.a_row0 = gp.b_row0 = 3 * (int)n * buf;
      gp.alpha = -1.f, gp.upper_only = 1;
      const int next_rows_sms = (int)((c0 - LDL_PB) / LDL_RR);
      const int cap = std::max(num_sms() / 2, num_sms() - LDL_FCTAS - next_rows_sms);
      QCHECK(split_gemm(ta, tb, gp, side.s, "k_gemm_split_tc[ldl]", cap));
      QCHECK(cudaEventRecord(side.join[p % kJoinRing], side.s));
    }
    Lin = Lout;
    lin0 = buf * (int)n;
  }
  QCHECK(cudaGetLastError());
  return QUIP_OK;
}

namespace {
struct LdlqRun {
  const float* Wt;
  float* A;
  const float* U;
  int64_t ldu, m, n;
  const float* lo;
  const float* sc;
  float qmax;
  uint8_t* codes;
  __nv_bfloat16* Es;
  CUtensorMap ta, tb, tb64, tb128, tacc, tut, tband, tw;
  cudaStream_t st;
  // optional: code_ev[c] is recorded once the block kernels of column blocks
  // [c code_every, (c + 1) code_every) have written their codes
  const cudaEvent_t* code_ev;
  int code_every;
};

constexpr int LDQ_BLK = 128;               // LDLQ block width (columns)
constexpr int64_t LQB_BLOCK_COLS = LDQ_BLK;

// One 32-row sub-group per CTA while that fits one wave of the GPU, else two
// (fewer waves of the rows' rounding chains).
cudaError_t ldlq_block(const LdlqRun& r, int64_t k0, int w) {
  const int64_t units = (r.m + LQB_ROWS - 1) / LQB_ROWS;
  cudaError_t e;
  {
    LaunchScope ls("k_ldlq_block", r.st);
    if (units <= num_sms())
      e = launch_pdl(k_ldlq_block<1>, dim3((unsigned)units), dim3(LQB_THREADS), (size_t)lqb_smem(1), r.st,
                     r.tacc, r.tut, r.tband, r.tw, r.m, r.n, k0, w, r.lo, r.sc, r.qmax, r.codes, r.Es, r.n);
    else
      e = launch_pdl(k_ldlq_block<2>, dim3((unsigned)((units + 1) / 2)), dim3(2 * LQB_THREADS),
                     (size_t)lqb_smem(2), r.st, r.tacc, r.tut, r.tband, r.tw, r.m, r.n, k0, w, r.lo, r.sc,
                     r.qmax, r.codes, r.Es, r.n);
  }
  if (e != cudaSuccess || !r.code_ev) return e;
  const int64_t blk = k0 / LQB_BLOCK_COLS;
  if ((blk + 1) % r.code_every == 0 || k0 + w >= r.n) e = cudaEventRecord(r.code_ev[blk / r.code_every], r.st);
  return e;
}

// Tensor maps of a run: the block kernel's (accumulator, weights, the
// transposed factor UTf, the factor's band) and, with gemm, the split
// GEMMs' (errors Es as A; UTs, the transposed factor's bf16 pieces, as B in
// 256-, 128- and 64-row boxes).
bool ldlq_maps(LdlqRun& r, const float* UTf, const __nv_bfloat16* UTs, bool gemm) {
  const uint64_t m = (uint64_t)r.m, n = (uint64_t)r.n;
  if (!make_tmap_f32_2d(&r.tacc, r.A, n, m, n * 4, LQB_S, LQB_ROWS) ||
      !make_tmap_f32_2d(&r.tw, r.Wt, n, m, n * 4, LQB_S, LQB_ROWS) ||
      !make_tmap_f32_2d(&r.tut, UTf, n, n, n * 4, LQB_S, 128) ||
      !make_tmap_f32_2d(&r.tband, r.U, n, n, (uint64_t)r.ldu * 4, 32, 16))
    return false;
  if (!gemm) return true;
  return make_tmap_bf16_2d(&r.ta, r.Es, n, 3 * m, n * 2, 64, sgemm::BM) &&
         make_tmap_bf16_2d(&r.tb, UTs, n, 3 * n, n * 2, 64, sgemm::BN) &&
         make_tmap_bf16_2d(&r.tb64, UTs, n, 3 * n, n * 2, 64, 64) &&
         make_tmap_bf16_2d(&r.tb128, UTs, n, 3 * n, n * 2, 64, 128);
}

void ldlq_block_attr() {
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(k_ldlq_block<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, lqb_smem(1));
    cudaFuncSetAttribute(k_ldlq_block<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, lqb_smem(2));
    attr = true;
  }
}

// Columns [a, b): left half, then A[:, mid:b] += Err[:, a:mid] Ů[a:mid, mid:b]
// in one split GEMM, then the right half.  Every column's feedback is the
// same sum as in the column-by-column definition, grouped differently.
cudaError_t ldlq_range(const LdlqRun& r, int64_t a, int64_t b) {
  const int64_t nb = (b - a + LDQ_BLK - 1) / LDQ_BLK;
  if (nb <= 1) return ldlq_block(r, a, (int)(b - a));
  const int64_t mid = a + ((nb + 1) / 2) * LDQ_BLK;
  cudaError_t e = ldlq_range(r, a, mid);
  if (e != cudaSuccess) return e;
  sgemm::Params gp{};
  gp.C = r.A + mid, gp.ldc = r.n, gp.M = (int)r.m, gp.N = (int)(b - mid), gp.K = (int)(mid - a);
  gp.a_piece_rows = (int)r.m, gp.a_k0 = (int)a;
  gp.b_piece_rows = (int)r.n, gp.b_row0 = (int)mid, gp.b_k0 = (int)a;
  gp.alpha = 1.f;
  e = split_gemm(r.ta, r.tb, gp, r.st, "k_gemm_split_tc[ldlq]", 0, &r.tb64, &r.tb128);
  if (e != cudaSuccess) return e;
  return ldlq_range(r, mid, b);
}
}  // namespace

}  // extern "C"

namespace {
// Argument checks of quip_ldlq_quantize that do not involve pointers.
quip_status ldlq_shape_ok(int64_t m, int64_t n, int bits, int64_t block) {
  if (bits < 1 || bits > 8) return QUIP_ERR_ARG;
  if (m <= 0 || n <= 0) return QUIP_ERR_SHAPE;
  if (!(block == 32 || block == 64 || block == 128) || n % block) return QUIP_ERR_SHAPE;
  // every block size is processed in 128-column blocks (the last one may be
  // 64 wide; same result), so n must be a multiple of 64
  if (n % 64) return QUIP_ERR_SHAPE;
  if (m > ((int64_t)1 << 20) || n > ((int64_t)1 << 16)) return QUIP_ERR_SHAPE;
  return QUIP_OK;
}

// The part of LDLQ that needs W~ only: the per-row grid and the accumulator's
// start A = W~ (m x n fp32).
cudaError_t ldlq_prepare(const float* W_t, int64_t m, int64_t n, int bits, float* lo, float* scale, float* A,
                         cudaStream_t st) {
  {
    LaunchScope ls("k_row_grid", st);
    k_row_grid<<<(unsigned)((m + 7) / 8), 256, 0, st>>>(W_t, m, n, (1 << bits) - 1, lo, scale);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return cudaMemcpyAsync(A, W_t, (size_t)m * n * sizeof(float), cudaMemcpyDeviceToDevice, st);
}

// The rest of LDLQ once ldlq_prepare has run: ws_rest holds the error pieces
// and the transposed factor (ldlq_ws_bytes less the accumulator).
quip_status ldlq_main(const float* W_t, const float* Uring, int64_t ldu, int64_t m, int64_t n, int bits,
                      uint8_t* codes, const float* lo, const float* scale, float* A, void* ws_rest,
                      cudaStream_t st, const cudaEvent_t* code_ev = nullptr, int code_every = 1) {
  LdlqRun r{};
  r.st = st;
  r.code_ev = code_ev, r.code_every = code_every;
  char* w8 = static_cast<char*>(ws_rest);
  r.A = A;
  r.Es = reinterpret_cast<__nv_bfloat16*>(w8);
  w8 += round256((size_t)3 * m * n * 2);
  __nv_bfloat16* UTs = reinterpret_cast<__nv_bfloat16*>(w8);
  w8 += round256((size_t)3 * n * n * 2);
  float* UTf = reinterpret_cast<float*>(w8);
  r.Wt = W_t, r.U = Uring, r.ldu = ldu, r.m = m, r.n = n, r.lo = lo, r.sc = scale;
  r.qmax = (float)((1 << bits) - 1), r.codes = codes;
  {
    const unsigned T = (unsigned)((n + 31) / 32);
    LaunchScope ls("k_split_upper_transposed", r.st);
    k_split_upper_transposed<<<dim3(T, T), 256, 0, r.st>>>(Uring, ldu, n, UTs, UTf);
  }
  if (!ldlq_maps(r, UTf, UTs, n > LDQ_BLK)) return QUIP_ERR_CUDA;
  ldlq_block_attr();
  QCHECK(ldlq_range(r, 0, n));
  return QUIP_OK;
}
}  // namespace

extern "C" {

quip_status quip_ldlq_quantize(const float* W_t, const float* Uring, int64_t ldu, int64_t m,
                               int64_t n, int bits, int64_t block, uint8_t* codes, float* lo,
                               float* scale, void* ws, size_t ws_bytes, void* stream) {
  if (!W_t || !Uring || !codes || !lo || !scale) return QUIP_ERR_ARG;
  quip_status s = ldlq_shape_ok(m, n, bits, block);
  if (s != QUIP_OK) return s;
  if (ldu < n) return QUIP_ERR_SHAPE;
  if ((ldu & 3) || (reinterpret_cast<uintptr_t>(Uring) & 15) || (reinterpret_cast<uintptr_t>(W_t) & 15))
    return QUIP_ERR_ARG;
  if ((s = check_ws(ws, ws_bytes, ldlq_ws_bytes(m, n, block))) != QUIP_OK) return s;
  cudaStream_t st = S(stream);
  float* A = static_cast<float*>(ws);
  QCHECK(ldlq_prepare(W_t, m, n, bits, lo, scale, A, st));
  return ldlq_main(W_t, Uring, ldu, m, n, bits, codes, lo, scale, A,
                   static_cast<char*>(ws) + round256((size_t)m * n * 4), st);
}

quip_status quip_nearest_quantize(const float* W_t, int64_t m, int64_t n, int bits, uint8_t* codes,
                                  float* lo, float* scale, void* stream) {
  if (!W_t || !codes || !lo || !scale) return QUIP_ERR_ARG;
  if (bits < 1 || bits > 8) return QUIP_ERR_ARG;
  if (m <= 0 || n <= 0) return QUIP_ERR_SHAPE;
  cudaStream_t st = S(stream);
  {
    LaunchScope ls("k_row_grid", st);
    k_row_grid<<<(unsigned)((m + 7) / 8), 256, 0, st>>>(W_t, m, n, (1 << bits) - 1, lo, scale);
  }
  const int vec = (n & 3) == 0 && (reinterpret_cast<uintptr_t>(codes) & 3) == 0 &&
                  (reinterpret_cast<uintptr_t>(W_t) & 15) == 0;
  const int64_t per_cta = (vec ? 4 : 1) * (int64_t)NR_THREADS;
  const unsigned gx = (unsigned)std::min<int64_t>((n + per_cta - 1) / per_cta, 1024);
  const unsigned gy = (unsigned)std::min<int64_t>(m, 65535);
  {
    LaunchScope ls("k_nearest", st);
    k_nearest<<<dim3(gx, gy), NR_THREADS, 0, st>>>(W_t, lo, scale, m, n, vec,
                                                    (float)((1 << bits) - 1), codes);
  }
  QCHECK(cudaGetLastError());
  return QUIP_OK;
}

quip_status quip_diag_order(const float* H, int64_t ldh, int64_t n, int32_t* perm, int32_t* iperm,
                            void* stream) {
  if (!H || !perm) return QUIP_ERR_ARG;
  if (n <= 0 || n > 65536 || ldh < n) return QUIP_ERR_SHAPE;
  cudaStream_t st = S(stream);
  {
    LaunchScope ls("k_diag_rank", st);
    k_diag_rank<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(H, ldh, n, perm, iperm);
  }
  QCHECK(cudaGetLastError());
  return QUIP_OK;
}

quip_status quip_permute(const void* in, int dtype, int64_t rows, int64_t cols, int64_t ldin,
                         const int32_t* row_perm, const int32_t* col_perm, void* out, int64_t ldout,
                         void* stream) {
  if (!in || !out) return QUIP_ERR_ARG;
  if (rows <= 0 || cols <= 0 || ldin < cols || ldout < cols) return QUIP_ERR_SHAPE;
  if (rows > INT32_MAX || cols > INT32_MAX) return QUIP_ERR_SHAPE;
  size_t es = 0;
  if (dtype == QUIP_F32) es = 4;
  else if (dtype == QUIP_BF16) es = 2;
  else if (dtype == QUIP_U8) es = 1;
  else return QUIP_ERR_ARG;
  // the two arrays may not overlap
  const char* a = static_cast<const char*>(in);
  const char* b = static_cast<const char*>(out);
  const size_t ea = es * (size_t)((rows - 1) * ldin + cols), eb = es * (size_t)((rows - 1) * ldout + cols);
  if (a < b + eb && b < a + ea) return QUIP_ERR_ARG;
  cudaStream_t st = S(stream);
  if (cols * (int64_t)es <= PERMUTE_STAGE_MAX) {
    cudaError_t e;
    if (es == 4)
      e = permute_staged(static_cast<const uint32_t*>(in), ldin, static_cast<uint32_t*>(out), ldout, rows,
                         cols, row_perm, col_perm, st, "k_permute");
    else if (es == 2)
      e = permute_staged(static_cast<const uint16_t*>(in), ldin, static_cast<uint16_t*>(out), ldout, rows,
                         cols, row_perm, col_perm, st, "k_permute");
    else
      e = permute_staged(static_cast<const uint8_t*>(in), ldin, static_cast<uint8_t*>(out), ldout, rows,
                         cols, row_perm, col_perm, st, "k_permute");
    QCHECK(e);
    return QUIP_OK;
  }
  const unsigned gx = (unsigned)std::min<int64_t>((cols + 255) / 256, 64);
  const unsigned gy = (unsigned)std::min<int64_t>(rows, 65535);
  LaunchScope ls("k_permute", st);
  if (es == 4)
    k_permute<uint32_t><<<dim3(gx, gy), 256, 0, st>>>(static_cast<const uint32_t*>(in), ldin,
                                                       static_cast<uint32_t*>(out), ldout, rows, cols,
                                                       row_perm, col_perm);
  else if (es == 2)
    k_permute<uint16_t><<<dim3(gx, gy), 256, 0, st>>>(static_cast<const uint16_t*>(in), ldin,
                                                       static_cast<uint16_t*>(out), ldout, rows, cols,
                                                       row_perm, col_perm);
  else
    k_permute<uint8_t><<<dim3(gx, gy), 256, 0, st>>>(static_cast<const uint8_t*>(in), ldin,
                                                      static_cast<uint8_t*>(out), ldout, rows, cols,
                                                      row_perm, col_perm);
  QCHECK(cudaGetLastError());
  return QUIP_OK;
}

quip_status quip_greedy_refine(const float* W_t, const float* H, int64_t ldh, int64_t m, int64_t n,
                               int bits, const float* lo, const float* scale, uint8_t* codes,
                               int passes, void* ws, size_t ws_bytes, void* stream) {
  if (!W_t || !H || !lo || !scale || !codes) return QUIP_ERR_ARG;
  if (bits < 1 || bits > 8 || passes < 0) return QUIP_ERR_ARG;
  if (m <= 0 || n <= 0 || ldh < n) return QUIP_ERR_SHAPE;
  if (n % 64) return QUIP_ERR_SHAPE;
  if (m > ((int64_t)1 << 20) || n > ((int64_t)1 << 16)) return QUIP_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(W_t) & 15) || (reinterpret_cast<uintptr_t>(codes) & 15))
    return QUIP_ERR_ARG;
  quip_status s = check_ws(ws, ws_bytes, greedy_ws_bytes(m, n));
  if (s != QUIP_OK) return s;
  if (passes == 0) return QUIP_OK;
  cudaStream_t st = S(stream);
  char* w8 = static_cast<char*>(ws);
  LdlqRun r{};
  r.st = st;
  r.A = reinterpret_cast<float*>(w8);
  w8 += round256((size_t)m * n * 4);
  r.Es = reinterpret_cast<__nv_bfloat16*>(w8);
  w8 += round256((size_t)3 * m * n * 2);
  __nv_bfloat16* UTs = reinterpret_cast<__nv_bfloat16*>(w8);
  w8 += round256((size_t)3 * n * n * 2);
  float* UTf = reinterpret_cast<float*>(w8);
  w8 += round256((size_t)n * n * 4);
  float* Ur = reinterpret_cast<float*>(w8);
  w8 += round256((size_t)n * n * 4);
  float* What = reinterpret_cast<float*>(w8);
  r.Wt = What, r.U = Ur, r.ldu = n, r.m = m, r.n = n, r.lo = lo, r.sc = scale;
  r.qmax = (float)((1 << bits) - 1), r.codes = codes;
  {
    const unsigned T = (unsigned)(n / 32);
    LaunchScope ls("k_greedy_factors", st);
    k_greedy_factors<<<dim3(T, T), 256, 0, st>>>(H, ldh, n, UTf, UTs, Ur);
  }
  if (!ldlq_maps(r, UTf, UTs, true)) return QUIP_ERR_CUDA;
  ldlq_block_attr();
  const unsigned gx = (unsigned)std::min<int64_t>((n + 1023) / 1024, 1024);
  const unsigned gy = (unsigned)std::min<int64_t>(m, 65535);
  for (int p = 0; p < passes; ++p) {
    {
      LaunchScope ls("k_greedy_start", st);
      k_greedy_start<<<dim3(gx, gy), 256, 0, st>>>(codes, lo, scale, W_t, m, n, What, r.A, r.Es);
    }
    // A = W^old - (E H) D^-1: every column's feedback from the pass's start
    sgemm::Params gp{};
    gp.C = r.A, gp.ldc = n, gp.M = (int)m, gp.N = (int)n, gp.K = (int)n;
    gp.a_piece_rows = (int)m, gp.b_piece_rows = (int)n;
    gp.alpha = -1.f;
    QCHECK(split_gemm(r.ta, r.tb, gp, st, "k_gemm_split_tc[greedy]", 0, &r.tb64, &r.tb128));
    // then LDLQ's recursion with weights W^old and factor U'_jk = H_jk / H_kk
    QCHECK(ldlq_range(r, 0, n));
  }
  return QUIP_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- static scratch

// Workspace of quip_ldlq_quantize_static: a fixed array in the library's own
// device memory, so that entry point never allocates.  Host code may not use
// the symbol as a pointer (on the host it is only a stand-in); its device
// address is looked up once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_ldlq_scratch[QUIP_LDLQ_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
void* g_ldlq_scratch_ptr[kMaxDevices] = {};
std::mutex g_ldlq_scratch_mu;

// Device address of g_ldlq_scratch on the current device.  Outside stream
// capture it is looked up on every call (cheap once the module is loaded), so
// a cudaDeviceReset, after which the module is loaded again and the array may
// sit elsewhere, never leaves a stale address behind; while `stream` is
// capturing, the address from the last call outside capture is used (and a
// device never looked up outside capture is an error).
quip_status ldlq_static_scratch(cudaStream_t stream, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QUIP_ERR_CUDA;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return QUIP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_ldlq_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ldlq_scratch) != cudaSuccess || !p) return QUIP_ERR_CUDA;
    g_ldlq_scratch_ptr[dev] = p;
  } else if (!g_ldlq_scratch_ptr[dev]) {
    return QUIP_ERR_CUDA;
  }
  *out = g_ldlq_scratch_ptr[dev];
  return QUIP_OK;
}
}  // namespace

extern "C" {

quip_status quip_ldlq_quantize_static(const float* W_t, const float* Uring, int64_t ldu, int64_t m,
                                      int64_t n, int bits, int64_t block, uint8_t* codes, float* lo,
                                      float* scale, void* stream) {
  size_t need = 0;
  if (m > 0 && n > 0 && block > 0) {
    quip_status s = quip_workspace_size(QUIP_OP_LDLQ, nullptr, m, n, block, &need);
    if (s != QUIP_OK) return s;
    if (need > (size_t)QUIP_LDLQ_STATIC_SCRATCH_BYTES) return QUIP_ERR_WORKSPACE;
  }
  void* ws = nullptr;
  quip_status s = ldlq_static_scratch(S(stream), &ws);
  if (s != QUIP_OK) return s;
  return quip_ldlq_quantize(W_t, Uring, ldu, m, n, bits, block, codes, lo, scale, ws,
                            (size_t)QUIP_LDLQ_STATIC_SCRATCH_BYTES, stream);
}

int64_t quip_packed_words(int64_t n, int bits) {
  if (n <= 0 || bits < 1 || bits > 8) return 0;
  return packed_row_words(n, bits);
}

quip_status quip_pack_codes(const uint8_t* codes, int64_t m, int64_t n, int bits, uint32_t* packed,
                            int64_t ldp, void* stream) {
  if (!codes || !packed) return QUIP_ERR_ARG;
  if (bits < 1 || bits > 8) return QUIP_ERR_ARG;
  if (m <= 0 || n <= 0) return QUIP_ERR_SHAPE;
  const int64_t Wd = packed_row_words(n, bits);
  if (ldp < Wd || (ldp & 3) || (reinterpret_cast<uintptr_t>(packed) & 15)) return QUIP_ERR_SHAPE;
  cudaStream_t st = S(stream);
  const unsigned grid = (unsigned)std::min<int64_t>((m * Wd + 255) / 256, (int64_t)num_sms() * 16);
  LaunchScope ls("k_pack_codes", st);
  switch (code_slot(bits)) {
    case 1: k_pack_codes<1><<<grid, 256, 0, st>>>(codes, m, n, Wd, packed, ldp); break;
    case 2: k_pack_codes<2><<<grid, 256, 0, st>>>(codes, m, n, Wd, packed, ldp); break;
    case 4: k_pack_codes<4><<<grid, 256, 0, st>>>(codes, m, n, Wd, packed, ldp); break;
    default: k_pack_codes<8><<<grid, 256, 0, st>>>(codes, m, n, Wd, packed, ldp); break;
  }
  QCHECK(cudaGetLastError());
  return QUIP_OK;
}

}  // extern "C"

namespace {
template <int SLOT, int BC>
cudaError_t qmatvec_launch(const uint32_t* packed, int64_t ldp, int64_t Wd, const float* lo,
                           const float* sc, int64_t m, int64_t n, const float* xs, int nb, float* z,
                           cudaStream_t st) {
  const int64_t tasks = (m + qmv_rows<BC>() - 1) / qmv_rows<BC>();
  const unsigned grid = (unsigned)std::max<int64_t>(
      1, std::min<int64_t>((tasks + QMV_WARPS - 1) / QMV_WARPS, (int64_t)num_sms() * 8));
  LaunchScope ls("k_qmatvec", st);
  k_qmatvec<SLOT, BC><<<grid, QMV_WARPS * 32, 0, st>>>(packed, ldp, Wd, lo, sc, m, n, xs, n, nb, z, m);
  return cudaGetLastError();
}

// The vectors in chunks of up to 8 (4 for 1-bit slots, whose 32 slots per
// word would need more registers).
template <int SLOT>
cudaError_t qmatvec_slot(const uint32_t* packed, int64_t ldp, int64_t Wd, const float* lo, const float* sc,
                         int64_t m, int64_t n, const float* xs, int64_t B, float* z, cudaStream_t st) {
  const int bc = SLOT == 1 ? 4 : 8;
  for (int64_t b0 = 0; b0 < B; b0 += bc) {
    const int nb = (int)std::min<int64_t>(bc, B - b0);
    const float* x = xs + b0 * n;
    float* zz = z + b0 * m;
    cudaError_t e;
    if (nb > 4) e = qmatvec_launch<SLOT, (SLOT == 1 ? 4 : 8)>(packed, ldp, Wd, lo, sc, m, n, x, nb, zz, st);
    else if (nb > 2) e = qmatvec_launch<SLOT, 4>(packed, ldp, Wd, lo, sc, m, n, x, nb, zz, st);
    else if (nb == 2) e = qmatvec_launch<SLOT, 2>(packed, ldp, Wd, lo, sc, m, n, x, nb, zz, st);
    else e = qmatvec_launch<SLOT, 1>(packed, ldp, Wd, lo, sc, m, n, x, nb, zz, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// A Kronecker side on a few fp32 vectors in one launch (k_kron_vec).
bool kron_vec_fits(const SideData& sd) {
  return sd.kind == QUIP_T_KRONECKER && sd.p <= 65535 && sd.q <= 1024;
}
cudaError_t kron_vec(const SideData& sd, bool inverse, const float* x, int64_t ldx, float* y, int64_t ldy,
                     int64_t B, cudaStream_t st) {
  LaunchScope ls("k_kron_vec", st);
  k_kron_vec<<<dim3((unsigned)sd.p, (unsigned)B), 256, 0, st>>>(sd.A, sd.B, (int)sd.p, (int)sd.q,
                                                                inverse ? 1 : 0, x, ldx, y, ldy);
  return cudaGetLastError();
}

// The one-launch product (k_qlinear) for Hadamard / identity sides without
// permutation: the vectors in chunks of BC (8, 4, 2 or 1, as many as fit
// BC x max(n, m) fp32 in shared memory).
constexpr int64_t QL_SMEM_MAX = 200 * 1024;

template <int SLOT, int BC, typename TX>
cudaError_t qlinear_launch(const uint32_t* packed, int64_t ldp, int64_t Wd, const float* lo, const float* sc,
                           int64_t m, int64_t n, const TX* x, int64_t ldx, int nb, const float* vs, float vscale,
                           const float* us, float uscale, float* z, unsigned* counter, float* y, int64_t ldy,
                           cudaStream_t st) {
  const size_t smem = (size_t)BC * ((std::max(m, n) + 3) / 4 * 4) * sizeof(float);
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_qlinear<SLOT, BC, TX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)QL_SMEM_MAX);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  // one CTA per SM at most: every CTA transforms the
  // vectors itself, so fewer, larger CTAs repeat that less
  const int64_t tasks = (m + qmv_rows<BC>() - 1) / qmv_rows<BC>();
  const unsigned grid = (unsigned)std::max<int64_t>(
      1, std::min<int64_t>((tasks + ql_warps<BC>() - 1) / ql_warps<BC>(), (int64_t)num_sms()));
  cudaError_t e = cudaMemsetAsync(counter, 0, sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  LaunchScope ls("k_qlinear", st);
  k_qlinear<SLOT, BC, TX><<<grid, ql_warps<BC>() * 32, smem, st>>>(packed, ldp, Wd, lo, sc, (int)m, (int)n, x, ldx,
                                                             nb, vs, vscale, us, uscale, z, counter, y, ldy);
  return cudaGetLastError();
}

template <int SLOT, typename TX>
cudaError_t qlinear_slot(const uint32_t* packed, int64_t ldp, int64_t Wd, const float* lo, const float* sc,
                         int64_t m, int64_t n, const TX* x, int64_t ldx, int64_t B, const float* vs,
                         float vscale, const float* us, float uscale, float* z, unsigned* counter, float* y,
                         int64_t ldy, int bc, cudaStream_t st) {
  for (int64_t b0 = 0; b0 < B; b0 += bc) {
    const int nb = (int)std::min<int64_t>(bc, B - b0);
    const TX* xx = x + b0 * ldx;
    float* yy = y + b0 * ldy;
    cudaError_t e;
#define QL_ARGS packed, ldp, Wd, lo, sc, m, n, xx, ldx, nb, vs, vscale, us, uscale, z, counter, yy, ldy, st
    if (bc == 8) e = qlinear_launch<SLOT, 8, TX>(QL_ARGS);
    else if (bc == 4) e = qlinear_launch<SLOT, 4, TX>(QL_ARGS);
    else if (bc == 2) e = qlinear_launch<SLOT, 2, TX>(QL_ARGS);
    else e = qlinear_launch<SLOT, 1, TX>(QL_ARGS);
#undef QL_ARGS
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename TX>
cudaError_t qlinear(int slot, const uint32_t* packed, int64_t ldp, int64_t Wd, const float* lo, const float* sc,
                    int64_t m, int64_t n, const TX* x, int64_t ldx, int64_t B, const float* vs, float vscale,
                    const float* us, float uscale, float* z, unsigned* counter, float* y, int64_t ldy, int bc,
                    cudaStream_t st) {
#define QL_ARGS packed, ldp, Wd, lo, sc, m, n, x, ldx, B, vs, vscale, us, uscale, z, counter, y, ldy, bc, st
  switch (slot) {
    case 1: return qlinear_slot<1, TX>(QL_ARGS);
    case 2: return qlinear_slot<2, TX>(QL_ARGS);
    case 4: return qlinear_slot<4, TX>(QL_ARGS);
    default: return qlinear_slot<8, TX>(QL_ARGS);
  }
#undef QL_ARGS
}
}  // namespace

extern "C" {

quip_status quip_qmatvec(const quip_transform* tf, const uint32_t* packed, int64_t ldp, const float* lo,
                         const float* scale, int bits, const void* x, int x_dtype, int64_t ldx, int64_t B,
                         float* y, int64_t ldy, void* ws, size_t ws_bytes, void* stream) {
  if (!tf || !packed || !lo || !scale || !x || !y) return QUIP_ERR_ARG;
  if (bits < 1 || bits > 8) return QUIP_ERR_ARG;
  if (x_dtype != QUIP_F32 && x_dtype != QUIP_BF16) return QUIP_ERR_ARG;
  const int64_t m = tf->m, n = tf->n;
  if (B <= 0 || ldx < n || ldy < m) return QUIP_ERR_SHAPE;
  const int slot = code_slot(bits);
  const int64_t Wd = packed_row_words(n, bits);
  if (ldp < Wd || (ldp & 3) || (reinterpret_cast<uintptr_t>(packed) & 15)) return QUIP_ERR_SHAPE;
  if (n % 4) return QUIP_ERR_SHAPE;
  const SideData &U = tf->side[0], &V = tf->side[1];
  if (V.kind == QUIP_T_HADAMARD && n >= 16 && !V.permute) {   // vector loads in the row kernel
    const size_t esz = x_dtype == QUIP_BF16 ? 2 : 4;
    if ((reinterpret_cast<uintptr_t>(x) % 16) || ((ldx * esz) % 16)) return QUIP_ERR_ARG;
  }
  quip_status s = check_ws(ws, ws_bytes, qmatvec_ws_bytes(m, n, B));
  if (s != QUIP_OK) return s;
  cudaStream_t st = S(stream);
  char* w8 = static_cast<char*>(ws);
  float* xs = reinterpret_cast<float*>(w8);
  w8 += round256((size_t)B * n * 4);
  float* z = reinterpret_cast<float*>(w8);
  w8 += round256((size_t)B * m * 4);
  float* tmp = reinterpret_cast<float*>(w8);
  unsigned* counter = reinterpret_cast<unsigned*>(reinterpret_cast<char*>(tmp) +
                                                 round256((size_t)B * std::max(m, n) * 4));
  // one launch per vector chunk (k_qlinear) when neither side permutes and a
  // chunk's vectors fit in shared memory: Hadamard / identity sides inside
  // the launch, a Kronecker side (k_kron_vec) as one more launch before
  // (V x into xs) or after (U^T z from tmp)
  const bool kin = V.kind == QUIP_T_KRONECKER, kout = U.kind == QUIP_T_KRONECKER;
  const bool simple = !U.permute && !V.permute && (!kin || (kron_vec_fits(V) && x_dtype == QUIP_F32)) &&
                      (!kout || kron_vec_fits(U));
  const int64_t dmax = (std::max(m, n) + 3) / 4 * 4;
  const int bc = std::min<int64_t>(B, 8) > 4 && 8 * dmax * 4 <= QL_SMEM_MAX ? 8
               : std::min<int64_t>(B, 8) > 2 && 4 * dmax * 4 <= QL_SMEM_MAX ? 4
               : std::min<int64_t>(B, 8) > 1 && 2 * dmax * 4 <= QL_SMEM_MAX ? 2
               : dmax * 4 <= QL_SMEM_MAX ? 1 : 0;
  if (simple && bc > 0 && m <= INT32_MAX && n <= INT32_MAX) {
    const float* vs = V.kind == QUIP_T_HADAMARD ? V.signs : nullptr;
    const float* us = U.kind == QUIP_T_HADAMARD ? U.signs : nullptr;
    const float vscale = vs ? (float)(1.0 / std::sqrt((double)n)) : 1.f;
    const float uscale = us ? (float)(1.0 / std::sqrt((double)m)) : 1.f;
    const void* xin = x;
    int64_t ldin = ldx;
    if (kin) {
      QCHECK(kron_vec(V, false, static_cast<const float*>(x), ldx, xs, n, B, st));
      xin = xs, ldin = n;
    }
    float* yout = kout ? tmp : y;
    const int64_t ldout = kout ? m : ldy;
    cudaError_t e;
    if (x_dtype == QUIP_BF16)
      e = qlinear<__nv_bfloat16>(slot, packed, ldp, Wd, lo, scale, m, n, static_cast<const __nv_bfloat16*>(xin),
                                 ldin, B, vs, vscale, us, uscale, z, counter, yout, ldout, bc, st);
    else
      e = qlinear<float>(slot, packed, ldp, Wd, lo, scale, m, n, static_cast<const float*>(xin), ldin, B, vs,
                         vscale, us, uscale, z, counter, yout, ldout, bc, st);
    QCHECK(e);
    if (kout) QCHECK(kron_vec(U, true, tmp, m, y, ldy, B, st));
    return QUIP_OK;
  }
  // x' = V x = T_n (P_n x), the vectors as rows
  if (V.permute) {
    if (x_dtype == QUIP_BF16)
      QCHECK(gather2d<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x), ldx, xs, n, B, n, nullptr, V.perm, st));
    else
      QCHECK(gather2d<float>(static_cast<const float*>(x), ldx, xs, n, B, n, nullptr, V.perm, st));
    QCHECK(side_rows<float>(V, false, xs, n, xs, B, tmp, st));
  } else if (x_dtype == QUIP_BF16) {
    QCHECK(side_rows<__nv_bfloat16>(V, false, static_cast<const __nv_bfloat16*>(x), ldx, xs, B, tmp, st));
  } else {
    QCHECK(side_rows<float>(V, false, static_cast<const float*>(x), ldx, xs, B, tmp, st));
  }
  // z = W~^ x'
  switch (slot) {
    case 1: QCHECK(qmatvec_slot<1>(packed, ldp, Wd, lo, scale, m, n, xs, B, z, st)); break;
    case 2: QCHECK(qmatvec_slot<2>(packed, ldp, Wd, lo, scale, m, n, xs, B, z, st)); break;
    case 4: QCHECK(qmatvec_slot<4>(packed, ldp, Wd, lo, scale, m, n, xs, B, z, st)); break;
    default: QCHECK(qmatvec_slot<8>(packed, ldp, Wd, lo, scale, m, n, xs, B, z, st)); break;
  }
  // y = U^T z = P_m^T (T_m^T z)
  if (U.permute || ldy != m) {
    QCHECK(side_rows<float>(U, true, z, m, z, B, tmp, st));
    QCHECK(gather2d<float>(z, m, y, ldy, B, m, nullptr, U.permute ? U.iperm : nullptr, st));
  } else {
    QCHECK(side_rows<float>(U, true, z, m, y, B, tmp, st));
  }
  return QUIP_OK;
}

quip_status quip_dequantize(const uint8_t* codes, const float* lo, const float* scale, int64_t m,
                            int64_t n, float* W_hat_t, void* stream) {
  if (!codes || !lo || !scale || !W_hat_t) return QUIP_ERR_ARG;
  if (m <= 0 || n <= 0) return QUIP_ERR_SHAPE;
  const int vec = (n & 3) == 0 && (reinterpret_cast<uintptr_t>(codes) & 3) == 0 &&
                  (reinterpret_cast<uintptr_t>(W_hat_t) & 15) == 0;
  const int64_t per_cta = (vec ? 16 : 1) * (int64_t)DQ_THREADS;
  const unsigned gx = (unsigned)std::min<int64_t>((n + per_cta - 1) / per_cta, 1024);
  const unsigned gy = (unsigned)std::min<int64_t>(m, 65535);
  {
    LaunchScope ls("k_dequant", S(stream));
    k_dequant<<<dim3(gx, gy), DQ_THREADS, 0, S(stream)>>>(codes, lo, scale, m, n, vec, W_hat_t);
  }
  QCHECK(cudaGetLastError());
  return QUIP_OK;
}

// ---------------------------------------------------------------- whole layer

namespace {
// A per-device stream for host <-> device copies of quip_quantize_layer_host,
// created on first use and kept for the process.
cudaError_t copy_stream(cudaStream_t* out) {
  static std::mutex mu;
  static cudaStream_t streams[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev]) {
    e = cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking);
    if (e != cudaSuccess) return e;
  }
  *out = streams[dev];
  return cudaSuccess;
}


// Device workspace of the whole-layer call: H (n x n), D (n), W~ (m x n),
// then one region shared by the stages (the largest stage workspace); the
// host variant adds device copies of W and X, and the device results: codes
// (m x n), lo and scale (m each) and W^ (m x n fp32).
struct LayerWs {
  size_t H, D, Wt, stage, wstage, Wd, Xd, codes, lo, sc, What, total;
};

// The events of one layer call, destroyed on every way out of it, error
// returns included (an event still pending is released once it completes).
struct CallEvents {
  std::vector<cudaEvent_t> e;
  explicit CallEvents(size_t k) : e(k, nullptr) {}
  ~CallEvents() {
    for (cudaEvent_t x : e)
      if (x) cudaEventDestroy(x);
  }
  CallEvents(const CallEvents&) = delete;
  CallEvents& operator=(const CallEvents&) = delete;
  cudaError_t create() {
    for (auto& x : e) {
      const cudaError_t r = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
      if (r != cudaSuccess) return r;
    }
    return cudaSuccess;
  }
};

quip_status layer_ws(const quip_transform* tf, int64_t N, int w_dtype, int x_dtype, int64_t block, bool host,
                     LayerWs* o) {
  const int64_t m = tf->m, n = tf->n;
  size_t st = 0, b = 0;
  quip_status s;
  const int ops[4] = {QUIP_OP_INCOHERENCE_FORWARD, QUIP_OP_INCOHERENCE_INVERSE, QUIP_OP_LDL, QUIP_OP_LDLQ};
  for (int op : ops) {
    if ((s = quip_workspace_size(op, tf, m, n, block, &b)) != QUIP_OK) return s;
    st = std::max(st, b);
  }
  const size_t wes = w_dtype == QUIP_BF16 ? 2 : 4, xes = x_dtype == QUIP_BF16 ? 2 : 4;
  *o = LayerWs{};
  o->H = round256((size_t)n * n * 4);
  o->D = round256((size_t)n * 4);
  o->Wt = round256((size_t)m * n * 4);
  o->stage = round256(std::max<size_t>(st, 256));
  // the W path's forward transform runs beside the Hessian path: its own
  // region, which then holds LDLQ's accumulator (started on the W path)
  if ((s = quip_workspace_size(QUIP_OP_INCOHERENCE_FORWARD, tf, m, n, block, &b)) != QUIP_OK) return s;
  o->wstage = round256(std::max<size_t>(std::max<size_t>(b, (size_t)m * n * 4), 256));
  if (host) {
    o->Wd = round256((size_t)m * n * wes);
    o->Xd = round256((size_t)std::max<int64_t>(N, 1) * n * xes);
    o->codes = round256((size_t)m * n);
    o->lo = o->sc = round256((size_t)m * 4);
    o->What = round256((size_t)m * n * 4);
  }
  o->total = o->H + o->D + o->Wt + o->stage + o->wstage + o->Wd + o->Xd + o->codes + o->lo + o->sc + o->What;
  return QUIP_OK;
}

quip_status layer_args(const quip_transform* tf, int w_dtype, int64_t ldw, int x_dtype, int64_t N, int64_t ldx,
                       int bits, int64_t block, float damp) {
  if (!tf) return QUIP_ERR_ARG;
  quip_status s = ldlq_shape_ok(tf->m, tf->n, bits, block);
  if (s != QUIP_OK) return s;
  if ((w_dtype != QUIP_F32 && w_dtype != QUIP_BF16) || (x_dtype != QUIP_F32 && x_dtype != QUIP_BF16))
    return QUIP_ERR_ARG;
  if (bits < 1 || bits > 8 || !(damp >= 0.f) || !std::isfinite(damp)) return QUIP_ERR_ARG;
  if (N < 1 || ldw < tf->n || ldx < tf->n) return QUIP_ERR_SHAPE;
  if (!(block == 32 || block == 64 || block == 128) || tf->n % block || tf->n % 64) return QUIP_ERR_SHAPE;
  return QUIP_OK;
}

// Token chunks of X in the host variant: X's copy lands in up to four
// pieces, each accumulated into H as soon as it is on the device.
// W~ = U W V^T and LDLQ's start (per-row grid, accumulator A = W~) for the
// layer call.  With bf16 W, a tensor-core Kronecker m side and an n-side
// Hadamard of 4096 or 8192 points, the Hadamard row kernel comes last and
// writes W~ twice (W_t and A) and the row grid while each row is in
// registers (no separate grid and copy passes); the values are those of
// quip_incoherence_forward then ldlq_prepare (the same operations in the
// same order; min and max are exact).  Otherwise those two calls.
quip_status forward_w_ldlq_start(const quip_transform* tf, const void* W, int w_dtype, int64_t ldw, float* W_t,
                                 int bits, float* lo, float* scale, float* A, void* ws, size_t ws_bytes,
                                 cudaStream_t st) {
  const int64_t m = tf->m, n = tf->n;
  const SideData &U = tf->side[0], &V = tf->side[1];
  const int L = n > 0 ? ilog2(n) : 0;
  const bool fused = w_dtype == QUIP_BF16 && (ldw % 8) == 0 && (reinterpret_cast<uintptr_t>(W) & 15) == 0 &&
                     V.kind == QUIP_T_HADAMARD && !V.permute && !U.permute && (L == 12 || L == 13) &&
                     (int64_t(1) << L) == n && kron_cols_tc_ok(U, n) && (reinterpret_cast<uintptr_t>(W_t) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(A) & 15) == 0;
  if (!fused) {
    quip_status r = quip_incoherence_forward(tf, W, w_dtype, ldw, W_t, nullptr, ws, ws_bytes, st);
    if (r != QUIP_OK) return r;
    QCHECK(ldlq_prepare(W_t, m, n, bits, lo, scale, A, st));
    return QUIP_OK;
  }
  size_t need = 0;
  quip_status s = quip_workspace_size(QUIP_OP_INCOHERENCE_FORWARD, tf, m, n, 0, &need);
  if (s != QUIP_OK) return s;
  if ((s = check_ws(ws, ws_bytes, need)) != QUIP_OK) return s;
  QCHECK(kron_cols_tc<__nv_bfloat16>(U, false, static_cast<const __nv_bfloat16*>(W), ldw, W_t, n, ws, st));
  RowSink sk{};
  sk.out = W_t, sk.out2 = A, sk.ld = n, sk.lo = lo, sk.sc = scale, sk.qmax = (float)((1 << bits) - 1);
  const float sc = (float)(1.0 / std::sqrt((double)n));
  {
    LaunchScope ls("k_fwht_rows", st);
    if (L == 13)
      k_fwht_row8192<float, ROW_GRID><<<(unsigned)m, 256, 0, st>>>(W_t, n, RowDequant{}, sk, V.signs, nullptr,
                                                                   nullptr, sc);
    else
      k_fwht_row4096<float, ROW_GRID><<<(unsigned)m, 256, 0, st>>>(W_t, n, RowDequant{}, sk, V.signs, nullptr,
                                                                   nullptr, sc);
  }
  QCHECK(cudaGetLastError());
  return QUIP_OK;
}

// W_hat = U^T (lo + s . codes) V, the layer call's last step.  With an
// n-side Hadamard of 4096 or 8192 points the dequantisation is folded into
// the row kernel (it reads the codes), and with a tensor-core Kronecker m
// side the row kernel writes the three bf16 pieces that the Kronecker
// products read: no fp32 W~^ and no separate split pass in between.  The
// arithmetic is that of quip_dequantize followed by quip_incoherence_inverse
// (the same fused multiply-add per code, the same butterflies, the same
// split), so W_hat is the same to the bit.  Other transforms take those two
// calls.  ws: QUIP_OP_INCOHERENCE_INVERSE.
quip_status inverse_from_codes(const quip_transform* tf, const uint8_t* codes, const float* lo,
                               const float* scale, float* W_hat, void* ws, size_t ws_bytes, cudaStream_t st) {
  const int64_t m = tf->m, n = tf->n;
  const SideData &U = tf->side[0], &V = tf->side[1];
  const int L = n > 0 ? ilog2(n) : 0;
  const bool fused = V.kind == QUIP_T_HADAMARD && !V.permute && !U.permute && (L == 12 || L == 13) &&
                     (int64_t(1) << L) == n && (reinterpret_cast<uintptr_t>(codes) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(W_hat) & 15) == 0;
  if (!fused) {
    quip_status r = quip_dequantize(codes, lo, scale, m, n, W_hat, st);
    if (r != QUIP_OK) return r;
    return quip_incoherence_inverse(tf, W_hat, W_hat, ws, ws_bytes, st);
  }
  size_t need = 0;
  quip_status s = quip_workspace_size(QUIP_OP_INCOHERENCE_INVERSE, tf, m, n, 0, &need);
  if (s != QUIP_OK) return s;
  if ((s = check_ws(ws, ws_bytes, need)) != QUIP_OK) return s;
  const float sc = (float)(1.0 / std::sqrt((double)n));
  const RowDequant dq{lo, scale};
  const bool tc = kron_cols_tc_ok(U, n);
  __nv_bfloat16* P1 = static_cast<__nv_bfloat16*>(ws);
  const int64_t pst = m * n;
  RowSink sk{};
  sk.ld = n;
  if (tc) sk.outp = P1, sk.pst = pst;
  else sk.out = W_hat;
  {
    LaunchScope ls("k_fwht_rows", st);
    if (L == 13 && tc)
      k_fwht_row8192<uint8_t, ROW_PIECES><<<(unsigned)m, 256, 0, st>>>(codes, n, dq, sk, nullptr, V.signs, nullptr, sc);
    else if (L == 13)
      k_fwht_row8192<uint8_t, ROW_F32><<<(unsigned)m, 256, 0, st>>>(codes, n, dq, sk, nullptr, V.signs, nullptr, sc);
    else if (tc)
      k_fwht_row4096<uint8_t, ROW_PIECES><<<(unsigned)m, 256, 0, st>>>(codes, n, dq, sk, nullptr, V.signs, nullptr, sc);
    else
      k_fwht_row4096<uint8_t, ROW_F32><<<(unsigned)m, 256, 0, st>>>(codes, n, dq, sk, nullptr, V.signs, nullptr, sc);
  }
  QCHECK(cudaGetLastError());
  if (tc) QCHECK(kron_cols_tc_x(U, true, P1, 3, n, W_hat, n, ws, st));
  else QCHECK(side_cols(U, true, W_hat, n, static_cast<float*>(ws), st));
  return QUIP_OK;
}

int64_t layer_x_chunk(int64_t N) {
  const int64_t c = (N + 3) / 4;
  return std::max<int64_t>(2048, (c + 2047) / 2048 * 2048);
}

// The device part of the layer from W, X on the device.  Two paths that
// meet before LDLQ: the Hessian path on the library's high-priority stream
// (draw V, H = X^T X / N, damping, H~, the LDL of H~) and the weight path
// on `st` (draw U, W~ = U W V^T, once V is drawn); then, on `st`, LDLQ and
// (W_hat non-NULL) W^.  x_ready, when given, is one event per token chunk
// of layer_x_chunk(N), waited for before that chunk is accumulated; w_ready
// is waited for before W is read; q_done is recorded once codes and grid
// are final.  Each path has its own workspace region.
quip_status layer_device(quip_transform* tf, uint64_t seed, const void* W, int w_dtype, int64_t ldw,
                         const void* X, int x_dtype, int64_t N, int64_t ldx, int bits, int64_t block,
                         float damp, uint8_t* codes, float* lo, float* scale, float* W_hat,
                         const LayerWs& L, char* ws, cudaStream_t st, const cudaEvent_t* x_ready,
                         cudaEvent_t w_ready, cudaEvent_t q_done, const cudaEvent_t* code_ev = nullptr,
                         int code_every = 1) {
  const int64_t m = tf->m, n = tf->n;
  float* H = reinterpret_cast<float*>(ws);
  float* D = reinterpret_cast<float*>(ws + L.H);
  float* Wt = reinterpret_cast<float*>(ws + L.H + L.D);
  void* sw = ws + L.H + L.D + L.Wt;
  void* sw2 = ws + L.H + L.D + L.Wt + L.stage;
  cudaStream_t hs = nullptr;
  QCHECK(hpath_stream(&hs));
  CallEvents evs(3);                                  // fork, V drawn, Hessian path done
  QCHECK(evs.create());
  cudaEvent_t* ev = evs.e.data();
  quip_status s = QUIP_OK;
  auto run = [&]() -> quip_status {
    quip_status r;
    QCHECK(cudaEventRecord(ev[0], st));
    QCHECK(cudaStreamWaitEvent(hs, ev[0], 0));
    // ---- Hessian path (hs)
    if ((r = draw_side(tf->side[1], seed, 1, hs)) != QUIP_OK) return r;
    QCHECK(cudaEventRecord(ev[1], hs));
    const size_t xes = x_dtype == QUIP_BF16 ? 2 : 4;
    if (x_ready) {
      const int64_t step = layer_x_chunk(N);
      int c = 0;
      for (int64_t a = 0; a < N; a += step, ++c) {
        QCHECK(cudaStreamWaitEvent(hs, x_ready[c], 0));
        const int64_t b = std::min(N, a + step);
        if ((r = quip_hessian_accumulate(static_cast<const char*>(X) + (size_t)a * ldx * xes, x_dtype, b - a, n,
                                         ldx, H, a > 0 ? 1 : 0, hs)) != QUIP_OK)
          return r;
      }
    } else if ((r = quip_hessian_accumulate(X, x_dtype, N, n, ldx, H, 0, hs)) != QUIP_OK) {
      return r;
    }
    if ((r = quip_hessian_finalize(H, n, N, damp, hs)) != QUIP_OK) return r;
    if ((r = quip_incoherence_forward(tf, nullptr, QUIP_F32, n, nullptr, H, sw, L.stage, hs)) != QUIP_OK) return r;
    // ---- weight path (st), enqueued before the LDL's many launches so that
    // its kernels start while the Hessian is accumulated
    if ((r = draw_side(tf->side[0], seed, 0, st)) != QUIP_OK) return r;
    if (w_ready) QCHECK(cudaStreamWaitEvent(st, w_ready, 0));
    QCHECK(cudaStreamWaitEvent(st, ev[1], 0));
    // W~, and LDLQ's grid and accumulator (they need W~ only): beside the
    // Hessian path.  A lives in the W path's region, after the transform's use.
    float* A = static_cast<float*>(sw2);
    if ((r = forward_w_ldlq_start(tf, W, w_dtype, ldw, Wt, bits, lo, scale, A, sw2, L.wstage, st)) != QUIP_OK)
      return r;
    // ---- Hessian path: the LDL of H~
    if ((r = quip_ldl(H, D, n, sw, L.stage, hs)) != QUIP_OK) return r;
    QCHECK(cudaEventRecord(ev[2], hs));
    // ---- both
    QCHECK(cudaStreamWaitEvent(st, ev[2], 0));
    if ((r = ldlq_main(Wt, H, n, m, n, bits, codes, lo, scale, A, sw, st, code_ev, code_every)) != QUIP_OK)
      return r;
    if (q_done) QCHECK(cudaEventRecord(q_done, st));
    if (W_hat) {
      if ((r = inverse_from_codes(tf, codes, lo, scale, W_hat, sw, L.stage, st)) != QUIP_OK) return r;
    }
    return QUIP_OK;
  };
  s = run();
  if (s != QUIP_OK) {
    // the caller's stream still waits for whatever was enqueued on hs
    cudaEventRecord(ev[2], hs);
    cudaStreamWaitEvent(st, ev[2], 0);
  }
  return s;
}
}  // namespace

extern "C" {

quip_status quip_layer_workspace_size(const quip_transform* tf, int64_t N, int w_dtype, int x_dtype,
                                      int64_t block, int host, size_t* bytes) {
  if (!tf || !bytes) return QUIP_ERR_ARG;
  *bytes = 0;
  LayerWs L;
  quip_status s = layer_ws(tf, N, w_dtype, x_dtype, block, host != 0, &L);
  if (s != QUIP_OK) return s;
  *bytes = L.total;
  return QUIP_OK;
}

quip_status quip_quantize_layer(quip_transform* tf, uint64_t seed, const void* W, int w_dtype, int64_t ldw,
                                const void* X, int x_dtype, int64_t N, int64_t ldx, int bits, int64_t block,
                                float damp, uint8_t* codes, float* lo, float* scale, float* W_hat, void* ws,
                                size_t ws_bytes, void* stream) {
  quip_status s = layer_args(tf, w_dtype, ldw, x_dtype, N, ldx, bits, block, damp);
  if (s != QUIP_OK) return s;
  if (!W || !X || !codes || !lo || !scale) return QUIP_ERR_ARG;
  LayerWs L;
  if ((s = layer_ws(tf, N, w_dtype, x_dtype, block, false, &L)) != QUIP_OK) return s;
  if ((s = check_ws(ws, ws_bytes, L.total)) != QUIP_OK) return s;
  return layer_device(tf, seed, W, w_dtype, ldw, X, x_dtype, N, ldx, bits, block, damp, codes, lo, scale, W_hat,
                      L, static_cast<char*>(ws), S(stream), nullptr, nullptr, nullptr);
}

quip_status quip_quantize_layer_host(quip_transform* tf, uint64_t seed, const void* W_host, int w_dtype,
                                     int64_t ldw, const void* X_host, int x_dtype, int64_t N, int64_t ldx,
                                     int bits, int64_t block, float damp, uint8_t* codes_host, float* lo_host,
                                     float* scale_host, float* W_hat_host, void* ws, size_t ws_bytes,
                                     void* stream) {
  quip_status s = layer_args(tf, w_dtype, ldw, x_dtype, N, ldx, bits, block, damp);
  if (s != QUIP_OK) return s;
  if (!W_host || !X_host || !codes_host || !lo_host || !scale_host) return QUIP_ERR_ARG;
  LayerWs L;
  if ((s = layer_ws(tf, N, w_dtype, x_dtype, block, true, &L)) != QUIP_OK) return s;
  if ((s = check_ws(ws, ws_bytes, L.total)) != QUIP_OK) return s;
  const int64_t m = tf->m, n = tf->n;
  const size_t wes = w_dtype == QUIP_BF16 ? 2 : 4, xes = x_dtype == QUIP_BF16 ? 2 : 4;
  char* Wd = static_cast<char*>(ws) + L.H + L.D + L.Wt + L.stage + L.wstage;
  char* Xd = Wd + L.Wd;
  uint8_t* codes = reinterpret_cast<uint8_t*>(Xd + L.Xd);
  float* lo = reinterpret_cast<float*>(reinterpret_cast<char*>(codes) + L.codes);
  float* sc = reinterpret_cast<float*>(reinterpret_cast<char*>(lo) + L.lo);
  float* What = reinterpret_cast<float*>(reinterpret_cast<char*>(sc) + L.sc);
  cudaStream_t st = S(stream), cp = nullptr;
  QCHECK(copy_stream(&cp));
  const int64_t step = layer_x_chunk(N);
  const int nch = (int)((N + step - 1) / step);
  // the codes go back in about eight column chunks, each as soon as LDLQ's
  // block kernels have finished its columns (they run in column order)
  const int64_t nblk = (n + LQB_BLOCK_COLS - 1) / LQB_BLOCK_COLS;
  const int every = (int)std::max<int64_t>(1, (nblk + 7) / 8);
  const int ncc = (int)((nblk + every - 1) / every);
  CallEvents evs((size_t)(nch + 4 + ncc));
  QCHECK(evs.create());
  std::vector<cudaEvent_t>& ev = evs.e;
  cudaEvent_t fork = ev[nch], w_ready = ev[nch + 1], q_done = ev[nch + 2], out_done = ev[nch + 3];
  const cudaEvent_t* code_ev = ev.data() + nch + 4;
  // the copies start after earlier work on the caller's stream, which may
  // still be reading this workspace
  QCHECK(cudaEventRecord(fork, st));
  QCHECK(cudaStreamWaitEvent(cp, fork, 0));
  int c = 0;
  for (int64_t a = 0; a < N; a += step, ++c) {
    const int64_t b = std::min(N, a + step);
    QCHECK(cudaMemcpy2DAsync(Xd + (size_t)a * n * xes, (size_t)n * xes,
                             static_cast<const char*>(X_host) + (size_t)a * ldx * xes, (size_t)ldx * xes,
                             (size_t)n * xes, (size_t)(b - a), cudaMemcpyHostToDevice, cp));
    QCHECK(cudaEventRecord(ev[c], cp));
  }
  QCHECK(cudaMemcpy2DAsync(Wd, (size_t)n * wes, W_host, (size_t)ldw * wes, (size_t)n * wes, (size_t)m,
                           cudaMemcpyHostToDevice, cp));
  QCHECK(cudaEventRecord(w_ready, cp));
  s = layer_device(tf, seed, Wd, w_dtype, n, Xd, x_dtype, N, n, bits, block, damp, codes, lo, sc, What, L,
                   static_cast<char*>(ws), st, ev.data(), w_ready, q_done, code_ev, every);
  if (s == QUIP_OK) {
    // the codes go back while LDLQ runs, one column chunk (all rows, a 2-D
    // copy) per event; the grid once LDLQ is done; W^ after it
    for (int c = 0; c < ncc; ++c) {
      const int64_t c0 = (int64_t)c * every * LQB_BLOCK_COLS, c1 = std::min(n, c0 + every * LQB_BLOCK_COLS);
      QCHECK(cudaStreamWaitEvent(cp, code_ev[c], 0));
      QCHECK(cudaMemcpy2DAsync(codes_host + c0, (size_t)n, codes + c0, (size_t)n, (size_t)(c1 - c0), (size_t)m,
                               cudaMemcpyDeviceToHost, cp));
    }
    QCHECK(cudaStreamWaitEvent(cp, q_done, 0));
    QCHECK(cudaMemcpyAsync(lo_host, lo, (size_t)m * 4, cudaMemcpyDeviceToHost, cp));
    QCHECK(cudaMemcpyAsync(scale_host, sc, (size_t)m * 4, cudaMemcpyDeviceToHost, cp));
    if (W_hat_host) QCHECK(cudaMemcpyAsync(W_hat_host, What, (size_t)m * n * 4, cudaMemcpyDeviceToHost, st));
  }
  // the caller's stream covers every copy: it waits for the copy stream
  QCHECK(cudaEventRecord(out_done, cp));
  QCHECK(cudaStreamWaitEvent(st, out_done, 0));
  return s;
}

}  // extern "C"

quip_status quip_timing_begin(void) {
  std::lock_guard<std::mutex> lk(g_timing_mu);
  for (const TimingRec& r : g_timing_recs) g_timing_pool.push_back({r.a, r.b});
  g_timing_recs.clear();
  g_timing_on.store(true);
  return QUIP_OK;
}

quip_status quip_timing_end(const char** names, uint64_t* launches, double* total_ms,
                            int max_entries, int* n_entries) {
  g_timing_on.store(false);
  std::lock_guard<std::mutex> lk(g_timing_mu);
  struct Agg {
    const char* name;
    uint64_t count;
    double ms;
  };
  std::vector<Agg> agg;
  quip_status st = QUIP_OK;
  for (const TimingRec& r : g_timing_recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
      st = QUIP_ERR_CUDA;
      continue;
    }
    size_t i = 0;
    while (i < agg.size() && std::strcmp(agg[i].name, r.name) != 0) ++i;
    if (i == agg.size()) agg.push_back({r.name, 0, 0.0});
    agg[i].count += 1;
    agg[i].ms += ms;
  }
  for (const TimingRec& r : g_timing_recs) g_timing_pool.push_back({r.a, r.b});
  g_timing_recs.clear();
  std::sort(agg.begin(), agg.end(), [](const Agg& x, const Agg& y) { return x.ms > y.ms; });
  if (n_entries) *n_entries = (int)agg.size();
  for (int i = 0; i < max_entries && i < (int)agg.size(); ++i) {
    if (names) names[i] = agg[i].name;
    if (launches) launches[i] = agg[i].count;
    if (total_ms) total_ms[i] = agg[i].ms;
  }
  return st;
}

quip_status quip_timing_trace(const char** names, double* start_ms, double* end_ms, int* stream_ids,
                              int max_entries, int* n_entries) {
  g_timing_on.store(false);
  std::lock_guard<std::mutex> lk(g_timing_mu);
  quip_status st = QUIP_OK;
  std::vector<cudaStream_t> streams;
  const int nrec = (int)g_timing_recs.size();
  if (n_entries) *n_entries = nrec;
  for (int i = 0; i < nrec && i < max_entries; ++i) {
    const TimingRec& r = g_timing_recs[i];
    float t0 = 0.f, t1 = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess ||
        cudaEventElapsedTime(&t0, g_timing_recs[0].a, r.a) != cudaSuccess ||
        cudaEventElapsedTime(&t1, g_timing_recs[0].a, r.b) != cudaSuccess) {
      st = QUIP_ERR_CUDA;
      continue;
    }
    size_t k = 0;
    while (k < streams.size() && streams[k] != r.st) ++k;
    if (k == streams.size()) streams.push_back(r.st);
    if (names) names[i] = r.name;
    if (start_ms) start_ms[i] = t0;
    if (end_ms) end_ms[i] = t1;
    if (stream_ids) stream_ids[i] = (int)k;
  }
  for (const TimingRec& r : g_timing_recs) g_timing_pool.push_back({r.a, r.b});
  g_timing_recs.clear();
  return st;
}

quip_status quip_sync_status(void* stream) {
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return QUIP_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return QUIP_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return QUIP_ERR_CUDA;
  return static_cast<quip_status>(v);
}

}  // extern "C"
