// Host launcher of the tcgen05 GEMM family and the tensor-map / status helpers.
#include <cstdlib>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <string>

#include "gemm.cuh"
#include "host.cuh"

namespace gptk {

// ------------------------------------------------------------ error string

static thread_local std::string g_last_error;

int set_error(int code, const std::string& msg) {
  g_last_error = msg;
  return code;
}
const char* last_error() { return g_last_error.c_str(); }

// ------------------------------------------------------------ device status word

// One status word per device, in a __device__ variable: the library allocates nothing.
__device__ unsigned int g_dev_status[4];
static unsigned int* g_status[64];
static std::once_flag g_status_once[64];
static unsigned long long g_timeout_ns = 2000000000ull;  // 2 s per wait

DevCtl device_ctl() {
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(g_status_once[dev & 63], [dev]() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_status) == cudaSuccess) g_status[dev & 63] = static_cast<unsigned int*>(p);
  });
  DevCtl c;
  c.status = g_status[dev & 63];
  c.timeout_ns = g_timeout_ns;
  return c;
}

void set_wait_timeout_ns(unsigned long long ns) { g_timeout_ns = ns; }

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (cached[dev & 63] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev & 63] = n > 0 ? n : 148;
  }
  return cached[dev & 63];
}

// ------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int make_tmap_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t ld,
                 uint32_t box_inner, uint32_t box_outer, int esize) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return set_error(ST_CUDA, "cuTensorMapEncodeTiled is not available");
  if ((reinterpret_cast<uintptr_t>(base) & 15) || ((ld * esize) & 15))
    return set_error(ST_INVALID_ARG, "tensor base must be 16-byte aligned and its pitch a multiple of 16 bytes");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * (uint64_t)esize};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  const CUtensorMapDataType dt = esize == 4   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : esize == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                              : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(ST_CUDA, "cuTensorMapEncodeTiled (2d) failed: " + std::to_string((int)r));
  return ST_OK;
}

int make_tmap_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                 uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return set_error(ST_CUDA, "cuTensorMapEncodeTiled is not available");
  if ((reinterpret_cast<uintptr_t>(base) & 15) || ((s1 * 2) & 15) || ((s2 * 2) & 15))
    return set_error(ST_INVALID_ARG, "tensor base must be 16-byte aligned and its pitches multiples of 16 bytes");
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1 * 2, s2 * 2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(ST_CUDA, "cuTensorMapEncodeTiled (3d) failed: " + std::to_string((int)r));
  return ST_OK;
}

// ------------------------------------------------------------ GEMM launcher

template <int BN, int EPI, bool LONGK, bool PAIR, bool F8 = false>
static int launch_gemm_t(const GemmMaps& maps, const GemmParams& p, cudaStream_t st) {
  using C = GemmCfg<BN, LONGK, PAIR>;
  auto kern = gemm_kernel<BN, EPI, LONGK, PAIR, F8>;
  static bool attr_set[64] = {false};
  static int max_pairs[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set[dev & 63]) {
    GPTK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    if (PAIR) {
      // how many CTA pairs fit at once (an SM whose GPC has no free partner SM stays out)
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
      cfg.blockDim = dim3(C::THREADS, 1, 1);
      cfg.dynamicSmemBytes = C::SMEM;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      GPTK_CUDA(cudaOccupancyMaxActiveClusters(&n, kern, &cfg));
      if (n < 1) return set_error(ST_UNSUPPORTED, "GEMM: no CTA pair fits on this device");
      max_pairs[dev & 63] = n;
    }
    attr_set[dev & 63] = true;
  }
  const int tiles = p.tile_start[p.n_prob];
  int grid = PAIR ? max_pairs[dev & 63] : num_sms();
  if (grid > tiles) grid = tiles;
  double flops = 0, bytes = 0;
  for (int q = 0; q < p.n_prob; ++q) {
    const double M = p.pM[q], N = p.pN[q], K = p.pK[q] > 0 ? p.pK[q] : p.K;
    double out_bytes = M * N * 2;
    if (EPI == EPI_F32 || EPI == EPI_RESID) out_bytes = M * N * 4 * (1 + (p.accumulate || EPI == EPI_RESID));
    if (EPI == EPI_UP) out_bytes = M * N * (p.out ? 4 : 2);
    if (EPI == EPI_ACTBWD) out_bytes = M * N * 4;
    if (EPI == EPI_CE_FWD) out_bytes = M * p.tiles_n * 8;
    flops += 2.0 * (p.pelems[q] > 0 ? p.pelems[q] : M * N) * K;
    bytes += (M * K + N * K) * (F8 ? 1 : 2) + out_bytes;
  }
  Prof prof(p.prof_kind > 0 ? p.prof_kind : PK_GEMM, flops, bytes, st);
  if (PAIR) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_pdl
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(2 * grid, 1, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    GPTK_CUDA(cudaLaunchKernelEx(&cfg, kern, maps, p));
  } else {
    GPTK_CUDA(launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM, st, maps, p));
  }
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

template <int BN, bool PAIR>
static int dispatch_epi(int epi, const GemmMaps& maps, const GemmParams& p, cudaStream_t st) {
  // reductions over all tokens (weight gradients) and over the vocabulary take the deep ring
  if (epi == EPI_F32 && p.K >= 8192) return launch_gemm_t<BN, EPI_F32, true, PAIR>(maps, p, st);
  switch (epi) {
    case EPI_BF16: return launch_gemm_t<BN, EPI_BF16, false, PAIR>(maps, p, st);
    case EPI_F32: return launch_gemm_t<BN, EPI_F32, false, PAIR>(maps, p, st);
    case EPI_RESID: return launch_gemm_t<BN, EPI_RESID, false, PAIR>(maps, p, st);
    case EPI_QKV:
      if (BN != 256 || !p.tma_out || p.qk_D % 256 != 0)
        return set_error(ST_UNSUPPORTED, "fused RoPE/QK-norm epilogue needs 256-column tiles over whole heads");
      return launch_gemm_t<BN, EPI_QKV, false, PAIR>(maps, p, st);
    case EPI_UP: return launch_gemm_t<BN, EPI_UP, false, PAIR>(maps, p, st);
    case EPI_ACTBWD: return launch_gemm_t<BN, EPI_ACTBWD, false, PAIR>(maps, p, st);
    case EPI_CE_FWD: return launch_gemm_t<BN, EPI_CE_FWD, false, PAIR>(maps, p, st);
    case EPI_CE_BWD: return launch_gemm_t<BN, EPI_CE_BWD, false, PAIR>(maps, p, st);
  }
  return set_error(ST_INVALID_ARG, "unknown GEMM epilogue");
}

template <int BN, bool PAIR>
static int dispatch_epi_f8(int epi, const GemmMaps& maps, const GemmParams& p, cudaStream_t st) {
  switch (epi) {
    case EPI_BF16: return launch_gemm_t<BN, EPI_BF16, false, PAIR, true>(maps, p, st);
    case EPI_F32: return launch_gemm_t<BN, EPI_F32, false, PAIR, true>(maps, p, st);
    case EPI_RESID: return launch_gemm_t<BN, EPI_RESID, false, PAIR, true>(maps, p, st);
    case EPI_QKV:
      if (BN != 256 || !p.tma_out || p.qk_D % 256 != 0)
        return set_error(ST_UNSUPPORTED, "fused RoPE/QK-norm epilogue needs 256-column tiles over whole heads");
      return launch_gemm_t<BN, EPI_QKV, false, PAIR, true>(maps, p, st);
    case EPI_UP: return launch_gemm_t<BN, EPI_UP, false, PAIR, true>(maps, p, st);
  }
  return set_error(ST_INVALID_ARG, "GEMM: this epilogue has no 8-bit operand variant");
}

static int dispatch(int epi, int bn, bool pair, const GemmMaps& maps, const GemmParams& p, cudaStream_t st) {
  if (p.f8_inv_a) {
    if (pair) return dispatch_epi_f8<256, true>(epi, maps, p, st);
    return bn == 256 ? dispatch_epi_f8<256, false>(epi, maps, p, st) : dispatch_epi_f8<128, false>(epi, maps, p, st);
  }
  if (pair) return dispatch_epi<256, true>(epi, maps, p, st);
  return bn == 256 ? dispatch_epi<256, false>(epi, maps, p, st) : dispatch_epi<128, false>(epi, maps, p, st);
}

// CTA pairs (256-row tiles) for N-256 tiles when the 256-row tiles still give every pair of SMs
// at least one tile; GPT_GEMM_PAIR=0 / 1 forces the choice (tuning and comparison).
static bool use_pair(int bn, long long tiles256) {
  static const int forced = []() {
    const char* e = std::getenv("GPT_GEMM_PAIR");
    return e ? std::atoi(e) : -1;
  }();
  if (bn != 256 || forced == 0) return false;
  if (forced == 1) return true;
  return tiles256 >= num_sms() / 2;
}

static bool aligned16(const void* ptr, long long ld, int esize) {
  return ptr != nullptr && (reinterpret_cast<uintptr_t>(ptr) & 15) == 0 && ((ld * esize) & 15) == 0;
}

// b_rows: B rows one CTA stages per K step (the tile's N, or half of it for CTA pairs).  8-bit
// operands (f8) are K-major only, with 128-element (128-byte) boxes along K.
static int operand_maps(const Operand& A, const Operand& B, int M, int N, int K, int b_rows, CUtensorMap* ta,
                        CUtensorMap* tb, bool f8 = false) {
  if (f8) {
    if (A.mn_major || B.mn_major) return set_error(ST_UNSUPPORTED, "GEMM: 8-bit operands must be K-major");
    GPTK_TRY(make_tmap_2d(ta, A.ptr, K, M, A.ld, 128, 128, 1));
    return make_tmap_2d(tb, B.ptr, K, N, B.ld, 128, b_rows, 1);
  }
  if (!A.mn_major) {
    GPTK_TRY(make_tmap_2d(ta, A.ptr, K, M, A.ld, 64, 128));
  } else {
    GPTK_TRY(make_tmap_2d(ta, A.ptr, M, K, A.ld, 64, 64));
  }
  if (!B.mn_major) {
    GPTK_TRY(make_tmap_2d(tb, B.ptr, K, N, B.ld, 64, b_rows));
  } else {
    GPTK_TRY(make_tmap_2d(tb, B.ptr, N, K, B.ld, 64, 64));
  }
  return ST_OK;
}

// band height: a few m-tiles whose A rows (tile_m x K bf16 each) stay within about 48 MB of L2
static int band_height(int tiles_m, int K, int tile_m) {
  const long long a_band_row = (long long)tile_m * K * 2;
  int gm = 8;  // measured best among 8, 16, 32 and the plain order on B200 (d20 shapes)
  const int gm_l2 = (int)((48LL << 20) / (a_band_row > 0 ? a_band_row : 1));
  if (gm > gm_l2) gm = gm_l2;
  // very long K (weight gradients): bands would be too thin to help; keep the plain order,
  // whose concurrent tiles share B columns while moving through K in step
  if (gm < 8) gm = tiles_m;
  // tuning override: GPT_GEMM_GROUP_M=<n> forces the band height (0 = plain order)
  static const int forced = []() {
    const char* e = std::getenv("GPT_GEMM_GROUP_M");
    return e ? std::atoi(e) : -1;
  }();
  if (forced == 0) gm = tiles_m;
  if (forced > 0) gm = forced < tiles_m ? forced : tiles_m;
  if (gm > tiles_m) gm = tiles_m;
  return gm < 1 ? 1 : gm;
}

int run_gemm(int epi, int bn, const Operand& A, const Operand& B, GemmParams& p, cudaStream_t st) {
  if (bn != 128 && bn != 256) return set_error(ST_INVALID_ARG, "GEMM tile N must be 128 or 256");
  if (p.M <= 0 || p.N <= 0 || p.K <= 0) return set_error(ST_INVALID_ARG, "GEMM with an empty dimension");
  GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const bool pair = use_pair(bn, (long long)((p.M + 255) / 256) * ((p.N + 255) / 256));
  const int tile_m = pair ? 256 : 128;
  const bool f8 = p.f8_inv_a != nullptr;
  if (f8 && (!p.f8_inv_b || p.f8_fmt_a < 0 || p.f8_fmt_a > 1 || p.f8_fmt_b < 0 || p.f8_fmt_b > 1))
    return set_error(ST_INVALID_ARG, "GEMM: 8-bit operands need both inverse scales and formats 0 (e4m3) / 1 (e5m2)");
  GPTK_TRY(operand_maps(A, B, p.M, p.N, p.K, pair ? bn / 2 : bn, &maps.a[0], &maps.b[0], f8));
  // output / input tensor maps of the TMA epilogue, where the layout allows one
  p.tma_out = 0;
  const bool f32out = (epi == EPI_F32 || epi == EPI_RESID);
  const int es = f32out ? 4 : 2;
  const unsigned bw = f32out ? 32 : 64;
  bool ok = epi != EPI_CE_FWD && (epi == EPI_UP ? (p.out == nullptr || aligned16(p.out, p.ldo, 2))
                                                  : aligned16(p.out, p.ldo, es)) &&
            (epi != EPI_BF16 || p.hd == p.hdp);
  if (ok && epi == EPI_RESID) ok = aligned16(p.resid, p.ldr, 4);
  if (ok && epi == EPI_UP) ok = aligned16(p.out2, p.ldo, 2);
  if (ok && epi == EPI_ACTBWD) ok = aligned16(p.aux, p.ld_aux, 2);
  if (ok) {
    if (p.out) GPTK_TRY(make_tmap_2d(&maps.c[0], p.out, p.N, p.M, p.ldo, bw, 32, es));
    if (epi == EPI_UP) GPTK_TRY(make_tmap_2d(&maps.c2, p.out2, p.N, p.M, p.ldo, 64, 32, 2));
    if (epi == EPI_RESID) GPTK_TRY(make_tmap_2d(&maps.r, p.resid, p.N, p.M, p.ldr, 32, 32, 4));
    if (epi == EPI_ACTBWD) GPTK_TRY(make_tmap_2d(&maps.r, p.aux, p.N, p.M, p.ld_aux, 64, 32, 2));
    p.tma_out = 1;
  }
  if (p.amax_h != nullptr && (epi != EPI_UP || !p.tma_out))
    return set_error(ST_UNSUPPORTED, "GEMM: max |h| is folded only by the MLP-up epilogue's TMA path");
  p.a_mn = A.mn_major;
  p.b_mn = B.mn_major;
  p.tiles_m = (p.M + tile_m - 1) / tile_m;
  p.tiles_n = (p.N + bn - 1) / bn;
  p.group_m = band_height(p.tiles_m, p.K, tile_m);
  p.n_prob = 1;
  p.tile_start[0] = 0;
  p.tile_start[1] = p.tiles_m * p.tiles_n;
  p.pM[0] = p.M;
  p.pN[0] = p.N;
  p.ptiles_m[0] = p.tiles_m;
  p.ptiles_n[0] = p.tiles_n;
  p.pgroup_m[0] = p.group_m;
  p.tile_rows = tile_m;
  p.tile_cols = bn;
  p.ctl = device_ctl();
  if (p.ctl.status == nullptr) return set_error(ST_CUDA, "device status word unavailable");
  return dispatch(epi, bn, pair, maps, p, st);
}

static int run_gemm_group_impl(int n, const GroupProblem* probs, int K, int a_mn, int b_mn, int bn, int prof_kind,
                               cudaStream_t st, int epi, int accumulate, const void* c, long long ldc,
                               long long c_rows, const int* c_row, float alpha, float beta);

int run_gemm_group(int n, const GroupProblem* probs, int K, int a_mn, int b_mn, int bn, int prof_kind,
                   cudaStream_t st, int epi, int accumulate) {
  return run_gemm_group_impl(n, probs, K, a_mn, b_mn, bn, prof_kind, st, epi, accumulate, nullptr, 0, 0, nullptr, 0.f,
                             0.f);
}

int run_gemm_group_axpby(int n, const GroupProblem* probs, int K, int a_mn, int b_mn, int prof_kind, const void* c,
                         long long ldc, long long c_rows, const int* c_row, float alpha, float beta, cudaStream_t st) {
  if (!c || !c_row) return set_error(ST_INVALID_ARG, "grouped GEMM: linear epilogue without its addend");
  return run_gemm_group_impl(n, probs, K, a_mn, b_mn, 256, prof_kind, st, EPI_ACTBWD, 0, c, ldc, c_rows, c_row,
                             alpha, beta);
}

static int run_gemm_group_impl(int n, const GroupProblem* probs, int K, int a_mn, int b_mn, int bn, int prof_kind,
                               cudaStream_t st, int epi, int accumulate, const void* c, long long ldc,
                               long long c_rows, const int* c_row, float alpha, float beta) {
  if (n < 1 || n > kMaxProblems) return set_error(ST_INVALID_ARG, "grouped GEMM: 1 to 8 problems");
  if (bn != 128 && bn != 256) return set_error(ST_INVALID_ARG, "GEMM tile N must be 128 or 256");
  if (!(epi == EPI_F32 || ((epi == EPI_BF16 || epi == EPI_ACTBWD) && !accumulate)))
    return set_error(ST_INVALID_ARG, "grouped GEMM: fp32 (stored or accumulated) or bf16 (stored) outputs");
  const int es = epi == EPI_F32 ? 4 : 2;
  GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.K = K;
  p.a_mn = a_mn;
  p.b_mn = b_mn;
  p.accumulate = accumulate;
  p.hd = p.hdp = 1;
  p.tma_out = 1;
  p.prof_kind = prof_kind;
  p.n_prob = n;
  long long tiles256 = 0;
  for (int q = 0; q < n; ++q) tiles256 += (long long)((probs[q].M + 255) / 256) * ((probs[q].N + 255) / 256);
  const bool pair = use_pair(bn, tiles256);
  const int tile_m = pair ? 256 : 128;
  int start = 0;
  for (int q = 0; q < n; ++q) {
    const GroupProblem& g = probs[q];
    if (g.M <= 0 || g.N <= 0 || g.K_ext < 0 || g.K_ext > K || !aligned16(g.out, g.ldo, es))
      return set_error(ST_INVALID_ARG, "grouped GEMM: bad problem");
    const int kq = g.K_ext > 0 ? g.K_ext : K;
    GPTK_TRY(operand_maps(Operand{g.a, g.lda, a_mn}, Operand{g.b, g.ldb, b_mn}, g.M, g.N, kq, pair ? bn / 2 : bn,
                          &maps.a[q], &maps.b[q]));
    p.pK[q] = kq;
    GPTK_TRY(make_tmap_2d(&maps.c[q], g.out, g.N, g.M, g.ldo, es == 4 ? 32 : 64, 32, es));
    p.pM[q] = g.M;
    p.pN[q] = g.N;
    p.ptiles_m[q] = (g.M + tile_m - 1) / tile_m;
    p.ptiles_n[q] = (g.N + bn - 1) / bn;
    p.pgroup_m[q] = band_height(p.ptiles_m[q], K, tile_m);
    p.tile_start[q] = start;
    if (g.upper) {
      if (g.M != g.N) return set_error(ST_INVALID_ARG, "grouped GEMM: an upper-triangle product must be square");
      // m-tile tm meets the upper triangle from n-tile tm * tile_m / bn on (tile_info's walk)
      p.ptri[q] = 1;
      double elems = 0;
      for (int tm = 0; tm < p.ptiles_m[q]; ++tm) {
        const int rows = std::min(tile_m, g.M - tm * tile_m);
        for (int tn = tm * tile_m / bn; tn < p.ptiles_n[q]; ++tn) {
          elems += (double)rows * std::min(bn, g.N - tn * bn);
          ++start;
        }
      }
      p.pelems[q] = elems;
    } else {
      start += p.ptiles_m[q] * p.ptiles_n[q];
    }
  }
  p.tile_rows = tile_m;
  p.tile_cols = bn;
  p.tile_start[n] = start;
  if (epi == EPI_ACTBWD) {  // the linear epilogue's addend: one stacked bf16 matrix, a row block per problem
    if (!aligned16(c, ldc, 2)) return set_error(ST_INVALID_ARG, "grouped GEMM: addend alignment");
    GPTK_TRY(make_tmap_2d(&maps.r, c, probs[0].N, c_rows, ldc, 64, 32, 2));
    for (int q = 0; q < n; ++q) p.prow[q] = c_row[q];
    p.act = 3;
    p.ax_alpha = alpha;
    p.ax_beta = beta;
  }
  p.M = p.pM[0];
  p.N = p.pN[0];
  p.tiles_m = p.ptiles_m[0];
  p.tiles_n = p.ptiles_n[0];
  p.group_m = p.pgroup_m[0];
  p.ctl = device_ctl();
  if (p.ctl.status == nullptr) return set_error(ST_CUDA, "device status word unavailable");
  return dispatch(epi, bn, pair, maps, p, st);
}

}  // namespace gptk
