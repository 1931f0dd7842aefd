// Host-side helpers shared by the launchers: error plumbing, tensor-map
// encoding, device properties.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <string>
#include <utility>

#include "ptx.cuh"

namespace gptk {

// status codes of the C ABI (mirrored in include/gpt.h)
enum : int {
  ST_OK = 0,
  ST_INVALID_ARG = 1,
  ST_UNSUPPORTED = 2,
  ST_WORKSPACE_TOO_SMALL = 3,
  ST_CUDA = 4,
  ST_DEVICE_TIMEOUT = 5,
};

// Records a message for gpt_last_error() (thread-local) and returns the code.
int set_error(int code, const std::string& msg);
const char* last_error();

// CUDA runtime check: records the call site and returns ST_CUDA on failure.
#define GPTK_CUDA(call)                                                                        \
  do {                                                                                         \
    cudaError_t e_ = (call);                                                                   \
    if (e_ != cudaSuccess)                                                                     \
      return ::gptk::set_error(::gptk::ST_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
  } while (0)

#define GPTK_TRY(expr)        \
  do {                        \
    int rc_ = (expr);         \
    if (rc_ != 0) return rc_; \
  } while (0)

// The device status word and wait limit used by every kernel launched on this device.
DevCtl device_ctl();
int num_sms();

// 2-D tensor map with 128-byte swizzle: inner extent `inner` (contiguous), outer
// extent `outer`, row pitch `ld` elements, box {box_inner, box_outer}; elements are
// bf16 (esize 2) or fp32 (esize 4).
int make_tmap_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t ld,
                 uint32_t box_inner, uint32_t box_outer, int esize = 2);
// 3-D bf16 tensor map: dims {d0 (contiguous), d1, d2}, pitches (elements) s1, s2, box {b0, b1, b2}.
int make_tmap_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                 uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2);

// One GEMM operand in global memory.  For a K-major operand `ld` is the pitch
// between consecutive M (or N) rows; for an MN-major operand it is the pitch
// between consecutive K rows.
struct Operand {
  const void* ptr;
  long long ld;
  int mn_major;
};

// ---- launch accounting and optional per-launch timing
// Every kernel launch site constructs a Prof scope: it counts the launch and, while
// profiling is on, brackets it with CUDA events on the launching stream together with
// the launch's algorithmic FLOPs and bytes.
enum ProfKind : int {
  PK_GEMM = 0, PK_ATTN_FWD, PK_ATTN_BWD_DKV, PK_ATTN_BWD_DQ, PK_NORM_FWD, PK_NORM_BWD, PK_EMBED_FWD,
  PK_EMBED_BWD, PK_CAST, PK_CE_COMBINE, PK_LOSS, PK_QK, PK_DELTA, PK_COLSUM, PK_MISC,
  // GEMM roles (the model tags each GEMM call; untagged calls count as PK_GEMM)
  PK_GEMM_QKV, PK_GEMM_O, PK_GEMM_UP, PK_GEMM_DOWN, PK_GEMM_LM_FWD, PK_GEMM_LM_BWD, PK_GEMM_DGRAD,
  PK_GEMM_WGRAD,
  PK_OPTIM,  // optimizer elementwise steps (gradient norm, AdamW update, Muon momentum and updates)
  PK_GEMM_MUON,  // the Newton-Schulz products of the Muon step
  PK_COUNT
};
class Prof {
 public:
  Prof(int kind, double flops, double bytes, cudaStream_t st);
  ~Prof();
 private:
  int idx_;
  cudaStream_t st_;
};

struct GemmParams;
// C[M,N] = A[M,K] B[N,K]^T with the fused epilogue `epi`; bn = 128 or 256.
int run_gemm(int epi, int bn, const Operand& A, const Operand& B, GemmParams& p, cudaStream_t st);

// One product of a grouped launch: out[M,N] (+)= A B^T (fp32, or bf16 when stored).  K_ext, when
// > 0, is the K extent this problem's operands really have (at most the launch's K): its
// tensor maps end there and the rest of the launch's K loop reads zeros, so one launch can
// hold the pieces of a split reduction whose last piece is shorter.
struct GroupProblem {
  const void* a;
  long long lda;
  const void* b;
  long long ldb;
  int M, N;
  void* out;
  long long ldo;
  int K_ext;
  // 1: the product is symmetric (M == N, e.g. X X^T); only the tiles that meet the upper
  // triangle (row <= column) are computed, the rest of out is left as it is
  int upper;
};
// Up to 8 products with the same K and operand layouts in one persistent launch (their tiles
// share one schedule, so small products do not leave SMs idle): fp32 outputs accumulated
// (epi EPI_F32, accumulate 1, the default) or stored (accumulate 0), or bf16 outputs stored
// (epi EPI_BF16).
int run_gemm_group(int n, const GroupProblem* probs, int K, int a_mn, int b_mn, int bn, int prof_kind,
                   cudaStream_t st, int epi = 1, int accumulate = 1);
// Grouped bf16 products with a linear epilogue: out_q = alpha (A_q B_q^T) + beta C_q, where the
// C_q are the row blocks of one stacked bf16 matrix c (problem q's rows start at c_row[q], pitch
// ldc); used where every product has its own addend of its own output's shape.
int run_gemm_group_axpby(int n, const GroupProblem* probs, int K, int a_mn, int b_mn, int prof_kind, const void* c,
                         long long ldc, long long c_rows, const int* c_row, float alpha, float beta, cudaStream_t st);

// Launch with programmatic stream serialization: the kernel may be scheduled while the previous
// kernel on the stream finishes (it must run pdl_wait() before touching global memory).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace gptk
