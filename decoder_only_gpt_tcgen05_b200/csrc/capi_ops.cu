// C ABI of the op-level entry points (include/gpt_ops.h).
#include <algorithm>
#include <string>

#include "gemm.cuh"
#include "gpt_ops.h"
#include "host.cuh"
#include "kernels.cuh"

using namespace gptk;

namespace gptk {
// Waits on an mbarrier that nothing arrives at, through the same bounded wait as every
// pipeline kernel: after ctl.timeout_ns it records DEV_ERR_TIMEOUT and returns.
__global__ void wait_probe_kernel(DevCtl ctl) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, ctl, &abort_flag, 99);
}

// The attention forward's two exponentials, element pairs (x[2i], x[2i+1]) -> out
__global__ void exp2_pair_kernel(const float* __restrict__ x, long long n_pairs, int poly, float* __restrict__ out) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_pairs; i += (long long)gridDim.x * blockDim.x) {
    const float2 v = reinterpret_cast<const float2*>(x)[i];
    reinterpret_cast<float2*>(out)[i] = poly ? exp2_poly2(v) : make_float2(ex2_approx(v.x), ex2_approx(v.y));
  }
}
}  // namespace gptk

extern "C" {

GPT_API int gpt_op_wait_probe(unsigned long long timeout_ns, void* stream) {
  set_error(ST_OK, "");
  if (timeout_ns == 0 || timeout_ns > 10000000000ull)
    return set_error(ST_INVALID_ARG, "wait_probe: timeout must be in (0, 10 s]");
  DevCtl ctl = device_ctl();
  if (!ctl.status) return set_error(ST_CUDA, "device status word unavailable");
  ctl.timeout_ns = timeout_ns;
  Prof prof(PK_MISC, 0, 0, static_cast<cudaStream_t>(stream));
  wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ctl);
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

GPT_API int gpt_op_exp2(const float* x, long long n, int poly, float* out, void* stream) {
  set_error(ST_OK, "");
  if (n < 0 || (n & 1)) return set_error(ST_INVALID_ARG, "exp2: n must be even and >= 0");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out)) & 7)
    return set_error(ST_INVALID_ARG, "exp2: x and out must be 8-byte aligned");
  if (n == 0) return ST_OK;
  Prof prof(PK_MISC, 0, 8.0 * n, static_cast<cudaStream_t>(stream));
  const long long pairs = n / 2;
  const int grid = static_cast<int>(std::min<long long>((pairs + 255) / 256, 4096));
  exp2_pair_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, pairs, poly, out);
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

GPT_API const char* gpt_last_error(void) { return last_error(); }

GPT_API int gpt_op_gemm(int epilogue, int bn, const void* a, long long lda, int a_mn, const void* b, long long ldb,
                        int b_mn, int M, int N, int K, void* out, long long ldo, const float* bias, int accumulate,
                        void* stream) {
  set_error(ST_OK, "");
  if (!a || !b || !out) return set_error(ST_INVALID_ARG, "gpt_op_gemm: null pointer");
  if (M < 1 || N < 1 || K < 1) return set_error(ST_INVALID_ARG, "gpt_op_gemm: M, N, K must be >= 1");
  if (epilogue != EPI_BF16 && epilogue != EPI_F32) return set_error(ST_INVALID_ARG, "gpt_op_gemm: bad epilogue");
  if (bn != 128 && bn != 256) return set_error(ST_INVALID_ARG, "gpt_op_gemm: bn must be 128 or 256");
  const long long need_a = a_mn ? M : K, need_b = b_mn ? N : K;
  if (lda < need_a || ldb < need_b || ldo < N) return set_error(ST_INVALID_ARG, "gpt_op_gemm: pitch too small");
  GemmParams p = {};
  p.M = M;
  p.N = N;
  p.K = K;
  p.out = out;
  p.ldo = ldo;
  p.bias = bias;
  p.accumulate = accumulate;
  p.hd = p.hdp = 1;
  Operand A{a, lda, a_mn ? 1 : 0};
  Operand B{b, ldb, b_mn ? 1 : 0};
  return run_gemm(epilogue, bn, A, B, p, static_cast<cudaStream_t>(stream));
}

static int check_attn_shape(int B, int T, int H, int hd) {
  if (B < 1 || T < 1 || H < 1) return set_error(ST_INVALID_ARG, "attention: B, T, H must be >= 1");
  if (hd != 64 && hd != 128) return set_error(ST_UNSUPPORTED, "attention: head dim must be 64 or 128");
  return ST_OK;
}

GPT_API int gpt_op_attention_fwd(const void* qkv, int B, int T, int H, int hd, int rope, int qk_norm, int window,
                                 float rope_base, float eps, void* qkv_norm, float* rstd_q, float* rstd_k,
                                 float* rope_cs, void* o, float* lse, void* stream) {
  set_error(ST_OK, "");
  GPTK_TRY(check_attn_shape(B, T, H, hd));
  if (window < -1) return set_error(ST_INVALID_ARG, "attention: window must be >= 0, or -1 for none");
  if (!qkv || !qkv_norm || !o || !lse) return set_error(ST_INVALID_ARG, "attention: null pointer");
  if (rope && !rope_cs) return set_error(ST_INVALID_ARG, "attention: rope needs rope_cs");
  if (qk_norm && (!rstd_q || !rstd_k)) return set_error(ST_INVALID_ARG, "attention: qk_norm needs rstd_q, rstd_k");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int M = B * T;
  float2* cs = reinterpret_cast<float2*>(rope_cs);
  if (rope) GPTK_TRY(launch_rope_table(cs, T, hd / 2, rope_base, st));
  GPTK_TRY(launch_qk_fwd(static_cast<const __nv_bfloat16*>(qkv), cs, M, T, H, hd, hd, rope, qk_norm, eps,
                         static_cast<__nv_bfloat16*>(qkv_norm), rstd_q, rstd_k, st));
  AttnShape s{B, T, H, hd, hd, 3LL * H * hd, window};
  return launch_attn_fwd(static_cast<const __nv_bfloat16*>(qkv_norm), s, static_cast<__nv_bfloat16*>(o),
                         (long long)H * hd, lse, st);
}

GPT_API int gpt_op_attention_bwd(const void* qkv_norm, const float* rstd_q, const float* rstd_k, const float* rope_cs,
                                 const void* o, const float* lse, const void* dout, int B, int T, int H, int hd,
                                 int rope, int qk_norm, int window, float* delta, void* dqkv, void* stream) {
  set_error(ST_OK, "");
  GPTK_TRY(check_attn_shape(B, T, H, hd));
  if (window < -1) return set_error(ST_INVALID_ARG, "attention: window must be >= 0, or -1 for none");
  if (!qkv_norm || !o || !lse || !dout || !delta || !dqkv) return set_error(ST_INVALID_ARG, "attention: null pointer");
  if (rope && !rope_cs) return set_error(ST_INVALID_ARG, "attention: rope needs rope_cs");
  if (qk_norm && (!rstd_q || !rstd_k)) return set_error(ST_INVALID_ARG, "attention: qk_norm needs rstd_q, rstd_k");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int M = B * T;
  const __nv_bfloat16* qn = static_cast<const __nv_bfloat16*>(qkv_norm);
  const __nv_bfloat16* dO = static_cast<const __nv_bfloat16*>(dout);
  __nv_bfloat16* dq = static_cast<__nv_bfloat16*>(dqkv);
  GPTK_TRY(launch_attn_delta(static_cast<const __nv_bfloat16*>(o), dO, B, T, H, hd, hd, delta, st));
  AttnShape s{B, T, H, hd, hd, 3LL * H * hd, window};
  GPTK_TRY(launch_attn_bwd(qn, dO, lse, delta, s, dq, st));
  // gradient w.r.t. the normalised q, k, v -> through QK-norm and RoPE, in place
  return launch_qk_bwd(dq, qn, rstd_q, rstd_k, reinterpret_cast<const float2*>(rope_cs), M, T, H, hd, hd, rope,
                       qk_norm, dq, st);
}

GPT_API size_t gpt_op_lmhead_ce_scratch_bytes(int M, int V) {
  if (M < 1 || V < 1) return 0;
  const size_t ntn = (size_t)(V + 255) / 256;
  return ((size_t)M * ntn * 8 + 255) / 256 * 256 + ((size_t)M * 4 + 255) / 256 * 256;
}

GPT_API int gpt_op_lmhead_ce_fwd(const void* x, const void* w, const int32_t* targets, int M, int D, int V, float* ell,
                                 float* lse, void* scratch, void* stream) {
  set_error(ST_OK, "");
  if (!x || !w || !targets || !ell || !lse || !scratch) return set_error(ST_INVALID_ARG, "lmhead_ce: null pointer");
  if (M < 1 || D < 1 || V < 1) return set_error(ST_INVALID_ARG, "lmhead_ce: M, D, V must be >= 1");
  if (D % 8) return set_error(ST_UNSUPPORTED, "lmhead_ce: D must be a multiple of 8");
  if (reinterpret_cast<uintptr_t>(scratch) & 255) return set_error(ST_INVALID_ARG, "lmhead_ce: scratch alignment");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int ntn = (V + 255) / 256;
  float2* part = static_cast<float2*>(scratch);
  float* zy = reinterpret_cast<float*>(static_cast<char*>(scratch) + ((size_t)M * ntn * 8 + 255) / 256 * 256);
  GemmParams p = {};
  p.M = M;
  p.N = V;
  p.K = D;
  p.hd = p.hdp = 1;
  p.targets = targets;
  p.ce_part = part;
  p.ce_zy = zy;
  GPTK_TRY(run_gemm(EPI_CE_FWD, 256, Operand{x, D, 0}, Operand{w, D, 0}, p, st));
  return launch_ce_combine(part, ntn, zy, targets, V, M, ell, lse, st);
}

}  // extern "C"
