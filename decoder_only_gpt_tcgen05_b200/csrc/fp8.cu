// 8-bit floating-point casts with a dynamic per-tensor scale ("Train your own ChatGPT", read the
// source fp8.py: scale = FP8_MAX / max(|tensor|), quantize, matmul, fold the inverse scales back
// in; e4m3 for activations and weights, e5m2 for gradients).
//
// Two HBM-bound launches per tensor: the absolute maximum (a float atomicMax on the bit pattern of
// |x|, exact and order-independent), then the cast of x * s with round-to-nearest-even and
// saturation (cvt.rn.satfinite), which also writes 1 / s for the product's epilogue.  Where the
// producer of x already folded max |x| into the same kind of slot (the model's FP8 forward: the
// norms, the attention output, the MLP-up epilogue), the cast runs alone (launch_fp8_cast).
#include <string>

#include "gemm.cuh"
#include "gpt_ops.h"
#include "host.cuh"
#include "kernels.cuh"

namespace gptk {

namespace {

constexpr float kMaxE4m3 = 448.f, kMaxE5m2 = 57344.f;

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// 8 elements per thread per step: one 16-byte load of bf16 (two of fp32)
template <typename T>
__device__ __forceinline__ void load8(const T* p, float* v);
template <>
__device__ __forceinline__ void load8<float>(const float* p, float* v) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
}

// n8 = n / 8 vectors, then the tail elements one by one
template <typename T>
__global__ void amax_kernel(const T* __restrict__ x, long long n, unsigned int* __restrict__ amax_bits) {
  float m = 0.f;
  const long long n8 = n / 8;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x, nth = (long long)gridDim.x * blockDim.x;
  for (long long i = tid; i < n8; i += nth) {
    float v[8];
    load8<T>(x + 8 * i, v);
#pragma unroll
    for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(v[k]));
  }
  for (long long i = 8 * n8 + tid; i < n; i += nth) m = fmaxf(m, fabsf(to_f(x[i])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // non-negative floats order like their bit patterns
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

template <typename T, int FMT>
__global__ void quantize_kernel(const T* __restrict__ x, long long n, const float* __restrict__ amax,
                                uint8_t* __restrict__ out, float* __restrict__ inv_scale) {
  pdl_trigger();
  const float fmax = FMT == 0 ? kMaxE4m3 : kMaxE5m2;
  const float a = *amax;
  const float s = a > 0.f ? fmax / a : 1.f;
  if (blockIdx.x == 0 && threadIdx.x == 0) *inv_scale = 1.f / s;
  auto cvt = [](float lo, float hi) -> uint32_t { return FMT == 0 ? cvt_e4m3x2(lo, hi) : cvt_e5m2x2(lo, hi); };
  const long long n8 = n / 8;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x, nth = (long long)gridDim.x * blockDim.x;
  long long i = tid;
  for (; i + nth < n8; i += 2 * nth) {  // two vectors in flight per thread
    float v[2][8];
    load8<T>(x + 8 * i, v[0]);
    load8<T>(x + 8 * (i + nth), v[1]);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      uint2 q;
      q.x = cvt(v[u][0] * s, v[u][1] * s) | (cvt(v[u][2] * s, v[u][3] * s) << 16);
      q.y = cvt(v[u][4] * s, v[u][5] * s) | (cvt(v[u][6] * s, v[u][7] * s) << 16);
      reinterpret_cast<uint2*>(out)[i + u * nth] = q;
    }
  }
  for (; i < n8; i += nth) {
    float v[8];
    load8<T>(x + 8 * i, v);
    uint2 q;
    q.x = cvt(v[0] * s, v[1] * s) | (cvt(v[2] * s, v[3] * s) << 16);
    q.y = cvt(v[4] * s, v[5] * s) | (cvt(v[6] * s, v[7] * s) << 16);
    reinterpret_cast<uint2*>(out)[i] = q;
  }
  for (long long i = 8 * n8 + tid; i < n; i += nth) out[i] = static_cast<uint8_t>(cvt(to_f(x[i]) * s, 0.f) & 0xffu);
}

}  // namespace

int launch_fp8_cast(const void* x, int x_fp32, long long n, int fmt, void* out, const float* amax, float* inv_scale,
                    cudaStream_t st) {
  if (n < 1) return set_error(ST_INVALID_ARG, "fp8_cast: n must be >= 1");
  if (fmt != 0 && fmt != 1) return set_error(ST_INVALID_ARG, "fp8_cast: format must be 0 (e4m3) or 1 (e5m2)");
  if (!x || !out || !amax || !inv_scale) return set_error(ST_INVALID_ARG, "fp8_cast: null pointer");
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(out) & 7))
    return set_error(ST_INVALID_ARG, "fp8_cast: x must be 16-byte and out 8-byte aligned");
  long long g = ((n + 7) / 8 + 255) / 256;
  int grid = (int)(g < num_sms() * 8 ? g : num_sms() * 8);
  Prof prof(PK_MISC, 0, (double)n * ((x_fp32 ? 4 : 2) + 1), st);
  uint8_t* o = static_cast<uint8_t*>(out);
  if (x_fp32) {
    const float* xf = static_cast<const float*>(x);
    if (fmt == 0) quantize_kernel<float, 0><<<grid, 256, 0, st>>>(xf, n, amax, o, inv_scale);
    else quantize_kernel<float, 1><<<grid, 256, 0, st>>>(xf, n, amax, o, inv_scale);
  } else {
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    if (fmt == 0) quantize_kernel<__nv_bfloat16, 0><<<grid, 256, 0, st>>>(xb, n, amax, o, inv_scale);
    else quantize_kernel<__nv_bfloat16, 1><<<grid, 256, 0, st>>>(xb, n, amax, o, inv_scale);
  }
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

int launch_fp8_quantize(const void* x, int x_fp32, long long n, int fmt, void* out, float* amax, float* inv_scale,
                        cudaStream_t st) {
  if (n < 1) return set_error(ST_INVALID_ARG, "fp8_quantize: n must be >= 1");
  if (fmt != 0 && fmt != 1) return set_error(ST_INVALID_ARG, "fp8_quantize: format must be 0 (e4m3) or 1 (e5m2)");
  if (!x || !out || !amax || !inv_scale) return set_error(ST_INVALID_ARG, "fp8_quantize: null pointer");
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(out) & 7))
    return set_error(ST_INVALID_ARG, "fp8_quantize: x must be 16-byte and out 8-byte aligned");
  GPTK_CUDA(cudaMemsetAsync(amax, 0, sizeof(float), st));
  long long g = ((n + 7) / 8 + 255) / 256;
  int grid = (int)(g < num_sms() * 8 ? g : num_sms() * 8);
  {
    Prof prof(PK_MISC, 0, (double)n * (x_fp32 ? 4 : 2), st);
    if (x_fp32) amax_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(x), n, reinterpret_cast<unsigned int*>(amax));
    else amax_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), n, reinterpret_cast<unsigned int*>(amax));
    GPTK_CUDA(cudaGetLastError());
  }
  return launch_fp8_cast(x, x_fp32, n, fmt, out, amax, inv_scale, st);
}

}  // namespace gptk

using namespace gptk;

extern "C" {

GPT_API int gpt_op_fp8_quantize(const void* x, int x_fp32, long long n, int fmt, void* out, float* amax,
                                float* inv_scale, void* stream) {
  set_error(ST_OK, "");
  return launch_fp8_quantize(x, x_fp32, n, fmt, out, amax, inv_scale, static_cast<cudaStream_t>(stream));
}

GPT_API int gpt_op_gemm_fp8(int epilogue, int bn, const void* a, long long lda, int fmt_a, const void* b,
                            long long ldb, int fmt_b, int M, int N, int K, const float* inv_a, const float* inv_b,
                            void* out, long long ldo, const float* bias, int accumulate, void* stream) {
  set_error(ST_OK, "");
  if (!a || !b || !out || !inv_a || !inv_b) return set_error(ST_INVALID_ARG, "gpt_op_gemm_fp8: null pointer");
  if (M < 1 || N < 1 || K < 1) return set_error(ST_INVALID_ARG, "gpt_op_gemm_fp8: M, N, K must be >= 1");
  if (epilogue != EPI_BF16 && epilogue != EPI_F32) return set_error(ST_INVALID_ARG, "gpt_op_gemm_fp8: bad epilogue");
  if (bn != 128 && bn != 256) return set_error(ST_INVALID_ARG, "gpt_op_gemm_fp8: bn must be 128 or 256");
  if ((fmt_a != 0 && fmt_a != 1) || (fmt_b != 0 && fmt_b != 1))
    return set_error(ST_INVALID_ARG, "gpt_op_gemm_fp8: formats must be 0 (e4m3) or 1 (e5m2)");
  if (lda < K || ldb < K || ldo < N) return set_error(ST_INVALID_ARG, "gpt_op_gemm_fp8: pitch too small");
  GemmParams p = {};
  p.M = M;
  p.N = N;
  p.K = K;
  p.out = out;
  p.ldo = ldo;
  p.bias = bias;
  p.accumulate = accumulate;
  p.hd = p.hdp = 1;
  p.f8_fmt_a = fmt_a;
  p.f8_fmt_b = fmt_b;
  p.f8_inv_a = inv_a;
  p.f8_inv_b = inv_b;
  return run_gemm(epilogue, bn, Operand{a, lda, 0}, Operand{b, ldb, 0}, p, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
