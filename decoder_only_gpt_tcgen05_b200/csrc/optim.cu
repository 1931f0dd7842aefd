// The optimizer step of nanoGPT's training loop on one flat fp32 parameter buffer
// ("nanoGPT - Karpathy's minimal GPT pretraining repo", How it works: model.py
// configure_optimizers builds AdamW with weight decay on every 2-D tensor and none on
// 1-D tensors; train.py clips the gradient at grad_clip with clip_grad_norm_ and scales
// it by 1 / the number of accumulated micro-steps).
//
// Two launches, both HBM-bound:
//   1. the squares of the gradient summed in fp64 over a fixed partition of the buffer
//      (kNormParts blocks, each a contiguous chunk), so the norm is bitwise the same on
//      every device and every run;
//   2. the update: every block sums those partials in one fixed order (all blocks get the
//      same bits), forms clip_grad_norm_'s factor min(1, clip / (norm + 1e-6)), and runs
//      the decoupled-weight-decay Adam step over float4 vectors:
//        g <- g * grad_scale * factor
//        m <- beta1 m + (1 - beta1) g,   v <- beta2 v + (1 - beta2) g^2
//        p <- p (1 - lr wd)  (decayed tensors only)
//        p <- p - lr / (1 - beta1^t) * m / (sqrt(v) / sqrt(1 - beta2^t) + eps)
// Algorithmic traffic: 4 bytes per element for the norm, 28 for the update (p, g, m, v
// read; p, m, v written).
#include <cmath>
#include <string>
#include <vector>

#include "gpt.h"
#include "host.cuh"
#include "kernels.cuh"

namespace gptk {

namespace {

constexpr int kNormParts = 1024;  // fixed partition of the norm reduction
constexpr int kMaxRuns = 128;     // decay runs per update launch; longer tables take several launches
constexpr int kThreads = 256;

// Element range of one update launch, split into runs of equal weight-decay flag.
struct DecayRuns {
  long long start[kMaxRuns + 1];  // run r covers [start[r], start[r + 1])
  unsigned int decay[kMaxRuns / 32];
  int n;
};

struct AdamWCoef {
  float beta1, one_m_beta1, beta2, one_m_beta2, eps;
  float decay_factor;  // 1 - lr * weight_decay
  float step_size;     // lr / (1 - beta1^t)
  float inv_sqrt_bc2;  // 1 / sqrt(1 - beta2^t)
  double grad_scale, grad_clip;
};

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum over the block in a fixed order (warp tree, then the warps in index order); the
// result is valid in thread 0.
__device__ __forceinline__ double block_sum_d(double s, double* red) {
  s = warp_sum_d(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < kThreads / 32; ++w) t += red[w];
  return t;
}

__global__ void __launch_bounds__(kThreads) grad_sqsum_kernel(const float* __restrict__ g, long long n,
                                                              double* __restrict__ part) {
  __shared__ double red[kThreads / 32];
  // chunk: a multiple of 4 elements, so every chunk starts on a 16-byte boundary
  const long long chunk = (((n + kNormParts - 1) / kNormParts) + 3) & ~3LL;
  const long long lo = blockIdx.x * chunk;
  const long long hi = lo + chunk < n ? lo + chunk : n;
  double s0 = 0.0, s1 = 0.0;
  if (lo < hi) {
    const long long nv = (hi - lo) >> 2;
    const float4* g4 = reinterpret_cast<const float4*>(g + lo);
    long long i = threadIdx.x;
    for (; i + kThreads < nv; i += 2 * kThreads) {  // two independent loads in flight per thread
      const float4 a = g4[i], b = g4[i + kThreads];
      s0 += (double)a.x * a.x + (double)a.y * a.y + (double)a.z * a.z + (double)a.w * a.w;
      s1 += (double)b.x * b.x + (double)b.y * b.y + (double)b.z * b.z + (double)b.w * b.w;
    }
    if (i < nv) {
      const float4 a = g4[i];
      s0 += (double)a.x * a.x + (double)a.y * a.y + (double)a.z * a.z + (double)a.w * a.w;
    }
    for (long long e = lo + (nv << 2) + threadIdx.x; e < hi; e += kThreads) {
      const double x = g[e];
      s1 += x * x;
    }
  }
  const double t = block_sum_d(s0 + s1, red);
  if (threadIdx.x == 0) part[blockIdx.x] = t;
}

__device__ __forceinline__ void adamw_elem(float& p, float g, float& m, float& v, bool decay, float gs,
                                           const AdamWCoef& c) {
  g *= gs;
  m = c.beta1 * m + c.one_m_beta1 * g;
  v = c.beta2 * v + c.one_m_beta2 * (g * g);
  if (decay) p *= c.decay_factor;
  p -= c.step_size * (m / (sqrtf(v) * c.inv_sqrt_bc2 + c.eps));
}

__global__ void __launch_bounds__(kThreads) adamw_kernel(float* __restrict__ p, const float* __restrict__ g,
                                                         float* __restrict__ m, float* __restrict__ v,
                                                         const double* __restrict__ part, DecayRuns runs,
                                                         AdamWCoef c, double* __restrict__ norm_out) {
  __shared__ long long s_start[kMaxRuns + 1];
  __shared__ unsigned int s_decay[kMaxRuns / 32];
  __shared__ double red[kThreads / 32];
  __shared__ float s_gs;
  for (int i = threadIdx.x; i <= runs.n; i += kThreads) s_start[i] = runs.start[i];
  if (threadIdx.x < kMaxRuns / 32) s_decay[threadIdx.x] = runs.decay[threadIdx.x];
  double t = 0.0;
  for (int i = threadIdx.x; i < kNormParts; i += kThreads) t += part[i];
  t = block_sum_d(t, red);
  if (threadIdx.x == 0) {
    const double norm = c.grad_scale * sqrt(t);
    double factor = 1.0;
    if (c.grad_clip > 0.0) {
      factor = c.grad_clip / (norm + 1e-6);
      if (factor > 1.0) factor = 1.0;
    }
    s_gs = (float)(c.grad_scale * factor);
    if (blockIdx.x == 0 && norm_out) *norm_out = norm;
  }
  __syncthreads();
  const float gs = s_gs;
  const int nr = runs.n;
  const long long lo = s_start[0], hi = s_start[nr];
  const long long q_end = (hi + 3) >> 2;
  for (long long q = (lo >> 2) + blockIdx.x * (long long)kThreads + threadIdx.x; q < q_end;
       q += (long long)gridDim.x * kThreads) {
    const long long e0 = q << 2;
    // the run holding the first in-range element of this vector: the last r with start[r] <= e
    const long long first = e0 > lo ? e0 : lo;
    int a = 0, b = nr - 1;
    while (a < b) {
      const int mid = (a + b + 1) >> 1;
      if (s_start[mid] <= first) a = mid; else b = mid - 1;
    }
    int r = a;
    if (e0 >= lo && e0 + 4 <= hi) {
      float4 pp = reinterpret_cast<float4*>(p)[q];
      const float4 gg = reinterpret_cast<const float4*>(g)[q];
      float4 mm = reinterpret_cast<float4*>(m)[q];
      float4 vv = reinterpret_cast<float4*>(v)[q];
      float* pe = &pp.x;
      const float* ge = &gg.x;
      float* me = &mm.x;
      float* ve = &vv.x;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        while (e0 + j >= s_start[r + 1]) ++r;
        adamw_elem(pe[j], ge[j], me[j], ve[j], (s_decay[r >> 5] >> (r & 31)) & 1u, gs, c);
      }
      reinterpret_cast<float4*>(p)[q] = pp;
      reinterpret_cast<float4*>(m)[q] = mm;
      reinterpret_cast<float4*>(v)[q] = vv;
    } else {
      // a vector cut by the launch's range: element by element, only those inside it
      for (int j = 0; j < 4; ++j) {
        const long long e = e0 + j;
        if (e < lo || e >= hi) continue;
        while (e >= s_start[r + 1]) ++r;
        float pe = p[e], me = m[e], ve = v[e];
        adamw_elem(pe, g[e], me, ve, (s_decay[r >> 5] >> (r & 31)) & 1u, gs, c);
        p[e] = pe;
        m[e] = me;
        v[e] = ve;
      }
    }
  }
}

inline bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }
inline bool is_finite(double x) { return std::isfinite(x); }

}  // namespace

size_t adamw_scratch_bytes() { return kNormParts * sizeof(double); }

int launch_adamw(float* params, const float* grads, float* m, float* v, long long n, const long long* run_start,
                 const unsigned char* run_decay, int n_runs, long long step, const gpt_adamw& h, void* scratch,
                 double* grad_norm, cudaStream_t st) {
  if (n < 0) return set_error(ST_INVALID_ARG, "adamw: n must be >= 0");
  if (step < 1) return set_error(ST_INVALID_ARG, "adamw: step must be >= 1");
  if (!is_finite(h.lr) || !is_finite(h.beta1) || !is_finite(h.beta2) || !is_finite(h.eps) ||
      !is_finite(h.weight_decay) || !is_finite(h.grad_scale) || !is_finite(h.grad_clip))
    return set_error(ST_INVALID_ARG, "adamw: hyperparameters must be finite");
  if (h.lr < 0.f || h.beta1 < 0.f || h.beta1 >= 1.f || h.beta2 < 0.f || h.beta2 >= 1.f || !(h.eps > 0.f) ||
      h.weight_decay < 0.f || !(h.grad_scale > 0.f) || h.grad_clip < 0.f || (double)h.lr * h.weight_decay > 1.0)
    return set_error(ST_INVALID_ARG,
                     "adamw: need lr >= 0, 0 <= beta < 1, eps > 0, weight_decay >= 0, lr * weight_decay <= 1, "
                     "grad_scale > 0, grad_clip >= 0");
  if (n == 0) {  // empty buffers may be null
    if (grad_norm) GPTK_CUDA(cudaMemsetAsync(grad_norm, 0, sizeof(double), st));
    return ST_OK;
  }
  if (!params || !grads || !m || !v || !scratch) return set_error(ST_INVALID_ARG, "adamw: null pointer");
  if (!aligned16(params) || !aligned16(grads) || !aligned16(m) || !aligned16(v))
    return set_error(ST_INVALID_ARG, "adamw: params, grads, m and v must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(scratch) & 7u) != 0)
    return set_error(ST_INVALID_ARG, "adamw: scratch must be 8-byte aligned");
  if (!run_start || !run_decay || n_runs < 1) return set_error(ST_INVALID_ARG, "adamw: empty run table");
  if (run_start[0] != 0) return set_error(ST_INVALID_ARG, "adamw: the first run must start at element 0");
  for (int r = 1; r < n_runs; ++r)
    if (run_start[r] <= run_start[r - 1] || run_start[r] >= n)
      return set_error(ST_INVALID_ARG, "adamw: run starts must increase strictly and stay below n");

  double* part = static_cast<double*>(scratch);
  {
    Prof prof(PK_OPTIM, 0, n * 4.0, st);
    grad_sqsum_kernel<<<kNormParts, kThreads, 0, st>>>(grads, n, part);
    GPTK_CUDA(cudaGetLastError());
  }
  AdamWCoef c;
  c.beta1 = h.beta1;
  c.one_m_beta1 = (float)(1.0 - (double)h.beta1);
  c.beta2 = h.beta2;
  c.one_m_beta2 = (float)(1.0 - (double)h.beta2);
  c.eps = h.eps;
  c.decay_factor = (float)(1.0 - (double)h.lr * h.weight_decay);
  c.step_size = (float)((double)h.lr / (1.0 - std::pow((double)h.beta1, (double)step)));
  c.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(1.0 - std::pow((double)h.beta2, (double)step)));
  c.grad_scale = h.grad_scale;
  c.grad_clip = h.grad_clip;
  const int max_grid = num_sms() * 8;
  for (int r0 = 0; r0 < n_runs; r0 += kMaxRuns) {
    const int r1 = r0 + kMaxRuns < n_runs ? r0 + kMaxRuns : n_runs;
    DecayRuns runs = {};
    runs.n = r1 - r0;
    for (int r = r0; r < r1; ++r) {
      runs.start[r - r0] = run_start[r];
      if (run_decay[r]) runs.decay[(r - r0) >> 5] |= 1u << ((r - r0) & 31);
    }
    runs.start[runs.n] = r1 < n_runs ? run_start[r1] : n;
    const long long vecs = ((runs.start[runs.n] + 3) >> 2) - (runs.start[0] >> 2);
    long long grid = (vecs + kThreads - 1) / kThreads;
    if (grid > max_grid) grid = max_grid;
    Prof prof(PK_OPTIM, 0, (runs.start[runs.n] - runs.start[0]) * 28.0, st);
    adamw_kernel<<<(int)grid, kThreads, 0, st>>>(params, grads, m, v, part, runs, c, r0 == 0 ? grad_norm : nullptr);
    GPTK_CUDA(cudaGetLastError());
  }
  return ST_OK;
}

}  // namespace gptk

// ====================================================================== C ABI

using namespace gptk;

extern "C" {

GPT_API int gpt_adamw_scratch_size(size_t* bytes) {
  set_error(ST_OK, "");
  if (!bytes) return set_error(ST_INVALID_ARG, "null output");
  *bytes = adamw_scratch_bytes();
  return ST_OK;
}

GPT_API size_t gpt_op_adamw_scratch_bytes(void) { return adamw_scratch_bytes(); }

GPT_API int gpt_op_adamw(float* params, const float* grads, float* m, float* v, int64_t n, const int64_t* run_start,
                         const uint8_t* run_decay, int32_t n_runs, int64_t step, const gpt_adamw* h, void* scratch,
                         double* grad_norm, void* stream) {
  set_error(ST_OK, "");
  if (!h) return set_error(ST_INVALID_ARG, "gpt_op_adamw: null hyperparameters");
  if (n_runs < 0 || n_runs > (1 << 20)) return set_error(ST_INVALID_ARG, "gpt_op_adamw: bad run count");
  std::vector<long long> starts(run_start ? (size_t)n_runs : 0);
  for (size_t r = 0; r < starts.size(); ++r) starts[r] = run_start[r];
  return launch_adamw(params, grads, m, v, n, starts.empty() ? nullptr : starts.data(), run_decay, n_runs, step, *h,
                      scratch, grad_norm, static_cast<cudaStream_t>(stream));
}

GPT_API int gpt_lr_schedule(int64_t it, int64_t warmup_iters, int64_t lr_decay_iters, double learning_rate,
                            double min_lr, double* lr_out) {
  set_error(ST_OK, "");
  if (!lr_out) return set_error(ST_INVALID_ARG, "null output");
  if (it < 0 || warmup_iters < 0 || lr_decay_iters < warmup_iters)
    return set_error(ST_INVALID_ARG, "lr_schedule: need it >= 0 and 0 <= warmup_iters <= lr_decay_iters");
  if (it < warmup_iters) {
    *lr_out = learning_rate * (double)it / (double)warmup_iters;
  } else if (it > lr_decay_iters) {
    *lr_out = min_lr;
  } else if (lr_decay_iters == warmup_iters) {
    *lr_out = learning_rate;
  } else {
    const double r = (double)(it - warmup_iters) / (double)(lr_decay_iters - warmup_iters);
    *lr_out = min_lr + 0.5 * (1.0 + std::cos(M_PI * r)) * (learning_rate - min_lr);
  }
  return ST_OK;
}

}  // extern "C"
