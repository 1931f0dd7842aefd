// Memory-bound kernels of the hot path: parameter cast, RoPE table, embedding,
// norms (forward / backward), column reductions, cross-entropy combine, loss and
// bits-per-byte reduction, QK-norm + RoPE (forward / backward), attention delta,
// and the counter-based initialiser.  Every reduction runs in a fixed order so
// results are bitwise reproducible run to run.
#include <cmath>
#include <string>

#include "host.cuh"
#include "kernels.cuh"

namespace gptk {

static inline int cdiv(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ------------------------------------------------------------------ cast

__global__ void cast_bf16_kernel(const float4* __restrict__ src, uint2* __restrict__ dst, long long n4) {
  pdl_trigger();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    float4 v = src[i];
    dst[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

int launch_cast_bf16(const float* src, __nv_bfloat16* dst, long long n, cudaStream_t st) {
  if (n % 4) return set_error(ST_INVALID_ARG, "cast: n must be a multiple of 4");
  long long n4 = n / 4;
  int grid = num_sms() * 8;
  if (n4 < (long long)grid * 256) grid = cdiv(n4, 256);
  if (grid < 1) return ST_OK;
  Prof prof(PK_CAST, 0, n * 6.0, st);
  cast_bf16_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const float4*>(src), reinterpret_cast<uint2*>(dst), n4);
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

// ------------------------------------------------------------------ RoPE table

__global__ void rope_table_kernel(float2* cs, int T, int half, double base) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * half) return;
  int t = i / half, j = i % half;
  double inv = pow(base, -static_cast<double>(j) / static_cast<double>(half));
  double s, c;
  sincos(static_cast<double>(t) * inv, &s, &c);
  cs[i] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

int launch_rope_table(float2* cs, int T, int half, double base, cudaStream_t st) {
  Prof prof(PK_MISC, 0, (double)T * half * 8, st);
  rope_table_kernel<<<cdiv((long long)T * half, 256), 256, 0, st>>>(cs, T, half, base);
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

// ------------------------------------------------------------------ embedding

__global__ void embed_fwd_kernel(const int* __restrict__ idx, const float* __restrict__ wte,
                                 const float* __restrict__ wpe, float* __restrict__ x, int M, int T, int D, int V,
                                 DevCtl ctl) {
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (int m = blockIdx.x * warps + (threadIdx.x >> 5); m < M; m += gridDim.x * warps) {
    int id = idx[m];
    if (id < 0 || id >= V) {
      if (lane == 0) dev_report(ctl, DEV_ERR_BAD_TOKEN, 0);
      id = 0;
    }
    const float4* e = reinterpret_cast<const float4*>(wte + (long long)id * D);
    const float4* p = wpe ? reinterpret_cast<const float4*>(wpe + (long long)(m % T) * D) : nullptr;
    float4* o = reinterpret_cast<float4*>(x + (long long)m * D);
    for (int c = lane; c < D / 4; c += 32) {
      float4 v = __ldg(e + c);
      if (p) {
        float4 q = __ldg(p + c);
        v.x += q.x; v.y += q.y; v.z += q.z; v.w += q.w;
      }
      o[c] = v;
    }
  }
}

int launch_embed_fwd(const int* idx, const float* wte, const float* wpe, float* x, int M, int T, int D, int V,
                     cudaStream_t st) {
  int grid = cdiv(M, 8);
  if (grid > num_sms() * 16) grid = num_sms() * 16;
  Prof prof(PK_EMBED_FWD, 0, (double)M * D * (wpe ? 12 : 8) + M * 4.0, st);
  embed_fwd_kernel<<<grid, 256, 0, st>>>(idx, wte, wpe, x, M, T, D, V, device_ctl());
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

// ------------------------------------------------------------------ norms
// One warp per row.  A row of D <= 128*NV floats lives in registers (NV float4 per lane).

// max over the block of each thread's am, rounded to bf16 (the values were stored as bf16, and the
// rounding is monotonic), into *amax_bits as a float bit pattern (non-negative floats order like
// their bits, so atomicMax is exact and order-independent)
__device__ __forceinline__ void block_amax(float am, unsigned int* amax_bits) {
  __shared__ float red[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = am;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.f;
    for (int i = 0; i < nw; ++i) m = fmaxf(m, red[i]);
    atomicMax(amax_bits, __float_as_uint(__bfloat162float(__float2bfloat16_rn(m))));
  }
}

template <int NV, bool LN>
__global__ void norm_fwd_kernel(const float* __restrict__ x, int M, int D, const float* __restrict__ g,
                                const float* __restrict__ b, float eps, __nv_bfloat16* __restrict__ y,
                                long long ldy, float* __restrict__ mean_out, float* __restrict__ rstd_out,
                                unsigned int* __restrict__ amax_bits) {
  pdl_trigger();
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  const int D4 = D / 4;
  float am = 0.f;  // max |y| of this thread's elements (for an 8-bit cast of y)
  for (int m = blockIdx.x * warps + (threadIdx.x >> 5); m < M; m += gridDim.x * warps) {
    const float4* xr = reinterpret_cast<const float4*>(x + (long long)m * D);
    float4 v[NV];
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      int c = i * 32 + lane;
      v[i] = c < D4 ? xr[c] : make_float4(0.f, 0.f, 0.f, 0.f);
      s += v[i].x + v[i].y + v[i].z + v[i].w;
    }
    float mu = 0.f;
    if (LN) mu = warp_sum(s) / D;
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      int c = i * 32 + lane;
      if (c < D4) {
        float a = v[i].x - mu, bb = v[i].y - mu, cc = v[i].z - mu, d = v[i].w - mu;
        ss += a * a + bb * bb + cc * cc + d * d;
      }
    }
    const float r = rsqrtf(warp_sum(ss) / D + eps);
    if (lane == 0) {
      rstd_out[m] = r;
      if (LN) mean_out[m] = mu;
    }
    uint2* yr = reinterpret_cast<uint2*>(y + (long long)m * ldy);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      int c = i * 32 + lane;
      if (c < D4) {
        float4 o = make_float4((v[i].x - mu) * r, (v[i].y - mu) * r, (v[i].z - mu) * r, (v[i].w - mu) * r);
        if (LN) {
          float4 gg = __ldg(reinterpret_cast<const float4*>(g) + c);
          o.x *= gg.x; o.y *= gg.y; o.z *= gg.z; o.w *= gg.w;
          if (b) {
            float4 bb = __ldg(reinterpret_cast<const float4*>(b) + c);
            o.x += bb.x; o.y += bb.y; o.z += bb.z; o.w += bb.w;
          }
        }
        yr[c] = make_uint2(pack_bf16x2(o.x, o.y), pack_bf16x2(o.z, o.w));
        am = fmaxf(am, fmaxf(fmaxf(fabsf(o.x), fabsf(o.y)), fmaxf(fabsf(o.z), fabsf(o.w))));
      }
    }
  }
  if (amax_bits) block_amax(am, amax_bits);
}

template <int NV, bool LN>
__global__ void norm_bwd_kernel(const float* __restrict__ dy, const float* __restrict__ x,
                                const float* __restrict__ mean, const float* __restrict__ rstd,
                                const float* __restrict__ g, int M, int D, float* __restrict__ dres, int dres_init,
                                __nv_bfloat16* __restrict__ dres_bf, float* __restrict__ dg_part,
                                float* __restrict__ db_part) {
  pdl_trigger();
  extern __shared__ float red[];  // [warps][2][D] (LayerNorm only)
  const int warps = blockDim.x >> 5;
  const int w = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int D4 = D / 4;
  float4 dg[LN ? NV : 1], db[LN ? NV : 1];
  if (LN) {
#pragma unroll
    for (int i = 0; i < NV; ++i) dg[i] = db[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int m = blockIdx.x * warps + w; m < M; m += gridDim.x * warps) {
    const float4* xr = reinterpret_cast<const float4*>(x + (long long)m * D);
    const float4* gr = reinterpret_cast<const float4*>(dy + (long long)m * D);
    const float mu = LN ? mean[m] : 0.f;
    const float r = rstd[m];
    float4 xh[NV], gh[NV];
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      int c = i * 32 + lane;
      if (c < D4) {
        float4 xv = xr[c], gv = gr[c];
        xh[i] = make_float4((xv.x - mu) * r, (xv.y - mu) * r, (xv.z - mu) * r, (xv.w - mu) * r);
        if (LN) {
          db[i].x += gv.x; db[i].y += gv.y; db[i].z += gv.z; db[i].w += gv.w;
          dg[i].x += gv.x * xh[i].x; dg[i].y += gv.y * xh[i].y; dg[i].z += gv.z * xh[i].z; dg[i].w += gv.w * xh[i].w;
          float4 gg = __ldg(reinterpret_cast<const float4*>(g) + c);
          gv.x *= gg.x; gv.y *= gg.y; gv.z *= gg.z; gv.w *= gg.w;
          s1 += gv.x + gv.y + gv.z + gv.w;
        }
        gh[i] = gv;
        s2 += gv.x * xh[i].x + gv.y * xh[i].y + gv.z * xh[i].z + gv.w * xh[i].w;
      } else {
        xh[i] = gh[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    const float m1 = LN ? warp_sum(s1) / D : 0.f;
    const float m2 = warp_sum(s2) / D;
    float4* dr = reinterpret_cast<float4*>(dres + (long long)m * D);
    uint2* db16 = reinterpret_cast<uint2*>(dres_bf + (long long)m * D);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      int c = i * 32 + lane;
      if (c < D4) {
        float4 o = make_float4(r * (gh[i].x - m1 - xh[i].x * m2), r * (gh[i].y - m1 - xh[i].y * m2),
                               r * (gh[i].z - m1 - xh[i].z * m2), r * (gh[i].w - m1 - xh[i].w * m2));
        if (!dres_init) {
          float4 prev = dr[c];
          o.x += prev.x; o.y += prev.y; o.z += prev.z; o.w += prev.w;
        }
        dr[c] = o;
        db16[c] = make_uint2(pack_bf16x2(o.x, o.y), pack_bf16x2(o.z, o.w));
      }
    }
  }
  if (!LN) return;
  // block-level reduction of the gain / bias partials in warp order
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    int c = i * 32 + lane;
    if (c < D4) {
      reinterpret_cast<float4*>(red + (size_t)w * 2 * D)[c] = dg[i];
      reinterpret_cast<float4*>(red + (size_t)w * 2 * D + D)[c] = db[i];
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float a = 0.f, bsum = 0.f;
    for (int k = 0; k < warps; ++k) {
      a += red[(size_t)k * 2 * D + c];
      bsum += red[(size_t)k * 2 * D + D + c];
    }
    dg_part[(size_t)blockIdx.x * D + c] = a;
    db_part[(size_t)blockIdx.x * D + c] = bsum;
  }
}

// NV = float4 per lane = ceil(D / 128): the row lives in registers without slack
template <typename F>
static int norm_dispatch(int D, F&& f) {
  if (D % 4) return set_error(ST_UNSUPPORTED, "norm: n_embd must be a multiple of 4");
  const int nv = (D + 127) / 128;
  switch (nv) {
    case 1: return f(std::integral_constant<int, 1>());
    case 2: return f(std::integral_constant<int, 2>());
    case 3: case 4: return f(std::integral_constant<int, 4>());
    case 5: case 6: return f(std::integral_constant<int, 6>());
    case 7: case 8: return f(std::integral_constant<int, 8>());
    case 9: case 10: return f(std::integral_constant<int, 10>());
    case 11: case 12: case 13: return f(std::integral_constant<int, 13>());
    case 14: case 15: case 16: return f(std::integral_constant<int, 16>());
  }
  if (nv <= 24) return f(std::integral_constant<int, 24>());
  if (nv <= 32) return f(std::integral_constant<int, 32>());
  return set_error(ST_UNSUPPORTED, "norm: n_embd above 4096");
}

int launch_norm_fwd(const float* x, int M, int D, const float* g, const float* b, int ln, float eps,
                    __nv_bfloat16* y, long long ldy, float* mean, float* rstd, cudaStream_t st, float* amax) {
  return norm_dispatch(D, [&](auto nv) {
    constexpr int NV = decltype(nv)::value;
    int grid = cdiv(M, 8);
    if (grid > num_sms() * 16) grid = num_sms() * 16;
    Prof prof(PK_NORM_FWD, 0, (double)M * D * 6 + M * 8.0, st);
    unsigned int* ab = reinterpret_cast<unsigned int*>(amax);
    if (ln)
      norm_fwd_kernel<NV, true><<<grid, 256, 0, st>>>(x, M, D, g, b, eps, y, ldy, mean, rstd, ab);
    else
      norm_fwd_kernel<NV, false><<<grid, 256, 0, st>>>(x, M, D, g, b, eps, y, ldy, mean, rstd, ab);
    GPTK_CUDA(cudaGetLastError());
    return (int)ST_OK;
  });
}

// RMSNorm backward from the saved bf16 output y = x r (the next GEMM's A operand, kept for the
// weight gradients) instead of x: dx = r (dy - y mean(dy y)); dres (+)= dx in fp32 and a bf16 copy.
// dy is bf16 (DYB) or fp32.  One warp per row, 8 elements per lane and step (16-byte loads of the
// bf16 rows); 14 bytes per element with a bf16 dy and accumulation (18 for the x-based kernel).
__device__ __forceinline__ void bf16x8(uint4 u, float* v) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
}

template <int NV8, bool DYB>
__global__ void rms_bwd_kernel(const void* __restrict__ dy_, const __nv_bfloat16* __restrict__ y,
                               const float* __restrict__ rstd, int M, int D, float* __restrict__ dres,
                               int dres_init, __nv_bfloat16* __restrict__ dres_bf) {
  pdl_trigger();
  const int warps = blockDim.x >> 5;
  const int w = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int D8 = D / 8;
  for (int m = blockIdx.x * warps + w; m < M; m += gridDim.x * warps) {
    const long long base = (long long)m * D;
    const float r = rstd[m];
    float yv[NV8][8], gv[NV8][8], dv[NV8][8];
    float s2 = 0.f;
#pragma unroll
    for (int i = 0; i < NV8; ++i) {
      const int c = i * 32 + lane;
      if (c < D8) {
        // the residual gradient is loaded with the row's other inputs, ahead of the reduction
        // (rows up to 1536 wide; wider rows load it afterwards, to stay within the registers)
        if (!dres_init && NV8 <= 6) {
          const float4* dr = reinterpret_cast<const float4*>(dres + base) + 2 * c;
          const float4 a = dr[0], b = dr[1];
          dv[i][0] = a.x; dv[i][1] = a.y; dv[i][2] = a.z; dv[i][3] = a.w;
          dv[i][4] = b.x; dv[i][5] = b.y; dv[i][6] = b.z; dv[i][7] = b.w;
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) dv[i][k] = 0.f;
        }
        bf16x8(reinterpret_cast<const uint4*>(y + base)[c], yv[i]);
        if (DYB) {
          bf16x8(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(dy_) + base)[c], gv[i]);
        } else {
          const float4* g4 = reinterpret_cast<const float4*>(static_cast<const float*>(dy_) + base) + 2 * c;
          const float4 a = g4[0], b = g4[1];
          gv[i][0] = a.x; gv[i][1] = a.y; gv[i][2] = a.z; gv[i][3] = a.w;
          gv[i][4] = b.x; gv[i][5] = b.y; gv[i][6] = b.z; gv[i][7] = b.w;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) s2 = fmaf(gv[i][k], yv[i][k], s2);
      }
    }
    const float m2 = warp_sum(s2) / D;
#pragma unroll
    for (int i = 0; i < NV8; ++i) {
      const int c = i * 32 + lane;
      if (c < D8) {
        float o[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] = r * (gv[i][k] - yv[i][k] * m2) + dv[i][k];
        float4* dr = reinterpret_cast<float4*>(dres + base) + 2 * c;
        if (!dres_init && NV8 > 6) {
          const float4 a = dr[0], b = dr[1];
          o[0] += a.x; o[1] += a.y; o[2] += a.z; o[3] += a.w; o[4] += b.x; o[5] += b.y; o[6] += b.z; o[7] += b.w;
        }
        dr[0] = make_float4(o[0], o[1], o[2], o[3]);
        dr[1] = make_float4(o[4], o[5], o[6], o[7]);
        reinterpret_cast<uint4*>(dres_bf + base)[c] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                                                 pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
      }
    }
  }
}

int launch_rms_bwd(const void* dy, int dy_bf16, const __nv_bfloat16* y, const float* rstd, int M, int D,
                   float* dres, int dres_init, __nv_bfloat16* dres_bf, cudaStream_t st) {
  if (D % 8) return set_error(ST_UNSUPPORTED, "rms_bwd: n_embd must be a multiple of 8");
  const int nv8 = (D + 255) / 256;
  auto run = [&](auto nvc) -> int {
    constexpr int NV8 = decltype(nvc)::value;
    int grid = cdiv(M, 4);
    if (grid > num_sms() * 32) grid = num_sms() * 32;
    Prof prof(PK_NORM_BWD, 0, (double)M * D * ((dy_bf16 ? 2 : 4) + 2 + 4 + 2 + (dres_init ? 0 : 4)) + M * 4.0, st);
    if (dy_bf16) rms_bwd_kernel<NV8, true><<<grid, 128, 0, st>>>(dy, y, rstd, M, D, dres, dres_init, dres_bf);
    else rms_bwd_kernel<NV8, false><<<grid, 128, 0, st>>>(dy, y, rstd, M, D, dres, dres_init, dres_bf);
    GPTK_CUDA(cudaGetLastError());
    return (int)ST_OK;
  };
  switch (nv8) {
    case 1: return run(std::integral_constant<int, 1>());
    case 2: return run(std::integral_constant<int, 2>());
    case 3: return run(std::integral_constant<int, 3>());
    case 4: return run(std::integral_constant<int, 4>());
    case 5: return run(std::integral_constant<int, 5>());
    case 6: return run(std::integral_constant<int, 6>());
    case 7: case 8: return run(std::integral_constant<int, 8>());
    case 9: case 10: case 11: case 12: return run(std::integral_constant<int, 12>());
    case 13: case 14: case 15: case 16: return run(std::integral_constant<int, 16>());
  }
  return set_error(ST_UNSUPPORTED, "rms_bwd: n_embd above 4096");
}

static const int kNormBwdBlocks = 296;

int launch_norm_bwd(const float* dy, const float* x, const float* mean, const float* rstd, const float* g, int ln,
                    int M, int D, float* dres, int dres_init, __nv_bfloat16* dres_bf, float* dg_part,
                    float* db_part, int* nblk_out, cudaStream_t st) {
  return norm_dispatch(D, [&](auto nv) {
    constexpr int NV = decltype(nv)::value;
    int grid = cdiv(M, 8);
    // LayerNorm keeps one gain/bias partial per block, so its grid is capped
    const int cap = ln ? kNormBwdBlocks : num_sms() * 16;
    if (grid > cap) grid = cap;
    Prof prof(PK_NORM_BWD, 0, (double)M * D * (dres_init ? 14 : 18), st);
    if (ln) {
      size_t smem = (size_t)8 * 2 * D * sizeof(float);
      if (smem > 48 * 1024)
        GPTK_CUDA(cudaFuncSetAttribute(norm_bwd_kernel<NV, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem));
      norm_bwd_kernel<NV, true><<<grid, 256, smem, st>>>(dy, x, mean, rstd, g, M, D, dres, dres_init, dres_bf,
                                                         dg_part, db_part);
    } else {
      norm_bwd_kernel<NV, false><<<grid, 256, 0, st>>>(dy, x, mean, rstd, g, M, D, dres, dres_init, dres_bf,
                                                       dg_part, db_part);
    }
    GPTK_CUDA(cudaGetLastError());
    if (nblk_out) *nblk_out = grid;
    return (int)ST_OK;
  });
}

int norm_bwd_max_blocks() { return kNormBwdBlocks; }

// ------------------------------------------------------------------ column reductions

__global__ void colreduce_kernel(const float* __restrict__ part, int R, int N, float* __restrict__ out,
                                 int accumulate) {
  int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= N) return;
  float s = 0.f;
  for (int r = 0; r < R; ++r) s += part[(size_t)r * N + c];
  out[c] = accumulate ? out[c] + s : s;
}

int launch_colreduce(const float* part, int R, int N, float* out, int accumulate, cudaStream_t st) {
  Prof prof(PK_COLSUM, 0, (double)R * N * 4, st);
  colreduce_kernel<<<cdiv(N, 256), 256, 0, st>>>(part, R, N, out, accumulate);
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

static const int kColsumChunks = 128;
int colsum_max_chunks() { return kColsumChunks; }

template <typename T>
__global__ void colsum_kernel(const T* __restrict__ a, long long lda, int M, int N, int rows_per, float* part) {
  int c = blockIdx.x * blockDim.x + threadIdx.x;
  int r0 = blockIdx.y * rows_per;
  if (c >= N) return;
  int r1 = min(M, r0 + rows_per);
  float s = 0.f;
  for (int r = r0; r < r1; ++r) s += static_cast<float>(a[(long long)r * lda + c]);
  part[(size_t)blockIdx.y * N + c] = s;
}

template <typename T>
static int colsum_t(const T* a, long long lda, int M, int N, float* part, int* R, cudaStream_t st) {
  int rows_per = cdiv(M, kColsumChunks);
  int chunks = cdiv(M, rows_per);
  dim3 grid(cdiv(N, 128), chunks);
  Prof prof(PK_COLSUM, 0, (double)M * N * sizeof(T), st);
  colsum_kernel<T><<<grid, 128, 0, st>>>(a, lda, M, N, rows_per, part);
  GPTK_CUDA(cudaGetLastError());
  *R = chunks;
  return ST_OK;
}

int launch_colsum_f32(const float* a, long long lda, int M, int N, float* part, int* R, cudaStream_t st) {
  return colsum_t(a, lda, M, N, part, R, st);
}
int launch_colsum_bf16(const __nv_bfloat16* a, long long lda, int M, int N, float* part, int* R, cudaStream_t st) {
  return colsum_t(a, lda, M, N, part, R, st);
}

// ------------------------------------------------------------------ cross-entropy combine

// A target outside [0, V) has no logit: the row's loss is NaN and the device status word records
// the bad id (the tile epilogues never match it, so its target-logit slot was not written).
__global__ void ce_combine_kernel(const float2* __restrict__ part, int ntiles, const float* __restrict__ zy,
                                  const int* __restrict__ targets, int V, int M, float* __restrict__ ell,
                                  float* __restrict__ lse, DevCtl ctl) {
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (int m = blockIdx.x * warps + (threadIdx.x >> 5); m < M; m += gridDim.x * warps) {
    const float2* p = part + (long long)m * ntiles;
    float mx = -INFINITY;
    for (int t = lane; t < ntiles; t += 32) mx = fmaxf(mx, p[t].x);
    mx = warp_max(mx);
    float s = 0.f;
    for (int t = lane; t < ntiles; t += 32) {
      float2 q = p[t];
      if (q.x != -INFINITY) s += q.y * ex2_approx(q.x - mx);
    }
    s = warp_sum(s);
    if (lane == 0) {
      float l = (mx + log2f(s)) * 0.6931471805599453f;
      lse[m] = l;
      const int y = targets[m];
      if (y < 0 || y >= V) {
        dev_report(ctl, DEV_ERR_BAD_TOKEN, 1);
        ell[m] = __int_as_float(0x7fc00000);
      } else {
        ell[m] = l - zy[m];
      }
    }
  }
}

int launch_ce_combine(const float2* part, int ntiles, const float* zy, const int* targets, int V, int M, float* ell,
                      float* lse, cudaStream_t st) {
  int grid = cdiv(M, 8);
  if (grid > num_sms() * 16) grid = num_sms() * 16;
  Prof prof(PK_CE_COMBINE, 0, (double)M * ntiles * 8 + M * 16.0, st);
  ce_combine_kernel<<<grid, 256, 0, st>>>(part, ntiles, zy, targets, V, M, ell, lse, device_ctl());
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

// ------------------------------------------------------------------ loss / bpb reduction

static const int kLossBlocks = 256;
int loss_reduce_blocks() { return kLossBlocks; }

// part_d: [blocks][2] (sum of loss, sum of loss over byte-bearing targets); part_i: [blocks][2] (bytes, count)
__global__ void loss_partial_kernel(const float* __restrict__ ell, const int* __restrict__ targets,
                                    const int* __restrict__ tb, int V, int M, double* part_d, long long* part_i) {
  __shared__ double sd[2][8];
  __shared__ long long si[2][8];
  int per = (M + gridDim.x - 1) / gridDim.x;
  int r0 = blockIdx.x * per, r1 = min(M, r0 + per);
  double a = 0.0, b = 0.0;
  long long nb = 0, cnt = 0;
  for (int r = r0 + threadIdx.x; r < r1; r += blockDim.x) {
    double l = ell[r];
    a += l;
    if (tb) {
      const int y = targets[r];
      const int bytes = (y >= 0 && y < V) ? tb[y] : 0;  // a bad id was reported by the combine kernel
      if (bytes > 0) {
        b += l;
        nb += bytes;
        cnt += 1;
      }
    }
  }
  a = warp_sum_d(a);
  b = warp_sum_d(b);
  nb = warp_sum_ll(nb);
  cnt = warp_sum_ll(cnt);
  int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sd[0][w] = a; sd[1][w] = b; si[0][w] = nb; si[1][w] = cnt;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double A = 0, Bs = 0;
    long long NB = 0, C = 0;
    for (int k = 0; k < (int)(blockDim.x >> 5); ++k) {
      A += sd[0][k]; Bs += sd[1][k]; NB += si[0][k]; C += si[1][k];
    }
    part_d[2 * blockIdx.x] = A;
    part_d[2 * blockIdx.x + 1] = Bs;
    part_i[2 * blockIdx.x] = NB;
    part_i[2 * blockIdx.x + 1] = C;
  }
}

__global__ void loss_final_kernel(const double* part_d, const long long* part_i, int nblk, int M, float* loss,
                                  double* sum_nats, long long* sum_bytes, float* bpb) {
  if (threadIdx.x != 0) return;
  double A = 0, Bs = 0;
  long long NB = 0;
  for (int k = 0; k < nblk; ++k) {
    A += part_d[2 * k];
    Bs += part_d[2 * k + 1];
    NB += part_i[2 * k];
  }
  if (loss) *loss = static_cast<float>(A / M);
  if (sum_nats) *sum_nats = Bs;
  if (sum_bytes) *sum_bytes = NB;
  if (bpb) *bpb = NB > 0 ? static_cast<float>(Bs / (0.6931471805599453 * (double)NB)) : NAN;
}

int launch_loss_reduce(const float* ell, const int* targets, const int* token_bytes, int V, int M, double* part_d,
                       long long* part_i, float* loss, double* sum_nats, long long* sum_bytes, float* bpb,
                       cudaStream_t st) {
  {
    Prof prof(PK_LOSS, 0, M * 12.0, st);
    loss_partial_kernel<<<kLossBlocks, 256, 0, st>>>(ell, targets, token_bytes, V, M, part_d, part_i);
    GPTK_CUDA(cudaGetLastError());
  }
  {
    Prof prof(PK_LOSS, 0, kLossBlocks * 32.0, st);
    loss_final_kernel<<<1, 32, 0, st>>>(part_d, part_i, kLossBlocks, M, loss, sum_nats, sum_bytes, bpb);
    GPTK_CUDA(cudaGetLastError());
  }
  return ST_OK;
}

// ------------------------------------------------------------------ QK-norm + RoPE
// One warp per (token, head).  Lane l owns pair indices i = l*PPL .. l*PPL+PPL-1 (i < hd/2)
// and their partners i + hd/2, so a RoPE pair never crosses lanes; with PPL = 2 the loads
// and stores are bf16x2.  src is [M, 3, H, hd]; dst is [M, 3, H, hdp] (may be src itself
// when hdp == hd, in which case v is left untouched).

template <int PPL>
__device__ __forceinline__ void ld_pairs(const __nv_bfloat16* p, int i, int half, float* a, float* b) {
  if (PPL == 2) {
    if (i < half) {
      const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(p + i);
      const __nv_bfloat162 y = *reinterpret_cast<const __nv_bfloat162*>(p + half + i);
      a[0] = __low2float(x); a[1] = __high2float(x);
      b[0] = __low2float(y); b[1] = __high2float(y);
    } else {
      a[0] = a[1] = b[0] = b[1] = 0.f;
    }
  } else {
    a[0] = i < half ? __bfloat162float(p[i]) : 0.f;
    b[0] = i < half ? __bfloat162float(p[half + i]) : 0.f;
  }
}

template <int PPL>
__device__ __forceinline__ void st_pairs(__nv_bfloat16* p, int i, int half, const float* a, const float* b) {
  if (i >= half) return;
  if (PPL == 2) {
    *reinterpret_cast<__nv_bfloat162*>(p + i) = __floats2bfloat162_rn(a[0], a[1]);
    *reinterpret_cast<__nv_bfloat162*>(p + half + i) = __floats2bfloat162_rn(b[0], b[1]);
  } else {
    p[i] = __float2bfloat16_rn(a[0]);
    p[half + i] = __float2bfloat16_rn(b[0]);
  }
}

// Every load of a (token, head) item is issued before its reductions and stores, so a warp
// keeps several independent loads in flight (the in-place form would otherwise stop the
// compiler from hoisting them past the stores).
template <int PPL>
__global__ void qk_fwd_kernel(const __nv_bfloat16* __restrict__ src, const float2* __restrict__ cs, int M, int T,
                              int H, int hd, int hdp, int rope, int qk_norm, float eps, __nv_bfloat16* dst,
                              float* __restrict__ rq, float* __restrict__ rk, int in_place) {
  pdl_trigger();
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  const int half = hd / 2;
  const int i = lane * PPL;
  const long long D = (long long)H * hd;
  const int total = M * H;
  for (int wid = blockIdx.x * warps + (threadIdx.x >> 5); wid < total; wid += gridDim.x * warps) {
    const int m = wid / H, h = wid - (wid / H) * H;
    const int t = m % T;
    const __nv_bfloat16* sp = src + (long long)m * 3 * D + (long long)h * hd;
    __nv_bfloat16* dp = dst + (long long)m * 3 * H * hdp + (long long)h * hdp;
    float a[3][PPL], b[3][PPL];
    ld_pairs<PPL>(sp, i, half, a[0], b[0]);
    ld_pairs<PPL>(sp + D, i, half, a[1], b[1]);
    if (!in_place) ld_pairs<PPL>(sp + 2 * D, i, half, a[2], b[2]);
    float2 e[PPL];
#pragma unroll
    for (int j = 0; j < PPL; ++j)
      e[j] = (rope && i + j < half) ? cs[(long long)t * half + i + j] : make_float2(1.f, 0.f);
#pragma unroll
    for (int sct = 0; sct < 2; ++sct) {
      float r = 1.f;
      if (qk_norm) {
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < PPL; ++j) ss += a[sct][j] * a[sct][j] + b[sct][j] * b[sct][j];
        r = rsqrtf(warp_sum(ss) / hd + eps);
        if (lane == 0) (sct == 0 ? rq : rk)[(long long)m * H + h] = r;
      }
#pragma unroll
      for (int j = 0; j < PPL; ++j) {
        const float x1 = a[sct][j], x2 = b[sct][j];
        a[sct][j] = (x1 * e[j].x - x2 * e[j].y) * r;
        b[sct][j] = (x1 * e[j].y + x2 * e[j].x) * r;
      }
    }
    st_pairs<PPL>(dp, i, half, a[0], b[0]);
    st_pairs<PPL>(dp + (long long)H * hdp, i, half, a[1], b[1]);
    if (!in_place) st_pairs<PPL>(dp + 2LL * H * hdp, i, half, a[2], b[2]);
  }
}

template <int PPL>
__global__ void qk_bwd_kernel(const __nv_bfloat16* dpad, const __nv_bfloat16* __restrict__ qpad,
                              const float* __restrict__ rq, const float* __restrict__ rk,
                              const float2* __restrict__ cs, int M, int T, int H, int hd, int hdp, int rope,
                              int qk_norm, __nv_bfloat16* dqkv) {
  pdl_trigger();
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  const int half = hd / 2;
  const int i = lane * PPL;
  const long long D = (long long)H * hd;
  const bool in_place = (const void*)dpad == (const void*)dqkv;
  const int total = M * H;
  for (int wid = blockIdx.x * warps + (threadIdx.x >> 5); wid < total; wid += gridDim.x * warps) {
    const int m = wid / H, h = wid - (wid / H) * H;
    const int t = m % T;
    const long long po = (long long)m * 3 * H * hdp + (long long)h * hdp;
    const long long ps = (long long)H * hdp;  // section pitch in the padded layout
    float a[3][PPL], b[3][PPL], ya[2][PPL], yb[2][PPL];
    ld_pairs<PPL>(dpad + po, i, half, a[0], b[0]);
    ld_pairs<PPL>(dpad + po + ps, i, half, a[1], b[1]);
    if (!in_place) ld_pairs<PPL>(dpad + po + 2 * ps, i, half, a[2], b[2]);
    if (qk_norm) {
      ld_pairs<PPL>(qpad + po, i, half, ya[0], yb[0]);
      ld_pairs<PPL>(qpad + po + ps, i, half, ya[1], yb[1]);
    }
    float r2[2] = {1.f, 1.f};
    if (qk_norm) {
      r2[0] = rq[(long long)m * H + h];
      r2[1] = rk[(long long)m * H + h];
    }
    float2 e[PPL];
#pragma unroll
    for (int j = 0; j < PPL; ++j)
      e[j] = (rope && i + j < half) ? cs[(long long)t * half + i + j] : make_float2(1.f, 0.f);
#pragma unroll
    for (int sct = 0; sct < 2; ++sct) {
      if (qk_norm) {
        // dx = r (dy - y mean(dy y)), y the normalised output that the forward saved
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < PPL; ++j) s += a[sct][j] * ya[sct][j] + b[sct][j] * yb[sct][j];
        const float mdy = warp_sum(s) / hd;
#pragma unroll
        for (int j = 0; j < PPL; ++j) {
          a[sct][j] = r2[sct] * (a[sct][j] - ya[sct][j] * mdy);
          b[sct][j] = r2[sct] * (b[sct][j] - yb[sct][j] * mdy);
        }
      }
      // the rotation is orthogonal: its reverse rotates by -phi
#pragma unroll
      for (int j = 0; j < PPL; ++j) {
        const float x1 = a[sct][j], x2 = b[sct][j];
        a[sct][j] = x1 * e[j].x + x2 * e[j].y;
        b[sct][j] = -x1 * e[j].y + x2 * e[j].x;
      }
    }
    __nv_bfloat16* dst = dqkv + (long long)m * 3 * D + (long long)h * hd;
    st_pairs<PPL>(dst, i, half, a[0], b[0]);
    st_pairs<PPL>(dst + D, i, half, a[1], b[1]);
    if (!in_place) st_pairs<PPL>(dst + 2 * D, i, half, a[2], b[2]);
  }
}

int launch_qk_fwd(const __nv_bfloat16* qkv, const float2* rope_cs, int M, int T, int H, int hd, int hdp, int rope,
                  int qk_norm, float eps, __nv_bfloat16* qkv_pad, float* rstd_q, float* rstd_k, cudaStream_t st) {
  if (hd % 2) return set_error(ST_UNSUPPORTED, "head_dim must be even");
  const int in_place = (const void*)qkv == (const void*)qkv_pad;
  if (in_place && hdp != hd) return set_error(ST_INVALID_ARG, "qk_fwd: in place needs an unpadded layout");
  long long work = (long long)M * H;
  int grid = cdiv(work, 8);
  if (grid > num_sms() * 32) grid = num_sms() * 32;
  Prof prof(PK_QK, 0, (double)M * (in_place ? 2 : 3) * H * hd * 4, st);
  if (hd <= 64)
    qk_fwd_kernel<1><<<grid, 256, 0, st>>>(qkv, rope_cs, M, T, H, hd, hdp, rope, qk_norm, eps, qkv_pad, rstd_q, rstd_k,
                                           in_place);
  else if (hd <= 128)
    qk_fwd_kernel<2><<<grid, 256, 0, st>>>(qkv, rope_cs, M, T, H, hd, hdp, rope, qk_norm, eps, qkv_pad, rstd_q, rstd_k,
                                           in_place);
  else
    return set_error(ST_UNSUPPORTED, "head_dim above 128");
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

// In-place QK-norm / RoPE backward for 64- or 128-wide unpadded heads: HD / 8 lanes per
// (token, head) item, each lane four consecutive pairs (i .. i+3 with i + HD/2 ..), 8-byte loads
// and stores, a segmented shuffle reduction; v is left as it is.
template <int HD>
__global__ void qk_bwd_vec_kernel(__nv_bfloat16* __restrict__ dqkv, const __nv_bfloat16* __restrict__ qpad,
                                  const float* __restrict__ rq, const float* __restrict__ rk,
                                  const float2* __restrict__ cs, int M, int T, int H, int rope, int qk_norm) {
  pdl_trigger();
  constexpr int HALF = HD / 2;
  constexpr int LPI = HD / 8;
  constexpr int IPW = 32 / LPI;
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPI, l8 = lane % LPI;
  const int i = 4 * l8;
  const long long total = (long long)M * H;
  const long long ps = (long long)H * HD;  // q -> k section pitch
  for (long long base = ((long long)blockIdx.x * warps + (threadIdx.x >> 5)) * IPW; base < total;
       base += (long long)gridDim.x * warps * IPW) {
    const long long w = base + sub;
    const bool live = w < total;
    const long long m = live ? w / H : 0;
    const int h = live ? (int)(w - m * H) : 0;
    const long long po = m * 3 * ps + (long long)h * HD;
    float a[2][4], b[2][4], ya[2][4], yb[2][4];
    auto ld4 = [&](const __nv_bfloat16* p, float* v) {
      const uint2 x = live ? __ldg(reinterpret_cast<const uint2*>(p)) : make_uint2(0u, 0u);
      v[0] = __uint_as_float(x.x << 16);
      v[1] = __uint_as_float(x.x & 0xffff0000u);
      v[2] = __uint_as_float(x.y << 16);
      v[3] = __uint_as_float(x.y & 0xffff0000u);
    };
#pragma unroll
    for (int sct = 0; sct < 2; ++sct) {
      ld4(dqkv + po + sct * ps + i, a[sct]);
      ld4(dqkv + po + sct * ps + HALF + i, b[sct]);
      if (qk_norm) {
        ld4(qpad + po + sct * ps + i, ya[sct]);
        ld4(qpad + po + sct * ps + HALF + i, yb[sct]);
      }
    }
    float2 e[4];
    if (rope && live) {
      const float4* c4 = reinterpret_cast<const float4*>(cs + (long long)(m % T) * HALF + i);
      const float4 c0 = __ldg(c4), c1 = __ldg(c4 + 1);
      e[0] = make_float2(c0.x, c0.y);
      e[1] = make_float2(c0.z, c0.w);
      e[2] = make_float2(c1.x, c1.y);
      e[3] = make_float2(c1.z, c1.w);
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) e[k] = make_float2(1.f, 0.f);
    }
    const float r2[2] = {(qk_norm && live) ? rq[m * H + h] : 1.f, (qk_norm && live) ? rk[m * H + h] : 1.f};
#pragma unroll
    for (int sct = 0; sct < 2; ++sct) {
      if (qk_norm) {
        // dx = r (dy - y mean(dy y)), y the normalised output that the forward saved
        float sm = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) sm += a[sct][k] * ya[sct][k] + b[sct][k] * yb[sct][k];
#pragma unroll
        for (int off = LPI / 2; off > 0; off >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, off);
        const float mdy = sm * (1.f / HD);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          a[sct][k] = r2[sct] * (a[sct][k] - ya[sct][k] * mdy);
          b[sct][k] = r2[sct] * (b[sct][k] - yb[sct][k] * mdy);
        }
      }
      // the rotation is orthogonal: its reverse rotates by -phi
      uint32_t wa[2], wb[2];
#pragma unroll
      for (int k2 = 0; k2 < 2; ++k2) {
        float oa[2], ob[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int k = 2 * k2 + q;
          oa[q] = a[sct][k] * e[k].x + b[sct][k] * e[k].y;
          ob[q] = -a[sct][k] * e[k].y + b[sct][k] * e[k].x;
        }
        wa[k2] = pack_bf16x2(oa[0], oa[1]);
        wb[k2] = pack_bf16x2(ob[0], ob[1]);
      }
      if (live) {
        *reinterpret_cast<uint2*>(dqkv + po + sct * ps + i) = make_uint2(wa[0], wa[1]);
        *reinterpret_cast<uint2*>(dqkv + po + sct * ps + HALF + i) = make_uint2(wb[0], wb[1]);
      }
    }
  }
}

int launch_qk_bwd(const __nv_bfloat16* dqkv_pad, const __nv_bfloat16* qkv_pad, const float* rstd_q,
                  const float* rstd_k, const float2* rope_cs, int M, int T, int H, int hd, int hdp, int rope,
                  int qk_norm, __nv_bfloat16* dqkv, cudaStream_t st) {
  if (hd % 2) return set_error(ST_UNSUPPORTED, "head_dim must be even");
  if ((const void*)dqkv_pad == (const void*)dqkv && hdp != hd)
    return set_error(ST_INVALID_ARG, "qk_bwd: in place needs an unpadded layout");
  long long work = (long long)M * H;
  if ((hd == 64 || hd == 128) && hdp == hd && (const void*)dqkv_pad == (const void*)dqkv) {
    // in place, unpadded: the vectorised form (v needs nothing)
    const int ipb = 8 * (32 / (hd / 8));  // items per 256-thread block and pass
    long long grid = (work + ipb - 1) / ipb;
    if (grid > (long long)num_sms() * 32) grid = num_sms() * 32;
    Prof prof(PK_QK, 0, (double)M * 2 * H * hd * 4 + (qk_norm ? (double)M * 2 * H * hd * 2 : 0), st);
    if (hd == 128)
      qk_bwd_vec_kernel<128><<<(int)grid, 256, 0, st>>>(dqkv, qkv_pad, rstd_q, rstd_k, rope_cs, M, T, H, rope, qk_norm);
    else
      qk_bwd_vec_kernel<64><<<(int)grid, 256, 0, st>>>(dqkv, qkv_pad, rstd_q, rstd_k, rope_cs, M, T, H, rope, qk_norm);
    GPTK_CUDA(cudaGetLastError());
    return ST_OK;
  }
  int grid = cdiv(work, 8);
  if (grid > num_sms() * 32) grid = num_sms() * 32;
  Prof prof(PK_QK, 0, (double)M * 3 * H * hd * 4 + (qk_norm ? (double)M * 2 * H * hd * 2 : 0), st);
  if (hd <= 64)
    qk_bwd_kernel<1><<<grid, 256, 0, st>>>(dqkv_pad, qkv_pad, rstd_q, rstd_k, rope_cs, M, T, H, hd, hdp, rope, qk_norm,
                                           dqkv);
  else if (hd <= 128)
    qk_bwd_kernel<2><<<grid, 256, 0, st>>>(dqkv_pad, qkv_pad, rstd_q, rstd_k, rope_cs, M, T, H, hd, hdp, rope, qk_norm,
                                           dqkv);
  else
    return set_error(ST_UNSUPPORTED, "head_dim above 128");
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

// ------------------------------------------------------------------ attention delta

// delta[b, h, t] = sum_d o[m, h hd + d] * dO[m, h hdp + d]: hd / 32 lanes per (token, head) item,
// each lane 32 elements of o and of dO in four 16-byte loads each (all eight issued first), a
// segmented shuffle reduction; 32 / (hd / 32) items per warp and pass.
template <int HD>
__global__ void attn_delta_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dpad, int B,
                                  int T, int H, int hdp, float* __restrict__ delta) {
  pdl_trigger();
  constexpr int LPI = HD / 32;  // lanes per item
  constexpr int IPW = 32 / LPI;
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPI, l8 = lane % LPI;
  const long long total = (long long)B * T * H;
  for (long long base = ((long long)blockIdx.x * warps + (threadIdx.x >> 5)) * IPW; base < total;
       base += (long long)gridDim.x * warps * IPW) {
    const long long w = base + sub;
    float s = 0.f;
    if (w < total) {
      const long long m = w / H;
      const int h = (int)(w - m * H);
      const uint4* ap = reinterpret_cast<const uint4*>(o + m * H * HD + (long long)h * HD) + 4 * l8;
      const uint4* dp = reinterpret_cast<const uint4*>(dpad + m * H * hdp + (long long)h * hdp) + 4 * l8;
      uint4 a[4], d[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = __ldg(ap + u);
        d[u] = __ldg(dp + u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t av[4] = {a[u].x, a[u].y, a[u].z, a[u].w}, dv[4] = {d[u].x, d[u].y, d[u].z, d[u].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          s = fmaf(__uint_as_float(av[k] << 16), __uint_as_float(dv[k] << 16), s);
          s = fmaf(__uint_as_float(av[k] & 0xffff0000u), __uint_as_float(dv[k] & 0xffff0000u), s);
        }
      }
    }
#pragma unroll
    for (int off = LPI / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (l8 == 0 && w < total) {
      const long long m = w / H;
      const int h = (int)(w - m * H);
      const long long b = m / T, t = m % T;
      delta[(b * H + h) * T + t] = s;
    }
  }
}

// any even head dim: one warp per (token, head)
__global__ void attn_delta_generic_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dpad,
                                          int B, int T, int H, int hd, int hdp, float* __restrict__ delta) {
  pdl_trigger();
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total = B * T * H;
  for (int wid = blockIdx.x * warps + (threadIdx.x >> 5); wid < total; wid += gridDim.x * warps) {
    const long long m = wid / H;
    const int h = wid - (wid / H) * H;
    const __nv_bfloat16* orow = o + m * H * hd + (long long)h * hd;
    const __nv_bfloat16* drow = dpad + m * H * hdp + (long long)h * hdp;
    float s = 0.f;
    for (int d = lane; d < hd; d += 32) s += __bfloat162float(orow[d]) * __bfloat162float(drow[d]);
    s = warp_sum(s);
    if (lane == 0) {
      const long long b = m / T, t = m % T;
      delta[(b * H + h) * T + t] = s;
    }
  }
}

int launch_attn_delta(const __nv_bfloat16* o, const __nv_bfloat16* do_pad, int B, int T, int H, int hd, int hdp,
                      float* delta, cudaStream_t st) {
  if (hd != 64 && hd != 128) {
    long long work = (long long)B * T * H;
    int grid = cdiv(work, 8);
    if (grid > num_sms() * 16) grid = num_sms() * 16;
    Prof prof(PK_DELTA, 0, (double)B * T * H * (hd * 2 + hdp * 2 + 4), st);
    attn_delta_generic_kernel<<<grid, 256, 0, st>>>(o, do_pad, B, T, H, hd, hdp, delta);
    GPTK_CUDA(cudaGetLastError());
    return ST_OK;
  }
  const long long items = (long long)B * T * H;
  const int ipb = 8 * (hd == 128 ? 8 : 16);  // items per 256-thread block and pass
  long long grid = (items + ipb - 1) / ipb;
  if (grid > (long long)num_sms() * 16) grid = num_sms() * 16;
  Prof prof(PK_DELTA, 0, (double)B * T * H * (hd * 2 + hdp * 2 + 4), st);
  if (hd == 128) attn_delta_kernel<128><<<(int)grid, 256, 0, st>>>(o, do_pad, B, T, H, hdp, delta);
  else attn_delta_kernel<64><<<(int)grid, 256, 0, st>>>(o, do_pad, B, T, H, hdp, delta);
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

// ------------------------------------------------------------------ initialisation
// SplitMix64 (Steele, Lea, Flood 2014): output n of the stream seeded with s is
// mix(s + (n+1) * golden_gamma).  Element i takes outputs 2i and 2i+1, turns their top
// 24 bits into u1 in (0,1] and u2 in [0,1), and Box-Muller gives sqrt(-2 ln u1) cos(2 pi u2).

__device__ __forceinline__ unsigned long long splitmix64_at(unsigned long long seed, unsigned long long n) {
  unsigned long long z = seed + (n + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void init_normal_kernel(float* __restrict__ p, long long off, long long n, unsigned long long seed,
                                   float stdv) {
  for (long long k = blockIdx.x * (long long)blockDim.x + threadIdx.x; k < n; k += (long long)gridDim.x * blockDim.x) {
    const unsigned long long i = static_cast<unsigned long long>(off + k);
    const unsigned long long r0 = splitmix64_at(seed, 2ull * i);
    const unsigned long long r1 = splitmix64_at(seed, 2ull * i + 1ull);
    const double u1 = (static_cast<double>(r0 >> 40) + 1.0) * (1.0 / 16777216.0);
    const double u2 = static_cast<double>(r1 >> 40) * (1.0 / 16777216.0);
    const double z = sqrt(-2.0 * log(u1)) * cospi(2.0 * u2);
    p[off + k] = static_cast<float>(static_cast<double>(stdv) * z);
  }
}

__global__ void fill_kernel(float* p, long long n, float v) {
  for (long long k = blockIdx.x * (long long)blockDim.x + threadIdx.x; k < n; k += (long long)gridDim.x * blockDim.x)
    p[k] = v;
}

int launch_init_normal(float* params, long long off, long long n, unsigned long long seed, float stdv,
                       cudaStream_t st) {
  if (n <= 0) return ST_OK;
  int grid = cdiv(n, 256);
  if (grid > num_sms() * 16) grid = num_sms() * 16;
  Prof prof(PK_MISC, 0, n * 4.0, st);
  init_normal_kernel<<<grid, 256, 0, st>>>(params, off, n, seed, stdv);
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

__global__ void sum_parts_kernel(const float* __restrict__ parts, int n_parts, size_t stride, size_t n4,
                                 float* __restrict__ out) {
  pdl_trigger();
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
    float4 a = reinterpret_cast<const float4*>(parts)[i];
    for (int p = 1; p < n_parts; ++p) {
      const float4 b = reinterpret_cast<const float4*>(parts + (size_t)p * stride)[i];
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    reinterpret_cast<float4*>(out)[i] = a;
  }
}

int launch_sum_parts(const float* parts, int n_parts, size_t stride, size_t n, float* out, cudaStream_t st) {
  if (n % 4 || stride % 4) return set_error(ST_INVALID_ARG, "sum_parts: sizes must be multiples of 4");
  int grid = (int)cdiv((long long)(n / 4), 256);
  if (grid > num_sms() * 8) grid = num_sms() * 8;
  Prof prof(PK_MISC, 0, (double)n * 4 * (n_parts + 1), st);
  sum_parts_kernel<<<grid, 256, 0, st>>>(parts, n_parts, stride, n / 4, out);
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

int launch_fill(float* p, long long n, float value, cudaStream_t st) {
  if (n <= 0) return ST_OK;
  int grid = cdiv(n, 256);
  if (grid > num_sms() * 16) grid = num_sms() * 16;
  Prof prof(PK_MISC, 0, n * 4.0, st);
  fill_kernel<<<grid, 256, 0, st>>>(p, n, value);
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

}  // namespace gptk
