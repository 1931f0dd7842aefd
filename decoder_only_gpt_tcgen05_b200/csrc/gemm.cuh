// Persistent tcgen05 GEMM for sm_100a:  C[M,N] = A[M,K] * B[N,K]^T  (bf16 in, fp32 accumulate).
//
// One CTA per SM walks output tiles of 128 x BN.  Warp roles:
//   warp 0      TMA producer: stages 128x64 A and BNx64 B tiles (128-byte swizzle) into a ring
//   warp 1      one thread issues tcgen05.mma (M=128, N=BN, K=16 per instruction); owns TMEM
//   warps 2..5  epilogue: tcgen05.ld the accumulator rows (one row per thread) and apply the
//               fused epilogue of the call (norm scale, bias, RoPE, QK-norm, residual add,
//               activation, activation gradient, cross-entropy partials or gradient)
// The accumulator is double buffered in tensor memory (2 x BN columns) so the epilogue of one
// tile overlaps the main loop of the next.
//
// Either operand may be K-major (rows of K contiguous elements: the usual [out,in] weight and
// [tokens,features] activation layouts) or MN-major (M or N contiguous: what the gradient GEMMs
// of a linear layer need), so forward, data-gradient and weight-gradient products all run on
// this one kernel without any transpose copies.
#pragma once

#include "ptx.cuh"

namespace gptk {

enum EpiKind : int {
  EPI_BF16 = 0,     // out bf16 = acc (+ bias), optional head-padded column map
  EPI_F32 = 1,      // out fp32 = acc (+ bias)  or  out += acc  (accumulate)
  EPI_RESID = 2,    // out fp32 = resid + acc (+ bias)
  EPI_QKV = 3,      // q,k,v bf16 (head padded), + bias, RoPE, per-head RMSNorm of q and k
  EPI_UP = 4,       // u = acc (+ bias) -> u bf16, h = act(u) bf16
  EPI_ACTBWD = 5,   // out bf16 = acc * act'(u)
  EPI_CE_FWD = 6,   // per-row (max, sum exp) partials over this tile's vocab columns + target logit
  EPI_CE_BWD = 7,   // out bf16 = (softmax - onehot) * scale
};

struct GemmParams {
  int M, N, K;
  int a_mn, b_mn;             // 1 = operand stored MN-major
  int tiles_m, tiles_n;
  DevCtl ctl;
  // generic output
  void* out;
  long long ldo;
  const float* bias;          // [N] or nullptr
  int accumulate;             // EPI_F32
  const float* resid;         // EPI_RESID
  long long ldr;
  void* out2;                 // EPI_UP: h
  const __nv_bfloat16* aux;   // EPI_ACTBWD: u
  long long ld_aux;
  int act;                    // 0 GELU(erf), 1 ReLU^2
  // head-padded layout of q/k/v (and of attention-gradient inputs): column c of a D-wide
  // block maps to (c / hd) * hdp + c % hd
  int hd, hdp;
  // QKV epilogue
  int d_model, n_head, T;
  int rope, qk_norm;
  float eps;
  const float2* rope_cs;      // [T][hd/2] (cos, sin)
  float* rstd_q;              // [M][H]
  float* rstd_k;
  // cross-entropy
  const int* targets;         // [M]
  float2* ce_part;            // [M][tiles_n]  (max log2, sum exp2)
  float* ce_zy;               // [M] target logit
  const float* ce_lse;        // [M] natural-log logsumexp (backward)
  float ce_scale;             // 1/M_total (backward)
};

template <int BN>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BK = 64;
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static constexpr int THREADS = 192;
};

// --------------------------------------------------------------- epilogue helpers

__device__ __forceinline__ float act_fwd(float u, int act) {
  if (act == 1) {
    float r = fmaxf(u, 0.f);
    return r * r;
  }
  return 0.5f * u * (1.f + erff(u * 0.70710678118654752f));
}

__device__ __forceinline__ float act_grad(float u, int act) {
  if (act == 1) return 2.f * fmaxf(u, 0.f);
  // d/du of 0.5 u (1 + erf(u/sqrt2)) = 0.5 (1 + erf(u/sqrt2)) + u * exp(-u^2/2) / sqrt(2 pi)
  return 0.5f * (1.f + erff(u * 0.70710678118654752f)) + u * expf(-0.5f * u * u) * 0.3989422804014327f;
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d[q] = w;
  }
}

__device__ __forceinline__ void add_bias32(float (&v)[32], const float* bias, int col0, int N) {
  if (bias == nullptr) return;
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (col0 + j < N) v[j] += __ldg(bias + col0 + j);
}

// Plain column-chunk epilogues: one 32-column chunk of one row.
template <int EPI>
__device__ __forceinline__ void epi_chunk(const GemmParams& p, float (&v)[32], int row, int col0, bool row_ok) {
  const bool full = (col0 + 32 <= p.N);
  if (EPI == EPI_BF16) {
    add_bias32(v, p.bias, col0, p.N);
    if (!row_ok) return;
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) + (long long)row * p.ldo;
    if (p.hd == p.hdp && full && (p.ldo % 8) == 0) {
      store_bf16x32(out + col0, v);
    } else {
      for (int j = 0; j < 32; ++j) {
        int c = col0 + j;
        if (c < p.N) out[(c / p.hd) * p.hdp + c % p.hd] = __float2bfloat16_rn(v[j]);
      }
    }
  } else if (EPI == EPI_F32) {
    add_bias32(v, p.bias, col0, p.N);
    if (!row_ok) return;
    float* out = reinterpret_cast<float*>(p.out) + (long long)row * p.ldo;
    if (full && (p.ldo % 4) == 0) {
      float4* o4 = reinterpret_cast<float4*>(out + col0);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float4 w = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        if (p.accumulate) {
          float4 o = o4[q];
          w.x += o.x; w.y += o.y; w.z += o.z; w.w += o.w;
        }
        o4[q] = w;
      }
    } else {
      for (int j = 0; j < 32; ++j) {
        int c = col0 + j;
        if (c < p.N) out[c] = p.accumulate ? out[c] + v[j] : v[j];
      }
    }
  } else if (EPI == EPI_RESID) {
    add_bias32(v, p.bias, col0, p.N);
    if (!row_ok) return;
    float* out = reinterpret_cast<float*>(p.out) + (long long)row * p.ldo;
    const float* res = p.resid + (long long)row * p.ldr;
    if (full && (p.ldo % 4) == 0 && (p.ldr % 4) == 0) {
      float4* o4 = reinterpret_cast<float4*>(out + col0);
      const float4* r4 = reinterpret_cast<const float4*>(res + col0);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float4 r = r4[q];
        o4[q] = make_float4(r.x + v[4 * q], r.y + v[4 * q + 1], r.z + v[4 * q + 2], r.w + v[4 * q + 3]);
      }
    } else {
      for (int j = 0; j < 32; ++j) {
        int c = col0 + j;
        if (c < p.N) out[c] = res[c] + v[j];
      }
    }
  } else if (EPI == EPI_UP) {
    add_bias32(v, p.bias, col0, p.N);
    if (!row_ok) return;
    __nv_bfloat16* u = reinterpret_cast<__nv_bfloat16*>(p.out) + (long long)row * p.ldo;
    __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(p.out2) + (long long)row * p.ldo;
    float hv[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) hv[j] = act_fwd(v[j], p.act);
    if (full && (p.ldo % 8) == 0) {
      store_bf16x32(u + col0, v);
      store_bf16x32(h + col0, hv);
    } else {
      for (int j = 0; j < 32; ++j) {
        int c = col0 + j;
        if (c < p.N) {
          u[c] = __float2bfloat16_rn(v[j]);
          h[c] = __float2bfloat16_rn(hv[j]);
        }
      }
    }
  } else if (EPI == EPI_ACTBWD) {
    if (!row_ok) return;
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) + (long long)row * p.ldo;
    const __nv_bfloat16* u = p.aux + (long long)row * p.ld_aux;
    if (full && (p.ldo % 8) == 0 && (p.ld_aux % 8) == 0) {
      const uint4* u4 = reinterpret_cast<const uint4*>(u + col0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 w = u4[q];
        const __nv_bfloat16* ub = reinterpret_cast<const __nv_bfloat16*>(&w);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[8 * q + e] *= act_grad(__bfloat162float(ub[e]), p.act);
      }
      store_bf16x32(out + col0, v);
    } else {
      for (int j = 0; j < 32; ++j) {
        int c = col0 + j;
        if (c < p.N) out[c] = __float2bfloat16_rn(v[j] * act_grad(__bfloat162float(u[c]), p.act));
      }
    }
  } else if (EPI == EPI_CE_BWD) {
    if (!row_ok) return;
    const float lse2 = p.ce_lse[row] * 1.4426950408889634f;
    const int y = p.targets[row];
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) + (long long)row * p.ldo;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      int c = col0 + j;
      float g = ex2_approx(fmaf(v[j], 1.4426950408889634f, -lse2));
      if (c == y) g -= 1.f;
      v[j] = g * p.ce_scale;
    }
    if (full && (p.ldo % 8) == 0) {
      store_bf16x32(out + col0, v);
    } else {
      for (int j = 0; j < 32; ++j)
        if (col0 + j < p.N) out[col0 + j] = __float2bfloat16_rn(v[j]);
    }
  }
}

// QKV epilogue for one head of q or k: RoPE on pairs (i, i + hd/2), then per-head RMSNorm.
// taddr points at this thread's row, column of the head's first element.
__device__ __forceinline__ void epi_qk_head(const GemmParams& p, uint32_t taddr, int row, bool row_ok, int col,
                                            int sect, int head) {
  const int hd = p.hd;
  const float* bias = p.bias ? p.bias + col : nullptr;
  float rstd = 1.f;
  if (p.qk_norm) {
    float ss = 0.f;
    for (int c = 0; c < hd; c += 32) {
      float v[32];
      tmem_ld32(taddr + c, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float x = v[j] + (bias ? __ldg(bias + c + j) : 0.f);
        ss = fmaf(x, x, ss);
      }
    }
    rstd = rsqrtf(ss / (float)hd + p.eps);
    if (row_ok) (sect == 0 ? p.rstd_q : p.rstd_k)[(long long)row * p.n_head + head] = rstd;
  }
  const int half = hd / 2;
  const int t = row % p.T;
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) + (long long)row * p.ldo +
                       (long long)sect * p.n_head * p.hdp + (long long)head * p.hdp;
  for (int c = 0; c < half; c += 32) {
    float x1[32], x2[32];
    tmem_ld32(taddr + c, x1);
    tmem_ld32(taddr + half + c, x2);
    if (bias) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        x1[j] += __ldg(bias + c + j);
        x2[j] += __ldg(bias + half + c + j);
      }
    }
    if (p.rope) {
      const float2* cs = p.rope_cs + (long long)t * half + c;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float2 e = __ldg(cs + j);
        float a = x1[j], b = x2[j];
        x1[j] = (a * e.x - b * e.y) * rstd;
        x2[j] = (a * e.y + b * e.x) * rstd;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        x1[j] *= rstd;
        x2[j] *= rstd;
      }
    }
    if (row_ok) {
      store_bf16x32(out + c, x1);
      store_bf16x32(out + half + c, x2);
    }
  }
}

// --------------------------------------------------------------- the kernel

template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ GemmParams p) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = bars + 2 * C::STAGES + 2;
  uint64_t* drain = bars + 2 * C::STAGES + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = p.tiles_m * p.tiles_n;
  const int num_k = (p.K + C::BK - 1) / C::BK;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t pending = 0;  // stages with a load in flight that the MMA has not yet released
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int tm = tile % p.tiles_m;
      const int tn = tile / p.tiles_m;
      for (int kb = 0; kb < num_k; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, p.ctl, abort_flag, 1)) {
          ok = false;
          break;
        }
        pending &= ~(1u << stage);
        mbar_expect_tx(&full[stage], C::STAGE_BYTES);
        uint8_t* a = sA + stage * C::A_BYTES;
        uint8_t* b = sB + stage * C::B_BYTES;
        if (!p.a_mn) {
          tma_load_2d(a, &tmA, &full[stage], kb * C::BK, tm * C::BM);
        } else {
#pragma unroll
          for (int c = 0; c < C::BM / 64; ++c) tma_load_2d(a + c * 8192, &tmA, &full[stage], tm * C::BM + c * 64, kb * C::BK);
        }
        if (!p.b_mn) {
          tma_load_2d(b, &tmB, &full[stage], kb * C::BK, tn * BN);
        } else {
#pragma unroll
          for (int c = 0; c < BN / 64; ++c) tma_load_2d(b + c * 8192, &tmB, &full[stage], tn * BN + c * 64, kb * C::BK);
        }
        pending |= 1u << stage;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) {
      // drain the copies still in flight before the CTA goes away (bounded as well)
      DevCtl c2 = p.ctl;
      volatile int never = 0;
      for (int s = 0; s < C::STAGES; ++s) {
        if (!(pending & (1u << s))) continue;
        // stage s was issued in the current or the previous lap of the ring
        uint32_t ph = (s < stage) ? phase : (phase ^ 1u);
        mbar_wait(&full[s], ph, c2, &never, 2);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------ MMA issuer
    constexpr uint32_t IDESC_KK = idesc_bf16(128, BN, 0, 0);
    const uint32_t idesc = IDESC_KK | (static_cast<uint32_t>(p.a_mn) << 15) | (static_cast<uint32_t>(p.b_mn) << 16);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    bool issued = false;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, p.ctl, abort_flag, 3)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int kb = 0; kb < num_k; ++kb) {
        if (!mbar_wait(&full[stage], phase, p.ctl, abort_flag, 4)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + stage * C::A_BYTES);
        const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::BK / 16; ++kk) {
          const uint64_t ad = p.a_mn ? sdesc_sw128(a0 + kk * 2048, 8192, 1024) : sdesc_sw128(a0 + kk * 32, 16, 1024);
          const uint64_t bd = p.b_mn ? sdesc_sw128(b0 + kk * 2048, 8192, 1024) : sdesc_sw128(b0 + kk * 32, 16, 1024);
          umma_bf16(d_tmem, ad, bd, idesc, (kb | kk) != 0);
        }
        umma_commit(&empty[stage]);
        issued = true;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      umma_commit(&tfull[acc]);
      issued = true;
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (!ok && issued) {
      // let the MMAs already issued finish before tensor memory is released
      volatile int never = 0;
      umma_commit(drain);
      mbar_wait(drain, 0, p.ctl, &never, 6);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int r_in_tile = quad * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int tm = tile % p.tiles_m;
      const int tn = tile / p.tiles_m;
      if (!mbar_wait(&tfull[acc], acc_phase, p.ctl, abort_flag, 5)) break;
      tc_fence_after();
      const int row = tm * 128 + r_in_tile;
      const bool row_ok = row < p.M;
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * BN;
      const int n0 = tn * BN;
      if (EPI == EPI_QKV) {
        const int D = p.d_model;
        // a tile never straddles q/k/v sections when hd divides BN and D
        for (int c = 0; c < BN; c += 32) {
          const int col = n0 + c;
          if (col >= p.N) break;
          const int sect = col / D;
          const int within = col - sect * D;
          if (sect < 2 && (p.rope || p.qk_norm)) {
            if (within % p.hd == 0 && c + p.hd <= BN) {
              epi_qk_head(p, trow + c, row, row_ok, col, sect, within / p.hd);
            }
            continue;  // columns of a head are handled by the head's first chunk
          }
          float v[32];
          tmem_ld32(trow + c, v);
          add_bias32(v, p.bias, col, p.N);
          if (row_ok) {
            __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) + (long long)row * p.ldo;
            for (int j = 0; j < 32; ++j) {
              const int cc = col + j;
              if (cc >= p.N) break;
              const int s = cc / D, w = cc - s * D;
              out[(long long)s * p.n_head * p.hdp + (w / p.hd) * p.hdp + (w % p.hd)] = __float2bfloat16_rn(v[j]);
            }
          }
        }
      } else if (EPI == EPI_CE_FWD) {
        const int y = row_ok ? p.targets[row] : -1;
        float m2 = -INFINITY, s = 0.f;
        for (int c = 0; c < BN; c += 32) {
          float v[32];
          tmem_ld32(trow + c, v);
          const int col0 = n0 + c;
          float cm = -INFINITY;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            v[j] = (col0 + j < p.N) ? v[j] * 1.4426950408889634f : -INFINITY;
            cm = fmaxf(cm, v[j]);
          }
          if (y >= col0 && y < col0 + 32 && row_ok) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j == y) p.ce_zy[row] = v[j] * 0.6931471805599453f;
          }
          if (cm != -INFINITY) {
            const float mn = fmaxf(m2, cm);
            float cs = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) cs += ex2_approx(v[j] - mn);
            s = s * ex2_approx(m2 - mn) + cs;
            m2 = mn;
          }
        }
        if (row_ok) p.ce_part[(long long)row * p.tiles_n + tn] = make_float2(m2, s);
      } else {
        for (int c = 0; c < BN; c += 32) {
          float v[32];
          tmem_ld32(trow + c, v);
          epi_chunk<EPI>(p, v, row, n0 + c, row_ok);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * BN);
  }
}

}  // namespace gptk
