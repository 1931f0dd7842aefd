// Persistent tcgen05 GEMM for sm_100a:  C[M,N] = A[M,K] * B[N,K]^T  (bf16 in, fp32 accumulate).
//
// One CTA per SM walks output tiles of 128 x BN.  Warp roles:
//   warp 0      TMA producer: stages 128x64 A and BNx64 B tiles (128-byte swizzle) into a ring
//   warp 1      one thread issues tcgen05.mma (M=128, N=BN, K=16 per instruction); owns TMEM
//   warps 2..9  epilogue: tcgen05.ld the accumulator rows (one row per thread; two warps per
//               TMEM lane quadrant, each taking half of the tile's columns), apply the fused
//               epilogue of the call (bias, residual add, activation, activation gradient,
//               cross-entropy partials or gradient), and write through shared memory with TMA
// The accumulator is double buffered in tensor memory (2 x BN columns) so the epilogue of one
// tile overlaps the main loop of the next.
//
// PAIR variant (cluster of two CTAs on two SMs): the pair walks 256 x BN tiles with one
// tcgen05.mma.cta_group::2 (M = 256) per K step, issued by the even CTA.  Each CTA stages its
// own 128 A rows and its own BN/2 B rows, so a K step moves half the B bytes per SM of the
// single-CTA form and the same shared memory holds a deeper ring.  Both CTAs' TMA loads
// complete on the even CTA's "full" barrier; its MMA commits release both CTAs' stages and
// accumulators; both CTAs' epilogues (each on its own 128 accumulator rows) arrive on the even
// CTA's "tempty" barrier.  Every cross-CTA arrival is waited for before the final cluster
// barrier, so neither CTA leaves while its peer may still touch its shared memory.
//
// Epilogue data path: each epilogue warp owns 32 rows x BN/2 columns and two 4 KB staging buffers.  A chunk of
// 32 fp32 or 64 bf16 columns (128-byte rows) goes registers -> swizzled shared memory -> one TMA
// tile store (or TMA reduce-add for accumulated gradients), so global writes are whole lines.
// Epilogue inputs (the residual stream, the saved pre-activation) arrive the same way by TMA
// load.  Rows and columns past M and N are clipped by the tensor maps.  The fused epilogues:
// bias; residual add (EPI_RESID); activation with the pre-activation kept or not (EPI_UP); its
// gradient (EPI_ACTBWD); RoPE + per-head RMSNorm of q and k on the fp32 accumulator, one 128-wide
// head per epilogue warp of a 256-column tile (EPI_QKV); the per-tile online logsumexp of the
// cross-entropy (EPI_CE_FWD) and its gradient softmax - onehot (EPI_CE_BWD).
//
// Variants: LONGK (reductions over all tokens, the weight gradients) has four epilogue warps and a
// deeper ring; a grouped launch runs up to eight products with the same K and operand layouts
// from one problem table (tile_start / pM / pN ...), their tiles in one persistent schedule (a
// symmetric product, ptri, takes only the tiles that meet its upper triangle); F8
// takes 8-bit operands (kind::f8f6f4, 128 K elements per stage) and scales every accumulator by
// the operands' inverse scales.
//
// Either operand may be K-major (rows of K contiguous elements: the usual [out,in] weight and
// [tokens,features] activation layouts) or MN-major (M or N contiguous: what the gradient GEMMs
// of a linear layer need), so forward, data-gradient and weight-gradient products all run on
// this one kernel without any transpose copies.
#pragma once

#include "ptx.cuh"

namespace gptk {

enum EpiKind : int {
  EPI_BF16 = 0,     // out bf16 = acc (+ bias); optional head-padded column map (generic path)
  EPI_F32 = 1,      // out fp32 = acc (+ bias)  or  out += acc  (accumulate)
  EPI_RESID = 2,    // out fp32 = resid + acc (+ bias)
  EPI_QKV = 3,      // out bf16 = acc, with RoPE + per-head RMSNorm applied to the q and k heads
  EPI_UP = 4,       // u = acc (+ bias) -> h = act(u) bf16 (out2), and u bf16 (out) unless out is null
  EPI_ACTBWD = 5,   // out bf16 = acc * act'(u); aux is u, or h = relu(u)^2 when act is ReLU^2;
                    // act 3: out bf16 = ax_alpha acc + ax_beta aux (a linear combination)
  EPI_CE_FWD = 6,   // per-row (max, sum exp) partials over this tile's vocab columns + target logit
  EPI_CE_BWD = 7,   // out bf16 = (softmax - onehot) * scale
};

struct GemmParams {
  int M, N, K;
  int a_mn, b_mn;             // 1 = operand stored MN-major
  int tiles_m, tiles_n;
  int tma_out;                // 1 = epilogue writes through the output tensor maps (fast path)
  int group_m;                // tile order: bands of group_m m-tiles sweep every n-tile
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
  int act;                    // 0 GELU(erf), 1 ReLU^2 (EPI_ACTBWD: 2 ReLU^2 from h, 3 linear)
  float ax_alpha, ax_beta;    // EPI_ACTBWD with act 3
  int prow[8];                // grouped launches: the epilogue input's first row for each problem
  // head-padded output layout (generic BF16 path): column c maps to (c / hd) * hdp + c % hd
  int hd, hdp;
  // cross-entropy
  const int* targets;         // [M]
  float2* ce_part;            // [M][tiles_n]  (max log2, sum exp2)
  float* ce_zy;               // [M] target logit
  const float* ce_lse;        // [M] natural-log logsumexp (backward)
  float ce_scale;             // 1/M_total (backward)
  // EPI_QKV (128-wide heads, 256-column tiles: one head per epilogue warp): columns [0, qk_D)
  // are q and [qk_D, 2 qk_D) are k; each head row gets r = rsqrt(mean(x^2) + qk_eps) (when
  // qk_norm; RoPE keeps the row norm, so the accumulator gives it) and the rotation of the pairs
  // (i, i + 64) by rope_cs[t][i] (when qk_rope), t = row % rope_T; r goes to rstd_q / rstd_k
  // [rows][qk_H].  Columns from 2 qk_D on (v) are stored as they are.
  const float2* rope_cs;
  int rope_T, qk_D, qk_H, qk_rope, qk_norm;
  float qk_eps;
  float* rstd_q;
  float* rstd_k;
  int prof_kind;              // host only: profiler family of this call (0 = generic GEMM)
  // grouped launch: up to kMaxProblems products with the same K, operand layouts and epilogue
  // share one persistent tile space; problem q owns tiles [tile_start[q], tile_start[q+1]).
  int n_prob;
  int tile_start[9];
  int pM[8], pN[8], ptiles_m[8], ptiles_n[8], pgroup_m[8];
  int pK[8];                  // host only: K extent of each problem (0 = K), for the FLOP count
  int ptri[8];                // 1: problem q computes only the tiles meeting its upper triangle
  int tile_rows, tile_cols;   // the launch's output tile (rows: 256 for CTA pairs, else 128)
  double pelems[8];           // host only: output elements problem q computes (0 = M N)
  // 8-bit operands (the F8 kernels): formats (0 = e4m3, 1 = e5m2) and the inverse scales that
  // multiply every accumulator (device scalars: the product is (a s_a)(b s_b)^T / (s_a s_b))
  int f8_fmt_a, f8_fmt_b;
  const float* f8_inv_a;
  const float* f8_inv_b;
  // EPI_UP: when set, max |h| over the stored (bf16) h is folded into *amax_h (a float bit
  // pattern; the caller zeroes it first) for an 8-bit cast of h that then needs no pass of its own
  unsigned int* amax_h;
};

constexpr int kMaxProblems = 8;

// Tensor maps of a launch: A and B (and the output C) per problem, plus the second output and
// the epilogue input of single-problem launches.
struct GemmMaps {
  CUtensorMap a[kMaxProblems], b[kMaxProblems], c[kMaxProblems];
  CUtensorMap c2, r;
};

// LONGK: the variant for very long reductions (weight gradients over all tokens), where the
// epilogue is rare and a deeper TMA ring matters more than epilogue parallelism.
template <int BN, bool LONGK = false, bool PAIR = false>
struct GemmCfg {
  static constexpr int BM = 128;                    // accumulator rows per CTA
  static constexpr int TILE_M = PAIR ? 256 : 128;   // output rows per tile
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN; // B rows staged per CTA
  static constexpr int BK = 64;
  static constexpr int STAGES = PAIR ? (LONGK ? 6 : 5) : (LONGK ? ((BN == 256) ? 4 : 6) : ((BN == 256) ? 3 : 5));
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_WARPS = LONGK ? 4 : 8;             // one or two per TMEM lane quadrant
  static constexpr int STAGING_BYTES = EPI_WARPS * 2 * 4096;  // 2 buffers of 32 rows x 128 B per warp
  static constexpr int BAR_BYTES = 512;
  static_assert((2 * STAGES + 5 + 2 * EPI_WARPS) * 8 + 8 <= BAR_BYTES, "barrier block too small");
  static constexpr int SMEM = STAGES * STAGE_BYTES + STAGING_BYTES + BAR_BYTES + 1024;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
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
  if (act == 2) return 2.f * sqrt_approx(fmaxf(u, 0.f));  // ReLU^2 given h = relu(u)^2: 2 relu(u) = 2 sqrt(h)
  // d/du of 0.5 u (1 + erf(u/sqrt2)) = 0.5 (1 + erf(u/sqrt2)) + u * exp(-u^2/2) / sqrt(2 pi)
  return 0.5f * (1.f + erff(u * 0.70710678118654752f)) + u * expf(-0.5f * u * u) * 0.3989422804014327f;
}

__device__ __forceinline__ void add_bias32(float* v, const float* bias, int col0, int N) {
  if (bias == nullptr) return;
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (col0 + j < N) v[j] += __ldg(bias + col0 + j);
}

// 16-byte unit `u` of row r in a 128-byte-swizzled staging buffer
__device__ __forceinline__ uint32_t stg_addr(uint32_t base, int r, int u) {
  return base + r * 128 + ((u ^ (r & 7)) << 4);
}
__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

// row r of a staging buffer <- 32 fp32 values
__device__ __forceinline__ void stage_f32(uint32_t buf, int r, const float* v) {
#pragma unroll
  for (int u = 0; u < 8; ++u)
    sts128(stg_addr(buf, r, u), __float_as_uint(v[4 * u]), __float_as_uint(v[4 * u + 1]),
           __float_as_uint(v[4 * u + 2]), __float_as_uint(v[4 * u + 3]));
}
// units u0 .. u0+3 (32 bf16 columns) of row r of a staging buffer <- 32 values
__device__ __forceinline__ void stage_bf16_half(uint32_t buf, int r, int u0, const float* v) {
#pragma unroll
  for (int u = 0; u < 4; ++u)
    sts128(stg_addr(buf, r, u0 + u), pack_bf16x2(v[8 * u], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
           pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
}
// row r of a staging buffer <- 64 bf16 values
__device__ __forceinline__ void stage_bf16(uint32_t buf, int r, const float* v) {
#pragma unroll
  for (int u = 0; u < 8; ++u)
    sts128(stg_addr(buf, r, u), pack_bf16x2(v[8 * u], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
           pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
}
__device__ __forceinline__ void unstage_f32(uint32_t buf, int r, float* v) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    uint4 x = lds128(stg_addr(buf, r, u));
    v[4 * u] = __uint_as_float(x.x);
    v[4 * u + 1] = __uint_as_float(x.y);
    v[4 * u + 2] = __uint_as_float(x.z);
    v[4 * u + 3] = __uint_as_float(x.w);
  }
}
__device__ __forceinline__ void unstage_bf16(uint32_t buf, int r, float* v) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    uint4 x = lds128(stg_addr(buf, r, u));
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[8 * u + 2 * k] = __uint_as_float(w[k] << 16);
      v[8 * u + 2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
}

// Generic (per-thread store) epilogue for one 32-column chunk of one row; used where the
// output is not a plain 2-D tile (head-padded layouts) or cannot be described by a tensor map.
template <int EPI>
__device__ __forceinline__ void epi_chunk_generic(const GemmParams& p, float* v, int row, int col0, bool row_ok) {
  if (EPI == EPI_BF16) {
    add_bias32(v, p.bias, col0, p.N);
    if (!row_ok) return;
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) + (long long)row * p.ldo;
    for (int j = 0; j < 32; ++j) {
      int c = col0 + j;
      if (c < p.N) out[(c / p.hd) * p.hdp + c % p.hd] = __float2bfloat16_rn(v[j]);
    }
  } else if (EPI == EPI_F32) {
    add_bias32(v, p.bias, col0, p.N);
    if (!row_ok) return;
    float* out = reinterpret_cast<float*>(p.out) + (long long)row * p.ldo;
    for (int j = 0; j < 32; ++j) {
      int c = col0 + j;
      if (c < p.N) out[c] = p.accumulate ? out[c] + v[j] : v[j];
    }
  } else if (EPI == EPI_RESID) {
    add_bias32(v, p.bias, col0, p.N);
    if (!row_ok) return;
    float* out = reinterpret_cast<float*>(p.out) + (long long)row * p.ldo;
    const float* res = p.resid + (long long)row * p.ldr;
    for (int j = 0; j < 32; ++j) {
      int c = col0 + j;
      if (c < p.N) out[c] = res[c] + v[j];
    }
  } else if (EPI == EPI_UP) {
    add_bias32(v, p.bias, col0, p.N);
    if (!row_ok) return;
    __nv_bfloat16* u = p.out ? reinterpret_cast<__nv_bfloat16*>(p.out) + (long long)row * p.ldo : nullptr;
    __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(p.out2) + (long long)row * p.ldo;
    for (int j = 0; j < 32; ++j) {
      int c = col0 + j;
      if (c < p.N) {
        if (u) u[c] = __float2bfloat16_rn(v[j]);
        h[c] = __float2bfloat16_rn(act_fwd(v[j], p.act));
      }
    }
  } else if (EPI == EPI_ACTBWD) {
    if (!row_ok) return;
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) + (long long)row * p.ldo;
    const __nv_bfloat16* u = p.aux + (long long)row * p.ld_aux;
    for (int j = 0; j < 32; ++j) {
      int c = col0 + j;
      if (c < p.N) out[c] = __float2bfloat16_rn(v[j] * act_grad(__bfloat162float(u[c]), p.act));
    }
  } else if (EPI == EPI_CE_BWD) {
    if (!row_ok) return;
    const float lse2 = p.ce_lse[row] * 1.4426950408889634f;
    const int y = p.targets[row];
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) + (long long)row * p.ldo;
    for (int j = 0; j < 32; ++j) {
      int c = col0 + j;
      float g = ex2_approx(fmaf(v[j], 1.4426950408889634f, -lse2));
      if (c == y) g -= 1.f;
      if (c < p.N) out[c] = __float2bfloat16_rn(g * p.ce_scale);
    }
  }
}

// Tile t -> (problem, tm, tn).  Within a problem, tiles are taken in bands of group_m m-tiles;
// inside a band the m index runs fastest, and the band sweeps every n-tile before the next
// band starts, so the A rows of a band stay in L2 while all of B passes by.
struct TileInfo {
  int prob, tm, tn, M, N;
};
__device__ __forceinline__ TileInfo tile_info(const GemmParams& p, int tile) {
  TileInfo t;
  int q = 0;
  while (q + 1 < p.n_prob && tile >= p.tile_start[q + 1]) ++q;
  t.prob = q;
  t.M = p.pM[q];
  t.N = p.pN[q];
  const int local = tile - p.tile_start[q];
  if (p.ptri[q]) {
    // upper-triangle problems: m-tile tm takes the n-tiles from the one holding column
    // tm * tile_rows (its first row) on, in row order
    int tm = 0, rest = local;
    for (;;) {
      const int cnt = p.ptiles_n[q] - tm * p.tile_rows / p.tile_cols;
      if (rest < cnt || tm + 1 >= p.ptiles_m[q]) break;
      rest -= cnt;
      ++tm;
    }
    t.tm = tm;
    t.tn = tm * p.tile_rows / p.tile_cols + rest;
    return t;
  }
  const int per_band = p.pgroup_m[q] * p.ptiles_n[q];
  const int band = local / per_band;
  const int first = band * p.pgroup_m[q];
  const int gm = min(p.pgroup_m[q], p.ptiles_m[q] - first);
  const int in_band = local - band * per_band;
  t.tm = first + in_band % gm;
  t.tn = in_band / gm;
  return t;
}

// --------------------------------------------------------------- the kernel

// F8: 8-bit operands (kind::f8f6f4, both K-major): a stage holds 128 K elements (the same 128
// bytes per row as 64 bf16 ones), four K = 32 MMAs, and the epilogue scales every accumulator.
template <int BN, int EPI, bool LONGK, bool PAIR, bool F8 = false>
__global__ void __launch_bounds__(GemmCfg<BN, LONGK, PAIR>::THREADS, 1)
    gemm_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmParams p) {
  using C = GemmCfg<BN, LONGK, PAIR>;
  constexpr int KE = F8 ? 2 * C::BK : C::BK;  // K elements per stage
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint8_t* staging = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + C::STAGING_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = bars + 2 * C::STAGES + 2;
  uint64_t* drain = bars + 2 * C::STAGES + 4;
  uint64_t* inbar = bars + 2 * C::STAGES + 5;  // [EPI_WARPS][2 buffers]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 5 + 2 * C::EPI_WARPS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  pdl_trigger();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA pairs: rank within the pair, and the pair's place in the persistent tile walk
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int tile0 = PAIR ? (int)cluster_id_x() : (int)blockIdx.x;
  const int tile_step = PAIR ? (int)cluster_count_x() : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], C::EPI_WARPS * (PAIR ? 2 : 1));
    }
    mbar_init(drain, 1);
    for (int i = 0; i < 2 * C::EPI_WARPS; ++i) mbar_init(&inbar[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
    for (int q = 0; q < p.n_prob; ++q) {
      prefetch_tmap(&maps.a[q]);
      prefetch_tmap(&maps.b[q]);
    }
  }
  if (PAIR) {
    // the peer's barriers must be initialised before anything is signalled across the pair
    cluster_sync();
    if (warp == 1) {
      tmem_alloc_pair(tmem_slot, 2 * BN);
      tmem_relinquish_pair();
    }
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // the operands and epilogue inputs come from the kernels before this one

  const int num_tiles = p.tile_start[p.n_prob];
  const int num_k = (p.K + KE - 1) / KE;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t pending = 0;  // stages with a load in flight that the MMA has not yet released
    bool ok = true;
    for (int tile = tile0; tile < num_tiles && ok; tile += tile_step) {
      const TileInfo ti = tile_info(p, tile);
      const int tm = ti.tm, tn = ti.tn;
      const CUtensorMap* tmA = &maps.a[ti.prob];
      const CUtensorMap* tmB = &maps.b[ti.prob];
      const int arow = tm * C::TILE_M + (int)rank * C::BM;     // this CTA's A rows
      const int brow = tn * BN + (int)rank * C::B_ROWS;        // this CTA's B rows
      for (int kb = 0; kb < num_k; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, p.ctl, abort_flag, 1)) {
          ok = false;
          break;
        }
        pending &= ~(1u << stage);
        uint8_t* a = sA + stage * C::A_BYTES;
        uint8_t* b = sB + stage * C::B_BYTES;
        if (PAIR) {
          // both CTAs' bytes complete on the even CTA's barrier, which expects all of them
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          if (rank == 0) mbar_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          if (!p.a_mn) {
            tma_load_2d_pair(a, tmA, fb, kb * KE, arow);
          } else {
#pragma unroll
            for (int c = 0; c < C::BM / 64; ++c) tma_load_2d_pair(a + c * 8192, tmA, fb, arow + c * 64, kb * KE);
          }
          if (!p.b_mn) {
            tma_load_2d_pair(b, tmB, fb, kb * KE, brow);
          } else {
#pragma unroll
            for (int c = 0; c < C::B_ROWS / 64; ++c)
              tma_load_2d_pair(b + c * 8192, tmB, fb, brow + c * 64, kb * KE);
          }
        } else {
          mbar_expect_tx(&full[stage], C::STAGE_BYTES);
          if (!p.a_mn) {
            tma_load_2d(a, tmA, &full[stage], kb * KE, arow);
          } else {
#pragma unroll
            for (int c = 0; c < C::BM / 64; ++c)
              tma_load_2d(a + c * 8192, tmA, &full[stage], arow + c * 64, kb * KE);
          }
          if (!p.b_mn) {
            tma_load_2d(b, tmB, &full[stage], kb * KE, brow);
          } else {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              tma_load_2d(b + c * 8192, tmB, &full[stage], brow + c * 64, kb * KE);
          }
        }
        pending |= 1u << stage;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (PAIR && ok) {
      // wait until the MMAs have released every stage, i.e. until the even CTA's last commits
      // to this CTA's "empty" barriers have landed
      for (int i = 0; i < C::STAGES && ok; ++i) {
        ok = mbar_wait(&empty[stage], phase ^ 1u, p.ctl, abort_flag, 8);
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok && (!PAIR || rank == 0)) {
      // drain the copies still in flight before the CTA goes away (bounded as well)
      volatile int never = 0;
      for (int s = 0; s < C::STAGES; ++s) {
        if (!(pending & (1u << s))) continue;
        // stage s was issued in the current or the previous lap of the ring
        uint32_t ph = (s < stage) ? phase : (phase ^ 1u);
        mbar_wait(&full[s], ph, p.ctl, &never, 2);
      }
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------------------------------ MMA issuer (the even CTA of a pair)
    constexpr uint32_t IDESC_KK = idesc_bf16(C::TILE_M, BN, 0, 0);
    const uint32_t idesc = F8 ? idesc_f8(C::TILE_M, BN, p.f8_fmt_a, p.f8_fmt_b)
                              : IDESC_KK | (static_cast<uint32_t>(p.a_mn) << 15) | (static_cast<uint32_t>(p.b_mn) << 16);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    bool issued = false;
    // stage-0 descriptors and the per-K-step advance, computed once: the four MMAs of a stage
    // then go out back to back (umma4_ss*)
    const uint64_t descA0 = p.a_mn ? sdesc_sw128(smem_u32(sA), 8192, 1024) : sdesc_sw128(smem_u32(sA), 16, 1024);
    const uint64_t descB0 = p.b_mn ? sdesc_sw128(smem_u32(sB), 8192, 1024) : sdesc_sw128(smem_u32(sB), 16, 1024);
    const uint32_t stepA = p.a_mn ? 2048u : 32u, stepB = p.b_mn ? 2048u : 32u;
    for (int tile = tile0; tile < num_tiles && ok; tile += tile_step) {
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
        const uint64_t da = sdesc_add(descA0, stage * C::A_BYTES);
        const uint64_t db = sdesc_add(descB0, stage * C::B_BYTES);
        static_assert(C::BK == 64, "one stage is four K = 16 MMAs");
        uint64_t aa[4], bb[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          aa[kk] = sdesc_add(da, kk * stepA);
          bb[kk] = sdesc_add(db, kk * stepB);
        }
        if (F8) {
          if (PAIR) umma4_f8_pair(d_tmem, aa, bb, idesc, kb == 0 ? 0xeu : 0xfu);
          else umma4_f8(d_tmem, aa, bb, idesc, kb == 0 ? 0xeu : 0xfu);
        } else {
          if (PAIR) umma4_ss_pair(d_tmem, aa, bb, idesc, kb == 0 ? 0xeu : 0xfu);
          else umma4_ss(d_tmem, aa, bb, idesc, kb == 0 ? 0xeu : 0xfu);
        }
        if (PAIR) {
          // the stage is free in both CTAs once these MMAs have read it
          const uint32_t eb = smem_u32(&empty[stage]);
          umma_commit_pair(eb);
          umma_commit_pair(mapa_shared(eb, 1));
        } else {
          umma_commit(&empty[stage]);
        }
        issued = true;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (PAIR) {
        const uint32_t tb = smem_u32(&tfull[acc]);
        umma_commit_pair(tb);
        umma_commit_pair(mapa_shared(tb, 1));
      } else {
        umma_commit(&tfull[acc]);
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (PAIR && ok) {
      // both CTAs' epilogues have finished with both accumulators: every arrival from the
      // peer on this CTA's "tempty" barriers has landed
      for (int i = 0; i < 2 && ok; ++i) {
        ok = mbar_wait(&tempty[acc], acc_phase ^ 1u, p.ctl, abort_flag, 9);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
    if (!ok && issued) {
      // let the MMAs already issued finish before tensor memory is released
      volatile int never = 0;
      if (PAIR) umma_commit_pair(smem_u32(drain));
      else umma_commit(drain);
      mbar_wait(drain, 0, p.ctl, &never, 6);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int ew = warp - 2;
    const int chalf = ew >> 2;  // which part of the tile's columns this warp writes
    uint8_t* stg_ptr = staging + ew * 8192;
    const uint32_t stg = smem_u32(stg_ptr);
    uint64_t* ibar = inbar + 2 * ew;
    uint32_t in_uses = 0;  // bit b flips on every use of input buffer b (its mbarrier parity)
    int chunk_ctr = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    constexpr bool F32OUT = (EPI == EPI_F32 || EPI == EPI_RESID);
    constexpr int CW = F32OUT ? 32 : 64;
    constexpr bool HAS_IN = (EPI == EPI_RESID || EPI == EPI_ACTBWD);
    constexpr int HALF = BN * 4 / C::EPI_WARPS;  // columns per epilogue warp
    const float f8_scale = F8 ? __ldg(p.f8_inv_a) * __ldg(p.f8_inv_b) : 1.f;
    float amax_h = 0.f;  // EPI_UP: max |h| of this thread's outputs over all its tiles
    for (int tile = tile0; tile < num_tiles; tile += tile_step) {
      const TileInfo ti = tile_info(p, tile);
      const int tm = ti.tm, tn = ti.tn;
      const int pN = ti.N;
      const CUtensorMap* tmC = &maps.c[ti.prob];
      const CUtensorMap* tmC2 = &maps.c2;
      const CUtensorMap* tmR = &maps.r;
      const int row0 = tm * C::TILE_M + (int)rank * C::BM + quad * 32;
      const int row = row0 + lane;
      const bool row_ok = row < ti.M;
      const int c_begin = chalf * HALF;
      const int n0 = tn * BN;
      const bool tma = p.tma_out && EPI != EPI_CE_FWD;
      // the first input chunk of the tile can load while the main loop still runs
      if (HAS_IN && tma && n0 + c_begin < pN && lane == 0) {
        const int b = chunk_ctr & 1;
        bulk_wait_read<1>();
        mbar_expect_tx(&ibar[b], 4096);
        tma_load_2d(stg_ptr + b * 4096, tmR, &ibar[b], n0 + c_begin, row0 + p.prow[ti.prob]);
      }
      if (!mbar_wait(&tfull[acc], acc_phase, p.ctl, abort_flag, 5)) break;
      tc_fence_after();
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * BN;
      bool ok = true;
      if (EPI == EPI_CE_FWD) {
        // both warps of a quadrant see the whole row; the lower-half warp reduces it
        if (chalf == 0) {
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
        }
      } else if (EPI == EPI_QKV && tma && n0 + c_begin < 2 * p.qk_D) {
        // one q or k head (128 columns) per warp: RMS of the row, then RoPE and the scale, both
        // halves of the head staged (buffer 0: columns 0-63, buffer 1: 64-127) and stored
        const int g0 = n0 + c_begin;
        const int part = g0 >= p.qk_D;
        const int hh = (g0 - part * p.qk_D) >> 7;
        float r = 1.f;
        if (p.qk_norm) {
          float ss = 0.f;
#pragma unroll 1
          for (int q4 = 0; q4 < 4; ++q4) {
            float v[32];
            tmem_ld32(trow + c_begin + 32 * q4, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (F8) v[j] *= f8_scale;
              ss = fmaf(v[j], v[j], ss);
            }
          }
          r = rsqrtf(ss * (1.f / 128.f) + p.qk_eps);
          if (row_ok) (part ? p.rstd_k : p.rstd_q)[(long long)row * p.qk_H + hh] = r;
        }
        if (lane == 0) bulk_wait_read<0>();  // both staging buffers free
        __syncwarp();
        const float4* csr = reinterpret_cast<const float4*>(p.rope_cs + (long long)(row_ok ? row % p.rope_T : 0) * 64);
#pragma unroll 1
        for (int rr = 0; rr < 2; ++rr) {
          float x1[32], x2[32];
          tmem_ld32(trow + c_begin + 32 * rr, x1);
          tmem_ld32(trow + c_begin + 64 + 32 * rr, x2);
          if (F8) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              x1[j] *= f8_scale;
              x2[j] *= f8_scale;
            }
          }
#pragma unroll
          for (int j2 = 0; j2 < 16; ++j2) {
            const float4 e = p.qk_rope ? __ldg(csr + 16 * rr + j2) : make_float4(1.f, 0.f, 1.f, 0.f);
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const int j = 2 * j2 + k;
              const float c = k ? e.z : e.x, sn = k ? e.w : e.y;
              const float a = x1[j], b = x2[j];
              x1[j] = (a * c - b * sn) * r;
              x2[j] = (a * sn + b * c) * r;
            }
          }
          stage_bf16_half(stg, lane, 4 * rr, x1);
          stage_bf16_half(stg + 4096, lane, 4 * rr, x2);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {  // one bulk group per buffer, so a later chunk waits only for its own
          tma_store_2d(tmC, stg_ptr, g0, row0);
          bulk_commit();
          tma_store_2d(tmC, stg_ptr + 4096, g0 + 64, row0);
          bulk_commit();
        }
        chunk_ctr += 2;
      } else if (!tma) {
        for (int c = c_begin; c < c_begin + HALF; c += 32) {
          float v[32];
          tmem_ld32(trow + c, v);
          if (F8) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= f8_scale;
          }
          epi_chunk_generic<EPI>(p, v, row, n0 + c, row_ok);
        }
      } else {
        // TMA path: chunks of 32 fp32 or 64 bf16 columns (128-byte staging rows)
        for (int c = c_begin; c < c_begin + HALF; c += CW) {
          const int col0 = n0 + c;
          if (col0 >= pN) break;
          const int b = chunk_ctr & 1;
          const uint32_t buf = stg + b * 4096;
          const bool two_out = (EPI == EPI_UP) && p.out != nullptr;
          if (!HAS_IN) {
            // the staging buffer must no longer be read by an earlier store
            if (lane == 0) {
              if (two_out) bulk_wait_read<0>();
              else bulk_wait_read<1>();
            }
            __syncwarp();
          }
          float v[CW];
          tmem_ld32(trow + c, *reinterpret_cast<float(*)[32]>(&v[0]));
          if (CW == 64) tmem_ld32(trow + c + 32, *reinterpret_cast<float(*)[32]>(&v[32 % CW]));
          if (F8) {
#pragma unroll
            for (int j = 0; j < CW; ++j) v[j] *= f8_scale;
          }
          if (EPI != EPI_ACTBWD && EPI != EPI_CE_BWD) {
            add_bias32(v, p.bias, col0, pN);
            if (CW == 64) add_bias32(v + (32 % CW), p.bias, col0 + 32, pN);
          }
          if (HAS_IN) {
            if (!mbar_wait(&ibar[b], (in_uses >> b) & 1u, p.ctl, abort_flag, 7)) {
              ok = false;
              break;
            }
            in_uses ^= 1u << b;
            float in[CW];
            if (EPI == EPI_RESID) {
              unstage_f32(buf, lane, in);
#pragma unroll
              for (int j = 0; j < CW; ++j) v[j] += in[j];
            } else if (p.act == 3) {  // EPI_ACTBWD, linear: alpha acc + beta aux
              unstage_bf16(buf, lane, in);
#pragma unroll
              for (int j = 0; j < CW; ++j) v[j] = fmaf(p.ax_beta, in[j], p.ax_alpha * v[j]);
            } else if (p.act == 2) {  // EPI_ACTBWD, ReLU^2 from h: 2 relu(u) = 2 sqrt(h)
              unstage_bf16(buf, lane, in);
#pragma unroll
              for (int j = 0; j < CW; ++j) v[j] *= 2.f * sqrt_approx(fmaxf(in[j], 0.f));
            } else if (p.act == 1) {  // ReLU^2 from u
              unstage_bf16(buf, lane, in);
#pragma unroll
              for (int j = 0; j < CW; ++j) v[j] *= 2.f * fmaxf(in[j], 0.f);
            } else {  // GELU from u
              unstage_bf16(buf, lane, in);
#pragma unroll
              for (int j = 0; j < CW; ++j) v[j] *= act_grad(in[j], 0);
            }
          }
          if (EPI == EPI_CE_BWD) {
            const float lse2 = row_ok ? p.ce_lse[row] * 1.4426950408889634f : 0.f;
            const int y = row_ok ? p.targets[row] : -1;
#pragma unroll
            for (int j = 0; j < CW; ++j) {
              float gv = ex2_approx(fmaf(v[j], 1.4426950408889634f, -lse2));
              if (col0 + j == y) gv -= 1.f;
              v[j] = gv * p.ce_scale;
            }
          }
          if (EPI == EPI_UP) {
            // h = act(u) to buffer b (tensor map tmC2); u itself to buffer b^1 when kept
            if (two_out) stage_bf16(stg + (b ^ 1) * 4096, lane, v);
            if (p.act == 1) {
#pragma unroll
              for (int j = 0; j < CW; ++j) {
                const float r = fmaxf(v[j], 0.f);
                v[j] = r * r;
              }
            } else {
#pragma unroll
              for (int j = 0; j < CW; ++j) v[j] = act_fwd(v[j], 0);
            }
            if (p.amax_h != nullptr && row_ok) {
#pragma unroll
              for (int j = 0; j < CW; ++j)
                if (col0 + j < pN) amax_h = fmaxf(amax_h, fabsf(v[j]));
            }
            stage_bf16(buf, lane, v);
          } else if (F32OUT) {
            stage_f32(buf, lane, v);
          } else {
            stage_bf16(buf, lane, v);
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (EPI == EPI_UP) {
              tma_store_2d(tmC2, stg_ptr + b * 4096, col0, row0);
              if (two_out) tma_store_2d(tmC, stg_ptr + (b ^ 1) * 4096, col0, row0);
            } else if (EPI == EPI_F32 && p.accumulate) {
              tma_reduce_add_2d(tmC, stg_ptr + b * 4096, col0, row0);
            } else {
              tma_store_2d(tmC, stg_ptr + b * 4096, col0, row0);
            }
            bulk_commit();
            // prefetch the next input chunk into the other buffer once its last store has read it
            if (HAS_IN && c + CW < c_begin + HALF && col0 + CW < pN) {
              bulk_wait_read<1>();
              mbar_expect_tx(&ibar[b ^ 1], 4096);
              tma_load_2d(stg_ptr + (b ^ 1) * 4096, tmR, &ibar[b ^ 1], col0 + CW, row0 + p.prow[ti.prob]);
            }
          }
          ++chunk_ctr;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
        else mbar_arrive(&tempty[acc]);
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
      if (!ok) break;
    }
    if (lane == 0) bulk_wait_all();
    if (EPI == EPI_UP && p.amax_h != nullptr) {
      // one atomic per epilogue warp; h is stored in bf16 and the rounding is monotonic
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax_h = fmaxf(amax_h, __shfl_xor_sync(0xffffffffu, amax_h, o));
      if (lane == 0) atomicMax(p.amax_h, __float_as_uint(__bfloat162float(__float2bfloat16_rn(amax_h))));
    }
  }

  __syncthreads();
  if (PAIR) {
    // neither CTA leaves while the other may still address its shared or tensor memory
    cluster_sync();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc_pair(tmem_base, 2 * BN);
    }
  } else if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * BN);
  }
}

}  // namespace gptk
