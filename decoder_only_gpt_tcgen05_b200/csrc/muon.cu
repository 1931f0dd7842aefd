// The split optimizer step of nanochat ("Train your own ChatGPT", read the source optim.py -- Muon
// + AdamW): every block matrix (w_qkv, w_o, w_up, w_down) takes a Muon step, which orthogonalizes
// its update, and every other tensor (embeddings, lm_head, LayerNorm gains, biases) an AdamW step.
//
// Muon, per matrix G [rows, cols] (the published form of its authors):
//   buf <- mu buf + (1 - mu) G;   U = (1 - mu) G + mu buf (Nesterov) or buf
//   X = U / (||U||_F + 1e-7), on the wide orientation (U^T when rows > cols), in bf16
//   ns_steps times:  A = X X^T;  M = b A + c A A;  X <- a X + M X     (a, b, c) = (3.4445, -4.7750, 2.0315)
//   W <- W - lr sqrt(max(1, rows / cols)) X   (X transposed back)
// Matrices of one shape are processed together, up to eight at a time: the three products of an
// iteration are grouped tcgen05 GEMM launches over all of them (a 1280 x 1280 product alone fills
// a third of the SM pairs), and the elementwise steps are one launch each.
//
// Launch sequence per chunk of same-shape matrices:
//   muon_momentum_kernel   buf update and the Nesterov input's squared norm (fp64 partials)
//   muon_prep_*_kernel     X = U / ||U|| in bf16 (transposed through shared memory when rows > cols)
//   ns_steps x { grouped GEMM A = X X^T (bf16; upper-triangle tiles only), muon_mirror_kernel,
//                grouped GEMM M = c (A A) + b A (bf16; the linear combination in the epilogue;
//                upper-triangle tiles only), muon_mirror_kernel,
//                grouped GEMM X' = (M X) + a X (bf16, into the other X buffer) }
//   muon_update_*_kernel   W -= lr scale X (transposed back through shared memory when rows > cols)
#include <algorithm>
#include <cmath>
#include <string>
#include <vector>

#include "gemm.cuh"
#include "gpt.h"
#include "host.cuh"
#include "kernels.cuh"

namespace gptk {

namespace {

constexpr int kParts = 256;             // fixed partition of each matrix's squared-norm sum
constexpr int kChunk = kMaxProblems;    // matrices per grouped launch
constexpr float kNsA = 3.4445f, kNsB = -4.7750f, kNsC = 2.0315f;

struct MatList {
  long long off[kChunk];  // element offsets of the chunk's matrices in the parameter buffer
};

__device__ __forceinline__ double warp_sum_dd(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// blockIdx.y: matrix of the chunk; blockIdx.x: its part (a contiguous range of n / kParts
// elements, a multiple of 4).  buf <- mu buf + (1 - mu) g, and the part's sum of u^2.
__global__ void __launch_bounds__(256) muon_momentum_kernel(const float* __restrict__ g, float* __restrict__ mom,
                                                            MatList ml, long long n, float mu, int nesterov,
                                                            double* __restrict__ part) {
  __shared__ double red[8];
  const long long base = ml.off[blockIdx.y];
  const long long chunk = (((n + kParts - 1) / kParts) + 3) & ~3LL;
  const long long lo = blockIdx.x * chunk;
  const long long hi = lo + chunk < n ? lo + chunk : n;
  const float omm = 1.f - mu;
  double s = 0.0;
  for (long long i = lo + 4LL * threadIdx.x; i < hi; i += 4LL * blockDim.x) {
    const float4 gv = *reinterpret_cast<const float4*>(g + base + i);
    float4 b = *reinterpret_cast<const float4*>(mom + base + i);
    b.x = fmaf(mu, b.x, omm * gv.x);
    b.y = fmaf(mu, b.y, omm * gv.y);
    b.z = fmaf(mu, b.z, omm * gv.z);
    b.w = fmaf(mu, b.w, omm * gv.w);
    *reinterpret_cast<float4*>(mom + base + i) = b;
    float4 u = b;
    if (nesterov) {
      u.x = fmaf(omm, gv.x, mu * b.x);
      u.y = fmaf(omm, gv.y, mu * b.y);
      u.z = fmaf(omm, gv.z, mu * b.z);
      u.w = fmaf(omm, gv.w, mu * b.w);
    }
    s += (double)u.x * u.x + (double)u.y * u.y + (double)u.z * u.z + (double)u.w * u.w;
  }
  s = warp_sum_dd(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    part[blockIdx.y * kParts + blockIdx.x] = t;
  }
}

// 1 / (||U||_F + 1e-7) of matrix q from its kParts partial sums, added in one fixed order (lane k
// sums parts 8 k .. 8 k + 7, then a fixed butterfly); called by a whole warp
__device__ __forceinline__ float muon_inv_norm(const double* __restrict__ part, int q) {
  static_assert(kParts == 256, "one warp, eight parts per lane");
  const int lane = threadIdx.x & 31;
  double t = 0.0;
#pragma unroll
  for (int k = 0; k < 8; ++k) t += part[q * kParts + 8 * lane + k];
  t = warp_sum_dd(t);
  return (float)(1.0 / (sqrt(t) + 1e-7));
}

// The Nesterov input (or buf) of four consecutive elements
__device__ __forceinline__ float4 muon_u4(const float* __restrict__ g, const float* __restrict__ mom, long long i,
                                          float mu, int nesterov) {
  const float4 b = *reinterpret_cast<const float4*>(mom + i);
  if (!nesterov) return b;
  const float4 gv = *reinterpret_cast<const float4*>(g + i);
  const float omm = 1.f - mu;
  return make_float4(fmaf(omm, gv.x, mu * b.x), fmaf(omm, gv.y, mu * b.y), fmaf(omm, gv.z, mu * b.z),
                     fmaf(omm, gv.w, mu * b.w));
}

// X[q] = U / (||U||_F + 1e-7) in bf16 for rows <= cols (X has U's layout): four elements per
// thread, blockIdx.y the matrix of the chunk
__global__ void __launch_bounds__(256) muon_prep_flat_kernel(const float* __restrict__ g, const float* __restrict__ mom,
                                                             MatList ml, long long n, float mu, int nesterov,
                                                             const double* __restrict__ part,
                                                             __nv_bfloat16* __restrict__ X) {
  pdl_trigger();
  __shared__ float s_inv;
  if (threadIdx.x < 32) {
    const float v = muon_inv_norm(part, blockIdx.y);
    if (threadIdx.x == 0) s_inv = v;
  }
  __syncthreads();
  const float inv = s_inv;
  const long long base = ml.off[blockIdx.y];
  __nv_bfloat16* Xq = X + (long long)blockIdx.y * n;
  for (long long i = 4LL * (blockIdx.x * blockDim.x + threadIdx.x); i < n; i += 4LL * gridDim.x * blockDim.x) {
    const float4 u = muon_u4(g, mom, base + i, mu, nesterov);
    *reinterpret_cast<uint2*>(Xq + i) = make_uint2(pack_bf16x2(u.x * inv, u.y * inv), pack_bf16x2(u.z * inv, u.w * inv));
  }
}

// X[q] [cols, rows] = U^T / (||U||_F + 1e-7) in bf16 for rows > cols: 32 x 32 tiles through
// shared memory (blockIdx.x: tile, blockIdx.y: matrix).  U is read as float4 along a row, X
// written four rows at a time along a column; both shared-memory passes are free of bank
// conflicts (row pitch 33).  Sides are multiples of 16, so a vector is in or out as a whole.
__global__ void __launch_bounds__(256) muon_prep_tr_kernel(const float* __restrict__ g, const float* __restrict__ mom,
                                                           MatList ml, int rows, int cols, float mu, int nesterov,
                                                           const double* __restrict__ part,
                                                           __nv_bfloat16* __restrict__ X) {
  pdl_trigger();
  __shared__ float tile[32][33];
  __shared__ float s_inv;
  if (threadIdx.x < 32) {
    const float v = muon_inv_norm(part, blockIdx.y);
    if (threadIdx.x == 0) s_inv = v;
  }
  const long long base = ml.off[blockIdx.y];
  const int tiles_c = (cols + 31) / 32;
  const int r0 = (blockIdx.x / tiles_c) * 32, c0 = (blockIdx.x % tiles_c) * 32;
  __syncthreads();
  const float inv = s_inv;
  {
    const int rr = threadIdx.x >> 3, cc = 4 * (threadIdx.x & 7);
    const int r = r0 + rr, c = c0 + cc;
    float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < rows && c < cols) u = muon_u4(g, mom, base + (long long)r * cols + c, mu, nesterov);
    tile[rr][cc] = u.x * inv;
    tile[rr][cc + 1] = u.y * inv;
    tile[rr][cc + 2] = u.z * inv;
    tile[rr][cc + 3] = u.w * inv;
  }
  __syncthreads();
  const int oc = threadIdx.x >> 3, orr = 4 * (threadIdx.x & 7);  // X row (a column of U), four rows of U
  const int c = c0 + oc, r = r0 + orr;
  if (c < cols && r < rows) {
    __nv_bfloat16* Xq = X + (long long)blockIdx.y * rows * cols;
    *reinterpret_cast<uint2*>(Xq + (long long)c * rows + r) =
        make_uint2(pack_bf16x2(tile[orr][oc], tile[orr + 1][oc]), pack_bf16x2(tile[orr + 2][oc], tile[orr + 3][oc]));
  }
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// W -= step * X for rows <= cols (X has W's layout): four elements per thread
__global__ void __launch_bounds__(256) muon_update_flat_kernel(float* __restrict__ params, MatList ml, long long n,
                                                               const __nv_bfloat16* __restrict__ X, float step) {
  const long long base = ml.off[blockIdx.y];
  const __nv_bfloat16* Xq = X + (long long)blockIdx.y * n;
  for (long long i = 4LL * (blockIdx.x * blockDim.x + threadIdx.x); i < n; i += 4LL * gridDim.x * blockDim.x) {
    const uint2 xv = *reinterpret_cast<const uint2*>(Xq + i);
    float4 w = *reinterpret_cast<const float4*>(params + base + i);
    w.x -= step * bf16lo(xv.x);
    w.y -= step * bf16hi(xv.x);
    w.z -= step * bf16lo(xv.y);
    w.w -= step * bf16hi(xv.y);
    *reinterpret_cast<float4*>(params + base + i) = w;
  }
}

// W[r][c] -= step * X[c][r] for rows > cols (X is [cols, rows]): 32 x 32 tiles through shared
// memory, X read four rows at a time along its rows, W updated as float4 along its rows
__global__ void __launch_bounds__(256) muon_update_tr_kernel(float* __restrict__ params, MatList ml, int rows, int cols,
                                                             const __nv_bfloat16* __restrict__ X, float step) {
  __shared__ float tile[32][33];  // tile[c][r]
  const long long base = ml.off[blockIdx.y];
  const int tiles_c = (cols + 31) / 32;
  const int r0 = (blockIdx.x / tiles_c) * 32, c0 = (blockIdx.x % tiles_c) * 32;
  const __nv_bfloat16* Xq = X + (long long)blockIdx.y * rows * cols;
  {
    const int oc = threadIdx.x >> 3, orr = 4 * (threadIdx.x & 7);
    const int c = c0 + oc, r = r0 + orr;
    uint2 xv = make_uint2(0u, 0u);
    if (c < cols && r < rows) xv = *reinterpret_cast<const uint2*>(Xq + (long long)c * rows + r);
    tile[oc][orr] = bf16lo(xv.x);
    tile[oc][orr + 1] = bf16hi(xv.x);
    tile[oc][orr + 2] = bf16lo(xv.y);
    tile[oc][orr + 3] = bf16hi(xv.y);
  }
  __syncthreads();
  const int rr = threadIdx.x >> 3, cc = 4 * (threadIdx.x & 7);
  const int r = r0 + rr, c = c0 + cc;
  if (r < rows && c < cols) {
    float4* wp = reinterpret_cast<float4*>(params + base + (long long)r * cols + c);
    float4 w = *wp;
    w.x -= step * tile[cc][rr];
    w.y -= step * tile[cc + 1][rr];
    w.z -= step * tile[cc + 2][rr];
    w.w -= step * tile[cc + 3][rr];
    *wp = w;
  }
}

// The strictly lower triangle of each symmetric m x m bf16 matrix of a stack of nq from its upper
// triangle (the grouped products A = X X^T and A A compute only the tiles that meet the upper
// one).  The blocks (bi, bj), bj <= bi, of 64 x 64 elements are dealt to the CTAs in turn; each goes
// through shared memory as fp32 (row pitch 65), read and written as 16-byte vectors.
constexpr int kMirrorCtas = 16;  // CTAs per SM at most (eight are resident: 16.6 KB of shared memory each)
__global__ void __launch_bounds__(256) muon_mirror_kernel(__nv_bfloat16* __restrict__ A, int m, int nq) {
  pdl_trigger();
  __shared__ float tile[64][65];
  const int nb = (m + 63) / 64;
  const int per = nb * (nb + 1) / 2;  // lower blocks of one matrix, the diagonal ones included
  const int rr = threadIdx.x >> 3, cc = 8 * (threadIdx.x & 7);  // 32 rows x 64 columns per pass
  for (int w = blockIdx.x; w < per * nq; w += gridDim.x) {
    const int q = w / per;
    int bi = 0, rest = w - q * per;
    while (rest > bi) {  // block row bi holds bi + 1 blocks
      rest -= bi + 1;
      ++bi;
    }
    const int bj = rest;
    __nv_bfloat16* Aq = A + (long long)q * m * m;
    // the upper block (bj, bi): rows bj*64 + rr (+32), columns bi*64 + cc .. cc + 7
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = bj * 64 + rr + 32 * h, c = bi * 64 + cc;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (r < m && c < m) v = *reinterpret_cast<const uint4*>(Aq + (long long)r * m + c);
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        tile[rr + 32 * h][cc + 2 * k] = __uint_as_float(wv[k] << 16);
        tile[rr + 32 * h][cc + 2 * k + 1] = __uint_as_float(wv[k] & 0xffff0000u);
      }
    }
    __syncthreads();
    // rows bi*64 + rr (+32), columns bj*64 + cc .. cc + 7 of the lower block: A[r][c] = A[c][r]
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int orow = rr + 32 * h;
      const int r = bi * 64 + orow, c = bj * 64 + cc;
      if (r < m && c < m) {
        __nv_bfloat16* d = Aq + (long long)r * m + c;
        if (bi > bj) {
          uint32_t wv[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) wv[k] = pack_bf16x2(tile[cc + 2 * k][orow], tile[cc + 2 * k + 1][orow]);
          *reinterpret_cast<uint4*>(d) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (c + k < r) d[k] = __float2bfloat16_rn(tile[cc + k][orow]);
        }
      }
    }
    __syncthreads();
  }
}

struct MuonGroup {
  int rows, cols;
  std::vector<long long> offs;
};

struct MuonScratch {
  size_t adam, part, x0, x1, a, m, total;
};

MuonScratch muon_scratch_plan(const std::vector<MuonGroup>& groups) {
  size_t mn = 0, mm = 0;
  for (const MuonGroup& g : groups) {
    const size_t m = (size_t)(g.rows < g.cols ? g.rows : g.cols);
    const size_t n = (size_t)(g.rows < g.cols ? g.cols : g.rows);
    if (m * n > mn) mn = m * n;
    if (m * m > mm) mm = m * m;
  }
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  MuonScratch s;
  size_t off = 0;
  s.adam = off;
  off += al(adamw_scratch_bytes());
  s.part = off;
  off += al((size_t)kChunk * kParts * 8);
  s.x0 = off;
  off += al((size_t)kChunk * mn * 2);
  s.x1 = off;
  off += al((size_t)kChunk * mn * 2);
  s.a = off;
  off += al((size_t)kChunk * mm * 2);
  s.m = off;
  off += al((size_t)kChunk * mm * 2);
  s.total = off;
  return s;
}

int muon_chunk(float* params, const float* grads, float* mom, const MuonGroup& grp, int first, int nq,
               const gpt_muon& h, void* scratch, const MuonScratch& sp, cudaStream_t st) {
  const int rows = grp.rows, cols = grp.cols;
  const int m = rows < cols ? rows : cols, n = rows < cols ? cols : rows;
  const long long elems = (long long)rows * cols;
  MatList ml = {};
  for (int q = 0; q < nq; ++q) ml.off[q] = grp.offs[first + q];
  char* base = static_cast<char*>(scratch);
  double* part = reinterpret_cast<double*>(base + sp.part);
  __nv_bfloat16* Xb[2] = {reinterpret_cast<__nv_bfloat16*>(base + sp.x0), reinterpret_cast<__nv_bfloat16*>(base + sp.x1)};
  __nv_bfloat16* A = reinterpret_cast<__nv_bfloat16*>(base + sp.a);
  __nv_bfloat16* M = reinterpret_cast<__nv_bfloat16*>(base + sp.m);
  __nv_bfloat16* X = Xb[0];
  const int nest = h.nesterov ? 1 : 0;
  {
    Prof prof(PK_OPTIM, 0, (double)nq * elems * 12, st);
    muon_momentum_kernel<<<dim3(kParts, nq), 256, 0, st>>>(grads, mom, ml, elems, h.momentum, nest, part);
    GPTK_CUDA(cudaGetLastError());
  }
  const int tiles = ((rows + 31) / 32) * ((cols + 31) / 32);
  const unsigned flat_blocks = (unsigned)std::min<long long>((elems + 1023) / 1024, 2048);
  {
    Prof prof(PK_OPTIM, 0, (double)nq * elems * 10, st);
    if (rows > cols)
      muon_prep_tr_kernel<<<dim3(tiles, nq), 256, 0, st>>>(grads, mom, ml, rows, cols, h.momentum, nest, part, X);
    else
      muon_prep_flat_kernel<<<dim3(flat_blocks, nq), 256, 0, st>>>(grads, mom, ml, elems, h.momentum, nest, part, X);
    GPTK_CUDA(cudaGetLastError());
  }
  int rows_of[kChunk];  // first row of matrix q in the stacked A and X buffers
  for (int q = 0; q < nq; ++q) rows_of[q] = q * m;
  for (int it = 0; it < h.ns_steps; ++it) {
    __nv_bfloat16* Xc = Xb[it & 1];
    __nv_bfloat16* Xn = Xb[(it + 1) & 1];
    GroupProblem gA[kChunk], gM[kChunk], gX[kChunk];
    for (int q = 0; q < nq; ++q) {
      __nv_bfloat16* Xq = Xc + (size_t)q * m * n;
      __nv_bfloat16* Aq = A + (size_t)q * m * m;
      __nv_bfloat16* Mq = M + (size_t)q * m * m;
      // A = X X^T and A A are symmetric: only their upper-triangle tiles are computed, and the
      // lower triangle is copied from the upper one
      gA[q] = GroupProblem{Xq, n, Xq, n, m, m, Aq, m, 0, 1};                   // A = X X^T
      gM[q] = GroupProblem{Aq, m, Aq, m, m, m, Mq, m, 0, 1};                   // A A (A^T = A)
      gX[q] = GroupProblem{Mq, m, Xq, n, m, n, Xn + (size_t)q * m * n, n, 0};  // M X (X read MN-major)
    }
    const int mirror_blocks = ((m + 63) / 64) * ((m + 63) / 64 + 1) / 2 * nq;
    const int mirror_grid = std::min(mirror_blocks, num_sms() * kMirrorCtas);  // every block resident at once
    GPTK_TRY(run_gemm_group(nq, gA, n, 0, 0, 256, PK_GEMM_MUON, st, EPI_BF16, 0));
    {
      Prof prof(PK_OPTIM, 0, (double)nq * m * m * 2, st);
      muon_mirror_kernel<<<mirror_grid, 256, 0, st>>>(A, m, nq);
      GPTK_CUDA(cudaGetLastError());
    }
    GPTK_TRY(run_gemm_group_axpby(nq, gM, m, 0, 0, PK_GEMM_MUON, A, m, (long long)nq * m, rows_of, kNsC, kNsB, st));
    {
      Prof prof(PK_OPTIM, 0, (double)nq * m * m * 2, st);
      muon_mirror_kernel<<<mirror_grid, 256, 0, st>>>(M, m, nq);
      GPTK_CUDA(cudaGetLastError());
    }
    GPTK_TRY(run_gemm_group_axpby(nq, gX, m, 0, 1, PK_GEMM_MUON, Xc, n, (long long)nq * m, rows_of, 1.f, kNsA, st));
  }
  X = Xb[h.ns_steps & 1];
  const float step = (float)(h.lr * std::sqrt(rows > cols ? (double)rows / cols : 1.0));
  {
    Prof prof(PK_OPTIM, 0, (double)nq * elems * 10, st);
    if (rows > cols)
      muon_update_tr_kernel<<<dim3(tiles, nq), 256, 0, st>>>(params, ml, rows, cols, X, step);
    else
      muon_update_flat_kernel<<<dim3(flat_blocks, nq), 256, 0, st>>>(params, ml, elems, X, step);
    GPTK_CUDA(cudaGetLastError());
  }
  return ST_OK;
}

}  // namespace

size_t muon_scratch_bytes(const std::vector<long long>& offs, const std::vector<int>& rows,
                          const std::vector<int>& cols) {
  std::vector<MuonGroup> groups;
  for (size_t i = 0; i < offs.size(); ++i) {
    bool found = false;
    for (MuonGroup& g : groups)
      if (g.rows == rows[i] && g.cols == cols[i]) {
        g.offs.push_back(offs[i]);
        found = true;
      }
    if (!found) groups.push_back(MuonGroup{rows[i], cols[i], {offs[i]}});
  }
  return muon_scratch_plan(groups).total;
}

int launch_muon(float* params, const float* grads, float* mom, const std::vector<long long>& offs,
                const std::vector<int>& rows, const std::vector<int>& cols, const gpt_muon& h, void* scratch,
                cudaStream_t st) {
  if (!(h.lr >= 0.f) || !(h.momentum >= 0.f && h.momentum < 1.f) || h.ns_steps < 1 || h.ns_steps > 32)
    return set_error(ST_INVALID_ARG, "muon: need lr >= 0, 0 <= momentum < 1 and 1 <= ns_steps <= 32");
  std::vector<MuonGroup> groups;
  for (size_t i = 0; i < offs.size(); ++i) {
    if ((rows[i] % 16) || (cols[i] % 16) || (offs[i] % 16))
      return set_error(ST_UNSUPPORTED, "muon: matrix sides and offsets must be multiples of 16");
    bool found = false;
    for (MuonGroup& g : groups)
      if (g.rows == rows[i] && g.cols == cols[i]) {
        g.offs.push_back(offs[i]);
        found = true;
      }
    if (!found) groups.push_back(MuonGroup{rows[i], cols[i], {offs[i]}});
  }
  const MuonScratch sp = muon_scratch_plan(groups);
  for (const MuonGroup& g : groups)
    for (int first = 0; first < (int)g.offs.size(); first += kChunk) {
      const int nq = (int)g.offs.size() - first < kChunk ? (int)g.offs.size() - first : kChunk;
      GPTK_TRY(muon_chunk(params, grads, mom, g, first, nq, h, scratch, sp, st));
    }
  return ST_OK;
}

}  // namespace gptk
