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
//   muon_prep_kernel       X = U / ||U|| in bf16, transposed through shared memory when needed
//   ns_steps x { grouped GEMM A = X X^T (bf16),
//                grouped GEMM M = c (A A) + b A (bf16; the linear combination in the epilogue),
//                grouped GEMM X' = (M X) + a X (bf16, into the other X buffer) }
//   muon_update_kernel     W -= lr scale X, transposed back through shared memory when needed
#include <cmath>
#include <string>
#include <vector>

#include "gemm.cuh"
#include "gpt.h"
#include "host.cuh"
#include "kernels.cuh"

namespace gptk {

namespace {

constexpr int kParts = 64;              // fixed partition of each matrix's squared-norm sum
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

// X[q] [m, n] bf16 = U / (||U||_F + 1e-7) with U [rows, cols] of matrix q; X = U^T when
// rows > cols.  32 x 32 tiles through shared memory (blockIdx.x: tile, blockIdx.y: matrix).
__global__ void __launch_bounds__(256) muon_prep_kernel(const float* __restrict__ g, const float* __restrict__ mom,
                                                        MatList ml, int rows, int cols, float mu, int nesterov,
                                                        const double* __restrict__ part,
                                                        __nv_bfloat16* __restrict__ X) {
  __shared__ float tile[32][33];
  __shared__ float s_inv;
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int k = 0; k < kParts; ++k) t += part[blockIdx.y * kParts + k];  // one fixed order
    s_inv = (float)(1.0 / (sqrt(t) + 1e-7));
  }
  const long long base = ml.off[blockIdx.y];
  const int tiles_c = (cols + 31) / 32;
  const int r0 = (blockIdx.x / tiles_c) * 32, c0 = (blockIdx.x % tiles_c) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 8 rows of 32 per pass
  const float omm = 1.f - mu;
  __syncthreads();
  const float inv = s_inv;
  const bool tr = rows > cols;
  __nv_bfloat16* Xq = X + (long long)blockIdx.y * rows * cols;
  for (int rr = ty; rr < 32; rr += 8) {
    const int r = r0 + rr, c = c0 + tx;
    float u = 0.f;
    if (r < rows && c < cols) {
      const long long i = base + (long long)r * cols + c;
      const float b = mom[i];
      u = nesterov ? fmaf(omm, g[i], mu * b) : b;
    }
    if (tr) tile[rr][tx] = u * inv;
    else if (r < rows && c < cols) Xq[(long long)r * cols + c] = __float2bfloat16_rn(u * inv);
  }
  if (!tr) return;
  __syncthreads();
  // X[c][r] = U[r][c]: X is [cols, rows]
  for (int cc = ty; cc < 32; cc += 8) {
    const int c = c0 + cc, r = r0 + tx;
    if (r < rows && c < cols) Xq[(long long)c * rows + r] = __float2bfloat16_rn(tile[tx][cc]);
  }
}

// W[r][c] -= step * X'[r][c] with X' = X (rows <= cols) or X^T (X is [cols, rows]); tiles of 32 x 32
__global__ void __launch_bounds__(256) muon_update_kernel(float* __restrict__ params, MatList ml, int rows, int cols,
                                                          const __nv_bfloat16* __restrict__ X, float step) {
  __shared__ float tile[32][33];
  const long long base = ml.off[blockIdx.y];
  const int tiles_c = (cols + 31) / 32;
  const int r0 = (blockIdx.x / tiles_c) * 32, c0 = (blockIdx.x % tiles_c) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const __nv_bfloat16* Xq = X + (long long)blockIdx.y * rows * cols;
  const bool tr = rows > cols;
  if (tr) {
    // read X[c][r] along r (contiguous), then update W[r][c] along c
    for (int cc = ty; cc < 32; cc += 8) {
      const int c = c0 + cc, r = r0 + tx;
      tile[tx][cc] = (r < rows && c < cols) ? __bfloat162float(Xq[(long long)c * rows + r]) : 0.f;
    }
    __syncthreads();
  }
  for (int rr = ty; rr < 32; rr += 8) {
    const int r = r0 + rr, c = c0 + tx;
    if (r < rows && c < cols) {
      const float x = tr ? tile[rr][tx] : __bfloat162float(Xq[(long long)r * cols + c]);
      params[base + (long long)r * cols + c] -= step * x;
    }
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
  {
    Prof prof(PK_OPTIM, 0, (double)nq * elems * 10, st);
    muon_prep_kernel<<<dim3(tiles, nq), 256, 0, st>>>(grads, mom, ml, rows, cols, h.momentum, nest, part, X);
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
      gA[q] = GroupProblem{Xq, n, Xq, n, m, m, Aq, m, 0};                   // A = X X^T
      gM[q] = GroupProblem{Aq, m, Aq, m, m, m, Mq, m, 0};                   // A A (A is symmetric: A^T = A)
      gX[q] = GroupProblem{Mq, m, Xq, n, m, n, Xn + (size_t)q * m * n, n, 0};  // M X (X read MN-major)
    }
    GPTK_TRY(run_gemm_group(nq, gA, n, 0, 0, 256, PK_GEMM_MUON, st, EPI_BF16, 0));
    GPTK_TRY(run_gemm_group_axpby(nq, gM, m, 0, 0, PK_GEMM_MUON, A, m, (long long)nq * m, rows_of, kNsC, kNsB, st));
    GPTK_TRY(run_gemm_group_axpby(nq, gX, m, 0, 1, PK_GEMM_MUON, Xc, n, (long long)nq * m, rows_of, 1.f, kNsA, st));
  }
  X = Xb[h.ns_steps & 1];
  const float step = (float)(h.lr * std::sqrt(rows > cols ? (double)rows / cols : 1.0));
  {
    Prof prof(PK_OPTIM, 0, (double)nq * elems * 10, st);
    muon_update_kernel<<<dim3(tiles, nq), 256, 0, st>>>(params, ml, rows, cols, X, step);
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
