// Deterministic backward of the token and position embeddings.
//
//   dwte[v] += sum over tokens m with idx[m] == v of dx[m]        (ascending m)
//   dwpe[t] += sum over b of dx[b*T + t]                          (ascending b)
//
// Token ids follow a Zipf law, so one id can own thousands of rows; floating-point
// atomics would make the sum order (and the result) vary run to run.  Instead the
// tokens are counting-sorted by id with a stable order:
//   1. chunks of 256 tokens: each token's rank among equal ids earlier in its chunk,
//      and the per-chunk count of every id
//   2. per id, an exclusive scan of the chunk counts over chunks (column scan)
//   3. an exclusive scan of the per-id totals (bucket offsets)
//   4. scatter: position = offset[id] + earlier chunks' count + rank in chunk
//   5. the sorted positions are cut into chunks of 256; each chunk sums the rows of
//      every id segment inside it in ascending token order and adds complete
//      buckets straight into dwte; a bucket that crosses chunk edges leaves one
//      partial per chunk, and the chunk where it starts adds them up in chunk
//      order (a fixed order, so the result is reproducible)
#include "host.cuh"
#include "kernels.cuh"

namespace gptk {

static constexpr int kChunk = 256;

static inline long long align256(long long x) { return (x + 255) & ~255LL; }

struct EmbedScratch {
  int* cnt;      // [G][V]
  int* total;    // [V]
  int* offs;     // [V]
  int* rank;     // [M]
  int* sorted;   // [M]
  float* head;   // [G][D]  sum of a chunk's first segment when its bucket began in an earlier chunk
  float* tail;   // [G][D]  sum of a chunk's last segment when its bucket begins here and goes on
};

static EmbedScratch carve(void* base, int M, int V, int D) {
  const int G = (M + kChunk - 1) / kChunk;
  char* p = static_cast<char*>(base);
  EmbedScratch s;
  s.cnt = reinterpret_cast<int*>(p);
  p += align256((long long)G * V * 4);
  s.total = reinterpret_cast<int*>(p);
  p += align256((long long)V * 4);
  s.offs = reinterpret_cast<int*>(p);
  p += align256((long long)V * 4);
  s.rank = reinterpret_cast<int*>(p);
  p += align256((long long)M * 4);
  s.sorted = reinterpret_cast<int*>(p);
  p += align256((long long)M * 4);
  s.head = reinterpret_cast<float*>(p);
  p += align256((long long)G * D * 4);
  s.tail = reinterpret_cast<float*>(p);
  return s;
}

long long embed_bwd_scratch_bytes(int M, int V, int D) {
  const long long G = (M + kChunk - 1) / kChunk;
  return align256(G * V * 4) + 2 * align256((long long)V * 4) + 2 * align256((long long)M * 4) +
         2 * align256(G * D * 4);
}

__global__ void chunk_rank_kernel(const int* __restrict__ idx, int M, int V, int* __restrict__ cnt,
                                  int* __restrict__ rank) {
  __shared__ int ids[kChunk];
  const int g = blockIdx.x;
  const int t = threadIdx.x;
  const int m = g * kChunk + t;
  int id = -1;
  if (m < M) {
    id = idx[m];
    if (id < 0 || id >= V) id = 0;  // out-of-range ids were reported by the forward embedding
  }
  ids[t] = id;
  __syncthreads();
  if (m >= M) return;
  int r = 0;
  bool last = true;
  for (int u = 0; u < kChunk; ++u) {
    const int o = ids[u];
    if (o == id) {
      if (u < t) ++r;
      if (u > t) last = false;
    }
  }
  rank[m] = r;
  if (last) cnt[(long long)g * V + id] = r + 1;
}

__global__ void col_scan_kernel(int* __restrict__ cnt, int G, int V, int* __restrict__ total) {
  const int v = blockIdx.x * blockDim.x + threadIdx.x;
  if (v >= V) return;
  int run = 0;
  int g = 0;
  for (; g + 8 <= G; g += 8) {  // eight independent loads in flight, then the running sum
    int c[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) c[u] = cnt[(long long)(g + u) * V + v];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      cnt[(long long)(g + u) * V + v] = run;
      run += c[u];
    }
  }
  for (; g < G; ++g) {
    const long long i = (long long)g * V + v;
    const int c = cnt[i];
    cnt[i] = run;
    run += c;
  }
  total[v] = run;
}

// single block, 1024 threads: exclusive scan of total[0..V), straight from global memory (any V)
__global__ void offsets_global_kernel(const int* __restrict__ total, int V, int* __restrict__ offs) {
  __shared__ int part[1024];
  const int t = threadIdx.x;
  const int per = (V + 1023) / 1024;
  const int v0 = t * per, v1 = min(V, v0 + per);
  int s = 0;
  for (int v = v0; v < v1; ++v) s += total[v];
  part[t] = s;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    int x = t >= o ? part[t - o] : 0;
    __syncthreads();
    part[t] += x;
    __syncthreads();
  }
  int run = t > 0 ? part[t - 1] : 0;
  for (int v = v0; v < v1; ++v) {
    offs[v] = run;
    run += total[v];
  }
}

// The same with total staged in shared memory by coalesced loads first (V up to kOffsSmemV), so that
// each thread's stretch is read from shared memory.
constexpr int kOffsSmemV = 53248;  // 208 KB

__global__ void offsets_kernel(const int* __restrict__ total, int V, int* __restrict__ offs) {
  __shared__ int part[1024];
  extern __shared__ int tot_s[];
  const int t = threadIdx.x;
  for (int v = t; v < V; v += 1024) tot_s[v] = total[v];
  __syncthreads();
  const int per = (V + 1023) / 1024;
  const int v0 = t * per, v1 = min(V, v0 + per);
  int s = 0;
  for (int v = v0; v < v1; ++v) s += tot_s[v];
  part[t] = s;
  __syncthreads();
  // Hillis-Steele inclusive scan over the 1024 partial sums
  for (int o = 1; o < 1024; o <<= 1) {
    int x = t >= o ? part[t - o] : 0;
    __syncthreads();
    part[t] += x;
    __syncthreads();
  }
  int run = t > 0 ? part[t - 1] : 0;
  for (int v = v0; v < v1; ++v) {
    const int c = tot_s[v];
    tot_s[v] = run;
    run += c;
  }
  __syncthreads();
  for (int v = t; v < V; v += 1024) offs[v] = tot_s[v];
}

__global__ void scatter_kernel(const int* __restrict__ idx, int M, int V, const int* __restrict__ cnt,
                               const int* __restrict__ offs, const int* __restrict__ rank, int* __restrict__ sorted) {
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  if (m >= M) return;
  int id = idx[m];
  if (id < 0 || id >= V) id = 0;
  const int g = m / kChunk;
  sorted[offs[id] + cnt[(long long)g * V + id] + rank[m]] = m;
}

__device__ __forceinline__ int clamp_id(int id, int V) { return (id < 0 || id >= V) ? 0 : id; }

// One block per (chunk of 256 sorted positions, 128 float4 columns): each thread owns one float4
// column and walks the chunk's segments; the rows of a segment are loaded eight at a time (the
// loads are independent) and added in ascending token order.
constexpr int kSegCols = 128;

__global__ void segsum_chunk_kernel(const int* __restrict__ idx, const float* __restrict__ dx, int M, int D, int V,
                                    const int* __restrict__ total, const int* __restrict__ offs,
                                    const int* __restrict__ sorted, float* __restrict__ dwte,
                                    float* __restrict__ head, float* __restrict__ tail) {
  const int c = blockIdx.x;
  const int p0 = c * kChunk, p1 = min(M, p0 + kChunk);
  const int D4 = D / 4;
  const int col = blockIdx.y * kSegCols + threadIdx.x;
  if (col >= D4) return;
  const float4* dx4 = reinterpret_cast<const float4*>(dx) + col;
  int pos = p0;
  while (pos < p1) {
    const int id = clamp_id(idx[sorted[pos]], V);
    const int bstart = offs[id], bend = bstart + total[id];
    const int send = min(bend, p1);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int q = pos;
    for (; q + 8 <= send; q += 8) {
      float4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = __ldg(dx4 + (long long)sorted[q + u] * D4);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        acc.x += x[u].x; acc.y += x[u].y; acc.z += x[u].z; acc.w += x[u].w;
      }
    }
    for (; q < send; ++q) {
      const float4 x = __ldg(dx4 + (long long)sorted[q] * D4);
      acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
    }
    if (bstart < p0) {
      reinterpret_cast<float4*>(head + (long long)c * D)[col] = acc;
    } else if (bend > p1) {
      reinterpret_cast<float4*>(tail + (long long)c * D)[col] = acc;
    } else {
      float4* w = reinterpret_cast<float4*>(dwte + (long long)id * D) + col;
      float4 cur = *w;
      cur.x += acc.x; cur.y += acc.y; cur.z += acc.z; cur.w += acc.w;
      *w = cur;
    }
    pos = send;
  }
}

// Buckets that start in chunk c and run past its end: tail[c] + head[c+1] + ... in chunk order.
__global__ void segsum_fixup_kernel(const int* __restrict__ idx, int M, int D, int V, const int* __restrict__ total,
                                    const int* __restrict__ offs, const int* __restrict__ sorted,
                                    float* __restrict__ dwte, const float* __restrict__ head,
                                    const float* __restrict__ tail) {
  const int c = blockIdx.x;
  const int p0 = c * kChunk, p1 = min(M, p0 + kChunk);
  const int id = clamp_id(idx[sorted[p1 - 1]], V);
  const int bstart = offs[id], bend = bstart + total[id];
  if (bstart < p0 || bend <= p1) return;
  const int D4 = D / 4;
  for (int col = threadIdx.x; col < D4; col += blockDim.x) {
    float4 acc = reinterpret_cast<const float4*>(tail + (long long)c * D)[col];
    for (int cc = c + 1; cc * kChunk < bend; ++cc) {
      const float4 h = reinterpret_cast<const float4*>(head + (long long)cc * D)[col];
      acc.x += h.x; acc.y += h.y; acc.z += h.z; acc.w += h.w;
    }
    float4* w = reinterpret_cast<float4*>(dwte + (long long)id * D) + col;
    float4 cur = *w;
    cur.x += acc.x; cur.y += acc.y; cur.z += acc.z; cur.w += acc.w;
    *w = cur;
  }
}

int launch_embed_bwd(const int* idx, const float* dx, int M, int D, int V, float* dwte, void* scratch,
                     cudaStream_t st) {
  if (D % 4) return set_error(ST_UNSUPPORTED, "embedding backward: n_embd must be a multiple of 4");
  const int G = (M + kChunk - 1) / kChunk;
  EmbedScratch s = carve(scratch, M, V, D);
  GPTK_CUDA(cudaMemsetAsync(s.cnt, 0, (size_t)G * V * sizeof(int), st));
  {
    Prof prof(PK_EMBED_BWD, 0, M * 8.0, st);
    chunk_rank_kernel<<<G, kChunk, 0, st>>>(idx, M, V, s.cnt, s.rank);
    GPTK_CUDA(cudaGetLastError());
  }
  {
    Prof prof(PK_EMBED_BWD, 0, (double)G * V * 8, st);
    col_scan_kernel<<<(V + 255) / 256, 256, 0, st>>>(s.cnt, G, V, s.total);
    GPTK_CUDA(cudaGetLastError());
  }
  {
    Prof prof(PK_EMBED_BWD, 0, V * 8.0, st);
    if (V <= kOffsSmemV) {
      GPTK_CUDA(cudaFuncSetAttribute(offsets_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kOffsSmemV * 4));
      offsets_kernel<<<1, 1024, (size_t)V * sizeof(int), st>>>(s.total, V, s.offs);
    } else {
      offsets_global_kernel<<<1, 1024, 0, st>>>(s.total, V, s.offs);
    }
    GPTK_CUDA(cudaGetLastError());
  }
  {
    Prof prof(PK_EMBED_BWD, 0, M * 20.0, st);
    scatter_kernel<<<(M + 255) / 256, 256, 0, st>>>(idx, M, V, s.cnt, s.offs, s.rank, s.sorted);
    GPTK_CUDA(cudaGetLastError());
  }
  const int threads = D / 4 < 256 ? ((D / 4 + 31) / 32) * 32 : 256;
  {
    Prof prof(PK_EMBED_BWD, 0, (double)M * D * 4 + M * 8.0, st);
    const dim3 grid(G, (D / 4 + kSegCols - 1) / kSegCols);
    const int seg_threads = D / 4 < kSegCols ? ((D / 4 + 31) / 32) * 32 : kSegCols;
    segsum_chunk_kernel<<<grid, seg_threads, 0, st>>>(idx, dx, M, D, V, s.total, s.offs, s.sorted, dwte, s.head,
                                                      s.tail);
    GPTK_CUDA(cudaGetLastError());
  }
  {
    Prof prof(PK_EMBED_BWD, 0, (double)G * D * 8, st);
    segsum_fixup_kernel<<<G, threads, 0, st>>>(idx, M, D, V, s.total, s.offs, s.sorted, dwte, s.head, s.tail);
    GPTK_CUDA(cudaGetLastError());
  }
  return ST_OK;
}

__global__ void pos_bwd_kernel(const float* __restrict__ dx, int B, int T, int D, float* __restrict__ dwpe,
                               int accumulate) {
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= (long long)T * D) return;
  const int t = static_cast<int>(i / D), d = static_cast<int>(i % D);
  float s = 0.f;
  for (int b = 0; b < B; ++b) s += dx[((long long)b * T + t) * D + d];
  dwpe[i] = accumulate ? dwpe[i] + s : s;
}

int launch_pos_bwd(const float* dx, int B, int T, int D, float* dwpe, int accumulate, cudaStream_t st) {
  const long long n = (long long)T * D;
  Prof prof(PK_EMBED_BWD, 0, (double)B * T * D * 4 + (double)T * D * 8, st);
  pos_bwd_kernel<<<(int)((n + 255) / 256), 256, 0, st>>>(dx, B, T, D, dwpe, accumulate);
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

}  // namespace gptk
