// Declarations of the launchers for the memory-bound kernels (kernels.cu,
// embed_bwd.cu) and the attention kernels (attention.cu).
#pragma once

#include "gpt.h"

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "ptx.cuh"

namespace gptk {

enum : unsigned int { DEV_ERR_BAD_TOKEN = 2u };

// fp32 -> bf16, n elements (n % 4 == 0, 16-byte aligned)
int launch_cast_bf16(const float* src, __nv_bfloat16* dst, long long n, cudaStream_t st);
// cs[t][i] = (cos, sin)(t * base^(-i/half)), computed in double
int launch_rope_table(float2* cs, int T, int half, double base, cudaStream_t st);
// x[m] = wte[idx[m]] (+ wpe[m % T])   (fp32 [M, D])
int launch_embed_fwd(const int* idx, const float* wte, const float* wpe, float* x, int M, int T, int D, int V,
                     cudaStream_t st);
// y = norm(x) as bf16 [M, ldy]; saves mean (LayerNorm only) and rstd per row
// amax (optional): max |y| over the output, as a float, atomically folded into *amax (which the
// caller zeroes first), for an 8-bit cast of y that then needs no pass of its own
int launch_norm_fwd(const float* x, int M, int D, const float* g, const float* b, int ln, float eps,
                    __nv_bfloat16* y, long long ldy, float* mean, float* rstd, cudaStream_t st,
                    float* amax = nullptr);
// dres (+)= norm'(x)^T dy ; also writes a bf16 copy of the result; LayerNorm gain/bias
// gradients go to per-block partials (dg_part, db_part: [nblk][D]) for launch_colreduce
int launch_norm_bwd(const float* dy, const float* x, const float* mean, const float* rstd, const float* g, int ln,
                    int M, int D, float* dres, int dres_init, __nv_bfloat16* dres_bf, float* dg_part,
                    float* db_part, int* nblk_out, cudaStream_t st);
// RMSNorm backward from the saved bf16 output y (= x rstd): dres (+)= rstd (dy - y mean(dy y)),
// with a bf16 copy; dy bf16 (dy_bf16 != 0) or fp32
int launch_rms_bwd(const void* dy, int dy_bf16, const __nv_bfloat16* y, const float* rstd, int M, int D,
                   float* dres, int dres_init, __nv_bfloat16* dres_bf, cudaStream_t st);
// out[i] = sum over p < n_parts of parts[p * stride + i], i < n, added in part order
int launch_sum_parts(const float* parts, int n_parts, size_t stride, size_t n, float* out, cudaStream_t st);
// out[c] (+)= sum_r part[r][c]  (fixed order)
int launch_colreduce(const float* part, int R, int N, float* out, int accumulate, cudaStream_t st);
// column sums of an [M, N] matrix into per-chunk partials (returns the number of chunks)
int launch_colsum_f32(const float* a, long long lda, int M, int N, float* part, int* R, cudaStream_t st);
int launch_colsum_bf16(const __nv_bfloat16* a, long long lda, int M, int N, float* part, int* R, cudaStream_t st);
int colsum_max_chunks();
// per-row cross-entropy from the vocab-tile partials: ell = lse - z_y (NaN, and a device status
// report, for a target outside [0, V))
int launch_ce_combine(const float2* part, int ntiles, const float* zy, const int* targets, int V, int M, float* ell,
                      float* lse, cudaStream_t st);
// deterministic reduction of per-token losses: loss = sum/M, and bpb sums over targets with bytes > 0
int launch_loss_reduce(const float* ell, const int* targets, const int* token_bytes, int V, int M, double* part_d,
                       long long* part_i, float* loss, double* sum_nats, long long* sum_bytes, float* bpb,
                       cudaStream_t st);
int loss_reduce_blocks();
// q,k,v (head padded) -> per-head RMSNorm / RoPE reverse -> dqkv [M, 3D] (unpadded)
int launch_qk_bwd(const __nv_bfloat16* dqkv_pad, const __nv_bfloat16* qkv_pad, const float* rstd_q,
                  const float* rstd_k, const float2* rope_cs, int M, int T, int H, int hd, int hdp, int rope,
                  int qk_norm, __nv_bfloat16* dqkv, cudaStream_t st);
// raw qkv [M, 3D] -> RoPE, per-head RMSNorm -> padded q,k,v
int launch_qk_fwd(const __nv_bfloat16* qkv, const float2* rope_cs, int M, int T, int H, int hd, int hdp, int rope,
                  int qk_norm, float eps, __nv_bfloat16* qkv_pad, float* rstd_q, float* rstd_k, cudaStream_t st);
// delta[b,h,t] = sum_d o[m, h*hd + d] * do[m, h, d]
int launch_attn_delta(const __nv_bfloat16* o, const __nv_bfloat16* do_pad, int B, int T, int H, int hd, int hdp,
                      float* delta, cudaStream_t st);
// params[off, off+n) = std * N(0,1) from the counter-based generator, or = value
int launch_init_normal(float* params, long long off, long long n, unsigned long long seed, float std,
                       cudaStream_t st);
int launch_fill(float* p, long long n, float value, cudaStream_t st);

// ---- embedding backward (embed_bwd.cu)
// scratch layout sizes for M tokens over V ids
long long embed_bwd_scratch_bytes(int M, int V, int D);
// dwte[v] += sum over tokens m with idx[m] == v of dx[m]  (deterministic order: ascending m)
int launch_embed_bwd(const int* idx, const float* dx, int M, int D, int V, float* dwte, void* scratch,
                     cudaStream_t st);
// dwpe[t] (+)= sum_b dx[b*T + t]
int launch_pos_bwd(const float* dx, int B, int T, int D, float* dwpe, int accumulate, cudaStream_t st);

// ---- optimizer step (optim.cu)
// fp64 partials of the gradient norm
size_t adamw_scratch_bytes();
// clip_grad_norm_ + AdamW over params[0, n): run r of the host table covers
// [run_start[r], run_start[r + 1]) (the last one up to n) and is weight-decayed when run_decay[r]
int launch_adamw(float* params, const float* grads, float* m, float* v, long long n, const long long* run_start,
                 const unsigned char* run_decay, int n_runs, long long step, const gpt_adamw& h, void* scratch,
                 double* grad_norm, cudaStream_t st);

// ---- Muon step of the block matrices (muon.cu): matrix q is params[offs[q] ...] with shape
// [rows[q], cols[q]]; mom holds the momentum at the same offsets
size_t muon_scratch_bytes(const std::vector<long long>& offs, const std::vector<int>& rows,
                          const std::vector<int>& cols);
int launch_muon(float* params, const float* grads, float* mom, const std::vector<long long>& offs,
                const std::vector<int>& rows, const std::vector<int>& cols, const gpt_muon& h, void* scratch,
                cudaStream_t st);

// ---- 8-bit casts (fp8.cu): amax = max |x|, s = FP8_MAX / amax, out = cast(x s), inv_scale = 1 / s
int launch_fp8_quantize(const void* x, int x_fp32, long long n, int fmt, void* out, float* amax, float* inv_scale,
                        cudaStream_t st);
// the cast alone, with *amax already computed (max |x| as a float, e.g. by the producer of x)
int launch_fp8_cast(const void* x, int x_fp32, long long n, int fmt, void* out, const float* amax, float* inv_scale,
                    cudaStream_t st);

// ---- attention (attention.cu)
struct AttnShape {
  int B, T, H, hd, hdp;
  long long ld_qkv;  // pitch (elements) between tokens in the padded q|k|v buffer: 3*H*hdp
  int win;           // left window: query i sees keys i - win .. i (-1: every key up to i)
};
// (query, key) pairs a causal attention of T tokens with left window win (-1: none) scores
double attn_pairs(int T, int win);
// amax (optional): max |o| folded into *amax as for launch_norm_fwd
int launch_attn_fwd(const __nv_bfloat16* qkv_pad, const AttnShape& s, __nv_bfloat16* o, long long ldo, float* lse,
                    cudaStream_t st, float* amax = nullptr);
int launch_attn_bwd(const __nv_bfloat16* qkv_pad, const __nv_bfloat16* do_pad, const float* lse,
                    const float* delta, const AttnShape& s, __nv_bfloat16* dqkv_pad, cudaStream_t st);

}  // namespace gptk
